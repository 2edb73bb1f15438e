"""KVSlimmer asymmetric KV merging -- plain CPU oracle (fp64, numpy).

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or links
this module; only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
legs of ``bench.py`` use it. It shares no code with the CUDA kernels: it takes
plain arrays and returns plain arrays, computed in fp64 in the order the pages
state the method, with no blocking, fusion or reordering.

Sources (cited by title and section):
  [KVS]  "论文专题讲解：KVSlimmer：非对称 KV 合并的数学与工程" -- blog deep dive of
         arXiv 2603.00907 (sections 数学主线二/三/四, 实验设置, 工程上怎么用).
  [ABS]  "KVSlimmer: Theoretical Insights and Practical Optimizations for
         Asymmetric KV Merging" -- abstract pages (fugumt / thelatestinai).
  [ASY]  "Homogeneous Keys, Heterogeneous Values: Exploiting Local KV Cache
         Asymmetry for Long-Context LLMs" -- related-paper entry on the fugumt
         page (AsymKV's "lossless value compression").

Readings taken where the pages are silent (each is listed again, with its
reason, in the design notes):
  R1 window statistics: the pages derive the Hessian for one query q. With a
     window of W recent queries of the G query heads sharing a KV head, the
     oracle averages the attention of those G*W queries (alpha_bar) and uses
     o_bar = mean_q o_q = sum_t alpha_bar_t v_t in the single-query formulas.
     For one query this is exactly the pages' expression. The alternative
     (reading B, stats="per_query") averages the single-query norms over the
     window queries instead; it too reduces to the pages' expression for one
     query.
  R2 candidates: disjoint adjacent pairs (c0+2p, c0+2p+1) of the candidate
     span [c0, len - n_recent); an odd leftover token is never merged.
  R3 score: a pair's score is the minimum value of the forward-only second
     order objective; lower scores merge first; ties go to the lower index;
     NaN counts as +inf.
  R4 budget: one round merges R = min(P, max(0, len - target)) pairs; rounds
     repeat until len == target (exact).
  R5 Value rule: Values are never averaged lossily. A merged group stores the
     count-weighted mean value and log(count) as a logit bias, which is
     exactly attention over the expanded cache in which every original
     position keeps its own value under the shared merged key.
  R6 degenerate pairs: when D = N11 - 2 N12 + N22 is not > 1e-6 (N11 + N22),
     or a term is not finite, the plain average (w = 1/2) is used and scored
     with the objective at w = 1/2.
  R7 merged key: k* = k_a + w_b (k_b - k_a), algebraically the pages' form.
  R8 window position: window query j sits at cache position len - W + j and
     attends positions <= its own (causal). Queries with a negative position
     are left out of the average.
  R9 storage: a cache is stored in its element type between rounds. Merged
     rows are rounded to that type (bf16: to fp32, then round-to-nearest-even
     on the upper 16 bits) and log counts to fp32 before the next round reads
     them; arithmetic inside a round stays fp64.
  R10 empty cache: decode attention over a head with no rows (and no appended
     row) returns the zero vector.
  R11 chunked prefill: each prompt chunk is appended with count 1; while a
     head is longer than the budget, a round runs with candidate span
     [sink, len - W), the chunk's last W queries as the window and the budget
     as the per-head target.
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np

DEGENERATE_REL = 1e-6


# ---------------------------------------------------------------------------
# Storage precision of a cache (reading R9)
# ---------------------------------------------------------------------------

def storage_round(x, storage="f64"):
    """Round fp64 values to what a cache of element type `storage` holds."""
    x = np.asarray(x, dtype=np.float64)
    if storage == "f64":
        return x
    f32 = x.astype(np.float32)
    if storage == "f32":
        return f32.astype(np.float64)
    if storage == "bf16":
        bits = f32.view(np.uint32).astype(np.uint64)
        nan = np.isnan(f32)
        lsb = (bits >> 16) & 1
        rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
        out = rounded.astype(np.uint32).view(np.float32)
        out = np.where(nan, np.float32(np.nan), out)
        return out.astype(np.float64)
    raise ValueError(storage)


# ---------------------------------------------------------------------------
# Attention forward and its exact derivatives  ([KVS] §数学主线三)
# ---------------------------------------------------------------------------

def attention_logits(q, K, log_n=None):
    """e_i = q k_i^T / sqrt(d_k)   ([KVS] §数学主线三, attention forward).

    ``log_n`` (log multiplicity of merged groups, reading R5) is added as a
    per-key logit bias; None means every key has count 1.
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    e = K @ q / math.sqrt(K.shape[-1])
    if log_n is not None:
        e = e + np.asarray(log_n, dtype=np.float64)
    return e


def softmax(e):
    """alpha_i = exp(e_i) / sum_t exp(e_t)   ([KVS] §数学主线三)."""
    e = np.asarray(e, dtype=np.float64)
    m = np.max(e)
    p = np.exp(e - m)
    return p / np.sum(p)


def attention_output(alpha, V):
    """o = sum_t alpha_t v_t   ([KVS] §数学主线三)."""
    return np.asarray(alpha, dtype=np.float64) @ np.asarray(V, dtype=np.float64)


def key_gradient(q, K, V, E, i, log_n=None):
    """g_i = (1/sqrt(d_k)) alpha_i [E^T (v_i - o)] q   ([KVS] §数学主线三, first-order term)."""
    q = np.asarray(q, dtype=np.float64)
    alpha = softmax(attention_logits(q, K, log_n))
    V = np.asarray(V, dtype=np.float64)
    o = attention_output(alpha, V)
    d_k = q.shape[0]
    return alpha[i] * float(np.dot(E, V[i] - o)) * q / math.sqrt(d_k)


def score_sensitivity(alpha, V, o, i, j):
    """d s_i / d e_j with s_i = alpha_i (v_i - o)   ([KVS] §数学主线三).

    diagonal:      alpha_i (1 - 2 alpha_i) (v_i - o)
    off-diagonal: -alpha_i alpha_j (v_i + v_j - 2 o)
    """
    V = np.asarray(V, dtype=np.float64)
    if i == j:
        return alpha[i] * (1.0 - 2.0 * alpha[i]) * (V[i] - o)
    return -alpha[i] * alpha[j] * (V[i] + V[j] - 2.0 * o)


def hessian_block(q, K, V, E, i, j, log_n=None):
    """h_ij = (1/d_k) [E^T ds_i/de_j] q q^T for the loss L = E^T o with fixed E
    ([KVS] §数学主线三, Hessian block)."""
    q = np.asarray(q, dtype=np.float64)
    alpha = softmax(attention_logits(q, K, log_n))
    o = attention_output(alpha, V)
    d_k = q.shape[0]
    sens = score_sensitivity(alpha, V, o, i, j)
    return float(np.dot(E, sens)) * np.outer(q, q) / d_k


# ---------------------------------------------------------------------------
# Pair objective and closed forms  ([KVS] §数学主线二, §数学主线四)
# ---------------------------------------------------------------------------

def forward_vectors(alpha_m, alpha_m1, v_m, v_m1, o):
    """c11, c22, c12 built from forward variables only   ([KVS] §数学主线四)."""
    v_m = np.asarray(v_m, dtype=np.float64)
    v_m1 = np.asarray(v_m1, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    c11 = alpha_m * (1.0 - 2.0 * alpha_m) * (v_m - o)
    c22 = alpha_m1 * (1.0 - 2.0 * alpha_m1) * (v_m1 - o)
    c12 = -alpha_m * alpha_m1 * (v_m + v_m1 - 2.0 * o)
    return c11, c22, c12


def pair_objective(k, k_m, k_m1, g11, g12, g22):
    """g11 |k-k_m|^2 + 2 g12 (k-k_m)^T (k-k_m1) + g22 |k-k_m1|^2   ([KVS] §数学主线二)."""
    k = np.asarray(k, dtype=np.float64)
    dm = k - np.asarray(k_m, dtype=np.float64)
    dm1 = k - np.asarray(k_m1, dtype=np.float64)
    return g11 * np.dot(dm, dm) + 2.0 * g12 * np.dot(dm, dm1) + g22 * np.dot(dm1, dm1)


def merged_key_hessian_form(g11, g12, g22, k_m, k_m1):
    """k* = [(g11+g12) k_m + (g12+g22) k_m1] / (g11 + 2 g12 + g22)   ([KVS] §数学主线二)."""
    return ((g11 + g12) * np.asarray(k_m, dtype=np.float64)
            + (g12 + g22) * np.asarray(k_m1, dtype=np.float64)) / (g11 + 2.0 * g12 + g22)


def forward_only_weights(n11, n12, n22):
    """(w_m, w_m1) from the norms |c11|, |c12|, |c22|   ([KVS] §数学主线四, forward-only k*).

    w_m  = (|c11| - |c12|) / (|c11| - 2|c12| + |c22|)
    w_m1 = (|c22| - |c12|) / (|c11| - 2|c12| + |c22|)
    """
    den = n11 - 2.0 * n12 + n22
    return (n11 - n12) / den, (n22 - n12) / den


def pair_norms(alpha_a, alpha_b, v_a, v_b, o):
    """N11 = |c11|, N12 = |c12|, N22 = |c22| for pairs (vectorised over leading axes).

    |c11| = |alpha_a (1 - 2 alpha_a)| |v_a - o|, |c22| likewise,
    |c12| = alpha_a alpha_b |v_a + v_b - 2 o|   ([KVS] §数学主线四).
    """
    alpha_a = np.asarray(alpha_a, dtype=np.float64)
    alpha_b = np.asarray(alpha_b, dtype=np.float64)
    v_a = np.asarray(v_a, dtype=np.float64)
    v_b = np.asarray(v_b, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    n11 = np.abs(alpha_a * (1.0 - 2.0 * alpha_a)) * np.linalg.norm(v_a - o, axis=-1)
    n22 = np.abs(alpha_b * (1.0 - 2.0 * alpha_b)) * np.linalg.norm(v_b - o, axis=-1)
    n12 = alpha_a * alpha_b * np.linalg.norm(v_a + v_b - 2.0 * o, axis=-1)
    return n11, n12, n22


FORMS = ("full", "diagonal")


def weight_and_score(n11, n12, n22, k_a, k_b, form="full"):
    """Merge weight w_b of the second key and the pair's score (vectorised).

    With the effective scalars (g11, g12, g22) = (N11, -N12, N22) -- the
    forward-only substitution of [KVS] §数学主线四 -- the objective of
    §数学主线二 has its minimiser at k* = k_a + w_b (k_b - k_a) with
    w_b = (N22 - N12) / D, D = N11 - 2 N12 + N22, and minimum value
    |k_b - k_a|^2 (N11 N22 - N12^2) / D (the score, reading R3).
    Degenerate pairs use w_b = 1/2 and the objective there,
    |k_b - k_a|^2 (N11 + 2 N12 + N22) / 4 (reading R6).

    form="diagonal" is the ablation without the coupling term (g12 = 0, the
    per-key weighting of AsymKV that §数学主线二 contrasts with): the objective
    N11 |k - k_a|^2 + N22 |k - k_b|^2 has its minimiser at
    k* = (N11 k_a + N22 k_b) / (N11 + N22), i.e. w_b = N22 / (N11 + N22), and
    minimum value |k_b - k_a|^2 N11 N22 / (N11 + N22); degenerate (N11 + N22 not
    positive or a term not finite): w_b = 1/2, score |k_b - k_a|^2 (N11 + N22) / 4.
    Returns (w_b, score, degenerate_mask, D).
    """
    if form not in FORMS:
        raise ValueError(form)
    n11 = np.asarray(n11, dtype=np.float64)
    n12 = np.asarray(n12, dtype=np.float64)
    n22 = np.asarray(n22, dtype=np.float64)
    delta = np.asarray(k_b, dtype=np.float64) - np.asarray(k_a, dtype=np.float64)
    delta_sq = np.sum(delta * delta, axis=-1)
    if form == "diagonal":
        D = n11 + n22
        with np.errstate(invalid="ignore", divide="ignore", over="ignore"):
            ok = np.isfinite(n11) & np.isfinite(n22) & np.isfinite(D) & (D > 0.0)
            safe_D = np.where(ok, D, 1.0)
            w_b = np.where(ok, n22 / safe_D, 0.5)
            score = np.where(ok, delta_sq * n11 * n22 / safe_D, delta_sq * D / 4.0)
        return w_b, score, ~ok, D
    D = n11 - 2.0 * n12 + n22
    with np.errstate(invalid="ignore", divide="ignore", over="ignore"):
        ok = (np.isfinite(n11) & np.isfinite(n12) & np.isfinite(n22) & np.isfinite(D)
              & (D > DEGENERATE_REL * (n11 + n22)))
        safe_D = np.where(ok, D, 1.0)
        w_b = np.where(ok, (n22 - n12) / safe_D, 0.5)
        score = np.where(ok, delta_sq * (n11 * n22 - n12 * n12) / safe_D,
                         delta_sq * (n11 + 2.0 * n12 + n22) / 4.0)
    return w_b, score, ~ok, D


# ---------------------------------------------------------------------------
# Window statistics (reading R1, R8)
# ---------------------------------------------------------------------------

def window_attention(Q_heads, K, V, log_n, length, W):
    """Attention rows of the window queries of one KV head.

    Q_heads: (G, W, d) -- the window queries of the G query heads sharing the
    KV head; query j sits at position length - W + j and attends positions
    0..length-W+j. Returns (A, O): A is (Qv, length) with one softmax row per
    valid query, O is (Qv, d) with the outputs o_q.
    """
    Q_heads = np.asarray(Q_heads, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)[:length]
    V = np.asarray(V, dtype=np.float64)[:length]
    ln = None if log_n is None else np.asarray(log_n, dtype=np.float64)[:length]
    rows, outs = [], []
    G = Q_heads.shape[0]
    for g in range(G):
        for j in range(W):
            pos = length - W + j
            if pos < 0:
                continue
            e = attention_logits(Q_heads[g, j], K[:pos + 1], None if ln is None else ln[:pos + 1])
            alpha = np.zeros(length)
            alpha[:pos + 1] = softmax(e)
            rows.append(alpha)
            outs.append(attention_output(alpha, V))
    d = K.shape[1] if K.ndim == 2 else Q_heads.shape[-1]
    if not rows:
        return np.zeros((0, length)), np.zeros((0, d))
    return np.array(rows), np.array(outs)


def window_statistics(Q_heads, K, V, log_n, length, W):
    """alpha_bar (length,) = mean over window queries of their attention;
    o_bar (d,) = mean over window queries of o_q (reading R1)."""
    A, O = window_attention(Q_heads, K, V, log_n, length, W)
    d = np.asarray(K).shape[-1]
    if A.shape[0] == 0:
        return np.zeros(length), np.zeros(d)
    return A.mean(axis=0), O.mean(axis=0)


def pair_norms_per_query(A, O, V, a, b):
    """Reading B of the window (the alternative to R1): the single-query norms of
    [KVS] §数学主线四 taken per window query and averaged,

        N11 = mean_q |a_qa (1 - 2 a_qa)| |v_a - o_q|,   N22 likewise,
        N12 = mean_q a_qa a_qb |v_a + v_b - 2 o_q|,

    from the window's attention rows A (Qv, len) and outputs O (Qv, d); a, b index the
    pairs' rows. With one window query it is exactly pair_norms of that query."""
    A = np.asarray(A, dtype=np.float64)
    O = np.asarray(O, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    a = np.asarray(a)
    b = np.asarray(b)
    if A.shape[0] == 0:
        z = np.zeros(a.shape)
        return z, z.copy(), z.copy()
    n11 = np.zeros(a.shape)
    n12 = np.zeros(a.shape)
    n22 = np.zeros(a.shape)
    for q in range(A.shape[0]):
        x11, x12, x22 = pair_norms(A[q, a], A[q, b], V[a], V[b], O[q])
        n11 += x11
        n12 += x12
        n22 += x22
    return n11 / A.shape[0], n12 / A.shape[0], n22 / A.shape[0]


STATS = ("mean", "per_query")


# ---------------------------------------------------------------------------
# One KV head: candidates, scores, selection, merge and compaction
# ---------------------------------------------------------------------------

def num_pairs(length, cand_begin, n_recent):
    """P = floor((len - n_recent - c0) / 2) disjoint adjacent pairs (reading R2)."""
    return max(0, (int(length) - int(n_recent) - int(cand_begin)) // 2)


@dataclass
class HeadScores:
    score: np.ndarray
    w_b: np.ndarray
    n11: np.ndarray
    n12: np.ndarray
    n22: np.ndarray
    D: np.ndarray
    degenerate: np.ndarray
    alpha_bar: np.ndarray
    o_bar: np.ndarray


def score_head(K, V, log_n, length, cand_begin, n_recent, Q_heads, W, form="full",
               stats="mean"):
    """Score every candidate pair of one KV head (form: see weight_and_score; stats:
    "mean" = reading R1, norms of the window-mean statistics; "per_query" = reading B,
    see pair_norms_per_query)."""
    if stats not in STATS:
        raise ValueError(stats)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    alpha_bar, o_bar = window_statistics(Q_heads, K, V, log_n, length, W)
    P = num_pairs(length, cand_begin, n_recent)
    a = int(cand_begin) + 2 * np.arange(P)
    b = a + 1
    if stats == "mean":
        n11, n12, n22 = pair_norms(alpha_bar[a], alpha_bar[b], V[a], V[b], o_bar)
    else:
        A, O = window_attention(Q_heads, K, V, log_n, length, W)
        n11, n12, n22 = pair_norms_per_query(A, O, V[:length], a, b)
    w_b, score, degen, D = weight_and_score(n11, n12, n22, K[a], K[b], form)
    return HeadScores(score=score, w_b=w_b, n11=n11, n12=n12, n22=n22, D=D,
                      degenerate=degen, alpha_bar=alpha_bar, o_bar=o_bar)


def select_pairs(score, R):
    """Boolean mask of the R entries with the smallest (score, index); NaN
    counts as +inf (reading R3)."""
    score = np.asarray(score, dtype=np.float64)
    n = score.shape[0]
    if R < 0 or R > n:
        raise ValueError(f"cannot select {R} of {n} pairs")
    key = np.where(np.isnan(score), np.inf, score)
    order = np.lexsort((np.arange(n), key))
    mask = np.zeros(n, dtype=bool)
    mask[order[:R]] = True
    return mask


@dataclass
class HeadMerge:
    K: np.ndarray
    V: np.ndarray
    log_n: np.ndarray
    length: int
    out_offset: np.ndarray      # output row of each pair's first (or merged) token
    k_merged: np.ndarray        # (P, d) merged keys (rows of unselected pairs are zero)


def merge_compact_head(K, V, log_n, length, cand_begin, n_recent, selected, w_b, storage="f64"):
    """Merge the selected pairs and compact one KV head, order preserved.

    Selected pair (a, b):  k* = k_a + w_b (k_b - k_a)      ([KVS] §数学主线四, reading R7)
                           v* = (n_a v_a + n_b v_b) / (n_a + n_b),
                           log n* = log(n_a + n_b)          (reading R5)
    Unselected pairs, protected prefix [0, c0), the odd leftover and the
    recent suffix are copied unchanged. Merged rows are rounded to `storage`
    (reading R9); ``k_merged`` keeps the unrounded fp64 keys.
    """
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    d = K.shape[1]
    ln = np.zeros(length) if log_n is None else np.asarray(log_n, dtype=np.float64)[:length]
    selected = np.asarray(selected, dtype=bool)
    P = selected.shape[0]
    c0 = int(cand_begin)
    out_K, out_V, out_ln = [], [], []
    out_offset = np.zeros(P, dtype=np.int64)
    k_merged = np.zeros((P, d))
    for t in range(min(c0, length)):
        out_K.append(K[t]); out_V.append(V[t]); out_ln.append(ln[t])
    for p in range(P):
        a, b = c0 + 2 * p, c0 + 2 * p + 1
        out_offset[p] = len(out_K)
        if selected[p]:
            k_star = K[a] + w_b[p] * (K[b] - K[a])
            n_a, n_b = math.exp(ln[a]), math.exp(ln[b])
            v_star = (n_a * V[a] + n_b * V[b]) / (n_a + n_b)
            k_merged[p] = k_star
            out_K.append(storage_round(k_star, storage))
            out_V.append(storage_round(v_star, storage))
            out_ln.append(float(storage_round(math.log(n_a + n_b), "f64" if storage == "f64" else "f32")))
        else:
            out_K.extend([K[a], K[b]]); out_V.extend([V[a], V[b]]); out_ln.extend([ln[a], ln[b]])
    for t in range(max(c0, 0) + 2 * P, length):
        out_K.append(K[t]); out_V.append(V[t]); out_ln.append(ln[t])
    n_out = len(out_K)
    return HeadMerge(K=np.array(out_K).reshape(n_out, d), V=np.array(out_V).reshape(n_out, d),
                     log_n=np.array(out_ln), length=n_out, out_offset=out_offset,
                     k_merged=k_merged)


# ---------------------------------------------------------------------------
# Whole caches [B, H_kv, T, d]: one round, the round driver, decode
# ---------------------------------------------------------------------------

@dataclass
class Cache:
    """A ragged cache in fp64: per (b, h) a (len, d) key/value array and log counts."""

    K: List[List[np.ndarray]]
    V: List[List[np.ndarray]]
    log_n: List[List[np.ndarray]]

    @property
    def B(self):
        return len(self.K)

    @property
    def H(self):
        return len(self.K[0])

    def length(self, b, h):
        return self.K[b][h].shape[0]

    def lengths(self):
        return np.array([[self.length(b, h) for h in range(self.H)] for b in range(self.B)])


def cache_from_arrays(K, V, lens, log_n=None):
    """Build a Cache from [B, H, T_cap, d] arrays and [B, H] lengths."""
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    lens = np.asarray(lens)
    B, H = lens.shape
    Ks, Vs, Ls = [], [], []
    for b in range(B):
        Ks.append([K[b, h, :lens[b, h]].copy() for h in range(H)])
        Vs.append([V[b, h, :lens[b, h]].copy() for h in range(H)])
        if log_n is None:
            Ls.append([np.zeros(lens[b, h]) for h in range(H)])
        else:
            Ls.append([np.asarray(log_n, dtype=np.float64)[b, h, :lens[b, h]].copy()
                       for h in range(H)])
    return Cache(Ks, Vs, Ls)


@dataclass
class RoundResult:
    cache: Cache
    scores: List[List[HeadScores]]
    selected: List[List[np.ndarray]]
    merges: List[List[HeadMerge]]
    R: np.ndarray                 # pairs merged per unit


def merge_round(cache, Q_win, W, cand_begin, n_recent, target, scope="head", storage="f64",
                form="full", stats="mean"):
    """One scoring + selection + merge round over a whole cache.

    Q_win: (B, H_q, W, d); query head hq belongs to KV head hq // G.
    cand_begin: (B, H) candidate-span starts; target: (B, H) for per-head
    scope or (B,) for pooled scope (total tokens of sequence b over its heads).
    Each unit merges R = min(P, max(0, len - target)) pairs (reading R4).
    """
    Q_win = np.asarray(Q_win, dtype=np.float64)
    B, H = cache.B, cache.H
    G = Q_win.shape[1] // H
    cand_begin = np.asarray(cand_begin).reshape(B, H)
    scores = [[score_head(cache.K[b][h], cache.V[b][h], cache.log_n[b][h], cache.length(b, h),
                          cand_begin[b, h], n_recent, Q_win[b, h * G:(h + 1) * G], W, form,
                          stats)
               for h in range(H)] for b in range(B)]
    selected = [[None] * H for _ in range(B)]
    if scope == "head":
        target = np.asarray(target).reshape(B, H)
        R = np.zeros((B, H), dtype=np.int64)
        for b in range(B):
            for h in range(H):
                P = scores[b][h].score.shape[0]
                R[b, h] = min(P, max(0, cache.length(b, h) - int(target[b, h])))
                selected[b][h] = select_pairs(scores[b][h].score, int(R[b, h]))
    elif scope == "pooled":
        target = np.asarray(target).reshape(B)
        R = np.zeros(B, dtype=np.int64)
        for b in range(B):
            pooled = np.concatenate([scores[b][h].score for h in range(H)])
            total = sum(cache.length(b, h) for h in range(H))
            R[b] = min(pooled.shape[0], max(0, total - int(target[b])))
            mask = select_pairs(pooled, int(R[b]))
            start = 0
            for h in range(H):
                P = scores[b][h].score.shape[0]
                selected[b][h] = mask[start:start + P]
                start += P
    else:
        raise ValueError(scope)
    merges = [[merge_compact_head(cache.K[b][h], cache.V[b][h], cache.log_n[b][h],
                                  cache.length(b, h), cand_begin[b, h], n_recent,
                                  selected[b][h], scores[b][h].w_b, storage)
               for h in range(H)] for b in range(B)]
    out = Cache([[m.K for m in row] for row in merges], [[m.V for m in row] for row in merges],
                [[m.log_n for m in row] for row in merges])
    return RoundResult(cache=out, scores=scores, selected=selected, merges=merges, R=R)


def compress(cache, Q_win, W, cand_begin, n_recent, target, scope="head", max_rounds=64,
             storage="f64", form="full", stats="mean"):
    """Repeat merge rounds until every unit reaches its budget exactly (reading R4)."""
    rounds = []
    for _ in range(max_rounds):
        lens = cache.lengths()
        if scope == "head":
            done = np.all(lens == np.asarray(target).reshape(lens.shape))
        else:
            done = np.all(lens.sum(axis=1) == np.asarray(target).reshape(-1))
        if done:
            return cache, rounds
        r = merge_round(cache, Q_win, W, cand_begin, n_recent, target, scope, storage, form,
                        stats)
        if np.all(r.R == 0):
            raise ValueError("budget unreachable: no candidate pairs left")
        rounds.append(r)
        cache = r.cache
    raise ValueError("budget not reached within max_rounds")


def decode_attention(q_heads, K, V, log_n, length):
    """out_g = sum_t softmax_t(q_g k_t^T / sqrt(d) + log n_t) v_t for the G
    query heads sharing one KV head ([KVS] §数学主线三 attention, reading R5 bias)."""
    q_heads = np.asarray(q_heads, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)[:length]
    V = np.asarray(V, dtype=np.float64)[:length]
    if length == 0:   # reading R10: attention over no rows is the zero vector
        return np.zeros_like(q_heads)
    ln = None if log_n is None else np.asarray(log_n, dtype=np.float64)[:length]
    return np.array([attention_output(softmax(attention_logits(q, K, ln)), V) for q in q_heads])


def decode_step(cache, q, k_new=None, v_new=None):
    """Append (k_new, v_new) with count 1 to every head, then attend.

    q: (B, H_q, d); k_new, v_new: (B, H, d) or None. Returns ((B, H_q, d), cache).
    """
    q = np.asarray(q, dtype=np.float64)
    B, H = cache.B, cache.H
    G = q.shape[1] // H
    if k_new is not None:
        k_new = np.asarray(k_new, dtype=np.float64)
        v_new = np.asarray(v_new, dtype=np.float64)
        for b in range(B):
            for h in range(H):
                cache.K[b][h] = np.vstack([cache.K[b][h], k_new[b, h][None]])
                cache.V[b][h] = np.vstack([cache.V[b][h], v_new[b, h][None]])
                cache.log_n[b][h] = np.append(cache.log_n[b][h], 0.0)
    out = np.zeros((B, q.shape[1], q.shape[2]))
    for b in range(B):
        for h in range(H):
            out[b, h * G:(h + 1) * G] = decode_attention(
                q[b, h * G:(h + 1) * G], cache.K[b][h], cache.V[b][h], cache.log_n[b][h],
                cache.length(b, h))
    return out, cache


def append_rows(cache, k_rows, v_rows):
    """Append n rows with count 1 (log n = 0) to every head; k_rows, v_rows (B, H, n, d).
    Returns a new Cache (the input is not modified)."""
    k_rows = np.asarray(k_rows, dtype=np.float64)
    v_rows = np.asarray(v_rows, dtype=np.float64)
    B, H = cache.B, cache.H
    n = k_rows.shape[2]
    return Cache([[np.vstack([cache.K[b][h], k_rows[b, h]]) for h in range(H)] for b in range(B)],
                 [[np.vstack([cache.V[b][h], v_rows[b, h]]) for h in range(H)] for b in range(B)],
                 [[np.append(cache.log_n[b][h], np.zeros(n)) for h in range(H)] for b in range(B)])


def prefill_chunk(cache, k_chunk, v_chunk, Q_win, W, budget, sink, storage="f64", form="full"):
    """One step of chunked streaming prefill compression ([KVS] §实验设置: context budget,
    chunk size and preserved initial tokens; reading R11): append the chunk to every head,
    then run merge rounds on heads longer than `budget` -- candidate span [sink, len - W),
    window queries Q_win (the chunk's last W positions), per-head target budget -- until
    every head holds min(len, budget) rows. Returns (cache, rounds)."""
    cache = append_rows(cache, k_chunk, v_chunk)
    lens = cache.lengths()
    target = np.minimum(lens, int(budget))
    cand = np.full(lens.shape, int(sink))
    return compress(cache, Q_win, W, cand, W, target, "head", storage=storage, form=form)


def budget(length, ratio):
    """Per-head token budget floor(len / ratio)."""
    return int(length) // int(ratio)
