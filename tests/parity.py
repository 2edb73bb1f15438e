"""Helpers for the GPU-vs-oracle parity tests.

Every comparison runs both sides on identical inputs: before each merge round the
oracle's cache is re-read from the GPU's cache (the rows the GPU stored, widened to
fp64), so a one-ulp difference in a stored row can never carry into a later round.

Tolerances (GPU arithmetic is fp32; the oracle is fp64):
  * selection flags and compaction offsets: bit-exact, except pairs whose oracle
    score is within 1e-5 relative of the unit's selection threshold; those are
    counted, the GPU's choice is checked to be a valid smallest-R selection under
    that tolerance, and the round is then compared against the oracle's merge of
    the GPU's own selection;
  * merged keys before rounding (fp32 debug output): per-row |dk| / |k| <= 1e-4;
  * copied rows: bit-exact; stored merged bf16 rows and bf16 decode outputs:
    |d| <= 1e-2 + 2e-2 |ref|; fp32 caches: merged rows per-row relative 1e-4,
    decode outputs 1e-4 + 1e-4 |ref|;
  * scores: relative 2e-4 and weights absolute 2e-4. A pair whose D sits within a
    factor 2 of the degenerate threshold 1e-6 (N11 + N22) may take either branch
    (a one-ulp change flips it); its score and weight must match the branch taken.
    The score is a product of ~10 fp32 operations on window statistics that are sums
    over up to 131072 rows; with fp32's 6e-8 unit roundoff and the statistics'
    blockwise summation the observed relative error stays near 1e-6, and 2e-4 leaves
    room for the cancellation in D = N11 - 2 N12 + N22.

Each test records its counts in REPORTS; tests/conftest.py prints one JSON line per
test at the end of the run, so the counts survive `pytest -q`.
"""

from __future__ import annotations

from dataclasses import asdict, dataclass

import numpy as np
import torch

import oracle
from asymmetric_kv_merging_b200 import kvs

NEAR_REL = 1e-5
REPORTS: list = []


@dataclass
class Stats:
    rounds: int = 0
    heads_compared: int = 0
    scores_compared: int = 0
    degenerate_pairs: int = 0        # the oracle took the plain-average branch
    degenerate_boundary: int = 0     # D within 2x of the branch threshold: either branch
    alpha_over_half: int = 0         # candidate rows with alpha_bar > 1/2
    extrapolating: int = 0           # pairs whose w_b lies outside [0, 1] (used as printed)
    selected: int = 0
    near_threshold: int = 0          # selection differences within 1e-5 of the threshold
    merged_compared: int = 0
    rows_compared: int = 0
    decode_steps: int = 0
    decode_outputs: int = 0
    max_score_rel: float = 0.0
    max_kmerged_rel: float = 0.0
    max_decode_err: float = 0.0      # max |d| / (atol + rtol |ref|) over decode outputs

    def report(self, name):
        line = dict(test=name, **asdict(self))
        REPORTS.append(line)
        return line


def storage_of(dtype: torch.dtype) -> str:
    return "bf16" if dtype == torch.bfloat16 else "f32"


class GpuCache:
    """A device cache [B, H_kv, T_cap, d] with lengths and log counts."""

    def __init__(self, K, V, lens, logn=None):
        self.K = K.contiguous()
        self.V = V.contiguous()
        self.lens = lens.reshape(-1).to(torch.int32).contiguous()
        B, H, T_cap, _ = K.shape
        self.logn = (logn if logn is not None
                     else torch.zeros(B, H, T_cap, dtype=torch.float32, device=K.device)).contiguous()

    @property
    def shape(self):
        return self.K.shape

    def clone(self):
        return GpuCache(self.K.clone(), self.V.clone(), self.lens.clone(), self.logn.clone())


def gpu_round(cache: GpuCache, H_q, Q_win, W, cand_begin, n_recent, target, scope, ws,
              T_cap_out=None, inplace=False, form=None):
    B, H, T_cap, d = cache.K.shape
    dev = cache.K.device
    desc = kvs.make_desc(B, H, H_q, d, T_cap, cache.K.dtype)
    npair = T_cap // 2
    score = torch.full((B, H, npair), float("nan"), dtype=torch.float32, device=dev)
    w_b = torch.full_like(score, float("nan"))
    kvs.score_pairs(desc, cache.K, cache.V, cache.logn, cache.lens, cand_begin, n_recent,
                    Q_win.contiguous(), W, score, w_b, ws, form=form)
    sel = torch.zeros(B, H, npair, dtype=torch.uint8, device=dev)
    off = torch.full((B, H, npair), -1, dtype=torch.int32, device=dev)
    km = torch.zeros(B, H, npair, d, dtype=torch.float32, device=dev)
    if inplace:
        out = cache
        kvs.merge_compact(desc, cache.K, cache.V, cache.logn, cache.lens, cand_begin, n_recent,
                          score, w_b, target, scope, T_cap, cache.K, cache.V, cache.logn,
                          cache.lens, ws, sel, off, km)
    else:
        T_out = T_cap_out or T_cap
        out = GpuCache(torch.zeros(B, H, T_out, d, dtype=cache.K.dtype, device=dev),
                       torch.zeros(B, H, T_out, d, dtype=cache.K.dtype, device=dev),
                       torch.zeros(B * H, dtype=torch.int32, device=dev),
                       torch.zeros(B, H, T_out, dtype=torch.float32, device=dev))
        kvs.merge_compact(desc, cache.K, cache.V, cache.logn, cache.lens, cand_begin, n_recent,
                          score, w_b, target, scope, T_out, out.K, out.V, out.logn, out.lens, ws,
                          sel, off, km)
    torch.cuda.synchronize()
    return out, dict(score=score.cpu().double(), w_b=w_b.cpu().double(), sel=sel.cpu().bool(),
                     off=off.cpu().long(), km=km.cpu().double())


def _rows(cache: GpuCache, bs):
    """fp64 copies of sequences `bs` of a device cache, trimmed to their longest head:
    (K, V, logn, lens)."""
    B, H = cache.K.shape[:2]
    lens = cache.lens.view(B, H).cpu().numpy()[bs]
    n = max(1, int(lens.max(initial=0)))
    idx = torch.tensor(bs, dtype=torch.long, device=cache.K.device)
    K = cache.K.index_select(0, idx)[:, :, :n].double().cpu().numpy()
    V = cache.V.index_select(0, idx)[:, :, :n].double().cpu().numpy()
    ln = cache.logn.index_select(0, idx)[:, :, :n].double().cpu().numpy()
    return K, V, ln, lens


def to_oracle_cache(cache: GpuCache, batch=None):
    """Copy (sequences `batch` of) a device cache to an oracle Cache (fp64)."""
    bs = list(range(cache.K.shape[0])) if batch is None else list(batch)
    K, V, ln, lens = _rows(cache, bs)
    return oracle.cache_from_arrays(K, V, lens, ln)


def _nan_inf(x):
    return np.where(np.isnan(x), np.inf, x)


def _unit_threshold(r, b, h, scope):
    """Largest oracle score among the oracle's selected pairs of the unit (None: none)."""
    if scope == "pooled":
        sc = np.concatenate([r.scores[b][hh].score for hh in range(len(r.scores[b]))])
        sl = np.concatenate([r.selected[b][hh] for hh in range(len(r.selected[b]))])
    else:
        sc, sl = r.scores[b][h].score, r.selected[b][h]
    if not sl.any():
        return None
    return _nan_inf(sc)[sl].max()


def _check_scores(hs, sg, wg, dd, form, stats, where):
    """GPU score / weight of every pair against the oracle; pairs at the degenerate
    boundary may match either branch."""
    P = hs.score.shape[0]
    if P == 0:
        return
    n11, n12, n22 = hs.n11, hs.n12, hs.n22
    if form == "diagonal":
        n12 = np.zeros_like(n12)
        ratio = np.full(P, np.inf)
        boundary = np.zeros(P, bool)
    else:
        with np.errstate(invalid="ignore", divide="ignore"):
            ratio = hs.D / (n11 + n22)
        boundary = ~np.isfinite(ratio) | ((ratio > 0.5e-6) & (ratio < 2e-6))
    stats.degenerate_pairs += int(hs.degenerate.sum())
    stats.degenerate_boundary += int(boundary.sum())
    stats.extrapolating += int(((hs.w_b < 0.0) | (hs.w_b > 1.0)).sum())
    strict = ~boundary
    scale = np.max(np.abs(hs.score[np.isfinite(hs.score)]), initial=0.0)
    np.testing.assert_allclose(sg[strict], hs.score[strict], rtol=2e-4, atol=1e-7 * scale,
                               err_msg=f"score {where}")
    np.testing.assert_allclose(wg[strict], hs.w_b[strict], rtol=0, atol=2e-4,
                               err_msg=f"w_b {where}")
    ok = strict & np.isfinite(hs.score) & (hs.score != 0)
    if ok.any():
        rel = np.abs(sg[ok] - hs.score[ok]) / np.abs(hs.score[ok])
        stats.max_score_rel = max(stats.max_score_rel, float(rel.max()))
    if boundary.any():
        # both branches of the oracle's own terms, in fp64
        Dn = n11 - 2.0 * n12 + n22
        with np.errstate(invalid="ignore", divide="ignore"):
            w_full = (n22 - n12) / Dn
            s_full = dd * (n11 * n22 - n12 * n12) / Dn
        w_avg = np.full(P, 0.5)
        s_avg = dd * (n11 + 2.0 * n12 + n22) / 4.0
        for i in np.flatnonzero(boundary):
            tol = lambda a, b, rt: abs(a - b) <= rt * abs(b) + 1e-7 * scale  # noqa: E731
            full_ok = (np.isfinite(s_full[i]) and tol(sg[i], s_full[i], 2e-4)
                       and abs(wg[i] - w_full[i]) <= 2e-4)
            avg_ok = tol(sg[i], s_avg[i], 2e-4) and wg[i] == 0.5
            assert full_ok or avg_ok, (f"boundary pair {i} {where}: gpu ({sg[i]}, {wg[i]}) "
                                       f"full ({s_full[i]}, {w_full[i]}) avg ({s_avg[i]}, 0.5)")
    stats.scores_compared += P


def compare_round(r, g, out: GpuCache, oin, dtype, scope="head", batch_map=None, stats=None,
                  cand_begin=None, n_recent=0, form="full"):
    """Compare one oracle round with one GPU round, head by head.

    r: oracle.merge_round on `oin`, an oracle copy of the GPU cache the round started
    from (identical inputs). g: the GPU round's debug outputs; out: its output cache.
    cand_begin: (B_o, H) candidate starts of the oracle's sequences; n_recent as passed.
    batch_map: oracle batch index -> GPU batch index (oracle run on a subset).
    """
    stats = stats or Stats()
    storage = storage_of(dtype)
    B_o = len(r.scores)
    H = len(r.scores[0])
    gb = [bo if batch_map is None else batch_map[bo] for bo in range(B_o)]
    Kg, Vg, Lg, lens_g = _rows(out, gb)           # indexed by the oracle's sequence index
    stats.rounds += 1
    # selection per unit: differences only near the threshold, same count per unit
    sel_g_all = {}
    for bo in range(B_o):
        bg = bo if batch_map is None else batch_map[bo]
        units = [list(range(H))] if scope == "pooled" else [[h] for h in range(H)]
        for heads in units:
            n_o = n_g = 0
            for h in heads:
                P = r.scores[bo][h].score.shape[0]
                sel_o = r.selected[bo][h]
                sel_g = g["sel"][bg, h, :P].numpy()
                sel_g_all[(bo, h)] = sel_g
                n_o += int(sel_o.sum())
                n_g += int(sel_g.sum())
                diff = sel_o != sel_g
                if diff.any():
                    thr = _unit_threshold(r, bo, h, scope)
                    assert thr is not None, f"GPU merged pairs the oracle did not b={bg} h={h}"
                    sc = _nan_inf(r.scores[bo][h].score)
                    near = np.abs(sc[diff] - thr) <= NEAR_REL * abs(thr)
                    assert near.all(), (f"selection differs away from the threshold b={bg} h={h}: "
                                        f"{np.flatnonzero(diff)[~near][:8]}")
                    # the GPU's choice is a smallest-R selection within the tolerance
                    lo, hi = thr - NEAR_REL * abs(thr), thr + NEAR_REL * abs(thr)
                    assert np.all(sc[sel_g] <= hi) and np.all(sc[~sel_g] >= lo)
                    stats.near_threshold += int(diff.sum())
            assert n_o == n_g, f"merged-pair count differs b={bg} heads={heads}: {n_g} vs {n_o}"
            stats.selected += n_g
    for bo in range(B_o):
        bg = bo if batch_map is None else batch_map[bo]
        for h in range(H):
            hs = r.scores[bo][h]
            P = hs.score.shape[0]
            L_in = oin.length(bo, h)
            c0 = int(cand_begin[bo, h]) if cand_begin is not None else (
                r.merges[bo][h].out_offset[0] if P else 0)
            a_rows = c0 + 2 * np.arange(P)
            Kin, Vin = oin.K[bo][h], oin.V[bo][h]
            dd = np.sum((Kin[a_rows + 1] - Kin[a_rows]) ** 2, axis=1) if P else np.zeros(0)
            _check_scores(hs, g["score"][bg, h, :P].numpy(), g["w_b"][bg, h, :P].numpy(), dd,
                          form, stats, f"b={bg} h={h}")
            if P:
                stats.alpha_over_half += int((hs.alpha_bar[c0:c0 + 2 * P] > 0.5).sum())
            sel_g = sel_g_all[(bo, h)]
            if np.array_equal(sel_g, r.selected[bo][h]):
                m = r.merges[bo][h]
            else:   # near-threshold swap: the oracle's merge of the GPU's selection
                m = oracle.merge_compact_head(Kin, Vin, oin.log_n[bo][h], L_in, c0, n_recent,
                                              sel_g, hs.w_b, storage)
            assert lens_g[bo, h] == m.length, (bg, h, lens_g[bo, h], m.length)
            np.testing.assert_array_equal(g["off"][bg, h, :P].numpy(), m.out_offset,
                                          err_msg=f"offsets b={bg} h={h}")
            n = m.length
            merged = np.zeros(n, bool)
            merged[m.out_offset[sel_g]] = True
            kg, vg = Kg[bo, h, :n], Vg[bo, h, :n]
            np.testing.assert_array_equal(kg[~merged], m.K[~merged], err_msg=f"K copy b={bg} h={h}")
            np.testing.assert_array_equal(vg[~merged], m.V[~merged], err_msg=f"V copy b={bg} h={h}")
            np.testing.assert_allclose(Lg[bo, h, :n], m.log_n, rtol=0, atol=2e-6,
                                       err_msg=f"logn b={bg} h={h}")
            if storage == "bf16":
                np.testing.assert_allclose(kg[merged], m.K[merged], rtol=2e-2, atol=1e-2)
                np.testing.assert_allclose(vg[merged], m.V[merged], rtol=2e-2, atol=1e-2)
            else:
                for a, o in ((kg[merged], m.K[merged]), (vg[merged], m.V[merged])):
                    if a.size:
                        rel = np.linalg.norm(a - o, axis=1) / np.maximum(np.linalg.norm(o, axis=1), 1e-30)
                        assert rel.max() <= 1e-4, f"merged rows rel {rel.max()} b={bg} h={h}"
            if sel_g.any():
                kmg = g["km"][bg, h, :P].numpy()[sel_g]
                kmo = m.k_merged[sel_g]
                rel = np.linalg.norm(kmg - kmo, axis=1) / np.maximum(np.linalg.norm(kmo, axis=1), 1e-30)
                assert rel.max() <= 1e-4, f"merged key rel {rel.max()} b={bg} h={h}"
                stats.max_kmerged_rel = max(stats.max_kmerged_rel, float(rel.max()))
                stats.merged_compared += int(sel_g.sum())
            stats.rows_compared += n
            stats.heads_compared += 1
    return stats


def compare_decode(out_o, out_g, dtype, stats=None, batch_map=None):
    """out_o: (B_o, H_q, d) oracle; out_g: (B, H_q, d) torch."""
    stats = stats or Stats()
    og = out_g.double().cpu().numpy()
    rtol, atol = (2e-2, 1e-2) if dtype == torch.bfloat16 else (1e-4, 1e-4)
    for bo in range(out_o.shape[0]):
        bg = bo if batch_map is None else batch_map[bo]
        np.testing.assert_allclose(og[bg], out_o[bo], rtol=rtol, atol=atol,
                                   err_msg=f"decode b={bg}")
        err = np.abs(og[bg] - out_o[bo]) / (atol + rtol * np.abs(out_o[bo]))
        stats.max_decode_err = max(stats.max_decode_err, float(err.max(initial=0.0)))
        stats.decode_outputs += out_o.shape[1]
    stats.decode_steps += 1
    return stats


def assert_same_rows(g: GpuCache, o, batch=None):
    """The GPU cache holds exactly the oracle cache's rows (lengths, K, V, log counts)."""
    oc = to_oracle_cache(g, batch)
    assert np.array_equal(oc.lengths(), o.lengths())
    for b in range(o.B):
        for h in range(o.H):
            assert np.array_equal(oc.K[b][h], o.K[b][h])
            assert np.array_equal(oc.V[b][h], o.V[b][h])
            np.testing.assert_allclose(oc.log_n[b][h], o.log_n[b][h], rtol=0, atol=0)
