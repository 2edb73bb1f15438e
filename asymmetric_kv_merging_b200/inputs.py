"""Seeded synthetic workloads for asymmetric KV merging.

This module only draws inputs. It holds none of the merging arithmetic, and it
is the one module that both the CUDA path's callers (tests, bench, smoke) and
the CPU oracle's callers share.

Recipe (per layer):
  * hidden states follow an AR(1) process over tokens,
        x_0 = eps_0 / sqrt(1 - rho^2),   x_t = rho * x_{t-1} + eps_t,   eps ~ N(0, I_dmodel);
  * W_K (one per KV head) and W_Q (one per query head) are U diag(s) V^T with
    U (d_model x d) and V (d x d) random orthogonal (QR of a Gaussian, sign fixed)
    and singular values s_i = i^-1.5: the concentrated spectrum the KVSlimmer
    deep dive ("论文专题讲解：KVSlimmer：非对称 KV 合并的数学与工程", §数学主线一)
    attributes to Q/K projections;
  * W_V (one per KV head) has flat singular values (s_i = 1), the dispersed
    spectrum the same section attributes to V projections;
  * K = x W_K, V = x W_V for the T prefill tokens; the observation window is
    the last W prefill rows of x times W_Q; decode steps continue the same
    hidden process (row T + s gives the step-s query, key and value).

The pages measure on trained models with LongBench; those are not available,
so these seeded tensors stand in for them with the shapes of the pages'
Llama-3.1-8B / Mistral-7B setting.

Seeds: config i uses seed i for its shape draws; layer l of config i uses
seed 1000*i + l (config 0, layer 0 uses seed 0).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Tuple

import torch


@dataclass(frozen=True)
class Workload:
    """Shape and schedule of one synthetic workload."""

    name: str
    index: int
    B: int
    layers: int
    H_kv: int
    H_q: int
    d: int
    T: int                      # prefill tokens per sequence (max when lengths vary)
    dtype: str                  # "f32" or "bf16"
    d_model: int
    rho: Tuple[float, float]    # AR(1) coefficient, or the [lo, hi) range drawn per layer
    W: int                      # observation window (recent queries)
    ratio: int                  # compression ratio: budget = floor(len / ratio) per head
    scope: str                  # "head" (budget per KV head) or "pooled" (per sequence)
    n_decode: int               # decode steps after compression
    remerge_every: int = 0      # re-merge the newest segment every this many steps (0: never)
    remerge_ratio: int = 8
    len_range: Optional[Tuple[int, int]] = None   # per-sequence prefill lengths U{lo..hi}
    sink: int = 32              # protected initial tokens
    description: str = ""

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def T_cap(self) -> int:
        """Cache capacity: prefill plus room for every decode append, rounded up to even."""
        c = self.T + self.n_decode
        return c + c % 2


WORKLOADS = [
    Workload("tiny_fp32_T512", 0, B=1, layers=1, H_kv=2, H_q=4, d=64, T=512, dtype="f32",
             d_model=256, rho=(0.9, 0.9), W=32, ratio=2, scope="head", n_decode=8,
             description="tiny CPU-checkable case, fp32"),
    Workload("llama8b_layer_T32K", 1, B=1, layers=1, H_kv=8, H_q=32, d=128, T=32768, dtype="bf16",
             d_model=4096, rho=(0.9, 0.9), W=32, ratio=2, scope="head", n_decode=128,
             description="Llama-3.1-8B single layer, 32K tokens, 2x"),
    Workload("llama8b_32L_T128K", 2, B=1, layers=32, H_kv=8, H_q=32, d=128, T=131072, dtype="bf16",
             d_model=4096, rho=(0.7, 0.95), W=32, ratio=4, scope="head", n_decode=128,
             description="Llama-3.1-8B full depth, 128K tokens, 4x"),
    Workload("mistral7b_32L_B8_T32K_pooled", 3, B=8, layers=32, H_kv=8, H_q=32, d=128, T=32768,
             dtype="bf16", d_model=4096, rho=(0.85, 0.85), W=32, ratio=2, scope="pooled",
             n_decode=1, description="Mistral-7B shapes, batch 8, pooled budget per sequence"),
    Workload("serving_B16_8K_64K", 4, B=16, layers=1, H_kv=8, H_q=32, d=128, T=65536, dtype="bf16",
             d_model=4096, rho=(0.9, 0.9), W=32, ratio=8, scope="head", n_decode=256,
             remerge_every=64, len_range=(8192, 65536),
             description="decode-heavy serving mix, ragged lengths, re-merge every 64 steps"),
]


def workload(i: int) -> Workload:
    return WORKLOADS[i]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def random_orthogonal(rows: int, cols: int, gen: torch.Generator, device) -> torch.Tensor:
    """rows x cols matrix with orthonormal columns (QR of a Gaussian, sign fixed)."""
    a = torch.randn(rows, cols, generator=gen, device=device, dtype=torch.float64)
    q, r = torch.linalg.qr(a)
    sign = torch.sign(torch.diagonal(r))
    sign[sign == 0] = 1.0
    return q * sign.unsqueeze(0)


def projection(d_model: int, d: int, flat: bool, gen: torch.Generator, device) -> torch.Tensor:
    """d_model x d projection U diag(s) V^T; s_i = i^-1.5 (decaying) or 1 (flat)."""
    u = random_orthogonal(d_model, d, gen, device)
    v = random_orthogonal(d, d, gen, device)
    if flat:
        s = torch.ones(d, dtype=torch.float64, device=device)
    else:
        s = torch.arange(1, d + 1, dtype=torch.float64, device=device) ** -1.5
    return (u * s.unsqueeze(0)) @ v.T


def ar1_hidden(T: int, d_model: int, rho: float, gen: torch.Generator, device,
               chunk: int = 256) -> torch.Tensor:
    """T x d_model stationary AR(1) hidden states (fp32).

    Evaluated chunk by chunk: inside a chunk the recurrence is a lower-triangular
    Toeplitz product with rho^(i-j); the previous chunk's last state enters
    through rho^(i+1).
    """
    eps = torch.randn(T, d_model, generator=gen, device=device, dtype=torch.float32)
    eps[0] *= 1.0 / math.sqrt(1.0 - rho * rho)
    n_chunks = (T + chunk - 1) // chunk
    pad = n_chunks * chunk - T
    if pad:
        eps = torch.cat([eps, torch.zeros(pad, d_model, device=device, dtype=torch.float32)])
    i = torch.arange(chunk, device=device, dtype=torch.float64)
    diff = i[:, None] - i[None, :]
    lower = torch.where(diff >= 0, torch.pow(torch.tensor(rho, dtype=torch.float64, device=device),
                                             diff.clamp(min=0)), torch.zeros_like(diff))
    lower = lower.to(torch.float32)
    y = torch.matmul(lower, eps.view(n_chunks, chunk, d_model))
    decay = (rho ** (i + 1)).to(torch.float32).unsqueeze(1)
    carry = torch.zeros(d_model, device=device, dtype=torch.float32)
    for c in range(n_chunks):
        if c:
            y[c] += decay * carry.unsqueeze(0)
        carry = y[c, -1].clone()
    return y.view(n_chunks * chunk, d_model)[:T]


def sequence_lengths(w: Workload, device="cpu") -> torch.Tensor:
    """Prefill length per sequence (int64, [B])."""
    if w.len_range is None:
        return torch.full((w.B,), w.T, dtype=torch.int64)
    g = _gen(w.index, "cpu")
    lo, hi = w.len_range
    return torch.randint(lo, hi + 1, (w.B,), generator=g, dtype=torch.int64)


def layer_rho(w: Workload, layer: int) -> float:
    lo, hi = w.rho
    if lo == hi:
        return lo
    g = _gen(1000 * w.index + layer, "cpu")
    return float(lo + (hi - lo) * torch.rand((), generator=g, dtype=torch.float64))


@dataclass
class LayerInputs:
    """One layer's tensors, cache layout [B, H_kv, T_cap, d] (row-major)."""

    K: torch.Tensor            # [B, H_kv, T_cap, d]
    V: torch.Tensor            # [B, H_kv, T_cap, d]
    lens: torch.Tensor         # [B, H_kv] int32 prefill lengths
    Q_win: torch.Tensor        # [B, H_q, W, d]
    q_dec: torch.Tensor        # [n_decode, B, H_q, d]
    k_new: torch.Tensor        # [n_decode, B, H_kv, d]
    v_new: torch.Tensor        # [n_decode, B, H_kv, d]
    rho: float = 0.0
    extra: dict = field(default_factory=dict)


def make_layer(w: Workload, layer: int = 0, device="cpu", T_cap: Optional[int] = None,
               lens: Optional[torch.Tensor] = None, q_scale: float = 1.0,
               window_ends: Optional[list] = None) -> LayerInputs:
    """Draw one layer of workload `w` on `device`.

    `q_scale` multiplies the queries (window and decode); values above 1 give
    peaked attention, a regime the default recipe does not reach.
    `window_ends` (positions e >= W, all <= the prefill length): also draw the W
    queries ending at each e, as extra["Q_ends"] [len(window_ends), B, H_q, W, d]
    (the window queries of a chunked prefill).
    """
    device = torch.device(device)
    gen = _gen(1000 * w.index + layer, device)
    rho = layer_rho(w, layer)
    if lens is None:
        lens = sequence_lengths(w)
    T_cap = T_cap if T_cap is not None else int(lens.max()) + w.n_decode
    T_cap += T_cap % 2            # caches hold an even number of rows (whole pairs)
    dt = w.torch_dtype
    W_K = [projection(w.d_model, w.d, False, gen, device) for _ in range(w.H_kv)]
    W_V = [projection(w.d_model, w.d, True, gen, device) for _ in range(w.H_kv)]
    W_Q = [projection(w.d_model, w.d, False, gen, device) for _ in range(w.H_q)]
    WK = torch.cat(W_K, dim=1).to(torch.float32)      # d_model x H_kv*d
    WV = torch.cat(W_V, dim=1).to(torch.float32)
    WQ = torch.cat(W_Q, dim=1).to(torch.float32)      # d_model x H_q*d

    K = torch.zeros(w.B, w.H_kv, T_cap, w.d, dtype=dt, device=device)
    V = torch.zeros_like(K)
    Q_win = torch.zeros(w.B, w.H_q, w.W, w.d, dtype=dt, device=device)
    q_dec = torch.zeros(w.n_decode, w.B, w.H_q, w.d, dtype=dt, device=device)
    k_new = torch.zeros(w.n_decode, w.B, w.H_kv, w.d, dtype=dt, device=device)
    v_new = torch.zeros_like(k_new)
    ends = list(window_ends or [])
    Q_ends = torch.zeros(len(ends), w.B, w.H_q, w.W, w.d, dtype=dt, device=device)
    for b in range(w.B):
        T_b = int(lens[b])
        x = ar1_hidden(T_b + w.n_decode, w.d_model, rho, gen, device)
        kb = (x @ WK).view(-1, w.H_kv, w.d)
        vb = (x @ WV).view(-1, w.H_kv, w.d)
        K[b, :, :T_b] = kb[:T_b].transpose(0, 1).to(dt)
        V[b, :, :T_b] = vb[:T_b].transpose(0, 1).to(dt)
        qw = (x[T_b - w.W:T_b] @ WQ).view(w.W, w.H_q, w.d) * q_scale
        Q_win[b] = qw.transpose(0, 1).to(dt)
        for i, e in enumerate(ends):
            qe = (x[e - w.W:e] @ WQ).view(w.W, w.H_q, w.d) * q_scale
            Q_ends[i, b] = qe.transpose(0, 1).to(dt)
        if w.n_decode:
            xd = x[T_b:]
            q_dec[:, b] = ((xd @ WQ).view(-1, w.H_q, w.d) * q_scale).to(dt)
            k_new[:, b] = kb[T_b:].to(dt)
            v_new[:, b] = vb[T_b:].to(dt)
        del x, kb, vb
    lens_bh = lens.to(torch.int32).view(w.B, 1).expand(w.B, w.H_kv).contiguous()
    return LayerInputs(K=K, V=V, lens=lens_bh.to(device), Q_win=Q_win, q_dec=q_dec,
                       k_new=k_new, v_new=v_new, rho=rho,
                       extra={"Q_ends": Q_ends} if ends else {})


def small_workload(base: Workload, **changes) -> Workload:
    """A copy of `base` with some fields changed (used for reduced test sizes)."""
    fields = dict(base.__dict__)
    fields.update(changes)
    return Workload(**fields)


def random_scores(n: int, seed: int, ties: bool = False, with_nan: bool = False,
                  device="cpu") -> torch.Tensor:
    """fp32 score-like values for selection tests (log-uniform magnitudes, some negative).

    With `ties`, values are drawn from a small set so equal keys occur; with
    `with_nan`, a few NaNs and infinities are planted.
    """
    g = _gen(seed, "cpu")
    if ties:
        s = torch.randint(-3, 6, (n,), generator=g).to(torch.float32)
    else:
        mag = torch.pow(10.0, torch.rand(n, generator=g, dtype=torch.float64) * 8 - 10)
        sign = torch.where(torch.rand(n, generator=g) < 0.1, -1.0, 1.0).to(torch.float64)
        s = (mag * sign).to(torch.float32)
    if with_nan and n:
        idx = torch.randperm(n, generator=g)[: max(1, n // 50)]
        s[idx[0::3]] = float("nan")
        s[idx[1::3]] = float("inf")
        s[idx[2::3]] = 0.0
    return s.to(device)


def random_weights(n: int, seed: int, device="cpu") -> torch.Tensor:
    """fp32 merge weights in roughly [-0.2, 1.2] for merge tests."""
    g = _gen(seed + 7, "cpu")
    return (torch.rand(n, generator=g) * 1.4 - 0.2).to(torch.float32).to(device)
