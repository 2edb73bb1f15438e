"""Helpers for the GPU-vs-oracle parity tests.

Tolerances (GPU arithmetic is fp32; the oracle is fp64):
  * selection flags and compaction offsets: bit-exact, except pairs whose oracle
    score is within 1e-5 relative of the unit's selection threshold (counted);
  * merged keys before rounding (fp32 debug output): per-row |dk| / |k| <= 1e-4;
  * stored bf16 rows and decode outputs: |d| <= 1e-2 + 2e-2 |ref|;
  * fp32 caches: stored rows per-row relative 1e-4, decode outputs 1e-4 + 1e-4 |ref|;
  * scores: relative 2e-4 and weights absolute 2e-4, except pairs whose D sits
    within a factor 2 of the degenerate threshold 1e-6 (N11 + N22), where a
    one-ulp change flips the branch. The score is a product of ~10 fp32
    operations on window statistics that are sums over up to 131072 rows; with
    fp32's 6e-8 unit roundoff and the statistics' blockwise summation the
    observed relative error stays near 1e-6, and 2e-4 leaves room for the
    cancellation in D = N11 - 2 N12 + N22.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

import oracle
from asymmetric_kv_merging_b200 import kvs

NEAR_REL = 1e-5


@dataclass
class Stats:
    near_threshold: int = 0
    input_divergent_selection: int = 0
    degenerate_boundary: int = 0
    input_rows_differing: int = 0
    diverged_heads: set = field(default_factory=set)
    compared_rows: int = 0
    merged_compared: int = 0
    merged_loose: int = 0
    scores_compared: int = 0

    def report(self):
        return (f"rows={self.compared_rows} merged={self.merged_compared} (+{self.merged_loose} "
                f"loose) scores={self.scores_compared} near_threshold={self.near_threshold} "
                f"input_divergent={self.input_divergent_selection} "
                f"degenerate_boundary={self.degenerate_boundary} "
                f"input_rows_differing={self.input_rows_differing} "
                f"diverged_heads={len(self.diverged_heads)}")


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


def to_oracle_cache(cache: GpuCache, heads=None, batch=None):
    """Copy (a subset of) a device cache to an oracle Cache (fp64)."""
    K = cache.K.double().cpu().numpy()
    V = cache.V.double().cpu().numpy()
    ln = cache.logn.double().cpu().numpy()
    B, H = K.shape[:2]
    lens = cache.lens.view(B, H).cpu().numpy()
    bs = range(B) if batch is None else batch
    return oracle.cache_from_arrays(K[list(bs)], V[list(bs)], lens[list(bs)], ln[list(bs)])


def _unit_threshold(r, b, h, scope):
    if scope == "pooled":
        sc = np.concatenate([r.scores[b][hh].score for hh in range(len(r.scores[b]))])
        sl = np.concatenate([r.selected[b][hh] for hh in range(len(r.selected[b]))])
    else:
        sc, sl = r.scores[b][h].score, r.selected[b][h]
    if not sl.any():
        return None
    key = np.where(np.isnan(sc), np.inf, sc)
    return key[sl].max()


def compare_round(r, g, out: GpuCache, gin: GpuCache, oin, dtype, scope="head", batch_map=None,
                  stats=None):
    """Compare one oracle round with one GPU round, head by head.

    gin / oin: the GPU and oracle caches the round started from. After a first
    round, a few merged bf16 rows can differ by one unit in the last place
    between the two sides (fp32 vs fp64 results rounding to different
    neighbours); the exact criteria apply to pairs and rows whose inputs agree
    bit for bit, the storage tolerance to the others (counted).
    batch_map: oracle batch index -> GPU batch index (oracle run on a subset).
    """
    stats = stats or Stats()
    storage = storage_of(dtype)
    B_o = len(r.scores)
    H = len(r.scores[0])
    Kg = out.K.double().cpu().numpy()
    Vg = out.V.double().cpu().numpy()
    Lg = out.logn.double().cpu().numpy()
    Kin = gin.K.double().cpu().numpy()
    Vin = gin.V.double().cpu().numpy()
    lens_g = out.lens.view(out.K.shape[0], H).cpu().numpy()
    for bo in range(B_o):
        bg = bo if batch_map is None else batch_map[bo]
        for h in range(H):
            if (bg, h) in stats.diverged_heads:
                continue
            L_in = oin.length(bo, h)
            row_eq = (np.all(Kin[bg, h, :L_in] == oin.K[bo][h], axis=1)
                      & np.all(Vin[bg, h, :L_in] == oin.V[bo][h], axis=1))
            stats.input_rows_differing += int((~row_eq).sum())
            hs = r.scores[bo][h]
            P = hs.score.shape[0]
            c0 = r.merges[bo][h].out_offset[0] if P else 0
            a_rows = c0 + 2 * np.arange(P)
            pair_eq = row_eq[a_rows] & row_eq[a_rows + 1] if P else np.zeros(0, bool)
            if P:
                n_sum = hs.n11 + hs.n22
                with np.errstate(invalid="ignore", divide="ignore"):
                    ratio = hs.D / n_sum
                boundary = ~np.isfinite(ratio) | ((ratio > 0.5e-6) & (ratio < 2e-6))
                stats.degenerate_boundary += int(boundary.sum())
                ok = ~boundary & pair_eq
                sg = g["score"][bg, h, :P].numpy()
                wg = g["w_b"][bg, h, :P].numpy()
                scale = np.max(np.abs(hs.score[ok]), initial=0.0)
                np.testing.assert_allclose(sg[ok], hs.score[ok], rtol=2e-4, atol=1e-7 * scale,
                                           err_msg=f"score b={bg} h={h}")
                np.testing.assert_allclose(wg[ok], hs.w_b[ok], rtol=0, atol=2e-4,
                                           err_msg=f"w_b b={bg} h={h}")
                stats.scores_compared += int(ok.sum())
            sel_o = r.selected[bo][h]
            sel_g = g["sel"][bg, h, :P].numpy()
            diff = sel_o != sel_g
            if diff.any():
                thr = _unit_threshold(r, bo, h, scope)
                sc = np.where(np.isnan(hs.score), np.inf, hs.score)
                near = np.abs(sc[diff] - thr) <= NEAR_REL * abs(thr)
                explained = near | ~pair_eq[diff]
                assert explained.all(), (f"selection differs away from the threshold b={bg} h={h}: "
                                         f"{np.flatnonzero(diff)[~explained][:8]}")
                stats.near_threshold += int(near.sum())
                stats.input_divergent_selection += int((~near).sum())
                stats.diverged_heads.add((bg, h))
                continue
            m = r.merges[bo][h]
            assert lens_g[bg, h] == m.length, (bg, h, lens_g[bg, h], m.length)
            np.testing.assert_array_equal(g["off"][bg, h, :P].numpy(), m.out_offset,
                                          err_msg=f"offsets b={bg} h={h}")
            n = m.length
            ko, vo = m.K, m.V
            kg, vg = Kg[bg, h, :n], Vg[bg, h, :n]
            # source input row of every copied output row
            src = np.full(n, -1, dtype=np.int64)
            src[:c0] = np.arange(min(c0, n))
            for p in np.flatnonzero(~sel_o):
                src[m.out_offset[p]] = a_rows[p]
                src[m.out_offset[p] + 1] = a_rows[p] + 1
            tail = L_in - (c0 + 2 * P)
            if tail:
                src[n - tail:] = np.arange(c0 + 2 * P, L_in)
            copied = src >= 0
            exact = copied.copy()
            exact[copied] = row_eq[src[copied]]
            np.testing.assert_array_equal(kg[exact], ko[exact], err_msg=f"K copy b={bg} h={h}")
            np.testing.assert_array_equal(vg[exact], vo[exact], err_msg=f"V copy b={bg} h={h}")
            np.testing.assert_allclose(Lg[bg, h, :n], m.log_n, rtol=0, atol=2e-6,
                                       err_msg=f"logn b={bg} h={h}")
            loose = ~exact
            if storage == "bf16":
                np.testing.assert_allclose(kg[loose], ko[loose], rtol=2e-2, atol=1e-2)
                np.testing.assert_allclose(vg[loose], vo[loose], rtol=2e-2, atol=1e-2)
            else:
                for a, o in ((kg[loose], ko[loose]), (vg[loose], vo[loose])):
                    if a.size:
                        rel = np.linalg.norm(a - o, axis=1) / np.maximum(np.linalg.norm(o, axis=1), 1e-30)
                        assert rel.max() <= 1e-4
            if sel_o.any():
                strict = sel_o & pair_eq
                kmg = g["km"][bg, h, :P].numpy()[strict]
                kmo = m.k_merged[strict]
                if kmo.size:
                    rel = np.linalg.norm(kmg - kmo, axis=1) / np.maximum(np.linalg.norm(kmo, axis=1), 1e-30)
                    assert rel.max() <= 1e-4, f"merged key rel {rel.max()} b={bg} h={h}"
                stats.merged_compared += int(strict.sum())
                stats.merged_loose += int((sel_o & ~pair_eq).sum())
            stats.compared_rows += n
    return stats


def compare_decode(out_o, out_g, dtype, heads_G, stats=None, batch_map=None):
    """out_o: (B_o, H_q, d) oracle; out_g: (B, H_q, d) torch."""
    stats = stats or Stats()
    og = out_g.double().cpu().numpy()
    for bo in range(out_o.shape[0]):
        bg = bo if batch_map is None else batch_map[bo]
        for hq in range(out_o.shape[1]):
            if (bg, hq // heads_G) in stats.diverged_heads:
                continue
            if dtype == torch.bfloat16:
                np.testing.assert_allclose(og[bg, hq], out_o[bo, hq], rtol=2e-2, atol=1e-2,
                                           err_msg=f"decode b={bg} hq={hq}")
            else:
                np.testing.assert_allclose(og[bg, hq], out_o[bo, hq], rtol=1e-4, atol=1e-4,
                                           err_msg=f"decode b={bg} hq={hq}")
    return stats
