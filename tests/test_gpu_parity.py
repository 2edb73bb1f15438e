"""GPU parity: the CUDA path through the C ABI against the fp64 oracle, on the
same seeded inputs, for all five workloads and the edge cases."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from asymmetric_kv_merging_b200 import inputs

from parity import (GpuCache, Stats, assert_same_rows, compare_decode, compare_round, gpu_round,
                    storage_of, to_oracle_cache)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvs():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from asymmetric_kv_merging_b200 import build
    build.build()
    from asymmetric_kv_merging_b200 import kvs as mod
    return mod


def _workspace(kvs, B, H, H_q, d, T_cap, dtype, W=32):
    return kvs.workspace(kvs.make_desc(B, H, H_q, d, T_cap, dtype), W)


def compress_both(kvs, w, li, batch=None, ratio=None, stats=None, Q_override=None, form=None):
    """Compress on the GPU (all sequences) and in the oracle (sequences `batch`),
    comparing every round; before each round the oracle's input is read back from the
    GPU's cache, so both sides always score the same rows."""
    dev = torch.device("cuda")
    B, H, T_cap, d = li.K.shape
    ratio = ratio or w.ratio
    batch = list(range(B)) if batch is None else list(batch)
    g = GpuCache(li.K.to(dev), li.V.to(dev), li.lens.to(dev))
    lens = li.lens.view(B, H).cpu().numpy().astype(np.int64)
    if w.scope == "pooled":
        target_np = (lens // ratio).sum(axis=1)
        scope, scope_code = "pooled", kvs.SCOPE_POOLED
    else:
        target_np = lens // ratio
        scope, scope_code = "head", kvs.SCOPE_HEAD
    target = torch.tensor(target_np.reshape(-1), dtype=torch.int32, device=dev)
    cand = torch.full((B * H,), w.sink, dtype=torch.int32, device=dev)
    cand_np = np.full((len(batch), H), w.sink)
    Q = (li.Q_win if Q_override is None else Q_override).to(dev)
    Qo = Q.double().cpu().numpy()[batch]
    ws = _workspace(kvs, B, H, w.H_q, d, T_cap, li.K.dtype, w.W)
    stats = stats or Stats()
    form_name = "diagonal" if (form or 0) & kvs.FORM_DIAGONAL else "full"
    stats_name = "per_query" if (form or 0) & kvs.FORM_PER_QUERY else "mean"
    for _ in range(16):
        cur = g.lens.view(B, H).cpu().numpy()
        done = (cur.sum(axis=1) <= target_np) if scope == "pooled" else (cur <= target_np)
        if np.all(done):
            break
        o = to_oracle_cache(g, batch)
        r = oracle.merge_round(o, Qo, w.W, cand_np, w.W, target_np[batch], scope,
                               storage_of(li.K.dtype), form_name, stats_name)
        gout, gres = gpu_round(g, w.H_q, Q, w.W, cand, w.W, target, scope_code, ws, form=form)
        compare_round(r, gres, gout, o, li.K.dtype, scope, batch, stats, cand_np, w.W, form_name)
        g = gout
    else:
        raise AssertionError("compression did not finish")
    lens_out = g.lens.view(B, H).cpu().numpy()
    if scope == "pooled":
        assert np.array_equal(lens_out.sum(axis=1), target_np)
    else:
        assert np.array_equal(lens_out, target_np)
    assert kvs.device_flags(ws) == 0
    return g, to_oracle_cache(g, batch), stats, ws


def decode_both(kvs, w, li, g, o, steps, batch=None, stats=None, ws=None):
    """Decode steps with append on both sides; every step's outputs are compared, and
    afterwards the GPU cache must hold exactly the oracle's rows (appends are copies)."""
    dev = torch.device("cuda")
    B, H, T_cap, d = g.K.shape
    batch = list(range(B)) if batch is None else list(batch)
    desc = kvs.make_desc(B, H, w.H_q, d, T_cap, g.K.dtype)
    ws = ws if ws is not None else kvs.workspace(desc, w.W)
    out = torch.empty(B, w.H_q, d, dtype=g.K.dtype, device=dev)
    for s in steps:
        q = li.q_dec[s].to(dev).contiguous()
        kn = li.k_new[s].to(dev).contiguous()
        vn = li.v_new[s].to(dev).contiguous()
        kvs.decode_attn(desc, q, g.K, g.V, g.logn, g.lens, out, ws, kn, vn)
        oo, o = oracle.decode_step(o, q.double().cpu().numpy()[batch],
                                   kn.double().cpu().numpy()[batch], vn.double().cpu().numpy()[batch])
        compare_decode(oo, out, g.K.dtype, stats, batch)
    assert kvs.device_flags(ws) == 0
    assert_same_rows(g, o, batch)
    return g, o


# --------------------------------------------------------------------------- workload 0

@pytest.mark.parametrize("q_scale", [1.0, 6.0])
def test_workload0_tiny_fp32_pipeline(kvs, q_scale):
    w = inputs.workload(0)
    li = inputs.make_layer(w, 0, q_scale=q_scale)
    g, o, stats, ws = compress_both(kvs, w, li)
    g, o = decode_both(kvs, w, li, g, o, range(w.n_decode), stats=stats, ws=ws)
    stats.report(f"workload0 q_scale={q_scale}")
    assert stats.merged_compared > 0 and stats.decode_steps == w.n_decode


def planted_sinks(w, plants, layer=0):
    """Workload inputs with attention sinks planted in the candidate span, so that the
    window attention concentrates where the recipe alone never puts it. plants: list of
    (KV head, rows, target alpha_bar per row); each planted row gets the key c u (u the
    normalised mean window query of the head, c found by bisection on the oracle's
    window statistics) plus 2% of its own key, and one shared value plus 5% of its own.
    Two rows of one pair at alpha_bar in (1/4, 1/2) each give D < 0 (no minimiser: the
    plain-average branch); one row above 1/2 gives alpha (1 - 2 alpha) < 0."""
    li = inputs.make_layer(w, layer)
    K, V, Q = li.K.clone(), li.V.clone(), li.Q_win
    L = int(li.lens[0, 0])
    G = w.G
    for h, rows, per_row in plants:
        u = Q[0, h * G:(h + 1) * G].reshape(-1, w.d).double().mean(0)
        u = u / u.norm()
        Kd, Vd = K[0, h].double(), V[0, h].double()
        v0 = Vd[rows[0]].clone()
        Qh = Q[0, h * G:(h + 1) * G].double().numpy()

        def setc(c):
            Kt, Vt = Kd.clone(), Vd.clone()
            for r in rows:
                Kt[r] = c * u + 0.02 * Kd[r]
                Vt[r] = v0 + 0.05 * Vd[r]
            return Kt.to(K.dtype), Vt.to(V.dtype)

        def abar(c):
            Kt, Vt = setc(c)
            a, _ = oracle.window_statistics(Qh, Kt.double().numpy(), Vt.double().numpy(), None,
                                            L, w.W)
            return float(np.mean(a[list(rows)]))

        lo, hi = 0.0, 200.0
        for _ in range(50):
            mid = 0.5 * (lo + hi)
            lo, hi = (mid, hi) if abar(mid) < per_row else (lo, mid)
        K[0, h], V[0, h] = setc(hi)
    return inputs.LayerInputs(K=K, V=V, lens=li.lens, Q_win=Q, q_dec=li.q_dec, k_new=li.k_new,
                              v_new=li.v_new)


@pytest.mark.parametrize("dtype,d,form", [("f32", 64, None), ("bf16", 128, None),
                                          ("bf16", 128, "per_query"), ("bf16", 64, "per_query")])
def test_peaked_attention_exercises_degenerate_pairs(kvs, dtype, d, form):
    """Planted attention sinks: a pair at alpha_bar ~ 0.35 per row (D < 0, the
    plain-average branch, in the window-mean reading) in KV head 0 and a row at alpha_bar
    ~ 0.7 (> 1/2) in KV head 1. Both must occur in the oracle's scoring, and the GPU must
    agree on them: fp32 on the CUDA-core window path, bf16 on the tensor-core passes. In
    the per-query form the branch depends on each query's own attention (no pair need be
    degenerate); there the sinks put window outputs next to the planted rows, the case in
    which the per-query distances are taken directly rather than by their expansion."""
    w = inputs.small_workload(inputs.workload(0), T=192, n_decode=2, dtype=dtype, d=d)
    li = planted_sinks(w, [(0, (52, 53), 0.35), (1, (60,), 0.7)])
    code = kvs.FORM_FULL | (kvs.FORM_PER_QUERY if form == "per_query" else 0)
    stats = Stats()
    g, o, stats, ws = compress_both(kvs, w, li, stats=stats, form=code)
    g, o = decode_both(kvs, w, li, g, o, range(w.n_decode), stats=stats, ws=ws)
    stats.report(f"planted sinks {dtype} d={d} {form or 'mean'} (degenerate branch, alpha > 1/2)")
    assert stats.alpha_over_half >= 2
    if form is None:
        assert stats.degenerate_pairs >= 1


# --------------------------------------------------------------------------- workload 1

def test_workload1_llama_layer_full_size(kvs):
    w = inputs.workload(1)
    li = inputs.make_layer(w, 0, device="cuda")
    g, o, stats, ws = compress_both(kvs, w, li)
    g, o = decode_both(kvs, w, li, g, o, range(w.n_decode), stats=stats, ws=ws)
    stats.report("workload1 llama layer 32K")
    assert stats.merged_compared > 8 * 16000
    assert stats.near_threshold <= 8


@pytest.mark.parametrize("wl", [0, 1])
def test_diagonal_form_pipeline(kvs, wl):
    """kvs_score_pairs_form with the diagonal-only form (the coupling term dropped):
    scores, weights, selection and the merged caches against the oracle's diagonal form,
    every round, then decode."""
    w = inputs.workload(wl)
    li = inputs.make_layer(w, 0, device="cuda")
    g, o, stats, ws = compress_both(kvs, w, li, form=kvs.FORM_DIAGONAL)
    g, o = decode_both(kvs, w, li, g, o, range(min(4, w.n_decode)), stats=stats, ws=ws)
    stats.report(f"diagonal form workload{wl}")
    assert stats.scores_compared > 0
    assert stats.near_threshold <= 8


@pytest.mark.parametrize("wl,T,H_kv", [(1, 4096, 2), (1, 32768, 8)])
def test_per_query_window_form(kvs, wl, T, H_kv):
    """kvs_score_pairs_form with KVS_FORM_PER_QUERY (the window read query by query: the
    one-query norms of every window query, averaged) against the oracle's per-query
    statistics, every round, then decode."""
    w = inputs.small_workload(inputs.workload(wl), T=T, H_kv=H_kv, H_q=4 * H_kv, n_decode=4)
    li = inputs.make_layer(w, 0, device="cuda")
    g, o, stats, ws = compress_both(kvs, w, li, form=kvs.FORM_FULL | kvs.FORM_PER_QUERY)
    g, o = decode_both(kvs, w, li, g, o, range(w.n_decode), stats=stats, ws=ws)
    stats.report(f"per-query window form T={T} H_kv={H_kv}")
    assert stats.scores_compared > 0
    assert stats.near_threshold <= 8


@pytest.mark.parametrize("form", ["full", "diagonal", "per_query"])
def test_head_dim_64_tensor_core_passes(kvs, form):
    """bf16 caches with d = 64 take the d = 64 instantiations of both tensor-core window
    passes (four-stage rings, one 64-column box per row): every form, several tiles per
    CTA in both passes, every round compared, then decode."""
    w = inputs.small_workload(inputs.workload(1), T=32768, H_kv=2, H_q=8, d=64, n_decode=4)
    li = inputs.make_layer(w, 0, device="cuda")
    code = {"full": kvs.FORM_FULL, "diagonal": kvs.FORM_DIAGONAL,
            "per_query": kvs.FORM_FULL | kvs.FORM_PER_QUERY}[form]
    g, o, stats, ws = compress_both(kvs, w, li, form=code)
    g, o = decode_both(kvs, w, li, g, o, range(w.n_decode), stats=stats, ws=ws)
    stats.report(f"bf16 d=64 {form} form T=32768 H_kv=2")
    assert stats.scores_compared > 0 and stats.merged_compared > 0
    assert stats.near_threshold <= 8


def test_per_query_form_needs_the_tensor_core_path(kvs):
    dev = torch.device("cuda")
    desc = kvs.make_desc(1, 2, 4, 64, 256, torch.float32)
    K = torch.randn(1, 2, 256, 64, device=dev)
    lens = torch.full((2,), 200, dtype=torch.int32, device=dev)
    cand = torch.full((2,), 32, dtype=torch.int32, device=dev)
    Q = torch.randn(1, 4, 32, 64, device=dev)
    score = torch.zeros(1, 2, 128, device=dev)
    ws = kvs.workspace(desc, 32)
    with pytest.raises(kvs.KvsError) as e:
        kvs.score_pairs(desc, K, K, None, lens, cand, 32, Q, 32, score, score.clone(), ws,
                        form=kvs.FORM_PER_QUERY)
    assert e.value.status == 2                  # KVS_ERR_UNSUPPORTED, nothing launched


def test_score_form_rejects_unknown_form(kvs):
    desc = kvs.make_desc(1, 1, 1, 64, 64, torch.float32)
    with pytest.raises(kvs.KvsError) as e:
        kvs.score_pairs(desc, None, None, None, None, None, 0, None, 1, None, None,
                        torch.zeros(16, dtype=torch.uint8), form=7)
    assert e.value.status == 1


# --------------------------------------------------------------------------- workload 2

@pytest.mark.parametrize("layer", [0, 31])
def test_workload2_128k_layer_sample(kvs, layer):
    """One layer of the 32-layer 128K workload, at full size: every round and 32
    decode steps (the bench times all 32 layers with the same kernels)."""
    w = inputs.workload(2)
    li = inputs.make_layer(w, layer, device="cuda")
    g, o, stats, ws = compress_both(kvs, w, li)
    g, o = decode_both(kvs, w, li, g, o, range(32), stats=stats, ws=ws)
    stats.report(f"workload2 128K layer {layer}")
    assert stats.near_threshold <= 8


# --------------------------------------------------------------------------- workload 3

@pytest.mark.parametrize("layer,batch", [(0, [0, 3, 5, 7]), (31, [1, 6])])
def test_workload3_pooled_budget_sample(kvs, layer, batch):
    """Batch 8 on the GPU, pooled budget per sequence; the oracle checks the listed
    sequences of the layer (every head, every round, then the decode step)."""
    w = inputs.workload(3)
    li = inputs.make_layer(w, layer, device="cuda")
    g, o, stats, ws = compress_both(kvs, w, li, batch=batch)
    lens = g.lens.view(w.B, w.H_kv).cpu().numpy()
    assert len(set(lens.reshape(-1).tolist())) > 1          # ragged per-head lengths
    g, o = decode_both(kvs, w, li, g, o, range(w.n_decode), batch=batch, stats=stats, ws=ws)
    stats.report(f"workload3 pooled layer {layer} sequences {batch}")
    assert stats.heads_compared == len(batch) * w.H_kv * stats.rounds
    assert stats.near_threshold <= 8


# --------------------------------------------------------------------------- workload 4

def test_workload4_serving_mix_sample(kvs):
    """Ragged batch of 16: 8x compression, 256 decode steps with an in-place
    re-merge of the newest 64 rows every 64 steps; the oracle follows sequences 0, 9
    and 13 through every round and every decode step."""
    w = inputs.workload(4)
    li = inputs.make_layer(w, 0, device="cuda")
    batch = [0, 9, 13]
    g, o, stats, ws = compress_both(kvs, w, li, batch=batch)
    dev = torch.device("cuda")
    B, H, T_cap, d = g.K.shape
    for seg in range(w.n_decode // w.remerge_every):
        s0 = seg * w.remerge_every
        g, o = decode_both(kvs, w, li, g, o, range(s0, s0 + w.remerge_every), batch=batch,
                           stats=stats, ws=ws)
        # re-merge the newest segment in place: 64 -> 8 rows, window = last 32 decode queries
        Qw = li.q_dec[s0 + w.remerge_every - w.W: s0 + w.remerge_every].to(dev)
        Qw = Qw.permute(1, 2, 0, 3).contiguous()                    # [B, H_q, W, d]
        Qo = Qw.double().cpu().numpy()[batch]
        for k in range(3):
            seg_len = w.remerge_every // (2 ** k)
            cand = (g.lens - seg_len).contiguous()
            lens_now = g.lens.view(B, H).cpu().numpy()
            target_np = lens_now - seg_len // 2
            target = torch.tensor(target_np.reshape(-1), dtype=torch.int32, device=dev)
            o = to_oracle_cache(g, batch)                             # the round's input
            oc = o.lengths() - seg_len
            r = oracle.merge_round(o, Qo, w.W, oc, 0, target_np[batch], "head",
                                   storage_of(g.K.dtype))
            gout, gres = gpu_round(g, w.H_q, Qw, w.W, cand, 0, target, kvs.SCOPE_HEAD, ws,
                                   inplace=True)
            compare_round(r, gres, gout, o, g.K.dtype, "head", batch, stats, oc, 0)
            g = gout
        o = to_oracle_cache(g, batch)
    stats.report(f"workload4 serving mix sequences {batch}")
    assert stats.decode_steps == w.n_decode
    assert stats.near_threshold <= 8
    assert kvs.device_flags(ws) == 0


# --------------------------------------------------------------------------- selection

def _selection_case(kvs, scope, B, H, L, c0, n_recent, R_list, ties, seed, dtype=torch.bfloat16, d=128):
    dev = torch.device("cuda")
    T_cap = L + 6 + L % 2
    g = torch.Generator().manual_seed(seed)
    K = torch.randn(B, H, T_cap, d, generator=g).to(dtype)
    V = torch.randn(B, H, T_cap, d, generator=g).to(dtype)
    logn = torch.log(torch.randint(1, 4, (B, H, T_cap), generator=g).float())
    lens = torch.full((B * H,), L, dtype=torch.int32)
    P = max(0, (L - n_recent - c0) // 2)
    score = torch.zeros(B, H, T_cap // 2)
    w_b = torch.zeros(B, H, T_cap // 2)
    for i in range(B * H):
        b, h = divmod(i, H)
        score[b, h, :P] = inputs.random_scores(P, seed * 100 + i, ties=ties, with_nan=True)
        w_b[b, h, :P] = inputs.random_weights(P, seed * 100 + i)
    desc = kvs.make_desc(B, H, 4 * H, d, T_cap, dtype)
    ws = kvs.workspace(desc, 32)
    cand = torch.full((B * H,), c0, dtype=torch.int32)
    for R in R_list:
        if scope == kvs.SCOPE_POOLED:
            target = torch.full((B,), H * L - R, dtype=torch.int32)
        else:
            target = torch.full((B * H,), L - R, dtype=torch.int32)
        outs = {}
        for inplace in (False, True):
            Kd, Vd, ld, lnd = K.to(dev), V.to(dev), lens.to(dev), logn.to(dev)
            sel = torch.zeros(B, H, T_cap // 2, dtype=torch.uint8, device=dev)
            off = torch.full((B, H, T_cap // 2), -1, dtype=torch.int32, device=dev)
            if inplace:
                Ko, Vo, lo, lno = Kd, Vd, ld, lnd
            else:
                Ko, Vo = torch.zeros_like(Kd), torch.zeros_like(Vd)
                lo, lno = torch.zeros_like(ld), torch.zeros_like(lnd)
            kvs.merge_compact(desc, Kd, Vd, lnd, ld, cand.to(dev), n_recent, score.to(dev),
                              w_b.to(dev), target.to(dev), scope, T_cap, Ko, Vo, lno, lo, ws,
                              sel, off)
            torch.cuda.synchronize()
            outs[inplace] = (Ko.cpu(), Vo.cpu(), lno.cpu(), lo.cpu(), sel.cpu(), off.cpu())
        assert kvs.device_flags(ws) == 0
        # oracle on the same fp32 scores: bit-exact selection and offsets
        Ko, Vo, lno, lo, sel, off = outs[False]
        for b in range(B):
            if scope == kvs.SCOPE_POOLED:
                pooled = np.concatenate([score[b, h, :P].double().numpy() for h in range(H)])
                mask = oracle.select_pairs(pooled, R).reshape(H, P)
            for h in range(H):
                sc = score[b, h, :P].double().numpy()
                m_sel = mask[h] if scope == kvs.SCOPE_POOLED else oracle.select_pairs(sc, R)
                np.testing.assert_array_equal(sel[b, h, :P].numpy().astype(bool), m_sel)
                m = oracle.merge_compact_head(K[b, h].double().numpy(), V[b, h].double().numpy(),
                                              logn[b, h].double().numpy(), L, c0, n_recent, m_sel,
                                              w_b[b, h, :P].double().numpy(),
                                              storage_of(dtype))
                np.testing.assert_array_equal(off[b, h, :P].numpy(), m.out_offset)
                assert int(lo[b * H + h]) == m.length
                n = m.length
                np.testing.assert_allclose(Ko[b, h, :n].double().numpy(), m.K, rtol=2e-2, atol=1e-2)
                np.testing.assert_allclose(Vo[b, h, :n].double().numpy(), m.V, rtol=2e-2, atol=1e-2)
                np.testing.assert_allclose(lno[b, h, :n].double().numpy(), m.log_n, atol=2e-6)
                merged = np.zeros(n, bool)
                merged[m.out_offset[m_sel]] = True
                np.testing.assert_array_equal(Ko[b, h, :n][~merged].double().numpy(), m.K[~merged])
        # in-place gives the same rows as out-of-place
        Ki, Vi, lni, li_, seli, offi = outs[True]
        assert torch.equal(li_, lo) and torch.equal(seli, sel) and torch.equal(offi, off)
        for b in range(B):
            for h in range(H):
                n = int(lo[b * H + h])
                assert torch.equal(Ki[b, h, :n], Ko[b, h, :n]) and torch.equal(Vi[b, h, :n], Vo[b, h, :n])
                assert torch.equal(lni[b, h, :n], lno[b, h, :n])
                assert torch.equal(Ki[b, h, :c0], K[b, h, :c0])


@pytest.mark.parametrize("ties", [False, True])
def test_selection_per_head_exact(kvs, ties):
    L, c0, nr = 700, 32, 32
    P = (L - nr - c0) // 2
    _selection_case(kvs, kvs.SCOPE_HEAD, 2, 3, L, c0, nr, [0, 1, 17, P // 2, P - 1, P], ties, 1)


@pytest.mark.parametrize("ties", [False, True])
def test_selection_pooled_exact(kvs, ties):
    L, c0, nr = 501, 7, 10
    P = (L - nr - c0) // 2
    _selection_case(kvs, kvs.SCOPE_POOLED, 2, 4, L, c0, nr, [0, 5, 4 * P // 3, 4 * P - 1, 4 * P],
                    ties, 2)


def test_selection_spans_many_blocks_fp32_d64(kvs):
    L = 128 * 2 * 9 + 77       # several merge blocks and a ragged tail
    _selection_case(kvs, kvs.SCOPE_HEAD, 1, 2, L, 32, 32, [300, 1000], False, 3,
                    dtype=torch.float32, d=64)


# --------------------------------------------------------------------------- decode

@pytest.mark.parametrize("dtype,d,G", [(torch.bfloat16, 128, 4), (torch.float32, 64, 2),
                                       (torch.bfloat16, 64, 8), (torch.float32, 128, 1)])
def test_decode_ragged_with_append(kvs, dtype, d, G):
    dev = torch.device("cuda")
    B, H = 3, 2
    lens = torch.tensor([[0, 1], [777, 64], [4097, 2000]], dtype=torch.int32)
    T_cap = 4200
    g = torch.Generator().manual_seed(7)
    K = (torch.randn(B, H, T_cap, d, generator=g)).to(dtype)
    V = torch.randn(B, H, T_cap, d, generator=g).to(dtype)
    logn = torch.log(torch.randint(1, 5, (B, H, T_cap), generator=g).float())
    q = (torch.randn(3, B, H * G, d, generator=g) * 3).to(dtype)
    kn = torch.randn(3, B, H, d, generator=g).to(dtype)
    vn = torch.randn(3, B, H, d, generator=g).to(dtype)
    gc = GpuCache(K.to(dev), V.to(dev), lens.to(dev), logn.to(dev))
    o = to_oracle_cache(gc)
    desc = kvs.make_desc(B, H, H * G, d, T_cap, dtype)
    ws = kvs.workspace(desc, 32)
    out = torch.empty(B, H * G, d, dtype=dtype, device=dev)
    # a step without append first
    kvs.decode_attn(desc, q[0].to(dev), gc.K, gc.V, gc.logn, gc.lens, out, ws)
    oo, _ = oracle.decode_step(o, q[0].double().numpy())
    compare_decode(oo, out, dtype)
    for s in range(3):
        kvs.decode_attn(desc, q[s].to(dev), gc.K, gc.V, gc.logn, gc.lens, out, ws,
                        kn[s].to(dev), vn[s].to(dev))
        oo, o = oracle.decode_step(o, q[s].double().numpy(), kn[s].double().numpy(),
                                   vn[s].double().numpy())
        compare_decode(oo, out, dtype)
    assert torch.equal(gc.lens.cpu().view(B, H), lens + 3)
    assert kvs.device_flags(ws) == 0


@pytest.mark.parametrize("B,H", [(1, 2), (40, 2)])      # few heads: cluster grid; many: split grid
@pytest.mark.parametrize("lead", [0, 1, 3])
def test_decode_log_counts_at_any_4_byte_offset(kvs, B, H, lead):
    """The log-counts may start at any 4-byte boundary (a view into a larger buffer):
    the TMA map over them starts at the 16-byte boundary below and skips `lead`."""
    dev = torch.device("cuda")
    d, G, T_cap = 128, 4, 1000
    g = torch.Generator().manual_seed(100 + lead)
    lens = torch.randint(0, T_cap - 1, (B, H), generator=g, dtype=torch.int32)
    lens[0, 0] = T_cap - 1
    K = torch.randn(B, H, T_cap, d, generator=g).to(torch.bfloat16)
    V = torch.randn(B, H, T_cap, d, generator=g).to(torch.bfloat16)
    logn = torch.log(torch.randint(1, 9, (B, H, T_cap), generator=g).float())
    buf = torch.zeros(B * H * T_cap + 4, device=dev)
    ln_view = buf[lead:lead + B * H * T_cap].view(B, H, T_cap)
    ln_view.copy_(logn.to(dev))
    assert (ln_view.data_ptr() % 16) == 4 * lead
    q = (torch.randn(B, H * G, d, generator=g) * 3).to(torch.bfloat16)
    kn = torch.randn(B, H, d, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, H, d, generator=g).to(torch.bfloat16)
    gc = GpuCache(K.to(dev), V.to(dev), lens.to(dev), ln_view)
    o = to_oracle_cache(gc)
    desc = kvs.make_desc(B, H, H * G, d, T_cap, torch.bfloat16)
    ws = kvs.workspace(desc, 32)
    out = torch.empty(B, H * G, d, dtype=torch.bfloat16, device=dev)
    kvs.decode_attn(desc, q.to(dev), gc.K, gc.V, ln_view, gc.lens, out, ws, kn.to(dev), vn.to(dev))
    oo, o = oracle.decode_step(o, q.double().numpy(), kn.double().numpy(), vn.double().numpy())
    compare_decode(oo, out, torch.bfloat16)
    assert torch.equal(gc.lens.cpu().view(B, H), lens + 1)
    assert kvs.device_flags(ws) == 0


def test_decode_append_at_capacity_sets_flag(kvs):
    dev = torch.device("cuda")
    desc = kvs.make_desc(1, 1, 4, 128, 64, torch.bfloat16)
    K = torch.randn(1, 1, 64, 128, device=dev).to(torch.bfloat16)
    V = torch.randn_like(K)
    lens = torch.tensor([64], dtype=torch.int32, device=dev)
    ws = kvs.workspace(desc, 32)
    out = torch.empty(1, 4, 128, dtype=torch.bfloat16, device=dev)
    kn = torch.randn(1, 1, 128, device=dev).to(torch.bfloat16)
    kvs.decode_attn(desc, torch.randn(1, 4, 128, device=dev).to(torch.bfloat16), K, V, None, lens,
                    out, ws, kn, kn)
    assert kvs.device_flags(ws, clear=True) == kvs.FLAG_OUT_CAPACITY
    assert int(lens.item()) == 64
    assert kvs.device_flags(ws) == 0


# --------------------------------------------------------------------------- edge cases

def test_edge_cases_short_and_empty_spans(kvs):
    """Heads with no candidate pairs, odd spans, a cache shorter than the window,
    and a budget already met, in one batch."""
    dev = torch.device("cuda")
    w = inputs.small_workload(inputs.workload(0), B=1, H_kv=6, H_q=12, T=200, n_decode=0)
    g0 = torch.Generator().manual_seed(3)
    T_cap = 256
    K = torch.randn(1, 6, T_cap, 64, generator=g0)
    V = torch.randn(1, 6, T_cap, 64, generator=g0)
    Q = torch.randn(1, 12, 32, 64, generator=g0) * 2
    lens = torch.tensor([[200, 65, 64, 20, 0, 97]], dtype=torch.int32)   # 64: P = 0; 20 < W
    li = inputs.LayerInputs(K=K, V=V, lens=lens, Q_win=Q, q_dec=None, k_new=None, v_new=None)
    gc = GpuCache(K.to(dev), V.to(dev), lens.to(dev))
    cand = torch.full((6,), 32, dtype=torch.int32, device=dev)
    cand_np = np.full((1, 6), 32)
    target_np = np.array([[100, 60, 64, 20, 0, 90]])
    target = torch.tensor(target_np.reshape(-1), dtype=torch.int32, device=dev)
    ws = kvs.workspace(kvs.make_desc(1, 6, 12, 64, T_cap, torch.float32), 32)
    stats = Stats()
    for _ in range(4):
        o = to_oracle_cache(gc)
        r = oracle.merge_round(o, Q.double().numpy(), 32, cand_np, 32, target_np, "head", "f32")
        gout, gres = gpu_round(gc, 12, Q.to(dev), 32, cand, 32, target, kvs.SCOPE_HEAD, ws)
        compare_round(r, gres, gout, o, torch.float32, "head", None, stats, cand_np, 32)
        gc = gout
        # the 65-row head has a one-row span (no pairs): its budget is unreachable, which
        # every round reports; the other heads reach theirs
        assert kvs.device_flags(ws, clear=True) == kvs.FLAG_BUDGET
    assert gc.lens.cpu().tolist() == [100, 65, 64, 20, 0, 90]
    stats.report("edge cases: short, empty and odd spans")


def test_bad_length_and_capacity_flags(kvs):
    dev = torch.device("cuda")
    desc = kvs.make_desc(1, 2, 4, 64, 128, torch.float32)
    K = torch.randn(1, 2, 128, 64, device=dev)
    V = torch.randn_like(K)
    lens = torch.tensor([129, 100], dtype=torch.int32, device=dev)      # head 0 invalid
    Q = torch.randn(1, 4, 32, 64, device=dev)
    cand = torch.full((2,), 32, dtype=torch.int32, device=dev)
    ws = kvs.workspace(desc, 32)
    score = torch.zeros(1, 2, 64, device=dev)
    w_b = torch.zeros_like(score)
    kvs.score_pairs(desc, K, V, None, lens, cand, 32, Q, 32, score, w_b, ws)
    assert kvs.device_flags(ws, clear=True) & kvs.FLAG_BAD_LENGTH
    lens = torch.tensor([128, 100], dtype=torch.int32, device=dev)
    kvs.score_pairs(desc, K, V, None, lens, cand, 32, Q, 32, score, w_b, ws)
    assert kvs.device_flags(ws) == 0
    # the output capacity (96 rows) is too small for head 0 (128 - 8 merged = 120 rows)
    Ko = torch.zeros(1, 2, 96, 64, device=dev)
    Vo = torch.zeros_like(Ko)
    lno = torch.zeros(1, 2, 96, device=dev)
    lo = torch.zeros(2, dtype=torch.int32, device=dev)
    target = torch.tensor([120, 50], dtype=torch.int32, device=dev)
    kvs.merge_compact(desc, K, V, None, lens, cand, 32, score, w_b, target, kvs.SCOPE_HEAD, 96,
                      Ko, Vo, lno, lo, ws)
    # head 0 does not fit; head 1's target (50) is below the 65 rows its 36-row span can
    # reach by repeated rounds
    assert kvs.device_flags(ws, clear=True) == kvs.FLAG_OUT_CAPACITY | kvs.FLAG_BUDGET
    assert int(lo[1]) == 82   # head 1: 100 rows, all 18 pairs merged
