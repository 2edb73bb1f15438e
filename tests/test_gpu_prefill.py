"""GPU parity of kvs_prefill_chunk (chunked streaming prefill compression) against the
oracle's loop, chunk by chunk.

Before every chunk the oracle takes the GPU cache as its input, so each chunk is
compared on identical inputs. Lengths must match exactly. Rows must match within the
bf16 / fp32 tolerances of the other parity tests, unless the oracle's own ranking
has a near-tie at the selection threshold of that head (a pair within 1e-5 relative
of the largest selected score), where the two sides may legitimately pick
different pairs; those heads are counted.
"""

import numpy as np
import pytest
import torch

import oracle
from parity import REPORTS, GpuCache, storage_of, to_oracle_cache

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvs():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from asymmetric_kv_merging_b200 import build
    build.build()
    from asymmetric_kv_merging_b200 import kvs as mod
    return mod


def _near_tie(rounds, b, h, rel=1e-5):
    for r in rounds:
        s = r.scores[b][h].score
        sel = r.selected[b][h]
        if sel.all() or not sel.any():
            continue
        thr = np.max(s[sel])
        nxt = np.min(s[~sel])
        if nxt - thr <= rel * max(abs(thr), 1e-30):
            return True
    return False


def _rows_match(go, oo, b, h, dtype):
    L = go.length(b, h)
    tol = dict(rtol=2e-2, atol=1e-2) if dtype == torch.bfloat16 else dict(rtol=1e-4, atol=1e-5)
    return (np.allclose(go.log_n[b][h][:L], oo.log_n[b][h][:L], rtol=0, atol=2e-6)
            and np.allclose(go.K[b][h][:L], oo.K[b][h][:L], **tol)
            and np.allclose(go.V[b][h][:L], oo.V[b][h][:L], **tol))


@pytest.mark.parametrize("dtype,d,G,T,chunk,budget", [
    (torch.bfloat16, 128, 4, 3072, 512, 1024),     # the pages' chunk size, budget halved
    (torch.float32, 64, 2, 2000, 256, 512),        # fp32 window path, ragged last chunk
])
def test_prefill_chunks_match_the_oracle(kvs, dtype, d, G, T, chunk, budget):
    from asymmetric_kv_merging_b200 import inputs
    dev = torch.device("cuda")
    sink, W = 32, 32
    base = inputs.workload(1 if dtype == torch.bfloat16 else 0)
    w = inputs.small_workload(base, B=2, H_kv=2, H_q=2 * G, d=d, T=T, W=W, n_decode=0)
    ends = [min(T, c + chunk) for c in range(0, T, chunk)]
    li = inputs.make_layer(w, 0, device=dev, window_ends=ends)
    B, H = w.B, w.H_kv
    T_cap = budget + chunk
    T_cap += T_cap % 2
    g = GpuCache(torch.zeros(B, H, T_cap, d, dtype=dtype, device=dev),
                 torch.zeros(B, H, T_cap, d, dtype=dtype, device=dev),
                 torch.zeros(B * H, dtype=torch.int32, device=dev),
                 torch.zeros(B, H, T_cap, dtype=torch.float32, device=dev))
    desc = kvs.make_desc(B, H, H * G, d, T_cap, dtype)
    ws = torch.zeros(kvs.workspace_size(desc, W, kvs.OP_PREFILL), dtype=torch.uint8, device=dev)
    L, ties, merged_chunks = 0, 0, 0
    for i, c0 in enumerate(range(0, T, chunk)):
        c1 = ends[i]
        kc = li.K[:, :, c0:c1].contiguous()
        vc = li.V[:, :, c0:c1].contiguous()
        Qw = li.extra["Q_ends"][i].contiguous()
        o_in = to_oracle_cache(g)
        o_out, rounds = oracle.prefill_chunk(o_in, kc.double().cpu().numpy(),
                                             vc.double().cpu().numpy(),
                                             Qw.double().cpu().numpy(), W, budget, sink,
                                             storage_of(dtype))
        L = kvs.prefill_chunk(desc, g.K, g.V, g.logn, g.lens, L, kc, vc, Qw, W, budget, sink, ws)
        torch.cuda.synchronize()
        assert L == min(c1, budget)
        g_out = to_oracle_cache(g)
        assert np.array_equal(g_out.lengths(), o_out.lengths())
        merged_chunks += bool(rounds)
        for b in range(B):
            for h in range(H):
                if not _rows_match(g_out, o_out, b, h, dtype):
                    assert _near_tie(rounds, b, h), f"chunk {i} b={b} h={h} differs without a tie"
                    ties += 1
    REPORTS.append(dict(test=f"prefill {str(dtype).split('.')[-1]} d={d}", chunks=len(ends),
                        chunks_with_rounds=merged_chunks, head_chunks=len(ends) * B * H,
                        near_tie_head_chunks=ties))
    assert merged_chunks >= 2
    assert ties <= 2
    assert kvs.device_flags(ws) == 0


def test_prefill_chunk_flags_a_head_with_another_length(kvs):
    dev = torch.device("cuda")
    B, H, G, d, T_cap = 1, 2, 4, 128, 1024
    desc = kvs.make_desc(B, H, H * G, d, T_cap, torch.bfloat16)
    K = torch.zeros(B, H, T_cap, d, dtype=torch.bfloat16, device=dev)
    V = torch.zeros_like(K)
    logn = torch.zeros(B, H, T_cap, device=dev)
    lens = torch.tensor([100, 96], dtype=torch.int32, device=dev)   # head 1 is not at L
    kc = torch.randn(B, H, 64, d, device=dev).to(torch.bfloat16)
    Qw = torch.randn(B, H * G, 32, d, device=dev).to(torch.bfloat16)
    ws = torch.zeros(kvs.workspace_size(desc, 32, kvs.OP_PREFILL), dtype=torch.uint8, device=dev)
    L = kvs.prefill_chunk(desc, K, V, logn, lens, 100, kc, kc, Qw, 32, 512, 32, ws)
    assert L == 164
    assert kvs.device_flags(ws, clear=True) == kvs.FLAG_BAD_LENGTH
    assert lens.tolist() == [164, 96]
    assert torch.equal(K[0, 0, 100:164], kc[0, 0]) and not K[0, 1].any()
