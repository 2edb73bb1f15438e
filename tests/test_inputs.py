"""The synthetic generator follows its stated recipe (spectra, AR(1), shapes, seeds)."""

import math

import torch

from asymmetric_kv_merging_b200 import inputs


def test_projection_spectra():
    g = torch.Generator().manual_seed(0)
    wk = inputs.projection(64, 16, False, g, "cpu")
    wv = inputs.projection(64, 16, True, g, "cpu")
    sk = torch.linalg.svdvals(wk)
    sv = torch.linalg.svdvals(wv)
    expect = torch.arange(1, 17, dtype=torch.float64) ** -1.5
    assert torch.allclose(sk, expect, rtol=1e-10)
    assert torch.allclose(sv, torch.ones(16, dtype=torch.float64), rtol=1e-10)


def test_ar1_recurrence_and_stationary_scale():
    g = torch.Generator().manual_seed(1)
    rho = 0.9
    T = 3000
    x = inputs.ar1_hidden(T, 64, rho, g, "cpu", chunk=128).double()
    g2 = torch.Generator().manual_seed(1)
    eps = torch.randn(T, 64, generator=g2, dtype=torch.float32).double()
    eps[0] /= math.sqrt(1 - rho * rho)
    ref = torch.zeros_like(eps)
    ref[0] = eps[0]
    for t in range(1, T):
        ref[t] = rho * ref[t - 1] + eps[t]
    assert torch.allclose(x, ref, rtol=1e-4, atol=1e-4)
    var = x.var().item()
    assert abs(var - 1 / (1 - rho * rho)) / (1 / (1 - rho * rho)) < 0.1


def test_layer_shapes_and_determinism():
    w = inputs.small_workload(inputs.WORKLOADS[0], T=96, n_decode=3)
    a = inputs.make_layer(w, 0)
    b = inputs.make_layer(w, 0)
    assert a.K.shape == (1, 2, 100, 64) and a.Q_win.shape == (1, 4, 32, 64)   # 96 + 3, even
    assert a.q_dec.shape == (3, 1, 4, 64) and a.k_new.shape == (3, 1, 2, 64)
    assert torch.equal(a.K, b.K) and torch.equal(a.Q_win, b.Q_win)
    assert torch.all(a.K[:, :, 96:] == 0)
    assert a.lens.tolist() == [[96, 96]]


def test_ragged_lengths_in_range():
    w = inputs.WORKLOADS[4]
    lens = inputs.sequence_lengths(w)
    assert lens.shape == (16,)
    assert int(lens.min()) >= 8192 and int(lens.max()) <= 65536
    assert len(set(lens.tolist())) > 8


def test_layer_rho_in_range():
    w = inputs.WORKLOADS[2]
    rhos = [inputs.layer_rho(w, l) for l in range(32)]
    assert all(0.7 <= r < 0.95 for r in rhos) and len(set(rhos)) == 32


def test_prefill_chunk_accounting():
    from asymmetric_kv_merging_b200 import accounting
    # the pages' setting at steady state: 2048 rows + a 512-row chunk, one round of 512
    b, rounds = accounting.prefill_chunk_bytes(2048, 512, 2048, 32, 32, 128, 2)
    assert rounds == 1
    row = 2 * 128 * 2
    want = (512 * (2 * row + 4)                                           # append
            + 2560 * (row + 4) + 2 * 1248 * (row + 4) + 1248 * 8         # the two window passes
            + (2560 - 32) * (row + 4) + (2048 - 32) * (row + 4))           # in-place merge
    assert b == want
    # the CUDA-core path of fp32 caches reads K once more for the window mass
    bf, _ = accounting.prefill_chunk_bytes(2048, 512, 2048, 32, 32, 128, 2, fused=False)
    assert bf - b == 2560 * (256 + 4 + 4)
    # under the budget: the append only
    assert accounting.prefill_chunk_bytes(0, 512, 2048, 32, 32, 128, 2) == (512 * (2 * row + 4), 0)
