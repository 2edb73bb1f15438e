"""Launch set-up that is cached on the host: kernel attributes (dynamic shared-memory
limits, cluster sizes) are set per device and per kernel, so the order in which shapes
and devices are first used cannot leave a later launch without the limit it needs."""

import numpy as np
import pytest
import torch

import oracle
from asymmetric_kv_merging_b200 import inputs
from parity import GpuCache, Stats, compare_decode, compare_round, gpu_round, to_oracle_cache

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvs():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from asymmetric_kv_merging_b200 import build
    build.build()
    from asymmetric_kv_merging_b200 import kvs as mod
    return mod


def _one_round(kvs, dev, d, H_kv, G, W, T, seed, stats, dtype="f32"):
    """One scoring + merge round and one decode step on `dev`, against the oracle."""
    w = inputs.small_workload(inputs.workload(0), H_kv=H_kv, H_q=H_kv * G, d=d, T=T, W=W,
                              n_decode=1, dtype=dtype)
    li = inputs.make_layer(w, seed)
    with torch.cuda.device(dev):
        g = GpuCache(li.K.to(dev), li.V.to(dev), li.lens.to(dev))
        B, H, T_cap, _ = g.K.shape
        target_np = li.lens.view(B, H).numpy() * 3 // 4
        target = torch.tensor(target_np.reshape(-1), dtype=torch.int32, device=dev)
        cand = torch.full((B * H,), 32, dtype=torch.int32, device=dev)
        cand_np = np.full((B, H), 32)
        dt = w.torch_dtype
        ws = kvs.workspace(kvs.make_desc(B, H, w.H_q, d, T_cap, dt), W, device=dev)
        o = to_oracle_cache(g)
        r = oracle.merge_round(o, li.Q_win.double().numpy(), W, cand_np, W, target_np, "head",
                               w.dtype)
        gout, gres = gpu_round(g, w.H_q, li.Q_win.to(dev), W, cand, W, target, kvs.SCOPE_HEAD, ws)
        compare_round(r, gres, gout, o, dt, "head", None, stats, cand_np, W)
        o = to_oracle_cache(gout)
        out = torch.empty(B, w.H_q, d, dtype=dt, device=dev)
        desc = kvs.make_desc(B, H, w.H_q, d, T_cap, dt)
        kvs.decode_attn(desc, li.q_dec[0].to(dev), gout.K, gout.V, gout.logn, gout.lens, out, ws,
                        li.k_new[0].to(dev), li.v_new[0].to(dev))
        oo, _ = oracle.decode_step(o, li.q_dec[0].double().numpy(), li.k_new[0].double().numpy(),
                                   li.v_new[0].double().numpy())
        compare_decode(oo, out, dt, stats)
        assert kvs.device_flags(ws) == 0


def test_fp32_window_head_dims_in_either_order(kvs):
    """The CUDA-core window kernels need more dynamic shared memory for d = 64 with
    G*W = 128 than for d = 128 with G*W = 64; running the second after the first in one
    process must still raise the limit for the kernel that needs it."""
    dev = torch.device("cuda", 0)
    stats = Stats()
    _one_round(kvs, dev, d=128, H_kv=2, G=2, W=32, T=700, seed=1, stats=stats)
    _one_round(kvs, dev, d=64, H_kv=2, G=4, W=32, T=700, seed=2, stats=stats)
    _one_round(kvs, dev, d=128, H_kv=2, G=4, W=32, T=700, seed=3, stats=stats)
    stats.report("fp32 window shapes in one process")
    assert stats.rounds == 3


def test_second_device_after_the_first(kvs):
    """Kernel attributes are per device: the same shapes on device 1 after device 0."""
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two CUDA devices")
    stats = Stats()
    for i in (0, 1):
        for dtype in ("f32", "bf16"):
            _one_round(kvs, torch.device("cuda", i), d=128, H_kv=2, G=4, W=32, T=700, seed=4,
                       stats=stats, dtype=dtype)
    stats.report("device 0 then device 1")
