"""Multi-process host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

With N GPUs every rank runs its own replica of the workload (weak scaling, no data
crosses GPUs); the only collectives are the barrier around the timed region and the
max-over-ranks reduction of the step time. Both are exercised here without a GPU.
"""

import os
import socket

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    from asymmetric_kv_merging_b200 import inputs
    r, w, local = bench.dist_setup(world)
    assert (r, w, local) == (rank, world, rank)
    bench.barrier(w)
    t = bench.max_over_ranks(10.0 + rank, w)      # each rank reports its own step time
    # each rank's replica draws its own layers (seed offset by the rank)
    wl = inputs.small_workload(inputs.workload(0), T=64, n_decode=0)
    li = inputs.make_layer(wl, 0 + rank * wl.layers)
    out[rank] = (t, float(li.K.double().sum()))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_ranks_barrier_max_and_distinct_replicas():
    ctx = mp.get_context("spawn")
    world = 2
    port = _free_port()
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=180)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][0] == res[1][0] == 11.0               # the max over ranks, on every rank
    assert res[0][1] != res[1][1]                       # different replicas


def test_round_plan_matches_the_budget():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.plan_rounds(131072, 32768, 32, 32) == [131072, 65568, 32816, 32768]
    assert bench.plan_rounds(32768, 16384, 32, 32) == [32768, 16416, 16384]
    assert torch.tensor(1).item() == 1


def test_round_plan_equals_the_oracle_rounds_for_any_budget():
    """The bench plans its graph of rounds on the host; every planned length must be what
    the oracle's round driver reaches on real data (R = min(P, len - target) per round)."""
    import sys
    sys.path.insert(0, ROOT)
    import numpy as np
    from hypothesis import given, settings, strategies as st

    import bench
    import oracle

    @settings(max_examples=25, deadline=None)
    @given(T=st.integers(70, 240), frac=st.floats(0.15, 1.0), sink=st.integers(0, 12),
           W=st.integers(1, 8))
    def check(T, frac, sink, W):
        target = max(sink + W + 1, int(T * frac))
        try:
            plan = bench.plan_rounds(T, target, sink, W)
        except ValueError:
            return
        rng = np.random.default_rng(T)
        K = rng.normal(size=(1, 1, T, 4))
        V = rng.normal(size=(1, 1, T, 4))
        Q = rng.normal(size=(1, 1, W, 4))
        cache = oracle.cache_from_arrays(K, V, np.array([[T]]))
        lens = [T]
        for _ in range(64):
            if lens[-1] == target:
                break
            r = oracle.merge_round(cache, Q, W, np.array([[sink]]), W, np.array([[target]]))
            cache = r.cache
            lens.append(cache.length(0, 0))
        assert lens == plan

    check()
