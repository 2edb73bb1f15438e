#!/usr/bin/env python
"""Benchmark of the KVSlimmer merging hot path on B200 -- one JSON line on stdout.

A step is one pass of the whole hot path over one batch of synthetic input:
every layer of the workload is scored, merged and compacted round by round to
its budget, then every layer runs the workload's decode steps over its merged
cache (GQA attention with the new row appended each step). The default
workload is the Llama-3.1-8B full-depth 128K case: 32 layers, 8 KV heads,
128K tokens, 4x compression, 128 decode steps per layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvs|reference]

With N > 1 the script runs under torchrun, one process per GPU; every rank
compresses and decodes its own replica (its own seeds), so per-GPU work is
fixed (weak scaling) and no data crosses GPUs; the step time is the maximum
over ranks. `--impl reference` times the fp64 CPU oracle on a bounded sample
of the same workload instead.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from asymmetric_kv_merging_b200 import accounting, inputs  # noqa: E402

METRIC = "merged KV tokens/s and decode µs/token at 128K; achieved HBM GB/s vs peak"
UNIT = "merged KV tokens/s"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["kvs", "reference"], default="kvs")
    ap.add_argument("--workload", type=int, default=2)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill", action="store_true",
                    help="time chunked streaming prefill compression instead (own JSON line)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# process group and clocks
# ---------------------------------------------------------------------------

def dist_setup(n_gpus):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda") if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """nvidia-smi samples of SM clock, power and throttle reasons (every 200 ms)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, local_rank):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [v for v in vis.split(",") if v.strip()]
        self.index = ids[local_rank] if local_rank < len(ids) and ids[local_rank].isdigit() else str(local_rank)
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", self.index], stdout=open(self.path, "w"),
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for name, val in zip(self.NAMES, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# the timed workload
# ---------------------------------------------------------------------------

def plan_rounds(T, target, sink, n_recent):
    """Per-head lengths after each merge round (every head is identical here)."""
    lens = [T]
    while lens[-1] > target:
        L = lens[-1]
        P = max(0, (L - n_recent - sink) // 2)
        R = min(P, L - target)
        if R == 0:
            raise ValueError("budget unreachable")
        lens.append(L - R)
    return lens


class Runner:
    """All device buffers of one replica of the workload, and its two CUDA graphs."""

    def __init__(self, w: inputs.Workload, rank: int, device):
        from asymmetric_kv_merging_b200 import kvs
        self.kvs = kvs
        self.w = w
        self.dev = device
        T = w.T
        self.target = T // w.ratio
        self.lens_plan = plan_rounds(T, self.target, w.sink, w.W)
        self.rounds = len(self.lens_plan) - 1
        # T_cap of the input cache, then of each round's output; the last round writes the
        # per-layer cache that decode appends to, so it keeps room for every decode row
        caps = [T + w.n_decode] + self.lens_plan[1:-1] + [self.target + w.n_decode]
        caps = [c + (c % 2) for c in caps]
        self.caps = caps
        self.layers = []
        for l in range(w.layers):
            li = inputs.make_layer(w, l + rank * w.layers, device=device, T_cap=caps[0])
            self.layers.append(li)
        torch.cuda.synchronize()
        B, H, d = w.B, w.H_kv, w.d
        dt = w.torch_dtype

        def cache(cap):
            return dict(K=torch.zeros(B, H, cap, d, dtype=dt, device=device),
                        V=torch.zeros(B, H, cap, d, dtype=dt, device=device),
                        logn=torch.zeros(B, H, cap, dtype=torch.float32, device=device),
                        lens=torch.zeros(B * H, dtype=torch.int32, device=device))
        self.scratch = [cache(c) for c in caps[1:-1]]           # rounds before the last
        self.final = [cache(caps[-1]) for _ in range(w.layers)]
        self.in_logn = torch.zeros(B, H, caps[0], dtype=torch.float32, device=device)
        self.in_lens = [li.lens.reshape(-1).to(torch.int32).contiguous() for li in self.layers]
        self.cand = torch.full((B * H,), w.sink, dtype=torch.int32, device=device)
        self.tgt = torch.full((B * H,), self.target, dtype=torch.int32, device=device)
        self.score = torch.zeros(B * H * (caps[0] // 2), dtype=torch.float32, device=device)
        self.w_b = torch.zeros_like(self.score)
        self.descs = [kvs.make_desc(B, H, w.H_q, d, c, dt) for c in caps]
        ws_bytes = max(kvs.workspace_size(dsc, w.W, op) for dsc in self.descs
                       for op in (kvs.OP_SCORE, kvs.OP_MERGE, kvs.OP_DECODE))
        self.ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=device)
        self.out = torch.zeros(w.layers, w.n_decode, B, w.H_q, d, dtype=dt, device=device)
        self.stream = torch.cuda.Stream(device)
        self.g_merge = None
        self.g_decode = None

    # one merge pass over every layer
    def merge_all(self):
        kvs, w = self.kvs, self.w
        for l, li in enumerate(self.layers):
            src = dict(K=li.K, V=li.V, logn=self.in_logn, lens=self.in_lens[l])
            for r in range(self.rounds):
                dst = self.final[l] if r == self.rounds - 1 else self.scratch[r]
                kvs.score_pairs(self.descs[r], src["K"], src["V"], src["logn"], src["lens"],
                                self.cand, w.W, li.Q_win, w.W, self.score, self.w_b, self.ws)
                kvs.merge_compact(self.descs[r], src["K"], src["V"], src["logn"], src["lens"],
                                  self.cand, w.W, self.score, self.w_b, self.tgt,
                                  kvs.SCOPE_HEAD, self.caps[r + 1], dst["K"], dst["V"],
                                  dst["logn"], dst["lens"], self.ws)
                src = dst

    # every decode step of every layer (new row appended each step)
    def decode_all(self):
        kvs, w = self.kvs, self.w
        dsc = self.descs[-1]
        for s in range(w.n_decode):
            for l, li in enumerate(self.layers):
                f = self.final[l]
                kvs.decode_attn(dsc, li.q_dec[s], f["K"], f["V"], f["logn"], f["lens"],
                                self.out[l, s], self.ws, li.k_new[s], li.v_new[s])

    def capture(self):
        with torch.cuda.stream(self.stream):
            self.merge_all()            # eager warm-up: first launches, attribute setup
            self.decode_all()
        self.stream.synchronize()
        c0 = self.kvs.launch_count()
        self.g_merge = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_merge, stream=self.stream):
            self.merge_all()
        c1 = self.kvs.launch_count()
        self.g_decode = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_decode, stream=self.stream):
            self.decode_all()
        c2 = self.kvs.launch_count()
        self.launches_merge = c1 - c0
        self.launches_decode = c2 - c1

    def step(self, ev=None):
        with torch.cuda.stream(self.stream):
            if ev:
                ev[0].record(self.stream)
            self.g_merge.replay()
            if ev:
                ev[1].record(self.stream)
            self.g_decode.replay()
            if ev:
                ev[2].record(self.stream)

    def tokens_per_step(self):
        return self.w.layers * self.w.B * self.w.T

    def decode_bytes_per_launch(self):
        w = self.w
        avg_len = self.target + (w.n_decode + 1) / 2.0
        return w.B * w.H_kv * avg_len * accounting.decode_bytes_per_token(w.d, w.elem_bytes)


def run_e2e(rn: Runner, steps, warmup):
    """The same step through the public API with host buffers: every step copies all of
    its inputs from pinned host memory (K, V and window queries of every layer, then the
    decode queries and new rows) and copies the decode outputs and final lengths back.

    Copies run on their own stream, as a serving loop would pipeline them: step k+1's
    K / V / window copies start once step k's merge phase has consumed its inputs (they
    overlap step k's decode phase); step k+1's decode inputs are copied once step k's
    decode phase is done. The timed region spans every copy of every timed step.
    """
    host_m, host_d = [], []
    h2d = 0
    for li in rn.layers:
        hm, hd = {}, {}
        for name, dst in (("K", hm), ("V", hm), ("Q_win", hm), ("q_dec", hd), ("k_new", hd),
                          ("v_new", hd)):
            t = getattr(li, name)
            hp = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
            hp.copy_(t)
            dst[name] = hp
            h2d += t.numel() * t.element_size()
        host_m.append(hm)
        host_d.append(hd)
    out_h = torch.empty(rn.out.shape, dtype=rn.out.dtype, pin_memory=True)
    lens_h = torch.empty(len(rn.final), rn.final[0]["lens"].numel(), dtype=torch.int32, pin_memory=True)
    d2h = out_h.numel() * out_h.element_size() + lens_h.numel() * 4
    st = rn.stream
    cp = torch.cuda.Stream(rn.dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731

    def copy_in(hosts, after):
        with torch.cuda.stream(cp):
            cp.wait_event(after)
            for li, hl in zip(rn.layers, hosts):
                for name, hp in hl.items():
                    getattr(li, name).copy_(hp, non_blocking=True)
            done = ev()
            done.record(cp)
        return done

    def run(n):
        start = ev()
        start.record(st)
        m_in = copy_in(host_m, start)
        d_in = copy_in(host_d, start)
        for k in range(n):
            with torch.cuda.stream(st):
                st.wait_event(m_in)
                rn.g_merge.replay()
                merged = ev()
                merged.record(st)
                if k + 1 < n:
                    m_in = copy_in(host_m, merged)         # overlaps this step's decode
                st.wait_event(d_in)
                rn.g_decode.replay()
                decoded = ev()
                decoded.record(st)
                out_h.copy_(rn.out, non_blocking=True)
                for i, f in enumerate(rn.final):
                    lens_h[i].copy_(f["lens"], non_blocking=True)
                if k + 1 < n:
                    d_in = copy_in(host_d, decoded)
        with torch.cuda.stream(st):
            st.wait_stream(cp)

    run(warmup)
    st.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(st):
        e0.record(st)
    run(steps)
    with torch.cuda.stream(st):
        e1.record(st)
    st.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del host_m, host_d
    return ms, h2d, d2h


# ---------------------------------------------------------------------------
# oracle timing (CPU baseline and reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(w: inputs.Workload, li, target, rounds_lens):
    """Time the fp64 oracle on one KV head of one layer (all rounds) and on two
    decode steps of one layer (all heads); scale to one full step of the workload."""
    import numpy as np
    import oracle
    from threadpoolctl import threadpool_info
    K = li.K[:1, :1].double().cpu().numpy()
    V = li.V[:1, :1].double().cpu().numpy()
    lens = np.array([[w.T]])
    Q = li.Q_win[:1, :w.G].double().cpu().numpy()
    cache = oracle.cache_from_arrays(K, V, lens)
    t0 = time.perf_counter()
    out, rounds = oracle.compress(cache, Q, w.W, np.array([[w.sink]]), w.W, np.array([[target]]),
                                  storage="bf16" if w.dtype == "bf16" else "f32")
    t_merge_head = time.perf_counter() - t0
    # two decode steps over one layer's compressed head, all query heads of that head
    qd = li.q_dec[:2, :1, :w.G].double().cpu().numpy()
    kn = li.k_new[:2, :1, :1].double().cpu().numpy()
    vn = li.v_new[:2, :1, :1].double().cpu().numpy()
    t0 = time.perf_counter()
    for s in range(2):
        _, out = oracle.decode_step(out, qd[s], kn[s], vn[s])
    t_dec_head = (time.perf_counter() - t0) / 2
    per_step = (w.layers * w.B * w.H_kv * t_merge_head
                + w.n_decode * w.layers * w.B * w.H_kv * t_dec_head)
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    sample = (f"oracle on KV head 0 of layer 0 (all {len(rounds)} rounds, {w.T} -> {target} rows: "
              f"{t_merge_head:.2f} s) and 2 decode steps of that head ({t_dec_head * 1e3:.1f} ms "
              f"each); scaled x{w.layers * w.B * w.H_kv} heads and x{w.n_decode} steps")
    return per_step, t_merge_head + 2 * t_dec_head, threads, sample


def reference_main(args, rank, world):
    if rank != 0:
        return
    w = inputs.workload(args.workload)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    li = inputs.make_layer(w, 0, device=dev)
    target = w.T // w.ratio
    lens = plan_rounds(w.T, target, w.sink, w.W)
    for _ in range(args.warmup):
        oracle_sample(w, li, target, lens)
    per = []
    threads, sample = 1, ""
    for _ in range(args.steps):
        per_step, _, threads, sample = oracle_sample(w, li, target, lens)
        per.append(per_step)
    ms = statistics.mean(per) * 1e3
    value = w.layers * w.B * w.T / (ms / 1e3)
    cores = threads
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


L2_BYTES = 126 * 1024 * 1024


def config_of(w, n_gpus):
    kv = 2 * w.layers * w.B * w.H_kv * w.T * w.d * w.elem_bytes
    dec = 2 * w.B * w.H_kv * (w.T // w.ratio) * w.d * w.elem_bytes
    l2 = (f"inputs larger than L2 ({kv / 2**30:.2f} GiB of K/V per replica; no flush needed)"
          if kv > L2_BYTES else f"inputs of {kv / 2**20:.1f} MiB fit in L2")
    if dec <= L2_BYTES and w.layers * dec > L2_BYTES:
        l2 += ("; decode rotates over the layers' merged caches "
               f"({w.layers} x {dec / 2**20:.1f} MiB), larger than L2 together")
    elif dec <= L2_BYTES:
        l2 += (f"; the merged decode cache ({dec / 2**20:.1f} MiB) fits in L2, so decode "
               "steps may hit it")
    return {"workload": w.name, "B": w.B, "layers": w.layers, "T": w.T, "H_kv": w.H_kv,
            "H_q": w.H_q, "d": w.d, "ratio": w.ratio, "budget_per_head": w.T // w.ratio,
            "decode_steps_per_layer": w.n_decode, "window": w.W, "sink": w.sink,
            "parallelism": f"replicas x{n_gpus}" if n_gpus > 1 else "single GPU", "l2": l2}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


PREFILL = dict(layers=32, T=131072, chunk=512, budget=2048, sink=32, W=32)


def prefill_main(args, rank, world, local):
    """Chunked streaming prefill compression (the pages' serving setting: budget 2048,
    chunk 512, 32 preserved initial tokens) of a 128K prompt in every layer of the
    Llama-3.1-8B-shaped model. After the forward pass of a chunk every layer's cache
    takes that chunk and is merged back to the budget before the next chunk, so the
    layers of one chunk go in one kvs_prefill_chunk call, stacked along the batch axis
    (B = layers). One step = the whole prompt (256 calls); the calls of a step are
    captured once into a CUDA graph and replayed."""
    from asymmetric_kv_merging_b200 import kvs
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    c = PREFILL
    w = inputs.small_workload(inputs.workload(2), layers=c["layers"], T=c["T"], n_decode=0)
    assert w.B == 1 and w.T % c["chunk"] == 0
    n_chunks = w.T // c["chunk"]
    ends = [(i + 1) * c["chunk"] for i in range(n_chunks)]
    T_cap = c["budget"] + c["chunk"]
    NL, H, Hq, d, ch = w.layers, w.H_kv, w.H_q, w.d, c["chunk"]
    desc = kvs.make_desc(NL, H, Hq, d, T_cap, torch.bfloat16)
    ws = torch.zeros(kvs.workspace_size(desc, c["W"], kvs.OP_PREFILL), dtype=torch.uint8,
                     device=dev)
    k_chunks = torch.empty(n_chunks, NL, H, ch, d, dtype=torch.bfloat16, device=dev)
    v_chunks = torch.empty_like(k_chunks)
    q_wins = torch.empty(n_chunks, NL, Hq, c["W"], d, dtype=torch.bfloat16, device=dev)
    for layer in range(NL):
        li = inputs.make_layer(w, layer + 1000 * rank, device=dev, window_ends=ends)
        k_chunks[:, layer] = li.K[0, :, :w.T].view(H, n_chunks, ch, d).transpose(0, 1)
        v_chunks[:, layer] = li.V[0, :, :w.T].view(H, n_chunks, ch, d).transpose(0, 1)
        q_wins[:, layer] = li.extra["Q_ends"][:, 0]
        del li
    cache = dict(K=torch.zeros(NL, H, T_cap, d, dtype=torch.bfloat16, device=dev),
                 V=torch.zeros(NL, H, T_cap, d, dtype=torch.bfloat16, device=dev),
                 logn=torch.zeros(NL, H, T_cap, device=dev),
                 lens=torch.zeros(NL * H, dtype=torch.int32, device=dev))
    stream = torch.cuda.Stream(device=dev)

    def step():
        cache["lens"].zero_()
        L = 0
        for i in range(n_chunks):
            L = kvs.prefill_chunk(desc, cache["K"], cache["V"], cache["logn"], cache["lens"], L,
                                  k_chunks[i], v_chunks[i], q_wins[i], c["W"], c["budget"],
                                  c["sink"], ws)
        assert L == c["budget"]

    with torch.cuda.stream(stream):
        step()                                   # eager pass: kernel attributes, first loads
    torch.cuda.synchronize()
    launches0 = kvs.launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    launches_per_step = kvs.launch_count() - launches0
    with torch.cuda.stream(stream):             # replays and events on the same stream
        for _ in range(args.warmup):
            graph.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    flags = kvs.device_flags(ws)
    tokens = NL * w.T * world
    step_bytes = prefill_step_bytes(w, c)
    peak, peak_kind = peaks()
    achieved = step_bytes / (ms / 1e3) / 1e9
    if rank == 0:
        print(json.dumps({
            "metric": "chunked prefill compression: prompt tokens/s", "value": tokens / (ms / 1e3),
            "unit": "prompt tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "llama8b_32L_prefill128K", "B": 1, "layers": NL,
                       "T": w.T, "H_kv": H, "H_q": Hq, "d": d, "budget": c["budget"],
                       "chunk": ch, "sink": c["sink"], "window": c["W"],
                       "calls_per_step": n_chunks, "layers_per_call": NL,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
            "us_per_chunk_call": ms * 1e3 / n_chunks,
            "gpu_launches": launches_per_step * args.steps, "device_flags": flags,
            "roofline": {"kernel": "whole chunk call (append, window passes, pair scoring, "
                                   "selection, in-place merge)", "bound": "hbm",
                         "achieved": achieved, "peak": peak, "peak_kind": peak_kind,
                         "unit": "GB/s", "frac": achieved / peak, "traffic": None,
                         "bytes_per_step": step_bytes},
            "clocks": clk}))


def prefill_step_bytes(w, c):
    """Algorithmic bytes of one prompt through the chunked prefill, all layers and
    heads of one replica (the per-head accounting of every chunk call)."""
    total, L = 0, 0
    for e in range(0, w.T, c["chunk"]):
        n = min(c["chunk"], w.T - e)
        b, _ = accounting.prefill_chunk_bytes(L, n, c["budget"], c["sink"], c["W"], w.d,
                                              w.elem_bytes)
        total += b
        L = min(L + n, c["budget"])
    return total * w.layers * w.B * w.H_kv


def main():
    args = parse_args()
    rank, world, local = dist_setup(args.gpus)
    if args.impl == "reference":
        reference_main(args, rank, world)
        return
    if args.prefill:
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA device (the kernels have no CPU path)")
        prefill_main(args, rank, world, local)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the kernels have no CPU path)")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = inputs.workload(args.workload)
    rn = Runner(w, rank, dev)
    rn.capture()
    for _ in range(args.warmup):
        rn.step()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for k in range(args.steps):
        rn.step(evs[k])
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    merge_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    decode_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    step_ms = evs[0][0].elapsed_time(evs[-1][2]) / args.steps
    step_ms = max_over_ranks(step_ms, world)
    merge_ms = max_over_ranks(merge_ms, world)
    decode_ms = max_over_ranks(decode_ms, world)
    tokens = rn.tokens_per_step() * world
    value = tokens / (step_ms / 1e3)

    peak, peak_kind = peaks()
    n_dec_launch = w.n_decode * w.layers
    dec_launch_ms = decode_ms / n_dec_launch
    achieved = rn.decode_bytes_per_launch() / (dec_launch_ms / 1e3) / 1e9
    traffic = None
    prof = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if os.path.exists(prof):
        # one ncu capture's DRAM bytes per launch, scaled by rows processed to this launch
        # (the capture shows traffic equal to the algorithmic bytes, so it scales in proportion)
        with open(prof) as f:
            tr = json.load(f)
        traffic = (tr["measured_dram_bytes_per_launch"] * rn.decode_bytes_per_launch()
                   / tr["measured_algorithmic_bytes_per_launch"])

    e2e = None
    if not args.no_e2e:
        e2e_ms, h2d, d2h = run_e2e(rn, max(3, args.steps), 1)
        e2e_ms = max_over_ranks(e2e_ms, world)
        e2e = {"value": tokens / (e2e_ms / 1e3), "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        per_step, spent, threads, sample = oracle_sample(w, rn.layers[0], rn.target, rn.lens_plan)
        cpu = {"value": rn.tokens_per_step() / per_step, "unit": UNIT, "cores": threads,
               "kind": "oracle", "sample": sample, "cpu_seconds_spent": round(spent, 2),
               "host_cpus": os.cpu_count()}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_of(w, world),
            "merge_ms_per_step": merge_ms, "decode_ms_per_step": decode_ms,
            "merge_tokens_per_s": tokens / (merge_ms / 1e3),
            "decode_us_per_token": decode_ms * 1e3 / w.n_decode,
            "decode_us_per_token_note": "one generated token = one decode step over all layers",
            "clocks": clk,
            "e2e": e2e,
            "gpu_launches": (rn.launches_merge + rn.launches_decode) * args.steps,
            "roofline": {"kernel": "decode_tc_kernel (GQA decode, one thread-block cluster per KV head)", "bound": "hbm",
                         "achieved": achieved, "peak": peak, "peak_kind": peak_kind,
                         "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                         "bytes_per_launch": rn.decode_bytes_per_launch(),
                         "launch_ms": dec_launch_ms},
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        del rn
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
