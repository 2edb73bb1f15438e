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
    ap.add_argument("--form", choices=["full", "diagonal", "per_query"], default="full",
                    help="scoring form: the full coupled form with the window mean (default), "
                         "the diagonal-only ablation, or the window read query by query")
    ap.add_argument("--layers", type=int, default=None,
                    help="fewer layers than the workload has (reduced runs for profiler captures)")
    ap.add_argument("--batch", type=int, default=None,
                    help="fewer sequences than the workload has (reduced runs for profiler captures)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill", action="store_true",
                    help="time chunked streaming prefill compression instead (own JSON line)")
    ap.add_argument("--fp32", action="store_true",
                    help="the workload with fp32 caches (the CUDA-core kernels), for profiling")
    ap.add_argument("--stream-ceiling", action="store_true",
                    help="time the decode's read pattern with no arithmetic (own JSON line)")
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

def reduced(w, args):
    """The workload with fewer layers or sequences, when asked for (profiler captures of
    a small case); its name says so."""
    ch = {}
    if args.layers is not None and args.layers < w.layers:
        ch["layers"] = args.layers
    if args.batch is not None and args.batch < w.B:
        ch["B"] = args.batch
    if not ch:
        return w
    tag = "".join(f"_{k}{v}" for k, v in ch.items())
    return inputs.small_workload(w, name=w.name + "_reduced" + tag, **ch)


def plan_rounds(T, target, sink, n_recent):
    """Per-head lengths after each merge round (a round merges R = min(P, len - target))."""
    lens = [T]
    while lens[-1] > target:
        L = lens[-1]
        P = max(0, (L - n_recent - sink) // 2)
        R = min(P, L - target)
        if R == 0:
            raise ValueError("budget unreachable")
        lens.append(L - R)
    return lens


def batch_plan(lens, target, scope, sink, n_recent):
    """Round plan of a batch of heads, on the host.

    lens: (B, H) lengths; target: (B, H) per head or (B,) per sequence (pooled).
    Returns a list with one entry per round: (len_in (B, H), len_out_upper (B, H),
    total_out (B,)). Per-head scope is exact. In pooled scope a round that merges every
    candidate pair of a sequence is exact too; a round that merges fewer leaves each
    head's length between len - P and len (the total is exact), so it must be the last.
    """
    import numpy as np
    L = np.asarray(lens, dtype=np.int64).copy()
    target = np.asarray(target, dtype=np.int64)
    rounds = []
    tot = L.sum(axis=1)
    partial = False
    for _ in range(64):
        if scope == "head":
            if np.all(L <= target):
                return rounds
            P = np.maximum(0, (L - n_recent - sink) // 2)
            R = np.minimum(P, np.maximum(0, L - target))
            if not R.any():
                raise ValueError("budget unreachable")
            rounds.append((L.copy(), L - R, (L - R).sum(axis=1)))
            L = L - R
        else:
            if np.all(tot <= target):
                return rounds
            if partial:
                raise ValueError("a partial pooled round must be the last")
            P = np.maximum(0, (L - n_recent - sink) // 2)
            Rs = np.minimum(P.sum(axis=1), np.maximum(0, tot - target))
            if not Rs.any():
                raise ValueError("budget unreachable")
            full = Rs == P.sum(axis=1)
            upper = np.where(full[:, None], L - P, L)
            rounds.append((L.copy(), upper, tot - Rs))
            partial = not full.all()
            L, tot = upper, tot - Rs
    raise ValueError("no plan within 64 rounds")


class Runner:
    """All device buffers of one replica of a workload, and its two CUDA graphs.

    One step = every layer merged round by round to its budget (the merge phase), then
    the decode phase: every layer's decode steps with the new row appended; with
    `remerge_every` (the serving mix) the newest `remerge_every` rows of every head are
    merged in place to 1/8 of their count after each such segment of decode steps.
    """

    def __init__(self, w: inputs.Workload, rank: int, device, form=None):
        import numpy as np
        from asymmetric_kv_merging_b200 import kvs
        self.kvs = kvs
        self.w = w
        self.dev = device
        self.form = form
        B, H, d = w.B, w.H_kv, w.d
        seq = inputs.sequence_lengths(w).numpy()
        self.seq_lens = seq
        lens0 = np.repeat(seq[:, None], H, axis=1)
        if w.scope == "pooled":
            self.target_np = (lens0 // w.ratio).sum(axis=1)
        else:
            self.target_np = lens0 // w.ratio
        self.scope = w.scope
        self.scope_code = kvs.SCOPE_POOLED if w.scope == "pooled" else kvs.SCOPE_HEAD
        self.plan = batch_plan(lens0, self.target_np, w.scope, w.sink, w.W)
        self.rounds = len(self.plan)
        final_upper = self.plan[-1][1]
        # decode-phase lengths per head (exact when the last round is exact)
        self.lens_after = final_upper
        extra = w.n_decode
        cap0 = int(seq.max()) + w.n_decode
        caps = [cap0] + [int(r[1].max()) for r in self.plan[:-1]] + [int(final_upper.max()) + extra]
        caps = [c + (c % 2) for c in caps]
        self.caps = caps
        self.layers = [inputs.make_layer(w, l + rank * w.layers, device=device, T_cap=caps[0])
                       for l in range(w.layers)]
        torch.cuda.synchronize()
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
        self.tgt = torch.tensor(self.target_np.reshape(-1), dtype=torch.int32, device=device)
        self.score = torch.zeros(B * H * (caps[0] // 2), dtype=torch.float32, device=device)
        self.w_b = torch.zeros_like(self.score)
        self.descs = [kvs.make_desc(B, H, w.H_q, d, c, dt) for c in caps]
        ws_bytes = max(kvs.workspace_size(dsc, w.W, op) for dsc in self.descs
                       for op in (kvs.OP_SCORE, kvs.OP_MERGE, kvs.OP_DECODE))
        self.ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=device)
        self.out = torch.zeros(w.layers, w.n_decode, B, w.H_q, d, dtype=dt, device=device)
        # serving mix: in-place re-merge of the newest rows after every segment
        self.remerge = []
        if w.remerge_every:
            if self.scope != "head":
                raise ValueError("re-merge is per head")
            seg = w.remerge_every
            L = final_upper.astype(np.int64).copy()
            for s0 in range(0, w.n_decode, seg):
                L = L + seg
                # the window: the last W decode queries of the segment, [B, H_q, W, d]
                Qw = [li.q_dec[s0 + seg - w.W:s0 + seg].permute(1, 2, 0, 3).contiguous()
                      for li in self.layers]
                subs = []
                n = seg
                while n > seg // w.remerge_ratio:
                    cand = L - n
                    tgt = L - n // 2
                    subs.append(dict(
                        cand=torch.tensor(cand.reshape(-1), dtype=torch.int32, device=device),
                        tgt=torch.tensor(tgt.reshape(-1), dtype=torch.int32, device=device),
                        L=L.copy(), n=n))
                    L = tgt
                    n //= 2
                self.remerge.append(dict(s0=s0, Qw=Qw, subs=subs))
        self.stream = torch.cuda.Stream(device)
        self.g_merge = None
        self.g_decode = None

    # one merge pass over every layer
    def merge_all(self, timer=None):
        kvs, w = self.kvs, self.w
        for l, li in enumerate(self.layers):
            src = dict(K=li.K, V=li.V, logn=self.in_logn, lens=self.in_lens[l])
            for r in range(self.rounds):
                dst = self.final[l] if r == self.rounds - 1 else self.scratch[r]
                with _timed(timer, "score"):
                    kvs.score_pairs(self.descs[r], src["K"], src["V"], src["logn"], src["lens"],
                                    self.cand, w.W, li.Q_win, w.W, self.score, self.w_b, self.ws,
                                    form=self.form)
                with _timed(timer, "merge"):
                    kvs.merge_compact(self.descs[r], src["K"], src["V"], src["logn"], src["lens"],
                                      self.cand, w.W, self.score, self.w_b, self.tgt,
                                      self.scope_code, self.caps[r + 1], dst["K"], dst["V"],
                                      dst["logn"], dst["lens"], self.ws)
                src = dst

    # every decode step of every layer (new row appended each step), with the re-merges
    def decode_all(self, timer=None):
        kvs, w = self.kvs, self.w
        dsc = self.descs[-1]
        seg = w.remerge_every or w.n_decode
        for s in range(w.n_decode):
            with _timed(timer, "decode"):
                for l, li in enumerate(self.layers):
                    f = self.final[l]
                    kvs.decode_attn(dsc, li.q_dec[s], f["K"], f["V"], f["logn"], f["lens"],
                                    self.out[l, s], self.ws, li.k_new[s], li.v_new[s])
            if self.remerge and (s + 1) % seg == 0:
                rm = self.remerge[s // seg]
                with _timed(timer, "remerge"):
                    for l in range(w.layers):
                        f = self.final[l]
                        for sub in rm["subs"]:
                            kvs.score_pairs(dsc, f["K"], f["V"], f["logn"], f["lens"], sub["cand"],
                                            0, rm["Qw"][l], w.W, self.score, self.w_b, self.ws,
                                            form=self.form)
                            kvs.merge_compact(dsc, f["K"], f["V"], f["logn"], f["lens"],
                                              sub["cand"], 0, self.score, self.w_b, sub["tgt"],
                                              kvs.SCOPE_HEAD, self.caps[-1], f["K"], f["V"],
                                              f["logn"], f["lens"], self.ws)

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

    def breakdown(self):
        """Device time of each kind of library call, from one eager pass of a step with
        CUDA events around every call on the launching stream. A sleep kernel first lets
        the host queue ahead of the device, so that the events time device work rather
        than host launch gaps. Returns {kind: ms per step}."""
        timer = {}
        with torch.cuda.stream(self.stream):
            torch.cuda._sleep(200_000_000)
            self.merge_all(timer)
            self.decode_all(timer)
        self.stream.synchronize()
        return {k: sum(a.elapsed_time(b) for a, b in v) for k, v in timer.items()}

    def tokens_per_step(self):
        return step_tokens(self.w)

    # ---- algorithmic bytes (per step, this replica) ----
    def score_bytes(self):
        w, eb = self.w, self.w.elem_bytes
        tot = 0
        for (L_in, _, _) in self.plan:
            P = (L_in - w.W - w.sink) // 2
            tot += sum(accounting.score_bytes(int(a), max(0, int(p)), w.d, eb, w.dtype == "bf16")
                       for a, p in zip(L_in.reshape(-1), P.reshape(-1)))
        return tot * w.layers

    def merge_bytes(self):
        w, eb = self.w, self.w.elem_bytes
        tot = 0
        for (L_in, _, tot_out) in self.plan:
            tot += accounting.merge_bytes(int(L_in.sum()), int(tot_out.sum()), w.d, eb)
        return tot * w.layers

    def decode_bytes(self):
        """Every decode launch reads, per head, its cached rows and the appended one
        (row totals per sequence are exact even where per-head lengths are not known)."""
        w = self.w
        per_tok = accounting.decode_bytes_per_token(w.d, w.elem_bytes)
        rows = float(self.plan[-1][2].sum())
        heads = w.B * w.H_kv
        seg = w.remerge_every or w.n_decode
        tot = 0.0
        for s in range(w.n_decode):
            rows += heads                       # the appended row of every head
            tot += rows * per_tok
            if self.remerge and (s + 1) % seg == 0:
                rows -= heads * (seg - seg // w.remerge_ratio)
        return tot * w.layers

    def remerge_bytes(self):
        w, eb = self.w, self.w.elem_bytes
        tot = 0
        for rm in self.remerge:
            for sub in rm["subs"]:
                n, L = sub["n"], sub["L"]
                P, R = n // 2, n // 2
                for Lh in L.reshape(-1):
                    tot += accounting.score_bytes(int(Lh), P, w.d, eb, w.dtype == "bf16")
                    tot += accounting.merge_bytes(n, n - R, w.d, eb)
        return tot * w.layers

    def decode_launches(self):
        return self.w.n_decode * self.w.layers

    def decode_bytes_per_launch(self):
        return self.decode_bytes() / self.decode_launches()


def step_tokens(w: inputs.Workload) -> int:
    """Merged KV tokens of one step: every input position of every sequence of every
    layer, plus the rows the re-merges take in (one token = one position of one
    sequence across all KV heads of one layer)."""
    t = int(inputs.sequence_lengths(w).sum()) * w.layers
    if w.remerge_every:
        t += (w.n_decode // w.remerge_every) * w.remerge_every * w.B * w.layers
    return t


class _timed:
    """Context manager that brackets library calls with CUDA events (no-op without a
    timer dict)."""

    def __init__(self, timer, kind):
        self.timer, self.kind = timer, kind

    def __enter__(self):
        if self.timer is not None:
            self.e0 = torch.cuda.Event(enable_timing=True)
            self.e0.record()
        return self

    def __exit__(self, *exc):
        if self.timer is not None:
            e1 = torch.cuda.Event(enable_timing=True)
            e1.record()
            self.timer.setdefault(self.kind, []).append((self.e0, e1))
        return False


def run_e2e(rn: Runner, steps, warmup):
    """The same step through the public API with host buffers: every step copies all of
    its inputs from pinned host memory (K, V and window queries of every layer, then the
    decode queries and new rows, and the re-merge windows) and copies the decode outputs
    and final lengths back.

    Copies run on their own stream, as a serving loop would pipeline them: step k+1's
    K / V / window copies start once step k's merge phase has consumed its inputs (they
    overlap step k's decode phase); step k+1's decode inputs are copied once step k's
    decode phase is done. The timed region spans every copy of every timed step.
    """
    host_m, host_d = [], []
    h2d = 0

    def pin(t):
        hp = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        hp.copy_(t)
        return hp

    for l, li in enumerate(rn.layers):
        hm, hd = {}, {}
        for name, dst in (("K", hm), ("V", hm), ("Q_win", hm), ("q_dec", hd), ("k_new", hd),
                          ("v_new", hd)):
            t = getattr(li, name)
            dst[(name, None)] = (t, pin(t))
            h2d += t.numel() * t.element_size()
        for i, rm in enumerate(rn.remerge):
            t = rm["Qw"][l]
            hd[("Qw", i)] = (t, pin(t))
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
            for hl in hosts:
                for dev_t, hp in hl.values():
                    dev_t.copy_(hp, non_blocking=True)
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

def _oracle_unit(job):
    """Worker (a spawned process): the fp64 oracle, single-threaded, on one selection unit
    (one KV head, or one sequence's heads in pooled scope): every merge round to the
    budget, then `n_dec` decode steps. Returns (merge s, decode s per step, rounds)."""
    path, W, sink, storage, scope, n_dec = job
    import numpy as np
    from threadpoolctl import threadpool_limits
    import oracle
    z = np.load(path)
    with threadpool_limits(1):
        cache = oracle.cache_from_arrays(z["K"], z["V"], z["lens"])
        t0 = time.perf_counter()
        out, rounds = oracle.compress(cache, z["Q"], W, z["cand"], W, z["target"], scope,
                                      storage=storage)
        t1 = time.perf_counter()
        for s in range(n_dec):
            _, out = oracle.decode_step(out, z["qd"][s], z["kn"][s], z["vn"][s])
        t2 = time.perf_counter()
    return t1 - t0, (t2 - t1) / max(n_dec, 1), len(rounds)


def oracle_units(w: inputs.Workload, layers, n_units):
    """The first n_units selection units of the workload (layer-major), as numpy files
    for the oracle workers: fp64 copies of the stored bf16 / fp32 inputs."""
    import numpy as np
    d = tempfile.mkdtemp(prefix="kvs_oracle_")
    paths = []
    G = w.G
    for li in layers:
        lens = li.lens.view(w.B, w.H_kv).cpu().numpy()
        for b in range(w.B):
            heads = [list(range(w.H_kv))] if w.scope == "pooled" else [[h] for h in range(w.H_kv)]
            for hs in heads:
                if len(paths) == n_units:
                    return paths, d
                T_b = int(lens[b, 0])
                h0, h1 = hs[0], hs[-1] + 1
                sl = lambda t: t[b:b + 1, h0:h1, :T_b].double().cpu().numpy()  # noqa: E731
                qd = li.q_dec[:2, b:b + 1, h0 * G:h1 * G].double().cpu().numpy()
                kn = li.k_new[:2, b:b + 1, h0:h1].double().cpu().numpy()
                vn = li.v_new[:2, b:b + 1, h0:h1].double().cpu().numpy()
                tgt = (np.array([[T_b // w.ratio] * len(hs)]) if w.scope == "head"
                       else np.array([(T_b // w.ratio) * len(hs)]))
                p = os.path.join(d, f"u{len(paths)}.npz")
                np.savez(p, K=sl(li.K), V=sl(li.V), lens=np.full((1, len(hs)), T_b),
                         Q=li.Q_win[b:b + 1, h0 * G:h1 * G].double().cpu().numpy(),
                         cand=np.full((1, len(hs)), w.sink), target=tgt, qd=qd, kn=kn, vn=vn)
                paths.append(p)
    return paths, d


def oracle_pool(w: inputs.Workload, paths, workers):
    """Run the oracle on every unit file with `workers` spawned single-threaded processes
    (spawn: safe after CUDA is initialised). Returns the per-unit results and wall s."""
    import multiprocessing as mp
    import shutil
    storage = "bf16" if w.dtype == "bf16" else "f32"
    n_dec = min(2, w.n_decode)
    jobs = [(p, w.W, w.sink, storage, w.scope, n_dec) for p in paths]
    t0 = time.perf_counter()
    with mp.get_context("spawn").Pool(workers) as pool:
        res = pool.map(_oracle_unit, jobs, chunksize=1)
    wall = time.perf_counter() - t0
    shutil.rmtree(os.path.dirname(paths[0]), ignore_errors=True)
    return res, wall


def units_per_step(w: inputs.Workload):
    return w.layers * w.B * (1 if w.scope == "pooled" else w.H_kv)


def oracle_step_seconds(w: inputs.Workload, res, workers):
    """One step of the workload on `workers` cores: every unit's merge rounds and
    n_decode decode steps, the units spread evenly over the cores."""
    t_merge = statistics.mean(r[0] for r in res)
    t_dec = statistics.mean(r[1] for r in res)
    waves = -(-units_per_step(w) // workers)          # a unit runs on one core
    return waves * (t_merge + w.n_decode * t_dec), t_merge, t_dec


def oracle_single_thread_workload0():
    """The oracle on the tiny fp32 workload (T = 512, 2 KV heads), single-threaded:
    merged tokens/s of its compression rounds."""
    import numpy as np
    from threadpoolctl import threadpool_limits
    import oracle
    w0 = inputs.workload(0)
    li = inputs.make_layer(w0, 0)
    B, H = w0.B, w0.H_kv
    with threadpool_limits(1):
        cache = oracle.cache_from_arrays(li.K.double().numpy(), li.V.double().numpy(),
                                         li.lens.numpy())
        t0 = time.perf_counter()
        oracle.compress(cache, li.Q_win.double().numpy(), w0.W, np.full((B, H), w0.sink), w0.W,
                        np.full((B, H), w0.T // w0.ratio), storage="f32")
        dt = time.perf_counter() - t0
    return B * w0.T / dt


def cpu_baseline(w: inputs.Workload, layers, tokens_per_step):
    """The oracle as it stands on the host's cores: one unit per core, run in parallel."""
    workers = max(1, os.cpu_count() or 1)
    n = min(workers, units_per_step(w))
    paths, _ = oracle_units(w, layers, n)
    res, wall = oracle_pool(w, paths, workers=len(paths))
    per_step, t_merge, t_dec = oracle_step_seconds(w, res, len(paths))
    return {"value": tokens_per_step / per_step, "unit": UNIT, "cores": len(paths),
            "kind": "oracle",
            "sample": (f"{len(paths)} selection units of layer 0 on, one per core in "
                       f"single-threaded processes ({res[0][2]} rounds each, mean {t_merge:.2f} s; "
                       f"then 2 decode steps, mean {t_dec * 1e3:.1f} ms each), {wall:.1f} s wall; "
                       f"scaled to {units_per_step(w)} units and {w.n_decode} decode steps "
                       f"spread over {len(paths)} cores"),
            "host_cpus": os.cpu_count(),
            "single_thread_workload0_tokens_per_s": oracle_single_thread_workload0()}


def reference_main(args, rank, world):
    """The reference arm: the oracle as it stands. Every step is one selection unit of
    the workload (all its merge rounds, then two decode steps), the units of all steps
    running in parallel single-threaded processes, one per host core; a step's time is
    scaled to the whole workload on those cores."""
    if rank != 0:
        return
    w = inputs.workload(args.workload)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    cores = max(1, os.cpu_count() or 1)
    # at least one unit per core, so that every unit is timed with all cores busy
    need = max(args.steps + args.warmup, cores)
    per_layer = w.B * (1 if w.scope == "pooled" else w.H_kv)
    layers = [inputs.make_layer(w, l, device=dev) for l in range((need + per_layer - 1) // per_layer)]
    paths, _ = oracle_units(w, layers, need)
    workers = cores
    res, wall = oracle_pool(w, paths, workers)
    res = res[args.warmup:]
    per_step, t_merge, t_dec = oracle_step_seconds(w, res, workers)
    ms = per_step * 1e3
    value = step_tokens(w) / per_step
    sample = (f"{len(paths)} selection units ({args.warmup} warm-up; at least one per step "
              f"and one per core), in {workers} single-threaded processes: merge rounds mean {t_merge:.2f} s, decode "
              f"step mean {t_dec * 1e3:.1f} ms; scaled to {units_per_step(w)} units and "
              f"{w.n_decode} decode steps over {workers} cores; {wall:.1f} s wall")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": workers, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


L2_BYTES = 126 * 1024 * 1024


def config_of(w, n_gpus):
    seq = inputs.sequence_lengths(w)
    kv = 2 * w.layers * int(seq.sum()) * w.H_kv * w.d * w.elem_bytes
    dec = 2 * w.H_kv * int((seq // w.ratio).sum()) * w.d * w.elem_bytes
    l2 = (f"inputs larger than L2 ({kv / 2**30:.2f} GiB of K/V per replica; no flush needed)"
          if kv > L2_BYTES else f"inputs of {kv / 2**20:.1f} MiB fit in L2")
    if dec <= L2_BYTES and w.layers * dec > L2_BYTES:
        l2 += ("; decode rotates over the layers' merged caches "
               f"({w.layers} x {dec / 2**20:.1f} MiB), larger than L2 together")
    elif dec <= L2_BYTES:
        l2 += (f"; the merged decode cache ({dec / 2**20:.1f} MiB) fits in L2, so decode "
               "steps may hit it")
    cfg = {"workload": w.name, "B": w.B, "layers": w.layers, "T": w.T, "H_kv": w.H_kv,
           "H_q": w.H_q, "d": w.d, "ratio": w.ratio, "scope": w.scope,
           "budget_per_head" if w.scope == "head" else "budget_per_sequence":
               w.T // w.ratio if w.scope == "head" else (w.T // w.ratio) * w.H_kv,
           "decode_steps_per_layer": w.n_decode, "window": w.W, "sink": w.sink,
           "parallelism": f"replicas x{n_gpus}" if n_gpus > 1 else "single GPU", "l2": l2}
    if w.len_range:
        cfg["T"] = f"per sequence U{{{w.len_range[0]}..{w.len_range[1]}}} (max {int(seq.max())})"
        cfg["total_prefill_tokens"] = int(seq.sum())
        cfg["budget_per_head"] = "floor(len / ratio) of its sequence"
    if w.remerge_every:
        cfg["remerge"] = (f"every {w.remerge_every} decode steps the newest {w.remerge_every} "
                          f"rows of every head are merged in place to "
                          f"{w.remerge_every // w.remerge_ratio} (window = the last {w.W} "
                          f"decode queries)")
    return cfg


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


def stream_ceiling_main(args, rank, world, local):
    """The read ceiling of one decode launch of the workload (kvs_stream_read): the bytes
    one launch reads (every cached K and V row of every head, plus the appended row), as
    rows of d bf16, streamed with the decode kernel's TMA loads on 80 to 148 CTAs and no
    arithmetic. Eight such buffers are rotated, so that no launch finds its rows in L2.
    One line per CTA count: the time a decode launch would take with free arithmetic."""
    from asymmetric_kv_merging_b200 import kvs
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = inputs.workload(args.workload)
    target = w.T // w.ratio
    rows_per_launch = int(w.B * w.H_kv * (target + (w.n_decode + 1) / 2.0) * 2)   # K and V rows
    bytes_per_launch = rows_per_launch * w.d * 2
    bufs = [torch.zeros(rows_per_launch, w.d, dtype=torch.bfloat16, device=dev) for _ in range(8)]
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    peak, peak_kind = peaks()
    stream = torch.cuda.Stream(dev)
    out = []
    for ctas in (80, 128, 144, 148):
        with torch.cuda.stream(stream):
            for i in range(8 * max(1, args.warmup)):
                kvs.stream_read(bufs[i % 8], w.d, ctas, ws)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            n = 64 * max(1, args.steps)
            e0.record(stream)
            for i in range(n):
                kvs.stream_read(bufs[i % 8], w.d, ctas, ws)
            e1.record(stream)
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / n
        ach = bytes_per_launch / (us / 1e6) / 1e9
        out.append({"ctas": ctas, "us_per_launch": us, "achieved": ach, "frac": ach / peak})
    if rank == 0:
        print(json.dumps({
            "metric": "decode read ceiling: one decode launch's bytes through the decode's TMA "
                      "loads with no arithmetic", "unit": "GB/s", "peak": peak,
            "peak_kind": peak_kind, "bytes_per_launch": bytes_per_launch,
            "config": {"workload": w.name, "rows_per_launch": rows_per_launch,
                       "buffers": "8 rotated, each larger than L2"},
            "device_flags": kvs.device_flags(ws), "by_ctas": out}), flush=True)


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
    if args.prefill or args.stream_ceiling:
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA device (the kernels have no CPU path)")
        (prefill_main if args.prefill else stream_ceiling_main)(args, rank, world, local)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the kernels have no CPU path)")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = inputs.workload(args.workload)
    if args.fp32:
        w = inputs.small_workload(w, dtype="f32", name=w.name + "_fp32")
    w = reduced(w, args)
    from asymmetric_kv_merging_b200 import kvs
    form_code = {"full": None, "diagonal": kvs.FORM_DIAGONAL,
                 "per_query": kvs.FORM_FULL | kvs.FORM_PER_QUERY}[args.form]
    rn = Runner(w, rank, dev, form=form_code)
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
    flags = rn.kvs.device_flags(rn.ws)

    # per-call device time of one eager step (CUDA events around every library call)
    parts = rn.breakdown()
    parts = {k: max_over_ranks(v, world) for k, v in sorted(parts.items())}
    if not rn.remerge:
        parts["decode"] = decode_ms          # the graph-replayed phase, exactly
    peak, peak_kind = peaks()
    algo = {"decode": rn.decode_bytes(), "score": rn.score_bytes(), "merge": rn.merge_bytes()}
    if rn.remerge:
        algo["remerge"] = rn.remerge_bytes()
    if w.dtype == "bf16":
        names = {
            "decode": "decode_tc_kernel (GQA decode; thread-block clusters per KV head when "
                      "they fit the GPU, else the split grid)",
            "score": "kvs_score_pairs: window_fa_kernel (S = Q K^T, O += P V), fa_query_kernel, "
                     "fa_center_kernel, window_score_kernel (window mass and pair scores)",
        }
    else:
        names = {
            "decode": "decode_kernel (fp32 GQA decode on CUDA cores, split grid)",
            "score": "kvs_score_pairs: window_partial_kernel, window_combine_kernel, "
                     "alpha_bar_kernel, pair_score_kernel (fp32, CUDA cores)",
        }
    names.update({
        "merge": "kvs_merge_compact: select_kernel + merge_kernel (out-of-place compaction)",
        "remerge": "in-place re-merge rounds: kvs_score_pairs + kvs_merge_compact "
                   "(merge_inplace_kernel)",
    })
    rooflines = {}
    for k, b in algo.items():
        ms = parts.get(k)
        if not ms:
            continue
        ach = b / (ms / 1e3) / 1e9
        rooflines[k] = {"kernel": names[k], "bound": "hbm", "achieved": ach, "peak": peak,
                        "peak_kind": peak_kind, "unit": "GB/s", "frac": ach / peak,
                        "algorithmic_bytes_per_step": b, "ms_per_step": ms,
                        "timing": ("graph replay, CUDA events" if k == "decode" and not rn.remerge
                                   else "eager pass, CUDA events around each call")}
    n_dec_launch = rn.decode_launches()
    dec_launch_ms = parts["decode"] / n_dec_launch
    traffic = None
    prof = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if os.path.exists(prof) and w.index == 2:
        # one ncu capture's DRAM bytes per launch, scaled by rows processed to this launch
        # (the capture shows traffic equal to the algorithmic bytes, so it scales in proportion)
        with open(prof) as f:
            tr = json.load(f)
        if tr.get("valid", True):          # false once the kernel changed after the capture
            traffic = (tr["measured_dram_bytes_per_launch"] * rn.decode_bytes_per_launch()
                       / tr["measured_algorithmic_bytes_per_launch"])
    dominant = max(rooflines, key=lambda k: rooflines[k]["ms_per_step"])
    roof = dict(rooflines[dominant])
    if dominant == "decode":
        roof.update(traffic=traffic, bytes_per_launch=rn.decode_bytes_per_launch(),
                    launch_ms=dec_launch_ms)
    else:
        roof["traffic"] = None
    merge_phase_bytes = algo["score"] + algo["merge"]

    e2e = None
    if not args.no_e2e:
        e2e_ms, h2d, d2h = run_e2e(rn, max(3, args.steps), 1)
        e2e_ms = max_over_ranks(e2e_ms, world)
        e2e = {"value": tokens / (e2e_ms / 1e3), "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, rn.layers, rn.tokens_per_step())

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": dict(config_of(w, world), form=args.form),
            "value_note": ("merged KV tokens per second of the whole step: the merge phase "
                           "(every layer to its budget) plus the decode phase"),
            "merge_ms_per_step": merge_ms, "decode_ms_per_step": decode_ms,
            "merge_tokens_per_s": tokens / (merge_ms / 1e3),
            "decode_us_per_token": decode_ms * 1e3 / w.n_decode,
            "decode_us_per_token_note": ("one generated token = one decode step over all layers"
                                         + (", re-merges included" if rn.remerge else "")),
            "merge_phase": {"algorithmic_bytes": merge_phase_bytes,
                            "achieved": merge_phase_bytes / (merge_ms / 1e3) / 1e9,
                            "frac": merge_phase_bytes / (merge_ms / 1e3) / 1e9 / peak,
                            "unit": "GB/s", "timing": "graph replay, CUDA events"},
            "clocks": clk,
            "e2e": e2e,
            "gpu_launches": (rn.launches_merge + rn.launches_decode) * args.steps,
            "device_flags": flags,
            "roofline": roof,
            "rooflines": rooflines,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        del rn
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
