#!/usr/bin/env python
"""Benchmark of the GlowQ corrected quantised linear layer on B200.

A step is one pass of the whole hot path over one batch of synthetic tokens:
the LLaMA-2-7B attention linears at decode T=1 -- the Q/K/V input-sharing
group (R = X B^T once, y_i = X w_hat_i^T + R A_i^T for Q, K, V) followed by the
solo o_proj (its own R inline), INT4 g128 weights, rank 64.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl glowq|reference]

Prints one JSON line (rank 0).  `value` is whole-job tokens/s from CUDA events
around exactly K steps (all ranks, max over ranks); weights are rotated over
enough replicas that every step streams its weights from HBM (inputs larger
than L2).  `e2e` is the same metric through the public API with the token
activations copied from pinned host memory and the outputs copied back each
step (enqueued eagerly; one CUDA graph replay per step beside it).  `--impl reference` times the CPU oracle (float64 C) on a bounded sample
of the same workload.  Multi-GPU runs are independent replicas (the layer has
no cross-GPU exchange): weak scaling, no data-path collective.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GlowQ linear tok/s (decode T=1, prefill T=2048); % of HBM / tensor roofline"
WORKLOAD = "llama2_7b_attn_decode"
DECODE_WORKLOAD = ("LLaMA-2-7B attention linears, decode T=1: Q/K/V group (3x4096x4096) + "
                   "o_proj solo (4096x4096), INT4 g128 asym, r=64 fp16 factors")
R_RANK = 64
D = 4096
QKV_OUTS = [4096, 4096, 4096]
O_OUTS = [4096]


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", 0)) or None, "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def group_bytes(outs, d, r, T, with_factors=True):
    """Algorithmic HBM bytes of one group call: INT4 codes + fp16 scales + u8 zeros,
    A_i (fp16) and B (fp16, once per group), X and R in, Y out."""
    O = sum(outs)
    b = O * d // 2 + O * (d // 128) * 3 + T * d * 2 + T * O * 2
    if with_factors and r:
        b += O * r * 2 + r * d * 2 + 2 * T * r * 2
    return b


def group_flops(outs, d, r, T):
    O = sum(outs)
    return 2 * T * O * d + (2 * T * r * d + 2 * T * O * r if r else 0)


# --------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v.lower() == "active"})
        loaded = [r[0] for r in rows if r[2] > 200.0] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(r[2] for r in rows)}


# ------------------------------------------------------------ replica ranks

class Ranks:
    """Cross-rank plumbing of a replica run (one process per GPU, no data-path
    collective): a barrier before every timed region, the max over ranks of
    every timed figure, and the whole-job rate from the max."""

    def __init__(self, dist=None, device=None):
        self.dist = dist
        self.device = device

    @property
    def world(self) -> int:
        return self.dist.get_world_size() if self.dist is not None else 1

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, *vals):
        """Max over ranks of each value (every rank calls this in the same order)."""
        if self.dist is None:
            out = [float(v) for v in vals]
        else:
            import torch
            t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=self.device)
            self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
            out = [float(x) for x in t.tolist()]
        return out if len(out) > 1 else out[0]

    def rate(self, units_per_rank: float, max_ms: float) -> float:
        """Whole-job units per second: every rank's units over the slowest rank's time."""
        return self.world * units_per_rank / (max_ms * 1e-3)


# ------------------------------------------------------------------ workload

def build_replicas(n_rep, T, device, seed=0):
    import torch
    from rank_error_correction_b200 import glowq, synth
    reps = []
    for i in range(n_rep):
        rep = {}
        for name, outs, sub in (("qkv", QKV_OUTS, 0), ("o_proj", O_OUTS, 10)):
            mods = []
            for j, O in enumerate(outs):
                W = synth.device_weights(O, D, seed, sub=1000 * i + sub + j, device=device)
                q, s, z = glowq.pack_int4(W)
                del W
                mods.append(glowq.QModule(q, s, z))
            As, B = synth.device_factors(outs, D, R_RANK, seed, sub=1000 * i + sub, device=device)
            for m, A in zip(mods, As):
                m.A = A
            rep[name] = (mods, B)
        reps.append(rep)
    torch.cuda.synchronize()
    return reps


def make_io(T, device, seed=0):
    import torch
    from rank_error_correction_b200 import glowq, synth
    X = torch.from_numpy(synth.activations(T, D, synth.ALPHA_QKV, seed=seed)).to(device)
    X2 = torch.from_numpy(synth.activations(T, D, synth.ALPHA_QKV, seed=seed, sub=1)).to(device)
    Yqkv = torch.empty((T, sum(QKV_OUTS)), dtype=torch.float16, device=device)
    Yo = torch.empty((T, O_OUTS[0]), dtype=torch.float16, device=device)
    R = torch.empty((T, R_RANK), dtype=torch.float16, device=device)
    ws = glowq.alloc_workspace(T, R_RANK, device)
    views, c = [], 0
    for O in QKV_OUTS:
        views.append(Yqkv[:, c:c + O])
        c += O
    return dict(X=X, X2=X2, Yqkv=Yqkv, views=views, Yo=Yo, R=R, ws=ws)


def run_step(rep, io, stream=None):
    from rank_error_correction_b200 import glowq
    mods, B = rep["qkv"]
    glowq.group_forward(mods, B, io["X"], Ys=io["views"], R_out=io["R"], workspace=io["ws"], stream=stream)
    mo, Bo = rep["o_proj"]
    glowq.solo_forward(mo[0], Bo, io["X2"], Y=io["Yo"], workspace=io["ws"], stream=stream)


def time_decode(T, steps, warmup, device, n_rep, gpu_index, want_clocks=True, ranks=None):
    """Time exactly `steps` decode steps replayed from one CUDA graph (value),
    then replay an instrumented copy with event nodes around each call to get
    the per-call durations used for the roofline (event nodes break the
    programmatic-dependent-launch overlap between calls, so they are kept out
    of the timed graph)."""
    import torch
    from rank_error_correction_b200 import glowq
    reps = build_replicas(n_rep, T, device)
    io = make_io(T, device)
    stream = torch.cuda.Stream(device=device)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(max(warmup, 3)):
            run_step(reps[i % n_rep], io)
    stream.synchronize()
    # timed graph: all steps back to back
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            run_step(reps[i % n_rep], io)
    with torch.cuda.stream(stream):
        g.replay()                     # warm replay on the same stream as the timed one
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(gpu_index) if want_clocks else None
    if sampler:
        sampler.__enter__()
    torch.cuda.synchronize()
    if ranks is not None:
        ranks.barrier()
    with torch.cuda.stream(stream):
        t0.record()
        g.replay()
        t1.record()
    stream.synchronize()
    if sampler:
        sampler.__exit__()
    total_ms = t0.elapsed_time(t1)
    del g
    # instrumented graph: event-record nodes around each call
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(steps)]
    gi = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gi, stream=stream):
        for i in range(steps):
            rep = reps[i % n_rep]
            mods, B = rep["qkv"]
            evs[i][0].record()
            glowq.group_forward(mods, B, io["X"], Ys=io["views"], R_out=io["R"], workspace=io["ws"])
            evs[i][1].record()
            mo, Bo = rep["o_proj"]
            glowq.solo_forward(mo[0], Bo, io["X2"], Y=io["Yo"], workspace=io["ws"])
            evs[i][2].record()
    with torch.cuda.stream(stream):
        gi.replay()                    # warm replay
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        gi.replay()                    # the replay whose event nodes are read
    torch.cuda.synchronize()
    qkv_ms = [evs[i][0].elapsed_time(evs[i][1]) for i in range(steps)]
    o_ms = [evs[i][1].elapsed_time(evs[i][2]) for i in range(steps)]
    del gi
    # steady-state duration of one Q/K/V group call: a graph of `steps` such
    # calls back to back (rotating weight replicas, PDL overlap kept), averaged
    gq = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gq, stream=stream):
        for i in range(steps):
            mods, B = reps[i % n_rep]["qkv"]
            glowq.group_forward(mods, B, io["X"], Ys=io["views"], R_out=io["R"], workspace=io["ws"])
    with torch.cuda.stream(stream):
        gq.replay()
    torch.cuda.synchronize()
    c0 = torch.cuda.Event(enable_timing=True)
    c1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        c0.record()
        gq.replay()
        c1.record()
    torch.cuda.synchronize()
    qkv_chain_ms = c0.elapsed_time(c1) / steps
    del gq
    return dict(total_ms=total_ms, qkv_ms=statistics.mean(qkv_ms), o_ms=statistics.mean(o_ms),
                qkv_ms_median=statistics.median(qkv_ms), qkv_chain_ms=qkv_chain_ms,
                clocks=sampler.summary() if sampler else None, reps=reps, io=io)


def time_e2e(T, steps, device, reps, io, ranks=None, graph=True):
    """Public-API steps with host<->device copies of the step's activations and
    outputs: one pinned H2D copy of both calls' inputs, the two calls as
    prepared plans (glowq.ForwardPlan: arguments marshalled once per replica),
    one D2H copy of both calls' outputs (Q/K/V and o_proj write column blocks
    of one T x 16384 buffer through ldY).  graph=True: each step is one replay
    of a CUDA graph captured from exactly those four operations (one graph per
    weight replica), the way a decode loop is driven; graph=False: the four
    operations are enqueued eagerly from Python every step."""
    import torch
    from rank_error_correction_b200 import glowq
    Xall = torch.empty((2, T, D), dtype=torch.float16, device=device)
    Xall[0].copy_(io["X"])
    Xall[1].copy_(io["X2"])
    ncol = sum(QKV_OUTS) + sum(O_OUTS)
    Yall = torch.empty((T, ncol), dtype=torch.float16, device=device)
    views, c = [], 0
    for O in QKV_OUTS:
        views.append(Yall[:, c:c + O])
        c += O
    Yo = Yall[:, c:c + O_OUTS[0]]
    stream = torch.cuda.Stream(device=device)
    plans = []
    for rep in reps:
        mods, B = rep["qkv"]
        mo, Bo = rep["o_proj"]
        plans.append((glowq.ForwardPlan(mods, B, Xall[0], views, R_out=io["R"], workspace=io["ws"], stream=stream),
                      glowq.ForwardPlan([mo[0]], Bo, Xall[1], [Yo], workspace=io["ws"], solo=True, stream=stream)))
    Xh = Xall.cpu().pin_memory()
    Yh = torch.empty((T, ncol), dtype=torch.float16).pin_memory()
    n = min(steps, 200)

    def one(i):
        Xall.copy_(Xh, non_blocking=True)
        pq, po = plans[i % len(plans)]
        pq()
        po()
        Yh.copy_(Yall, non_blocking=True)

    with torch.cuda.stream(stream):
        for i in range(3):
            one(i)
    stream.synchronize()
    graphs = []
    if graph:
        for i in range(len(plans)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                one(i)
            graphs.append(g)
        with torch.cuda.stream(stream):
            for g in graphs:
                g.replay()
    torch.cuda.synchronize()
    if ranks is not None:
        ranks.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record()
        for i in range(n):
            if graph:
                graphs[i % len(graphs)].replay()
            else:
                one(i)
        t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / n
    del graphs
    h2d = Xh.numel() * 2
    d2h = Yh.numel() * 2
    return ms, h2d, d2h, n


# ------------------------------------------------------------------ prefill

MLP_D, MLP_FFN = 4096, 11008


def time_prefill(T, steps, warmup, device, n_rep=2, seed=0, eager_steps=None, ranks=None):
    """LLaMA-2-7B MLP linears at T tokens: gate/up group + down_proj solo (tcgen05 path).
    With `eager_steps`, run that many plain steps and return None (profiling)."""
    import torch
    from rank_error_correction_b200 import glowq, synth
    reps = []
    for i in range(n_rep):
        gu = []
        for j in range(2):
            W = synth.device_weights(MLP_FFN, MLP_D, seed, sub=5000 + 100 * i + j, device=device)
            q, s, z = glowq.pack_int4(W)
            del W
            gu.append(glowq.QModule(q, s, z))
        As, Bg = synth.device_factors([MLP_FFN] * 2, MLP_D, R_RANK, seed, sub=5000 + i, device=device)
        for m, A in zip(gu, As):
            m.A = A
        W = synth.device_weights(MLP_D, MLP_FFN, seed, sub=6000 + i, device=device)
        q, s, z = glowq.pack_int4(W)
        del W
        Ad, Bd = synth.device_factors([MLP_D], MLP_FFN, R_RANK, seed, sub=6000 + i, device=device)
        reps.append((gu, Bg, glowq.QModule(q, s, z, Ad[0]), Bd))
    torch.cuda.synchronize()
    X = torch.from_numpy(synth.activations(T, MLP_D, synth.ALPHA_MLP, seed=seed)).to(device)
    Xd = torch.from_numpy(synth.activations(T, MLP_FFN, synth.ALPHA_MLP, seed=seed, sub=1)).to(device)
    Ygu = torch.empty((T, 2 * MLP_FFN), dtype=torch.float16, device=device)
    views = [Ygu[:, :MLP_FFN], Ygu[:, MLP_FFN:]]
    Yd = torch.empty((T, MLP_D), dtype=torch.float16, device=device)
    R = torch.empty((T, R_RANK), dtype=torch.float16, device=device)
    ws = glowq.alloc_workspace(T, R_RANK, device)
    stream = torch.cuda.Stream(device=device)

    def step(i):
        gu, Bg, dn, Bd = reps[i % n_rep]
        glowq.group_forward(gu, Bg, X, Ys=views, R_out=R, workspace=ws)
        glowq.solo_forward(dn, Bd, Xd, Y=Yd, workspace=ws)

    if eager_steps is not None:
        for i in range(eager_steps):
            step(i)
        return None

    with torch.cuda.stream(stream):
        for i in range(max(warmup, 3)):
            step(i)
    stream.synchronize()
    # timed graph: all steps back to back, no event nodes inside (they would
    # break the programmatic-dependent-launch overlap between calls)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            step(i)
    with torch.cuda.stream(stream):
        g.replay()                     # warm replay on the same stream as the timed one
    torch.cuda.synchronize()
    if ranks is not None:
        ranks.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record()
        g.replay()
        t1.record()
    torch.cuda.synchronize()
    total_ms = t0.elapsed_time(t1)
    del g
    # per-call durations (roofline): a second graph with event nodes around each call
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(steps)]
    gi = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gi, stream=stream):
        for i in range(steps):
            gu, Bg, dn, Bd = reps[i % n_rep]
            evs[i][0].record()
            glowq.group_forward(gu, Bg, X, Ys=views, R_out=R, workspace=ws)
            evs[i][1].record()
            glowq.solo_forward(dn, Bd, Xd, Y=Yd, workspace=ws)
            evs[i][2].record()
    with torch.cuda.stream(stream):
        gi.replay()                    # warm replay
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        gi.replay()                    # the replay whose event nodes are read
    torch.cuda.synchronize()
    gu_ms = statistics.mean(evs[i][0].elapsed_time(evs[i][1]) for i in range(steps))
    dn_ms = statistics.mean(evs[i][1].elapsed_time(evs[i][2]) for i in range(steps))
    del gi
    return dict(total_ms=total_ms, gu_ms=gu_ms, dn_ms=dn_ms)


# ------------------------------------------------------------ oracle timing

_ORACLE_STEP = None


def oracle_step_inputs(T=1, seed=0):
    """Host inputs of one whole decode step for the CPU oracle: the Q/K/V group
    (3 x 4096 x 4096) and the o_proj solo (4096 x 4096), INT4 g128 packed by
    the oracle's own quantiser, r = 64 stand-in factors of the solve's
    magnitude, X of T tokens.  Built once per process."""
    global _ORACLE_STEP
    if _ORACLE_STEP is None:
        import numpy as np
        import oracle
        from rank_error_correction_b200 import synth
        X = synth.bits(synth.activations(T, D, synth.ALPHA_QKV, seed=seed))
        X2 = synth.bits(synth.activations(T, D, synth.ALPHA_QKV, seed=seed, sub=1))
        units = []
        for name, outs, sub in (("qkv", QKV_OUTS, 0), ("o_proj", O_OUTS, 10)):
            mods = []
            As, B = synth.random_factors(outs, D, R_RANK, seed=seed, sub=sub)
            for j, O in enumerate(outs):
                W = synth.weights(O, D, seed=seed, stream_sub=sub + j)
                q, s, z = oracle.quantize_int4(W)
                del W
                mods.append((q, s, z, synth.bits(As[j])))
            units.append((name, mods, synth.bits(B)))
        _ORACLE_STEP = (X, X2, units)
    return _ORACLE_STEP


def oracle_step(threads):
    """One whole decode step through the oracle (float64 C): the Q/K/V group
    with one shared R, then the o_proj solo with its own R.  Returns seconds."""
    import oracle
    X, X2, units = oracle_step_inputs()
    oracle.set_threads(threads)
    t0 = time.perf_counter()
    (_, mods, B), (_, omods, Bo) = units
    oracle.group_forward(mods, B, X)
    q, s, z, A = omods[0]
    oracle.solo_forward(q, s, z, A, Bo, X2)
    return time.perf_counter() - t0


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline_figures(budget_s=12.0):
    """The oracle as it stands on this host's cores: whole decode steps with
    every core (OpenMP over output rows), and with one thread."""
    ncores = host_cores()
    oracle_step(ncores)                     # warm: pages, thread pool
    t_all, t_start = [], time.perf_counter()
    while time.perf_counter() - t_start < budget_s * 0.5 and len(t_all) < 50:
        t_all.append(oracle_step(ncores))
    t_one, t_start = [], time.perf_counter()
    while time.perf_counter() - t_start < budget_s * 0.5 and len(t_one) < 5:
        t_one.append(oracle_step(1))
    import oracle
    oracle.set_threads(ncores)
    all_s, one_s = statistics.median(t_all), statistics.median(t_one)
    return {"value": 1.0 / all_s, "unit": "tok/s", "cores": ncores, "kind": "oracle",
            "nproc": os.cpu_count(), "threads": ncores,
            "single_thread_value": 1.0 / one_s, "ms_per_step_all_cores": all_s * 1e3,
            "ms_per_step_single_thread": one_s * 1e3,
            "sample": f"the whole decode step (T=1: Q/K/V group 3x4096x4096 with one shared R + o_proj solo "
                      f"4096x4096, r=64), float64 C oracle; {len(t_all)} steps on {ncores} threads "
                      f"(median), {len(t_one)} steps on 1 thread (median)"}


def decode_config(replicas, world):
    """The config dict of the decode line (shared by both arms)."""
    return {"workload": DECODE_WORKLOAD, "tokens": 1, "replicas": replicas,
            "l2": f"inputs larger than L2: {replicas} weight replicas rotated ({replicas * 38.4:.0f} MB)",
            "graph": "one CUDA graph of all timed steps (per-call roofline times from a second, "
                     "event-instrumented replay)",
            "parallelism": "replicas" if world > 1 else "single GPU"}


def run_reference(args, rank, world):
    """The oracle as the reference arm: every step is the whole decode step
    (nothing sampled or extrapolated), timed on the host's cores."""
    if rank != 0:
        return 0
    T = 1
    ncores = host_cores()
    for _ in range(args.warmup):
        oracle_step(ncores)
    times = [oracle_step(ncores) for _ in range(args.steps)]
    total_s = sum(times)
    value = T * args.steps / total_s
    line = {"metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_s / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": decode_config(args.replicas, world),
            "cpu_baseline": {"value": value, "unit": "tok/s", "cores": ncores, "kind": "oracle",
                             "nproc": os.cpu_count(),
                             "sample": f"every step is the whole decode step (Q/K/V group + o_proj, T=1), "
                                       f"{args.steps} timed steps after {args.warmup} warm-up steps, "
                                       f"float64 C oracle, OpenMP over output rows on {ncores} threads"},
            "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------- 40-layer LLaMA-2-13B linear stack

S13_D, S13_FFN, S13_LAYERS = 5120, 13824, 40
# (unit, output features of its modules, input dimension, activation alpha)
S13_UNITS = [("qkv", [5120, 5120, 5120], 5120, "qkv"), ("o_proj", [5120], 5120, "qkv"),
             ("gate_up", [13824, 13824], 5120, "mlp"), ("down_proj", [5120], 13824, "mlp")]
# The pages' Table 3 (LLaMA-2-7B time to first batch on their RTX 4090), context only.
PAGES_TABLE3_TTFB_MS = {"layerwise": 88.45, "glowq": 82.66, "glowq_s": 66.68}


def build_stack13b(device, layers=S13_LAYERS, seed=0):
    """Random-init INT4 g128 weights of a LLaMA-2-13B linear stack, r = 64 factors:
    a shared B per unit (GlowQ) and an own B_i per module (layerwise), device
    error norms and the GlowQ-S top-50% mask by g_ner."""
    import numpy as np
    import torch
    from rank_error_correction_b200 import glowq, synth
    units, e2, w2, layer_idx, kind = [], [], [], [], []
    for l in range(layers):
        for k, (name, outs, d, _) in enumerate(S13_UNITS):
            mods, e_u, w_u = [], 0.0, 0.0
            for i, O in enumerate(outs):
                W = synth.device_weights(O, d, seed, sub=100000 + 100 * l + 10 * k + i, device=device)
                q, s, z = glowq.pack_int4(W)
                en = glowq.error_norms(W, q, s, z).sum(dim=0)
                e_u, w_u = e_u + en[0], w_u + en[1]
                del W
                mods.append((q, s, z))
            As, B = synth.device_factors(outs, d, R_RANK, seed, sub=200000 + 10 * l + k, device=device)
            own = [synth.device_factors([O], d, R_RANK, seed, sub=300000 + 100 * l + 10 * k + i, device=device)
                   for i, O in enumerate(outs)]
            units.append(dict(name=name, d=d, outs=outs, packed=mods, As=As, B=B,
                              own=[(a[0], b) for a, b in own]))
            e2.append(e_u)
            w2.append(w_u)
            layer_idx.append(l)
            kind.append(k)
    torch.cuda.synchronize()
    e2 = np.array([float(x) for x in e2])
    w2 = np.array([float(x) for x in w2])
    mask, _, _ = glowq.select_restore(e2, w2, np.array(layer_idx, np.int32), np.array(kind, np.int32),
                                      len(units) // 2)
    for u, m in zip(units, mask):
        u["restore"] = bool(m)
    return units


def time_stack13b(units, T, steps, warmup, device, mode, seed=0, ranks=None):
    """One token batch through every linear of the stack, captured in one CUDA
    graph.  mode: 'layerwise' (every module its own R_i = X B_i^T), 'glowq'
    (R shared per group, all units corrected) or 'glowq_s' (only the restored
    units corrected).  Every unit reads a fixed synthetic input of its width
    (the stack's data flow between layers is not modelled; the inputs are the
    timing-only device draws of synth.device_activations).  Returns ms/batch."""
    import torch
    from rank_error_correction_b200 import glowq, synth
    # timing-only inputs (iid, unit power per coordinate): one per unit kind
    Xs = {n: synth.device_activations(T, d, seed, sub=500 + k, device=device)
          for k, (n, _, d, _) in enumerate(S13_UNITS)}
    Ys = {n: [torch.empty((T, O), dtype=torch.float16, device=device) for O in outs]
          for n, outs, _, _ in S13_UNITS}
    # one workspace for every unit: the largest any unit's call can use
    wsn = max(glowq.workspace_bytes_for(T, R_RANK, d, outs) for _, outs, d, _ in S13_UNITS)
    ws = torch.zeros(max(wsn, 16), dtype=torch.uint8, device=device)
    calls = []
    for u in units:
        a = u["name"]
        X = Xs[a]
        if mode == "layerwise":
            for (q, s, z), (A, B), Y in zip(u["packed"], u["own"], Ys[a]):
                calls.append(("solo", glowq.QModule(q, s, z, A), B, X, Y))
        else:
            on = mode == "glowq" or u["restore"]
            mods = [glowq.QModule(q, s, z, A if on else None) for (q, s, z), A in zip(u["packed"], u["As"])]
            B = u["B"] if on else None
            if len(mods) > 1:
                calls.append(("group", mods, B, X, Ys[a]))
            else:
                calls.append(("solo", mods[0], B, X, Ys[a][0]))
    R = torch.empty((T, R_RANK), dtype=torch.float16, device=device)

    def one():
        for kindc, m, B, X, Y in calls:
            if kindc == "group":
                glowq.group_forward(m, B, X, Ys=Y, R_out=R if B is not None else None, workspace=ws)
            else:
                glowq.solo_forward(m, B, X, Y=Y, workspace=ws)

    stream = torch.cuda.Stream(device=device)
    with torch.cuda.stream(stream):
        for _ in range(max(warmup, 1)):
            one()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(steps):
            one()
    with torch.cuda.stream(stream):
        g.replay()                     # warm replay on the same stream as the timed one
    torch.cuda.synchronize()
    if ranks is not None:
        ranks.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record()
        g.replay()
        t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    del g
    return ranks.max(ms) if ranks is not None else ms


def stack13b_line(device, warmup, ranks=None):
    units = build_stack13b(device)
    out = {"workload": "LLaMA-2-13B-shaped linear stack, 40 layers x (Q/K/V group 3x5120x5120, o_proj 5120x5120, "
                       "gate/up group 2x13824x5120, down_proj 5120x13824), INT4 g128 asym, r=64, random-init "
                       "weights, GlowQ-S restoring the top 50% of units by g_ner",
           "units": len(units), "restored_units": sum(u["restore"] for u in units),
           "context_pages_table3_ttfb_ms_llama2_7b": PAGES_TABLE3_TTFB_MS}
    for T, steps in ((1, 10), (2048, 2)):
        ms = {mode: time_stack13b(units, T, steps, warmup, device, mode, ranks=ranks)
              for mode in ("layerwise", "glowq", "glowq_s")}
        world = ranks.world if ranks is not None else 1
        out[f"T{T}"] = {"ms_per_batch": ms, "tok_s": {k: world * T / (v * 1e-3) for k, v in ms.items()},
                        "speedup_vs_layerwise": {k: ms["layerwise"] / v for k, v in ms.items()}}
    del units
    return out


# ------------------------------------------------ per-unit lines (configs)

# LLaMA-3.1-8B-shaped GQA layer: (unit, module output features, input dim)
L31_UNITS = [("qkv", [4096, 1024, 1024], 4096), ("o_proj", [4096], 4096),
             ("gate_up", [14336, 14336], 4096), ("down_proj", [4096], 14336)]
# LLaMA-2-13B-shaped layer units
S13_UNIT_SHAPES = [("qkv", [5120, 5120, 5120], 5120), ("o_proj", [5120], 5120),
                   ("gate_up", [13824, 13824], 5120), ("down_proj", [5120], 13824)]
L2_BYTES = 126 * 1024 * 1024


def build_unit(outs, d, seed, sub, device):
    """One unit (group or solo) of random-init INT4 g128 modules with r = 64 factors."""
    from rank_error_correction_b200 import glowq, synth
    mods = []
    for j, O in enumerate(outs):
        W = synth.device_weights(O, d, seed, sub=sub + j, device=device)
        q, s, z = glowq.pack_int4(W)
        del W
        mods.append(glowq.QModule(q, s, z))
    As, B = synth.device_factors(outs, d, R_RANK, seed, sub=sub, device=device)
    for m, A in zip(mods, As):
        m.A = A
    return mods, B


def time_unit_chain(reps, X, T, calls, device, ranks=None):
    """Average duration of one call of a unit in a CUDA graph of `calls`
    back-to-back calls over the weight replicas `reps` (CUDA events around the
    graph on the launching stream).  Returns microseconds per call."""
    import torch
    from rank_error_correction_b200 import glowq
    mods0, _ = reps[0]
    Ys = [torch.empty((T, m.out_features), dtype=torch.float16, device=device) for m in mods0]
    R = torch.empty((T, R_RANK), dtype=torch.float16, device=device)
    ws = glowq.alloc_workspace(T, R_RANK, device, mods0[0].in_features, [m.out_features for m in mods0])

    def call(i):
        mods, B = reps[i % len(reps)]
        if len(mods) > 1:
            glowq.group_forward(mods, B, X, Ys=Ys, R_out=R, workspace=ws)
        else:
            glowq.solo_forward(mods[0], B, X, Y=Ys[0], workspace=ws)

    stream = torch.cuda.Stream(device=device)
    with torch.cuda.stream(stream):
        for i in range(3):
            call(i)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(calls):
            call(i)
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    if ranks is not None:
        ranks.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record()
        g.replay()
        t1.record()
    torch.cuda.synchronize()
    us = t0.elapsed_time(t1) * 1e3 / calls
    del g
    st = glowq.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after a timed chain (T={T}, {len(mods0)} modules, "
                           f"d={mods0[0].in_features})")
    return ranks.max(us) if ranks is not None else us


def unit_lines(shapes, tokens, device, hbm_peak, tf_peak, seed=0, sub0=0, ranks=None):
    """Per-unit throughput of one layer's linears at each token count: decode
    counts (T <= 64) rotate enough weight replicas that every call streams its
    weights from HBM (more than 2x L2 per chain); T >= 512 rotate two."""
    import torch
    from rank_error_correction_b200 import synth
    out = {}
    for k, (name, outs, d) in enumerate(shapes):
        ubytes = group_bytes(outs, d, R_RANK, 1)
        n_dec = max(2, min(8, -(-2 * L2_BYTES // ubytes)))
        reps = [build_unit(outs, d, seed, sub0 + 1000 * i + 10 * k, device) for i in range(n_dec)]
        for T in tokens:
            X = synth.device_activations(T, d, seed, sub=700 + k, device=device)
            calls = 64 if T <= 64 else 6
            use = reps if T <= 64 else reps[:2]
            us = time_unit_chain(use, X, T, calls, device, ranks=ranks)
            b = group_bytes(outs, d, R_RANK, T)
            f = group_flops(outs, d, R_RANK, T)
            e = {"us_per_call": us, "GBps": b / (us * 1e-6) / 1e9, "hbm_frac": b / (us * 1e-6) / 1e9 / hbm_peak,
                 "TFLOPs": f / (us * 1e-6) / 1e12, "tensor_frac": f / (us * 1e-6) / 1e12 / tf_peak,
                 "algorithmic_bytes": b, "algorithmic_flops": f, "replicas": len(use)}
            out.setdefault(f"T{T}", {})[name] = e
            del X
        del reps
        torch.cuda.empty_cache()
    for key, units in out.items():
        T = int(key[1:])
        tot = sum(u["us_per_call"] for u in units.values())
        units["layer"] = {"us": tot, "tok_s": (ranks.world if ranks is not None else 1) * T / (tot * 1e-6)}
    return out


# ----------------------------------------------------- offline solve (GPU)

def solve_line(device, r=64, p=16, q=2, seed=0):
    """The offline whitened group solve on the GPU for one LLaMA-2-7B Q/K/V
    group (3 x 4096 x 4096, r = 64, p = 16, q = 2), float64.  Context: the
    pages' Table 11 times the randomised SVD of the covariance-aligned core
    per layer on an A100.  Synthetic inputs: random-init weights and a
    diagonal power-law Sx^{1/2} (alpha = 1.19) stored dense."""
    import torch
    from rank_error_correction_b200 import glowq, synth
    d, outs = D, QKV_OUTS
    Ws, packs = [], []
    for j, O in enumerate(outs):
        W = synth.device_weights(O, d, seed, sub=7000 + j, device=device)
        Ws.append(W)
        packs.append(glowq.pack_int4(W))
    lam = torch.from_numpy(synth.power_law_spectrum(d, synth.ALPHA_QKV)).to(device)
    Sh = torch.diag(lam.sqrt()).contiguous()
    Shp = torch.diag(1.0 / lam.sqrt()).contiguous()
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    Om = torch.randn((d, r + p), generator=g, device=device, dtype=torch.float64)
    glowq.group_solve(Ws, packs, Sh, Shp, r, p, q, Om)          # warm (module load, attributes)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    _, _, sing, gec, _, _ = glowq.group_solve(Ws, packs, Sh, Shp, r, p, q, Om)
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    st = glowq.device_status()
    M = sum(outs)
    l = r + p
    flops = 2 * M * d * d + 2 * (2 * q + 2) * M * d * l
    return {"workload": "whitened shared-B solve of one LLaMA-2-7B Q/K/V group (12288 x 4096 stacked error), "
                        "r=64, p=16, q=2, float64 on the GPU",
            "ms": ms, "fp64_GFLOP": flops / 1e9, "fp64_TFLOPs": flops / (ms * 1e-3) / 1e12,
            "g_ec": float(gec.cpu()[0]), "sigma_1": float(sing.cpu()[0]), "status": st,
            "context_pages_table11": "randomised SVD per layer 0.09 s, LLaMA-3.2-3B, A100 (thelatestinai.com "
                                     "GlowQ page, Table 11)"}


# ------------------------------------------------------------ profile cases

def profile_case(case, device, steps=4):
    """A few untimed steps of one bench workload (no JSON line): the command
    that the ncu summaries under profiles/ are captured from.  Launch order per
    step -- decode: corrected_gemv (Q/K/V group), corrected_gemv (o_proj);
    prefill: rproj_tc, rproj_sum, corrected_gemm
    (gate/up), rproj_tc, rproj_sum, corrected_gemm (down_proj); small
    (LLaMA-2-13B o_proj and down_proj solos at decode batch T = 64, k-split
    64-token tiles): rproj_tc, rproj_sum, corrected_gemm (o_proj), rproj_tc,
    rproj_sum, corrected_gemm (down_proj)."""
    import torch
    from rank_error_correction_b200 import glowq, synth
    if case == "decode":
        reps = build_replicas(8, 1, device)
        io = make_io(1, device)
        for i in range(steps):
            run_step(reps[i % len(reps)], io)
    elif case == "small":
        T = 64
        units = []
        for k, (outs, d) in enumerate((([5120], 5120), ([5120], 13824))):
            mods, B = build_unit(outs, d, 0, 10 * k, device)
            X = synth.device_activations(T, d, 0, sub=700 + k, device=device)
            ws = torch.zeros(max(glowq.workspace_bytes_for(T, R_RANK, d, outs), 16), dtype=torch.uint8,
                             device=device)
            Y = torch.empty((T, outs[0]), dtype=torch.float16, device=device)
            units.append((mods[0], B, X, Y, ws))
        for i in range(steps):
            for m, B, X, Y, ws in units:
                glowq.solo_forward(m, B, X, Y=Y, workspace=ws)
    else:
        time_prefill(2048, 1, 0, device, n_rep=1, eager_steps=steps)
    torch.cuda.synchronize()
    print(f"profile case {case}: {steps} steps done", flush=True)
    return 0


# --------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="glowq", choices=["glowq", "reference"])
    ap.add_argument("--replicas", type=int, default=8)
    ap.add_argument("--no-extra", action="store_true", help="skip the T=4/16 decode lines")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-prefill", action="store_true", help="skip the T=2048 prefill line")
    ap.add_argument("--no-stack", action="store_true", help="skip the 40-layer LLaMA-2-13B stack line")
    ap.add_argument("--no-solve", action="store_true", help="skip the GPU offline solve line")
    ap.add_argument("--no-units", action="store_true",
                    help="skip the per-unit lines (LLaMA-3.1-8B layer, LLaMA-2-13B decode batches)")
    ap.add_argument("--profile-case", choices=["decode", "prefill", "small"],
                    help="run a few untimed steps of one workload and exit (for ncu captures)")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    from rank_error_correction_b200 import build, glowq
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if rank == 0 or not os.path.exists(glowq.LIB_PATH):
        build.build()
    ranks = Ranks()
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
        ranks = Ranks(dist, device)
        ranks.barrier()
    glowq.lib()

    if args.profile_case:
        return profile_case(args.profile_case, device)

    hbm_peak, tf_peak, tf_sust, peak_src = _peaks()
    T = 1
    res = time_decode(T, args.steps, args.warmup, device, args.replicas, local, want_clocks=(rank == 0),
                      ranks=ranks)
    total_ms, qkv_ms, o_ms, qkv_chain_ms = ranks.max(res["total_ms"], res["qkv_ms"], res["o_ms"],
                                                     res["qkv_chain_ms"])
    ms_step = total_ms / args.steps
    value = ranks.rate(T * args.steps, total_ms)
    qkv_bytes = group_bytes(QKV_OUTS, D, R_RANK, T)
    achieved = qkv_bytes / (qkv_chain_ms * 1e-3) / 1e9
    launches_per_step = 1 + 1          # one corrected_gemv launch per call (R computed inside it)
    e2e_ms, h2d, d2h, _ = time_e2e(T, args.steps, device, res["reps"], res["io"], ranks=ranks, graph=False)
    e2e_ms = ranks.max(e2e_ms)
    e2e_graph_ms, _, _, _ = time_e2e(T, args.steps, device, res["reps"], res["io"], ranks=ranks, graph=True)
    e2e_graph_ms = ranks.max(e2e_graph_ms)

    extra = []
    if not args.no_extra:
        for Tx in (4, 16):
            r2 = time_decode(Tx, min(args.steps, 100), args.warmup, device, args.replicas, local, want_clocks=False,
                             ranks=ranks)
            tot2, q2, o2 = ranks.max(r2["total_ms"], r2["qkv_ms"], r2["o_ms"])
            b = group_bytes(QKV_OUTS, D, R_RANK, Tx)
            extra.append({"tokens": Tx, "tok_s": ranks.rate(Tx * min(args.steps, 100), tot2),
                          "ms_per_step": tot2 / min(args.steps, 100),
                          "qkv_group_us": q2 * 1e3, "o_proj_us": o2 * 1e3,
                          "qkv_group_GBps": b / (q2 * 1e-3) / 1e9,
                          "qkv_group_hbm_frac": b / (q2 * 1e-3) / 1e9 / hbm_peak})
            del r2

    prefill = None
    if not args.no_prefill:
        Tp, sp = 2048, min(args.steps, 20)
        pr = time_prefill(Tp, sp, args.warmup, device, ranks=ranks)
        pr["total_ms"], pr["gu_ms"], pr["dn_ms"] = ranks.max(pr["total_ms"], pr["gu_ms"], pr["dn_ms"])
        tf_gu = group_flops([MLP_FFN] * 2, MLP_D, R_RANK, Tp) / (pr["gu_ms"] * 1e-3) / 1e12
        tf_dn = group_flops([MLP_D], MLP_FFN, R_RANK, Tp) / (pr["dn_ms"] * 1e-3) / 1e12
        prefill = {"workload": "LLaMA-2-7B MLP linears, prefill T=2048: gate/up group (2x11008x4096) + "
                               "down_proj solo (4096x11008), INT4 g128, r=64",
                   "tokens": Tp, "steps": sp, "tok_s": ranks.rate(Tp * sp, pr["total_ms"]),
                   "ms_per_step": pr["total_ms"] / sp,
                   "gate_up_us": pr["gu_ms"] * 1e3, "down_us": pr["dn_ms"] * 1e3,
                   "roofline": {"bound": "tensor", "kernel": "glowq_group_forward (gate/up, T=2048)",
                                "achieved": tf_gu, "peak": tf_peak, "peak_source": peak_src, "unit": "TFLOP/s",
                                "frac": tf_gu / tf_peak, "down_proj_TFLOPs": tf_dn,
                                "algorithmic_flops": group_flops([MLP_FFN] * 2, MLP_D, R_RANK, Tp)}}

    stack = None
    if not args.no_stack:
        stack = stack13b_line(device, args.warmup, ranks=ranks)

    solve = None
    if not args.no_solve:
        solve = solve_line(device)
    l31 = s13b = None
    if not args.no_units:
        l31 = unit_lines(L31_UNITS, (1, 4096), device, hbm_peak, tf_peak, sub0=20000, ranks=ranks)
        l31["workload"] = ("LLaMA-3.1-8B-shaped GQA layer: Q/K/V group 4096/1024/1024 x 4096, o_proj 4096x4096, "
                           "gate/up group 2x14336x4096, down_proj 4096x14336; INT4 g128, r=64; per unit, "
                           "CUDA graph of back-to-back calls")
        s13b = unit_lines(S13_UNIT_SHAPES, (16, 32, 64), device, hbm_peak, tf_peak, sub0=40000, ranks=ranks)
        s13b["workload"] = ("LLaMA-2-13B-shaped layer units at decode batches 16/32/64 (T <= 16: weight-streaming "
                            "decode kernel; T > 16: tcgen05 kernel); INT4 g128, r=64; per unit")

    cpu = None
    if rank == 0 and not args.no_cpu:
        cpu = cpu_baseline_figures()

    if rank == 0:
        # DRAM bytes per launch from the committed ncu captures (profiles/)
        traffic = traffic_pf = None
        tr_path = os.path.join(ROOT, "profiles", "traffic.json")
        if os.path.exists(tr_path):
            try:
                tr = json.load(open(tr_path))
                # an entry whose kernel changed after its capture reports null
                dec = tr.get("decode qkv T=1 group call", {})
                pf = tr.get("prefill gate_up T=2048 corrected_gemm", {})
                traffic = None if dec.get("stale") else dec.get("bytes")
                traffic_pf = None if pf.get("stale") else pf.get("bytes")
            except Exception:
                traffic = traffic_pf = None
        if prefill is not None:
            prefill["roofline"]["traffic"] = traffic_pf
        line = {
            "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp16 x int4 -> fp32 acc", "data": "synthetic",
            "config": decode_config(args.replicas, world),
            "roofline": {"bound": "hbm", "kernel": "glowq_group_forward (Q/K/V, T=1): corrected_gemv with the anchor projection inside",
                         "achieved": achieved, "peak": hbm_peak, "peak_source": peak_src, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "traffic": traffic, "algorithmic_bytes": qkv_bytes,
                         "us_per_launch": qkv_chain_ms * 1e3,
                         "timing": "average call in a graph of back-to-back Q/K/V calls (CUDA events around the "
                                   "graph on the launching stream)",
                         "us_per_launch_isolated": qkv_ms * 1e3},
            "o_proj_us": o_ms * 1e3,
            "e2e": {"value": ranks.rate(T, e2e_ms), "unit": "tok/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "driven_by": "pinned H2D copy, the two ForwardPlan calls and a D2H copy to pinned host "
                                 "memory, enqueued from Python every step",
                    "graph": {"value": ranks.rate(T, e2e_graph_ms), "ms_per_step": e2e_graph_ms,
                              "driven_by": "the same four operations replayed as one CUDA graph per step"}},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": res["clocks"],
            "cpu_baseline": cpu,
            "extra": extra,
            "prefill": prefill,
            "stack13b": stack,
            "llama31_8b_layer": l31,
            "offline_solve": solve,
            "llama2_13b_units_decode_batches": s13b,
        }
        print(json.dumps(line), flush=True)
    if ranks.dist is not None:
        ranks.barrier()
        ranks.dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
