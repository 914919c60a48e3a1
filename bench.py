#!/usr/bin/env python
"""Throughput of the STAPLE embedding-augmented SwiGLU FFN layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Default workload: one OLMo-2-1B-shaped layer decoding a batch of 64 tokens
(d_model 2048, d_ff 8192, vocab 100352, bf16, the whole table E in HBM).  A
step is one forward pass of the layer over one batch: the gate/up GEMM with
the E-row add and SiLU gating fused in, then the down GEMM.  Four weight sets
(403 MB, more than the 126 MB L2) and 64 token batches rotate from step to
step, so no step finds its weights in L2.  The training layer (16384 tokens,
host table with a 5% HBM cache, forward + full backward incl. the unique-row
table gradient) is timed as well and reported under "train_layer", next to
the same build's dense run (E path disabled).

Multi-GPU (torchrun): every rank runs its own replica on its own batches (no
collective on the data path); the time is the max over ranks.

--impl reference times the CPU oracle (the plain fp64 definition) on a bounded
sample of the same workload: each step is one token's forward restricted to a
256-feature slice of d_ff, i.e. 1/32 of a token; tokens/s is scaled to match.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthetic as syn  # noqa: E402

METRIC = "STAPLE FFN layer tokens/s (fwd+bwd and decode) at 1 B200; % of roofline"
DEFAULT_WORKLOAD = "olmo2-1b-decode-layer"
REF_SLICE = 256


# --------------------------------------------------------------------------
# Plumbing: ranks, peaks, clocks
# --------------------------------------------------------------------------

def dist_init(backend: str | None = None):
    """Ranks from the torchrun environment.  For more than one rank the
    process group uses NCCL (one GPU per rank) unless `backend` says
    otherwise (gloo runs the same plumbing on CPU)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        backend = backend or "nccl"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """The largest of the ranks' values (each rank's device time): the job
    takes as long as its slowest rank."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(units_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time (weak scaling: every rank runs its own replica)."""
    return world * units_per_rank / (ms_max / 1000.0)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons while it runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((int(parts[1]), int(parts[2]), float(parts[3]), parts[4:]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        # samples taken while the timed region ran: the ones drawing power
        load = [r for r in rows if r[2] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in load for n, v in zip(names, r[3][1:]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(load), "reasons": reasons}


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch,
# from the ncu capture summarised in the named profile.  It describes the
# kernel as captured, so it is reported only while the kernel's sources hash
# to the captured value; otherwise the roofline's traffic is null.
CAPTURED_TRAFFIC = {
    "k5k6_decode_fused": {
        "bytes": 103_393_280,   # mean of two launches: 104,610,304 and 102,176,256
        # (file, first marker, end marker): the decode launcher's part of ffn_tc.cu sets the grid
        "sources": [("token_indexed_sparse_staple_b200/csrc/decode_fused.cuh", None, None),
                    ("token_indexed_sparse_staple_b200/csrc/common.cuh", None, None),
                    ("token_indexed_sparse_staple_b200/csrc/ffn_tc.cu",
                     "// ---------------------------------------------------------------- decode",
                     "staple_status tc_ffn_fwd(")],
        "sha256": "cf520aacfa4d1fd5cff8432d22cd0ce2dd8c032b819af63ac5fdecb827823a73",
        "profile": "profiles/decode_fused_olmo2_1b_T64.md",
    },
}


def captured_traffic(kernel):
    c = CAPTURED_TRAFFIC.get(kernel)
    if c is None:
        return None, "no capture"
    h = hashlib.sha256()
    for f, first, end in c["sources"]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            text = fh.read()
        if first is not None:
            i = text.find(first.encode())
            j = text.find(end.encode(), i)
            if i < 0 or j < 0:
                return None, "decode launcher not found for the capture in " + c["profile"]
            text = text[i:j]
        h.update(text)
    if h.hexdigest() != c["sha256"]:
        return None, "kernel changed since the capture in " + c["profile"]
    return c["bytes"], c["profile"]


def bf16_randn(shape, std, seed):
    """Seeded N(0, std) draws made on the GPU, rounded to bf16 (used for the
    big tensors; the parity tests use the numpy generator of `synthetic`)."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device="cuda", dtype=torch.float32) * std).to(torch.bfloat16)


def kernel_table(trace, steps_seen):
    out = {}
    for name, ms in trace:
        if ms < 0:
            continue
        d = out.setdefault(name, {"launches": 0, "total_ms": 0.0})
        d["launches"] += 1
        d["total_ms"] += ms
    tot = sum(d["total_ms"] for d in out.values()) or 1.0
    for d in out.values():
        d["avg_us"] = round(1000.0 * d["total_ms"] / d["launches"], 3)
        d["share"] = round(d["total_ms"] / tot, 4)
        d["total_ms"] = round(d["total_ms"], 4)
    return out


# --------------------------------------------------------------------------
# Decode layer (device table)
# --------------------------------------------------------------------------

def decode_setup(stp, w, local):
    import torch
    R, S = 4, 64
    T, D, F, V = w.T, w.D, w.F, w.V
    st = {"R": R, "S": S}
    st["wg"] = [bf16_randn((F, D), w.w_std, syn.SEED_W + 3 * r) for r in range(R)]
    st["wu"] = [bf16_randn((F, D), w.w_std, syn.SEED_W + 3 * r + 1) for r in range(R)]
    st["wd"] = [bf16_randn((D, F), w.w_std, syn.SEED_W + 3 * r + 2) for r in range(R)]
    st["table"] = bf16_randn((V, F), w.e_std, syn.SEED_E)
    ids = np.stack([syn.zipf_ids(T, V, w.zipf_s, seed=syn.SEED_IDS + w.index + 7919 * s)
                    for s in range(S)])
    st["ids_host"] = torch.from_numpy(ids).pin_memory()
    st["ids"] = st["ids_host"].cuda()
    st["x"] = bf16_randn((S, T, D), w.x_std, syn.SEED_ACT)
    st["x_host"] = st["x"].cpu().pin_memory()
    st["z"] = torch.empty((T, F), dtype=torch.bfloat16, device="cuda")
    st["y"] = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")
    st["y_host"] = torch.empty((S, T, D), dtype=torch.bfloat16).pin_memory()
    st["emb"] = [stp.make_embed(stp.STAPLE_EMBED_TABLE, st["table"], F, st["ids"][s], V)
                 for s in range(S)]
    st["emb_none"] = stp.make_embed(stp.STAPLE_EMBED_NONE)
    st["emb_stem"] = [stp.make_embed(stp.STAPLE_EMBED_TABLE, st["table"], F, st["ids"][s], V,
                                     flags=stp.STAPLE_EMBED_REPLACE_UP) for s in range(S)]
    st["wsb"] = stp.staple_workspace_bytes(T, D, F)
    st["ws"] = torch.zeros(st["wsb"], dtype=torch.uint8, device="cuda")
    return st


def decode_step(stp, ctx, w, st, s, stream, mode="staple"):
    """One decode step.  mode: "staple" (row added), "dense" (E path off) or
    "stem" (row replaces the up-projection; W_up not passed)."""
    r = s % st["R"]
    b = s % st["S"]
    emb = {"staple": st["emb"], "stem": st["emb_stem"]}[mode][b] if mode != "dense" else st["emb_none"]
    stp.staple_ffn_fwd(ctx, stp.STAPLE_BF16, w.T, w.D, w.F, st["x"][b], emb, st["wg"][r],
                       None if mode == "stem" else st["wu"][r], st["wd"][r], st["z"], st["y"],
                       None, None, st["ws"], st["wsb"], stream=stream)


def capture_steps(step, n, stream):
    """One CUDA graph of n consecutive steps (step(s) for s in [0, n))."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for s in range(n):
            step(s)
    return g


def time_graph_steps(step, K, G, stream, warmup, world, local):
    """Exactly K steps: a captured graph of G steps replayed K // G times, then
    a graph of the K % G remaining steps.  Untraced; CUDA events on the
    launching stream, max over ranks.  Returns (ms_max, ms_local, clocks)."""
    import torch
    full = capture_steps(step, G, stream) if K >= G else None
    rem = capture_steps(step, K % G, stream) if K % G else None
    with torch.cuda.stream(stream):       # replay() launches on the current stream
        for _ in range(max(1, warmup // G)):
            for g in (full, rem):
                if g is not None:
                    g.replay()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    with Clocks(local) as clk:
        torch.cuda.synchronize()
        t0 = time.time()
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for _ in range(K // G):
                full.replay()
            if rem is not None:
                rem.replay()
            ev1.record(stream)
        torch.cuda.synchronize()
        t1 = time.time()
    ms = ev0.elapsed_time(ev1)
    del full, rem
    return max_over_ranks(ms, world), ms, clk.summary(t0, t1)


def run_decode(stp, ctx, w, args, world, local):
    import torch
    st = decode_setup(stp, w, local)
    stream = torch.cuda.Stream()
    G = st["R"] * st["S"] // 4   # steps per captured graph (cycles weights 16x)
    K = max(1, args.steps)
    out = {}
    for mode in ("staple", "dense", "stem"):
        def step(s, mode=mode):
            decode_step(stp, ctx, w, st, s, stream, mode)

        with torch.cuda.stream(stream):
            for s in range(max(args.warmup, 3)):
                step(s)
        torch.cuda.synchronize()
        assert stp.staple_get_error(ctx, stream) == 0
        ms_max, ms, clocks = time_graph_steps(step, K, G, stream, args.warmup, world, local)
        assert stp.staple_get_error(ctx, stream) == 0
        out[mode] = {"ms": ms_max, "ms_local": ms, "clocks": clocks}
    res = {"K": K, "ms": out["staple"]["ms"], "ms_local": out["staple"]["ms_local"],
           "clocks": out["staple"]["clocks"], "dense_ms": out["dense"]["ms"],
           "dense_clocks": out["dense"]["clocks"], "stem_ms": out["stem"]["ms"],
           "stem_ms_local": out["stem"]["ms_local"]}
    # the same steps again with per-kernel CUDA events recorded around every
    # launch: the kernel list and shares (events between launches stop the
    # programmatic overlap of consecutive launches, so these steps are slower)
    stp.staple_trace_enable(ctx, True)
    tgraph = capture_steps(lambda s: decode_step(stp, ctx, w, st, s, stream), G, stream)
    with torch.cuda.stream(stream):
        for _ in range(4):
            tgraph.replay()
    torch.cuda.synchronize()
    trace = stp.staple_trace_read(ctx)
    stp.staple_trace_enable(ctx, False)
    assert stp.staple_get_error(ctx, stream) == 0
    del tgraph
    kern = kernel_table(trace, G)
    res["kernels"] = kern
    # a captured launch holds one pair of trace events, re-recorded by every
    # replay: the records cover the G captured steps once
    res["launches_per_step"] = sum(d["launches"] for d in kern.values()) / G
    # end to end through the public call with host buffers: every step copies
    # its x and ids in from pinned memory and its y out.  As a serving loop
    # would, the copies run on two copy streams in chunks of C steps, with the
    # device inputs and outputs double-buffered by chunk: chunk c's copies in
    # overlap chunk c-1's layer calls and chunk c-1's copies out overlap
    # chunk c's, and only the first call of a chunk waits on a copy, so the
    # other calls follow one another as programmatic dependents.  The steps
    # are captured in CUDA graphs of up to 512 steps (the first chunk's copies
    # in and the last chunk's copies out of a graph are not overlapped).
    Ke = K
    h2d = st["x"][0].numel() * 2 + st["ids"][0].numel() * 4
    d2h = st["y"].numel() * 2
    C = 16
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    xd = [torch.empty_like(st["x"][0]) for _ in range(2 * C)]
    idd = [torch.empty_like(st["ids"][0]) for _ in range(2 * C)]
    yd = [torch.empty_like(st["y"]) for _ in range(2 * C)]
    embd = [stp.make_embed(stp.STAPLE_EMBED_TABLE, st["table"], w.F, idd[i], w.V)
            for i in range(2 * C)]
    ev_in, ev_used, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def e2e_chunk(s0, n):
        """Steps s0 .. s0+n-1 (n <= C), one chunk; buffers half (s0 // C) % 2."""
        h = (s0 // C) % 2
        cin.wait_event(ev_used[h])        # the chunk two back has read these inputs
        with torch.cuda.stream(cin):
            for k in range(n):
                b = (s0 + k) % st["S"]
                xd[h * C + k].copy_(st["x_host"][b], non_blocking=True)
                idd[h * C + k].copy_(st["ids_host"][b], non_blocking=True)
        ev_in[h].record(cin)
        stream.wait_event(ev_in[h])
        stream.wait_event(ev_out[h])      # the chunk two back's outputs are on the host
        for k in range(n):
            r = (s0 + k) % st["R"]
            stp.staple_ffn_fwd(ctx, stp.STAPLE_BF16, w.T, w.D, w.F, xd[h * C + k], embd[h * C + k],
                               st["wg"][r], st["wu"][r], st["wd"][r], st["z"], yd[h * C + k],
                               None, None, st["ws"], st["wsb"], stream=stream)
        ev_used[h].record(stream)
        cout.wait_event(ev_used[h])
        with torch.cuda.stream(cout):
            for k in range(n):
                st["y_host"][(s0 + k) % st["S"]].copy_(yd[h * C + k], non_blocking=True)
        ev_out[h].record(cout)

    def e2e_graph(n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for e in ev_used + ev_out:     # fork the copy streams into the capture
                e.record(stream)
            for s0 in range(0, n, C):
                e2e_chunk(s0, min(C, n - s0))
            stream.wait_stream(cin)        # and join them before it ends
            stream.wait_stream(cout)
        return g

    G = min(512, Ke)
    full = e2e_graph(G)
    rem = e2e_graph(Ke % G) if Ke % G else None
    with torch.cuda.stream(stream):
        for _ in range(max(1, args.warmup // G)):
            full.replay()
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(Ke // G):
            full.replay()
        if rem is not None:
            rem.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    del full, rem
    e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    res["e2e"] = {"K": Ke, "ms": e_ms, "h2d": h2d, "d2h": d2h}
    # dominant (and only) kernel: the fused decode launch.  Algorithmic bytes
    # of one launch: the three weight matrices, x, the T gathered E rows, ids,
    # and the z and y outputs
    T, D, F = w.T, w.D, w.F
    res["roofline_kernel"] = "k5k6_decode_fused"
    res["alg_bytes"] = 3 * F * D * 2 + T * D * 2 + T * F * 2 + T * 4 + T * F * 2 + T * D * 2
    res["alg_note"] = ("k5k6_decode_fused bytes per launch: W_gate + W_up + W_down (3*F*D*2) + "
                       "x (T*D*2) + E rows (T*F*2) + ids (T*4) + z (T*F*2) + y (T*D*2)")
    return res


# --------------------------------------------------------------------------
# Training layer (host table + 5% cache)
# --------------------------------------------------------------------------

def run_decode_layer(stp, ctx, spec, args, world, local):
    """Decode steps of one layer of another shape ("D,F": T = 64, vocabulary
    8192, table in HBM, four rotating weight sets), untraced graph replays:
    a small case for per-kernel profiling (the 7B shape, 4096,11008, runs the
    one-launch cluster path).  Prints its own JSON line, not the bench line."""
    import torch
    D, F = (int(v) for v in spec.split(","))
    w = syn.Workload(f"decode-layer-{D}x{F}", T=64, D=D, F=F, V=8192, layers=1, dtype="bf16",
                     w_std=0.02, e_std=0.01, x_std=1.0, dy_std=1.0, table="device",
                     cache_frac=0.0, group=1, training=False)
    st = decode_setup(stp, w, local)
    stream = torch.cuda.Stream()
    K = args.steps
    ms, _, clocks = time_graph_steps(lambda s: decode_step(stp, ctx, w, st, s, stream), K,
                                     min(64, K), stream, args.warmup, world, local)
    status = stp.staple_get_error(ctx, stream)
    alg = 3 * F * D * 2 + w.T * D * 2 + 2 * w.T * F * 2 + 4 * w.T + w.T * D * 2
    us = ms * 1000.0 / K
    return {"profile": w.name, "T": w.T, "d_model": D, "d_ff": F, "steps": K,
            "us_per_step": r3(us), "alg_bytes_per_step": alg,
            "achieved_gbs": r3(alg / (us * 1e-6) / 1e9), "clocks": clocks, "status": status}


def run_dw_down(stp, ctx, args, world, local):
    """The training layer's dW_down GEMM alone (staple_ffn_bwd with only
    dw_down: dW_down = dY^T z, T = 16384, D = 2048, F = 8192), L2 flushed
    between calls: a small case for capturing it under ncu (about 1 GB on
    the device).  Prints its own JSON line, not the bench line."""
    import torch
    w = syn.WORKLOADS["olmo2-1b-train-layer"]
    T, D, F = w.T, w.D, w.F
    dy = bf16_randn((T, D), 1.0, syn.SEED_ACT)
    z = bf16_randn((T, F), 1.0, syn.SEED_ACT + 1)
    # x and dgh are passed as the call requires; only dx and dW_gate/up read them
    x = torch.zeros((T, D), dtype=torch.bfloat16, device="cuda")
    dgh = torch.zeros((T, 2 * F), dtype=torch.bfloat16, device="cuda")
    dwd = torch.empty((D, F), dtype=torch.float32, device="cuda")
    wsb = stp.staple_workspace_bytes(T, D, F)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def call():
        stp.staple_ffn_bwd(ctx, stp.STAPLE_BF16, T, D, F, dy, x, z, dgh, None, None, None,
                           None, None, dwd, stream=stream)

    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize()
    ts = []
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1000.0)
    us = statistics.median(ts)
    return {"profile": "dw-down", "T": T, "d_model": D, "d_ff": F, "calls": args.steps,
            "us_median": r3(us), "tflops": r3(2.0 * T * D * F / (us * 1e-6) / 1e12),
            "status": stp.staple_get_error(ctx, stream)}


def run_train(stp, ctx, w, steps, warmup, world, local):
    import torch
    T, D, F, V = w.T, w.D, w.F, w.V
    S = 4
    wg = bf16_randn((F, D), w.w_std, syn.SEED_W)
    wu = bf16_randn((F, D), w.w_std, syn.SEED_W + 1)
    wd = bf16_randn((D, F), w.w_std, syn.SEED_W + 2)
    table_host = bf16_randn((V, F), w.e_std, syn.SEED_E).cpu().pin_memory()
    tab = stp.staple_table_register(ctx, table_host, V * F * 2, V, F, 1, stp.STAPLE_BF16,
                                    stp.STAPLE_TABLE_HOST_PINNED)
    freq = syn.calibration_freq(V)
    cache = stp.staple_cache_build(ctx, tab, freq, w.cache_frac)
    ids = torch.from_numpy(np.stack([syn.zipf_ids(T, V, w.zipf_s, seed=syn.SEED_IDS + w.index + 7919 * s)
                                     for s in range(S)])).cuda()
    x = [bf16_randn((T, D), w.x_std, syn.SEED_ACT + 2 * s) for s in range(S)]
    dy = [bf16_randn((T, D), w.dy_std, syn.SEED_ACT + 2 * s + 1) for s in range(S)]
    i32 = dict(dtype=torch.int32, device="cuda")

    class Retrieval:
        """One microbatch's retrieval outputs (two of them alternate)."""

        def __init__(self):
            self.unique, self.inverse, self.sorted_pos, self.slot, self.miss = (
                torch.empty(T, **i32) for _ in range(5))
            self.seg, self.U, self.mc = (torch.empty(T + 1, **i32), torch.empty(1, **i32),
                                         torch.empty(1, **i32))
            self.rows = torch.empty((T, F), dtype=torch.bfloat16, device="cuda")
            self.emb = stp.make_embed(stp.STAPLE_EMBED_ROWS, self.rows, F, self.inverse, T)
            self.emb_stem = stp.make_embed(stp.STAPLE_EMBED_ROWS, self.rows, F, self.inverse, T,
                                           flags=stp.STAPLE_EMBED_REPLACE_UP)
            self.ready = torch.cuda.Event()   # rows gathered (prefetch streams)
            self.free = torch.cuda.Event()    # last reader done (main stream)

    buf = [Retrieval(), Retrieval()]
    z, g, h = (torch.empty((T, F), dtype=torch.bfloat16, device="cuda") for _ in range(3))
    y = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")
    dgh = torch.empty((T, 2 * F), dtype=torch.bfloat16, device="cuda")
    dE = torch.empty((T, F), dtype=torch.float32, device="cuda")
    dx = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")
    dwg, dwu = (torch.empty((F, D), dtype=torch.float32, device="cuda") for _ in range(2))
    dwd = torch.empty((D, F), dtype=torch.float32, device="cuda")
    wsb = stp.staple_workspace_bytes(T, D, F)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    pf, pf_side = torch.cuda.Stream(), torch.cuda.Stream()   # prefetch: main and miss streams
    emb_none = stp.make_embed(stp.STAPLE_EMBED_NONE)

    def prefetch(s):
        """Retrieval for microbatch s (dedup, probe, hit and miss gathers) on
        the prefetch streams, into the buffer whose previous reader (step
        s - 2) has finished.  Successive microbatches are pipelined this way
        (retrieval-path table, Prefill row); there is no optimizer in this
        layer benchmark, so no row the prefetch reads is updated in between."""
        r = buf[s % 2]
        pf.wait_event(r.free)
        stp.staple_gather_rows(ctx, cache, tab, ids[s % S], T, r.unique, r.inverse, r.seg,
                               r.sorted_pos, r.U, r.slot, r.miss, r.mc, r.rows, stream=pf,
                               side=pf_side)
        r.ready.record(pf)

    def step(s, staple=True, stem=False):
        """staple: the E path on (with stem: the row replaces the
        up-projection, no W_up in the forward or backward); else the dense run."""
        b = s % S
        r = buf[s % 2]
        if staple:
            prefetch(s + 1)
            stream.wait_event(r.ready)
        emb = (r.emb_stem if stem else r.emb) if staple else emb_none
        stp.staple_ffn_fwd(ctx, stp.STAPLE_BF16, T, D, F, x[b], emb, wg, None if stem else wu, wd,
                           z, y, g, h, ws, wsb, stream=stream)
        stp.staple_embed_bwd(ctx, stp.STAPLE_BF16, T, D, F, dy[b], g, h, wd, r.sorted_pos,
                             r.inverse, r.seg, r.U, dgh, dE if staple else None, ws, wsb,
                             stream=stream)
        if staple:
            r.free.record(stream)
        stp.staple_ffn_bwd(ctx, stp.STAPLE_BF16, T, D, F, dy[b], x[b], z, dgh, wg,
                           None if stem else wu, dx, dwg, None if stem else dwu, dwd, stream=stream)

    out = {}

    def timed(staple, stem, s0, n):
        """n consecutive steps from step s0, CUDA events on the layer's stream
        around them.  The first step's retrieval is done before the events (as
        for a pipeline already running), every later one, up to the prefetch of
        the step after the last, falls inside; nothing of another run is still
        on the GPU when the first event is recorded."""
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            if staple:
                prefetch(s0)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for s in range(s0, s0 + n):
                step(s, staple, stem)
            if staple:
                stream.wait_event(buf[(s0 + n) % 2].ready)
            ev1.record(stream)
        return ev0, ev1

    def warm(staple, stem, s0):
        nw = max(warmup, 3)
        with torch.cuda.stream(stream):
            if staple:
                prefetch(s0)
            for s in range(s0, s0 + nw):
                step(s, staple, stem)
            if staple:
                stream.wait_event(buf[(s0 + nw) % 2].ready)
        torch.cuda.synchronize()
        assert stp.staple_get_error(ctx, stream) == 0

    try:
        # The E-path and dense runs alternate in rounds of steps, so that both
        # see the same clocks under the power cap, and the mode that goes
        # first alternates from round to round (ABBA), so that a drift of the
        # clock over the run does not favour either; all of these steps run
        # untraced.  (name, E path on, STEM, SMs the GEMMs leave to the
        # prefetch kernels)
        rounds = 10 if steps >= 10 else 1
        per = [steps // rounds + (1 if r < steps % rounds else 0) for r in range(rounds)]
        stp.staple_set_sm_reserve(ctx, 0)
        warm(True, False, 0)
        warm(False, False, 0)
        barrier(world)
        evs = {"staple_r0": [], "dense": []}
        s_next = 16
        with Clocks(local) as clk:
            torch.cuda.synchronize()
            t0 = time.time()
            for r in range(rounds):
                order = (("staple_r0", True), ("dense", False))
                for mode, staple in (order if r % 2 == 0 else order[::-1]):
                    evs[mode].append(timed(staple, False, s_next, per[r]))
                    s_next += per[r] + 2
            torch.cuda.synchronize()
            t1 = time.time()
        assert stp.staple_get_error(ctx, stream) == 0
        clocks = clk.summary(t0, t1)
        for mode in ("staple_r0", "dense"):
            ms = sum(e0.elapsed_time(e1) for e0, e1 in evs[mode])
            out[mode] = {"ms": max_over_ranks(ms, world), "clocks": clocks, "sm_reserve": 0}
        # one reserved SM, and STEM: timed on their own
        for mode, stem, reserve in (("staple", False, 1), ("stem", True, 1)):
            stp.staple_set_sm_reserve(ctx, reserve)
            warm(True, stem, s_next)
            s_next += 16
            barrier(world)
            with Clocks(local) as clk:
                torch.cuda.synchronize()
                t0 = time.time()
                e0, e1 = timed(True, stem, s_next, steps)
                torch.cuda.synchronize()
                t1 = time.time()
            s_next += steps + 2
            assert stp.staple_get_error(ctx, stream) == 0
            out[mode] = {"ms": max_over_ranks(e0.elapsed_time(e1), world),
                         "clocks": clk.summary(t0, t1), "sm_reserve": reserve}
        # the kernel tables: a separate traced run of a few steps per mode
        stp.staple_set_sm_reserve(ctx, 0)
        nt = min(steps, 10)
        for mode, staple in (("staple_r0", True), ("dense", False)):
            stp.staple_trace_enable(ctx, True)
            timed(staple, False, s_next, nt)
            torch.cuda.synchronize()
            out[mode]["kernels"] = kernel_table(stp.staple_trace_read(ctx), nt)
            stp.staple_trace_enable(ctx, False)
            s_next += nt + 2
        out["U"] = int(buf[0].U.item())
        out["misses"] = int(buf[0].mc.item())
        # the pages' prefill route for the misses on the last batch: packed on
        # the host, bulk copy, scatter (wall time of the whole call, waited for)
        r = buf[0]
        staging_h = torch.empty((T, F), dtype=torch.bfloat16).pin_memory()
        staging_d = torch.empty((T, F), dtype=torch.bfloat16, device="cuda")
        list_h = torch.empty(1 + 2 * T, dtype=torch.int32).pin_memory()
        by_chunk = {}
        for chunk in (64, 128, 256, 512):
            times = []
            for _ in range(6):
                torch.cuda.synchronize()
                t0 = time.perf_counter()
                stp.staple_gather_unique_rows_bulk(ctx, cache, tab, r.unique, r.U, T, r.slot,
                                                   r.miss, r.mc, r.rows, staging_h, staging_d,
                                                   list_h, chunk_rows=chunk, threads=0,
                                                   stream=stream)
                stream.synchronize()
                times.append(time.perf_counter() - t0)
            by_chunk[chunk] = statistics.median(times[1:])
        assert stp.staple_get_error(ctx, stream) == 0
        best = min(by_chunk, key=by_chunk.get)
        t_bulk = by_chunk[best]
        nb = int(r.mc.item()) * F * 2
        out["bulk_misses"] = {"ms": t_bulk * 1e3, "miss_bytes": nb, "gbs": nb / t_bulk / 1e9,
                              "chunk_rows": best,
                              "ms_by_chunk_rows": {c: round(t * 1e3, 3) for c, t in by_chunk.items()},
                              "how": "probe + hits + host pack (all threads) + bulk H2D chunk by "
                                     "chunk + scatter, wall time, median of 5 per chunk size"}
    finally:
        stp.staple_set_sm_reserve(ctx, 0)
        stp.staple_cache_free(cache)
        stp.staple_table_unregister(tab)
    return out


# --------------------------------------------------------------------------
# Stacks of layers (tables grouped G layers per host row)
# --------------------------------------------------------------------------

def pinned_group_tables(n_groups, G, V, F, std, seed0, chunk_rows=4096):
    """Page-locked host tables, one [V][G * F] bf16 array per group (layer
    G*k + j in columns [j F, (j+1) F)).  Values are seeded N(0, std) draws
    made on the GPU (one generator per layer, seed seed0 + layer), rounded to
    bf16 and copied down in row chunks."""
    import torch
    out = []
    for gi in range(n_groups):
        t = torch.empty((V, G * F), dtype=torch.bfloat16, pin_memory=True)
        gens = []
        for j in range(G):
            g = torch.Generator(device="cuda")
            g.manual_seed(seed0 + gi * G + j)
            gens.append(g)
        blk = torch.empty((chunk_rows, G, F), dtype=torch.bfloat16, device="cuda")
        for r0 in range(0, V, chunk_rows):
            n = min(chunk_rows, V - r0)
            for j in range(G):
                blk[:n, j] = (torch.randn((n, F), generator=gens[j], device="cuda") * std).to(torch.bfloat16)
            t[r0:r0 + n].copy_(blk[:n].view(n, G * F))
        out.append(t)
    torch.cuda.synchronize()
    return out


def measure_host_link(nbytes=1 << 30, reps=5):
    """Copy-engine bandwidth between pinned host memory and HBM, each way
    (best of `reps` copies of `nbytes`, CUDA events).  The host link's peak is
    not in the measured-peaks file, so the bench measures it here."""
    import torch
    h = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    d = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out = {}
    for name, dst, src in (("h2d_gbs", d, h), ("d2h_gbs", h, d)):
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            dst.copy_(src, non_blocking=True)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        out[name] = nbytes / (best * 1e-3) / 1e9
    del h, d
    out["bytes"] = nbytes
    return out


def measure_host_adamw(stp, w, U=4529, steps=3):
    """The host AdamW (staple_adamw_rows) on U distinct rows of one layer's
    bf16 table with fp32 moments, all in host memory as the pages keep them:
    per element it reads and writes the weight (2 + 2 bytes) and both moments
    (8 + 8) and reads the fp32 gradient (4).  All host threads."""
    rng = np.random.default_rng(5)
    table = np.zeros((w.V, w.F), np.uint16)            # touched rows only are paged in
    m = np.zeros((w.V, w.F), np.float32)
    v = np.zeros((w.V, w.F), np.float32)
    ids = np.sort(rng.choice(w.V, U, replace=False)).astype(np.int32)
    grad = (rng.standard_normal((U, w.F)) * 0.01).astype(np.float32)
    stp.staple_adamw_rows(table, w.F, stp.STAPLE_BF16, w.F, ids, U, grad, w.F, m, v, w.F,
                          lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, step=1)
    t0 = time.perf_counter()
    for s in range(steps):
        stp.staple_adamw_rows(table, w.F, stp.STAPLE_BF16, w.F, ids, U, grad, w.F, m, v, w.F,
                              lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0,
                              step=s + 2)
    dt = (time.perf_counter() - t0) / steps
    nbytes = U * w.F * 24
    return {"rows": U, "F": w.F, "ms_per_step": dt * 1e3, "rows_per_s": U / dt,
            "gbs": nbytes / dt / 1e9, "threads": os.cpu_count(),
            "bytes_per_step": nbytes, "note": "host memory traffic of one layer's update"}


def release_pinned():
    """Return cached page-locked host blocks to the system (torch keeps freed
    pinned blocks for reuse)."""
    import gc

    import torch
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    f = getattr(torch._C, "_host_emptyCache", None)
    if f is not None:
        f()


def stack_weights(L, D, F, std, seed0=syn.SEED_W):
    from token_indexed_sparse_staple_b200.stack import LayerWeights
    return [LayerWeights(bf16_randn((F, D), std, seed0 + 3 * l), bf16_randn((F, D), std, seed0 + 3 * l + 1),
                         bf16_randn((D, F), std, seed0 + 3 * l + 2)) for l in range(L)]


def run_stack_decode(stp, ctx, w, steps, world, local):
    """16 stacked 7B-shaped layers decoding 64 tokens per step: one dedup and
    four group gathers (side streams) per step, the 16 fused decode layers,
    the whole step replayed from one CUDA graph."""
    import torch

    from token_indexed_sparse_staple_b200.stack import DecodeStack, GroupedTables
    T, D, F, V, L, G = w.T, w.D, w.F, w.V, w.layers, w.group
    t0 = time.time()
    W = stack_weights(L, D, F, w.w_std)
    host = pinned_group_tables(L // G, G, V, F, w.e_std, syn.SEED_E)
    setup_s = time.time() - t0
    freq = syn.calibration_freq(V)
    tables = GroupedTables(ctx, host, V, F, G, freq, w.cache_frac)
    S = 64
    try:
        s = DecodeStack(ctx, W, tables, T, D, F, V)
        ids = torch.from_numpy(np.stack([syn.zipf_ids(T, V, w.zipf_s, seed=syn.SEED_IDS + w.index + 7919 * k)
                                         for k in range(S)])).cuda()
        xs = bf16_randn((S, T, D), w.x_std, syn.SEED_ACT)
        st = torch.cuda.Stream()
        with torch.cuda.stream(st):
            s.ids_buf.copy_(ids[0])
            s.xs[0].copy_(xs[0])
            s.run(st)
        torch.cuda.synchronize()
        assert stp.staple_get_error(ctx, st) == 0
        # one graph per recorded batch: each step's graph copies that batch's ids and x in
        graphs = [s.capture(st, ids[k], xs[k]) for k in range(S)]

        def one(k):
            graphs[k % S].replay()

        with torch.cuda.stream(st):
            for k in range(8):
                one(k)
        torch.cuda.synchronize()
        barrier(world)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with Clocks(local) as clk:
            torch.cuda.synchronize()
            c0 = time.time()
            with torch.cuda.stream(st):
                ev0.record(st)
                for k in range(steps):
                    one(k)
                ev1.record(st)
            torch.cuda.synchronize()
            c1 = time.time()
        assert stp.staple_get_error(ctx, st) == 0
        ms = max_over_ranks(ev0.elapsed_time(ev1), world)
        misses = [int(m.item()) for m in s.r.mc]
        U = int(s.r.U.item())
        s.release()
        del graphs
        # a few steps outside the graph with per-launch CUDA events
        stp.staple_trace_enable(ctx, True)
        with torch.cuda.stream(st):
            for k in range(4):
                s.ids_buf.copy_(ids[k])
                s.run(st)
        torch.cuda.synchronize()
        kern = kernel_table(stp.staple_trace_read(ctx), 4)
        stp.staple_trace_enable(ctx, False)
    finally:
        tables.close()
    step_ms = ms / steps
    wbytes = L * 3 * D * F * 2
    clocks = clk.summary(c0, c1)
    return {"workload": w.name, "layers": L, "groups_of": G, "T": T, "d_model": D, "d_ff": F,
            "steps": steps, "ms_per_step": step_ms, "tokens_per_s": job_value(T * steps, ms, world),
            "U_last_step": U, "misses_last_step_per_group": misses,
            "weight_bytes_per_step": wbytes, "weight_gbs": wbytes / (step_ms * 1e-3) / 1e9,
            "weight_frac": wbytes / (step_ms * 1e-3) / 1e9 / peaks()["hbm_gbs"],
            "sm_mhz": clocks.get("sm_mhz"),
            "table_bytes_host": L * V * F * 2, "setup_s": setup_s,
            "graph": ("one CUDA graph per step (one per recorded batch): the batch's ids and x "
                      "copied in, dedup, 4 group gathers on side streams, 16 layers"),
            "clocks": clocks, "kernels_4_traced_steps": kern}


def run_stack_train(stp, ctx, w, steps, world, local):
    """12 stacked 1B-shaped layers, training: one dedup per step, three group
    gathers (side streams), forward, backward in reverse with every layer's dE
    returned to host memory while the backward continues."""
    import torch

    from token_indexed_sparse_staple_b200.stack import GroupedTables, TrainStack
    T, D, F, V, L, G = w.T, w.D, w.F, w.V, w.layers, w.group
    t0 = time.time()
    W = stack_weights(L, D, F, w.w_std)
    host = pinned_group_tables(L // G, G, V, F, w.e_std, syn.SEED_E)
    setup_s = time.time() - t0
    freq = syn.calibration_freq(V)
    tables = GroupedTables(ctx, host, V, F, G, freq, w.cache_frac)
    S = 4
    # one SM is left to the next step's dedup and first gather, which run
    # beside the backward's GEMMs on the prefetch streams
    stp.staple_set_sm_reserve(ctx, 1)
    try:
        s = TrainStack(ctx, W, tables, T, D, F, V)
        ids = [torch.from_numpy(syn.zipf_ids(T, V, w.zipf_s, seed=syn.SEED_IDS + w.index + 7919 * k)).cuda()
               for k in range(S)]
        x0 = [bf16_randn((T, D), w.x_std, syn.SEED_ACT + 2 * k) for k in range(S)]
        dyt = [bf16_randn((T, D), w.dy_std, syn.SEED_ACT + 2 * k + 1) for k in range(S)]
        st = torch.cuda.Stream()
        k = 0

        def one():
            nonlocal k
            r = s.step(ids[k % S], x0[k % S], dyt[k % S], next_ids=ids[(k + 1) % S], stream=st)
            k += 1
            return r

        with torch.cuda.stream(st):
            for _ in range(2):
                one()
        torch.cuda.synchronize()
        assert stp.staple_get_error(ctx, st) == 0
        barrier(world)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with Clocks(local) as clk:
            torch.cuda.synchronize()
            c0 = time.time()
            with torch.cuda.stream(st):
                ev0.record(st)
                for _ in range(steps):
                    r = one()
                st.wait_event(s.host_ready)   # the last step's dE rows are on the host
                ev1.record(st)
            torch.cuda.synchronize()
            c1 = time.time()
        assert stp.staple_get_error(ctx, st) == 0
        ms = max_over_ranks(ev0.elapsed_time(ev1), world)
        U = int(r.U.item())
        misses = [int(m.item()) for m in r.mc]
        # one more step with per-launch CUDA events: the kernel list
        stp.staple_trace_enable(ctx, True)
        with torch.cuda.stream(st):
            one()
        torch.cuda.synchronize()
        kern = kernel_table(stp.staple_trace_read(ctx), 1)
        stp.staple_trace_enable(ctx, False)
    finally:
        stp.staple_set_sm_reserve(ctx, 0)
        tables.close()
    step_ms = ms / steps
    flops = 18 * T * D * F * L
    h2d = sum(misses) * G * F * 2          # zero-copy miss rows of all groups
    d2h = L * (U * F * 4 + U * 4 + 4)      # dE rows, ids and U of every layer
    pk = peaks()
    tf = flops / (step_ms * 1e-3) / 1e12
    clocks = clk.summary(c0, c1)
    return {"workload": w.name, "layers": L, "groups_of": G, "T": T, "d_model": D, "d_ff": F,
            "steps": steps, "ms_per_step": step_ms, "tokens_per_s": job_value(T * steps, ms, world),
            "U_last_step": U, "misses_last_step_per_group": misses,
            "tflops": tf, "tensor_frac_sustained": tf / pk["bf16_tflops_sustained"],
            "sm_mhz": clocks.get("sm_mhz"),
            "host_link": {"h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                          "h2d_gbs": h2d / (step_ms * 1e-3) / 1e9,
                          "d2h_gbs": d2h / (step_ms * 1e-3) / 1e9},
            "table_bytes_host": L * V * F * 2, "setup_s": setup_s,
            "clocks": clocks, "kernels_one_traced_step": kern}


def train_flops(w):
    return 18 * w.T * w.D * w.F   # 3 forward + 6 backward GEMMs of 2*T*D*F


# --------------------------------------------------------------------------
# CPU oracle legs
# --------------------------------------------------------------------------

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def decode_config(w):
    """The `config` of the decode workload, shared by both arms."""
    return {"workload": w.name, "T": w.T, "d_model": w.D, "d_ff": w.F, "vocab": w.V,
            "table": "device (1.64 GB in HBM)", "weights": "random N(0,0.02) bf16",
            "l2": "inputs larger than L2: 4 rotating weight sets (403 MB) and 64 token batches",
            "graph": "steps replayed from captured CUDA graphs of 64 steps (+ the remainder)"}


def oracle_decode_batch(w):
    """One decode batch for the oracle, fp64: x, the three weights and the T
    tokens' gathered table rows (the oracle needs only those rows)."""
    inp = syn.make_layer_inputs(w, with_table=False)
    x, wg, wu, wd = (inp.f64(k) for k in ("x", "w_gate", "w_up", "w_down"))
    E_rows = syn.bf16_normal((w.T, w.F), w.e_std, syn.SEED_E)[1].astype(np.float64)
    return x, wg, wu, wd, E_rows


def oracle_decode_tokens(batch, n):
    """The oracle's forward of the batch's first n tokens."""
    import oracle
    x, wg, wu, wd, E_rows = batch
    oracle.ffn_forward(x[:n], np.arange(n), wg, wu, wd, E_rows[:n])


def cpu_baseline_decode(w, seconds=12.0):
    """The oracle's forward on whole 64-token batches for ~seconds of CPU time."""
    batch = oracle_decode_batch(w)
    n = 0
    t0 = time.time()
    while time.time() - t0 < seconds or n == 0:
        oracle_decode_tokens(batch, w.T)
        n += 1
    dt = time.time() - t0
    return {"value": n * w.T / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} full decode batches of {w.T} tokens (fp64 numpy oracle), {dt:.1f} s"}


def cpu_baseline_train(w, seconds=12.0, n=256):
    """The oracle's forward and full backward (dx, dW_gate, dW_up, dW_down, dE)
    on the first n tokens of the training microbatch, repeated for ~seconds.
    The layer's cost grows linearly with its token count, so tokens/s over the
    sample stands for the whole 16384-token microbatch (an extrapolation)."""
    import oracle
    inp = syn.make_layer_inputs(w, T=n, with_table=False, with_dy=True)
    x, wg, wu, wd, dy = (inp.f64(k) for k in ("x", "w_gate", "w_up", "w_down", "dy"))
    E_rows = syn.bf16_normal((n, w.F), w.e_std, syn.SEED_E)[1].astype(np.float64)
    ids = np.arange(n)
    reps = 0
    t0 = time.time()
    while time.time() - t0 < seconds or reps == 0:
        fw = oracle.ffn_forward(x, ids, wg, wu, wd, E_rows)
        oracle.ffn_backward(dy, x, ids, wg, wu, wd, fw)
        reps += 1
    dt = time.time() - t0
    return {"value": reps * n / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{reps} x fwd+bwd of {n} of the {w.T} tokens (fp64 numpy oracle), "
                      f"{dt:.1f} s; extrapolated to the microbatch (cost linear in tokens)"}


def cpu_baseline_stack_decode(w, seconds=8.0):
    """The oracle's forward of one of the stack's layers on a whole decode
    batch, repeated for ~seconds; a step runs w.layers such layers, so the
    step's tokens/s is the layer's divided by the layer count (an
    extrapolation: the cost is linear in layers)."""
    one = syn.Workload(w.name + "-one-layer", T=w.T, D=w.D, F=w.F, V=w.V, layers=1,
                       dtype="bf16", w_std=w.w_std, e_std=w.e_std, x_std=w.x_std,
                       dy_std=w.dy_std, table="device", cache_frac=0.0, group=1, training=False)
    batch = oracle_decode_batch(one)
    reps = 0
    t0 = time.time()
    while time.time() - t0 < seconds or reps == 0:
        oracle_decode_tokens(batch, w.T)
        reps += 1
    dt = time.time() - t0
    return {"value": w.T * reps / (dt * w.layers), "unit": "tokens/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"{reps} forwards of one {w.D} x {w.F} layer on a {w.T}-token batch (fp64 "
                      f"numpy oracle), {dt:.1f} s; extrapolated to {w.layers} layers (cost "
                      f"linear in layers)"}


def reference_arm(w, args, budget_s=60.0):
    """--impl reference: the oracle on the decode workload (same config, metric
    and step count as the CUDA arm).  A step is the oracle's forward of the
    step's batch; when K whole batches would take more than budget_s, each
    step is bounded to the batch's first n tokens (n from one timed batch),
    and tokens/s counts the tokens actually computed."""
    batch = oracle_decode_batch(w)
    t0 = time.time()
    oracle_decode_tokens(batch, w.T)
    t_batch = max(time.time() - t0, 1e-6)
    K, W = max(1, args.steps), max(0, args.warmup)
    n = int(max(1, min(w.T, w.T * budget_s / ((K + W) * t_batch))))
    for _ in range(W):
        oracle_decode_tokens(batch, n)
    t0 = time.time()
    for _ in range(K):
        oracle_decode_tokens(batch, n)
    dt = time.time() - t0
    v = K * n / dt
    sample = (f"per step: the forward of {n} of the batch's {w.T} tokens "
              f"({'the whole batch' if n == w.T else 'bounded sample'}), fp64 numpy oracle")
    return {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": K, "warmup": W, "ms_per_step": 1000 * dt / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference", "config": decode_config(w),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "kind": "oracle",
                             "cores": blas_threads(), "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def r3(v):
    return None if v is None else float(f"{v:.4g}")


# --------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60000)
    ap.add_argument("--warmup", type=int, default=256)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=[DEFAULT_WORKLOAD])
    ap.add_argument("--train-steps", type=int, default=200)
    ap.add_argument("--no-train", action="store_true")
    ap.add_argument("--no-stacks", action="store_true")
    ap.add_argument("--stack-decode-steps", type=int, default=256)
    ap.add_argument("--stack-train-steps", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--dw-down", action="store_true",
                    help="only time the training layer's dW_down GEMM (profiling case)")
    ap.add_argument("--decode-layer", default=None, metavar="D,F",
                    help="only time decode steps of one layer of this shape (profiling case)")
    ap.add_argument("--detail", default=None,
                    help="also write every per-kernel table and sub-measurement to this JSON file")
    args = ap.parse_args()
    w = syn.WORKLOADS[args.workload]

    # the reference arm runs on host cores only, so its ranks need no GPU
    rank, world, local = dist_init("gloo" if args.impl == "reference" else None)
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(w, args)), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    import torch

    import token_indexed_sparse_staple_b200 as stp
    torch.cuda.set_device(local)
    ctx = stp.staple_context_create(local)
    pk = peaks()
    detail = {}
    if args.decode_layer or args.dw_down:
        out = (run_dw_down(stp, ctx, args, world, local) if args.dw_down
               else run_decode_layer(stp, ctx, args.decode_layer, args, world, local))
        if rank == 0:
            print(json.dumps(out), flush=True)
        stp.staple_context_destroy(ctx)
        if world > 1:
            import torch.distributed as dist
            barrier(world)
            dist.destroy_process_group()
        return
    dec = run_decode(stp, ctx, w, args, world, local)
    K = dec["K"]
    value = job_value(w.T * K, dec["ms"], world)
    kd = dec["kernels"].get(dec["roofline_kernel"], {})
    # Every launch of a step belongs to the decode layer (the fused kernel and
    # its split-k sum kernel): the untraced timed step bounds the dominant
    # kernel's duration from above; the traced averages are reported beside
    # it (trace events between launches stop their programmatic overlap).
    own = set(dec["kernels"]) <= {"k5k6_decode_fused", "k6r_decode_reduce"}
    one = own and kd
    launch_us = dec["ms_local"] * 1000.0 / K if one else kd.get("avg_us", float("nan"))
    ach = dec["alg_bytes"] / (launch_us * 1e-6) / 1e9
    traffic, traffic_src = captured_traffic(dec["roofline_kernel"])
    dense_us = dec["dense_ms"] * 1000.0 / K
    stem_us = dec["stem_ms_local"] * 1000.0 / K
    stem_bytes = dec["alg_bytes"] - w.F * w.D * 2      # no W_up
    step_us = dec["ms"] * 1000.0 / K
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": dec["ms"] / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": decode_config(w),
        "roofline": {"bound": "hbm", "kernel": dec["roofline_kernel"], "achieved": r3(ach),
                     "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": r3(ach / pk["hbm_gbs"]),
                     "traffic": traffic, "traffic_source": traffic_src,
                     "peak_source": pk["source"] + " (copy bandwidth)",
                     "alg_bytes_per_launch": dec["alg_bytes"], "launch_us": r3(launch_us),
                     "traced_launch_us": kd.get("avg_us"),
                     "traced_reduce_us": dec["kernels"].get("k6r_decode_reduce", {}).get("avg_us"),
                     "duration": ("untraced timed step (the decode kernel and its split-k sum "
                                  "kernel)" if one else "traced per-launch CUDA events")},
        "e2e": {"value": r3(job_value(w.T * dec["e2e"]["K"], dec["e2e"]["ms"], world)),
                "unit": "tokens/s", "h2d_bytes_per_step": dec["e2e"]["h2d"],
                "d2h_bytes_per_step": dec["e2e"]["d2h"], "steps": dec["e2e"]["K"],
                "how": ("per step: pinned H2D of x and ids on a copy stream, staple_ffn_fwd, "
                        "D2H of y on another copy stream; copies in chunks of 16 steps, "
                        "double-buffered by chunk, steps in CUDA graphs of 512")},
        "gpu_launches": int(round(dec["launches_per_step"] * K)),
        "clocks": dec["clocks"],
        "decode_dense": {"us_per_step": r3(dense_us), "us_per_step_staple": r3(step_us),
                         "e_path_overhead": r3((step_us - dense_us) / dense_us),
                         "how": "same kernel and steps with STAPLE_EMBED_NONE (no E rows)"},
        "decode_stem": {"tokens_per_s": r3(job_value(w.T * K, dec["stem_ms"], world)),
                        "us_per_step": r3(stem_us),
                        "hbm_frac": r3(stem_bytes / (stem_us * 1e-6) / 1e9 / pk["hbm_gbs"]),
                        "how": "same steps, STAPLE_EMBED_REPLACE_UP: the row replaces W_up "
                               "(2*F*D*2 weight bytes per step)"},
    }
    detail["decode_kernels"] = dec["kernels"]
    detail["decode_dense_clocks"] = dec["dense_clocks"]
    detail["roofline_note"] = dec["alg_note"]
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_decode(w)
    train = None
    if not args.no_train:
        try:
            wt = syn.WORKLOADS["olmo2-1b-train-layer"]
            tr = run_train(stp, ctx, wt, args.train_steps, 5, world, local)
            # the E-path and dense runs timed in alternating rounds (the same
            # clocks), untraced; the kernel tables come from a separate traced run
            st_ms = tr["staple_r0"]["ms"] / args.train_steps
            de_ms = tr["dense"]["ms"] / args.train_steps
            kern = tr["staple_r0"]["kernels"]
            gemm_flops = {"k5_gateup": 4, "k6_down": 2, "k7_dz": 2, "k9_dx": 4, "k10_dw_gate_up": 4,
                          "k10_dw_down": 2}
            # the dominant kernel of the step's own stream: the largest GEMM (the
            # miss gather runs on a side stream under the previous microbatch's
            # GEMMs and is rated against the host link below)
            top = max(((k, v) for k, v in kern.items() if k in gemm_flops),
                      key=lambda kv: kv[1]["total_ms"])
            tf = gemm_flops[top[0]] * wt.T * wt.D * wt.F / (top[1]["avg_us"] * 1e-6) / 1e12
            link = measure_host_link()
            adamw = measure_host_adamw(stp, wt)
            k4 = kern.get("k4_gather_misses")
            if k4:
                zc = tr["misses"] * wt.F * 2 / (k4["avg_us"] * 1e-6) / 1e9
                link["k4_zero_copy_gbs"] = zc
                link["k4_frac_of_h2d"] = zc / link["h2d_gbs"]
            layer_tf = train_flops(wt) / (st_ms / 1000.0) / 1e12
            train = {
                "workload": wt.name, "tokens_per_s": r3(job_value(wt.T, st_ms, world)),
                "ms_per_step": r3(st_ms), "dense_ms_per_step": r3(de_ms),
                "e_path_overhead": r3((st_ms - de_ms) / de_ms), "steps": args.train_steps,
                "sm_reserve": 0,
                "timing": ("E path and dense run alternated in 10 rounds of steps, the first mode "
                           "alternating (ABBA), untraced"),
                "ms_by_sm_reserve": {str(tr[m]["sm_reserve"]): r3(tr[m]["ms"] / args.train_steps)
                                     for m in ("staple_r0", "staple")},
                "stem_ms_per_step": r3(tr["stem"]["ms"] / args.train_steps),
                "stem_tokens_per_s": r3(job_value(wt.T, tr["stem"]["ms"] / args.train_steps,
                                                  world)),
                "U": tr["U"], "misses": tr["misses"],
                "tflops": r3(layer_tf),
                "layer_frac_sustained": r3(layer_tf / pk["bf16_tflops_sustained"]),
                "roofline": {"bound": "tensor", "kernel": top[0], "achieved": r3(tf),
                             "peak": pk["bf16_tflops_sustained"], "unit": "TFLOP/s",
                             "frac": None if tf is None else r3(tf / pk["bf16_tflops_sustained"]),
                             "peak_source": pk["source"] + " (cuBLAS bf16, sustained)"},
                "clocks": tr["staple_r0"]["clocks"],
            }
            detail["train_layer"] = {"kernels": kern, "kernels_dense": tr["dense"].get("kernels"),
                                     "host_link": link, "host_adamw": adamw,
                                     "bulk_misses": tr.get("bulk_misses"),
                                     "dense_clocks": tr["dense"]["clocks"]}
        except Exception as ex:  # the decode line must still print
            train = {"error": repr(ex)}
        release_pinned()
        if world == 1 and rank == 0 and not args.no_cpu_baseline and "error" not in train:
            train["cpu_baseline"] = cpu_baseline_train(syn.WORKLOADS["olmo2-1b-train-layer"])
    if not args.no_stacks:
        for key, fn, name, n in (("stack_decode", run_stack_decode, "olmo2-7b-decode-16l",
                                  args.stack_decode_steps),
                                 ("stack_train", run_stack_train, "olmo2-1b-train-12l",
                                  args.stack_train_steps)):
            try:
                full = fn(stp, ctx, syn.WORKLOADS[name], n, world, local)
                detail[key] = full
                line[key] = {k: (r3(v) if isinstance(v, float) else v) for k, v in full.items()
                             if k in STACK_KEYS}
            except Exception as ex:  # the headline line must still print
                line[key] = {"error": repr(ex)}
            release_pinned()
        if world == 1 and rank == 0 and not args.no_cpu_baseline:
            sd = line.get("stack_decode", {})
            if "error" not in sd:
                sd["cpu_baseline"] = cpu_baseline_stack_decode(syn.WORKLOADS["olmo2-7b-decode-16l"])
            stt, tb = line.get("stack_train", {}), (train or {}).get("cpu_baseline")
            if "error" not in stt and tb:
                nl = syn.WORKLOADS["olmo2-1b-train-12l"].layers
                stt["cpu_baseline"] = {
                    "value": tb["value"] / nl, "unit": "tokens/s", "cores": tb["cores"],
                    "kind": "oracle",
                    "sample": f"the training layer's oracle sample ({tb['value']:.0f} tokens/s "
                              f"fwd+bwd for one layer) over {nl} layers (cost linear in layers)"}
    if train is not None:
        line["train_layer"] = train   # last, so that a tail of the output holds it
    stp.staple_context_destroy(ctx)
    if rank == 0:
        if args.detail:
            with open(args.detail, "w") as f:
                json.dump({"line": line, "detail": detail}, f, indent=1)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()


# keys of a stack's result that go into the printed line (the rest: --detail)
STACK_KEYS = ("workload", "layers", "steps", "ms_per_step", "tokens_per_s", "weight_gbs",
              "weight_frac", "tflops", "tensor_frac_sustained", "sm_mhz")


if __name__ == "__main__":
    main()
