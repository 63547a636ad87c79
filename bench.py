#!/usr/bin/env python3
"""Benchmark of the tensor-parallel MLP hot path on B200.

Default workload: the 7B-shaped SwiGLU MLP, forward + backward: hidden 4096,
ffn 11008 (gate and up fused into column shards of 2 x 11008/p), tokens
8 x 4096 = 32768, p = 8 shards held as separate buffers on one GPU, bf16
storage with fp32 accumulation. One step = column GEMM (+SwiGLU) -> row GEMM
-> sum over shards (+bias once) -> row backward (dSwiGLU fused) -> column
backward -> sum of the dX partials.

--variant fused (default): the sums over shards happen inside the row GEMM and
the column-backward dX GEMM (one TMEM accumulator over all shards' K slices).
--variant partials: the row GEMM writes p full-shape partials and the reduce
kernel sums them (and likewise for dX). In both variants the standalone
partial-reduce kernel's HBM GB/s is reported: measured inside the step for
"partials", and in its own timed loop over the same partial sizes for "fused".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). For N > 1 (torchrun, one process per GPU) the
p = 8 shards of the one workload split over the N ranks, 8/N per GPU
(dist.DistTPMLP): inside a GPU the shards' sums run in the fused GEMMs, between
GPUs the row layer's all-reduce and the dX all-reduce are NCCL collectives
(strong scaling: the total work is fixed). --replicas instead runs one
independent full replica per GPU (weak scaling, no data-path collective).
Time is the max over ranks of the device-timed region.

--impl reference times the CPU oracle (fp64 numpy, the machine's host cores) on
a bounded sample of the same workload: each step is the full forward and
backward of the MLP on a fixed sample of token rows.
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

HIDDEN, FFN, TOKENS, P = 4096, 11008, 8 * 4096, 8
METRIC = "sharded MLP fwd+bwd TFLOP/s at p shards on 1 B200; partial-reduce HBM GB/s"
WORKLOAD = "7B-shaped SwiGLU MLP fwd+bwd: hidden 4096, ffn 11008, tokens 8x4096, p=8 shards on one GPU"


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    """The measured peaks file (copy GB/s, bf16 TFLOP/s burst and sustained)
    when present and readable, else the fallback figures; a figure the file
    lacks is taken from the fallback (the sustained one scaled from the
    measured burst), and `source` says which."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        got = {k: float(d[k]) for k in FALLBACK_PEAKS if isinstance(d.get(k), (int, float)) and d[k] > 0}
    except Exception:
        got = {}
    if not got:
        return dict(FALLBACK_PEAKS, source="fallback")
    out = dict(FALLBACK_PEAKS)
    out.update(got)
    if "bf16_tflops_sustained" not in got and "bf16_tflops" in got:
        out["bf16_tflops_sustained"] = got["bf16_tflops"] * (FALLBACK_PEAKS["bf16_tflops_sustained"] /
                                                             FALLBACK_PEAKS["bf16_tflops"])
    missing = [k for k in FALLBACK_PEAKS if k not in got]
    out["source"] = "measured" if not missing else "measured (" + ", ".join(missing) + " from the fallback)"
    return out


def mlp_flops(T, h, f):
    # SwiGLU: forward 2*T*h*(2f) + 2*T*f*h; backward twice the forward.
    return 3.0 * (2.0 * T * h * 2 * f + 2.0 * T * f * h)


def gemm_algorithmic_bytes(T, h, f):
    """Bytes each of the six GEMM launches of the fused step must move at least
    once (bf16): its operands read once and its outputs written once.
      column fwd + SwiGLU: X, W1 -> Z, H;   row fwd (shard sum fused): H, W2 -> Y;
      row bwd dgrad + dSwiGLU: dY, W2, Z -> dZ;   dW2: dY, H -> dW2;
      dW1: dZ, X -> dW1;   column bwd dX (shard sum fused): dZ, W1 -> dX."""
    X = Y = dY = dX = T * h * 2
    Z = dZ = T * 2 * f * 2
    H = T * f * 2
    W1 = dW1 = 2 * f * h * 2
    W2 = dW2 = h * f * 2
    return [X + W1 + Z + H, H + W2 + Y, dY + W2 + Z + dZ, dY + H + dW2, dZ + X + dW1, dZ + W1 + dX]


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """Max of a per-rank float over all ranks (device tensor for NCCL, host for gloo)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(flops_per_step, steps, ms_local, world):
    """Whole-job throughput (TFLOP/s) of N weak-scaling replicas: every rank
    processes the same work, and the job takes as long as the slowest rank."""
    ms = max_over_ranks(ms_local, world)
    return world * flops_per_step * steps / (ms / 1e3) / 1e12, ms


# --------------------------------------------------------------- CPU oracle leg
def oracle_sample(rows, seed=0):
    """Inputs for the oracle sample: the first `rows` token rows of the same
    seeded draw and the full weights."""
    import torch
    import tp_synth
    inp = tp_synth.draw_mlp(TOKENS, HIDDEN, FFN, "swiglu", torch.bfloat16, seed=seed)
    import oracle as O
    return (O.f64(inp.X[:rows]), O.f64(inp.W1), O.f64(inp.W2), O.f64(inp.dY[:rows]))


def oracle_step(X, W1, W2, dY):
    import oracle as O
    fwd = O.mlp_fwd(X, W1, None, W2, None, "swiglu")
    O.mlp_bwd(X, W1, W2, fwd["Z"], fwd["H"], dY, "swiglu")


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=1)
    except Exception:
        return os.cpu_count() or 1


def run_cpu_baseline(rows=256, seed=0):
    X, W1, W2, dY = oracle_sample(rows, seed)
    t0 = time.perf_counter()
    oracle_step(X, W1, W2, dY)
    dt = time.perf_counter() - t0
    fl = mlp_flops(rows, HIDDEN, FFN)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": f"full fwd+bwd of the MLP on {rows} of the {TOKENS} token rows (fp64 numpy), "
                      f"{dt:.1f} s"}


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    rows = args.ref_rows
    X, W1, W2, dY = oracle_sample(rows)
    fl = mlp_flops(rows, HIDDEN, FFN)
    for _ in range(args.warmup):
        oracle_step(X, W1, W2, dY)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(X, W1, W2, dY)
    dt = time.perf_counter() - t0
    value = fl * args.steps / dt / 1e12
    cores = oracle_threads()
    sample = f"each step: full fwd+bwd of the MLP on {rows} of the {TOKENS} token rows (fp64 numpy)"
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded; tp_synth)",
           "config": {"workload": WORKLOAD, "hidden": HIDDEN, "ffn": FFN, "tokens": TOKENS, "p": P,
                      "act": "swiglu", "sample_rows": rows},
           "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    return 0


# ------------------------------------------------------------------- GPU leg
def run_dist(args, world, rank, local):
    """The 7B SwiGLU MLP with its p = 8 shards split over the N ranks (8/N per
    GPU), NCCL all-reduces between them; strong scaling."""
    import torch
    import tp_synth
    from megatron_tensor_transformer_gemm_b200 import tp
    from megatron_tensor_transformer_gemm_b200.dist import DistTPMLP

    if P % world:
        raise SystemExit(f"--gpus {world}: the {P} shards do not split over {world} GPUs")
    peaks = load_peaks()
    dev = torch.device("cuda", local)
    T = args.tokens
    inp = tp_synth.draw_mlp(T, HIDDEN, FFN, "swiglu", torch.bfloat16, seed=0)  # replicated input
    m = DistTPMLP(HIDDEN, FFN, P, "swiglu", device=dev, comm=args.comm)
    m.load_weights(inp.W1, inp.W2)
    X_h, dY_h = inp.X.pin_memory(), inp.dY.pin_memory()
    del inp
    X, dY = X_h.to(dev), dY_h.to(dev)
    m.alloc(T)
    stream = torch.cuda.current_stream()
    pl = m.plan
    peer = args.comm == "peer"
    gemm_calls = ("column_fwd", "row_fwd_push_peer", "row_bwd", "column_bwd_push_peer") if peer else \
        ("column_fwd", "row_fwd_reduce", "row_bwd", "column_bwd_reduce")
    orig = {n: getattr(pl, n) for n in gemm_calls}
    gemm_ev, comm_ev = [], []

    def timed(fn, bucket):
        def wrapper(*a, **k):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            out = fn(*a, **k)
            e1.record(stream)
            bucket.append((e0, e1))
            return out
        return wrapper

    import megatron_tensor_transformer_gemm_b200.dist as D
    orig_sum = D.sum_over_ranks
    orig_peer = m.peer.reduce if peer else None

    def step(instrument=False):
        for n in gemm_calls:
            setattr(pl, n, timed(orig[n], gemm_ev) if instrument else orig[n])
        if peer:   # the reduce + wait steps (the pushes are inside the GEMMs)
            m.peer.reduce = timed(orig_peer, comm_ev) if instrument else orig_peer
        else:
            D.sum_over_ranks = timed(orig_sum, comm_ev) if instrument else orig_sum
        m.forward(X)
        m.backward(dY)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    tp.launch_count(reset=True)
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(args.steps):
        step(instrument=True)
    s1.record(stream)
    torch.cuda.synchronize()
    launches = tp.launch_count(reset=True)
    barrier(world)
    clk = clocks.stop()
    for n in gemm_calls:
        setattr(pl, n, orig[n])
    D.sum_over_ranks = orig_sum
    if peer:
        m.peer.reduce = orig_peer
    flops = m.flops(T)
    ms = max_over_ranks(s0.elapsed_time(s1), world)
    value = flops * args.steps / (ms / 1e3) / 1e12
    gemm_ms = sum(a.elapsed_time(b) for a, b in gemm_ev)
    comm_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in comm_ev), world)
    gemm_tflops = (flops / world) * args.steps / (gemm_ms / 1e3) / 1e12
    # end to end: every rank copies X and dY in from pinned memory and Y and dX out
    Y_h = torch.empty(T, HIDDEN, dtype=torch.bfloat16).pin_memory()
    dX_h = torch.empty(T, HIDDEN, dtype=torch.bfloat16).pin_memory()
    e2e = None
    if not args.skip_e2e:
        barrier(world)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            X.copy_(X_h, non_blocking=True)
            dY.copy_(dY_h, non_blocking=True)
            Y = m.forward(X)
            Y_h.copy_(Y, non_blocking=True)
            dX = m.backward(dY)
            dX_h.copy_(dX, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        nb = X_h.numel() * 2
        e2e = {"value": flops * args.steps / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": 2 * nb * world, "d2h_bytes_per_step": 2 * nb * world,
               "ms_per_step": e2e_ms / args.steps}
    status = tp.device_status()
    barrier(world)   # no rank frees its peer memory while another may still write into it
    if peer:
        m.close_peer()
    if rank != 0:
        return 0
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded tp_synth draws: X, dY ~ N(0,1), W ~ N(0,0.02))",
        "config": {"workload": WORKLOAD.replace("on one GPU", f"over {world} GPUs"), "hidden": HIDDEN,
                   "ffn": FFN, "tokens": T, "p": P, "act": "swiglu", "global_batch": 8, "seq_len": 4096,
                   "parallelism": f"tp{world}: {P // world} of the {P} shards per GPU, "
                                  + ("peer-memory all-reduce" if peer else "NCCL all-reduce"),
                   "l2": "inputs larger than L2 (X and dY 268 MB each); no flush"},
        "roofline": {"bound": "tensor", "kernel": "tp_gemm_kernel (tcgen05)", "achieved": gemm_tflops,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": gemm_tflops / peaks["bf16_tflops"],
                     "peak_kind": f"bf16 burst ({peaks['source']}), per GPU", "traffic": None},
        "comm": {"collective": ("peer memory: row blocks pushed from the GEMM epilogues into the owners' "
                                "receive buffers, reduced once and pushed to every rank (all-reduce of Y and dX)")
                 if peer else "NCCL all-reduce of Y and dX ([T, 4096] bf16) per step",
                 "ms_per_step": comm_ms / args.steps,
                 "bytes_per_rank_per_step": 2 * 2 * (world - 1) / world * T * HIDDEN * 2},
        "e2e": e2e, "gpu_launches": launches, "clocks": clk, "device_status": status,
        "cpu_baseline": None,
    }
    print(json.dumps(out), flush=True)
    return 0


def run_ours(args, world, rank, local):
    import torch
    import tp_synth
    from megatron_tensor_transformer_gemm_b200 import tp
    from megatron_tensor_transformer_gemm_b200.block import TPMLP

    peaks = load_peaks()
    dev = torch.device("cuda", local)
    T = args.tokens
    inp = tp_synth.draw_mlp(T, HIDDEN, FFN, "swiglu", torch.bfloat16, seed=rank)
    X_h = inp.X.pin_memory()
    dY_h = inp.dY.pin_memory()
    fused = args.variant == "fused"
    m = TPMLP(HIDDEN, FFN, P, "swiglu", "bf16", dev, fused=fused,
              overlap_chunks=4 if args.variant == "overlap" else 0,
              group_wgrad=args.wgrad_grouping)
    m.load_weights(inp.W1.to(dev), inp.W2.to(dev))
    del inp
    X = X_h.to(dev)
    dY = dY_h.to(dev)
    m.alloc(T)
    stream = torch.cuda.current_stream()

    # Per-launch CUDA events around the GEMM and reduce calls (same stream).
    gemm_ev, red_ev = [], []
    pl = m.plan
    gemm_calls = ("column_fwd", "row_fwd_partial", "row_bwd", "column_bwd", "row_fwd_reduce",
                  "column_bwd_reduce")
    orig = {name: getattr(pl, name) for name in gemm_calls + ("reduce_partials",)}

    n_gemm = [0]

    def timed(name, bucket):
        fn = orig[name]

        def wrapper(*a, **k):
            if bucket is None:
                return fn(*a, **k)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            c0 = tp.launch_count()
            e0.record(stream)
            fn(*a, **k)
            e1.record(stream)
            if bucket is gemm_ev:
                n_gemm[0] += tp.launch_count() - c0
            bucket.append((name, e0, e1))
        return wrapper

    def step(instrument=False):
        g = gemm_ev if instrument else None
        # the overlapped variant launches its reduces on a side stream, where
        # events on this stream would not bracket them: time those standalone
        r = red_ev if instrument and args.variant != "overlap" else None
        for name in gemm_calls:
            setattr(pl, name, timed(name, g))
        pl.reduce_partials = timed("reduce_partials", r)
        m.forward(X)
        m.backward(dY)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- device-timed region
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    tp.launch_count(reset=True)
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(args.steps):
        step(instrument=True)
    s1.record(stream)
    torch.cuda.synchronize()
    launches = tp.launch_count(reset=True)
    barrier(world)
    clk = clocks.stop()
    ms_local = s0.elapsed_time(s1)
    flops = mlp_flops(T, HIDDEN, FFN)
    value, ms = aggregate(flops, args.steps, ms_local, world)

    # GEMM launches (the dominant kernel): algorithmic FLOPs / summed launch time.
    # The row_bwd and column_bwd calls each hold two GEMM launches plus a small
    # column-sum (db) only when biases exist (not in this workload).
    gemm_ms = sum(e0.elapsed_time(e1) for _, e0, e1 in gemm_ev)
    n_gemm_launches = n_gemm[0]
    gemm_tflops = flops * args.steps / (gemm_ms / 1e3) / 1e12
    red_bytes_launch = P * T * HIDDEN * 2 + T * HIDDEN * 2
    if red_ev:
        red_ms = sum(e0.elapsed_time(e1) for _, e0, e1 in red_ev)
        red_gbs = red_bytes_launch * len(red_ev) / (red_ms / 1e3) / 1e9
        red_where = "inside the timed steps (2 per step)"
    else:
        red_gbs = time_standalone_reduce(pl, T, args.steps, stream)
        red_where = "standalone loop over the same partial sizes (p=8 x [T, 4096] bf16)"
    red_bytes = red_bytes_launch

    # ---- end-to-end through the public API with host buffers
    e2e = None
    if not args.skip_e2e:
        e2e = run_e2e(m, X_h, dY_h, T, flops, args, world, stream)
    coll = None if args.skip_collectives else time_sp_collectives(peaks, stream, rank)
    others = None
    if not args.skip_workloads and world == 1:
        # free the 7B buffers first; every other configuration, briefly
        del m, X, dY
        torch.cuda.empty_cache()
        others = {}
        for wl, graph in (("sp", False), ("attn", False), ("stack", True)):
            sub = argparse.Namespace(**vars(args))
            sub.workload, sub.steps, sub.warmup, sub.graph = wl, 10, 3, graph
            o = measure_other(sub, world, rank, local, sample_clocks=False)
            keep = ("value", "unit", "ms_per_step", "frac_of_burst_peak", "roofline", "gpu_launches",
                    "device_status")
            others[wl] = {"workload": o["config"]["workload"], "cuda_graph": graph, "l2": o["config"]["l2"],
                          **{k: o[k] for k in keep}}
    status = tp.device_status()
    if rank != 0:
        return 0
    return report(args, world, T, ms, value, flops, gemm_tflops, n_gemm_launches, peaks,
                  red_gbs, red_bytes, e2e, launches, clk, status, red_where, coll, others)


def time_standalone_reduce(pl, T, steps, stream):
    """HBM GB/s of tp_reduce_partials summing p = 8 bf16 partials [T, 4096]."""
    import torch
    Pt = [torch.randn(T, HIDDEN, device="cuda", dtype=torch.bfloat16) for _ in range(P)]
    Y = torch.empty(T, HIDDEN, device="cuda", dtype=torch.bfloat16)
    for _ in range(3):
        pl.reduce_partials(T, Pt, None, None, Y)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    n = max(2 * steps, 4)
    e0.record(stream)
    for _ in range(n):
        pl.reduce_partials(T, Pt, None, None, Y)
    e1.record(stream)
    torch.cuda.synchronize()
    nbytes = (P + 1) * T * HIDDEN * 2
    gbs = nbytes * n / (e0.elapsed_time(e1) / 1e3) / 1e9
    del Pt, Y
    torch.cuda.empty_cache()
    return gbs


def time_sp_collectives(peaks, stream, rank):
    """HBM GB/s of the Megatron-SP collectives at the SP workload's sizes (seq
    8192, hidden 8192, p 8, bf16): S4' reduce-scatter of the row partials, S9
    all-gather of dY, S1 LayerNorm fused with the sequence all-gather. Each is
    timed as a replayed CUDA graph of 10 launches (algorithmic bytes / device
    time); every buffer set is larger than L2."""
    import torch
    from megatron_tensor_transformer_gemm_b200 import tp
    from megatron_tensor_transformer_gemm_b200.block import CapturedStep
    T, h, p = 8192, 8192, 8
    t = T // p
    g = torch.Generator(device="cpu").manual_seed(500 + rank)
    plan = tp.Plan(h, 0, 0, p, "bf16", "none")
    dev = torch.device("cuda", torch.cuda.current_device())
    bf = torch.bfloat16
    parts = [torch.randn(T, h, generator=g).to(bf).to(dev) for _ in range(p)]
    outs = [torch.empty(t, h, dtype=bf, device=dev) for _ in range(p)]
    full = torch.empty(T, h, dtype=bf, device=dev)
    xs = [torch.randn(t, h, generator=g).to(bf).to(dev) for _ in range(p)]
    gam = (1 + 0.1 * torch.randn(h, generator=g)).to(bf).to(dev)
    bet = (0.1 * torch.randn(h, generator=g)).to(bf).to(dev)
    mean = torch.empty(T, dtype=torch.float32, device=dev)
    rstd = torch.empty(T, dtype=torch.float32, device=dev)
    cases = [
        ("reduce_scatter", "reduce_kernel (S4' reduce-scatter of 8 partials [8192, 8192])",
         lambda: plan.reduce_scatter_seq(T, parts, None, None, outs), p * T * h * 2 + T * h * 2),
        ("all_gather", "gather_kernel (S9 all-gather of dY, 8 x [1024, 8192])",
         lambda: plan.reduce_scatter_seq_bwd(T, outs, full), 2 * T * h * 2),
        ("ln_all_gather", "ln_fwd_kernel (S1 LayerNorm fused with the sequence all-gather)",
         lambda: plan.layernorm_all_gather_seq(T, xs, gam, bet, full, mean, rstd), 2 * T * h * 2 + T * 8),
    ]
    # reference only (not on the path): a plain device copy of the same bytes,
    # the ceiling an all-gather of this size meets
    src_full = torch.randn(T, h, generator=g).to(bf).to(dev)
    cases.append(("copy_reference", "torch copy_ of [8192, 8192] bf16 (reference, not on the path)",
                  lambda: full.copy_(src_full), 2 * T * h * 2))
    res = {}
    reps = 10
    for key, kname, fn, nbytes in cases:
        def rep(fn=fn):
            for _ in range(reps):
                fn()
        graph = CapturedStep(rep)
        for _ in range(2):
            graph()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(3):
            graph()
        e1.record(stream)
        torch.cuda.synchronize()
        sec = e0.elapsed_time(e1) / 1e3 / (3 * reps)
        gbs = nbytes / sec / 1e9
        res[key] = {"kernel": kname, "achieved": gbs, "unit": "GB/s", "us": sec * 1e6,
                    "bytes_per_launch": nbytes, "frac": gbs / peaks["hbm_gbs"],
                    "frac_of_8TBs": gbs / 8000.0}
        del graph
    del parts, outs, full, xs, src_full
    torch.cuda.empty_cache()
    return res


def run_e2e(m, X_h, dY_h, T, flops, args, world, stream):
    """Every step copies X and dY in from pinned host memory and Y and dX
    out, through HostStepPipeline (the copies of one step overlap the GEMMs
    of its neighbours); the timed region ends when the last copy-out has
    landed."""
    import torch
    from megatron_tensor_transformer_gemm_b200.block import HostStepPipeline
    Y_h = torch.empty(T, HIDDEN, dtype=torch.bfloat16).pin_memory()
    dX_h = torch.empty(T, HIDDEN, dtype=torch.bfloat16).pin_memory()
    pipe = HostStepPipeline(m, T)
    for _ in range(2):
        pipe.step(X_h, dY_h, Y_h, dX_h)
    pipe.finish()
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    pipe.h2d.wait_stream(stream)  # the first copy-in starts inside the timed region
    for _ in range(args.steps):
        pipe.step(X_h, dY_h, Y_h, dX_h)
    pipe.finish()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_value, e2e_ms = aggregate(flops, args.steps, e0.elapsed_time(e1), world)
    h2d = X_h.numel() * 2 + dY_h.numel() * 2
    d2h = Y_h.numel() * 2 + dX_h.numel() * 2
    return {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps}


def gemm_source_hash():
    """sha256 of the GEMM kernel sources: ncu traffic figures taken on other
    sources are not reported."""
    import hashlib
    h = hashlib.sha256()
    for f in ("tp_gemm_sm100.cu", "tp_device.cuh"):
        with open(os.path.join(ROOT, "megatron_tensor_transformer_gemm_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(T, variant):
    """DRAM bytes per GEMM launch (mean over the six launches of one step) from
    the committed ncu capture, if it was taken on this workload, variant and
    kernel source; None otherwise."""
    path = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    try:
        d = json.load(open(path))
    except Exception:
        return None
    if d.get("tokens") != T or d.get("variant") != variant or d.get("source_sha256") != gemm_source_hash():
        return None
    return d.get("bytes_per_launch"), d.get("per_launch_bytes")


def report(args, world, T, ms, value, flops, gemm_tflops, n_gemm_launches, peaks, red_gbs,
           red_bytes, e2e, launches, clk, status, red_where, coll, others=None):
    traffic, per_launch = measured_traffic(T, args.variant) or (None, None)
    alg = gemm_algorithmic_bytes(T, HIDDEN, FFN)
    alg_mean = sum(alg) / len(alg)
    ratios = None
    if per_launch and len(per_launch) == len(alg) and args.variant == "fused":
        ratios = [round(m / a, 2) for m, a in zip(per_launch, alg)]
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = run_cpu_baseline(rows=args.cpu_rows)
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded tp_synth draws: X, dY ~ N(0,1), W ~ N(0,0.02))",
        "config": {"workload": WORKLOAD if T == TOKENS else WORKLOAD.replace("tokens 8x4096", f"tokens {T}"),
                   "hidden": HIDDEN, "ffn": FFN, "tokens": T, "p": P,
                   "act": "swiglu", "global_batch": world * 8, "seq_len": 4096,
                   "parallelism": f"{P} TP shards per GPU x {world} replicas",
                   "variant": args.variant,
                   "l2": "inputs larger than L2 (X and dY 268 MB each); no flush"},
        "roofline": {"bound": "tensor", "kernel": "tp_gemm_kernel (tcgen05)",
                     "achieved": gemm_tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": gemm_tflops / peaks["bf16_tflops"],
                     "peak_kind": f"bf16 burst ({peaks['source']}): the timed region lasts under a second",
                     "frac_of_sustained_peak": gemm_tflops / peaks["bf16_tflops_sustained"],
                     "launches_timed": n_gemm_launches, "traffic": traffic,
                     "algorithmic_bytes_per_launch": alg_mean,
                     "traffic_ratio": None if traffic is None else traffic / alg_mean,
                     "traffic_ratio_per_launch": ratios},
        "reduce": {"kernel": "reduce_kernel", "achieved": red_gbs, "unit": "GB/s",
                   "peak": peaks["hbm_gbs"], "frac": red_gbs / peaks["hbm_gbs"],
                   "peak_kind": f"HBM copy ({peaks['source']})",
                   "frac_of_8TBs": red_gbs / 8000.0, "bytes_per_launch": red_bytes,
                   "measured": red_where},
        "collectives": coll,
        "workloads": others,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk,
        "device_status": status,
        "cpu_baseline": cpu,
    }
    print(json.dumps(out), flush=True)
    return 0


def run_other(args, world, rank, local):
    """--workload attn|sp|stack: one of the other configurations, printed as
    the JSON line of measure_other."""
    out = measure_other(args, world, rank, local)
    if rank == 0:
        print(json.dumps(out), flush=True)
    return 0


def measure_other(args, world, rank, local, sample_clocks=True):
    """Device-timed throughput of the other workloads (parity cases of the
    suite): the attention block forward (hidden 4096, 32 heads x 128, seq
    4096, batch 2, p 8) with its attention core forward and backward timed
    alone, the Megatron-SP SwiGLU MLP fwd+bwd (hidden 8192, ffn 28672, seq
    8192, p 8) and the 12-layer stack fwd+bwd (hidden 512, MLP 2048, 8 heads,
    tokens 8x512, p 4). Returns the JSON-line dict."""
    import torch
    import tp_synth
    from megatron_tensor_transformer_gemm_b200 import tp
    from megatron_tensor_transformer_gemm_b200.block import CapturedStep, SPMLP, TPAttention, TPLayer

    peaks = load_peaks()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    if args.workload == "attn":
        b, s, h, H, p = 2, 4096, 4096, 32, 8
        a = tp_synth.draw_attn_block(b, s, h, torch.bfloat16, seed=rank)
        blk = TPAttention(h, H, p, dev, fused=args.variant == "fused")
        blk.load_weights(a.Wqkv.to(dev), a.Wo.to(dev))
        X = a.X.to(dev)
        flops = blk.flops_fwd(b, s)
        step = lambda: blk.forward(X, b, s, residual=X)
        name = "attention block fwd: hidden 4096, 32 heads x 128, seq 4096, batch 2, p=8, causal"
        l2 = "inputs larger than L2 (X 67 MB, Wqkv 101 MB, the shards' QKV 201 MB); no flush"
        # attention-core launches alone, for the roofline of the dominant kernel
        core = lambda: blk.plan.attention_fwd(b, s, blk.QKV, blk.O, blk.LSE)
        core_flops = 4.0 * b * H * (s * (s + 1) / 2) * (h // H)
    elif args.workload == "sp":
        s_, h, f, p = 8192, 8192, 28672, 8
        X, g, be, W1, W2, dY = tp_synth.draw_sp_mlp(s_, h, f, p, torch.bfloat16, seed=rank)
        sp = SPMLP(h, f, p, "swiglu", dev, fused=args.variant == "fused")
        sp.mlp.load_weights(W1.to(dev), W2.to(dev))
        t = s_ // p
        Xs = [X[j * t:(j + 1) * t].to(dev) for j in range(p)]
        dYs = [dY[j * t:(j + 1) * t].to(dev) for j in range(p)]
        flops = sp.flops(s_)

        def step():
            sp.forward(Xs)
            sp.backward(dYs)
        name = "Megatron-SP SwiGLU MLP fwd+bwd: hidden 8192, ffn 28672, seq 8192, batch 1, p=8"
        l2 = "inputs larger than L2 (W1 940 MB, W2 470 MB, gathered X 134 MB); no flush"
        core, core_flops = None, None
    else:
        L, b, s_, h, f, H, p = 12, 8, 512, 512, 2048, 8, 4
        X, layers, dY = tp_synth.draw_block_stack(L, b, s_, h, f, torch.bfloat16, seed=rank)
        lays = []
        for prm in layers:
            lay = TPLayer(h, f, H, p, dev, fused=args.variant == "fused")
            lay.load(type(prm)(**{k: getattr(prm, k).to(dev) for k in prm.__dataclass_fields__}))
            lays.append(lay)
        Xd, dYd = X.to(dev), dY.to(dev)
        T = b * s_
        per_layer = (3.0 * (2.0 * T * h * f * 2) + 3.0 * (2.0 * T * h * 3 * h + 2.0 * T * h * h)
                     + 3.0 * 4.0 * b * H * (s_ * (s_ + 1) / 2) * (h // H) * 1.0)
        flops = L * per_layer

        def step():
            x = Xd
            for lay in lays:
                x = lay.forward(x, b, s_)
            g = dYd
            for lay in reversed(lays):  # weight gradients joined once, after the last layer
                g = lay.backward(g, b, s_, join=False)
            tp.backward_join()
        name = "12-layer block stack fwd+bwd: hidden 512, MLP 2048, 8 heads x 64, tokens 8x512, p=4"
        # a layer keeps about 65 MB of activations for its backward (LN outputs, QKV,
        # attention output, Z and H of the MLP), so the step's data is well over L2
        l2 = "a step touches about 0.8 GB (12 layers' saved activations), larger than L2; no flush"
        core, core_flops = None, None
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    graph = None
    if args.graph:
        graph = CapturedStep(step)
        step = graph
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
    clocks = ClockSampler(local)
    if sample_clocks:
        clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    tp.launch_count(reset=True)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    launches = tp.launch_count(reset=True)
    if graph is not None:
        launches = graph.launches * args.steps  # replays launch the captured kernels
    clk = clocks.stop() if sample_clocks else None
    value, ms = aggregate(flops, args.steps, e0.elapsed_time(e1), world)
    roof = None
    if core is not None:
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(args.steps):
            core()
        c1.record(stream)
        torch.cuda.synchronize()
        ach = core_flops * args.steps / (c0.elapsed_time(c1) / 1e3) / 1e12
        roof = {"bound": "tensor", "kernel": "attn_fwd_kernel (tcgen05)", "achieved": ach,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"],
                "peak_kind": f"bf16 burst ({peaks['source']}; timed alone)", "traffic": None}
        if args.workload == "attn":
            # The attention backward core alone (D prep + dK/dV + dQ launches):
            # 2.5x the forward's FLOPs (S recomputed, dV, dP, dQ, dK).
            blk.alloc_bwd()
            g = torch.Generator(device="cpu").manual_seed(7 + rank)
            for x in blk.dO:
                x.copy_(torch.randn(x.shape, generator=g).to(torch.bfloat16))
            bwd = lambda: blk.plan.attention_bwd(b, s, blk.QKV, blk.O, blk.dO, blk.LSE, blk.dQKV)
            for _ in range(3):
                bwd()
            torch.cuda.synchronize()
            c0.record(stream)
            for _ in range(args.steps):
                bwd()
            c1.record(stream)
            torch.cuda.synchronize()
            achb = 2.5 * core_flops * args.steps / (c0.elapsed_time(c1) / 1e3) / 1e12
            roof["backward"] = {"kernel": "attn_bwd_prep + attn_bwd_dkdv_st + attn_bwd_dq_gemm (tcgen05)",
                                "achieved": achb, "unit": "TFLOP/s", "frac": achb / peaks["bf16_tflops"],
                                "flops_per_launch_set": 2.5 * core_flops}
    out = {"metric": f"{args.workload} TFLOP/s on 1 B200", "value": value, "unit": "TFLOP/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded tp_synth)",
           "config": {"workload": name, "variant": args.variant,
                      "cuda_graph": bool(args.graph), "l2": l2}, "roofline": roof,
           "frac_of_burst_peak": value / peaks["bf16_tflops"],
           "gpu_launches": launches, "clocks": clk,
           "device_status": tp.device_status()}
    if graph is not None:
        del graph
    torch.cuda.empty_cache()
    return out


def run_peer_emul(args, world, rank, local):
    """The peer-memory all-reduce of the 7B row layer (hidden 4096, ffn 11008,
    tokens 8x4096) with 8 ranks of one shard each emulated on this GPU: every
    rank's receive buffer, flags and output are local, and each step is taken
    for all 8 ranks before the next (push GEMMs, then reduces, then waits), so
    no kernel waits for a later launch. Times each step over the 8 ranks
    beside the single-GPU fused row GEMM of the same FLOPs; the reduce's
    algorithmic bytes per rank: 8 slots read + 8 output blocks written."""
    import torch
    from megatron_tensor_transformer_gemm_b200 import tp
    from megatron_tensor_transformer_gemm_b200.dist import bf16_view

    peaks = load_peaks()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    T, h, f, W = args.tokens, HIDDEN, FFN, P
    t, fp = T // W, f // W
    g = torch.Generator(device="cpu").manual_seed(2000 + rank)
    H = [torch.randn(T, fp, generator=g).to(torch.bfloat16).to(dev) for _ in range(W)]
    W2 = [(torch.randn(h, fp, generator=g) * 0.02).to(torch.bfloat16).to(dev) for _ in range(W)]
    fused = tp.Plan(h, f, 0, W, "bf16", "none")
    Y = torch.empty(T, h, dtype=torch.bfloat16, device=dev)
    plans = [tp.Plan(h, fp, 0, 1, "bf16", "none") for _ in range(W)]
    mem, outs = [], []
    try:
        for _ in range(W):
            mem.append(tp.peer_alloc(tp.PEER_FLAG_BYTES + 2 * T * h)[0])
            outs.append(tp.peer_alloc(2 * T * h)[0])
        grp = [tp.peer_group(W, r, T * h, mem, [q + tp.PEER_FLAG_BYTES for q in mem]) for r in range(W)]
        blocks = [[q + r * t * h * 2 for q in outs] for r in range(W)]
        epoch = 1
        steps = {
            "fused row GEMM, one GPU (tp_row_fwd_reduce, 8 shards in one accumulator)":
                lambda: fused.row_fwd_reduce("mlp", T, H, W2, None, None, Y),
            "push: 8 x tp_gemm_kernel (1 shard each, row blocks stored into 8 receive buffers) + peer_signal":
                lambda: [plans[r].row_fwd_push_peer("mlp", T, [H[r]], [W2[r]], grp[r], epoch) for r in range(W)],
            "reduce: 8 x peer_reduce_kernel (8 slots summed, block pushed to 8 outputs) + peer_signal":
                lambda: [tp.peer_reduce(grp[r], T, h, None, None, blocks[r], epoch) for r in range(W)],
            "wait: 8 x peer_wait_kernel":
                lambda: [tp.peer_wait(grp[r], epoch) for r in range(W)],
        }
        for fn in steps.values():
            for _ in range(args.warmup):
                fn()
        torch.cuda.synchronize()
        if tp.lib.tp_get_device_status(None, None) != 0:
            raise SystemExit("a peer wait gave up in the warm-up")
        clocks = ClockSampler(local)
        clocks.start()
        tp.launch_count(reset=True)
        per = []
        for name, fn in steps.items():
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                fn()
            e1.record(stream)
            torch.cuda.synchronize()
            per.append({"step": name, "ms": e0.elapsed_time(e1) / args.steps})
        launches = tp.launch_count(reset=True)
        clk = clocks.stop()
        status = tp.device_status()
    finally:
        torch.cuda.synchronize()
        for q in mem + outs:
            tp.peer_free(q)
    flops = 2.0 * T * h * f
    red_bytes = W * (W * t * h * 2 + W * t * h * 2)
    per[0]["tflops"] = flops / (per[0]["ms"] / 1e3) / 1e12
    per[1]["tflops"] = flops / (per[1]["ms"] / 1e3) / 1e12
    per[2]["bytes"] = red_bytes
    per[2]["gbs"] = red_bytes / (per[2]["ms"] / 1e3) / 1e9
    if rank != 0:
        return 0
    gbs = per[2]["gbs"]
    print(json.dumps({
        "metric": "peer all-reduce steps of the 7B row layer, 8 ranks emulated on 1 B200: reduce GB/s",
        "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sum(x["ms"] for x in per[1:]), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded torch draws)",
        "config": {"workload": f"row layer hidden {h}, ffn {f}, tokens {T}, 8 ranks x 1 shard, emulated on one GPU "
                               "(peer stores land in local HBM; NVLink is not exercised)",
                   "l2": "every buffer set larger than L2; no flush"},
        "roofline": {"bound": "hbm", "kernel": "peer_reduce_kernel", "achieved": gbs, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "peak_kind": f"HBM copy ({peaks['source']})",
                     "traffic": None},
        "steps_timed": per, "gpu_launches": launches, "clocks": clk, "device_status": status}), flush=True)
    return 0


def run_hbm(args, world, rank, local):
    """Device-timed HBM throughput of the memory-bound rows, each kernel timed
    on its own over the same buffers (algorithmic bytes / event time; sp_hbm:
    the sequence-parallel collectives and LayerNorm of the SP config):
    vocab -- embedding lookup, vocab-parallel cross-entropy (loss + dlogits,
    in place) and embedding gradient; Llama-7B shapes: vocab 32000, hidden
    4096, tokens 8x4096, p 8.
    norm -- hidden-sharded RMSNorm and LayerNorm forward + backward; hidden
    8192 split over p 8, tokens 8x4096."""
    import torch
    from megatron_tensor_transformer_gemm_b200 import tp

    peaks = load_peaks()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    g = torch.Generator(device="cpu").manual_seed(1000 + rank)
    kernels = []   # (name, fn, algorithmic bytes per launch)
    if args.workload == "vocab":
        T, V, h, p = args.tokens, 32000, 4096, 8
        plan = tp.Plan(h, 0, 0, p, "bf16", "none")
        Vp = plan.set_vocab(V)
        Vs = Vp // p
        E = [(torch.randn(Vs, h, generator=g) * 0.02).to(torch.bfloat16).to(dev) for _ in range(p)]
        ids = torch.randint(0, V, (T,), generator=g, dtype=torch.int32).to(dev)
        Y = torch.empty(T, h, dtype=torch.bfloat16, device=dev)
        L = [(torch.randn(T, Vs, generator=g) * 2).to(torch.bfloat16).to(dev) for _ in range(p)]
        loss = torch.empty(T, dtype=torch.float32, device=dev)
        lse = torch.empty(T, dtype=torch.float32, device=dev)
        dY = torch.randn(T, h, generator=g).to(torch.bfloat16).to(dev)
        dE = [torch.empty(Vs, h, dtype=torch.bfloat16, device=dev) for _ in range(p)]
        kernels = [
            ("vocab_ce_kernel", lambda: plan.vocab_cross_entropy(T, L, ids, 1.0 / T, loss, lse, L),
             T * Vp * 2 * 2 + T * 12),
            ("embed_fwd_kernel", lambda: plan.embedding_fwd(T, ids, E, Y), T * h * 2 * 2 + T * 4),
            ("embed_bwd_kernel", lambda: plan.embedding_bwd(T, ids, dY, dE), T * h * 2 + Vp * h * 2 + T * 4),
        ]
        name = f"vocab-parallel embedding + cross-entropy: vocab 32000 (padded to a multiple of 8p), hidden 4096, tokens {T}, p=8"
    elif args.workload == "sp_hbm":
        # Megatron-SP's memory-bound steps at the SP config's sizes (seq 8192,
        # hidden 8192, p 8): S1 LayerNorm fused with the sequence all-gather,
        # S4' reduce-scatter of the row partials, S9 all-gather of dY, S8's
        # reduce-scatter of the dX partials, and a LayerNorm backward over all
        # rows (every buffer set larger than L2).
        T, h, p = min(args.tokens, 8192), 8192, 8
        t = T // p
        plan = tp.Plan(h, 0, 0, p, "bf16", "none")
        xs = [torch.randn(t, h, generator=g).to(torch.bfloat16).to(dev) for _ in range(p)]
        gam = (1 + 0.1 * torch.randn(h, generator=g)).to(torch.bfloat16).to(dev)
        bet = (0.1 * torch.randn(h, generator=g)).to(torch.bfloat16).to(dev)
        U = torch.empty(T, h, dtype=torch.bfloat16, device=dev)
        mean = torch.empty(T, dtype=torch.float32, device=dev)
        rstd = torch.empty(T, dtype=torch.float32, device=dev)
        parts = [torch.randn(T, h, generator=g).to(torch.bfloat16).to(dev) for _ in range(p)]
        outs = [torch.empty(t, h, dtype=torch.bfloat16, device=dev) for _ in range(p)]
        full = torch.empty(T, h, dtype=torch.bfloat16, device=dev)
        dxf = torch.empty(T, h, dtype=torch.bfloat16, device=dev)
        dgam = torch.empty(h, dtype=torch.float32, device=dev)
        dbet = torch.empty(h, dtype=torch.float32, device=dev)
        plan.layernorm_all_gather_seq(T, xs, gam, bet, U, mean, rstd)
        kernels = [
            ("ln_fwd_kernel (LayerNorm + sequence all-gather)",
             lambda: plan.layernorm_all_gather_seq(T, xs, gam, bet, U, mean, rstd), T * h * 2 * 2 + T * 8),
            ("reduce_kernel (reduce-scatter of the row partials)",
             lambda: plan.reduce_scatter_seq(T, parts, None, None, outs), p * T * h * 2 + T * h * 2),
            ("gather_kernel (all-gather of dY)",
             lambda: plan.reduce_scatter_seq_bwd(T, outs, full), T * h * 2 * 2),
            ("reduce_kernel (reduce-scatter of the dX partials)",
             lambda: plan.all_gather_seq_bwd(T, parts, outs), p * T * h * 2 + T * h * 2),
            ("ln_bwd (all T rows: dx + dgamma, dbeta)",
             lambda: plan.layernorm_bwd(T, full, gam, U, mean, rstd, dxf, dgam, dbet),
             T * h * 2 * 3 + T * 8),
        ]
        name = f"Megatron-SP memory-bound steps: seq {T}, hidden 8192, p=8 (LN+AG, RS, AG, RS, LN bwd)"
    else:
        T, h, p = args.tokens, 8192, 8
        plan = tp.Plan(h, 0, 0, p, "bf16", "none")
        hs = h // p
        X = [torch.randn(T, hs, generator=g).to(torch.bfloat16).to(dev) for _ in range(p)]
        gam = [(1 + 0.1 * torch.randn(hs, generator=g)).to(torch.bfloat16).to(dev) for _ in range(p)]
        bet = [(0.1 * torch.randn(hs, generator=g)).to(torch.bfloat16).to(dev) for _ in range(p)]
        Yn = [torch.empty_like(x) for x in X]
        dYn = [torch.randn(T, hs, generator=g).to(torch.bfloat16).to(dev) for _ in range(p)]
        dXn = [torch.empty_like(x) for x in X]
        dg = [torch.empty(hs, dtype=torch.float32, device=dev) for _ in range(p)]
        db = [torch.empty(hs, dtype=torch.float32, device=dev) for _ in range(p)]
        mean = torch.empty(T, dtype=torch.float32, device=dev)
        rstd = torch.empty(T, dtype=torch.float32, device=dev)
        kernels = [
            ("norm_hsh_row_fwd_kernel (rms)", lambda: plan.norm_sharded_fwd("rms", T, X, gam, None, Yn, None, rstd),
             T * h * 2 * 2 + T * 4),
            ("norm_hsh_bwd (rms)", lambda: plan.norm_sharded_bwd("rms", T, X, gam, dYn, None, rstd, dXn, dg),
             T * h * 2 * 3 + T * 4),
            ("norm_hsh_row_fwd_kernel (layer)", lambda: plan.norm_sharded_fwd("layer", T, X, gam, bet, Yn, mean, rstd),
             T * h * 2 * 2 + T * 8),
            ("norm_hsh_bwd (layer)", lambda: plan.norm_sharded_bwd("layer", T, X, gam, dYn, mean, rstd, dXn, dg, db),
             T * h * 2 * 3 + T * 8),
        ]
        name = f"hidden-sharded RMSNorm + LayerNorm fwd+bwd: hidden 8192 over p=8, tokens {T}"

    def step():
        for _, fn, _ in kernels:
            fn()
    step_bytes = sum(b for _, _, b in kernels)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    tp.launch_count(reset=True)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    launches = tp.launch_count(reset=True)
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    value = step_bytes * args.steps * world / (ms / 1e3) / 1e9
    from megatron_tensor_transformer_gemm_b200.block import CapturedStep

    def timed(fn):
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(args.steps):
            fn()
        c1.record(stream)
        torch.cuda.synchronize()
        return c0.elapsed_time(c1) / 1e3 / args.steps

    # Each kernel's device time comes from replaying it as a captured graph:
    # a kernel of a few tens of microseconds is otherwise shorter than the
    # Python + ctypes call that launches it, and the eager loop (us_eager)
    # then times the host.
    per = []
    for kname, fn, nbytes in kernels:
        eager = timed(fn)
        sec = timed(CapturedStep(fn))
        per.append({"kernel": kname, "bytes_per_launch": nbytes, "us": sec * 1e6, "us_eager": eager * 1e6,
                    "achieved": nbytes / sec / 1e9, "frac": nbytes / sec / 1e9 / peaks["hbm_gbs"]})
    top = per[0]
    if rank != 0:
        return 0
    print(json.dumps({"metric": f"{args.workload} algorithmic HBM GB/s on 1 B200", "value": value,
                      "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                      "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
                      "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded torch draws)",
                      "config": {"workload": name, "l2": "every buffer set larger than L2; no flush",
                                 "kernel_timing": "CUDA-graph replay of each kernel (eager loop: us_eager)"},
                      "roofline": {"bound": "hbm", "kernel": top["kernel"], "achieved": top["achieved"],
                                   "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": top["frac"],
                                   "peak_kind": f"HBM copy ({peaks['source']})", "traffic": None},
                      "kernels": per, "gpu_launches": launches, "clocks": clk,
                      "device_status": tp.device_status()}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=8192, help="token rows in the oracle baseline sample")
    ap.add_argument("--ref-rows", type=int, default=1024, help="token rows per oracle step (--impl reference)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=TOKENS,
                    help="token rows (default 8x4096; smaller values are for profiling only)")
    ap.add_argument("--skip-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--skip-collectives", action="store_true",
                    help="skip the Megatron-SP collective GB/s measurements")
    ap.add_argument("--skip-workloads", action="store_true",
                    help="skip the brief runs of the other configurations (SP, attention, stack)")
    ap.add_argument("--variant", choices=["fused", "partials", "overlap"], default="fused",
                    help="sum over shards inside the GEMMs (fused), via p partials + reduce, "
                         "or partials with each token block's reduce overlapped with the next "
                         "block's GEMM (overlap)")
    ap.add_argument("--workload", choices=["mlp7b", "attn", "sp", "stack", "vocab", "norm", "sp_hbm", "peer"],
                    default="mlp7b",
                    help="mlp7b (the metric's workload) or another config of the suite")
    ap.add_argument("--replicas", action="store_true",
                    help="N > 1: one independent replica per GPU (weak scaling) instead of the "
                         "shards split over the GPUs")
    ap.add_argument("--comm", choices=["nccl", "peer"], default="nccl",
                    help="N > 1, mlp7b: the all-reduces of Y and dX through NCCL, or through libtp's "
                         "peer-memory steps (push from the GEMM epilogue, reduce, wait)")
    ap.add_argument("--wgrad-grouping", action="store_true",
                    help="mlp7b: launch the row and column backward's weight gradients as one "
                         "grouped GEMM instead of two")
    ap.add_argument("--graph", action="store_true",
                    help="replay each step as one captured CUDA graph (other workloads)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = (1, int(os.environ.get("RANK", "0")), 0)
    if args.impl == "reference":
        # The oracle runs on rank 0's host cores only; no GPU or process group needed.
        return run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
    world, rank, local = dist_setup()
    if args.workload == "mlp7b":
        rc = run_dist(args, world, rank, local) if world > 1 and not args.replicas else \
            run_ours(args, world, rank, local)
    elif args.workload in ("vocab", "norm", "sp_hbm"):
        rc = run_hbm(args, world, rank, local)
    elif args.workload == "peer":
        rc = run_peer_emul(args, world, rank, local)
    else:
        rc = run_other(args, world, rank, local)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
