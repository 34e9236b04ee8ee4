#!/usr/bin/env python
"""Benchmark of the NABLA block-sparse attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input at
the 720p-like training shape (B=1, 40 heads, 20 x 48 x 80 latent = 76,800
tokens, head dim 128, p = 0.7, STA 3x3x3):
    flatten Q, K, V (grid -> flattened order)
    build the block mask (pool, pooled scores, CDF cut, STA, row + column lists)
    block-sparse attention forward (O, LSE)
    block-sparse attention backward (dQ, dK, dV)
    unflatten O, dQ, dK, dV (flattened -> grid order)

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl nabla|reference]

Prints one JSON line (rank 0).  `value` is effective TFLOP/s on kept blocks
(forward 4*64*64*D + backward 10*64*64*D FLOP per kept block pair), whole job.
Timing: CUDA events on the launching stream, barrier + synchronize around the
K timed steps, max over ranks.  Every input tensor (786 MB) is larger than the
126 MB L2, so no flush is needed between steps.
"""
import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "block-sparse attn fwd/bwd ms & eff. TFLOP/s at 76.8K tokens; mask-build GB/s"
WORKLOAD = "train"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch, per
# head, from one ncu capture of `bench.py --heads 8` (same shape, 8 heads;
# heads are independent, so the traffic scales with their number), with the
# SHA-256 (first 12 hex digits) of the kernel sources it was taken from.  When
# the sources no longer match, the bench reports no traffic rather than a
# stale figure.
NCU_DRAM = {
    # pre 317.0 + 4.0 MB, dK/dV 653.4 + 292.6 MB, dQ 649.9 + 142.5 MB at 8 heads
    ("train", "attn_bwd"): {"bytes_per_head": (317.04e6 + 3.97e6 + 653.38e6 + 292.59e6
                                               + 649.92e6 + 142.47e6) / 8,
                            "sources_sha": "aae2a86a0837"},
    # 475.7 + 140.4 MB at 8 heads
    ("train", "attn_fwd"): {"bytes_per_head": (475.69e6 + 140.43e6) / 8,
                            "sources_sha": "9ea9d3d0ece4"},
}
KERNEL_SOURCES = {
    "attn_bwd": ("attn_bwd_sm100.cu", "sm100.cuh", "common.cuh"),
    "attn_fwd": ("attn_fwd_sm100.cu", "sm100.cuh", "common.cuh"),
}
# dense bf16 tensor-core work of one SM per clock: two M=128 x N=128 x K=128
# MMAs (2 x 4.19 MFLOP) take 1024 cycles
TENSOR_FLOP_PER_CLK_SM = 8192
NUM_SMS = 148


def sources_sha(op):
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[op]:
        with open(os.path.join(ROOT, "adaptive_block_sparse_fractal_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def tensor_peak_at_clock(sm_mhz):
    """TFLOP/s of the tensor pipes of all SMs at the given SM clock."""
    return NUM_SMS * TENSOR_FLOP_PER_CLK_SM * sm_mhz * 1e6 / 1e12 if sm_mhz else None


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("nabla", "reference"), default="nabla")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the long-clip p sweep (kept fraction vs time) added to the line")
    ap.add_argument("--workload", default=WORKLOAD, choices=("train", "long"),
                    help="train: 720p-like training step (the benchmark); long: 92,160-token clip")
    ap.add_argument("--heads", type=int, default=None,
                    help="run fewer heads (profiling captures only; not a benchmark result)")
    return ap.parse_args(argv)


def workload_of(args):
    import dataclasses
    from adaptive_block_sparse_fractal_b200 import synth
    w = synth.WORKLOADS[args.workload]
    if args.workload == "long":
        w = dataclasses.replace(w, backward=True)
    if args.heads is not None:
        w = dataclasses.replace(w, heads=args.heads)
    return w


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_config(w):
    return {
        "workload": "%s: B=%d heads=%d T*H*W=%dx%dx%d (%d tokens, %d blocks of 64) D=%d "
                    "p=%.2f STA %dx%dx%d; flatten + mask + fwd + bwd + unflatten"
                    % ("train-720p" if w.name == "train" else w.name, w.B, w.heads, w.T, w.H, w.W,
                       w.N, w.nb, w.D, w.p, *w.window),
        "global_batch": w.B,
        "seq_len": w.N,
        "heads": w.heads,
        "head_dim": w.D,
        "p": w.p,
        "sta_window": list(w.window),
        "cell": list(w.cell),
        "l2": "no flush: every input tensor (%.0f MB) exceeds the 126 MB L2" % (w.BH * w.N * w.D * 2 / 1e6),
    }


# --------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------
class Clocks:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.QUERY,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# --------------------------------------------------------------------------
# CPU oracle timing (bounded sample)
# --------------------------------------------------------------------------
def oracle_sample(w, n_fwd=8, n_dq=4, seed=0):
    """The oracle on a bounded sample of one head of the workload, timed, and
    extrapolated to one whole step (all heads, mask + forward + backward).

    Timed: the mask of the head (every row), the forward of n_fwd sampled query
    blocks, and the backward of n_dq sampled query blocks (dQ) plus one key
    block (dK, dV).  The oracle's backward recomputes the
    forward rows it needs (LSE and D of every query block the selection
    touches), so its FLOPs are counted as it performs them.  The key block is
    the one with the shortest column list of the head, which bounds the rows
    it needs; the rates measured are per FLOP, so the choice does not bias
    the extrapolation:
      forward      4 * 64 * 64 * D per kept block pair of a selected row,
      LSE rows     4 * 64 * 64 * D per kept pair of every needed query block,
      dQ           6 * 64 * 64 * D per kept pair (S, dP, dQ),
      dK, dV       8 * 64 * 64 * D per kept pair of the column (S, dP, dV, dK).
    A whole step in the oracle is then, per head, the mask plus every kept
    pair at 4 (forward) + 18 (backward: LSE rows, dQ loop, dK/dV loop) units,
    each part at the rate measured on its sample.  Returns a dict with the
    extrapolated seconds per step, the step's kept-pair FLOP count (the metric's
    14 units per pair, as on the GPU) and a description."""
    import numpy as np
    import oracle
    from adaptive_block_sparse_fractal_b200 import synth
    w1 = synth.Workload(w.name, 1, 1, w.T, w.H, w.W, w.D, w.cell, w.p, w.window)
    inp = synth.make_inputs(w1, seed, with_dout=True)
    flat = {n: oracle.flatten_tokens(synth.bits(inp[n]).reshape(1, w.N, w.D), w.T, w.H, w.W, w.P)
            for n in ("q", "k", "v")}
    dout = synth.bits(inp["dout"]).reshape(1, w.N, w.D)
    t0 = time.perf_counter()
    m = oracle.build_mask(flat["q"], flat["k"], w.grid_blocks, w.p, w.scale, w.window, cols=True)
    t_mask = time.perf_counter() - t0
    q, k, v = (oracle.bf16_bits_to_f64(flat[n]) for n in ("q", "k", "v"))
    do = oracle.bf16_bits_to_f64(dout)
    rc, cc = m["row_cnt"][0], m["col_cnt"][0]
    unit = 64.0 * 64 * w.D
    rng = np.random.default_rng(seed)
    fsel = [int(i) for i in rng.choice(w.nb, n_fwd, replace=False)]
    t0 = time.perf_counter()
    oracle.attn_fwd(q, k, v, m["row_idx"], m["row_cnt"], w.scale, sel=[(0, i) for i in fsel])
    t_fwd = time.perf_counter() - t0
    rate_fwd = 4 * unit * float(rc[fsel].sum()) / t_fwd
    qsel = [int(i) for i in rng.choice(w.nb, n_dq, replace=False)]
    kj = int(np.argmin(cc))
    need = set(qsel) | set(int(i) for i in m["col_idx"][0, kj, :cc[kj]])
    bwd_flop = unit * (4 * float(sum(int(rc[i]) for i in need)) + 6 * float(rc[qsel].sum())
                       + 8 * float(cc[kj]))
    t0 = time.perf_counter()
    oracle.attn_bwd(q, k, v, do, m["row_idx"], m["row_cnt"], m["col_idx"], m["col_cnt"],
                    w.scale, dq_sel=[(0, i) for i in qsel], kv_sel=[(0, kj)])
    t_bwd = time.perf_counter() - t0
    rate_bwd = bwd_flop / t_bwd
    kept_head = float(rc.sum())
    s_step = w.BH * (t_mask + kept_head * (4 * unit / rate_fwd + 18 * unit / rate_bwd))
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    desc = ("oracle (float64 C, OpenMP, %d threads) on one head of the same workload: mask for all "
            "%d rows (%.2f s), forward of %d sampled query blocks (%.2f s, %.1f GFLOP/s), backward "
            "of %d sampled query blocks + 1 key block with the forward rows it recomputes "
            "(%d query blocks; %.2f s, %.1f GFLOP/s); extrapolated to %d heads x all %d kept "
            "pairs per head: %.0f s per step" % (cores, w.nb, t_mask, n_fwd, t_fwd, rate_fwd / 1e9,
                                                 n_dq, len(need), t_bwd, rate_bwd / 1e9, w.BH,
                                                 int(kept_head), s_step))
    return {"s_step": s_step, "flop_step": 14 * unit * kept_head * w.BH, "cores": cores,
            "desc": desc, "sample_s": t_mask + t_fwd + t_bwd}


# --------------------------------------------------------------------------
# distributed plumbing
# --------------------------------------------------------------------------
def dist_init(n):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d" % (n, world))
    return rank, world, local


def max_over_ranks(x, world, device):
    """Maximum of a per-rank scalar over all ranks (every rank gets it)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def head_range(heads, world, rank):
    """Heads [h0, h1) of every batch element that rank `rank` of `world` owns:
    the heads are split into equal contiguous runs, one per GPU (masks,
    forward and backward are independent per head, so no data moves between
    the GPUs)."""
    if heads % world:
        raise SystemExit("%d heads do not split evenly over %d GPUs" % (heads, world))
    n = heads // world
    return rank * n, (rank + 1) * n


def sum_over_ranks(x, world, device):
    """Sum of a per-rank scalar over all ranks (every rank gets it)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def whole_job_tflops(flop_all_ranks, ms_per_step):
    """Strong scaling over a head partition: the job's FLOPs (all ranks'
    heads of the one problem) in the slowest rank's time."""
    return flop_all_ranks / (ms_per_step * 1e-3) / 1e12


def long_p_sweep(dev, reps=5, warmup=3):
    """Kept-block fraction against time on the long clip (92,160 tokens,
    12 heads, 1,440 blocks) for each p of its sweep: mask build from the
    flattened Q, K and the block-sparse forward, each timed with CUDA events
    (median of `reps` after `warmup`)."""
    import statistics as st
    import torch
    from adaptive_block_sparse_fractal_b200 import nabla, synth
    w = synth.WORKLOADS["long"]
    shape = nabla.shape_of(w.B, w.heads, w.T, w.H, w.W, w.D, w.P)
    grid = synth.make_inputs_device(w, 0, dev, with_dout=False)
    q, k, v = (nabla.flatten(grid[n], w.T, w.H, w.W, w.P) for n in ("q", "k", "v"))
    del grid
    stream = torch.cuda.current_stream(dev)
    mask = nabla.alloc_mask(shape, dev, cols=False)
    ws_m = nabla.workspace(shape, nabla.OP_BUILD_MASK, dev)
    ws_f = nabla.workspace(shape, nabla.OP_ATTN_FWD, dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.BH, w.N), dtype=torch.float32, device=dev)

    def timed(fn):
        for _ in range(warmup):
            fn()
        out = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            out.append(a.elapsed_time(b))
        return st.median(out)

    rows = []
    for p in w.p_sweep:
        prm = nabla.params_of(p, w.window, D=w.D)
        t_mask = timed(lambda: nabla.build_mask(shape, prm, q, k, mask=mask, ws=ws_m))
        t_fwd = timed(lambda: nabla.attn_fwd(shape, prm, q, k, v, mask, o=o, lse=lse, ws=ws_f))
        kept = int(mask["row_cnt"].sum().item())
        rows.append({"p": p, "kept_fraction": kept / (w.BH * w.nb * w.nb),
                     "build_mask_ms": t_mask, "attn_fwd_ms": t_fwd,
                     "attn_fwd_tflops": 4.0 * 64 * 64 * w.D * kept / (t_fwd * 1e-3) / 1e12})
    return {"workload": "long: B=1 heads=12 T*H*W=60x32x48 (92160 tokens, 1440 blocks) D=128 "
                        "STA 3x3x3, cell 2x4x4; mask from flattened Q,K + forward per p",
            "rows": rows}


def config_timings(dev, reps=20, warmup=5):
    """The two small workloads, each call timed on its own with CUDA events
    (median of `reps` after `warmup`), with a 256 MB write between repetitions
    so that every timed call starts from a cold L2 (their inputs fit in it):
      tiny   (2 heads, 4 x 16 x 16, D = 64, p = 0.9): flatten of Q, mask build
             from the flattened Q and K, forward;
      small  (24 heads, 8 x 32 x 32, D = 128, p = 0.8): mask build, forward."""
    import statistics as st
    import torch
    from adaptive_block_sparse_fractal_b200 import nabla, synth
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def timed(fn):
        for _ in range(warmup):
            fn()
        out = []
        for _ in range(reps):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            out.append(a.elapsed_time(b))
        return st.median(out)

    res = {}
    for name in ("tiny", "small"):
        w = synth.WORKLOADS[name]
        shape = nabla.shape_of(w.B, w.heads, w.T, w.H, w.W, w.D, w.P)
        prm = nabla.params_of(w.p, w.window, D=w.D)
        grid = synth.make_inputs_device(w, 0, dev, with_dout=False)
        q, k, v = (nabla.flatten(grid[n], w.T, w.H, w.W, w.P) for n in ("q", "k", "v"))
        mask = nabla.alloc_mask(shape, dev, cols=False)
        ws_m = nabla.workspace(shape, nabla.OP_BUILD_MASK, dev)
        ws_f = nabla.workspace(shape, nabla.OP_ATTN_FWD, dev)
        o = torch.empty_like(q)
        lse = torch.empty((w.BH, w.N), dtype=torch.float32, device=dev)
        fq = torch.empty_like(q)
        row = {"workload": "%s: B=%d heads=%d T*H*W=%dx%dx%d (%d tokens, %d blocks) D=%d p=%.2f "
                           "STA %dx%dx%d" % (name, w.B, w.heads, w.T, w.H, w.W, w.N, w.nb, w.D, w.p,
                                             *w.window),
               "l2": "256 MB write before every timed call"}
        if name == "tiny":
            t = timed(lambda: nabla.flatten(grid["q"], w.T, w.H, w.W, w.P, out=fq))
            row["flatten_ms"] = t
            row["flatten_gbs"] = 2.0 * q.numel() * 2 / (t * 1e-3) / 1e9
        t_mask = timed(lambda: nabla.build_mask(shape, prm, q, k, mask=mask, ws=ws_m))
        t_fwd = timed(lambda: nabla.attn_fwd(shape, prm, q, k, v, mask, o=o, lse=lse, ws=ws_f))
        kept = int(mask["row_cnt"].sum().item())
        mask_bytes = 4.0 * w.N * w.D * w.BH + 16.0 * w.nb * w.D * w.BH + w.nb * w.nb * w.BH / 8.0 \
            + 2.0 * kept + 4.0 * w.BH * w.nb
        row.update({"build_mask_ms": t_mask, "build_mask_gbs": mask_bytes / (t_mask * 1e-3) / 1e9,
                    "attn_fwd_ms": t_fwd, "kept_fraction": kept / (w.BH * w.nb * w.nb),
                    "attn_fwd_tflops": 4.0 * 64 * 64 * w.D * kept / (t_fwd * 1e-3) / 1e12})
        res[name] = row
        del grid, q, k, v, mask, ws_m, ws_f, o, lse, fq
    del flush
    torch.cuda.empty_cache()
    return res


def run_reference(args):
    rank, world, _ = dist_init(args.gpus)
    if rank != 0:
        return 0
    w = workload_of(args)
    steps = []
    for s in range(args.warmup + args.steps):
        r = oracle_sample(w, seed=s)
        if s >= args.warmup:
            steps.append(r)
    s_step = sum(r["s_step"] for r in steps) / len(steps)
    value = sum(r["flop_step"] for r in steps) / sum(r["s_step"] for r in steps) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * s_step, "ms_per_step_kind": "extrapolated from a timed sample",
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": steps[-1]["cores"],
                         "kind": "oracle", "sample": steps[-1]["desc"],
                         "extrapolated_ms_per_step": 1e3 * s_step},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_nabla(args):
    import torch
    import torch.distributed as dist
    from adaptive_block_sparse_fractal_b200 import nabla, synth

    rank, world, local = dist_init(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    nabla.lib()
    import dataclasses
    w_job = workload_of(args)
    h0, h1 = head_range(w_job.heads, world, rank)
    w = dataclasses.replace(w_job, heads=h1 - h0)  # this rank's share of the problem
    shape = nabla.shape_of(w.B, w.heads, w.T, w.H, w.W, w.D, w.P)
    prm = nabla.params_of(w.p, w.window, D=w.D, flags=nabla.EMIT_COLS)

    grid = synth.make_inputs_device(w_job, args.seed, dev, with_dout=True, head_range=(h0, h1))
    B = {
        "flat": {n: torch.empty_like(grid[n]) for n in ("q", "k", "v")},
        "o": torch.empty_like(grid["q"]),
        "lse": torch.empty((w.BH, w.N), dtype=torch.float32, device=dev),
        "dq": torch.empty_like(grid["q"]), "dk": torch.empty_like(grid["q"]),
        "dv": torch.empty_like(grid["q"]),
        "out": {n: torch.empty_like(grid["q"]) for n in ("o", "dq", "dk", "dv")},
        "mask": nabla.alloc_mask(shape, dev, cols=True),
        "ws_mask": nabla.workspace(shape, nabla.OP_BUILD_MASK, dev),
        "ws_fwd": nabla.workspace(shape, nabla.OP_ATTN_FWD, dev),
        "ws_bwd": nabla.workspace(shape, nabla.OP_ATTN_BWD, dev),
    }
    stream = torch.cuda.current_stream(dev)

    def step(src, ev=None, out=None):
        out = B["out"] if out is None else out
        nabla.flatten(src["v"], w.T, w.H, w.W, w.P, out=B["flat"]["v"])
        if ev: ev[1].record(stream)
        # Q and K are flattened by the mask build itself (pooling in the same pass)
        nabla.build_mask_grid(shape, prm, src["q"], src["k"], q=B["flat"]["q"], k=B["flat"]["k"],
                              mask=B["mask"], ws=B["ws_mask"])
        if ev: ev[2].record(stream)
        nabla.attn_fwd(shape, prm, B["flat"]["q"], B["flat"]["k"], B["flat"]["v"], B["mask"],
                       o=B["o"], lse=B["lse"], ws=B["ws_fwd"])
        if ev: ev[3].record(stream)
        nabla.attn_bwd(shape, prm, B["flat"]["q"], B["flat"]["k"], B["flat"]["v"], B["o"],
                       src["dout"], B["lse"], B["mask"], dq=B["dq"], dk=B["dk"], dv=B["dv"],
                       ws=B["ws_bwd"])
        if ev: ev[4].record(stream)
        for n in ("o", "dq", "dk", "dv"):
            nabla.flatten(B[n], w.T, w.H, w.W, w.P, inverse=True, out=out[n])

    # flatten v; the persistent front end (flatten + pool of Q, K with scores and
    # cut) and the column lists; fwd; pre, dK/dV, dQ; 4 unflattens
    launches_per_step = 1 + 2 + 1 + 3 + 4

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)


    for _ in range(args.warmup):
        step(grid)
    barrier()
    kept = int(B["mask"]["row_cnt"].sum().item())
    kept_all = sum_over_ranks(kept, world, dev)  # kept pairs of the whole problem
    kept_frac = kept_all / (w_job.BH * w.nb * w.nb)

    # ---- device-resident timed region
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for s in range(args.steps):
        evs[s][0].record(stream)
        step(grid, evs[s])
        evs[s][5].record(stream)
    stop.record(stream)
    barrier()
    clk = clocks.stop()
    total_ms = max_over_ranks(start.elapsed_time(stop), world, dev)
    phase = [0.0] * 5
    for s in range(args.steps):
        for p in range(5):
            phase[p] += evs[s][p].elapsed_time(evs[s][p + 1])
    phase = [x / args.steps for x in phase]
    ms_step = total_ms / args.steps

    fwd_flop = 4.0 * 64 * 64 * w.D * kept  # this rank's share
    bwd_flop = 10.0 * 64 * 64 * w.D * kept
    job_flop = 14.0 * 64 * 64 * w.D * kept_all
    value = whole_job_tflops(job_flop, ms_step)
    N, D, BH, nb = w.N, w.D, w.BH, w.nb
    # flatten of Q and K (read grid, write flattened) + pooled means (write + read)
    # + bit rows + row and column lists
    mask_bytes = (2 * 4.0 * N * D * BH + 16.0 * nb * D * BH + nb * nb * BH / 8.0
                  + 2 * 2.0 * kept + 2 * 4.0 * BH * nb)
    mask_gbs = mask_bytes / (phase[1] * 1e-3) / 1e9
    flat_gbs = 2.0 * BH * N * D * 2 / (phase[0] * 1e-3) / 1e9

    pk, pk_src = peaks()
    ops = {"attn_bwd": (phase[3], bwd_flop), "attn_fwd": (phase[2], fwd_flop)}
    dom = max(ops, key=lambda k: ops[k][0])
    achieved = ops[dom][1] / (ops[dom][0] * 1e-3) / 1e12
    peak = pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    traffic, traffic_note = None, "no ncu capture recorded for this kernel"
    cap = NCU_DRAM.get((args.workload, dom))
    if cap is not None and cap["bytes_per_head"] is not None:
        if cap["sources_sha"] == sources_sha(dom):
            traffic = cap["bytes_per_head"] * w.heads
            traffic_note = ("ncu capture of bench.py --heads 8 (kernel sources %s), scaled to %d "
                            "heads" % (cap["sources_sha"], w.heads))
        else:
            traffic_note = "stale: the kernel sources changed since the ncu capture"
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic, "traffic_note": traffic_note,
                "kernel": dom, "peak_source": "bf16 sustained (of %s)" % pk_src,
                "flop_per_launch": ops[dom][1], "ms_per_launch": ops[dom][0],
                "frac_of_burst": achieved / pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])}
    clk_peak = tensor_peak_at_clock(clk.get("sm_mhz"))
    if clk_peak:
        # the same work against the tensor pipes' own rate at this run's clock
        roofline["frac_at_clock"] = achieved / clk_peak
        roofline["peak_at_clock"] = clk_peak

    # ---- end to end through the C ABI with host buffers (pinned).  Every step
    # uploads its inputs from pinned host memory and downloads its results, all
    # inside the timed region.  As a training loop would, the step runs in
    # chunks of (batch, head) rows -- heads are independent -- so copies
    # overlap compute: the inputs of the next chunk upload on one copy stream
    # and the outputs of the previous chunk download on another while the
    # current chunk computes (chunk buffers double-buffered on the device).
    e2e = None
    if not args.no_e2e:
        host_in = {n: torch.empty(grid[n].shape, dtype=grid[n].dtype, pin_memory=True)
                   for n in ("q", "k", "v", "dout")}
        for n in host_in:
            host_in[n].copy_(grid[n])
        host_out = {n: torch.empty(grid["q"].shape, dtype=torch.bfloat16, pin_memory=True)
                    for n in ("o", "dq", "dk", "dv")}
        nch = max(c for c in range(1, 9) if w.BH % c == 0)  # chunks per step
        hc = w.BH // nch                                     # (batch, head) rows per chunk
        shape_c = nabla.shape_of(1, hc, w.T, w.H, w.W, w.D, w.P)
        rows = lambda t, c: t.view(w.BH, w.N, w.D)[c * hc:(c + 1) * hc]
        like = lambda t: torch.empty((hc, w.N, w.D), dtype=t.dtype, device=dev)
        C = {"flat": {n: like(grid[n]) for n in ("q", "k", "v")},
             "o": like(grid["q"]), "lse": torch.empty((hc, w.N), dtype=torch.float32, device=dev),
             "dq": like(grid["q"]), "dk": like(grid["q"]), "dv": like(grid["q"]),
             "mask": nabla.alloc_mask(shape_c, dev, cols=True),
             "ws_mask": nabla.workspace(shape_c, nabla.OP_BUILD_MASK, dev),
             "ws_fwd": nabla.workspace(shape_c, nabla.OP_ATTN_FWD, dev),
             "ws_bwd": nabla.workspace(shape_c, nabla.OP_ATTN_BWD, dev)}
        dev_in = [{n: like(grid[n]) for n in host_in} for _ in range(2)]
        dev_out = [{n: like(grid["q"]) for n in host_out} for _ in range(2)]
        h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()
        in_ready = [ev(), ev()]    # inputs of buffer b uploaded
        in_free = [ev(), ev()]     # chunk using input buffer b finished reading it
        out_ready = [ev(), ev()]   # outputs of buffer b written
        out_free = [ev(), ev()]    # outputs of buffer b downloaded

        def chunk_step(src, out):
            nabla.flatten(src["v"], w.T, w.H, w.W, w.P, out=C["flat"]["v"])
            nabla.build_mask_grid(shape_c, prm, src["q"], src["k"], q=C["flat"]["q"],
                                  k=C["flat"]["k"], mask=C["mask"], ws=C["ws_mask"])
            nabla.attn_fwd(shape_c, prm, C["flat"]["q"], C["flat"]["k"], C["flat"]["v"], C["mask"],
                           o=C["o"], lse=C["lse"], ws=C["ws_fwd"])
            nabla.attn_bwd(shape_c, prm, C["flat"]["q"], C["flat"]["k"], C["flat"]["v"], C["o"],
                           src["dout"], C["lse"], C["mask"], dq=C["dq"], dk=C["dk"], dv=C["dv"],
                           ws=C["ws_bwd"])
            for n in ("o", "dq", "dk", "dv"):
                nabla.flatten(C[n], w.T, w.H, w.W, w.P, inverse=True, out=out[n])

        def upload(u, first):
            b, c = u % 2, u % nch
            with torch.cuda.stream(h2d_s):
                if not first:
                    h2d_s.wait_event(in_free[b])
                for n in host_in:
                    dev_in[b][n].copy_(rows(host_in[n], c), non_blocking=True)
                in_ready[b].record(h2d_s)

        def download(u):
            b, c = u % 2, u % nch
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(out_ready[b])
                for n in host_out:
                    rows(host_out[n], c).copy_(dev_out[b][n], non_blocking=True)
                out_free[b].record(d2h_s)

        def run(nsteps):
            units = nsteps * nch
            upload(0, True)
            for u in range(units):
                b = u % 2
                if u + 1 < units:
                    upload(u + 1, u == 0)
                stream.wait_event(in_ready[b])
                if u >= 2:
                    stream.wait_event(out_free[b])
                chunk_step(dev_in[b], dev_out[b])
                in_free[b].record(stream)
                out_ready[b].record(stream)
                download(u)
            for cs in (h2d_s, d2h_s):
                done = ev()
                done.record(cs)
                stream.wait_event(done)

        run(max(2, args.warmup // 2))
        barrier()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        h2d_s.wait_event(a)
        d2h_s.wait_event(a)
        run(args.steps)
        b_.record(stream)
        barrier()
        e2e_ms = max_over_ranks(a.elapsed_time(b_), world, dev) / args.steps
        h2d = sum(t.numel() * t.element_size() for t in host_in.values())
        d2h = sum(t.numel() * t.element_size() for t in host_out.values())
        # the chunked calls must give the device-resident step's results, bit for bit
        same = all(torch.equal(host_out[n], B["out"][n].cpu()) for n in host_out)
        e2e = {"value": whole_job_tflops(job_flop, e2e_ms), "unit": "TFLOP/s",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d * world,
               "d2h_bytes_per_step": d2h * world, "outputs_match_device_step": same,
               "copies": "pinned host <-> device in %d chunks of %d (batch, head) rows per step, "
                         "uploads and downloads on two copy streams overlapped with the "
                         "neighbouring chunks' compute" % (nch, hc)}
        del dev_in, dev_out, C

    sweep, small_cfgs = None, None
    if rank == 0 and world == 1 and not args.no_sweep:
        B.clear()  # free this workload's buffers first
        torch.cuda.empty_cache()
        sweep = long_p_sweep(dev)
        small_cfgs = config_timings(dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        r = oracle_sample(w)
        cpu = {"value": r["flop_step"] / r["s_step"] / 1e12, "unit": "TFLOP/s",
               "cores": r["cores"], "kind": "oracle", "sample": r["desc"],
               "extrapolated_ms_per_step": 1e3 * r["s_step"]}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded cell-correlated bf16 Q/K/V (cell 2x8x8, noise 0.5), dO ~ "
                    "N(0,1), one seed per (batch, head)",
            "config": dict(workload_config(w_job),
                           parallelism="heads split over %d GPU(s), %d per GPU, no exchange"
                                       % (world, w.heads)),
            "breakdown_ms": {"flatten_v": phase[0], "flatten_qk_build_mask": phase[1],
                             "attn_fwd": phase[2], "attn_bwd": phase[3],
                             "unflatten_out": phase[4]},
            "kept_blocks": int(kept_all), "kept_fraction": kept_frac,
            "attn_fwd_tflops": fwd_flop / (phase[2] * 1e-3) / 1e12,
            "attn_bwd_tflops": bwd_flop / (phase[3] * 1e-3) / 1e12,
            "attn_fwd_frac_at_clock": (fwd_flop / (phase[2] * 1e-3) / 1e12 / clk_peak
                                       if clk_peak else None),
            "attn_bwd_frac_at_clock": (bwd_flop / (phase[3] * 1e-3) / 1e12 / clk_peak
                                       if clk_peak else None),
            "flatten_qk_build_mask_gbs": mask_gbs,
            "flatten_qk_build_mask_frac_hbm": mask_gbs / pk["hbm_gbs"],
            "flatten_v_gbs": flat_gbs,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
            "long_p_sweep": sweep, "small_configs": small_cfgs,
            "gpu_launches": launches_per_step * args.steps,
        }
        print(json.dumps(line), flush=True)
    B.clear()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_nabla(args)


if __name__ == "__main__":
    sys.exit(main())
