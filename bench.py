#!/usr/bin/env python3
"""Benchmark of the fused smooth-rotate-MXFP4 path on B200.

One step = one pass of the whole hot path over one batch: a single launch of
the fused kernel.  That launch loads X, applies the optional smoothing, the
32x32 rotation on the tensor cores, the absmax, the E8M0 scale, the E2M1
rounding and the packed stores.  The workload is the down-projection input,
8192 x 14336 bf16: Student-t(3) entries, 8 tokens carrying 1e3-1e4 outliers in
4 channels, a random orthogonal R̂, no smoothing.

Metric: GB/s of algorithmic traffic per step.  That is 2 B of bf16 read plus
0.5 B of codes and 1/32 B of scale written, per element: 2.53125 B/elem.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mine|reference]

With N > 1, launch it under torch.distributed.run, one rank per GPU.  Each rank
quantises its own batch of the same shape (weak scaling, no collective on the
data path).  The timing is the max over ranks.  ``--impl reference`` times the
CPU oracle on the host cores on a bounded sample of the same workload.
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
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import synth  # noqa: E402

CFG = 3
ROWS, COLS = synth.CONFIG_SHAPES[CFG]
BYTES_PER_ELEM = 2.0 + 0.5 + 1.0 / 32.0
METRIC = "rotate+MXFP4-quantize GB/s and % of HBM roofline, 1×B200, down-proj shape"
UNIT = "GB/s"
WORKLOAD = ("down-proj input 8192x14336 bf16 (Student-t(3), 8 tokens x 4 channels of 1e3-1e4 outliers), "
            "random orthogonal 32x32 R, no smoothing -> MXFP4 codes + E8M0 scales")
FALLBACK_HBM_GBS = 6650.0
_CSRC = "mxfp4_block_rotation_b200/csrc/"
_COMMON = [_CSRC + "pipeline_sm100.cuh", _CSRC + "sm100_ptx.cuh", _CSRC + "sm100_bulk.cuh",
           _CSRC + "mxq_internal.h"]
# The device code each timed kernel is built from: a DRAM-traffic record under profiles/ is
# reported only while the hash of these files matches the one it was taken with.
KERNEL_SOURCES = {
    "rotate_flat": [_CSRC + "rotate_flat_sm100.cu"] + _COMMON,
    "rotate_cols": [_CSRC + "rotate_cols_sm100.cu", _CSRC + "tile_order.cuh"] + _COMMON,
    "dequant_rot": [_CSRC + "dequant_sm100.cu"] + _COMMON,
}
# profiles/traffic_<row>.json: ncu's dram__bytes_read.sum + dram__bytes_write.sum of one launch
TRAFFIC_KERNEL = {
    "qkv_o_proj_input_8192x4096": "rotate_flat",
    "down_proj_input_8192x14336": "rotate_flat",
    "large_prefill_65536x8192_hadamard": "rotate_flat",
    "smoothing_32768x14336_quantize": "rotate_cols",
    "smoothing_32768x14336_dequantize_round_trip": "dequant_rot",
}


def algorithmic_bytes(rows: int, cols: int) -> float:
    return rows * cols * BYTES_PER_ELEM


def kernel_source_hash(kernel: str = "rotate_flat") -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def _bf16_peak_tflops() -> float:
    """Measured dense bf16 burst TFLOP/s (MEASURED_PEAKS.json), else the recipe's fallback 1590."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except (OSError, KeyError, ValueError):
        return 1590.0


def recorded_traffic(row: str = "down_proj_input_8192x14336"):
    """DRAM bytes per launch of a row's kernel from its committed ncu record, or None when there
    is no record or the kernel's source has changed since it was taken."""
    try:
        with open(os.path.join(ROOT, "profiles", f"traffic_{row}.json")) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("kernel_source_sha256") != kernel_source_hash(TRAFFIC_KERNEL[row]):
        return None
    return rec.get("dram_bytes_per_launch")


def max_over_ranks(values, dist=None, device=None):
    """Element-wise max of a list of floats over all ranks (identity without a process group)."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def weak_scaling_value(world: int, bytes_per_rank: float, ms_per_step: float) -> float:
    """Whole-job GB/s: every rank moves bytes_per_rank per step; the step time is the slowest rank's."""
    return world * bytes_per_rank / (ms_per_step * 1e-3) / 1e9


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sms, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sms.append(float(parts[1]))
                    maxes.append(float(parts[2]))
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        busy = [s for s in sms if s > 0.5 * max(sms)] or sms
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(maxes), "reasons": sorted(reasons),
                "samples": len(sms)}


# ----------------------------------------------------------------------------- CPU oracle leg

def oracle_rate(x_bits: np.ndarray, rhat_bits: np.ndarray, target_s: float, threads: int):
    """Time the oracle on a row sample sized for about target_s seconds (whole passes over the
    workload are repeated if one pass is shorter); returns (GB/s, elements processed, seconds)."""
    import oracle
    probe = min(x_bits.shape[0], max(8, threads * 2))
    t0 = time.perf_counter()
    oracle.smooth_rotate_quantize(x_bits[:probe], rhat_bits, None, threads=threads)
    dt = max(time.perf_counter() - t0, 1e-6)
    n = int(min(x_bits.shape[0], max(probe, probe * target_s / dt)))
    done, t0 = 0, time.perf_counter()
    while True:
        oracle.smooth_rotate_quantize(x_bits[:n], rhat_bits, None, threads=threads)
        done += n
        dt = time.perf_counter() - t0
        if dt >= 0.5 * target_s:
            break
    return algorithmic_bytes(done, x_bits.shape[1]) / dt / 1e9, done * x_bits.shape[1], dt


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    w = synth.make_config(CFG)
    xb = synth.bf16_bits(w.x)
    rb = synth.bf16_bits(w.rhat)
    threads = host_cores()
    per_step_s = max(0.05, min(args.cpu_seconds, 150.0 / max(1, args.steps + args.warmup)))
    probe = min(ROWS, max(8, threads * 2))
    t0 = time.perf_counter()
    oracle.smooth_rotate_quantize(xb[:probe], rb, None, threads=threads)
    n_rows = int(min(ROWS, max(probe, probe * per_step_s / max(time.perf_counter() - t0, 1e-6))))
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.smooth_rotate_quantize(xb[:n_rows], rb, None, threads=threads)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    value = algorithmic_bytes(n_rows, COLS) / sec / 1e9
    sample = f"first {n_rows} of {ROWS} rows of the workload per step ({n_rows * COLS} elements)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "rows": ROWS, "cols": COLS, "lambda": None},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU leg

def run_mine(args):
    import mxfp4_block_rotation_b200 as mxq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}; launch N>1 under torch.distributed.run")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    w = synth.make_config(CFG)
    rows, cols = w.rows, w.cols
    n_bytes = algorithmic_bytes(rows, cols)
    # two input/output sets alternated: each X (235 MB) already exceeds the 126 MB L2
    xs = [w.x.to(dev), w.x.to(dev)]
    rhat = w.rhat.to(dev)
    outs = [(torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev),
             torch.empty((rows, cols // 32), dtype=torch.uint8, device=dev)) for _ in range(2)]
    stream = torch.cuda.current_stream(dev)

    def step(i):
        c, s = outs[i & 1]
        mxq.smooth_rotate_quantize(xs[i & 1], rhat, None, codes=c, scales=s, stream=stream)

    # Timed region: K back-to-back launches on one stream, bracketed by two events (no
    # events between launches, so programmatic dependent launch can overlap each
    # launch's set-up with the previous one's tail).  The kernel's average launch
    # duration is therefore the region's time / K.  The clock sampler starts before the
    # warm-up, so the GPU does not sit idle between the warm-up and the timed region.
    k = args.steps
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        for i in range(args.warmup):
            step(i)
        torch.cuda.synchronize(dev)
        mxq.sync_check()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)
        t_begin.record(stream)
        h0 = time.perf_counter()
        for i in range(k):
            step(i)
        h1 = time.perf_counter()
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
    mxq.sync_check()
    host_us_per_call = (h1 - h0) / k * 1e6
    total_ms = max_over_ranks([t_begin.elapsed_time(t_end)], dist, dev)[0]
    kern_avg_ms = total_ms / k
    ms_per_step = total_ms / k
    value = weak_scaling_value(world, n_bytes, ms_per_step)

    # end to end through the public API: pinned host X -> device -> kernel -> codes/scales back to host
    e2e = None if args.no_e2e else run_e2e(mxq, w, rhat, dev, stream, args, dist)
    extras = None if (args.no_extras or world > 1) else run_extras(mxq, w, xs, rhat, outs, dev, stream,
                                                                    k=max(1, args.extras_steps))
    del xs, outs
    per_config = None if (args.no_configs or world > 1) else run_configs(mxq, dev, stream,
                                                                         k=max(1, args.extras_steps))

    if rank == 0:
        peak, peak_kind = hbm_peak()
        achieved = n_bytes / (kern_avg_ms * 1e-3) / 1e9
        traffic = recorded_traffic()
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": k, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "rows": rows, "cols": cols, "lambda": None,
                       "elements_per_gpu": rows * cols, "bytes_per_step_per_gpu": n_bytes,
                       "l2": "inputs larger than L2: two 235 MB X buffers alternated (L2 126 MB)",
                       "parallelism": f"dp{world} (independent row batches, no collective)"},
            "elements_per_s": world * rows * cols / (ms_per_step * 1e-3),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                         if peak_kind == "measured" else "fallback 6.65 TB/s",
                         "kernel": "rotate_flat_kernel<Quant> (no smoothing)", "kernel_ms": kern_avg_ms},
            "e2e": e2e,
            "gpu_launches": k,
            "host_submit_us_per_call": host_us_per_call,
            "clocks": clocks.summary(),
        }
        if per_config is not None:
            line["per_config"] = per_config
        if extras is not None:
            line["other_rows"] = extras
        if world == 1 and not args.no_cpu_baseline:
            import oracle
            oracle.build()
            threads = host_cores()
            gbs, n_el, sec = oracle_rate(synth.bf16_bits(w.x), synth.bf16_bits(w.rhat), args.cpu_seconds,
                                         threads)
            # the same at one thread (a fifth of the time budget), for the per-core rate
            gbs1, n_el1, sec1 = oracle_rate(synth.bf16_bits(w.x), synth.bf16_bits(w.rhat),
                                            max(1.0, args.cpu_seconds / 5), 1)
            line["cpu_baseline"] = {"value": gbs, "unit": UNIT, "cores": threads, "kind": "oracle",
                                    "elements_per_s": n_el / sec,
                                    "sample": f"{n_el} elements (leading rows of the workload, whole "
                                              f"passes repeated) in {sec:.1f} s of oracle time",
                                    "one_thread": {"value": gbs1, "unit": UNIT, "elements_per_s": n_el1 / sec1,
                                                   "sample": f"{n_el1} elements in {sec1:.1f} s"}}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def _timed(fn, k, stream, dev):
    for i in range(5):
        fn(i)
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(k):
        fn(i)
    b.record(stream)
    torch.cuda.synchronize(dev)
    return a.elapsed_time(b) / k


def run_extras(mxq, w, xs, rhat, outs, dev, stream, k=300):
    """The other rows of the path on the same workload, each timed back to back."""
    rows, cols = w.rows, w.cols
    peak, _ = hbm_peak()
    lam = synth.smoothing_scale(w.x).to(dev)   # the smoothing recipe: clip(max|X_j|^0.5, 1e-2, 1e2)
    res = {}

    def row(name, ms, nbytes, what):
        gbs = nbytes / (ms * 1e-3) / 1e9
        res[name] = {"what": what, "ms": ms, "GB/s": gbs, "frac_of_hbm_peak": gbs / peak,
                     "bytes_per_launch": nbytes}

    def quant_lam(i):
        c, s = outs[i & 1]
        mxq.smooth_rotate_quantize(xs[i & 1], rhat, lam, codes=c, scales=s, stream=stream)
    row("smooth_rotate_quantize_with_lambda", _timed(quant_lam, k, stream, dev),
        algorithmic_bytes(rows, cols) + 4 * cols,
        "same X, Lambda_j = clip(max_t|X_tj|^0.5, 1e-2, 1e2) (rotate_cols_kernel)")
    deq = [torch.empty((rows, cols), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    deq_bytes = rows * cols * (0.5 + 1.0 / 32.0 + 2.0)

    def dq_plain(i):
        c, s = outs[i & 1]
        mxq.dequantize(c, s, out=deq[i & 1], stream=stream)
    row("dequantize", _timed(dq_plain, k, stream, dev), deq_bytes, "codes + scales -> bf16 (rotated domain)")

    def dq_rot(i):
        c, s = outs[i & 1]
        mxq.dequantize(c, s, rhat, out=deq[i & 1], stream=stream)
    row("dequantize_inverse_rotation", _timed(dq_rot, k, stream, dev), deq_bytes, "codes + scales -> v * R^T -> bf16")

    def dq_inv(i):
        c, s = outs[i & 1]
        mxq.dequantize(c, s, rhat, lam, out=deq[i & 1], stream=stream)
    row("dequantize_inverse_rotation_and_smoothing", _timed(dq_inv, k, stream, dev), deq_bytes + 4 * cols,
        "codes + scales -> (v * R^T) * Lambda -> bf16")
    errs = torch.empty((rows, cols // 32), dtype=torch.float32, device=dev)
    mean = torch.empty((), dtype=torch.float64, device=dev)
    for lam_q in (None, lam):
        ws = torch.empty(mxq.lib().mxq_quant_error_workspace_bytes(rows, cols, int(lam_q is not None)),
                         dtype=torch.uint8, device=dev)

        def qerr(i, lam_q=lam_q, ws=ws):
            import ctypes
            st = mxq.lib().mxq_quant_error(ctypes.c_void_p(xs[i & 1].data_ptr()), rows, cols,
                                           ctypes.c_void_p(rhat.data_ptr()),
                                           None if lam_q is None else ctypes.c_void_p(lam_q.data_ptr()),
                                           ctypes.c_void_p(errs.data_ptr()), ctypes.c_void_p(mean.data_ptr()),
                                           ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                                           ctypes.c_void_p(stream.cuda_stream))
            assert st == 0
        lam_bytes = 0.0 if lam_q is None else 4.0 * cols
        row("quant_error_per_group_and_mean" + ("" if lam_q is None else "_with_lambda"),
            _timed(qerr, k, stream, dev), rows * cols * 2.0 + rows * (cols // 32) * 4.0 + lam_bytes,
            "per-group ||Q(y)-y||/||y|| (fp32 out) and its mean: reads X, writes 4 B per group" +
            ("" if lam_q is None else "; y = X Lambda^-1 R (rotate_cols_kernel<Err>)"))
    # the rotation-block-size variants on the same X (no smoothing): B = 16, 64, 128
    for blk in (16, 64, 128):
        rblk = synth.rhat_tensor(synth.haar_orthogonal(300 + blk, n=blk)).to(dev)

        def quant_blk(i, rblk=rblk):
            c, s = outs[i & 1]
            mxq.rotate_quantize_block(xs[i & 1], rblk, codes=c, scales=s, stream=stream)
        row(f"rotate_quantize_block{blk}", _timed(quant_blk, k, stream, dev), algorithmic_bytes(rows, cols),
            f"rotation blocks of {blk} columns, MXFP4 groups of 32 "
            f"({'rotate_flat_kernel with diag(R16, R16)' if blk == 16 else 'rotate_block_kernel'})")
    # the NVFP4 variant (16-value blocks, E4M3 block scales, an fp32 tensor scale on the device)
    nv_scales = [torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev) for _ in range(2)]
    s_t = torch.tensor([float(w.x.abs().max().float()) * 32 ** 0.5 / (6 * 448)], dtype=torch.float32, device=dev)
    nv_bytes = rows * cols * (2.0 + 0.5 + 1.0 / 16.0) + 32 * 32 * 2 + 4
    for name, lam_nv, kern in (("nvfp4_rotate_quantize", None, "rotate_flat_kernel"),
                               ("nvfp4_rotate_quantize_with_lambda", lam, "rotate_cols_kernel")):
        def quant_nv(i, lam_nv=lam_nv):
            mxq.smooth_rotate_quantize_nvfp4(xs[i & 1], rhat, s_t, lam_nv, codes=outs[i & 1][0],
                                             scales=nv_scales[i & 1], stream=stream)
        row(name, _timed(quant_nv, k, stream, dev), nv_bytes + (4 * cols if lam_nv is not None else 0),
            f"NVFP4: blocks of 16, E4M3 scales [rows, cols/16], fp32 tensor scale ({kern})")
    del nv_scales
    # the consumer GEMM of the down-projection: MXFP4(X R) [8192 x 14336] times the absorbed weight
    # MXFP4(W^T R) [4096 x 14336] (synthetic N(0, 1/K) weight), bf16 out, on the block-scaled tensor cores
    n_out = 4096
    wt = synth.random_bf16(n_out, cols, seed=77, scale=1.0 / cols ** 0.5).to(dev)
    cb, sb = mxq.weight_rotate_quantize(wt, rhat, None, stream=stream)
    ca, sa = outs[0]
    sfa = mxq.scales_to_mma_layout(sa, stream=stream)
    sfb = mxq.scales_to_mma_layout(sb, stream=stream)
    y = torch.empty((rows, n_out), dtype=torch.bfloat16, device=dev)
    flops = 2.0 * rows * n_out * cols
    fp4_peak = _bf16_peak_tflops() * 4.0

    def gemm(i):
        mxq.mxfp4_gemm(ca, sfa, cb, sfb, out=y, stream=stream)
    ms = _timed(gemm, max(1, min(50, k)), stream, dev)
    res["mxfp4_gemm_downproj"] = {
        "what": f"Y[{rows}x{n_out}] = MXFP4(X R) MXFP4(W^T R)^T, K = {cols}, bf16 out (mxfp4_gemm_kernel)",
        "ms": ms, "TFLOP/s": flops / (ms * 1e-3) / 1e12, "peak_TFLOP/s": fp4_peak,
        "frac_of_fp4_peak": flops / (ms * 1e-3) / 1e12 / fp4_peak,
        "peak_source": "measured bf16 burst (MEASURED_PEAKS.json bf16_tflops) x 4, the nominal fp4/bf16 ratio"}

    # the NVFP4 consumer GEMM on the same shape: operands quantised by the NVFP4 path (tensor
    # scales from the bound amax <= sqrt(32) max|x|), E4M3 scales per 16 k
    ts_a = torch.tensor([float(w.x.abs().max().float()) * 32 ** 0.5 / (6 * 448)], dtype=torch.float32, device=dev)
    ts_b = torch.tensor([float(wt.abs().max().float()) * 32 ** 0.5 / (6 * 448)], dtype=torch.float32, device=dev)
    nca, nsa = mxq.smooth_rotate_quantize_nvfp4(xs[0], rhat, ts_a, stream=stream)
    ncb, nsb = mxq.smooth_rotate_quantize_nvfp4(wt, rhat, ts_b, stream=stream)
    nsfa = mxq.nvfp4_scales_to_mma_layout(nsa, stream=stream)
    nsfb = mxq.nvfp4_scales_to_mma_layout(nsb, stream=stream)

    def gemm_nv(i):
        mxq.nvfp4_gemm(nca, nsfa, ts_a, ncb, nsfb, ts_b, out=y, stream=stream)
    ms = _timed(gemm_nv, max(1, min(50, k)), stream, dev)
    res["nvfp4_gemm_downproj"] = {
        "what": f"Y[{rows}x{n_out}] = NVFP4(X R) NVFP4(W^T R)^T, K = {cols}, bf16 out (mxfp4_gemm_kernel<NVFP4>)",
        "ms": ms, "TFLOP/s": flops / (ms * 1e-3) / 1e12, "peak_TFLOP/s": fp4_peak,
        "frac_of_fp4_peak": flops / (ms * 1e-3) / 1e12 / fp4_peak,
        "peak_source": "measured bf16 burst (MEASURED_PEAKS.json bf16_tflops) x 4, the nominal fp4/bf16 ratio"}
    # the NVFP4 layer: quantise X (tensor scale on the device), lay out its scales, GEMM; and with
    # the quantiser writing its E4M3 scales straight into the MMA layout
    nv_codes = [torch.empty_like(nca) for _ in range(2)]
    nv_rows = [torch.empty_like(nsa) for _ in range(2)]
    nv_sf = [torch.empty_like(nsfa) for _ in range(2)]

    def layer_nv(i):
        mxq.smooth_rotate_quantize_nvfp4(xs[i & 1], rhat, ts_a, codes=nv_codes[i & 1], scales=nv_rows[i & 1],
                                         stream=stream)
        mxq.nvfp4_scales_to_mma_layout(nv_rows[i & 1], out=nv_sf[i & 1], stream=stream)
        mxq.nvfp4_gemm(nv_codes[i & 1], nv_sf[i & 1], ts_a, ncb, nsfb, ts_b, out=y, stream=stream)
    ms = _timed(layer_nv, max(1, min(50, k)), stream, dev)
    res["nvfp4_layer_quantize_plus_gemm"] = {
        "what": "the NVFP4 layer: rotate+quantise X, scale layout, NVFP4 GEMM (3 launches)", "ms": ms,
        "TFLOP/s": flops / (ms * 1e-3) / 1e12}

    def layer_nv_fused(i):
        mxq.smooth_rotate_quantize_nvfp4_mma(xs[i & 1], rhat, ts_a, codes=nv_codes[i & 1], sf=nv_sf[i & 1],
                                             stream=stream)
        mxq.nvfp4_gemm(nv_codes[i & 1], nv_sf[i & 1], ts_a, ncb, nsfb, ts_b, out=y, stream=stream)
    ms = _timed(layer_nv_fused, max(1, min(50, k)), stream, dev)
    res["nvfp4_layer_fused_scales_plus_gemm"] = {
        "what": "the NVFP4 layer with the quantiser writing MMA-layout E4M3 scales, then the GEMM (2 launches)",
        "ms": ms, "TFLOP/s": flops / (ms * 1e-3) / 1e12}
    del nca, nsa, ncb, nsb, nsfa, nsfb, nv_codes, nv_rows, nv_sf

    def layer(i):
        c, s = outs[i & 1]
        mxq.smooth_rotate_quantize(xs[i & 1], rhat, None, codes=c, scales=s, stream=stream)
        mxq.scales_to_mma_layout(s, out=sfa, stream=stream)
        mxq.mxfp4_gemm(c, sfa, cb, sfb, out=y, stream=stream)
    ms = _timed(layer, max(1, min(50, k)), stream, dev)
    res["downproj_layer_quantize_plus_gemm"] = {
        "what": "the whole layer: rotate+quantise X, scale layout, MXFP4 GEMM (3 launches)", "ms": ms,
        "TFLOP/s": flops / (ms * 1e-3) / 1e12}
    # the same layer with the quantiser writing its scales in the MMA layout (2 launches)
    sfa2 = [torch.empty_like(sfa) for _ in range(2)]

    def layer_fused(i):
        c = outs[i & 1][0]
        mxq.smooth_rotate_quantize_mma(xs[i & 1], rhat, None, codes=c, sf=sfa2[i & 1], stream=stream)
        mxq.mxfp4_gemm(c, sfa2[i & 1], cb, sfb, out=y, stream=stream)
    ms = _timed(layer_fused, max(1, min(50, k)), stream, dev)
    res["downproj_layer_fused_scales_plus_gemm"] = {
        "what": "the whole layer with the quantiser writing MMA-layout scales, then the MXFP4 GEMM (2 launches)",
        "ms": ms, "TFLOP/s": flops / (ms * 1e-3) / 1e12}
    del wt, cb, sb, sfa, sfb, y, sfa2
    # the offline rotation search on the same activations, smoothed: K = 128 steps, 64 angles per pair
    sws = torch.empty(mxq.lib().mxq_rotation_search_workspace_bytes(rows, cols, 32), dtype=torch.uint8, device=dev)
    found = {}

    def search(i):
        found["out"] = mxq.rotation_search(xs[i & 1], lam, max_steps=128, n_angle=32, workspace=sws, stream=stream)
    ms = _timed(search, max(1, min(10, k)), stream, dev)
    res["rotation_search_K128"] = {
        "what": "greedy Givens search for R^ on X / Lambda (worst group by column maxima, 128 steps, 64 angles)",
        "ms": ms, "steps": int(found["out"]["steps"]), "launches": 2 * 128 + 6,
        "bound": "latency: two dependent launches per step"}
    # §4.1 / Figure 1 on the synthetic activations: the mean per-group MXFP4 error under the identity,
    # a random-sign Hadamard, a random orthogonal R and the searched R (on X / Lambda: the searched
    # R's own target) -- the write-up's comparison, on the down-proj and QKV-input shapes
    fig1 = {}
    qkv = synth.make_config(2)
    for name, xw in (("down_proj", xs[0]), ("qkv_input", qkv.x.to(dev))):
        lam_w = synth.smoothing_scale(w.x if name == "down_proj" else qkv.x).to(dev)
        mats = {"identity": synth.rhat_tensor(np.eye(32)).to(dev),
                "hadamard_random_signs": synth.rhat_tensor(synth.hadamard_rhat(5)).to(dev),
                "random_orthogonal": synth.rhat_tensor(synth.haar_orthogonal(6)).to(dev)}
        fig1[name] = {}
        for key, lam_k in (("no_smoothing", None), ("smoothed", lam_w)):
            # the searched R is found on the very input it rotates (X, or X / Lambda)
            mats["searched_K128"] = mxq.rotation_search(xw, lam_k, max_steps=128, n_angle=32, stream=stream)["rhat"]
            fig1[name][key] = {}
            for rn, rm in mats.items():
                _, mean = mxq.quant_error(xw, rm, lam_k, per_group=False, stream=stream)
                fig1[name][key][rn] = float(mean.item())
        del xw
    res["figure1_mean_group_error"] = {
        "what": "mean over groups of ||Q(y) - y|| / ||y|| (MXFP4), y = X Lambda^-1 R; the searched R is found "
                "on the same X (or X / Lambda), K = 128, 64 angles", **fig1}
    mxq.sync_check()
    return res


L2_BYTES = 126 * 2 ** 20


def _sets_for(set_bytes: float) -> int:
    """Input/output sets to rotate so that a launch never finds its buffers in L2: the sets
    together hold at least three times the L2 capacity (at least two sets)."""
    return max(2, -(-int(3 * L2_BYTES) // int(set_bytes)))


# The workloads of the write-up's layer inputs (§4.1 / Figure 1: QKV-in, O-in and Down-in), each
# timed as its own row: (config, what the launch does, kernel)
CONFIG_ROWS = {
    "qkv_o_proj_input_8192x4096": (2, "quantize", "rotate_flat_kernel<Quant>"),
    "down_proj_input_8192x14336": (3, "quantize", "rotate_flat_kernel<Quant>"),
    "large_prefill_65536x8192_hadamard": (4, "quantize", "rotate_flat_kernel<Quant>"),
    "smoothing_32768x14336_quantize": (5, "quantize", "rotate_cols_kernel<Quant>"),
    "smoothing_32768x14336_dequantize_round_trip": (5, "dequantize", "dequant_rot_kernel<2>"),
}


def _config_row(mxq, name, w, dev, stream, k, codes_scales=None):
    """One CONFIG_ROWS row, K back-to-back launches on rotating sets; returns (row, codes, scales)."""
    cfg, what, kern = CONFIG_ROWS[name]
    rows, cols = w.rows, w.cols
    peak, _ = hbm_peak()
    rhat = w.rhat.to(dev)
    lam = None if w.lam is None else w.lam.to(dev)
    lam_bytes = 0 if lam is None else 4 * cols
    if what == "quantize":
        n_bytes = algorithmic_bytes(rows, cols) + lam_bytes
        n_sets = _sets_for(n_bytes)
        x0 = w.x.to(dev)
        xs = [x0] + [x0.clone() for _ in range(n_sets - 1)]
        outs = [(torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev),
                 torch.empty((rows, cols // 32), dtype=torch.uint8, device=dev)) for _ in range(n_sets)]

        def fn(i):
            c, s = outs[i % n_sets]
            mxq.smooth_rotate_quantize(xs[i % n_sets], rhat, lam, codes=c, scales=s, stream=stream)
        keep = outs[0]
    else:
        c0, s0 = codes_scales
        n_bytes = rows * cols * (0.5 + 1.0 / 32.0 + 2.0) + lam_bytes
        n_sets = _sets_for(n_bytes)
        ins = [(c0, s0)] + [(c0.clone(), s0.clone()) for _ in range(n_sets - 1)]
        outs = [torch.empty((rows, cols), dtype=torch.bfloat16, device=dev) for _ in range(n_sets)]

        def fn(i):
            c, s = ins[i % n_sets]
            mxq.dequantize(c, s, rhat, lam, out=outs[i % n_sets], stream=stream)
        keep = None
    ms = _timed(fn, k, stream, dev)
    mxq.sync_check()
    gbs = n_bytes / (ms * 1e-3) / 1e9
    row = {"config": cfg, "shape": [rows, cols], "what": what, "kernel": kern, "ms": ms, "GB/s": gbs,
           "frac_of_hbm_peak": gbs / peak, "elements_per_s": rows * cols / (ms * 1e-3),
           "bytes_per_launch": n_bytes, "traffic": recorded_traffic(name), "lambda": lam is not None,
           "launches": k,
           "l2": f"{n_sets} input/output sets rotated ({n_bytes / 1e6:.0f} MB each; L2 126 MB)"}
    return row, keep


def run_configs(mxq, dev, stream, k=300):
    """Every workload's own row (CONFIG_ROWS), each against the HBM roofline."""
    res = {}
    for cfg in (2, 3, 4, 5):
        w = synth.make_config(cfg)
        keep = None
        for name, (c, what, _) in CONFIG_ROWS.items():
            if c != cfg:
                continue
            res[name], got = _config_row(mxq, name, w, dev, stream, k, keep)
            keep = got if got is not None else keep
        del w, keep
        torch.cuda.empty_cache()
    return res


def run_row_only(args):
    """Profiling aid: one CONFIG_ROWS row alone, --warmup + --steps launches, then its time."""
    import mxfp4_block_rotation_b200 as mxq
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream(dev)
    cfg, what, _ = CONFIG_ROWS[args.row]
    w = synth.make_config(cfg, rows=args.row_rows)   # the row's recipe, optionally cut to fewer rows
    keep = None
    if what == "dequantize":
        keep = mxq.smooth_rotate_quantize(w.x.to(dev), w.rhat.to(dev), None if w.lam is None else w.lam.to(dev),
                                          stream=stream)
    row, _ = _config_row(mxq, args.row, w, dev, stream, max(1, args.steps), keep)
    print(json.dumps({args.row: row}), flush=True)
    return 0


def run_e2e(mxq, w, rhat, dev, stream, args, dist):
    rows, cols = w.rows, w.cols
    x_host = w.x.pin_memory()
    c_host = torch.empty((rows, cols // 2), dtype=torch.uint8).pin_memory()
    s_host = torch.empty((rows, cols // 32), dtype=torch.uint8).pin_memory()
    x_dev = torch.empty_like(x_host, device=dev)
    c_dev = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    s_dev = torch.empty((rows, cols // 32), dtype=torch.uint8, device=dev)

    # A step moves the whole batch: host -> device, quantise, codes and scales -> host.  The rows
    # are independent, so the batch goes in row chunks over three streams and the copies in both
    # directions overlap each other and the kernels (PCIe is full duplex).  Steps do not overlap:
    # each starts after the previous one's results are on the host.
    n_chunks = 8
    bounds = [(i * rows // n_chunks, (i + 1) * rows // n_chunks) for i in range(n_chunks)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def step():
        s_in.wait_stream(stream)
        for lo, hi in bounds:
            with torch.cuda.stream(s_in):
                x_dev[lo:hi].copy_(x_host[lo:hi], non_blocking=True)
            stream.wait_stream(s_in)
            mxq.smooth_rotate_quantize(x_dev[lo:hi], rhat, None, codes=c_dev[lo:hi], scales=s_dev[lo:hi],
                                       stream=stream)
            s_out.wait_stream(stream)
            with torch.cuda.stream(s_out):
                c_host[lo:hi].copy_(c_dev[lo:hi], non_blocking=True)
                s_host[lo:hi].copy_(s_dev[lo:hi], non_blocking=True)
        stream.wait_stream(s_out)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    k = max(3, min(50, args.steps // 2))
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    a.record(stream)
    for _ in range(k):
        step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks([a.elapsed_time(b) / k], dist, dev)[0]
    world = dist.get_world_size() if dist is not None else 1
    return {"value": weak_scaling_value(world, algorithmic_bytes(rows, cols), ms), "unit": UNIT,
            "h2d_bytes_per_step": x_host.numel() * 2,
            "d2h_bytes_per_step": c_host.numel() + s_host.numel(), "ms_per_step": ms, "steps": k,
            "pipeline": f"{n_chunks} row chunks over three streams (H2D, kernel, D2H)"}


def run_gemm_only(args):
    """The consumer GEMM alone at a chosen shape (small cases for ncu captures): MXFP4, or NVFP4
    with --gemm-nvfp4 (E4M3 block scales in [0x30, 0x40), tensor scales 0.5 and 0.25)."""
    import mxfp4_block_rotation_b200 as mxq
    M, N, K = (int(v) for v in args.gemm_only.split(","))
    dev = torch.device("cuda:0")
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    a = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev, generator=g)
    b = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=g)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    if args.gemm_nvfp4:
        sfa = mxq.nvfp4_scales_to_mma_layout(
            torch.randint(0x30, 0x40, (M, K // 16), dtype=torch.uint8, device=dev, generator=g))
        sfb = mxq.nvfp4_scales_to_mma_layout(
            torch.randint(0x30, 0x40, (N, K // 16), dtype=torch.uint8, device=dev, generator=g))
        ta = torch.tensor([0.5], device=dev)
        tb = torch.tensor([0.25], device=dev)

        def gemm():
            mxq.nvfp4_gemm(a, sfa, ta, b, sfb, tb, out=y)
    else:
        sfa = mxq.scales_to_mma_layout(
            torch.randint(120, 134, (M, K // 32), dtype=torch.uint8, device=dev, generator=g))
        sfb = mxq.scales_to_mma_layout(
            torch.randint(120, 134, (N, K // 32), dtype=torch.uint8, device=dev, generator=g))

        def gemm():
            mxq.mxfp4_gemm(a, sfa, b, sfb, out=y)
    for _ in range(3):
        gemm()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        gemm()
    e1.record()
    torch.cuda.synchronize(dev)
    mxq.sync_check()
    ms = e0.elapsed_time(e1) / max(args.steps, 1)
    print(json.dumps({"gemm": [M, N, K], "format": "nvfp4" if args.gemm_nvfp4 else "mxfp4", "ms": ms,
                      "TFLOP/s": 2.0 * M * N * K / (ms * 1e-3) / 1e12}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["mine", "reference"], default="mine")
    ap.add_argument("--cpu-seconds", type=float, default=8.0,
                    help="oracle seconds: the cpu_baseline sample (rank 0, N=1) and each --impl reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg (profiling runs)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip other_rows: the other rows of the path, the GEMMs, the search and the error comparison")
    ap.add_argument("--extras-steps", type=int, default=300,
                    help="timed launches per extra row (the search row times min(10, this) runs)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip per_config: the other workloads' rows (QKV/O-proj, large prefill, smoothing)")
    ap.add_argument("--row", choices=sorted(CONFIG_ROWS),
                    help="profiling aid: run only this per_config row, --steps launches after 5 warm-up "
                         "launches, print its time and exit")
    ap.add_argument("--row-rows", type=int, default=None,
                    help="with --row: the same recipe with this many rows (smaller cases for full ncu captures)")
    ap.add_argument("--gemm-only", metavar="M,N,K",
                    help="profiling aid: run only the MXFP4 GEMM, 3 + --steps launches on random operands of this "
                         "shape (bf16 out), print its time and exit")
    ap.add_argument("--gemm-nvfp4", action="store_true", help="with --gemm-only: the NVFP4 GEMM instead")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.gemm_only:
        return run_gemm_only(args)
    if args.row:
        return run_row_only(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_mine(args)


if __name__ == "__main__":
    sys.exit(main())
