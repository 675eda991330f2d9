#!/usr/bin/env python
"""Benchmark of the block-scaled weight quantization hot path on B200.

One step = the whole path over one batch of synthetic input:
  1. h pass        h_j = E_r[x_rj^2] over X [R, K] (bf16)        -- mxq_act_sqmean
  2. search        NVFP4 (E2M1) block 16, H-optimal over all 126 E4M3 scales
                   on W [N, K] (bf16), codes + scales            -- mxq_quantize
  3. metrics       weight error and h-weighted error sums         -- mxq_error
Default workload: the "full calibration" shape of the qwantize results page
(W 2560x9728, X 244449x9728, both bf16), synthetic data.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
With N > 1 (launched by torch.distributed.run, one rank per GPU) every rank owns its own
X and W of that shape (weak scaling); the h pass becomes per-rank column sums, one NCCL
all-gather of those sums and a fixed-order finalize, so every rank quantizes with the
global h. ``--impl reference`` times the CPU oracle (bounded sample) instead.
Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import collections
import dataclasses
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "G weights/s quantized (H-opt NVFP4 blk16) + h-pass GB/s; % of roofline"
UNIT = "G weights/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
# Plain-ALU peak of the search kernel: 148 SMs x 4 sub-partitions x 32 FP32 lanes x
# 1965 MHz (max SM clock) = lane-operations per second, an FMA counted as one operation.
ALU_PEAK_TOPS = 148 * 128 * 1.965e9 / 1e12
# Oracle samples, in weight rows of the first weight (with the matching share of activation
# rows): the cpu_baseline leg (about 10-30 s of CPU work) and each step of the reference arm
# (a fraction of a second, so that a long --steps run stays short).
CPU_W_ROWS = 1024
GPTQ_CPU_X_ROWS, GPTQ_CPU_W_ROWS = 4096, 16
Quantizer = collections.namedtuple("Quantizer", "fmt block mode window sfmt")
HEADLINE_Q = Quantizer("nvfp4", 16, "hopt", -1, "e4m3")
REF_X_ROWS, REF_W_ROWS = 2048, 64


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="mxq", choices=["mxq", "reference"])
    ap.add_argument("--workload", default="nvfp4_full_calib")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--block", type=int, default=0, help="block size (default: the workload's)")
    ap.add_argument("--mode", default="",
                    choices=["", "naive", "sse", "hopt", "bhopt", "gptq", "gptq-ord"],
                    help="bhopt: the block-Hessian objective d^T G_b d (Gram pass on the "
                         "tensor cores instead of the h pass); gptq: GPTQ with the H-optimal "
                         "quantizer as its inner step (NVFP4 / INT4: full Hessian; E4M3: "
                         "64 x 64 tiles); gptq-ord: ordered GPTQ (NVFP4 / INT4)")
    ap.add_argument("--fmt", default="", choices=["", "nvfp4", "int4", "int8", "e4m3"],
                    help="element format (default: the workload's)")
    ap.add_argument("--scale-fmt", default="", choices=["", "e4m3", "ue4m4", "ue5m3", "ue8m0"],
                    help="block-scale grid of nvfp4 / int4 elements (ue8m0 = MXFP4)")
    ap.add_argument("--x-rows", type=int, default=0,
                    help="use only this many activation rows (profiling captures)")
    ap.add_argument("--serial", action="store_true",
                    help="time the steps back to back on one stream (no overlap of a step's "
                         "search with the next step's h pass)")
    return ap.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def measured_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def executed_for(kernel):
    """Executed thread instructions per launch (and active lanes per warp instruction) from a
    committed ncu capture, if the kernel source is unchanged."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)[kernel]
        src = os.path.join(ROOT, rec["source"])
        if source_sha(src) != rec["source_sha"] or "thread_inst_per_launch" not in rec:
            return None
        return {"thread_inst": rec["thread_inst_per_launch"], "lanes": rec.get("lanes_per_inst"),
                "candidates_per_block": rec.get("candidates_per_block")}
    except Exception:
        return None


def traffic_for(kernel):
    """DRAM bytes per launch from a committed ncu capture, if the kernel source is unchanged."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)[kernel]
        src = os.path.join(ROOT, rec["source"])
        if source_sha(src) != rec["source_sha"]:
            return None
        return rec["dram_bytes_per_launch"]
    except Exception:
        return None


class ClockSampler:
    """Polls NVML (SM clock, max clock, throttle reasons) every 10 ms while active."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception as e:  # NVML unavailable: report no clocks
            self.error = repr(e)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        self._stop.clear()                    # re-entrant: samples accumulate across regions
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._ok:
            self._t.join()

    def summary(self):
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def quant_name(q):
    """Short name of a quantizer: the element format, or MXFP4 / NVINT4 / E2M1-on-UE4M4 ..."""
    if q.fmt == "nvfp4":
        return {"e4m3": "nvfp4", "ue8m0": "mxfp4"}.get(q.sfmt, f"e2m1-{q.sfmt}")
    if q.fmt == "int4":
        return "nvint4" if q.sfmt == "e4m3" else f"int4-{q.sfmt}"
    return q.fmt


def workload_desc(wl, q, x_rows=None):
    """One-line description of what a step computes (both arms print the same)."""
    fmt, block, mode, window = q.fmt, q.block, q.mode, q.window
    x_rows = x_rows or [r for r, _ in wl.x_shapes]
    dt = "bf16" if wl.w_dtype == torch.bfloat16 else "f32"
    shapes = ", ".join(f"{nm} {n}x{k}" for nm, n, k in wl.weights)
    xsh = ", ".join(f"{r}x{k}" for r, (_, k) in zip(x_rows, wl.x_shapes))
    sg = q.sfmt.upper()
    ncand = {"e4m3": 126, "ue4m4": 255, "ue5m3": 255, "ue8m0": 255}[q.sfmt]
    grid = ("64-point log grid" if fmt == "e4m3" else
            f"all {ncand} {sg} scales" if window < 0 else f"{sg} scales within +-{window} codes")
    if full_gptq(q):
        kind = "ordered" if mode == "gptq-ord" else "sequential"
        return (f"{wl.name}: W {shapes} {dt}; X {xsh} {dt}; {quant_name(q)} block {block}, "
                f"{kind} GPTQ over the full input dimension: h = mean of X^2, H = X^T X / R, "
                f"float64 factor of (H + lambda I)^-1 (damp {GPTQ_DAMP}), sweep with the hopt "
                f"block search on the {grid}; then weight/h-weighted error sums")
    if mode == "gptq":
        return (f"{wl.name}: W {shapes} {dt}; X {xsh} {dt}; e4m3 64x64 tiles: Gram blocks of X "
                f"(h = their diagonal), GPTQ factors (damp {GPTQ_DAMP}), tile scales by the "
                f"hopt search on the {grid}, GPTQ sweep; then weight/h-weighted error sums")
    return (f"{wl.name}: W {shapes} {dt}; X {xsh} {dt}; {quant_name(q)} block {block}, {mode}, "
            f"{grid}; then weight/h-weighted error sums")


# ---------------------------------------------------------------------------------------
# oracle (CPU) timing: the cpu_baseline leg and the reference arm
# ---------------------------------------------------------------------------------------

def oracle_step_sample(X_bits, W_bits, h_np, n_threads, R_full, N_full, q):
    """Time the oracle on a bounded sample (X_bits: the first rows of X, W_bits: the first
    rows of W, bf16 bits; q the quantizer) and scale each part to the full
    workload (R_full rows of X, N_full rows of W, in units of the sample's row widths).
    Returns (seconds for a full step, measured seconds per part)."""
    import numpy as np
    from oracle import oracle as orc
    fmt, block, mode, window = q.fmt, q.block, q.mode, q.window
    x_rows, K = X_bits.shape
    w_rows = W_bits.shape[0]
    if full_gptq(q):
        t0 = time.perf_counter()
        H = orc.gram(X_bits)
        h = orc.act_sqmean(X_bits, n_threads=n_threads)
        t1 = time.perf_counter()
        if mode == "gptq-ord":
            perm = orc.block_order(orc.block_losses(W_bits, h, fmt, "hopt", block, sfmt=q.sfmt,
                                                    window=window))
        else:
            perm = np.arange(K // block, dtype=np.int32)
        t2 = time.perf_counter()
        cols = (perm[:, None] * block + np.arange(block)[None, :]).reshape(-1)
        U = orc.gptq_prepare(np.ascontiguousarray(H[np.ix_(cols, cols)])[None], GPTQ_DAMP)[0]
        t3 = time.perf_counter()
        r = orc.gptq_blocks(W_bits, U, h, fmt, "hopt", block, sfmt=q.sfmt, window=window,
                            perm=perm, n_threads=n_threads)
        What = orc.dequant(r.codes, r.scales, fmt, block, w_rows, K, sfmt=q.sfmt)
        orc.error_sums(W_bits, What, h)
        t4 = time.perf_counter()
        full = ((t1 - t0) * (R_full / x_rows) + (t2 - t1) * (N_full / w_rows) + (t3 - t2)
                + (t4 - t3) * (N_full / w_rows))
        return full, {"h_s": t1 - t0 + t3 - t2, "quant_s": t2 - t1 + t4 - t3}
    t0 = time.perf_counter()
    if mode in ("bhopt", "gptq"):
        G = orc.block_gram(X_bits, block)
    else:
        orc.act_sqmean(X_bits, n_threads=n_threads)
    t1 = time.perf_counter()
    if mode == "gptq":                     # per column block: independent of the rows
        U = orc.gptq_prepare(G)
        h_np = np.diagonal(G, axis1=1, axis2=2).reshape(-1).copy()
    tp = time.perf_counter()
    if mode == "bhopt":
        r = orc.quantize_gram(W_bits, fmt, block, G, window=window, n_threads=n_threads,
                              sfmt=q.sfmt)
    else:
        r = orc.quantize(W_bits, fmt, "hopt" if mode == "gptq" else mode, block, h=h_np,
                         window=window, n_threads=n_threads, sfmt=q.sfmt)
    codes = orc.gptq_tiles(W_bits, U, r.scales) if mode == "gptq" else r.codes
    What = orc.dequant(codes, r.scales, fmt, block, w_rows, K, sfmt=q.sfmt)
    orc.error_sums(W_bits, What, h_np)
    t2 = time.perf_counter()
    full = (t1 - t0) * (R_full / x_rows) + (tp - t1) + (t2 - tp) * (N_full / w_rows)
    return full, {"h_s": t1 - t0 + tp - t1, "quant_s": t2 - tp}


def bits_of(t):
    """Host copy for the oracle: bf16 as its raw 16-bit patterns, float32 as is."""
    import numpy as np
    if t.dtype == torch.float32:
        return t.contiguous().numpy()
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def proportional_rows(wl, w_rows):
    """Rows of the first activation matrix and of the first weight that make the same
    fraction of the workload: w_rows of the weights' rows (in units of the first weight's
    width) and the matching share of the activation rows (in units of the first activation
    matrix's width), so that a sample's time is that fraction of a full step's."""
    (_, n, k), (R, kx) = wl.weights[0], wl.x_shapes[0]
    n_equiv = sum(nn * kk for _, nn, kk in wl.weights) / k
    r_equiv = sum(r * kk for r, kk in wl.x_shapes) / kx
    w_rows = min(w_rows, n)
    x_rows = max(1, min(R, round(w_rows * r_equiv / n_equiv)))
    return x_rows, w_rows, w_rows / n_equiv


def reference_arm(args):
    """The CPU oracle, as it stands, timed on the host cores. Each step is the whole path on
    a proportional sample of the workload -- REF_W_ROWS weight rows and the matching share of
    the activation rows (h pass, search, error sums) -- so ms_per_step is the step's own
    measured time and the throughput is the sample's weights over it. GPTQ modes (whose
    factor does not shrink with the rows) time a smaller sample and scale it."""
    rank, world, _ = dist_env()
    if world > 1 and rank != 0:
        return
    from block_scaled_weight_b200 import synth
    from oracle import oracle as orc
    wl = synth.WORKLOADS[args.workload]
    q = quantizer_for(wl, args)
    (_, n, k), (R, _) = wl.weights[0], wl.x_shapes[0]
    nt = os.cpu_count() or 1
    weights = sum(nn * kk for _, nn, kk in wl.weights)
    headline = args.workload == "nvfp4_full_calib" and q == HEADLINE_Q
    metric = METRIC if headline else metric_for(q)
    times = []
    if full_gptq(q):
        x_rows, w_rows = min(REF_X_ROWS, R), min(GPTQ_CPU_W_ROWS, n)
        X = bits_of(synth.workload_activations(wl, 0, rows=x_rows))
        W = bits_of(synth.workload_weight(wl, 0, rows=w_rows))
        h = orc.act_sqmean(X)
        R_full = sum(r * kk for r, kk in wl.x_shapes) / k
        for i in range(args.warmup + args.steps):
            full, _ = oracle_step_sample(X, W, h, nt, R_full, weights / k, q)
            if i >= args.warmup:
                times.append(full)
        step_s = statistics.mean(times)
        value = weights / step_s / 1e9
        sample = (f"oracle on {x_rows} of {R} X rows and {w_rows} of {n} W rows per step, "
                  f"{nt} threads; times scaled to the full workload")
    else:
        w_rows = REF_W_ROWS
        if q.fmt == "e4m3":
            w_rows = max(w_rows - w_rows % q.block, q.block)
        x_rows, w_rows, frac = proportional_rows(wl, w_rows)
        X = bits_of(synth.workload_activations(wl, 0, rows=x_rows))
        W = bits_of(synth.workload_weight(wl, 0, rows=w_rows))
        for i in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            oracle_path(X, W, nt, q)
            if i >= args.warmup:
                times.append(time.perf_counter() - t0)
        step_s = statistics.mean(times)
        value = frac * weights / step_s / 1e9
        sample = (f"oracle, whole path per step on {x_rows} of {R} X rows and {w_rows} of "
                  f"{n} W rows (the same {frac:.2%} share of the activations and of the "
                  f"weights), {nt} threads; per-step time measured, not scaled")
    line = {"impl": "reference", "metric": metric, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(wl, q)},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": nt, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def oracle_path(X_bits, W_bits, n_threads, q):
    """One pass of the whole path through the oracle on host inputs: h pass (or Gram blocks),
    search (or tile GPTQ), dequantisation and the error sums."""
    import numpy as np
    from oracle import oracle as orc
    fmt, block, mode, window = q.fmt, q.block, q.mode, q.window
    w_rows, K = W_bits.shape
    if mode in ("bhopt", "gptq"):
        G = orc.block_gram(X_bits, block)
        h = np.diagonal(G, axis1=1, axis2=2).reshape(-1).copy()
    else:
        h = orc.act_sqmean(X_bits, n_threads=n_threads)
    if mode == "bhopt":
        r = orc.quantize_gram(W_bits, fmt, block, G, window=window, n_threads=n_threads,
                              sfmt=q.sfmt)
        codes = r.codes
    elif mode == "gptq":
        r = orc.quantize(W_bits, fmt, "hopt", block, h=h, window=window, n_threads=n_threads,
                         sfmt=q.sfmt)
        codes = orc.gptq_tiles(W_bits, orc.gptq_prepare(G), r.scales)
    else:
        r = orc.quantize(W_bits, fmt, mode, block, h=h if mode == "hopt" else None,
                         window=window, n_threads=n_threads, sfmt=q.sfmt)
        codes = r.codes
    What = orc.dequant(codes, r.scales, fmt, block, w_rows, K, sfmt=q.sfmt)
    return orc.error_sums(W_bits, What, h)


# ---------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------

def quantizer_for(wl, args):
    """The quantizer the bench times for a workload (its own, or the command line's)."""
    block = args.block or wl.blocks[0]
    mode = args.mode or ("hopt" if "hopt" in wl.modes else wl.modes[-1])
    fmt = args.fmt or wl.fmt
    if mode == "gptq" and fmt == "e4m3" and block != 64:
        raise SystemExit("--mode gptq on E4M3 elements uses 64 x 64 tiles")
    if mode.startswith("gptq") and fmt not in ("e4m3", "nvfp4", "int4"):
        raise SystemExit("--mode gptq: NVFP4 / INT4 blocks or E4M3 64 x 64 tiles")
    if mode == "gptq-ord" and fmt == "e4m3":
        raise SystemExit("--mode gptq-ord: NVFP4 / INT4 blocks")
    return Quantizer(fmt, block, mode, wl.window, args.scale_fmt or "e4m3")


def full_gptq(q):
    """GPTQ over the whole input dimension (NVFP4 / INT4 blocks), not the E4M3 tiles."""
    return q.mode in ("gptq", "gptq-ord") and q.fmt in ("nvfp4", "int4")


def sweep_ops_per_weight(q, k):
    """Algorithmic lane-operations per weight of the GPTQ sweep: the block's scale search
    (C candidates x 6 + 4, as the plain search), its own quantisation, residual and division
    (6), and the updates it receives from every earlier column -- one product and one
    difference from each earlier column of its block, one fma from each column of every
    earlier block plus one difference per earlier block: on average (k / 2)(1 + 1/B)."""
    return ops_per_weight(q.fmt, "hopt", q.window, q.sfmt, q.block) + 6 + (k / 2) * (1 + 1 / q.block)


def metric_for(q):
    return (f"G weights/s quantized ({q.mode} {quant_name(q)} blk{q.block}) + h-pass GB/s; "
            f"% of roofline")


def ops_per_weight(fmt, mode, window, sfmt="e4m3", block=16):
    """Algorithmic lane-operations per weight of a scale search: C candidates x 6 (quotient,
    projection, dequantise, subtract, h-multiply, square-accumulate; 5 without h) + 4
    (amax, naive quotient, final projection, pack)."""
    full = 126 if sfmt == "e4m3" else 255
    C = 64 if fmt == "e4m3" else (full if window < 0 else 2 * window + 1)
    if mode == "bhopt":      # quotient, round, dequantise, sign + B FMAs of the form
        return C * (block + 4) + 4
    return C * (6 if mode == "hopt" else 5) + 4


# The GPTQ sweep per weight: quotient, round, dequantise, residual, division by U_cc, pack
# (6), and its residual's propagation into the 63 - c later columns of the tile row, one
# product and one difference each (2 x 31.5 on average over c = 0 .. 63).
GPTQ_SWEEP_OPS = 6 + 63
GPTQ_DAMP = 0.01          # lambda = 0.01 x mean(diag G_b), GPTQ's customary damping


def code_bytes(fmt, block):
    """Bytes of codes + scales per weight."""
    if fmt in ("nvfp4", "int4"):
        return 0.5 + 1.0 / block
    if fmt == "int8":
        return 1.0 + 1.0 / block
    return 1.0 + 4.0 / (block * block)


def gpu_arm(args):
    import torch.distributed as dist
    from block_scaled_weight_b200 import mxq, synth
    from block_scaled_weight_b200.dist import distributed_h
    rank, world, local = dist_env()
    wl = synth.WORKLOADS[args.workload]
    q = quantizer_for(wl, args)
    if full_gptq(q):
        return gpu_arm_gptq(args, wl, q)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    fmt, block, mode, window = q.fmt, q.block, q.mode, q.window
    bh, gq = mode == "bhopt", mode == "gptq"
    gram = bh or gq                       # the Gram pass replaces the h pass
    if gram and world > 1:
        raise SystemExit(f"--mode {mode} runs on one GPU")
    p = mxq.params(fmt, "hopt" if gram else mode, block, window=window, scale_fmt=q.sfmt)
    # for the overlapped steps below, when the h pass is long enough to hide it: the search
    # holds one CTA per SM, leaving the other SM slots to the next batch's h pass beside it
    p_overlap = mxq.params(fmt, "hopt" if gram else mode, block, window=window,
                           scale_fmt=q.sfmt, ctas_per_sm=1)
    # inputs: every rank draws its own shard (weak scaling)
    wl_r = dataclasses.replace(wl, seed=wl.seed + 1000 * rank)
    # activations and their h, one per activation width
    Xs, hs, wss, cols, Gs, Us = [], [], [], [], [], []
    for xi, (R, k) in enumerate(wl.x_shapes):
        R = min(R, args.x_rows) if args.x_rows else R
        X = torch.empty(R, k, dtype=wl.w_dtype, device=dev)
        synth.workload_activations(wl_r, xi, device=dev, rows=R, out=X)
        Xs.append(X)
        hs.append(torch.empty(k, dtype=torch.float32, device=dev))
        wss.append(torch.empty(mxq.mxq_act_block_gram_workspace(R, k, block) if gram else
                               mxq.mxq_act_sqmean_workspace(R, k), dtype=torch.uint8, device=dev))
        cols.append(torch.empty(k, dtype=torch.float64, device=dev))
        Gs.append(torch.empty(k // block, block, block, dtype=torch.float32, device=dev)
                  if gram else None)
        Us.append(torch.empty(k // block, block, block, dtype=torch.float32, device=dev)
                  if gq else None)
    # weights and their outputs (codes, scales, error sums, error workspace, which h)
    Ws, outs = [], []
    for wi, (_, n, k) in enumerate(wl.weights):
        Ws.append(synth.workload_weight(wl_r, wi, device=dev))
        cs, cd, ss, sd = mxq.output_shapes(p, n, k)
        ews = max(mxq.mxq_error_workspace(n, k), mxq.mxq_quantize_err_workspace(n, k, p),
                  mxq.mxq_quantize_err_workspace(n, k, p_overlap))
        outs.append((torch.empty(cs, dtype=cd, device=dev), torch.empty(ss, dtype=sd, device=dev),
                     torch.empty(4, dtype=torch.float64, device=dev),
                     torch.empty(ews, dtype=torch.uint8, device=dev),
                     synth.x_index_for_weight(wl, wi)))
    stream = torch.cuda.current_stream(dev)
    # The NVFP4 search with E4M3 scales adds the error sums itself (mxq_quantize_err: search,
    # exact pass, combine); every other quantizer runs the error pass after it.
    fused = fmt == "nvfp4" and q.sfmt == "e4m3" and mode in ("sse", "hopt")
    # our kernels per step: h pass or Gram pass (2 per activation matrix; 3 with the sharded
    # finalize), search (+ exact fixup for NVFP4 / INT8 searches), error sums + combine (2)
    # per weight (fused: the combine only); GPTQ adds the factor (1 per activation matrix)
    # and the sweep (1 per weight)
    fixup = 1 if mode != "naive" and fmt != "e4m3" else 0
    launches_per_step = len(Xs) * (2 if world == 1 else 3) + len(Ws) * (
        1 + fixup + (1 if fused else 2))
    if gq:
        launches_per_step += len(Xs) + len(Ws)

    def h_phase():
        for X, h, ws, colsum, G in zip(Xs, hs, wss, cols, Gs):
            if gram:
                mxq.mxq_act_block_gram(X, block, G, h, workspace=ws)
            elif world == 1:
                mxq.mxq_act_sqmean(X, h, workspace=ws)
            else:
                # per-rank column sums -> rank-ordered all-gather -> fixed-order finalize
                distributed_h(X, lambda x, c=colsum, w=ws: mxq.mxq_act_sqsum(x, c, workspace=w),
                              lambda pp, r, hh=h: mxq.mxq_act_sqmean_finalize(pp, r, hh),
                              X.shape[0] * world)

    def prepare_phase():
        for G, U in zip(Gs, Us):
            mxq.mxq_gptq_prepare(G, GPTQ_DAMP, U=U)

    def quantize_phase():
        for W, (codes, scales, sums, ews, xi) in zip(Ws, outs):
            if fused:
                mxq.mxq_quantize_err(W, p, hs[xi], codes=codes, scales=scales, sums=sums,
                                     workspace=ews)
            elif bh:
                mxq.mxq_quantize_gram(W, p, Gs[xi], codes=codes, scales=scales)
            else:
                mxq.mxq_quantize(W, p, hs[xi], codes=codes, scales=scales)

    def sweep_phase():
        for W, (codes, scales, _, _, xi) in zip(Ws, outs):
            mxq.mxq_gptq_tiles(W, Us[xi], scales, codes=codes)

    def error_phase():
        for W, (codes, scales, sums, ews, xi) in zip(Ws, outs):
            mxq.mxq_error(W, codes, scales, p, hs[xi], sums=sums, workspace=ews)

    hname = "block_gram" if gram else "act_sqmean"
    phases = [(hname, h_phase)]
    if gq:
        phases.append(("gptq_prepare", prepare_phase))
    phases.append(("quantize", quantize_phase))
    if gq:
        phases.append(("gptq_tiles", sweep_phase))
    if not fused:
        phases.append(("error", error_phase))

    def step(ev=None):
        for i, (_, fn) in enumerate(phases):
            if ev is not None:
                ev[i].record(stream)
            fn()
        if ev is not None:
            ev[-1].record(stream)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    # Inputs smaller than a few L2s would be served from L2 on the next step: flush L2
    # between steps (a write of twice its size) and time the steps alone.
    in_bytes = sum(t.numel() * t.element_size() for t in Xs + Ws)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) \
        if in_bytes < 4 * L2_BYTES else None

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(phases) + 1)]
           for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    barrier()
    torch.cuda.synchronize(dev)
    with sampler:
        t_start.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()
            step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    ms_total = t_start.elapsed_time(t_end) if flush is None else \
        sum(e[0].elapsed_time(e[-1]) for e in evs)
    k_ph = [sum(e[i].elapsed_time(e[i + 1]) for e in evs) / args.steps
            for i in range(len(phases))]
    t = torch.tensor([ms_total] + k_ph, dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_total, *k_ph = t.tolist()
    k_of = {nm: kk for (nm, _), kk in zip(phases, k_ph)}
    k_h, k_q, k_e = k_of[hname], k_of["quantize"], k_of.get("error")
    ms_step = ms_total / args.steps
    ms_step_serial = ms_step
    weights = sum(W.numel() for W in Ws)

    # ---- pipelined steps: step i's search and error sums (one stream) overlap step i+1's h
    # pass (another stream; h in two alternating buffers). The h pass is HBM-bound, the search
    # ALU-bound. Every step still does all of its work; only consecutive steps overlap.
    pipelined = world == 1 and not gram and flush is None and not args.serial
    # a search held to one CTA per SM runs about 1.7 x longer alone: worth it only when the
    # h pass it runs beside is longer still
    p_pipe = p_overlap if k_h >= 1.8 * k_q else p
    if pipelined:
        # the search stream at the higher priority: its CTAs take SM slots first as the h
        # pass's free up
        s_h, s_q = torch.cuda.Stream(dev), torch.cuda.Stream(dev, priority=-1)
        hb = [hs, [torch.empty_like(h) for h in hs]]
        # a fresh pair of events per step, so that no event is recorded again while a wait
        # on its earlier record may still be queued (the host runs many steps ahead)
        ev_h = [torch.cuda.Event() for _ in range(max(args.warmup, args.steps))]
        ev_q = [torch.cuda.Event() for _ in range(max(args.warmup, args.steps))]

        def pstep(i, wait_free):
            b = i & 1
            with torch.cuda.stream(s_h):
                if wait_free:
                    s_h.wait_event(ev_q[i - 2])
                for X, h, ws in zip(Xs, hb[b], wss):
                    mxq.mxq_act_sqmean(X, h, workspace=ws)
                ev_h[i].record(s_h)
            with torch.cuda.stream(s_q):
                s_q.wait_event(ev_h[i])
                for W, (codes, scales, sums, ews, xi) in zip(Ws, outs):
                    if fused:
                        mxq.mxq_quantize_err(W, p_pipe, hb[b][xi], codes=codes,
                                             scales=scales, sums=sums, workspace=ews)
                    else:
                        mxq.mxq_quantize(W, p, hb[b][xi], codes=codes, scales=scales)
                        mxq.mxq_error(W, codes, scales, p, hb[b][xi], sums=sums, workspace=ews)
                ev_q[i].record(s_q)

        for i in range(args.warmup):
            pstep(i, i >= 2)
        torch.cuda.synchronize(dev)
        # The K timed steps as one CUDA graph (both streams forked from and joined into the
        # capture stream), launched once: the overlap of the two streams then does not
        # depend on the host staying ahead of the GPU. Should capture fail, the steps are
        # enqueued one by one instead.
        cap = torch.cuda.Stream(dev)
        graph = None
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                fork = torch.cuda.Event()
                fork.record(cap)
                s_h.wait_event(fork)
                s_q.wait_event(fork)
                for i in range(args.steps):
                    pstep(i, i >= 2)
                cap.wait_stream(s_h)
                cap.wait_stream(s_q)
            graph = g
        except Exception as e:  # noqa: BLE001 -- reported in the JSON line, eager steps used
            graph_note = f"graph capture failed ({type(e).__name__}); steps enqueued one by one"
        torch.cuda.synchronize(dev)
        p_start = torch.cuda.Event(enable_timing=True)
        p_end = torch.cuda.Event(enable_timing=True)
        if graph is not None:
            graph_note = "the K timed steps captured as one CUDA graph and launched once"
            with torch.cuda.stream(cap):
                graph.replay()                  # untimed: the graph's first launch
            torch.cuda.synchronize(dev)
            with sampler:
                with torch.cuda.stream(cap):
                    p_start.record(cap)
                    graph.replay()
                    p_end.record(cap)
                torch.cuda.synchronize(dev)
        else:
            with sampler:
                p_start.record(s_h)
                s_q.wait_event(p_start)
                for i in range(args.steps):
                    pstep(i, i >= 2)
                p_end.record(s_q)
                torch.cuda.synchronize(dev)
        ms_step = p_start.elapsed_time(p_end) / args.steps
        # the last step's outputs are the ones the e2e and metric reads below use
    value = world * weights / (ms_step * 1e-3) / 1e9

    # ---- end to end through the public API, host buffers -----------------------------
    Xh = [torch.empty(X.shape, dtype=X.dtype, pin_memory=True) for X in Xs]
    Wh = [torch.empty(W.shape, dtype=W.dtype, pin_memory=True) for W in Ws]
    for th, td in zip(Xh + Wh, Xs + Ws):
        th.copy_(td)
    oh = [tuple(torch.empty(td.shape, dtype=td.dtype, pin_memory=True) for td in o[:3])
          for o in outs]
    h2d = sum(th.numel() * th.element_size() for th in Xh + Wh)
    d2h = sum(th.numel() * th.element_size() for o in oh for th in o)

    def e2e_step():
        for td, th in zip(Xs + Ws, Xh + Wh):
            td.copy_(th, non_blocking=True)
        step()
        for o, ho in zip(outs, oh):
            for td, th in zip(o[:3], ho):
                th.copy_(td, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    t2 = torch.tensor([a.elapsed_time(b)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t2, op=dist.ReduceOp.MAX)
    e2e_ms = t2.item() / args.e2e_steps
    e2e_value = world * weights / (e2e_ms * 1e-3) / 1e9
    metrics = mxq.mxq_metrics_from_sums(oh[0][2])
    # The pages' output error ||X_s Wq^T - X_s W^T||_F / ||X_s W^T||_F on 512 sampled rows of
    # X, for the first weight (tensor cores; outside the timed region).
    out_rel = None
    if fmt in ("nvfp4", "int4") and Xs[0].dtype == torch.bfloat16:
        W0, (c0_, s0_, _, _, xi0) = Ws[0], outs[0]
        rows = synth.sample_rows(Xs[xi0].shape[0], 512, wl.seed + 7).to(dev)
        Xsmp = Xs[xi0].index_select(0, rows).contiguous()
        osum = mxq.mxq_output_error(Xsmp, W0, c0_, s0_, p).cpu()
        out_rel = float((osum[0] / osum[1]).sqrt())

    # ---- roofline ------------------------------------------------------------------------
    hbm, hbm_kind = measured_peaks()
    headline = args.workload == "nvfp4_full_calib" and q == HEADLINE_Q and not args.x_rows
    x_bytes = sum(X.numel() * X.element_size() + 4 * X.shape[1] * (block if gram else 1)
                  for X in Xs)
    w_bytes = sum(W.numel() * W.element_size() for W in Ws)
    h_gbs = x_bytes / (k_h * 1e-3) / 1e9
    kernels = {hname: {"ms": k_h, "bound": "hbm", "achieved": h_gbs, "peak": hbm,
                       "unit": "GB/s", "frac": h_gbs / hbm, "algorithmic_bytes": x_bytes,
                       "traffic": traffic_for("act_sqmean") if headline else None}}
    if mode == "naive":
        q_bytes = w_bytes + weights * code_bytes(fmt, block)
        q_gbs = q_bytes / (k_q * 1e-3) / 1e9
        kernels["quantize"] = {"ms": k_q, "bound": "hbm", "achieved": q_gbs, "peak": hbm,
                               "unit": "GB/s", "frac": q_gbs / hbm, "algorithmic_bytes": q_bytes,
                               "traffic": None}
    else:
        ops = ops_per_weight(fmt, mode, window, q.sfmt, block) * weights
        q_tops = ops / (k_q * 1e-3) / 1e12
        kernels["quantize"] = {"ms": k_q, "bound": "alu", "achieved": q_tops,
                               "peak": ALU_PEAK_TOPS, "unit": "T lane-op/s",
                               "frac": q_tops / ALU_PEAK_TOPS, "algorithmic_ops": ops,
                               "traffic": traffic_for("quantize") if headline else None}
        if fused:
            kernels["quantize"]["includes"] = ("the error sums at the winning scales (added "
                                               "inside the search and its exact pass)")
        ex = executed_for("quantize") if headline else None
        if ex:
            # the hardware's view: thread instructions the search kernels executed per launch
            # (an ncu capture of this build) over the launch time, against the lane peak
            kernels["quantize"]["executed"] = {
                "thread_inst_per_launch": ex["thread_inst"],
                "achieved": ex["thread_inst"] / (k_q * 1e-3) / 1e12,
                "frac_executed": ex["thread_inst"] / (k_q * 1e-3) / 1e12 / ALU_PEAK_TOPS,
                "active_lanes_per_inst": ex["lanes"],
                "candidates_scored_per_block": ex.get("candidates_per_block")}
    if gq:
        u_bytes = sum(2 * 4 * X.shape[1] * block for X in Xs)     # G read, U written
        kernels["gptq_prepare"] = {
            "ms": k_of["gptq_prepare"], "bound": "hbm",
            "achieved": u_bytes / (k_of["gptq_prepare"] * 1e-3) / 1e9, "peak": hbm,
            "unit": "GB/s", "frac": u_bytes / (k_of["gptq_prepare"] * 1e-3) / 1e9 / hbm,
            "algorithmic_bytes": u_bytes, "traffic": None}
        s_ops = GPTQ_SWEEP_OPS * weights
        s_tops = s_ops / (k_of["gptq_tiles"] * 1e-3) / 1e12
        kernels["gptq_tiles"] = {"ms": k_of["gptq_tiles"], "bound": "alu", "achieved": s_tops,
                                 "peak": ALU_PEAK_TOPS, "unit": "T lane-op/s",
                                 "frac": s_tops / ALU_PEAK_TOPS, "algorithmic_ops": s_ops,
                                 "traffic": None}
    if k_e is not None:
        e_bytes = w_bytes + weights * code_bytes(fmt, block) + sum(4 * W.shape[1] for W in Ws)
        e_gbs = e_bytes / (k_e * 1e-3) / 1e9
        kernels["error"] = {"ms": k_e, "bound": "hbm", "achieved": e_gbs, "peak": hbm,
                            "unit": "GB/s", "frac": e_gbs / hbm, "algorithmic_bytes": e_bytes,
                            "traffic": traffic_for("error") if headline else None}
    dom = max(kernels, key=lambda kk: kernels[kk]["ms"])
    dk = kernels[dom]
    roofline = {"kernel": dom, "bound": dk["bound"], "achieved": dk["achieved"],
                "peak": dk["peak"], "unit": dk["unit"], "frac": dk["frac"],
                "traffic": dk["traffic"],
                "peak_source": ("MEASURED_PEAKS.json hbm_gbs (" + hbm_kind + ")")
                if dk["bound"] == "hbm" else "148 SM x 128 FP32 lanes x 1965 MHz"}
    metric = METRIC if (args.workload == "nvfp4_full_calib" and q == HEADLINE_Q) \
        else metric_for(q)
    line = {"metric": metric, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "ms_per_step_serial": ms_step_serial,
            "pipelined": ("step i's search and error sums overlap step i+1's h pass (two "
                          "streams, h double-buffered; search occupancy: "
                          + ("one CTA per SM beside the h pass's two, mxq_params.ctas_per_sm "
                             "= 1" if p_pipe is p_overlap else "all SM slots") +
                          "; " + graph_note + "); kernel times below are from the serial timed "
                          "region")
            if pipelined else None,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": workload_desc(wl, q, [X.shape[0] for X in Xs]),
                       "weights_per_gpu": weights,
                       "x_rows_per_gpu": Xs[0].shape[0] if len(Xs) == 1 else
                       [X.shape[0] for X in Xs],
                       "parallelism": f"dp{world}" + (" (rows of X and W per rank; one "
                                                      "all-gather of column sums)" if world > 1 else ""),
                       "l2": ("inputs larger than L2: X (%.2f GB) is streamed every step"
                              % (sum(X.numel() * X.element_size() for X in Xs) / 1e9))
                       if flush is None else
                       ("L2 flushed between steps (a %d MB write, outside the step's events); "
                        "inputs %.0f MB" % (2 * L2_BYTES >> 20, in_bytes / 1e6))},
            "h_pass_gbs": h_gbs, "h_pass_frac_of_hbm": h_gbs / hbm,
            "roofline": roofline, "kernels": kernels,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": args.e2e_steps},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": sampler.summary(),
            "result": {"weight_rel": metrics["weight_rel"], "h_rel": metrics["h_rel"],
                       "output_rel_512_rows": out_rel}}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        X0, W0 = Xs[0], Ws[0]
        R0, n0 = X0.shape[0], W0.shape[0]
        # the whole path on a proportional sample: the same share of X's rows and W's rows
        w_rows = CPU_W_ROWS // (8 if fmt == "e4m3" or mode == "bhopt" else 1)
        if fmt == "e4m3":
            w_rows = max(w_rows - w_rows % block, block)
        x_rows, w_rows, frac = proportional_rows(wl, w_rows)
        x_rows = min(x_rows, R0)
        Xb = bits_of(X0[:x_rows].cpu())
        Wb = bits_of(W0[:w_rows].cpu())
        from oracle import oracle as orc
        nt = os.cpu_count() or 1
        t0 = time.perf_counter()
        oracle_path(Xb, Wb, nt, q)
        t_cpu = time.perf_counter() - t0
        line["cpu_baseline"] = {
            "value": frac * weights / t_cpu / 1e9, "unit": UNIT, "cores": nt, "kind": "oracle",
            "sample": (f"oracle, whole path on {x_rows} of {R0} X rows and {w_rows} of {n0} W "
                       f"rows (the same {frac:.2%} share of the activations and the weights), "
                       f"{nt} threads, {t_cpu:.1f} s measured")}
        line["result"]["parity_sample"] = sampled_parity(orc, synth, wl, q, p, Ws[0], outs[0],
                                                         hs[outs[0][4]], nt)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def sampled_parity(orc, synth, wl, q, p, W, out, h, nt, n_rows=32):
    """The timed step's own outputs for sampled rows of the first weight against the oracle
    run on the same bytes (the same weight rows, the GPU's h): blocks compared, blocks whose
    scale or codes differ, and near ties -- blocks whose two best candidate errors differ by
    less than 1e-6 relative, which the acceptance rule counts and excludes. 1-D block
    quantizers with a diagonal objective only (null otherwise)."""
    import numpy as np
    if q.fmt == "e4m3" or q.mode not in ("naive", "sse", "hopt"):
        return None
    codes, scales = out[0], out[1]
    n = W.shape[0]
    rows = synth.sample_rows(n, min(n_rows, n), wl.seed + 11)
    ri = rows.to(W.device)
    r = orc.quantize(bits_of(W.index_select(0, ri).cpu()), q.fmt, q.mode, q.block,
                     h=h.cpu().numpy() if q.mode == "hopt" else None, window=q.window,
                     sfmt=q.sfmt, n_threads=nt)
    g_s = scales.index_select(0, ri).cpu().numpy()
    g_c = codes.index_select(0, ri).cpu().numpy().view(np.uint8)
    bpr = g_s.shape[1]
    cpb = g_c.shape[1] // bpr                        # code bytes per block
    code_bad = (g_c.reshape(len(rows), bpr, cpb) !=
                r.codes.view(np.uint8).reshape(len(rows), bpr, cpb)).any(axis=2)
    bad = (g_s != r.scales) | code_bad
    near = orc.near_tie(r.best, r.second) if q.mode != "naive" else np.zeros_like(bad)
    return {"rows": int(len(rows)), "blocks": int(bad.size),
            "differing_blocks": int(bad.sum()), "near_tie_blocks": int(near.sum()),
            "differing_outside_near_ties": int((bad & ~near).sum()),
            "h": "the GPU's h of the timed step (the oracle gets the same bytes)"}


def gptq_launches(k, ordered, panel_tiles=4):
    """Our kernels per GPTQ step: h pass 2, the Hessian 3 (the tensor-core product, the sums
    of the last wave's row chunks, the transpose onto the lower triangle), [order: search,
    fixup, block losses, sort], factor (lambda, load, per tile column: panel update (not the
    panel's first), diagonal tile, tiles below (not the last); per panel but the last: the
    next panel's columns and, while any remain, everything beyond; 2 per doubling level;
    store), sweep (init, 64-position panels, trailing updates), error 2."""
    nt = (k + 63) // 64
    f = 2 + 1
    for p0 in range(0, nt, panel_tiles):
        pe = min(p0 + panel_tiles, nt)
        for p in range(p0, pe):
            f += (p > p0) + 1 + (p < nt - 1)
        if pe < nt:
            f += 1 + (min(pe + panel_tiles, nt) < nt)
    s = 1
    while s < nt:
        f += 2
        s *= 2
    panels = (k + 63) // 64
    return 2 + 3 + (4 if ordered else 0) + f + 1 + panels + (panels - 1) + 2


def bf16_peak():
    try:
        with open(PEAKS_FILE) as f:
            pk = json.load(f)
        return float(pk["bf16_tflops_sustained"]), "measured, sustained"
    except Exception:
        return 1400.0, "fallback, sustained"


# FP64 FMA peak of the factorisation kernels: 148 SMs x 64 FP64 lanes x 2 flops x 1965 MHz.
FP64_PEAK_TFLOPS = 148 * 64 * 2 * 1.965e9 / 1e12


def gpu_arm_gptq(args, wl, q):
    """GPTQ over the whole input dimension with the H-optimal quantizer as its inner step
    (sequential or ordered) on one GPU: h pass, Gram matrix, [block order], factor, sweep,
    error sums."""
    from block_scaled_weight_b200 import mxq, synth
    rank, world, local = dist_env()
    if world > 1:
        raise SystemExit(f"--mode {q.mode} runs on one GPU")
    if len(wl.weights) != 1:
        raise SystemExit(f"--mode {q.mode}: workloads with one weight matrix")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ordered = q.mode == "gptq-ord"
    B = q.block
    p = mxq.params(q.fmt, "hopt", B, window=q.window, scale_fmt=q.sfmt)
    (_, n, k), (R, _) = wl.weights[0], wl.x_shapes[0]
    R = min(R, args.x_rows) if args.x_rows else R
    X = torch.empty(R, k, dtype=wl.w_dtype, device=dev)
    synth.workload_activations(wl, 0, device=dev, rows=R, out=X)
    W = synth.workload_weight(wl, 0, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    u8 = dict(dtype=torch.uint8, device=dev)
    h = torch.empty(k, **f32)
    H = torch.empty(k, k, **f32)
    gws = torch.empty(max(mxq.mxq_act_gram_workspace(R, k), 8), **u8)
    U = torch.empty(k, k, **f32)
    perm = torch.arange(k // B, dtype=torch.int32, device=dev)
    hws = torch.empty(mxq.mxq_act_sqmean_workspace(R, k), **u8)
    fws = torch.empty(mxq.mxq_gptq_factor_workspace(k), **u8)
    ows = torch.empty(max(mxq.mxq_gptq_order_workspace(n, k, p), 8), **u8)
    sws = torch.empty(mxq.mxq_gptq_workspace(n, k), **u8)
    cs, cd, ss, sd = mxq.output_shapes(p, n, k)
    codes, scales = torch.empty(cs, dtype=cd, device=dev), torch.empty(ss, dtype=sd, device=dev)
    sums = torch.empty(4, dtype=torch.float64, device=dev)
    ews = torch.empty(mxq.mxq_error_workspace(n, k), **u8)
    pv = perm if ordered else None
    phases = [("act_sqmean", lambda: mxq.mxq_act_sqmean(X, h, workspace=hws)),
              ("gram", lambda: mxq.mxq_act_gram(X, H, workspace=gws))]
    if ordered:
        phases.append(("gptq_order", lambda: mxq.mxq_gptq_order(W, h, p, perm=perm,
                                                                workspace=ows)))
    phases += [("gptq_factor", lambda: mxq.mxq_gptq_factor(H, B, pv, GPTQ_DAMP, U=U,
                                                           workspace=fws)),
               ("gptq_sweep", lambda: mxq.mxq_gptq(W, U, p, h, pv, codes=codes, scales=scales,
                                                   workspace=sws)),
               ("error", lambda: mxq.mxq_error(W, codes, scales, p, h, sums=sums,
                                               workspace=ews))]
    stream = torch.cuda.current_stream(dev)
    launches_per_step = gptq_launches(k, ordered)

    def step(ev=None):
        for i, (_, fn) in enumerate(phases):
            if ev is not None:
                ev[i].record(stream)
            fn()
        if ev is not None:
            ev[-1].record(stream)

    in_bytes = X.numel() * X.element_size() + W.numel() * W.element_size()
    flush = torch.empty(2 * L2_BYTES, **u8) if in_bytes < 4 * L2_BYTES else None
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(phases) + 1)]
           for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    torch.cuda.synchronize(dev)
    with sampler:
        t_start.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()
            step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    ms_total = t_start.elapsed_time(t_end) if flush is None else \
        sum(e[0].elapsed_time(e[-1]) for e in evs)
    k_of = {nm: sum(e[i].elapsed_time(e[i + 1]) for e in evs) / args.steps
            for i, (nm, _) in enumerate(phases)}
    ms_step = ms_total / args.steps
    weights = W.numel()
    value = weights / (ms_step * 1e-3) / 1e9

    # ---- end to end through the public API, host buffers -----------------------------
    Xh = torch.empty(X.shape, dtype=X.dtype, pin_memory=True)
    Wh = torch.empty(W.shape, dtype=W.dtype, pin_memory=True)
    Xh.copy_(X)
    Wh.copy_(W)
    oh = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (codes, scales, sums)]
    h2d = Xh.numel() * Xh.element_size() + Wh.numel() * Wh.element_size()
    d2h = sum(t.numel() * t.element_size() for t in oh)

    def e2e_step():
        X.copy_(Xh, non_blocking=True)
        W.copy_(Wh, non_blocking=True)
        step()
        for td, th in zip((codes, scales, sums), oh):
            th.copy_(td, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = a.elapsed_time(b) / args.e2e_steps
    metrics = mxq.mxq_metrics_from_sums(oh[2])
    rows = synth.sample_rows(R, 512, wl.seed + 7).to(dev)
    Xsmp = X.index_select(0, rows).contiguous()
    osum = mxq.mxq_output_error(Xsmp, W, codes, scales, p).cpu()
    out_rel = float((osum[0] / osum[1]).sqrt())

    # ---- roofline ------------------------------------------------------------------------
    hbm, hbm_kind = measured_peaks()
    bfp, bf_kind = bf16_peak()
    x_bytes = X.numel() * X.element_size() + 4 * k
    w_bytes = W.numel() * W.element_size()

    def kern(nm, bound, amount, peak, unit):
        ach = amount / (k_of[nm] * 1e-3) / (1e9 if unit == "GB/s" else 1e12)
        return {"ms": k_of[nm], "bound": bound, "achieved": ach, "peak": peak, "unit": unit,
                "frac": ach / peak, ("algorithmic_bytes" if unit == "GB/s" else
                                     "algorithmic_ops"): amount, "traffic": None}
    kernels = {"act_sqmean": kern("act_sqmean", "hbm", x_bytes, hbm, "GB/s"),
               # H is symmetric: the work that defines it is one triangle, diagonal included
               "gram": kern("gram", "tensor", 1.0 * R * k * (k + 1), bfp, "TFLOP/s")}
    if ordered:
        kernels["gptq_order"] = kern("gptq_order", "alu",
                                     ops_per_weight(q.fmt, "hopt", q.window, q.sfmt, B) * weights,
                                     ALU_PEAK_TOPS, "T lane-op/s")
    kernels["gptq_factor"] = kern("gptq_factor", "fp64", 2.0 / 3.0 * k ** 3, FP64_PEAK_TFLOPS,
                                  "TFLOP/s")
    kernels["gptq_sweep"] = kern("gptq_sweep", "alu", sweep_ops_per_weight(q, k) * weights,
                                 ALU_PEAK_TOPS, "T lane-op/s")
    kernels["error"] = kern("error", "hbm", w_bytes + weights * code_bytes(q.fmt, B) + 4 * k, hbm,
                            "GB/s")
    dom = max(kernels, key=lambda kk: kernels[kk]["ms"])
    dk = kernels[dom]
    src = {"hbm": "MEASURED_PEAKS.json hbm_gbs (" + hbm_kind + ")",
           "tensor": "MEASURED_PEAKS.json bf16_tflops_sustained (" + bf_kind + ")",
           "alu": "148 SM x 128 FP32 lanes x 1965 MHz",
           "fp64": "148 SM x 64 FP64 lanes x 2 x 1965 MHz"}[dk["bound"]]
    roofline = {"kernel": dom, "bound": dk["bound"], "achieved": dk["achieved"],
                "peak": dk["peak"], "unit": dk["unit"], "frac": dk["frac"],
                "traffic": None, "peak_source": src}
    line = {"metric": metric_for(q), "value": value, "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": workload_desc(wl, q, [R]), "weights_per_gpu": weights,
                       "x_rows_per_gpu": R, "parallelism": "dp1",
                       "l2": ("inputs larger than L2: X (%.2f GB) is streamed every step"
                              % (X.numel() * X.element_size() / 1e9)) if flush is None else
                       ("L2 flushed between steps (a %d MB write, outside the step's events); "
                        "inputs %.0f MB" % (2 * L2_BYTES >> 20, in_bytes / 1e6))},
            "roofline": roofline, "kernels": kernels,
            "e2e": {"value": weights / (e2e_ms * 1e-3) / 1e9, "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "steps": args.e2e_steps},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": sampler.summary(),
            "result": {"weight_rel": metrics["weight_rel"], "h_rel": metrics["h_rel"],
                       "output_rel_512_rows": out_rel}}
    if not args.no_cpu_baseline:
        x_rows = min(GPTQ_CPU_X_ROWS, R)
        w_rows = min(GPTQ_CPU_W_ROWS, n)
        Xb = bits_of(X[:x_rows].cpu())
        Wb = bits_of(W[:w_rows].cpu())
        nt_cpu = os.cpu_count() or 1
        full, d = oracle_step_sample(Xb, Wb, None, nt_cpu, R, n, q)
        line["cpu_baseline"] = {
            "value": weights / full / 1e9, "unit": UNIT, "cores": nt_cpu, "kind": "oracle",
            "sample": (f"oracle on {x_rows} of {R} X rows (Gram, h) and {w_rows} of {n} W rows "
                       f"({q.mode} sweep + error), the factor of the full {k} x {k} Hessian, "
                       f"{nt_cpu} threads; times scaled to the full workload ({d['h_s']:.1f} s "
                       f"+ {d['quant_s']:.1f} s measured)")}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        reference_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
