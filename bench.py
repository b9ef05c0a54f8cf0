#!/usr/bin/env python
"""Benchmark of the QAM-W codec hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Workload: one Llama-7B-shaped 4096x4096 bf16 weight matrix, Student-t(5) x 0.02,
lognormal(0,1) activation statistic with 1% outlier channels x20, alpha 0.5,
Hadamard block 128, K = 2048 codebook (~5.5 bpw).  All inputs are seeded and
synthetic (no checkpoints or datasets).

One step = the whole per-matrix hot path, each stage one C-ABI call:
  channel scales -> pair calibration (eq. 1) -> row encode (steps 1-6)
  -> decode to BF16 -> fused decode-GEMV (batch 1).
The K=2048 codebook (Lloyd, 2^20 samples, 50 iterations) and its prefilter
table are per-codec constants, built once per run and timed on their own.

Timing: CUDA events on the launching stream around each stage; the L2 (126 MB)
is flushed before every step (256 MB written, then another 256 MB read, so that
no write-back of the flush itself falls in the timed region), outside the events;
K steps are bracketed by barrier + synchronize; multi-GPU numbers are the max
over ranks.  Under torchrun each rank encodes its own matrix (weak scaling,
no data-path collective).  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode BF16 GB/s, encode Mweights/s, decode-GEMV GB/s; % HBM/FP32 roofline"
WORKLOAD = "4096x4096 bf16 Student-t(5)x0.02 weight matrix, K=2048 (bits 11), block 128, alpha 0.5"
D_OUT = D_IN = 4096
BITS, BLOCK, ALPHA = 11, 128, 0.5
TRAIN_N, TRAIN_ITERS = 1 << 20, 50
GEMV_BATCH = 1
L2_FLUSH_BYTES = 256 << 20
FP32_LANES_PER_SM = 128
SMS = 148

# DRAM bytes (read + write) of one k_encode launch on this workload, from one
# ncu capture (profiles/k_encode_4096x4096_k2048.md), valid while the encoder's
# sources hash to the recorded sha256; otherwise the roofline reports traffic
# null.
ENCODE_TRAFFIC = {"bytes": 35311616 + 4608,
                  "sha256": "1f7e056fda94e64066c0105216993430be7fcc058e375719dcb48c9b4913154f"}
ENCODE_SOURCES = ("vector_quantization_codec_b200/csrc/encode.cu",
                  "vector_quantization_codec_b200/csrc/common.cuh",
                  "vector_quantization_codec_b200/csrc/launch.cuh")


def sources_sha256(paths) -> str:
    import hashlib
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def encode_traffic():
    if ENCODE_TRAFFIC["bytes"] is None:
        return None
    return ENCODE_TRAFFIC["bytes"] if sources_sha256(ENCODE_SOURCES) == ENCODE_TRAFFIC["sha256"] else None


# ------------------------------------------------------------------ host logic

def rank_env() -> tuple[int, int, int]:
    """(rank, world_size, local_rank) from the torchrun environment (1 GPU default)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def rank_seed(rank: int) -> int:
    """Each rank encodes its own matrix: seeds differ per rank (weak scaling)."""
    return 1000 + rank


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over the process group (identity at world 1)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def algorithmic_bytes(d_out: int, d_in: int, bits: int, batch: int) -> dict:
    """Bytes each stage must move at minimum (inputs read once, outputs written once).

    decode:  packed indices + binary16 r, sigma, s + fp32 codebook + BF16 output.
    gemv:    packed indices + binary16 r, sigma, s + codebook + x (bf16) + y (bf16).
    encode:  W (bf16) + s, sigma, codebook in + packed indices + r out.
    """
    K = 1 << bits
    rb = ((d_in // 2) * bits + 127) // 128 * 16
    side = 2 * d_out + 2 * (d_in // 2) + 2 * d_in + 8 * K
    packed = d_out * rb
    return dict(
        decode=packed + side + 2 * d_out * d_in,
        gemv=packed + side + 2 * batch * d_in + 2 * batch * d_out,
        encode=2 * d_out * d_in + side + packed,
    )


def encode_flops(d_out: int, d_in: int, block: int, candidates: int) -> float:
    """fp32 operations of the row encoder (one FMA = 2).

    Per pair: channel scale 2, sum of squares 4, Hadamard butterflies
    2 log2(block), normalisation 4, grid cell 4; per candidate codeword
    evaluated (|c|^2 - 2 p.c, two FMAs) 4.  `candidates` is the total number of
    codewords the kernel scored for this matrix (counted on the device)."""
    import math
    pairs = d_out * d_in // 2
    per_pair = 2 + 4 + 2 * math.log2(block) + 4 + 4
    return pairs * per_pair + 4.0 * candidates


def fp32_peak_tflops(sm_mhz: float, sms: int = SMS) -> float:
    """FP32 FMA peak: SMs x 128 lanes x 2 flops x clock."""
    return sms * FP32_LANES_PER_SM * 2 * sm_mhz * 1e6 / 1e12


def parse_clocks(csv_text: str) -> dict:
    """Median SM clock under load, max clock and the throttle reasons seen, from
    `nvidia-smi --query-gpu=index,clocks.sm,clocks.max.sm,power.draw,
    clocks_event_reasons.active,...hw_slowdown,...hw_thermal_slowdown,
    ...sw_thermal_slowdown,...sw_power_cap --format=csv` samples."""
    sm, smax, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in csv_text.strip().splitlines():
        f = [x.strip() for x in line.split(",")]
        if len(f) < 9 or not f[1].split()[0].isdigit():
            continue
        sm.append(float(f[1].split()[0]))
        smax.append(float(f[2].split()[0]))
        for name, v in zip(names, f[5:9]):
            if v.lower().startswith("active"):
                reasons.add(name)
    if not sm:
        return dict(sm_mhz=None, sm_max_mhz=None, reasons=[], samples=0)
    loaded = [v for v in sm if v > 0.5 * max(sm)] or sm
    return dict(sm_mhz=statistics.median(loaded), sm_max_mhz=max(smax), reasons=sorted(reasons),
                samples=len(sm))


class ClockSampler:
    """nvidia-smi sampling (every 100 ms) of one GPU during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = ""

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()
        return False

    def summary(self) -> dict:
        return parse_clocks(self.out)


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm_gbs=6650.0, source="fallback")


# ------------------------------------------------------------------ GPU arm

def make_inputs(seed: int):
    from vector_quantization_codec_b200 import synth
    W = synth.student_t_weights(D_OUT, D_IN, seed)
    act = synth.act_stat_lognormal(D_IN, seed)
    x = synth.gemv_x(GEMV_BATCH, D_IN, seed)
    return W, act, x


def run_gpu(args) -> dict | None:
    import torch
    import torch.distributed as dist

    from vector_quantization_codec_b200 import qamw, synth

    rank, world, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    stream = torch.cuda.current_stream()

    # ---- per-codec constants: codebook (Lloyd on N(0, I_2)) and prefilter table
    K = 1 << BITS
    samples = torch.from_numpy(synth.circular_gaussian_samples(TRAIN_N, seed=7)).to(dev)
    codebook = torch.empty((K, 2), dtype=torch.float32, device=dev)
    distortion = torch.empty(TRAIN_ITERS, dtype=torch.float64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    qamw.qamw_train_codebook(samples, BITS, TRAIN_ITERS, codebook, distortion, status=status)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    qamw.qamw_train_codebook(samples, BITS, TRAIN_ITERS, codebook, distortion, status=status)
    t1.record(stream)
    prefilter = qamw.qamw_build_prefilter(codebook, BITS)
    torch.cuda.synchronize()
    train_ms = t0.elapsed_time(t1)

    # ---- per-rank matrix, resident in HBM
    W_np, act_np, x_np = make_inputs(rank_seed(rank))
    W = torch.from_numpy(W_np).to(torch.bfloat16).to(dev)
    act = torch.from_numpy(act_np).to(dev)
    x = torch.from_numpy(x_np).to(torch.bfloat16).to(dev)
    m = qamw.EncodedMatrix.empty(D_OUT, D_IN, BLOCK, BITS, codebook, 0, prefilter)
    ws_cal = torch.empty(qamw.qamw_workspace_bytes(qamw.QAMW_OP_CALIBRATE, D_OUT, D_IN, BITS),
                         dtype=torch.uint8, device=dev)
    ws_gemv = torch.empty(qamw.qamw_workspace_bytes(qamw.QAMW_OP_GEMV, D_OUT, D_IN, BITS,
                                                    GEMV_BATCH), dtype=torch.uint8, device=dev)
    W_hat = torch.empty((D_OUT, D_IN), dtype=torch.bfloat16, device=dev)
    y = torch.empty((GEMV_BATCH, D_OUT), dtype=torch.bfloat16, device=dev)
    # L2 flush: write one buffer larger than L2, then read another, so that the
    # written lines are evicted (and written back) before the timed region and
    # L2 holds only clean lines of an unrelated buffer when the step starts
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        flush.fill_(1.0)
        return flush_rd.sum()

    stages = ["scales", "calibrate", "encode", "decode", "gemv"]

    # one step: the five C-ABI calls, each on the current stream (the capture
    # stream while a graph is recorded)
    stage_calls = [
        lambda: qamw.qamw_channel_scales(D_IN, act, ALPHA, m.chan_scale, status=status),
        lambda: qamw.qamw_calibrate_sigma(W, m, workspace=ws_cal, status=status),
        lambda: qamw.qamw_encode_rows(W, m, status=status),
        lambda: qamw.qamw_decode(m, W_hat, status=status),
        lambda: qamw.qamw_decode_gemv(m, x, y, workspace=ws_gemv, status=status),
    ]

    def step():
        for call in stage_calls:
            call()

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()
    if status.item() != 0:
        raise RuntimeError(f"status flags after warm-up: {qamw.status_string(status.item())}")

    # candidate codewords the encoder scores on this matrix (for the flop count)
    cand = torch.zeros(1, dtype=torch.int64, device=dev)
    qamw.qamw_encode_rows(W, m, status=status, stream=stream, candidates=cand)
    torch.cuda.synchronize()
    candidates = int(cand.item())

    # the step and each stage as CUDA graphs of the same C-ABI calls (device
    # time; the host only replays); the L2 flush stays outside the events
    torch.cuda.synchronize()
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        step()
    g_stage = []
    for call in stage_calls:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call()
        g_stage.append(g)
    for _ in range(args.warmup):
        flush_l2()
        g_step.replay()
    torch.cuda.synchronize()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        wall0 = time.perf_counter()
        for k in range(args.steps):
            flush_l2()
            ev[k][0].record(stream)
            g_step.replay()
            ev[k][1].record(stream)
        torch.cuda.synchronize()
        wall1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    mean_step = sum(step_ms) / len(step_ms)
    mean_step_max = max_over_ranks(mean_step, world, dev)
    # each stage alone (after the same flush), for the breakdown
    stage_ms = {s: [] for s in stages}
    for s, g in zip(stages, g_stage):
        for k in range(args.steps):
            flush_l2()
            ev[k][0].record(stream)
            g.replay()
            ev[k][1].record(stream)
        torch.cuda.synchronize()
        stage_ms[s] = [a.elapsed_time(b) for a, b in ev]
    mean_stage = {s: sum(v) / len(v) for s, v in stage_ms.items()}

    # ---- end to end through the public API with host buffers
    e2e = run_e2e(args, W_np, act_np, x_np, m, ws_cal, ws_gemv, W_hat, y, status, stream, world, dev)

    if status.item() != 0:
        raise RuntimeError(f"status flags: {qamw.status_string(status.item())}")
    clocks = clk.summary()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    peaks = measured_peaks()
    hbm = peaks["hbm_gbs"]
    ab = algorithmic_bytes(D_OUT, D_IN, BITS, GEMV_BATCH)
    weights = D_OUT * D_IN
    sm_mhz = clocks["sm_mhz"] or 1965.0
    flops = encode_flops(D_OUT, D_IN, BLOCK, candidates)
    comp = {
        "scales": dict(ms=mean_stage["scales"]),
        "calibrate": dict(ms=mean_stage["calibrate"], rows=1024),
        "encode": dict(ms=mean_stage["encode"],
                       Mweights_per_s=weights / (mean_stage["encode"] * 1e-3) / 1e6,
                       fp32_tflops=flops / (mean_stage["encode"] * 1e-3) / 1e12,
                       frac_fp32_at_max_clock=flops / (mean_stage["encode"] * 1e-3) / 1e12 /
                       fp32_peak_tflops(1965.0),
                       frac_fp32_at_run_clock=flops / (mean_stage["encode"] * 1e-3) / 1e12 /
                       fp32_peak_tflops(sm_mhz),
                       candidates_per_pair=candidates / (weights / 2),
                       hbm_floor_frac=ab["encode"] / (mean_stage["encode"] * 1e-3) / 1e9 / hbm),
        "decode": dict(ms=mean_stage["decode"],
                       GB_per_s=ab["decode"] / (mean_stage["decode"] * 1e-3) / 1e9,
                       frac_hbm=ab["decode"] / (mean_stage["decode"] * 1e-3) / 1e9 / hbm),
        "decode_gemv": dict(ms=mean_stage["gemv"], batch=GEMV_BATCH,
                            GB_per_s=ab["gemv"] / (mean_stage["gemv"] * 1e-3) / 1e9,
                            frac_hbm=ab["gemv"] / (mean_stage["gemv"] * 1e-3) / 1e9 / hbm),
        "train": dict(ms=train_ms, samples=TRAIN_N, iters=TRAIN_ITERS, K=K,
                      note="per-codec constant, outside the step"),
    }
    dominant = max(["calibrate", "encode", "decode", "gemv"], key=lambda s: mean_stage[s])
    if dominant == "encode":
        # the encoder's bound is the larger of bytes / HBM and algorithmic
        # flops / FP32 peak; for this workload the bytes (see components)
        t_bytes = ab["encode"] / (hbm * 1e9)
        t_flops = flops / (fp32_peak_tflops(sm_mhz) * 1e12)
        if t_bytes >= t_flops:
            achieved = ab["encode"] / (mean_stage["encode"] * 1e-3) / 1e9
            roofline = dict(bound="hbm", kernel="k_encode (qamw_encode_rows)", achieved=achieved,
                            peak=hbm, unit="GB/s", frac=achieved / hbm,
                            traffic=encode_traffic(),
                            peak_source=peaks["source"] + " MEASURED_PEAKS.json hbm_gbs")
        else:
            achieved = flops / (mean_stage["encode"] * 1e-3) / 1e12
            peak = fp32_peak_tflops(sm_mhz)
            roofline = dict(bound="alu", kernel="k_encode (qamw_encode_rows)", achieved=achieved,
                            peak=peak, unit="TFLOP/s", frac=achieved / peak,
                            traffic=encode_traffic(),
                            peak_source=f"148 SM x 128 FP32 lanes x 2 x {sm_mhz:.0f} MHz (run clock)")
    else:
        key = {"decode": "decode", "gemv": "gemv", "calibrate": "encode"}[dominant]
        achieved = ab[key] / (mean_stage[dominant] * 1e-3) / 1e9
        roofline = dict(bound="hbm", kernel=dominant, achieved=achieved, peak=hbm, unit="GB/s",
                        frac=achieved / hbm, traffic=None,
                        peak_source=peaks["source"] + " MEASURED_PEAKS.json hbm_gbs")
    value = world * weights / (mean_step_max * 1e-3) / 1e6
    out = {
        "metric": METRIC,
        "value": value,
        "unit": "Mweights/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": mean_step_max,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded Student-t weights, lognormal activation statistics)",
        "config": {"workload": WORKLOAD, "d_out": D_OUT, "d_in": D_IN, "bits": BITS,
                   "block": BLOCK, "alpha": ALPHA, "gemv_batch": GEMV_BATCH,
                   "step": "scales+calibrate+encode_rows+decode+decode_gemv",
                   "l2": "flushed before every step (256 MB written, then another 256 MB read), outside the timed events",
                   "timing": "CUDA events around a CUDA-graph replay of the step's five C-ABI calls",
                   "parallelism": f"{world} independent matrices (one per GPU)"},
        "components": comp,
        "roofline": roofline,
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": args.steps * LAUNCHES_PER_STEP,
        "wall_s_timed": wall1 - wall0,
    }
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = run_cpu_baseline(args.cpu_rows)
        out["cpu_baseline"] = cpu
    return out


# kernels one step launches: scales 1, calibrate 3 (rows, extension, finish),
# encode 1, decode 1, decode-GEMV 1 (batch 1)
LAUNCHES_PER_STEP = 7


def run_e2e(args, W_np, act_np, x_np, m, ws_cal, ws_gemv, W_hat, y, status, stream, world, dev):
    """Same step through the public API from pinned host buffers: H2D of W, the
    statistic and x; D2H of the encoded matrix (indices, r, sigma, s) and y."""
    import torch

    from vector_quantization_codec_b200 import qamw
    Wh = torch.from_numpy(W_np).to(torch.bfloat16).pin_memory()
    ah = torch.from_numpy(act_np).pin_memory()
    xh = torch.from_numpy(x_np).to(torch.bfloat16).pin_memory()
    Wd = torch.empty_like(Wh, device=dev)
    ad = torch.empty_like(ah, device=dev)
    xd = torch.empty_like(xh, device=dev)
    outs = [m.packed, m.row_norm, m.sigma, m.chan_scale, y]
    outs_h = [torch.empty_like(t, device="cpu").pin_memory() for t in outs]
    h2d = sum(t.numel() * t.element_size() for t in (Wh, ah, xh))
    d2h = sum(t.numel() * t.element_size() for t in outs)

    def step():
        Wd.copy_(Wh, non_blocking=True)
        ad.copy_(ah, non_blocking=True)
        xd.copy_(xh, non_blocking=True)
        qamw.qamw_channel_scales(D_IN, ad, ALPHA, m.chan_scale, status=status, stream=stream)
        qamw.qamw_calibrate_sigma(Wd, m, workspace=ws_cal, status=status, stream=stream)
        qamw.qamw_encode_rows(Wd, m, status=status, stream=stream)
        qamw.qamw_decode(m, W_hat, status=status, stream=stream)
        qamw.qamw_decode_gemv(m, xd, y, workspace=ws_gemv, status=status, stream=stream)
        for hd, dd in zip(outs_h, outs):
            hd.copy_(dd, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms, world, dev)
    return dict(value=world * D_OUT * D_IN / (ms * 1e-3) / 1e6, unit="Mweights/s",
                ms_per_step=ms, h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h)


# ------------------------------------------------------------------ CPU oracle

def oracle_step_sample(rows: int, seed: int = 1000) -> dict:
    """The oracle on a bounded sample of the same workload: eq. (1) over the
    matrix's 1024 calibration rows (a fixed per-matrix cost), then encode,
    decode and GEMV of `rows` rows; the full-matrix step time is extrapolated
    as t_cal + t_rows * 4096 / rows."""
    import numpy as np

    import oracle
    from vector_quantization_codec_b200 import synth
    import torch
    W, act, x = make_inputs(seed)
    W64 = torch.from_numpy(W).to(torch.bfloat16).double().numpy()
    x64 = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    # a codebook of the same size (the exhaustive search costs the same for any values)
    cb = np.asarray(synth.circular_gaussian_samples(1 << BITS, seed=7), dtype=np.float64)
    threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    s = oracle.channel_scales(act.astype(np.float64), D_IN, ALPHA)
    sig = oracle.calibrate_sigma(W64[:1024], BLOCK, s)
    t1 = time.perf_counter()
    enc = oracle.encode(W64[:rows], BITS, BLOCK, cb, s_half=s, sigma_half=sig, threads=threads)
    What = oracle.decode(enc, cb, threads=threads)
    oracle.gemv(What, x64, threads=threads)
    t2 = time.perf_counter()
    full_s = (t1 - t0) + (t2 - t1) * D_OUT / rows
    return dict(value=D_OUT * D_IN / full_s / 1e6, unit="Mweights/s", cores=threads,
                kind="oracle", seconds=t2 - t0,
                sample=f"eq.(1) on 1024 rows ({t1 - t0:.1f} s) + encode/decode/GEMV of "
                       f"{rows} of 4096 rows ({t2 - t1:.1f} s), extrapolated to the matrix")


def run_cpu_baseline(rows: int) -> dict:
    return oracle_step_sample(rows)


def run_reference(args) -> dict | None:
    rank, world, _ = rank_env()
    if rank != 0:
        return None
    vals = []
    for _ in range(args.warmup):
        oracle_step_sample(args.cpu_rows // 4 or 8)
    for _ in range(args.steps):
        vals.append(oracle_step_sample(args.cpu_rows // 4 or 8))
    v = statistics.mean(r["value"] for r in vals)
    cpu = dict(vals[-1])
    cpu["value"] = v
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "Mweights/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": D_OUT * D_IN / (v * 1e6) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "step": "scales+calibrate+encode+decode+gemv (oracle)"},
        "cpu_baseline": cpu,
        "e2e": {"value": v, "unit": "Mweights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_single_stage(args) -> dict:
    """One stage alone on a d_out = args.rows x 4096 matrix (same distributions),
    for kernel profiling and sweeps: `warmup` untimed then `steps` timed calls."""
    import torch

    from vector_quantization_codec_b200 import qamw, synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    rows = args.rows
    K = 1 << BITS
    samples = torch.from_numpy(synth.circular_gaussian_samples(TRAIN_N, seed=7)).to(dev)
    codebook = torch.empty((K, 2), dtype=torch.float32, device=dev)
    iters = TRAIN_ITERS if args.only != "train" else 1
    if args.only != "train":
        qamw.qamw_train_codebook(samples, BITS, iters, codebook)
    prefilter = qamw.qamw_build_prefilter(codebook, BITS) if args.only != "train" else None
    g = synth.rng(args.seed, 9)
    W = torch.from_numpy((g.standard_t(5.0, size=(rows, D_IN)) * 0.02).astype("float32"))
    W = W.to(torch.bfloat16).to(dev)
    act = torch.from_numpy(synth.act_stat_lognormal(D_IN, args.seed)).to(dev)
    x = torch.from_numpy(synth.gemv_x(args.batch, D_IN, args.seed)).to(torch.bfloat16).to(dev)
    m = qamw.EncodedMatrix.empty(rows, D_IN, BLOCK, BITS, codebook, 0, prefilter)
    if args.only != "train":
        qamw.qamw_encode(W, m, act, ALPHA)
    ws_cal = torch.empty(qamw.qamw_workspace_bytes(qamw.QAMW_OP_CALIBRATE, rows, D_IN, BITS),
                         dtype=torch.uint8, device=dev)
    ws_g = torch.empty(qamw.qamw_workspace_bytes(qamw.QAMW_OP_GEMV, rows, D_IN, BITS, args.batch),
                       dtype=torch.uint8, device=dev)
    W_hat = torch.empty((rows, D_IN), dtype=torch.bfloat16, device=dev)
    y = torch.empty((args.batch, rows), dtype=torch.bfloat16, device=dev)
    fns = {
        "encode": lambda: qamw.qamw_encode_rows(W, m),
        "calibrate": lambda: qamw.qamw_calibrate_sigma(W, m, workspace=ws_cal),
        "decode": lambda: qamw.qamw_decode(m, W_hat),
        "gemv": lambda: qamw.qamw_decode_gemv(m, x, y, workspace=ws_g),
        "train": lambda: qamw.qamw_train_codebook(samples, BITS, 1, codebook),
    }
    fn = fns[args.only]
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if args.eager:
        e0.record()
        for _ in range(args.steps):
            fn()
        e1.record()
    else:
        # `steps` back-to-back calls captured in one CUDA graph: device time only,
        # no host launch overhead between calls (the warm-up filled the library's
        # launch-shape caches, so capture sees launches only)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(args.steps):
                fn()
        graph.replay()
        torch.cuda.synchronize()
        e0.record()
        graph.replay()
        e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    ab = algorithmic_bytes(rows, D_IN, BITS, args.batch)
    key = {"encode": "encode", "calibrate": "encode", "decode": "decode", "gemv": "gemv"}.get(args.only)
    out = dict(stage=args.only, rows=rows, d_in=D_IN, batch=args.batch, ms=ms,
               timing="eager" if args.eager else "cuda graph of back-to-back calls",
               Mweights_per_s=rows * D_IN / (ms * 1e-3) / 1e6)
    if key:
        out["GB_per_s"] = ab[key] / (ms * 1e-3) / 1e9
    return out


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="qamw", choices=["qamw", "reference"])
    ap.add_argument("--cpu-rows", type=int, default=64, help="rows of the CPU oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["encode", "calibrate", "decode", "gemv", "train"],
                    help="profiling mode: time one stage alone (no step, no JSON contract)")
    ap.add_argument("--rows", type=int, default=16384, help="--only: rows of the d_in=4096 matrix")
    ap.add_argument("--batch", type=int, default=1, help="--only gemv: batch columns")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--eager", action="store_true", help="--only: time eager calls, not a graph")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.only:
        print(json.dumps(run_single_stage(args)), flush=True)
        return 0
    out = run_reference(args) if args.impl == "reference" else run_gpu(args)
    if out is not None:
        print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
