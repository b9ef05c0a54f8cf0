#!/usr/bin/env python
"""Benchmark of the QAM-W codec hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Workload (the step): every linear weight of 32 Llama-2-7B-shaped layers -- per
layer q, k, v, o (4096x4096), gate, up (11008x4096) and down (4096x11008), 224
matrices and 6.48e9 weights -- bf16 Student-t(5) x 0.02, a lognormal(0,1)
activation statistic with 1% outlier channels x20 per layer input, alpha 0.5,
Hadamard block 128, K = 2048 codebook (~5.5 bpw).  All inputs are seeded and
synthetic (no checkpoints or datasets).

One step = the whole hot path over all 224 matrices, each stage one C-ABI call
per matrix, in four phases:
  channel scales + pair calibration (eq. 1)  ->  row encode (section 3.1)
  ->  decode to BF16 (section 3.2)  ->  fused decode-GEMV at batch 1.
The K=2048 codebook (Lloyd, 2^20 samples, 50 iterations) and its search table
are per-codec constants, built once per run and timed on their own.

Timing: each phase is one CUDA graph of its calls; CUDA events on the launching
stream bracket every phase of every step, so the per-phase times (and the
rooflines) are measured inside the timed region.  The step's inputs (12.95 GB of
weights, 4.45 GB of indices) are far larger than the 126 MB L2, and each phase
streams all 224 matrices, so no phase reads what the one before left in L2; no
flush is needed.  K steps are bracketed by barrier + synchronize; multi-GPU
numbers are the max over ranks (each rank encodes its own copy of the workload
with its own seeds: weak scaling, no data-path collective).

Also measured, outside the step and reported under `components`:
  * decode-GEMV on the 11008x4096 and 4096x11008 matrices at batch 1, 4 and 16,
    cycling through the 32 layers' gate (resp. down) matrices;
  * the prefill-size decode-GEMM (tensor cores) on the same matrices at 64 and
    128 tokens;
  * the 3.5 bpw variant: every linear weight of 40 13B-shaped layers with a
    K = 128 codebook, encode and decode, and the polar amplitude x phase
    quantiser of the same K as the comparison path.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode BF16 GB/s, encode Mweights/s, decode-GEMV GB/s; % HBM/FP32 roofline"
BITS, BLOCK, ALPHA = 11, 128, 0.5
BITS_35 = 7
LAYERS, LAYERS_13B = 32, 40
WL_7B, WL_13B = 3, 4  # workload ids in the input seeds
TRAIN_N, TRAIN_ITERS = 1 << 20, 50
GEMV_BATCHES = (1, 4, 16)
GEMM_TOKENS = (64, 128)
FP32_LANES_PER_SM = 128
SMS = 148

# DRAM bytes (read + write) of one k_encode launch on a 4096x4096 bf16 matrix
# (K = 2048), from one ncu capture, valid while the encoder's sources hash to
# the recorded sha256 (otherwise the roofline reports traffic null).  The
# traffic of an average launch of the workload is this figure scaled by the
# weights the launch encodes (encode traffic grows in proportion to the rows).
ENCODE_TRAFFIC = {"bytes": 35317760 + 1024, "weights": 4096 * 4096,
                  "sha256": "9f222a2a7f678e3f471d60039db22e988fe8a982d7ba3f8ceabc830460b41e8e"}
ENCODE_SOURCES = ("vector_quantization_codec_b200/csrc/encode.cu",
                  "vector_quantization_codec_b200/csrc/common.cuh",
                  "vector_quantization_codec_b200/csrc/launch.cuh")


def sources_sha256(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def encode_traffic(weights_per_launch: float):
    """ncu DRAM bytes of an average encode launch, or None when stale."""
    if ENCODE_TRAFFIC["bytes"] is None or sources_sha256(ENCODE_SOURCES) != ENCODE_TRAFFIC["sha256"]:
        return None
    return ENCODE_TRAFFIC["bytes"] * weights_per_launch / ENCODE_TRAFFIC["weights"]


# ------------------------------------------------------------------ host logic

def rank_env() -> tuple[int, int, int]:
    """(rank, world_size, local_rank) from the torchrun environment (1 GPU default)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def rank_seed(rank: int) -> int:
    """Each rank encodes its own copy of the workload: seeds differ per rank."""
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


def workload_matrices(layers: int = LAYERS, rank: int = 0, shapes: str = "7b") -> list[dict]:
    """The matrices of the workload (layer-major), with the seeds of their
    weights and activation statistics for this rank."""
    from vector_quantization_codec_b200 import synth
    if shapes == "7b":
        mats = synth.layer_matrices(synth.llama2_7b_layer_shapes(), layers, WL_7B)
    else:
        mats = synth.layer_matrices(synth.llama_13b_layer_shapes(), layers, WL_13B)
    for m in mats:
        m["w_seed"] = (rank_seed(rank),) + m["w_seed"]
        m["act_seed"] = (rank_seed(rank),) + m["act_seed"]
    return mats


def make_inputs(seed: int, d_out: int = 64, d_in: int = 4096):
    """Host inputs of one small matrix of the workload's distributions (the
    multi-rank host test checks that ranks draw different inputs)."""
    from vector_quantization_codec_b200 import synth
    W = synth.student_t_weights(d_out, d_in, seed)
    act = synth.act_stat_lognormal(d_in, seed)
    x = synth.gemv_x(1, d_in, seed)
    return W, act, x


def row_bytes(d_in: int, bits: int) -> int:
    return ((d_in // 2) * bits + 127) // 128 * 16


def algorithmic_bytes(d_out: int, d_in: int, bits: int, batch: int) -> dict:
    """Bytes each stage must move at minimum (inputs read once, outputs written once).

    decode:  packed indices + binary16 r, sigma, s + fp32 codebook + BF16 output.
    gemv:    packed indices + binary16 r, sigma, s + codebook + x (bf16) + y (bf16).
    encode:  W (bf16) + s, sigma, codebook in + packed indices + r out.
    """
    K = 1 << bits
    side = 2 * d_out + 2 * (d_in // 2) + 2 * d_in + 8 * K
    packed = d_out * row_bytes(d_in, bits)
    return dict(
        decode=packed + side + 2 * d_out * d_in,
        gemv=packed + side + 2 * batch * d_in + 2 * batch * d_out,
        encode=2 * d_out * d_in + side + packed,
    )


def total_bytes(mats: list[dict], bits: int, batch: int = 1) -> dict:
    out = dict(decode=0, gemv=0, encode=0)
    for m in mats:
        for k, v in algorithmic_bytes(m["d_out"], m["d_in"], bits, batch).items():
            out[k] += v
    return out


def encode_flops(d_out: int, d_in: int, block: int, candidates: int) -> float:
    """fp32 operations of the row encoder (one FMA = 2).

    Per pair: channel scale 2, sum of squares 4, Hadamard butterflies
    2 log2(block), normalisation 4, grid cell 4; per candidate codeword
    evaluated (|c|^2 - 2 p.c, two FMAs) 4.  `candidates` is the total number of
    codewords the kernel scored for these matrices (counted on the device)."""
    import math
    pairs = d_out * d_in // 2
    per_pair = 2 + 4 + 2 * math.log2(block) + 4 + 4
    return pairs * per_pair + 4.0 * candidates


def fp32_peak_tflops(sm_mhz: float, sms: int = SMS) -> float:
    """FP32 FMA peak: SMs x 128 lanes x 2 flops x clock."""
    return sms * FP32_LANES_PER_SM * 2 * sm_mhz * 1e6 / 1e12


def encoder_roofline(bytes_: float, flops: float, ms: float, hbm_gbs: float, sm_mhz: float) -> dict:
    """The encoder's bound is the larger of bytes / HBM and flops / FP32 peak."""
    t_bytes = bytes_ / (hbm_gbs * 1e9)
    t_flops = flops / (fp32_peak_tflops(sm_mhz) * 1e12)
    if t_bytes >= t_flops:
        achieved = bytes_ / (ms * 1e-3) / 1e9
        return dict(bound="hbm", achieved=achieved, peak=hbm_gbs, unit="GB/s",
                    frac=achieved / hbm_gbs)
    achieved = flops / (ms * 1e-3) / 1e12
    peak = fp32_peak_tflops(sm_mhz)
    return dict(bound="alu", achieved=achieved, peak=peak, unit="TFLOP/s", frac=achieved / peak)


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
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p.get("bf16_tflops", 1590.0)),
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, source="fallback")


def workload_config(layers: int, world: int) -> dict:
    """`config` of the JSON line (the same for both arms)."""
    return {"workload": f"Llama-2-7B-shaped linear weights of {layers} layers "
                        f"({7 * layers} matrices: q,k,v,o 4096x4096, gate,up 11008x4096, "
                        f"down 4096x11008), bf16 Student-t(5)x0.02, K=2048 (bits 11), "
                        f"block 128, alpha 0.5",
            "layers": layers, "matrices": 7 * layers,
            "weights": sum(m["d_out"] * m["d_in"] for m in workload_matrices(layers)),
            "bits": BITS, "block": BLOCK, "alpha": ALPHA, "gemv_batch": 1,
            "step": "per matrix: channel scales, eq.(1) calibration, row encode, decode to "
                    "BF16, decode-GEMV batch 1 (phases over all matrices)",
            "parallelism": f"{world} independent replicas of the workload (one per GPU)"}


# ------------------------------------------------------------------ GPU arm

class Workload:
    """Device buffers of one workload: weights, statistics, encoded matrices,
    decoded outputs and GEMV vectors, all resident in HBM."""

    def __init__(self, mats, bits, codebook, prefilter, dev, gemv_batch=1, polar_codebook=None):
        import torch

        from vector_quantization_codec_b200 import qamw, synth
        self.mats = mats
        self.bits = bits
        self.W, self.act, self.m, self.out, self.x, self.y, self.m_polar = [], [], [], [], [], [], []
        for i, d in enumerate(mats):
            W = synth.student_t_weights_device(d["d_out"], d["d_in"], d["w_seed"], dev)
            self.W.append(W)
            self.act.append(torch.from_numpy(synth.act_stat_for(d["act_seed"], d["d_in"])).to(dev))
            m = qamw.EncodedMatrix.empty(d["d_out"], d["d_in"], BLOCK, bits, codebook, i, prefilter)
            self.m.append(m)
            self.out.append(torch.empty((d["d_out"], d["d_in"]), dtype=torch.bfloat16, device=dev))
            xs = synth.gemv_x(gemv_batch, d["d_in"], seed=1000 * d["layer"] + synth.LAYER_INPUT[d["name"]])
            self.x.append(torch.from_numpy(xs).to(torch.bfloat16).to(dev))
            self.y.append(torch.empty((gemv_batch, d["d_out"]), dtype=torch.bfloat16, device=dev))
            if polar_codebook is not None:
                # same side values (s, sigma), own indices and row norms
                mp = qamw.EncodedMatrix(d["d_out"], d["d_in"], BLOCK, bits, i,
                                        torch.empty_like(m.packed), torch.empty_like(m.row_norm),
                                        m.sigma, m.chan_scale, polar_codebook, None)
                self.m_polar.append(mp)
        self.ws_cal = torch.empty(qamw.qamw_calibrate_many_workspace_bytes(self.m), dtype=torch.uint8,
                                  device=dev)
        gw = max(qamw.qamw_workspace_bytes(qamw.QAMW_OP_GEMV, d["d_out"], d["d_in"], bits, 16)
                 for d in mats)
        self.ws_gemv = torch.empty(gw, dtype=torch.uint8, device=dev)
        # the batch-1 products of all matrices in one list call, in d_in order
        # (matrices of one d_in share launches)
        self.gemv_order = sorted(range(len(mats)), key=lambda i: mats[i]["d_in"])
        self.ws_gemv_many = torch.empty(
            max(16, qamw.qamw_decode_gemv_many_workspace_bytes([self.m[i] for i in self.gemv_order])),
            dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.encode_streams = []

    @property
    def weights(self) -> int:
        return sum(d["d_out"] * d["d_in"] for d in self.mats)

    # the calls of each stage, on the current stream
    def calibrate(self, stream=None):
        # channel scales and eq. (1) of every matrix in one call
        from vector_quantization_codec_b200 import qamw
        qamw.qamw_calibrate_many(self.W, self.m, self.act, ALPHA, workspace=self.ws_cal,
                                 status=self.status, stream=stream)

    def encode(self, stream=None, candidates=None):
        # the matrices' encodes are independent: with several streams they go
        # round-robin over them, so that the SMs a launch's last rows leave idle
        # take the CTAs of the next matrix (one CTA fills an SM)
        import torch

        from vector_quantization_codec_b200 import qamw
        if not self.encode_streams or stream is not None:
            for W, m in zip(self.W, self.m):
                qamw.qamw_encode_rows(W, m, status=self.status, stream=stream, candidates=candidates)
            return
        cur = torch.cuda.current_stream()
        for s in self.encode_streams:
            s.wait_stream(cur)
        for i, (W, m) in enumerate(zip(self.W, self.m)):
            s = self.encode_streams[i % len(self.encode_streams)]
            with torch.cuda.stream(s):
                qamw.qamw_encode_rows(W, m, status=self.status, stream=s, candidates=candidates)
        for s in self.encode_streams:
            cur.wait_stream(s)

    def encode_polar(self, stream=None):
        from vector_quantization_codec_b200 import qamw
        for W, m in zip(self.W, self.m_polar):
            qamw.qamw_encode_rows_polar(W, m, status=self.status, stream=stream)

    def decode(self, stream=None, polar=False):
        # one call for all matrices (one launch per 64 matrices)
        from vector_quantization_codec_b200 import qamw
        qamw.qamw_decode_many(self.m_polar if polar else self.m, self.out, status=self.status,
                              stream=stream)

    def gemv(self, stream=None):
        from vector_quantization_codec_b200 import qamw
        if self.x[0].shape[0] == 1:
            o = self.gemv_order
            qamw.qamw_decode_gemv_many([self.m[i] for i in o], [self.x[i] for i in o],
                                       [self.y[i] for i in o], workspace=self.ws_gemv_many,
                                       status=self.status, stream=stream)
            return
        for m, x, y in zip(self.m, self.x, self.y):
            qamw.qamw_decode_gemv(m, x, y, workspace=self.ws_gemv, status=self.status, stream=stream)

    def check_status(self, what: str):
        from vector_quantization_codec_b200 import qamw
        v = int(self.status.item())
        if v != 0:
            raise RuntimeError(f"status flags after {what}: {qamw.status_string(v)}")


def capture(fn):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def time_graph(g, reps: int, stream) -> float:
    """Mean device ms of one replay of g over `reps` back-to-back replays."""
    import torch
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def train_codebook(bits: int, dev):
    """Per-codec constant: Lloyd codebook on 2^20 N(0, I_2) samples, 50
    iterations, and its search table; returns (codebook, table, ms)."""
    import torch

    from vector_quantization_codec_b200 import qamw, synth
    samples = torch.from_numpy(synth.circular_gaussian_samples(TRAIN_N, seed=7)).to(dev)
    cb = torch.empty((1 << bits, 2), dtype=torch.float32, device=dev)
    dist_ = torch.empty(TRAIN_ITERS, dtype=torch.float64, device=dev)
    qamw.qamw_train_codebook(samples, bits, TRAIN_ITERS, cb, dist_)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    qamw.qamw_train_codebook(samples, bits, TRAIN_ITERS, cb, dist_)
    e1.record()
    table = qamw.qamw_build_prefilter(cb, bits)
    torch.cuda.synchronize()
    return cb, table, e0.elapsed_time(e1)


def run_gpu(args) -> dict | None:
    import torch
    import torch.distributed as dist

    rank, world, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    stream = torch.cuda.current_stream()
    peaks = measured_peaks()
    hbm = peaks["hbm_gbs"]

    codebook, table, train_ms = train_codebook(BITS, dev)
    mats = workload_matrices(args.layers, rank)
    wl = Workload(mats, BITS, codebook, table, dev)
    if args.encode_streams > 1:
        wl.encode_streams = [torch.cuda.Stream(device=dev) for _ in range(args.encode_streams)]
    weights = wl.weights
    nm = len(mats)
    torch.cuda.synchronize()

    phases = ["calibrate", "encode", "decode", "gemv"]
    calls = {"calibrate": wl.calibrate, "encode": wl.encode, "decode": wl.decode, "gemv": wl.gemv}
    # warm-up eagerly (fills the library's launch-shape caches), then capture
    for _ in range(args.warmup):
        for p in phases:
            calls[p]()
    torch.cuda.synchronize()
    wl.check_status("warm-up")
    # candidate codewords the encoder scores on these matrices (for the flop count)
    cand = torch.zeros(1, dtype=torch.int64, device=dev)
    wl.encode(candidates=cand)
    torch.cuda.synchronize()
    candidates = int(cand.item())
    graphs = {p: capture(calls[p]) for p in phases}
    for _ in range(args.warmup):
        for p in phases:
            graphs[p].replay()
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(phases) + 1)]
          for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        wall0 = time.perf_counter()
        for k in range(args.steps):
            ev[k][0].record(stream)
            for i, p in enumerate(phases):
                graphs[p].replay()
                ev[k][i + 1].record(stream)
        torch.cuda.synchronize()
        wall1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    step_ms = [e[0].elapsed_time(e[-1]) for e in ev]
    phase_ms = {p: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in ev)
                for i, p in enumerate(phases)}
    mean_step = statistics.mean(step_ms)
    mean_step_max = max_over_ranks(mean_step, world, dev)
    clocks = clk.summary()
    wl.check_status("timed steps")
    for g in graphs.values():
        del g
    graphs.clear()

    # ---- decode-GEMV on the MLP shapes at batch 1 / 4 / 16 (cycling 32 layers)
    gemv_lines = run_gemv_lines(args, wl, dev, stream, hbm)
    gemm_lines = run_gemm_lines(args, wl, dev, stream, hbm, peaks["bf16_tflops"])
    dense_context = run_dense_context(args, wl, dev, stream, hbm)
    # ---- end to end through the public API with host buffers
    e2e = run_e2e(args, wl, stream, world, dev)
    del wl
    torch.cuda.empty_cache()
    # ---- the 3.5 bpw variant on 13B shapes, joint 2-D and polar
    c35 = run_35bpw(args, dev, stream, hbm, rank) if not args.skip_35 else None

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    ab = total_bytes(mats, BITS)
    sm_mhz = clocks["sm_mhz"] or 1965.0
    flops = sum(encode_flops(d["d_out"], d["d_in"], BLOCK, 0) for d in mats) + 4.0 * candidates
    enc_ms, dec_ms, gemv_ms = phase_ms["encode"], phase_ms["decode"], phase_ms["gemv"]
    enc_roof = encoder_roofline(ab["encode"], flops, enc_ms, hbm, sm_mhz)
    comp = {
        "calibrate": dict(ms=phase_ms["calibrate"], launches=4 * ((nm + 63) // 64),
                          note="channel scales + eq.(1) over the first 1024 rows of every matrix "
                               "(qamw_calibrate_many)"),
        "encode": dict(ms=enc_ms, Mweights_per_s=weights / (enc_ms * 1e-3) / 1e6,
                       fp32_tflops=flops / (enc_ms * 1e-3) / 1e12,
                       frac_fp32_at_run_clock=flops / (enc_ms * 1e-3) / 1e12 / fp32_peak_tflops(sm_mhz),
                       frac_fp32_at_max_clock=flops / (enc_ms * 1e-3) / 1e12 / fp32_peak_tflops(1965.0),
                       hbm_GB_per_s=ab["encode"] / (enc_ms * 1e-3) / 1e9,
                       frac_hbm=ab["encode"] / (enc_ms * 1e-3) / 1e9 / hbm,
                       candidates_per_pair=candidates / (weights / 2), bound=enc_roof["bound"],
                       streams=max(1, args.encode_streams),
                       note="one qamw_encode_rows call per matrix; the calls go round-robin over "
                            "the streams (independent matrices)"),
        "decode": dict(ms=dec_ms, GB_per_s=ab["decode"] / (dec_ms * 1e-3) / 1e9,
                       frac_hbm=ab["decode"] / (dec_ms * 1e-3) / 1e9 / hbm,
                       bytes=ab["decode"]),
        "decode_gemv_b1_all": dict(ms=gemv_ms, GB_per_s=ab["gemv"] / (gemv_ms * 1e-3) / 1e9,
                                   frac_hbm=ab["gemv"] / (gemv_ms * 1e-3) / 1e9 / hbm),
        "decode_gemv_mlp": gemv_lines,
        "decode_gemm_prefill": gemm_lines,
        "gpu_context_dense_bf16": dense_context,
        "train": dict(ms=train_ms, samples=TRAIN_N, iters=TRAIN_ITERS, K=1 << BITS,
                      note="per-codec constant, outside the step"),
    }
    if c35 is not None:
        comp["bpw3.5_13b"] = c35
    # the dominant kernel of the step: the phase with the most time
    dom = max(["encode", "decode", "gemv"], key=lambda p: phase_ms[p])
    if dom == "encode":
        roofline = dict(enc_roof, kernel="k_encode (qamw_encode_rows)",
                        traffic=encode_traffic(weights / nm),
                        per_launch=(f"the encode phase's algorithmic bytes over its event time: "
                                    f"{nm} launches on {max(1, args.encode_streams)} stream(s), "
                                    f"consecutive launches overlapping at their tails"))
    else:
        key = {"decode": "decode", "gemv": "gemv"}[dom]
        achieved = ab[key] / (phase_ms[dom] * 1e-3) / 1e9
        roofline = dict(bound="hbm", kernel=dom, achieved=achieved, peak=hbm, unit="GB/s",
                        frac=achieved / hbm, traffic=None)
    roofline["peak_source"] = (peaks["source"] + " MEASURED_PEAKS.json hbm_gbs" if roofline["bound"] == "hbm"
                               else f"148 SM x 128 FP32 lanes x 2 x {sm_mhz:.0f} MHz (run clock)")
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
        "config": dict(workload_config(args.layers, world),
                       l2="inputs (12.95 GB of weights, 4.45 GB of indices) far larger than L2; "
                          "each phase streams every matrix; no flush",
                       timing="CUDA events on the launching stream around each phase (one CUDA "
                              "graph of the phase's C-ABI calls) of every step"),
        "components": comp,
        "roofline": roofline,
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": args.steps * launches_per_step(mats),
        "wall_s_timed": wall1 - wall0,
    }
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args)
    return out


# kernels of one step: per matrix, encode 1 and decode-GEMV 1 (batch 1); per
# group of 64 matrices, calibration 4 (scales, rows, extension, finish) and
# decode 1
def launches_per_step(mats) -> int:
    """Kernel launches of one step: an encoder launch per matrix; per run of up
    to 64 matrices, four of calibration and one of decoding; per run of up to 64
    matrices of one d_in, two of the batch-1 products (x_bar, then the GEMV)."""
    n = len(mats)
    runs = (n + 63) // 64
    by_din = {}
    for d in mats:
        by_din[d["d_in"]] = by_din.get(d["d_in"], 0) + 1
    gemv_runs = sum((k + 63) // 64 for k in by_din.values())
    return n + 5 * runs + 2 * gemv_runs


def run_gemv_lines(args, wl, dev, stream, hbm) -> dict:
    """decode-GEMV on the 11008x4096 (gate) and 4096x11008 (down) matrices of the
    workload at batch 1, 4 and 16: each line is one CUDA graph of the calls on
    all layers' matrices of that shape (distinct matrices, 1 GB of indices per
    pass, so each call reads its indices from HBM)."""
    import torch

    from vector_quantization_codec_b200 import qamw, synth
    lines = {}
    for name in ("gate", "down"):
        sel = [i for i, d in enumerate(wl.mats) if d["name"] == name]
        d0 = wl.mats[sel[0]]
        for b in GEMV_BATCHES:
            xs = [torch.from_numpy(synth.gemv_x(b, d0["d_in"], seed=7000 + i)).to(torch.bfloat16).to(dev)
                  for i in sel]
            ys = [torch.empty((b, d0["d_out"]), dtype=torch.bfloat16, device=dev) for _ in sel]

            def calls():
                for i, x, y in zip(sel, xs, ys):
                    qamw.qamw_decode_gemv(wl.m[i], x, y, workspace=wl.ws_gemv, status=wl.status)

            calls()
            torch.cuda.synchronize()
            g = capture(calls)
            g.replay()
            ms = time_graph(g, max(3, args.steps // 2), stream) / len(sel)
            del g
            ab = algorithmic_bytes(d0["d_out"], d0["d_in"], BITS, b)["gemv"]
            lines[f"{d0['d_out']}x{d0['d_in']}_b{b}"] = dict(
                us_per_call=ms * 1e3, GB_per_s=ab / (ms * 1e-3) / 1e9,
                frac_hbm=ab / (ms * 1e-3) / 1e9 / hbm,
                gflops=2.0 * b * d0["d_out"] * d0["d_in"] / (ms * 1e-3) / 1e9,
                matrices_cycled=len(sel))
    wl.check_status("decode-GEMV lines")
    return lines


def run_dense_context(args, wl, dev, stream, hbm) -> dict:
    """Context on the GPU, not the target: torch's dense BF16 product x @ W^T on
    the same 11008x4096 and 4096x11008 weights (BF16, 90 MB each) at the batches
    of the decode-GEMV lines and the token counts of the decode-GEMM lines, and
    a BF16 copy of the same bytes (W into a scratch buffer).  Each line is one
    CUDA graph over the 32 layers' matrices of that shape."""
    import torch

    from vector_quantization_codec_b200 import synth
    lines = {}
    for name in ("gate", "down"):
        sel = [i for i, d in enumerate(wl.mats) if d["name"] == name]
        d0 = wl.mats[sel[0]]
        wbytes = 2 * d0["d_out"] * d0["d_in"]
        for b in tuple(GEMV_BATCHES) + tuple(GEMM_TOKENS):
            xs = [torch.from_numpy(synth.gemv_x(b, d0["d_in"], seed=7000 + i)).to(torch.bfloat16).to(dev)
                  for i in sel]
            ys = [torch.empty((b, d0["d_out"]), dtype=torch.bfloat16, device=dev) for _ in sel]

            def calls():
                for i, x, y in zip(sel, xs, ys):
                    torch.matmul(x, wl.W[i].t(), out=y)

            calls()
            torch.cuda.synchronize()
            g = capture(calls)
            g.replay()
            ms = time_graph(g, max(3, args.steps // 2), stream) / len(sel)
            del g
            byts = wbytes + 2 * b * (d0["d_in"] + d0["d_out"])
            lines[f"{d0['d_out']}x{d0['d_in']}_dense_bf16_m{b}"] = dict(
                us_per_call=ms * 1e3, GB_per_s=byts / (ms * 1e-3) / 1e9,
                tflops=2.0 * b * d0["d_out"] * d0["d_in"] / (ms * 1e-3) / 1e12)
        scratch = torch.empty_like(wl.W[sel[0]])

        def copies():
            for i in sel:
                scratch.copy_(wl.W[i])

        copies()
        torch.cuda.synchronize()
        g = capture(copies)
        g.replay()
        ms = time_graph(g, max(3, args.steps // 2), stream) / len(sel)
        del g
        lines[f"{d0['d_out']}x{d0['d_in']}_bf16_copy"] = dict(
            us_per_call=ms * 1e3, GB_per_s=2 * wbytes / (ms * 1e-3) / 1e9,
            frac_hbm=2 * wbytes / (ms * 1e-3) / 1e9 / hbm)
        del scratch
    lines["note"] = ("torch.matmul (cuBLAS) on the uncompressed BF16 weights, and torch copy_ of "
                     "them: context for the decode-GEMV and decode-GEMM lines, not their target; "
                     "the dense path reads 2 B/weight, the codec 11/16 B/weight")
    return lines


def run_gemm_lines(args, wl, dev, stream, hbm, bf16_tflops) -> dict:
    """Prefill-size decode-GEMM (qamw_decode_gemm, tensor cores) on the 11008x4096
    and 4096x11008 matrices at 64 and 128 tokens, each line one CUDA graph of
    the calls on all layers' matrices of that shape."""
    import torch

    from vector_quantization_codec_b200 import qamw, synth
    lines = {}
    for name in ("gate", "down"):
        sel = [i for i, d in enumerate(wl.mats) if d["name"] == name]
        d0 = wl.mats[sel[0]]
        for M in GEMM_TOKENS:
            ws = torch.empty(qamw.qamw_workspace_bytes(qamw.QAMW_OP_GEMM, d0["d_out"], d0["d_in"], BITS, M),
                             dtype=torch.uint8, device=dev)
            xs = [torch.from_numpy(synth.gemv_x(M, d0["d_in"], seed=9000 + i)).to(torch.bfloat16).to(dev)
                  for i in sel]
            ys = [torch.empty((M, d0["d_out"]), dtype=torch.bfloat16, device=dev) for _ in sel]

            def calls():
                for i, x, y in zip(sel, xs, ys):
                    qamw.qamw_decode_gemm(wl.m[i], x, y, workspace=ws, status=wl.status)

            calls()
            torch.cuda.synchronize()
            g = capture(calls)
            g.replay()
            ms = time_graph(g, max(3, args.steps // 2), stream) / len(sel)
            del g
            flops = 2.0 * M * d0["d_out"] * d0["d_in"]
            lines[f"{d0['d_out']}x{d0['d_in']}_m{M}"] = dict(
                us_per_call=ms * 1e3, useful_tflops=flops / (ms * 1e-3) / 1e12,
                executed_tflops=3 * flops / (ms * 1e-3) / 1e12,
                frac_bf16_peak_executed=3 * flops / (ms * 1e-3) / 1e12 / bf16_tflops,
                index_GB_per_s=d0["d_out"] * row_bytes(d0["d_in"], BITS) / (ms * 1e-3) / 1e9,
                matrices_cycled=len(sel),
                note="three binary16 MMAs per product (hi.hi, lo.hi, hi.lo)")
    wl.check_status("decode-GEMM lines")
    return lines


def run_35bpw(args, dev, stream, hbm, rank) -> dict:
    """The 3.5 bpw variant: every linear weight of 40 13B-shaped layers, K = 128
    (bits 7), joint 2-D codebook and the polar quantiser of the same K."""
    import torch

    from vector_quantization_codec_b200 import qamw
    cb, table, train_ms = train_codebook(BITS_35, dev)
    pcb = qamw.qamw_polar_codebook(BITS_35)
    mats = workload_matrices(args.layers_13b, rank, shapes="13b")
    wl = Workload(mats, BITS_35, cb, table, dev, polar_codebook=pcb)
    if args.encode_streams > 1:
        wl.encode_streams = [torch.cuda.Stream(device=dev) for _ in range(args.encode_streams)]
    wl.calibrate()
    wl.encode()
    wl.decode()
    wl.encode_polar()
    wl.decode(polar=True)
    torch.cuda.synchronize()
    wl.check_status("3.5 bpw warm-up")
    reps = 3
    out = {"workload": f"13B-shaped linear weights of {args.layers_13b} layers ({len(mats)} matrices: "
                       "q,k,v,o 5120x5120, gate,up 13824x5120, down 5120x13824), bf16 Student-t(5)x0.02, "
                       "K=128 (bits 7), block 128, alpha 0.5",
           "weights": wl.weights, "train_ms": train_ms}
    ab = total_bytes(mats, BITS_35)
    for label, fns in (("joint", (wl.calibrate, wl.encode, wl.decode)),
                       ("polar", (None, wl.encode_polar, lambda: wl.decode(polar=True)))):
        res = {}
        for key, fn in zip(("calibrate", "encode", "decode"), fns):
            if fn is None:
                continue
            g = capture(fn)
            g.replay()
            ms = time_graph(g, reps, stream)
            del g
            res[key] = dict(ms=ms)
        res["encode"]["Mweights_per_s"] = wl.weights / (res["encode"]["ms"] * 1e-3) / 1e6
        res["encode"]["frac_hbm"] = ab["encode"] / (res["encode"]["ms"] * 1e-3) / 1e9 / hbm
        res["decode"]["GB_per_s"] = ab["decode"] / (res["decode"]["ms"] * 1e-3) / 1e9
        res["decode"]["frac_hbm"] = res["decode"]["GB_per_s"] / hbm
        out[label] = res
    wl.check_status("3.5 bpw")
    # reconstruction error of both paths on layer 0's q matrix (joint 2-D vs polar)
    W0 = wl.W[0].float()
    dj = wl.out[0]
    qamw.qamw_decode(wl.m[0], dj)
    torch.cuda.synchronize()
    err_joint = float(((dj.float() - W0).norm() / W0.norm()).item())
    qamw.qamw_decode(wl.m_polar[0], dj)
    torch.cuda.synchronize()
    err_polar = float(((dj.float() - W0).norm() / W0.norm()).item())
    out["rel_fro_error_layer0_q"] = dict(joint=err_joint, polar=err_polar)
    del wl
    torch.cuda.empty_cache()
    return out


def run_e2e(args, wl, stream, world, dev) -> dict:
    """The step through the public API from pinned host buffers: every step
    copies each matrix's weights, statistic and x host -> device (copy stream),
    runs the five calls (compute stream, waiting on that matrix's copies) and
    reads back the encoded matrix (indices, r, sigma, s) and y (third stream)."""
    import torch

    from vector_quantization_codec_b200 import qamw
    def pinned(t):
        return torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t)

    # pinned host copies of the whole workload when the host has room for them
    # (twice over), else of as many leading matrices as fit; the line says which
    per_mat = [W.numel() * 2 + m.packed.numel() + 16 * m.d_in for W, m in zip(wl.W, wl.m)]
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except ImportError:
        avail = 1 << 40
    n, acc = 0, 0
    for b in per_mat:
        if 2 * (acc + b) > avail:
            break
        acc += b
        n += 1
    n = max(n, 1)
    Wh = [pinned(W) for W in wl.W[:n]]
    ah = [pinned(a) for a in wl.act[:n]]
    xh = [pinned(x) for x in wl.x[:n]]
    outs = [[m.packed, m.row_norm, m.sigma, m.chan_scale, y] for m, y in zip(wl.m[:n], wl.y[:n])]
    outs_h = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in o] for o in outs]
    h2d = sum(t.numel() * t.element_size() for ts in (Wh, ah, xh) for t in ts)
    d2h = sum(t.numel() * t.element_size() for o in outs for t in o)
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    weights = sum(W.numel() for W in wl.W[:n])
    ev_in = [torch.cuda.Event() for _ in range(n)]
    ev_done = [torch.cuda.Event() for _ in range(n)]

    def step():
        for i in range(n):
            with torch.cuda.stream(s_in):
                wl.W[i].copy_(Wh[i], non_blocking=True)
                wl.act[i].copy_(ah[i], non_blocking=True)
                wl.x[i].copy_(xh[i], non_blocking=True)
                ev_in[i].record(s_in)
        for i in range(n):
            stream.wait_event(ev_in[i])
            m = wl.m[i]
            qamw.qamw_channel_scales(m.d_in, wl.act[i], ALPHA, m.chan_scale, status=wl.status, stream=stream)
            qamw.qamw_calibrate_sigma(wl.W[i], m, workspace=wl.ws_cal, status=wl.status, stream=stream)
            qamw.qamw_encode_rows(wl.W[i], m, status=wl.status, stream=stream)
            qamw.qamw_decode(m, wl.out[i], status=wl.status, stream=stream)
            qamw.qamw_decode_gemv(m, wl.x[i], wl.y[i], workspace=wl.ws_gemv, status=wl.status,
                                  stream=stream)
            ev_done[i].record(stream)
        for i in range(n):
            s_out.wait_event(ev_done[i])
            with torch.cuda.stream(s_out):
                for hd, dd in zip(outs_h[i], outs[i]):
                    hd.copy_(dd, non_blocking=True)
        # the next step's copies overwrite W: wait for this step's kernels
        s_in.wait_stream(stream)
        stream.wait_stream(s_out)

    step()
    torch.cuda.synchronize()
    steps = max(1, args.e2e_steps)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    s_in.wait_stream(stream)
    e0.record(s_in)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    wl.check_status("e2e")
    ms = e0.elapsed_time(e1) / steps
    ms = max_over_ranks(ms, world, dev)
    return dict(value=world * weights / (ms * 1e-3) / 1e6, unit="Mweights/s", ms_per_step=ms,
                steps=steps, matrices=n, h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h,
                host_mem_available=avail,
                note="weights, statistics and x copied host->device and the encoded matrices and "
                     "y read back every step (pinned buffers; copies overlap the kernels on separate streams)")


# ------------------------------------------------------------------ CPU oracle

ORACLE_SAMPLE_ROWS = 1024


def oracle_sample(name: str, layer: int = 0, rows: int = ORACLE_SAMPLE_ROWS,
                  threads: int | None = None) -> dict:
    """The oracle on a bounded piece of the workload: rows 0..rows-1 of layer
    `layer`'s `name` matrix (weights drawn on the host with the same
    distributions): channel scales, eq. (1) over those rows (the first 1024
    rows of the matrix are the rows eq. (1) reads), then encode, decode and the
    GEMV of the same rows.  Returns the weights processed and the seconds."""
    import numpy as np
    import torch

    import oracle
    from vector_quantization_codec_b200 import synth
    shapes = dict((n, (o, i)) for n, o, i in synth.llama2_7b_layer_shapes())
    d_out, d_in = shapes[name]
    rows = min(rows, d_out)
    t = [n for n, _, _ in synth.llama2_7b_layer_shapes()].index(name)
    W = synth.student_t_weights(rows, d_in, seed=10000 * WL_7B + 10 * layer + t)
    W64 = torch.from_numpy(W).to(torch.bfloat16).double().numpy()
    act = synth.act_stat_for((WL_7B, layer, 100 + synth.LAYER_INPUT[name]), d_in).astype(np.float64)
    x64 = torch.from_numpy(synth.gemv_x(1, d_in, seed=layer)).to(torch.bfloat16).double().numpy()
    cb = np.asarray(synth.circular_gaussian_samples(1 << BITS, seed=7), dtype=np.float64)
    threads = threads or (os.cpu_count() or 1)
    t0 = time.perf_counter()
    s = oracle.channel_scales(act, d_in, ALPHA)
    sig = oracle.calibrate_sigma(W64, BLOCK, s)
    enc = oracle.encode(W64, BITS, BLOCK, cb, s_half=s, sigma_half=sig, threads=threads)
    What = oracle.decode(enc, cb, threads=threads)
    oracle.gemv(What, x64, threads=threads)
    secs = time.perf_counter() - t0
    return dict(weights=rows * d_in, seconds=secs, name=name, rows=rows, d_in=d_in)


def cpu_baseline(args) -> dict:
    """The oracle as it stands on this host's cores: rows 0..1023 of layer 0's
    q (4096x4096), gate (11008x4096) and down (4096x11008) matrices, all
    threads (about 10-30 s of CPU work); plus the same q rows on one thread
    (encode/decode/GEMV of 64 rows) for the per-core rate."""
    threads = os.cpu_count() or 1
    runs = [oracle_sample(n, threads=threads) for n in ("q", "gate", "down")]
    w = sum(r["weights"] for r in runs)
    s = sum(r["seconds"] for r in runs)
    one = oracle_sample("q", rows=64, threads=1)
    return dict(value=w / s / 1e6, unit="Mweights/s", cores=threads, kind="oracle", seconds=s,
                sample="rows 0..1023 of layer 0's q, gate and down matrices: channel scales, eq.(1) "
                       "over those rows, encode, decode and GEMV (batch 1) of the same rows; "
                       f"{w} weights in {s:.1f} s on {threads} threads",
                single_thread=dict(value=one["weights"] / one["seconds"] / 1e6, unit="Mweights/s",
                                   sample="rows 0..63 of layer 0's q matrix (eq.(1) over those rows), "
                                          "1 thread", seconds=one["seconds"]))


def run_reference(args) -> dict | None:
    """The reference arm: the oracle (the only implementation the pages
    define) timed on this host's cores.  Each step is one bounded sample of the
    workload, cycling through layer 0's seven matrices (rows 0..1023 each);
    `value` is the weights processed over the time taken, `ms_per_step` the
    mean measured time of one sample step (nothing is extrapolated)."""
    rank, world, _ = rank_env()
    if rank != 0:
        return None
    from vector_quantization_codec_b200 import synth
    names = [n for n, _, _ in synth.llama2_7b_layer_shapes()]
    threads = os.cpu_count() or 1
    for k in range(args.warmup):
        oracle_sample(names[k % len(names)], rows=args.ref_rows, threads=threads)
    runs = [oracle_sample(names[k % len(names)], rows=args.ref_rows, threads=threads)
            for k in range(args.steps)]
    w = sum(r["weights"] for r in runs)
    s = sum(r["seconds"] for r in runs)
    v = w / s / 1e6
    sample = (f"each step: rows 0..{args.ref_rows - 1} of one of layer 0's seven matrices (cycled), "
              "channel scales, eq.(1) over those rows, encode, decode and GEMV of the same rows; "
              f"{w} weights in {s:.1f} s over {args.steps} steps")
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "Mweights/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": s / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(args.layers, world),
                       sample=sample),
        "cpu_baseline": dict(value=v, unit="Mweights/s", cores=threads, kind="oracle", sample=sample),
        "e2e": {"value": v, "unit": "Mweights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# ------------------------------------------------------------------ profiling

def run_single_stage(args) -> dict:
    """One stage alone on a d_out = args.rows x args.din matrix (same
    distributions), for kernel profiling and sweeps: `warmup` untimed then
    `steps` timed calls."""
    import torch

    from vector_quantization_codec_b200 import qamw, synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    rows, d_in, bits = args.rows, args.din, args.bits
    K = 1 << bits
    samples = torch.from_numpy(synth.circular_gaussian_samples(TRAIN_N, seed=7)).to(dev)
    codebook = torch.empty((K, 2), dtype=torch.float32, device=dev)
    if args.only != "train":
        qamw.qamw_train_codebook(samples, bits, TRAIN_ITERS, codebook)
    prefilter = qamw.qamw_build_prefilter(codebook, bits) if args.only != "train" else None
    W = synth.student_t_weights_device(rows, d_in, (9, args.seed), dev)
    act = torch.from_numpy(synth.act_stat_lognormal(d_in, args.seed)).to(dev)
    x = torch.from_numpy(synth.gemv_x(args.batch, d_in, args.seed)).to(torch.bfloat16).to(dev)
    m = qamw.EncodedMatrix.empty(rows, d_in, BLOCK, bits, codebook, 0, prefilter)
    if args.only != "train":
        qamw.qamw_encode(W, m, act, ALPHA)
    ws_cal = torch.empty(qamw.qamw_workspace_bytes(qamw.QAMW_OP_CALIBRATE, rows, d_in, bits),
                         dtype=torch.uint8, device=dev)
    ws_g = torch.empty(qamw.qamw_workspace_bytes(qamw.QAMW_OP_GEMV, rows, d_in, bits, min(args.batch, 16)),
                       dtype=torch.uint8, device=dev)
    ws_gm = torch.empty(qamw.qamw_workspace_bytes(qamw.QAMW_OP_GEMM, rows, d_in, bits, args.batch),
                        dtype=torch.uint8, device=dev)
    W_hat = torch.empty((rows, d_in), dtype=torch.bfloat16, device=dev)
    y = torch.empty((args.batch, rows), dtype=torch.bfloat16, device=dev)
    count = args.count if args.only in ("gemv_many", "calibrate_many") else 1
    if args.only == "gemv_many":
        # `count` distinct encodings of W (own index buffers: more than L2 holds)
        mlist = [m]
        for i in range(1, count):
            mi = qamw.EncodedMatrix.empty(rows, d_in, BLOCK, bits, codebook, i, prefilter)
            qamw.qamw_encode(W, mi, act, ALPHA)
            mlist.append(mi)
        xl = [x[:1].clone() for _ in range(count)]
        yl = [torch.empty((1, rows), dtype=torch.bfloat16, device=dev) for _ in range(count)]
        ws_many = torch.empty(max(16, qamw.qamw_decode_gemv_many_workspace_bytes(mlist)),
                              dtype=torch.uint8, device=dev)
    if args.only == "calibrate_many":
        # `count` matrices calibrated from the same W (own s and sigma)
        clist = [m] + [qamw.EncodedMatrix.empty(rows, d_in, BLOCK, bits, codebook, i, prefilter)
                       for i in range(1, count)]
        ws_cm = torch.empty(max(16, qamw.qamw_calibrate_many_workspace_bytes(clist)),
                            dtype=torch.uint8, device=dev)
    fns = {
        "encode": lambda: qamw.qamw_encode_rows(W, m),
        "calibrate": lambda: qamw.qamw_calibrate_sigma(W, m, workspace=ws_cal),
        "decode": lambda: qamw.qamw_decode(m, W_hat),
        "gemv": lambda: qamw.qamw_decode_gemv(m, x, y, workspace=ws_g),
        "gemm": lambda: qamw.qamw_decode_gemm(m, x, y, workspace=ws_gm),
        "gemv_many": lambda: qamw.qamw_decode_gemv_many(mlist, xl, yl, workspace=ws_many),
        "calibrate_many": lambda: qamw.qamw_calibrate_many([W] * count, clist, [act] * count, ALPHA,
                                                           workspace=ws_cm),
        "train": lambda: qamw.qamw_train_codebook(samples, bits, 1, codebook),
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
        # `steps` back-to-back calls captured in one CUDA graph: device time only
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
    ab = algorithmic_bytes(rows, d_in, bits, args.batch)
    key = {"encode": "encode", "calibrate": "encode", "decode": "decode", "gemv": "gemv",
           "gemm": "gemv", "gemv_many": "gemv"}.get(args.only)
    out = dict(stage=args.only, rows=rows, d_in=d_in, bits=bits, batch=args.batch, ms=ms,
               timing="eager" if args.eager else "cuda graph of back-to-back calls",
               Mweights_per_s=count * rows * d_in / (ms * 1e-3) / 1e6)
    if count > 1:
        out["matrices"] = count
    if key:
        out["GB_per_s"] = count * ab[key] / (ms * 1e-3) / 1e9
    return out


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="qamw", choices=["qamw", "reference"])
    ap.add_argument("--layers", type=int, default=LAYERS,
                    help="layers of the Llama-2-7B-shaped workload (32; fewer only for profiling)")
    ap.add_argument("--layers-13b", type=int, default=LAYERS_13B,
                    help="layers of the 13B-shaped 3.5 bpw workload (40)")
    ap.add_argument("--skip-35", action="store_true", help="skip the 3.5 bpw workload")
    ap.add_argument("--encode-streams", type=int, default=2,
                    help="streams the encode phase's independent per-matrix calls go round-robin over")
    ap.add_argument("--e2e-steps", type=int, default=3, help="steps of the end-to-end leg")
    ap.add_argument("--ref-rows", type=int, default=ORACLE_SAMPLE_ROWS,
                    help="--impl reference: rows of each sample step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["encode", "calibrate", "calibrate_many", "decode", "gemv",
                                       "gemv_many", "gemm", "train"],
                    help="profiling mode: time one stage alone (no step, no JSON contract)")
    ap.add_argument("--rows", type=int, default=16384, help="--only: rows of the matrix")
    ap.add_argument("--din", type=int, default=4096, help="--only: columns of the matrix")
    ap.add_argument("--bits", type=int, default=BITS, help="--only: bits per pair")
    ap.add_argument("--batch", type=int, default=1, help="--only gemv / gemm: batch columns / tokens")
    ap.add_argument("--count", type=int, default=16,
                    help="--only gemv_many / calibrate_many: matrices in the list")
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
