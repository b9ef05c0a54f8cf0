"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Sizes: small enough for the oracle to finish in seconds, spanning several
CTAs / grid-stride iterations with ragged tails (row counts that are not
multiples of anything, d_in = 192 = 3 chunks, 11008 = 172 chunks), every
Hadamard block layout (b = 1, 16, 64, 128, 1024), bits 1..11, fp32 and bf16 W.
The full 4096x4096 K=2048 matrix is checked on sampled rows.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from tests.parity import bf16_to_f64, check_close, check_indices, halves, to_half_tensor, ulp_diff
from vector_quantization_codec_b200 import qamw, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"

_CB_CACHE: dict = {}


def codebook(bits: int) -> np.ndarray:
    """fp32 codebook from the oracle's Lloyd on seeded N(0, I_2) samples."""
    if bits not in _CB_CACHE:
        K = 1 << bits
        n = max(64 * K, 4096) if bits <= 8 else 32 * K
        s = synth.circular_gaussian_samples(n, seed=100 + bits).astype(np.float64)
        cb, _ = oracle.lloyd(s, K, 12 if bits <= 8 else 6)
        _CB_CACHE[bits] = cb.astype(np.float32)
    return _CB_CACHE[bits]


def weights(d_out, d_in, seed, dtype):
    W = synth.student_t_weights(d_out, d_in, seed)
    W[seed % d_out] *= 10.0
    if dtype == "bf16":
        Wt = torch.from_numpy(W).to(torch.bfloat16)
        return Wt.to(DEV), Wt.double().numpy()
    return torch.from_numpy(W).to(DEV), W.astype(np.float64)


def gpu_encode(Wt, d_in, block, bits, cb, act=None, alpha=0.0, seed=0, flags=0, m=None,
               prefilter=True):
    cbt = torch.from_numpy(cb).to(DEV)
    pf = qamw.qamw_build_prefilter(cbt, bits) if prefilter else None
    if m is None:
        m = qamw.EncodedMatrix.empty(Wt.shape[0], d_in, block, bits, cbt, seed, pf)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    a = None if act is None else torch.from_numpy(act).to(DEV)
    qamw.qamw_encode(Wt, m, a, alpha, flags=flags, status=st)
    torch.cuda.synchronize()
    return m, int(st.item())


CASES = [
    # d_out, d_in, block, bits, dtype, alpha
    (256, 512, 64, 8, "f32", 0.5),
    (300, 1024, 128, 11, "bf16", 0.5),
    (97, 4096, 1024, 7, "bf16", 0.5),
    (64, 192, 64, 3, "f32", 0.5),
    (50, 256, 16, 5, "f32", 0.0),
    (17, 128, 1, 1, "f32", 0.5),
    (24, 11008, 128, 11, "bf16", 0.5),
    (33, 640, 128, 9, "bf16", 0.3),
    (41, 384, 128, 6, "f32", 1.0),
    (19, 1024, 256, 10, "bf16", 0.5),
    (12, 256, 32, 2, "f32", 0.5),
    (9, 320, 64, 4, "bf16", 0.5),
    (16, 20480, 128, 11, "bf16", 0.5),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}x{c[1]}_b{c[2]}_B{c[3]}_{c[4]}")
def test_encode_matches_oracle(case):
    d_out, d_in, block, bits, dtype, alpha = case
    cb = codebook(bits)
    Wt, W = weights(d_out, d_in, d_out + bits, dtype)
    act = synth.act_stat_lognormal(d_in, seed=bits)
    m, status = gpu_encode(Wt, d_in, block, bits, cb, act, alpha, seed=5)
    assert status == 0
    s_g, r_g, sig_g = halves(m.chan_scale), halves(m.row_norm), halves(m.sigma)
    # channel scales and pair scales: within one binary16 ulp of the oracle's
    s_o = oracle.channel_scales(act.astype(np.float64), d_in, alpha)
    assert ulp_diff(s_g, s_o).max() <= 1
    sig_o = oracle.calibrate_sigma(W, block, s_g, 5)
    assert ulp_diff(sig_g, sig_o).max() <= 1
    # indices with the GPU's binary16 side values given to the oracle
    enc = oracle.encode(W, bits, block, cb, mask_seed=5, s_half=s_g, sigma_half=sig_g,
                        want_points=True)
    assert ulp_diff(r_g, enc["rnorm_half"]).max() <= 1
    packed = m.packed.cpu().numpy()
    idx_g = oracle.unpack(packed, d_in // 2, bits)
    check_indices(idx_g, enc["idx"], enc["points"], cb)
    # padding bits of every row are zero
    used = (d_in // 2) * bits
    stream = np.unpackbits(packed, axis=1, bitorder="little")
    assert not stream[:, used:].any()


DECODE_CASES = [(256, 512, 64, 8), (300, 1024, 128, 11), (97, 4096, 1024, 7), (64, 192, 64, 3),
                (50, 256, 16, 5), (17, 128, 1, 1), (24, 11008, 128, 11), (19, 1024, 256, 10)]


@pytest.mark.parametrize("case", DECODE_CASES, ids=lambda c: f"{c[0]}x{c[1]}_b{c[2]}_B{c[3]}")
def test_decode_matches_oracle(case):
    # oracle-encoded stream -> GPU decode vs oracle decode (fp64)
    d_out, d_in, block, bits = case
    cb = codebook(bits)
    W = synth.student_t_weights(d_out, d_in, seed=d_in).astype(np.float64)
    W[3 % d_out] = 0.0  # a zero row decodes to exact zeros
    act = synth.act_stat_lognormal(d_in, seed=1).astype(np.float64)
    enc = oracle.encode(W, bits, block, cb, mask_seed=9, act_stat=act, alpha=0.5)
    ref = oracle.decode(enc, cb)
    cbt = torch.from_numpy(cb).to(DEV)
    m = qamw.EncodedMatrix(d_out, d_in, block, bits, 9,
                           torch.from_numpy(enc["packed"]).to(DEV),
                           to_half_tensor(enc["rnorm_half"], DEV),
                           to_half_tensor(enc["sigma_half"], DEV),
                           to_half_tensor(enc["s_half"], DEV), cbt)
    out = qamw.qamw_decode(m)
    torch.cuda.synchronize()
    got = bf16_to_f64(out)
    assert np.all(got[3 % d_out] == 0.0)
    check_close(got, ref, what="decode")


GEMV_CASES = [(256, 512, 64, 8, 1), (300, 1024, 128, 11, 4), (97, 4096, 1024, 7, 16),
              (64, 192, 64, 3, 3), (24, 11008, 128, 11, 13), (33, 640, 128, 9, 8),
              (17, 128, 1, 1, 1), (16, 20480, 128, 11, 1), (10, 20480, 256, 8, 5),
              (40, 2048, 128, 11, 9), (12, 16384, 128, 11, 2), (20, 6144, 128, 11, 3),
              (21, 6144, 128, 11, 6)]


@pytest.mark.parametrize("case", GEMV_CASES, ids=lambda c: f"{c[0]}x{c[1]}_b{c[2]}_B{c[3]}_n{c[4]}")
def test_decode_gemv_matches_oracle(case):
    d_out, d_in, block, bits, batch = case
    cb = codebook(bits)
    Wt, W = weights(d_out, d_in, 7 + d_out, "bf16")
    act = synth.act_stat_lognormal(d_in, seed=2)
    m, status = gpu_encode(Wt, d_in, block, bits, cb, act, 0.5, seed=3)
    assert status == 0
    enc = dict(packed=m.packed.cpu().numpy(), rnorm_half=halves(m.row_norm),
               sigma_half=halves(m.sigma), s_half=halves(m.chan_scale), d_out=d_out, d_in=d_in,
               block=block, bits=bits, mask_seed=3)
    What = oracle.decode(enc, cb)
    x32 = synth.gemv_x(batch, d_in, seed=batch)
    xt = torch.from_numpy(x32).to(torch.bfloat16)
    xref = xt.double().numpy()
    yref = oracle.gemv(What, xref)
    y = qamw.qamw_decode_gemv(m, xt.to(DEV))
    torch.cuda.synchronize()
    got = bf16_to_f64(y)
    for t in range(batch):
        check_close(got[t], yref[t], what=f"gemv col {t}")


def test_train_first_iteration_matches_oracle():
    bits, n = 8, 1 << 16
    K = 1 << bits
    s = synth.circular_gaussian_samples(n, seed=41)
    cb_g = torch.empty((K, 2), dtype=torch.float32, device=DEV)
    dist_g = torch.empty(1, dtype=torch.float64, device=DEV)
    qamw.qamw_train_codebook(torch.from_numpy(s).to(DEV), bits, 1, cb_g, dist_g)
    torch.cuda.synchronize()
    s64 = s.astype(np.float64)
    cb_o, dist_o = oracle.lloyd(s64, K, 1)
    # The samples and initial codewords are exact fp32 values, so the kernel's
    # fp32 scores differ from the exact distances only by rounding (~2^-20 of
    # 1 + |p|^2).  Cells that a sample within that gap of a tie could have
    # gone to are not compared.
    c0 = s64[:K]
    d = ((s64[:, None, :] - c0[None]) ** 2).sum(-1)
    part = np.partition(d, 1, axis=1)
    tol = 2e-6 * (1 + (s64 ** 2).sum(1))
    tie = (part[:, 1] - part[:, 0]) <= tol
    excluded = set()
    for t in np.nonzero(tie)[0]:
        excluded.update(np.nonzero(d[t] <= part[t, 0] + tol[t])[0].tolist())
    keep = np.array([j not in excluded for j in range(K)])
    assert keep.sum() >= K // 2
    got = cb_g.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got[keep] - cb_o[keep])) <= 1e-6
    assert float(dist_g.item()) == pytest.approx(dist_o[0], rel=1e-5)


def test_train_lloyd_conditions_and_determinism():
    bits, n, iters = 8, 1 << 18, 40
    K = 1 << bits
    s = synth.circular_gaussian_samples(n, seed=42)
    st = torch.from_numpy(s).to(DEV)
    out = []
    for _ in range(2):
        cb = torch.empty((K, 2), dtype=torch.float32, device=DEV)
        dist = torch.empty(iters, dtype=torch.float64, device=DEV)
        qamw.qamw_train_codebook(st, bits, iters, cb, dist)
        torch.cuda.synchronize()
        out.append((cb.cpu().numpy(), dist.cpu().numpy()))
    assert np.array_equal(out[0][0], out[1][0])  # bitwise reproducible
    cb, dist = out[0]
    assert np.all(np.diff(dist) <= 1e-6 * dist[:-1])
    s64 = s.astype(np.float64)
    a = oracle.nearest(s64, cb.astype(np.float64))
    means = np.array([s64[a == j].mean(0) for j in range(K)])
    assert np.max(np.abs(means - cb)) < 2e-2
    held = synth.circular_gaussian_samples(1 << 16, seed=43).astype(np.float64)
    mse = ((held - cb[oracle.nearest(held, cb.astype(np.float64))]) ** 2).sum(1).mean()
    ratio = mse / (2 * (5 / (36 * np.sqrt(3))) * 8 * np.pi / K)
    assert 0.95 <= ratio <= 1.10, ratio


def test_zero_row_nonfinite_and_bad_stat_flags():
    d_in, bits, block = 256, 6, 64
    cb = codebook(bits)
    W = synth.student_t_weights(8, d_in, seed=1)
    W[2] = 0.0
    m, status = gpu_encode(torch.from_numpy(W).to(DEV), d_in, block, bits, cb)
    assert status == 0
    assert halves(m.row_norm)[2] == 0
    assert not m.packed[2].any().item()
    assert not qamw.qamw_decode(m)[2].float().abs().sum().item()
    W[5, 7] = np.nan
    _, status = gpu_encode(torch.from_numpy(W).to(DEV), d_in, block, bits, cb)
    assert status & qamw.QAMW_STATUS_NONFINITE
    act = np.ones(d_in, dtype=np.float32)
    act[3] = 0.0
    W[5, 7] = 0.0
    m, status = gpu_encode(torch.from_numpy(W).to(DEV), d_in, block, bits, cb, act, 0.5)
    assert status == qamw.QAMW_STATUS_BAD_STAT
    assert halves(m.chan_scale)[3] == 0x3C00


def test_empty_and_single_row():
    bits, d_in, block = 4, 128, 64
    cb = codebook(bits)
    cbt = torch.from_numpy(cb).to(DEV)
    m0 = qamw.EncodedMatrix.empty(0, d_in, block, bits, cbt)
    qamw.qamw_encode(torch.empty((0, d_in), device=DEV), m0)
    qamw.qamw_decode(m0)
    W = synth.student_t_weights(1, d_in, seed=3)
    m, status = gpu_encode(torch.from_numpy(W).to(DEV), d_in, block, bits, cb)
    assert status == 0
    enc = oracle.encode(W.astype(np.float64), bits, block, cb, s_half=halves(m.chan_scale),
                        sigma_half=halves(m.sigma), want_points=True)
    check_indices(oracle.unpack(m.packed.cpu().numpy(), d_in // 2, bits), enc["idx"],
                  enc["points"], cb)


def test_without_prefilter_table_matches_with_it():
    d_out, d_in, block, bits = 64, 1024, 128, 11
    cb = codebook(bits)
    Wt, _ = weights(d_out, d_in, 77, "bf16")
    m1, _ = gpu_encode(Wt, d_in, block, bits, cb, prefilter=True)
    m2, _ = gpu_encode(Wt, d_in, block, bits, cb, prefilter=False)
    assert torch.equal(m1.packed, m2.packed)


def test_full_size_4096_square_sampled_rows():
    # The 4096x4096 bf16 Student-t matrix with K = 2048, block 128, alpha 0.5:
    # whole-matrix side values, then sampled rows of indices, decode and GEMV.
    case = synth.llama_square_case(seed=0)
    d_out, d_in, block, bits = case["d_out"], case["d_in"], case["block"], case["bits"]
    cb = codebook(bits)
    Wt = torch.from_numpy(case["W"]).to(torch.bfloat16)
    W = Wt.double().numpy()
    m, status = gpu_encode(Wt.to(DEV), d_in, block, bits, cb, case["act_stat"], case["alpha"])
    assert status == 0
    s_g, sig_g, r_g = halves(m.chan_scale), halves(m.sigma), halves(m.row_norm)
    assert ulp_diff(s_g, oracle.channel_scales(case["act_stat"].astype(np.float64), d_in,
                                               case["alpha"])).max() <= 1
    assert ulp_diff(sig_g, oracle.calibrate_sigma(W[:1024], block, s_g)).max() <= 1
    rows = np.unique(np.concatenate([[0, 1, 1023, 1024, 2047, 4095],
                                     np.random.default_rng(0).choice(d_out, 58, replace=False)]))
    enc = oracle.encode(W[rows], bits, block, cb, s_half=s_g, sigma_half=sig_g, want_points=True)
    assert ulp_diff(r_g[rows], enc["rnorm_half"]).max() <= 1
    packed = m.packed.cpu().numpy()[rows]
    check_indices(oracle.unpack(packed, d_in // 2, bits), enc["idx"], enc["points"], cb)
    # decode of the GPU stream on those rows
    sub = dict(packed=packed, rnorm_half=r_g[rows], sigma_half=sig_g, s_half=s_g, d_out=len(rows),
               d_in=d_in, block=block, bits=bits, mask_seed=0)
    ref = oracle.decode(sub, cb)
    got = bf16_to_f64(qamw.qamw_decode(m))[rows]
    check_close(got, ref, what="decode 4096^2")
    for batch in (1, 4, 16):
        xt = torch.from_numpy(synth.gemv_x(batch, d_in, seed=batch)).to(torch.bfloat16)
        y = bf16_to_f64(qamw.qamw_decode_gemv(m, xt.to(DEV)))[:, rows]
        yref = oracle.gemv(ref, xt.double().numpy())
        for t in range(batch):
            check_close(y[t], yref[t], what=f"gemv 4096^2 b{batch} col {t}")


def test_stage_calls_equal_composite_encode():
    # qamw_channel_scales + qamw_calibrate_sigma + qamw_encode_rows == qamw_encode
    d_out, d_in, block, bits = 150, 2048, 128, 11
    cb = codebook(bits)
    Wt, _ = weights(d_out, d_in, 5, "bf16")
    act = synth.act_stat_lognormal(d_in, seed=9)
    m1, st1 = gpu_encode(Wt, d_in, block, bits, cb, act, 0.5, seed=4)
    cbt = torch.from_numpy(cb).to(DEV)
    m2 = qamw.EncodedMatrix.empty(d_out, d_in, block, bits, cbt, 4, qamw.qamw_build_prefilter(cbt, bits))
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    qamw.qamw_channel_scales(d_in, torch.from_numpy(act).to(DEV), 0.5, m2.chan_scale, status=st)
    qamw.qamw_calibrate_sigma(Wt, m2, status=st)
    cand = torch.zeros(1, dtype=torch.int64, device=DEV)
    qamw.qamw_encode_rows(Wt, m2, status=st, candidates=cand)
    torch.cuda.synchronize()
    assert st1 == 0 and st.item() == 0
    for a, b in [(m1.packed, m2.packed), (m1.row_norm, m2.row_norm), (m1.sigma, m2.sigma),
                 (m1.chan_scale, m2.chan_scale)]:
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    pairs = d_out * d_in // 2
    assert pairs <= cand.item() <= pairs * 64  # at least one codeword scored per pair
    # without a prefilter table the search is exhaustive: K per pair, same indices
    m3 = qamw.EncodedMatrix(d_out, d_in, block, bits, 4, torch.empty_like(m2.packed),
                            torch.empty_like(m2.row_norm), m2.sigma, m2.chan_scale, cbt, None)
    cand.zero_()
    qamw.qamw_encode_rows(Wt, m3, candidates=cand)
    torch.cuda.synchronize()
    assert cand.item() == pairs * (1 << bits)
    assert torch.equal(m3.packed, m2.packed)


def test_encode_is_deterministic():
    d_out, d_in, block, bits = 300, 1024, 128, 11
    cb = codebook(bits)
    Wt, _ = weights(d_out, d_in, 8, "bf16")
    act = synth.act_stat_lognormal(d_in, seed=8)
    a, _ = gpu_encode(Wt, d_in, block, bits, cb, act, 0.5)
    b, _ = gpu_encode(Wt, d_in, block, bits, cb, act, 0.5)
    for x, y in [(a.packed, b.packed), (a.row_norm, b.row_norm), (a.sigma, b.sigma)]:
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


@pytest.mark.parametrize("bits", [7, 11])
def test_far_points_use_exact_sector_lists(bits):
    # sigma given 20x too small pushes normalised pairs to |p| ~ 20-60, far off
    # the prefilter grid: the angular-sector lists must give the oracle's
    # indices, and score few codewords (no exhaustive fallback).
    d_out, d_in, block = 64, 1024, 128
    cb = codebook(bits)
    Wt, W = weights(d_out, d_in, 21, "bf16")
    m, _ = gpu_encode(Wt, d_in, block, bits, cb)
    sig = (m.sigma.float() / 20).half()
    m2 = qamw.EncodedMatrix(d_out, d_in, block, bits, 0, torch.empty_like(m.packed),
                            torch.empty_like(m.row_norm), sig, m.chan_scale, m.codebook, m.prefilter)
    cand = torch.zeros(1, dtype=torch.int64, device=DEV)
    qamw.qamw_encode_rows(Wt, m2, candidates=cand)
    torch.cuda.synchronize()
    enc = oracle.encode(W, bits, block, cb, s_half=halves(m.chan_scale), sigma_half=halves(sig),
                        want_points=True)
    assert np.median(np.linalg.norm(enc["points"], axis=-1)) > 15
    check_indices(oracle.unpack(m2.packed.cpu().numpy(), d_in // 2, bits), enc["idx"],
                  enc["points"], cb)
    pairs = d_out * d_in // 2
    assert cand.item() < 40 * pairs


def test_calibration_rows_past_the_first_scan():
    # Rows 0..2047 hold only 80 non-zero rows, so the first 1024 non-zero rows
    # of eq. (1) reach past the rows whose norms are computed up front.
    d_out, d_in, block, bits = 3000, 256, 64, 6
    W = synth.student_t_weights(d_out, d_in, seed=12)
    keep = np.zeros(d_out, dtype=bool)
    keep[np.random.default_rng(0).choice(2048, 80, replace=False)] = True
    keep[2048:] = True
    keep[2100:2110] = False
    W[~keep] = 0.0
    cb = codebook(bits)
    m, status = gpu_encode(torch.from_numpy(W).to(DEV), d_in, block, bits, cb)
    assert status == 0
    sig_o = oracle.calibrate_sigma(W.astype(np.float64), block, halves(m.chan_scale))
    assert ulp_diff(halves(m.sigma), sig_o).max() <= 1
    # and rows of only zeros anywhere: all calibration rows zero -> sigma = 1
    m0, _ = gpu_encode(torch.zeros((5, d_in), device=DEV), d_in, block, bits, cb)
    assert np.all(halves(m0.sigma) == 0x3C00)
