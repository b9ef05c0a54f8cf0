"""Pins of the oracle's d = 1 scalar ablation (QAM-W paper, section 2, "parallel
work": the d = 1 versus d = 2 comparison named as the first follow-up).

The N(0, 1) Lloyd-Max levels are checked against closed forms (one level: 0,
MSE 1; two levels: +-sqrt(2/pi), MSE 1 - 2/pi), against Max's 1960 table, and
against the centroid conditions evaluated by scipy's numerical integration;
the quantiser against brute-force nearest levels and against the exhaustive 2D
search over its own product table (which pins the index layout i_x L + i_y);
the encoder by a lossless round trip; and the paper's claim that the joint 2D
code beats the scalar one at equal bits, on samples of N(0, I_2).
"""
import math

import numpy as np
import pytest
import scipy.integrate

import oracle
from vector_quantization_codec_b200 import synth


def phi(x):
    return math.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)


def test_one_and_two_levels_closed_forms():
    lv1 = oracle.gauss_lloyd_max(1)
    assert lv1[0] == pytest.approx(0.0, abs=1e-15)
    assert oracle.gauss_mse(lv1) == pytest.approx(1.0, abs=1e-14)
    lv2 = oracle.gauss_lloyd_max(2)
    c = math.sqrt(2 / math.pi)
    assert lv2 == pytest.approx([-c, c], abs=1e-14)
    assert oracle.gauss_mse(lv2) == pytest.approx(1 - 2 / math.pi, abs=1e-14)


def test_max_1960_table(golden):
    rows = golden("lloyd_max_gaussian.txt")
    for r in rows:
        N, kind, vals = int(r[0]), r[1], [float(v) for v in r[2:]]
        lv = oracle.gauss_lloyd_max(N)
        if kind == "levels":
            # four significant digits as printed
            assert np.allclose(lv[N // 2:], vals, rtol=6e-4, atol=6e-5), (N, lv[N // 2:])
        else:
            assert oracle.gauss_mse(lv) == pytest.approx(vals[0], rel=6e-4), N


@pytest.mark.parametrize("N", [2, 3, 5, 8, 16, 32])
def test_lloyd_max_conditions_by_quadrature(N):
    lv = oracle.gauss_lloyd_max(N)
    assert np.all(np.diff(lv) > 0)
    assert np.allclose(lv, -lv[::-1], atol=1e-12)  # symmetric
    t = np.concatenate([[-np.inf], 0.5 * (lv[1:] + lv[:-1]), [np.inf]])
    mse = 0.0
    for i in range(N):
        m, _ = scipy.integrate.quad(phi, t[i], t[i + 1])
        mom, _ = scipy.integrate.quad(lambda x: x * phi(x), t[i], t[i + 1])
        sq, _ = scipy.integrate.quad(lambda x: (x - lv[i]) ** 2 * phi(x), t[i], t[i + 1])
        assert lv[i] == pytest.approx(mom / m, rel=1e-9, abs=1e-12)
        mse += sq
    assert oracle.gauss_mse(lv) == pytest.approx(mse, rel=1e-8)


def test_distortion_falls_toward_the_high_rate_formula():
    # Panter-Dite: N^2 MSE -> pi sqrt(3) / 2 = 2.7207 as N grows, from below
    prev = None
    for N in (4, 8, 16, 32):
        r = oracle.gauss_mse(oracle.gauss_lloyd_max(N)) * N * N / (math.pi * math.sqrt(3) / 2)
        assert 0.5 < r < 1.0
        if prev is not None:
            assert r > prev
        prev = r
    assert prev > 0.92


@pytest.mark.parametrize("bits", [2, 4, 6, 8, 10])
def test_index_is_nearest_level_per_coordinate(bits):
    L = 1 << (bits // 2)
    lv = oracle.scalar_levels(bits)
    g = np.random.default_rng(bits)
    pts = g.standard_normal((3000, 2)) * 1.3
    got = oracle.scalar_index(pts, lv, bits)
    ix = np.argmin(np.abs(pts[:, :1] - lv[None, :]), axis=1)
    iy = np.argmin(np.abs(pts[:, 1:] - lv[None, :]), axis=1)
    assert np.array_equal(got, ix * L + iy)
    # 0 lies exactly between the two middle levels +-l: the lower index wins
    if L >= 2:
        assert oracle.scalar_index(np.zeros((1, 2)), lv, bits)[0] == (L // 2 - 1) * (L + 1)


@pytest.mark.parametrize("bits", [4, 8])
def test_index_equals_the_2d_search_over_the_product_table(bits):
    lv = oracle.scalar_levels(bits)
    cb = oracle.scalar_codebook(bits, lv)
    L = 1 << (bits // 2)
    assert np.array_equal(cb[:, 0], np.repeat(lv, L)) and np.array_equal(cb[:, 1], np.tile(lv, L))
    pts = np.random.default_rng(7).standard_normal((4000, 2))
    assert np.array_equal(oracle.scalar_index(pts, lv, bits), oracle.nearest(pts, cb))


def test_encode_scalar_lossless_round_trip():
    # One row built from product-table codewords, W = R_inv(sigma * c_idx), with
    # sigma chosen so that ||sigma * c_idx|| = 1 up to binary16 rounding: then
    # r ~ 1 and p_k = c_idx_k (1 +- 1e-3), far from every decision midpoint, so
    # encoding with the same sigma recovers idx exactly and decoding gives back
    # r_hat * W.
    bits, d_in, b, seed = 6, 256, 64, 3
    K, P = 1 << bits, d_in // 2
    lv = oracle.scalar_levels(bits)
    cb = oracle.scalar_codebook(bits, lv)
    g = np.random.default_rng(9)
    idx = g.integers(0, K, size=(1, P), dtype=np.int32)
    raw = g.uniform(0.5, 1.5, P)
    raw /= np.linalg.norm(raw[:, None] * cb[idx[0]])
    sigma = oracle.f64_to_halves(raw)
    sg = oracle.halves_to_f64(sigma)
    y = (sg[:, None] * cb[idx[0]]).reshape(-1)
    W = oracle.rotate_inv(y, b, seed)[None, :]
    one = oracle.f64_to_halves(np.ones(d_in))
    enc = oracle.encode_scalar(W, bits, b, lv, mask_seed=seed, s_half=one, sigma_half=sigma)
    assert np.array_equal(enc["idx"], idx)
    rhat = oracle.halves_to_f64(enc["rnorm_half"])[0]
    assert abs(rhat - 1.0) < 2e-3
    Wd = oracle.decode(enc, cb)
    assert np.allclose(Wd, rhat * W, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("bits,n", [(4, 1 << 16), (6, 1 << 17)])
def test_joint_2d_beats_scalar_at_equal_bits(bits, n):
    # about 2000 training samples per codeword, so that the 2D codebook is a
    # Lloyd codebook of N(0, I_2) rather than of its sample; measured on fresh
    # samples the joint code's MSE is ~0.92 (B = 4) and ~0.87 (B = 6) of the
    # scalar code's
    K = 1 << bits
    train = synth.circular_gaussian_samples(n, seed=60 + bits).astype(np.float64)
    cb2d, _ = oracle.lloyd(train, K, 60)
    test = synth.circular_gaussian_samples(1 << 16, seed=70 + bits).astype(np.float64)
    mse2d = ((test - cb2d[oracle.nearest(test, cb2d)]) ** 2).sum(1).mean()
    lv = oracle.scalar_levels(bits)
    cb1d = oracle.scalar_codebook(bits, lv)
    mse1d = ((test - cb1d[oracle.scalar_index(test, lv, bits)]) ** 2).sum(1).mean()
    # the scalar code's per-pair MSE is twice the per-coordinate Lloyd-Max MSE
    assert mse1d == pytest.approx(2 * oracle.gauss_mse(lv), rel=0.03)
    assert mse2d < 0.95 * mse1d, (mse2d, mse1d)
