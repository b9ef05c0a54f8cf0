"""Pins of the oracle's polar baseline (QAM-W paper section 3.5).

The amplitude codebook is checked against the Rayleigh mean (closed form for
one level) and against the Lloyd-Max conditions evaluated by scipy's numerical
integration; the quantiser against brute-force nearest level / nearest angle;
and the paper's comparison "joint 2D beats polar at equal bits" on samples of
the unit circular Gaussian.
"""
import math

import numpy as np
import pytest
import scipy.integrate

import oracle
from vector_quantization_codec_b200 import synth


def rayleigh_pdf(r):
    return r * math.exp(-0.5 * r * r)


def test_single_level_is_the_rayleigh_mean():
    assert oracle.rayleigh_lloyd_max(1)[0] == pytest.approx(math.sqrt(math.pi / 2), abs=1e-15)


@pytest.mark.parametrize("N", [2, 3, 8, 32])
def test_lloyd_max_conditions_by_quadrature(N):
    lv = oracle.rayleigh_lloyd_max(N)
    assert np.all(np.diff(lv) > 0)
    t = np.concatenate([[0.0], 0.5 * (lv[1:] + lv[:-1]), [np.inf]])
    for i in range(N):
        m, _ = scipy.integrate.quad(rayleigh_pdf, t[i], t[i + 1])
        mom, _ = scipy.integrate.quad(lambda r: r * rayleigh_pdf(r), t[i], t[i + 1])
        assert lv[i] == pytest.approx(mom / m, rel=1e-9, abs=1e-12)


def test_more_levels_less_distortion():
    def mse(lv):
        t = np.concatenate([[0.0], 0.5 * (lv[1:] + lv[:-1]), [np.inf]])
        return sum(scipy.integrate.quad(lambda r, a=a: (r - a) ** 2 * rayleigh_pdf(r), t[i],
                                        t[i + 1])[0] for i, a in enumerate(lv))
    d = [mse(oracle.rayleigh_lloyd_max(N)) for N in (1, 2, 4, 8)]
    assert d[0] == pytest.approx(2 - math.pi / 2, rel=1e-9)  # Var of the Rayleigh law
    assert all(a > b for a, b in zip(d, d[1:]))


@pytest.mark.parametrize("bits", [3, 7, 11])
def test_polar_index_is_nearest_level_and_nearest_angle(bits):
    ba, bp = oracle.polar_split(bits)
    assert (ba, bp) == (bits // 2, bits - bits // 2)
    Na, Np = 1 << ba, 1 << bp
    lv = oracle.polar_levels(bits)
    g = np.random.default_rng(bits)
    p = g.standard_normal((4000, 2)) * 1.3
    got = oracle.polar_index(p, lv, bits)
    r = np.hypot(p[:, 0], p[:, 1])
    ia = np.abs(r[:, None] - lv[None, :]).argmin(1)
    th = np.arctan2(p[:, 1], p[:, 0])
    centres = 2 * np.pi * np.arange(Np) / Np
    dang = np.abs(np.angle(np.exp(1j * (th[:, None] - centres[None, :]))))
    ip = dang.argmin(1)
    assert np.array_equal(got, ia * Np + ip)
    cb = oracle.polar_codebook(bits, lv)
    assert np.allclose(np.hypot(cb[:, 0], cb[:, 1]), np.repeat(lv, Np))
    assert np.allclose(np.arctan2(cb[1:Np, 1], cb[1:Np, 0]) % (2 * np.pi), centres[1:])


@pytest.mark.parametrize("bits", [7, 8])
def test_joint_2d_beats_polar_at_equal_bits(bits):
    # Section 3.6 / abstract: the joint 2D codebook beats the polar baseline at
    # the same bits per pair (on the unit circular Gaussian the codec targets).
    K = 1 << bits
    train = synth.circular_gaussian_samples(64 * K, seed=70 + bits).astype(np.float64)
    cb_joint, _ = oracle.lloyd(train, K, 40)
    held = synth.circular_gaussian_samples(1 << 15, seed=80 + bits).astype(np.float64)
    mse_joint = ((held - cb_joint[oracle.nearest(held, cb_joint)]) ** 2).sum(1).mean()
    lv = oracle.polar_levels(bits)
    cb_polar = oracle.polar_codebook(bits, lv)
    mse_polar = ((held - cb_polar[oracle.polar_index(held, lv, bits)]) ** 2).sum(1).mean()
    assert mse_joint < 0.95 * mse_polar, (mse_joint, mse_polar)


def test_polar_encode_matches_definition_on_rows():
    bits, d_in, b = 7, 256, 64
    lv = oracle.polar_levels(bits)
    W = synth.student_t_weights(5, d_in, seed=3).astype(np.float64)
    s = oracle.channel_scales(None, d_in, 0.0)
    sig = oracle.calibrate_sigma(W, b, s)
    enc = oracle.encode_polar(W, bits, b, lv, s_half=s, sigma_half=sig, want_points=True)
    assert np.array_equal(enc["idx"].ravel(),
                          oracle.polar_index(enc["points"].reshape(-1, 2), lv, bits))
    dec = oracle.decode(enc, oracle.polar_codebook(bits, lv))
    rel = np.linalg.norm(dec - W) / np.linalg.norm(W)
    assert rel < 0.15
