"""Pins of the fp64 oracle against what the QAM-W paper and mathematics fix.

None of these compares the oracle with itself: each check is a closed form, a
library routine (numpy float16, scipy's Sylvester Hadamard, numpy argmin and
matrix products), a value the paper prints (tests/golden), a mathematical
invariant, or brute force on a tiny input.
"""
import math

import numpy as np
import pytest
import scipy.linalg

import oracle
from vector_quantization_codec_b200 import synth


# ---------------------------------------------------------------- storage formats

def test_half_decode_matches_numpy_all_patterns():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float64)
    got = oracle.halves_to_f64(pats)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_half_rounding_matches_numpy():
    g = np.random.default_rng(1)
    x = np.concatenate([
        g.standard_normal(4000) * 10.0 ** g.uniform(-9, 5, 4000),
        # exact binary16 midpoints (ties to even) and the overflow edge
        (np.arange(1024, 1100) + 0.5) * 2.0 ** -10,
        np.array([65504.0, 65519.99, 65520.0, 1e9, -0.0, 2.0 ** -25, 2.0 ** -24 * 1.5, 6.1e-5]),
    ])
    with np.errstate(over="ignore"):
        want = x.astype(np.float16).view(np.uint16)
    got = oracle.f64_to_halves(x)
    assert np.array_equal(got, want)


def test_splitmix64_published_output(golden):
    for counter, hexout in golden("splitmix64.txt"):
        assert oracle.splitmix64(int(counter)) == int(hexout, 16)


def test_sign_mask_is_balanced_and_seeded():
    d = 4096
    m0 = oracle.sign_mask(0, d)
    m1 = oracle.sign_mask(1, d)
    assert set(np.unique(m0)) == {-1, 1}
    assert abs(m0.mean()) < 4.0 / math.sqrt(d)
    assert (m0 != m1).mean() > 0.4


def test_pack_hand_worked_example(golden):
    rows = {r[0]: r[1:] for r in golden("pack_example.txt")}
    bits = int(rows["bits"][0])
    idx = np.array([[int(v) for v in rows["indices"]]], dtype=np.int32)
    want = np.array([int(v) for v in rows["bytes"]], dtype=np.uint8)
    rb = oracle.row_bytes(2 * idx.shape[1], bits)
    assert rb == 16
    got = oracle.pack(idx, bits, rb)[0]
    assert np.array_equal(got, want)


@pytest.mark.parametrize("bits", list(range(1, 12)))
def test_pack_unpack_roundtrip(bits):
    g = np.random.default_rng(bits)
    d_in = 320
    idx = g.integers(0, 1 << bits, size=(5, d_in // 2), dtype=np.int32)
    rb = oracle.row_bytes(d_in, bits)
    assert rb % 16 == 0 and rb * 8 >= (d_in // 2) * bits and rb * 8 - (d_in // 2) * bits < 128
    packed = oracle.pack(idx, bits, rb)
    assert np.array_equal(oracle.unpack(packed, d_in // 2, bits), idx)
    # the stream as one little-endian bit string, checked with numpy's unpackbits
    stream = np.unpackbits(packed[0], bitorder="little")
    vals = [int(sum(int(stream[k * bits + t]) << t for t in range(bits))) for k in range(d_in // 2)]
    assert vals == idx[0].tolist()


def test_row_bytes_of_workload_shapes():
    # (d_in, bits) -> bytes per row; all already multiples of 16
    for d_in, bits, want in [(512, 8, 256), (4096, 11, 2816), (11008, 11, 7568),
                             (5120, 7, 2240), (13824, 7, 6048)]:
        assert oracle.row_bytes(d_in, bits) == want


def test_bitrate_eq3(golden):
    for d_in, bits, printed in golden("bitrate_eq3.txt"):
        bpw = oracle.bits_per_weight(int(d_in), int(bits))
        assert round(bpw, 2) == float(printed)
    assert oracle.bits_per_weight(2048, 11) == pytest.approx(5.5078125, abs=0)


def test_block_rule(golden):
    for d_in, block in golden("block_rule.txt"):
        assert oracle.default_block(int(d_in)) == int(block)
    assert oracle.default_block(4096) == 1024      # capped
    assert oracle.default_block(11008) == 256       # 11008 = 2^8 * 43
    assert oracle.default_block(96) == 32


# ---------------------------------------------------------------- rotation

@pytest.mark.parametrize("b", [1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024])
def test_hadamard_is_sylvester_and_orthogonal(b):
    H = oracle.hadamard(b).astype(np.int64)
    assert np.array_equal(H, scipy.linalg.hadamard(b))
    assert np.array_equal(H @ H.T, b * np.eye(b, dtype=np.int64))


@pytest.mark.parametrize("b,d", [(64, 512), (128, 1024), (1024, 2048), (2, 16)])
def test_rotation_is_the_sign_masked_block_hadamard(b, d):
    seed = 7
    D = oracle.sign_mask(seed, d).astype(np.float64)
    Hs = scipy.linalg.hadamard(b).astype(np.float64) / math.sqrt(b)
    R = scipy.linalg.block_diag(*([Hs] * (d // b))) @ np.diag(D)
    g = np.random.default_rng(b)
    u = g.standard_normal(d)
    y = oracle.rotate_fwd(u, b, seed)
    assert np.allclose(y, R @ u, rtol=0, atol=1e-12)
    # Lemma 1: exact isometry; R_inv undoes R_fwd
    assert abs(np.linalg.norm(y) - np.linalg.norm(u)) <= 1e-14 * np.linalg.norm(u) * math.sqrt(d)
    assert np.allclose(oracle.rotate_inv(y, b, seed), u, rtol=0, atol=1e-13)
    assert np.allclose(oracle.rotate_inv(u, b, seed), R.T @ u, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- scales

def test_channel_scales():
    assert np.all(oracle.channel_scales(None, 8, 0.5) == 0x3C00)
    assert np.all(oracle.channel_scales(np.ones(8), 8, 0.0) == 0x3C00)
    s = oracle.channel_scales(np.array([1.0, 3.0]), 2, 1.0)  # mean 2 -> (0.5, 1.5)
    assert oracle.halves_to_f64(s).tolist() == [0.5, 1.5]
    s = oracle.channel_scales(np.array([1.0, 1.0, 1.0, 9.0]), 4, 0.5)  # mean 3
    want = np.array([1 / 3, 1 / 3, 1 / 3, 3.0]) ** 0.5
    assert np.array_equal(s, want.astype(np.float16).view(np.uint16))
    with pytest.raises(ValueError):
        oracle.channel_scales(np.array([1.0, 0.0]), 2, 0.5)
    with pytest.raises(ValueError):
        oracle.channel_scales(np.array([1.0, np.nan]), 2, 0.5)


# ---------------------------------------------------------------- calibration

def test_sigma_is_rayleigh_mean_of_unit_gaussian_rows():
    # Eq. (1): for iid Gaussian rows, unit-normalised and rotated, each pair is
    # circular Gaussian with per-coordinate std 1/sqrt(d_in); sigma*sqrt(d) ~ 1.
    d_out, d_in, b = 1024, 512, 128
    W = np.random.default_rng(3).standard_normal((d_out, d_in))
    s = oracle.channel_scales(None, d_in, 0.0)
    sig = oracle.halves_to_f64(oracle.calibrate_sigma(W, b, s, 5))
    est = sig * math.sqrt(d_in)
    assert abs(est.mean() - 1.0) < 0.01
    assert np.all(np.abs(est - 1.0) < 6 * 0.523 / math.sqrt(d_out))  # per-pair spread


def test_sigma_uses_first_1024_nonzero_rows():
    g = np.random.default_rng(4)
    d_in, b = 128, 64
    W = g.standard_normal((1500, d_in))
    W[0] = 0.0
    W[10] = 0.0
    W[1026:] *= 0.0
    W[1026:, 0] = 1.0  # rows past the calibration set: all energy in one column
    s = oracle.channel_scales(None, d_in, 0.0)
    a = oracle.calibrate_sigma(W, b, s)
    assert np.array_equal(a, oracle.calibrate_sigma(W[:1026], b, s))
    assert not np.array_equal(a, oracle.calibrate_sigma(W[:1025], b, s))
    # row scale is irrelevant (rows are unit-normalised first)
    W2 = W.copy()
    W2[5] *= 1e3
    assert np.array_equal(a, oracle.calibrate_sigma(W2, b, s))
    # a matrix with no non-zero row gets sigma = 1
    assert np.all(oracle.calibrate_sigma(np.zeros((4, d_in)), b, s) == 0x3C00)


# ---------------------------------------------------------------- nearest codeword

@pytest.mark.parametrize("K", [2, 4, 8, 16])
def test_nearest_equals_exhaustive_argmin(K):
    g = np.random.default_rng(K)
    cb = g.standard_normal((K, 2))
    p = g.standard_normal((5000, 2)) * 1.5
    d = ((p[:, None, :] - cb[None, :, :]) ** 2).sum(-1)
    assert np.array_equal(oracle.nearest(p, cb), d.argmin(1))


def test_nearest_ties_go_to_lowest_index():
    cb = np.array([[1.0, 0.0], [-1.0, 0.0], [0.0, 1.0], [1.0, 0.0]])
    p = np.array([[0.0, 0.0], [0.0, -5.0], [2.0, 0.0], [0.0, 0.5]])
    # origin: 0,1,2 tie -> 0; (0,-5): 0 and 1 tie -> 0; (2,0): 0 and 3 tie -> 0
    assert oracle.nearest(p, cb).tolist() == [0, 0, 0, 2]


# ---------------------------------------------------------------- Lloyd, eq. (2)

@pytest.fixture(scope="module")
def cb128():
    s = synth.circular_gaussian_samples(1 << 16, seed=11).astype(np.float64)
    cb, dist = oracle.lloyd(s, 128, 60)
    return cb, dist


def test_lloyd_distortion_non_increasing_and_conditions(cb128):
    cb, dist = cb128
    assert np.all(np.diff(dist) <= 1e-12)
    # nearest-neighbour condition by brute force, centroid condition approx.
    s = synth.circular_gaussian_samples(1 << 16, seed=11).astype(np.float64)
    d = ((s[:, None, :] - cb[None, :, :]) ** 2).sum(-1)
    a = d.argmin(1)
    assert np.array_equal(oracle.nearest(s, cb), a)
    means = np.array([s[a == j].mean(0) for j in range(cb.shape[0])])
    assert np.max(np.abs(means - cb)) < 2e-2


def test_lloyd_first_iteration_by_hand():
    s = synth.circular_gaussian_samples(4096, seed=2).astype(np.float64)
    cb1, dist = oracle.lloyd(s, 16, 1)
    c0 = s[:16]
    d = ((s[:, None, :] - c0[None]) ** 2).sum(-1)
    a = d.argmin(1)
    assert dist[0] == pytest.approx(d.min(1).mean(), rel=1e-12)
    want = np.array([s[a == j].mean(0) if np.any(a == j) else c0[j] for j in range(16)])
    assert np.allclose(cb1, want, rtol=0, atol=1e-12)


def test_lloyd_closed_form_K2():
    # Two cells split by a line through the origin: centroids +-sqrt(2/pi) along
    # the normal; per-pair MSE 2 - 2/pi.
    s = synth.circular_gaussian_samples(1 << 17, seed=21).astype(np.float64)
    cb, dist = oracle.lloyd(s, 2, 40)
    r = np.linalg.norm(cb, axis=1)
    assert np.allclose(r, math.sqrt(2 / math.pi), atol=0.01)
    assert np.linalg.norm(cb[0] + cb[1]) < 0.02
    assert dist[-1] == pytest.approx(2 - 2 / math.pi, abs=0.01)


def test_lloyd_closed_form_K4():
    # Four quadrant cells: centroids at radius 2/sqrt(pi), 90 degrees apart;
    # per-pair MSE 2 - 4/pi.
    s = synth.circular_gaussian_samples(1 << 17, seed=22).astype(np.float64)
    cb, dist = oracle.lloyd(s, 4, 60)
    r = np.linalg.norm(cb, axis=1)
    assert np.allclose(r, 2 / math.sqrt(math.pi), atol=0.015)
    ang = np.sort(np.mod(np.arctan2(cb[:, 1], cb[:, 0]), 2 * math.pi))
    gaps = np.diff(np.concatenate([ang, ang[:1] + 2 * math.pi]))
    assert np.allclose(gaps, math.pi / 2, atol=0.02)
    assert dist[-1] == pytest.approx(2 - 4 / math.pi, abs=0.01)


def test_lloyd_high_rate_distortion(cb128):
    # Zador/Gersho in 2D with the hexagonal cell (G = 5/(36 sqrt 3)):
    # per-pair MSE ~ 2 G (int f^(1/2))^2 / K = 2 G 8 pi / K on N(0, I_2).
    cb, _ = cb128
    held = synth.circular_gaussian_samples(1 << 16, seed=12).astype(np.float64)
    a = oracle.nearest(held, cb)
    mse = ((held - cb[a]) ** 2).sum(1).mean()
    G = 5 / (36 * math.sqrt(3))
    ratio = mse / (2 * G * 8 * math.pi / 128)
    assert 0.95 <= ratio <= 1.10, ratio


# ---------------------------------------------------------------- codec, end to end

def _rand_codebook(K, seed):
    g = np.random.default_rng(seed)
    return g.standard_normal((K, 2)) * 1.2


def test_lossless_roundtrip_on_codeword_rows():
    # One row built from codewords: W = R_inv(sigma * c_idx) with sigma chosen so
    # that ||sigma * c_idx|| = 1 up to binary16 rounding.  Then r ~ 1 and
    # p_k = c_idx_k * (1 +- 1e-3), so encoding with the same sigma recovers idx
    # exactly on a codebook with spacing 0.25, and decoding gives back r_hat * W.
    bits, d_in, b, seed = 8, 256, 64, 3
    K, P = 1 << bits, d_in // 2
    ax = (np.arange(16) - 7.5) * 0.25
    cb = np.stack(np.meshgrid(ax, ax, indexing="ij"), -1).reshape(K, 2)
    g = np.random.default_rng(9)
    idx = g.integers(0, K, size=(1, P), dtype=np.int32)
    raw = g.uniform(0.5, 1.5, P)
    raw /= np.linalg.norm(raw[:, None] * cb[idx[0]])
    sigma = oracle.f64_to_halves(raw)
    sg = oracle.halves_to_f64(sigma)
    y = (sg[:, None] * cb[idx[0]]).reshape(-1)
    W = oracle.rotate_inv(y, b, seed)[None, :]
    enc = oracle.encode(W, bits, b, cb, mask_seed=seed, sigma_half=sigma)
    assert np.array_equal(enc["idx"], idx)
    rhat = oracle.halves_to_f64(enc["rnorm_half"])[0]
    assert abs(rhat - 1.0) < 2e-3
    Wd = oracle.decode(enc, cb)
    assert np.allclose(Wd, rhat * W, rtol=1e-12, atol=1e-15)


def test_zero_row_is_encoded_as_zero_row():
    cb = _rand_codebook(16, 1)
    W = np.random.default_rng(0).standard_normal((3, 64))
    W[1] = 0.0
    enc = oracle.encode(W, 4, 64, cb)
    assert np.all(enc["idx"][1] == 0) and enc["rnorm_half"][1] == 0
    assert np.all(oracle.decode(enc, cb)[1] == 0.0)


def test_end_to_end_mse_on_gaussian_rows(cb128):
    # sum_k sigma_k^2 MSE_pair ~ MSE_pair/2 for unit rows (2.015/K at high rate)
    cb, _ = cb128
    d_in, b = 1024, 128
    W = np.random.default_rng(31).standard_normal((64, d_in))
    enc = oracle.encode(W, 7, b, cb, mask_seed=1)
    Wd = oracle.decode(enc, cb)
    U = W / np.linalg.norm(W, axis=1, keepdims=True)
    Ud = Wd / np.linalg.norm(W, axis=1, keepdims=True)
    rel = ((U - Ud) ** 2).sum(1).mean()
    held = synth.circular_gaussian_samples(1 << 15, seed=13).astype(np.float64)
    mse_pair = ((held - cb[oracle.nearest(held, cb)]) ** 2).sum(1).mean()
    assert 0.85 <= rel / (mse_pair / 2) <= 1.2


def test_gemv_and_trace_identity():
    g = np.random.default_rng(8)
    W = g.standard_normal((40, 64))
    X = g.standard_normal((5, 64))
    assert np.allclose(oracle.gemv(W, X), X @ W.T, rtol=1e-13, atol=1e-12)
    dW = g.standard_normal((40, 64)) * 1e-2
    lhs = (oracle.gemv(dW, X) ** 2).sum()
    rhs = np.trace(dW @ (X.T @ X) @ dW.T)
    assert lhs == pytest.approx(rhs, rel=1e-12)


def test_activation_aware_scaling_lowers_output_error():
    # The layer-output error ||X dW^T||^2 = Tr(dW Mx dW^T) weights column j by the
    # activation energy of channel j; scaling W by s_j ~ a_j^alpha before
    # quantisation (and dividing after) lowers it when a few channels dominate.
    d_out, d_in, b = 96, 512, 128
    W = synth.student_t_weights(d_out, d_in, seed=4).astype(np.float64)
    a = synth.act_stat_lognormal(d_in, seed=4).astype(np.float64)
    cb = oracle.lloyd(synth.circular_gaussian_samples(1 << 14, 6).astype(np.float64), 64, 25)[0]
    err = {}
    for alpha in (0.0, 0.5):
        enc = oracle.encode(W, 6, b, cb, act_stat=a, alpha=alpha, mask_seed=2)
        dW = oracle.decode(enc, cb) - W
        err[alpha] = np.sum(dW ** 2 * (a ** 2)[None, :])
    assert err[0.5] < 0.8 * err[0.0], err
