"""Normalised points of a matrix on the GPU against the oracle, and a codebook
trained on them (the per-checkpoint codebook that the explainer page's
"Significance and Claims" suggests in place of the unit circular Gaussian).

Rule: the points are z_k / sigma_k in fp32 from the same s and sigma as the
oracle's fp64 points; they agree to 2e-5 (1 + |p|) (a few fp32 ulps of the
rotation and the two normalisations).
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import halves, log_stats
from vector_quantization_codec_b200 import qamw, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def gaussian_codebook(bits):
    # a quick Lloyd codebook of N(0, I_2) from the oracle (small K only)
    K = 1 << bits
    train = synth.circular_gaussian_samples(64 * K, seed=bits).astype(np.float64)
    cb, _ = oracle.lloyd(train, K, 20)
    return cb


@pytest.mark.parametrize("case", [(40, 1024, 128, 8, "bf16"), (23, 576, 64, 6, "f32")],
                         ids=lambda c: f"{c[0]}x{c[1]}_b{c[2]}_{c[4]}")
def test_normalised_pairs_match_oracle(case):
    d_out, d_in, block, bits, dtype = case
    W32 = synth.student_t_weights(d_out, d_in, seed=d_in)
    W32[3] = 0.0  # a zero row: NaN points
    Wt = torch.from_numpy(W32).to(torch.bfloat16) if dtype == "bf16" else torch.from_numpy(W32)
    W = Wt.double().numpy()
    cbt = torch.from_numpy(gaussian_codebook(bits)).float().to(DEV)
    m = qamw.EncodedMatrix.empty(d_out, d_in, block, bits, cbt, 5)
    act = torch.from_numpy(synth.act_stat_lognormal(d_in, seed=1)).to(DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    qamw.qamw_encode(Wt.to(DEV), m, act, 0.5, status=st)
    pts = qamw.qamw_normalised_pairs(Wt.to(DEV), m, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    got = pts.cpu().numpy().astype(np.float64)
    enc = oracle.encode(W, bits, block, cbt.cpu().numpy().astype(np.float64), mask_seed=5,
                        s_half=halves(m.chan_scale), sigma_half=halves(m.sigma), want_points=True)
    want = enc["points"]
    assert np.isnan(got[3]).all()
    ok = np.delete(np.arange(d_out), 3)
    err = np.abs(got[ok] - want[ok])
    ratio = float((err / (2e-5 * (1.0 + np.abs(want[ok])))).max())
    log_stats("normalised pairs", dict(max_ratio=ratio))
    assert ratio <= 1.0, ratio
    # a row range is the same slice of the whole
    part = qamw.qamw_normalised_pairs(Wt.to(DEV), m, row0=7, nrows=11)
    torch.cuda.synchronize()
    assert torch.equal(part, pts[7:18])


def test_codebook_trained_on_matrix_points():
    d_out, d_in, block, bits = 256, 1024, 128, 6
    Wt = torch.from_numpy(synth.student_t_weights(d_out, d_in, seed=11)).to(torch.bfloat16).to(DEV)
    cb_g = torch.from_numpy(gaussian_codebook(bits)).float().to(DEV)
    m = qamw.EncodedMatrix.empty(d_out, d_in, block, bits, cb_g)
    qamw.qamw_encode(Wt, m, torch.from_numpy(synth.act_stat_lognormal(d_in, seed=2)).to(DEV), 0.5)
    pts = qamw.qamw_normalised_pairs(Wt, m).reshape(-1, 2).contiguous()
    K, iters = 1 << bits, 30
    cb_m = torch.empty((K, 2), dtype=torch.float32, device=DEV)
    dist = torch.empty(iters, dtype=torch.float64, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    qamw.qamw_train_codebook(pts, bits, iters, cb_m, dist, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    d = dist.cpu().numpy()
    assert np.all(np.diff(d) <= 1e-12 * d[0]), d
    # fitted to this matrix's own points, it beats the Gaussian codebook on them
    P = pts.cpu().numpy().astype(np.float64)[::7]
    mse = []
    for cb in (cb_m, cb_g):
        c = cb.cpu().numpy().astype(np.float64)
        mse.append(float(((P - c[oracle.nearest(P, c)]) ** 2).sum(1).mean()))
    log_stats("per-matrix codebook", dict(mse_matrix=mse[0], mse_gaussian=mse[1]))
    assert mse[0] < mse[1], mse
