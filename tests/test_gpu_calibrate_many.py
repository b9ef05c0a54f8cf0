"""qamw_calibrate_many (channel scales and eq. (1) of many matrices in four
launches per 64) against the fp64 oracle and against the single calls.

The matrices differ in shape, Hadamard block, mask seed and statistic; one has
zero rows past its first 1024 (the in-order extension of eq. (1)), one has no
statistic (s = 1), one is wider than 11008 columns, and one call holds more
matrices than one launch takes."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from tests.parity import halves, ulp_diff
from tests.test_gpu_parity import codebook
from vector_quantization_codec_b200 import qamw, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def make(d_out, d_in, block, seed, zero_head=False):
    W = synth.student_t_weights(d_out, d_in, seed=seed)
    if zero_head:  # rows 0..1999 zero except 50: eq. (1) reads on past row 1024
        keep = np.zeros(d_out, dtype=bool)
        keep[np.random.default_rng(seed).choice(2000, 50, replace=False)] = True
        keep[2000:] = True
        W[~keep] = 0.0
    Wt = torch.from_numpy(W).to(torch.bfloat16)
    return Wt.to(DEV), Wt.double().numpy()


@pytest.mark.parametrize("ncopies", [1, 10])
def test_calibrate_many_matches_oracle_and_single_calls(ncopies):
    bits = 7
    cbt = torch.from_numpy(codebook(bits)).to(DEV)
    shapes = [(300, 1024, 128, False, True), (2600, 256, 64, True, True), (64, 11008, 128, False, True),
              (40, 4096, 1024, False, False), (17, 16384, 256, False, True), (9, 192, 64, False, True)]
    shapes = shapes * ncopies  # 60 matrices: one launch group; 6: a short one
    Ws, W64, acts, ms, ms1 = [], [], [], [], []
    for i, (d_out, d_in, block, zh, has_stat) in enumerate(shapes):
        Wt, W = make(d_out, d_in, block, 40 + i, zh)
        Ws.append(Wt)
        W64.append(W)
        acts.append(torch.from_numpy(synth.act_stat_lognormal(d_in, seed=i)).to(DEV) if has_stat else None)
        ms.append(qamw.EncodedMatrix.empty(d_out, d_in, block, bits, cbt, 7 + i))
        ms1.append(qamw.EncodedMatrix.empty(d_out, d_in, block, bits, cbt, 7 + i))
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    qamw.qamw_calibrate_many(Ws, ms, acts, 0.5, status=st)
    for Wt, a, m in zip(Ws, acts, ms1):
        qamw.qamw_channel_scales(m.d_in, a, 0.5, m.chan_scale, status=st)
        qamw.qamw_calibrate_sigma(Wt, m, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0, qamw.status_string(st.item())
    for i, (m, m1, W, a) in enumerate(zip(ms, ms1, W64, acts)):
        s_g, sig_g = halves(m.chan_scale), halves(m.sigma)
        assert np.array_equal(s_g, halves(m1.chan_scale)), i
        assert np.array_equal(sig_g, halves(m1.sigma)), i
        s_o = oracle.channel_scales(None if a is None else a.cpu().numpy().astype(np.float64),
                                    m.d_in, 0.5)
        assert ulp_diff(s_g, s_o).max() <= 1, i
        sig_o = oracle.calibrate_sigma(W, m.block, s_g, m.mask_seed)
        assert ulp_diff(sig_g, sig_o).max() <= 1, i


def test_calibrate_many_workspace_and_argument_errors():
    bits = 7
    cbt = torch.from_numpy(codebook(bits)).to(DEV)
    ms = [qamw.EncodedMatrix.empty(8, 256, 64, bits, cbt), qamw.EncodedMatrix.empty(8, 4096, 128, bits, cbt)]
    Ws = [torch.zeros((8, 256), dtype=torch.bfloat16, device=DEV),
          torch.zeros((8, 4096), dtype=torch.bfloat16, device=DEV)]
    need = qamw.qamw_calibrate_many_workspace_bytes(ms)
    one = sum(qamw.qamw_workspace_bytes(qamw.QAMW_OP_CALIBRATE, m.d_out, m.d_in, bits) for m in ms)
    assert need == one
    small = torch.empty(need - 16, dtype=torch.uint8, device=DEV)
    with pytest.raises(qamw.QamwError) as e:
        qamw.qamw_calibrate_many(Ws, ms, None, 0.5, workspace=small)
    assert e.value.rc == qamw.QAMW_ERR_WORKSPACE
    with pytest.raises(qamw.QamwError) as e:  # a weight pointer off the 16-byte grid
        qamw.qamw_calibrate_many([Ws[0].view(-1)[1:], Ws[1]], ms, None, 0.5)
    assert e.value.rc == qamw.QAMW_ERR_ALIGN
    # all-zero matrices: sigma = 1, scales 1 without a statistic
    qamw.qamw_calibrate_many(Ws, ms, None, 0.5)
    torch.cuda.synchronize()
    for m in ms:
        assert np.all(halves(m.sigma) == 0x3C00) and np.all(halves(m.chan_scale) == 0x3C00)
