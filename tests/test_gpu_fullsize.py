"""Parity at the benchmarked shapes, on sampled rows the oracle can compute.

* The 11008x4096 MLP matrix (K = 2048, block 128, alpha 0.5) in full on the
  GPU: side values against the oracle, then indices, decode and decode-GEMV at
  batch 1, 4 and 16 on sampled rows (first, last, around row 1024, random).
* The 13B shapes of the 3.5 bpw workload (d_in = 5120 and 13824, K = 128,
  block 128): joint 2-D codebook and the polar quantiser of the same K, on a
  few dozen rows -- 80 and 216 chunks a row, so the last 2048-column slice is
  ragged (16 and 24 chunks).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from tests.parity import bf16_to_f64, check_close, check_indices, halves, ulp_diff
from tests.test_gpu_parity import codebook, gpu_encode
from tests.test_gpu_polar import check_polar_indices
from vector_quantization_codec_b200 import qamw, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_full_size_11008x4096_sampled_rows():
    d_out, d_in, block, bits, alpha = 11008, 4096, 128, 11, 0.5
    cb = codebook(bits)
    Wt = torch.from_numpy(synth.student_t_weights(d_out, d_in, seed=31)).to(torch.bfloat16)
    act = synth.act_stat_lognormal(d_in, seed=31)
    m, status = gpu_encode(Wt.to(DEV), d_in, block, bits, cb, act, alpha, seed=6)
    assert status == 0
    W = Wt[:1024].double().numpy()
    s_g, sig_g, r_g = halves(m.chan_scale), halves(m.sigma), halves(m.row_norm)
    assert ulp_diff(s_g, oracle.channel_scales(act.astype(np.float64), d_in, alpha)).max() <= 1
    assert ulp_diff(sig_g, oracle.calibrate_sigma(W, block, s_g, 6)).max() <= 1
    rows = np.unique(np.concatenate([[0, 1, 1023, 1024, 5503, 11006, 11007],
                                     np.random.default_rng(1).choice(d_out, 41, replace=False)]))
    Wr = Wt[rows].double().numpy()
    enc = oracle.encode(Wr, bits, block, cb, mask_seed=6, s_half=s_g, sigma_half=sig_g,
                        want_points=True)
    assert ulp_diff(r_g[rows], enc["rnorm_half"]).max() <= 1
    packed = m.packed.cpu().numpy()[rows]
    check_indices(oracle.unpack(packed, d_in // 2, bits), enc["idx"], enc["points"], cb)
    sub = dict(packed=packed, rnorm_half=r_g[rows], sigma_half=sig_g, s_half=s_g, d_out=len(rows),
               d_in=d_in, block=block, bits=bits, mask_seed=6)
    ref = oracle.decode(sub, cb)
    check_close(bf16_to_f64(qamw.qamw_decode(m))[rows], ref, what="decode 11008x4096")
    for batch in (1, 4, 16):
        xt = torch.from_numpy(synth.gemv_x(batch, d_in, seed=100 + batch)).to(torch.bfloat16)
        y = bf16_to_f64(qamw.qamw_decode_gemv(m, xt.to(DEV)))[:, rows]
        yref = oracle.gemv(ref, xt.double().numpy())
        for t in range(batch):
            check_close(y[t], yref[t], what=f"gemv 11008x4096 b{batch} col {t}")


@pytest.mark.parametrize("d_in", [5120, 13824])
def test_13b_shapes_k128_joint(d_in):
    d_out, block, bits = 37, 128, 7
    cb = codebook(bits)
    Wt = torch.from_numpy(synth.student_t_weights(d_out, d_in, seed=d_in)).to(torch.bfloat16)
    W = Wt.double().numpy()
    act = synth.act_stat_lognormal(d_in, seed=d_in)
    m, status = gpu_encode(Wt.to(DEV), d_in, block, bits, cb, act, 0.5, seed=9)
    assert status == 0
    s_g, sig_g = halves(m.chan_scale), halves(m.sigma)
    assert ulp_diff(sig_g, oracle.calibrate_sigma(W, block, s_g, 9)).max() <= 1
    enc = oracle.encode(W, bits, block, cb, mask_seed=9, s_half=s_g, sigma_half=sig_g,
                        want_points=True)
    assert ulp_diff(halves(m.row_norm), enc["rnorm_half"]).max() <= 1
    check_indices(oracle.unpack(m.packed.cpu().numpy(), d_in // 2, bits), enc["idx"],
                  enc["points"], cb)
    enc["packed"] = m.packed.cpu().numpy()
    enc["rnorm_half"] = halves(m.row_norm)
    ref = oracle.decode(enc, cb)
    check_close(bf16_to_f64(qamw.qamw_decode(m)), ref, what=f"decode 13b {d_in}")
    for batch in (1, 4, 16):
        xt = torch.from_numpy(synth.gemv_x(batch, d_in, seed=batch)).to(torch.bfloat16)
        y = bf16_to_f64(qamw.qamw_decode_gemv(m, xt.to(DEV)))
        yref = oracle.gemv(ref, xt.double().numpy())
        for t in range(batch):
            check_close(y[t], yref[t], what=f"gemv 13b {d_in} b{batch} col {t}")


@pytest.mark.parametrize("d_in", [5120, 13824])
def test_13b_shapes_k128_polar(d_in):
    d_out, block, bits = 29, 128, 7
    Np = 1 << oracle.polar_split(bits)[1]
    cbt = qamw.qamw_polar_codebook(bits)
    cb = cbt.cpu().numpy().astype(np.float64)
    levels = cb[::Np, 0].copy()
    Wt = torch.from_numpy(synth.student_t_weights(d_out, d_in, seed=d_in + 1)).to(torch.bfloat16)
    W = Wt.double().numpy()
    act = synth.act_stat_lognormal(d_in, seed=d_in + 1)
    m = qamw.EncodedMatrix.empty(d_out, d_in, block, bits, cbt, 4)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    qamw.qamw_encode(Wt.to(DEV), m, torch.from_numpy(act).to(DEV), 0.5, flags=qamw.QAMW_POLAR,
                     status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    s_g, sig_g = halves(m.chan_scale), halves(m.sigma)
    enc = oracle.encode_polar(W, bits, block, levels, mask_seed=4, s_half=s_g, sigma_half=sig_g,
                              want_points=True)
    check_polar_indices(oracle.unpack(m.packed.cpu().numpy(), d_in // 2, bits), enc["idx"],
                        enc["points"], levels, bits)
    enc["packed"] = m.packed.cpu().numpy()
    enc["rnorm_half"] = halves(m.row_norm)
    ref = oracle.decode(enc, cb)
    check_close(bf16_to_f64(qamw.qamw_decode(m)), ref, what=f"polar decode 13b {d_in}")
    xt = torch.from_numpy(synth.gemv_x(4, d_in, seed=3)).to(torch.bfloat16)
    y = bf16_to_f64(qamw.qamw_decode_gemv(m, xt.to(DEV)))
    yref = oracle.gemv(ref, xt.double().numpy())
    for t in range(4):
        check_close(y[t], yref[t], what=f"polar gemv 13b {d_in} col {t}")
