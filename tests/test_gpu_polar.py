"""Polar baseline on the GPU (QAM-W paper section 3.5) against the oracle.

Index rule: the amplitude and phase parts of an index must equal the oracle's,
except where the oracle's fp64 point lies within fp32 rounding of a decision
boundary -- an amplitude midway between two levels (| |r-a_g| - |r-a_o| |
<= 1e-5 (1 + r)) or a phase midway between two bin centres (the bin
coordinate u = theta Np / 2 pi within 1e-4 of a half-integer).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.parity import bf16_to_f64, check_close, halves, log_stats, ulp_diff
from vector_quantization_codec_b200 import qamw, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("bits", [1, 3, 7, 8, 11])
def test_polar_codebook_matches_oracle(bits):
    got = qamw.qamw_polar_codebook(bits).cpu().numpy().astype(np.float64)
    want = oracle.polar_codebook(bits)
    assert np.max(np.abs(got - want)) <= 2e-6


def check_polar_indices(got, want, points, levels, bits):
    Np = 1 << oracle.polar_split(bits)[1]
    diff = got != want
    r_, k_ = np.nonzero(diff)
    bad = 0
    for i, k in zip(r_, k_):
        p = points[i, k]
        r = math.hypot(p[0], p[1])
        ga, gp = divmod(int(got[i, k]), Np)
        oa, op = divmod(int(want[i, k]), Np)
        ok = True
        if ga != oa:
            ok &= abs(abs(r - levels[ga]) - abs(r - levels[oa])) <= 1e-5 * (1 + r)
        if gp != op:
            u = math.atan2(p[1], p[0]) * Np / (2 * math.pi)
            ok &= abs((u - math.floor(u)) - 0.5) <= 1e-4
        bad += not ok
    stats = dict(n=int(diff.size), mismatches=int(diff.sum()), bad=bad)
    log_stats("polar indices", stats)
    assert bad == 0, stats
    assert stats["mismatches"] <= max(8, 1e-4 * diff.size), stats
    return stats


@pytest.mark.parametrize("case", [(64, 1024, 128, 7, "bf16"), (33, 4096, 128, 11, "bf16"),
                                  (20, 512, 64, 8, "f32"), (9, 192, 64, 3, "f32")],
                         ids=lambda c: f"{c[0]}x{c[1]}_B{c[3]}_{c[4]}")
def test_polar_encode_decode_match_oracle(case):
    d_out, d_in, block, bits, dtype = case
    Np = 1 << oracle.polar_split(bits)[1]
    cbt = qamw.qamw_polar_codebook(bits)
    cb = cbt.cpu().numpy().astype(np.float64)
    levels = cb[::Np, 0].copy()
    W32 = synth.student_t_weights(d_out, d_in, seed=d_in + bits)
    Wt = torch.from_numpy(W32).to(torch.bfloat16) if dtype == "bf16" else torch.from_numpy(W32)
    W = Wt.double().numpy()
    act = synth.act_stat_lognormal(d_in, seed=bits)
    m = qamw.EncodedMatrix.empty(d_out, d_in, block, bits, cbt, 2)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    qamw.qamw_encode(Wt.to(DEV), m, torch.from_numpy(act).to(DEV), 0.5, flags=qamw.QAMW_POLAR,
                     status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    s_g, sig_g = halves(m.chan_scale), halves(m.sigma)
    assert ulp_diff(sig_g, oracle.calibrate_sigma(W, block, s_g, 2)).max() <= 1
    enc = oracle.encode_polar(W, bits, block, levels, mask_seed=2, s_half=s_g, sigma_half=sig_g,
                              want_points=True)
    assert ulp_diff(halves(m.row_norm), enc["rnorm_half"]).max() <= 1
    idx_g = oracle.unpack(m.packed.cpu().numpy(), d_in // 2, bits)
    check_polar_indices(idx_g, enc["idx"], enc["points"], levels, bits)
    # the polar table is an ordinary codebook for the decoder and the GEMV
    enc["packed"] = m.packed.cpu().numpy()
    enc["rnorm_half"] = halves(m.row_norm)
    ref = oracle.decode(enc, cb)
    check_close(bf16_to_f64(qamw.qamw_decode(m)), ref, what="polar decode")
    xt = torch.from_numpy(synth.gemv_x(2, d_in, seed=1)).to(torch.bfloat16)
    y = bf16_to_f64(qamw.qamw_decode_gemv(m, xt.to(DEV)))
    yref = oracle.gemv(ref, xt.double().numpy())
    for t in range(2):
        check_close(y[t], yref[t], what=f"polar gemv col {t}")


def test_polar_stage_call_equals_composite():
    d_out, d_in, block, bits = 40, 1024, 128, 11
    cbt = qamw.qamw_polar_codebook(bits)
    Wt = torch.from_numpy(synth.student_t_weights(d_out, d_in, seed=5)).to(torch.bfloat16).to(DEV)
    m1 = qamw.EncodedMatrix.empty(d_out, d_in, block, bits, cbt)
    qamw.qamw_encode(Wt, m1, flags=qamw.QAMW_POLAR)
    m2 = qamw.EncodedMatrix(d_out, d_in, block, bits, 0, torch.empty_like(m1.packed),
                            torch.empty_like(m1.row_norm), m1.sigma, m1.chan_scale, cbt)
    qamw.qamw_encode_rows_polar(Wt, m2)
    torch.cuda.synchronize()
    assert torch.equal(m1.packed, m2.packed)
