"""The d = 1 scalar ablation on the GPU (QAM-W paper section 2, "parallel work")
against the oracle.

Index rule: each coordinate's level must equal the oracle's, except where the
oracle's fp64 coordinate lies within fp32 rounding of the midpoint between the
two levels (| |v - l_g| - |v - l_o| | <= 1e-5 (1 + |v|)); every such case is
counted.  Decoded weights and GEMV outputs follow the 1e-2 rule of the other
parity tests (the product table is an ordinary codebook for those kernels).
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import bf16_to_f64, check_close, halves, log_stats, ulp_diff
from tests.test_gpu_parity import codebook
from vector_quantization_codec_b200 import qamw, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("bits", [2, 4, 6, 8, 10])
def test_scalar_codebook_matches_oracle(bits):
    got = qamw.qamw_scalar_codebook(bits).cpu().numpy().astype(np.float64)
    want = oracle.scalar_codebook(bits)
    assert np.max(np.abs(got - want)) <= 2e-6


def check_scalar_indices(got, want, points, levels, bits):
    L = 1 << (bits // 2)
    diff = got != want
    r_, k_ = np.nonzero(diff)
    bad = 0
    for i, k in zip(r_, k_):
        p = points[i, k]
        g2, o2 = divmod(int(got[i, k]), L), divmod(int(want[i, k]), L)
        for v, gl, ol in ((p[0], g2[0], o2[0]), (p[1], g2[1], o2[1])):
            if gl != ol:
                bad += abs(abs(v - levels[gl]) - abs(v - levels[ol])) > 1e-5 * (1 + abs(v))
    stats = dict(n=int(diff.size), mismatches=int(diff.sum()), bad=int(bad))
    log_stats("scalar indices", stats)
    assert bad == 0, stats
    assert stats["mismatches"] <= max(8, 1e-4 * diff.size), stats
    return stats


@pytest.mark.parametrize("case", [(64, 1024, 128, 8, "bf16"), (33, 4096, 128, 10, "bf16"),
                                  (20, 512, 64, 6, "f32"), (9, 192, 64, 2, "f32"),
                                  (17, 5120, 128, 6, "bf16"), (5, 13824, 128, 4, "bf16")],
                         ids=lambda c: f"{c[0]}x{c[1]}_B{c[3]}_{c[4]}")
def test_scalar_encode_decode_gemv_match_oracle(case):
    d_out, d_in, block, bits, dtype = case
    L = 1 << (bits // 2)
    cbt = qamw.qamw_scalar_codebook(bits)
    cb = cbt.cpu().numpy().astype(np.float64)
    levels = cb[::L, 0].copy()
    W32 = synth.student_t_weights(d_out, d_in, seed=d_in + bits)
    Wt = torch.from_numpy(W32).to(torch.bfloat16) if dtype == "bf16" else torch.from_numpy(W32)
    W = Wt.double().numpy()
    act = synth.act_stat_lognormal(d_in, seed=bits)
    m = qamw.EncodedMatrix.empty(d_out, d_in, block, bits, cbt, 2)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    qamw.qamw_encode(Wt.to(DEV), m, torch.from_numpy(act).to(DEV), 0.5, flags=qamw.QAMW_SCALAR,
                     status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    s_g, sig_g = halves(m.chan_scale), halves(m.sigma)
    assert ulp_diff(sig_g, oracle.calibrate_sigma(W, block, s_g, 2)).max() <= 1
    enc = oracle.encode_scalar(W, bits, block, levels, mask_seed=2, s_half=s_g, sigma_half=sig_g,
                               want_points=True)
    assert ulp_diff(halves(m.row_norm), enc["rnorm_half"]).max() <= 1
    idx_g = oracle.unpack(m.packed.cpu().numpy(), d_in // 2, bits)
    check_scalar_indices(idx_g, enc["idx"], enc["points"], levels, bits)
    enc["packed"] = m.packed.cpu().numpy()
    enc["rnorm_half"] = halves(m.row_norm)
    ref = oracle.decode(enc, cb)
    check_close(bf16_to_f64(qamw.qamw_decode(m)), ref, what="scalar decode")
    for batch in (1, 5):
        xt = torch.from_numpy(synth.gemv_x(batch, d_in, seed=batch)).to(torch.bfloat16)
        y = bf16_to_f64(qamw.qamw_decode_gemv(m, xt.to(DEV)))
        yref = oracle.gemv(ref, xt.double().numpy())
        for t in range(batch):
            check_close(y[t], yref[t], what=f"scalar gemv b{batch} col {t}")


def test_scalar_stage_call_equals_composite():
    d_out, d_in, block, bits = 40, 1024, 128, 8
    cbt = qamw.qamw_scalar_codebook(bits)
    Wt = torch.from_numpy(synth.student_t_weights(d_out, d_in, seed=5)).to(torch.bfloat16).to(DEV)
    m1 = qamw.EncodedMatrix.empty(d_out, d_in, block, bits, cbt)
    qamw.qamw_encode(Wt, m1, flags=qamw.QAMW_SCALAR)
    m2 = qamw.EncodedMatrix(d_out, d_in, block, bits, 0, torch.empty_like(m1.packed),
                            torch.empty_like(m1.row_norm), m1.sigma, m1.chan_scale, cbt)
    qamw.qamw_encode_rows_scalar(Wt, m2)
    torch.cuda.synchronize()
    assert torch.equal(m1.packed, m2.packed)


@pytest.mark.parametrize("bits", [6, 8])
def test_joint_2d_beats_scalar_on_the_gpu_at_equal_bits(bits):
    # the same matrix encoded with the joint K = 2^bits codebook (Lloyd on
    # N(0, I_2)) and with the scalar code of bits / 2 bits per coordinate: the
    # joint code reconstructs it with less error
    d_out, d_in, block = 512, 2048, 128
    K = 1 << bits
    samples = torch.from_numpy(synth.circular_gaussian_samples(2048 * K, seed=80 + bits)).to(DEV)
    cb2d = torch.empty((K, 2), dtype=torch.float32, device=DEV)
    qamw.qamw_train_codebook(samples, bits, 40, cb2d)
    cb1d = qamw.qamw_scalar_codebook(bits)
    Wt = torch.from_numpy(synth.student_t_weights(d_out, d_in, seed=bits)).to(torch.bfloat16).to(DEV)
    errs = {}
    for name, cb, flags in (("joint", cb2d, 0), ("scalar", cb1d, qamw.QAMW_SCALAR)):
        m = qamw.EncodedMatrix.empty(d_out, d_in, block, bits, cb, 1,
                                     qamw.qamw_build_prefilter(cb, bits) if flags == 0 else None)
        qamw.qamw_encode(Wt, m, flags=flags)
        out = qamw.qamw_decode(m)
        torch.cuda.synchronize()
        errs[name] = float(((out.float() - Wt.float()).norm() / Wt.float().norm()) ** 2)
    log_stats("joint vs scalar rel mse", dict(bits=bits, **errs))
    assert errs["joint"] < 0.97 * errs["scalar"], errs


def test_scalar_arguments():
    cbt = qamw.qamw_scalar_codebook(4)
    m = qamw.EncodedMatrix.empty(4, 128, 64, 7, cbt)
    W = torch.zeros((4, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(qamw.QamwError) as e:
        qamw.qamw_encode_rows_scalar(W, m)  # odd bits
    assert e.value.rc == qamw.QAMW_ERR_INVALID
    with pytest.raises(qamw.QamwError) as e:
        qamw.qamw_scalar_codebook(7)
    assert e.value.rc == qamw.QAMW_ERR_INVALID
    m4 = qamw.EncodedMatrix.empty(4, 128, 64, 4, cbt)
    with pytest.raises(qamw.QamwError) as e:
        qamw.qamw_encode(W, m4, flags=qamw.QAMW_SCALAR | qamw.QAMW_POLAR)
    assert e.value.rc == qamw.QAMW_ERR_INVALID
