"""The prefill-size decode-GEMM on the tensor cores (tcgen05, accumulator in
tensor memory) against the fp64 oracle's dense product Y = X W_hat^T.

Token counts of one and two 64-token tiles and a ragged count; shapes with one
and several 128-row tiles and a ragged last tile; K ranges split over CTAs;
the full 4096x4096 and 11008x4096 K = 2048 matrices on sampled rows.  The rule
is the 1e-2 rule of the other product tests, per token (column of the output's
transpose)."""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import bf16_to_f64, check_close, halves
from tests.test_gpu_parity import codebook, gpu_encode, weights
from vector_quantization_codec_b200 import qamw, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def oracle_What(m, cb, rows=None):
    packed = m.packed.cpu().numpy()
    rn = halves(m.row_norm)
    if rows is not None:
        packed, rn = packed[rows], rn[rows]
    enc = dict(packed=packed, rnorm_half=rn, sigma_half=halves(m.sigma), s_half=halves(m.chan_scale),
               d_out=packed.shape[0], d_in=m.d_in, block=m.block, bits=m.bits, mask_seed=m.mask_seed)
    return oracle.decode(enc, cb)


CASES = [(300, 1024, 128, 11, 64), (300, 1024, 128, 11, 128), (97, 4096, 1024, 7, 100),
         (24, 11008, 128, 11, 64), (130, 2048, 64, 9, 3), (64, 192, 64, 3, 70)]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}x{c[1]}_b{c[2]}_B{c[3]}_t{c[4]}")
def test_decode_gemm_matches_oracle(case):
    d_out, d_in, block, bits, ntok = case
    cb = codebook(bits)
    Wt, _ = weights(d_out, d_in, 11 + d_out, "bf16")
    act = synth.act_stat_lognormal(d_in, seed=4)
    m, status = gpu_encode(Wt, d_in, block, bits, cb, act, 0.5, seed=7)
    assert status == 0
    What = oracle_What(m, cb)
    xt = torch.from_numpy(synth.gemv_x(ntok, d_in, seed=ntok)).to(torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = qamw.qamw_decode_gemm(m, xt.to(DEV), status=st)
    torch.cuda.synchronize()
    assert st.item() == 0, qamw.status_string(st.item())
    got = bf16_to_f64(y)
    ref = oracle.gemv(What, xt.double().numpy())
    for t in range(ntok):
        check_close(got[t], ref[t], what=f"gemm token {t}")


@pytest.mark.parametrize("d_out,ntok", [(4096, 64), (4096, 128), (11008, 128)])
def test_decode_gemm_full_size_sampled_rows(d_out, ntok):
    d_in, block, bits = 4096, 128, 11
    cb = codebook(bits)
    Wt = torch.from_numpy(synth.student_t_weights(d_out, d_in, seed=d_out)).to(torch.bfloat16)
    act = synth.act_stat_lognormal(d_in, seed=5)
    m, status = gpu_encode(Wt.to(DEV), d_in, block, bits, cb, act, 0.5, seed=2)
    assert status == 0
    rows = np.unique(np.concatenate([[0, 127, 128, d_out - 1],
                                     np.random.default_rng(d_out).choice(d_out, 44, replace=False)]))
    What = oracle_What(m, cb, rows)
    xt = torch.from_numpy(synth.gemv_x(ntok, d_in, seed=3)).to(torch.bfloat16)
    y = bf16_to_f64(qamw.qamw_decode_gemm(m, xt.to(DEV)))[:, rows]
    torch.cuda.synchronize()
    ref = oracle.gemv(What, xt.double().numpy())
    # the rms floor of the rule is taken over the sampled rows of each token
    for t in range(ntok):
        check_close(y[t], ref[t], what=f"gemm {d_out} token {t}")


def test_decode_gemm_arguments():
    bits = 7
    cb = torch.from_numpy(codebook(bits)).to(DEV)
    m = qamw.EncodedMatrix.empty(16, 256, 64, bits, cb)
    x = torch.zeros((8, 256), dtype=torch.bfloat16, device=DEV)
    need = qamw.qamw_workspace_bytes(qamw.QAMW_OP_GEMM, 16, 256, bits, 8)
    assert need > 0
    assert qamw.qamw_workspace_bytes(qamw.QAMW_OP_GEMM, 16, 256, bits, 0) == 0
    with pytest.raises(qamw.QamwError) as e:
        qamw.qamw_decode_gemm(m, x, workspace=torch.empty(need - 16, dtype=torch.uint8, device=DEV))
    assert e.value.rc == qamw.QAMW_ERR_WORKSPACE
    with pytest.raises(qamw.QamwError) as e:
        qamw.qamw_decode_gemm(m, x[:0])
    assert e.value.rc == qamw.QAMW_ERR_INVALID
