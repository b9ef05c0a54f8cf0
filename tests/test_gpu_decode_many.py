"""qamw_decode_many (one launch over many matrices) against the fp64 oracle and
against qamw_decode of each matrix alone.

The matrices of one call differ in shape, Hadamard block, mask seed and side
values; they include a ragged last slice (11008 columns = 172 chunks), a matrix
narrower than one slice (192 columns), a block of 1 (which starts a second
launch group: its table is not folded), an empty matrix, and more matrices than
one launch takes (70 > 64)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from tests.parity import bf16_to_f64, check_close, to_half_tensor
from tests.test_gpu_parity import codebook
from vector_quantization_codec_b200 import qamw, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def oracle_matrix(d_out, d_in, block, bits, seed, cbt, cb):
    if d_out == 0:
        m = qamw.EncodedMatrix.empty(0, d_in, block, bits, cbt, seed)
        m.sigma.fill_(1.0)
        m.chan_scale.fill_(1.0)
        return m, np.zeros((0, d_in))
    W = synth.student_t_weights(d_out, d_in, seed=seed).astype(np.float64)
    if d_out > 3:
        W[3] = 0.0
    act = synth.act_stat_lognormal(d_in, seed=seed).astype(np.float64)
    enc = oracle.encode(W, bits, block, cb, mask_seed=seed, act_stat=act, alpha=0.5)
    m = qamw.EncodedMatrix(d_out, d_in, block, bits, seed,
                           torch.from_numpy(enc["packed"]).to(DEV).reshape(d_out, -1),
                           to_half_tensor(enc["rnorm_half"], DEV),
                           to_half_tensor(enc["sigma_half"], DEV),
                           to_half_tensor(enc["s_half"], DEV), cbt)
    return m, oracle.decode(enc, cb)


@pytest.mark.parametrize("bits", [11, 7])
def test_decode_many_matches_oracle_and_single_calls(bits):
    cb = codebook(bits)
    cbt = torch.from_numpy(cb).to(DEV)
    shapes = [(300, 1024, 128), (24, 11008, 128), (0, 4096, 128), (97, 4096, 1024),
              (64, 192, 64), (17, 128, 1), (33, 2048, 256), (9, 5120, 128)]
    mats, refs = [], []
    for i, (d_out, d_in, block) in enumerate(shapes):
        m, ref = oracle_matrix(d_out, d_in, block, bits, 11 + i, cbt, cb)
        mats.append(m)
        refs.append(ref)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    outs = qamw.qamw_decode_many(mats, status=st)
    singles = [qamw.qamw_decode(m) for m in mats]
    torch.cuda.synchronize()
    assert st.item() == 0
    for (d_out, d_in, block), o, s, ref in zip(shapes, outs, singles, refs):
        assert torch.equal(o.view(torch.int16), s.view(torch.int16)), (d_out, d_in, block)
        if d_out:
            got = bf16_to_f64(o)
            if d_out > 3:
                assert np.all(got[3] == 0.0)
            check_close(got, ref, what=f"decode_many {d_out}x{d_in} b{block}")


def test_decode_many_more_matrices_than_one_launch():
    bits = 11
    cb = codebook(bits)
    cbt = torch.from_numpy(cb).to(DEV)
    mats, refs = [], []
    for i in range(70):
        d_out, d_in = 3 + (i % 5), 128 * (1 + i % 3)
        m, ref = oracle_matrix(d_out, d_in, 64 if i % 2 else 128, bits, 200 + i, cbt, cb)
        mats.append(m)
        refs.append(ref)
    outs = qamw.qamw_decode_many(mats)
    torch.cuda.synchronize()
    for o, ref in zip(outs, refs):
        check_close(bf16_to_f64(o), ref, what="decode_many x70")


def test_decode_many_rejects_bad_arguments_before_enqueueing():
    bits = 11
    cbt = torch.from_numpy(codebook(bits)).to(DEV)
    good = qamw.EncodedMatrix.empty(8, 256, 64, bits, cbt)
    bad = qamw.EncodedMatrix.empty(8, 256, 64, bits, cbt)
    bad.d_in = 100  # not a multiple of 64
    out = torch.zeros((8, 256), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(qamw.QamwError) as e:
        qamw.qamw_decode_many([good, bad], [out, out])
    assert e.value.rc == qamw.QAMW_ERR_SHAPE
    torch.cuda.synchronize()
    assert not out.any()  # nothing ran
