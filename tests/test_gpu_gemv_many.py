"""The batch-1 decode-GEMV of a list of matrices (qamw_decode_gemv_many) against
single qamw_decode_gemv calls -- bit for bit, since the list call forms x_bar
with the same arithmetic and sums the same partial products in the same order
-- and against the fp64 oracle's product within the 1e-2 rule of the other
product tests.

Lists mix runs that share a launch (same d_in, block, bits and codebook) with
matrices that start a new run (another d_in, bits or codebook), empty matrices,
ragged last tiles, more than 64 matrices of one kind (two launches), and the
full 11008 x 4096 / 4096 x 11008 shapes at K = 2048."""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import bf16_to_f64, check_close, halves
from tests.test_gpu_parity import codebook, gpu_encode, weights
from vector_quantization_codec_b200 import qamw, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def encode_list(specs, shared):
    """Matrices for (d_out, d_in, block, bits) specs; `shared` codebook tensors
    per bits (one pointer per bits, so runs can form)."""
    ms = []
    for i, (d_out, d_in, block, bits) in enumerate(specs):
        cbt = shared.setdefault(bits, torch.from_numpy(codebook(bits)).to(DEV))
        m = qamw.EncodedMatrix.empty(d_out, d_in, block, bits, cbt, 3 + i,
                                     qamw.qamw_build_prefilter(cbt, bits))
        if d_out > 0:
            Wt, _ = weights(d_out, d_in, 5 + i, "bf16")
            act = synth.act_stat_lognormal(d_in, seed=i)
            m, st = gpu_encode(Wt, d_in, block, bits, codebook(bits), act, 0.5, m=m)
            assert st == 0
        ms.append(m)
    return ms


def xs_for(ms, seed):
    return [torch.from_numpy(synth.gemv_x(1, m.d_in, seed=seed + i)).to(torch.bfloat16).to(DEV)
            for i, m in enumerate(ms)]


def singles(ms, xs):
    return [qamw.qamw_decode_gemv(m, x) if m.d_out > 0 else
            torch.empty((1, 0), dtype=torch.bfloat16, device=DEV) for m, x in zip(ms, xs)]


def oracle_product(m, x):
    cb = m.codebook.cpu().numpy().astype(np.float64)
    enc = dict(packed=m.packed.cpu().numpy(), rnorm_half=halves(m.row_norm), sigma_half=halves(m.sigma),
               s_half=halves(m.chan_scale), d_out=m.d_out, d_in=m.d_in, block=m.block, bits=m.bits,
               mask_seed=m.mask_seed)
    return oracle.gemv(oracle.decode(enc, cb), x.double().cpu().numpy())


MIXED = [(300, 1024, 128, 11), (24, 1024, 128, 11), (0, 1024, 128, 11), (97, 1024, 128, 11),
         (130, 4096, 1024, 11), (64, 4096, 1024, 11), (40, 192, 64, 3), (33, 192, 64, 3),
         (129, 1024, 128, 9), (17, 1024, 64, 11)]


def test_gemv_many_equals_single_calls_bitwise():
    ms = encode_list(MIXED, {})
    xs = xs_for(ms, 40)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    got = qamw.qamw_decode_gemv_many(ms, xs, status=st)
    want = singles(ms, xs)
    torch.cuda.synchronize()
    assert st.item() == 0, qamw.status_string(st.item())
    for i, (g, w) in enumerate(zip(got, want)):
        assert torch.equal(g, w), f"matrix {i} {MIXED[i]}"


def test_gemv_many_matches_oracle():
    specs = [(300, 1024, 128, 11), (130, 4096, 1024, 11), (40, 192, 64, 3)]
    ms = encode_list(specs, {})
    xs = xs_for(ms, 7)
    ys = qamw.qamw_decode_gemv_many(ms, xs)
    torch.cuda.synchronize()
    for i, (m, x, y) in enumerate(zip(ms, xs, ys)):
        check_close(bf16_to_f64(y)[0], oracle_product(m, x.view(1, -1))[0], what=f"gemv many {i}")


def test_gemv_many_more_than_one_launch_per_run():
    # 70 matrices of one kind: a run of 64 and a run of 6, plus a codebook
    # change in the middle (another tensor with the same values)
    shared = {}
    specs = [(40 + (i % 5), 256, 64, 7) for i in range(70)]
    ms = encode_list(specs, shared)
    other = torch.from_numpy(codebook(7)).to(DEV)
    ms[35] = qamw.EncodedMatrix(ms[35].d_out, ms[35].d_in, ms[35].block, ms[35].bits,
                                ms[35].mask_seed, ms[35].packed, ms[35].row_norm, ms[35].sigma,
                                ms[35].chan_scale, other)
    xs = xs_for(ms, 100)
    got = qamw.qamw_decode_gemv_many(ms, xs)
    want = singles(ms, xs)
    torch.cuda.synchronize()
    for i, (g, w) in enumerate(zip(got, want)):
        assert torch.equal(g, w), f"matrix {i}"


def test_gemv_many_full_size_shapes():
    d_in_a, bits = 4096, 11
    cbt = torch.from_numpy(codebook(bits)).to(DEV)
    ms = []
    for i, (d_out, d_in) in enumerate([(11008, 4096), (4096, 4096), (4096, 11008), (11008, 4096)]):
        Wt = torch.from_numpy(synth.student_t_weights(d_out, d_in, seed=60 + i)).to(torch.bfloat16)
        m = qamw.EncodedMatrix.empty(d_out, d_in, 128, bits, cbt, i, qamw.qamw_build_prefilter(cbt, bits))
        m, st = gpu_encode(Wt.to(DEV), d_in, 128, bits, codebook(bits),
                           synth.act_stat_lognormal(d_in, seed=i), 0.5, m=m)
        assert st == 0
        ms.append(m)
    assert ms[0].d_in == d_in_a
    xs = xs_for(ms, 9)
    got = qamw.qamw_decode_gemv_many(ms, xs)
    want = singles(ms, xs)
    torch.cuda.synchronize()
    for i, (g, w) in enumerate(zip(got, want)):
        assert torch.equal(g, w), f"matrix {i}"


def test_gemv_many_arguments():
    ms = encode_list([(16, 256, 64, 7), (8, 256, 64, 7)], {})
    xs = xs_for(ms, 1)
    need = qamw.qamw_decode_gemv_many_workspace_bytes(ms)
    assert need >= 2 * 256 * 4
    with pytest.raises(qamw.QamwError) as e:
        qamw.qamw_decode_gemv_many(ms, xs, workspace=torch.empty(need - 16, dtype=torch.uint8,
                                                                  device=DEV))
    assert e.value.rc == qamw.QAMW_ERR_WORKSPACE
    with pytest.raises(qamw.QamwError) as e:  # an unaligned activation
        qamw.qamw_decode_gemv_many(ms, [xs[0], torch.zeros(264, dtype=torch.bfloat16,
                                                           device=DEV)[4:]])
    assert e.value.rc == qamw.QAMW_ERR_ALIGN
    assert qamw.qamw_decode_gemv_many([], []) == []
