"""The allocation-free decode-GEMV entry point against the regular one.

qamw_decode_gemv_noalloc serves callers that cannot allocate device memory
(plugin interfaces that pass only input/output pointers, engines that have
reserved all free memory for their own pools, loops that must not synchronise
the device through cudaMalloc/cudaFree): its scratch is a fixed array inside
the library instead of a caller workspace.  This test calls it through the C
ABI twice in a row -- the second call with a smaller batch, so stale scratch
from the first call would show up -- and compares each result with
qamw_decode_gemv on the same inputs and with the fp64 oracle's product, within
the tolerance of the other parity tests.  Problems that fill the scratch
exactly (batch 9-16 with d_in 16384, batch 5-8 with d_in 32768) are checked the
same way, the smallest problem past the limit is refused, and the Python wrapper is called
too.  The file name makes pytest collect it last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
from tests.parity import bf16_to_f64, check_close, halves
from vector_quantization_codec_b200 import qamw, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _encoded_matrix(d_out, d_in, block, bits):
    K = 1 << bits
    s = synth.circular_gaussian_samples(32 * K, seed=5).astype(np.float64)
    cb = torch.from_numpy(oracle.lloyd(s, K, 4)[0].astype(np.float32)).to(DEV)
    m = qamw.EncodedMatrix.empty(d_out, d_in, block, bits, cb, 1, qamw.qamw_build_prefilter(cb, bits))
    W = torch.from_numpy(synth.student_t_weights(d_out, d_in, seed=3)).to(torch.bfloat16).to(DEV)
    act = torch.from_numpy(synth.act_stat_lognormal(d_in, seed=3)).to(DEV)
    qamw.qamw_encode(W, m, act, 0.5)
    return m


def _oracle_product(m, x):
    """The fp64 oracle's x W_hat^T for the GPU-encoded matrix m."""
    cb = m.codebook.cpu().numpy().astype(np.float64)
    enc = dict(packed=m.packed.cpu().numpy(), rnorm_half=halves(m.row_norm),
               sigma_half=halves(m.sigma), s_half=halves(m.chan_scale), d_out=m.d_out,
               d_in=m.d_in, block=m.block, bits=m.bits, mask_seed=m.mask_seed)
    return oracle.gemv(oracle.decode(enc, cb), x.double().cpu().numpy())


def _noalloc_call(m, x, y, status):
    st = m.struct()
    rc = qamw.lib().qamw_decode_gemv_noalloc(C.byref(st), C.c_void_p(x.data_ptr()), x.shape[0],
                                             C.c_void_p(y.data_ptr()),
                                             C.c_void_p(status.data_ptr()),
                                             C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == qamw.QAMW_OK, qamw.status_string(rc)


def test_noalloc_gemv_matches_regular_entry_point_twice():
    d_out, d_in, block, bits = 1000, 4096, 128, 11
    m = _encoded_matrix(d_out, d_in, block, bits)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    for call, batch in enumerate((16, 3)):
        x = torch.from_numpy(synth.gemv_x(batch, d_in, seed=10 + call)).to(torch.bfloat16).to(DEV)
        y_new = torch.full((batch, d_out), float("nan"), dtype=torch.bfloat16, device=DEV)
        _noalloc_call(m, x, y_new, status)
        y_ref = qamw.qamw_decode_gemv(m, x)
        torch.cuda.synchronize()
        assert status.item() == 0
        got, ref = bf16_to_f64(y_new), bf16_to_f64(y_ref)
        want = _oracle_product(m, x)
        for t in range(batch):
            check_close(got[t], ref[t], what=f"noalloc call {call} col {t}")
            check_close(got[t], want[t], what=f"noalloc call {call} col {t} vs oracle")


@pytest.mark.parametrize("batch,d_in", [(13, 16384), (7, 32768)])
def test_noalloc_gemv_at_the_scratch_limit(batch, d_in):
    # padded batch x d_in / 2 = 131072 pairs: the whole scratch array
    m = _encoded_matrix(24, d_in, 128, 9)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    x = torch.from_numpy(synth.gemv_x(batch, d_in, seed=batch)).to(torch.bfloat16).to(DEV)
    y_new = torch.full((batch, m.d_out), float("nan"), dtype=torch.bfloat16, device=DEV)
    qamw.qamw_decode_gemv_noalloc(m, x, y_new, status=status)  # through the Python wrapper
    y_ref = qamw.qamw_decode_gemv(m, x)
    torch.cuda.synchronize()
    assert status.item() == 0
    got, ref, want = bf16_to_f64(y_new), bf16_to_f64(y_ref), _oracle_product(m, x)
    for t in range(batch):
        check_close(got[t], ref[t], what=f"noalloc limit col {t}")
        check_close(got[t], want[t], what=f"noalloc limit col {t} vs oracle")
    # the wrapper refuses a wrong output buffer before calling the library
    with pytest.raises(ValueError):
        qamw.qamw_decode_gemv_noalloc(m, x, y_new[:, :-1])


def test_noalloc_gemv_rejects_sizes_beyond_its_scratch():
    m = _encoded_matrix(8, 32768, 128, 4)
    x = torch.zeros((16, 32768), dtype=torch.bfloat16, device=DEV)
    y = torch.zeros((16, 8), dtype=torch.bfloat16, device=DEV)
    st = m.struct()
    rc = qamw.lib().qamw_decode_gemv_noalloc(C.byref(st), C.c_void_p(x.data_ptr()), 16,
                                             C.c_void_p(y.data_ptr()), None, None)
    assert rc == qamw.QAMW_ERR_SHAPE
    # the smallest problem past the limit: batch 9-16 with d_in 16384 + 64 (16 x 8224 pairs)
    m2 = _encoded_matrix(8, 16384 + 64, 64, 4)
    x2 = torch.zeros((9, 16384 + 64), dtype=torch.bfloat16, device=DEV)
    st2 = m2.struct()
    rc = qamw.lib().qamw_decode_gemv_noalloc(C.byref(st2), C.c_void_p(x2.data_ptr()), 9,
                                             C.c_void_p(y.data_ptr()), None, None)
    assert rc == qamw.QAMW_ERR_SHAPE
    # batch 1 with the same d_in fits (16384 pairs)
    _noalloc_call(m, x[:1], y[:1], torch.zeros(1, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
