"""The allocation-free decode-GEMV entry point against the regular one.

qamw_decode_gemv_noalloc serves callers that cannot allocate device memory
(plugin interfaces that pass only input/output pointers, engines that have
reserved all free memory for their own pools, loops that must not synchronise
the device through cudaMalloc/cudaFree): its scratch is a fixed array inside
the library instead of a caller workspace.  This test calls it through the C
ABI twice in a row -- the second call with a smaller batch, so stale scratch
from the first call would show up -- and compares each result with
qamw_decode_gemv on the same inputs, within the tolerance of the other parity
tests.  The file name makes pytest collect it last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
from tests.parity import bf16_to_f64, check_close
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
        for t in range(batch):
            check_close(got[t], ref[t], what=f"noalloc call {call} col {t}")


def test_noalloc_gemv_rejects_sizes_beyond_its_scratch():
    m = _encoded_matrix(8, 32768, 128, 4)
    x = torch.zeros((16, 32768), dtype=torch.bfloat16, device=DEV)
    y = torch.zeros((16, 8), dtype=torch.bfloat16, device=DEV)
    st = m.struct()
    rc = qamw.lib().qamw_decode_gemv_noalloc(C.byref(st), C.c_void_p(x.data_ptr()), 16,
                                             C.c_void_p(y.data_ptr()), None, None)
    assert rc == qamw.QAMW_ERR_SHAPE
    # batch 1 with the same d_in fits (16384 pairs)
    _noalloc_call(m, x[:1], y[:1], torch.zeros(1, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
