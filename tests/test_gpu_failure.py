"""Failure path of the bounded waits, on the GPU without a fault: a wait that
nothing completes must give up, flag QAMW_STATUS_TIMEOUT, and leave the CUDA
context usable (a decode-GEMV before and after gives the same result)."""
import numpy as np
import pytest
import torch

from tests.parity import log_stats
from vector_quantization_codec_b200 import qamw, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_bounded_wait_times_out_and_context_stays_usable():
    d_out, d_in, block, bits = 64, 512, 64, 6
    K = 1 << bits
    cb = torch.from_numpy(synth.circular_gaussian_samples(K, seed=3)).float().to(DEV)
    W = torch.from_numpy(synth.student_t_weights(d_out, d_in, seed=4)).to(torch.bfloat16).to(DEV)
    m = qamw.EncodedMatrix.empty(d_out, d_in, block, bits, cb)
    qamw.qamw_encode(W, m)
    x = torch.from_numpy(synth.gemv_x(1, d_in, seed=5)).to(torch.bfloat16).to(DEV)
    y_before = qamw.qamw_decode_gemv(m, x).clone()

    tries = 4096
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    cycles = torch.zeros(1, dtype=torch.int64, device=DEV)
    qamw.qamw_selftest_wait_timeout(tries, st, cycles)
    torch.cuda.synchronize()
    assert st.item() & qamw.QAMW_STATUS_TIMEOUT
    per_try = cycles.item() / tries
    # the kernels' own limit, 2^18 polls, at the B200's top clock of 1.965 GHz:
    # about a second
    full_s = per_try * (1 << 18) / 1.965e9
    log_stats("bounded wait", dict(cycles_per_try=per_try, full_limit_s=full_s))
    assert 0 < per_try and full_s < 2.5, (per_try, full_s)

    st2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    y_after = qamw.qamw_decode_gemv(m, x, status=st2)
    torch.cuda.synchronize()
    assert st2.item() == 0
    assert torch.equal(y_before, y_after)
