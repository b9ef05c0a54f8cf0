"""Host-side checks of libqamw.so: it loads without a GPU, exports every entry
point include/qamw.h declares, its size helpers follow the paper, and argument
errors are rejected on the host before anything reaches the GPU.

The error-path calls pass made-up device addresses: each is rejected by the
argument checks, which run before any CUDA call (no GPU is touched here).
"""
import ctypes as C
import os
import re

import pytest

import oracle
from vector_quantization_codec_b200 import qamw

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "qamw.h")).read()
    return sorted(set(re.findall(r"QAMW_API[^;(]*?\b(qamw_\w+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_symbols() == sorted(qamw.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = C.CDLL(qamw.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_header_compiles_as_plain_c(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "qamw.h"\nint main(void){ return (int)qamw_row_bytes(64, 1) - 16; }\n')
    exe = tmp_path / "t"
    import subprocess
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           str(src), qamw.LIB_PATH, "-o", str(exe),
                           f"-Wl,-rpath,{os.path.dirname(qamw.LIB_PATH)}"])
    assert subprocess.run([str(exe)]).returncode == 0


@pytest.mark.parametrize("d_in", [64, 128, 512, 2048, 4096, 5120, 5632, 11008, 13824])
@pytest.mark.parametrize("bits", list(range(1, 12)))
def test_row_bytes_and_bitrate_match_oracle(d_in, bits):
    assert qamw.qamw_row_bytes(d_in, bits) == oracle.row_bytes(d_in, bits)
    assert qamw.qamw_bits_per_weight(d_in, bits) == oracle.bits_per_weight(d_in, bits)


def test_default_block_rule(golden):
    for d_in, block in golden("block_rule.txt"):
        assert qamw.qamw_default_block(int(d_in)) == int(block)
    for d_in in [1, 64, 96, 4096, 11008, 13824, 3 * 2048]:
        assert qamw.qamw_default_block(d_in) == oracle.default_block(d_in)
    assert qamw.qamw_default_block(0) == 0


def test_workspace_sizes():
    assert qamw.qamw_workspace_bytes(qamw.QAMW_OP_TRAIN, 0, 0, 11) >= 3 * 2048 * 8
    enc = qamw.qamw_workspace_bytes(qamw.QAMW_OP_ENCODE, 4096, 4096, 11)
    assert enc >= 4096 * 4 + qamw.qamw_prefilter_bytes(11)
    assert qamw.qamw_workspace_bytes(qamw.QAMW_OP_GEMV, 4096, 4096, 11, 16) >= 16 * 2048 * 8
    assert qamw.qamw_workspace_bytes(qamw.QAMW_OP_GEMV, 4096, 4096, 11, 17) == 0
    assert qamw.qamw_workspace_bytes(qamw.QAMW_OP_ENCODE, 4096, 100, 11) == 0
    assert qamw.qamw_workspace_bytes(7, 4096, 4096, 11) == 0
    assert qamw.qamw_workspace_bytes(qamw.QAMW_OP_TRAIN, 0, 0, 12) == 0


FAKE = 0x7F0000000000  # a 16-byte aligned address that is never dereferenced


def _matrix(d_out=8, d_in=128, block=64, bits=4, **kw):
    m = qamw.qamw_matrix(d_out, d_in, block, bits, 0, oracle.row_bytes(d_in, bits),
                         FAKE, FAKE, FAKE, FAKE, FAKE, None)
    for k, v in kw.items():
        setattr(m, k, v)
    return m


def _encode(m, W=FAKE, dtype=qamw.QAMW_DTYPE_BF16, flags=0, ws=FAKE, ws_bytes=1 << 40, alpha=0.5):
    return qamw.lib().qamw_encode(C.c_void_p(W), dtype, None, alpha, flags, C.byref(m),
                                  C.c_void_p(ws), ws_bytes, None, None)


@pytest.mark.parametrize("kw,rc", [
    (dict(bits=0), qamw.QAMW_ERR_INVALID),
    (dict(bits=12), qamw.QAMW_ERR_INVALID),
    (dict(d_in=100), qamw.QAMW_ERR_SHAPE),
    (dict(d_in=0), qamw.QAMW_ERR_SHAPE),
    (dict(d_in=32768 + 64), qamw.QAMW_ERR_SHAPE),
    (dict(d_out=-1), qamw.QAMW_ERR_SHAPE),
    (dict(block=48), qamw.QAMW_ERR_SHAPE),
    (dict(block=2048, d_in=4096), qamw.QAMW_ERR_SHAPE),
    (dict(block=256), qamw.QAMW_ERR_SHAPE),  # 256 does not divide 128
    (dict(row_bytes=17), qamw.QAMW_ERR_INVALID),
    (dict(packed=None), qamw.QAMW_ERR_INVALID),
    (dict(codebook=None), qamw.QAMW_ERR_INVALID),
    (dict(packed=FAKE + 8), qamw.QAMW_ERR_ALIGN),
    (dict(codebook=FAKE + 4), qamw.QAMW_ERR_ALIGN),
    (dict(sigma=FAKE + 2), qamw.QAMW_ERR_ALIGN),
    (dict(chan_scale=FAKE + 8), qamw.QAMW_ERR_ALIGN),
])
def test_matrix_argument_errors(kw, rc):
    m = _matrix(**kw)
    assert _encode(m) == rc
    assert qamw.lib().qamw_decode_gemv_noalloc(C.byref(m), C.c_void_p(FAKE), 1, C.c_void_p(FAKE),
                                               None, None) == rc
    assert qamw.lib().qamw_decode(C.byref(m), C.c_void_p(FAKE), None, None) == rc
    assert qamw.lib().qamw_decode_gemv(C.byref(m), C.c_void_p(FAKE), 1, C.c_void_p(FAKE),
                                       C.c_void_p(FAKE), 1 << 40, None, None) == rc
    assert qamw.lib().qamw_decode_gemm(C.byref(m), C.c_void_p(FAKE), 64, C.c_void_p(FAKE),
                                       C.c_void_p(FAKE), 1 << 40, None, None) == rc
    one = (qamw.qamw_matrix * 1)(m)
    assert qamw.lib().qamw_decode_gemv_many(one, 1, (C.c_void_p * 1)(FAKE), (C.c_void_p * 1)(FAKE),
                                            C.c_void_p(FAKE), 1 << 40, None, None) == rc


def test_encode_argument_errors():
    m = _matrix()
    assert _encode(m, dtype=5) == qamw.QAMW_ERR_INVALID
    assert _encode(m, flags=0x10) == qamw.QAMW_ERR_INVALID
    assert _encode(m, W=0) == qamw.QAMW_ERR_INVALID
    assert _encode(m, W=FAKE + 2) == qamw.QAMW_ERR_ALIGN
    assert _encode(m, ws=0) == qamw.QAMW_ERR_WORKSPACE
    assert _encode(m, ws_bytes=64) == qamw.QAMW_ERR_WORKSPACE
    assert _encode(m, alpha=float("nan")) == qamw.QAMW_ERR_INVALID
    # an empty matrix is a no-op that needs no buffers
    assert _encode(_matrix(d_out=0, packed=None, codebook=None), W=0, ws=0, ws_bytes=0) == qamw.QAMW_OK


def test_gemv_and_train_argument_errors():
    m = _matrix()
    L = qamw.lib()
    for batch in (0, 17):
        assert L.qamw_decode_gemv(C.byref(m), C.c_void_p(FAKE), batch, C.c_void_p(FAKE),
                                  C.c_void_p(FAKE), 1 << 40, None, None) == qamw.QAMW_ERR_INVALID
    assert L.qamw_decode_gemv(C.byref(m), C.c_void_p(FAKE), 4, C.c_void_p(FAKE),
                              C.c_void_p(FAKE), 100, None, None) == qamw.QAMW_ERR_WORKSPACE
    assert L.qamw_decode_gemv(C.byref(m), C.c_void_p(FAKE + 2), 4, C.c_void_p(FAKE),
                              C.c_void_p(FAKE), 1 << 40, None, None) == qamw.QAMW_ERR_ALIGN
    T = L.qamw_train_codebook
    assert T(C.c_void_p(FAKE), 1 << 20, 12, 5, C.c_void_p(FAKE), None, C.c_void_p(FAKE), 1 << 30,
             None, None) == qamw.QAMW_ERR_INVALID
    assert T(C.c_void_p(FAKE), 100, 8, 5, C.c_void_p(FAKE), None, C.c_void_p(FAKE), 1 << 30,
             None, None) == qamw.QAMW_ERR_SHAPE
    assert T(C.c_void_p(FAKE), 1 << 20, 8, -1, C.c_void_p(FAKE), None, C.c_void_p(FAKE), 1 << 30,
             None, None) == qamw.QAMW_ERR_INVALID
    assert T(C.c_void_p(FAKE), 1 << 20, 8, 5, C.c_void_p(FAKE), None, C.c_void_p(FAKE), 10,
             None, None) == qamw.QAMW_ERR_WORKSPACE
    assert L.qamw_build_prefilter(C.c_void_p(FAKE), 11, C.c_void_p(FAKE), 10, None) == \
        qamw.QAMW_ERR_WORKSPACE
    # the bounded-wait check takes 1 .. 2^18 polls and a status word
    S = L.qamw_selftest_wait_timeout
    assert S(0, C.c_void_p(FAKE), None, None) == qamw.QAMW_ERR_INVALID
    assert S((1 << 18) + 1, C.c_void_p(FAKE), None, None) == qamw.QAMW_ERR_INVALID
    assert S(16, None, None, None) == qamw.QAMW_ERR_INVALID
    # the row range of the point export must lie inside the matrix
    P = L.qamw_normalised_pairs
    assert P(C.c_void_p(FAKE), qamw.QAMW_DTYPE_BF16, C.byref(m), 90, 20, C.c_void_p(FAKE), None,
             None) == qamw.QAMW_ERR_SHAPE


def _gemm_plan_bytes(d_out, d_in, ntok, sms=148):
    """Workspace of qamw_decode_gemm re-derived from its stated plan: 64-column
    chunks, token groups of 64 (<= 64 tokens) or 128, 128-row tiles, the units
    shared equally over min(SMs, units / 4) CTAs, x_bar images (2 parts x 8 KB
    per chunk and 64 tokens) and one fp32 partial sum per (CTA share of a row
    tile and token group)."""
    C = d_in // 64
    NT = 128 if ntok > 64 else 64
    TG = (ntok + NT - 1) // NT
    ntt = TG * NT // 64
    U = ((d_out + 127) // 128) * TG * C
    G = min(sms, max(1, U // 4))
    per = max(1, U // G)
    segmax = min(G, (C - 1 + per - 1) // per + 1)
    return C * 2 * ntt * 8192 + segmax * ntt * 64 * d_out * 4


@pytest.mark.parametrize("d_out,d_in,ntok", [(11008, 4096, 128), (4096, 4096, 64), (4096, 11008, 3),
                                             (300, 1024, 100), (24, 11008, 256), (64, 192, 70)])
def test_gemm_workspace_follows_the_plan(d_out, d_in, ntok):
    # without a device the library plans for 148 SMs
    assert qamw.qamw_workspace_bytes(qamw.QAMW_OP_GEMM, d_out, d_in, 11, ntok) == \
        _gemm_plan_bytes(d_out, d_in, ntok)


def test_gemv_many_workspace_sizes():
    ms = [_matrix(d_in=4096), _matrix(d_in=11008), _matrix(d_out=0, d_in=4096), _matrix(d_in=192)]
    arr = (qamw.qamw_matrix * 4)(*ms)
    # x_bar of every non-empty matrix, fp32, each rounded up to 256 bytes
    assert qamw.lib().qamw_decode_gemv_many_workspace_bytes(arr, 4) == 4096 * 4 + 11008 * 4 + 768
    assert qamw.lib().qamw_decode_gemv_many_workspace_bytes(arr, 0) == 0


def test_gemm_and_gemv_many_argument_errors():
    L = qamw.lib()
    m = _matrix()
    G = L.qamw_decode_gemm
    for ntok in (0, 65537):
        assert G(C.byref(m), C.c_void_p(FAKE), ntok, C.c_void_p(FAKE), C.c_void_p(FAKE), 1 << 40,
                 None, None) == qamw.QAMW_ERR_INVALID
    assert G(C.byref(m), None, 64, C.c_void_p(FAKE), C.c_void_p(FAKE), 1 << 40, None, None) == \
        qamw.QAMW_ERR_INVALID
    assert G(C.byref(m), C.c_void_p(FAKE + 2), 64, C.c_void_p(FAKE), C.c_void_p(FAKE), 1 << 40,
             None, None) == qamw.QAMW_ERR_ALIGN
    assert G(C.byref(m), C.c_void_p(FAKE), 64, C.c_void_p(FAKE), C.c_void_p(FAKE), 100, None,
             None) == qamw.QAMW_ERR_WORKSPACE
    assert G(C.byref(m), C.c_void_p(FAKE), 64, C.c_void_p(FAKE), C.c_void_p(FAKE + 8), 1 << 40,
             None, None) == qamw.QAMW_ERR_ALIGN
    empty = _matrix(d_out=0)
    assert G(C.byref(empty), None, 64, None, None, 0, None, None) == qamw.QAMW_OK
    M = L.qamw_decode_gemv_many
    arr = (qamw.qamw_matrix * 2)(_matrix(), _matrix(d_in=256))
    xs = (C.c_void_p * 2)(FAKE, FAKE)
    ys = (C.c_void_p * 2)(FAKE, FAKE)
    assert M(arr, -1, xs, ys, C.c_void_p(FAKE), 1 << 40, None, None) == qamw.QAMW_ERR_INVALID
    assert M(arr, 2, None, ys, C.c_void_p(FAKE), 1 << 40, None, None) == qamw.QAMW_ERR_INVALID
    assert M(arr, 2, (C.c_void_p * 2)(FAKE, None), ys, C.c_void_p(FAKE), 1 << 40, None, None) == \
        qamw.QAMW_ERR_INVALID
    assert M(arr, 2, (C.c_void_p * 2)(FAKE, FAKE + 2), ys, C.c_void_p(FAKE), 1 << 40, None, None) == \
        qamw.QAMW_ERR_ALIGN
    assert M(arr, 2, xs, ys, C.c_void_p(FAKE), 100, None, None) == qamw.QAMW_ERR_WORKSPACE
    assert M(arr, 2, xs, ys, None, 1 << 40, None, None) == qamw.QAMW_ERR_WORKSPACE
    assert M(arr, 0, None, None, None, 0, None, None) == qamw.QAMW_OK
    # a bad matrix anywhere in the list is reported before anything is enqueued
    bad = (qamw.qamw_matrix * 2)(_matrix(), _matrix(bits=12))
    assert M(bad, 2, xs, ys, C.c_void_p(FAKE), 1 << 40, None, None) == qamw.QAMW_ERR_INVALID


def test_status_strings():
    for rc in (0, -1, -2, -3, -4, -5, 1, 2, 4):
        assert qamw.status_string(rc)
