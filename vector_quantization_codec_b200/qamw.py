"""Python binding of libqamw.so (QAM-W codec on B200).

Argument marshalling only: every function here passes device pointers taken
from torch tensors (and the current CUDA stream) to the C ABI declared in
include/qamw.h, and raises QamwError on a non-zero return code.  The codec's
arithmetic runs entirely in the library's CUDA kernels; there is no CPU or
PyTorch fallback, and importing this module fails if the library is missing.

Names follow the C ABI: qamw_train_codebook, qamw_build_prefilter,
qamw_encode (= qamw_channel_scales + qamw_calibrate_sigma + qamw_encode_rows),
qamw_decode, qamw_decode_gemv and the size helpers.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libqamw.so")

QAMW_OK = 0
QAMW_ERR_INVALID = -1
QAMW_ERR_SHAPE = -2
QAMW_ERR_ALIGN = -3
QAMW_ERR_WORKSPACE = -4
QAMW_ERR_CUDA = -5
QAMW_STATUS_NONFINITE = 0x1
QAMW_STATUS_RANGE = 0x2
QAMW_STATUS_BAD_STAT = 0x4
QAMW_STATUS_TIMEOUT = 0x8
QAMW_DTYPE_F32 = 0
QAMW_DTYPE_BF16 = 1
QAMW_SIGMA_GIVEN = 0x1
QAMW_SCALES_GIVEN = 0x2
QAMW_POLAR = 0x4
QAMW_SCALAR = 0x8
QAMW_OP_TRAIN = 0
QAMW_OP_ENCODE = 1
QAMW_OP_GEMV = 2
QAMW_OP_CALIBRATE = 3
QAMW_OP_GEMM = 4

# Every symbol include/qamw.h declares (checked by the test suite).
EXPORTS = ("qamw_row_bytes", "qamw_default_block", "qamw_bits_per_weight",
           "qamw_workspace_bytes", "qamw_prefilter_bytes", "qamw_status_string",
           "qamw_train_codebook", "qamw_build_prefilter", "qamw_encode", "qamw_channel_scales",
           "qamw_calibrate_sigma", "qamw_calibrate_many", "qamw_calibrate_many_workspace_bytes",
           "qamw_encode_rows", "qamw_decode", "qamw_decode_many",
           "qamw_decode_gemv", "qamw_decode_gemv_many", "qamw_decode_gemv_many_workspace_bytes",
           "qamw_decode_gemm",
           "qamw_decode_gemv_noalloc", "qamw_polar_codebook", "qamw_encode_rows_polar",
           "qamw_scalar_codebook", "qamw_encode_rows_scalar",
           "qamw_normalised_pairs", "qamw_selftest_wait_timeout")


class QamwError(RuntimeError):
    def __init__(self, fn: str, rc: int):
        super().__init__(f"{fn} returned {rc}: {status_string(rc)}")
        self.rc = rc


class qamw_matrix(C.Structure):
    _fields_ = [("d_out", C.c_int32), ("d_in", C.c_int32), ("block", C.c_int32),
                ("bits", C.c_int32), ("mask_seed", C.c_uint64), ("row_bytes", C.c_int64),
                ("packed", C.c_void_p), ("row_norm", C.c_void_p), ("sigma", C.c_void_p),
                ("chan_scale", C.c_void_p), ("codebook", C.c_void_p), ("prefilter", C.c_void_p)]


def _load() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m vector_quantization_codec_b200.build` (no fallback exists)")
    lib = C.CDLL(LIB_PATH)
    V, I, I64, SZ, D = C.c_void_p, C.c_int, C.c_int64, C.c_size_t, C.c_double
    sig = {
        "qamw_row_bytes": (I64, [I, I]),
        "qamw_default_block": (I, [I]),
        "qamw_bits_per_weight": (D, [I, I]),
        "qamw_workspace_bytes": (SZ, [I, I, I, I, I]),
        "qamw_prefilter_bytes": (SZ, [I]),
        "qamw_status_string": (C.c_char_p, [I]),
        "qamw_train_codebook": (I, [V, I64, I, I, V, V, V, SZ, V, V]),
        "qamw_build_prefilter": (I, [V, I, V, SZ, V]),
        "qamw_encode": (I, [V, I, V, C.c_float, I, C.POINTER(qamw_matrix), V, SZ, V, V]),
        "qamw_channel_scales": (I, [V, I, C.c_float, V, V, V]),
        "qamw_calibrate_sigma": (I, [V, I, C.POINTER(qamw_matrix), V, SZ, V, V]),
        "qamw_calibrate_many": (I, [C.POINTER(C.c_void_p), I, C.POINTER(C.c_void_p), C.c_float,
                                    C.POINTER(qamw_matrix), I, V, SZ, V, V]),
        "qamw_calibrate_many_workspace_bytes": (SZ, [C.POINTER(qamw_matrix), I]),
        "qamw_encode_rows": (I, [V, I, C.POINTER(qamw_matrix), V, V, V]),
        "qamw_decode": (I, [C.POINTER(qamw_matrix), V, V, V]),
        "qamw_decode_many": (I, [C.POINTER(qamw_matrix), I, C.POINTER(C.c_void_p), V, V]),
        "qamw_decode_gemv": (I, [C.POINTER(qamw_matrix), V, I, V, V, SZ, V, V]),
        "qamw_decode_gemv_many": (I, [C.POINTER(qamw_matrix), I, C.POINTER(C.c_void_p),
                                      C.POINTER(C.c_void_p), V, SZ, V, V]),
        "qamw_decode_gemv_many_workspace_bytes": (SZ, [C.POINTER(qamw_matrix), I]),
        "qamw_decode_gemm": (I, [C.POINTER(qamw_matrix), V, I, V, V, SZ, V, V]),
        "qamw_decode_gemv_noalloc": (I, [C.POINTER(qamw_matrix), V, I, V, V, V]),
        "qamw_polar_codebook": (I, [I, V, V]),
        "qamw_encode_rows_polar": (I, [V, I, C.POINTER(qamw_matrix), V, V]),
        "qamw_scalar_codebook": (I, [I, V, V]),
        "qamw_encode_rows_scalar": (I, [V, I, C.POINTER(qamw_matrix), V, V]),
        "qamw_normalised_pairs": (I, [V, I, C.POINTER(qamw_matrix), I64, I64, V, V, V]),
        "qamw_selftest_wait_timeout": (I, [C.c_uint, V, V, V]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def lib() -> C.CDLL:
    return _lib


def _p(t: torch.Tensor | None):
    return None if t is None else C.c_void_p(t.data_ptr())


def _s(stream) -> C.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn: str, rc: int) -> None:
    if rc != QAMW_OK:
        raise QamwError(fn, rc)


# ------------------------------------------------------------------ helpers

def qamw_row_bytes(d_in: int, bits: int) -> int:
    return int(_lib.qamw_row_bytes(d_in, bits))


def qamw_default_block(d_in: int) -> int:
    return int(_lib.qamw_default_block(d_in))


def qamw_bits_per_weight(d_in: int, bits: int) -> float:
    return float(_lib.qamw_bits_per_weight(d_in, bits))


def qamw_workspace_bytes(op: int, d_out: int, d_in: int, bits: int, batch: int = 0) -> int:
    return int(_lib.qamw_workspace_bytes(op, d_out, d_in, bits, batch))


def qamw_prefilter_bytes(bits: int) -> int:
    return int(_lib.qamw_prefilter_bytes(bits))


def status_string(code: int) -> str:
    return _lib.qamw_status_string(int(code)).decode()


qamw_status_string = status_string


# ------------------------------------------------------------------ matrix

@dataclass
class EncodedMatrix:
    """Device buffers of one encoded matrix (all torch tensors on one GPU)."""
    d_out: int
    d_in: int
    block: int
    bits: int
    mask_seed: int
    packed: torch.Tensor       # uint8 [d_out, row_bytes]
    row_norm: torch.Tensor     # int16 view of binary16 [d_out]
    sigma: torch.Tensor        # binary16 [d_in/2]
    chan_scale: torch.Tensor   # binary16 [d_in]
    codebook: torch.Tensor     # float32 [K, 2]
    prefilter: torch.Tensor | None = None  # uint8 table

    @staticmethod
    def empty(d_out: int, d_in: int, block: int, bits: int, codebook: torch.Tensor,
              mask_seed: int = 0, prefilter: torch.Tensor | None = None) -> "EncodedMatrix":
        dev = codebook.device
        rb = qamw_row_bytes(d_in, bits)
        return EncodedMatrix(d_out, d_in, block, bits, mask_seed,
                             torch.empty((d_out, rb), dtype=torch.uint8, device=dev),
                             torch.empty(d_out, dtype=torch.float16, device=dev),
                             torch.empty(d_in // 2, dtype=torch.float16, device=dev),
                             torch.empty(d_in, dtype=torch.float16, device=dev),
                             codebook, prefilter)

    @property
    def row_bytes(self) -> int:
        return qamw_row_bytes(self.d_in, self.bits)

    def struct(self) -> qamw_matrix:
        return qamw_matrix(self.d_out, self.d_in, self.block, self.bits, self.mask_seed,
                           self.row_bytes, self.packed.data_ptr(), self.row_norm.data_ptr(),
                           self.sigma.data_ptr(), self.chan_scale.data_ptr(),
                           self.codebook.data_ptr(),
                           None if self.prefilter is None else self.prefilter.data_ptr())


def _dtype_code(W: torch.Tensor) -> int:
    if W.dtype == torch.float32:
        return QAMW_DTYPE_F32
    if W.dtype == torch.bfloat16:
        return QAMW_DTYPE_BF16
    raise TypeError(f"W must be float32 or bfloat16, not {W.dtype}")


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ calls

def qamw_train_codebook(samples: torch.Tensor, bits: int, iters: int, codebook: torch.Tensor,
                        distortion: torch.Tensor | None = None,
                        workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
                        stream=None) -> None:
    """Lloyd iterations (paper section 3.6 eq. 2); samples float32 [n, 2] on the GPU."""
    if workspace is None:
        workspace = _workspace(qamw_workspace_bytes(QAMW_OP_TRAIN, 0, 0, bits), samples.device)
    rc = _lib.qamw_train_codebook(_p(samples), samples.shape[0], bits, iters, _p(codebook),
                                  _p(distortion), _p(workspace), workspace.numel(), _p(status),
                                  _s(stream))
    _check("qamw_train_codebook", rc)


def qamw_build_prefilter(codebook: torch.Tensor, bits: int, table: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    if table is None:
        table = _workspace(qamw_prefilter_bytes(bits), codebook.device)
    rc = _lib.qamw_build_prefilter(_p(codebook), bits, _p(table), table.numel(), _s(stream))
    _check("qamw_build_prefilter", rc)
    return table


def qamw_encode(W: torch.Tensor, m: EncodedMatrix, act_stat: torch.Tensor | None = None,
                alpha: float = 0.0, flags: int = 0, workspace: torch.Tensor | None = None,
                status: torch.Tensor | None = None, stream=None) -> EncodedMatrix:
    """Encoder of paper section 3.1 with activation-aware channel scaling; fills m."""
    if workspace is None:
        workspace = _workspace(qamw_workspace_bytes(QAMW_OP_ENCODE, m.d_out, m.d_in, m.bits),
                               W.device)
    st = m.struct()
    rc = _lib.qamw_encode(_p(W), _dtype_code(W), _p(act_stat), float(alpha), int(flags),
                          C.byref(st), _p(workspace), workspace.numel(), _p(status), _s(stream))
    _check("qamw_encode", rc)
    return m


def qamw_channel_scales(d_in: int, act_stat: torch.Tensor | None, alpha: float,
                        scale: torch.Tensor, status: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    rc = _lib.qamw_channel_scales(_p(act_stat), d_in, float(alpha), _p(scale), _p(status),
                                  _s(stream))
    _check("qamw_channel_scales", rc)
    return scale


def qamw_calibrate_sigma(W: torch.Tensor, m: EncodedMatrix, workspace: torch.Tensor | None = None,
                         status: torch.Tensor | None = None, stream=None) -> EncodedMatrix:
    if workspace is None:
        workspace = _workspace(qamw_workspace_bytes(QAMW_OP_CALIBRATE, m.d_out, m.d_in, m.bits),
                               W.device)
    st = m.struct()
    rc = _lib.qamw_calibrate_sigma(_p(W), _dtype_code(W), C.byref(st), _p(workspace),
                                   workspace.numel(), _p(status), _s(stream))
    _check("qamw_calibrate_sigma", rc)
    return m


def _matrix_array(ms: list):
    return (qamw_matrix * max(len(ms), 1))(*[m.struct() for m in ms])


def qamw_calibrate_many_workspace_bytes(ms: list) -> int:
    return int(_lib.qamw_calibrate_many_workspace_bytes(_matrix_array(ms), len(ms)))


def qamw_calibrate_many(Ws: list, ms: list, act_stats: list | None = None, alpha: float = 0.0,
                        workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
                        stream=None) -> list:
    """Channel scales and eq. (1) of every matrix of `ms` (weights `Ws`) in one call."""
    n = len(ms)
    if len(Ws) != n or (act_stats is not None and len(act_stats) != n):
        raise ValueError("one weight tensor (and statistic) per matrix")
    dtypes = {_dtype_code(W) for W in Ws}
    if len(dtypes) != 1:
        raise TypeError("all weights must have the same dtype")
    arr = _matrix_array(ms)
    if workspace is None:
        workspace = _workspace(int(_lib.qamw_calibrate_many_workspace_bytes(arr, n)), Ws[0].device)
    wp = (C.c_void_p * max(n, 1))(*[W.data_ptr() for W in Ws])
    ap = None if act_stats is None else (C.c_void_p * max(n, 1))(
        *[None if a is None else a.data_ptr() for a in act_stats])
    rc = _lib.qamw_calibrate_many(wp, dtypes.pop(), ap, float(alpha), arr, n, _p(workspace),
                                  workspace.numel(), _p(status), _s(stream))
    _check("qamw_calibrate_many", rc)
    return ms


def qamw_encode_rows(W: torch.Tensor, m: EncodedMatrix, status: torch.Tensor | None = None,
                     stream=None, candidates: torch.Tensor | None = None) -> EncodedMatrix:
    """Steps 1-6 of section 3.1 with the side values already in m.  `candidates`
    (int64 [1], optional) accumulates the number of codewords scored."""
    st = m.struct()
    rc = _lib.qamw_encode_rows(_p(W), _dtype_code(W), C.byref(st), _p(candidates), _p(status),
                               _s(stream))
    _check("qamw_encode_rows", rc)
    return m


def qamw_polar_codebook(bits: int, codebook: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """Expanded [2^bits, 2] table of the polar baseline (section 3.5)."""
    if codebook is None:
        codebook = torch.empty((1 << bits, 2), dtype=torch.float32, device="cuda")
    _check("qamw_polar_codebook", _lib.qamw_polar_codebook(bits, _p(codebook), _s(stream)))
    return codebook


def qamw_encode_rows_polar(W: torch.Tensor, m: EncodedMatrix, status: torch.Tensor | None = None,
                           stream=None) -> EncodedMatrix:
    """Steps 1-6 of section 3.1 with the polar quantiser of section 3.5."""
    st = m.struct()
    rc = _lib.qamw_encode_rows_polar(_p(W), _dtype_code(W), C.byref(st), _p(status), _s(stream))
    _check("qamw_encode_rows_polar", rc)
    return m


def qamw_scalar_codebook(bits: int, codebook: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """Product table [2^bits, 2] of the d = 1 scalar ablation (section 2)."""
    if codebook is None:
        codebook = torch.empty((1 << bits, 2), dtype=torch.float32, device="cuda")
    _check("qamw_scalar_codebook", _lib.qamw_scalar_codebook(bits, _p(codebook), _s(stream)))
    return codebook


def qamw_encode_rows_scalar(W: torch.Tensor, m: EncodedMatrix, status: torch.Tensor | None = None,
                            stream=None) -> EncodedMatrix:
    """Steps 1-6 of section 3.1 with the d = 1 scalar quantiser."""
    st = m.struct()
    rc = _lib.qamw_encode_rows_scalar(_p(W), _dtype_code(W), C.byref(st), _p(status), _s(stream))
    _check("qamw_encode_rows_scalar", rc)
    return m


def qamw_normalised_pairs(W: torch.Tensor, m: EncodedMatrix, row0: int = 0,
                          nrows: int | None = None, out: torch.Tensor | None = None,
                          status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The normalised points z_k / sigma_k of rows [row0, row0 + nrows) as a float32
    [nrows, d_in / 2, 2] tensor (the encoder's points, bitwise; NaN for rows whose
    norm is zero or not finite): samples for a per-checkpoint codebook."""
    if nrows is None:
        nrows = m.d_out - row0
    if out is None:
        out = torch.empty((nrows, m.d_in // 2, 2), dtype=torch.float32, device=W.device)
    st = m.struct()
    rc = _lib.qamw_normalised_pairs(_p(W), _dtype_code(W), C.byref(st), row0, nrows, _p(out),
                                    _p(status), _s(stream))
    _check("qamw_normalised_pairs", rc)
    return out


def qamw_selftest_wait_timeout(tries: int, status: torch.Tensor, cycles: torch.Tensor | None = None,
                               stream=None) -> None:
    """Bounded-wait failure check: a wait that nothing completes gives up after
    `tries` polls and flags QAMW_STATUS_TIMEOUT in `status`."""
    _check("qamw_selftest_wait_timeout",
           _lib.qamw_selftest_wait_timeout(tries, _p(status), _p(cycles), _s(stream)))


def qamw_decode(m: EncodedMatrix, out: torch.Tensor | None = None,
                status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Decoder of paper section 3.2 into a bf16 [d_out, d_in] tensor."""
    if out is None:
        out = torch.empty((m.d_out, m.d_in), dtype=torch.bfloat16, device=m.packed.device)
    st = m.struct()
    rc = _lib.qamw_decode(C.byref(st), _p(out), _p(status), _s(stream))
    _check("qamw_decode", rc)
    return out


def qamw_decode_many(ms: list, outs: list | None = None, status: torch.Tensor | None = None,
                     stream=None) -> list:
    """qamw_decode of every matrix of `ms` in one call (bf16 [d_out, d_in] each)."""
    if outs is None:
        outs = [torch.empty((m.d_out, m.d_in), dtype=torch.bfloat16, device=m.packed.device)
                for m in ms]
    n = len(ms)
    arr = _matrix_array(ms)
    ptrs = (C.c_void_p * max(n, 1))(*[o.data_ptr() for o in outs])
    rc = _lib.qamw_decode_many(arr, n, ptrs, _p(status), _s(stream))
    _check("qamw_decode_many", rc)
    return outs


def qamw_decode_gemv(m: EncodedMatrix, x: torch.Tensor, y: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """y = x W_hat^T (bf16 [batch, d_out]) decoding the weights on the fly."""
    x2 = x if x.dim() == 2 else x.view(1, -1)
    batch = x2.shape[0]
    if y is None:
        y = torch.empty((batch, m.d_out), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = _workspace(qamw_workspace_bytes(QAMW_OP_GEMV, m.d_out, m.d_in, m.bits, batch),
                               x.device)
    st = m.struct()
    rc = _lib.qamw_decode_gemv(C.byref(st), _p(x2), batch, _p(y), _p(workspace), workspace.numel(),
                               _p(status), _s(stream))
    _check("qamw_decode_gemv", rc)
    return y


def qamw_decode_gemv_many_workspace_bytes(ms: list) -> int:
    return int(_lib.qamw_decode_gemv_many_workspace_bytes(_matrix_array(ms), len(ms)))


def qamw_decode_gemv_many(ms: list, xs: list, ys: list | None = None,
                          workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
                          stream=None) -> list:
    """Batch-1 y_i = x_i W_hat_i^T of every matrix of `ms` in one call (x_i: bf16
    [d_in] or [1, d_in]; y_i: bf16 [1, d_out])."""
    n = len(ms)
    if len(xs) != n or (ys is not None and len(ys) != n):
        raise ValueError("one activation (and output) per matrix")
    if ys is None:
        ys = [torch.empty((1, m.d_out), dtype=torch.bfloat16, device=x.device) for m, x in zip(ms, xs)]
    arr = _matrix_array(ms)
    if workspace is None:
        workspace = _workspace(int(_lib.qamw_decode_gemv_many_workspace_bytes(arr, n)),
                               xs[0].device if n else torch.device("cuda"))
    xp = (C.c_void_p * max(n, 1))(*[x.data_ptr() for x in xs])
    yp = (C.c_void_p * max(n, 1))(*[y.data_ptr() for y in ys])
    rc = _lib.qamw_decode_gemv_many(arr, n, xp, yp, _p(workspace), workspace.numel(), _p(status),
                                    _s(stream))
    _check("qamw_decode_gemv_many", rc)
    return ys


def qamw_decode_gemm(m: EncodedMatrix, x: torch.Tensor, y: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Y = X W_hat^T (bf16 [ntok, d_out]) for many tokens on the tensor cores."""
    ntok = x.shape[0]
    if y is None:
        y = torch.empty((ntok, m.d_out), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = _workspace(qamw_workspace_bytes(QAMW_OP_GEMM, m.d_out, m.d_in, m.bits, ntok),
                               x.device)
    st = m.struct()
    rc = _lib.qamw_decode_gemm(C.byref(st), _p(x), ntok, _p(y), _p(workspace), workspace.numel(),
                               _p(status), _s(stream))
    _check("qamw_decode_gemm", rc)
    return y


def qamw_decode_gemv_noalloc(m: EncodedMatrix, x: torch.Tensor, y: torch.Tensor,
                             status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """qamw_decode_gemv without a workspace, for callers that cannot allocate
    device memory: the rotated activation lives in a fixed array inside the
    library (limit: padded batch x d_in/2 <= 131072 pairs).  `y` must be given
    (this wrapper allocates nothing either).  Calls that overlap on the GPU
    share that array and must be serialised."""
    x2 = x if x.dim() == 2 else x.view(1, -1)
    batch = x2.shape[0]
    if x2.dtype != torch.bfloat16 or not x2.is_contiguous() or x2.shape[1] != m.d_in:
        raise ValueError("x must be a contiguous bf16 [batch, d_in] tensor")
    if (y.dtype != torch.bfloat16 or not y.is_contiguous() or tuple(y.shape) != (batch, m.d_out)
            or y.device != x2.device):
        raise ValueError("y must be a contiguous bf16 [batch, d_out] tensor on x's device")
    st = m.struct()
    rc = _lib.qamw_decode_gemv_noalloc(C.byref(st), _p(x2), batch, _p(y), _p(status), _s(stream))
    _check("qamw_decode_gemv_noalloc", rc)
    return y
