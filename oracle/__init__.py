"""fp64 CPU oracle of the QAM-W codec (TEST INFRASTRUCTURE).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The library path (``libqamw.so`` and its
Python binding) never imports, links or calls it, and the two share no code.

The arithmetic lives in ``qamw_oracle.c`` (plain C, fp64).  This module only
builds that file with gcc, marshals numpy arrays into it, and splits rows over
threads (ctypes drops the GIL during each call; every row is computed by the
same single-threaded C code, so the split does not change any result).

Sections cited below refer to "QAM-W: Joint 2D Codebook Quantization for LLM
Weights via Hadamard Rotation and Activation-Aware Scaling" (Sharma & Dobek).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qamw_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libqamw_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile qamw_oracle.c into a shared library (gcc, fp64, no FMA contraction)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_DEFAULT_SOURCE", "-ffp-contract=off",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = C.CDLL(build())
    P, I, I64, D, U64 = C.c_void_p, C.c_int, C.c_int64, C.c_double, C.c_uint64
    sig = {
        "ref_half_to_double": (D, [C.c_uint16]),
        "ref_double_to_half": (C.c_uint16, [D]),
        "ref_splitmix64": (U64, [U64]),
        "ref_sign": (I, [U64, I64]),
        "ref_default_block": (I, [I]),
        "ref_bits_per_weight": (D, [I, I]),
        "ref_row_bytes": (I64, [I, I]),
        "ref_hadamard": (None, [I, P]),
        "ref_rotate_fwd": (None, [P, I, I, U64, P]),
        "ref_rotate_inv": (None, [P, I, I, U64, P]),
        "ref_channel_scales": (I, [P, I, D, P]),
        "ref_calibrate_sigma": (None, [P, I, I, I, U64, P, P]),
        "ref_nearest": (I, [D, D, P, I]),
        "ref_nearest_batch": (None, [P, I64, P, I, P]),
        "ref_encode_rows": (None, [P, I, I, I, U64, P, P, P, I, I, I, P, P, P]),
        "ref_pack_rows": (None, [P, I, I, I, I64, P]),
        "ref_unpack_rows": (None, [P, I, I, I, I64, P]),
        "ref_decode_rows": (None, [P, I64, I, I, I, U64, P, P, P, P, I, I, P]),
        "ref_gemv": (None, [P, I, I, P, I, I, I, P]),
        "ref_lloyd": (None, [P, I64, I, I, P, P]),
        "ref_rayleigh_lloyd_max": (None, [I, I, P]),
        "ref_polar_codebook": (None, [I, P, P]),
        "ref_polar_index": (I, [D, D, P, I]),
        "ref_encode_rows_polar": (None, [P, I, I, I, U64, P, P, P, I, I, I, P, P, P]),
        "ref_gauss_lloyd_max": (None, [I, I, P]),
        "ref_gauss_mse": (D, [I, P]),
        "ref_scalar_codebook": (None, [I, P, P]),
        "ref_scalar_index": (I, [D, D, P, I]),
        "ref_encode_rows_scalar": (None, [P, I, I, I, U64, P, P, P, I, I, I, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def _row_split(n: int, parts: int):
    parts = max(1, min(parts, n))
    edges = np.linspace(0, n, parts + 1).astype(int)
    return [(int(edges[t]), int(edges[t + 1])) for t in range(parts) if edges[t + 1] > edges[t]]


def _parallel_rows(n_rows: int, fn, threads: int | None):
    spans = _row_split(n_rows, threads or _threads())
    if len(spans) == 1:
        fn(*spans[0])
        return
    with ThreadPoolExecutor(len(spans)) as ex:
        list(ex.map(lambda s: fn(*s), spans))


# ---------------------------------------------------------------- scalars

def half_to_double(h: int) -> float:
    return _load().ref_half_to_double(int(h))


def double_to_half(x: float) -> int:
    return int(_load().ref_double_to_half(float(x)))


def halves_to_f64(h: np.ndarray) -> np.ndarray:
    lib = _load()
    return np.array([lib.ref_half_to_double(int(v)) for v in np.asarray(h).ravel()],
                    dtype=np.float64).reshape(np.shape(h))


def f64_to_halves(x: np.ndarray) -> np.ndarray:
    lib = _load()
    return np.array([lib.ref_double_to_half(float(v)) for v in np.asarray(x).ravel()],
                    dtype=np.uint16).reshape(np.shape(x))


def splitmix64(counter: int) -> int:
    return int(_load().ref_splitmix64(counter & 0xFFFFFFFFFFFFFFFF))


def sign_mask(mask_seed: int, d: int) -> np.ndarray:
    lib = _load()
    return np.array([lib.ref_sign(mask_seed, j) for j in range(d)], dtype=np.int8)


def default_block(d_in: int) -> int:
    """Section 3.3 block rule."""
    return int(_load().ref_default_block(d_in))


def bits_per_weight(d_in: int, bits: int) -> float:
    """Section 3.7 eq. (3)."""
    return float(_load().ref_bits_per_weight(d_in, bits))


def row_bytes(d_in: int, bits: int) -> int:
    return int(_load().ref_row_bytes(d_in, bits))


def hadamard(b: int) -> np.ndarray:
    H = np.empty((b, b), dtype=np.int8)
    _load().ref_hadamard(b, _p(H))
    return H


def rotate_fwd(u: np.ndarray, block: int, mask_seed: int = 0) -> np.ndarray:
    """y = R_fwd u per block (section 3.1 step 2); u is one row of length d."""
    u = np.ascontiguousarray(u, dtype=np.float64)
    y = np.empty_like(u)
    _load().ref_rotate_fwd(_p(u), u.size, block, mask_seed, _p(y))
    return y


def rotate_inv(y: np.ndarray, block: int, mask_seed: int = 0) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.float64)
    u = np.empty_like(y)
    _load().ref_rotate_inv(_p(y), y.size, block, mask_seed, _p(u))
    return u


def channel_scales(act_stat: np.ndarray | None, d_in: int, alpha: float) -> np.ndarray:
    """binary16 s_j = (a_j / mean a)^alpha (explainer, activation-aware scaling)."""
    s = np.empty(d_in, dtype=np.uint16)
    a = None if act_stat is None else np.ascontiguousarray(act_stat, dtype=np.float64)
    rc = _load().ref_channel_scales(_p(a), d_in, float(alpha), _p(s))
    if rc != 0:
        raise ValueError("activation statistic must be positive and finite")
    return s


def calibrate_sigma(W: np.ndarray, block: int, s_half: np.ndarray, mask_seed: int = 0) -> np.ndarray:
    """binary16 sigma_k of section 3.4 eq. (1)."""
    W = np.ascontiguousarray(W, dtype=np.float64)
    d_out, d_in = W.shape
    sig = np.empty(d_in // 2, dtype=np.uint16)
    s_half = np.ascontiguousarray(s_half, dtype=np.uint16)
    _load().ref_calibrate_sigma(_p(W), d_out, d_in, block, mask_seed, _p(s_half), _p(sig))
    return sig


def nearest(points: np.ndarray, codebook: np.ndarray) -> np.ndarray:
    """Brute-force nearest codeword, lowest index on ties (section 3.6)."""
    pts = np.ascontiguousarray(points, dtype=np.float64).reshape(-1, 2)
    cb = np.ascontiguousarray(codebook, dtype=np.float64).reshape(-1, 2)
    out = np.empty(pts.shape[0], dtype=np.int32)
    lib = _load()

    def run(a, b):
        lib.ref_nearest_batch(_p(pts) + 16 * a, b - a, _p(cb), cb.shape[0], _p(out) + 4 * a)

    _parallel_rows(pts.shape[0], run, None)
    return out


def encode(W: np.ndarray, bits: int, block: int, codebook: np.ndarray, *, mask_seed: int = 0,
           act_stat: np.ndarray | None = None, alpha: float = 0.0,
           s_half: np.ndarray | None = None, sigma_half: np.ndarray | None = None,
           want_points: bool = False, threads: int | None = None) -> dict:
    """Encoder of section 3.1 (steps 1-6) with activation-aware scaling.

    ``s_half`` / ``sigma_half`` (binary16 bit patterns) replace the computed
    channel scales / pair scales when given.
    """
    W = np.ascontiguousarray(W, dtype=np.float64)
    d_out, d_in = W.shape
    P = d_in // 2
    cb = np.ascontiguousarray(codebook, dtype=np.float64).reshape(-1, 2)
    K = cb.shape[0]
    assert K == 1 << bits
    if s_half is None:
        s_half = channel_scales(act_stat, d_in, alpha)
    s_half = np.ascontiguousarray(s_half, dtype=np.uint16)
    if sigma_half is None:
        sigma_half = calibrate_sigma(W, block, s_half, mask_seed)
    sigma_half = np.ascontiguousarray(sigma_half, dtype=np.uint16)
    rnorm = np.zeros(d_out, dtype=np.uint16)
    idx = np.zeros((d_out, P), dtype=np.int32)
    pts = np.zeros((d_out, P, 2), dtype=np.float64) if want_points else None
    lib = _load()

    def run(a, b):
        lib.ref_encode_rows(_p(W), d_out, d_in, block, mask_seed, _p(s_half), _p(sigma_half),
                            _p(cb), K, a, b, _p(rnorm), _p(idx), _p(pts))

    _parallel_rows(d_out, run, threads)
    rb = row_bytes(d_in, bits)
    packed = pack(idx, bits, rb)
    out = dict(s_half=s_half, sigma_half=sigma_half, rnorm_half=rnorm, idx=idx, packed=packed,
               row_bytes=rb, bits=bits, block=block, mask_seed=mask_seed, d_in=d_in, d_out=d_out)
    if want_points:
        out["points"] = pts
    return out


def pack(idx: np.ndarray, bits: int, row_bytes_: int) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    n, P = idx.shape
    out = np.empty((n, row_bytes_), dtype=np.uint8)
    _load().ref_pack_rows(_p(idx), n, P, bits, row_bytes_, _p(out))
    return out


def unpack(packed: np.ndarray, P: int, bits: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    n, rb = packed.shape
    out = np.empty((n, P), dtype=np.int32)
    _load().ref_unpack_rows(_p(packed), n, P, bits, rb, _p(out))
    return out


def decode(enc: dict, codebook: np.ndarray, threads: int | None = None) -> np.ndarray:
    """Decoder of section 3.2 in fp64, from the packed stream."""
    packed = np.ascontiguousarray(enc["packed"], dtype=np.uint8)
    d_out, d_in = enc["d_out"], enc["d_in"]
    cb = np.ascontiguousarray(codebook, dtype=np.float64).reshape(-1, 2)
    rn = np.ascontiguousarray(enc["rnorm_half"], dtype=np.uint16)
    sg = np.ascontiguousarray(enc["sigma_half"], dtype=np.uint16)
    sh = np.ascontiguousarray(enc["s_half"], dtype=np.uint16)
    out = np.empty((d_out, d_in), dtype=np.float64)
    lib = _load()

    def run(a, b):
        lib.ref_decode_rows(_p(packed), packed.shape[1], d_in, enc["block"], enc["bits"],
                            enc["mask_seed"], _p(rn), _p(sg), _p(sh), _p(cb), a, b, _p(out))

    _parallel_rows(d_out, run, threads)
    return out


def gemv(W: np.ndarray, x: np.ndarray, threads: int | None = None) -> np.ndarray:
    """y = x W^T by the dense definition; x is [batch, d_in]."""
    W = np.ascontiguousarray(W, dtype=np.float64)
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float64)
    d_out, d_in = W.shape
    batch = x.shape[0]
    y = np.empty((batch, d_out), dtype=np.float64)
    lib = _load()

    def run(a, b):
        lib.ref_gemv(_p(W), d_out, d_in, _p(x), batch, a, b, _p(y))

    _parallel_rows(d_out, run, threads)
    return y


def lloyd(samples: np.ndarray, K: int, iters: int):
    """Lloyd iterations of section 3.6 eq. (2) from the first K samples.

    Returns (codebook [K,2] fp64, distortion per iteration [iters])."""
    s = np.ascontiguousarray(samples, dtype=np.float64).reshape(-1, 2)
    cb = np.empty((K, 2), dtype=np.float64)
    dist = np.empty(max(iters, 1), dtype=np.float64)
    _load().ref_lloyd(_p(s), s.shape[0], K, iters, _p(cb), _p(dist))
    return cb, dist[:iters]


# ------------------------------------------------------------- polar baseline

def rayleigh_lloyd_max(N: int, iters: int = 20000) -> np.ndarray:
    """Section 3.5: N-level Lloyd-Max codebook of the unit Rayleigh density."""
    lv = np.empty(N, dtype=np.float64)
    _load().ref_rayleigh_lloyd_max(N, iters, _p(lv))
    return lv


def polar_split(bits: int) -> tuple[int, int]:
    """(amplitude bits, phase bits) = (floor(B/2), B - floor(B/2))."""
    return bits // 2, bits - bits // 2


def polar_levels(bits: int, iters: int = 20000) -> np.ndarray:
    return rayleigh_lloyd_max(1 << polar_split(bits)[0], iters)


def polar_codebook(bits: int, levels: np.ndarray | None = None) -> np.ndarray:
    """Expanded K-entry table: entry ia * Np + ip = a_ia (cos 2 pi ip/Np, sin 2 pi ip/Np)."""
    if levels is None:
        levels = polar_levels(bits)
    lv = np.ascontiguousarray(levels, dtype=np.float64)
    cb = np.empty((1 << bits, 2), dtype=np.float64)
    _load().ref_polar_codebook(bits, _p(lv), _p(cb))
    return cb


def polar_index(points: np.ndarray, levels: np.ndarray, bits: int) -> np.ndarray:
    lib = _load()
    lv = np.ascontiguousarray(levels, dtype=np.float64)
    pts = np.asarray(points, dtype=np.float64).reshape(-1, 2)
    return np.array([lib.ref_polar_index(float(x), float(y), _p(lv), bits) for x, y in pts],
                    dtype=np.int32)


def encode_polar(W: np.ndarray, bits: int, block: int, levels: np.ndarray, *, mask_seed: int = 0,
                 s_half: np.ndarray, sigma_half: np.ndarray, want_points: bool = False,
                 threads: int | None = None) -> dict:
    """Encoder of section 3.1 with the polar quantiser of section 3.5 (given s, sigma)."""
    W = np.ascontiguousarray(W, dtype=np.float64)
    d_out, d_in = W.shape
    P = d_in // 2
    lv = np.ascontiguousarray(levels, dtype=np.float64)
    s_half = np.ascontiguousarray(s_half, dtype=np.uint16)
    sigma_half = np.ascontiguousarray(sigma_half, dtype=np.uint16)
    rnorm = np.zeros(d_out, dtype=np.uint16)
    idx = np.zeros((d_out, P), dtype=np.int32)
    pts = np.zeros((d_out, P, 2), dtype=np.float64) if want_points else None
    lib = _load()

    def run(a, b):
        lib.ref_encode_rows_polar(_p(W), d_out, d_in, block, mask_seed, _p(s_half),
                                  _p(sigma_half), _p(lv), bits, a, b, _p(rnorm), _p(idx), _p(pts))

    _parallel_rows(d_out, run, threads)
    rb = row_bytes(d_in, bits)
    out = dict(s_half=s_half, sigma_half=sigma_half, rnorm_half=rnorm, idx=idx,
               packed=pack(idx, bits, rb), row_bytes=rb, bits=bits, block=block,
               mask_seed=mask_seed, d_in=d_in, d_out=d_out)
    if want_points:
        out["points"] = pts
    return out


# ------------------------------------------------------------- d = 1 ablation

def gauss_lloyd_max(L: int, iters: int = 20000) -> np.ndarray:
    """Section 2 (parallel work), the d = 1 ablation: L-level Lloyd-Max quantiser of N(0, 1)."""
    lv = np.empty(L, dtype=np.float64)
    _load().ref_gauss_lloyd_max(L, iters, _p(lv))
    return lv


def gauss_mse(levels: np.ndarray) -> float:
    """Mean squared error of the midpoint quantiser with these levels on N(0, 1)."""
    lv = np.ascontiguousarray(levels, dtype=np.float64)
    return float(_load().ref_gauss_mse(len(lv), _p(lv)))


def scalar_levels(bits: int, iters: int = 20000) -> np.ndarray:
    """The 2^(bits/2) levels of the scalar code with `bits` (even) per pair."""
    if bits % 2:
        raise ValueError("the scalar code needs an even number of bits per pair")
    return gauss_lloyd_max(1 << (bits // 2), iters)


def scalar_codebook(bits: int, levels: np.ndarray | None = None) -> np.ndarray:
    """Product table: entry ix * L + iy = (l_ix, l_iy)."""
    if levels is None:
        levels = scalar_levels(bits)
    lv = np.ascontiguousarray(levels, dtype=np.float64)
    cb = np.empty((1 << bits, 2), dtype=np.float64)
    _load().ref_scalar_codebook(bits, _p(lv), _p(cb))
    return cb


def scalar_index(points: np.ndarray, levels: np.ndarray, bits: int) -> np.ndarray:
    lib = _load()
    lv = np.ascontiguousarray(levels, dtype=np.float64)
    pts = np.asarray(points, dtype=np.float64).reshape(-1, 2)
    return np.array([lib.ref_scalar_index(float(x), float(y), _p(lv), bits) for x, y in pts],
                    dtype=np.int32)


def encode_scalar(W: np.ndarray, bits: int, block: int, levels: np.ndarray, *, mask_seed: int = 0,
                  s_half: np.ndarray, sigma_half: np.ndarray, want_points: bool = False,
                  threads: int | None = None) -> dict:
    """Encoder of section 3.1 with the d = 1 scalar quantiser (given s, sigma)."""
    W = np.ascontiguousarray(W, dtype=np.float64)
    d_out, d_in = W.shape
    P = d_in // 2
    lv = np.ascontiguousarray(levels, dtype=np.float64)
    s_half = np.ascontiguousarray(s_half, dtype=np.uint16)
    sigma_half = np.ascontiguousarray(sigma_half, dtype=np.uint16)
    rnorm = np.zeros(d_out, dtype=np.uint16)
    idx = np.zeros((d_out, P), dtype=np.int32)
    pts = np.zeros((d_out, P, 2), dtype=np.float64) if want_points else None
    lib = _load()

    def run(a, b):
        lib.ref_encode_rows_scalar(_p(W), d_out, d_in, block, mask_seed, _p(s_half),
                                   _p(sigma_half), _p(lv), bits, a, b, _p(rnorm), _p(idx), _p(pts))

    _parallel_rows(d_out, run, threads)
    rb = row_bytes(d_in, bits)
    out = dict(s_half=s_half, sigma_half=sigma_half, rnorm_half=rnorm, idx=idx,
               packed=pack(idx, bits, rb), row_bytes=rb, bits=bits, block=block,
               mask_seed=mask_seed, d_in=d_in, d_out=d_out)
    if want_points:
        out["points"] = pts
    return out
