"""Comparison rules between the CUDA path and the fp64 oracle.

Indices: equal, except where the oracle and the kernel land on different
codewords at a near-tie.  The kernel decides in fp32 (scores |c|^2 - 2 p.c);
a differing index is accepted only when, in fp64 at the oracle's point p,
    | |p - c_gpu|^2 - |p - c_oracle|^2 | <= 1e-5 (1 + |p|^2),
about five times the fp32 rounding of the kernel's point and score.  Every
accepted mismatch is counted and reported.

Decoded weights and GEMV outputs: elementwise |got - ref| <= 1e-2 max(|ref|,
rms of the row), and relative Frobenius error <= 1e-2 (the 1e-2 relative
tolerance of the codec's parity target).

binary16 side values (s, sigma, r): at most one unit in the last place.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

TIE_TOL = 1e-5
REL_TOL = 1e-2


def halves(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def to_half_tensor(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(
        torch.float16).to(device)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def ulp_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """|a - b| in binary16 ulps for non-negative finite halves given as bit patterns."""
    return np.abs(a.astype(np.int64) - b.astype(np.int64))


def check_indices(got: np.ndarray, want: np.ndarray, points: np.ndarray, codebook: np.ndarray,
                  rows_mask: np.ndarray | None = None) -> dict:
    """got/want [rows, P] indices; points [rows, P, 2] oracle fp64 points."""
    cb = np.asarray(codebook, dtype=np.float64).reshape(-1, 2)
    diff = got != want
    if rows_mask is not None:
        diff &= rows_mask[:, None]
    r, k = np.nonzero(diff)
    p = points[r, k]
    dg = ((p - cb[got[r, k]]) ** 2).sum(-1)
    do = ((p - cb[want[r, k]]) ** 2).sum(-1)
    gap = np.abs(dg - do)
    tol = TIE_TOL * (1.0 + (p ** 2).sum(-1))
    bad = gap > tol
    stats = dict(n=int(diff.size), mismatches=int(diff.sum()),
                 max_gap=float(gap.max()) if gap.size else 0.0, bad=int(bad.sum()))
    log_stats("indices", stats)
    assert stats["bad"] == 0, (stats, list(zip(r[bad][:5], k[bad][:5], gap[bad][:5])))
    assert stats["mismatches"] <= max(8, 1e-4 * diff.size), stats
    return stats


def log_stats(kind: str, stats: dict) -> None:
    """Append parity statistics to $QAMW_PARITY_LOG (JSON lines) when it is set."""
    path = os.environ.get("QAMW_PARITY_LOG")
    if path:
        test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
        with open(path, "a") as f:
            f.write(json.dumps(dict(test=test, kind=kind, **stats)) + "\n")


def check_close(got: np.ndarray, ref: np.ndarray, axis_rms: int = -1, what: str = "") -> dict:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = np.sqrt((ref ** 2).mean(axis=axis_rms, keepdims=True))
    bound = REL_TOL * np.maximum(np.abs(ref), rms)
    err = np.abs(got - ref)
    worst = float((err / np.where(bound > 0, bound, 1.0)).max()) if err.size else 0.0
    fro = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    log_stats("close:" + what, dict(max_elem_ratio=worst, rel_fro=fro))
    assert np.all(err <= bound), (what, worst, fro)
    assert fro <= REL_TOL, (what, fro)
    return dict(max_elem_ratio=worst, rel_fro=fro)
