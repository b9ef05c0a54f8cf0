"""Seeded synthetic inputs for the QAM-W codec workloads.

This module draws random numbers and nothing else: it holds none of the codec's
arithmetic, so both the CUDA path's tests/benchmark and the CPU oracle's tests
can take their inputs from it.  Every array comes from ``numpy.random.Generator``
(PCG64) seeded by a (workload, layer, tensor) tuple, so a given call returns the
same values on every machine.

The shapes and distributions stand in for the LLM checkpoints and WikiText-2
activations that the QAM-W paper evaluates on (TinyLlama-1.1B ... 13B models),
which are not used here:

* weights: Student-t with 5 degrees of freedom times 0.02 (heavy-tailed, like
  trained linear layers), or N(0, 0.02^2) with a few rows scaled up;
* activation statistics: lognormal magnitudes with 1% outlier channels x20
  (the per-channel activation statistic that drives the AWQ-style scaling);
* codebook training samples: the unit circular Gaussian N(0, I_2) of the
  paper's eq. (2);
* GEMV inputs: N(0, 1) activations with 1% outlier channels x20.
"""
from __future__ import annotations

import numpy as np

# Tensor ids used in seeds.
T_WEIGHT, T_ACT, T_X, T_SAMPLES, T_ROWS = 1, 2, 3, 4, 5


def rng(*key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(k) for k in key]))


def circular_gaussian_samples(n: int, seed: int = 0) -> np.ndarray:
    """n draws from N(0, I_2) as float32 [n, 2]."""
    return rng(seed, T_SAMPLES).standard_normal((n, 2), dtype=np.float64).astype(np.float32)


def gaussian_weights(d_out: int, d_in: int, seed: int = 0, scale: float = 0.02,
                     n_big_rows: int = 4, big: float = 10.0) -> np.ndarray:
    """float32 N(0, scale^2) matrix with `n_big_rows` seeded rows multiplied by `big`."""
    g = rng(seed, T_WEIGHT)
    W = (g.standard_normal((d_out, d_in)) * scale).astype(np.float32)
    if n_big_rows:
        rows = rng(seed, T_ROWS).choice(d_out, size=min(n_big_rows, d_out), replace=False)
        W[rows] *= np.float32(big)
    return W


def student_t_weights(d_out: int, d_in: int, seed: int = 0, scale: float = 0.02,
                      nu: float = 5.0) -> np.ndarray:
    """float32 Student-t(nu) * scale matrix."""
    return (rng(seed, T_WEIGHT).standard_t(nu, size=(d_out, d_in)) * scale).astype(np.float32)


def act_stat_lognormal(d_in: int, seed: int = 0, sigma: float = 1.0, outlier_frac: float = 0.01,
                       outlier_mult: float = 20.0) -> np.ndarray:
    """Positive per-channel activation statistic: lognormal(0, sigma) with
    round(outlier_frac * d_in) seeded channels multiplied by outlier_mult."""
    g = rng(seed, T_ACT)
    a = g.lognormal(0.0, sigma, size=d_in)
    n_out = int(round(outlier_frac * d_in))
    if n_out:
        a[g.choice(d_in, size=n_out, replace=False)] *= outlier_mult
    return a.astype(np.float32)


def gemv_x(batch: int, d_in: int, seed: int = 0, outlier_frac: float = 0.01,
           outlier_mult: float = 20.0) -> np.ndarray:
    """float32 [batch, d_in] N(0,1) activations with outlier channels."""
    g = rng(seed, T_X)
    x = g.standard_normal((batch, d_in))
    n_out = int(round(outlier_frac * d_in))
    if n_out:
        x[:, g.choice(d_in, size=n_out, replace=False)] *= outlier_mult
    return x.astype(np.float32)


# ----------------------------------------------------------------- workloads
# Each returns a dict of host arrays; `name` says what it is.

def tiny_case(seed: int = 0) -> dict:
    """One 256x512 fp32 matrix, N(0, 0.02^2) with 4 rows x10; mean|x| statistic
    lognormal(0, 0.5); alpha 0.5; block 64; K = 256 (4 bits/weight); codebook
    trained by 50 Lloyd iterations on 2^20 N(0, I_2) samples."""
    return dict(name="256x512 fp32 N(0,0.02^2), K=256, block 64", d_out=256, d_in=512,
                W=gaussian_weights(256, 512, seed), dtype="f32",
                act_stat=act_stat_lognormal(512, seed, sigma=0.5, outlier_frac=0.0),
                alpha=0.5, block=64, bits=8, train_n=1 << 20, train_iters=50, seed=seed)


def llama_square_case(seed: int = 0) -> dict:
    """One 4096x4096 bf16 Student-t(5) x0.02 matrix; lognormal(0,1) statistic with
    1% outlier channels x20; alpha 0.5; block 128; K = 2048 (~5.5 bpw)."""
    return dict(name="4096x4096 bf16 Student-t(5)x0.02, K=2048, block 128", d_out=4096,
                d_in=4096, W=student_t_weights(4096, 4096, seed), dtype="bf16",
                act_stat=act_stat_lognormal(4096, seed), alpha=0.5, block=128, bits=11,
                train_n=1 << 20, train_iters=50, seed=seed)


def llama2_7b_layer_shapes() -> list[tuple[str, int, int]]:
    """(name, d_out, d_in) of the seven linear weights of one Llama-2-7B layer."""
    return [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
            ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]


def llama_13b_layer_shapes() -> list[tuple[str, int, int]]:
    """(name, d_out, d_in) of the seven linear weights of one 13B-shaped layer."""
    return [("q", 5120, 5120), ("k", 5120, 5120), ("v", 5120, 5120), ("o", 5120, 5120),
            ("gate", 13824, 5120), ("up", 13824, 5120), ("down", 5120, 13824)]


# The input each linear weight of a transformer layer sees: q/k/v share the
# attention input, gate/up share the MLP input, o and down see their own.  One
# activation statistic is drawn per (layer, input).
LAYER_INPUT = {"q": 0, "k": 0, "v": 0, "o": 1, "gate": 2, "up": 2, "down": 3}


def layer_matrices(shapes: list[tuple[str, int, int]], layers: int, workload: int) -> list[dict]:
    """Every linear weight of `layers` layers in order (layer-major), each with
    the seeds of its weights and of its activation statistic."""
    out = []
    for layer in range(layers):
        for t, (name, d_out, d_in) in enumerate(shapes):
            out.append(dict(layer=layer, name=name, d_out=d_out, d_in=d_in,
                            w_seed=(workload, layer, t),
                            act_seed=(workload, layer, 100 + LAYER_INPUT[name])))
    return out


def act_stat_for(key: tuple, d_in: int) -> np.ndarray:
    """act_stat_lognormal seeded by a (workload, layer, input) key."""
    g = rng(*key, T_ACT)
    a = g.lognormal(0.0, 1.0, size=d_in)
    n_out = int(round(0.01 * d_in))
    if n_out:
        a[g.choice(d_in, size=n_out, replace=False)] *= 20.0
    return a.astype(np.float32)


def student_t_weights_device(d_out: int, d_in: int, key: tuple, device, out=None,
                             scale: float = 0.02, nu: int = 5):
    """Student-t(nu) * scale weights drawn on a CUDA device by torch's Philox
    generator (for workloads too large to draw on the host): t = Z / sqrt(V / nu)
    with V the sum of nu squared standard normals.  Returns bf16 [d_out, d_in]
    (written into `out` when given).  Seeded by `key`; the values differ from
    student_t_weights' (another generator) but follow the same distribution."""
    import torch
    seed = int(np.random.SeedSequence([int(k) for k in key]).generate_state(1, np.uint64)[0] >> 1)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    if out is None:
        out = torch.empty((d_out, d_in), dtype=torch.bfloat16, device=device)
    rows = max(1, (1 << 26) // d_in)  # bounded temporaries
    for r0 in range(0, d_out, rows):
        n = min(rows, d_out - r0)
        z = torch.randn((n, d_in), generator=g, device=device)
        v = torch.zeros_like(z)
        for _ in range(nu):
            e = torch.randn((n, d_in), generator=g, device=device)
            v.addcmul_(e, e)
        out[r0:r0 + n] = (z * torch.rsqrt(v / nu) * scale).to(torch.bfloat16)
    return out
