"""Seeded synthetic inputs for the five LLM-layer workloads.

This module draws random numbers and rounds them to bf16; it holds none of
the method's arithmetic (no pruning, scaling, quantisation or GEMM), so both
the CUDA path and the CPU oracle can consume exactly the same bytes.

Recipe: ``numpy.random.default_rng([seed, cfg, stream, *extra])`` with
seed 0, ``cfg`` the workload number 1-5 and ``stream`` 0 for W, 1 for X and
2 for the outlier-column permutation.  Values are drawn in float64 and
rounded to bf16 (round to nearest even) by ``ml_dtypes``; tensors are
returned as ``uint16`` bf16 bit patterns.

The shapes follow LLM linear layers: a Llama-7B-like MLP up-projection
4096 -> 11008 (decode-shaped, M tokens in {1, 8, 32, 64}), a fused QKV
projection 4096 -> 12288 at prefill (M = 4096, with 1% of the activation
columns scaled by 20 as outliers), an MLP down-projection 14336 -> 4096 with
heavy-tailed (Student-t, nu = 3) weights, and a 4096 x 4096 layer for the
6:8 sliding-window case.  They stand in for real model weights and
activations, which this project does not ship.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import ml_dtypes
import numpy as np

SEED = 0


@dataclass(frozen=True)
class Workload:
    cfg: int
    name: str
    n: int
    k: int
    ms: tuple
    w_dist: str = "normal"          # "normal" (sd 0.02) or "student_t3" (x 0.02)
    x_outlier_frac: float = 0.0     # fraction of X columns scaled by 20
    pattern: str = "2:4"            # "2:4" or "6:8"
    notes: str = ""
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    1: Workload(1, "tiny 2:4 FP8 GEMM M16 K256 N256", 256, 256, (16,)),
    2: Workload(2, "decode MLP up-proj W[11008,4096]", 11008, 4096, (1, 8, 32, 64)),
    3: Workload(3, "prefill fused QKV M4096 N12288 K4096", 12288, 4096, (4096,),
                x_outlier_frac=0.01),
    4: Workload(4, "MLP down-proj M256 N4096 K14336", 4096, 14336, (256,),
                w_dist="student_t3"),
    5: Workload(5, "6:8 sliding-window W[4096,4096] K'=6144", 4096, 4096, (64, 2048),
                pattern="6:8"),
}


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (nearest even) and return the bit patterns."""
    return np.asarray(x, dtype=np.float64).astype(ml_dtypes.bfloat16).view(np.uint16)


def weight_bits(cfg: int, n: int | None = None, k: int | None = None, layer: int = 0) -> np.ndarray:
    """W [n, k] as bf16 bits for workload ``cfg`` (defaults to its full shape).

    ``layer`` selects an independent draw (used to build several distinct
    layers of the same shape).
    """
    wl = WORKLOADS[cfg]
    n = wl.n if n is None else n
    k = wl.k if k is None else k
    extra = [] if layer == 0 else [layer]
    rng = np.random.default_rng([SEED, cfg, 0, *extra])
    if wl.w_dist == "normal":
        w = rng.normal(0.0, 0.02, size=(n, k))
    elif wl.w_dist == "student_t3":
        w = rng.standard_t(3.0, size=(n, k)) * 0.02
    else:
        raise ValueError(wl.w_dist)
    return to_bf16_bits(w)


def activation_bits(cfg: int, m: int, k: int | None = None) -> np.ndarray:
    """X [m, k] as bf16 bits for workload ``cfg``; N(0, 1), with the
    workload's outlier columns (a seeded permutation) scaled by 20."""
    wl = WORKLOADS[cfg]
    k = wl.k if k is None else k
    rng = np.random.default_rng([SEED, cfg, 1, m])
    x = rng.normal(0.0, 1.0, size=(m, k))
    if wl.x_outlier_frac > 0:
        n_out = int(round(wl.x_outlier_frac * k))
        perm = np.random.default_rng([SEED, cfg, 2]).permutation(k)
        x[:, perm[:n_out]] *= 20.0
    return to_bf16_bits(x)


def random_bits(shape, seed, scale=1.0, dist="normal") -> np.ndarray:
    """Generic seeded bf16 tensor for parity cases beyond the five workloads."""
    rng = np.random.default_rng([SEED, 99, *np.atleast_1d(seed).tolist()])
    if dist == "normal":
        x = rng.normal(0.0, scale, size=shape)
    elif dist == "student_t3":
        x = rng.standard_t(3.0, size=shape) * scale
    elif dist == "ties":
        # small integer magnitudes with random signs: many exact ties and zeros
        x = rng.integers(-2, 3, size=shape).astype(np.float64) * scale
    else:
        raise ValueError(dist)
    return to_bf16_bits(x)
