"""Seeded synthetic inputs for the IQ8R rotated W8A8 linear.

This module is shared by the CPU oracle and the CUDA path. It draws random
numbers and casts them to the bf16 input format; it holds none of the
method's arithmetic (no rotation, no scales, no quantisation).

The pages measure on a whole model (Qwen3.8-27B) and a public
quantisation-challenge dataset ("Qwen3.8-27B IQ8R + DFlash2 -- radiance
container", sections "Quality" and "Speed"). Neither is available, so these
generators stand in for them with tensors of the pages' shapes.

Recipe, in this fixed order, from ``numpy.random.default_rng(seed)`` (PCG64):

1. W = sigma_w * standard_normal((N, K), float32), sigma_w = 0.02;
2. if ``w_outlier_frac`` > 0: cols = rng.choice(K, round(frac * K),
   replace=False); W[:, cols] *= 8;
3. x = standard_normal((M, K), float32);
4. ch = rng.choice(K, x_outliers, replace=False); x[:, ch] *= 20;
5. both cast to bf16 with round-to-nearest-even.

bf16 tensors are returned as ``uint16`` bit patterns (numpy has no bf16).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "f32_to_bf16_bits",
    "bf16_bits_to_f32",
    "gen_weight",
    "gen_act",
    "gen_workload",
]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Cast float32 values to bf16 bit patterns, round-to-nearest-even.

    Only finite inputs are produced by the generators, so NaN handling is
    not needed here.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, weight format and generator knobs."""

    name: str
    m: int
    k: int
    n: int
    fmt: str  # "g256" (trunk: u8 per 256 under a bf16 row scale), "g128" (bf16 per 128), "cb4" (codebook)
    seed: int
    w_outlier_frac: float
    x_outliers: int
    sigma_w: float = 0.02
    x_outlier_mult: float = 20.0
    w_outlier_mult: float = 8.0


# Shapes of the pages' workloads: the 27B trunk's hidden size 5120, its MLP
# width 17408 (gate/up output, down-projection input) and the 151936-entry
# vocabulary. M spans a decode step, a speculative-verify block and an
# 8K-token prefill ("Speed" on the IQ8R container page).
WORKLOADS: dict[str, Workload] = {
    "pr1": Workload("pr1", m=4, k=512, n=256, fmt="g256", seed=0, w_outlier_frac=0.0, x_outliers=2),
    "decode": Workload("decode", m=1, k=5120, n=17408, fmt="g256", seed=1, w_outlier_frac=0.01, x_outliers=8),
    "verify8": Workload("verify8", m=8, k=17408, n=5120, fmt="g256", seed=2, w_outlier_frac=0.01, x_outliers=8),
    "verify16": Workload("verify16", m=16, k=17408, n=5120, fmt="g256", seed=2, w_outlier_frac=0.01, x_outliers=8),
    "verify128": Workload("verify128", m=128, k=17408, n=5120, fmt="g256", seed=2, w_outlier_frac=0.01, x_outliers=8),
    "prefill": Workload("prefill", m=8192, k=5120, n=17408, fmt="g256", seed=3, w_outlier_frac=0.01, x_outliers=8),
    # the trunk in the earlier IQ8R format: a bf16 scale per (row, 128 of K)
    # instead of u8 under a bf16 row scale (IQ8R page, introduction)
    "decode_g128": Workload("decode_g128", m=1, k=5120, n=17408, fmt="g128", seed=1, w_outlier_frac=0.01,
                            x_outliers=8),
    "prefill_g128": Workload("prefill_g128", m=8192, k=5120, n=17408, fmt="g128", seed=3, w_outlier_frac=0.01,
                             x_outliers=8),
    # the drafter's linears in their codebook format, at the trunk's shape
    "draft_cb4": Workload("draft_cb4", m=1, k=5120, n=17408, fmt="cb4", seed=5, w_outlier_frac=0.01, x_outliers=8),
    "lm_head1": Workload("lm_head1", m=1, k=5120, n=151936, fmt="g128", seed=4, w_outlier_frac=0.0, x_outliers=8),
    "lm_head8": Workload("lm_head8", m=8, k=5120, n=151936, fmt="g128", seed=4, w_outlier_frac=0.0, x_outliers=8),
}


def gen_weight(rng: np.random.Generator, n: int, k: int, sigma_w: float = 0.02,
               w_outlier_frac: float = 0.0, w_outlier_mult: float = 8.0) -> np.ndarray:
    """Steps 1-2 of the recipe; returns float32 [n, k] (not yet cast)."""
    w = rng.standard_normal((n, k), dtype=np.float32)
    w *= np.float32(sigma_w)
    n_cols = int(round(w_outlier_frac * k))
    if n_cols > 0:
        cols = rng.choice(k, n_cols, replace=False)
        w[:, cols] *= np.float32(w_outlier_mult)
    return w


def gen_act(rng: np.random.Generator, m: int, k: int, x_outliers: int = 0,
            x_outlier_mult: float = 20.0) -> np.ndarray:
    """Steps 3-4 of the recipe; returns float32 [m, k] (not yet cast)."""
    x = rng.standard_normal((m, k), dtype=np.float32)
    if x_outliers > 0:
        ch = rng.choice(k, x_outliers, replace=False)
        x[:, ch] *= np.float32(x_outlier_mult)
    return x


def gen_workload(wl: Workload | str, m: int | None = None, n: int | None = None,
                 k: int | None = None, seed: int | None = None):
    """Generate (x_bf16_bits [M, K], w_bf16_bits [N, K]) for a workload.

    ``m``, ``n``, ``k`` and ``seed`` override the workload's own values so a
    test can draw a smaller tensor with the same value distribution.
    """
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    m = wl.m if m is None else m
    n = wl.n if n is None else n
    k = wl.k if k is None else k
    seed = wl.seed if seed is None else seed
    rng = np.random.default_rng(seed)
    w = gen_weight(rng, n, k, wl.sigma_w, wl.w_outlier_frac, wl.w_outlier_mult)
    x = gen_act(rng, m, k, wl.x_outliers, wl.x_outlier_mult)
    return f32_to_bf16_bits(x), f32_to_bf16_bits(w)
