"""Seeded synthetic inputs for the UFP4 hot path (shared by tests, smoke and bench).

This module generates operands only: it holds none of the method's arithmetic
(no rotation, scaling, rounding or contraction).  Every tensor is a bf16 bit
pattern (``numpy.uint16``) produced from a seeded PCG64 stream, rounded to
bf16 with round-to-nearest-even, so the oracle and the CUDA library see the
same bits.

Shapes and distributions are the workloads the paper's recipe targets: one
linear layer's X / W / dY, heavy-tailed tensors for the quantizer sweep and a
Zipf-routed mixture-of-experts layer.  "N(0, s)" means standard deviation s.
Outlier channels multiply whole input channels (columns of X) by a factor, the
structure RHT is meant to spread ([PL] §3.2 "outlier-heavy training tensors").
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

SEED_X, SEED_W, SEED_DY, SEED_OUTLIER, SEED_STUDENT, SEED_ZIPF = 1, 2, 3, 4, 5, 6


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern, round to nearest even (finite inputs)."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal(rows: int, cols: int, std: float, seed: int) -> np.ndarray:
    g = _rng(seed)
    a = g.standard_normal((rows, cols), dtype=np.float32)
    a *= np.float32(std)
    return bf16_bits(a)


def normal_with_outlier_channels(rows: int, cols: int, std: float, n_out: int,
                                 factor: float, seed: int = SEED_X,
                                 seed_out: int = SEED_OUTLIER) -> np.ndarray:
    """N(0, std) with ``n_out`` seeded columns (input channels) scaled by ``factor``."""
    g = _rng(seed)
    a = g.standard_normal((rows, cols), dtype=np.float32)
    a *= np.float32(std)
    cols_out = _rng(seed_out).choice(cols, size=n_out, replace=False)
    a[:, cols_out] *= np.float32(factor)
    return bf16_bits(a)


def student_t(rows: int, cols: int, nu: float = 4.0, scale: float = 0.1,
              seed: int = SEED_STUDENT) -> np.ndarray:
    g = _rng(seed)
    a = g.standard_t(nu, size=(rows, cols)).astype(np.float32)
    a *= np.float32(scale)
    return bf16_bits(a)


# --------------------------------------------------------------- named sets
@dataclass
class LayerShape:
    M: int  # tokens
    K: int  # input channels
    N: int  # output channels
    x_outlier_frac: float
    x_outlier_factor: float
    w_std: float
    dy_std: float


TINY = LayerShape(M=256, K=512, N=512, x_outlier_frac=0.0, x_outlier_factor=20.0,
                  w_std=0.02, dy_std=1e-3)
LAYER = LayerShape(M=8192, K=2048, N=8192, x_outlier_frac=0.005, x_outlier_factor=30.0,
                   w_std=0.02, dy_std=1e-3)
LARGE = LayerShape(M=16384, K=8192, N=28672, x_outlier_frac=0.01, x_outlier_factor=50.0,
                   w_std=0.01, dy_std=1e-4)


_LAYER_CACHE: dict = {}


def layer_inputs(shape: LayerShape, want_dy: bool = True, n_outliers: int | None = None,
                 cache: bool = True):
    """X [M, K], W [N, K], dY [M, N] as bf16 bit patterns (memoised per shape)."""
    key = (shape.M, shape.K, shape.N, want_dy, n_outliers)
    if cache and key in _LAYER_CACHE:
        return _LAYER_CACHE[key]
    out = _layer_inputs(shape, want_dy, n_outliers)
    if cache:
        _LAYER_CACHE.clear()
        _LAYER_CACHE[key] = out
    return out


def _layer_inputs(shape: LayerShape, want_dy: bool, n_outliers: int | None):
    if n_outliers is None:
        n_outliers = int(round(shape.x_outlier_frac * shape.K))
    if shape is TINY:
        n_outliers = 4
    X = normal_with_outlier_channels(shape.M, shape.K, 1.0, n_outliers,
                                     shape.x_outlier_factor)
    W = normal(shape.N, shape.K, shape.w_std, SEED_W)
    dY = normal(shape.M, shape.N, shape.dy_std, SEED_DY) if want_dy else None
    return X, W, dY


QUANT_SWEEP_SHAPES = [(4096, 4096), (16384, 8192), (32768, 16384)]


# --------------------------------------------------------------- MoE routing
@dataclass
class MoEShape:
    tokens: int = 16384
    hidden: int = 2048
    ffn: int = 1408
    experts: int = 64
    topk: int = 6
    zipf_s: float = 1.2


MOE = MoEShape()


def moe_expert_counts(shape: MoEShape = MOE, seed: int = SEED_ZIPF) -> np.ndarray:
    """Rows routed to each expert: Zipf(s) over expert rank, total tokens*topk.

    No expert can receive a token twice, so each count is capped at ``tokens``;
    the excess is redistributed over the uncapped experts in proportion to their
    Zipf weight (water filling), counts are rounded by largest remainder, and
    ranks are assigned to experts by a seeded permutation.
    """
    total = shape.tokens * shape.topk
    w = np.arange(1, shape.experts + 1, dtype=np.float64) ** (-shape.zipf_s)
    target = np.zeros(shape.experts)
    capped = np.zeros(shape.experts, dtype=bool)
    remaining = float(total)
    while True:
        free = ~capped
        share = w[free] / w[free].sum() * remaining
        over = share > shape.tokens
        if not over.any():
            target[free] = share
            break
        idx = np.flatnonzero(free)[over]
        target[idx] = shape.tokens
        capped[idx] = True
        remaining = total - target[capped].sum()
    base = np.floor(target).astype(np.int64)
    short = total - int(base.sum())
    order = np.argsort(-(target - base), kind="stable")
    base[order[:short]] += 1
    perm = _rng(seed).permutation(shape.experts)
    counts = np.empty(shape.experts, dtype=np.int64)
    counts[perm] = base
    return counts


def padded_offsets(counts: np.ndarray, align: int = 64):
    """Start row of each expert segment when every segment is zero-padded to
    a multiple of ``align`` rows; returns (starts, padded_counts, total)."""
    padded = (counts + align - 1) // align * align
    starts = np.concatenate([[0], np.cumsum(padded)[:-1]]).astype(np.int64)
    return starts, padded.astype(np.int64), int(padded.sum())
