"""Quantization diagnostics of the oracle (test infrastructure only, like the
rest of ``oracle/``).

What the pages measure (paperlayer.ai summary §5 "Q1: Grid geometry and RHT",
Appendix A "RHT-Induced SQNR Changes in Tensors and GEMM Outputs"; gist.science
"Kwantisatie en GEMM Diagnostiek"): the signal-to-quantization-noise ratio of a
quantized tensor and of a GEMM output, its change under the RHT, the
"effective bucket" use of the 4-bit codes, and the signed rounding error of the
grid's levels (the Shrinkage Bias of §3.1).  The pages print no formulas for
these; the readings taken here:

* tensor SQNR: 10 log10(sum u^2 / sum (u - deq)^2) over the logical K columns of
  the operand, u the rotated values the quantizer rounds and deq the
  dequantized codes (same rotated domain; the RHT is orthogonal up to a factor
  n, so the ratio equals the one of the original domain);
* per-level signed error, in grid units: for elements coded with magnitude
  index k in a block of step sigma > 0, lvl(k) - |u| / sigma (negative =
  shrinkage), summed per k together with its element count;
* code occupancy: the 16-bin histogram of the 4-bit codes; the effective bucket
  ratio is the share of the grid's codes (15, or 9 for the restricted E2M1
  grid) whose occupancy exceeds 1/(15 * 16) of the elements;
* underflow ratio: the share of nonzero rotated values coded 0;
* GEMM output SQNR: 10 log10(sum ref^2 / sum (test - ref)^2).

Everything is plain numpy in float64 on top of ``oracle.quantize``.
"""
from __future__ import annotations

import numpy as np

import oracle


def _steps(q: oracle.QTensor) -> np.ndarray:
    """Per-element block step sigma (float64): s, e_b * S, or 2^(E - 127) (exact in fp64)."""
    B = q.cfg.block
    if q.scales is not None:
        per_block = q.scales.astype(np.float64)
    elif q.cfg.scale_fmt == oracle.SCALE_UE8M0:
        per_block = np.ldexp(1.0, q.escales.astype(np.int64) - 127)
    else:
        table = np.array([oracle.e4m3_value(b) for b in range(256)], dtype=np.float64)
        per_block = table[q.escales] * float(np.float32(q.S))
    return np.repeat(per_block, B, axis=1)


def quant_stats(q: oracle.QTensor, u: np.ndarray) -> dict:
    """Sums and counts over the logical columns [0, q.k) of an operand quantized
    by ``oracle.quantize(..., want_u=True)``."""
    K = q.k
    codes = q.codes[:, :K].astype(np.int64)
    uu = u[:, :K].astype(np.float64)
    deq = q.dequantize()[:, :K]
    sigma = _steps(q)[:, :K]
    mag = codes & 7
    lv = oracle.levels(q.cfg.grid)
    full = np.array([oracle.level(q.cfg.grid, k) for k in range(8)])
    live = sigma > 0
    err = np.zeros_like(uu)
    err[live] = full[mag[live]] - np.abs(uu[live]) / sigma[live]
    level_err = np.array([err[(mag == k) & live].sum() for k in range(8)])
    level_n = np.array([np.count_nonzero((mag == k) & live) for k in range(8)], dtype=np.int64)
    nz = uu != 0
    return {
        "signal": float(np.sum(uu * uu)),
        "noise": float(np.sum((uu - deq) ** 2)),
        "level_err": level_err,
        "level_n": level_n,
        "code_count": np.bincount(codes.ravel(), minlength=16).astype(np.int64),
        "nonzero": int(np.count_nonzero(nz)),
        "underflow": int(np.count_nonzero(nz & (mag == 0))),
        "grid_codes": 2 * (len(lv) - 1) + 1,
    }


def sqnr_db(signal: float, noise: float) -> float:
    return float("inf") if noise == 0 else 10.0 * np.log10(signal / noise)


def summary(st: dict) -> dict:
    """Derived figures: SQNR (dB), effective bucket ratio, underflow ratio and
    the mean signed error of each magnitude level (NaN where unused)."""
    total = int(st["code_count"].sum())
    occupied = int(np.count_nonzero(st["code_count"] * 240 > total)) if total else 0
    with np.errstate(invalid="ignore", divide="ignore"):
        mean_err = st["level_err"] / st["level_n"]
    return {
        "sqnr_db": sqnr_db(st["signal"], st["noise"]),
        "bucket_ratio": occupied / st["grid_codes"],
        "underflow_ratio": st["underflow"] / st["nonzero"] if st["nonzero"] else 0.0,
        "level_mean_err": mean_err,
    }


def gemm_sqnr_sums(ref: np.ndarray, test: np.ndarray) -> tuple[float, float]:
    """(sum ref^2, sum (test - ref)^2) in float64."""
    r = np.asarray(ref, dtype=np.float64)
    t = np.asarray(test, dtype=np.float64)
    return float(np.sum(r * r)), float(np.sum((t - r) ** 2))
