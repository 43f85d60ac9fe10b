"""Small single-kernel cases for ncu captures (inputs larger than L2, a few
hundred MB on the device at most), so that a full-metric capture of one
launch ends quickly.  Each case runs its kernel twice: a warm-up launch and
the launch to capture.

    python -m fp4_quantized_gemms_b200.profile_cases gemm --m 4096 --n 4096 --k 2048 --grid e1m2
    python -m fp4_quantized_gemms_b200.profile_cases gemm --m 4096 --n 8192 --k 8192 --mx
    python -m fp4_quantized_gemms_b200.profile_cases gemm --m 4096 --n 4096 --k 2048 --fp32-scales
    python -m fp4_quantized_gemms_b200.profile_cases grouped --tokens 4096
    python -m fp4_quantized_gemms_b200.profile_cases quantize --rows 8192 --cols 8192 --axis rows --sr
    python -m fp4_quantized_gemms_b200.profile_cases quantize --rows 8192 --cols 2048 --dual
    python -m fp4_quantized_gemms_b200.profile_cases stats --rows 8192 --cols 8192 --axis rows
"""
from __future__ import annotations

import argparse

import numpy as np
import torch

from fp4_quantized_gemms_b200 import ufp4
from fp4_quantized_gemms_b200 import workloads as wl


def _dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def gemm_case(m: int, n: int, k: int, grid: int, path: int, mx: bool = False, fp32: bool = False) -> None:
    """Quantize X [m, k] and W [n, k] (RHT16; two-level scales with block 16,
    or with `mx` UE8M0 scales with block 32 and the E4M3 element planes, or
    with `fp32` fp32 scales with block 16), then run the FPROP GEMM twice."""
    if mx:
        cfg = ufp4.QuantConfig(grid=grid, hadamard_n=16, block=32, scale_fmt=ufp4.SCALE_UE8M0)
    elif fp32:
        cfg = ufp4.QuantConfig(grid=grid, hadamard_n=16, block=16, scale_fmt=ufp4.SCALE_FP32)
    else:
        cfg = ufp4.QuantConfig(grid=grid, hadamard_n=16, block=16, scale_fmt=ufp4.SCALE_E4M3_X_FP32)
    qx = ufp4.rht_quantize(_dev(wl.normal(m, k, 1.0, 1)), ufp4.ALONG_COLS, cfg)
    qw = ufp4.rht_quantize(_dev(wl.normal(n, k, 0.02, 2)), ufp4.ALONG_COLS, cfg)
    ufp4.set_two_level_gemm_path(path)
    out = torch.empty((m, n), dtype=torch.float32, device="cuda")
    for _ in range(2):
        ufp4.gemm_fprop(qx, qw, out)
    torch.cuda.synchronize()
    if ufp4.check_device_status() != ufp4.OK:
        raise RuntimeError("device error word set")


def grouped_case(tokens: int, experts: int, hidden: int, ffn: int) -> None:
    """The gate/up FPROP of a mixture-of-experts layer: tokens x top-6 routed
    rows in Zipf(1.2) expert segments (zero-padded to 64 rows), two-level
    scales, one grouped GEMM over the device group table, twice."""
    shp = wl.MoEShape(tokens=tokens, hidden=hidden, ffn=ffn, experts=experts, topk=6, zipf_s=1.2)
    counts = wl.moe_expert_counts(shp)
    starts, _, total = wl.padded_offsets(counts, 64)
    x = wl.normal(total, hidden, 1.0, 1)
    mask = np.zeros(total, dtype=bool)
    for s0, c in zip(starts, counts):
        mask[s0:s0 + c] = True
    x[~mask] = 0
    cfg = ufp4.QuantConfig(grid=ufp4.GRID_E1M2, hadamard_n=16, block=16, scale_fmt=ufp4.SCALE_E4M3_X_FP32)
    qx = ufp4.rht_quantize(_dev(x), ufp4.ALONG_COLS, cfg)
    qw = ufp4.rht_quantize(_dev(wl.normal(experts * 2 * ffn, hidden, 0.02, 2)), ufp4.ALONG_COLS, cfg)
    groups = [(counts[e], 2 * ffn, hidden, starts[e], 0, e * 2 * ffn, 0, starts[e], 0) for e in range(experts)]
    g = torch.tensor(np.array(groups, dtype=np.int64), device="cuda")
    out = torch.empty((total, 2 * ffn), dtype=torch.float32, device="cuda")
    for _ in range(2):
        ufp4.grouped_gemm(qx, qw, g, out)
    torch.cuda.synchronize()
    if ufp4.check_device_status() != ufp4.OK:
        raise RuntimeError("device error word set")


def quantize_case(rows: int, cols: int, axis: int, sr: bool, two_level: bool, dual: bool = False) -> None:
    """Rotated amax + quantize of one bf16 operand, twice (with `dual`: both
    layouts from one read, through the dual-output kernel)."""
    fmt = ufp4.SCALE_E4M3_X_FP32 if two_level else ufp4.SCALE_FP32
    cfg = ufp4.QuantConfig(grid=ufp4.GRID_E1M2, rounding=ufp4.ROUND_SR if sr else ufp4.ROUND_RTNE,
                           sr_seed=1234, hadamard_n=16, block=16, scale_fmt=fmt)
    x = _dev(wl.normal(rows, cols, 1e-3, 3))
    q = None
    for _ in range(2):
        if dual:
            q = ufp4.rht_quantize_dual(x, cfg, cfg.with_(sr_stream=1), out=q)
        else:
            q = ufp4.rht_quantize(x, axis, cfg, out=q)
    torch.cuda.synchronize()
    if ufp4.check_device_status() != ufp4.OK:
        raise RuntimeError("device error word set")


def stats_case(rows: int, cols: int, axis: int) -> None:
    """Quantize once, then the diagnostics kernel on the operand, twice."""
    cfg = ufp4.QuantConfig(grid=ufp4.GRID_E1M2, hadamard_n=16, block=16,
                           scale_fmt=ufp4.SCALE_E4M3_X_FP32)
    x = _dev(wl.normal(rows, cols, 1e-3, 3))
    q = ufp4.rht_quantize(x, axis, cfg)
    buf = None
    for _ in range(2):
        buf = ufp4.quant_stats_launch(x, axis, q, out=buf)
    torch.cuda.synchronize()
    if ufp4.check_device_status() != ufp4.OK:
        raise RuntimeError("device error word set")


def main() -> None:
    ap = argparse.ArgumentParser()
    sub = ap.add_subparsers(dest="case", required=True)
    g = sub.add_parser("gemm")
    g.add_argument("--m", type=int, default=4096)
    g.add_argument("--n", type=int, default=4096)
    g.add_argument("--k", type=int, default=2048)
    g.add_argument("--grid", choices=["e1m2", "e2m1"], default="e1m2")
    g.add_argument("--path", type=int, default=ufp4.GEMM_PATH_AUTO)
    g.add_argument("--mx", action="store_true", help="UE8M0 block-32 scales (the MX path)")
    g.add_argument("--fp32-scales", action="store_true", help="fp32 block-16 scales (the fp32-scale kernel)")
    m = sub.add_parser("grouped")
    m.add_argument("--tokens", type=int, default=4096)
    m.add_argument("--experts", type=int, default=64)
    m.add_argument("--hidden", type=int, default=2048)
    m.add_argument("--ffn", type=int, default=1408)
    q = sub.add_parser("quantize")
    q.add_argument("--rows", type=int, default=8192)
    q.add_argument("--cols", type=int, default=8192)
    q.add_argument("--axis", choices=["cols", "rows"], default="cols")
    q.add_argument("--sr", action="store_true")
    q.add_argument("--fp32-scales", action="store_true")
    q.add_argument("--dual", action="store_true")
    t = sub.add_parser("stats")
    t.add_argument("--rows", type=int, default=8192)
    t.add_argument("--cols", type=int, default=8192)
    t.add_argument("--axis", choices=["cols", "rows"], default="rows")
    a = ap.parse_args()
    if a.case == "gemm":
        gemm_case(a.m, a.n, a.k, ufp4.GRID_E1M2 if a.grid == "e1m2" else ufp4.GRID_E2M1, a.path, a.mx,
                  a.fp32_scales)
    elif a.case == "grouped":
        grouped_case(a.tokens, a.experts, a.hidden, a.ffn)
    elif a.case == "stats":
        stats_case(a.rows, a.cols, ufp4.ALONG_COLS if a.axis == "cols" else ufp4.ALONG_ROWS)
    else:
        quantize_case(a.rows, a.cols, ufp4.ALONG_COLS if a.axis == "cols" else ufp4.ALONG_ROWS,
                      a.sr, not a.fp32_scales, a.dual)
    print("ok")


if __name__ == "__main__":
    main()
