"""Benchmark of the UFP4 hot path on B200.

One step = the whole data-parallel hot path of one large linear layer of LLM
pretraining under the UFP4 recipe: RHT + block-scale + 4-bit quantize of every
GEMM operand along its reduction dimension (X and W: RTNE; dY: stochastic
rounding, Philox seed 1234) and the three training GEMMs
    FPROP Y = X W^T,  DGRAD dX = dY W,  WGRAD dW = dY^T X
on X [16384, 8192] ~ N(0,1) with 82 (1%) outlier channels x50, W [28672, 8192]
~ N(0, 0.01), dY [16384, 28672] ~ N(0, 1e-4); RHT16, scale block 16, E1M2 grid
with two-level (E4M3 block x fp32 tensor) scales.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--scale two-level|fp32] [--workload large|layer] [--quick]

Prints one JSON line (rank 0).  `value` is the effective UFP4 GEMM throughput of
the whole step: 3 * 2*M*N*K / step time (quantization included).  The line also
carries the E2M1-RTNE baseline of the same layer, the quantizer sweep over the
three sweep tensors, the fused-vs-unfused RHT ratio, the grouped MoE GEMMs, the
quantization diagnostics, the MX block-32 FPROP, the end-to-end figure through
host buffers and the CPU oracle baseline.  Multi-GPU runs are independent
replicas (the path has no exchange step): weak scaling, time = max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from fp4_quantized_gemms_b200 import workloads as wl  # noqa: E402

METRIC = "UFP4 GEMM TFLOPS & % tensor peak; RHT-quantize HBM GB/s & % of 8 TB/s"
SHAPES = {"large": wl.LARGE, "layer": wl.LAYER}
SR_SEED = 1234
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
HBM_SPEC_GBS = 8000.0
L2_BYTES = 126 * 1024 * 1024
FP4_OVER_BF16 = 4.0          # nominal dense fp4 / bf16 tensor rates (9 / 2.25 PFLOP/s)


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of the ranks' values; every rank takes part (NCCL on the
    GPU machine, any backend the process group was created with)."""
    if world <= 1:
        return x
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, flops_per_step: float, ms_per_step: float) -> float:
    """Whole-job throughput of `world` replicas each doing `flops_per_step` per
    step, the step time being the slowest rank's."""
    return world * flops_per_step / (ms_per_step * 1e-3) / 1e12


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(shape, scale: str) -> dict:
    s = shape
    n_out = int(round(s.x_outlier_frac * s.K))
    name = "large dense layer" if s is wl.LARGE else "one linear layer"
    return {
        "workload": (f"{name}, all three GEMMs: X bf16 {s.M}x{s.K} ~N(0,1) with {n_out} "
                     f"({s.x_outlier_frac:.1%}) outlier channels x{s.x_outlier_factor:g}, W bf16 "
                     f"{s.N}x{s.K} ~N(0,{s.w_std:g}), dY bf16 {s.M}x{s.N} ~N(0,{s.dy_std:g}); RHT16 on "
                     f"every operand along its K, block 16, E1M2; RTNE X/W, SR (Philox seed {SR_SEED}) dY"),
        "scales": "E4M3 block x fp32 tensor (two-level)" if scale == "two-level" else "fp32 per block",
        "M": s.M, "K": s.K, "N": s.N,
        "gemm_flops_per_step": 3 * 2 * s.M * s.N * s.K,
        "l2": "inputs larger than L2: every operand and output of a step is larger than the 126 MB L2",
    }


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out = ""

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        loaded = [v for v in sm if v > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ device arm
def to_dev(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


class LayerStep:
    """Preallocated buffers and one call sequence of the hot path of a layer:
    grid E1M2 (the recipe: RTNE on X and W, SR on dY) or E2M1 (the baseline
    grid, RTNE on every operand)."""

    def __init__(self, device, scale: str, shape, inputs, grid: int | None = None):
        from fp4_quantized_gemms_b200 import ufp4
        self.u = ufp4
        self.dev = device
        self.shape = shape
        self.grid = ufp4.GRID_E1M2 if grid is None else grid
        two = scale == "two-level"
        fmt = ufp4.SCALE_E4M3_X_FP32 if two else ufp4.SCALE_FP32
        base = ufp4.QuantConfig(grid=self.grid, hadamard_n=16, block=16, scale_fmt=fmt)
        self.two = two
        self.c_rtne = base
        if self.grid == ufp4.GRID_E1M2:
            self.c_sr0 = base.with_(rounding=ufp4.ROUND_SR, sr_seed=SR_SEED, sr_stream=0)
            self.c_sr1 = base.with_(rounding=ufp4.ROUND_SR, sr_seed=SR_SEED, sr_stream=1)
        else:
            self.c_sr0 = self.c_sr1 = base
        s = shape
        self.X, self.W, self.dY = inputs
        C, R = ufp4.ALONG_COLS, ufp4.ALONG_ROWS
        E = ufp4.empty_qtensor
        # Per-lane factor tiles only on the GEMMs' first operands.
        self.qx = E(s.M, s.K, self.c_rtne, device)                    # FPROP A
        self.qw = E(s.N, s.K, self.c_rtne, device, with_lanes=False)  # FPROP B
        self.qdy = E(s.M, s.N, self.c_sr0, device)                    # DGRAD A
        self.qwt = E(s.K, s.N, self.c_rtne, device, with_lanes=False)  # DGRAD B
        self.qdyt = E(s.N, s.M, self.c_sr1, device)                   # WGRAD A
        self.qxt = E(s.K, s.M, self.c_rtne, device, with_lanes=False)  # WGRAD B
        # Each tensor feeds two GEMMs, one along each axis: one quantization
        # call per operand (two single-output calls measured faster than the
        # dual-output pass at these sizes).  The rotated amaxes of all six
        # operands come from one dual amax pass per tensor.
        self.ops = self._ops()
        self.amax = torch.zeros(6, dtype=torch.float32, device=device)   # [cols, rows] per tensor
        self.Y = torch.empty((s.M, s.N), dtype=torch.float32, device=device)
        self.dX = torch.empty((s.M, s.K), dtype=torch.float32, device=device)
        self.dW = torch.empty((s.N, s.K), dtype=torch.float32, device=device)
        self.launches = (3 if two else 0) + len(self.ops) + 3
        self.tensor_elems = self.X.numel() + self.W.numel() + self.dY.numel()
        self.quant_elems = 2 * self.tensor_elems         # elements quantized per step

    def _ops(self):
        """(input, axis, output, amax slot) of the six quantizations."""
        C, R = self.u.ALONG_COLS, self.u.ALONG_ROWS
        return [(self.X, C, self.qx, 0), (self.X, R, self.qxt, 1), (self.W, C, self.qw, 2),
                (self.W, R, self.qwt, 3), (self.dY, C, self.qdy, 4), (self.dY, R, self.qdyt, 5)]

    def bind(self, X, W, dY, Y, dX, dW):
        """Point the step at other input / output buffers of the same shapes."""
        self.X, self.W, self.dY, self.Y, self.dX, self.dW = X, W, dY, Y, dX, dW
        self.ops = self._ops()

    def quantize_all(self):
        u = self.u
        sm = self.c_rtne.rht_sign_mask
        if self.two:
            for i, x in enumerate((self.X, self.W, self.dY)):
                u.rht_amax_dual(x, 16, sm, out=self.amax[2 * i:2 * i + 2])
        for x, axis, q, slot in self.ops:
            am = self.amax[slot:slot + 1] if self.two else None
            u.rht_quantize(x, axis, q.cfg, tensor_amax=am, out=q)

    def gemms(self, events=None):
        u = self.u
        if events:
            events[0].record()
        u.gemm_fprop(self.qx, self.qw, out=self.Y)
        if events:
            events[1].record()
        u.gemm_dgrad(self.qdy, self.qwt, out=self.dX)
        if events:
            events[2].record()
        u.gemm_wgrad(self.qdyt, self.qxt, out=self.dW)
        if events:
            events[3].record()

    def step(self, events=None):
        if events:
            events[0].record()
        self.quantize_all()
        self.gemms(events[1:] if events else None)

    def free(self):
        for name in ("qx", "qw", "qdy", "qwt", "qdyt", "qxt", "Y", "dX", "dW", "amax"):
            setattr(self, name, None)


def quant_bytes(step: LayerStep) -> float:
    """Algorithmic bytes of the step's quantization: each quantized element
    writes its code and its share of a block scale (fp32, or E4M3); every
    quantization call reads its bf16 input once; with two-level scales the
    dual amax pass reads each tensor once more.  The E1M2 correction planes
    the GEMM reads are not counted."""
    out_per = 0.5 + (4 / 16 if not step.two else 1 / 16)
    total = step.quant_elems * out_per
    total += sum(x.numel() for x, _, _, _ in step.ops) * 2
    if step.two:
        total += step.tensor_elems * 2
    return total


def time_steps(step: LayerStep, steps: int, warmup: int, world: int, device, clocks: bool):
    """Device-timed steps: CUDA events on the launching stream, bracketed by a
    barrier and a synchronize on both sides; per-phase event splits."""
    stream = torch.cuda.current_stream(device)
    for _ in range(warmup):
        step.step()
    torch.cuda.synchronize(device)
    if step.u.check_device_status() != step.u.OK:
        raise RuntimeError("device error word set during warm-up")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    clk = ClockSampler(device.index if device.index is not None else 0) if clocks else None
    if clk:
        clk.__enter__()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(steps):
        step.step(ev[i])
    end.record(stream)
    torch.cuda.synchronize(device)
    if clk:
        clk.__exit__()
    if world > 1:
        torch.distributed.barrier()
    total_ms = max_over_ranks(start.elapsed_time(end), world, device)
    q_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(steps))
    g_ms = [statistics.mean(ev[i][1 + j].elapsed_time(ev[i][2 + j]) for i in range(steps)) for j in range(3)]
    return total_ms / steps, q_ms, g_ms, (clk.summary() if clk else None)


# ------------------------------------------------------------------ quantizer sweep
def _timed(fn, flush, reps: int = 5, warm: int = 2) -> float:
    """Median of `reps` CUDA-event timings of fn, L2 flushed (256 MB write)
    before each."""
    for _ in range(warm):
        fn()
    ts = []
    for _ in range(reps):
        flush.add_(1.0)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    ts.sort()
    return ts[len(ts) // 2]


def sweep_input(rows: int, cols: int, device) -> torch.Tensor:
    """0.1 * Student-t(nu = 4) bf16 tensor of the sweep, drawn on the device
    from a seeded generator (the parity tests draw the same distribution with
    the host generator of `workloads.student_t`)."""
    g = torch.Generator(device=device)
    g.manual_seed(wl.SEED_STUDENT)
    z = torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32)
    chi2 = torch.empty((rows, cols), device=device, dtype=torch.float32)
    # chi-square with 4 degrees of freedom as -2 log(u1 u2) (two exponentials)
    u1 = torch.rand((rows, cols), generator=g, device=device, dtype=torch.float32).clamp_(min=1e-30)
    u2 = torch.rand((rows, cols), generator=g, device=device, dtype=torch.float32).clamp_(min=1e-30)
    torch.mul(u1, u2, out=chi2).log_().mul_(-2.0)
    del u1, u2
    z.mul_(torch.rsqrt(chi2.div_(4.0))).mul_(0.1)
    del chi2
    return z.to(torch.bfloat16)


def run_sweep(device, peaks, quick: bool = False) -> dict:
    """The quantizer sweep: bf16 4096x4096, 16384x8192, 32768x16384 ~0.1 t(4);
    Hadamard 16/32/64, block 16/32; E1M2 RTNE, E1M2 SR, E2M1 RTNE; fp32
    scales; both axes (plus the dual-output call at n = 16, block 16).  GB/s
    of algorithmic bytes: 2 (bf16 in) + 0.5 (codes) + 4/B (fp32 scales) per
    element of each output (dual: 2 + 2 (0.5 + 4/B))."""
    from fp4_quantized_gemms_b200 import ufp4 as u
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    rows_out = []
    shapes = wl.QUANT_SWEEP_SHAPES[-1:] if quick else wl.QUANT_SWEEP_SHAPES
    modes = [("e1m2_rtne", u.GRID_E1M2, u.ROUND_RTNE), ("e1m2_sr", u.GRID_E1M2, u.ROUND_SR),
             ("e2m1_rtne", u.GRID_E2M1, u.ROUND_RTNE)]
    ratio = None
    for (R, C) in shapes:
        x = sweep_input(R, C, device)
        for n in (16, 32, 64):
            for blk in (16, 32):
                for mode, grid, rnd in modes:
                    cfg = u.QuantConfig(grid=grid, rounding=rnd, sr_seed=SR_SEED, hadamard_n=n, block=blk,
                                        scale_fmt=u.SCALE_FP32)
                    for axis in (u.ALONG_COLS, u.ALONG_ROWS):
                        q = u.rht_quantize(x, axis, cfg)
                        ms = _timed(lambda: u.rht_quantize(x, axis, cfg, out=q), flush)
                        gbs = R * C * (2.5 + 4 / blk) / (ms * 1e-3) / 1e9
                        rows_out.append({"shape": [R, C], "n": n, "block": blk, "mode": mode,
                                         "axis": ("cols", "rows")[axis], "ms": round(ms, 4),
                                         "GBps": round(gbs, 1)})
                        del q
                    if n == 16 and blk == 16:
                        qq = u.rht_quantize_dual(x, cfg)
                        ms = _timed(lambda: u.rht_quantize_dual(x, cfg, out=qq), flush)
                        gbs = R * C * (2 + 2 * (0.5 + 4 / blk)) / (ms * 1e-3) / 1e9
                        rows_out.append({"shape": [R, C], "n": n, "block": blk, "mode": mode,
                                         "axis": "dual", "ms": round(ms, 4), "GBps": round(gbs, 1)})
                        del qq
        if (R, C) == wl.QUANT_SWEEP_SHAPES[-1]:
            ratio = fused_vs_unfused(x, flush)
        del x
        torch.cuda.empty_cache()
    big = [r for r in rows_out if r["shape"] == list(wl.QUANT_SWEEP_SHAPES[-1])]

    def best(pred):
        sel = [r for r in big if pred(r)]
        return max(sel, key=lambda r: r["GBps"]) if sel else None

    def worst(pred):
        sel = [r for r in big if pred(r)]
        return min(sel, key=lambda r: r["GBps"]) if sel else None

    rec = [r for r in big if r["n"] == 16 and r["block"] == 16 and r["mode"] == "e1m2_rtne"
           and r["axis"] in ("cols", "rows")]
    rec_gbs = min(r["GBps"] for r in rec) if rec else None
    summary = {
        "largest_tensor": list(wl.QUANT_SWEEP_SHAPES[-1]),
        "recipe_e1m2_rtne_n16_b16_GBps": rec_gbs,
        "recipe_frac_of_8TBps": round(rec_gbs / HBM_SPEC_GBS, 4) if rec_gbs else None,
        "recipe_frac_of_measured_hbm": round(rec_gbs / hbm, 4) if rec_gbs else None,
        "best": best(lambda r: r["axis"] != "dual"),
        "worst": worst(lambda r: r["axis"] != "dual"),
        "e1m2_sr_worst": worst(lambda r: r["mode"] == "e1m2_sr" and r["axis"] != "dual"),
    }
    return {"workload": ("quantizer sweep: bf16 4096x4096, 16384x8192, 32768x16384 ~0.1 Student-t(4) "
                         "(device generator, seed 5); RHT 16/32/64, block 16/32; E1M2 RTNE, E1M2 SR "
                         "(seed 1234), E2M1 RTNE; fp32 scales; both axes; L2 flushed between runs"),
            "bytes_per_element": "2 + 0.5 + 4/B (dual: 2 + 2 (0.5 + 4/B))",
            "hbm_peak_GBps": hbm, "summary": summary, "fused_vs_unfused": ratio, "rows": rows_out}


def fused_vs_unfused(x: torch.Tensor, flush) -> dict:
    """The pages' kernel-fusion comparison on the largest sweep tensor, row-wise,
    E1M2 RTNE, block 16, fp32 scales: quantization alone (n = 0), the fused
    RHT16 + quantization, and the unfused pair (a separate RHT pass writing
    bf16, then quantization with n = 0)."""
    from fp4_quantized_gemms_b200 import ufp4 as u
    cfg16 = u.QuantConfig(hadamard_n=16, block=16)
    cfg0 = cfg16.with_(hadamard_n=0)
    q = u.rht_quantize(x, u.ALONG_COLS, cfg16)
    y = torch.empty_like(x)
    t_fused = _timed(lambda: u.rht_quantize(x, u.ALONG_COLS, cfg16, out=q), flush)
    t_plain = _timed(lambda: u.rht_quantize(x, u.ALONG_COLS, cfg0, out=q), flush)
    t_rht = _timed(lambda: u.rht_bf16(x, 16, out=y), flush)
    u.rht_bf16(x, 16, out=y)
    t_q_rot = _timed(lambda: u.rht_quantize(y, u.ALONG_COLS, cfg0, out=q), flush)
    t_unfused = t_rht + t_q_rot
    del y, q
    return {"tensor": list(x.shape), "quantize_only_ms": round(t_plain, 4), "fused_rht16_ms": round(t_fused, 4),
            "rht_pass_ms": round(t_rht, 4), "quantize_of_rotated_ms": round(t_q_rot, 4),
            "unfused_ms": round(t_unfused, 4),
            "fused_over_quantize_only": round(t_fused / t_plain, 3),
            "unfused_over_quantize_only": round(t_unfused / t_plain, 3),
            "pages": "fused ~1.06-1.07x, unfused ~1.4-1.6x of standalone quantization (SM90/SM100, "
                     "shapes not stated; context only)"}


# ------------------------------------------------------------------ side measurements
def run_mx(step: LayerStep, reps: int = 3) -> dict:
    """The layer's FPROP with MX block scales (UE8M0, block 32): X and W are
    quantized by the dual calls, which also write the E4M3 element planes, and
    the GEMM runs the block-scaled FP8 MMA on CTA pairs.  Both timed with CUDA
    events (reported, not in `value`)."""
    u = step.u
    cfg = u.QuantConfig(grid=u.GRID_E1M2, hadamard_n=16, block=32, scale_fmt=u.SCALE_UE8M0)
    s = step.shape
    qx, qxr = u.rht_quantize_dual(step.X, cfg)
    qw, qwr = u.rht_quantize_dual(step.W, cfg)
    out = torch.empty((s.M, s.N), dtype=torch.float32, device=step.dev)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=step.dev)
    t_g = _timed(lambda: u.gemm_fprop(qx, qw, out), flush, reps=reps, warm=1)
    t_q = _timed(lambda: u.rht_quantize_dual(step.X, cfg, out=(qx, qxr)), flush, reps=reps, warm=1)
    del out, qx, qw, qxr, qwr, flush
    return {"fprop_ms": round(t_g, 4),
            "fprop_TFLOPs": round(2 * s.M * s.N * s.K / (t_g * 1e-3) / 1e12, 1),
            "quantize_X_dual_ms": round(t_q, 4),
            "kernel": "gemm_pair_kernel<3> (kind::mxf8f6f4 block32, E4M3 elements, UE8M0 factors)"}


def run_f32s(step: LayerStep, peaks: dict, reps: int = 3) -> dict:
    """The layer's FPROP with fp32 block scales (E1M2, RHT16, block 16): X and W
    quantized once (untimed), the GEMM on the fp32-scale kernel (per-block
    K = 16 partials in TMEM, s_a * s_b accumulated on the CUDA cores), timed
    with CUDA events; reported beside the bf16 rate (not in `value`)."""
    u = step.u
    cfg = u.QuantConfig(grid=u.GRID_E1M2, hadamard_n=16, block=16, scale_fmt=u.SCALE_FP32)
    s = step.shape
    qx = u.rht_quantize(step.X, u.ALONG_COLS, cfg)
    qw = u.rht_quantize(step.W, u.ALONG_COLS, cfg)
    out = torch.empty((s.M, s.N), dtype=torch.float32, device=step.dev)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=step.dev)
    t_g = _timed(lambda: u.gemm_fprop(qx, qw, out), flush, reps=reps, warm=1)
    del out, qx, qw, flush
    tf = 2 * s.M * s.N * s.K / (t_g * 1e-3) / 1e12
    bf16 = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    return {"fprop_ms": round(t_g, 4), "fprop_TFLOPs": round(tf, 1),
            "frac_of_bf16": round(tf / bf16, 4),
            "kernel": "gemm_f32s_kernel (fp16-expanded codes, K = 16 kind::f16 partials, s_a * s_b * partial accumulated in fp32 registers)"}


def run_moe(device, two_level: bool, reps: int = 10):
    """The grouped (mixture-of-experts) GEMMs of one expert FFN: 16384 tokens,
    top-6 of 64 experts (Zipf(1.2) counts, segments padded to 64 rows), hidden
    2048, FFN 1408.  Operands are quantized once (untimed); the three grouped
    GEMMs are timed with CUDA events over `reps` launches each."""
    from fp4_quantized_gemms_b200 import ufp4
    shp = wl.MOE
    counts = wl.moe_expert_counts(shp)
    starts, padded, total = wl.padded_offsets(counts, 64)
    E, Hd, F = shp.experts, shp.hidden, shp.ffn
    rng_rows = np.zeros(total, dtype=bool)
    for s0, c in zip(starts, counts):
        rng_rows[s0:s0 + c] = True

    def routed(cols, std, seed):
        a = wl.normal(total, cols, std, seed)
        a[~rng_rows] = 0
        return to_dev(a, device)

    fmt = ufp4.SCALE_E4M3_X_FP32 if two_level else ufp4.SCALE_FP32
    rt = ufp4.QuantConfig(grid=ufp4.GRID_E1M2, hadamard_n=16, block=16, scale_fmt=fmt)
    sr0 = rt.with_(rounding=ufp4.ROUND_SR, sr_seed=SR_SEED, sr_stream=0)
    sr1 = rt.with_(rounding=ufp4.ROUND_SR, sr_seed=SR_SEED, sr_stream=1)
    C, R = ufp4.ALONG_COLS, ufp4.ALONG_ROWS
    X = routed(Hd, 1.0, 1)
    dY = routed(Hd, 1e-3, 3)
    H = routed(F, 1.0, 5)
    Wgu = to_dev(wl.normal(E * 2 * F, Hd, 0.02, 2), device)
    Wd = to_dev(wl.normal(E * Hd, F, 0.02, 4), device)
    q = ufp4.rht_quantize
    jobs = {
        "fprop_gate_up": (q(X, C, rt), q(Wgu, C, rt),
                          [(counts[e], 2 * F, Hd, starts[e], 0, e * 2 * F, 0, starts[e], 0) for e in range(E)],
                          (total, 2 * F)),
        "dgrad_down": (q(dY, C, sr0), q(Wd, R, rt),
                       [(counts[e], F, Hd, starts[e], 0, 0, e * Hd, starts[e], 0) for e in range(E)],
                       (total, F)),
        "wgrad_down": (q(dY, R, sr1), q(H, R, rt),
                       [(Hd, F, padded[e], 0, starts[e], 0, starts[e], e * Hd, 0) for e in range(E)],
                       (E * Hd, F)),
    }
    out = {}
    for name, (qa, qb, groups, oshape) in jobs.items():
        g = torch.tensor(np.array(groups, dtype=np.int64), device=device)
        c = torch.empty(oshape, dtype=torch.float32, device=device)
        flops = sum(2 * m * n * k for (m, n, k, *_r) in groups)
        for _ in range(3):
            ufp4.grouped_gemm(qa, qb, g, c)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(device)
        e0.record()
        for _ in range(reps):
            ufp4.grouped_gemm(qa, qb, g, c)
        e1.record()
        torch.cuda.synchronize(device)
        ms = e0.elapsed_time(e1) / reps
        out[name] = {"ms": round(ms, 4), "TFLOPs": round(flops / (ms * 1e-3) / 1e12, 1),
                     "GFLOP": round(flops / 1e9, 1)}
    if ufp4.check_device_status() != ufp4.OK:
        raise RuntimeError("device error word set in the MoE measurement")
    out["workload"] = ("16384 tokens, top-6 of 64 experts (Zipf 1.2 counts, 64-row padded segments), "
                       "hidden 2048, FFN 1408; grouped GEMMs over a device group table")
    return out


def _occupancy(code_count, grid: int) -> dict:
    """Code-occupancy histogram (share of elements per magnitude code, both
    signs) and its entropy in bits, beside the bucket ratio."""
    mags = [code_count[k] + (code_count[8 + k] if k else 0) for k in range(8)]
    tot = float(sum(mags)) or 1.0
    p = [m / tot for m in mags]
    ent = -sum(q * math.log2(q) for q in p if q > 0)
    return {"magnitude_share": [round(q, 5) for q in p], "entropy_bits": round(ent, 4)}


def run_diag(step: LayerStep, reps: int = 5) -> dict:
    """Diagnostics of the step's six operands (SQNR, bucket ratio, code
    occupancy, underflow ratio from ufp4_quant_stats) and the time of the two
    diagnostics kernels on the largest tensors: quant_stats of dY^T and the
    GEMM-output SQNR sums of Y against a copy of it (both read from HBM)."""
    u = step.u
    C, R = u.ALONG_COLS, u.ALONG_ROWS
    out = {}
    for name, x, axis, q in (("X", step.X, C, step.qx), ("W", step.W, C, step.qw),
                             ("dY", step.dY, C, step.qdy), ("dY^T", step.dY, R, step.qdyt),
                             ("W^T", step.W, R, step.qwt), ("X^T", step.X, R, step.qxt)):
        st = u.quant_stats(x, axis, q)
        out[name] = {"sqnr_db": round(st["sqnr_db"], 3), "bucket_ratio": round(st["bucket_ratio"], 4),
                     "underflow_ratio": round(st["underflow_ratio"], 5),
                     **_occupancy(st["code_count"], q.cfg.grid)}
    buf = torch.zeros(64, dtype=torch.float64, device=step.dev)
    sums = torch.zeros(2, dtype=torch.float64, device=step.dev)
    ref = step.Y
    test = step.Y.clone()
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=step.dev)
    t_stats = _timed(lambda: u.quant_stats_launch(step.dY, R, step.qdyt, out=buf), flush, reps=reps)
    t_sqnr = _timed(lambda: u.sqnr_sums(ref, test, out=sums), flush, reps=reps)
    n = step.dY.numel()
    per = 2 + 0.5 + (1 / 16 if step.two else 4 / 16)
    out["quant_stats_dYT"] = {"ms": round(t_stats, 4), "GBps": round(n * per / (t_stats * 1e-3) / 1e9, 1),
                              "bytes_per_element": per}
    m = ref.numel()
    out["sqnr_sums_Y"] = {"ms": round(t_sqnr, 4), "GBps": round(m * 8 / (t_sqnr * 1e-3) / 1e9, 1)}
    del test, flush
    return out


def run_e2e(step: LayerStep, host_inputs, args, device):
    """Same step through the public API with HOST inputs and outputs, the way
    a training loop streams batches: every step copies X, W, dY in from
    pinned host memory and Y, dX, dW back out, all inside the timed region.
    Copies run on their own streams (host-to-device and device-to-host use
    separate copy engines) and overlap the compute of neighbouring steps:
    inputs and outputs are double-buffered on the device, an input set is
    refilled once its step's quantization is done (the GEMMs read only the
    quantized operands), an output set is rewritten once its copies out have
    landed, and each GEMM's output leaves as soon as that GEMM ends."""
    s = step.shape
    X, W, dY = host_inputs
    hX = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).pin_memory()
    hW = torch.from_numpy(W.view(np.int16)).view(torch.bfloat16).pin_memory()
    hdY = torch.from_numpy(dY.view(np.int16)).view(torch.bfloat16).pin_memory()
    hY = torch.empty(step.Y.shape, dtype=torch.float32).pin_memory()
    hdX = torch.empty(step.dX.shape, dtype=torch.float32).pin_memory()
    hdW = torch.empty(step.dW.shape, dtype=torch.float32).pin_memory()
    h2d = (hX.numel() + hW.numel() + hdY.numel()) * 2
    d2h = (hY.numel() + hdX.numel() + hdW.numel()) * 4
    u = step.u
    comp = torch.cuda.current_stream(device)
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ins = [(step.X, step.W, step.dY), tuple(torch.empty_like(t) for t in (step.X, step.W, step.dY))]
    outs = [(step.Y, step.dX, step.dW), tuple(torch.empty_like(t) for t in (step.Y, step.dX, step.dW))]
    q_done = [None, None]     # quantization of the last step that read input set b
    out_free = [None, None]   # copies out of the last step that wrote output set b

    def ev(stream):
        e = torch.cuda.Event()
        e.record(stream)
        return e

    def h2d_issue(i, start=None):
        b = i % 2
        with torch.cuda.stream(s_in):
            if start is not None:
                s_in.wait_event(start)
            if q_done[b] is not None:
                s_in.wait_event(q_done[b])
            for dst, src in zip(ins[b], (hX, hW, hdY)):
                dst.copy_(src, non_blocking=True)
            return ev(s_in)

    def compute(i, landed):
        b = i % 2
        comp.wait_event(landed)
        if out_free[b] is not None:
            comp.wait_event(out_free[b])
        step.bind(*ins[b], *outs[b])
        step.quantize_all()
        q_done[b] = ev(comp)
        Yb, dXb, dWb = outs[b]
        for fn, qa, qb, dev_out, host_out in ((u.gemm_fprop, step.qx, step.qw, Yb, hY),
                                              (u.gemm_dgrad, step.qdy, step.qwt, dXb, hdX),
                                              (u.gemm_wgrad, step.qdyt, step.qxt, dWb, hdW)):
            fn(qa, qb, out=dev_out)
            done = ev(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done)
                host_out.copy_(dev_out, non_blocking=True)
        out_free[b] = ev(s_out)

    def run(n, start=None):
        landed = h2d_issue(0, start)
        for i in range(n):
            nxt = h2d_issue(i + 1) if i + 1 < n else None
            compute(i, landed)
            landed = nxt
        comp.wait_event(out_free[(n - 1) % 2])

    run(max(1, min(args.warmup, 3)))
    torch.cuda.synchronize(device)
    n = max(2, min(args.steps, 8))
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(comp)
    run(n, start=a)
    b.record(comp)
    torch.cuda.synchronize(device)
    step.bind(*ins[0], *outs[0])
    ms = a.elapsed_time(b) / n
    flops = 3 * 2 * s.M * s.N * s.K
    return {"value": round(flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": n, "pipelined": "copies in and out on their own streams, overlapping neighbouring steps"}


# DRAM bytes (read + write) per launch of the large layer's three GEMMs with
# two-level E1M2 operands, from one ncu capture of the bench's own launches
# (dram__bytes_read.sum + dram__bytes_write.sum, a one-pass metric set): the
# CTA-pair kernel with factor atoms and the banded tile order.  Valid only for
# that kernel and workload; re-capture when either changes.
LARGE_E1M2_GEMM_DRAM_BYTES = {"fprop": 2.890e9 + 1.855e9, "dgrad": 5.663e9 + 0.524e9, "wgrad": 5.115e9 + 0.924e9}


def gemm_roofline(g_ms, shape, peaks, peak_kind, two: bool, grid: int) -> dict:
    """Roofline of the dominant (slowest) GEMM of a step: useful flops 2MNK
    over its CUDA-event time, against the peak of the MMA kind it runs on."""
    s = shape
    tf = [2 * s.M * s.N * s.K / (g * 1e-3) / 1e12 for g in g_ms]
    dom = int(np.argmax(g_ms))
    # the GEMMs are timed inside a long step loop under the power cap: the
    # sustained bf16 figure is the denominator
    bf16 = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    if two:
        peak = bf16 * FP4_OVER_BF16
        kern = ("gemm_pair_kernel (CTA pairs, 256x256 tiles, factor atoms copied by tcgen05.cp), "
                "tcgen05.mma kind::mxf4nvf4.block_scale.block16"
                + (" (E1M2 as two E2M1 planes: four MMAs per K step)" if grid == 0 else ""))
        src = f"{peak_kind} sustained bf16 dense x 4 (nominal fp4 / bf16 dense ratio)"
    else:
        peak = bf16
        kern = "gemm_f32s_kernel, tcgen05.mma kind::f16 (fp16 operands, fp32 block-scale accumulate)"
        src = f"{peak_kind} sustained bf16 dense (fp16 runs at the bf16 rate)"
    r = {"kernel": f"{kern} ({('fprop', 'dgrad', 'wgrad')[dom]})", "bound": "tensor",
         "achieved": round(tf[dom], 1), "peak": round(peak, 1), "unit": "TFLOP/s",
         "frac": round(tf[dom] / peak, 4), "traffic": None, "peak_source": src,
         "achieved_is": "useful flops 2MNK / CUDA-event time of the dominant GEMM"}
    if two and grid == 0:
        r["frac_of_bf16_rate_ceiling"] = round(tf[dom] / bf16, 4)
        r["ceiling_note"] = ("an exact E1M2 product needs four FP4 MMAs per K step (no native uniform-grid "
                             "kind), so its ceiling is the FP4 rate / 4 = the bf16 rate")
        r["issued_fp4_TFLOPs"] = round(4 * tf[dom], 1)
    name = ("fprop", "dgrad", "wgrad")[dom]
    if two and grid == 0 and shape is wl.LARGE:
        r["traffic"] = LARGE_E1M2_GEMM_DRAM_BYTES[name]
        r["traffic_note"] = ("DRAM bytes read + written per launch from one ncu capture of these launches at "
                             "full size; algorithmic bytes (operands + output) are 2.30 / 1.03 / 1.61 GB for "
                             "FPROP / DGRAD / WGRAD")
    else:
        r["traffic_note"] = "null: no capture of this kernel at this size"
    return r


def run_device(args, rank, world, device):
    from fp4_quantized_gemms_b200 import ufp4
    peaks, peak_kind = load_peaks()
    shape = SHAPES[args.workload]
    s = shape
    flops = 3 * 2 * s.M * s.N * s.K
    host = wl.layer_inputs(shape)
    dev_inputs = tuple(to_dev(b, device) for b in host)
    step = LayerStep(device, args.scale, shape, dev_inputs)
    ms_per_step, q_ms, g_ms, clk = time_steps(step, args.steps, args.warmup, world, device, clocks=True)
    status = ufp4.check_device_status()
    value = job_tflops(world, flops, ms_per_step)
    qbytes = quant_bytes(step)
    q_gbs = qbytes / (q_ms * 1e-3) / 1e9
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    gemm_tf = [2 * s.M * s.N * s.K / (g * 1e-3) / 1e12 for g in g_ms]
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("e1m2 codes as two e2m1 planes (ue4m3 block-16 factors), fp32 accumulate"
                  if step.two else "e1m2 codes, fp16 tensor-core operands, fp32 accumulate"),
        "data": "synthetic (seeded PCG64 inputs of the workload's shapes and distributions)",
        "config": {**workload_desc(shape, args.scale), "parallelism": f"replicas x{world}"},
        "gpu_launches": step.launches * args.steps,
        "kernels": {
            "quantize_all_ms": round(q_ms, 4),
            "quantize_GBps": round(q_gbs, 1),
            "quantize_frac_of_8TBps": round(q_gbs / HBM_SPEC_GBS, 4),
            "quantize_frac_of_measured_hbm": round(q_gbs / hbm, 4),
            "gemm_ms": {k: round(v, 4) for k, v in zip(("fprop", "dgrad", "wgrad"), g_ms)},
            "gemm_TFLOPs": {k: round(v, 1) for k, v in zip(("fprop", "dgrad", "wgrad"), gemm_tf)},
        },
        "roofline": gemm_roofline(g_ms, shape, peaks, peak_kind, step.two, step.grid),
        "device_status": ufp4.status_string(status),
        "clocks": clk,
    }
    if rank == 0 and not args.quick:
        result["diagnostics"] = run_diag(step)
        result["mx_block32"] = run_mx(step)
        result["fp32_scales"] = run_f32s(step, peaks)
    result["e2e"] = run_e2e(step, host, args, device)
    step.free()
    del step
    torch.cuda.empty_cache()
    if not args.quick:
        # the E2M1 baseline grid of the same layer, RTNE on every operand
        b = LayerStep(device, args.scale, shape, dev_inputs, grid=ufp4.GRID_E2M1)
        ms_b, q_b, g_b, _ = time_steps(b, max(3, args.steps // 4), 3, 1, device, clocks=False)
        result["e2m1_baseline"] = {
            "recipe": "E2M1 grid, RTNE on X, W and dY, RHT16, block 16, two-level scales",
            "ms_per_step": round(ms_b, 4), "value": round(flops / (ms_b * 1e-3) / 1e12, 2),
            "quantize_all_ms": round(q_b, 4),
            "gemm_TFLOPs": {k: round(2 * s.M * s.N * s.K / (g * 1e-3) / 1e12, 1)
                            for k, g in zip(("fprop", "dgrad", "wgrad"), g_b)},
            "roofline": gemm_roofline(g_b, shape, peaks, peak_kind, b.two, b.grid),
        }
        b.free()
        del b
        torch.cuda.empty_cache()
    del dev_inputs
    torch.cuda.empty_cache()
    if rank == 0 and not args.quick:
        result["moe_grouped"] = run_moe(device, args.scale == "two-level")
        result["quantize_sweep"] = run_sweep(device, peaks)
    if ufp4.check_device_status() != ufp4.OK:
        raise RuntimeError("device error word set")
    return result


# ------------------------------------------------------------------ oracle arm
class OracleSample:
    """The oracle as it stands, on the host cores, in the GPU arm's
    configuration (`scale`): it quantizes sampled output rows of every operand
    (full reduction length) and contracts a sampled block of each GEMM.  The
    inputs and, with two-level scales, the six rotated tensor amaxes are
    prepared once, outside any timed region."""

    MASK = 0x09F1FD9D03F0A9B4       # the binding's default D sign mask

    def __init__(self, scale: str, shape):
        import oracle
        self.oracle = oracle
        oracle.build()
        self.shape = shape
        self.X, self.W, self.dY = wl.layer_inputs(shape)
        self.two = scale == "two-level"
        fmt = oracle.SCALE_E4M3_X_FP32 if self.two else oracle.SCALE_FP32
        base = dict(grid=0, hadamard_n=16, block=16, sign_mask=self.MASK, scale_fmt=fmt)
        self.rt = oracle.QuantCfg(**base)
        self.sr0 = oracle.QuantCfg(rounding=1, sr_seed=SR_SEED, sr_stream=0, **base)
        self.sr1 = oracle.QuantCfg(rounding=1, sr_seed=SR_SEED, sr_stream=1, **base)
        self.amax = {}
        for name, bits in (("X", self.X), ("W", self.W), ("dY", self.dY)):
            for ax in (0, 1):
                self.amax[name, ax] = oracle.rht_amax(bits, ax, 16, self.MASK) if self.two else 0.0

    def step(self, rng, n_rows: int, n_cols: int):
        """One sampled step: returns (elements quantized, quantize seconds,
        GEMM flops of the sampled entries, GEMM seconds)."""
        oracle = self.oracle
        s = self.shape
        gemms = [(("X", 0, self.rt, s.M), ("W", 0, self.rt, s.N), s.K),
                 (("dY", 0, self.sr0, s.M), ("W", 1, self.rt, s.K), s.N),
                 (("dY", 1, self.sr1, s.N), ("X", 1, self.rt, s.K), s.M)]
        bits = {"X": self.X, "W": self.W, "dY": self.dY}

        def rows_q(name, ax, cfg, picks):
            parts = [oracle.quantize(bits[name], ax, cfg, tensor_amax=self.amax[name, ax], r0=int(r), nr=1)
                     for r in picks]
            q = parts[0]
            q.codes = np.concatenate([p.codes for p in parts])
            if q.scales is not None:
                q.scales = np.concatenate([p.scales for p in parts])
            else:
                q.escales = np.concatenate([p.escales for p in parts])
            return q

        elems = flops = 0.0
        tq = tg = 0.0
        for (an, aax, acfg, arows), (bn, bax, bcfg, brows), K in gemms:
            t0 = time.perf_counter()
            qa = rows_q(an, aax, acfg, rng.choice(arows, n_rows, replace=False))
            qb = rows_q(bn, bax, bcfg, rng.choice(brows, n_cols, replace=False))
            t1 = time.perf_counter()
            ii = np.repeat(np.arange(n_rows), n_cols)
            jj = np.tile(np.arange(n_cols), n_rows)
            out = oracle.gemm_tn_entries(qa, qb, ii, jj)
            t2 = time.perf_counter()
            elems += (n_rows + n_cols) * K
            flops += 2.0 * K * out.size
            tq += t1 - t0
            tg += t2 - t1
        return elems, tq, flops, tg


def oracle_rates(smp: OracleSample, rng, budget_s: float, n_rows: int, n_cols: int, max_steps: int):
    """Runs sampled steps until `budget_s` of CPU work; returns the oracle's
    quantize rate (elements/s), GEMM rate (flop/s), the steps run and the
    seconds spent."""
    E = Q = F = G = 0.0
    n = 0
    while (Q + G) < budget_s and n < max_steps:
        e, q, f, g = smp.step(rng, n_rows, n_cols)
        E, Q, F, G = E + e, Q + q, F + f, G + g
        n += 1
    return E / Q, F / G, n, Q + G


def oracle_step_figures(shape, two: bool, q_rate: float, g_rate: float) -> dict:
    """The oracle's whole-step throughput in the GPU arm's unit, from its
    measured rates: a step quantizes every operand in full (2 (MK + NK + MN)
    elements) and contracts the three GEMMs (3 * 2MNK flops)."""
    s = shape
    elems = 2 * (s.M * s.K + s.N * s.K + s.M * s.N)
    flops = 3 * 2 * s.M * s.N * s.K
    t = elems / q_rate + flops / g_rate
    per = 2.5 + (1 / 16 if two else 4 / 16)
    return {"step_s": t, "value": flops / t / 1e12,
            "quantize_GBps": q_rate * per / 1e9, "gemm_GFLOPs": g_rate / 1e9}


def run_reference(args, world):
    shape = SHAPES[args.workload]
    smp = OracleSample(args.scale, shape)       # inputs and tensor amaxes outside the timed region
    rng = np.random.default_rng(0)
    for _ in range(args.warmup):
        smp.step(rng, 2, 2)
    cores = smp.oracle.num_threads()
    n_rows = max(2, min(16, cores))
    times = []
    Eq = Tq = Fg = Tg = 0.0
    for _ in range(args.steps):
        e, q, f, g = smp.step(rng, n_rows, n_rows)
        Eq, Tq, Fg, Tg = Eq + e, Tq + q, Fg + f, Tg + g
        times.append(q + g)
    fig = oracle_step_figures(shape, smp.two, Eq / Tq, Fg / Tg)
    sample = (f"per step: {n_rows} sampled output rows of each of the 6 quantized operands "
              f"(full reduction length) and the {n_rows}x{n_rows} sampled block of each GEMM; "
              "value = full-step flops / (elements of a step / measured quantize rate + flops of a step / "
              "measured GEMM rate)" + ("; the rotated tensor amaxes are computed once before the timed steps"
                                       if smp.two else ""))
    value = fig["value"]
    res = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": fig["step_s"] * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 oracle (fp32 RHT, exact rounding decisions)", "data": "synthetic",
        "config": {**workload_desc(shape, args.scale), "parallelism": f"replicas x{world}"},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample, "quantize_GBps": round(fig["quantize_GBps"], 4),
                         "gemm_GFLOPs": round(fig["gemm_GFLOPs"], 3),
                         "sampled_wall_s": round(sum(times), 3)},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return res


def cpu_baseline(scale: str, shape, budget_s: float = 10.0) -> dict:
    """The oracle as it stands on the host cores (rank 0), in the GPU arm's
    configuration: quantize GB/s on sampled full-K rows of the large layer's
    six operands, GEMM GFLOP/s on the sampled entries of its three GEMMs, the
    full tiny FPROP as a second GEMM figure, and the modeled whole-step
    throughput in the GPU arm's unit."""
    import oracle
    smp = OracleSample(scale, shape)
    cores = smp.oracle.num_threads()
    rng = np.random.default_rng(1)
    smp.step(rng, 2, 2)                     # warm caches / page in
    n_rows = max(8, 2 * cores)
    q_rate, g_rate, n, secs = oracle_rates(smp, rng, budget_s, n_rows, n_rows, 50)
    fig = oracle_step_figures(shape, smp.two, q_rate, g_rate)
    # the tiny FPROP in full (256 x 512 x 512)
    t = wl.TINY
    X, W, _ = wl.layer_inputs(t, want_dy=False, cache=False)
    cfg = oracle.QuantCfg(grid=0, hadamard_n=16, block=16, sign_mask=OracleSample.MASK)
    t0 = time.perf_counter()
    qa = oracle.quantize(X, 0, cfg)
    qb = oracle.quantize(W, 0, cfg)
    t1 = time.perf_counter()
    oracle.gemm_tn(qa, qb)
    t2 = time.perf_counter()
    tiny_gflops = 2 * t.M * t.N * t.K / (t2 - t1) / 1e9
    # the quantizer sweep's largest tensor (32768 x 16384 ~0.1 Student-t(4)),
    # recipe configuration (E1M2 RTNE, n 16, block 16, fp32 scales): full-K
    # rows quantized along the columns (rows are independent with fp32 scales)
    sweep_rows = min(4096, 256 * cores)
    Xs = wl.student_t(sweep_rows, 16384, seed=5)
    t3 = time.perf_counter()
    oracle.quantize(Xs, 0, oracle.QuantCfg(grid=0, hadamard_n=16, block=16, sign_mask=OracleSample.MASK))
    t4 = time.perf_counter()
    sweep_gbps = sweep_rows * 16384 * (2 + 0.5 + 4 / 16) / (t4 - t3) / 1e9
    return {"value": fig["value"], "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": (f"{n} sampled steps of the large layer ({secs:.1f} s of CPU work): {n_rows} output rows "
                       f"of each of the 6 quantized operands (full K) and a {n_rows}x{n_rows} block of each "
                       "GEMM; value = full-step flops / (step elements / quantize rate + step flops / GEMM rate)"
                       + ("; tensor amaxes computed before timing" if smp.two else "")),
            "quantize_GBps": round(fig["quantize_GBps"], 4),
            "gemm_GFLOPs": round(fig["gemm_GFLOPs"], 3),
            "tiny_fprop_full": {"shape": [t.M, t.K, t.N], "gemm_GFLOPs": round(tiny_gflops, 3),
                                "quantize_ms": round((t1 - t0) * 1e3, 2)},
            "quantize_sweep_tensor": {"shape": [32768, 16384], "sample_rows": sweep_rows,
                                      "recipe": "E1M2 RTNE, RHT16, block 16, fp32 scales, along columns",
                                      "GBps": round(sweep_gbps, 4), "seconds": round(t4 - t3, 2)}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ufp4", choices=["ufp4", "reference"])
    ap.add_argument("--scale", default="two-level", choices=["two-level", "fp32"])
    ap.add_argument("--workload", default="large", choices=sorted(SHAPES))
    ap.add_argument("--quick", action="store_true", help="the timed step and e2e only")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return

    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from fp4_quantized_gemms_b200 import build as ufp4_build
    ufp4_build.build()
    res = run_device(args, rank, world, device)
    if rank == 0:
        if not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(args.scale, SHAPES[args.workload])
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
