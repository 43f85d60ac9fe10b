"""CPU oracle of the UFP4 quantize + GEMM hot path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  It shares no
code with the CUDA library; the two meet only in the seeded input generators
(``fp4_quantized_gemms_b200.workloads``), which hold none of the method's
arithmetic.

The arithmetic lives in plain C (``ufp4_oracle.c``, built with
``-O2 -ffp-contract=off -fno-fast-math``); this module only marshals numpy
arrays.  Every function cites its source section in the C file.

Pinned by ``tests/test_oracle_pins.py`` (closed forms, invariants, brute force,
library routines).  One function is "parity unpinned" against an external
source on the CPU: the Philox4x32-10 stream (see ``philox4x32_10``), which a
GPU test pins against cuRAND's independent implementation.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ufp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libufp4_oracle.so")

GRID_E1M2, GRID_E2M1, GRID_E2M1_MAX2 = 0, 1, 2
ROUND_RTNE, ROUND_SR = 0, 1
SCALE_FP32, SCALE_E4M3_X_FP32, SCALE_UE8M0 = 0, 1, 2
ALONG_COLS, ALONG_ROWS = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle shared library in place (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= max(os.path.getmtime(_SRC),
                                                   os.path.getmtime(_SRC[:-2] + ".h"))):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-std=c11",
           "-Wall", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Cfg(ctypes.Structure):
    _fields_ = [("grid", ctypes.c_int), ("rounding", ctypes.c_int),
                ("sr_seed", ctypes.c_uint64), ("sr_stream", ctypes.c_uint32),
                ("hadamard_n", ctypes.c_int), ("sign_mask", ctypes.c_uint64),
                ("block", ctypes.c_int), ("scale_fmt", ctypes.c_int)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i64, u64, u32, i32 = ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int
        L.uo_level.restype = ctypes.c_double
        L.uo_level.argtypes = [i32, i32]
        L.uo_gmax.restype = ctypes.c_double
        L.uo_ue8m0_scale.restype = ctypes.c_uint8
        L.uo_ue8m0_scale.argtypes = [i32, ctypes.c_float]
        L.uo_ue8m0_value.restype = ctypes.c_double
        L.uo_ue8m0_value.argtypes = [ctypes.c_uint8]
        L.uo_gmax.argtypes = [i32]
        L.uo_top_code.restype = i32
        L.uo_top_code.argtypes = [i32]
        L.uo_fwht_f32.argtypes = [P, i32]
        L.uo_fwht_f64.argtypes = [P, i32]
        L.uo_e4m3_rne_satfinite.restype = ctypes.c_uint8
        L.uo_e4m3_rne_satfinite.argtypes = [ctypes.c_float]
        L.uo_e4m3_value.restype = ctypes.c_double
        L.uo_e4m3_value.argtypes = [ctypes.c_uint8]
        L.uo_philox4x32_10.argtypes = [P, P, P]
        L.uo_sr_u16.restype = u32
        L.uo_sr_u16.argtypes = [u64, u32, u64]
        L.uo_round_rtne.restype = i32
        L.uo_round_rtne.argtypes = [i32, ctypes.c_double, ctypes.c_double]
        L.uo_round_sr.restype = i32
        L.uo_round_sr.argtypes = [i32, ctypes.c_double, ctypes.c_double, u32]
        L.uo_tensor_scale.restype = ctypes.c_float
        L.uo_tensor_scale.argtypes = [i32, ctypes.c_float]
        L.uo_block_decode_base.restype = ctypes.c_float
        L.uo_block_decode_base.argtypes = [i32, ctypes.c_float]
        L.uo_kpad.restype = i64
        L.uo_kpad.argtypes = [i64]
        L.uo_rht_amax.restype = ctypes.c_float
        L.uo_rht_amax.argtypes = [P, i64, i64, i64, i32, i32, u64]
        L.uo_quantize.restype = i32
        L.uo_quantize.argtypes = [P, i64, i64, i64, i32, ctypes.POINTER(_Cfg), ctypes.c_float,
                                  i64, i64, P, P, P, P, P]
        L.uo_dequantize.argtypes = [P, P, P, ctypes.c_float, i64, i64, i32, i32, i32, P]
        L.uo_gemm_tn_f64.argtypes = [P, P, i64, i64, i64, ctypes.c_double, P, i64]
        L.uo_gemm_tn_f64_entries.argtypes = [P, P, i64, ctypes.c_double, P, P, i64, P]
        L.uo_num_threads.restype = i32
        L.uo_e4m3_rne_satfinite_array.argtypes = [P, i64, P]
        L.uo_sr_u16_array.argtypes = [u64, u32, P, i64, P]
        L.uo_sr_u16_seeds.argtypes = [P, i64, u32, u64, P]
        L.uo_round_rtne_array.argtypes = [i32, P, ctypes.c_double, i64, P]
        L.uo_round_sr_array.argtypes = [i32, P, ctypes.c_double, P, i64, P]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- scalars
def level(grid: int, k: int) -> float:
    return lib().uo_level(grid, k)


def top_code(grid: int) -> int:
    """Largest magnitude code the grid uses (7; 4 for E2M1 with max 2.0)."""
    return int(lib().uo_top_code(grid))


def levels(grid: int) -> np.ndarray:
    """Magnitudes of codes 0 .. top_code(grid), indexed by code."""
    return np.array([level(grid, k) for k in range(top_code(grid) + 1)])


def gmax(grid: int) -> float:
    return lib().uo_gmax(grid)


def ue8m0_scale(grid: int, amax: float) -> int:
    """MX block-scale byte (biased exponent) of a block maximum."""
    return int(lib().uo_ue8m0_scale(grid, float(np.float32(amax))))


def ue8m0_value(e: int) -> float:
    return lib().uo_ue8m0_value(e)


def kpad(k: int) -> int:
    return int(lib().uo_kpad(k))


def num_threads() -> int:
    return int(lib().uo_num_threads())


def fwht_f32(v: np.ndarray) -> np.ndarray:
    out = np.ascontiguousarray(v, dtype=np.float32).copy()
    lib().uo_fwht_f32(_p(out), out.size)
    return out


def fwht_f64(v: np.ndarray) -> np.ndarray:
    out = np.ascontiguousarray(v, dtype=np.float64).copy()
    lib().uo_fwht_f64(_p(out), out.size)
    return out


def e4m3(x) -> np.ndarray:
    xa = np.ascontiguousarray(np.atleast_1d(x), dtype=np.float32)
    out = np.empty(xa.size, dtype=np.uint8)
    lib().uo_e4m3_rne_satfinite_array(_p(xa), xa.size, _p(out))
    return out


def e4m3_value(b: int) -> float:
    return lib().uo_e4m3_value(int(b))


def philox4x32_10(ctr, key) -> np.ndarray:
    """Philox4x32-10 block function.  Parity unpinned on the CPU against an
    external source (no published known-answer vectors are in this tree); the
    GPU test pins it against cuRAND's Philox4_32_10."""
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.empty(4, dtype=np.uint32)
    lib().uo_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def sr_u16(seed: int, stream: int, L) -> np.ndarray:
    La = np.ascontiguousarray(np.atleast_1d(L), dtype=np.uint64)
    out = np.empty(La.size, dtype=np.uint32)
    lib().uo_sr_u16_array(seed, stream, _p(La), La.size, _p(out))
    return out


def sr_u16_over_seeds(seeds, stream: int, L: int) -> np.ndarray:
    sa = np.ascontiguousarray(seeds, dtype=np.uint64)
    out = np.empty(sa.size, dtype=np.uint32)
    lib().uo_sr_u16_seeds(_p(sa), sa.size, stream, L, _p(out))
    return out


def round_rtne(grid: int, au, s: float) -> np.ndarray:
    a = np.ascontiguousarray(np.atleast_1d(au), dtype=np.float64)
    out = np.empty(a.size, dtype=np.int32)
    lib().uo_round_rtne_array(grid, _p(a), float(s), a.size, _p(out))
    return out


def round_sr(grid: int, au, s: float, r16) -> np.ndarray:
    a = np.ascontiguousarray(np.atleast_1d(au), dtype=np.float64)
    r = np.ascontiguousarray(np.broadcast_to(np.atleast_1d(r16), a.shape), dtype=np.uint32)
    out = np.empty(a.size, dtype=np.int32)
    lib().uo_round_sr_array(grid, _p(a), float(s), _p(r), a.size, _p(out))
    return out


def tensor_scale(grid: int, amax_t: float) -> float:
    return float(lib().uo_tensor_scale(grid, amax_t))


def block_decode_base(grid: int, S: float) -> float:
    return float(lib().uo_block_decode_base(grid, S))


# ---------------------------------------------------------------- operands
@dataclass
class QuantCfg:
    grid: int = GRID_E1M2
    rounding: int = ROUND_RTNE
    sr_seed: int = 0
    sr_stream: int = 0
    hadamard_n: int = 16
    sign_mask: int = 0
    block: int = 16
    scale_fmt: int = SCALE_FP32

    def _c(self) -> _Cfg:
        return _Cfg(self.grid, self.rounding, self.sr_seed, self.sr_stream,
                    self.hadamard_n, self.sign_mask, self.block, self.scale_fmt)


@dataclass
class QTensor:
    """Logical (unpacked) quantized operand, K-major: ``codes[r][k]`` nibbles,
    ``scales[r][b]`` (fp32 mode) or ``escales[r][b]`` E4M3 bytes plus ``S``."""
    codes: np.ndarray
    scales: np.ndarray | None
    escales: np.ndarray | None
    S: float
    cfg: QuantCfg
    k: int
    kpad: int
    row0: int = 0

    def dequantize(self) -> np.ndarray:
        nr = self.codes.shape[0]
        out = np.empty((nr, self.kpad), dtype=np.float64)
        sc = self.scales if self.scales is not None else np.zeros(1, np.float32)
        es = self.escales if self.escales is not None else np.zeros(1, np.uint8)
        lib().uo_dequantize(_p(self.codes), _p(sc), _p(es), self.S, nr, self.kpad,
                            self.cfg.grid, self.cfg.block, self.cfg.scale_fmt, _p(out))
        return out


def _as_bf16_bits(x) -> np.ndarray:
    a = np.asarray(x)
    if a.dtype == np.uint16:
        return np.ascontiguousarray(a)
    raise TypeError("oracle inputs are bf16 bit patterns (uint16 arrays)")


def rht_amax(x, axis: int, hadamard_n: int, sign_mask: int) -> float:
    xb = _as_bf16_bits(x)
    rows, cols = xb.shape
    return float(lib().uo_rht_amax(_p(xb), rows, cols, cols, axis, hadamard_n, sign_mask))


def quantize(x, axis: int, cfg: QuantCfg, tensor_amax: float = 0.0,
             r0: int = 0, nr: int | None = None, want_u: bool = False):
    """Quantize output rows [r0, r0+nr) of the K-major view of bf16 ``x``.

    Returns a QTensor (and the rotated fp32 values when ``want_u``)."""
    xb = _as_bf16_bits(x)
    rows, cols = xb.shape
    K = cols if axis == ALONG_COLS else rows
    nout = rows if axis == ALONG_COLS else cols
    if nr is None:
        nr = nout - r0
    kp = kpad(K)
    nb = kp // cfg.block
    codes = np.zeros((nr, kp), dtype=np.int8)
    scales = np.zeros((nr, nb), dtype=np.float32)
    escales = np.zeros((nr, nb), dtype=np.uint8)
    S = np.zeros(1, dtype=np.float32)
    u = np.zeros((nr, kp), dtype=np.float32) if want_u else None
    c = cfg._c()
    rc = lib().uo_quantize(_p(xb), rows, cols, cols, axis, ctypes.byref(c), float(tensor_amax),
                           r0, nr, _p(codes), _p(scales), _p(escales), _p(S),
                           _p(u) if want_u else None)
    if rc != 0:
        raise ValueError(f"oracle quantize rejected the configuration (code {rc})")
    two = cfg.scale_fmt == SCALE_E4M3_X_FP32
    byte_scales = cfg.scale_fmt != SCALE_FP32      # E4M3 bytes, or UE8M0 exponent bytes
    q = QTensor(codes=codes, scales=None if byte_scales else scales,
                escales=escales if byte_scales else None,
                S=float(S[0]) if two else 1.0, cfg=cfg, k=K, kpad=kp, row0=r0)
    return (q, u) if want_u else q


def gemm_tn(a: QTensor, b: QTensor) -> np.ndarray:
    """C[i][j] = (1/n) sum_k deq(a)[i][k] deq(b)[j][k] in fp64 (full output)."""
    A = a.dequantize()
    B = b.dequantize()
    assert A.shape[1] == B.shape[1]
    M, K = A.shape
    N = B.shape[0]
    n = a.cfg.hadamard_n
    inv_n = 1.0 / n if n else 1.0
    C = np.empty((M, N), dtype=np.float64)
    lib().uo_gemm_tn_f64(_p(A), _p(B), M, N, K, inv_n, _p(C), N)
    return C


def gemm_dequantized(A: np.ndarray, B: np.ndarray, inv_n: float) -> np.ndarray:
    """C = inv_n * A B^T for dequantized fp64 operands (rows of A, B along K)."""
    A = np.ascontiguousarray(A, dtype=np.float64)
    B = np.ascontiguousarray(B, dtype=np.float64)
    M, K = A.shape
    N = B.shape[0]
    C = np.empty((M, N), dtype=np.float64)
    lib().uo_gemm_tn_f64(_p(A), _p(B), M, N, K, float(inv_n), _p(C), N)
    return C


def gemm_tn_entries(a: QTensor, b: QTensor, ii, jj) -> np.ndarray:
    """Selected entries; ``ii``/``jj`` index the rows held in ``a``/``b``."""
    A = a.dequantize()
    B = b.dequantize()
    ia = np.ascontiguousarray(ii, dtype=np.int64)
    ja = np.ascontiguousarray(jj, dtype=np.int64)
    out = np.empty(ia.size, dtype=np.float64)
    n = a.cfg.hadamard_n
    inv_n = 1.0 / n if n else 1.0
    lib().uo_gemm_tn_f64_entries(_p(A), _p(B), A.shape[1], inv_n, _p(ia), _p(ja), ia.size,
                                 _p(out))
    return out
