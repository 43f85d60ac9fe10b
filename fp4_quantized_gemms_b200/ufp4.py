"""Thin Python binding of libufp4.so (argument marshalling only).

Every function here maps one-to-one onto an ``extern "C"`` entry point of
``include/ufp4.h``; tensors are torch CUDA tensors (device memory and streams
come from PyTorch), results are computed by the library's kernels.  There is
no CPU path: loading raises if the shared library is missing, and every call
that launches work raises if the tensors are not on a CUDA device.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, replace

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libufp4.so")

# enums (include/ufp4.h)
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_ALIGNMENT, ERR_OPERAND_MISMATCH, ERR_CUDA, \
    ERR_DEVICE_TIMEOUT = range(7)
GRID_E1M2, GRID_E2M1, GRID_E2M1_MAX2 = 0, 1, 2
ROUND_RTNE, ROUND_SR = 0, 1
SCALE_FP32, SCALE_E4M3_X_FP32, SCALE_UE8M0 = 0, 1, 2
ALONG_COLS, ALONG_ROWS = 0, 1
DEFAULT_SIGN_MASK = 0x09F1FD9D03F0A9B4

EXPORTED = [
    "ufp4_qtensor_layout", "ufp4_rht_amax", "ufp4_rht_quantize", "ufp4_gemm_fprop",
    "ufp4_gemm_dgrad", "ufp4_gemm_wgrad", "ufp4_grouped_gemm", "ufp4_check_device_status",
    "ufp4_status_string", "ufp4_version", "ufp4_set_two_level_gemm_path",
    "ufp4_get_two_level_gemm_path", "ufp4_rht_quantize_dual", "ufp4_rht_amax_dual",
    "ufp4_quant_stats", "ufp4_qstats_summarize", "ufp4_sqnr_sums", "ufp4_rht_bf16",
    "ufp4_sf_atoms_layout", "ufp4_sf_lanes_layout", "ufp4_test_set_quantize_wait_limit",
]


class UFP4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class QuantCfgC(ctypes.Structure):
    _fields_ = [("grid", ctypes.c_int32), ("rounding", ctypes.c_int32),
                ("sr_seed", ctypes.c_uint64), ("sr_stream", ctypes.c_uint32),
                ("hadamard_n", ctypes.c_int32), ("rht_sign_mask", ctypes.c_uint64),
                ("block", ctypes.c_int32), ("scale_fmt", ctypes.c_int32)]


class QTensorC(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("tensor_scale", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("k", ctypes.c_int64), ("kpad", ctypes.c_int64), ("scale_ld", ctypes.c_int64),
                ("cfg", QuantCfgC), ("corr", ctypes.c_void_p), ("elems8", ctypes.c_void_p),
                ("sf_atoms", ctypes.c_void_p), ("sf_lanes", ctypes.c_void_p)]


class GroupC(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in
                ("m", "n", "k", "a_row", "a_col", "b_row", "b_col", "c_row", "c_col")]


class QStatsC(ctypes.Structure):
    _fields_ = [("signal", ctypes.c_double), ("noise", ctypes.c_double),
                ("level_err", ctypes.c_double * 8), ("level_n", ctypes.c_uint64 * 8),
                ("code_count", ctypes.c_uint64 * 16), ("nonzero", ctypes.c_uint64),
                ("underflow", ctypes.c_uint64)]


class QStatsSummaryC(ctypes.Structure):
    _fields_ = [("sqnr_db", ctypes.c_double), ("bucket_ratio", ctypes.c_double),
                ("underflow_ratio", ctypes.c_double), ("level_mean_err", ctypes.c_double * 8)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libufp4.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m fp4_quantized_gemms_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i64, i32, u64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint64
        st = ctypes.c_int
        L.ufp4_status_string.restype = ctypes.c_char_p
        L.ufp4_status_string.argtypes = [st]
        L.ufp4_version.restype = i32
        L.ufp4_qtensor_layout.restype = st
        L.ufp4_qtensor_layout.argtypes = [i64, i64, ctypes.POINTER(QuantCfgC),
                                          ctypes.POINTER(i64), ctypes.POINTER(i64),
                                          ctypes.POINTER(ctypes.c_size_t),
                                          ctypes.POINTER(ctypes.c_size_t)]
        L.ufp4_rht_amax.restype = st
        L.ufp4_rht_amax.argtypes = [P, i64, i64, i64, i32, i32, u64, P, P]
        L.ufp4_rht_bf16.restype = st
        L.ufp4_rht_bf16.argtypes = [P, i64, i64, i64, i32, u64, P, i64, P]
        L.ufp4_rht_quantize.restype = st
        L.ufp4_rht_quantize.argtypes = [P, i64, i64, i64, i32, P, ctypes.POINTER(QTensorC), P]
        L.ufp4_quant_stats.restype = st
        L.ufp4_quant_stats.argtypes = [P, i64, i64, i64, i32, ctypes.POINTER(QTensorC), P, P]
        L.ufp4_qstats_summarize.restype = st
        L.ufp4_qstats_summarize.argtypes = [ctypes.POINTER(QStatsC), i32, ctypes.POINTER(QStatsSummaryC)]
        L.ufp4_sqnr_sums.restype = st
        L.ufp4_sqnr_sums.argtypes = [P, i64, P, i64, i64, i64, P, P]
        L.ufp4_rht_amax_dual.restype = st
        L.ufp4_rht_amax_dual.argtypes = [P, i64, i64, i64, i32, u64, P, P, P]
        L.ufp4_rht_quantize_dual.restype = st
        L.ufp4_rht_quantize_dual.argtypes = [P, i64, i64, i64, P, P, ctypes.POINTER(QTensorC),
                                             ctypes.POINTER(QTensorC), P]
        for name in ("ufp4_gemm_fprop", "ufp4_gemm_dgrad", "ufp4_gemm_wgrad"):
            f = getattr(L, name)
            f.restype = st
            f.argtypes = [ctypes.POINTER(QTensorC), ctypes.POINTER(QTensorC), P, i64, P]
        L.ufp4_grouped_gemm.restype = st
        L.ufp4_grouped_gemm.argtypes = [ctypes.POINTER(QTensorC), ctypes.POINTER(QTensorC), P,
                                        i32, P, i64, P]
        L.ufp4_check_device_status.restype = st
        L.ufp4_check_device_status.argtypes = []
        L.ufp4_sf_atoms_layout.restype = st
        L.ufp4_sf_atoms_layout.argtypes = [i64, i64, ctypes.POINTER(QuantCfgC), ctypes.POINTER(i64),
                                           ctypes.POINTER(ctypes.c_size_t)]
        L.ufp4_sf_lanes_layout.restype = st
        L.ufp4_sf_lanes_layout.argtypes = [i64, i64, ctypes.POINTER(QuantCfgC), ctypes.POINTER(ctypes.c_size_t)]
        L.ufp4_test_set_quantize_wait_limit.restype = st
        L.ufp4_test_set_quantize_wait_limit.argtypes = [u64]
        L.ufp4_set_two_level_gemm_path.restype = st
        L.ufp4_set_two_level_gemm_path.argtypes = [i32]
        L.ufp4_get_two_level_gemm_path.restype = i32
        L.ufp4_get_two_level_gemm_path.argtypes = []
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().ufp4_status_string(status).decode()


def _check(status: int, where: str):
    if status != OK:
        raise UFP4Error(status, where)


def _stream_ptr(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _require_cuda(*tensors):
    for t in tensors:
        if t is not None and not t.is_cuda:
            raise RuntimeError("ufp4 kernels need CUDA tensors (there is no CPU path)")


# ---------------------------------------------------------------- operands
@dataclass(frozen=True)
class QuantConfig:
    grid: int = GRID_E1M2
    rounding: int = ROUND_RTNE
    sr_seed: int = 0
    sr_stream: int = 0
    hadamard_n: int = 16
    rht_sign_mask: int = DEFAULT_SIGN_MASK
    block: int = 16
    scale_fmt: int = SCALE_FP32

    def c(self) -> QuantCfgC:
        return QuantCfgC(self.grid, self.rounding, self.sr_seed, self.sr_stream, self.hadamard_n,
                         self.rht_sign_mask, self.block, self.scale_fmt)

    def with_(self, **kw) -> "QuantConfig":
        return replace(self, **kw)


def layout(rows: int, k: int, cfg: QuantConfig):
    kpad, sld = ctypes.c_int64(), ctypes.c_int64()
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    c = cfg.c()
    _check(lib().ufp4_qtensor_layout(rows, k, ctypes.byref(c), ctypes.byref(kpad),
                                     ctypes.byref(sld), ctypes.byref(cb), ctypes.byref(sb)),
           "ufp4_qtensor_layout")
    return kpad.value, sld.value, cb.value, sb.value


@dataclass
class QTensor:
    """A quantized operand: K-major packed codes + block-major scales."""
    codes: torch.Tensor          # uint8 [rows, kpad/2]
    scales: torch.Tensor         # float32 or uint8 [kpad/block, scale_ld]
    tensor_scale: torch.Tensor | None   # float32 [1] (two-level only)
    rows: int
    k: int
    kpad: int
    scale_ld: int
    cfg: QuantConfig
    corr: torch.Tensor | None = None    # uint8 [rows, kpad/2]: E1M2 correction plane
    elems8: torch.Tensor | None = None  # uint8 [rows, kpad]: E4M3 element plane (MX path)
    sf_atoms: torch.Tensor | None = None  # uint8 [ceil(rows/128), atoms_k, 512]: factor atoms
    sf_lanes: torch.Tensor | None = None  # uint8 [ceil(rows/128), ceil(kpad/128), 4096]: per-lane
                                          # factor tiles of a first GEMM operand (E1M2, E4M3 factors)

    def c(self) -> QTensorC:
        return QTensorC(self.codes.data_ptr(), self.scales.data_ptr(),
                        self.tensor_scale.data_ptr() if self.tensor_scale is not None else None,
                        self.rows, self.k, self.kpad, self.scale_ld, self.cfg.c(),
                        self.corr.data_ptr() if self.corr is not None else None,
                        self.elems8.data_ptr() if self.elems8 is not None else None,
                        self.sf_atoms.data_ptr() if self.sf_atoms is not None else None,
                        self.sf_lanes.data_ptr() if self.sf_lanes is not None else None)


def wants_corr(cfg: QuantConfig) -> bool:
    """Operands the native block-scaled GEMM reads as two E2M1 planes."""
    return cfg.grid == GRID_E1M2 and cfg.scale_fmt == SCALE_E4M3_X_FP32


def wants_elems8(cfg: QuantConfig) -> bool:
    """Operands the block-scaled FP8 GEMM reads as E4M3 elements (MX path)."""
    return cfg.grid == GRID_E1M2 and cfg.scale_fmt == SCALE_UE8M0


def wants_atoms(cfg: QuantConfig) -> bool:
    """Byte block scales: the CTA-pair GEMMs copy factor atoms into tensor
    memory directly."""
    return cfg.scale_fmt != SCALE_FP32


def wants_lanes(cfg: QuantConfig) -> bool:
    """E1M2 operands with E4M3 factors: per-lane factor tiles save the
    CTA-pair GEMM a tensor-memory copy per stage when the operand is its
    first (A) operand."""
    return cfg.grid == GRID_E1M2 and cfg.scale_fmt == SCALE_E4M3_X_FP32


def sf_lanes_layout(rows: int, k: int, cfg: QuantConfig) -> int:
    """Bytes of the per-lane factor tiles of a [rows, k] operand."""
    nb = ctypes.c_size_t()
    c = cfg.c()
    _check(lib().ufp4_sf_lanes_layout(rows, k, ctypes.byref(c), ctypes.byref(nb)), "ufp4_sf_lanes_layout")
    return nb.value


def sf_atoms_layout(rows: int, k: int, cfg: QuantConfig) -> tuple[int, int]:
    """(atoms_k, bytes) of the factor-atom plane of a [rows, k] operand."""
    ak, nb = ctypes.c_int64(), ctypes.c_size_t()
    c = cfg.c()
    _check(lib().ufp4_sf_atoms_layout(rows, k, ctypes.byref(c), ctypes.byref(ak), ctypes.byref(nb)),
           "ufp4_sf_atoms_layout")
    return ak.value, nb.value


def empty_qtensor(rows: int, k: int, cfg: QuantConfig, device="cuda",
                  with_corr: bool | None = None, with_elems8: bool | None = None,
                  with_atoms: bool | None = None, with_lanes: bool | None = None) -> QTensor:
    """Device buffers of a quantized operand.  The optional planes default
    to what the GEMMs use: the correction plane and per-lane factor tiles
    for E1M2 operands with two-level scales, the element plane for MX
    operands, factor atoms for byte block scales.  Pass with_lanes=False for
    an operand that is only ever a GEMM's second operand."""
    kpad, sld, _, _ = layout(rows, k, cfg)
    nblk = kpad // cfg.block
    if with_corr is None:
        with_corr = wants_corr(cfg)
    # codes and the correction plane in one allocation ([2][rows][kpad/2]):
    # the GEMM then fetches both planes of a tile with one copy
    planes = torch.empty((2 if with_corr else 1, rows, kpad // 2), dtype=torch.uint8, device=device)
    codes = planes[0]
    if cfg.scale_fmt == SCALE_FP32:
        scales = torch.empty((nblk, sld), dtype=torch.float32, device=device)
        ts = None
    else:
        scales = torch.empty((nblk, sld), dtype=torch.uint8, device=device)
        ts = torch.empty(1, dtype=torch.float32, device=device) if cfg.scale_fmt == SCALE_E4M3_X_FP32 else None
    corr = planes[1] if with_corr else None
    if with_elems8 is None:
        with_elems8 = wants_elems8(cfg)
    e8 = torch.empty((rows, kpad), dtype=torch.uint8, device=device) if with_elems8 else None
    if with_atoms is None:
        with_atoms = wants_atoms(cfg)
    atoms = None
    if with_atoms:
        ak, _ = sf_atoms_layout(rows, k, cfg)
        atoms = torch.empty(((rows + 127) // 128, ak, 512), dtype=torch.uint8, device=device)
    if with_lanes is None:
        with_lanes = wants_lanes(cfg) and atoms is not None
    lanes = None
    if with_lanes:
        lanes = torch.empty(((rows + 127) // 128, -(-kpad // 128), 4096), dtype=torch.uint8, device=device)
        assert lanes.numel() == sf_lanes_layout(rows, k, cfg)
    return QTensor(codes, scales, ts, rows, k, kpad, sld, cfg, corr, e8, atoms, lanes)


# ---------------------------------------------------------------- entry points
def rht_amax(x: torch.Tensor, axis: int, hadamard_n: int,
             sign_mask: int = DEFAULT_SIGN_MASK, out: torch.Tensor | None = None) -> torch.Tensor:
    """max |H_n D x| over the operand's K-major view -> float32 [1] on device."""
    _require_cuda(x)
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    rows, cols = x.shape
    _check(lib().ufp4_rht_amax(ctypes.c_void_p(x.data_ptr()), rows, cols, x.stride(0), axis,
                               hadamard_n, sign_mask, ctypes.c_void_p(out.data_ptr()),
                               _stream_ptr(x.device)), "ufp4_rht_amax")
    return out


def rht_bf16(x: torch.Tensor, hadamard_n: int, sign_mask: int = DEFAULT_SIGN_MASK,
             out: torch.Tensor | None = None) -> torch.Tensor:
    """Unfused RHT along the columns: bf16(H_n D x) of every n-block of every
    row (the separate pass the fused quantizer is compared with)."""
    _require_cuda(x)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    if out is None:
        out = torch.empty_like(x, memory_format=torch.contiguous_format)
    rows, cols = x.shape
    _check(lib().ufp4_rht_bf16(ctypes.c_void_p(x.data_ptr()), rows, cols, x.stride(0), hadamard_n,
                               sign_mask, ctypes.c_void_p(out.data_ptr()), out.stride(0),
                               _stream_ptr(x.device)), "ufp4_rht_bf16")
    return out


def rht_quantize(x: torch.Tensor, axis: int, cfg: QuantConfig,
                 tensor_amax: torch.Tensor | None = None, out: QTensor | None = None,
                 with_corr: bool | None = None, with_elems8: bool | None = None,
                 with_atoms: bool | None = None, with_lanes: bool | None = None) -> QTensor:
    """Fused RHT + block scale + 4-bit rounding + packing of a bf16 operand
    (plus the E1M2 correction plane when with_corr, by default for E1M2
    operands with two-level scales; the MX element plane; factor atoms, by
    default for byte block scales; per-lane factor tiles, by default with
    the correction plane's operands)."""
    _require_cuda(x, tensor_amax)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    orows, k = (rows, cols) if axis == ALONG_COLS else (cols, rows)
    if out is None:
        out = empty_qtensor(orows, k, cfg, device=x.device, with_corr=with_corr, with_elems8=with_elems8,
                            with_atoms=with_atoms, with_lanes=with_lanes)
    if cfg.scale_fmt == SCALE_E4M3_X_FP32 and tensor_amax is None:
        tensor_amax = rht_amax(x, axis, cfg.hadamard_n, cfg.rht_sign_mask)
    qc = out.c()
    _check(lib().ufp4_rht_quantize(ctypes.c_void_p(x.data_ptr()), rows, cols, x.stride(0), axis,
                                   ctypes.c_void_p(tensor_amax.data_ptr()) if tensor_amax is not None else None,
                                   ctypes.byref(qc), _stream_ptr(x.device)), "ufp4_rht_quantize")
    return out


def rht_amax_dual(x: torch.Tensor, hadamard_n: int, sign_mask: int = DEFAULT_SIGN_MASK,
                  out: torch.Tensor | None = None) -> torch.Tensor:
    """Both rotated amaxes from one read -> float32 [2] on device:
    [ALONG_COLS, ALONG_ROWS]."""
    _require_cuda(x)
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    if out is None:
        out = torch.empty(2, dtype=torch.float32, device=x.device)
    rows, cols = x.shape
    _check(lib().ufp4_rht_amax_dual(ctypes.c_void_p(x.data_ptr()), rows, cols, x.stride(0), hadamard_n,
                                    sign_mask, ctypes.c_void_p(out[0:1].data_ptr()),
                                    ctypes.c_void_p(out[1:2].data_ptr()), _stream_ptr(x.device)),
           "ufp4_rht_amax_dual")
    return out


def rht_quantize_dual(x: torch.Tensor, cfg_cols: QuantConfig, cfg_rows: QuantConfig | None = None,
                      tensor_amax: torch.Tensor | None = None,
                      out: tuple[QTensor, QTensor] | None = None,
                      with_corr: bool | None = None,
                      with_elems8: bool | None = None,
                      with_atoms: bool | None = None) -> tuple[QTensor, QTensor]:
    """Both quantizations of x from one read: (ALONG_COLS result, ALONG_ROWS
    result).  cfg_rows defaults to cfg_cols; the two may differ in sr_stream
    only.  tensor_amax: float32 [2] device tensor from rht_amax_dual (two-level
    scales; computed here when None)."""
    _require_cuda(x, tensor_amax)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    cfg_rows = cfg_cols if cfg_rows is None else cfg_rows
    rows, cols = x.shape
    if out is None:
        out = (empty_qtensor(rows, cols, cfg_cols, device=x.device, with_corr=with_corr,
                             with_elems8=with_elems8, with_atoms=with_atoms),
               empty_qtensor(cols, rows, cfg_rows, device=x.device, with_corr=with_corr,
                             with_elems8=with_elems8, with_atoms=with_atoms))
    if cfg_cols.scale_fmt == SCALE_E4M3_X_FP32 and tensor_amax is None:
        tensor_amax = rht_amax_dual(x, cfg_cols.hadamard_n, cfg_cols.rht_sign_mask)
    qc, qr = out[0].c(), out[1].c()
    am_c = ctypes.c_void_p(tensor_amax[0:1].data_ptr()) if tensor_amax is not None else None
    am_r = ctypes.c_void_p(tensor_amax[1:2].data_ptr()) if tensor_amax is not None else None
    _check(lib().ufp4_rht_quantize_dual(ctypes.c_void_p(x.data_ptr()), rows, cols, x.stride(0), am_c, am_r,
                                        ctypes.byref(qc), ctypes.byref(qr), _stream_ptr(x.device)),
           "ufp4_rht_quantize_dual")
    return out


def quant_stats_launch(x: torch.Tensor, axis: int, q: QTensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """Enqueue ufp4_quant_stats; returns the device buffer holding the
    ufp4_qstats_t (float64 words)."""
    _require_cuda(x, q.codes)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    if out is None:
        out = torch.zeros(ctypes.sizeof(QStatsC) // 8, dtype=torch.float64, device=x.device)
    rows, cols = x.shape
    qc = q.c()
    _check(lib().ufp4_quant_stats(ctypes.c_void_p(x.data_ptr()), rows, cols, x.stride(0), axis,
                                  ctypes.byref(qc), ctypes.c_void_p(out.data_ptr()), _stream_ptr(x.device)),
           "ufp4_quant_stats")
    return out


def quant_stats(x: torch.Tensor, axis: int, q: QTensor, out: torch.Tensor | None = None) -> dict:
    """Diagnostics sums of operand q quantized from x along axis (a host copy
    of ufp4_qstats_t as a dict, plus its ufp4_qstats_summarize figures)."""
    out = quant_stats_launch(x, axis, q, out)
    host = QStatsC.from_buffer_copy(out.cpu().numpy().tobytes())
    sm = QStatsSummaryC()
    _check(lib().ufp4_qstats_summarize(ctypes.byref(host), q.cfg.grid, ctypes.byref(sm)),
           "ufp4_qstats_summarize")
    return {
        "signal": host.signal, "noise": host.noise, "level_err": list(host.level_err),
        "level_n": list(host.level_n), "code_count": list(host.code_count),
        "nonzero": host.nonzero, "underflow": host.underflow,
        "sqnr_db": sm.sqnr_db, "bucket_ratio": sm.bucket_ratio, "underflow_ratio": sm.underflow_ratio,
        "level_mean_err": list(sm.level_mean_err),
    }


def sqnr_sums(ref: torch.Tensor, test: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """[sum ref^2, sum (test - ref)^2] (float64 [2] on device) of two fp32 matrices."""
    _require_cuda(ref, test)
    assert ref.dtype == torch.float32 and test.dtype == torch.float32 and ref.shape == test.shape
    assert ref.stride(1) == 1 and test.stride(1) == 1
    if out is None:
        out = torch.empty(2, dtype=torch.float64, device=ref.device)
    rows, cols = ref.shape
    _check(lib().ufp4_sqnr_sums(ctypes.c_void_p(ref.data_ptr()), ref.stride(0),
                                ctypes.c_void_p(test.data_ptr()), test.stride(0), rows, cols,
                                ctypes.c_void_p(out.data_ptr()), _stream_ptr(ref.device)), "ufp4_sqnr_sums")
    return out


def _gemm(name: str, a: QTensor, b: QTensor, out: torch.Tensor | None) -> torch.Tensor:
    _require_cuda(a.codes, b.codes)
    if out is None:
        out = torch.empty((a.rows, b.rows), dtype=torch.float32, device=a.codes.device)
    ac, bc = a.c(), b.c()
    _check(getattr(lib(), name)(ctypes.byref(ac), ctypes.byref(bc), ctypes.c_void_p(out.data_ptr()),
                                out.stride(0), _stream_ptr(out.device)), name)
    return out


def gemm_fprop(xq: QTensor, wq: QTensor, out=None) -> torch.Tensor:
    """Y = X W^T from X, W both quantized ALONG_COLS."""
    return _gemm("ufp4_gemm_fprop", xq, wq, out)


def gemm_dgrad(dyq: QTensor, wtq: QTensor, out=None) -> torch.Tensor:
    """dX = dY W from dY quantized ALONG_COLS and W quantized ALONG_ROWS."""
    return _gemm("ufp4_gemm_dgrad", dyq, wtq, out)


def gemm_wgrad(dytq: QTensor, xtq: QTensor, out=None) -> torch.Tensor:
    """dW = dY^T X from dY and X both quantized ALONG_ROWS."""
    return _gemm("ufp4_gemm_wgrad", dytq, xtq, out)


def grouped_gemm(a: QTensor, b: QTensor, groups: torch.Tensor, out: torch.Tensor) -> torch.Tensor:
    """groups: int64 CUDA tensor [G, 9] rows (m, n, k, a_row, a_col, b_row, b_col, c_row, c_col)."""
    _require_cuda(a.codes, b.codes, groups, out)
    assert groups.dtype == torch.int64 and groups.dim() == 2 and groups.shape[1] == 9
    groups = groups.contiguous()
    ac, bc = a.c(), b.c()
    _check(lib().ufp4_grouped_gemm(ctypes.byref(ac), ctypes.byref(bc),
                                   ctypes.c_void_p(groups.data_ptr()), groups.shape[0],
                                   ctypes.c_void_p(out.data_ptr()), out.stride(0),
                                   _stream_ptr(out.device)), "ufp4_grouped_gemm")
    return out


GEMM_PATH_AUTO, GEMM_PATH_NATIVE_FP4, GEMM_PATH_NATIVE_FP4_PAIR256 = 0, 3, 5


def set_two_level_gemm_path(path: int) -> None:
    """Process-wide kernel family for GEMMs on two-level-scaled operands."""
    _check(lib().ufp4_set_two_level_gemm_path(path), "ufp4_set_two_level_gemm_path")


def get_two_level_gemm_path() -> int:
    return lib().ufp4_get_two_level_gemm_path()


def check_device_status() -> int:
    """Reads and clears the kernels' device error word (synchronises)."""
    return lib().ufp4_check_device_status()


def set_quantize_wait_limit_for_tests(limit_ns: int) -> None:
    """Test support: the quantizer producer's wait limit in ns (0: default)."""
    _check(lib().ufp4_test_set_quantize_wait_limit(limit_ns), "ufp4_test_set_quantize_wait_limit")
