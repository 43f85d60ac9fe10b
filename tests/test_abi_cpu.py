"""C ABI checks that need no GPU: the library builds and loads, exports every
function ``include/ufp4.h`` declares, the ctypes mirrors match the C struct
layouts, and host-side validation rejects bad arguments before any launch."""
import ctypes
import math
import os
import re
import subprocess

import numpy as np
import pytest
import torch

from fp4_quantized_gemms_b200 import build as ufp4_build
from fp4_quantized_gemms_b200 import ufp4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ufp4.h")


@pytest.fixture(scope="module")
def L():
    ufp4_build.build()
    return ufp4.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ufp4_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert set(names) == set(ufp4.EXPORTED)
    nm = subprocess.run(["nm", "-D", "--defined-only", ufp4.LIB_PATH], capture_output=True,
                        text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(ufp4_\w+)", nm))
    for n in names:
        assert n in exported, n
        assert hasattr(L, n)


def test_struct_layouts_match_header(tmp_path):
    """sizeof / offsetof from the C compiler == the ctypes mirrors."""
    src = tmp_path / "layout.c"
    src.write_text("""
#include <stdio.h>
#include <stddef.h>
#include "ufp4.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu\\n", sizeof(ufp4_quant_cfg_t), offsetof(ufp4_quant_cfg_t, sr_seed),
         offsetof(ufp4_quant_cfg_t, rht_sign_mask), offsetof(ufp4_quant_cfg_t, scale_fmt), 0);
  printf("%zu %zu %zu %zu %zu %zu %zu %zu\\n", sizeof(ufp4_qtensor_t), offsetof(ufp4_qtensor_t, rows),
         offsetof(ufp4_qtensor_t, scale_ld), offsetof(ufp4_qtensor_t, cfg),
         offsetof(ufp4_qtensor_t, corr), offsetof(ufp4_qtensor_t, elems8), offsetof(ufp4_qtensor_t, sf_atoms),
         offsetof(ufp4_qtensor_t, sf_lanes));
  printf("%zu %zu\\n", sizeof(ufp4_group_t), offsetof(ufp4_group_t, c_col));
  printf("%zu %zu %zu %zu %zu\\n", sizeof(ufp4_qstats_t), offsetof(ufp4_qstats_t, level_n),
         offsetof(ufp4_qstats_t, code_count), offsetof(ufp4_qstats_t, underflow),
         sizeof(ufp4_qstats_summary_t));
  return 0;
}
""")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    c1 = list(map(int, out[0].split()))
    c2 = list(map(int, out[1].split()))
    c3 = list(map(int, out[2].split()))
    c4 = list(map(int, out[3].split()))
    Q, T, G = ufp4.QuantCfgC, ufp4.QTensorC, ufp4.GroupC
    St, Sm = ufp4.QStatsC, ufp4.QStatsSummaryC
    assert c4 == [ctypes.sizeof(St), St.level_n.offset, St.code_count.offset, St.underflow.offset,
                  ctypes.sizeof(Sm)]
    assert c1[:4] == [ctypes.sizeof(Q), Q.sr_seed.offset, Q.rht_sign_mask.offset, Q.scale_fmt.offset]
    assert c2 == [ctypes.sizeof(T), T.rows.offset, T.scale_ld.offset, T.cfg.offset, T.corr.offset,
                  T.elems8.offset, T.sf_atoms.offset, T.sf_lanes.offset]
    assert c3 == [ctypes.sizeof(G), G.c_col.offset]


def test_status_strings_and_version(L):
    assert ufp4.status_string(ufp4.OK) == "UFP4_OK"
    assert ufp4.status_string(ufp4.ERR_OPERAND_MISMATCH) == "UFP4_ERR_OPERAND_MISMATCH"
    assert L.ufp4_version() >= 100


@pytest.mark.parametrize("k,block,fmt,kpad,codes,scales", [
    (512, 16, ufp4.SCALE_FP32, 512, 256 * 256, 32 * 256 * 4),
    (500, 16, ufp4.SCALE_FP32, 512, 256 * 256, 32 * 256 * 4),
    (2048, 32, ufp4.SCALE_E4M3_X_FP32, 2048, 256 * 1024, 64 * 256),
    (0, 16, ufp4.SCALE_FP32, 0, 0, 0),
    (1000, 32, ufp4.SCALE_UE8M0, 1024, 256 * 512, 32 * 256),
])
def test_layout(L, k, block, fmt, kpad, codes, scales):
    cfg = ufp4.QuantConfig(block=block, scale_fmt=fmt)
    kp, sld, cb, sb = ufp4.layout(256, k, cfg)
    assert (kp, sld, cb, sb) == (kpad, 256, codes, scales)
    assert ufp4.layout(300, 64, cfg)[1] == 320


@pytest.mark.parametrize("rows,k,block,fmt,atoms_k,nbytes", [
    (256, 512, 16, ufp4.SCALE_E4M3_X_FP32, 8, 2 * 8 * 512),
    (300, 200, 32, ufp4.SCALE_E4M3_X_FP32, 4, 3 * 4 * 512),     # kpad 256: 16 slots of 16
    (129, 1000, 32, ufp4.SCALE_UE8M0, 8, 2 * 8 * 512),          # kpad 1024: 32 slots of 32
    (1, 136, 32, ufp4.SCALE_UE8M0, 2, 1 * 2 * 512),             # kpad 192: 6 slots, 2 atoms
    (0, 64, 16, ufp4.SCALE_E4M3_X_FP32, 1, 0),
])
def test_sf_atoms_layout(L, rows, k, block, fmt, atoms_k, nbytes):
    """Factor-atom plane size: ceil(rows/128) row groups x ceil(kpad / 4W)
    atoms of 512 bytes (W = 16 for E4M3 factors, 32 for UE8M0); none for
    fp32 scales."""
    cfg = ufp4.QuantConfig(block=block, scale_fmt=fmt)
    assert ufp4.sf_atoms_layout(rows, k, cfg) == (atoms_k, nbytes)
    c = ufp4.QuantConfig(scale_fmt=ufp4.SCALE_FP32).c()
    assert L.ufp4_sf_atoms_layout(64, 64, ctypes.byref(c), None, None) == ufp4.ERR_UNSUPPORTED
    c = cfg.c()
    assert L.ufp4_sf_atoms_layout(-1, 64, ctypes.byref(c), None, None) == ufp4.ERR_INVALID_ARG
    assert L.ufp4_sf_atoms_layout(64, 64, None, None, None) == ufp4.ERR_INVALID_ARG


@pytest.mark.parametrize("rows,k,block,grid,fmt,nbytes", [
    (256, 512, 16, ufp4.GRID_E1M2, ufp4.SCALE_E4M3_X_FP32, 2 * 4 * 4096),
    (300, 200, 32, ufp4.GRID_E1M2, ufp4.SCALE_E4M3_X_FP32, 3 * 2 * 4096),   # kpad 256
    (130, 64, 16, ufp4.GRID_E1M2, ufp4.SCALE_E4M3_X_FP32, 2 * 1 * 4096),    # kpad 64: half a tile used
    (0, 64, 16, ufp4.GRID_E1M2, ufp4.SCALE_E4M3_X_FP32, 0),
    (256, 512, 16, ufp4.GRID_E2M1, ufp4.SCALE_E4M3_X_FP32, None),           # other grids: no tiles
    (256, 512, 32, ufp4.GRID_E1M2, ufp4.SCALE_UE8M0, None),
    (256, 512, 16, ufp4.GRID_E1M2, ufp4.SCALE_FP32, None),
])
def test_sf_lanes_layout(L, rows, k, block, grid, fmt, nbytes):
    """Per-lane factor tiles: ceil(rows/128) x ceil(kpad/128) tiles of 4096
    bytes, E1M2 operands with E4M3 x fp32 scales only (else UNSUPPORTED)."""
    cfg = ufp4.QuantConfig(grid=grid, block=block, scale_fmt=fmt)
    c = cfg.c()
    nb = ctypes.c_size_t()
    st = L.ufp4_sf_lanes_layout(rows, k, ctypes.byref(c), ctypes.byref(nb))
    if nbytes is None:
        assert st == ufp4.ERR_UNSUPPORTED
    else:
        assert st == ufp4.OK and nb.value == nbytes
        assert ufp4.sf_lanes_layout(rows, k, cfg) == nbytes
    assert L.ufp4_sf_lanes_layout(rows, k, ctypes.byref(c), None) == ufp4.ERR_INVALID_ARG
    assert L.ufp4_sf_lanes_layout(-1, k, ctypes.byref(c), ctypes.byref(nb)) == ufp4.ERR_INVALID_ARG


def _q(rows=128, k=256, **kw):
    cfg = ufp4.QuantConfig(**kw).c()
    kp = (k + 63) // 64 * 64
    return ufp4.QTensorC(16 * 1024, 32 * 1024, 48 * 1024 if kw.get("scale_fmt") else None,
                         rows, k, kp, (rows + 63) // 64 * 64, cfg)


def _gemm(L, a, b, c_ptr=64 * 1024, ldc=128):
    return L.ufp4_gemm_fprop(ctypes.byref(a), ctypes.byref(b), ctypes.c_void_p(c_ptr), ldc, None)


def test_gemm_validation_rejects_before_launch(L):
    """Every rejection below happens on the host: no CUDA call is made."""
    assert _gemm(L, _q(grid=0), _q(grid=1)) == ufp4.ERR_OPERAND_MISMATCH
    assert _gemm(L, _q(grid=1), _q(grid=2)) == ufp4.ERR_OPERAND_MISMATCH
    assert _gemm(L, _q(grid=3), _q(grid=3)) == ufp4.ERR_INVALID_ARG
    assert _gemm(L, _q(block=16), _q(block=32)) == ufp4.ERR_OPERAND_MISMATCH
    assert _gemm(L, _q(hadamard_n=16), _q(hadamard_n=32)) == ufp4.ERR_OPERAND_MISMATCH
    assert _gemm(L, _q(rht_sign_mask=1), _q(rht_sign_mask=2)) == ufp4.ERR_OPERAND_MISMATCH
    # sign-mask bits beyond n do not matter
    a, b = _q(hadamard_n=16, rht_sign_mask=0x1_0001), _q(hadamard_n=16, rht_sign_mask=0x2_0001)
    assert _gemm(L, a, b, c_ptr=64 * 1024 + 2) == ufp4.ERR_ALIGNMENT
    assert _gemm(L, _q(k=256), _q(k=192)) == ufp4.ERR_OPERAND_MISMATCH
    assert _gemm(L, _q(scale_fmt=0), _q(scale_fmt=1)) == ufp4.ERR_OPERAND_MISMATCH
    assert _gemm(L, _q(scale_fmt=2, block=32), _q(scale_fmt=0, block=32)) == ufp4.ERR_OPERAND_MISMATCH
    assert _gemm(L, _q(scale_fmt=2, block=16), _q(scale_fmt=2, block=16)) == ufp4.ERR_INVALID_ARG  # MX: 32
    bad = _q()
    bad.kpad = 100
    assert _gemm(L, bad, _q()) == ufp4.ERR_INVALID_ARG
    bad = _q()
    bad.codes = 16 * 1024 + 8
    assert _gemm(L, bad, _q()) == ufp4.ERR_ALIGNMENT
    bad = _q(scale_fmt=1)
    bad.tensor_scale = None
    assert _gemm(L, bad, _q(scale_fmt=1)) == ufp4.ERR_INVALID_ARG
    assert _gemm(L, _q(), _q(), ldc=64) == ufp4.ERR_INVALID_ARG    # ldc < N
    assert _gemm(L, _q(), _q(), c_ptr=64 * 1024 + 1) == ufp4.ERR_ALIGNMENT
    bad_cfg = _q()
    bad_cfg.cfg.hadamard_n = 8
    assert _gemm(L, bad_cfg, _q()) == ufp4.ERR_INVALID_ARG
    assert L.ufp4_gemm_fprop(None, ctypes.byref(_q()), None, 128, None) == ufp4.ERR_INVALID_ARG
    assert L.ufp4_grouped_gemm(ctypes.byref(_q()), ctypes.byref(_q()), None, 3, None, 128,
                               None) == ufp4.ERR_INVALID_ARG
    assert L.ufp4_grouped_gemm(ctypes.byref(_q()), ctypes.byref(_q()), None, -1, None, 128,
                               None) == ufp4.ERR_INVALID_ARG


def test_quantize_validation_rejects_before_launch(L):
    out = _q(rows=64, k=128)
    x = ctypes.c_void_p(4096)
    Q = L.ufp4_rht_quantize
    assert Q(None, 64, 128, 128, 0, None, ctypes.byref(out), None) == ufp4.ERR_INVALID_ARG
    assert Q(x, 64, 128, 100, 0, None, ctypes.byref(out), None) == ufp4.ERR_INVALID_ARG   # ld < cols
    assert Q(x, 64, 120, 124, 0, None, ctypes.byref(_q(rows=64, k=120)), None) == ufp4.ERR_ALIGNMENT
    assert Q(ctypes.c_void_p(4098), 64, 128, 128, 0, None, ctypes.byref(out), None) == ufp4.ERR_ALIGNMENT
    assert Q(x, 64, 128, 128, 2, None, ctypes.byref(out), None) == ufp4.ERR_INVALID_ARG   # axis
    assert Q(x, 64, 128, 128, 1, None, ctypes.byref(out), None) == ufp4.ERR_INVALID_ARG   # shape
    two = _q(rows=64, k=128, scale_fmt=1)
    assert Q(x, 64, 128, 128, 0, None, ctypes.byref(two), None) == ufp4.ERR_INVALID_ARG   # no amax
    am = ctypes.c_void_p(8192)
    fp = _q(rows=64, k=128)
    fp.sf_atoms = 64 * 1024
    assert Q(x, 64, 128, 128, 0, None, ctypes.byref(fp), None) == ufp4.ERR_INVALID_ARG    # atoms, fp32 scales
    two.sf_atoms = 64 * 1024 + 8
    assert Q(x, 64, 128, 128, 0, am, ctypes.byref(two), None) == ufp4.ERR_ALIGNMENT       # atoms alignment
    assert L.ufp4_rht_amax(x, 64, 128, 128, 0, 8, 0, ctypes.c_void_p(4096), None) == ufp4.ERR_UNSUPPORTED
    assert L.ufp4_rht_amax(x, 64, 128, 128, 0, 16, 0, None, None) == ufp4.ERR_INVALID_ARG
    R = L.ufp4_rht_bf16
    y = ctypes.c_void_p(8192)
    assert R(x, 64, 128, 128, 8, 0, y, 128, None) == ufp4.ERR_UNSUPPORTED       # n
    assert R(x, 64, 136, 136, 16, 0, y, 136, None) == ufp4.ERR_UNSUPPORTED     # cols % 64
    assert R(x, 64, 128, 128, 16, 0, None, 128, None) == ufp4.ERR_INVALID_ARG   # no output
    assert R(x, 64, 128, 128, 16, 0, y, 64, None) == ufp4.ERR_INVALID_ARG       # ldy < cols
    assert R(x, 64, 128, 128, 16, 0, ctypes.c_void_p(8200), 128, None) == ufp4.ERR_ALIGNMENT
    assert R(x, 0, 128, 128, 16, 0, None, 0, None) == ufp4.OK                   # empty: no launch


def test_dual_quantize_validation_rejects_before_launch(L):
    """The dual quantizer checks both descriptors and that their recipes agree
    (all but sr_stream) before any CUDA call."""
    x = ctypes.c_void_p(4096)
    D = L.ufp4_rht_quantize_dual

    def call(oc, orr, rows=64, cols=128, ld=128, am=None):
        return D(x, rows, cols, ld, am, am, ctypes.byref(oc), ctypes.byref(orr), None)

    assert call(_q(rows=64, k=128), _q(rows=128, k=128)) == ufp4.ERR_INVALID_ARG   # rows-out shape
    assert call(_q(rows=128, k=64), _q(rows=128, k=64)) == ufp4.ERR_INVALID_ARG    # cols-out shape
    for kw in ({"grid": 1}, {"rounding": 1}, {"hadamard_n": 32}, {"block": 32}, {"sr_seed": 5},
               {"hadamard_n": 16, "rht_sign_mask": 0x1}):
        base = {"hadamard_n": 16, "rht_sign_mask": 0x2} if "rht_sign_mask" in kw else {}
        assert call(_q(rows=64, k=128, **base), _q(rows=128, k=64, **kw)) == ufp4.ERR_UNSUPPORTED, kw
    two_c, two_r = _q(rows=64, k=128, scale_fmt=1), _q(rows=128, k=64, scale_fmt=1)
    assert call(two_c, two_r) == ufp4.ERR_INVALID_ARG                              # no amax
    assert D(None, 64, 128, 128, None, None, ctypes.byref(_q(rows=64, k=128)),
             ctypes.byref(_q(rows=128, k=64)), None) == ufp4.ERR_INVALID_ARG
    # empty input: validated, nothing to launch
    assert call(_q(rows=0, k=128), _q(rows=128, k=0), rows=0) == ufp4.OK
    A = L.ufp4_rht_amax_dual
    assert A(x, 64, 128, 128, 8, 0, x, x, None) == ufp4.ERR_UNSUPPORTED
    assert A(x, 64, 128, 128, 16, 0, None, x, None) == ufp4.ERR_INVALID_ARG
    assert A(x, 64, 120, 124, 16, 0, x, x, None) == ufp4.ERR_ALIGNMENT


def test_two_level_gemm_path_selector(L):
    """The path setting is host state: it round-trips and rejects unknown values."""
    old = ufp4.get_two_level_gemm_path()
    try:
        for p in (ufp4.GEMM_PATH_NATIVE_FP4, ufp4.GEMM_PATH_NATIVE_FP4_PAIR256, ufp4.GEMM_PATH_AUTO):
            ufp4.set_two_level_gemm_path(p)
            assert ufp4.get_two_level_gemm_path() == p
        for bad in (-1, 1, 2, 4, 6, 99):   # 1, 2, 4: removed kernel families
            with pytest.raises(ufp4.UFP4Error):
                ufp4.set_two_level_gemm_path(bad)
        assert ufp4.get_two_level_gemm_path() == ufp4.GEMM_PATH_AUTO
    finally:
        ufp4.set_two_level_gemm_path(old)


def test_qstats_summarize_host_arithmetic(L):
    """The summary is plain host arithmetic: closed-form values of a made-up
    set of sums, and the argument checks."""
    st = ufp4.QStatsC()
    st.signal, st.noise = 1000.0, 10.0                  # 20 dB
    for c, n in {0: 500, 1: 300, 9: 150, 7: 40, 15: 9, 3: 1}.items():
        st.code_count[c] = n                            # 1000 elements; threshold 1000/240
    st.level_err[1], st.level_n[1] = -4.5, 450
    st.nonzero, st.underflow = 800, 300
    sm = ufp4.QStatsSummaryC()
    assert L.ufp4_qstats_summarize(ctypes.byref(st), 0, ctypes.byref(sm)) == ufp4.OK
    assert sm.sqnr_db == 20.0
    assert sm.bucket_ratio == 5 / 15                     # codes 0, 1, 9, 7, 15 (9 > 4.17)
    assert sm.underflow_ratio == 300 / 800
    assert sm.level_mean_err[1] == -0.01 and math.isnan(sm.level_mean_err[2])
    assert L.ufp4_qstats_summarize(ctypes.byref(st), 2, ctypes.byref(sm)) == ufp4.OK
    assert sm.bucket_ratio == 5 / 9
    st.noise = 0.0
    assert L.ufp4_qstats_summarize(ctypes.byref(st), 1, ctypes.byref(sm)) == ufp4.OK
    assert math.isinf(sm.sqnr_db)
    assert L.ufp4_qstats_summarize(ctypes.byref(st), 3, ctypes.byref(sm)) == ufp4.ERR_INVALID_ARG
    assert L.ufp4_qstats_summarize(None, 0, ctypes.byref(sm)) == ufp4.ERR_INVALID_ARG


def test_diagnostics_validation_rejects_before_launch(L):
    x = ctypes.c_void_p(4096)
    q = _q(rows=64, k=128)
    st = ctypes.c_void_p(8192)
    S = L.ufp4_quant_stats
    assert S(x, 64, 128, 128, 0, ctypes.byref(q), None, None) == ufp4.ERR_INVALID_ARG
    assert S(x, 64, 128, 128, 0, ctypes.byref(q), ctypes.c_void_p(8196), None) == ufp4.ERR_ALIGNMENT
    assert S(x, 64, 128, 128, 1, ctypes.byref(q), st, None) == ufp4.ERR_INVALID_ARG   # shape
    assert S(x, 64, 128, 100, 0, ctypes.byref(q), st, None) == ufp4.ERR_INVALID_ARG   # ld < cols
    assert S(None, 64, 128, 128, 0, ctypes.byref(q), st, None) == ufp4.ERR_INVALID_ARG
    Q = L.ufp4_sqnr_sums
    assert Q(x, 128, x, 128, 4, 128, None, None) == ufp4.ERR_INVALID_ARG
    assert Q(x, 100, x, 128, 4, 128, st, None) == ufp4.ERR_INVALID_ARG
    assert Q(None, 128, x, 128, 4, 128, st, None) == ufp4.ERR_INVALID_ARG
    assert Q(x, 128, x, 128, -1, 128, st, None) == ufp4.ERR_INVALID_ARG


def test_product_path_fails_loudly_without_the_library_or_cuda(tmp_path):
    """No CPU fallback: a missing library raises on first use, and CPU tensors
    are refused before any call."""
    import sys
    code = ("import sys; sys.path.insert(0, %r)\n"
            "from fp4_quantized_gemms_b200 import ufp4\n"
            "ufp4.LIB_PATH = %r\n"
            "try:\n    ufp4.lib()\nexcept RuntimeError as e:\n    print('raised', 'missing' in str(e))\n"
            % (ROOT, str(tmp_path / "absent.so")))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert r.stdout.strip() == "raised True", r.stderr
    import torch
    x = torch.zeros((16, 64), dtype=torch.bfloat16)
    with pytest.raises(RuntimeError, match="CUDA"):
        ufp4.rht_quantize(x, ufp4.ALONG_COLS, ufp4.QuantConfig())
    with pytest.raises(RuntimeError, match="CUDA"):
        ufp4.rht_quantize_dual(x, ufp4.QuantConfig())


@pytest.mark.parametrize("grid,fmt,block", [
    (ufp4.GRID_E1M2, ufp4.SCALE_FP32, 16), (ufp4.GRID_E1M2, ufp4.SCALE_E4M3_X_FP32, 16),
    (ufp4.GRID_E2M1, ufp4.SCALE_E4M3_X_FP32, 32), (ufp4.GRID_E2M1_MAX2, ufp4.SCALE_UE8M0, 32),
    (ufp4.GRID_E1M2, ufp4.SCALE_UE8M0, 32),
])
def test_binding_allocates_what_the_layout_call_sizes(grid, fmt, block):
    """empty_qtensor (host tensors here) matches ufp4_qtensor_layout: codes,
    block-major scales of the format's element size, the E1M2 correction plane
    for two-level operands only, a tensor scale for two-level only."""
    cfg = ufp4.QuantConfig(grid=grid, block=block, scale_fmt=fmt)
    kpad, sld, cbytes, sbytes = ufp4.layout(300, 200, cfg)
    q = ufp4.empty_qtensor(300, 200, cfg, device="cpu")
    assert q.codes.numel() == cbytes and q.scales.numel() * q.scales.element_size() == sbytes
    assert q.scales.shape == (kpad // block, sld) and sld % 64 == 0 and sld >= 300
    assert (q.corr is not None) == (grid == ufp4.GRID_E1M2 and fmt == ufp4.SCALE_E4M3_X_FP32)
    assert (q.tensor_scale is not None) == (fmt == ufp4.SCALE_E4M3_X_FP32)
    if fmt == ufp4.SCALE_FP32:
        assert q.sf_atoms is None
    else:
        assert q.sf_atoms.numel() == ufp4.sf_atoms_layout(300, 200, cfg)[1]
    c = q.c()
    assert c.rows == 300 and c.k == 200 and c.kpad == kpad and c.scale_ld == sld
    assert c.cfg.scale_fmt == fmt and c.cfg.block == block and c.cfg.grid == grid


def test_mx_element_table_is_the_e4m3_encoding():
    """The MX element plane's byte table (E1M2 level k/4 -> E4M3 byte, used by
    the GPU tests) equals torch's float8_e4m3fn encoding of k/4, and negation
    sets bit 7 only."""
    from tests.gpu_util import E4M3_OF_E1M2, expected_elems8
    vals = torch.tensor([k / 4 for k in range(8)], dtype=torch.float32)
    assert list(vals.to(torch.float8_e4m3fn).view(torch.uint8).numpy()) == E4M3_OF_E1M2
    neg = (-vals[1:]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert list(expected_elems8(np.arange(9, 16))) == list(neg)
    assert list(expected_elems8(np.arange(0, 8))) == E4M3_OF_E1M2
