"""Parity of the diagnostics kernels with the oracle's diagnostics: integer
counts bit-exact, fp sums within 1e-5 relative (the kernel sums 64-element
segments in fp32 before fp64; the oracle sums in fp64), on ragged shapes of
every grid, RHT size, rounding, scale format and axis; full-size properties;
GEMM-output SQNR sums."""
import numpy as np
import pytest
import torch

import oracle
from oracle import diagnostics as dg
from fp4_quantized_gemms_b200 import ufp4
from fp4_quantized_gemms_b200 import workloads as wl
from tests.gpu_util import needs_gpu, oracle_cfg, to_dev

pytestmark = needs_gpu

RTOL = 1e-5
AXES = [ufp4.ALONG_COLS, ufp4.ALONG_ROWS]


def _check(got: dict, want: dict):
    assert got["code_count"] == list(want["code_count"])
    assert got["level_n"] == list(want["level_n"])
    assert got["nonzero"] == want["nonzero"] and got["underflow"] == want["underflow"]
    assert got["signal"] == pytest.approx(want["signal"], rel=RTOL)
    assert got["noise"] == pytest.approx(want["noise"], rel=RTOL)
    # a level's error sum is a sum of terms of either sign: bound by its count
    for k in range(8):
        assert abs(got["level_err"][k] - want["level_err"][k]) <= RTOL * (want["level_n"][k] + 1)


def _run(X, axis, cfg):
    x = to_dev(X)
    q = ufp4.rht_quantize(x, axis, cfg)
    got = ufp4.quant_stats(x, axis, q)
    amax = 0.0
    if cfg.scale_fmt == ufp4.SCALE_E4M3_X_FP32:
        amax = oracle.rht_amax(X, axis, cfg.hadamard_n, cfg.rht_sign_mask)
    rq, ru = oracle.quantize(X, axis, oracle_cfg(cfg), tensor_amax=amax, want_u=True)
    want = dg.quant_stats(rq, ru)
    _check(got, want)
    sm = dg.summary(want)
    assert got["sqnr_db"] == pytest.approx(sm["sqnr_db"], abs=1e-4)
    assert got["bucket_ratio"] == sm["bucket_ratio"]
    assert got["underflow_ratio"] == sm["underflow_ratio"]
    assert ufp4.check_device_status() == ufp4.OK
    return got


@pytest.mark.parametrize("axis", AXES)
@pytest.mark.parametrize("n,block", [(0, 16), (16, 16), (32, 32), (64, 16)])
@pytest.mark.parametrize("grid", [ufp4.GRID_E1M2, ufp4.GRID_E2M1, ufp4.GRID_E2M1_MAX2])
@pytest.mark.parametrize("fmt", [ufp4.SCALE_FP32, ufp4.SCALE_E4M3_X_FP32])
def test_quant_stats_match_oracle(axis, n, block, grid, fmt):
    """200 x 136 outlier-heavy input: ragged rows and a ragged K tail."""
    X = wl.normal_with_outlier_channels(200, 136, 1.0, 3, 30.0)
    for rounding in (ufp4.ROUND_RTNE, ufp4.ROUND_SR):
        cfg = ufp4.QuantConfig(grid=grid, rounding=rounding, sr_seed=99, hadamard_n=n, block=block,
                               scale_fmt=fmt)
        _run(X, axis, cfg)


def test_quant_stats_underflow_and_zero_blocks():
    """Tiny values beside a large one in each block (E4M3 block factors that
    underflow to 0 in two-level mode), an all-zero row."""
    x = np.full((64, 256), 1e-6, dtype=np.float32)
    x[:, ::16] = 5.0
    x[:, 100:116] = 1e-30
    x[7, :] = 0.0
    X = wl.bf16_bits(x)
    for fmt in (ufp4.SCALE_FP32, ufp4.SCALE_E4M3_X_FP32):
        for axis in AXES:
            got = _run(X, axis, ufp4.QuantConfig(hadamard_n=0, block=16, scale_fmt=fmt))
            # Along the columns every block mixes 5.0 with tiny values, which
            # round to 0.  Along the rows a block is part of one column, whose
            # values are all alike: no underflow with fp32 scales, but with
            # two-level scales the E4M3 factor of a 1e-6 column (1e-6 / G with
            # G = 5/448) underflows to 0 and takes the whole block with it.
            two = fmt == ufp4.SCALE_E4M3_X_FP32
            assert (got["underflow"] > 0) == (axis == ufp4.ALONG_COLS or two)


def test_rht_flips_the_grid_ranking_on_the_gpu():
    """The pages' diagnostic claim through the CUDA path on a synthetic
    outlier-heavy tensor (the same ranking as the oracle's CPU check)."""
    X = wl.normal_with_outlier_channels(1024, 2048, 1.0, 16, 30.0)
    x = to_dev(X)
    s = {}
    for grid in (ufp4.GRID_E1M2, ufp4.GRID_E2M1):
        for n in (0, 16):
            cfg = ufp4.QuantConfig(grid=grid, hadamard_n=n, block=16, scale_fmt=ufp4.SCALE_E4M3_X_FP32)
            q = ufp4.rht_quantize(x, ufp4.ALONG_COLS, cfg)
            s[grid, n] = ufp4.quant_stats(x, ufp4.ALONG_COLS, q)["sqnr_db"]
    E1, E2 = ufp4.GRID_E1M2, ufp4.GRID_E2M1
    assert s[E2, 0] > s[E1, 0] and s[E1, 16] > s[E2, 16]
    assert s[E1, 16] > s[E1, 0] and s[E2, 16] < s[E2, 0]


@pytest.mark.parametrize("axis", AXES)
def test_quant_stats_full_size_properties(axis):
    """dY of the layer workload (8192 x 8192, SR, two-level): every element
    counted once, no 0x8 code, level counts consistent with the codes, and
    Parseval: sum u^2 = 16 sum x^2 (x summed in fp64 by torch)."""
    dY = wl.normal(8192, 8192, 1e-3, 3)
    x = to_dev(dY)
    cfg = ufp4.QuantConfig(rounding=ufp4.ROUND_SR, sr_seed=1234, hadamard_n=16, block=16,
                           scale_fmt=ufp4.SCALE_E4M3_X_FP32)
    q = ufp4.rht_quantize(x, axis, cfg)
    st = ufp4.quant_stats(x, axis, q)
    cc = st["code_count"]
    assert sum(cc) == 8192 * 8192 and cc[8] == 0
    assert st["level_n"][0] <= cc[0] and all(st["level_n"][k] == cc[k] + cc[8 + k] for k in range(1, 8))
    x2 = torch.sum(x.double() ** 2).item()
    assert st["signal"] == pytest.approx(16 * x2, rel=1e-5)
    assert 0 < st["sqnr_db"] < 40
    assert ufp4.check_device_status() == ufp4.OK


@pytest.mark.parametrize("rows,cols", [(1, 1), (37, 300), (512, 1024)])
def test_sqnr_sums_match_oracle(rows, cols):
    rng = np.random.default_rng(rows)
    ref = rng.standard_normal((rows, cols)).astype(np.float32)
    test = (ref + 0.01 * rng.standard_normal((rows, cols))).astype(np.float32)
    pad = np.zeros((rows, cols + 5), dtype=np.float32)       # a row pitch > cols
    pad[:, :cols] = test
    r = torch.from_numpy(ref).cuda()
    t = torch.from_numpy(pad).cuda()[:, :cols]
    got = ufp4.sqnr_sums(r, t).cpu().numpy()
    want = dg.gemm_sqnr_sums(ref, test)
    assert got[0] == pytest.approx(want[0], rel=1e-12)
    assert got[1] == pytest.approx(want[1], rel=1e-12)


@pytest.mark.parametrize("axis", AXES)
@pytest.mark.parametrize("grid", [ufp4.GRID_E1M2, ufp4.GRID_E2M1, ufp4.GRID_E2M1_MAX2])
def test_quant_stats_ue8m0(axis, grid):
    """Diagnostics of MX (UE8M0, block 32) operands against the oracle."""
    X = wl.normal_with_outlier_channels(200, 136, 1.0, 3, 30.0)
    cfg = ufp4.QuantConfig(grid=grid, hadamard_n=16, block=32, scale_fmt=ufp4.SCALE_UE8M0)
    _run(X, axis, cfg)
