"""Parity of the three training GEMMs with the oracle.

The CUDA path (GPU quantize -> GPU GEMM) and the oracle path (oracle quantize
-> fp64 contraction of the dequantized operands) start from the same seeded
bf16 inputs; the GPU's codes are checked bit-exactly and its fp32 output
within GEMM_RTOL relative Frobenius error of the fp64 result."""
import numpy as np
import pytest
import torch

import oracle
from fp4_quantized_gemms_b200 import ufp4
from fp4_quantized_gemms_b200 import workloads as wl
from tests.gpu_util import (GEMM_RTOL, assert_quant_equal, needs_gpu, oracle_cfg, rel_fro,
                            to_dev)

pytestmark = needs_gpu

C, R = ufp4.ALONG_COLS, ufp4.ALONG_ROWS


def _quant_both(bits, axis, cfg, rows=None, with_elems8=None):
    """GPU and oracle quantization of the same operand (optionally only some
    output rows on the oracle side)."""
    x = to_dev(bits)
    amax_d, amax_o = None, 0.0
    if cfg.scale_fmt == ufp4.SCALE_E4M3_X_FP32:
        amax_d = ufp4.rht_amax(x, axis, cfg.hadamard_n, cfg.rht_sign_mask)
        amax_o = oracle.rht_amax(bits, axis, cfg.hadamard_n, cfg.rht_sign_mask)
    q = ufp4.rht_quantize(x, axis, cfg, tensor_amax=amax_d, with_elems8=with_elems8)
    oc = oracle_cfg(cfg)
    if rows is None:
        ref = oracle.quantize(bits, axis, oc, tensor_amax=amax_o)
    else:
        parts = [oracle.quantize(bits, axis, oc, tensor_amax=amax_o, r0=int(r), nr=1) for r in rows]
        ref = parts[0]
        ref.codes = np.concatenate([p.codes for p in parts])
        if ref.scales is not None:
            ref.scales = np.concatenate([p.scales for p in parts])
        else:
            ref.escales = np.concatenate([p.escales for p in parts])
    return q, ref


def _check_full(qa, ra, qb, rb, fn):
    out = fn(qa, qb)
    torch.cuda.synchronize()
    assert ufp4.check_device_status() == ufp4.OK
    assert_quant_equal(qa, ra)
    assert_quant_equal(qb, rb)
    ref = oracle.gemm_tn(ra, rb)
    got = out.cpu().numpy()
    assert got.shape == ref.shape
    err = rel_fro(got, ref)
    assert err <= GEMM_RTOL, err
    return err


def _cfg(grid=0, fmt=0, n=16, block=16, rounding=0, stream=0):
    return ufp4.QuantConfig(grid=grid, rounding=rounding, sr_seed=1234, sr_stream=stream,
                            hadamard_n=n, block=block, scale_fmt=fmt)


@pytest.mark.parametrize("grid", [ufp4.GRID_E1M2, ufp4.GRID_E2M1, ufp4.GRID_E2M1_MAX2])
@pytest.mark.parametrize("fmt", [ufp4.SCALE_FP32, ufp4.SCALE_E4M3_X_FP32])
def test_fprop_tiny_config(grid, fmt):
    """X 256x512 with 4 outlier columns x20, W 512x512 ~ N(0, 0.02), RHT16, block 16."""
    X, W, _ = wl.layer_inputs(wl.TINY, want_dy=False)
    cfg = _cfg(grid=grid, fmt=fmt)
    qx, rx = _quant_both(X, C, cfg)
    qw, rw = _quant_both(W, C, cfg)
    _check_full(qx, rx, qw, rw, ufp4.gemm_fprop)


@pytest.mark.parametrize("M,N,K", [(300, 200, 200), (128, 256, 64), (1, 1, 8), (129, 257, 136),
                                   (640, 520, 1000)])
@pytest.mark.parametrize("fmt", [ufp4.SCALE_FP32, ufp4.SCALE_E4M3_X_FP32])
@pytest.mark.parametrize("grid,n,block", [(0, 16, 16), (1, 32, 32), (0, 64, 32), (1, 0, 16),
                                          (0, 0, 32)])
def test_fprop_ragged_shapes(M, N, K, fmt, grid, n, block):
    """Partial M / N tiles, K tails padded inside the quantizer, degenerate sizes."""
    X = wl.normal_with_outlier_channels(M, K, 1.0, min(2, K), 20.0)
    W = wl.normal(N, K, 0.02, 2)
    cfg = _cfg(grid=grid, fmt=fmt, n=n, block=block)
    qx, rx = _quant_both(X, C, cfg)
    qw, rw = _quant_both(W, C, cfg)
    _check_full(qx, rx, qw, rw, ufp4.gemm_fprop)


@pytest.mark.parametrize("fmt", [ufp4.SCALE_FP32, ufp4.SCALE_E4M3_X_FP32])
@pytest.mark.parametrize("grid", [ufp4.GRID_E1M2, ufp4.GRID_E2M1, ufp4.GRID_E2M1_MAX2])
def test_layer_dgrad_wgrad_small(fmt, grid):
    """The full recipe on a small layer: RHT on every operand along its GEMM's
    K, RTNE for X / W, SR on dY (stream 0 for DGRAD, 1 for WGRAD).  With the
    restricted E2M1 grid this is the full-RHT max_fpx = 2.0 ablation."""
    M, K, N = 384, 320, 264
    X = wl.normal_with_outlier_channels(M, K, 1.0, 3, 30.0)
    W = wl.normal(N, K, 0.02, 2)
    dY = wl.normal(M, N, 1e-3, 3)
    rtne, sr0, sr1 = _cfg(grid=grid, fmt=fmt), _cfg(grid=grid, fmt=fmt, rounding=1, stream=0), \
        _cfg(grid=grid, fmt=fmt, rounding=1, stream=1)
    qdy, rdy = _quant_both(dY, C, sr0)          # [M, N], K = N
    qwt, rwt = _quant_both(W, R, rtne)          # W^T [K, N]
    _check_full(qdy, rdy, qwt, rwt, ufp4.gemm_dgrad)
    qdyt, rdyt = _quant_both(dY, R, sr1)        # dY^T [N, M]
    qxt, rxt = _quant_both(X, R, rtne)          # X^T [K, M]
    _check_full(qdyt, rdyt, qxt, rxt, ufp4.gemm_wgrad)


def _sampled(shape: wl.LayerShape, fmt, grid, gemm, n_rows=96, n_cols=96, block=16):
    """One GEMM of a full-size layer in the production launch; the oracle
    computes a sampled row x column block of the output."""
    X, W, dY = wl.layer_inputs(shape, want_dy=True)
    rng = np.random.default_rng(17)
    if gemm == "fprop":
        a_bits, a_axis, a_cfg = X, C, _cfg(grid=grid, fmt=fmt, block=block)
        b_bits, b_axis, b_cfg = W, C, _cfg(grid=grid, fmt=fmt, block=block)
        fn = ufp4.gemm_fprop
    elif gemm == "dgrad":
        a_bits, a_axis, a_cfg = dY, C, _cfg(grid=grid, fmt=fmt, rounding=1, stream=0, block=block)
        b_bits, b_axis, b_cfg = W, R, _cfg(grid=grid, fmt=fmt, block=block)
        fn = ufp4.gemm_dgrad
    else:
        a_bits, a_axis, a_cfg = dY, R, _cfg(grid=grid, fmt=fmt, rounding=1, stream=1, block=block)
        b_bits, b_axis, b_cfg = X, R, _cfg(grid=grid, fmt=fmt, block=block)
        fn = ufp4.gemm_wgrad
    ma = a_bits.shape[0] if a_axis == C else a_bits.shape[1]
    nb = b_bits.shape[0] if b_axis == C else b_bits.shape[1]
    ii = np.unique(np.concatenate([[0, ma - 1], rng.choice(ma, n_rows, replace=False)]))
    jj = np.unique(np.concatenate([[0, nb - 1], rng.choice(nb, n_cols, replace=False)]))
    qa, ra = _quant_both(a_bits, a_axis, a_cfg, rows=ii)
    qb, rb = _quant_both(b_bits, b_axis, b_cfg, rows=jj)
    out = fn(qa, qb)
    torch.cuda.synchronize()
    assert ufp4.check_device_status() == ufp4.OK
    assert_quant_equal(qa, ra, ii)
    assert_quant_equal(qb, rb, jj)
    ref = oracle.gemm_tn(ra, rb)                       # [len(ii), len(jj)]
    got = out[torch.as_tensor(ii, device="cuda")][:, torch.as_tensor(jj, device="cuda")].cpu().numpy()
    err = rel_fro(got, ref)
    assert err <= GEMM_RTOL, err
    return err


@pytest.mark.parametrize("gemm", ["fprop", "dgrad", "wgrad"])
@pytest.mark.parametrize("fmt", [ufp4.SCALE_FP32, ufp4.SCALE_E4M3_X_FP32, ufp4.SCALE_UE8M0])
def test_layer_config_sampled(gemm, fmt):
    """X 8192x2048 (10 outlier channels x30), W 8192x2048, dY 8192x8192
    (MX scales: block 32, the block-scaled FP8 path)."""
    _sampled(wl.LAYER, fmt, ufp4.GRID_E1M2, gemm, block=32 if fmt == ufp4.SCALE_UE8M0 else 16)


@pytest.mark.parametrize("gemm", ["fprop", "dgrad", "wgrad"])
@pytest.mark.parametrize("fmt,grid", [(ufp4.SCALE_E4M3_X_FP32, ufp4.GRID_E1M2),
                                      (ufp4.SCALE_FP32, ufp4.GRID_E1M2),
                                      (ufp4.SCALE_E4M3_X_FP32, ufp4.GRID_E2M1),
                                      (ufp4.SCALE_UE8M0, ufp4.GRID_E1M2)])
def test_large_config_sampled(gemm, fmt, grid):
    """M=16384, K=8192, N=28672 (1% outlier channels x50): the largest layer."""
    _sampled(wl.LARGE, fmt, grid, gemm, n_rows=64, n_cols=64,
             block=32 if fmt == ufp4.SCALE_UE8M0 else 16)


@pytest.mark.parametrize("path", [ufp4.GEMM_PATH_NATIVE_FP4, ufp4.GEMM_PATH_NATIVE_FP4_PAIR256])
@pytest.mark.parametrize("corr", [True, False])
@pytest.mark.parametrize("grid", [ufp4.GRID_E1M2, ufp4.GRID_E2M1, ufp4.GRID_E2M1_MAX2])
def test_two_level_kernel_families(path, corr, grid):
    """Every kernel family for two-level scales gives the oracle's result, with
    the E1M2 correction planes stored by the quantizer or derived in the GEMM;
    shapes with partial tiles in M, N (224-wide tiles) and a K tail."""
    if grid != ufp4.GRID_E1M2 and corr:
        pytest.skip("correction planes exist for E1M2 only")
    old = ufp4.get_two_level_gemm_path()
    ufp4.set_two_level_gemm_path(path)
    try:
        for (M, N, K) in [(520, 700, 448), (130, 230, 200)]:
            X = wl.normal_with_outlier_channels(M, K, 1.0, 2, 20.0)
            W = wl.normal(N, K, 0.02, 2)
            cfg = _cfg(grid=grid, fmt=ufp4.SCALE_E4M3_X_FP32)
            x, w = to_dev(X), to_dev(W)
            qx = ufp4.rht_quantize(x, C, cfg, with_corr=corr)
            qw = ufp4.rht_quantize(w, C, cfg, with_corr=corr)
            oc = oracle_cfg(cfg)
            rx = oracle.quantize(X, C, oc, tensor_amax=oracle.rht_amax(X, C, 16, cfg.rht_sign_mask))
            rw = oracle.quantize(W, C, oc, tensor_amax=oracle.rht_amax(W, C, 16, cfg.rht_sign_mask))
            assert (qx.corr is not None) == corr
            _check_full(qx, rx, qw, rw, ufp4.gemm_fprop)
    finally:
        ufp4.set_two_level_gemm_path(old)


@pytest.mark.parametrize("grid,fmt,block", [
    (ufp4.GRID_E1M2, ufp4.SCALE_E4M3_X_FP32, 16), (ufp4.GRID_E1M2, ufp4.SCALE_E4M3_X_FP32, 32),
    (ufp4.GRID_E2M1, ufp4.SCALE_E4M3_X_FP32, 16), (ufp4.GRID_E2M1_MAX2, ufp4.SCALE_E4M3_X_FP32, 32),
    (ufp4.GRID_E1M2, ufp4.SCALE_UE8M0, 32)])
def test_factor_atoms_path_equals_factor_warps(grid, fmt, block):
    """Dense CTA-pair GEMMs whose operands carry factor atoms (the MMA issuer
    copies them into tensor memory) give bit-for-bit the output of the same
    kernel building the factors from the block-major scales, and the
    oracle's result; partial 256-wide tiles, one-row operands, K tails of 64
    and of 128 + 64 (E2M1 stages 256 K: tails of 64, 192 and 256).  E1M2
    operands also carry per-lane factor tiles, which the kernel uses for A:
    A with and without them gives the same bits too."""
    import dataclasses
    cfg = _cfg(grid=grid, fmt=fmt, block=block)
    for (M, N, K) in [(520, 700, 448), (130, 230, 200), (1, 1, 8), (300, 513, 1000)]:
        X = wl.normal_with_outlier_channels(M, K, 1.0, 2, 20.0)
        W = wl.normal(N, K, 0.02, 2)
        qx, rx = _quant_both(X, C, cfg)
        qw, rw = _quant_both(W, C, cfg)
        assert qx.sf_atoms is not None and qw.sf_atoms is not None
        _check_full(qx, rx, qw, rw, ufp4.gemm_fprop)
        with_atoms = ufp4.gemm_fprop(qx, qw)
        plain = ufp4.gemm_fprop(dataclasses.replace(qx, sf_atoms=None), dataclasses.replace(qw, sf_atoms=None))
        if qx.sf_lanes is not None:
            no_lanes = ufp4.gemm_fprop(dataclasses.replace(qx, sf_lanes=None), qw)
            torch.cuda.synchronize()
            assert torch.equal(with_atoms, no_lanes), (M, N, K)
        torch.cuda.synchronize()
        assert ufp4.check_device_status() == ufp4.OK
        assert torch.equal(with_atoms, plain), (M, N, K)


@pytest.mark.parametrize("fmt", [ufp4.SCALE_FP32, ufp4.SCALE_E4M3_X_FP32])
def test_e2m1_reference_recipe_layer(fmt):
    """The comparison recipe of the pages (E2M1 grid, RHT on the WGRAD
    operands only, SR on dY, RTNE elsewhere): all three GEMMs of a small
    layer against the oracle."""
    M, K, N = 384, 320, 264
    X = wl.normal_with_outlier_channels(M, K, 1.0, 3, 30.0)
    W = wl.normal(N, K, 0.02, 2)
    dY = wl.normal(M, N, 1e-3, 3)
    plain = _cfg(grid=ufp4.GRID_E2M1, fmt=fmt, n=0)
    sr_plain = _cfg(grid=ufp4.GRID_E2M1, fmt=fmt, n=0, rounding=1, stream=0)
    rot = _cfg(grid=ufp4.GRID_E2M1, fmt=fmt, n=16)
    sr_rot = _cfg(grid=ufp4.GRID_E2M1, fmt=fmt, n=16, rounding=1, stream=1)
    qx, rx = _quant_both(X, C, plain)
    qw, rw = _quant_both(W, C, plain)
    _check_full(qx, rx, qw, rw, ufp4.gemm_fprop)
    qdy, rdy = _quant_both(dY, C, sr_plain)
    qwt, rwt = _quant_both(W, R, plain)
    _check_full(qdy, rdy, qwt, rwt, ufp4.gemm_dgrad)
    qdyt, rdyt = _quant_both(dY, R, sr_rot)
    qxt, rxt = _quant_both(X, R, rot)
    _check_full(qdyt, rdyt, qxt, rxt, ufp4.gemm_wgrad)


# ------------------------------------------------------------------ MX block scales
@pytest.mark.parametrize("grid,e8", [(ufp4.GRID_E1M2, True), (ufp4.GRID_E1M2, False),
                                     (ufp4.GRID_E2M1, False), (ufp4.GRID_E2M1_MAX2, False)])
def test_ue8m0_gemms(grid, e8):
    """UE8M0 (MX, block 32) operands: E1M2 with E4M3 element planes on the
    block-scaled FP8 MMA (factors in the MMA), otherwise through the
    fp32-scale kernel.  FPROP on ragged shapes (partial 256-wide tiles, K
    tails of 64), and DGRAD / WGRAD of a small layer with SR on dY."""
    for (M, N, K) in [(300, 200, 200), (129, 257, 136), (1, 1, 8), (520, 700, 448)]:
        X = wl.normal_with_outlier_channels(M, K, 1.0, 2, 20.0)
        W = wl.normal(N, K, 0.02, 2)
        cfg = _cfg(grid=grid, fmt=ufp4.SCALE_UE8M0, block=32)
        qx, rx = _quant_both(X, C, cfg, with_elems8=e8)
        qw, rw = _quant_both(W, C, cfg, with_elems8=e8)
        assert (qx.elems8 is not None) == e8
        _check_full(qx, rx, qw, rw, ufp4.gemm_fprop)
    M, K, N = 384, 320, 264
    X = wl.normal_with_outlier_channels(M, K, 1.0, 3, 30.0)
    W = wl.normal(N, K, 0.02, 2)
    dY = wl.normal(M, N, 1e-3, 3)
    rt = _cfg(grid=grid, fmt=ufp4.SCALE_UE8M0, block=32)
    sr0 = _cfg(grid=grid, fmt=ufp4.SCALE_UE8M0, block=32, rounding=1, stream=0)
    sr1 = _cfg(grid=grid, fmt=ufp4.SCALE_UE8M0, block=32, rounding=1, stream=1)
    qdy, rdy = _quant_both(dY, C, sr0, with_elems8=e8)
    qwt, rwt = _quant_both(W, R, rt, with_elems8=e8)
    _check_full(qdy, rdy, qwt, rwt, ufp4.gemm_dgrad)
    qdyt, rdyt = _quant_both(dY, R, sr1, with_elems8=e8)
    qxt, rxt = _quant_both(X, R, rt, with_elems8=e8)
    _check_full(qdyt, rdyt, qxt, rxt, ufp4.gemm_wgrad)
