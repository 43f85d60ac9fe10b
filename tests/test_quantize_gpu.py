"""Parity of the fused RHT + quantize kernel with the oracle: bit-exact codes,
block scales, tensor scales and SR draws, on shapes that span several work
units and ragged tails, and on the quantizer-sweep sizes (sampled rows)."""
import itertools

import numpy as np
import pytest
import torch

import oracle
from fp4_quantized_gemms_b200 import ufp4
from fp4_quantized_gemms_b200 import workloads as wl
from tests.gpu_util import assert_quant_equal, needs_gpu, oracle_cfg, to_dev

pytestmark = needs_gpu

AXES = [ufp4.ALONG_COLS, ufp4.ALONG_ROWS]


def _run(x_bits, axis, cfg, rows=None):
    x = to_dev(x_bits)
    amax_o = 0.0
    amax_d = None
    if cfg.scale_fmt == ufp4.SCALE_E4M3_X_FP32:
        amax_o = oracle.rht_amax(x_bits, axis, cfg.hadamard_n, cfg.rht_sign_mask)
        amax_d = ufp4.rht_amax(x, axis, cfg.hadamard_n, cfg.rht_sign_mask)
        assert np.float32(amax_d.item()) == np.float32(amax_o)
    q = ufp4.rht_quantize(x, axis, cfg, tensor_amax=amax_d)
    torch.cuda.synchronize()
    oc = oracle_cfg(cfg)
    if rows is None:
        ref = oracle.quantize(x_bits, axis, oc, tensor_amax=amax_o)
    else:
        refs = [oracle.quantize(x_bits, axis, oc, tensor_amax=amax_o, r0=int(r), nr=1) for r in rows]
        ref = refs[0]
        ref.codes = np.concatenate([r.codes for r in refs])
        if ref.scales is not None:
            ref.scales = np.concatenate([r.scales for r in refs])
        else:
            ref.escales = np.concatenate([r.escales for r in refs])
    assert_quant_equal(q, ref, rows)
    return q


GRID_ROUND_FMT = list(itertools.product([ufp4.GRID_E1M2, ufp4.GRID_E2M1, ufp4.GRID_E2M1_MAX2],
                                        [ufp4.ROUND_RTNE, ufp4.ROUND_SR],
                                        [ufp4.SCALE_FP32, ufp4.SCALE_E4M3_X_FP32]))


@pytest.mark.parametrize("axis", AXES)
@pytest.mark.parametrize("n,block", [(0, 16), (16, 16), (16, 32), (32, 16), (32, 32), (64, 16),
                                     (64, 32), (0, 32)])
@pytest.mark.parametrize("grid,rounding,fmt", GRID_ROUND_FMT)
def test_quantize_matches_oracle_small(axis, n, block, grid, rounding, fmt):
    """200 x 136: ragged rows (not a multiple of 8 / 64) and a ragged K tail."""
    X = wl.student_t(200, 136, seed=11)
    cfg = ufp4.QuantConfig(grid=grid, rounding=rounding, sr_seed=1234, sr_stream=axis,
                           hadamard_n=n, block=block, scale_fmt=fmt)
    _run(X, axis, cfg)


@pytest.mark.parametrize("axis", AXES)
@pytest.mark.parametrize("grid", [ufp4.GRID_E1M2, ufp4.GRID_E2M1, ufp4.GRID_E2M1_MAX2])
def test_quantize_exact_ties_and_zero_blocks(axis, grid):
    """n = 0 with values on grid midpoints (exact RTNE ties), level values (SR
    must not move them), all-zero blocks and a block whose max is tiny."""
    rng = np.random.default_rng(3)
    lv = oracle.levels(grid)
    mids = (lv[:-1] + lv[1:]) / 2
    vals = np.concatenate([mids, lv, -mids, -lv])
    X = rng.choice(vals, size=(64, 128)).astype(np.float32) * np.float32(0.5)
    X[:, 0::16] = np.float32(lv[-1] * 0.5)          # block max = gmax * 0.5 -> s = 0.5 (exact)
    X[5, :] = 0.0
    X[9, 32:48] = 0.0
    X[11, 64:80] = np.float32(1e-30)
    X[13, 96:112] = np.float32(3e-39) * rng.integers(-5, 6, 16)   # subnormal block scale
    bits = wl.bf16_bits(X)
    for rounding in (ufp4.ROUND_RTNE, ufp4.ROUND_SR):
        cfg = ufp4.QuantConfig(grid=grid, rounding=rounding, sr_seed=7, hadamard_n=0)
        _run(bits, axis, cfg)


@pytest.mark.parametrize("axis", AXES)
def test_quantize_medium_with_outliers(axis):
    X = wl.normal_with_outlier_channels(1000, 1000, 1.0, 5, 30.0)
    for grid, rnd in [(0, 0), (0, 1), (1, 0), (2, 0), (2, 1)]:
        cfg = ufp4.QuantConfig(grid=grid, rounding=rnd, sr_seed=1234, hadamard_n=16, block=16)
        _run(X, axis, cfg)


@pytest.mark.parametrize("axis", AXES)
def test_sr_draws_independent_of_launch_shape(axis):
    """SR bits are a function of (seed, stream, output row, column) only: a
    separate call on a leading block of the output rows (a row prefix of X
    along its columns, a column prefix of X, as a strided view, along its
    rows) runs on another grid with other work units per CTA, yet gives
    exactly the codes and scales of those rows in the call on the whole
    tensor.  A different seed gives different codes."""
    X = to_dev(wl.student_t(1024, 768, seed=12))
    cfg = ufp4.QuantConfig(rounding=ufp4.ROUND_SR, sr_seed=99, sr_stream=axis, hadamard_n=32)
    full = ufp4.rht_quantize(X, axis, cfg)
    for lead in (8, 200, 520):
        part_x = X[:lead] if axis == ufp4.ALONG_COLS else X[:, :lead]
        part = ufp4.rht_quantize(part_x, axis, cfg)
        assert part.rows == lead and part.kpad == full.kpad
        assert torch.equal(part.codes, full.codes[:lead])
        assert torch.equal(part.scales[:, :lead], full.scales[:, :lead])
    other = ufp4.rht_quantize(X, axis, cfg.with_(sr_seed=100))
    assert not torch.equal(full.codes, other.codes)


@pytest.mark.parametrize("shape", wl.QUANT_SWEEP_SHAPES)
@pytest.mark.parametrize("axis", AXES)
def test_quantize_sweep_sizes_sampled(shape, axis):
    """Full quantizer-sweep sizes in the production launch; 48 sampled output
    rows (plus the first and last) checked against the oracle row by row."""
    rows, cols = shape
    X = wl.student_t(rows, cols)
    nout = rows if axis == ufp4.ALONG_COLS else cols
    rng = np.random.default_rng(rows + axis)
    sample = np.unique(np.concatenate([[0, nout - 1], rng.choice(nout, 48, replace=False)]))
    for grid, rnd, n, block in [(0, 0, 16, 16), (0, 1, 64, 32), (1, 0, 32, 16)]:
        cfg = ufp4.QuantConfig(grid=grid, rounding=rnd, sr_seed=1234, hadamard_n=n, block=block)
        _run(X, axis, cfg, rows=sample)
    cfg = ufp4.QuantConfig(hadamard_n=16, block=16, scale_fmt=ufp4.SCALE_E4M3_X_FP32)
    _run(X, axis, cfg, rows=sample)


# ------------------------------------------------------------------ dual output
def _oracle_ref(x_bits, axis, cfg, amax, rows=None):
    oc = oracle_cfg(cfg)
    if rows is None:
        return oracle.quantize(x_bits, axis, oc, tensor_amax=amax)
    refs = [oracle.quantize(x_bits, axis, oc, tensor_amax=amax, r0=int(r), nr=1) for r in rows]
    ref = refs[0]
    ref.codes = np.concatenate([r.codes for r in refs])
    if ref.scales is not None:
        ref.scales = np.concatenate([r.scales for r in refs])
    else:
        ref.escales = np.concatenate([r.escales for r in refs])
    return ref


def _run_dual(x_bits, cfg_c, cfg_r, rows_c=None, rows_r=None, with_corr=None):
    """One dual call against the oracle on both outputs (and both amaxes)."""
    x = to_dev(x_bits)
    am_c = am_r = 0.0
    am_d = None
    if cfg_c.scale_fmt == ufp4.SCALE_E4M3_X_FP32:
        am_c = oracle.rht_amax(x_bits, ufp4.ALONG_COLS, cfg_c.hadamard_n, cfg_c.rht_sign_mask)
        am_r = oracle.rht_amax(x_bits, ufp4.ALONG_ROWS, cfg_c.hadamard_n, cfg_c.rht_sign_mask)
        am_d = ufp4.rht_amax_dual(x, cfg_c.hadamard_n, cfg_c.rht_sign_mask)
        got = am_d.cpu().numpy()
        assert got[0] == np.float32(am_c) and got[1] == np.float32(am_r)
    qc, qr = ufp4.rht_quantize_dual(x, cfg_c, cfg_r, tensor_amax=am_d, with_corr=with_corr)
    torch.cuda.synchronize()
    assert ufp4.check_device_status() == ufp4.OK
    assert_quant_equal(qc, _oracle_ref(x_bits, ufp4.ALONG_COLS, cfg_c, am_c, rows_c), rows_c)
    assert_quant_equal(qr, _oracle_ref(x_bits, ufp4.ALONG_ROWS, cfg_r, am_r, rows_r), rows_r)
    return qc, qr


@pytest.mark.parametrize("n,block", [(0, 16), (16, 16), (16, 32), (32, 16), (64, 32)])
@pytest.mark.parametrize("grid,rounding,fmt", GRID_ROUND_FMT)
def test_dual_quantize_matches_oracle_small(n, block, grid, rounding, fmt):
    """300 x 600: five 64-row K segments for the row-wise output (ragged last)
    and three 256-column blocks (the last with only two of its four 64-column
    K segments inside the padded width)."""
    X = wl.student_t(300, 600, seed=13)
    cfg = ufp4.QuantConfig(grid=grid, rounding=rounding, sr_seed=1234, sr_stream=0,
                           hadamard_n=n, block=block, scale_fmt=fmt)
    _run_dual(X, cfg, cfg.with_(sr_stream=1))


def test_dual_quantize_equals_two_single_calls():
    """The dual call writes exactly what two single calls write (layer recipe:
    dY with SR, streams 0 and 1, two-level scales, correction planes)."""
    dY = wl.normal(520, 712, 1e-3, 3)
    x = to_dev(dY)
    cfg = ufp4.QuantConfig(rounding=ufp4.ROUND_SR, sr_seed=77, hadamard_n=16, block=16,
                           scale_fmt=ufp4.SCALE_E4M3_X_FP32)
    qc, qr = ufp4.rht_quantize_dual(x, cfg, cfg.with_(sr_stream=1))
    sc = ufp4.rht_quantize(x, ufp4.ALONG_COLS, cfg)
    sr = ufp4.rht_quantize(x, ufp4.ALONG_ROWS, cfg.with_(sr_stream=1))
    torch.cuda.synchronize()
    for d, s in ((qc, sc), (qr, sr)):
        # scale columns past the operand's rows (up to scale_ld) are padding
        # that neither call writes
        assert torch.equal(d.codes, s.codes)
        assert torch.equal(d.scales[:, :d.rows], s.scales[:, :s.rows])
        assert torch.equal(d.corr, s.corr) and torch.equal(d.tensor_scale, s.tensor_scale)


@pytest.mark.parametrize("shape", [wl.QUANT_SWEEP_SHAPES[0], wl.QUANT_SWEEP_SHAPES[-1]])
def test_dual_quantize_full_size_sampled(shape):
    """Quantizer-sweep sizes through the dual kernel, 40 sampled output rows of
    each result (plus the first and last) against the oracle."""
    rows, cols = shape
    X = wl.student_t(rows, cols)
    rng = np.random.default_rng(rows + cols)
    rc = np.unique(np.concatenate([[0, rows - 1], rng.choice(rows, 40, replace=False)]))
    rr = np.unique(np.concatenate([[0, cols - 1], rng.choice(cols, 40, replace=False)]))
    cfg = ufp4.QuantConfig(rounding=ufp4.ROUND_SR, sr_seed=1234, hadamard_n=16, block=16,
                           scale_fmt=ufp4.SCALE_E4M3_X_FP32)
    _run_dual(X, cfg, cfg.with_(sr_stream=1), rows_c=rc, rows_r=rr)
    cfg = ufp4.QuantConfig(hadamard_n=16, block=16)
    _run_dual(X, cfg, cfg, rows_c=rc, rows_r=rr)


# ------------------------------------------------------------------ MX block scales
@pytest.mark.parametrize("axis", AXES)
@pytest.mark.parametrize("n", [0, 16, 64])
@pytest.mark.parametrize("grid", [ufp4.GRID_E1M2, ufp4.GRID_E2M1, ufp4.GRID_E2M1_MAX2])
@pytest.mark.parametrize("rounding", [ufp4.ROUND_RTNE, ufp4.ROUND_SR])
def test_quantize_ue8m0_matches_oracle(axis, n, grid, rounding):
    """UE8M0 (MX) block scales, block 32: exponent bytes and codes bit-exact on
    a 200 x 136 outlier tensor, ragged in rows and K."""
    X = wl.normal_with_outlier_channels(200, 136, 1.0, 3, 30.0)
    cfg = ufp4.QuantConfig(grid=grid, rounding=rounding, sr_seed=321, sr_stream=axis, hadamard_n=n,
                           block=32, scale_fmt=ufp4.SCALE_UE8M0)
    _run(X, axis, cfg)


@pytest.mark.parametrize("grid", [ufp4.GRID_E1M2, ufp4.GRID_E2M1, ufp4.GRID_E2M1_MAX2])
def test_quantize_ue8m0_exponent_edges(grid):
    """Block maxima exactly at gmax * 2^k, one ulp either side, tiny (clamped
    at 2^-127), huge, and zero blocks, without RHT (n = 0) so the maxima are
    the inputs themselves."""
    gm = oracle.gmax(grid)
    rng = np.random.default_rng(7)
    rows = []
    for k in range(-120, 120, 9):
        tb = int(wl.bf16_bits(np.array([gm * 2.0 ** k], np.float32))[0])
        for bb in (tb - 1, tb, tb + 1):             # the bf16 neighbours of gmax * 2^k
            v = np.float32(wl.bf16_to_f32(np.array([bb], np.uint16))[0])
            r = rng.uniform(-1, 1, 64).astype(np.float32) * v
            r[5] = v
            r[40] = -v
            rows.append(r)
    rows.append(np.full(64, 1e-40, np.float32))
    rows.append(np.zeros(64, np.float32))
    rows.append(np.full(64, 3.0e38, np.float32))
    X = wl.bf16_bits(np.stack(rows))
    for rounding in (ufp4.ROUND_RTNE, ufp4.ROUND_SR):
        cfg = ufp4.QuantConfig(grid=grid, rounding=rounding, sr_seed=3, hadamard_n=0, block=32,
                               scale_fmt=ufp4.SCALE_UE8M0)
        _run(X, ufp4.ALONG_COLS, cfg)


# ------------------------------------------------------------------ unfused RHT
@pytest.mark.parametrize("n", [0, 16, 32, 64])
def test_rht_bf16_matches_oracle_rotation(n):
    """The unfused RHT pass equals the oracle's rotated values (the same fp32
    butterflies) rounded to bf16 with round-to-nearest-even, bit for bit, on a
    ragged row count with outlier channels and a strided input view."""
    X = wl.normal_with_outlier_channels(200, 320, 1.0, 4, 30.0)
    cfg = ufp4.QuantConfig(hadamard_n=n)
    x_full = to_dev(np.concatenate([X, np.zeros((200, 64), np.uint16)], axis=1))
    x = x_full[:, :320]                       # ld = 384, cols = 320
    y = ufp4.rht_bf16(x, n, cfg.rht_sign_mask)
    torch.cuda.synchronize()
    _, u = oracle.quantize(X, oracle.ALONG_COLS, oracle_cfg(cfg), want_u=True)
    want = wl.bf16_bits(u[:, :320])
    got = y.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)
    with pytest.raises(ufp4.UFP4Error):
        ufp4.rht_bf16(to_dev(X[:, :136]), n)          # cols not a multiple of 64
