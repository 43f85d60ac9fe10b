"""Pins of the oracle's quantization diagnostics (CPU).

Each check compares ``oracle.diagnostics`` with something it does not compute
itself: Parseval's identity and the inverse transform (scipy's Hadamard
matrix), the uniform-quantizer noise law, the conditional bias printed on the
pages (``tests/golden``), hand-built inputs with known codes, and a closed-form
SQNR of a scaled copy.
"""
import numpy as np
import pytest
import scipy.linalg

import oracle
from oracle import diagnostics as dg
from fp4_quantized_gemms_b200 import workloads as wl
from tests.conftest import read_golden

E1M2, E2M1, MAX2 = oracle.GRID_E1M2, oracle.GRID_E2M1, oracle.GRID_E2M1_MAX2
C = oracle.ALONG_COLS


def _quant(X, **kw):
    cfg = oracle.QuantCfg(**kw)
    amax = 0.0
    if cfg.scale_fmt == oracle.SCALE_E4M3_X_FP32:
        amax = oracle.rht_amax(X, C, cfg.hadamard_n, cfg.sign_mask)
    return oracle.quantize(X, C, cfg, tensor_amax=amax, want_u=True)


@pytest.mark.parametrize("grid", [E1M2, E2M1, MAX2])
@pytest.mark.parametrize("n", [16, 32, 64])
def test_signal_and_noise_match_the_original_domain(grid, n):
    """Parseval: sum u^2 = n sum x^2, and the noise measured on u equals n times
    the noise of x against the inverse-transformed dequantized values
    (x_hat = D H deq / n with scipy's Hadamard matrix)."""
    X = wl.normal_with_outlier_channels(24, 4 * n, 1.0, 2, 20.0)
    mask = 0x9E3779B97F4A7C15 & ((1 << n) - 1)
    q, u = _quant(X, grid=grid, hadamard_n=n, sign_mask=mask, block=16)
    st = dg.quant_stats(q, u)
    x = wl.bf16_to_f32(X).astype(np.float64)
    assert st["signal"] == pytest.approx(n * np.sum(x * x), rel=1e-6)
    H = scipy.linalg.hadamard(n).astype(np.float64)
    d = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(n)])
    deq = q.dequantize()[:, :x.shape[1]].reshape(x.shape[0], -1, n)
    x_hat = (deq @ H.T) * d / n                   # D H deq / n per block (H symmetric)
    noise_x = np.sum((x.reshape(x_hat.shape) - x_hat) ** 2)
    assert st["noise"] == pytest.approx(n * noise_x, rel=1e-4)


def test_uniform_grid_noise_law():
    """E1M2 without RHT on uniform inputs with every block maximum 1: the step
    is 1/7, every bin (the half-bins at 0 and at the top included) has error
    variance step^2 / 12, and the block maxima are exact, so the noise is
    (15/16) N step^2 / 12 (a closed form, to 0.05 dB)."""
    rng = np.random.default_rng(8)
    x = rng.uniform(-1, 1, (512, 256)).astype(np.float32)
    x[:, ::16] = 1.0                               # every block maximum is exactly 1
    X = wl.bf16_bits(x)
    q, u = _quant(X, grid=E1M2, hadamard_n=0, block=16)
    st = dg.quant_stats(q, u)
    step = 1.0 / 7.0                               # 1.75 / 7 per unit block max
    xb = wl.bf16_to_f32(X).astype(np.float64)
    signal = np.sum(xb * xb)
    noise = (xb.size * 15 / 16) * step ** 2 / 12   # the maxima carry no error
    assert st["signal"] == signal
    assert dg.sqnr_db(st["signal"], st["noise"]) == pytest.approx(dg.sqnr_db(signal, noise), abs=0.05)


def test_level_error_reproduces_the_printed_shrinkage_bias():
    """RTNE of values spread uniformly over each E2M1 bin: the mean signed
    error per level is (l - r)/2, -0.125 at level 2 (printed on the pages) and
    -0.25 at level 4; zero at the interior E1M2 levels."""
    g = read_golden("shrinkage_bias_e2m1.txt")
    rng = np.random.default_rng(4)
    for grid, checks in ((E2M1, {4: float(g["conditional_bias"]), 6: -0.25, 2: 0.0}),
                         (E1M2, {2: 0.0, 4: 0.0, 6: 0.0})):
        gm = oracle.gmax(grid)
        x = rng.uniform(0, gm, (2048, 256)).astype(np.float32)
        x[:, ::16] = gm                            # step = 1 exactly (power of two)
        q, u = _quant(wl.bf16_bits(x), grid=grid, hadamard_n=0, block=16)
        sm = dg.summary(dg.quant_stats(q, u))
        lv = list(oracle.levels(grid))
        for k, want in checks.items():
            # bf16 inputs put only ~50 values in a bin (8-bit mantissa), and
            # ties at its edges go to the even level: up to ~1e-2 of bias
            assert sm["level_mean_err"][k] == pytest.approx(want, abs=1e-2), (grid, lv[k])


def test_counts_on_hand_built_blocks():
    """Blocks of one large value and fifteen tiny ones: the tiny values all
    underflow to code 0, the large one takes the top code; counts are exact."""
    x = np.full((8, 64), 1e-4, dtype=np.float32)
    x[:, ::16] = -3.0
    x[3, 16:32] = 0.0                              # one all-zero block
    X = wl.bf16_bits(x)
    for grid in (E1M2, E2M1, MAX2):
        q, u = _quant(X, grid=grid, hadamard_n=0, block=16)
        st = dg.quant_stats(q, u)
        top = len(oracle.levels(grid)) - 1
        assert st["code_count"][8 + top] == 8 * 4 - 1
        assert st["code_count"][0] == 8 * 64 - (8 * 4 - 1)
        assert st["code_count"].sum() == 8 * 64 and st["code_count"][8] == 0
        assert st["nonzero"] == 8 * 64 - 16
        assert st["underflow"] == 8 * 64 - 16 - (8 * 4 - 1)
        assert st["level_n"][0] == 8 * 64 - 16 - (8 * 4 - 1)     # zero block excluded
        sm = dg.summary(st)
        assert sm["bucket_ratio"] == pytest.approx(2 / st["grid_codes"])


def test_padding_columns_are_not_counted():
    X = wl.normal(16, 72, 1.0, 5)                  # kpad 128: 56 padded zeros per row
    q, u = _quant(X, grid=E1M2, hadamard_n=16, block=16)
    st = dg.quant_stats(q, u)
    assert st["code_count"].sum() == 16 * 72


def test_rht_flips_the_grid_ranking_on_outlier_tensors():
    """The qualitative claim of the pages' diagnostics on a synthetic
    outlier-heavy tensor: E2M1 leads E1M2 before rotation, E1M2 leads after,
    and the RHT raises E1M2's SQNR while it lowers E2M1's."""
    X = wl.normal_with_outlier_channels(256, 1024, 1.0, 8, 30.0)
    s = {}
    for grid in (E1M2, E2M1):
        for n in (0, 16):
            q, u = _quant(X, grid=grid, hadamard_n=n, sign_mask=0x5EED, block=16)
            s[grid, n] = dg.summary(dg.quant_stats(q, u))["sqnr_db"]
    assert s[E2M1, 0] > s[E1M2, 0] and s[E1M2, 16] > s[E2M1, 16]
    assert s[E1M2, 16] > s[E1M2, 0] and s[E2M1, 16] < s[E2M1, 0]


def test_gemm_sqnr_of_a_scaled_copy():
    """test = ref (1 + eps) has SQNR exactly -20 log10(eps)."""
    rng = np.random.default_rng(2)
    ref = rng.standard_normal((64, 48))
    sig, noi = dg.gemm_sqnr_sums(ref, ref * (1 + 2.0 ** -10))
    assert dg.sqnr_db(sig, noi) == pytest.approx(-20 * np.log10(2.0 ** -10), abs=1e-9)
