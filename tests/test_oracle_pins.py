"""Pins of the CPU oracle against what the pages and the mathematics fix.

Every test here runs without a GPU.  None of them retypes an oracle formula:
each compares the oracle with a closed form, an invariant, a library routine,
a value printed on the pages (``tests/golden``) or exact brute force
(``fractions.Fraction``).
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg

import oracle
from fp4_quantized_gemms_b200 import workloads as wl
from tests.conftest import read_golden

E1M2, E2M1, MAX2 = oracle.GRID_E1M2, oracle.GRID_E2M1, oracle.GRID_E2M1_MAX2
ALL_GRIDS = [E1M2, E2M1, MAX2]


# ------------------------------------------------------------------ RHT (C1)
@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64])
def test_fwht_reproduces_sylvester_matrix(n):
    """P2: the butterflies applied to unit vectors give H_n with
    H[i][j] = (-1)^popcount(i & j), which is also scipy's Sylvester construction."""
    H = np.stack([oracle.fwht_f64(np.eye(n)[j]) for j in range(n)], axis=1)
    closed = np.array([[(-1) ** bin(i & j).count("1") for j in range(n)] for i in range(n)])
    assert np.array_equal(H, closed)
    assert np.array_equal(H, scipy.linalg.hadamard(n))
    # P1: H^T H = n I exactly (integer arithmetic)
    Hi = H.astype(np.int64)
    assert np.array_equal(Hi.T @ Hi, n * np.eye(n, dtype=np.int64))


@pytest.mark.parametrize("n", [16, 32, 64])
def test_rht_norm_preservation_and_inverse(n):
    """P2/P3: ||H D x||^2 = n ||x||^2; x = D H (H D x) / n."""
    rng = np.random.default_rng(7)
    for _ in range(20):
        x = rng.standard_normal(n)
        d = np.where(rng.integers(0, 2, n) == 1, -1.0, 1.0)
        u = oracle.fwht_f64(d * x)
        assert np.isclose(u @ u, n * (x @ x), rtol=1e-13)
        back = d * oracle.fwht_f64(u) / n
        assert np.allclose(back, x, rtol=0, atol=1e-13)


@pytest.mark.parametrize("n", [16, 32, 64])
def test_rht_cancels_in_gemm(n):
    """P4: (A D H)(B D H)^T / n = A B^T with H applied block-diagonally along K."""
    rng = np.random.default_rng(11)
    M, N, K = 5, 7, 4 * n
    A = rng.standard_normal((M, K))
    B = rng.standard_normal((N, K))
    d = np.where(rng.integers(0, 2, n) == 1, -1.0, 1.0)

    def rot(X):
        out = np.empty_like(X)
        for r in range(X.shape[0]):
            for b0 in range(0, K, n):
                out[r, b0:b0 + n] = oracle.fwht_f64(d * X[r, b0:b0 + n])
        return out

    assert np.allclose(rot(A) @ rot(B).T / n, A @ B.T, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("n", [16, 32, 64])
def test_fwht_f32_matches_exact_transform(n):
    """fp32 butterflies: exact on small integers, within n*2^-24 relative otherwise."""
    rng = np.random.default_rng(3)
    ints = rng.integers(-1000, 1000, n).astype(np.float64)
    assert np.array_equal(oracle.fwht_f32(ints).astype(np.float64), oracle.fwht_f64(ints))
    x = rng.standard_normal(n).astype(np.float32)
    f32 = oracle.fwht_f32(x).astype(np.float64)
    f64 = oracle.fwht_f64(x.astype(np.float64))
    scale = np.abs(x).astype(np.float64).sum()
    assert np.max(np.abs(f32 - f64)) <= n * 2.0 ** -24 * scale


# ------------------------------------------------------------------ grids (C2)
def test_e1m2_grid_is_uniform():
    """P5: E1M2 levels are equally spaced, so l_i = r_i at every interior level."""
    lv = oracle.levels(E1M2)
    assert np.all(np.diff(lv) == 0.25)
    assert lv[0] == 0.0 and oracle.gmax(E1M2) == 1.75


def test_e2m1_range_restricted_prefix_matches_pages():
    """P7: the pages' range-restricted set (max_fpx = 2.0) is the E2M1 prefix."""
    g = read_golden("e2m1_range_restricted.txt")
    printed = [float(v) for v in g["levels"].split(",")]
    lv = oracle.levels(E2M1)
    assert list(lv[lv <= float(g["max_fpx"])]) == printed
    assert oracle.gmax(E2M1) == 6.0
    # the restricted grid itself: exactly the printed set, topped at max_fpx,
    # with the E2M1 code points (code k means the same magnitude in both)
    assert list(oracle.levels(MAX2)) == printed
    assert oracle.gmax(MAX2) == float(g["max_fpx"]) and oracle.top_code(MAX2) == 4
    assert list(oracle.levels(MAX2)) == list(lv[:5])


def test_e2m1_range_restricted_grid_is_uniform():
    """The restricted set is uniform (step 0.5): no geometric asymmetry, so no
    conditional RTNE bias at its interior levels (checked by Monte Carlo below)."""
    assert np.all(np.diff(oracle.levels(MAX2)) == 0.5)


def _half_widths(grid, i):
    lv = oracle.levels(grid)
    return (lv[i] - lv[i - 1]) / 2, (lv[i + 1] - lv[i]) / 2


def test_shrinkage_bias_worked_example_matches_pages():
    """P6: the printed E2M1 example (q=2: widths 0.25 / 0.5, bias -0.125)."""
    g = read_golden("shrinkage_bias_e2m1.txt")
    lv = list(oracle.levels(E2M1))
    i = lv.index(float(g["level"]))
    left, right = _half_widths(E2M1, i)
    assert left == float(g["left_width"]) and right == float(g["right_width"])
    assert (left - right) / 2 == float(g["conditional_bias"])


@pytest.mark.parametrize("grid,level,expect", [
    (E2M1, 0.5, 0.0), (E2M1, 1.0, 0.0), (E2M1, 1.5, 0.0), (E2M1, 2.0, -0.125),
    (E2M1, 3.0, 0.0), (E2M1, 4.0, -0.25),
    (E1M2, 0.25, 0.0), (E1M2, 0.5, 0.0), (E1M2, 0.75, 0.0), (E1M2, 1.0, 0.0),
    (E1M2, 1.25, 0.0), (E1M2, 1.5, 0.0),
    (MAX2, 0.5, 0.0), (MAX2, 1.0, 0.0), (MAX2, 1.5, 0.0),
])
def test_rtne_conditional_bias_monte_carlo(grid, level, expect):
    """P6: uniform draws inside the RTNE bin of a level, rounded by the oracle,
    have mean error (l - r)/2: negative ("Shrinkage Bias") for E2M1 at 2 and 4,
    zero for every interior E1M2 level."""
    lv = list(oracle.levels(grid))
    i = lv.index(level)
    left, right = _half_widths(grid, i)
    assert (left - right) / 2 == expect
    rng = np.random.default_rng(1000 + i + 10 * grid)
    nsamp = 1_000_000
    x = rng.uniform(level - left, level + right, nsamp)
    k = oracle.round_rtne(grid, x, 1.0)
    q = oracle.levels(grid)[k]
    err = q - x
    sigma = err.std() / np.sqrt(nsamp)
    assert abs(err.mean() - expect) < 5 * sigma + 1e-12


# ------------------------------------------------------------------ rounding (C4, C5)
def _brute_rtne(grid, u, s):
    """argmin over all 15 codes of |u - s*lvl(c)|, exact rationals, ties to the
    even magnitude index, canonical zero."""
    uf, sf = Fraction(u), Fraction(s)
    lv = [Fraction(v) for v in oracle.levels(grid)]
    best = None
    for k in range(len(lv)):
        for sign in (1, -1):
            if k == 0 and sign == -1:
                continue
            d = abs(uf - sign * sf * lv[k])
            key = (d, k % 2)  # smaller distance, then even index
            if best is None or key < best[0]:
                best = (key, k, sign)
    return best[1]


@pytest.mark.parametrize("grid", ALL_GRIDS)
def test_rtne_matches_brute_force_sweep(grid):
    """P9: dense sweep of |u|/s across every bin, exact ties and both edges."""
    lv = oracle.levels(grid)
    s = 2.0 ** -3  # power of two: every midpoint * s is an fp32 value
    mids = (lv[:-1] + lv[1:]) / 2
    pts = []
    for m in mids:
        t = np.float32(m * s)
        pts += [t, np.nextafter(t, np.float32(0)), np.nextafter(t, np.float32(1e9))]
    pts += list(np.float32(np.linspace(0, 1.2 * lv[-1] * s, 4001)))
    pts = np.array(pts, dtype=np.float32).astype(np.float64)
    got = oracle.round_rtne(grid, pts, s)
    want = [_brute_rtne(grid, float(p), s) for p in pts]
    assert list(got) == want


@pytest.mark.parametrize("grid", ALL_GRIDS)
def test_rtne_matches_brute_force_random_blocks(grid):
    """P9 on random 16-blocks with non-power-of-two fp32 scales."""
    rng = np.random.default_rng(5)
    for _ in range(200):
        u = rng.standard_normal(16).astype(np.float32)
        amax = np.float32(np.abs(u).max())
        s = np.float32(amax / np.float32(oracle.gmax(grid)))
        got = oracle.round_rtne(grid, np.abs(u).astype(np.float64), float(s))
        want = [_brute_rtne(grid, float(abs(v)), float(s)) for v in u]
        assert list(got) == want
        # P8: the block maximum maps to gmax (no clipping)
        assert got.max() == len(oracle.levels(grid)) - 1


@pytest.mark.parametrize("grid", ALL_GRIDS)
def test_sr_is_unbiased_over_seeds(grid):
    """P10: the mean of SR-dequantized values over 2^20 seeds equals x within
    Delta*2^-16 + 4 sigma; P11: every result is one of the two adjacent levels."""
    lv = oracle.levels(grid)
    rng = np.random.default_rng(17 + grid)
    seeds = np.arange(1 << 20, dtype=np.uint64)
    for lo in [0, 2, 4, 5] if grid != MAX2 else [0, 1, 2, 3]:
        x = rng.uniform(lv[lo], lv[lo + 1])
        delta = lv[lo + 1] - lv[lo]
        r16 = oracle.sr_u16_over_seeds(seeds, 0, 12345)
        k = oracle.round_sr(grid, np.full(seeds.size, x), 1.0, r16)
        assert set(np.unique(k)) <= {lo, lo + 1}
        q = lv[k]
        sigma = q.std() / np.sqrt(seeds.size)
        assert abs(q.mean() - x) <= delta * 2.0 ** -16 + 4 * sigma


@pytest.mark.parametrize("grid", ALL_GRIDS)
def test_sr_never_moves_values_on_a_level(grid):
    """P12: a value exactly on a level stays there for every uniform draw."""
    lv = oracle.levels(grid)
    r16 = np.arange(65536, dtype=np.uint32)
    for k in range(len(lv)):
        got = oracle.round_sr(grid, np.full(r16.size, lv[k] * 0.375), 0.375, r16)
        assert np.all(got == k)


def test_sr_uniforms_are_uniform():
    """The 16-bit draws behave like uniforms (chi-square over 256 cells, and no
    repeated 64-element windows between two streams)."""
    L = np.arange(1 << 18, dtype=np.uint64)
    r = oracle.sr_u16(1234, 0, L)
    hist = np.bincount(r >> 8, minlength=256)
    expected = L.size / 256
    chi2 = ((hist - expected) ** 2 / expected).sum()
    assert chi2 < 256 + 6 * np.sqrt(2 * 256)
    r1 = oracle.sr_u16(1234, 1, L)
    assert np.mean(r == r1) < 1e-3
    assert np.all(r < 65536)


# ------------------------------------------------------------------ scales (C3, C6)
def test_e4m3_conversion_matches_torch():
    """The OCP E4M3 conversion agrees with torch's float8_e4m3fn cast (a library
    routine) on every fp32 value of a dense sweep within range, and saturates."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(9)
    xs = np.concatenate([
        np.exp2(rng.uniform(-12, np.log2(448.0), 200_000)),
        np.array([oracle.e4m3_value(b) for b in range(0x7F)]),           # exact values
        np.array([(oracle.e4m3_value(b) + oracle.e4m3_value(b + 1)) / 2  # exact ties
                  for b in range(0x7E)]),
    ]).astype(np.float32)
    ours = oracle.e4m3(xs)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    assert np.all(oracle.e4m3(np.array([448.0, 460.0, 1e6], np.float32)) == 0x7E)
    assert oracle.e4m3_value(0x7E) == 448.0 and oracle.e4m3_value(1) == 2.0 ** -9


def test_e4m3_times_e1m2_code_is_exact_in_bf16():
    """C6 pin: e_b * lvl is representable in bf16 for every E4M3 block scale
    and every E1M2 / E2M1 level (what lets a 16-bit MMA take it exactly)."""
    for grid in (E1M2, E2M1):
        for b in range(0x7F):
            for lvl in oracle.levels(grid):
                v = np.float32(oracle.e4m3_value(b) * lvl)
                bits = wl.bf16_bits(np.array([v]))
                assert wl.bf16_to_f32(bits)[0] == v


# ------------------------------------------------------------------ whole operand
def _cfg(**kw):
    return oracle.QuantCfg(**kw)


@pytest.mark.parametrize("grid", ALL_GRIDS)
@pytest.mark.parametrize("axis", [oracle.ALONG_COLS, oracle.ALONG_ROWS])
def test_quantize_structure(grid, axis):
    """Canonical zero, |k| <= 7, fp32 scale = RN(amax/gmax) of the rotated block,
    every nonzero block reaches gmax (P8), padding is zero."""
    X = wl.normal_with_outlier_channels(40, 72, 1.0, 2, 20.0)
    cfg = _cfg(grid=grid, hadamard_n=16, sign_mask=0xB3A5, block=16)
    q, u = oracle.quantize(X, axis, cfg, want_u=True)
    K = 72 if axis == oracle.ALONG_COLS else 40
    assert q.kpad == (128 if K == 72 else 64) and q.k == K
    top = len(oracle.levels(grid)) - 1
    assert not np.any(q.codes == 8)
    assert np.all((q.codes & 7) <= top)
    nb = q.kpad // 16
    amax = np.abs(u.reshape(u.shape[0], nb, 16)).max(axis=2)
    want = (amax / np.float32(oracle.gmax(grid))).astype(np.float32)
    assert np.array_equal(q.scales, want)
    mags = (q.codes & 7).reshape(q.codes.shape[0], nb, 16).max(axis=2)
    assert np.all(mags[amax > 0] == top)
    assert np.all(u[:, ((K + 15) // 16) * 16:] == 0)


@pytest.mark.parametrize("grid", [E1M2, E2M1])
def test_gemm_oracle_equals_numpy_matmul(grid):
    """P13: the fp64 contraction equals numpy's float64 matmul of the same
    dequantized operands (times 1/n)."""
    X = wl.normal_with_outlier_channels(24, 100, 1.0, 2, 20.0)
    W = wl.normal(16, 100, 0.02, 2)
    cfg = _cfg(grid=grid, hadamard_n=32, sign_mask=0x1234ABCD, block=32)
    a = oracle.quantize(X, oracle.ALONG_COLS, cfg)
    b = oracle.quantize(W, oracle.ALONG_COLS, cfg)
    C = oracle.gemm_tn(a, b)
    A, B = a.dequantize(), b.dequantize()
    ref = A @ B.T / 32
    # both sum exact fp64 products; they may differ only by summation order
    bound = 2 * A.shape[1] * 2.0 ** -53 * (np.abs(A) @ np.abs(B).T) / 32
    assert np.all(np.abs(C - ref) <= bound)
    ii = np.array([0, 5, 23]); jj = np.array([15, 0, 7])
    assert np.array_equal(oracle.gemm_tn_entries(a, b, ii, jj), C[ii, jj])


def test_gemm_oracle_exact_on_grid_values():
    """P14: with n = 0 and operands already on the E1M2 grid with power-of-two
    block maxima, quantization is lossless and the oracle GEMM is the exact
    integer GEMM."""
    rng = np.random.default_rng(21)
    M, N, K = 12, 9, 128
    def on_grid(rows):
        k = rng.integers(-7, 8, (rows, K))
        k[:, ::16] = 7                                   # every block reaches gmax
        e = rng.integers(-4, 5, (rows, K // 16)).repeat(16, axis=1)
        return k, (k / 4.0) * np.exp2(e)
    ka, A = on_grid(M)
    kb, B = on_grid(N)
    cfg = _cfg(grid=E1M2, hadamard_n=0, block=16)
    qa = oracle.quantize(wl.bf16_bits(A.astype(np.float32)), oracle.ALONG_COLS, cfg)
    qb = oracle.quantize(wl.bf16_bits(B.astype(np.float32)), oracle.ALONG_COLS, cfg)
    assert np.array_equal(qa.dequantize(), A) and np.array_equal(qb.dequantize(), B)
    exact = np.array([[sum(Fraction(float(A[i, t])) * Fraction(float(B[j, t])) for t in range(K))
                       for j in range(N)] for i in range(M)], dtype=object)
    C = oracle.gemm_tn(qa, qb)
    assert all(Fraction(float(C[i, j])) == exact[i, j] for i in range(M) for j in range(N))


@pytest.mark.parametrize("grid", ALL_GRIDS)
@pytest.mark.parametrize("scale_fmt", [oracle.SCALE_FP32, oracle.SCALE_E4M3_X_FP32, oracle.SCALE_UE8M0])
def test_quantized_gemm_tracks_bf16_gemm(grid, scale_fmt):
    """End to end: the oracle's quantized FPROP approximates the fp64 X W^T of
    the bf16 inputs to 4-bit accuracy.  A dropped 1/n, a sign mask on one side
    only or a transposed operand all fail this by orders of magnitude."""
    X = wl.normal_with_outlier_channels(64, 256, 1.0, 4, 20.0)
    W = wl.normal(48, 256, 0.02, 2)
    block = 32 if scale_fmt == oracle.SCALE_UE8M0 else 16      # MX blocks are 32 long
    cfg = _cfg(grid=grid, hadamard_n=16, sign_mask=0x5EED, block=block, scale_fmt=scale_fmt)
    amx = oracle.rht_amax(X, oracle.ALONG_COLS, 16, 0x5EED)
    amw = oracle.rht_amax(W, oracle.ALONG_COLS, 16, 0x5EED)
    a = oracle.quantize(X, oracle.ALONG_COLS, cfg, tensor_amax=amx)
    b = oracle.quantize(W, oracle.ALONG_COLS, cfg, tensor_amax=amw)
    C = oracle.gemm_tn(a, b)
    ref = wl.bf16_to_f32(X).astype(np.float64) @ wl.bf16_to_f32(W).astype(np.float64).T
    rel = np.linalg.norm(C - ref) / np.linalg.norm(ref)
    # power-of-two block scales leave the block maximum anywhere in
    # (gmax/2, gmax]: with the 5-level restricted grid that costs ~0.29
    bound = 0.35 if (grid == MAX2 and scale_fmt == oracle.SCALE_UE8M0) else 0.25
    assert rel < bound
    if scale_fmt == oracle.SCALE_E4M3_X_FP32:
        assert a.escales.max() <= 0x7E and a.S > 0


def test_two_level_scales_follow_hierarchy():
    """C6: S from the rotated tensor amax; the largest block lands near the top of
    E4M3 (<= 448) and dequantized blocks stay within half a grid step."""
    X = wl.student_t(32, 256)
    cfg = _cfg(grid=E1M2, hadamard_n=16, sign_mask=0x5EED, block=16,
               scale_fmt=oracle.SCALE_E4M3_X_FP32)
    amax = oracle.rht_amax(X, oracle.ALONG_COLS, 16, 0x5EED)
    q, u = oracle.quantize(X, oracle.ALONG_COLS, cfg, tensor_amax=amax, want_u=True)
    assert q.S == np.float32(amax / np.float32(784.0))
    top = max(oracle.e4m3_value(b) for b in np.unique(q.escales))
    assert 384.0 <= top <= 448.0
    deq = q.dequantize()
    e = np.array([[oracle.e4m3_value(b) for b in row] for row in q.escales]).repeat(16, axis=1)
    top_level = 1.75 * e * q.S
    sat = np.abs(u) > top_level
    assert np.all(np.abs(deq[sat]) == top_level[sat])
    step = e * q.S * 0.25
    assert np.all(np.abs(deq - u)[~sat] <= step[~sat] / 2 * (1 + 1e-6))


# ------------------------------------------------------------------ restricted E2M1
def test_restricted_e2m1_rounding_is_scaled_e1m2_rounding_capped():
    """The restricted levels are 2x the E1M2 levels of codes 0..4, so rounding
    |u| at scale s onto them must pick the E1M2 code of |u| at scale 2s, capped
    at 4 (both rules are exact-quotient; both break ties to even codes).  A
    wrong top code, a stale loop bound or a missed saturation fails this."""
    rng = np.random.default_rng(33)
    s = 0.375
    au = np.concatenate([rng.uniform(0, 3.0 * s, 200_000),
                         s * np.arange(0, 2.5, 0.25)])           # levels and midpoints
    want = np.minimum(oracle.round_rtne(E1M2, au, 2 * s), 4)
    assert np.array_equal(oracle.round_rtne(MAX2, au, s), want)
    r16 = rng.integers(0, 65536, au.size).astype(np.uint32)
    got = oracle.round_sr(MAX2, au, s, r16)
    inside = au <= 2.0 * s
    assert np.array_equal(got[inside], oracle.round_sr(E1M2, au[inside], 2 * s, r16[inside]))
    assert np.all(got[~inside] == 4)


def test_restricted_e2m1_block_maximum_is_exact():
    """P8 with max_fpx = 2.0: the fp32 scale is amax/2 (exact), so the element
    that sets the block maximum dequantizes to itself, code 4."""
    X = wl.normal_with_outlier_channels(16, 64, 1.0, 2, 20.0)
    cfg = _cfg(grid=MAX2, hadamard_n=16, sign_mask=0x9A3C, block=16)
    q, u = oracle.quantize(X, oracle.ALONG_COLS, cfg, want_u=True)
    deq = q.dequantize()
    blocks = np.abs(u).reshape(u.shape[0], -1, 16)
    arg = blocks.argmax(axis=2)
    r = np.arange(u.shape[0])[:, None]
    c = np.arange(blocks.shape[1])[None, :] * 16 + arg
    assert np.array_equal(np.abs(deq[r, c]), blocks.max(axis=2).astype(np.float64))
    assert np.all((q.codes[r, c] & 7) == 4)


def test_restricted_e2m1_two_level_tensor_scale():
    """Two-level scales with max_fpx = 2.0: S maps the rotated tensor amax to
    2.0 x 448; blocks whose E4M3 factor rounds down saturate at code 4."""
    X = wl.student_t(32, 256)
    cfg = _cfg(grid=MAX2, hadamard_n=16, sign_mask=0x5EED, block=16,
               scale_fmt=oracle.SCALE_E4M3_X_FP32)
    amax = oracle.rht_amax(X, oracle.ALONG_COLS, 16, 0x5EED)
    q, u = oracle.quantize(X, oracle.ALONG_COLS, cfg, tensor_amax=amax, want_u=True)
    assert q.S == np.float32(amax / np.float32(896.0))
    assert np.all((q.codes & 7) <= 4)
    e = np.array([[oracle.e4m3_value(b) for b in row] for row in q.escales]).repeat(16, axis=1)
    top_level = 2.0 * e * q.S
    deq = q.dequantize()
    sat = np.abs(u) > top_level
    assert np.all(np.abs(deq[sat]) == top_level[sat])
    assert np.all(np.abs(deq - u)[~sat] <= (0.25 * e * q.S)[~sat] * (1 + 1e-6))


# ------------------------------------------------------------------ MX block scales
def _ue8m0_closed_form(gmax: float, amax: float) -> int:
    """X = e_a - e_g + (m_a > m_g) from frexp mantissas (both in [0.5, 1)):
    the smallest X with amax <= gmax 2^X, then clamped; 0 for amax = 0."""
    if amax == 0:
        return 0
    ma, ea = math.frexp(amax)
    mg, eg = math.frexp(gmax)
    X = ea - eg + (1 if ma > mg else 0)
    return min(max(X, -127), 127) + 127


@pytest.mark.parametrize("grid", ALL_GRIDS)
def test_ue8m0_scale_matches_closed_form(grid):
    """The MX scale byte against the frexp closed form, on random magnitudes,
    exact multiples of gmax by powers of two and their fp32 neighbours, and
    the clamped ends (subnormal and huge block maxima)."""
    rng = np.random.default_rng(41 + grid)
    gm = oracle.gmax(grid)
    vals = list(np.float32(np.exp2(rng.uniform(-140, 127, 3000))))
    for k in range(-130, 126, 7):
        t = np.float32(gm * 2.0 ** k)
        vals += [t, np.nextafter(t, np.float32(0)), np.nextafter(t, np.float32(np.inf))]
    vals += [np.float32(1e-45), np.float32(3.4e38), np.float32(0)]
    for v in vals:
        v = float(v)
        assert oracle.ue8m0_scale(grid, v) == _ue8m0_closed_form(gm, v), (grid, v)
    assert oracle.ue8m0_value(127) == 1.0 and oracle.ue8m0_value(0) == 2.0 ** -127


@pytest.mark.parametrize("grid", ALL_GRIDS)
@pytest.mark.parametrize("rounding", [oracle.ROUND_RTNE, oracle.ROUND_SR])
def test_ue8m0_quantize_structure(grid, rounding):
    """MX blocks of 32: every scale a power of two with the block maximum in
    (gmax/2, gmax] of it (no clipping, tight), RTNE within half a step, and
    block 16 rejected."""
    X = wl.normal_with_outlier_channels(48, 256, 1.0, 3, 30.0)
    cfg = _cfg(grid=grid, rounding=rounding, sr_seed=5, hadamard_n=16, sign_mask=0x5EED, block=32,
               scale_fmt=oracle.SCALE_UE8M0)
    q, u = oracle.quantize(X, oracle.ALONG_COLS, cfg, want_u=True)
    assert q.scales is None and q.escales.shape == (48, 256 // 32)
    s = np.ldexp(1.0, q.escales.astype(np.int64) - 127)
    amax = np.abs(u.astype(np.float64)).reshape(48, -1, 32).max(axis=2)
    gm = oracle.gmax(grid)
    nz = amax > 0
    assert np.all(amax[nz] <= gm * s[nz]) and np.all(amax[nz] > gm * s[nz] / 2)
    deq = q.dequantize()
    step = np.repeat(s, 32, axis=1)
    if rounding == oracle.ROUND_RTNE:
        lv = oracle.levels(grid)
        half = np.max(np.diff(lv)) / 2
        assert np.all(np.abs(deq - u) <= half * step * (1 + 1e-12))
    with pytest.raises(ValueError):
        oracle.quantize(X, oracle.ALONG_COLS, _cfg(grid=grid, block=16, scale_fmt=oracle.SCALE_UE8M0))


# ------------------------------------------------------------------ rotated amax and the row-wise view
def _rotated_f64(X_bits: np.ndarray, axis: int, n: int, mask: int) -> np.ndarray:
    """u = H_n D x of every row of the operand's K-major view, computed
    independently of the oracle: scipy's Sylvester matrix times the sign-
    flipped block, in fp64, with K zero-padded to a multiple of 64."""
    x = wl.bf16_to_f32(X_bits).astype(np.float64)
    if axis == oracle.ALONG_ROWS:
        x = x.T
    rows, K = x.shape
    kp = (K + 63) // 64 * 64
    v = np.zeros((rows, kp))
    v[:, :K] = x
    if n == 0:
        return v
    d = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(n)])
    H = scipy.linalg.hadamard(n).astype(np.float64)
    blocks = v.reshape(rows, kp // n, n) * d
    return (blocks @ H.T).reshape(rows, kp)


@pytest.mark.parametrize("n", [0, 16, 32, 64])
@pytest.mark.parametrize("axis", [oracle.ALONG_COLS, oracle.ALONG_ROWS])
def test_rht_amax_matches_independent_hadamard(n, axis):
    """The oracle's rotated tensor amax equals max |H_n D x| from scipy's
    Hadamard matrix in fp64, to the fp32 butterflies' error bound, on a
    non-square tensor with outlier channels (there the rotated amax differs
    from the raw amax and from the other axis's, so an amax taken before the
    rotation, along the wrong axis or over part of the blocks fails)."""
    mask = 0x09F1FD9D03F0A9B4
    X = wl.normal_with_outlier_channels(72, 136, 1.0, 3, 30.0)
    got = oracle.rht_amax(X, axis, n, mask)
    u = _rotated_f64(X, axis, n, mask)
    want = np.abs(u).max()
    x = wl.bf16_to_f32(X).astype(np.float64)
    xa = np.abs(x.T if axis == oracle.ALONG_ROWS else x)
    # |fp32 butterflies - exact| <= n 2^-24 sum|x| over the block (see the
    # fp32 FWHT pin above); the largest block sum bounds every block
    kp = u.shape[1]
    pad = np.zeros((xa.shape[0], kp))
    pad[:, :xa.shape[1]] = xa
    bsum = pad.reshape(pad.shape[0], -1, max(n, 1)).sum(axis=2).max() if n else 0.0
    assert abs(got - want) <= n * 2.0 ** -24 * bsum
    if n == 0:
        assert got == np.float32(np.abs(x).max())
    else:
        raw = np.abs(x).max()
        other = np.abs(_rotated_f64(X, 1 - axis, n, mask)).max()
        margin = n * 2.0 ** -24 * bsum
        assert abs(want - raw) > 10 * margin and abs(want - other) > 10 * margin


@pytest.mark.parametrize("grid", ALL_GRIDS)
@pytest.mark.parametrize("rounding", [oracle.ROUND_RTNE, oracle.ROUND_SR])
@pytest.mark.parametrize("scale_fmt", [oracle.SCALE_FP32, oracle.SCALE_E4M3_X_FP32, oracle.SCALE_UE8M0])
def test_quantize_along_rows_is_transpose_of_along_cols(grid, rounding, scale_fmt):
    """Quantizing X along its rows (the strided dimension, output transposed)
    gives exactly what quantizing the explicit transpose along its columns
    gives: codes, scales, tensor scale and the SR draws (both index the draws
    by output row and column).  With a non-square X whose row count is not a
    multiple of 64, a mix-up of row pitch and row count, a missing transpose or
    a draw index taken from the input layout fails this."""
    X = wl.normal_with_outlier_channels(100, 72, 1.0, 3, 25.0)
    XT = np.ascontiguousarray(X.T)
    block = 32 if scale_fmt == oracle.SCALE_UE8M0 else 16
    cfg = _cfg(grid=grid, rounding=rounding, sr_seed=1234, sr_stream=1, hadamard_n=16,
               sign_mask=0x09F1FD9D03F0A9B4, block=block, scale_fmt=scale_fmt)
    am_r = oracle.rht_amax(X, oracle.ALONG_ROWS, 16, cfg.sign_mask)
    am_c = oracle.rht_amax(XT, oracle.ALONG_COLS, 16, cfg.sign_mask)
    assert am_r == am_c
    a, ua = oracle.quantize(X, oracle.ALONG_ROWS, cfg, tensor_amax=am_r, want_u=True)
    b, ub = oracle.quantize(XT, oracle.ALONG_COLS, cfg, tensor_amax=am_c, want_u=True)
    assert a.k == b.k == 100 and a.kpad == b.kpad == 128 and a.codes.shape == (72, 128)
    assert np.array_equal(ua, ub)
    assert np.array_equal(a.codes, b.codes)
    if scale_fmt == oracle.SCALE_FP32:
        assert np.array_equal(a.scales, b.scales)
    else:
        assert np.array_equal(a.escales, b.escales)
    assert a.S == b.S
    # the transposed view really is the other axis: quantizing X along its
    # columns gives a different operand
    c = oracle.quantize(X, oracle.ALONG_COLS, cfg,
                        tensor_amax=oracle.rht_amax(X, oracle.ALONG_COLS, 16, cfg.sign_mask))
    assert c.codes.shape == (100, 128)


@pytest.mark.parametrize("grid", ALL_GRIDS)
@pytest.mark.parametrize("scale_fmt", [oracle.SCALE_FP32, oracle.SCALE_E4M3_X_FP32])
def test_quantized_backward_gemms_track_bf16_gemms(grid, scale_fmt):
    """End to end for the two backward GEMMs, with the recipe's operands:
    DGRAD dX = dY W from dY along its columns (SR, stream 0) and W along its
    rows; WGRAD dW = dY^T X from dY (SR, stream 1) and X both along their rows.
    Each approximates the fp64 product of the bf16 inputs to 4-bit accuracy; a
    transposed operand, a row-wise read along the wrong axis or a missing 1/n
    is off by orders of magnitude."""
    M, K, N = 128, 96, 80
    X = wl.normal_with_outlier_channels(M, K, 1.0, 3, 20.0)
    W = wl.normal(N, K, 0.02, 2)
    dY = wl.normal(M, N, 1e-3, 3)
    mask = 0x5EED
    base = dict(grid=grid, hadamard_n=16, sign_mask=mask, block=16, scale_fmt=scale_fmt)
    rt = _cfg(**base)
    sr0 = _cfg(rounding=oracle.ROUND_SR, sr_seed=1234, sr_stream=0, **base)
    sr1 = _cfg(rounding=oracle.ROUND_SR, sr_seed=1234, sr_stream=1, **base)
    C, R = oracle.ALONG_COLS, oracle.ALONG_ROWS

    def q(bits, axis, cfg):
        return oracle.quantize(bits, axis, cfg, tensor_amax=oracle.rht_amax(bits, axis, 16, mask))

    f = lambda b: wl.bf16_to_f32(b).astype(np.float64)  # noqa: E731
    dX = oracle.gemm_tn(q(dY, C, sr0), q(W, R, rt))
    dW = oracle.gemm_tn(q(dY, R, sr1), q(X, R, rt))
    ref_dX = f(dY) @ f(W)
    ref_dW = f(dY).T @ f(X)
    assert dX.shape == ref_dX.shape == (M, K) and dW.shape == ref_dW.shape == (N, K)
    # measured 0.14-0.17 (E1M2, E2M1) and 0.25-0.26 for the 5-level restricted grid
    bound = 0.35 if grid == MAX2 else 0.22
    for got, ref in ((dX, ref_dX), (dW, ref_dW)):
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert rel < bound, rel
