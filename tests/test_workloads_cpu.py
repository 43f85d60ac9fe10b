"""The seeded input generators (shared by the oracle and the GPU tests) and
the MoE routing counts: determinism, shapes, and the invariants of the
water-filling count rule."""
import numpy as np

from fp4_quantized_gemms_b200 import workloads as wl


def test_generators_are_seeded_bf16():
    a = wl.normal(64, 48, 0.5, 7)
    b = wl.normal(64, 48, 0.5, 7)
    c = wl.normal(64, 48, 0.5, 8)
    assert a.dtype == np.uint16 and a.shape == (64, 48)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    x = wl.bf16_to_f32(wl.normal_with_outlier_channels(512, 256, 1.0, 4, 30.0))
    col = np.abs(x).mean(axis=0)
    assert np.sum(col > 10 * np.median(col)) == 4          # exactly the outlier channels


def test_bf16_rounding_is_nearest_even():
    v = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 0.0], dtype=np.float32)
    back = wl.bf16_to_f32(wl.bf16_bits(v))
    assert list(back) == [1.0, 1.0 + 2 * 2.0 ** -7, -2.5, 0.0]   # ties to even mantissa


def test_moe_counts_water_filling():
    s = wl.MOE
    counts = wl.moe_expert_counts(s)
    assert counts.sum() == s.tokens * s.topk
    assert counts.max() <= s.tokens and counts.min() >= 0
    assert np.array_equal(counts, wl.moe_expert_counts(s))
    # by Zipf rank the counts never increase (the seeded permutation only relabels)
    ranked = np.sort(counts)[::-1]
    w = np.arange(1, s.experts + 1, dtype=np.float64) ** (-s.zipf_s)
    free = ranked < s.tokens
    # uncapped experts follow the Zipf weights to within one row
    ratio = ranked[free] / w[free]
    assert ratio.max() - ratio.min() <= (1.0 / w[free]).max()
    starts, padded, total = wl.padded_offsets(counts)
    assert np.all(starts % 64 == 0) and np.all(padded >= counts) and np.all(padded - counts < 64)
    assert total == padded.sum() and starts[-1] + padded[-1] == total
