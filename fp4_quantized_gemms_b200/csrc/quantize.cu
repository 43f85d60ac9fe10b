// quantize.cu -- fused RHT + block absmax + scale + 4-bit rounding + packing
// (ufp4_rht_quantize) and the rotated-domain tensor amax (ufp4_rht_amax).
//
// Method: arXiv 2606.20381, paperlayer.ai summary §2 "Random Hadamard
// transforms", "Blockwise quantization", "Rounding rules"; §4 UFP4 recipe;
// gist.science "Efficiëntie" (RHT fused with the quantizer).
//
// Work decomposition.  A warp owns a 64-long segment of the reduction
// dimension K for 8 output rows (row-wise, K contiguous) or for 64 output rows
// (column-wise, K strided: the operand is transposed on the fly).  Inside a
// warp, lane = 4*g + j: j picks the 16-element chunk [16j, 16j+16) of the
// segment, so a 32- or 64-point Hadamard block spans lanes j^1 / j^2 and is
// finished with shuffles.  Every lane holds whole 16-element chunks in
// registers: loads are 16-byte vectors, coalesced along K (row-wise) or along
// the contiguous input columns (column-wise), the "transpose" is free because
// each bf16 is widened to fp32 individually anyway.
//
// Exactness.  The butterflies are the same fp32 adds in the same stage order
// as the definition; every rounding decision compares |u| with
// (threshold * m1) * b by one fma, whose sign is exact (threshold * m1 is an
// exact fp32 value, b the fp32 scale), so codes match the exact-quotient rule
// bit for bit.  An fp32 estimate picks the candidate; the fma tests fix it.

#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define UFP4_PIPELINE_KERNELS 1
#include "ufp4_device.cuh"
#include "ufp4_internal.h"

namespace ufp4 {

namespace {

constexpr int kThreads = 256;

// Grids: 0 = E1M2 (levels k/4, k <= 7), 1 = E2M1 (OCP FP4 magnitudes),
// 2 = E2M1 restricted to max_fpx = 2.0 (the E2M1 codes 0..4, levels k/2).
// Grids 0 and 2 are uniform: level k = k / kUnit.
template <int GRID>
constexpr int top_of() { return GRID == 2 ? 4 : 7; }
template <int GRID>
constexpr float unit_of() { return GRID == 0 ? 4.0f : 2.0f; }

template <int GRID>
__device__ __forceinline__ float level_of(int k) {
    if (GRID != 1) return static_cast<float>(k) * (1.0f / unit_of<GRID>());
    return k <= 4 ? static_cast<float>(k) * 0.5f : (k == 5 ? 3.0f : (k == 6 ? 4.0f : 6.0f));
}

// Midpoint between level j and level j+1 (j < top), exact in fp32.
template <int GRID>
__device__ __forceinline__ float mid_of(int j) {
    if (GRID != 1) return static_cast<float>(2 * j + 1) * (0.5f / unit_of<GRID>());
    return j <= 3 ? static_cast<float>(2 * j + 1) * 0.25f
                  : (j == 4 ? 2.5f : (j == 5 ? 3.5f : 5.0f));
}

template <int GRID>
__device__ __forceinline__ float gmax_of() {
    return GRID == 0 ? 1.75f : (GRID == 1 ? 6.0f : 2.0f);
}

// Nearest level index of an approximate quotient y (within one of the truth).
template <int GRID>
__device__ __forceinline__ int estimate_nearest(float y) {
    if (GRID != 1) return min(max(__float2int_rn(y * unit_of<GRID>()), 0), top_of<GRID>());
    return (y > 0.25f) + (y > 0.75f) + (y > 1.25f) + (y > 1.75f) + (y > 2.5f) + (y > 3.5f) +
           (y > 5.0f);
}

// Largest level index whose level is <= y (approximate, within one).
template <int GRID>
__device__ __forceinline__ int estimate_floor(float y) {
    if (GRID != 1) return min(max(__float2int_rd(y * unit_of<GRID>()), 0), top_of<GRID>());
    return (y >= 0.5f) + (y >= 1.0f) + (y >= 1.5f) + (y >= 2.0f) + (y >= 3.0f) + (y >= 4.0f) +
           (y >= 6.0f);
}

// sign(au - t * m1 * b), exact: t * m1 is an exact fp32 product.
__device__ __forceinline__ float exact_diff(float au, float t, float m1, float b) {
    return __fmaf_rn(-(t * m1), b, au);
}

// RTNE on the exact quotient au / (m1 * b), ties to the even index,
// saturating at gmax.  [PL] §2 "Rounding rules".
template <int GRID>
__device__ __forceinline__ int round_rtne(float au, float m1, float b, float inv) {
    if (!(fabsf(inv) < INFINITY)) {
        // Subnormal step: no usable reciprocal, count the boundaries passed.
        int k = 0;
#pragma unroll
        for (int j = 0; j < top_of<GRID>(); ++j) {
            const float d = exact_diff(au, mid_of<GRID>(j), m1, b);
            if (d > 0.0f || (d == 0.0f && (j & 1))) k = j + 1;
        }
        return k;
    }
    int k = estimate_nearest<GRID>(au * inv);
    if (k > 0) {
        const float d = exact_diff(au, mid_of<GRID>(k - 1), m1, b);
        if (d < 0.0f || (d == 0.0f && (k & 1))) --k;
    }
    if (k < top_of<GRID>()) {
        const float d = exact_diff(au, mid_of<GRID>(k), m1, b);
        if (d > 0.0f || (d == 0.0f && (k & 1))) ++k;
    }
    return k;
}

// Stochastic rounding between the adjacent levels lo <= au/s < hi: up iff
// au > (lo + r16 * 2^-16 * (hi - lo)) * s.
template <int GRID>
__device__ __forceinline__ int round_sr(float au, float m1, float b, float inv, uint32_t r16) {
    int lo;
    if (!(fabsf(inv) < INFINITY)) {
        lo = 0;
#pragma unroll
        for (int j = 1; j <= top_of<GRID>(); ++j)
            if (exact_diff(au, level_of<GRID>(j), m1, b) >= 0.0f) lo = j;
    } else {
        lo = estimate_floor<GRID>(au * inv);
        if (lo > 0 && exact_diff(au, level_of<GRID>(lo), m1, b) < 0.0f) {
            --lo;
        } else if (lo < top_of<GRID>() && exact_diff(au, level_of<GRID>(lo + 1), m1, b) >= 0.0f) {
            ++lo;
        }
    }
    if (lo >= top_of<GRID>()) return top_of<GRID>();
    const float l0 = level_of<GRID>(lo);
    const float step = level_of<GRID>(lo + 1) - l0;
    const float c = __fmaf_rn(static_cast<float>(r16), step * (1.0f / 65536.0f), l0);
    return exact_diff(au, c, m1, b) > 0.0f ? lo + 1 : lo;
}


// Reciprocal for the fp32 estimate only (every decision it feeds is either
// certified by the 2^-16 margin or re-decided exactly): rcp.approx has at
// most 1 ulp error; a subnormal argument flushes to zero and gives +inf,
// which sends the block to the exact path.
__device__ __forceinline__ float approx_rcp(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

struct ScaleOut {
    float m1;    // factor folded into the threshold (1 or e_b)
    float b;     // fp32 scale multiplied inside the fma (s or S)
    float inv;   // approximate 1 / (m1 * b) for the estimate
    bool zero;   // block step is zero: every code 0
    uint32_t stored;  // fp32 bits of s, or the E4M3 byte
};

// MX block-scale exponent: the smallest X with amax <= gmax * 2^X, clamped to
// [-127, 127] (-127 for amax = 0).  With amax = ma 2^ea and gmax = mg 2^eg
// (mantissas in [1, 2)) it is ea - eg, plus one when ma > mg; the comparison
// is exact on the scaled-down mantissas.
template <int GRID>
__device__ __forceinline__ int ue8m0_exponent(float amax) {
    if (!(amax > 0.0f)) return -127;
    const int ea = ilogbf(amax);
    const int eg = GRID == 0 ? 0 : (GRID == 1 ? 2 : 1);     // 1.75, 6 = 1.5 * 4, 2 = 1 * 2
    const float mg = GRID == 0 ? 1.75f : (GRID == 1 ? 1.5f : 1.0f);
    const float ma = ldexpf(amax, -ea);                      // exact, in [1, 2)
    const int X = ea - eg + (ma > mg ? 1 : 0);
    return X < -127 ? -127 : (X > 127 ? 127 : X);
}

template <int GRID>
__device__ __forceinline__ ScaleOut block_scale(float amax, int scale_fmt, float S, float G) {
    ScaleOut o;
    if (scale_fmt == 2) {
        // power-of-two step: every quotient |u| / 2^X is exact
        const int X = ue8m0_exponent<GRID>(amax);
        o.m1 = 1.0f;
        o.b = ldexpf(1.0f, X);
        o.zero = !(amax > 0.0f);
        o.inv = ldexpf(1.0f, -X);
        o.stored = static_cast<uint32_t>(X + 127);
        return o;
    }
    if (scale_fmt == 0) {
        const float s = __fdiv_rn(amax, gmax_of<GRID>());
        o.m1 = 1.0f;
        o.b = s;
        o.zero = !(s > 0.0f);
        o.inv = o.zero ? 0.0f : approx_rcp(s);
        o.stored = __float_as_uint(s);
    } else {
        const float q = __fdiv_rn(amax, G);
        const __nv_fp8_storage_t e8 = __nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3);
        const float e = e4m3_to_f32(e8);
        o.m1 = e;
        o.b = S;
        o.zero = !(e > 0.0f);
        o.inv = o.zero ? 0.0f : approx_rcp(e * S);
        o.stored = e8;
    }
    return o;
}

// Keeps the sign bit of a nibble only when its magnitude is nonzero, for
// the 8 nibbles of a word at once (mag + 7 sets bit 3 iff mag >= 1, and never
// carries into the next nibble).  Zero is always coded 0x0.
__device__ __forceinline__ uint32_t canonical_zero(uint32_t w) {
    const uint32_t mag = w & 0x77777777u;
    return w & (0x77777777u | ((mag + 0x77777777u) & 0x88888888u));
}

// x + 1.5*2^23 rounds x to an integer (ties to even) in the low mantissa bits.
constexpr float kRound = 12582912.0f;
// A candidate closer than this (in units of the grid step) to a decision
// boundary is re-decided by the exact path.  The estimate's error is below
// 2^-20 steps (two roundings of a quotient below 8).
constexpr float kMargin = 1.0f / 65536.0f;

// E2M1 RTNE of (b, a) -> one byte, low nibble = a (OCP FP4 encoding, sign kept).
__device__ __forceinline__ uint32_t cvt_e2m1x4(float a0, float a1, float a2, float a3, float a4,
                                               float a5, float a6, float a7) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(a0), "f"(a1), "f"(a2), "f"(a3), "f"(a4), "f"(a5), "f"(a6), "f"(a7));
    return out;
}

// The 16 values and 8 random words of a chunk, passed by value so that the
// out-of-line exact path below keeps them in registers.
struct Chunk16 {
    float4 v0, v1, v2, v3;
};
// Where a chunk's SR words come from: Philox key (seed) and counter base.
struct RandSrc {
    uint64_t seed;
    uint64_t L0;
    uint32_t stream;
};

// Exact path: every element decided by the fma boundary tests.
template <int GRID, int RND>
__device__ __noinline__ uint2 round_pack_exact(const Chunk16 c, const ScaleOut sc, const RandSrc src) {
    const float v[16] = {c.v0.x, c.v0.y, c.v0.z, c.v0.w, c.v1.x, c.v1.y, c.v1.z, c.v1.w,
                         c.v2.x, c.v2.y, c.v2.z, c.v2.w, c.v3.x, c.v3.y, c.v3.z, c.v3.w};
    // the chunk's SR words again (this path is rare)
    uint32_t rnd[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (RND == 1) {
        const PhiloxKeys keys = philox_keys(src.seed);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint64_t g = (src.L0 >> 3) + h;
            const uint4 r = philox4x32_10(
                make_uint4(static_cast<uint32_t>(g), static_cast<uint32_t>(g >> 32), src.stream, 0u), keys);
            rnd[4 * h] = r.x, rnd[4 * h + 1] = r.y, rnd[4 * h + 2] = r.z, rnd[4 * h + 3] = r.w;
        }
    }
    uint32_t w0 = 0, w1 = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float u = v[i];
        const float au = fabsf(u);
        int k;
        if (RND == 0) {
            k = round_rtne<GRID>(au, sc.m1, sc.b, sc.inv);
        } else {
            const uint32_t word = rnd[i >> 1];
            const uint32_t r16 = (i & 1) ? (word >> 16) : (word & 0xFFFFu);
            k = round_sr<GRID>(au, sc.m1, sc.b, sc.inv, r16);
        }
        const uint32_t code = static_cast<uint32_t>(k) | ((__float_as_uint(u) >> 28) & 8u);
        if (i < 8) w0 |= code << (4 * i);
        else w1 |= code << (4 * (i - 8));
    }
    return make_uint2(canonical_zero(w0), canonical_zero(w1));
}

// Round the 16 rotated values of one chunk and pack them (2 codes / byte,
// low nibble = lower K index).  A certified fast path decides each element
// from an fp32 estimate of |u|/s; when any element of the chunk lies within
// kMargin of a decision boundary the chunk is re-decided exactly, so the
// result always equals the exact-quotient rule.
template <int GRID, int RND>
__device__ __forceinline__ uint2 round_pack(const float (&v)[16], const ScaleOut &sc,
                                            const PhiloxKeys &keys, uint32_t stream, uint64_t L0,
                                            uint64_t seed) {
    uint32_t rnd[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (RND == 1) {
        const uint64_t g0 = L0 >> 3;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint64_t g = g0 + c;
            const uint4 r = philox4x32_10(
                make_uint4(static_cast<uint32_t>(g), static_cast<uint32_t>(g >> 32), stream, 0u), keys);
            rnd[4 * c + 0] = r.x;
            rnd[4 * c + 1] = r.y;
            rnd[4 * c + 2] = r.z;
            rnd[4 * c + 3] = r.w;
        }
    }
    if (sc.zero) return make_uint2(0u, 0u);
    uint32_t w[2] = {0u, 0u};
    bool risky = !(sc.inv * 4.0f < INFINITY);   // tiny (subnormal) step: exact path
    constexpr float kTop = static_cast<float>(top_of<GRID>());
    if (GRID != 1 && RND == 0) {
        // Uniform grid RTNE: k = rint(min(|u| * unit/s, top)).
        const float inv4 = sc.inv * unit_of<GRID>();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float u = v[i];
            const float y = fminf(fabsf(u) * inv4, kTop);
            const float f = y + kRound;
            risky |= fabsf(y - (f - kRound)) > 0.5f - kMargin;
            const uint32_t code = (__float_as_uint(f) & 7u) | ((__float_as_uint(u) >> 28) & 8u);
            w[i >> 3] |= code << (4 * (i & 7));
        }
    } else if (GRID != 1 && RND == 1) {
        // Uniform grid SR.  With q = |u|/(s/unit) and r = r16 * 2^-16, "lo =
        // floor(q), up iff q > lo + r" is exactly k = ceil(q - r): for q =
        // lo + f the value q - r lies in (lo, lo+1) when f > r and in
        // (lo-1, lo] otherwise.  q >= top gives top (clamp first).  ceil(t) =
        // rint(t + 1/2) except when t is (near) an integer, which the margin
        // test sends to the exact path.
        const float inv4 = sc.inv * unit_of<GRID>();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float u = v[i];
            const float y = fminf(fabsf(u) * inv4, kTop);
            const uint32_t word = rnd[i >> 1];
            const uint32_t r16 = (i & 1) ? (word >> 16) : (word & 0xFFFFu);
            const float rf = __uint_as_float(0x4B000000u | r16) - 8388608.0f;   // r16 exactly
            const float th = __fmaf_rn(rf, -1.0f / 65536.0f, y) + 0.5f;          // q - r + 1/2
            const float f = th + kRound;
            risky |= fabsf(th - (f - kRound)) > 0.5f - kMargin;
            const uint32_t code = (__float_as_uint(f) & 7u) | ((__float_as_uint(u) >> 28) & 8u);
            w[i >> 3] |= code << (4 * (i & 7));
        }
    } else if (GRID == 1 && RND == 0) {
        // E2M1 RTNE: the hardware E2M1 conversion of u/s (ties to even); the
        // distance to the nearest midpoint is measured in a scale where the
        // midpoints are half-integers (x2 below 2, x1 below 4, x0.5 above).
        float y[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            y[i] = v[i] * sc.inv;
            const float ay = fminf(fabsf(y[i]), 6.0f);
            const float scl = ay < 2.0f ? 2.0f : (ay < 4.0f ? 1.0f : 0.5f);
            const float m = __fmaf_rn(ay, scl, -0.5f);
            risky |= fabsf(m - ((m + kRound) - kRound)) < kMargin;
        }
        w[0] = cvt_e2m1x4(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
        w[1] = cvt_e2m1x4(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
    } else {
        risky = true;   // E2M1 SR: exact path only
    }
    if (risky) {
        const Chunk16 c{make_float4(v[0], v[1], v[2], v[3]), make_float4(v[4], v[5], v[6], v[7]),
                        make_float4(v[8], v[9], v[10], v[11]), make_float4(v[12], v[13], v[14], v[15])};
        return round_pack_exact<GRID, RND>(c, sc, RandSrc{seed, L0, stream});
    }
    return make_uint2(canonical_zero(w[0]), canonical_zero(w[1]));
}

// ---------------------------------------------------------------------------
// Two chunks at once in packed fp32x2 arithmetic (lane x = chunk a, lane y =
// chunk b): the same IEEE operations per lane as the scalar code.

// Butterfly on two lanes: (x0 + x1, x0 - x1); fma(x1, -1, x0) rounds x0 - x1
// exactly like a subtraction.
__device__ __forceinline__ void bfly2(float2 &x0, float2 &x1) {
    const float2 s = __fadd2_rn(x0, x1);
    const float2 d = __ffma2_rn(x1, make_float2(-1.0f, -1.0f), x0);
    x0 = s;
    x1 = d;
}

// 0x4B000000 | (16 bits of w): the float 2^23 + r16 (lo or hi half).
__device__ __forceinline__ float r16_magic(uint32_t w, bool hi) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(w), "r"(0x4B000000u), "r"(hi ? 0x7432u : 0x7410u));
    return __uint_as_float(d);
}

// A uniform grid (E1M2 or restricted E2M1), RTNE or SR, for two chunks with
// their own block scales: the fast paths of round_pack (same decisions, same
// certification) with the fp32 adds / fmas done two lanes at a time.
template <int GRID, int RND>
__device__ __forceinline__ void round_pack2_uniform(const float (&va)[16], const float (&vb)[16],
                                                 const ScaleOut &sa, const ScaleOut &sb,
                                                 const PhiloxKeys &keys, uint32_t stream, uint64_t seed,
                                                 uint64_t L0a, uint64_t L0b, uint2 &outa, uint2 &outb) {
    constexpr float kTop = static_cast<float>(top_of<GRID>());
    const float inv4a = sa.inv * unit_of<GRID>(), inv4b = sb.inv * unit_of<GRID>();
    // min(|u| * inv4, top) as top * sat(|u| * inv4 / top): a saturating
    // multiply on the fma pipe instead of a min (the estimate moves by a few
    // ulp, far inside the 2^-16 margin; at and above top both give top).
    const float c7a = inv4a * (1.0f / kTop), c7b = inv4b * (1.0f / kTop);
    float deva = 0.0f, devb = 0.0f;      // largest distance from a rint half-way point
    uint32_t wa[2] = {0u, 0u}, wb[2] = {0u, 0u};
    const float2 kR = make_float2(kRound, kRound);
    const float2 kRn = make_float2(-kRound, -kRound);
    const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        // SR words of elements 8 hf .. 8 hf + 7 of each chunk (one Philox call each)
        uint4 ra = make_uint4(0, 0, 0, 0), rb = make_uint4(0, 0, 0, 0);
        if (RND == 1) {
            const uint64_t ga = (L0a >> 3) + hf, gb = (L0b >> 3) + hf;
            ra = philox4x32_10(make_uint4(static_cast<uint32_t>(ga), static_cast<uint32_t>(ga >> 32), stream, 0u),
                               keys);
            rb = philox4x32_10(make_uint4(static_cast<uint32_t>(gb), static_cast<uint32_t>(gb >> 32), stream, 0u),
                               keys);
        }
        const uint32_t rwa[4] = {ra.x, ra.y, ra.z, ra.w}, rwb[4] = {rb.x, rb.y, rb.z, rb.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int i = 8 * hf + e;
            const float2 y7 = make_float2(__saturatef(fabsf(va[i]) * c7a), __saturatef(fabsf(vb[i]) * c7b));
            float2 h;
            if (RND == 1) {
                // h = y - r16 * 2^-16 + 1/2 (k = ceil(q - r) = rint(h) off the
                // integers, which the margin test sends to the exact path)
                const float2 rf = __fadd2_rn(make_float2(r16_magic(rwa[e >> 1], e & 1), r16_magic(rwb[e >> 1], e & 1)),
                                             make_float2(-8421376.0f, -8421376.0f));   // r16 - 2^15
                const float2 rt = __fmul2_rn(rf, make_float2(-1.0f / 65536.0f, -1.0f / 65536.0f));   // exact
                h = __ffma2_rn(y7, make_float2(kTop, kTop), rt);
            } else {
                h = __fmul2_rn(y7, make_float2(kTop, kTop));
            }
            const float2 f = __fadd2_rn(h, kR);
            const float2 g = __fadd2_rn(f, kRn);
            const float2 d = __ffma2_rn(g, m1, h);       // h - rint(h), in [-1/2, 1/2]
            deva = fmaxf(deva, fabsf(d.x));
            devb = fmaxf(devb, fabsf(d.y));
            const uint32_t ca = (__float_as_uint(f.x) & 7u) | ((__float_as_uint(va[i]) >> 28) & 8u);
            const uint32_t cb = (__float_as_uint(f.y) & 7u) | ((__float_as_uint(vb[i]) >> 28) & 8u);
            // nibbles do not overlap: a multiply-add places them
            wa[hf] = ca * (1u << (4 * e)) + wa[hf];
            wb[hf] = cb * (1u << (4 * e)) + wb[hf];
        }
    }
    const bool riska = !(inv4a < INFINITY) || deva > 0.5f - kMargin;
    const bool riskb = !(inv4b < INFINITY) || devb > 0.5f - kMargin;
    outa = sa.zero ? make_uint2(0u, 0u) : make_uint2(canonical_zero(wa[0]), canonical_zero(wa[1]));
    outb = sb.zero ? make_uint2(0u, 0u) : make_uint2(canonical_zero(wb[0]), canonical_zero(wb[1]));
    if (riska && !sa.zero) {
        const Chunk16 c{make_float4(va[0], va[1], va[2], va[3]), make_float4(va[4], va[5], va[6], va[7]),
                        make_float4(va[8], va[9], va[10], va[11]), make_float4(va[12], va[13], va[14], va[15])};
        outa = round_pack_exact<GRID, RND>(c, sa, RandSrc{seed, L0a, stream});
    }
    if (riskb && !sb.zero) {
        const Chunk16 c{make_float4(vb[0], vb[1], vb[2], vb[3]), make_float4(vb[4], vb[5], vb[6], vb[7]),
                        make_float4(vb[8], vb[9], vb[10], vb[11]), make_float4(vb[12], vb[13], vb[14], vb[15])};
        outb = round_pack_exact<GRID, RND>(c, sb, RandSrc{seed, L0b, stream});
    }
}

// ---------------------------------------------------------------------------
// Kernel.  A CTA of 256 compute threads plus one producer warp takes units of
// 256 x 64 bf16 elements, staged in shared memory by TMA with the 128-byte
// swizzle and double-buffered across the CTA's units.  Every compute thread
// quantizes 64 consecutive K elements of one output row, so any Hadamard size
// up to 64 and either block size stays inside the thread:
//   AXIS 0 (row-wise)    one 64 (K) x 256 (rows) box; thread t reads row t,
//                        eight 16-byte chunks (chunk c of row t sits at chunk
//                        c ^ (t & 7)).
//   AXIS 1 (column-wise) four 64 (columns) x 64 (K rows) boxes side by side;
//                        thread t reads column t, one bf16 per K row; a warp
//                        reads 32 consecutive columns of one K row.
//   AXIS 2 (both)        the AXIS 1 tile quantized twice: column-wise into
//                        `a` exactly as AXIS 1, then row-wise into `a2`, where
//                        thread t takes row t & 63 of box t >> 6 (64 columns
//                        of one input row).  One read of the tensor serves
//                        both of its GEMM operands.
// Codes (32 bytes per thread) and block-major scales (a warp writes 32
// consecutive rows of each block) go straight to global memory.
constexpr int kUnitRows = 256;
constexpr int kStageBytes = kUnitRows * 64 * 2;   // 32 KB of bf16
constexpr int kStages = 2;
constexpr int kComputeWarps = kThreads / 32;
constexpr int kCtaThreads = kThreads + 32;        // + one producer warp
constexpr int kQuantSmem = kStages * kStageBytes + 1024 + 64;
// Resident CTAs per SM: three for one output (72 registers a thread); the
// dual kernel does twice the work per staged tile and keeps more state, two.
template <int AXIS>
constexpr int ctas_per_sm() { return AXIS == 2 ? 2 : 3; }

// Two-level tensor scale of one output: S maps the rotated tensor amax to
// gmax * 448 (the top of E4M3), G = gmax * S is the block-scale divisor.
template <int GRID>
__device__ __forceinline__ void tensor_scale(const QuantArgs &q, float &S, float &G) {
    const float amax_t = *q.amax_t;
    S = amax_t > 0.0f ? __fdiv_rn(amax_t, gmax_of<GRID>() * 448.0f) : 1.0f;
    G = __fmul_rn(gmax_of<GRID>(), S);
    if (blockIdx.x == 0 && threadIdx.x == 0 && q.S_out) *q.S_out = S;
}

// Quantizes K elements [k0, k0 + 64) of output row orow of `a`:
//   RD 0: they are one swizzled 128-byte row at src (chunk c at (c ^ swz) << 4);
//   RD 1: they are one column of the four-box tile at src, K row kr at
//         src + col_off[kr & 7] + kr * 128.
// The rotated values' amax goes to amax_acc (AMAX_ONLY) or the codes and
// scales to `a` (rows beyond a.out_rows are computed but not stored).
template <int RD, int NH, int BLK, int GRID, int RND, bool AMAX_ONLY>
__device__ __forceinline__ void quantize64(const QuantArgs &a, const uint8_t *src, int swz,
                                           const uint32_t (&col_off)[8], int64_t orow, int64_t k0,
                                           float S, float G, const PhiloxKeys &keys,
                                           const uint32_t (&smask)[16], uint32_t pat_lo,
                                           uint32_t pat_hi, float &amax_acc) {
    // Per group of GS elements (the Hadamard block and the scale block both
    // lie inside one group): load, D, H, block scales, round, pack.
    constexpr int GS = (NH > BLK ? NH : BLK) > 16 ? (NH > BLK ? NH : BLK) : 16;
    uint32_t codes[8];
    uint32_t stored[4];
    if constexpr (GS == 16) {
        // Groups g and g + 16 side by side as the two lanes of fp32x2
        // values: same positions mod 16, so the same signs of D; the
        // butterflies and the rounding arithmetic run two lanes at a time.
        // Not unrolled: one copy of the body keeps the kernel small.
#pragma unroll 1
        for (int gp = 0; gp < 64; gp += 32) {
            float va[16], vb[16];
            if (RD == 0) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const uint4 qa = *reinterpret_cast<const uint4 *>(src + (((gp / 8 + c) ^ swz) << 4));
                    const uint4 qb = *reinterpret_cast<const uint4 *>(src + (((gp / 8 + 2 + c) ^ swz) << 4));
                    const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w}, wb[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i0 = 8 * c + 2 * e;
                        va[i0] = __uint_as_float((wa[e] << 16) + smask[i0]);
                        va[i0 + 1] = __uint_as_float((wa[e] & 0xFFFF0000u) ^ smask[i0 + 1]);
                        vb[i0] = __uint_as_float((wb[e] << 16) + smask[i0]);
                        vb[i0 + 1] = __uint_as_float((wb[e] & 0xFFFF0000u) ^ smask[i0 + 1]);
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int ka = gp + i, kb = gp + 16 + i;
                    const uint32_t ba = *reinterpret_cast<const uint16_t *>(src + col_off[ka & 7] + ka * 128);
                    const uint32_t bb = *reinterpret_cast<const uint16_t *>(src + col_off[kb & 7] + kb * 128);
                    va[i] = __uint_as_float((ba << 16) + smask[i]);
                    vb[i] = __uint_as_float((bb << 16) + smask[i]);
                }
            }
            if (NH == 16) {
                float2 pr[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pr[i] = make_float2(va[i], vb[i]);
#pragma unroll
                for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (!(i & h)) bfly2(pr[i], pr[i + h]);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    va[i] = pr[i].x;
                    vb[i] = pr[i].y;
                }
            }
            if (AMAX_ONLY) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    amax_acc = fmaxf(amax_acc, fmaxf(fabsf(va[i]), fabsf(vb[i])));
                continue;
            }
            float ama = 0.0f, amb = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                ama = fmaxf(ama, fabsf(va[i]));
                amb = fmaxf(amb, fabsf(vb[i]));
            }
            const ScaleOut sa = block_scale<GRID>(ama, a.scale_fmt, S, G);
            const ScaleOut sb = block_scale<GRID>(amb, a.scale_fmt, S, G);
            const uint64_t L0a = static_cast<uint64_t>(orow) * static_cast<uint64_t>(a.kpad) +
                                 static_cast<uint64_t>(k0 + gp);
            uint2 pa, pb;
            if (GRID != 1) {
                round_pack2_uniform<GRID, RND>(va, vb, sa, sb, keys, a.stream, a.seed, L0a, L0a + 16,
                                               pa, pb);
            } else {
                pa = round_pack<GRID, RND>(va, sa, keys, a.stream, L0a, a.seed);
                pb = round_pack<GRID, RND>(vb, sb, keys, a.stream, L0a + 16, a.seed);
            }
            if (gp == 0) {
                codes[0] = pa.x, codes[1] = pa.y, codes[2] = pb.x, codes[3] = pb.y;
                stored[0] = sa.stored, stored[1] = sb.stored;
            } else {
                codes[4] = pa.x, codes[5] = pa.y, codes[6] = pb.x, codes[7] = pb.y;
                stored[2] = sa.stored, stored[3] = sb.stored;
            }
        }
    } else {
#pragma unroll
        for (int g0 = 0; g0 < 64; g0 += GS) {
            float v[GS];
            if (RD == 0) {
#pragma unroll
                for (int c = 0; c < GS / 8; ++c) {
                    const int cg = g0 / 8 + c;
                    const uint4 q = *reinterpret_cast<const uint4 *>(src + ((cg ^ swz) << 4));
                    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        v[8 * c + 2 * e] = __uint_as_float(w[e] << 16);
                        v[8 * c + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < GS; ++i) {
                    const int kr = g0 + i;
                    const uint16_t b = *reinterpret_cast<const uint16_t *>(src + col_off[kr & 7] + kr * 128);
                    v[i] = __uint_as_float(static_cast<uint32_t>(b) << 16);
                }
            }
            if (NH > 0) {
#pragma unroll
                for (int i = 0; i < GS; ++i) {
                    const int p = g0 + i;
                    const uint32_t bit = p < 32 ? (pat_lo >> p) & 1u : (pat_hi >> (p - 32)) & 1u;
                    v[i] = __uint_as_float(__float_as_uint(v[i]) ^ (bit << 31));
                }
#pragma unroll
                for (int h = 1; h < NH; h <<= 1) {
#pragma unroll
                    for (int i = 0; i < GS; ++i) {
                        if (i & h) continue;
                        const float x0 = v[i], x1 = v[i + h];
                        v[i] = __fadd_rn(x0, x1);
                        v[i + h] = __fsub_rn(x0, x1);
                    }
                }
            }
            if constexpr (AMAX_ONLY) {
#pragma unroll
                for (int i = 0; i < GS; ++i) amax_acc = fmaxf(amax_acc, fabsf(v[i]));
            } else {
#pragma unroll
            for (int b0 = 0; b0 < GS; b0 += BLK) {
                float am = 0.0f;
#pragma unroll
                for (int i = 0; i < BLK; ++i) am = fmaxf(am, fabsf(v[b0 + i]));
                const ScaleOut sc = block_scale<GRID>(am, a.scale_fmt, S, G);
                stored[(g0 + b0) / BLK] = sc.stored;
#pragma unroll
                for (int c0 = 0; c0 < BLK; c0 += 16) {
                    float chunk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) chunk[i] = v[b0 + c0 + i];
                    const int kc = g0 + b0 + c0;
                    const uint64_t L0 = static_cast<uint64_t>(orow) * static_cast<uint64_t>(a.kpad) +
                                        static_cast<uint64_t>(k0 + kc);
                    const uint2 pk = round_pack<GRID, RND>(chunk, sc, keys, a.stream, L0, a.seed);
                    codes[kc / 8] = pk.x;
                    codes[kc / 8 + 1] = pk.y;
                }
            }
            }
        }
    }
    if constexpr (!AMAX_ONLY) {
        if (orow >= a.out_rows) return;
        uint4 *dst = reinterpret_cast<uint4 *>(a.codes + orow * (a.kpad / 2) + k0 / 2);
        dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
        dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
        if (GRID == 0 && a.corr != nullptr) {
            // E1M2 correction plane for the block-scaled FP4 GEMM
            uint4 *cdst = reinterpret_cast<uint4 *>(a.corr + orow * (a.kpad / 2) + k0 / 2);
            cdst[0] = make_uint4(e1m2_correction(codes[0]), e1m2_correction(codes[1]),
                                 e1m2_correction(codes[2]), e1m2_correction(codes[3]));
            cdst[1] = make_uint4(e1m2_correction(codes[4]), e1m2_correction(codes[5]),
                                 e1m2_correction(codes[6]), e1m2_correction(codes[7]));
        }
        constexpr int kBlocks = 64 / BLK;
#pragma unroll
        for (int b = 0; b < kBlocks; ++b) {
            const int64_t blk = k0 / BLK + b;
            if (a.scale_fmt == 0)
                reinterpret_cast<uint32_t *>(a.scales)[blk * a.scale_ld + orow] = stored[b];
            else
                reinterpret_cast<uint8_t *>(a.scales)[blk * a.scale_ld + orow] = static_cast<uint8_t>(stored[b]);
        }
    }
}

// `a` drives the units (AXIS 0: row-wise output; AXIS 1 and 2: column-wise
// output); `a2` is the row-wise output of AXIS 2 and unused otherwise.
template <int AXIS, int NH, int BLK, int GRID, int RND, bool AMAX_ONLY>
__global__ void __launch_bounds__(kCtaThreads, ctas_per_sm<AXIS>()) rht_quantize_kernel(const __grid_constant__ QuantArgs a,
                                                                  const __grid_constant__ QuantArgs a2,
                                                                  const __grid_constant__ CUtensorMap tmap) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * kStageBytes);
    uint64_t *empty = full + kStages;
    volatile uint32_t *abort_flag =
        reinterpret_cast<volatile uint32_t *>(smem + kStages * kStageBytes + 16 * kStages);
    const int t = threadIdx.x;
    const int lane = t & 31;
    const int warp = t >> 5;
    const int64_t nseg = a.kpad / 64;
    const int64_t nrb = (a.out_rows + kUnitRows - 1) / kUnitRows;
    const int64_t nunits = nseg * nrb;

    auto unit_coords = [&](int64_t u, int64_t &rb, int64_t &seg) {
        if (AXIS == 0) {
            rb = u / nseg;
            seg = u % nseg;
        } else {
            seg = u / nrb;
            rb = u % nrb;
        }
    };
    auto issue = [&](int64_t u, int s) {
        int64_t rb, seg;
        unit_coords(u, rb, seg);
        uint8_t *dst = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        if (AXIS == 0) {
            tma_load_2d(dst, &tmap, &full[s], static_cast<int32_t>(seg * 64),
                        static_cast<int32_t>(rb * kUnitRows));
        } else {
#pragma unroll
            for (int b = 0; b < 4; ++b)
                tma_load_2d(dst + b * 8192, &tmap, &full[s], static_cast<int32_t>(rb * kUnitRows + 64 * b),
                            static_cast<int32_t>(seg * 64));
        }
    };

    if (t == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kComputeWarps);
        }
        *abort_flag = 0u;
        fence_barrier_init();
    }
    __syncthreads();
    const int64_t u0 = blockIdx.x;
    if (warp == kComputeWarps) {
        // Producer warp: refills a stage once every compute warp released it.
        if (lane == 0) {
            uint32_t it = 0;
            for (int64_t u = u0; u < nunits; u += gridDim.x, ++it) {
                const int s = it % kStages;
                if (it >= kStages &&
                    !mbar_wait(&empty[s], ((it / kStages) - 1) & 1, kErrTimeoutProducer, abort_flag))
                    break;
                issue(u, s);
            }
            // Drain: the last copies have landed before the CTA exits.
            for (uint32_t d = 0; d < kStages && d < it; ++d) {
                const uint32_t idx = it - 1 - d;
                uint32_t dummy = 0;
                mbar_wait(&full[idx % kStages], (idx / kStages) & 1, kErrTimeoutDrain,
                          reinterpret_cast<volatile uint32_t *>(&dummy));
            }
        }
        return;
    }

    float S = 1.0f, G = 0.0f, S2 = 1.0f, G2 = 0.0f;
    if (!AMAX_ONLY && a.scale_fmt == 1) tensor_scale<GRID>(a, S, G);
    if (AXIS == 2 && !AMAX_ONLY && a2.scale_fmt == 1) tensor_scale<GRID>(a2, S2, G2);
    // D for the 64 positions of a segment (K offsets are multiples of 64).
    uint64_t pat = 0;
    if (NH > 0) {
        const uint64_t m = NH == 64 ? a.sign_mask : (a.sign_mask & ((1ull << NH) - 1));
#pragma unroll
        for (int off = 0; off < 64; off += (NH > 0 ? NH : 64)) pat |= m << off;
    }
    const uint32_t pat_lo = static_cast<uint32_t>(pat), pat_hi = static_cast<uint32_t>(pat >> 32);
    // Sign of D at position i mod 16 as an fp32 sign bit (NH <= 16; adding it
    // to a widened bf16 flips the sign bit like an xor) and the Philox round
    // keys: both from the parameter bank, no registers held.
    const uint32_t (&smask)[16] = a.smask;
    const PhiloxKeys &keys = a.keys;
    float amax_acc = 0.0f, amax_acc2 = 0.0f;

    // Column-wise: byte offset of column cc (= t & 63) within K row r of a
    // 64-column box for r % 8 (the 128-byte swizzle XORs the 16-byte chunk
    // index with the row mod 8).
    uint32_t col_off[8];
    {
        const int cc = t & 63;
#pragma unroll
        for (int r = 0; r < 8; ++r)
            col_off[r] = static_cast<uint32_t>((t >> 6) * 8192 + ((((cc >> 3) ^ r) & 7) << 4) + (cc & 7) * 2);
    }
    uint32_t it = 0;
    for (int64_t u = u0; u < nunits; u += gridDim.x, ++it) {
        const int s = it % kStages;
        if (!warp_wait(&full[s], (it / kStages) & 1, kErrTimeoutTransform, abort_flag)) break;
        int64_t rb, seg;
        unit_coords(u, rb, seg);
        const uint8_t *tile = smem + s * kStageBytes;
        if (AXIS == 0) {
            quantize64<0, NH, BLK, GRID, RND, AMAX_ONLY>(a, tile + t * 128, t & 7, col_off, rb * kUnitRows + t,
                                                         seg * 64, S, G, keys, smask, pat_lo, pat_hi,
                                                         amax_acc);
        } else {
            quantize64<1, NH, BLK, GRID, RND, AMAX_ONLY>(a, tile, 0, col_off, rb * kUnitRows + t, seg * 64, S,
                                                         G, keys, smask, pat_lo, pat_hi, amax_acc);
            if (AXIS == 2) {
                // Row-wise output: input row 64 seg + (t & 63), K columns from
                // 256 rb + 64 (t >> 6).  Boxes past the padded K (the last
                // column block of a ragged width) are skipped, per warp.
                const int64_t k0 = rb * kUnitRows + 64 * (t >> 6);
                if (k0 < a2.kpad)
                    quantize64<0, NH, BLK, GRID, RND, AMAX_ONLY>(a2, tile + (t >> 6) * 8192 + (t & 63) * 128, t & 7,
                                                                 col_off, seg * 64 + (t & 63), k0, S2, G2, keys,
                                                                 smask, pat_lo, pat_hi, amax_acc2);
            }
        }
        __syncwarp();      // this warp is done with stage s
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (AMAX_ONLY) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            amax_acc = fmaxf(amax_acc, __shfl_xor_sync(0xFFFFFFFFu, amax_acc, off));
            if (AXIS == 2) amax_acc2 = fmaxf(amax_acc2, __shfl_xor_sync(0xFFFFFFFFu, amax_acc2, off));
        }
        if (lane == 0 && amax_acc > 0.0f)
            atomicMax(reinterpret_cast<unsigned int *>(a.amax_out), __float_as_uint(amax_acc));
        if (AXIS == 2 && lane == 0 && amax_acc2 > 0.0f)
            atomicMax(reinterpret_cast<unsigned int *>(a2.amax_out), __float_as_uint(amax_acc2));
    }
}

// Host side of the per-call constants: Philox round keys of the seed and the
// D sign bits of positions 0..15 (used by the kernels with NH <= 16).
void fill_call_constants(QuantArgs &a, int hadamard_n) {
    uint32_t kx = static_cast<uint32_t>(a.seed), ky = static_cast<uint32_t>(a.seed >> 32);
    for (int r = 0; r < 10; ++r) {
        a.keys.x[r] = kx;
        a.keys.y[r] = ky;
        kx += 0x9E3779B9u;
        ky += 0xBB67AE85u;
    }
    for (int i = 0; i < 16; ++i)
        a.smask[i] = hadamard_n > 0 ? static_cast<uint32_t>((a.sign_mask >> i) & 1u) << 31 : 0u;
}

template <int AXIS, int NH, int BLK, int GRID, int RND, bool AMAX_ONLY>
cudaError_t launch_one(const QuantArgs &a, const QuantArgs &a2, const CUtensorMap &tmap, int num_sms,
                       cudaStream_t stream) {
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(rht_quantize_kernel<AXIS, NH, BLK, GRID, RND, AMAX_ONLY>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kQuantSmem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const int64_t nunits = (a.kpad / 64) * ((a.out_rows + kUnitRows - 1) / kUnitRows);
    const int64_t cap = static_cast<int64_t>(num_sms) * ctas_per_sm<AXIS>();
    const int grid = static_cast<int>(nunits < cap ? nunits : cap);
    if (grid <= 0) return cudaSuccess;
    rht_quantize_kernel<AXIS, NH, BLK, GRID, RND, AMAX_ONLY><<<grid, kCtaThreads, kQuantSmem, stream>>>(a, a2, tmap);
    return cudaGetLastError();
}

template <int AXIS, int NH, int BLK, bool AMAX_ONLY>
cudaError_t dispatch_grid_round(const QuantArgs &a, const QuantArgs &a2, const CUtensorMap &m, int grid_kind,
                                int rnd, int num_sms, cudaStream_t stream) {
    if (AMAX_ONLY) return launch_one<AXIS, NH, BLK, 0, 0, true>(a, a2, m, num_sms, stream);
    if (grid_kind == 0) {
        return rnd == 0 ? launch_one<AXIS, NH, BLK, 0, 0, false>(a, a2, m, num_sms, stream)
                        : launch_one<AXIS, NH, BLK, 0, 1, false>(a, a2, m, num_sms, stream);
    }
    if (grid_kind == 2) {
        return rnd == 0 ? launch_one<AXIS, NH, BLK, 2, 0, false>(a, a2, m, num_sms, stream)
                        : launch_one<AXIS, NH, BLK, 2, 1, false>(a, a2, m, num_sms, stream);
    }
    return rnd == 0 ? launch_one<AXIS, NH, BLK, 1, 0, false>(a, a2, m, num_sms, stream)
                    : launch_one<AXIS, NH, BLK, 1, 1, false>(a, a2, m, num_sms, stream);
}

template <int AXIS, bool AMAX_ONLY>
cudaError_t dispatch_nh_blk(const QuantArgs &a, const QuantArgs &a2, const CUtensorMap &m, int nh, int blk,
                            int grid_kind, int rnd, int num_sms, cudaStream_t stream) {
#define UFP4_CASE(N, B)                                                                          \
    if (nh == N && blk == B)                                                                     \
        return dispatch_grid_round<AXIS, N, B, AMAX_ONLY>(a, a2, m, grid_kind, rnd, num_sms, stream);
    UFP4_CASE(0, 16)
    UFP4_CASE(0, 32)
    UFP4_CASE(16, 16)
    UFP4_CASE(16, 32)
    UFP4_CASE(32, 16)
    UFP4_CASE(32, 32)
    UFP4_CASE(64, 16)
    UFP4_CASE(64, 32)
#undef UFP4_CASE
    return cudaErrorInvalidValue;
}

// bf16 input as a 2-D tensor map: rows x cols, row pitch ld; 128-byte swizzle,
// box 64 x 256 (row-wise: K x rows) or 64 x 64 (column-wise and dual:
// columns x K).
cudaError_t make_input_map(const QuantArgs &a, CUtensorMap *m) {
    const uint32_t box_outer = a.axis == 0 ? kUnitRows : 64;
    CUresult r = encode_tensor_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x,
                                      static_cast<uint64_t>(a.cols), static_cast<uint64_t>(a.rows),
                                      static_cast<uint64_t>(a.ld) * 2, 64, box_outer,
                                      CU_TENSOR_MAP_SWIZZLE_128B);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_rht_quantize(QuantArgs a, int hadamard_n, int block, int grid_kind,
                                int rounding, int num_sms, cudaStream_t stream) {
    fill_call_constants(a, hadamard_n);
    CUtensorMap m;
    cudaError_t e = make_input_map(a, &m);
    if (e != cudaSuccess) return e;
    if (a.axis == 0)
        return dispatch_nh_blk<0, false>(a, a, m, hadamard_n, block, grid_kind, rounding, num_sms, stream);
    return dispatch_nh_blk<1, false>(a, a, m, hadamard_n, block, grid_kind, rounding, num_sms, stream);
}

cudaError_t launch_rht_quantize_dual(QuantArgs a_rows, QuantArgs a_cols, int hadamard_n, int block,
                                     int grid_kind, int rounding, int num_sms, cudaStream_t stream) {
    fill_call_constants(a_rows, hadamard_n);
    fill_call_constants(a_cols, hadamard_n);
    CUtensorMap m;
    cudaError_t e = make_input_map(a_rows, &m);
    if (e != cudaSuccess) return e;
    return dispatch_nh_blk<2, false>(a_rows, a_cols, m, hadamard_n, block, grid_kind, rounding, num_sms,
                                     stream);
}

cudaError_t launch_rht_amax(QuantArgs a, int hadamard_n, int num_sms, cudaStream_t stream) {
    fill_call_constants(a, hadamard_n);
    cudaError_t e = cudaMemsetAsync(a.amax_out, 0, sizeof(float), stream);
    if (e != cudaSuccess) return e;
    CUtensorMap m;
    e = make_input_map(a, &m);
    if (e != cudaSuccess) return e;
    if (a.axis == 0) return dispatch_nh_blk<0, true>(a, a, m, hadamard_n, 16, 0, 0, num_sms, stream);
    return dispatch_nh_blk<1, true>(a, a, m, hadamard_n, 16, 0, 0, num_sms, stream);
}

cudaError_t launch_rht_amax_dual(QuantArgs a_rows, QuantArgs a_cols, int hadamard_n, int num_sms,
                                 cudaStream_t stream) {
    fill_call_constants(a_rows, hadamard_n);
    fill_call_constants(a_cols, hadamard_n);
    cudaError_t e = cudaMemsetAsync(a_rows.amax_out, 0, sizeof(float), stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(a_cols.amax_out, 0, sizeof(float), stream);
    if (e != cudaSuccess) return e;
    CUtensorMap m;
    e = make_input_map(a_rows, &m);
    if (e != cudaSuccess) return e;
    return dispatch_nh_blk<2, true>(a_rows, a_cols, m, hadamard_n, 16, 0, 0, num_sms, stream);
}

cudaError_t quantize_read_and_clear_error_word(uint32_t *out) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(out, g_error_word, sizeof(uint32_t));
    if (e != cudaSuccess) return e;
    const uint32_t zero = 0;
    return cudaMemcpyToSymbol(g_error_word, &zero, sizeof(uint32_t));
}

}  // namespace ufp4
