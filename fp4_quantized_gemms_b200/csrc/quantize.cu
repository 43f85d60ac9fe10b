// quantize.cu -- fused RHT + block absmax + scale + 4-bit rounding + packing
// (ufp4_rht_quantize) and the rotated-domain tensor amax (ufp4_rht_amax).
//
// Method: arXiv 2606.20381, paperlayer.ai summary §2 "Random Hadamard
// transforms", "Blockwise quantization", "Rounding rules"; §4 UFP4 recipe;
// gist.science "Efficiëntie" (RHT fused with the quantizer).
//
// Work decomposition.  A persistent CTA (8 compute warps + one TMA producer
// warp) takes units of 256 output rows x 64 K elements whose bf16 tile a TMA copy stages in shared memory (3-stage
// ring).  Every compute thread quantizes 64 elements of a unit as 32
// "entries", each a pair of fp32 values held as the two lanes of an fp32x2
// register: lane x and lane y are two 32-long runs along K that share their
// D signs position by position, so the butterflies, the rounding estimate and
// the packing run two elements per instruction:
//   row map   (K contiguous)  one output row, K [0, 32) in x, [32, 64) in y;
//   col2 map  (K strided, n <= 32)  two adjacent output rows (input columns
//             c, c + 1: one 32-bit shared load gives both), 32 K each;
//   col1 map  (K strided, n = 64)  one output row, K [0, 32) in x, [32, 64) in y.
//
// Exactness.  The butterflies are the same fp32 adds in the same stage order
// as the definition.  Codes come from an fp32 estimate of u / s that is
// certified: every decision whose estimate lies within 2^-18 grid steps of a
// boundary (the estimate's error is below 2^-19 steps), and every block whose
// step is subnormal or could saturate, sends the thread's 64 elements to the
// exact path, which the warp runs cooperatively and which decides each
// element by fma sign tests against exact thresholds, so codes always equal
// the exact-quotient rule bit for bit.

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define UFP4_PIPELINE_KERNELS 1
#include "ufp4_device.cuh"
#include "ufp4_internal.h"

namespace ufp4 {

namespace {


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
// certified by the 2^-18 margin or re-decided exactly): rcp.approx has at
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
// 2^-19 steps: a quotient below 8 with a relative error under 2^-22 (the
// reciprocal's ulp, the product's rounding, and for two-level scales the
// rounding of e_b * S).
constexpr float kMargin = 1.0f / 262144.0f;

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

// ---------------------------------------------------------------------------
// Packed fp32x2 arithmetic: the same IEEE operation per lane as the scalar
// code.  The butterfly's difference is fma(x1, -1, x0), rounded exactly like
// x0 - x1.
__device__ __forceinline__ void bfly2(float2 &x0, float2 &x1) {
    const float2 s = __fadd2_rn(x0, x1);
    const float2 d = __ffma2_rn(x1, make_float2(-1.0f, -1.0f), x0);
    x0 = s;
    x1 = d;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// 0x4B000000 | (16 bits of w): the float 2^23 + r16 (lo or hi half).
__device__ __forceinline__ float r16_magic(uint32_t w, bool hi) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(w), "r"(0x4B000000u), "r"(hi ? 0x7432u : 0x7410u));
    return __uint_as_float(d);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Offset-binary nibbles o = g + 8 (g in [-7, 7]) -> sign-magnitude codes:
// g >= 0 gives o ^ 8 = g; g < 0 (o < 8) gives (o ^ 15) + 1 = 8 + |g|.  Eight
// nibbles at once, no carries between them; g = 0 gives 0 (canonical zero).
__device__ __forceinline__ uint32_t offset_to_sign_magnitude(uint32_t o) {
    const uint32_t neg = (~o & 0x88888888u) >> 3;     // 1 in each negative nibble
    return (o ^ (neg * 15u | 0x88888888u)) + neg;
}

// bf16 -> fp32 with the D sign s (0 or 0x80000000) applied: adding s flips
// the sign bit like an xor.
__device__ __forceinline__ float lo_f(uint32_t w, uint32_t s) { return __uint_as_float((w << 16) + s); }
__device__ __forceinline__ float hi_f(uint32_t w, uint32_t s) {
    return __uint_as_float((w & 0xFFFF0000u) ^ s);
}

// Grid constants of the runtime-selected grid (the two uniform grids share
// one kernel): gmax, grid units per step (u / s * unit is the level index),
// the top index, and frexp-style (mantissa in [1, 2), exponent) of gmax.
struct GridK {
    float gmax, unit, top, mg;
    int eg;
};

__device__ __forceinline__ GridK grid_constants(int grid) {
    if (grid == 0) return GridK{1.75f, 4.0f, 7.0f, 1.75f, 0};   // E1M2: k / 4
    if (grid == 1) return GridK{6.0f, 1.0f, 7.0f, 1.5f, 2};     // E2M1 (unit unused)
    return GridK{2.0f, 2.0f, 4.0f, 1.0f, 1};                    // E2M1, max_fpx 2: k / 2
}

// block_scale with the grid taken at run time: the same stored scales and
// steps as the templated version.  For two-level scales the quotient amax / G
// comes from rG = RN(1 / G) (one product, within 2 ulp of the exact quotient,
// 2.5 ulp of its rounding) instead of a division; the E4M3 byte depends only
// on the side of the quotient's rounding midpoints (fraction bits below the
// third = 1000...0) it falls on, so a product within 4 ulp of a midpoint, or
// below the smallest normal E4M3 value (2^-6, where the midpoints are spaced
// differently), sets `risky` and the exact path decides the block (so does
// a NaN product, e.g. amax = 0 times an infinite rG).
__device__ __forceinline__ ScaleOut block_scale_rt(float amax, int scale_fmt, float S, float G, float rG,
                                                   const GridK &gk, bool &risky) {
    ScaleOut o;
    if (scale_fmt == 2) {
        int X = -127;
        if (amax > 0.0f) {
            const int ea = ilogbf(amax);
            const float ma = ldexpf(amax, -ea);
            X = ea - gk.eg + (ma > gk.mg ? 1 : 0);
            X = X < -127 ? -127 : (X > 127 ? 127 : X);
        }
        o.m1 = 1.0f;
        o.b = ldexpf(1.0f, X);
        o.zero = !(amax > 0.0f);
        o.inv = ldexpf(1.0f, -X);
        o.stored = static_cast<uint32_t>(X + 127);
        return o;
    }
    if (scale_fmt == 0) {
        const float s = __fdiv_rn(amax, gk.gmax);
        o.m1 = 1.0f;
        o.b = s;
        o.zero = !(s > 0.0f);
        o.inv = o.zero ? 0.0f : approx_rcp(s);
        o.stored = __float_as_uint(s);
    } else {
        const float q = __fmul_rn(amax, rG);
        risky |= (__float_as_uint(q) & 0xFFFFFu) - 0x7FFFCu < 9u || !(q >= 0.015625f || q == 0.0f);
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

// ---------------------------------------------------------------------------
// Work unit and thread maps.
constexpr int kComputeWarps = 8;
constexpr int kUnitRows = 256;
constexpr int kStageBytes = kUnitRows * 64 * 2;   // 32 KB of bf16
constexpr int kStages = 3;
constexpr int kCtasPerSm = 2;
constexpr int kCtaThreads = 32 * (kComputeWarps + 1);   // + one producer warp
constexpr int kQuantSmem = kStages * kStageBytes + 8 * 2 * kStages + 16 + 1024;   // + barriers, abort word, alignment

enum { MAP_ROW = 0, MAP_COL2 = 1, MAP_COL1 = 2 };

// Where a thread reads its 64 bf16 values in the staged tile.
//   row:  p = the thread's 128-byte tile row, off8[0] = its swizzle (row & 7);
//   col2: p = the box's first K row of this half, off8[j] = byte offset of the
//         thread's column pair in a K row r with r % 8 == j (without the
//         swizzle every off8[j] is off8[0]);
//   col1: p = the box, off8[j] = the same for the thread's single column.
struct Src {
    const uint8_t *p;
    uint32_t off8[8];
};

// Output rows and first output column of the lane-x and lane-y runs
// (callers validate rows and kpad below 2^31).  Either row_y = row_x and
// k_y = k_x + 32 (row and col1 maps) or row_y = row_x + 1 and k_y = k_x
// (col2 map).
struct Site {
    int32_t row_x, row_y, k_x, k_y;
};

// D sign bit of lane-run position p (p < 64; the launcher stores the mask
// pattern repeated with period n), 0 without a rotation.
template <int NH>
__device__ __forceinline__ uint32_t dsign(const QuantArgs &a, int p) {
    return NH == 0 ? 0u : a.smask[p];
}

// Entries processed together: 16 when both the Hadamard block and the scale
// block fit in 16 positions, else the whole run of 32.
template <int NH, int BLK>
constexpr int ent_of() { return (NH <= 16 && BLK == 16) ? 16 : 32; }

// Entries [E0, E0 + ENT) of the thread's run pair.
template <int MAP, bool SWZ, int NH, int E0, int ENT>
__device__ __forceinline__ void load_entries(const QuantArgs &a, const Src &src, float2 (&v)[ENT]) {
    if constexpr (MAP == MAP_ROW) {
        const uint32_t swz = src.off8[0];
#pragma unroll
        for (int c = E0 / 8; c < (E0 + ENT) / 8; ++c) {
            const uint4 qx = *reinterpret_cast<const uint4 *>(src.p + ((c ^ swz) << 4));
            const uint4 qy = *reinterpret_cast<const uint4 *>(src.p + (((c + 4) ^ swz) << 4));
            const uint32_t wx[4] = {qx.x, qx.y, qx.z, qx.w}, wy[4] = {qy.x, qy.y, qy.z, qy.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = 8 * c + 2 * e;
                v[i - E0] = make_float2(lo_f(wx[e], dsign<NH>(a, i)), lo_f(wy[e], dsign<NH>(a, i + 32)));
                v[i + 1 - E0] =
                    make_float2(hi_f(wx[e], dsign<NH>(a, i + 1)), hi_f(wy[e], dsign<NH>(a, i + 33)));
            }
        }
    } else if constexpr (MAP == MAP_COL2) {
#pragma unroll
        for (int i = E0; i < E0 + ENT; ++i) {
            const uint32_t off = SWZ ? src.off8[i & 7] : src.off8[0];
            const uint32_t w = *reinterpret_cast<const uint32_t *>(src.p + i * 128 + off);
            v[i - E0] = make_float2(lo_f(w, dsign<NH>(a, i)), hi_f(w, dsign<NH>(a, i)));
        }
    } else {
#pragma unroll
        for (int i = E0; i < E0 + ENT; ++i) {
            const uint32_t off = SWZ ? src.off8[i & 7] : src.off8[0];
            const uint32_t bx = *reinterpret_cast<const uint16_t *>(src.p + i * 128 + off);
            const uint32_t by = *reinterpret_cast<const uint16_t *>(src.p + (i + 32) * 128 + off);
            v[i - E0] = make_float2(lo_f(bx, dsign<NH>(a, i)), lo_f(by, dsign<NH>(a, i + 32)));
        }
    }
}

// u = H_n (D x) per n-block along each lane's run (stages h = 1, 2, ..., n/2;
// for n = 64 the last stage pairs lane x with lane y, positions i and i + 32).
template <int NH, int ENT>
__device__ __forceinline__ void rht_entries(float2 (&v)[ENT]) {
    constexpr int HI = NH > 32 ? 32 : NH;
#pragma unroll
    for (int h = 1; h < HI; h <<= 1) {
#pragma unroll
        for (int i = 0; i < ENT; ++i)
            if (!(i & h)) bfly2(v[i], v[i + h]);
    }
    if constexpr (NH == 64) {
#pragma unroll
        for (int i = 0; i < ENT; ++i) {
            const float x0 = v[i].x, x1 = v[i].y;
            v[i] = make_float2(__fadd_rn(x0, x1), __fsub_rn(x0, x1));
        }
    }
}

// Block amaxes of both lanes: am[b] lane x, am[NB + b] lane y (two partial
// maxima per lane: shorter dependency chains).
template <int BLK, int ENT>
__device__ __forceinline__ void block_amax(const float2 (&v)[ENT], float (&am)[2 * ENT / BLK]) {
    constexpr int NB = ENT / BLK;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        float mx0 = 0.0f, my0 = 0.0f, mx1 = 0.0f, my1 = 0.0f;
#pragma unroll
        for (int i = b * BLK; i < (b + 1) * BLK; i += 4) {
            mx0 = max3(mx0, fabsf(v[i].x), fabsf(v[i + 1].x));
            my0 = max3(my0, fabsf(v[i].y), fabsf(v[i + 1].y));
            mx1 = max3(mx1, fabsf(v[i + 2].x), fabsf(v[i + 3].x));
            my1 = max3(my1, fabsf(v[i + 2].y), fabsf(v[i + 3].y));
        }
        am[b] = fmaxf(mx0, mx1);
        am[NB + b] = fmaxf(my0, my1);
    }
}

// E4M3 bytes of 8 E1M2 codes (nibble i -> byte i, the MX element plane): the
// magnitude k/4 from a byte table (0x00 0x28 0x30 0x34 0x38 0x3A 0x3C 0x3E
// for k = 0..7), the sign moved from bit 3 of the nibble to bit 7 of the byte.
// Codes 0..3 of the low 16 bits of w16 (higher bits ignored).
__device__ __forceinline__ uint32_t e1m2_to_e4m3x4(uint32_t w16) {
    const uint32_t mag = prmt(0x34302800u, 0x3E3C3A38u, w16 & 0x7777u);
    uint32_t v = w16 & 0xFFFFu;
    v = (v | (v << 8)) & 0x00FF00FFu;                   // nibbles n0 n1 | n2 n3 in bytes 0 and 2
    v = (v | (v << 4)) & 0x0F0F0F0Fu;                   // one nibble per byte
    return mag | ((v & 0x08080808u) << 4);
}

// Factor atoms: byte 16 (r % 32) + 4 ((r / 32) % 4) + slot % 4 of the
// 512-byte atom (r / 128, slot / 4) holds the factor of K slot `slot` of row
// r (slots of 16 elements for E4M3 factors, 32 for UE8M0).
__device__ __forceinline__ uint8_t *atom_byte(const QuantArgs &a, int32_t row, int32_t slot) {
    return a.sf_atoms + (static_cast<int64_t>(row >> 7) * a.atoms_k + (slot >> 2)) * 512 + 16 * (row & 31) +
           4 * ((row >> 5) & 3) + (slot & 3);
}

// The atom bytes of one block factor (stored value `sv`) of block `blk_idx`:
// UE8M0 fills one 32-element slot, an E4M3 factor of a 16-block one slot,
// of a 32-block its two 16-element slots.
template <int BLK>
__device__ __forceinline__ void store_atom(const QuantArgs &a, int32_t row, int32_t blk_idx, uint32_t sv) {
    const uint32_t b = sv & 0xFFu;
    if (a.scale_fmt == 2 || BLK == 16)
        *atom_byte(a, row, blk_idx) = static_cast<uint8_t>(b);
    else
        *reinterpret_cast<uint16_t *>(atom_byte(a, row, 2 * blk_idx)) = static_cast<uint16_t>(b | (b << 8));
}

// Per-lane factor tiles (E1M2 operands with E4M3 factors): the factor of
// 16-element slot s of row r sits in tile (r / 128, s / 8), half
// j = (s / 4) % 2 (the K step), lane L = r % 128, byte 4 (L / 32) + s % 4 of
// the lane's 16 bytes: byte 2048 j + 16 L + 4 (L / 32) + s % 4.
__device__ __forceinline__ uint8_t *lane_byte(const QuantArgs &a, int32_t row, int32_t slot) {
    const int32_t L = row & 127;
    return a.sf_lanes + (static_cast<int64_t>(row >> 7) * a.lane_groups + (slot >> 3)) * kLaneTileBytes +
           2048 * ((slot >> 2) & 1) + 16 * L + 4 * (L >> 5) + (slot & 3);
}

template <int BLK>
__device__ __forceinline__ void store_lanes(const QuantArgs &a, int32_t row, int32_t blk_idx, uint32_t sv) {
    const uint32_t b = sv & 0xFFu;
    if (BLK == 16)
        *lane_byte(a, row, blk_idx) = static_cast<uint8_t>(b);
    else
        *reinterpret_cast<uint16_t *>(lane_byte(a, row, 2 * blk_idx)) = static_cast<uint16_t>(b | (b << 8));
}

// Stores the 16 code bytes (and the E1M2 correction plane, the MX element
// plane) and the block scales (and factor atoms) of one lane run.
// The whole 16-byte lane record of row `row` for the K step at k0 (a
// multiple of 64): the step's four factors at bytes 4 (L / 32) .. + 3, zeros
// elsewhere, one full-sector-friendly store.  st: the two runs' stored
// scales (lane x, then lane y).
template <int BLK>
__device__ __forceinline__ void store_lane_record(const QuantArgs &a, int32_t row, int32_t k0, const uint32_t *st) {
    const uint32_t f = BLK == 16 ? ((st[0] & 0xFFu) | ((st[1] & 0xFFu) << 8) | ((st[2] & 0xFFu) << 16) |
                                    ((st[3] & 0xFFu) << 24))
                                 : ((st[0] & 0xFFu) * 0x0101u) | (((st[1] & 0xFFu) * 0x0101u) << 16);
    const int q = (row & 127) >> 5;
    uint4 v = make_uint4(q == 0 ? f : 0u, q == 1 ? f : 0u, q == 2 ? f : 0u, q == 3 ? f : 0u);
    *reinterpret_cast<uint4 *>(lane_byte(a, row, k0 / 16) - 4 * q) = v;
}

template <int BLK>
__device__ __forceinline__ void store_run(const QuantArgs &a, int32_t row, int32_t k0, const uint32_t *w,
                                          const uint32_t *st, bool lane_bytes = true) {
    if (row >= a.out_rows) return;
    const int64_t off = static_cast<int64_t>(row) * (a.kpad / 2) + k0 / 2;
    *reinterpret_cast<uint4 *>(a.codes + off) = make_uint4(w[0], w[1], w[2], w[3]);
    if (a.corr != nullptr)
        *reinterpret_cast<uint4 *>(a.corr + off) = make_uint4(e1m2_correction(w[0]), e1m2_correction(w[1]),
                                                              e1m2_correction(w[2]), e1m2_correction(w[3]));
    if (a.elems8 != nullptr) {
        uint4 *e = reinterpret_cast<uint4 *>(a.elems8 + static_cast<int64_t>(row) * a.kpad + k0);
        e[0] = make_uint4(e1m2_to_e4m3x4(w[0]), e1m2_to_e4m3x4(w[0] >> 16), e1m2_to_e4m3x4(w[1]),
                          e1m2_to_e4m3x4(w[1] >> 16));
        e[1] = make_uint4(e1m2_to_e4m3x4(w[2]), e1m2_to_e4m3x4(w[2] >> 16), e1m2_to_e4m3x4(w[3]),
                          e1m2_to_e4m3x4(w[3] >> 16));
    }
#pragma unroll
    for (int b = 0; b < 32 / BLK; ++b) {
        const int64_t at = static_cast<int64_t>(k0 / BLK + b) * a.scale_ld + row;
        if (a.scale_fmt == 0)
            reinterpret_cast<uint32_t *>(a.scales)[at] = st[b];
        else
            reinterpret_cast<uint8_t *>(a.scales)[at] = static_cast<uint8_t>(st[b]);
    }
    if (a.sf_atoms != nullptr) {
        if (BLK == 16 && a.scale_fmt != 2)   // two adjacent 16-slots: one 16-bit store
            *reinterpret_cast<uint16_t *>(atom_byte(a, row, k0 / 16)) =
                static_cast<uint16_t>((st[0] & 0xFFu) | ((st[1] & 0xFFu) << 8));
        else
            store_atom<BLK>(a, row, k0 / BLK, st[0]);
    }
    if (a.sf_lanes != nullptr && lane_bytes) {
        if (BLK == 16)   // the run's two adjacent 16-slots: one 16-bit store
            *reinterpret_cast<uint16_t *>(lane_byte(a, row, k0 / 16)) =
                static_cast<uint16_t>((st[0] & 0xFFu) | ((st[1] & 0xFFu) << 8));
        else
            store_lanes<BLK>(a, row, k0 / BLK, st[0]);
    }
}

// Exact path, cooperative: the warp re-derives the 64 elements of each of
// its threads whose fast decision was not certified ("owners"), from the
// staged tile that is still in place.  Lane l holds run position l of the
// owner (its lane-x and lane-y elements as one fp32x2 value), so the
// butterflies become shuffles (the lower partner forms a + b, the upper one
// a - b: the same IEEE operations), block maxima are shuffle reductions, and
// every lane decides its two codes by the fma boundary tests.  Few registers,
// no call: the fast path keeps its registers.
template <int MAP, bool SWZ, int NH>
__device__ __forceinline__ float2 load_entry(const QuantArgs &a, const uint8_t *p, const uint32_t (&off8)[8], int l) {
    const uint32_t off = SWZ ? off8[l & 7] : off8[0];
    if constexpr (MAP == MAP_ROW) {
        const uint32_t swz = off8[0], c = static_cast<uint32_t>(l >> 3), e = static_cast<uint32_t>(l & 7);
        const uint32_t bx = *reinterpret_cast<const uint16_t *>(p + ((c ^ swz) << 4) + 2 * e);
        const uint32_t by = *reinterpret_cast<const uint16_t *>(p + (((c + 4) ^ swz) << 4) + 2 * e);
        return make_float2(lo_f(bx, dsign<NH>(a, l)), lo_f(by, dsign<NH>(a, l + 32)));
    } else if constexpr (MAP == MAP_COL2) {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(p + l * 128 + off);
        return make_float2(lo_f(w, dsign<NH>(a, l)), hi_f(w, dsign<NH>(a, l)));
    } else {
        const uint32_t bx = *reinterpret_cast<const uint16_t *>(p + l * 128 + off);
        const uint32_t by = *reinterpret_cast<const uint16_t *>(p + (l + 32) * 128 + off);
        return make_float2(lo_f(bx, dsign<NH>(a, l)), lo_f(by, dsign<NH>(a, l + 32)));
    }
}

template <int MAP, bool SWZ, int NH, int BLK, int GRID, int RND>
__device__ __forceinline__ void coop_exact(const QuantArgs &a, const uint8_t *tile, uint32_t pofs,
                                        const uint32_t (&off8)[8], Site site, float S, float G,
                                        uint32_t owners) {
    const int lane = threadIdx.x & 31;
    while (owners != 0u) {
        const int o = __ffs(owners) - 1;
        owners &= owners - 1u;
        uint32_t off[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) off[j] = __shfl_sync(0xFFFFFFFFu, off8[j], o);
        const uint8_t *p = tile + __shfl_sync(0xFFFFFFFFu, pofs, o);
        Site so;
        so.row_x = __shfl_sync(0xFFFFFFFFu, site.row_x, o);
        so.row_y = __shfl_sync(0xFFFFFFFFu, site.row_y, o);
        so.k_x = __shfl_sync(0xFFFFFFFFu, site.k_x, o);
        so.k_y = __shfl_sync(0xFFFFFFFFu, site.k_y, o);
        float2 v = load_entry<MAP, SWZ, NH>(a, p, off, lane);
        constexpr int HI = NH > 32 ? 32 : NH;
#pragma unroll
        for (int h = 1; h < HI; h <<= 1) {
            const float px = __shfl_xor_sync(0xFFFFFFFFu, v.x, h), py = __shfl_xor_sync(0xFFFFFFFFu, v.y, h);
            if (lane & h) v = make_float2(__fsub_rn(px, v.x), __fsub_rn(py, v.y));
            else v = make_float2(__fadd_rn(v.x, px), __fadd_rn(v.y, py));
        }
        if (NH == 64) v = make_float2(__fadd_rn(v.x, v.y), __fsub_rn(v.x, v.y));
        float mx = fabsf(v.x), my = fabsf(v.y);
#pragma unroll
        for (int m = 1; m < BLK; m <<= 1) {
            mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, m));
            my = fmaxf(my, __shfl_xor_sync(0xFFFFFFFFu, my, m));
        }
        uint32_t nib[2];
        uint32_t stv[2];
#pragma unroll
        for (int ln = 0; ln < 2; ++ln) {
            const float u = ln ? v.y : v.x;
            const ScaleOut sc = block_scale<GRID>(ln ? my : mx, a.scale_fmt, S, G);
            stv[ln] = sc.stored;
            int k = 0;
            if (!sc.zero) {
                if (RND == 0) {
                    k = round_rtne<GRID>(fabsf(u), sc.m1, sc.b, sc.inv);
                } else {
                    const int64_t row = ln ? so.row_y : so.row_x, k0 = ln ? so.k_y : so.k_x;
                    const uint64_t g = ((static_cast<uint64_t>(row) * static_cast<uint64_t>(a.kpad) +
                                         static_cast<uint64_t>(k0)) >> 3) + (lane >> 3);
                    const uint4 r = philox4x32_10(make_uint4(static_cast<uint32_t>(g),
                                                             static_cast<uint32_t>(g >> 32), a.stream, 0u),
                                                  a.keys);
                    const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
                    const uint32_t word = rw[(lane >> 1) & 3];
                    const uint32_t r16 = (lane & 1) ? (word >> 16) : (word & 0xFFFFu);
                    k = round_sr<GRID>(fabsf(u), sc.m1, sc.b, sc.inv, r16);
                }
            }
            nib[ln] = k == 0 ? 0u : (static_cast<uint32_t>(k) | ((__float_as_uint(u) >> 28) & 8u));
        }
        // 8 lanes' nibbles -> one code word; lane 8j stores word j of each run
        uint32_t wx = nib[0] << (4 * (lane & 7)), wy = nib[1] << (4 * (lane & 7));
#pragma unroll
        for (int m = 1; m < 8; m <<= 1) {
            wx |= __shfl_xor_sync(0xFFFFFFFFu, wx, m);
            wy |= __shfl_xor_sync(0xFFFFFFFFu, wy, m);
        }
#pragma unroll
        for (int ln = 0; ln < 2; ++ln) {
            const int32_t row = ln ? so.row_y : so.row_x, k0 = ln ? so.k_y : so.k_x;
            if (row >= a.out_rows) continue;
            const uint32_t w = ln ? wy : wx;
            if ((lane & 7) == 0) {
                const int64_t at = static_cast<int64_t>(row) * (a.kpad / 2) + k0 / 2 + 4 * (lane >> 3);
                *reinterpret_cast<uint32_t *>(a.codes + at) = w;
                if (a.corr != nullptr) *reinterpret_cast<uint32_t *>(a.corr + at) = e1m2_correction(w);
                if (a.elems8 != nullptr)
                    *reinterpret_cast<uint2 *>(a.elems8 + static_cast<int64_t>(row) * a.kpad + k0 + 8 * (lane >> 3)) =
                        make_uint2(e1m2_to_e4m3x4(w), e1m2_to_e4m3x4(w >> 16));
            }
            if (lane % BLK == 0) {
                const int64_t at = static_cast<int64_t>(k0 / BLK + lane / BLK) * a.scale_ld + row;
                if (a.scale_fmt == 0) reinterpret_cast<uint32_t *>(a.scales)[at] = stv[ln];
                else reinterpret_cast<uint8_t *>(a.scales)[at] = static_cast<uint8_t>(stv[ln]);
                if (a.sf_atoms != nullptr) store_atom<BLK>(a, row, k0 / BLK + lane / BLK, stv[ln]);
                if (a.sf_lanes != nullptr) store_lanes<BLK>(a, row, k0 / BLK + lane / BLK, stv[ln]);
            }
        }
    }
}

// Perturbation of the E2M1 estimate (relative): far above its error (a few
// ulp) and far below the distance that separates grid decisions.
constexpr float kE2m1Eps = 1.0f / 1048576.0f;
// Start value of a code accumulator: 2^23 + 0x8888 (offset 8 per nibble).
constexpr float kPackBase = 8423560.0f;

// One thread's 64 elements: load, rotate, block scales, certified fast
// rounding and packing into cw (codes: lane x words 0..3, lane y words 4..7)
// and st (stored scales: lane x, then lane y).  Returns whether a decision
// is not certified (the warp then decides the thread's elements again on the
// exact path).  GRID 0 = the uniform grids (E1M2, restricted E2M1; a.grid
// picks the constants), GRID 1 = E2M1.
template <int MAP, bool SWZ, int NH, int BLK, int GRID, int RND>
__device__ __forceinline__ bool quant_thread(const QuantArgs &a, const Src &src, const Site &site, float S,
                                             float G, float rG, const GridK &gk, uint32_t (&cw)[8],
                                             uint32_t (&st)[64 / BLK]) {
    constexpr int ENT = ent_of<NH, BLK>();
    constexpr int NBP = ENT / BLK;          // blocks per lane in a pass
    constexpr int NB = 32 / BLK;            // blocks per lane run
    bool risky = (GRID == 1 && RND == 1);   // E2M1 SR: exact path
    // Philox counter of the runs' first 8 elements; lane y's is a fixed
    // distance away (the next 32 K of the row, or the next row).
    uint64_t gx = 0;
    if (RND == 1 && GRID == 0)
        gx = (static_cast<uint64_t>(site.row_x) * static_cast<uint64_t>(a.kpad) +
              static_cast<uint64_t>(site.k_x)) >> 3;
    const uint64_t dgy = MAP == MAP_COL2 ? static_cast<uint64_t>(a.kpad) >> 3 : 4u;
#pragma unroll
    for (int p = 0; p < 32 / ENT; ++p) {
        float2 v[ENT];
        if (p == 0) load_entries<MAP, SWZ, NH, 0, ENT>(a, src, v);
        else load_entries<MAP, SWZ, NH, (32 / ENT > 1 ? ENT : 0), ENT>(a, src, v);
        rht_entries<NH, ENT>(v);
        float am[2 * NBP];
        block_amax<BLK, ENT>(v, am);
        float inv[2 * NBP];
#pragma unroll
        for (int j = 0; j < 2 * NBP; ++j) {
            const ScaleOut sc = block_scale_rt(am[j], a.scale_fmt, S, G, rG, gk, risky);
            st[(j / NBP) * NB + p * NBP + (j % NBP)] = sc.stored;
            const float iv = sc.zero ? 0.0f : (GRID == 1 ? sc.inv : sc.inv * gk.unit);
            inv[j] = iv;
            risky |= !(iv < INFINITY);              // subnormal step: no usable reciprocal
            // RTNE without a clamp: the block maximum must stay below top + 1/2
            if (RND == 0 && GRID == 0) risky |= am[j] * iv >= gk.top + 0.4921875f;
        }
        if constexpr (GRID == 1) {
            // E2M1 RTNE: the hardware E2M1 conversion (ties to even,
            // saturating at 6) of the estimate scaled up and down by
            // kE2m1Eps; equal codes certify every quotient in between.
#pragma unroll
            for (int j = 0; j < ENT / 8; ++j) {
                float y1[2][8], y2[2][8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int i = 8 * j + e;
                    const int b = i / BLK;
                    const float2 p1 = __fmul2_rn(v[i], make_float2(inv[b] * (1.0f + kE2m1Eps),
                                                                  inv[NBP + b] * (1.0f + kE2m1Eps)));
                    const float2 p2 = __fmul2_rn(v[i], make_float2(inv[b] * (1.0f - kE2m1Eps),
                                                                  inv[NBP + b] * (1.0f - kE2m1Eps)));
                    y1[0][e] = p1.x, y1[1][e] = p1.y, y2[0][e] = p2.x, y2[1][e] = p2.y;
                }
#pragma unroll
                for (int ln = 0; ln < 2; ++ln) {
                    const uint32_t c1 = cvt_e2m1x4(y1[ln][0], y1[ln][1], y1[ln][2], y1[ln][3], y1[ln][4],
                                                   y1[ln][5], y1[ln][6], y1[ln][7]);
                    const uint32_t c2 = cvt_e2m1x4(y2[ln][0], y2[ln][1], y2[ln][2], y2[ln][3], y2[ln][4],
                                                   y2[ln][5], y2[ln][6], y2[ln][7]);
                    risky |= c1 != c2;
                    cw[4 * ln + p * (ENT / 8) + j] = canonical_zero(c1);
                }
            }
        } else {
            // Uniform grids: g = rint(t) with t = u/s in grid units (RTNE) or
            // t = sign(u) (min(|u|/s, top) + 1/2 - r) (SR: ceil(|q| - r) off
            // the integers), by the 1.5 * 2^23 rint; d = t - g certifies it.
            // The signed g are packed four per fp32 accumulator as
            // offset-binary nibbles (exact integer fmas), then turned into
            // sign-magnitude codes.
            const float2 kR2 = make_float2(kRound, kRound), kRn2 = make_float2(-kRound, -kRound);
            const float2 m1 = make_float2(-1.0f, -1.0f);
            float2 acc[ENT / 4];
#pragma unroll
            for (int j = 0; j < ENT / 4; ++j) acc[j] = make_float2(kPackBase, kPackBase);
            // Distance maximum: two chains for RTNE (shorter dependency
            // chain); one for SR, whose Philox words already crowd the
            // register file.
            constexpr int NDEV = RND == 0 ? 2 : 1;
            float dev[2] = {0.0f, 0.0f};
#pragma unroll
            for (int j = 0; j < ENT / 8; ++j) {
                uint4 rx = make_uint4(0u, 0u, 0u, 0u), ry = rx;
                if (RND == 1) {
                    const uint64_t cx = gx + p * (ENT / 8) + j, cy = cx + dgy;
                    rx = philox4x32_10(make_uint4(static_cast<uint32_t>(cx), static_cast<uint32_t>(cx >> 32),
                                                  a.stream, 0u), a.keys);
                    ry = philox4x32_10(make_uint4(static_cast<uint32_t>(cy), static_cast<uint32_t>(cy >> 32),
                                                  a.stream, 0u), a.keys);
                }
                const uint32_t wx[4] = {rx.x, rx.y, rx.z, rx.w}, wy[4] = {ry.x, ry.y, ry.z, ry.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int i = 8 * j + e;
                    const int b = i / BLK;
                    const float2 y = __fmul2_rn(v[i], make_float2(inv[b], inv[NBP + b]));
                    float2 t;
                    if (RND == 1) {
                        const float2 ya = make_float2(fminf(fabsf(y.x), gk.top), fminf(fabsf(y.y), gk.top));
                        const float2 rf =
                            make_float2(r16_magic(wx[e >> 1], e & 1), r16_magic(wy[e >> 1], e & 1));
                        // 1/2 - r16 2^-16, exact: (2^23 + r16) 2^-16 = 128 + r16 2^-16
                        const float2 c = __ffma2_rn(rf, make_float2(-1.0f / 65536.0f, -1.0f / 65536.0f),
                                                    make_float2(128.5f, 128.5f));
                        const float2 ta = __fadd2_rn(ya, c);
                        t = make_float2(
                            __uint_as_float(__float_as_uint(ta.x) ^ (__float_as_uint(v[i].x) & 0x80000000u)),
                            __uint_as_float(__float_as_uint(ta.y) ^ (__float_as_uint(v[i].y) & 0x80000000u)));
                    } else {
                        t = y;
                    }
                    const float2 f = __fadd2_rn(t, kR2);
                    const float2 g = __fadd2_rn(f, kRn2);
                    const float2 d = __ffma2_rn(g, m1, t);
                    dev[e % NDEV] = max3(dev[e % NDEV], fabsf(d.x), fabsf(d.y));
                    const float wgt = static_cast<float>(1 << (4 * (i & 3)));
                    acc[i >> 2] = __ffma2_rn(g, make_float2(wgt, wgt), acc[i >> 2]);
                }
            }
            risky |= fmaxf(dev[0], dev[1]) > 0.5f - kMargin;
#pragma unroll
            for (int j = 0; j < ENT / 8; ++j) {
                cw[p * (ENT / 8) + j] = offset_to_sign_magnitude(
                    prmt(__float_as_uint(acc[2 * j].x), __float_as_uint(acc[2 * j + 1].x), 0x5410u));
                cw[4 + p * (ENT / 8) + j] = offset_to_sign_magnitude(
                    prmt(__float_as_uint(acc[2 * j].y), __float_as_uint(acc[2 * j + 1].y), 0x5410u));
            }
        }
    }
    return risky;
}

template <int MAP, bool SWZ, int NH>
__device__ __forceinline__ float amax_thread(const QuantArgs &a, const Src &src) {
    constexpr int ENT = NH <= 16 ? 16 : 32;
    float m = 0.0f;
#pragma unroll
    for (int p = 0; p < 32 / ENT; ++p) {
        float2 v[ENT];
        if (p == 0) load_entries<MAP, SWZ, NH, 0, ENT>(a, src, v);
        else load_entries<MAP, SWZ, NH, (32 / ENT > 1 ? ENT : 0), ENT>(a, src, v);
        rht_entries<NH, ENT>(v);
#pragma unroll
        for (int i = 0; i < ENT; ++i) m = max3(m, fabsf(v[i].x), fabsf(v[i].y));
    }
    return m;
}

// Two-level tensor scale of one output: S maps the rotated tensor amax to
// gmax * 448 (the top of E4M3), G = gmax * S is the block-scale divisor and
// rG = RN(1 / G) its reciprocal for the certified quotient estimate.
__device__ __forceinline__ void tensor_scale(const QuantArgs &q, const GridK &gk, float &S, float &G, float &rG) {
    const float amax_t = *q.amax_t;
    S = amax_t > 0.0f ? __fdiv_rn(amax_t, gk.gmax * 448.0f) : 1.0f;
    G = __fmul_rn(gk.gmax, S);
    rG = __frcp_rn(G);
    if (blockIdx.x == 0 && threadIdx.x == 0 && q.S_out) *q.S_out = S;
}

// One thread's part of a unit over the staged tile; `q` is the output it
// fills.  Warp-uniform call: threads whose fast decision was not certified
// are decided again by the whole warp.
template <int MAP, bool SWZ, int NH, int BLK, int GRID, int RND, bool AMAX_ONLY>
__device__ __forceinline__ void unit_part(const QuantArgs &q, const uint8_t *tile, const Src &src, const Site &site,
                                          float S, float G, float rG, const GridK &gk, float &amax_acc) {
    if constexpr (AMAX_ONLY) {
        amax_acc = fmaxf(amax_acc, amax_thread<MAP, SWZ, NH>(q, src));
    } else {
        uint32_t cw[8], st[64 / BLK];
        const bool risky = quant_thread<MAP, SWZ, NH, BLK, GRID, RND>(q, src, site, S, G, rG, gk, cw, st);
        if (!risky) {
            // Row map: both runs are one K step of one row, so the thread
            // writes that row's whole per-lane factor record at once.
            constexpr bool kRecord = MAP == MAP_ROW;
            store_run<BLK>(q, site.row_x, site.k_x, cw, st, !kRecord);
            store_run<BLK>(q, site.row_y, site.k_y, cw + 4, st + 32 / BLK, !kRecord);
            if (kRecord && q.sf_lanes != nullptr && site.row_x < q.out_rows)
                store_lane_record<BLK>(q, site.row_x, site.k_x, st);
        }
        const uint32_t owners = __ballot_sync(0xFFFFFFFFu, risky);
        if (owners != 0u) {
            const uint32_t pofs = static_cast<uint32_t>(src.p - tile);
            if (GRID == 1) coop_exact<MAP, SWZ, NH, BLK, 1, RND>(q, tile, pofs, src.off8, site, S, G, owners);
            else if (q.grid == 0) coop_exact<MAP, SWZ, NH, BLK, 0, RND>(q, tile, pofs, src.off8, site, S, G, owners);
            else coop_exact<MAP, SWZ, NH, BLK, 2, RND>(q, tile, pofs, src.off8, site, S, G, owners);
        }
    }
}

// `a` drives the units (AXIS 0: row-wise output; AXIS 1 and 2: column-wise
// output); `a2` is the row-wise output of AXIS 2 and unused otherwise.
//   AXIS 0  one 64 (K) x 256 (rows) box, 128-byte swizzle: thread t takes
//           tile row t (row map);
//   AXIS 1  four 64 (columns) x 64 (K rows) boxes, no swizzle (a warp's
//           32-bit loads of one K row are 128 consecutive bytes): warp w
//           takes box w & 3, K half w >> 2, lane l columns 2l, 2l + 1 (col2),
//           or for n = 64 thread t takes column t & 63 of box t >> 6 (col1);
//   AXIS 2  the AXIS 1 tile with the 128-byte swizzle quantized twice:
//           column-wise into `a` as AXIS 1, then row-wise into `a2` (thread t
//           takes row t & 63 of box t >> 6: 64 columns of one input row).
//           One read of the tensor serves both of its GEMM operands.

// A CTA's walk over a grid of `slow` x `fast` units (fast fastest), visiting
// units blockIdx.x, blockIdx.x + gridDim.x, ...: advanced without a division.
struct UnitWalk {
    int32_t slow, fast, dslow, dfast, nfast;
    __device__ UnitWalk(uint32_t first, uint32_t step, int32_t nfast_)
        : slow(static_cast<int32_t>(first / static_cast<uint32_t>(nfast_))),
          fast(static_cast<int32_t>(first % static_cast<uint32_t>(nfast_))),
          dslow(static_cast<int32_t>(step / static_cast<uint32_t>(nfast_))),
          dfast(static_cast<int32_t>(step % static_cast<uint32_t>(nfast_))),
          nfast(nfast_) {}
    __device__ __forceinline__ void next() {
        fast += dfast;
        slow += dslow;
        if (fast >= nfast) {
            fast -= nfast;
            ++slow;
        }
    }
};

// Limit of the producer's wait for a free stage (ns).  Only test support
// lowers it, to make that bounded wait run out on purpose; the drain and the
// compute warps keep the normal bound.
static __device__ uint64_t g_producer_wait_limit_ns = kWaitLimitNs;

template <int AXIS, int NH, int BLK, int GRID, int RND, bool AMAX_ONLY>
__global__ void __launch_bounds__(kCtaThreads, kCtasPerSm)
    rht_quantize_kernel(const __grid_constant__ QuantArgs a, const __grid_constant__ QuantArgs a2,
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
    const int32_t nseg = static_cast<int32_t>(a.kpad / 64);
    const int32_t nrb = static_cast<int32_t>((a.out_rows + kUnitRows - 1) / kUnitRows);
    constexpr bool kSwz = AXIS != 1;
    // Units in order (row block major for AXIS 0, K segment major otherwise).
    const UnitWalk walk0(blockIdx.x, gridDim.x, AXIS == 0 ? nseg : nrb);
    const int32_t nslow = AXIS == 0 ? nrb : nseg;
    auto coords = [&](const UnitWalk &w, int32_t &rb, int32_t &seg) {
        rb = AXIS == 0 ? w.slow : w.fast;
        seg = AXIS == 0 ? w.fast : w.slow;
    };

    auto issue = [&](const UnitWalk &w, int s) {
        int32_t rb, seg;
        coords(w, rb, seg);
        uint8_t *dst = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        if (AXIS == 0) {
            tma_load_2d(dst, &tmap, &full[s], seg * 64, rb * kUnitRows);
        } else {
#pragma unroll
            for (int b = 0; b < 4; ++b)
                tma_load_2d(dst + b * 8192, &tmap, &full[s], rb * kUnitRows + 64 * b, seg * 64);
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
    if (warp == kComputeWarps) {
        // Producer warp: refills a stage once every compute warp released it.
        if (lane == 0) {
            uint32_t it = 0;
            for (UnitWalk w = walk0; w.slow < nslow; w.next(), ++it) {
                const int s = it % kStages;
                if (it >= kStages && !mbar_wait(&empty[s], ((it / kStages) - 1) & 1, kErrTimeoutProducer,
                                                abort_flag, g_producer_wait_limit_ns))
                    break;
                issue(w, s);
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
    const GridK gk = grid_constants(a.grid);
    float S = 1.0f, G = 0.0f, rG = 0.0f, S2 = 1.0f, G2 = 0.0f, rG2 = 0.0f;
    if (!AMAX_ONLY && a.scale_fmt == 1) tensor_scale(a, gk, S, G, rG);
    if (AXIS == 2 && !AMAX_ONLY && a2.scale_fmt == 1) tensor_scale(a2, gk, S2, G2, rG2);
    float amax_acc = 0.0f, amax_acc2 = 0.0f;

    // Column maps: byte offsets of the thread's column(s) within a K row r
    // of a 64-column box, for r % 8 = j (the 128-byte swizzle XORs the
    // 16-byte chunk index with the row mod 8).
    constexpr int CMAP = NH == 64 ? MAP_COL1 : MAP_COL2;
    Src csrc;
    csrc.p = nullptr;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int jj = kSwz ? j : 0;
        csrc.off8[j] = CMAP == MAP_COL2
                           ? static_cast<uint32_t>((((lane >> 2) ^ jj) << 4) + 4 * (lane & 3))
                           : static_cast<uint32_t>(((((t & 63) >> 3) ^ jj) << 4) + 2 * (t & 7));
    }
    uint32_t it = 0;
    for (UnitWalk w = walk0; w.slow < nslow; w.next(), ++it) {
        const int s = it % kStages;
        if (!warp_wait(&full[s], (it / kStages) & 1, kErrTimeoutTransform, abort_flag)) break;
        int32_t rb, seg;
        coords(w, rb, seg);
        const uint8_t *tile = smem + s * kStageBytes;
        if (AXIS == 0) {
            Src src;
            src.p = tile + t * 128;
            src.off8[0] = static_cast<uint32_t>(t & 7);
            const int32_t row = rb * kUnitRows + t, k0 = seg * 64;
            const Site site{row, row, k0, k0 + 32};
            unit_part<MAP_ROW, true, NH, BLK, GRID, RND, AMAX_ONLY>(a, tile, src, site, S, G, rG, gk, amax_acc);
        } else {
            Src src = csrc;
            Site site;
            if (CMAP == MAP_COL2) {
                const int box = warp & 3, half = warp >> 2;
                src.p = tile + box * 8192 + half * 32 * 128;
                const int32_t row = rb * kUnitRows + 64 * box + 2 * lane, k0 = seg * 64 + 32 * half;
                site = Site{row, row + 1, k0, k0};
            } else {
                src.p = tile + (t >> 6) * 8192;
                const int32_t row = rb * kUnitRows + t, k0 = seg * 64;
                site = Site{row, row, k0, k0 + 32};
            }
            unit_part<CMAP, kSwz, NH, BLK, GRID, RND, AMAX_ONLY>(a, tile, src, site, S, G, rG, gk, amax_acc);
            if (AXIS == 2) {
                // Row-wise output: input row 64 seg + (t & 63), K columns from
                // 256 rb + 64 (t >> 6).  Boxes past the padded K (the last
                // column block of a ragged width) are skipped, per warp.
                const int64_t k0 = static_cast<int64_t>(rb) * kUnitRows + 64 * (t >> 6);
                if (k0 < a2.kpad) {
                    Src rs;
                    rs.p = tile + (t >> 6) * 8192 + (t & 63) * 128;
                    rs.off8[0] = static_cast<uint32_t>(t & 7);
                    const int32_t row = seg * 64 + (t & 63);
                    const Site rsite{row, row, static_cast<int32_t>(k0), static_cast<int32_t>(k0 + 32)};
                    unit_part<MAP_ROW, true, NH, BLK, GRID, RND, AMAX_ONLY>(a2, tile, rs, rsite, S2, G2, rG2, gk,
                                                                             amax_acc2);
                }
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


// ---------------------------------------------------------------------------
// Unfused RHT (the baseline the fused kernel is compared with, [GS]
// "Efficiëntie"): y = bf16_RN(H_n D x) along the contiguous dimension, the
// same fp32 butterflies as the quantizer, one 64-element row segment per
// thread (global loads and stores of 128 contiguous bytes), grid-stride.
template <int NH>
__global__ void __launch_bounds__(256) rht_bf16_kernel(const __grid_constant__ QuantArgs a, uint16_t *y,
                                                        int64_t ldy) {
    const int64_t nseg = a.cols / 64;
    const int64_t total = a.rows * nseg;
    for (int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; w < total;
         w += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = w / nseg, seg = w % nseg;
        const uint4 *src = reinterpret_cast<const uint4 *>(a.x + r * a.ld + seg * 64);
        float v[64];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint4 q = src[c];
            const uint32_t wd[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = 8 * c + 2 * e;
                v[i] = lo_f(wd[e], NH ? a.smask[i] : 0u);
                v[i + 1] = hi_f(wd[e], NH ? a.smask[i + 1] : 0u);
            }
        }
#pragma unroll
        for (int h = 1; h < NH; h <<= 1) {
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                if (i & h) continue;
                const float x0 = v[i], x1 = v[i + h];
                v[i] = __fadd_rn(x0, x1);
                v[i + h] = __fsub_rn(x0, x1);
            }
        }
        uint4 *dst = reinterpret_cast<uint4 *>(y + r * ldy + seg * 64);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 b = __floats2bfloat162_rn(v[8 * c + 2 * e], v[8 * c + 2 * e + 1]);
                o[e] = *reinterpret_cast<const uint32_t *>(&b);
            }
            dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// Host side of the per-call constants: Philox round keys of the seed and the
// D sign bit of every position 0..63 of a lane run (the n-bit mask repeated
// with period n).
void fill_call_constants(QuantArgs &a, int hadamard_n) {
    uint32_t kx = static_cast<uint32_t>(a.seed), ky = static_cast<uint32_t>(a.seed >> 32);
    for (int r = 0; r < 10; ++r) {
        a.keys.x[r] = kx;
        a.keys.y[r] = ky;
        kx += 0x9E3779B9u;
        ky += 0xBB67AE85u;
    }
    for (int p = 0; p < 64; ++p)
        a.smask[p] = hadamard_n > 0 ? static_cast<uint32_t>((a.sign_mask >> (p % hadamard_n)) & 1u) << 31 : 0u;
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
    const int64_t cap = static_cast<int64_t>(num_sms) * kCtasPerSm;
    const int grid = static_cast<int>(nunits < cap ? nunits : cap);
    if (grid <= 0) return cudaSuccess;
    rht_quantize_kernel<AXIS, NH, BLK, GRID, RND, AMAX_ONLY>
        <<<grid, kCtaThreads, kQuantSmem, stream>>>(a, a2, tmap);
    return cudaGetLastError();
}

// grid_kind: 0 E1M2, 1 E2M1, 2 restricted E2M1 (the uniform grids share GRID 0).
template <int AXIS, int NH, int BLK, bool AMAX_ONLY>
cudaError_t dispatch_grid_round(const QuantArgs &a, const QuantArgs &a2, const CUtensorMap &m, int grid_kind,
                                int rnd, int num_sms, cudaStream_t stream) {
    if (AMAX_ONLY) return launch_one<AXIS, NH, BLK, 0, 0, true>(a, a2, m, num_sms, stream);
    if (grid_kind != 1) {
        return rnd == 0 ? launch_one<AXIS, NH, BLK, 0, 0, false>(a, a2, m, num_sms, stream)
                        : launch_one<AXIS, NH, BLK, 0, 1, false>(a, a2, m, num_sms, stream);
    }
    return rnd == 0 ? launch_one<AXIS, NH, BLK, 1, 0, false>(a, a2, m, num_sms, stream)
                    : launch_one<AXIS, NH, BLK, 1, 1, false>(a, a2, m, num_sms, stream);
}

template <int AXIS, bool AMAX_ONLY>
cudaError_t dispatch_nh_blk(const QuantArgs &a, const QuantArgs &a2, const CUtensorMap &m, int nh, int blk,
                            int grid_kind, int rnd, int num_sms, cudaStream_t stream) {
    // The amax pass has no blocks: one instantiation per Hadamard size.
    if (AMAX_ONLY) blk = 16;
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

// bf16 input as a 2-D tensor map: rows x cols, row pitch ld; box 64 x 256
// (row-wise: K x rows, 128-byte swizzle) or 64 x 64 (column-wise: columns x
// K, no swizzle; dual: 128-byte swizzle).
cudaError_t make_input_map(const QuantArgs &a, CUtensorMap *m, bool dual) {
    const uint32_t box_outer = a.axis == 0 ? kUnitRows : 64;
    const CUtensorMapSwizzle swz =
        (a.axis == 0 || dual) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
    CUresult r = encode_tensor_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x,
                                      static_cast<uint64_t>(a.cols), static_cast<uint64_t>(a.rows),
                                      static_cast<uint64_t>(a.ld) * 2, 64, box_outer, swz);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_rht_quantize(QuantArgs a, int hadamard_n, int block, int grid_kind,
                                int rounding, int num_sms, cudaStream_t stream) {
    fill_call_constants(a, hadamard_n);
    a.grid = grid_kind;
    CUtensorMap m;
    cudaError_t e = make_input_map(a, &m, false);
    if (e != cudaSuccess) return e;
    if (a.axis == 0)
        return dispatch_nh_blk<0, false>(a, a, m, hadamard_n, block, grid_kind, rounding, num_sms, stream);
    return dispatch_nh_blk<1, false>(a, a, m, hadamard_n, block, grid_kind, rounding, num_sms, stream);
}

cudaError_t launch_rht_quantize_dual(QuantArgs a_rows, QuantArgs a_cols, int hadamard_n, int block,
                                     int grid_kind, int rounding, int num_sms, cudaStream_t stream) {
    fill_call_constants(a_rows, hadamard_n);
    fill_call_constants(a_cols, hadamard_n);
    a_rows.grid = a_cols.grid = grid_kind;
    CUtensorMap m;
    cudaError_t e = make_input_map(a_rows, &m, true);
    if (e != cudaSuccess) return e;
    return dispatch_nh_blk<2, false>(a_rows, a_cols, m, hadamard_n, block, grid_kind, rounding, num_sms,
                                     stream);
}

cudaError_t launch_rht_amax(QuantArgs a, int hadamard_n, int num_sms, cudaStream_t stream) {
    fill_call_constants(a, hadamard_n);
    a.grid = 0;
    cudaError_t e = cudaMemsetAsync(a.amax_out, 0, sizeof(float), stream);
    if (e != cudaSuccess) return e;
    CUtensorMap m;
    e = make_input_map(a, &m, false);
    if (e != cudaSuccess) return e;
    if (a.axis == 0) return dispatch_nh_blk<0, true>(a, a, m, hadamard_n, 16, 0, 0, num_sms, stream);
    return dispatch_nh_blk<1, true>(a, a, m, hadamard_n, 16, 0, 0, num_sms, stream);
}

cudaError_t launch_rht_amax_dual(QuantArgs a_rows, QuantArgs a_cols, int hadamard_n, int num_sms,
                                 cudaStream_t stream) {
    fill_call_constants(a_rows, hadamard_n);
    fill_call_constants(a_cols, hadamard_n);
    a_rows.grid = a_cols.grid = 0;
    cudaError_t e = cudaMemsetAsync(a_rows.amax_out, 0, sizeof(float), stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(a_cols.amax_out, 0, sizeof(float), stream);
    if (e != cudaSuccess) return e;
    CUtensorMap m;
    e = make_input_map(a_rows, &m, true);
    if (e != cudaSuccess) return e;
    return dispatch_nh_blk<2, true>(a_rows, a_cols, m, hadamard_n, 16, 0, 0, num_sms, stream);
}

cudaError_t launch_rht_bf16(QuantArgs a, int hadamard_n, uint16_t *y, int64_t ldy, int num_sms,
                            cudaStream_t stream) {
    fill_call_constants(a, hadamard_n);
    const int64_t total = a.rows * (a.cols / 64);
    if (total == 0) return cudaSuccess;
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    const int64_t need = (total + 255) / 256;
    const int grid = static_cast<int>(need < cap ? need : cap);
    switch (hadamard_n) {
        case 0: rht_bf16_kernel<0><<<grid, 256, 0, stream>>>(a, y, ldy); break;
        case 16: rht_bf16_kernel<16><<<grid, 256, 0, stream>>>(a, y, ldy); break;
        case 32: rht_bf16_kernel<32><<<grid, 256, 0, stream>>>(a, y, ldy); break;
        case 64: rht_bf16_kernel<64><<<grid, 256, 0, stream>>>(a, y, ldy); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t quantize_set_producer_wait_limit(uint64_t limit_ns) {
    const uint64_t v = limit_ns == 0 ? kWaitLimitNs : limit_ns;
    return cudaMemcpyToSymbol(g_producer_wait_limit_ns, &v, sizeof(v));
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
