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

#include "ufp4_device.cuh"
#include "ufp4_internal.h"

namespace ufp4 {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <int GRID>
__device__ __forceinline__ float level_of(int k) {
    if (GRID == 0) return static_cast<float>(k) * 0.25f;
    return k <= 4 ? static_cast<float>(k) * 0.5f : (k == 5 ? 3.0f : (k == 6 ? 4.0f : 6.0f));
}

// Midpoint between level j and level j+1 (j in 0..6), exact in fp32.
template <int GRID>
__device__ __forceinline__ float mid_of(int j) {
    if (GRID == 0) return static_cast<float>(2 * j + 1) * 0.125f;
    return j <= 3 ? static_cast<float>(2 * j + 1) * 0.25f
                  : (j == 4 ? 2.5f : (j == 5 ? 3.5f : 5.0f));
}

template <int GRID>
__device__ __forceinline__ float gmax_of() {
    return GRID == 0 ? 1.75f : 6.0f;
}

// Nearest level index of an approximate quotient y (within one of the truth).
template <int GRID>
__device__ __forceinline__ int estimate_nearest(float y) {
    if (GRID == 0) return min(max(__float2int_rn(y * 4.0f), 0), 7);
    return (y > 0.25f) + (y > 0.75f) + (y > 1.25f) + (y > 1.75f) + (y > 2.5f) + (y > 3.5f) +
           (y > 5.0f);
}

// Largest level index whose level is <= y (approximate, within one).
template <int GRID>
__device__ __forceinline__ int estimate_floor(float y) {
    if (GRID == 0) return min(max(__float2int_rd(y * 4.0f), 0), 7);
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
    int k = estimate_nearest<GRID>(au * inv);
    if (k > 0) {
        const float d = exact_diff(au, mid_of<GRID>(k - 1), m1, b);
        if (d < 0.0f || (d == 0.0f && (k & 1))) --k;
    }
    if (k < 7) {
        const float d = exact_diff(au, mid_of<GRID>(k), m1, b);
        if (d > 0.0f || (d == 0.0f && (k & 1))) ++k;
    }
    return k;
}

// Stochastic rounding between the adjacent levels lo <= au/s < hi: up iff
// au > (lo + r16 * 2^-16 * (hi - lo)) * s.
template <int GRID>
__device__ __forceinline__ int round_sr(float au, float m1, float b, float inv, uint32_t r16) {
    int lo = estimate_floor<GRID>(au * inv);
    if (lo > 0 && exact_diff(au, level_of<GRID>(lo), m1, b) < 0.0f) {
        --lo;
    } else if (lo < 7 && exact_diff(au, level_of<GRID>(lo + 1), m1, b) >= 0.0f) {
        ++lo;
    }
    if (lo >= 7) return 7;
    const float l0 = level_of<GRID>(lo);
    const float step = level_of<GRID>(lo + 1) - l0;
    const float c = __fmaf_rn(static_cast<float>(r16), step * (1.0f / 65536.0f), l0);
    return exact_diff(au, c, m1, b) > 0.0f ? lo + 1 : lo;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// In-place unnormalised Walsh-Hadamard transform of one 16-chunk plus the
// cross-lane stages of a 32 / 64 block.  Stage order h = 1, 2, ..., NH/2.
template <int NH>
__device__ __forceinline__ void fwht_chunk(float (&v)[16], int j) {
    if constexpr (NH > 0) {
#pragma unroll
        for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if (i & h) continue;
                const float a = v[i], b = v[i + h];
                v[i] = __fadd_rn(a, b);
                v[i + h] = __fsub_rn(a, b);
            }
        }
    }
    if constexpr (NH >= 32) {
        const bool upper = (j & 1) != 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float p = __shfl_xor_sync(0xFFFFFFFFu, v[i], 1);
            v[i] = upper ? __fsub_rn(p, v[i]) : __fadd_rn(v[i], p);
        }
    }
    if constexpr (NH >= 64) {
        const bool upper = (j & 2) != 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float p = __shfl_xor_sync(0xFFFFFFFFu, v[i], 2);
            v[i] = upper ? __fsub_rn(p, v[i]) : __fadd_rn(v[i], p);
        }
    }
}

// Signs of D for this lane's 16 positions (bit i: position i of the chunk).
template <int NH>
__device__ __forceinline__ uint32_t lane_sign_bits(uint64_t mask, int j) {
    if (NH == 0) return 0u;
    const int off = 16 * (j & (NH / 16 - 1));
    return static_cast<uint32_t>(mask >> off) & 0xFFFFu;
}

struct ScaleOut {
    float m1;    // factor folded into the threshold (1 or e_b)
    float b;     // fp32 scale multiplied inside the fma (s or S)
    float inv;   // approximate 1 / (m1 * b) for the estimate
    bool zero;   // block step is zero: every code 0
    uint32_t stored;  // fp32 bits of s, or the E4M3 byte
};

template <int GRID>
__device__ __forceinline__ ScaleOut block_scale(float amax, int scale_fmt, float S, float G) {
    ScaleOut o;
    if (scale_fmt == 0) {
        const float s = __fdiv_rn(amax, gmax_of<GRID>());
        o.m1 = 1.0f;
        o.b = s;
        o.zero = !(s > 0.0f);
        o.inv = o.zero ? 0.0f : __frcp_rn(s);
        o.stored = __float_as_uint(s);
    } else {
        const float q = __fdiv_rn(amax, G);
        const __nv_fp8_storage_t e8 = __nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3);
        const float e = e4m3_to_f32(e8);
        o.m1 = e;
        o.b = S;
        o.zero = !(e > 0.0f);
        o.inv = o.zero ? 0.0f : __frcp_rn(e * S);
        o.stored = e8;
    }
    return o;
}

// Round the 16 rotated values of one chunk and pack them (2 codes / byte,
// low nibble = lower K index).  Returns the 8 packed bytes.
template <int GRID, int RND>
__device__ __forceinline__ uint2 round_pack(const float (&v)[16], const ScaleOut &sc,
                                            uint64_t seed, uint32_t stream, uint64_t L0) {
    uint32_t rnd[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (RND == 1) {
        const uint2 key = make_uint2(static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
        const uint64_t g0 = L0 >> 3;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint64_t g = g0 + c;
            const uint4 r = philox4x32_10(
                make_uint4(static_cast<uint32_t>(g), static_cast<uint32_t>(g >> 32), stream, 0u), key);
            rnd[4 * c + 0] = r.x;
            rnd[4 * c + 1] = r.y;
            rnd[4 * c + 2] = r.z;
            rnd[4 * c + 3] = r.w;
        }
    }
    uint32_t w0 = 0, w1 = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float u = v[i];
        const float au = fabsf(u);
        int k = 0;
        if (!sc.zero) {
            if (RND == 0) {
                k = round_rtne<GRID>(au, sc.m1, sc.b, sc.inv);
            } else {
                const uint32_t word = rnd[i >> 1];
                const uint32_t r16 = (i & 1) ? (word >> 16) : (word & 0xFFFFu);
                k = round_sr<GRID>(au, sc.m1, sc.b, sc.inv, r16);
            }
        }
        uint32_t code = static_cast<uint32_t>(k);
        if (k != 0 && (__float_as_uint(u) >> 31)) code |= 8u;
        if (i < 8) w0 |= code << (4 * i);
        else w1 |= code << (4 * (i - 8));
    }
    return make_uint2(w0, w1);
}

struct Loaded {
    uint4 q[16];
};

// Row-wise: lane loads elements [k0, k0+16) of its row.
__device__ __forceinline__ void load_rowwise(const QuantArgs &a, int64_t row, int64_t k0,
                                             uint4 &q0, uint4 &q1) {
    q0 = make_uint4(0, 0, 0, 0);
    q1 = make_uint4(0, 0, 0, 0);
    if (row >= a.rows) return;
    const uint16_t *p = a.x + row * a.ld + k0;
    if (k0 < a.cols) q0 = __ldg(reinterpret_cast<const uint4 *>(p));
    if (k0 + 8 < a.cols) q1 = __ldg(reinterpret_cast<const uint4 *>(p + 8));
}

// Column-wise: lane loads input rows [k0, k0+16) x columns [c0, c0+8).
__device__ __forceinline__ void load_colwise(const QuantArgs &a, int64_t k0, int64_t c0,
                                             uint4 (&q)[16]) {
    const bool col_ok = c0 < a.cols;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        q[i] = make_uint4(0, 0, 0, 0);
        if (col_ok && k0 + i < a.rows)
            q[i] = __ldg(reinterpret_cast<const uint4 *>(a.x + (k0 + i) * a.ld + c0));
    }
}

__device__ __forceinline__ uint32_t pick_word(const uint4 &q, int w) {
    return w == 0 ? q.x : (w == 1 ? q.y : (w == 2 ? q.z : q.w));
}

template <int AXIS, int NH, int BLK, int GRID, int RND, bool AMAX_ONLY>
__global__ void __launch_bounds__(kThreads) rht_quantize_kernel(const QuantArgs a) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int j = lane & 3;
    const int g = lane >> 2;
    const int64_t nseg = a.kpad / 64;

    float S = 1.0f, G = 0.0f;
    if (!AMAX_ONLY && a.scale_fmt == 1) {
        const float amax_t = *a.amax_t;
        S = amax_t > 0.0f ? __fdiv_rn(amax_t, gmax_of<GRID>() * 448.0f) : 1.0f;
        G = __fmul_rn(gmax_of<GRID>(), S);
        if (blockIdx.x == 0 && threadIdx.x == 0 && a.S_out) *a.S_out = S;
    }
    const uint32_t sgn = lane_sign_bits<NH>(a.sign_mask, j);
    float amax_acc = 0.0f;

    const int64_t total_warps = static_cast<int64_t>(gridDim.x) * kWarps;
    for (int64_t unit = static_cast<int64_t>(blockIdx.x) * kWarps + warp; unit < a.num_units;
         unit += total_warps) {
        int64_t seg, rbase;
        if (AXIS == 0) {
            seg = unit % nseg;
            rbase = (unit / nseg) * 8;
        } else {
            const int64_t ncb = (a.out_rows + 63) / 64;
            seg = unit / ncb;
            rbase = (unit % ncb) * 64;
        }
        const int64_t k0 = seg * 64 + 16 * j;

        uint4 q[16];
        if (AXIS == 0) {
            load_rowwise(a, rbase + g, k0, q[0], q[1]);
        } else {
            load_colwise(a, k0, rbase + 8 * g, q);
        }

        constexpr int kRowsPerLane = AXIS == 0 ? 1 : 8;
        float col_scales[8];
#pragma unroll
        for (int rr = 0; rr < kRowsPerLane; ++rr) {
            float v[16];
            if (AXIS == 0) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t w0 = pick_word(q[0], i >> 1);
                    const uint32_t w1 = pick_word(q[1], i >> 1);
                    v[i] = (i & 1) ? bf16_hi(w0) : bf16_lo(w0);
                    v[i + 8] = (i & 1) ? bf16_hi(w1) : bf16_lo(w1);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint32_t w = pick_word(q[i], rr >> 1);
                    v[i] = (rr & 1) ? bf16_hi(w) : bf16_lo(w);
                }
            }
            // D: exact negation where the sign mask bit is set.
#pragma unroll
            for (int i = 0; i < 16; ++i)
                v[i] = __uint_as_float(__float_as_uint(v[i]) ^ (((sgn >> i) & 1u) << 31));
            fwht_chunk<NH>(v, j);

            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
            if (AMAX_ONLY) {
                amax_acc = fmaxf(amax_acc, amax);
                continue;
            }
            if (BLK == 32) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));

            const ScaleOut sc = block_scale<GRID>(amax, a.scale_fmt, S, G);
            const int64_t orow = AXIS == 0 ? rbase + g : rbase + 8 * g + rr;
            const uint64_t L0 = static_cast<uint64_t>(orow) * static_cast<uint64_t>(a.kpad) +
                                static_cast<uint64_t>(k0);
            const uint2 packed = round_pack<GRID, RND>(v, sc, a.seed, a.stream, L0);

            if (orow < a.out_rows) {
                *reinterpret_cast<uint2 *>(a.codes + orow * (a.kpad / 2) + k0 / 2) = packed;
                const int64_t blk = k0 / BLK;
                const bool writer = (BLK == 16) || ((j & 1) == 0);
                if (AXIS == 0 && writer) {
                    if (a.scale_fmt == 0)
                        reinterpret_cast<uint32_t *>(a.scales)[blk * a.scale_ld + orow] = sc.stored;
                    else
                        reinterpret_cast<uint8_t *>(a.scales)[blk * a.scale_ld + orow] =
                            static_cast<uint8_t>(sc.stored);
                }
            }
            col_scales[rr] = __uint_as_float(sc.stored);
        }
        if (!AMAX_ONLY && AXIS == 1) {
            // 8 consecutive output rows of one block: one 32-byte (fp32) or
            // 8-byte (E4M3) store per lane.
            const int64_t c0 = rbase + 8 * g;
            const int64_t blk = k0 / BLK;
            const bool writer = (BLK == 16) || ((j & 1) == 0);
            if (writer && c0 < a.out_rows) {
                if (a.scale_fmt == 0) {
                    float4 *dst = reinterpret_cast<float4 *>(
                        reinterpret_cast<float *>(a.scales) + blk * a.scale_ld + c0);
                    dst[0] = make_float4(col_scales[0], col_scales[1], col_scales[2], col_scales[3]);
                    dst[1] = make_float4(col_scales[4], col_scales[5], col_scales[6], col_scales[7]);
                } else {
                    uint32_t lo = 0, hi = 0;
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        lo |= (__float_as_uint(col_scales[r]) & 0xFFu) << (8 * r);
                        hi |= (__float_as_uint(col_scales[r + 4]) & 0xFFu) << (8 * r);
                    }
                    *reinterpret_cast<uint2 *>(reinterpret_cast<uint8_t *>(a.scales) +
                                               blk * a.scale_ld + c0) = make_uint2(lo, hi);
                }
            }
        }
    }
    if (AMAX_ONLY) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            amax_acc = fmaxf(amax_acc, __shfl_xor_sync(0xFFFFFFFFu, amax_acc, off));
        if (lane == 0 && amax_acc > 0.0f)
            atomicMax(reinterpret_cast<unsigned int *>(a.amax_out), __float_as_uint(amax_acc));
    }
}

template <int AXIS, int NH, int BLK, int GRID, int RND, bool AMAX_ONLY>
cudaError_t launch_one(const QuantArgs &a, int num_sms, cudaStream_t stream) {
    const int64_t blocks_needed = (a.num_units + kWarps - 1) / kWarps;
    const int64_t cap = static_cast<int64_t>(num_sms) * (AXIS == 0 ? 8 : 4);
    const int grid = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
    if (grid <= 0) return cudaSuccess;
    rht_quantize_kernel<AXIS, NH, BLK, GRID, RND, AMAX_ONLY><<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

template <int AXIS, int NH, int BLK, bool AMAX_ONLY>
cudaError_t dispatch_grid_round(const QuantArgs &a, int grid_kind, int rnd, int num_sms,
                                cudaStream_t stream) {
    if (AMAX_ONLY) return launch_one<AXIS, NH, BLK, 0, 0, true>(a, num_sms, stream);
    if (grid_kind == 0) {
        return rnd == 0 ? launch_one<AXIS, NH, BLK, 0, 0, false>(a, num_sms, stream)
                        : launch_one<AXIS, NH, BLK, 0, 1, false>(a, num_sms, stream);
    }
    return rnd == 0 ? launch_one<AXIS, NH, BLK, 1, 0, false>(a, num_sms, stream)
                    : launch_one<AXIS, NH, BLK, 1, 1, false>(a, num_sms, stream);
}

template <int AXIS, bool AMAX_ONLY>
cudaError_t dispatch_nh_blk(const QuantArgs &a, int nh, int blk, int grid_kind, int rnd,
                            int num_sms, cudaStream_t stream) {
#define UFP4_CASE(N, B)                                                                     \
    if (nh == N && blk == B)                                                                \
        return dispatch_grid_round<AXIS, N, B, AMAX_ONLY>(a, grid_kind, rnd, num_sms, stream);
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

}  // namespace

cudaError_t launch_rht_quantize(QuantArgs a, int hadamard_n, int block, int grid_kind,
                                int rounding, int num_sms, cudaStream_t stream) {
    if (a.axis == 0) {
        a.num_units = ((a.out_rows + 7) / 8) * (a.kpad / 64);
        return dispatch_nh_blk<0, false>(a, hadamard_n, block, grid_kind, rounding, num_sms, stream);
    }
    a.num_units = ((a.out_rows + 63) / 64) * (a.kpad / 64);
    return dispatch_nh_blk<1, false>(a, hadamard_n, block, grid_kind, rounding, num_sms, stream);
}

cudaError_t launch_rht_amax(QuantArgs a, int hadamard_n, int num_sms, cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(a.amax_out, 0, sizeof(float), stream);
    if (e != cudaSuccess) return e;
    if (a.axis == 0) {
        a.num_units = ((a.out_rows + 7) / 8) * (a.kpad / 64);
        return dispatch_nh_blk<0, true>(a, hadamard_n, 16, 0, 0, num_sms, stream);
    }
    a.num_units = ((a.out_rows + 63) / 64) * (a.kpad / 64);
    return dispatch_nh_blk<1, true>(a, hadamard_n, 16, 0, 0, num_sms, stream);
}

}  // namespace ufp4
