// gemm.cu -- block-scaled 4-bit TN contraction on tcgen05 tensor cores.
//
// C[i][j] = (1/n) * sum_k deq(A)[i][k] * deq(B)[j][k]   (fp32 accumulate)
//
// Both operands arrive K-major as packed sign-magnitude nibbles plus block
// scales, exactly as ufp4_rht_quantize writes them.  FPROP, DGRAD and WGRAD
// are the same kernels: the quantizer already laid every operand out along its
// GEMM's reduction dimension (paperlayer.ai summary §2, "for the three
// training GEMMs, RHT acts along the shared reduction dimension").
//
// Kernel families (all persistent over output tiles, warp-specialised, every
// wait bounded: a stuck pipeline sets the device error word and the CTA
// unwinds, drains its copies and frees TMEM):
//   gemm_pair_kernel<0/1>  two-level (E4M3 x fp32) scales, the default: CTA
//       pairs (cta_group::2) with 256 x 256 tiles on the block-scaled FP4 MMA
//       (kind::mxf4nvf4, UE4M3 factors per 16 elements).  E1M2 codes split
//       exactly into two E2M1 planes, four MMAs per K step.  The factors come
//       as the quantizer's factor atoms and the MMA issuer copies them into
//       TMEM (tcgen05.cp), or, for grouped problems and operands without
//       atoms, factor warps build them from the block-major scales.
//   gemm_pair_kernel<3>    MX operands (UE8M0, block 32): the E4M3 element
//       planes on the block-scaled FP8 MMA (kind::mxf8f6f4), factors in the MMA.
//   gemm_fp4_kernel        two-level scales with one CTA per 128 x 192 tile
//       (E1M2 operands whose correction planes are not stored next to their
//       codes, or when the caller picks it).
//   gemm_f32s_kernel       fp32 or UE8M0 block scales without element planes:
//       codes expanded to fp16, one K = 16 MMA per block into its own TMEM
//       partial, s_a * s_b * partial accumulated in fp32 registers.

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#define UFP4_PIPELINE_KERNELS 1
#include "ufp4_device.cuh"
#include "ufp4_internal.h"

namespace ufp4 {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;             // K elements per pipeline stage
constexpr int kCodeRow = BK / 2;   // packed bytes per row per stage
constexpr int kOpRow = BK * 2;     // fp16 bytes per row per stage (= 128)

// fp32 (or UE8M0) block scales: no MMA kind applies an fp32 factor per block,
// so every 16-element K block is one K = 16 fp16 MMA into its own TMEM partial
// buffer (an exact partial: a sum of at most 16 products on a 1/16 lattice,
// E1M2 as k, E2M1 as its level), and the epilogue warps accumulate
// s_a * s_b * partial in fp32 registers.  The loop is bound by the round trip
// of a partial buffer (MMA -> commit -> epilogue load -> release -> MMA) over
// the four buffers TMEM holds, not by either pipe's throughput.
// One CTA per SM per 128 x 128 output tile, persistent over tiles.
struct F32sCfg {
    static constexpr int BN = 128;    // B rows staged per stage (= tile columns)
    static constexpr int TM = 128;
    static constexpr int TN = 128;
    static constexpr int NT = 2;      // transform warps: codes -> fp16
    static constexpr int NE = 8;      // epilogue warps: 2 per TMEM lane quarter, 64 columns each
    static constexpr int NC = 4;      // code ring slots
    static constexpr int NO = 3;      // fp16 operand ring slots
    static constexpr int NS = 4;      // scale ring slots
    static constexpr int NP = 4;      // TMEM partial buffers (BN columns each)
    static constexpr int kOpA = BM * kOpRow;
    static constexpr int kOpB = BN * kOpRow;
    static constexpr int kCodeA = BM * kCodeRow;
    static constexpr int kCodeB = BN * kCodeRow;
    // fp32 scales of the smallest block (16): BK / 16 blocks per stage
    static constexpr int kScA = BM * (BK / 16) * 4;
    static constexpr int kScB = BN * (BK / 16) * 4;
    // code slots start on 1024-byte boundaries (the 32-byte TMA swizzle)
    static constexpr int kCodeSlot = (kCodeA + kCodeB + 1023) / 1024 * 1024;
    static constexpr int kScSlot = kScA + kScB;
    static constexpr int off_op = 0;
    static constexpr int off_code = off_op + NO * (kOpA + kOpB);
    static constexpr int off_sc = off_code + NC * kCodeSlot;
    static constexpr int off_bar = (off_sc + NS * kScSlot + 127) / 128 * 128;
    // barriers: code_full, code_empty, op_full, op_empty, sc_full, sc_empty,
    //           p_full, p_empty, drain
    static constexpr int kNumBars = 2 * NC + 2 * NO + 2 * NS + 2 * NP + 1;
    static constexpr int off_misc = off_bar + kNumBars * 8;
    static constexpr int kAlloc = off_misc + 64 + 1024;   // slack for 1024-byte alignment
    static constexpr int kThreads = 32 * (2 + NT + NE);
    static constexpr int kTmemCols = 512;
    static_assert(NP * BN <= kTmemCols, "TMEM budget");
    static_assert(kThreads % 128 == 0, "whole warp quads");
    static_assert(NE == 8, "epilogue: 2 warps per lane quarter, 64 columns each");
    static_assert(kAlloc <= 232448, "shared memory budget");
};

struct Tile {
    GemmGroup g;
    int64_t m0, n0;
    int nks;   // K stages
};

__device__ __forceinline__ bool group_ok(const GemmGroup &g) {
    return g.m >= 0 && g.n >= 0 && g.k >= 0 && (g.k % 64) == 0 && (g.a_col % 64) == 0 &&
           (g.b_col % 64) == 0 && (g.a_row % 16) == 0 && (g.b_row % 16) == 0 && g.a_row >= 0 &&
           g.b_row >= 0 && g.c_row >= 0 && g.c_col >= 0;
}

template <int TM, int TN>
__device__ __forceinline__ int64_t tiles_of(const GemmGroup &g) {
    if (!group_ok(g)) return 0;
    return ((g.m + TM - 1) / TM) * ((g.n + TN - 1) / TN);
}

__device__ __forceinline__ GemmGroup load_group(const GemmArgs &a, int i) {
    if (a.groups == nullptr) return a.single;
    GemmGroup g;
    const int64_t *p = reinterpret_cast<const int64_t *>(a.groups + i);
    g.m = __ldg(p + 0);
    g.n = __ldg(p + 1);
    g.k = __ldg(p + 2);
    g.a_row = __ldg(p + 3);
    g.a_col = __ldg(p + 4);
    g.b_row = __ldg(p + 5);
    g.b_col = __ldg(p + 6);
    g.c_row = __ldg(p + 7);
    g.c_col = __ldg(p + 8);
    return g;
}

template <int TM, int TN>
__device__ int64_t total_tiles(const GemmArgs &a) {
    const int ng = a.groups == nullptr ? 1 : a.num_groups;
    int64_t t = 0;
    for (int i = 0; i < ng; ++i) t += tiles_of<TM, TN>(load_group(a, i));
    return t;
}

// Tile t of the concatenated schedule (groups in order).  Inside a problem
// the M tiles go in bands of a.band rows of tiles, each band swept across all
// of N with M fastest inside it: the tiles in flight at once (one per SM or
// SM pair) then share a few operand panels in L2, and a panel is read from
// HBM about once per band instead of once per column of tiles.  In a step
// that runs at the power cap the saved DRAM traffic is clock headroom.
// Tile t (of nt) of one problem g.
template <int TM, int TN>
__device__ __forceinline__ Tile tile_in_group(const GemmArgs &a, const GemmGroup &g, int64_t t, int64_t nt) {
    Tile tl;
    const int64_t mt = (g.m + TM - 1) / TM;
    int64_t mi = t % mt, ni = t / mt;
    if (a.band > 0 && mt > a.band) {
        const int64_t per = static_cast<int64_t>(a.band) * (nt / mt);   // tiles of a full band
        const int64_t b = t / per, r = t - b * per;
        const int64_t h = min(static_cast<int64_t>(a.band), mt - b * a.band);   // rows of tiles in band b
        mi = b * a.band + r % h;
        ni = r / h;
    }
    tl.g = g;
    tl.m0 = mi * TM;
    tl.n0 = ni * TN;
    tl.nks = static_cast<int>(g.k / BK);
    return tl;
}

template <int TM, int TN>
__device__ Tile get_tile(const GemmArgs &a, int64_t t) {
    const int ng = a.groups == nullptr ? 1 : a.num_groups;
    for (int i = 0; i < ng; ++i) {
        const GemmGroup g = load_group(a, i);
        const int64_t nt = tiles_of<TM, TN>(g);
        if (t < nt) return tile_in_group<TM, TN>(a, g, t, nt);
        t -= nt;
    }
    Tile tl;
    tl.g = a.single;
    tl.m0 = tl.n0 = 0;
    tl.nks = 0;
    return tl;
}

// A grouped schedule precomputed in shared memory: order[r] is the group
// scheduled r-th and cum[r] the number of tiles of the groups before it
// (cum[ng] = all tiles).  Tile t is found by binary search.
struct GroupSchedule {
    const uint16_t *order;
    const int64_t *cum;
    int ng;
};

template <int TM, int TN>
__device__ Tile get_tile(const GemmArgs &a, int64_t t, const GroupSchedule &gs) {
    if (gs.order == nullptr) return get_tile<TM, TN>(a, t);
    int lo = 0, hi = gs.ng;              // largest r with cum[r] <= t
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (gs.cum[mid] <= t) lo = mid;
        else hi = mid;
    }
    const GemmGroup g = load_group(a, gs.order[lo]);
    return tile_in_group<TM, TN>(a, g, t - gs.cum[lo], gs.cum[lo + 1] - gs.cum[lo]);
}

// ---------------------------------------------------------------------------
// 4-bit code -> fp16 expansion.  A 32-bit word holds 8 codes (nibble i = K
// index i).  Output word i (i = 0..3) holds the fp16 pair (code i, code i+4):
// the same K permutation inside every 8-element chunk of both operands, which
// leaves every dot product (and every 16-block) unchanged.
//
// E1M2 carries the magnitude index k (the level is k/4; the 1/4 moves to the
// epilogue); E2M1 carries the level itself.  Both are exact in fp16.

// Sign bits of codes i and i+4 (nibble bit 3) moved to fp16 bits 15 and 31.
template <int I>
__device__ __forceinline__ uint32_t sign_pair(uint32_t w) {
    return (w << (12 - 4 * I)) & 0x80008000u;
}

// k of codes I and I+4 placed in mantissa bits 7..9 of fp16 8.0 (0x4800):
// the pair (8 + k_I, 8 + k_{I+4}).
template <int I>
__device__ __forceinline__ uint32_t eight_plus_k(uint32_t w) {
    const uint32_t t = (I <= 1) ? (w << (7 - 4 * I)) : (w >> (4 * I - 7));
    return (t & 0x03800380u) | 0x48004800u;
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

// Expansion of 8 codes: k (E1M2) or lvl (E2M1).
template <int GRID>
__device__ __forceinline__ void expand_unscaled(uint32_t w, uint32_t (&o)[4]) {
    if (GRID == 0) {
        const __half2 eight = __half2(__ushort_as_half(0x4800), __ushort_as_half(0x4800));
        o[0] = h2_bits(__hsub2(bits_h2(eight_plus_k<0>(w)), eight)) ^ sign_pair<0>(w);
        o[1] = h2_bits(__hsub2(bits_h2(eight_plus_k<1>(w)), eight)) ^ sign_pair<1>(w);
        o[2] = h2_bits(__hsub2(bits_h2(eight_plus_k<2>(w)), eight)) ^ sign_pair<2>(w);
        o[3] = h2_bits(__hsub2(bits_h2(eight_plus_k<3>(w)), eight)) ^ sign_pair<3>(w);
    } else {
        // fp16 high byte of {0,.5,1,1.5,2,3,4,6}; the low byte is always 0.
        const uint32_t m = w & 0x77777777u;
        const uint32_t lo = __byte_perm(0x3E3C3800u, 0x46444240u, m);
        const uint32_t hi = __byte_perm(0x3E3C3800u, 0x46444240u, m >> 16);
        o[0] = (__byte_perm(lo, hi, 0x4000u) & 0xFF00FF00u) ^ sign_pair<0>(w);
        o[1] = (__byte_perm(lo, hi, 0x5010u) & 0xFF00FF00u) ^ sign_pair<1>(w);
        o[2] = (__byte_perm(lo, hi, 0x6020u) & 0xFF00FF00u) ^ sign_pair<2>(w);
        o[3] = (__byte_perm(lo, hi, 0x7030u) & 0xFF00FF00u) ^ sign_pair<3>(w);
    }
}

// ---------------------------------------------------------------------------
// 2^(E - 127) of a UE8M0 byte E <= 254: the byte is the fp32 exponent field
// (E = 0 is the subnormal 2^-127).
__device__ __forceinline__ float ue8m0_to_f32(uint32_t e) {
    return __uint_as_float(e ? (e << 23) : 0x00400000u);
}

template <int GRID, bool UE8>
__global__ void __launch_bounds__(F32sCfg::kThreads, 1)
    gemm_f32s_kernel(const __grid_constant__ GemmArgs args) {
    using C = F32sCfg;
    constexpr int BN = C::BN, TM = C::TM, TN = C::TN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::off_bar);
    uint64_t *code_full = bars;
    uint64_t *code_empty = code_full + C::NC;
    uint64_t *op_full = code_empty + C::NC;
    uint64_t *op_empty = op_full + C::NO;
    uint64_t *sc_full = op_empty + C::NO;
    uint64_t *sc_empty = sc_full + C::NS;
    uint64_t *p_full = sc_empty + C::NS;
    uint64_t *p_empty = p_full + C::NP;
    uint64_t *drain = p_empty + C::NP;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::off_misc);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + C::off_misc + 4);

    auto op_a = [&](int s) { return smem + C::off_op + s * (C::kOpA + C::kOpB); };
    auto op_b = [&](int s) { return op_a(s) + C::kOpA; };
    auto code_a = [&](int s) { return smem + C::off_code + s * C::kCodeSlot; };
    auto code_b = [&](int s) { return code_a(s) + C::kCodeA; };
    auto sc_a = [&](int s) { return smem + C::off_sc + s * C::kScSlot; };
    auto sc_b = [&](int s) { return sc_a(s) + C::kScA; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nblk_stage = BK / args.block;
    const int64_t unit = blockIdx.x;
    const int64_t nunits = gridDim.x;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NC; ++i) {
            mbar_init(&code_full[i], 1);
            mbar_init(&code_empty[i], C::NT);
        }
        for (int i = 0; i < C::NO; ++i) {
            mbar_init(&op_full[i], C::NT);
            mbar_init(&op_empty[i], 1);
        }
        for (int i = 0; i < C::NS; ++i) {
            mbar_init(&sc_full[i], 1);
            mbar_init(&sc_empty[i], C::NE);
        }
        for (int i = 0; i < C::NP; ++i) {
            mbar_init(&p_full[i], 1);
            mbar_init(&p_empty[i], C::NE);
        }
        mbar_init(drain, 1);
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&args.tm_a_codes);
        tma_prefetch_desc(&args.tm_b_codes);
        tma_prefetch_desc(&args.tm_a_scales);
        tma_prefetch_desc(&args.tm_b_scales);
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int64_t ntiles = total_tiles<TM, TN>(args);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t it = 0, sit = 0;
            bool ok = true;
            for (int64_t t = unit; t < ntiles && ok; t += nunits) {
                const Tile tl = get_tile<TM, TN>(args, t);
                const int32_t arow = static_cast<int32_t>(tl.g.a_row + tl.m0);
                const int32_t brow = static_cast<int32_t>(tl.g.b_row + tl.n0);
                for (int ks = 0; ks < tl.nks; ++ks, ++it) {
                    const int s = it % C::NC;
                    const uint32_t use = it / C::NC;
                    if (!mbar_wait(&code_empty[s], (use & 1) ^ 1, kErrTimeoutProducer, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int32_t acol = static_cast<int32_t>(tl.g.a_col + ks * BK);
                    const int32_t bcol = static_cast<int32_t>(tl.g.b_col + ks * BK);
                    mbar_arrive_expect_tx(&code_full[s], C::kCodeA + C::kCodeB);
                    tma_load_2d(code_a(s), &args.tm_a_codes, &code_full[s], acol / 2, arow);
                    tma_load_2d(code_b(s), &args.tm_b_codes, &code_full[s], bcol / 2, brow);
                    const int ss = sit % C::NS;
                    const uint32_t suse = sit / C::NS;
                    if (!mbar_wait(&sc_empty[ss], (suse & 1) ^ 1, kErrTimeoutProducer, abort_flag)) {
                        ok = false;
                        ++it;   // the code copies of this stage were issued
                        break;
                    }
                    mbar_arrive_expect_tx(&sc_full[ss], (BM + BN) * nblk_stage * (args.scale_ue8m0 ? 1 : 4));
                    tma_load_2d(sc_a(ss), &args.tm_a_scales, &sc_full[ss], arow, acol / args.block);
                    tma_load_2d(sc_b(ss), &args.tm_b_scales, &sc_full[ss], brow, bcol / args.block);
                    ++sit;
                }
            }
            // Drain: wait (time-bounded, regardless of abort) until the last
            // copy issued into every slot has landed.
            for (int s = 0; s < C::NC; ++s) {
                if (it > static_cast<uint32_t>(s)) {
                    const uint32_t last = (it - 1 - s) / C::NC * C::NC + s;
                    uint32_t dummy = 0;
                    mbar_wait(&code_full[s], (last / C::NC) & 1, kErrTimeoutDrain,
                              reinterpret_cast<volatile uint32_t *>(&dummy));
                }
            }
            for (int s = 0; s < C::NS; ++s) {
                if (sit > static_cast<uint32_t>(s)) {
                    const uint32_t last = (sit - 1 - s) / C::NS * C::NS + s;
                    uint32_t dummy = 0;
                    mbar_wait(&sc_full[s], (last / C::NS) & 1, kErrTimeoutDrain,
                              reinterpret_cast<volatile uint32_t *>(&dummy));
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ UMMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_f16_f32(BM, BN);
            uint32_t it = 0, pq = 0;
            bool ok = true;
            for (int64_t t = unit; t < ntiles && ok; t += nunits) {
                const Tile tl = get_tile<TM, TN>(args, t);
                for (int ks = 0; ks < tl.nks && ok; ++ks, ++it) {
                    const int s = it % C::NO;
                    if (!mbar_wait(&op_full[s], (it / C::NO) & 1, kErrTimeoutMma, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_addr(op_a(s));
                    const uint32_t b0 = smem_addr(op_b(s));
                    const int slices = args.block / 16;
                    for (int bi = 0; bi < nblk_stage; ++bi, ++pq) {
                        const int p = pq % C::NP;
                        if (!mbar_wait(&p_empty[p], ((pq / C::NP) & 1) ^ 1, kErrTimeoutMma, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        for (int sl = 0; sl < slices; ++sl) {
                            const int kk = bi * slices + sl;
                            umma_f16(tmem_base + p * BN, umma_desc_sw128(a0 + kk * 32), umma_desc_sw128(b0 + kk * 32),
                                     idesc, sl > 0 ? 1u : 0u);
                        }
                        umma_commit(&p_full[p]);
                    }
                    umma_commit(&op_empty[s]);
                }
            }
            // Drain: every MMA issued by this thread completes before TMEM is freed.
            umma_commit(drain);
            uint32_t dummy = 0;
            mbar_wait(drain, 0, kErrTimeoutDrain, reinterpret_cast<volatile uint32_t *>(&dummy));
        }
    } else if (warp < 2 + C::NT) {
        // ------------------------------------------------------------ transform
        // One operand row (64 codes, 32 bytes) per thread per pass.  The code
        // tiles arrive with the 32-byte TMA swizzle: the two 16-byte halves of
        // row r are swapped when bit 2 of r is set, so the lanes of a quarter
        // warp read distinct banks.
        const int tt = threadIdx.x - 64;
        constexpr int kRows = BM + BN;
        uint32_t it = 0;
        bool ok = true;
        for (int64_t t = unit; t < ntiles && ok; t += nunits) {
            const Tile tl = get_tile<TM, TN>(args, t);
            for (int ks = 0; ks < tl.nks; ++ks, ++it) {
                const int cs = it % C::NC;
                const int os = it % C::NO;
                if (!warp_wait(&code_full[cs], (it / C::NC) & 1, kErrTimeoutTransform, abort_flag) ||
                    !warp_wait(&op_empty[os], ((it / C::NO) & 1) ^ 1, kErrTimeoutTransform, abort_flag)) {
                    ok = false;
                    break;
                }
                const uint8_t *ca = code_a(cs);
                const uint8_t *cb = code_b(cs);
                uint8_t *oa = op_a(os);
                uint8_t *ob = op_b(os);
#pragma unroll 1
                for (int row = tt; row < kRows; row += C::NT * 32) {
                    const bool isA = row < BM;
                    const int r = isA ? row : row - BM;
                    const uint8_t *src = (isA ? ca : cb) + r * kCodeRow;
                    const int flip = (r >> 2) & 1;
                    const uint4 h0 = *reinterpret_cast<const uint4 *>(src + (flip << 4));
                    const uint4 h1 = *reinterpret_cast<const uint4 *>(src + ((flip ^ 1) << 4));
                    const uint32_t words[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
                    uint8_t *dst = (isA ? oa : ob) + r * 128;
                    const uint32_t sw = static_cast<uint32_t>(r & 7);
#pragma unroll
                    for (int wi = 0; wi < 8; ++wi) {
                        uint32_t o[4];
                        expand_unscaled<GRID>(words[wi], o);
                        *reinterpret_cast<uint4 *>(dst + ((static_cast<uint32_t>(wi) ^ sw) << 4)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&op_full[os]);
                    mbar_arrive(&code_empty[cs]);
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // acc += (s_a * s_b) * partial per 16/32-block: thread = accumulator
        // row (its TMEM lane), 64 columns per warp.
        const int ew = warp - 2 - C::NT;      // 0 .. NE-1
        const int q = warp & 3;               // TMEM lane quarter of this warp
        const int cs = ew >> 2;               // column half: 64 columns
        const int row_in_tile = 32 * q + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
        const float mult = args.inv_n * (GRID == 0 ? (1.0f / 16.0f) : 1.0f);
        uint32_t it = 0, pq = 0;
        bool ok = true;
        for (int64_t t = unit; t < ntiles && ok; t += nunits) {
            const Tile tl = get_tile<TM, TN>(args, t);
            float2 acc[32];   // columns 2i, 2i + 1 of the warp's 64
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[i] = make_float2(0.0f, 0.0f);
            for (int ks = 0; ks < tl.nks && ok; ++ks, ++it) {
                const int ss = it % C::NS;
                if (!warp_wait(&sc_full[ss], (it / C::NS) & 1, kErrTimeoutEpilogue, abort_flag)) {
                    ok = false;
                    break;
                }
                const float *sa_tile = reinterpret_cast<const float *>(sc_a(ss));
                const float *sb_tile = reinterpret_cast<const float *>(sc_b(ss));
                // UE8M0 scales: exponent bytes in the same slots, 2^(E - 127)
                const uint8_t *sa_u8 = sc_a(ss);
                const uint8_t *sb_u8 = sc_b(ss);
                for (int bi = 0; bi < nblk_stage; ++bi, ++pq) {
                    const int p = pq % C::NP;
                    if (!warp_wait(&p_full[p], (pq / C::NP) & 1, kErrTimeoutEpilogue, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const float sa = UE8 ? ue8m0_to_f32(sa_u8[bi * BM + row_in_tile]) : sa_tile[bi * BM + row_in_tile];
                    const float2 sa2 = make_float2(sa, sa);
                    const float4 *sb4 = reinterpret_cast<const float4 *>(sb_tile + bi * BN + cs * 64);
                    const uchar4 *sb4u = reinterpret_cast<const uchar4 *>(sb_u8 + bi * BN + cs * 64);
                    const uint32_t ta = tmem_base + p * BN + cs * 64 + lane_addr;
                    uint32_t r[2][32];
                    tmem_ld_32x32b_x32(ta, r[0]);
                    tmem_ld_32x32b_x32(ta + 32, r[1]);
                    tmem_wait_ld();
                    // partial buffer p read: the MMAs may refill it
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&p_empty[p]);
                    // Two columns per packed fp32x2 operation: the same
                    // per-lane IEEE product s_a s_b and fused accumulate.
#pragma unroll
                    for (int c4 = 0; c4 < 16; ++c4) {
                        float4 sb;
                        if constexpr (UE8) {
                            const uchar4 e = sb4u[c4];
                            sb = make_float4(ue8m0_to_f32(e.x), ue8m0_to_f32(e.y), ue8m0_to_f32(e.z),
                                             ue8m0_to_f32(e.w));
                        } else {
                            sb = sb4[c4];
                        }
                        const uint32_t *rr = r[c4 >> 3] + 4 * (c4 & 7);
                        const float2 s01 = __fmul2_rn(sa2, make_float2(sb.x, sb.y));
                        const float2 s23 = __fmul2_rn(sa2, make_float2(sb.z, sb.w));
                        acc[2 * c4] = __ffma2_rn(s01, make_float2(__uint_as_float(rr[0]), __uint_as_float(rr[1])),
                                                 acc[2 * c4]);
                        acc[2 * c4 + 1] = __ffma2_rn(
                            s23, make_float2(__uint_as_float(rr[2]), __uint_as_float(rr[3])), acc[2 * c4 + 1]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sc_empty[ss]);
            }
            if (!ok) break;
            const int64_t row = tl.m0 + row_in_tile;
            if (row < tl.g.m) {
                const int64_t col0 = tl.n0 + 64 * cs;
                float *dst = args.c + (tl.g.c_row + row) * args.ldc + tl.g.c_col + col0;
                const bool vec = (col0 + 64 <= tl.g.n) && ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0);
                if (vec) {
#pragma unroll
                    for (int i = 0; i < 32; i += 2)
                        *reinterpret_cast<float4 *>(dst + 2 * i) = make_float4(
                            acc[i].x * mult, acc[i].y * mult, acc[i + 1].x * mult, acc[i + 1].y * mult);
                } else {
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        if (col0 + i < tl.g.n) dst[i] = (i & 1 ? acc[i >> 1].y : acc[i >> 1].x) * mult;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Native block-scaled FP4 path for two-level scales, one CTA per tile (mode 3).
//
// kind::mxf4nvf4 multiplies E2M1 operands scaled per 16 elements by UE4M3
// factors, which is exactly an E2M1 operand under the two-level scales (the
// block scale e_b is a non-negative E4M3 byte).  E2M1 codes go from TMA
// straight to the tensor core.  An E1M2 code with magnitude k (value k/4 of
// the step) splits exactly into two E2M1 operands: the code bits read as an
// E2M1 number e(k) = {0, .5, 1, 1.5, 2, 3, 4, 6}[k], plus a correction plane
// d(k) = k - e(k) = {0, .5, 1, 1.5, 2, 2, 2, 1}[k], which is E2M1 as well.
// Then sum k_a k_b = sum (e_a + d_a)(e_b + d_b): four native MMAs with the
// same scale factors, the raw code tiles used as they arrived and only the
// correction planes written by the transform warps (a per-byte bit function).
//
// Tiles: 128 x 192 on one CTA.  192 columns let
// two accumulators share TMEM with one scale-factor slot per TMA stage, so the
// epilogue of one tile overlaps the MMAs of the next and the transform runs
// ahead of the MMAs as far as the TMA ring allows.  A stage covers 128 K elements
// (64-byte code rows, 64-byte TMA swizzle).
//
// The transform warps write the scale factors into TMEM themselves
// (tcgen05.st), so the tensor pipe runs MMAs only: for each 128-row group and
// K step, lane i of every 32-lane quarter holds, in 4 consecutive columns,
// the 4 block factors of rows i, 32 + i, 64 + i and 96 + i (the layout the
// MMA reads, the same in all four quarters); a warp builds an atom with a
// 4x4 byte transpose per 4 rows in its scratch, and two groups of transform
// warps take alternate stages.  E1M2 correction planes are loaded with the
// codes
// when the quantizer stored them, else the transform builds them.  Scale
// factors and built planes use two-slot rings, refilled once the MMAs two
// stages back have completed.  The epilogue stages 128 x 32 fp32 chunks in
// shared memory and writes them with coalesced 16-byte stores.
template <int GRID, bool CIN>
struct Fp4Cfg {
    static constexpr int BN = kNativeTileN;         // tile columns (B rows)
    static constexpr int BNh = BN;                  // B code rows staged per CTA
    static constexpr int TM = BM;                   // tile rows
    static constexpr int BKE = 128;                 // K elements per stage
    static constexpr int kRow = BKE / 2;            // code bytes per row per stage
    static constexpr int KST = BKE / 64;            // MMA K steps per stage
    static constexpr int NT = 8;                    // transform warps
    static constexpr int NE = 4;                    // epilogue warps
    // E1M2 correction planes: loaded with the codes (CIN) or built by the
    // transform warps into a two-slot ring
    static constexpr int ND = (GRID == 0 && !CIN) ? 2 : 0;
    static constexpr int kCodesA = BM * kRow;
    static constexpr int kCodesB = BNh * kRow;
    static constexpr int kRawA = BM * (BKE / 16);
    static constexpr int kRawB = BN * (BKE / 16);
    static constexpr int kIn = CIN ? 2 : 1;         // code planes loaded per stage
    // Code stage: [codes A | planes A | codes B | planes B] (the planes only
    // with CIN: a 3-D box fills an operand's two tiles).
    static constexpr int o_codes_a = 0;
    static constexpr int o_cin_a = o_codes_a + kCodesA;         // CIN only
    static constexpr int o_codes_b = o_codes_a + kIn * kCodesA;
    static constexpr int o_cin_b = o_codes_b + kCodesB;         // CIN only
    static constexpr int kStage = (kIn * (kCodesA + kCodesB) + 1023) / 1024 * 1024;
    static constexpr int kCorr = (kCodesA + kCodesB + 1023) / 1024 * 1024;  // one slot
    // Scale factors run in their own ring, one TMEM slot per raw-scale smem
    // slot ([raw scales A | raw scales B]), ahead of the code stages.
    static constexpr int o_raw_a = 0;                           // within a raw slot
    static constexpr int o_raw_b = kRawA;
    static constexpr int kRawSlot = (kRawA + kRawB + 127) / 128 * 128;
    // scale-factor atoms per stage: K step j, kind 0 = SFA, 1 / 2 = SFB rows
    // [0, 128) / [128, BN)
    static constexpr int kAtoms = 3 * KST;
    static constexpr int kGroupWarps = NT / 2;      // transform warps per stage
    static constexpr int kScr = NT * kAtoms * 512;  // per-warp atom scratch
    static constexpr int kAccCols = BN;             // one accumulator
    static constexpr int kSfCols = KST * 12;        // scale factors of one stage
    static constexpr int kSfBase = 2 * kAccCols;
    static constexpr int kBudget = 232448 - 2048;   // barriers, alignment slack
    static constexpr int kOutChunk = BM * 32 * 4;   // epilogue staging: 128 rows x 32 fp32
    // Code stages, capped by the TMEM scale-factor slots: slot s serves code
    // stage s, so the stage's release (empty) also frees its factors.
    static constexpr int kNsTmem = (512 - kSfBase) / kSfCols;
    static constexpr int kNsSmem = (kBudget - ND * kCorr - kOutChunk - kScr - kNsTmem * kRawSlot) / kStage;
    static constexpr int NS = kNsSmem < kNsTmem ? kNsSmem : kNsTmem;
    static constexpr int NSF = NS;                              // raw-scale slots
    // E1M2 (eight MMAs a stage): a scale producer warp streams the raw scales
    // ahead of the code tiles.  E2M1 (two MMAs a stage): the code producer
    // issues them just before each stage's codes (fewer TMA streams).
    static constexpr bool kAheadScales = GRID == 0;
    static constexpr int o_corr = NS * kStage;
    static constexpr int o_out = o_corr + ND * kCorr;
    static constexpr int o_scr = o_out + kOutChunk;
    static constexpr int o_raw = o_scr + kScr;
    static constexpr int o_bar = o_raw + NSF * kRawSlot;
    // code ring: full, empty; scale-factor ring: sfull, sraw_free, sf_ready;
    // acc_full[2], acc_empty[2], drain
    static constexpr int kNumBars = 2 * NS + 3 * NSF + 5;
    static constexpr int o_misc = o_bar + kNumBars * 8;
    static constexpr int kAlloc = o_misc + 64 + 1024;
    // producer, MMA issuer, transform warps, epilogue warps, scale producer
    static constexpr int kThreads = 32 * (3 + NT + NE);
    static_assert(kGroupWarps == 4, "one warp per TMEM lane quarter in each transform group");
    static_assert(NS >= 4 && NSF >= 4, "pipeline depth");
    static_assert(kSfBase + NSF * kSfCols <= 512, "TMEM budget");
    static_assert(kAlloc <= 232448, "shared memory budget");
    static_assert(o_corr % 1024 == 0 && o_out % 1024 == 0, "swizzle alignment");
    static_assert(BN % 32 == 0 && BN > 128 && BN <= 256, "two SFB row groups, 32-column chunks");
    static_assert(BN % 8 == 0, "B rows per CTA");
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// 4 x 4 byte transpose: out_i holds byte i of w0, w1, w2, w3 (low to high).
__device__ __forceinline__ void transpose4x4(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3,
                                             uint32_t (&o)[4]) {
    const uint32_t t0 = prmt(w0, w1, 0x5140u), t1 = prmt(w0, w1, 0x7362u);
    const uint32_t t2 = prmt(w2, w3, 0x5140u), t3 = prmt(w2, w3, 0x7362u);
    o[0] = prmt(t0, t2, 0x5410u);
    o[1] = prmt(t0, t2, 0x7632u);
    o[2] = prmt(t1, t3, 0x5410u);
    o[3] = prmt(t1, t3, 0x7632u);
}

template <int GRID, bool CIN>
__global__ void __launch_bounds__(Fp4Cfg<GRID, CIN>::kThreads, 1)
    gemm_fp4_kernel(const __grid_constant__ GemmArgs args) {
    using C = Fp4Cfg<GRID, CIN>;
    constexpr int BN = C::BN;
    constexpr int TM = C::TM;
    constexpr int NS = C::NS;
    constexpr int NSF = C::NSF;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    // code ring (index s = it % NS)
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::o_bar);   // code tiles landed
    uint64_t *empty = full + NS;          // MMAs done with the stage (multicast commit)
    // scale-factor ring (index j = it % NSF)
    uint64_t *sfull = empty + NS;         // raw scale factors landed
    uint64_t *sraw_free = sfull + NSF;    // transform read the raw slot
    uint64_t *sf_ready = sraw_free + NSF; // in CTA 0: factors in TMEM (all CTAs)
    uint64_t *acc_full = sf_ready + NSF;  // [2]
    uint64_t *acc_empty = acc_full + 2;   // [2], in CTA 0: accumulator drained (all CTAs)
    uint64_t *drain = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::o_misc);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + C::o_misc + 4);
    auto stage = [&](int s) { return smem + s * C::kStage; };
    auto raw_slot = [&](int j) { return smem + C::o_raw + j * C::kRawSlot; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int blk = args.block;                       // 16 or 32
    const int nraw = C::BKE / blk;                    // raw scale rows per stage
    const int64_t unit = blockIdx.x;
    const int64_t nunits = gridDim.x;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < NSF; ++i) {
            mbar_init(&sfull[i], 1);
            mbar_init(&sraw_free[i], C::kGroupWarps);
            mbar_init(&sf_ready[i], C::kGroupWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], C::NE);
        }
        mbar_init(drain, 1);
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&args.tm_a_codes);
        tma_prefetch_desc(&args.tm_b_codes);
        tma_prefetch_desc(&args.tm_a_scales);
        tma_prefetch_desc(&args.tm_b_scales);
        if (CIN) {
            tma_prefetch_desc(&args.tm_a_corr);
            tma_prefetch_desc(&args.tm_b_corr);
        }
    }
    if (warp == 1) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int64_t ntiles = total_tiles<TM, BN>(args);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_last();
            uint32_t it = 0;
            bool ok = true;
            for (int64_t t = unit; t < ntiles && ok; t += nunits) {
                const Tile tl = get_tile<TM, BN>(args, t);
                const int nks = static_cast<int>((tl.g.k + C::BKE - 1) / C::BKE);
                const int32_t arow = static_cast<int32_t>(tl.g.a_row + tl.m0);
                const int32_t brow = static_cast<int32_t>(tl.g.b_row + tl.n0);
                for (int ks = 0; ks < nks; ++ks, ++it) {
                    const int s = it % NS;
                    if (!mbar_wait(&empty[s], ((it / NS) & 1) ^ 1, kErrTimeoutProducer, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int32_t acol = static_cast<int32_t>(tl.g.a_col + ks * C::BKE);
                    const int32_t bcol = static_cast<int32_t>(tl.g.b_col + ks * C::BKE);
                    uint8_t *st = stage(s);
                    if constexpr (!C::kAheadScales) {
                        uint8_t *rs = raw_slot(s);
                        mbar_arrive_expect_tx(&sfull[s], (BM + BN) * nraw);
                        tma_load_2d_hint(rs + C::o_raw_a, &args.tm_a_scales, &sfull[s], arow, acol / blk, pol);
                        tma_load_2d_hint(rs + C::o_raw_b, &args.tm_b_scales, &sfull[s], brow, bcol / blk, pol);
                    }
                    mbar_arrive_expect_tx(&full[s], C::kIn * (C::kCodesA + C::kCodesB));
                    const int32_t brow_h = brow;
                    // Operand tiles are read by many CTAs: keep them in L2
                    // ahead of the streamed output.
                    if (CIN && args.planes3d) {
                        tma_load_3d_hint(st + C::o_codes_a, &args.tm_a_corr, &full[s], acol / 2, arow, 0, pol);
                        tma_load_3d_hint(st + C::o_codes_b, &args.tm_b_corr, &full[s], bcol / 2, brow_h, 0, pol);
                    } else {
                        tma_load_2d_hint(st + C::o_codes_a, &args.tm_a_codes, &full[s], acol / 2, arow, pol);
                        tma_load_2d_hint(st + C::o_codes_b, &args.tm_b_codes, &full[s], bcol / 2, brow_h, pol);
                        if (CIN) {
                            tma_load_2d_hint(st + C::o_cin_a, &args.tm_a_corr, &full[s], acol / 2, arow, pol);
                            tma_load_2d_hint(st + C::o_cin_b, &args.tm_b_corr, &full[s], bcol / 2, brow_h, pol);
                        }
                    }
                }
            }
            // Drain: the last copy into each stage has landed before exit.
            for (int s = 0; s < NS; ++s) {
                if (it > static_cast<uint32_t>(s)) {
                    const uint32_t last = (it - 1 - s) / NS * NS + s;
                    uint32_t dummy = 0;
                    mbar_wait(&full[s], (last / NS) & 1, kErrTimeoutDrain,
                              reinterpret_cast<volatile uint32_t *>(&dummy));
                    if constexpr (!C::kAheadScales)
                        mbar_wait(&sfull[s], (last / NS) & 1, kErrTimeoutDrain,
                                  reinterpret_cast<volatile uint32_t *>(&dummy));
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ UMMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_fp4_bs(TM, BN);
            auto wait_any = [&](uint64_t *bar, uint32_t parity) {
                return mbar_wait(bar, parity, kErrTimeoutMma, abort_flag);
            };
            uint32_t it = 0, tcount = 0;
            bool ok = true;
            for (int64_t t = unit; t < ntiles && ok; t += nunits, ++tcount) {
                const Tile tl = get_tile<TM, BN>(args, t);
                const int nks = static_cast<int>((tl.g.k + C::BKE - 1) / C::BKE);
                const int ab = tcount & 1;
                if (!wait_any(&acc_empty[ab], ((tcount >> 1) & 1) ^ 1)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + ab * C::kAccCols;
                bool first = true;
                for (int ks = 0; ks < nks && ok; ++ks, ++it) {
                    const int s = it % NS;
                    const int j = it % NSF;
                    // factors in TMEM, then the code tiles
                    if (!wait_any(&sf_ready[j], (it / NSF) & 1) ||
                        !mbar_wait(&full[s], (it / NS) & 1, kErrTimeoutMma, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint8_t *st = stage(s);
                    // scale factors of K step j: SFA at 12 j, SFB rows 0-127
                    // at 12 j + 4, rows 128+ at 12 j + 8 of the stage's slot
                    // (written by the transform warps of each CTA)
                    const uint32_t sf0 = tmem_base + C::kSfBase + j * C::kSfCols;
                    // K steps of 64 in this stage (a tail uses only its own)
                    const int64_t rem = tl.g.k - static_cast<int64_t>(ks) * C::BKE;
                    const int steps = rem >= C::BKE ? C::KST : static_cast<int>((rem + 63) / 64);
                    const uint32_t a0 = smem_addr(st + C::o_codes_a), b0 = smem_addr(st + C::o_codes_b);
                    const uint32_t ac = CIN ? smem_addr(st + C::o_cin_a)
                                            : smem_addr(smem + C::o_corr + (it & 1) * C::kCorr);
                    const uint32_t bc = CIN ? smem_addr(st + C::o_cin_b) : ac + C::kCodesA;
                    for (int j = 0; j < steps; ++j) {
                        const uint32_t sfa = sf0 + 12 * j, sfb = sfa + 4;
                        const uint32_t dk = 32 * j;
                        umma_fp4_bs(d_tmem, umma_desc_sw64(a0 + dk), umma_desc_sw64(b0 + dk), idesc,
                                           sfa, sfb, first ? 0u : 1u);
                        first = false;
                        if (GRID == 0) {
                            umma_fp4_bs(d_tmem, umma_desc_sw64(a0 + dk), umma_desc_sw64(bc + dk),
                                               idesc, sfa, sfb, 1u);
                            umma_fp4_bs(d_tmem, umma_desc_sw64(ac + dk), umma_desc_sw64(b0 + dk),
                                               idesc, sfa, sfb, 1u);
                            umma_fp4_bs(d_tmem, umma_desc_sw64(ac + dk), umma_desc_sw64(bc + dk),
                                               idesc, sfa, sfb, 1u);
                        }
                    }
                    umma_commit(&empty[s]);
                }
                if (ok) umma_commit(&acc_full[ab]);
            }
            // Drain: every MMA issued here completes before TMEM is freed.
            umma_commit(drain);
            uint32_t dummy = 0;
            mbar_wait(drain, 0, kErrTimeoutDrain, reinterpret_cast<volatile uint32_t *>(&dummy));
        }
    } else if (warp < 2 + C::NT) {
        // ------------------------------------------------------------ transform
        // Two groups of four warps (one per TMEM lane quarter) take alternate
        // iterations.  Each warp builds every scale-factor atom of its
        // iteration for its lane quarter (a 4x4 byte transpose per 4 rows into
        // its scratch) and stores it with tcgen05.st into TMEM slot it % NS,
        // once the MMAs that last read that slot (and released the code stage
        // of the same index) are done.  The raw scales arrive in their own
        // ring, ahead of the code tiles.
        const int tw = warp - 2;
        const int grp = tw >> 2;
        const int gt = (tw & 3) * 32 + lane;            // thread index within the group
        constexpr int kGrpThr = 32 * C::kGroupWarps;
        constexpr int kChunks = (C::kCodesA + C::kCodesB) / 16;   // correction pieces
        constexpr int kPer = (kChunks + kGrpThr - 1) / kGrpThr;
        uint8_t *scr = smem + C::o_scr + tw * (C::kAtoms * 512);
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
        uint32_t it = 0;
        bool ok = true;
        for (int64_t t = unit; t < ntiles && ok; t += nunits) {
            const Tile tl = get_tile<TM, BN>(args, t);
            const int nks = static_cast<int>((tl.g.k + C::BKE - 1) / C::BKE);
            for (int ks = 0; ks < nks; ++ks, ++it) {
                if (static_cast<int>(it & 1) != grp) continue;
                const int s = it % NS;
                const int j = it % NSF;
                const uint32_t jph = (it / NSF) & 1;
                constexpr bool kBuild = GRID == 0 && !CIN;   // correction planes here
                // The factors need the raw scales and a free TMEM slot;
                // building correction planes needs the codes.
                if (!warp_wait(&sfull[j], jph, kErrTimeoutTransform, abort_flag) ||
                    !warp_wait(&empty[j], jph ^ 1, kErrTimeoutTransform, abort_flag) ||
                    (kBuild && !warp_wait(&full[s], (it / NS) & 1, kErrTimeoutTransform, abort_flag))) {
                    ok = false;
                    break;
                }
                // Correction slot it & 1 was last read by the MMAs of it - 2.
                if (kBuild && it >= 2) {
                    const uint32_t p = it - 2;
                    if (!warp_wait(&empty[p % NS], (p / NS) & 1, kErrTimeoutTransform, abort_flag)) {
                        ok = false;
                        break;
                    }
                }
                const uint8_t *st = stage(s);
                // Loads first: raw scale words (lane builds rows 4 lane ..
                // 4 lane + 3 of a 128-row group) and the code pieces to correct.
                uint32_t w[C::kAtoms][4];
#pragma unroll
                for (int a = 0; a < C::kAtoms; ++a) {
                    const int jk = a / 3, kind = a % 3;
                    const int rows = kind == 0 ? BM : BN;
                    const int r = 4 * lane + (kind == 2 ? 128 : 0);
                    const uint8_t *raw = raw_slot(j) + (kind == 0 ? C::o_raw_a : C::o_raw_b) + r;
                    if (r < rows) {
                        if (blk == 16) {
#pragma unroll
                            for (int kb = 0; kb < 4; ++kb)
                                w[a][kb] = *reinterpret_cast<const uint32_t *>(raw + (4 * jk + kb) * rows);
                        } else {
                            w[a][0] = w[a][1] = *reinterpret_cast<const uint32_t *>(raw + (2 * jk) * rows);
                            w[a][2] = w[a][3] =
                                *reinterpret_cast<const uint32_t *>(raw + (2 * jk + 1) * rows);
                        }
                    } else {
                        w[a][0] = w[a][1] = w[a][2] = w[a][3] = 0u;
                    }
                }
                // raw slot j read: the scale producer may refill it
                __syncwarp();
                if (lane == 0) mbar_arrive(&sraw_free[j]);
                uint4 cw[kBuild ? kPer : 1];
                if constexpr (kBuild) {
#pragma unroll
                    for (int i = 0; i < kPer; ++i) {
                        const int idx = gt + i * kGrpThr;
                        if (idx < kChunks) cw[i] = *reinterpret_cast<const uint4 *>(st + 16 * idx);
                    }
                }
                // Atom byte 16 (r % 32) + 4 (r / 32) + kb holds the factor of
                // 16-element block 4 jk + kb of row r of the group.
#pragma unroll
                for (int a = 0; a < C::kAtoms; ++a) {
                    uint32_t o[4];
                    transpose4x4(w[a][0], w[a][1], w[a][2], w[a][3], o);
                    uint8_t *dst = scr + a * 512 + 16 * ((4 * lane) & 31) + 4 * ((4 * lane) >> 5);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) *reinterpret_cast<uint32_t *>(dst + 16 * q4) = o[q4];
                }
                if constexpr (kBuild) {
                    // Correction planes of both code tiles (same swizzled
                    // offsets; the function is per byte).
                    uint8_t *corr = smem + C::o_corr + (it & 1) * C::kCorr;
#pragma unroll
                    for (int i = 0; i < kPer; ++i) {
                        const int idx = gt + i * kGrpThr;
                        if (idx < kChunks) {
                            const uint4 d = make_uint4(e1m2_correction(cw[i].x), e1m2_correction(cw[i].y),
                                                       e1m2_correction(cw[i].z), e1m2_correction(cw[i].w));
                            *reinterpret_cast<uint4 *>(corr + 16 * idx) = d;
                        }
                    }
                }
                __syncwarp();
                const uint32_t sfw = lane_base + C::kSfBase + j * C::kSfCols;
#pragma unroll
                for (int a = 0; a < C::kAtoms; ++a) {
                    const uint4 row = *reinterpret_cast<const uint4 *>(scr + a * 512 + 16 * lane);
                    tmem_st_32x32b_x4(sfw + 12 * (a / 3) + 4 * (a % 3), row.x, row.y, row.z, row.w);
                }
                tmem_wait_st();
                __syncwarp();
                tc_fence_before();
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_ready[j]);
            }
        }
    } else if (warp < 2 + C::NT + C::NE) {
        // ------------------------------------------------------------ epilogue
        // Thread = accumulator row.  Each 128 x 32 fp32 chunk is staged in
        // shared memory (128-byte rows, 16-byte pieces XOR-swizzled by row)
        // and written 4 whole rows per warp instruction, keeping the load /
        // store unit free for the transform warps.  The double-buffered
        // accumulator lets these stores overlap the next tile.
        const int q = warp & 3;
        const int et = threadIdx.x - 32 * (2 + C::NT);   // 0 .. 127
        const int row_in_tile = 32 * q + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
        constexpr uint32_t kEpiThreads = 32 * C::NE;
        uint8_t *buf = smem + C::o_out;
        // E1M2 operands carry k = 4 * level on both sides: 1/16 (exact).
        const float mult = __fmul_rn(__fmul_rn(*args.a_S, *args.b_S),
                                     args.inv_n * (GRID == 0 ? (1.0f / 16.0f) : 1.0f));
        uint32_t tcount = 0;
        for (int64_t t = unit; t < ntiles; t += nunits, ++tcount) {
            const Tile tl = get_tile<TM, BN>(args, t);
            const int ab = tcount & 1;
            const bool ok = warp_wait(&acc_full[ab], (tcount >> 1) & 1, kErrTimeoutEpilogue, abort_flag);
            // one decision for the four epilogue warps (they share barrier 1)
            if (named_bar_or(1, kEpiThreads, !ok)) break;
            tc_fence_after();
            const int64_t m0 = tl.m0;                 // accumulator rows of the tile
            const int64_t row = m0 + row_in_tile;
            const bool row_ok = row < tl.g.m;
            float *crow = args.c + (tl.g.c_row + row) * args.ldc + tl.g.c_col + tl.n0;
            const bool vec_tile = args.c_vec && (tl.g.c_col & 3) == 0;
            const uint32_t acc = tmem_base + ab * C::kAccCols + lane_addr;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(acc + 32 * c, r);
                tmem_wait_ld();
                if (c == BN / 32 - 1) {
                    // accumulator drained: the MMAs of tile t + 2 may start
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acc_empty[ab]);
                }
                const int64_t col0 = tl.n0 + 32 * c;
                if (col0 >= tl.g.n) continue;             // the same for all threads
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    v[i] = tl.g.k > 0 ? __fmul_rn(__uint_as_float(r[i]), mult) : 0.0f;
                if (vec_tile) {
                    uint8_t *rowp = buf + row_in_tile * 128;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        *reinterpret_cast<float4 *>(rowp + ((ch ^ (row_in_tile & 7)) << 4)) =
                            make_float4(v[4 * ch], v[4 * ch + 1], v[4 * ch + 2], v[4 * ch + 3]);
                    named_bar_sync(1, kEpiThreads);          // chunk staged
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int p = et + 128 * k;
                        const int rr = p >> 3, c16 = p & 7;
                        const float4 val =
                            *reinterpret_cast<const float4 *>(buf + rr * 128 + ((c16 ^ (rr & 7)) << 4));
                        const int64_t grow = m0 + rr;
                        const int64_t gcol = col0 + 4 * c16;
                        if (grow < tl.g.m && gcol < tl.g.n) {
                            float *dst = args.c + (tl.g.c_row + grow) * args.ldc + tl.g.c_col + gcol;
                            if (gcol + 4 <= tl.g.n) {
                                __stcs(reinterpret_cast<float4 *>(dst), val);   // streamed: evict first
                            } else {
                                const float e4[4] = {val.x, val.y, val.z, val.w};
                                for (int e = 0; e < 4 && gcol + e < tl.g.n; ++e) dst[e] = e4[e];
                            }
                        }
                    }
                    named_bar_sync(1, kEpiThreads);          // chunk read out
                } else if (row_ok) {
                    float *dst = crow + 32 * c;
                    for (int i = 0; i < 32; ++i)
                        if (col0 + i < tl.g.n) dst[i] = v[i];
                }
            }
        }
    } else {
        // ------------------------------------------------------------ scale producer
        // Streams each iteration's raw scale factors (A rows of this CTA, all
        // BN B rows) into raw slot it % NSF once the transform has read the
        // slot's previous contents.
        if (C::kAheadScales && lane == 0) {
            const uint64_t pol = l2_policy_evict_last();
            uint32_t it = 0;
            bool ok = true;
            for (int64_t t = unit; t < ntiles && ok; t += nunits) {
                const Tile tl = get_tile<TM, BN>(args, t);
                const int nks = static_cast<int>((tl.g.k + C::BKE - 1) / C::BKE);
                const int32_t arow = static_cast<int32_t>(tl.g.a_row + tl.m0);
                const int32_t brow = static_cast<int32_t>(tl.g.b_row + tl.n0);
                for (int ks = 0; ks < nks; ++ks, ++it) {
                    const int j = it % NSF;
                    if (!mbar_wait(&sraw_free[j], ((it / NSF) & 1) ^ 1, kErrTimeoutProducer, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int32_t acol = static_cast<int32_t>(tl.g.a_col + ks * C::BKE);
                    const int32_t bcol = static_cast<int32_t>(tl.g.b_col + ks * C::BKE);
                    uint8_t *rs = raw_slot(j);
                    mbar_arrive_expect_tx(&sfull[j], (BM + BN) * nraw);
                    tma_load_2d_hint(rs + C::o_raw_a, &args.tm_a_scales, &sfull[j], arow, acol / blk, pol);
                    tma_load_2d_hint(rs + C::o_raw_b, &args.tm_b_scales, &sfull[j], brow, bcol / blk, pol);
                }
            }
            // Drain: the last copy into each slot has landed before exit.
            for (int j = 0; j < NSF; ++j) {
                if (it > static_cast<uint32_t>(j)) {
                    const uint32_t last = (it - 1 - j) / NSF * NSF + j;
                    uint32_t dummy = 0;
                    mbar_wait(&sfull[j], (last / NSF) & 1, kErrTimeoutDrain,
                              reinterpret_cast<volatile uint32_t *>(&dummy));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

// ---------------------------------------------------------------------------
// CTA-pair native kernel for two-level scales (mode 5): 256 x 256 output
// tiles on a CTA pair with cta_group::2 MMAs of M = 256, N = 256, K = 64.
// Rank r of the pair stages A rows [128 r, +128) and B rows [128 r, +128) of
// the tile (E1M2: codes and correction planes, one 3-D box per operand) and
// holds accumulator rows [128 r, +128) x 256 fp32 columns of TMEM.  Per SM
// that is half the operand bytes per flop of a one-CTA 128 x 256 tile.  The
// other 256 TMEM columns hold the scale factors of up to ten stages in
// flight (slot s of stage s, freed by the same MMA commit that frees the
// stage's shared memory).
//   warp 0     producer: each stage's code tiles (completion counted on the
//              leader CTA's barrier, which expects both CTAs' bytes) and
//              this CTA's raw block-major factors (A rows, all 256 B rows);
//   warp 1     TMEM owner; in the leader, the single-thread MMA issuer;
//   warps 4-7  factor writers, one per TMEM lane quarter: build the stage's
//              atoms (lane i of a quarter holds the 4 block factors of rows
//              i, 32 + i, 64 + i, 96 + i of a 128-row group) by 4 x 4 byte
//              transposes and store them with tcgen05.st;
//   warps 8-11 epilogue: TMEM -> registers -> x S_a S_b / (16 n) -> staged
//              in shared memory -> coalesced 16-byte stores.
// One accumulator per CTA.  Without factor atoms the epilogue reads TMEM in
// 32-column pieces between its stores, and the next tile's MMAs wait for the
// last piece.  With factor atoms (no factor writers) warps 4-11 drain the
// accumulator into registers, 128 columns each, release TMEM at once and
// then scale and store while the next tile's MMAs run.
// GRID 3 is the MX path: E1M2 operands as their E4M3 element planes (one
// byte per element, 128-byte rows, 128-byte swizzle), UE8M0 factors per 32
// elements applied in the MMA (kind::mxf8f6f4, K = 32 per MMA, four MMAs per
// stage picking byte j of the same factor atom).
template <int GRID, bool ATOMS, bool LANES = false>
struct PairCfg {
    static constexpr bool kMx = GRID == 3;
    static constexpr int TM = 256;
    static constexpr int BN = 256;
    static constexpr int BKE = kMx ? 128 : pair_stage_k(GRID, ATOMS);   // K elements per stage
    static constexpr int KST = kMx ? 1 : BKE / 64;  // factor atom groups per stage
    static constexpr int kRow = kMx ? BKE : BKE / 2;   // operand bytes per row per stage
    static constexpr int kPlanes = GRID == 0 ? 2 : 1;
    static constexpr int kTile = 128 * kRow;        // one plane of a 128-row tile
    static constexpr int o_a = 0;                   // [codes | corr] of A
    static constexpr int o_b = kPlanes * kTile;     // [codes | corr] of this CTA's B half
    static constexpr int kCodeBytes = 2 * kPlanes * kTile;   // per CTA per stage
    static constexpr int kRawRows = kMx ? BKE / 32 : BKE / 16;   // factor rows per stage (most)
    // E1M2 with factor atoms and per-lane tiles on A: the A factors of a
    // stage arrive as one per-lane tile (4 KB) and leave for TMEM in one copy.
    static constexpr bool kLaneA = GRID == 0 && ATOMS && LANES;
    static constexpr int o_raw_a = kCodeBytes;      // raw factors: [blocks][128 rows]
    static constexpr int kRawA = kLaneA ? kLaneTileBytes : 128 * kRawRows;
    static constexpr int o_raw_b = o_raw_a + kRawA; // [blocks][256 rows]
    static constexpr int kRawB = 256 * kRawRows;
    static constexpr int kStage = (kCodeBytes + kRawA + kRawB + 1023) / 1024 * 1024;
    static constexpr int kAtoms = 3 * KST;          // SFA, SFB rows 0-127, SFB rows 128-255 per K step
    static constexpr int kScr = ATOMS ? 0 : 4 * kAtoms * 512;   // one atom scratch per factor warp
    static constexpr int kOutBytes = (ATOMS ? 8 : 4) * 4096;   // epilogue staging: 4 KB per epilogue warp
    static constexpr int kSfBase = 256;             // TMEM column of the first factor slot
    static constexpr int kSfCols = 12 * KST;        // TMEM columns of one stage's factors
    static_assert(!kLaneA || (BKE == kLaneK && 8 + 8 * KST <= kSfCols), "per-lane A factors: one tile per stage");
    static constexpr int kNsTmem = (512 - kSfBase) / kSfCols;
    static constexpr int kBudget = 232448 - 2048;
    static constexpr int kNsSmem = (kBudget - kScr - kOutBytes) / kStage;
    static constexpr int NS = kNsSmem < kNsTmem ? kNsSmem : kNsTmem;
    static constexpr int o_out = NS * kStage;
    static constexpr int o_scr = o_out + kOutBytes;
    static constexpr int o_bar = o_scr + kScr;
    // full[NS], empty[NS], sfull[NS], sfready[NS], sflocal[NS], acc_full,
    // acc_empty, drain
    static constexpr int kNumBars = 5 * NS + 3;
    static constexpr int o_misc = o_bar + kNumBars * 8;
    static constexpr int kMaxOrder = 256;           // grouped problems: a schedule of up to 256 groups
    static constexpr int o_cum = o_misc + 64;       // int64 [kMaxOrder + 1]
    static constexpr int o_order = o_cum + 8 * (kMaxOrder + 1);   // u16 [kMaxOrder]
    static constexpr int kAlloc = o_order + 2 * kMaxOrder + 1024;
    static constexpr int kThreads = 32 * 12;
    static_assert(NS >= 4, "pipeline depth");
    static_assert(kAlloc <= 232448, "shared memory budget");
    static_assert(kSfBase + NS * kSfCols <= 512, "TMEM budget");
};

// Copy of one 512-byte factor atom (32 rows of 16 bytes, row i at byte 16 i)
// from shared memory into TMEM columns [taddr, taddr + 4) of all four lane
// quarters, in both CTAs of the pair (each from its own shared memory at the
// same address).  Descriptor: no swizzle, K-major, core matrices of 8 rows x
// 16 bytes at a stride of 128 bytes (SBO); one core matrix along K (LBO unused).
__device__ __forceinline__ void tmem_cp_atom_pair(uint32_t taddr, uint32_t smem_byte_addr) {
    const uint64_t d = static_cast<uint64_t>((smem_byte_addr >> 4) & 0x3FFFu) |
                       (static_cast<uint64_t>(128u >> 4) << 32) | (static_cast<uint64_t>(1u) << 46);
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
}

// Copy of one per-lane factor tile (128 lanes x 32 bytes, two 2048-byte halves
// of 16 bytes per lane) into TMEM columns [taddr, taddr + 8) of both CTAs of
// the pair.  Descriptor: no swizzle, K-major, core matrices of 8 rows x 16
// bytes at a stride of 128 bytes (SBO) along the lanes and 2048 bytes (LBO)
// between the two halves.
__device__ __forceinline__ void tmem_cp_lanes_pair(uint32_t taddr, uint32_t smem_byte_addr) {
    const uint64_t d = static_cast<uint64_t>((smem_byte_addr >> 4) & 0x3FFFu) |
                       (static_cast<uint64_t>(2048u >> 4) << 16) | (static_cast<uint64_t>(128u >> 4) << 32) |
                       (static_cast<uint64_t>(1u) << 46);
    asm volatile("tcgen05.cp.cta_group::2.128x256b [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
}

// TMA tile loads whose completion is counted on a barrier of the leader CTA
// of the pair (`bar_cluster`: a shared::cluster address from mapa).  The
// destination is this CTA's shared memory.  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void *smem_dst, const CUtensorMap *map, uint32_t bar_cluster,
                                                 int32_t x, int32_t y, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_addr(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(void *smem_dst, const CUtensorMap *map, uint32_t bar_cluster,
                                                 int32_t x, int32_t y, int32_t z, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_addr(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y), "r"(z), "l"(policy)
        : "memory");
}

// shared::cluster address of the same-offset object in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
    return r;
}

// Block-scaled FP8 MMA on a CTA pair: E4M3 operands, UE8M0 factors per 32
// elements (byte sf_id of each factor word, chosen in the instruction
// descriptor), fp32 accumulate, K = 32.
__device__ __forceinline__ void umma_mxf8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Instruction descriptor, kind::mxf8f6f4 block-scaled: A = B = E4M3, UE8M0
// factors, fp32 accumulate, both K-major; factor byte sf_id of A and B.
__host__ __device__ constexpr uint32_t umma_idesc_mxf8(int M, int N, uint32_t sf_id) {
    return (sf_id << 4)                               // B factor byte
           | (0u << 7) | (0u << 10)                   // A, B: E4M3
           | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
           | (1u << 23)                               // factor format UE8M0
           | (static_cast<uint32_t>(M >> 4) << 24)    // M / 16
           | (sf_id << 29);                           // A factor byte
}

// Epilogue piece of one warp: accumulator rows m0 + lane (thread = row) x
// columns [col0, col0 + 32), scaled by mult (zero: the group has k = 0 and
// no MMA wrote the accumulator) and written to C.  With 16-byte aligned rows
// the piece is transposed through the warp's 4 KB buffer (16-byte units
// XORed with the row mod 8, conflict-free both ways) so that eight lanes
// write one row's 128 bytes per store.
__device__ __forceinline__ void store_piece(const GemmArgs &args, const Tile &tl, uint8_t *buf, int lane,
                                            int64_t m0, int64_t col0, uint32_t (&r)[32], float mult, bool zero,
                                            bool vec_tile) {
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = zero ? 0.0f : __fmul_rn(__uint_as_float(r[i]), mult);
    if (vec_tile) {
        uint8_t *rowp = buf + lane * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
            *reinterpret_cast<float4 *>(rowp + ((ch ^ (lane & 7)) << 4)) =
                make_float4(v[4 * ch], v[4 * ch + 1], v[4 * ch + 2], v[4 * ch + 3]);
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int rr = 4 * k + (lane >> 3), c16 = lane & 7;
            const float4 val = *reinterpret_cast<const float4 *>(buf + rr * 128 + ((c16 ^ (rr & 7)) << 4));
            const int64_t grow = m0 + rr;
            const int64_t gcol = col0 + 4 * c16;
            if (grow < tl.g.m && gcol < tl.g.n) {
                float *dst = args.c + (tl.g.c_row + grow) * args.ldc + tl.g.c_col + gcol;
                if (gcol + 4 <= tl.g.n) {
                    *reinterpret_cast<float4 *>(dst) = val;   // default L2 policy: fewer operand re-reads than evict-first
                } else {
                    const float e4[4] = {val.x, val.y, val.z, val.w};
                    for (int e = 0; e < 4 && gcol + e < tl.g.n; ++e) dst[e] = e4[e];
                }
            }
        }
        __syncwarp();                                 // buffer read out before the next piece
    } else {
        const int64_t row = m0 + lane;
        if (row < tl.g.m) {
            float *dst = args.c + (tl.g.c_row + row) * args.ldc + tl.g.c_col + col0;
            for (int i = 0; i < 32; ++i)
                if (col0 + i < tl.g.n) dst[i] = v[i];
        }
    }
}

template <int GRID, bool ATOMS, bool LANES>
__global__ void __launch_bounds__(PairCfg<GRID, ATOMS, LANES>::kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ GemmArgs args) {
    using C = PairCfg<GRID, ATOMS, LANES>;
    constexpr int TM = C::TM, BN = C::BN, NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::o_bar);   // leader: both CTAs' code tiles landed
    uint64_t *empty = full + NS;          // MMAs done with stage s (commit to both CTAs)
    uint64_t *sfull = empty + NS;         // this CTA's raw factors of stage s landed
    uint64_t *sfready = sfull + NS;       // leader: factors of stage s in both CTAs' TMEM
    uint64_t *sflocal = sfready + NS;     // peer: its four factor warps wrote stage s
    uint64_t *acc_full = sflocal + NS;    // accumulator complete (commit to both CTAs)
    uint64_t *acc_empty = acc_full + 1;   // leader: both CTAs' epilogues drained TMEM (8 or 16 warps)
    uint64_t *drain = acc_empty + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::o_misc);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + C::o_misc + 4);
    auto stage = [&](int s) { return smem + s * C::kStage; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int blk = args.block;                       // 16 or 32
    const int nraw = C::BKE / blk;                    // raw factor rows per stage
    const uint32_t rank = cluster_ctarank();
    const int64_t unit = blockIdx.x >> 1;
    const int64_t nunits = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
            mbar_init(&sfull[i], 1);
            mbar_init(&sfready[i], 5);     // the leader's four factor warps + the peer's relay
            mbar_init(&sflocal[i], 4);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, ATOMS ? 16 : 8);
        mbar_init(drain, 1);
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(GRID == 0 ? &args.tm_a_corr : (C::kMx ? &args.tm_a_e8 : &args.tm_a_codes));
        tma_prefetch_desc(GRID == 0 ? &args.tm_b_corr : (C::kMx ? &args.tm_b_e8 : &args.tm_b_codes));
        tma_prefetch_desc(ATOMS ? &args.tm_a_atoms : &args.tm_a_scales);
        tma_prefetch_desc(ATOMS ? &args.tm_b_atoms : &args.tm_b_scales);
    }
    if (warp == 1) tmem_alloc_pair(tmem_slot, 512);
    // Grouped problems: the schedule goes group by group in decreasing K
    // (ties by index), so the longest tiles start first and the persistent
    // CTA pairs finish together (ragged K per group, as in an expert WGRAD),
    // and the tile -> group lookup is a binary search over prefix counts in
    // shared memory.  Every CTA builds the same schedule: group g's rank
    // counts the groups scheduled before it.
    uint16_t *order_s = reinterpret_cast<uint16_t *>(smem + C::o_order);
    int64_t *cum_s = reinterpret_cast<int64_t *>(smem + C::o_cum);
    const bool scheduled = args.groups != nullptr && args.num_groups <= C::kMaxOrder;
    if (scheduled) {
        if (static_cast<int>(threadIdx.x) < args.num_groups) {
            const int gi = threadIdx.x;
            const GemmGroup g = load_group(args, gi);
            int rankv = 0;
            for (int j = 0; j < args.num_groups; ++j) {
                const int64_t kj = load_group(args, j).k;
                rankv += (kj > g.k || (kj == g.k && j < gi)) ? 1 : 0;
            }
            order_s[rankv] = static_cast<uint16_t>(gi);
            cum_s[rankv + 1] = tiles_of<TM, BN>(g);      // tiles of the rank-th group, summed below
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            cum_s[0] = 0;
            for (int r = 1; r <= args.num_groups; ++r) cum_s[r] += cum_s[r - 1];
        }
    }
    const GroupSchedule sched{scheduled ? order_s : nullptr, cum_s, args.num_groups};
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int64_t ntiles = scheduled ? cum_s[args.num_groups] : total_tiles<TM, BN>(args);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_last();
            uint32_t it = 0;
            bool ok = true;
            for (int64_t t = unit; t < ntiles && ok; t += nunits) {
                const Tile tl = get_tile<TM, BN>(args, t, sched);
                const int nks = static_cast<int>((tl.g.k + C::BKE - 1) / C::BKE);
                const int32_t arow = static_cast<int32_t>(tl.g.a_row + tl.m0 + 128 * rank);
                const int32_t brow = static_cast<int32_t>(tl.g.b_row + tl.n0);
                const int32_t brow_h = brow + 128 * static_cast<int32_t>(rank);
                for (int ks = 0; ks < nks; ++ks, ++it) {
                    const int s = it % NS;
                    if (it >= static_cast<uint32_t>(NS) &&
                        !mbar_wait(&empty[s], ((it / NS) - 1) & 1, kErrTimeoutProducer, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int32_t acol = static_cast<int32_t>(tl.g.a_col + ks * C::BKE);
                    const int32_t bcol = static_cast<int32_t>(tl.g.b_col + ks * C::BKE);
                    uint8_t *st = stage(s);
                    const uint32_t fb = cluster_addr(&full[s], 0);
                    if constexpr (ATOMS) {
                        // factor atoms of this CTA's A rows and of all 256 B rows, with the
                        // code tiles on the leader's barrier: 128 K elements per box
                        if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * (C::kCodeBytes + C::kRawA + C::kRawB));
                        // 64 u64 per atom of kAtomK K elements (dense problems: acol = bcol)
                        constexpr int kAtomK = C::kMx ? 128 : 64;
                        const int32_t ax = 64 * (acol / kAtomK), bx = 64 * (bcol / kAtomK);
                        if constexpr (C::kLaneA)   // this CTA's 128 A rows: the stage's per-lane tile
                            tma_load_3d_pair(st + C::o_raw_a, &args.tm_a_atoms, fb, 0, 0,
                                             (arow / 128) * args.lane_groups + acol / kLaneK, pol);
                        else
                            tma_load_2d_pair(st + C::o_raw_a, &args.tm_a_atoms, fb, ax, arow / 128, pol);
                        tma_load_2d_pair(st + C::o_raw_b, &args.tm_b_atoms, fb, bx, brow / 128, pol);
                    } else {
                        // this CTA's raw factors
                        mbar_arrive_expect_tx(&sfull[s], (128 + 256) * nraw);
                        tma_load_2d_hint(st + C::o_raw_a, &args.tm_a_scales, &sfull[s], arow, acol / blk, pol);
                        tma_load_2d_hint(st + C::o_raw_b, &args.tm_b_scales, &sfull[s], brow, bcol / blk, pol);
                        // code tiles of both CTAs complete on the leader's barrier
                        if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * C::kCodeBytes);
                    }
                    if (GRID == 0) {
                        tma_load_3d_pair(st + C::o_a, &args.tm_a_corr, fb, acol / 2, arow, 0, pol);
                        tma_load_3d_pair(st + C::o_b, &args.tm_b_corr, fb, bcol / 2, brow_h, 0, pol);
                    } else if (C::kMx) {
                        tma_load_2d_pair(st + C::o_a, &args.tm_a_e8, fb, acol, arow, pol);
                        tma_load_2d_pair(st + C::o_b, &args.tm_b_e8, fb, bcol, brow_h, pol);
                    } else {
                        tma_load_2d_pair(st + C::o_a, &args.tm_a_codes, fb, acol / 2, arow, pol);
                        tma_load_2d_pair(st + C::o_b, &args.tm_b_codes, fb, bcol / 2, brow_h, pol);
                    }
                }
            }
            // Drain: this CTA's factor copies have landed before it exits
            // (the leader's MMAs consumed every code stage it issued).
            for (uint32_t d = 0; d < static_cast<uint32_t>(NS) && d < it; ++d) {
                const uint32_t idx = it - 1 - d;
                uint32_t dummy = 0;
                if (!ATOMS)
                    mbar_wait(&sfull[idx % NS], (idx / NS) & 1, kErrTimeoutDrain,
                              reinterpret_cast<volatile uint32_t *>(&dummy));
                if (rank == 0)
                    mbar_wait_cluster(&full[idx % NS], (idx / NS) & 1, kErrTimeoutDrain,
                                      reinterpret_cast<volatile uint32_t *>(&dummy));
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = umma_idesc_fp4_bs(TM, BN);
            uint32_t it = 0, tcount = 0;
            bool ok = true;
            for (int64_t t = unit; t < ntiles && ok; t += nunits, ++tcount) {
                const Tile tl = get_tile<TM, BN>(args, t, sched);
                const int nks = static_cast<int>((tl.g.k + C::BKE - 1) / C::BKE);
                if (!mbar_wait_cluster(acc_empty, (tcount & 1) ^ 1, kErrTimeoutMma, abort_flag)) break;
                tc_fence_after();
                bool first = true;
                for (int ks = 0; ks < nks; ++ks, ++it) {
                    const int s = it % NS;
                    if (!mbar_wait(&full[s], (it / NS) & 1, kErrTimeoutMma, abort_flag) ||
                        (!ATOMS && !mbar_wait_cluster(&sfready[s], (it / NS) & 1, kErrTimeoutMma, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint8_t *st = stage(s);
                    const uint32_t sf0 = tmem_base + C::kSfBase + s * C::kSfCols;
                    if constexpr (ATOMS) {
                        // the stage's factor atoms into TMEM slot s of both CTAs (each from its
                        // own shared memory; the copies run before the MMAs issued after them,
                        // and after the MMAs that last read the slot)
                        if constexpr (C::kLaneA) {
                            // A: columns sf0 + 4 j + q (K step j, lane quarter q); B of K step j:
                            // columns sf0 + 8 + 8 j (rows 0-127) and + 4 (rows 128-255)
                            tmem_cp_lanes_pair(sf0, smem_addr(st + C::o_raw_a));
#pragma unroll
                            for (int j = 0; j < C::KST; ++j) {
                                tmem_cp_atom_pair(sf0 + 8 + 8 * j, smem_addr(st + C::o_raw_b + 512 * j));
                                tmem_cp_atom_pair(sf0 + 12 + 8 * j, smem_addr(st + C::o_raw_b + 512 * (C::KST + j)));
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < C::KST; ++j) {
                                tmem_cp_atom_pair(sf0 + 12 * j, smem_addr(st + C::o_raw_a + 512 * j));
                                tmem_cp_atom_pair(sf0 + 12 * j + 4, smem_addr(st + C::o_raw_b + 512 * j));
                                tmem_cp_atom_pair(sf0 + 12 * j + 8,
                                                  smem_addr(st + C::o_raw_b + 512 * (C::KST + j)));
                            }
                        }
                    }
                    const int64_t rem = tl.g.k - static_cast<int64_t>(ks) * C::BKE;
                    const int steps = rem >= C::BKE ? C::KST : static_cast<int>((rem + 63) / 64);
                    const uint32_t a0 = smem_addr(st + C::o_a), b0 = smem_addr(st + C::o_b);
                    const uint32_t ac = a0 + C::kTile, bc = b0 + C::kTile;
                    if constexpr (C::kMx) {
                        // K = 32 MMAs (32 bytes of the 128-byte rows), factor byte j:
                        // four per full stage (a K tail of 64 takes two)
                        const int nk32 = rem >= C::BKE ? C::BKE / 32 : static_cast<int>(rem / 32);
                        for (int j = 0; j < nk32; ++j) {
                            umma_mxf8_pair(tmem_base, umma_desc_sw128(a0 + 32 * j), umma_desc_sw128(b0 + 32 * j),
                                           umma_idesc_mxf8(TM, BN, static_cast<uint32_t>(j)), sf0, sf0 + 4,
                                           first ? 0u : 1u);
                            first = false;
                        }
                    } else {
                        // code rows of 64 bytes (64-byte swizzle) or, for 256-K stages, 128 bytes
                        auto desc = [](uint32_t addr) {
                            return C::kRow == 128 ? umma_desc_sw128(addr) : umma_desc_sw64(addr);
                        };
                        for (int j = 0; j < steps; ++j) {
                            const uint32_t sfa = C::kLaneA ? sf0 + 4 * j : sf0 + 12 * j;
                            const uint32_t sfb = C::kLaneA ? sf0 + 8 + 8 * j : sfa + 4;
                            const uint32_t dk = 32 * j;
                            umma_fp4_bs_pair(tmem_base, desc(a0 + dk), desc(b0 + dk), idesc, sfa, sfb,
                                             first ? 0u : 1u);
                            first = false;
                            if (GRID == 0) {
                                umma_fp4_bs_pair(tmem_base, desc(a0 + dk), desc(bc + dk), idesc, sfa, sfb, 1u);
                                umma_fp4_bs_pair(tmem_base, desc(ac + dk), desc(b0 + dk), idesc, sfa, sfb, 1u);
                                umma_fp4_bs_pair(tmem_base, desc(ac + dk), desc(bc + dk), idesc, sfa, sfb, 1u);
                            }
                        }
                    }
                    umma_commit_pair_mc(&empty[s], 0x3);
                }
                if (ok) umma_commit_pair_mc(acc_full, 0x3);
            }
            // Drain: every MMA issued here completes before TMEM is freed.
            umma_commit_pair(drain);
            uint32_t dummy = 0;
            mbar_wait(drain, 0, kErrTimeoutDrain, reinterpret_cast<volatile uint32_t *>(&dummy));
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ factor relay (peer)
        // One cluster-scope arrive per stage on the leader's barrier once the
        // peer's four factor warps are done (their arrives stay CTA-local).
        if (!ATOMS && lane == 0 && rank == 1) {
            const uint32_t ready = cluster_addr(&sfready[0], 0);
            uint32_t it = 0;
            bool ok = true;
            for (int64_t t = unit; t < ntiles && ok; t += nunits) {
                const Tile tl = get_tile<TM, BN>(args, t, sched);
                const int nks = static_cast<int>((tl.g.k + C::BKE - 1) / C::BKE);
                for (int ks = 0; ks < nks; ++ks, ++it) {
                    const int s = it % NS;
                    if (!mbar_wait(&sflocal[s], (it / NS) & 1, kErrTimeoutTransform, abort_flag)) {
                        ok = false;
                        break;
                    }
                    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                                     ready + static_cast<uint32_t>(s) * 8u)
                                 : "memory");
                }
            }
        }
    } else if (!ATOMS && warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ factor writers
        uint8_t *scr = smem + C::o_scr + (warp - 4) * (C::kAtoms * 512);
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
        uint32_t it = 0;
        bool ok = true;
        for (int64_t t = unit; t < ntiles && ok; t += nunits) {
            const Tile tl = get_tile<TM, BN>(args, t, sched);
            const int nks = static_cast<int>((tl.g.k + C::BKE - 1) / C::BKE);
            for (int ks = 0; ks < nks; ++ks, ++it) {
                const int s = it % NS;
                // the raw factors landed, and the MMAs that last read TMEM slot s are done
                if (!warp_wait(&sfull[s], (it / NS) & 1, kErrTimeoutTransform, abort_flag) ||
                    (it >= static_cast<uint32_t>(NS) &&
                     !warp_wait(&empty[s], ((it / NS) - 1) & 1, kErrTimeoutTransform, abort_flag))) {
                    ok = false;
                    break;
                }
                const uint8_t *st = stage(s);
                uint32_t w[C::kAtoms][4];
#pragma unroll
                for (int a = 0; a < C::kAtoms; ++a) {
                    const int jk = a / 3, kind = a % 3;
                    const int rows = kind == 0 ? 128 : 256;
                    const int r = 4 * lane + (kind == 2 ? 128 : 0);
                    const uint8_t *raw = st + (kind == 0 ? C::o_raw_a : C::o_raw_b) + r;
                    if (C::kMx || blk == 16) {
                        // four factor rows per atom: 16-element blocks 4 jk .. 4 jk + 3,
                        // or (MX) the stage's four 32-element blocks
#pragma unroll
                        for (int kb = 0; kb < 4; ++kb)
                            w[a][kb] = *reinterpret_cast<const uint32_t *>(raw + (4 * jk + kb) * rows);
                    } else {
                        w[a][0] = w[a][1] = *reinterpret_cast<const uint32_t *>(raw + (2 * jk) * rows);
                        w[a][2] = w[a][3] = *reinterpret_cast<const uint32_t *>(raw + (2 * jk + 1) * rows);
                    }
                }
                // Atom byte 16 (r % 32) + 4 (r / 32) + kb holds the factor of
                // 16-element block 4 jk + kb of row r of the group.
#pragma unroll
                for (int a = 0; a < C::kAtoms; ++a) {
                    uint32_t o[4];
                    transpose4x4(w[a][0], w[a][1], w[a][2], w[a][3], o);
                    uint8_t *dst = scr + a * 512 + 16 * ((4 * lane) & 31) + 4 * ((4 * lane) >> 5);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) *reinterpret_cast<uint32_t *>(dst + 16 * q4) = o[q4];
                }
                __syncwarp();
                const uint32_t sfw = lane_base + C::kSfBase + s * C::kSfCols;
#pragma unroll
                for (int a = 0; a < C::kAtoms; ++a) {
                    const uint4 row = *reinterpret_cast<const uint4 *>(scr + a * 512 + 16 * lane);
                    tmem_st_32x32b_x4(sfw + 12 * (a / 3) + 4 * (a % 3), row.x, row.y, row.z, row.w);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                // the leader's warps arrive on its barrier directly; the
                // peer's on a local one that its relay forwards
                if (lane == 0) mbar_arrive(rank == 0 ? &sfready[s] : &sflocal[s]);
            }
        }
    } else if (ATOMS ? warp >= 4 : warp >= 8) {
        // ------------------------------------------------------------ epilogue
        // Warp w reads TMEM lane quarter w % 4 (accumulator rows 32 (w % 4) +
        // lane of this CTA's 128).  With factor atoms (no factor writers)
        // warps 4-11 drain the accumulator, 128 columns each (h = (w - 4) / 4
        // picks the half): all of them go to registers and TMEM is released
        // at once, so the next tile's MMAs overlap this tile's scaling and
        // stores.  Otherwise warps 8-11 take both halves, one after the
        // other, and release TMEM once the second half is in registers.
        const int q = warp & 3;
        const int h0 = ATOMS ? (warp - 4) >> 2 : 0;
        constexpr int kHalves = ATOMS ? 1 : 2;
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
        const uint32_t empty_acc = cluster_addr(acc_empty, 0);
        uint8_t *buf = smem + C::o_out + (warp - (ATOMS ? 4 : 8)) * 4096;
        // E1M2 operands carry k = 4 * level on both sides: 1/16 (exact).  The
        // MX path's E4M3 elements are the levels and its factors are in the
        // MMA: only 1/n.
        const float mult = C::kMx ? args.inv_n
                                  : __fmul_rn(__fmul_rn(*args.a_S, *args.b_S),
                                              args.inv_n * (GRID == 0 ? (1.0f / 16.0f) : 1.0f));
        uint32_t tcount = 0;
        for (int64_t t = unit; t < ntiles; t += nunits, ++tcount) {
            const Tile tl = get_tile<TM, BN>(args, t, sched);
            if (!warp_wait(acc_full, tcount & 1, kErrTimeoutEpilogue, abort_flag)) break;
            tc_fence_after();
            const int64_t m0 = tl.m0 + 128 * rank + 32 * q;   // this warp's accumulator rows
            const bool vec_tile = args.c_vec && (tl.g.c_col & 3) == 0;
            const bool zero = tl.g.k == 0;             // no MMA wrote the accumulator
#pragma unroll
            for (int hh = 0; hh < kHalves; ++hh) {
                const int h = h0 + hh;
                uint32_t r[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tmem_base + lane_addr + 128 * h + 32 * c, r[c]);
                tmem_wait_ld();
                if (hh == kHalves - 1) {
                    // accumulator drained by this warp: the next tile's MMAs
                    // may start once every epilogue warp of the pair arrived
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(empty_acc)
                                     : "memory");
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int64_t col0 = tl.n0 + 128 * h + 32 * c;
                    if (col0 >= tl.g.n) break;            // the same for the whole warp
                    store_piece(args, tl, buf, lane, m0, col0, r[c], mult, zero, vec_tile);
                }
            }
        }
    }

    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 512);
    }
}

template <int GRID, bool ATOMS, bool LANES = false>
cudaError_t launch_pair(const GemmArgs &args, int num_sms, cudaStream_t stream) {
    using C = PairCfg<GRID, ATOMS, LANES>;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemm_pair_kernel<GRID, ATOMS, LANES>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::kAlloc);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    int units = num_sms / 2;
    if (args.groups == nullptr) {
        const GemmGroup &g = args.single;
        const int64_t tiles = ((g.m + C::TM - 1) / C::TM) * ((g.n + C::BN - 1) / C::BN);
        if (tiles < units) units = static_cast<int>(tiles);
    }
    if (units <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(units * 2, 1, 1);
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemm_pair_kernel<GRID, ATOMS, LANES>, args);
}

template <int GRID, bool CIN>
cudaError_t launch_fp4(const GemmArgs &args, int num_sms, cudaStream_t stream) {
    using C = Fp4Cfg<GRID, CIN>;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemm_fp4_kernel<GRID, CIN>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::kAlloc);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    int units = num_sms;
    if (args.groups == nullptr) {
        const GemmGroup &g = args.single;
        const int64_t tiles = ((g.m + C::TM - 1) / C::TM) * ((g.n + C::BN - 1) / C::BN);
        if (tiles < units) units = static_cast<int>(tiles);
    }
    if (units <= 0) return cudaSuccess;
    gemm_fp4_kernel<GRID, CIN><<<units, C::kThreads, C::kAlloc, stream>>>(args);
    return cudaGetLastError();
}

template <int GRID, bool UE8>
cudaError_t launch_f32s_fmt(const GemmArgs &args, int num_sms, cudaStream_t stream) {
    using C = F32sCfg;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemm_f32s_kernel<GRID, UE8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kAlloc);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    int units = num_sms;
    if (args.groups == nullptr) {
        const GemmGroup &g = args.single;
        const int64_t tiles = ((g.m + C::TM - 1) / C::TM) * ((g.n + C::TN - 1) / C::TN);
        if (tiles < units) units = static_cast<int>(tiles);
    }
    if (units <= 0) return cudaSuccess;
    gemm_f32s_kernel<GRID, UE8><<<units, C::kThreads, C::kAlloc, stream>>>(args);
    return cudaGetLastError();
}

// fp32 or UE8M0 block scales: the scale decode is a compile-time choice.
template <int GRID>
cudaError_t launch_f32s(const GemmArgs &args, int num_sms, cudaStream_t stream) {
    return args.scale_ue8m0 ? launch_f32s_fmt<GRID, true>(args, num_sms, stream)
                            : launch_f32s_fmt<GRID, false>(args, num_sms, stream);
}

}  // namespace

cudaError_t launch_gemm(const GemmArgs &args, int mode, int grid_kind, int num_sms,
                        cudaStream_t stream) {
    switch (mode) {
        case 0:
            return grid_kind == 0 ? launch_f32s<0>(args, num_sms, stream) : launch_f32s<1>(args, num_sms, stream);
        case 3:
            if (grid_kind == 1) return launch_fp4<1, false>(args, num_sms, stream);
            return args.corr_in ? launch_fp4<0, true>(args, num_sms, stream) : launch_fp4<0, false>(args, num_sms, stream);
        case 5:
            if (args.atoms)
                return grid_kind == 1 ? launch_pair<1, true>(args, num_sms, stream)
                                      : (args.lanes ? launch_pair<0, true, true>(args, num_sms, stream)
                                                    : launch_pair<0, true, false>(args, num_sms, stream));
            return grid_kind == 1 ? launch_pair<1, false>(args, num_sms, stream)
                                  : launch_pair<0, false>(args, num_sms, stream);
        case 6:
            return args.atoms ? launch_pair<3, true>(args, num_sms, stream) : launch_pair<3, false>(args, num_sms, stream);
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace ufp4

namespace ufp4 {

// Host side of ufp4_check_device_status (the error word lives in this
// translation unit).  Synchronises the current device.
cudaError_t read_and_clear_error_word(uint32_t *out) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(out, g_error_word, sizeof(uint32_t));
    if (e != cudaSuccess) return e;
    const uint32_t zero = 0;
    return cudaMemcpyToSymbol(g_error_word, &zero, sizeof(uint32_t));
}

}  // namespace ufp4
