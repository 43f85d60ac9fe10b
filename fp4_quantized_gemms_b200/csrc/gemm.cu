// gemm.cu -- block-scaled 4-bit TN contraction on tcgen05 tensor cores.
//
// C[i][j] = (1/n) * sum_k deq(A)[i][k] * deq(B)[j][k]   (fp32 accumulate)
//
// Both operands arrive K-major as packed sign-magnitude nibbles plus block
// scales, exactly as ufp4_rht_quantize writes them.  FPROP, DGRAD and WGRAD
// are this one kernel: the quantizer already laid every operand out along its
// GEMM's reduction dimension (paperlayer.ai summary §2, "for the three
// training GEMMs, RHT acts along the shared reduction dimension").
//
// No tcgen05 MMA kind consumes a uniform 4-bit grid, and none applies an fp32
// scale per 16 elements.  Both 4-bit grids are exact in fp16, so the kernel
// expands codes to fp16 in shared memory and runs kind::f16:
//   mode 1 (E4M3 x fp32 two-level scales): e_b * lvl has at most 7
//     significant bits and lies in [2^-11, 2688], so it is exact in fp16; the
//     scale is folded into the operand and one fp32 accumulation runs over
//     all of K.  The tensor scales S_a * S_b / n are applied in the epilogue.
//   mode 0 (fp32 block scales): each 16-block is one K=16 MMA into its own
//     TMEM buffer (an exact partial: sums of at most 32 products on a 1/16
//     lattice); epilogue warps add s_a * s_b * partial into fp32 registers.
//
// Pipeline (one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: packed codes (+ scales) of each 64-wide K stage
//   warp 1      TMEM owner and single-thread UMMA issuer
//   transform   codes -> fp16 in the 128-byte-swizzled UMMA layout
//   epilogue    TMEM -> registers -> (scale) -> global fp32
// Every wait is bounded (see ufp4_device.cuh); a stuck pipeline sets the
// device error word and the CTA unwinds, drains its copies, frees TMEM.

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define UFP4_PIPELINE_KERNELS 1
#include "ufp4_device.cuh"
#include "ufp4_internal.h"

namespace ufp4 {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;             // K elements per pipeline stage
constexpr int kCodeRow = BK / 2;   // packed bytes per row per stage
constexpr int kOpRow = BK * 2;     // fp16 bytes per row per stage (= 128)

template <int MODE>
struct Cfg;

template <>
struct Cfg<1> {
    static constexpr int BN = 256;
    static constexpr int NT = 8;   // transform warps
    static constexpr int NE = 4;   // epilogue warps
    static constexpr int NC = 4;   // code ring slots
    static constexpr int NO = 3;   // fp16 operand ring slots
    static constexpr int NS = 0;   // separate scale ring slots
    static constexpr int NP = 2;   // TMEM accumulators (BN columns each)
    static constexpr int kScaleElt = 1;
};

template <>
struct Cfg<0> {
    static constexpr int BN = 128;
    static constexpr int NT = 2;
    static constexpr int NE = 8;
    static constexpr int NC = 4;
    static constexpr int NO = 3;
    static constexpr int NS = 4;
    static constexpr int NP = 4;   // TMEM partial buffers (BN columns each)
    static constexpr int kScaleElt = 4;
};

template <int MODE>
struct Layout {
    using C = Cfg<MODE>;
    static constexpr int BN = C::BN;
    static constexpr int kOpA = BM * kOpRow;
    static constexpr int kOpB = BN * kOpRow;
    static constexpr int kCodeA = BM * kCodeRow;
    static constexpr int kCodeB = BN * kCodeRow;
    // scales per stage for the smallest block (16): BK/16 = 4 blocks
    static constexpr int kScA = BM * (BK / 16) * C::kScaleElt;
    static constexpr int kScB = BN * (BK / 16) * C::kScaleElt;
    static constexpr int kCodeSlot = MODE == 1 ? kCodeA + kCodeB + kScA + kScB : kCodeA + kCodeB;
    static constexpr int kScSlot = MODE == 0 ? kScA + kScB : 0;

    static constexpr int off_op = 0;
    static constexpr int off_code = off_op + C::NO * (kOpA + kOpB);
    static constexpr int off_sc = off_code + C::NC * kCodeSlot;
    static constexpr int off_bar = (off_sc + C::NS * kScSlot + 127) / 128 * 128;
    // barriers: code_full, code_empty, op_full, op_empty, sc_full, sc_empty,
    //           p_full, p_empty, drain
    static constexpr int kNumBars = 2 * C::NC + 2 * C::NO + 2 * C::NS + 2 * C::NP + 1;
    static constexpr int off_misc = off_bar + kNumBars * 8;
    static constexpr int kBytes = off_misc + 64;
    static constexpr int kAlloc = kBytes + 1024;   // slack for 1024-byte alignment
    static constexpr int kThreads = 32 * (2 + C::NT + C::NE);
    static constexpr int kTmemCols = 512;
    static_assert(C::NP * BN <= kTmemCols, "TMEM budget");
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

template <int BN>
__device__ __forceinline__ int64_t tiles_of(const GemmGroup &g) {
    if (!group_ok(g)) return 0;
    return ((g.m + BM - 1) / BM) * ((g.n + BN - 1) / BN);
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

template <int BN>
__device__ int64_t total_tiles(const GemmArgs &a) {
    const int ng = a.groups == nullptr ? 1 : a.num_groups;
    int64_t t = 0;
    for (int i = 0; i < ng; ++i) t += tiles_of<BN>(load_group(a, i));
    return t;
}

// Tile t of the concatenated schedule (groups in order, M fastest inside).
template <int BN>
__device__ Tile get_tile(const GemmArgs &a, int64_t t) {
    const int ng = a.groups == nullptr ? 1 : a.num_groups;
    Tile tl;
    for (int i = 0; i < ng; ++i) {
        const GemmGroup g = load_group(a, i);
        const int64_t nt = tiles_of<BN>(g);
        if (t < nt) {
            const int64_t mt = (g.m + BM - 1) / BM;
            tl.g = g;
            tl.m0 = (t % mt) * BM;
            tl.n0 = (t / mt) * BN;
            tl.nks = static_cast<int>(g.k / BK);
            return tl;
        }
        t -= nt;
    }
    tl.g = a.single;
    tl.m0 = tl.n0 = 0;
    tl.nks = 0;
    return tl;
}

// ---------------------------------------------------------------------------
// 4-bit code -> fp16 expansion.  A 32-bit word holds 8 codes (nibble i = K
// index i).  Output word i (i = 0..3) holds the fp16 pair (code i, code i+4):
// the same K permutation inside every 8-element chunk of both operands, which
// leaves every dot product (and every 16-block) unchanged.
__device__ __forceinline__ uint32_t sign_pair(uint32_t t) { return (t << 12) & 0x80008000u; }

// E1M2: magnitude index k itself (the level is k/4; the 1/4 goes to the scale).
__device__ __forceinline__ void expand_e1m2(uint32_t w, uint32_t (&o)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t t = w >> (4 * i);
        const uint32_t mag = (t & 0x00070007u) | 0x64006400u;   // fp16 1024 + k
        const __half2 h = __hsub2(*reinterpret_cast<const __half2 *>(&mag),
                                  __half2(__ushort_as_half(0x6400), __ushort_as_half(0x6400)));
        o[i] = *reinterpret_cast<const uint32_t *>(&h) ^ sign_pair(t);
    }
}

// E2M1: fp16 of the level {0,.5,1,1.5,2,3,4,6}; only the high byte is nonzero.
__device__ __forceinline__ void expand_e2m1(uint32_t w, uint32_t (&o)[4]) {
    const uint32_t m = w & 0x77777777u;
    const uint32_t lo = __byte_perm(0x3E3C3800u, 0x46444240u, m);
    const uint32_t hi = __byte_perm(0x3E3C3800u, 0x46444240u, m >> 16);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t sel = ((4u + i) << 12) | (static_cast<uint32_t>(i) << 4);
        o[i] = (__byte_perm(lo, hi, sel) & 0xFF00FF00u) ^ sign_pair(w >> (4 * i));
    }
}

template <int GRID>
__device__ __forceinline__ void expand(uint32_t w, uint32_t (&o)[4]) {
    if (GRID == 0) expand_e1m2(w, o);
    else expand_e2m1(w, o);
}

__device__ __forceinline__ uint32_t hmul2_bits(uint32_t x, __half2 s) {
    const __half2 r = __hmul2(*reinterpret_cast<const __half2 *>(&x), s);
    return *reinterpret_cast<const uint32_t *>(&r);
}

// ---------------------------------------------------------------------------
template <int MODE, int GRID>
__global__ void __launch_bounds__(Layout<MODE>::kThreads, 1)
    gemm_tn_kernel(const __grid_constant__ GemmArgs args) {
    using C = Cfg<MODE>;
    using Lay = Layout<MODE>;
    constexpr int BN = C::BN;
    constexpr int NSr = C::NS > 0 ? C::NS : 1;   // scale-ring modulus (mode 0 only)
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::off_bar);
    uint64_t *code_full = bars;
    uint64_t *code_empty = code_full + C::NC;
    uint64_t *op_full = code_empty + C::NC;
    uint64_t *op_empty = op_full + C::NO;
    uint64_t *sc_full = op_empty + C::NO;
    uint64_t *sc_empty = sc_full + C::NS;
    uint64_t *p_full = sc_empty + C::NS;
    uint64_t *p_empty = p_full + C::NP;
    uint64_t *drain = p_empty + C::NP;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::off_misc);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + Lay::off_misc + 4);

    auto op_a = [&](int s) { return smem + Lay::off_op + s * (Lay::kOpA + Lay::kOpB); };
    auto op_b = [&](int s) { return op_a(s) + Lay::kOpA; };
    auto code_a = [&](int s) { return smem + Lay::off_code + s * Lay::kCodeSlot; };
    auto code_b = [&](int s) { return code_a(s) + Lay::kCodeA; };
    // mode 1: scales ride in the code slot; mode 0: separate scale ring
    auto sc_a = [&](int s) {
        return MODE == 1 ? code_b(s) + Lay::kCodeB : smem + Lay::off_sc + s * Lay::kScSlot;
    };
    auto sc_b = [&](int s) { return sc_a(s) + Lay::kScA; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nblk_stage = BK / args.block;

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
    if (warp == 1) tmem_alloc(tmem_slot, Lay::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int64_t ntiles = total_tiles<BN>(args);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t it = 0, sit = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                const Tile tl = get_tile<BN>(args, t);
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
                    uint32_t bytes = Lay::kCodeA + Lay::kCodeB;
                    if (MODE == 1) bytes += (BM + BN) * nblk_stage;
                    mbar_arrive_expect_tx(&code_full[s], bytes);
                    tma_load_2d(code_a(s), &args.tm_a_codes, &code_full[s], acol / 2, arow);
                    tma_load_2d(code_b(s), &args.tm_b_codes, &code_full[s], bcol / 2, brow);
                    if (MODE == 1) {
                        tma_load_2d(sc_a(s), &args.tm_a_scales, &code_full[s], arow, acol / args.block);
                        tma_load_2d(sc_b(s), &args.tm_b_scales, &code_full[s], brow, bcol / args.block);
                    } else {
                        const int ss = sit % NSr;
                        const uint32_t suse = sit / NSr;
                        if (!mbar_wait(&sc_empty[ss], (suse & 1) ^ 1, kErrTimeoutProducer, abort_flag)) {
                            ok = false;
                            ++it;   // the code copies of this stage were issued
                            break;
                        }
                        mbar_arrive_expect_tx(&sc_full[ss], (BM + BN) * nblk_stage * 4);
                        tma_load_2d(sc_a(ss), &args.tm_a_scales, &sc_full[ss], arow, acol / args.block);
                        tma_load_2d(sc_b(ss), &args.tm_b_scales, &sc_full[ss], brow, bcol / args.block);
                        ++sit;
                    }
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
                    const uint32_t last = (sit - 1 - s) / NSr * NSr + s;
                    uint32_t dummy = 0;
                    mbar_wait(&sc_full[s], (last / NSr) & 1, kErrTimeoutDrain,
                              reinterpret_cast<volatile uint32_t *>(&dummy));
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ UMMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_f16_f32(BM, BN);
            uint32_t it = 0, pq = 0, tcount = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tcount) {
                const Tile tl = get_tile<BN>(args, t);
                uint32_t acc_col = 0;
                if (MODE == 1) {
                    const int b = tcount & 1;
                    if (!mbar_wait(&p_empty[b], ((tcount >> 1) & 1) ^ 1, kErrTimeoutMma, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    acc_col = b * BN;
                }
                for (int ks = 0; ks < tl.nks && ok; ++ks, ++it) {
                    const int s = it % C::NO;
                    if (!mbar_wait(&op_full[s], (it / C::NO) & 1, kErrTimeoutMma, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_addr(op_a(s));
                    const uint32_t b0 = smem_addr(op_b(s));
                    if (MODE == 1) {
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            umma_f16(tmem_base + acc_col, umma_desc_sw128(a0 + kk * 32),
                                     umma_desc_sw128(b0 + kk * 32), idesc,
                                     (ks > 0 || kk > 0) ? 1u : 0u);
                        }
                    } else {
                        const int slices = args.block / 16;
                        for (int bi = 0; bi < nblk_stage; ++bi, ++pq) {
                            const int p = pq % C::NP;
                            if (!mbar_wait(&p_empty[p], ((pq / C::NP) & 1) ^ 1, kErrTimeoutMma,
                                           abort_flag)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            for (int sl = 0; sl < slices; ++sl) {
                                const int kk = bi * slices + sl;
                                umma_f16(tmem_base + p * BN, umma_desc_sw128(a0 + kk * 32),
                                         umma_desc_sw128(b0 + kk * 32), idesc, sl > 0 ? 1u : 0u);
                            }
                            umma_commit(&p_full[p]);
                        }
                    }
                    umma_commit(&op_empty[s]);
                }
                if (MODE == 1 && ok) umma_commit(&p_full[tcount & 1]);
            }
            // Drain: every MMA issued by this thread completes before TMEM is freed.
            umma_commit(drain);
            uint32_t dummy = 0;
            mbar_wait(drain, 0, kErrTimeoutDrain, reinterpret_cast<volatile uint32_t *>(&dummy));
        }
    } else if (warp < 2 + C::NT) {
        // ------------------------------------------------------------ transform
        const int tt = threadIdx.x - 64;
        constexpr int kUnits = (BM + BN) * 2;   // (row, 32-code half)
        const __half2 unit2 = __float2half2_rn(GRID == 0 ? 0.25f : 1.0f);
        uint32_t it = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const Tile tl = get_tile<BN>(args, t);
            for (int ks = 0; ks < tl.nks; ++ks, ++it) {
                const int cs = it % C::NC;
                const int os = it % C::NO;
                if (!warp_wait(&code_full[cs], (it / C::NC) & 1, kErrTimeoutTransform, abort_flag) ||
                    !warp_wait(&op_empty[os], ((it / C::NO) & 1) ^ 1, kErrTimeoutTransform,
                               abort_flag)) {
                    ok = false;
                    break;
                }
                const uint8_t *ca = code_a(cs);
                const uint8_t *cb = code_b(cs);
                uint8_t *oa = op_a(os);
                uint8_t *ob = op_b(os);
                for (int u = tt; u < kUnits; u += C::NT * 32) {
                    const int row = u >> 1;
                    const int half = u & 1;
                    const bool isA = row < BM;
                    const int r = isA ? row : row - BM;
                    const uint4 w =
                        *reinterpret_cast<const uint4 *>((isA ? ca : cb) + r * kCodeRow + half * 16);
                    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
                    uint8_t *dst = isA ? oa : ob;
#pragma unroll
                    for (int wi = 0; wi < 4; ++wi) {
                        uint32_t o[4];
                        expand<GRID>(words[wi], o);
                        if (MODE == 1) {
                            const int blk = (half * 32 + wi * 8) / args.block;
                            const uint8_t e8 = isA ? sc_a(cs)[blk * BM + r] : sc_b(cs)[blk * BN + r];
                            const __half2 s2 = __hmul2(__float2half2_rn(e4m3_to_f32(e8)), unit2);
#pragma unroll
                            for (int q = 0; q < 4; ++q) o[q] = hmul2_bits(o[q], s2);
                        }
                        *reinterpret_cast<uint4 *>(dst + sw128_offset(r, half * 4 + wi)) =
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
        const int ew = warp - 2 - C::NT;      // 0 .. NE-1
        const int q = warp & 3;               // TMEM lane quarter of this warp
        const int row_in_tile = 32 * q + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
        if (MODE == 1) {
            const float mult = __fmul_rn(__fmul_rn(*args.a_S, *args.b_S), args.inv_n);
            uint32_t tcount = 0;
            for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++tcount) {
                const Tile tl = get_tile<BN>(args, t);
                const int b = tcount & 1;
                if (!warp_wait(&p_full[b], (tcount >> 1) & 1, kErrTimeoutEpilogue, abort_flag)) break;
                tc_fence_after();
                const int64_t row = tl.m0 + row_in_tile;
                const bool row_ok = row < tl.g.m;
                float *crow = args.c + (tl.g.c_row + row) * args.ldc + tl.g.c_col + tl.n0;
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tmem_base + b * BN + 32 * c + lane_addr, r);
                    tmem_wait_ld();
                    if (c == BN / 32 - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&p_empty[b]);
                    }
                    if (!row_ok) continue;
                    const int64_t col0 = tl.n0 + 32 * c;
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        v[i] = tl.nks > 0 ? __fmul_rn(__uint_as_float(r[i]), mult) : 0.0f;
                    float *dst = crow + 32 * c;
                    const bool vec = (col0 + 32 <= tl.g.n) &&
                                     ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0);
                    if (vec) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            *reinterpret_cast<float4 *>(dst + i) =
                                make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                    } else {
                        for (int i = 0; i < 32; ++i)
                            if (col0 + i < tl.g.n) dst[i] = v[i];
                    }
                }
            }
        } else {
            // fp32 block scales: acc += (s_a * s_b) * partial, per 16/32-block.
            const int h = ew >> 2;            // column half (64 columns)
            const float mult = args.inv_n * (GRID == 0 ? (1.0f / 16.0f) : 1.0f);
            uint32_t it = 0, pq = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                const Tile tl = get_tile<BN>(args, t);
                float acc[64];
#pragma unroll
                for (int i = 0; i < 64; ++i) acc[i] = 0.0f;
                for (int ks = 0; ks < tl.nks && ok; ++ks, ++it) {
                    const int ss = it % NSr;
                    if (!warp_wait(&sc_full[ss], (it / NSr) & 1, kErrTimeoutEpilogue, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const float *sa_tile = reinterpret_cast<const float *>(sc_a(ss));
                    const float *sb_tile = reinterpret_cast<const float *>(sc_b(ss));
                    for (int bi = 0; bi < nblk_stage; ++bi, ++pq) {
                        const int p = pq % C::NP;
                        if (!warp_wait(&p_full[p], (pq / C::NP) & 1, kErrTimeoutEpilogue, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const float sa = sa_tile[bi * BM + row_in_tile];
                        const float4 *sb4 = reinterpret_cast<const float4 *>(sb_tile + bi * BN + h * 64);
                        const uint32_t ta = tmem_base + p * BN + h * 64 + lane_addr;
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            uint32_t r[32];
                            tmem_ld_32x32b_x32(ta + 32 * half, r);
                            tmem_wait_ld();
                            if (half == 1) {
                                tc_fence_before();
                                __syncwarp();
                                if (lane == 0) mbar_arrive(&p_empty[p]);
                            }
#pragma unroll
                            for (int c4 = 0; c4 < 8; ++c4) {
                                const float4 sb = sb4[8 * half + c4];
                                float *ac = acc + 32 * half + 4 * c4;
                                ac[0] = __fmaf_rn(__fmul_rn(sa, sb.x), __uint_as_float(r[4 * c4 + 0]), ac[0]);
                                ac[1] = __fmaf_rn(__fmul_rn(sa, sb.y), __uint_as_float(r[4 * c4 + 1]), ac[1]);
                                ac[2] = __fmaf_rn(__fmul_rn(sa, sb.z), __uint_as_float(r[4 * c4 + 2]), ac[2]);
                                ac[3] = __fmaf_rn(__fmul_rn(sa, sb.w), __uint_as_float(r[4 * c4 + 3]), ac[3]);
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sc_empty[ss]);
                }
                if (!ok) break;
                const int64_t row = tl.m0 + row_in_tile;
                if (row < tl.g.m) {
                    const int64_t col0 = tl.n0 + h * 64;
                    float *dst = args.c + (tl.g.c_row + row) * args.ldc + tl.g.c_col + col0;
                    const bool vec = (col0 + 64 <= tl.g.n) &&
                                     ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0);
                    if (vec) {
#pragma unroll
                        for (int i = 0; i < 64; i += 4)
                            *reinterpret_cast<float4 *>(dst + i) =
                                make_float4(acc[i] * mult, acc[i + 1] * mult, acc[i + 2] * mult,
                                            acc[i + 3] * mult);
                    } else {
#pragma unroll
                        for (int i = 0; i < 64; ++i)
                            if (col0 + i < tl.g.n) dst[i] = acc[i] * mult;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Lay::kTmemCols);
    }
}

template <int MODE, int GRID>
cudaError_t launch_impl(const GemmArgs &args, int num_sms, cudaStream_t stream) {
    using Lay = Layout<MODE>;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemm_tn_kernel<MODE, GRID>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kAlloc);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    int grid = num_sms;
    if (args.groups == nullptr) {
        const GemmGroup &g = args.single;
        const int64_t tiles = ((g.m + BM - 1) / BM) * ((g.n + Lay::BN - 1) / Lay::BN);
        if (tiles < grid) grid = static_cast<int>(tiles);
    }
    if (grid <= 0) return cudaSuccess;
    gemm_tn_kernel<MODE, GRID><<<grid, Lay::kThreads, Lay::kAlloc, stream>>>(args);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const GemmArgs &args, int mode, int grid_kind, int num_sms,
                        cudaStream_t stream) {
    if (mode == 1) {
        return grid_kind == 0 ? launch_impl<1, 0>(args, num_sms, stream)
                              : launch_impl<1, 1>(args, num_sms, stream);
    }
    return grid_kind == 0 ? launch_impl<0, 0>(args, num_sms, stream)
                          : launch_impl<0, 1>(args, num_sms, stream);
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
