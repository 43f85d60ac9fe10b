// diag.cu -- quantization diagnostics: statistics of a quantized operand
// against the rotated values it was rounded from, and GEMM-output SQNR sums.
//
// The quantities are the ones the diagnostics of "Rethinking Shrinkage Bias in
// LLM FP4 Pretraining" report (paperlayer.ai summary §5 "Q1: Grid geometry and
// RHT", Appendix A; gist.science "Kwantisatie en GEMM Diagnostiek"): SQNR of
// tensors and GEMM outputs, bucket use of the codes and the signed error of
// each grid level.  Their definitions are stated in ufp4.h.
//
// quant_stats_kernel: one thread per (output row, 64-column segment), as in
// the quantizer.  The thread rebuilds the rotated values with the quantizer's
// fp32 arithmetic (D, then butterflies h = 1, 2, ..., n/2), reads its 32 code
// bytes and the block steps, and accumulates in fp32 over the segment:
// signal and noise in registers, the level errors and the code counts in
// thread-private shared-memory columns (index [j][thread]: a warp's 32
// accesses fall in 32 banks whatever j is).  Segment sums go to fp64
// registers; a block reduction and one atomic per quantity finish.  Reads
// 2 + 0.5 + scale bytes per element; the per-element work (about 30
// instructions) makes it issue-bound, not HBM-bound.
#include <cuda_runtime.h>
#include <stdint.h>

#include "ufp4.h"
#include "ufp4_device.cuh"
#include "ufp4_internal.h"

namespace ufp4 {

namespace {

constexpr int kDiagThreads = 256;
constexpr int kDiagWarps = kDiagThreads / 32;
// Reduced quantities: signal, noise, level_err[8] (fp64); level_n[8],
// code_count[16], nonzero, underflow (integers).
constexpr int kNumF = 10;
constexpr int kNumI = 26;

template <int AXIS, int NH>
__global__ void __launch_bounds__(kDiagThreads) quant_stats_kernel(const __grid_constant__ DiagArgs a) {
    __shared__ float s_err[8][kDiagThreads];
    __shared__ uint32_t s_cnt[16][kDiagThreads];
    __shared__ uint32_t s_dead[8][kDiagThreads];      // elements in blocks with step 0
    __shared__ float s_lv[8];
    __shared__ double s_redf[kDiagWarps][kNumF];
    __shared__ unsigned long long s_redi[kDiagWarps][kNumI];
    const int t = threadIdx.x;
    const int lane = t & 31, warp = t >> 5;
    if (t < 8) {
        const float e2m1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
        s_lv[t] = a.grid == 0 ? 0.25f * static_cast<float>(t) : e2m1[t];
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        s_err[j][t] = 0.0f;
        s_dead[j][t] = 0u;
    }
#pragma unroll
    for (int c = 0; c < 16; ++c) s_cnt[c][t] = 0u;
    __syncthreads();

    double signal = 0.0, noise = 0.0, lerr[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) lerr[j] = 0.0;
    uint32_t nonzero = 0, underflow = 0;
    const float S = a.scale_fmt == 1 ? *a.S : 1.0f;   // two-level only
    const int64_t nseg = a.kpad / 64;
    const int64_t units = nseg * a.out_rows;
    for (int64_t u = static_cast<int64_t>(blockIdx.x) * kDiagThreads + t; u < units;
         u += static_cast<int64_t>(gridDim.x) * kDiagThreads) {
        const int64_t r = u % a.out_rows, seg = u / a.out_rows;
        const int64_t k0 = seg * 64;
        const int nvalid = static_cast<int>(a.K - k0 < 64 ? a.K - k0 : 64);
        float v[64];
        if (AXIS == 0) {
            // row r of x, columns k0 .. k0 + 63 (cols % 8 == 0: whole uint4s)
            const uint16_t *src = a.x + r * a.ld + k0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                uint4 q = make_uint4(0u, 0u, 0u, 0u);
                if (8 * j < nvalid) q = *reinterpret_cast<const uint4 *>(src + 8 * j);
                const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    v[8 * j + 2 * e] = __uint_as_float(w[e] << 16);
                    v[8 * j + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
                }
            }
        } else {
            // column r of x, rows k0 .. k0 + 63
            const uint16_t *src = a.x + k0 * a.ld + r;
#pragma unroll
            for (int i = 0; i < 64; ++i)
                v[i] = i < nvalid ? __uint_as_float(static_cast<uint32_t>(src[i * a.ld]) << 16) : 0.0f;
        }
        if constexpr (NH > 0) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
                if ((a.sign_mask >> (i % NH)) & 1u) v[i] = __uint_as_float(__float_as_uint(v[i]) ^ 0x80000000u);
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
        }
        const uint4 *cp = reinterpret_cast<const uint4 *>(a.codes + r * (a.kpad / 2) + k0 / 2);
        const uint4 c0 = cp[0], c1 = cp[1];
        const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        // Block steps of the segment's four 16-element quarters as m * b:
        // (1, s), or (e_b, S).  lvl * m is exact in fp32 (3 x 4 significant
        // bits), so u - lvl * m * b below is one fma with a single rounding.
        float sm[4], sb[4], inv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t b = (k0 + 16 * j) / a.block;
            if (a.scale_fmt == 0) {
                sm[j] = 1.0f;
                sb[j] = reinterpret_cast<const float *>(a.scales)[b * a.scale_ld + r];
            } else if (a.scale_fmt == 2) {           // UE8M0: 2^(E - 127), exact
                sm[j] = 1.0f;
                sb[j] = ldexpf(1.0f, static_cast<int>(reinterpret_cast<const uint8_t *>(a.scales)[b * a.scale_ld + r]) - 127);
            } else {
                sm[j] = e4m3_to_f32(reinterpret_cast<const uint8_t *>(a.scales)[b * a.scale_ld + r]);
                sb[j] = S;
            }
            const float sv = __fmul_rn(sm[j], sb[j]);
            inv[j] = sv > 0.0f ? __frcp_rn(sv) : 0.0f;
        }
        float sig_acc = 0.0f, noi_acc = 0.0f;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            if (i < nvalid) {
                const uint32_t code = (cw[i >> 3] >> (4 * (i & 7))) & 15u;
                const uint32_t mag = code & 7u;
                const float lv = s_lv[mag];
                const float lm = __fmul_rn(lv, sm[i >> 4]);               // exact
                const float uf = v[i];
                const float d = __fmaf_rn((code & 8u) ? lm : -lm, sb[i >> 4], uf);
                sig_acc = __fmaf_rn(uf, uf, sig_acc);
                noi_acc = __fmaf_rn(d, d, noi_acc);
                if (inv[i >> 4] > 0.0f)
                    s_err[mag][t] += __fmaf_rn(-fabsf(uf), inv[i >> 4], lv);
                else
                    s_dead[mag][t] += 1u;
                s_cnt[code][t] += 1u;
                nonzero += uf != 0.0f;
                underflow += (uf != 0.0f) & (mag == 0u);
            }
        }
        signal += static_cast<double>(sig_acc);
        noise += static_cast<double>(noi_acc);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            lerr[j] += static_cast<double>(s_err[j][t]);
            s_err[j][t] = 0.0f;
        }
    }

    // Block reduction: warp shuffles, one row per warp in shared memory, then
    // one thread per quantity sums the rows and issues its atomic.
    double f[kNumF];
    unsigned long long iv[kNumI];
    f[0] = signal;
    f[1] = noise;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        f[2 + j] = lerr[j];
        const uint32_t live = s_cnt[j][t] + s_cnt[8 + j][t] - s_dead[j][t];
        iv[j] = live;
    }
#pragma unroll
    for (int c = 0; c < 16; ++c) iv[8 + c] = s_cnt[c][t];
    iv[24] = nonzero;
    iv[25] = underflow;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
        for (int j = 0; j < kNumF; ++j) f[j] += __shfl_xor_sync(0xFFFFFFFFu, f[j], off);
#pragma unroll
        for (int j = 0; j < kNumI; ++j) iv[j] += __shfl_xor_sync(0xFFFFFFFFu, iv[j], off);
    }
    if (lane == 0) {
#pragma unroll
        for (int j = 0; j < kNumF; ++j) s_redf[warp][j] = f[j];
#pragma unroll
        for (int j = 0; j < kNumI; ++j) s_redi[warp][j] = iv[j];
    }
    __syncthreads();
    if (t < kNumF) {
        double sum = 0.0;
        for (int w = 0; w < kDiagWarps; ++w) sum += s_redf[w][t];
        double *dst = t == 0 ? &a.out->signal : (t == 1 ? &a.out->noise : &a.out->level_err[t - 2]);
        if (sum != 0.0) atomicAdd(dst, sum);
    } else if (t >= 32 && t < 32 + kNumI) {
        const int j = t - 32;
        unsigned long long sum = 0;
        for (int w = 0; w < kDiagWarps; ++w) sum += s_redi[w][j];
        unsigned long long *dst = reinterpret_cast<unsigned long long *>(
            j < 8 ? &a.out->level_n[j]
                  : (j < 24 ? &a.out->code_count[j - 8] : (j == 24 ? &a.out->nonzero : &a.out->underflow)));
        if (sum != 0) atomicAdd(dst, sum);
    }
}

// sum ref^2 and sum (test - ref)^2 over a rows x cols region, fp64: one
// block per row at a time, threads over the columns (coalesced).
__global__ void __launch_bounds__(kDiagThreads) sqnr_sums_kernel(const float *ref, int64_t ld_ref,
                                                                 const float *test, int64_t ld_test,
                                                                 int64_t rows, int64_t cols, double *sums) {
    __shared__ double s_red[kDiagWarps][2];
    double sr = 0.0, sn = 0.0;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const float *pr = ref + r * ld_ref;
        const float *pt = test + r * ld_test;
        for (int64_t c = threadIdx.x; c < cols; c += kDiagThreads) {
            const double x = pr[c], y = pt[c];
            const double d = y - x;
            sr = fma(x, x, sr);
            sn = fma(d, d, sn);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        sr += __shfl_xor_sync(0xFFFFFFFFu, sr, off);
        sn += __shfl_xor_sync(0xFFFFFFFFu, sn, off);
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) {
        s_red[warp][0] = sr;
        s_red[warp][1] = sn;
    }
    __syncthreads();
    if (threadIdx.x < 2) {
        double s = 0.0;
        for (int w = 0; w < kDiagWarps; ++w) s += s_red[w][threadIdx.x];
        if (s != 0.0) atomicAdd(&sums[threadIdx.x], s);
    }
}

template <int AXIS>
cudaError_t launch_stats_axis(const DiagArgs &a, int hadamard_n, int num_sms, cudaStream_t stream) {
    const int64_t units = (a.kpad / 64) * a.out_rows;
    int64_t blocks = (units + kDiagThreads - 1) / kDiagThreads;
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks <= 0) return cudaSuccess;
    const int g = static_cast<int>(blocks);
    switch (hadamard_n) {
        case 0: quant_stats_kernel<AXIS, 0><<<g, kDiagThreads, 0, stream>>>(a); break;
        case 16: quant_stats_kernel<AXIS, 16><<<g, kDiagThreads, 0, stream>>>(a); break;
        case 32: quant_stats_kernel<AXIS, 32><<<g, kDiagThreads, 0, stream>>>(a); break;
        case 64: quant_stats_kernel<AXIS, 64><<<g, kDiagThreads, 0, stream>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant_stats(const DiagArgs &a, int hadamard_n, int num_sms, cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(a.out, 0, sizeof(ufp4_qstats_t), stream);
    if (e != cudaSuccess) return e;
    return a.axis == 0 ? launch_stats_axis<0>(a, hadamard_n, num_sms, stream)
                       : launch_stats_axis<1>(a, hadamard_n, num_sms, stream);
}

cudaError_t launch_sqnr_sums(const float *ref, int64_t ld_ref, const float *test, int64_t ld_test,
                             int64_t rows, int64_t cols, double *sums, int num_sms, cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(sums, 0, 2 * sizeof(double), stream);
    if (e != cudaSuccess || rows == 0 || cols == 0) return e;
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    const int g = static_cast<int>(rows < cap ? rows : cap);
    sqnr_sums_kernel<<<g, kDiagThreads, 0, stream>>>(ref, ld_ref, test, ld_test, rows, cols, sums);
    return cudaGetLastError();
}

}  // namespace ufp4
