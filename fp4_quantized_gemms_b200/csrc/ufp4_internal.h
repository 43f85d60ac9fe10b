// ufp4_internal.h -- launch interfaces between the C ABI layer and kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ufp4.h"

namespace ufp4 {

// Bits of the device error word: a bounded wait of that role gave up
// (kernels OR them in; the host reads and clears the word in
// ufp4_check_device_status).
enum : uint32_t {
    kErrTimeoutProducer = 1u << 0,
    kErrTimeoutTransform = 1u << 1,
    kErrTimeoutMma = 1u << 2,
    kErrTimeoutEpilogue = 1u << 3,
    kErrTimeoutDrain = 1u << 4,
};

}  // namespace ufp4

namespace ufp4 {

// The ten round keys of a Philox4x32-10 key: (x, y)_r = key + r * (the two
// Weyl constants), the schedule of Salmon et al. (SC'11).
struct PhiloxKeys {
    uint32_t x[10], y[10];
};

struct QuantArgs {
    const uint16_t *x;   // bf16 input [rows][ld]
    int64_t rows, cols, ld;
    int axis;            // 0: reduce along cols, 1: along rows (transposed out)
    int64_t out_rows;    // rows of the K-major output
    int64_t K, kpad, scale_ld;
    uint8_t *codes;      // [out_rows][kpad/2]
    uint8_t *corr;       // E1M2 correction plane, same layout, or nullptr
    uint8_t *elems8;     // E4M3 element plane [out_rows][kpad] (MX path), or nullptr
    uint8_t *sf_atoms;   // factor atoms [ceil(out_rows/128)][atoms_k][512], or nullptr
    int64_t atoms_k;     // atoms along K (kpad / 64 for E4M3 factors, kpad / 128 rounded up for UE8M0)
    uint8_t *sf_lanes;   // per-lane factor tiles [ceil(out_rows/128)][lane_groups][4096], or nullptr
    int64_t lane_groups; // 128-K groups along K (ceil(kpad / 128))
    void *scales;        // block-major [kpad/B][scale_ld], fp32 or E4M3
    float *S_out;        // two-level: receives S
    const float *amax_t; // two-level: rotated tensor amax
    float *amax_out;     // amax kernel output
    uint64_t seed;
    uint32_t stream;
    uint64_t sign_mask;
    int scale_fmt;
    int grid;            // ufp4_grid_t (filled by the launcher)
    int64_t num_units;   // filled by the launcher
    // Per-call constants the kernels read from the parameter bank instead of
    // holding in registers (filled by the launcher from seed / sign_mask):
    PhiloxKeys keys;     // round keys of `seed`
    uint32_t smask[64];  // D sign of lane-run position p (period n), fp32 sign bit
};

cudaError_t launch_rht_quantize(QuantArgs a, int hadamard_n, int block, int grid_kind,
                                int rounding, int num_sms, cudaStream_t stream);
cudaError_t launch_rht_amax(QuantArgs a, int hadamard_n, int num_sms, cudaStream_t stream);
// Unfused RHT: y = bf16(H_n D x) along cols (cols % 64 == 0).
cudaError_t launch_rht_bf16(QuantArgs a, int hadamard_n, uint16_t *y, int64_t ldy, int num_sms,
                            cudaStream_t stream);
// One read of the input, both outputs: a_rows (axis 1, drives the units) and
// a_cols (axis 0); same grid / rounding / RHT / block for both.
cudaError_t launch_rht_quantize_dual(QuantArgs a_rows, QuantArgs a_cols, int hadamard_n, int block,
                                     int grid_kind, int rounding, int num_sms, cudaStream_t stream);
cudaError_t launch_rht_amax_dual(QuantArgs a_rows, QuantArgs a_cols, int hadamard_n, int num_sms,
                                 cudaStream_t stream);

// Statistics of one quantized operand (diag.cu).
struct DiagArgs {
    const uint16_t *x;      // bf16 input [rows][ld]
    int64_t rows, cols, ld;
    int axis;
    int64_t out_rows, K, kpad, scale_ld;
    const uint8_t *codes;   // [out_rows][kpad/2]
    const void *scales;     // block-major, fp32 or E4M3
    const float *S;         // two-level tensor scale (device)
    int scale_fmt, grid, block;
    uint64_t sign_mask;
    ufp4_qstats_t *out;     // device
};

cudaError_t launch_quant_stats(const DiagArgs &a, int hadamard_n, int num_sms, cudaStream_t stream);
cudaError_t launch_sqnr_sums(const float *ref, int64_t ld_ref, const float *test, int64_t ld_test,
                             int64_t rows, int64_t cols, double *sums, int num_sms, cudaStream_t stream);

// One contraction problem (a group of the grouped GEMM, or the whole GEMM).
struct GemmGroup {
    int64_t m, n, k;
    int64_t a_row, a_col;
    int64_t b_row, b_col;
    int64_t c_row, c_col;
};

struct GemmArgs {
    CUtensorMap tm_a_codes, tm_b_codes;   // u8 [rows][kpad/2]
    CUtensorMap tm_a_scales, tm_b_scales; // [nblk][scale_ld], fp32 or u8
    const float *a_S, *b_S;               // two-level tensor scales (device)
    float *c;
    int64_t ldc;
    float inv_n;                          // 1/n of the Hadamard size (1 if none)
    int block;                            // 16 or 32
    const GemmGroup *groups;              // device table or nullptr
    int num_groups;
    GemmGroup single;                     // used when groups == nullptr
    int c_vec;                            // c 16-byte aligned and ldc % 4 == 0
    CUtensorMap tm_a_corr, tm_b_corr;     // E1M2 correction planes (corr_in); with
                                          // planes3d: 3-D maps over {codes, corr}
    int corr_in;                          // both operands carry correction planes
    int scale_ue8m0;                      // mode 0: scales are UE8M0 exponent bytes
    int planes3d;                         // corr = codes + rows * kpad / 2 for both
    CUtensorMap tm_a_e8, tm_b_e8;         // MX path: E4M3 element planes [rows][kpad]
    CUtensorMap tm_a_atoms, tm_b_atoms;   // factor atoms as u64 [row groups][64 atoms_k]; for
                                          // E1M2 the A map covers the per-lane tiles instead
                                          // (u64 [tiles][2][256])
    int32_t lane_groups;                  // per-lane tiles per 128-row group of A (E1M2)
    int lanes;                            // A carries per-lane factor tiles (E1M2 pair kernel)
    int atoms;                            // both operands carry factor atoms (pair kernels, dense)
    int band;                             // tile order: rows of tiles per band (0: M fastest)
};

// Tile columns (B rows) of the native block-scaled FP4 kernels (modes 3, 4).
constexpr int kNativeTileN = 192;
constexpr int kTileBand = 8;   // rows of output tiles per band of the GEMM tile order
// Per-lane factor tiles (E1M2 operands with E4M3 factors): the A-operand
// factors of 128 rows x 128 K in the image of one 128-lane x 256-bit tensor
// memory copy.  Each 32-lane quarter q of the block-scaled MMA reads the
// factors of its rows from column (factor base + q), and the factor base is
// a multiple of 4 columns; with bases c and c + 4 for K steps 0 and 1, lane
// L (row L of the group, q = L / 32) holds the four factors of K step j in
// column c + 4 j + q.  One copy then serves both K steps, where the
// factor atoms (32 rows, copied to every quarter) take one copy each.
// Tile layout: two halves of 2048 bytes (K steps 0 and 1), lane L's 16
// bytes of a half at 16 L, the factors at bytes 4 q .. 4 q + 3 of them.
constexpr int kLaneK = 128;
constexpr int kLaneTileBytes = 4096;
// K elements per pipeline stage of the CTA-pair kernels: 256 for E2M1
// operands with factor atoms (one MMA per 64 K: a longer stage spreads the
// issuer's per-stage waits, fences and commits over more MMAs), else 128.
constexpr int pair_stage_k(int grid_kind, bool atoms) { return (grid_kind == 1 && atoms) ? 256 : 128; }

// mode 0: fp32 block scales (per-block partial products, CUDA-core scaling)
// mode 1: E4M3 x fp32 two-level scales (scales folded into fp16 operands)
// mode 2: mode 1 on a CTA pair (cta_group::2, 256 x 256 tiles)
// mode 3: two-level scales on the native block-scaled FP4 MMA (kind::mxf4nvf4)
cudaError_t launch_gemm(const GemmArgs &args, int mode, int grid_kind, int num_sms,
                        cudaStream_t stream);

// Driver entry point for tensor-map encoding (resolved once at run time).
CUresult encode_tensor_map_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base,
                              uint64_t inner, uint64_t outer, uint64_t row_bytes,
                              uint32_t box_inner, uint32_t box_outer,
                              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE);
// 3-D map without swizzle: dims innermost first, strides of dims 1 and 2 in bytes.
CUresult encode_tensor_map_3d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base,
                              const cuuint64_t (&dims)[3], const cuuint64_t (&strides)[2],
                              const cuuint32_t (&box)[3]);
// u8 planes [planes][outer][inner] (plane_bytes apart), boxes of every plane.
CUresult encode_tensor_map_planes(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                                  uint64_t planes, uint64_t plane_bytes, uint32_t box_inner,
                                  uint32_t box_outer, CUtensorMapSwizzle swizzle);

}  // namespace ufp4
