// api.cu -- the C ABI of libufp4.so (declared in include/ufp4.h): argument
// validation on the host, tensor-map encoding, kernel dispatch.  No call
// allocates, frees or synchronises (ufp4_check_device_status excepted).

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <cmath>
#include <mutex>

#include "ufp4.h"
#include "ufp4_internal.h"

namespace ufp4 {

cudaError_t read_and_clear_error_word(uint32_t *out);            // gemm.cu
cudaError_t quantize_read_and_clear_error_word(uint32_t *out);   // quantize.cu
cudaError_t quantize_set_producer_wait_limit(uint64_t limit_ns);  // quantize.cu

namespace {

constexpr int64_t kKAlign = 64;
constexpr int64_t kScaleLdAlign = 64;

int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool cfg_valid(const ufp4_quant_cfg_t &c) {
    if (c.grid != UFP4_GRID_E1M2 && c.grid != UFP4_GRID_E2M1 && c.grid != UFP4_GRID_E2M1_MAX2)
        return false;
    if (c.rounding != UFP4_ROUND_RTNE && c.rounding != UFP4_ROUND_SR) return false;
    if (!(c.hadamard_n == 0 || c.hadamard_n == 16 || c.hadamard_n == 32 || c.hadamard_n == 64))
        return false;
    if (c.block != 16 && c.block != 32) return false;
    if (c.scale_fmt != UFP4_SCALE_FP32 && c.scale_fmt != UFP4_SCALE_E4M3_X_FP32 &&
        c.scale_fmt != UFP4_SCALE_UE8M0)
        return false;
    if (c.scale_fmt == UFP4_SCALE_UE8M0 && c.block != 32) return false;   // MX blocks are 32 long
    return true;
}

int sm_count() {
    static int cache[64];
    static std::once_flag flags[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::call_once(flags[dev], [dev] {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev] = n;
    });
    return cache[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Common checks of one quantized operand descriptor.
// Factor-atom slot width along K: 16 for E4M3 factors (the block16 MMA
// granularity), 32 for UE8M0; 0 = fp32 scales (no atoms).
int atom_slot(const ufp4_quant_cfg_t &c) {
    return c.scale_fmt == UFP4_SCALE_E4M3_X_FP32 ? 16 : c.scale_fmt == UFP4_SCALE_UE8M0 ? 32 : 0;
}

int64_t atoms_k_of(int64_t kpad, const ufp4_quant_cfg_t &c) {
    const int64_t w = 4 * atom_slot(c);
    return (kpad + w - 1) / w;
}

// E1M2 operands with E4M3 factors may carry per-lane factor tiles (the
// A-operand factor layout of the CTA-pair kernel).
bool has_lane_tiles(const ufp4_quant_cfg_t &c) {
    return c.grid == UFP4_GRID_E1M2 && c.scale_fmt == UFP4_SCALE_E4M3_X_FP32;
}

int64_t lane_groups_of(int64_t kpad) { return (kpad + kLaneK - 1) / kLaneK; }

// Bytes of the factor atoms.
int64_t atom_bytes_of(int64_t rows, int64_t kpad, const ufp4_quant_cfg_t &c) {
    return (rows + 127) / 128 * atoms_k_of(kpad, c) * 512;
}

ufp4_status_t check_qtensor(const ufp4_qtensor_t *q) {
    if (q == nullptr) return UFP4_ERR_INVALID_ARG;
    if (!cfg_valid(q->cfg)) return UFP4_ERR_INVALID_ARG;
    if (q->rows < 0 || q->k < 0) return UFP4_ERR_INVALID_ARG;
    if (q->kpad != round_up(q->k, kKAlign)) return UFP4_ERR_INVALID_ARG;
    if (q->scale_ld < q->rows || q->scale_ld % kScaleLdAlign != 0) return UFP4_ERR_INVALID_ARG;
    if (q->rows > 0 && q->kpad > 0) {
        if (q->codes == nullptr || q->scales == nullptr) return UFP4_ERR_INVALID_ARG;
        if (!aligned16(q->codes) || !aligned16(q->scales)) return UFP4_ERR_ALIGNMENT;
    }
    if (q->cfg.scale_fmt == UFP4_SCALE_E4M3_X_FP32 && q->tensor_scale == nullptr)
        return UFP4_ERR_INVALID_ARG;
    if (q->corr != nullptr) {   // E1M2 correction plane: same layout as codes
        if (q->cfg.grid != UFP4_GRID_E1M2) return UFP4_ERR_INVALID_ARG;
        if (!aligned16(q->corr)) return UFP4_ERR_ALIGNMENT;
    }
    if (q->elems8 != nullptr) {   // E4M3 element plane of an MX (UE8M0) E1M2 operand
        if (q->cfg.grid != UFP4_GRID_E1M2 || q->cfg.scale_fmt != UFP4_SCALE_UE8M0) return UFP4_ERR_INVALID_ARG;
        if (!aligned16(q->elems8)) return UFP4_ERR_ALIGNMENT;
    }
    if (q->sf_atoms != nullptr) {   // factor atoms: byte block scales only
        if (atom_slot(q->cfg) == 0) return UFP4_ERR_INVALID_ARG;
        if (!aligned16(q->sf_atoms)) return UFP4_ERR_ALIGNMENT;
    }
    if (q->sf_lanes != nullptr) {   // per-lane factor tiles: E1M2 with E4M3 factors only
        if (!has_lane_tiles(q->cfg)) return UFP4_ERR_INVALID_ARG;
        if (!aligned16(q->sf_lanes)) return UFP4_ERR_ALIGNMENT;
    }
    if (q->rows > (int64_t(1) << 31) || q->kpad > (int64_t(1) << 31)) return UFP4_ERR_UNSUPPORTED;
    return UFP4_OK;
}

// D agrees on its n positions (mask bits beyond n are unused).
bool same_signs(uint64_t x, uint64_t y, int n) {
    const uint64_t m = n == 64 ? ~uint64_t(0) : ((uint64_t(1) << n) - 1);
    return (x & m) == (y & m);
}

ufp4_status_t check_pair(const ufp4_qtensor_t *a, const ufp4_qtensor_t *b, bool same_k) {
    ufp4_status_t s = check_qtensor(a);
    if (s != UFP4_OK) return s;
    s = check_qtensor(b);
    if (s != UFP4_OK) return s;
    const ufp4_quant_cfg_t &x = a->cfg, &y = b->cfg;
    if (x.grid != y.grid || x.block != y.block || x.scale_fmt != y.scale_fmt ||
        x.hadamard_n != y.hadamard_n)
        return UFP4_ERR_OPERAND_MISMATCH;
    if (x.hadamard_n > 0 && !same_signs(x.rht_sign_mask, y.rht_sign_mask, x.hadamard_n))
        return UFP4_ERR_OPERAND_MISMATCH;
    if (same_k && (a->k != b->k || a->kpad != b->kpad)) return UFP4_ERR_OPERAND_MISMATCH;
    return UFP4_OK;
}

std::atomic<int32_t> g_two_level_path{UFP4_GEMM_PATH_AUTO};

ufp4_status_t encode_operand_maps(const ufp4_qtensor_t *q, int code_rows, int scale_rows, int mode, int k_stage,
                                  CUtensorMap *codes, CUtensorMap *scales) {
    const int64_t rows_t = q->rows > 0 ? q->rows : 1;
    // Code rows of k_stage / 2 bytes per pipeline stage, swizzled by their
    // width: the fp32-scale kernel stages 64 K elements (32-byte rows), the
    // FP4 kernels 128 (64-byte rows) or 256 (128-byte rows).
    const uint32_t row_bytes = static_cast<uint32_t>(k_stage / 2);
    const CUtensorMapSwizzle swz = row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                   : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                     : CU_TENSOR_MAP_SWIZZLE_32B;
    CUresult r = encode_tensor_map_2d(codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, q->codes,
                                      static_cast<uint64_t>(q->kpad / 2),
                                      static_cast<uint64_t>(rows_t),
                                      static_cast<uint64_t>(q->kpad / 2), row_bytes,
                                      static_cast<uint32_t>(code_rows), swz);
    if (r != CUDA_SUCCESS) return UFP4_ERR_CUDA;
    const int nblk_stage = k_stage / q->cfg.block;
    const uint64_t nblk = static_cast<uint64_t>(q->kpad / q->cfg.block);
    if (mode != 0 || q->cfg.scale_fmt == UFP4_SCALE_UE8M0) {   // byte scales
        r = encode_tensor_map_2d(scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, q->scales,
                                 static_cast<uint64_t>(q->scale_ld), nblk,
                                 static_cast<uint64_t>(q->scale_ld), static_cast<uint32_t>(scale_rows),
                                 static_cast<uint32_t>(nblk_stage));
    } else {
        r = encode_tensor_map_2d(scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, q->scales,
                                 static_cast<uint64_t>(q->scale_ld), nblk,
                                 static_cast<uint64_t>(q->scale_ld) * 4,
                                 static_cast<uint32_t>(scale_rows), static_cast<uint32_t>(nblk_stage));
    }
    return r == CUDA_SUCCESS ? UFP4_OK : UFP4_ERR_CUDA;
}

ufp4_status_t run_gemm(const ufp4_qtensor_t *a, const ufp4_qtensor_t *b,
                       const ufp4_group_t *groups_dev, int32_t num_groups, float *c, int64_t ldc,
                       int64_t m, int64_t n, void *stream) {
    // Grouped problems pick their own K window of each operand (a_col, b_col,
    // k per group), so only the quantization settings must agree there.
    ufp4_status_t s = check_pair(a, b, groups_dev == nullptr);
    if (s != UFP4_OK) return s;
    if (c == nullptr && (m > 0 && n > 0)) return UFP4_ERR_INVALID_ARG;
    if (ldc < n || ldc < 1) return UFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(c) & 3u) != 0) return UFP4_ERR_ALIGNMENT;
    if (groups_dev != nullptr && (reinterpret_cast<uintptr_t>(groups_dev) & 7u))
        return UFP4_ERR_ALIGNMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // fp32 or UE8M0 block scales: per-block partials (mode 0).  Two-level
    // scales: the block-scaled FP4 kernel on CTA pairs with 256 x 256 tiles
    // (mode 5) or with one CTA per 128 x 192 tile (mode 3).  MX operands with
    // E4M3 element planes: the block-scaled FP8 kernel on CTA pairs (mode 6).
    int mode = 0;
    if (a->cfg.scale_fmt == UFP4_SCALE_E4M3_X_FP32) {
        // The CTA-pair kernel (mode 5) takes E1M2 operands whose correction
        // planes follow their codes in one allocation, and E2M1 operands.
        auto adjacent_planes = [](const ufp4_qtensor_t *q) {
            const uint64_t plane = static_cast<uint64_t>(q->rows) * static_cast<uint64_t>(q->kpad / 2);
            return q->rows > 0 && q->corr != nullptr &&
                   reinterpret_cast<uintptr_t>(q->corr) == reinterpret_cast<uintptr_t>(q->codes) + plane;
        };
        const bool pair_ok = a->cfg.grid != UFP4_GRID_E1M2 || (adjacent_planes(a) && adjacent_planes(b));
        mode = (g_two_level_path.load() == UFP4_GEMM_PATH_NATIVE_FP4 || !pair_ok) ? 3 : 5;
    }
    // MX operands that carry E4M3 element planes: the block-scaled FP8 MMA
    // on CTA pairs (mode 6); otherwise the fp32-block-scale kernel.
    if (a->cfg.scale_fmt == UFP4_SCALE_UE8M0 && a->cfg.grid == UFP4_GRID_E1M2 && a->elems8 != nullptr &&
        b->elems8 != nullptr)
        mode = 6;
    if (groups_dev == nullptr) {
        if (m == 0 || n == 0) return UFP4_OK;
        if (a->kpad == 0) {
            cudaError_t e = cudaMemset2DAsync(c, static_cast<size_t>(ldc) * 4, 0,
                                              static_cast<size_t>(n) * 4, static_cast<size_t>(m), st);
            return e == cudaSuccess ? UFP4_OK : UFP4_ERR_CUDA;
        }
    } else if (num_groups == 0 || a->kpad == 0 || a->rows == 0 || b->rows == 0) {
        return UFP4_OK;
    }
    if (encode_fn() == nullptr) return UFP4_ERR_CUDA;

    GemmArgs args;
    memset(&args, 0, sizeof(args));
    args.scale_ue8m0 = a->cfg.scale_fmt == UFP4_SCALE_UE8M0 ? 1 : 0;
    // B code rows staged per CTA: fp32-scale kernel 128, one-CTA FP4 kernel
    // 192, CTA-pair kernels 128 (with the scales of all 256 B rows of a tile
    // in each CTA).
    int bn = 128, bscale = 128;
    switch (mode) {
        case 3: bn = bscale = kNativeTileN; break;
        case 5:
        case 6: bn = 128; bscale = 256; break;
        default: bn = bscale = 128; break;
    }
    // Dense problems on the CTA-pair kernels whose operands both carry factor
    // atoms: each stage's atoms come with its code tiles and the MMA issuer
    // copies them into tensor memory.  Grouped problems keep the
    // factor-building warps (measured faster there: short K per tile, ragged
    // groups).
    const bool use_atoms = (mode == 5 || mode == 6) && groups_dev == nullptr && a->sf_atoms != nullptr &&
                           b->sf_atoms != nullptr && a->rows > 0 && b->rows > 0;
    // The restricted E2M1 grid stores E2M1 codes (0..4): the E2M1 kernels.
    const int grid_kind = a->cfg.grid == UFP4_GRID_E1M2 ? 0 : 1;
    // K elements per pipeline stage of the chosen kernel.
    const int k_stage = mode == 0 ? 64 : (mode == 5 ? pair_stage_k(grid_kind, use_atoms) : 128);
    s = encode_operand_maps(a, 128, 128, mode, k_stage, &args.tm_a_codes, &args.tm_a_scales);
    if (s != UFP4_OK) return s;
    s = encode_operand_maps(b, bn, bscale, mode, k_stage, &args.tm_b_codes, &args.tm_b_scales);
    if (s != UFP4_OK) return s;
    if (mode == 6) {   // E4M3 element planes: 128-byte rows (128 K per stage), 128-byte swizzle
        const int64_t ra = a->rows > 0 ? a->rows : 1, rb = b->rows > 0 ? b->rows : 1;
        CUresult r = encode_tensor_map_2d(&args.tm_a_e8, CU_TENSOR_MAP_DATA_TYPE_UINT8, a->elems8,
                                          static_cast<uint64_t>(a->kpad), static_cast<uint64_t>(ra),
                                          static_cast<uint64_t>(a->kpad), 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
        if (r != CUDA_SUCCESS) return UFP4_ERR_CUDA;
        r = encode_tensor_map_2d(&args.tm_b_e8, CU_TENSOR_MAP_DATA_TYPE_UINT8, b->elems8,
                                 static_cast<uint64_t>(b->kpad), static_cast<uint64_t>(rb),
                                 static_cast<uint64_t>(b->kpad), 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
        if (r != CUDA_SUCCESS) return UFP4_ERR_CUDA;
    }
    args.a_S = a->tensor_scale;
    args.b_S = b->tensor_scale;
    args.c = c;
    args.ldc = ldc;
    args.inv_n = a->cfg.hadamard_n > 0 ? 1.0f / static_cast<float>(a->cfg.hadamard_n) : 1.0f;
    args.block = a->cfg.block;
    args.groups = reinterpret_cast<const GemmGroup *>(groups_dev);
    args.num_groups = num_groups;
    args.single.m = m;
    args.single.n = n;
    args.single.k = a->kpad;
    // E1M2 operands that carry correction planes: the native kernels load
    // them with the codes (same box, same swizzle).
    if (mode >= 3 && a->cfg.grid == UFP4_GRID_E1M2 && a->corr != nullptr && b->corr != nullptr) {
        // When each operand's plane follows its codes in one allocation
        // ([2][rows][kpad/2]), one 3-D box per operand fetches both.
        auto adjacent = [](const ufp4_qtensor_t *q) {
            const uint64_t plane = static_cast<uint64_t>(q->rows) * static_cast<uint64_t>(q->kpad / 2);
            return q->rows > 0 && reinterpret_cast<uintptr_t>(q->corr) ==
                                      reinterpret_cast<uintptr_t>(q->codes) + plane;
        };
        if (adjacent(a) && adjacent(b)) {
            const uint64_t pa = static_cast<uint64_t>(a->rows) * static_cast<uint64_t>(a->kpad / 2);
            const uint64_t pb = static_cast<uint64_t>(b->rows) * static_cast<uint64_t>(b->kpad / 2);
            CUresult r = encode_tensor_map_planes(&args.tm_a_corr, a->codes, static_cast<uint64_t>(a->kpad / 2),
                                                  static_cast<uint64_t>(a->rows), 2, pa, 64, 128,
                                                  CU_TENSOR_MAP_SWIZZLE_64B);
            if (r != CUDA_SUCCESS) return UFP4_ERR_CUDA;
            r = encode_tensor_map_planes(&args.tm_b_corr, b->codes, static_cast<uint64_t>(b->kpad / 2),
                                         static_cast<uint64_t>(b->rows), 2, pb, 64, static_cast<uint32_t>(bn),
                                         CU_TENSOR_MAP_SWIZZLE_64B);
            if (r != CUDA_SUCCESS) return UFP4_ERR_CUDA;
            args.planes3d = 1;
        } else {
            ufp4_qtensor_t ac = *a, bc = *b;
            ac.codes = a->corr;
            bc.codes = b->corr;
            CUtensorMap scratch;
            s = encode_operand_maps(&ac, 128, 128, mode, k_stage, &args.tm_a_corr, &scratch);
            if (s != UFP4_OK) return s;
            s = encode_operand_maps(&bc, bn, bscale, mode, k_stage, &args.tm_b_corr, &scratch);
            if (s != UFP4_OK) return s;
        }
        args.corr_in = 1;
    }
    // Factor atoms: one u64 box of a stage's K elements per 128-row group
    // (k_stage / 64 atoms of E4M3 factors, k_stage / 128 of UE8M0).
    if (use_atoms) {
        const int64_t ak = atoms_k_of(a->kpad, a->cfg), bk = atoms_k_of(b->kpad, b->cfg);
        const uint32_t box_k = static_cast<uint32_t>(64 * (k_stage / (4 * atom_slot(a->cfg))));
        CUresult r;
        if (mode == 5 && grid_kind == 0 && a->sf_lanes != nullptr) {
            // E1M2 with per-lane tiles on A: one 4 KB box per 128 rows and
            // 128 K, u64 [tiles][2 halves][256]
            const int64_t sg = lane_groups_of(a->kpad);
            const uint8_t *base = static_cast<const uint8_t *>(a->sf_lanes);
            const cuuint64_t dims[3] = {256, 2, static_cast<cuuint64_t>((a->rows + 127) / 128 * sg)};
            const cuuint64_t strides[2] = {2048, kLaneTileBytes};
            const cuuint32_t box[3] = {256, 2, 1};
            r = encode_tensor_map_3d(&args.tm_a_atoms, CU_TENSOR_MAP_DATA_TYPE_UINT64, base, dims, strides, box);
            args.lane_groups = static_cast<int32_t>(sg);
            args.lanes = 1;
        } else {
            r = encode_tensor_map_2d(&args.tm_a_atoms, CU_TENSOR_MAP_DATA_TYPE_UINT64, a->sf_atoms,
                                     static_cast<uint64_t>(64 * ak), static_cast<uint64_t>((a->rows + 127) / 128),
                                     static_cast<uint64_t>(ak) * 512, box_k, 1, CU_TENSOR_MAP_SWIZZLE_NONE);
        }
        if (r != CUDA_SUCCESS) return UFP4_ERR_CUDA;
        r = encode_tensor_map_2d(&args.tm_b_atoms, CU_TENSOR_MAP_DATA_TYPE_UINT64, b->sf_atoms,
                                 static_cast<uint64_t>(64 * bk), static_cast<uint64_t>((b->rows + 127) / 128),
                                 static_cast<uint64_t>(bk) * 512, box_k, 2, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (r != CUDA_SUCCESS) return UFP4_ERR_CUDA;
        args.atoms = 1;
    }
    // Tile order: bands of 8 rows of tiles (measured on the large layer's
    // step at the power cap: 1030 against 953 TFLOP/s for M-fastest order,
    // SM clock 1965 against 1650 MHz, from the HBM traffic saved).
    args.band = kTileBand;
    // Native kernels store 16-byte pieces when the output allows it.
    args.c_vec = (aligned16(c) && ldc % 4 == 0) ? 1 : 0;
    cudaError_t e = launch_gemm(args, mode, grid_kind, sm_count(), st);
    return e == cudaSuccess ? UFP4_OK : UFP4_ERR_CUDA;
}

ufp4_status_t check_input(const void *x, int64_t rows, int64_t cols, int64_t ld, int32_t axis) {
    if (rows < 0 || cols < 0) return UFP4_ERR_INVALID_ARG;
    if (axis != UFP4_ALONG_COLS && axis != UFP4_ALONG_ROWS) return UFP4_ERR_INVALID_ARG;
    if (rows > 0 && cols > 0) {
        if (x == nullptr) return UFP4_ERR_INVALID_ARG;
        if (ld < cols) return UFP4_ERR_INVALID_ARG;
        if (!aligned16(x) || ld % 8 != 0 || cols % 8 != 0) return UFP4_ERR_ALIGNMENT;
    }
    return UFP4_OK;
}

// Validates `out` against the input shape and fills the kernel arguments of
// one quantization (x along `axis`).
ufp4_status_t fill_quant_args(const void *x_dev, int64_t rows, int64_t cols, int64_t ld, int32_t axis,
                              const float *tensor_amax_dev, const ufp4_qtensor_t *out, QuantArgs *a) {
    ufp4_status_t s = check_qtensor(out);
    if (s != UFP4_OK) return s;
    const int64_t out_rows = axis == UFP4_ALONG_COLS ? rows : cols;
    const int64_t K = axis == UFP4_ALONG_COLS ? cols : rows;
    if (out->rows != out_rows || out->k != K) return UFP4_ERR_INVALID_ARG;
    const bool two_level = out->cfg.scale_fmt == UFP4_SCALE_E4M3_X_FP32;
    if (two_level && tensor_amax_dev == nullptr) return UFP4_ERR_INVALID_ARG;
    memset(a, 0, sizeof(*a));
    a->x = static_cast<const uint16_t *>(x_dev);
    a->rows = rows;
    a->cols = cols;
    a->ld = ld;
    a->axis = axis;
    a->out_rows = out_rows;
    a->K = K;
    a->kpad = out->kpad;
    a->scale_ld = out->scale_ld;
    a->codes = static_cast<uint8_t *>(out->codes);
    a->corr = static_cast<uint8_t *>(out->corr);
    a->elems8 = static_cast<uint8_t *>(out->elems8);
    a->sf_atoms = static_cast<uint8_t *>(out->sf_atoms);
    a->atoms_k = out->sf_atoms != nullptr ? atoms_k_of(out->kpad, out->cfg) : 0;
    if (out->sf_lanes != nullptr) {
        a->sf_lanes = static_cast<uint8_t *>(out->sf_lanes);
        a->lane_groups = lane_groups_of(out->kpad);
    }
    a->scales = out->scales;
    a->S_out = two_level ? out->tensor_scale : nullptr;
    a->amax_t = two_level ? tensor_amax_dev : nullptr;
    a->seed = out->cfg.sr_seed;
    a->stream = out->cfg.sr_stream;
    a->sign_mask = out->cfg.rht_sign_mask;
    a->scale_fmt = out->cfg.scale_fmt;
    return UFP4_OK;
}

}  // namespace

CUresult encode_tensor_map_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base,
                              uint64_t inner, uint64_t outer, uint64_t row_bytes,
                              uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (fn == nullptr) return CUDA_ERROR_NOT_INITIALIZED;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estride[2] = {1, 1};
    return fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estride,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

CUresult encode_tensor_map_3d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base,
                              const cuuint64_t (&dims)[3], const cuuint64_t (&strides)[2],
                              const cuuint32_t (&box)[3]) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (fn == nullptr) return CUDA_ERROR_NOT_INITIALIZED;
    const cuuint32_t estride[3] = {1, 1, 1};
    return fn(map, dtype, 3, const_cast<void *>(base), dims, strides, box, estride,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

CUresult encode_tensor_map_planes(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                                  uint64_t planes, uint64_t plane_bytes, uint32_t box_inner,
                                  uint32_t box_outer, CUtensorMapSwizzle swizzle) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (fn == nullptr) return CUDA_ERROR_NOT_INITIALIZED;
    const cuuint64_t dims[3] = {inner, outer, planes};
    const cuuint64_t strides[2] = {inner, plane_bytes};
    const cuuint32_t box[3] = {box_inner, box_outer, static_cast<cuuint32_t>(planes)};
    const cuuint32_t estride[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estride,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

}  // namespace ufp4

using namespace ufp4;

extern "C" {

int32_t ufp4_version(void) { return 100; }

const char *ufp4_status_string(ufp4_status_t s) {
    switch (s) {
        case UFP4_OK: return "UFP4_OK";
        case UFP4_ERR_INVALID_ARG: return "UFP4_ERR_INVALID_ARG";
        case UFP4_ERR_UNSUPPORTED: return "UFP4_ERR_UNSUPPORTED";
        case UFP4_ERR_ALIGNMENT: return "UFP4_ERR_ALIGNMENT";
        case UFP4_ERR_OPERAND_MISMATCH: return "UFP4_ERR_OPERAND_MISMATCH";
        case UFP4_ERR_CUDA: return "UFP4_ERR_CUDA";
        case UFP4_ERR_DEVICE_TIMEOUT: return "UFP4_ERR_DEVICE_TIMEOUT";
    }
    return "UFP4_ERR_UNKNOWN";
}

ufp4_status_t ufp4_qtensor_layout(int64_t rows, int64_t k, const ufp4_quant_cfg_t *cfg,
                                  int64_t *kpad, int64_t *scale_ld, size_t *codes_bytes,
                                  size_t *scales_bytes) {
    if (cfg == nullptr || rows < 0 || k < 0 || !cfg_valid(*cfg)) return UFP4_ERR_INVALID_ARG;
    const int64_t kp = round_up(k, kKAlign);
    const int64_t sl = round_up(rows > 0 ? rows : 1, kScaleLdAlign);
    const int64_t elt = cfg->scale_fmt == UFP4_SCALE_FP32 ? 4 : 1;
    if (kpad) *kpad = kp;
    if (scale_ld) *scale_ld = sl;
    if (codes_bytes) *codes_bytes = static_cast<size_t>(rows * (kp / 2));
    if (scales_bytes) *scales_bytes = static_cast<size_t>((kp / cfg->block) * sl * elt);
    return UFP4_OK;
}

ufp4_status_t ufp4_sf_atoms_layout(int64_t rows, int64_t k, const ufp4_quant_cfg_t *cfg, int64_t *atoms_k,
                                   size_t *bytes) {
    if (cfg == nullptr || rows < 0 || k < 0 || !cfg_valid(*cfg)) return UFP4_ERR_INVALID_ARG;
    if (atom_slot(*cfg) == 0) return UFP4_ERR_UNSUPPORTED;
    const int64_t ak = atoms_k_of(round_up(k, kKAlign), *cfg);
    if (atoms_k) *atoms_k = ak;
    if (bytes) *bytes = static_cast<size_t>(atom_bytes_of(rows, round_up(k, kKAlign), *cfg));
    return UFP4_OK;
}

ufp4_status_t ufp4_sf_lanes_layout(int64_t rows, int64_t k, const ufp4_quant_cfg_t *cfg, size_t *bytes) {
    if (cfg == nullptr || bytes == nullptr || rows < 0 || k < 0 || !cfg_valid(*cfg)) return UFP4_ERR_INVALID_ARG;
    if (!has_lane_tiles(*cfg)) return UFP4_ERR_UNSUPPORTED;
    *bytes = static_cast<size_t>((rows + 127) / 128 * lane_groups_of(round_up(k, kKAlign)) * kLaneTileBytes);
    return UFP4_OK;
}

ufp4_status_t ufp4_rht_amax(const void *x_dev, int64_t rows, int64_t cols, int64_t ld,
                            int32_t axis, int32_t hadamard_n, uint64_t rht_sign_mask,
                            float *amax_dev, void *stream) {
    ufp4_status_t s = check_input(x_dev, rows, cols, ld, axis);
    if (s != UFP4_OK) return s;
    if (amax_dev == nullptr) return UFP4_ERR_INVALID_ARG;
    if (!(hadamard_n == 0 || hadamard_n == 16 || hadamard_n == 32 || hadamard_n == 64))
        return UFP4_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    QuantArgs a;
    memset(&a, 0, sizeof(a));
    a.x = static_cast<const uint16_t *>(x_dev);
    a.rows = rows;
    a.cols = cols;
    a.ld = ld;
    a.axis = axis;
    a.out_rows = axis == UFP4_ALONG_COLS ? rows : cols;
    a.K = axis == UFP4_ALONG_COLS ? cols : rows;
    a.kpad = round_up(a.K, kKAlign);
    a.amax_out = amax_dev;
    a.sign_mask = rht_sign_mask;
    if (a.out_rows == 0 || a.kpad == 0) {
        return cudaMemsetAsync(amax_dev, 0, sizeof(float), st) == cudaSuccess ? UFP4_OK : UFP4_ERR_CUDA;
    }
    cudaError_t e = launch_rht_amax(a, hadamard_n, sm_count(), st);
    return e == cudaSuccess ? UFP4_OK : UFP4_ERR_CUDA;
}

ufp4_status_t ufp4_rht_bf16(const void *x_dev, int64_t rows, int64_t cols, int64_t ld, int32_t hadamard_n,
                            uint64_t rht_sign_mask, void *y_dev, int64_t ldy, void *stream) {
    ufp4_status_t s = check_input(x_dev, rows, cols, ld, UFP4_ALONG_COLS);
    if (s != UFP4_OK) return s;
    if (!(hadamard_n == 0 || hadamard_n == 16 || hadamard_n == 32 || hadamard_n == 64))
        return UFP4_ERR_UNSUPPORTED;
    if (cols % 64 != 0) return UFP4_ERR_UNSUPPORTED;
    if (rows > 0 && cols > 0) {
        if (y_dev == nullptr) return UFP4_ERR_INVALID_ARG;
        if (ldy < cols) return UFP4_ERR_INVALID_ARG;
        if (!aligned16(y_dev) || ldy % 8 != 0) return UFP4_ERR_ALIGNMENT;
        if ((ld % 8) != 0) return UFP4_ERR_ALIGNMENT;
    }
    if (rows == 0 || cols == 0) return UFP4_OK;
    QuantArgs a;
    memset(&a, 0, sizeof(a));
    a.x = static_cast<const uint16_t *>(x_dev);
    a.rows = rows;
    a.cols = cols;
    a.ld = ld;
    a.sign_mask = rht_sign_mask;
    cudaError_t e = launch_rht_bf16(a, hadamard_n, static_cast<uint16_t *>(y_dev), ldy, sm_count(),
                                    static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? UFP4_OK : UFP4_ERR_CUDA;
}

ufp4_status_t ufp4_rht_quantize(const void *x_dev, int64_t rows, int64_t cols, int64_t ld,
                                int32_t axis, const float *tensor_amax_dev, ufp4_qtensor_t *out,
                                void *stream) {
    ufp4_status_t s = check_input(x_dev, rows, cols, ld, axis);
    if (s != UFP4_OK) return s;
    QuantArgs a;
    s = fill_quant_args(x_dev, rows, cols, ld, axis, tensor_amax_dev, out, &a);
    if (s != UFP4_OK) return s;
    if (a.out_rows == 0 || a.kpad == 0) return UFP4_OK;
    cudaError_t e = launch_rht_quantize(a, out->cfg.hadamard_n, out->cfg.block, out->cfg.grid,
                                        out->cfg.rounding, sm_count(),
                                        static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? UFP4_OK : UFP4_ERR_CUDA;
}

ufp4_status_t ufp4_rht_amax_dual(const void *x_dev, int64_t rows, int64_t cols, int64_t ld,
                                 int32_t hadamard_n, uint64_t rht_sign_mask, float *amax_cols_dev,
                                 float *amax_rows_dev, void *stream) {
    ufp4_status_t s = check_input(x_dev, rows, cols, ld, UFP4_ALONG_COLS);
    if (s != UFP4_OK) return s;
    if (amax_cols_dev == nullptr || amax_rows_dev == nullptr) return UFP4_ERR_INVALID_ARG;
    if (!(hadamard_n == 0 || hadamard_n == 16 || hadamard_n == 32 || hadamard_n == 64))
        return UFP4_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (rows == 0 || cols == 0) {
        if (cudaMemsetAsync(amax_cols_dev, 0, sizeof(float), st) != cudaSuccess ||
            cudaMemsetAsync(amax_rows_dev, 0, sizeof(float), st) != cudaSuccess)
            return UFP4_ERR_CUDA;
        return UFP4_OK;
    }
    QuantArgs ar, ac;
    memset(&ar, 0, sizeof(ar));
    ar.x = static_cast<const uint16_t *>(x_dev);
    ar.rows = rows;
    ar.cols = cols;
    ar.ld = ld;
    ar.sign_mask = rht_sign_mask;
    ac = ar;
    ar.axis = UFP4_ALONG_ROWS;
    ar.out_rows = cols;
    ar.K = rows;
    ar.kpad = round_up(rows, kKAlign);
    ar.amax_out = amax_rows_dev;
    ac.axis = UFP4_ALONG_COLS;
    ac.out_rows = rows;
    ac.K = cols;
    ac.kpad = round_up(cols, kKAlign);
    ac.amax_out = amax_cols_dev;
    cudaError_t e = launch_rht_amax_dual(ar, ac, hadamard_n, sm_count(), st);
    return e == cudaSuccess ? UFP4_OK : UFP4_ERR_CUDA;
}

ufp4_status_t ufp4_rht_quantize_dual(const void *x_dev, int64_t rows, int64_t cols, int64_t ld,
                                     const float *tensor_amax_cols_dev,
                                     const float *tensor_amax_rows_dev, ufp4_qtensor_t *out_cols,
                                     ufp4_qtensor_t *out_rows, void *stream) {
    ufp4_status_t s = check_input(x_dev, rows, cols, ld, UFP4_ALONG_COLS);
    if (s != UFP4_OK) return s;
    QuantArgs ac, ar;
    s = fill_quant_args(x_dev, rows, cols, ld, UFP4_ALONG_COLS, tensor_amax_cols_dev, out_cols, &ac);
    if (s != UFP4_OK) return s;
    s = fill_quant_args(x_dev, rows, cols, ld, UFP4_ALONG_ROWS, tensor_amax_rows_dev, out_rows, &ar);
    if (s != UFP4_OK) return s;
    // One kernel computes both: the same recipe on both sides, except the
    // SR stream (DGRAD and WGRAD draw independent bits from one tensor).
    const ufp4_quant_cfg_t &c = out_cols->cfg, &r = out_rows->cfg;
    if (c.grid != r.grid || c.rounding != r.rounding || c.hadamard_n != r.hadamard_n ||
        c.block != r.block || c.scale_fmt != r.scale_fmt || c.sr_seed != r.sr_seed ||
        (c.hadamard_n > 0 && !same_signs(c.rht_sign_mask, r.rht_sign_mask, c.hadamard_n)))
        return UFP4_ERR_UNSUPPORTED;
    if (rows == 0 || cols == 0) return UFP4_OK;
    cudaError_t e = launch_rht_quantize_dual(ar, ac, c.hadamard_n, c.block, c.grid, c.rounding, sm_count(),
                                             static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? UFP4_OK : UFP4_ERR_CUDA;
}

ufp4_status_t ufp4_quant_stats(const void *x_dev, int64_t rows, int64_t cols, int64_t ld,
                               int32_t axis, const ufp4_qtensor_t *q, ufp4_qstats_t *stats_dev,
                               void *stream) {
    ufp4_status_t s = check_input(x_dev, rows, cols, ld, axis);
    if (s != UFP4_OK) return s;
    s = check_qtensor(q);
    if (s != UFP4_OK) return s;
    if (stats_dev == nullptr) return UFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(stats_dev) & 7u) != 0) return UFP4_ERR_ALIGNMENT;
    const int64_t out_rows = axis == UFP4_ALONG_COLS ? rows : cols;
    const int64_t K = axis == UFP4_ALONG_COLS ? cols : rows;
    if (q->rows != out_rows || q->k != K) return UFP4_ERR_INVALID_ARG;
    DiagArgs a;
    memset(&a, 0, sizeof(a));
    a.x = static_cast<const uint16_t *>(x_dev);
    a.rows = rows;
    a.cols = cols;
    a.ld = ld;
    a.axis = axis;
    a.out_rows = out_rows;
    a.K = K;
    a.kpad = q->kpad;
    a.scale_ld = q->scale_ld;
    a.codes = static_cast<const uint8_t *>(q->codes);
    a.scales = q->scales;
    a.S = q->tensor_scale;
    a.scale_fmt = q->cfg.scale_fmt;
    a.grid = q->cfg.grid == UFP4_GRID_E1M2 ? 0 : 1;   // level table: E1M2 or E2M1 codes
    a.block = q->cfg.block;
    a.sign_mask = q->cfg.rht_sign_mask;
    a.out = stats_dev;
    cudaError_t e = launch_quant_stats(a, q->cfg.hadamard_n, sm_count(), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? UFP4_OK : UFP4_ERR_CUDA;
}

ufp4_status_t ufp4_qstats_summarize(const ufp4_qstats_t *st, int32_t grid, ufp4_qstats_summary_t *out) {
    if (st == nullptr || out == nullptr) return UFP4_ERR_INVALID_ARG;
    if (grid != UFP4_GRID_E1M2 && grid != UFP4_GRID_E2M1 && grid != UFP4_GRID_E2M1_MAX2)
        return UFP4_ERR_INVALID_ARG;
    out->sqnr_db = st->noise > 0.0 ? 10.0 * log10(st->signal / st->noise) : HUGE_VAL;
    uint64_t total = 0;
    for (int c = 0; c < 16; ++c) total += st->code_count[c];
    int occupied = 0;
    for (int c = 0; c < 16; ++c)
        if (total > 0 && st->code_count[c] * 240.0 > static_cast<double>(total)) ++occupied;
    const int grid_codes = grid == UFP4_GRID_E2M1_MAX2 ? 9 : 15;
    out->bucket_ratio = static_cast<double>(occupied) / grid_codes;
    out->underflow_ratio = st->nonzero ? static_cast<double>(st->underflow) / st->nonzero : 0.0;
    for (int k = 0; k < 8; ++k)
        out->level_mean_err[k] = st->level_n[k] ? st->level_err[k] / st->level_n[k] : NAN;
    return UFP4_OK;
}

ufp4_status_t ufp4_sqnr_sums(const float *ref_dev, int64_t ld_ref, const float *test_dev,
                             int64_t ld_test, int64_t rows, int64_t cols, double *sums_dev,
                             void *stream) {
    if (rows < 0 || cols < 0 || sums_dev == nullptr) return UFP4_ERR_INVALID_ARG;
    if (rows > 0 && cols > 0 && (ref_dev == nullptr || test_dev == nullptr || ld_ref < cols || ld_test < cols))
        return UFP4_ERR_INVALID_ARG;
    cudaError_t e = launch_sqnr_sums(ref_dev, ld_ref, test_dev, ld_test, rows, cols, sums_dev, sm_count(),
                                     static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? UFP4_OK : UFP4_ERR_CUDA;
}

ufp4_status_t ufp4_gemm_fprop(const ufp4_qtensor_t *xq, const ufp4_qtensor_t *wq, float *y_dev,
                              int64_t ldy, void *stream) {
    if (xq == nullptr || wq == nullptr) return UFP4_ERR_INVALID_ARG;
    return run_gemm(xq, wq, nullptr, 0, y_dev, ldy, xq->rows, wq->rows, stream);
}

ufp4_status_t ufp4_gemm_dgrad(const ufp4_qtensor_t *dyq, const ufp4_qtensor_t *wtq, float *dx_dev,
                              int64_t lddx, void *stream) {
    if (dyq == nullptr || wtq == nullptr) return UFP4_ERR_INVALID_ARG;
    return run_gemm(dyq, wtq, nullptr, 0, dx_dev, lddx, dyq->rows, wtq->rows, stream);
}

ufp4_status_t ufp4_gemm_wgrad(const ufp4_qtensor_t *dytq, const ufp4_qtensor_t *xtq,
                              float *dw_dev, int64_t lddw, void *stream) {
    if (dytq == nullptr || xtq == nullptr) return UFP4_ERR_INVALID_ARG;
    return run_gemm(dytq, xtq, nullptr, 0, dw_dev, lddw, dytq->rows, xtq->rows, stream);
}

ufp4_status_t ufp4_grouped_gemm(const ufp4_qtensor_t *a, const ufp4_qtensor_t *b,
                                const ufp4_group_t *groups_dev, int32_t num_groups, float *c_dev,
                                int64_t ldc, void *stream) {
    if (a == nullptr || b == nullptr || num_groups < 0) return UFP4_ERR_INVALID_ARG;
    if (num_groups > 0 && groups_dev == nullptr) return UFP4_ERR_INVALID_ARG;
    if (num_groups == 0) return UFP4_OK;
    if (c_dev == nullptr) return UFP4_ERR_INVALID_ARG;
    return run_gemm(a, b, groups_dev, num_groups, c_dev, ldc, 0, 0, stream);
}

ufp4_status_t ufp4_set_two_level_gemm_path(int32_t path) {
    if (path != UFP4_GEMM_PATH_AUTO && path != UFP4_GEMM_PATH_NATIVE_FP4 && path != UFP4_GEMM_PATH_NATIVE_FP4_PAIR256)
        return UFP4_ERR_INVALID_ARG;
    g_two_level_path.store(path);
    return UFP4_OK;
}

int32_t ufp4_get_two_level_gemm_path(void) { return g_two_level_path.load(); }

ufp4_status_t ufp4_test_set_quantize_wait_limit(uint64_t limit_ns) {
    return quantize_set_producer_wait_limit(limit_ns) == cudaSuccess ? UFP4_OK : UFP4_ERR_CUDA;
}

ufp4_status_t ufp4_check_device_status(void) {
    uint32_t w = 0;
    if (read_and_clear_error_word(&w) != cudaSuccess) return UFP4_ERR_CUDA;
    uint32_t wq = 0;
    if (quantize_read_and_clear_error_word(&wq) != cudaSuccess) return UFP4_ERR_CUDA;
    w |= wq;
    return w == 0 ? UFP4_OK : UFP4_ERR_DEVICE_TIMEOUT;
}

}  // extern "C"
