/*
 * ufp4.h -- C ABI of libufp4.so: the data-parallel hot path of the UFP4
 * 4-bit training recipe on NVIDIA B200 (sm_100a).
 *
 * Method: arXiv 2606.20381, "Rethinking Shrinkage Bias in LLM FP4 Pretraining:
 * Geometric Origin, Systemic Impact, and UFP4 Recipe".  Citations name the
 * paperlayer.ai per-section summary of the paper as [PL], the gist.science
 * technical summary as [GS] and the author's dreamwings.cn post as [DW].
 *
 * What the library computes ([PL] §2 Preliminaries, §4 UFP4):
 *   1. ufp4_rht_quantize: for each row of an operand's K-major view (K = the
 *      GEMM's reduction dimension), apply a random sign diagonal D and an
 *      unnormalised Sylvester Hadamard H_n per n-block, take the absolute
 *      maximum of each scale block, derive the block scale, round every
 *      element to the 4-bit grid (RTNE, or stochastic rounding from a
 *      Philox4x32-10 stream) and pack two codes per byte.
 *   2. ufp4_gemm_{fprop,dgrad,wgrad}: C[i][j] = (1/n) sum_k A[i][k] B[j][k]
 *      over the dequantized operands, fp32 accumulation, fp32 output.
 *   3. ufp4_grouped_gemm: the same contraction for a table of independent
 *      sub-problems (mixture-of-experts layers).
 *   4. ufp4_rht_quantize_dual / ufp4_rht_amax_dual: both quantizations (both
 *      rotated amaxes) of one tensor from a single read of it.
 *   5. ufp4_quant_stats / ufp4_qstats_summarize / ufp4_sqnr_sums: the
 *      quantization diagnostics of [PL] §5 and Appendix A (SQNR, level error,
 *      code occupancy, underflow).
 *
 * Conventions shared by every call:
 *   - All pointers named *_dev, and every pointer inside ufp4_qtensor_t, are
 *     device pointers owned by the caller.  The library never allocates,
 *     frees or synchronises; work is enqueued on `stream` (a cudaStream_t
 *     passed as void*; NULL = legacy default stream) and returns at once.
 *   - Arguments are validated on the host before any launch; a failed check
 *     returns an error status and enqueues nothing.
 *   - Inputs are assumed finite; NaN/Inf inputs give unspecified codes.
 *   - Outputs are overwritten (no accumulation into C).
 *
 * Quantized operand layout (ufp4_qtensor_t), for `rows` output rows and
 * reduction length `k`:
 *   kpad      = k rounded up to a multiple of 64; positions >= k hold zeros.
 *   codes     u8 [rows][kpad/2], row-major.  Byte j of a row holds element 2j
 *             in its low nibble and element 2j+1 in its high nibble.  A nibble
 *             is sign-magnitude: bit 3 = sign, bits 0..2 = magnitude index k
 *             of the grid (E1M2: k/4; E2M1: {0,.5,1,1.5,2,3,4,6}[k]; the
 *             restricted E2M1 grid uses k <= 4 of the E2M1 list).  Zero is
 *             always 0x0, never 0x8.
 *   scales    block-major: entry (row r, block b) at scales[b*scale_ld + r],
 *             scale_ld = rows rounded up to a multiple of 64.
 *             UFP4_SCALE_FP32:         fp32, s = RN(amax_b / gmax).
 *             UFP4_SCALE_E4M3_X_FP32:  u8 OCP E4M3 e_b; the step of the block
 *                                      is e_b * S with S = *tensor_scale.
 *             UFP4_SCALE_UE8M0:        u8 biased exponent E; the step of the
 *                                      block is 2^(E - 127) (tensor_scale
 *                                      unused); GEMMs run the block-scaled
 *                                      FP8 MMA when both operands carry an
 *                                      elems8 plane, else the fp32-scale kernel.
 *   The dequantized (rotated) value of element (r, t) is s * lvl(code); the
 *   Hadamard normalisation 1/n is applied once in the GEMM (n = 0: none).
 *   corr      optional, E1M2 only: the same layout as codes, each nibble the
 *             E2M1 code of d(k) = k - e(k), where e(k) is the code's bits read
 *             as an E2M1 number (d = {0,.5,1,1.5,2,2,2,1}[k] as E2M1 codes
 *             {0,1,2,3,4,4,4,2}, sign bit copied).  k = e(k) + d(k) exactly,
 *             so the block-scaled FP4 GEMM multiplies E1M2 operands as two
 *             E2M1 planes.  ufp4_rht_quantize writes it when non-NULL; the
 *             GEMMs read it when both operands carry one (else they derive it
 *             on the fly).  Must be NULL for E2M1 operands.
 *   elems8    optional, E1M2 with UE8M0 scales only (the MX path): u8
 *             [rows][kpad], byte t of a row the OCP E4M3 encoding of element
 *             t's grid value +-k/4 (0x00 for zero; magnitudes 0x28, 0x30,
 *             0x34, 0x38, 0x3A, 0x3C, 0x3E for k = 1..7; sign in bit 7), an
 *             exact remap of the code.  ufp4_rht_quantize writes it when
 *             non-NULL; when both GEMM operands carry one, the GEMM runs on the
 *             block-scaled FP8 MMA with the UE8M0 factors applied in the MMA
 *             (else on the fp32-scale kernel).  Must be NULL otherwise.
 *   sf_atoms  optional, byte block scales only (E4M3 x fp32 or UE8M0): the
 *             same factors again, in the layout the block-scaled tensor-core
 *             MMA reads its scale factors from (a copy per 32-lane quarter of
 *             tensor memory; a hardware layout, not part of the method).  Factors are
 *             per "slot" of W elements along K: W = 16 for E4M3 factors
 *             (a block-32 factor fills both of its slots), W = 32 for UE8M0.
 *             u8 [ceil(rows/128)][atoms_k][512] with atoms_k =
 *             ceil(kpad / (4 W)); byte 16 (r % 32) + 4 ((r / 32) % 4) + s % 4
 *             of atom (r / 128, s / 4) holds the factor of slot s of row r.
 *             Bytes of rows >= rows and of slots at or beyond kpad / W are
 *             not written and feed no stored GEMM output.  ufp4_sf_atoms_layout
 *             gives atoms_k and the size.  ufp4_rht_quantize writes it when
 *             non-NULL; when both operands of a dense GEMM on a CTA-pair path
 *             carry one, the MMA issuer copies each stage's factors into
 *             tensor memory itself (no factor-building warps).  Must be NULL
 *             for fp32 scales.  16-byte aligned.
 *   sf_lanes  optional, E1M2 with E4M3 x fp32 scales only: the same factors
 *             once more, as per-lane tiles for the first operand (A) of a
 *             CTA-pair GEMM: u8 [ceil(rows/128)][ceil(kpad/128)][4096], the
 *             factor of slot s (16 elements) of row r at byte
 *             2048 ((s / 4) % 2) + 16 L + 4 (L / 32) + s % 4 of tile
 *             (r / 128, s / 8), L = r % 128.  A tile is the tensor-memory
 *             image of one 128-lane copy holding the factors of two 64-K
 *             steps (a hardware layout, not part of the method); the other
 *             bytes of a lane's 16 are zero or not written.  Factor atoms
 *             reach each 32-lane quarter by a broadcast copy per K step, so
 *             an A operand that carries these tiles saves one copy per stage.
 *             ufp4_rht_quantize writes it when non-NULL (about 5% more time
 *             per call); a dense GEMM uses it when A carries it and both
 *             operands carry factor atoms, and ignores it on B.  ufp4_sf_lanes_layout gives the size.  16-byte
 *             aligned.
 */
#ifndef UFP4_H
#define UFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    UFP4_OK = 0,
    UFP4_ERR_INVALID_ARG = 1,      /* null pointer, bad size or enum value       */
    UFP4_ERR_UNSUPPORTED = 2,      /* valid but not implemented combination      */
    UFP4_ERR_ALIGNMENT = 3,        /* pointer / leading dimension alignment      */
    UFP4_ERR_OPERAND_MISMATCH = 4, /* GEMM operands quantized incompatibly       */
    UFP4_ERR_CUDA = 5,             /* a CUDA runtime/driver call failed          */
    UFP4_ERR_DEVICE_TIMEOUT = 6    /* a kernel's bounded wait gave up            */
} ufp4_status_t;

/* 4-bit grids, [PL] §2 "FP4 formats" and §4.  INT4 is the E1M2 grid (same
 * codes under absmax scaling).  UFP4_GRID_E2M1_MAX2 is the range-restricted
 * E2M1 variant of [PL] §5 "Q4: Recipe ablations" (max_fpx = 2.0): block
 * scales map the block maximum to 2.0 and only the E2M1 magnitudes
 * {0, 0.5, 1, 1.5, 2} (codes 0..4) are used; its codes are E2M1 codes, so its
 * operands run on the E2M1 GEMM kernels.  Operands of one GEMM must share a
 * grid (else UFP4_ERR_OPERAND_MISMATCH). */
typedef enum {
    UFP4_GRID_E1M2 = 0,
    UFP4_GRID_E2M1 = 1,
    UFP4_GRID_E2M1_MAX2 = 2
} ufp4_grid_t;
/* Rounding rules, [PL] §2 "Rounding rules": RTNE for X and W, SR on dY. */
typedef enum { UFP4_ROUND_RTNE = 0, UFP4_ROUND_SR = 1 } ufp4_round_t;
/* Block scale formats: plain fp32 per block, or the two-level hierarchy of
 * NVFP4 ([PL] §6 "FP4 formats, block scaling, and scale hierarchy") that UFP4
 * inherits ([DW]: the NVFP4 recipe with the grid swapped), or the MX-style
 * power-of-two scale of the MXFP4 lineage that [PL] §6 also names: per block of
 * 32 (block must be 32) the smallest 2^X with amax <= gmax * 2^X, X clamped to
 * [-127, 127], stored as the biased exponent byte X + 127 (UE8M0; 0 for an
 * all-zero block), no tensor scale. */
typedef enum {
    UFP4_SCALE_FP32 = 0,
    UFP4_SCALE_E4M3_X_FP32 = 1,
    UFP4_SCALE_UE8M0 = 2
} ufp4_scale_fmt_t;
/* Which input dimension is the GEMM's reduction dimension ([PL] §2: input
 * channels for fwd_y, output channels for bwd_dx, tokens for bwd_dw).
 * ALONG_COLS: the contiguous dimension; output row r = input row r.
 * ALONG_ROWS: the strided dimension; output row r = input column r (the
 *             quantized operand is the transpose, K-major). */
typedef enum { UFP4_ALONG_COLS = 0, UFP4_ALONG_ROWS = 1 } ufp4_axis_t;

/* Quantizer configuration.  Fixed-width fields (C ABI stable). */
typedef struct {
    int32_t grid;           /* ufp4_grid_t                                   */
    int32_t rounding;       /* ufp4_round_t                                  */
    uint64_t sr_seed;       /* Philox4x32-10 key (SR only)                   */
    uint32_t sr_stream;     /* Philox counter word 2 (SR only)               */
    int32_t hadamard_n;     /* 0 (no RHT), 16, 32 or 64                      */
    uint64_t rht_sign_mask; /* bit i set => D_ii = -1, i < hadamard_n        */
    int32_t block;          /* scale block length along K: 16 or 32          */
    int32_t scale_fmt;      /* ufp4_scale_fmt_t                              */
} ufp4_quant_cfg_t;

/* A quantized operand: plain descriptor, owns nothing. */
typedef struct {
    void *codes;            /* device u8 [rows][kpad/2]                      */
    void *scales;           /* device, block-major, see layout above         */
    float *tensor_scale;    /* device fp32 S (two-level only, else NULL)     */
    int64_t rows;           /* output rows of the K-major view               */
    int64_t k;              /* logical reduction length                      */
    int64_t kpad;           /* k rounded up to 64                            */
    int64_t scale_ld;       /* rows rounded up to 64                         */
    ufp4_quant_cfg_t cfg;   /* how it was quantized                          */
    void *corr;             /* device u8 [rows][kpad/2] or NULL, see above   */
    void *elems8;           /* device u8 [rows][kpad] or NULL, see above     */
    void *sf_atoms;         /* device u8 factor atoms or NULL, see above     */
    void *sf_lanes;         /* device u8 per-lane factor tiles or NULL, see above */
} ufp4_qtensor_t;

/* One sub-problem of ufp4_grouped_gemm:
 *   C[c_row+i][c_col+j] = (1/n) sum_{t<k} A[a_row+i][a_col+t] * B[b_row+j][b_col+t]
 * for 0 <= i < m, 0 <= j < n.  k, a_col and b_col are multiples of 64. */
typedef struct {
    int64_t m, n, k;
    int64_t a_row, a_col;
    int64_t b_row, b_col;
    int64_t c_row, c_col;
} ufp4_group_t;

/* Default RHT sign mask: bits of splitmix64(0x5EED), any fixed choice works
 * as long as both operands of a GEMM use the same one. */
#define UFP4_DEFAULT_SIGN_MASK 0x09F1FD9D03F0A9B4ull

/* Sizes of a quantized operand.  Fills kpad, scale_ld and the byte counts of
 * the codes and scales buffers the caller must provide.  Any output pointer
 * may be NULL.  Errors: UFP4_ERR_INVALID_ARG (rows < 0, k < 0, bad cfg). */
ufp4_status_t ufp4_qtensor_layout(int64_t rows, int64_t k, const ufp4_quant_cfg_t *cfg,
                                  int64_t *kpad, int64_t *scale_ld,
                                  size_t *codes_bytes, size_t *scales_bytes);

/* Size of the optional factor-atom plane (sf_atoms) of a quantized operand:
 * atoms_k = ceil(kpad / (4 W)) atoms along K (W = 16 for E4M3 x fp32 scales,
 * 32 for UE8M0), bytes = ceil(rows / 128) * atoms_k * 512.  Either output may
 * be NULL.  Errors: INVALID_ARG (rows < 0, k < 0, bad cfg), UNSUPPORTED (fp32
 * scales: no atoms). */
ufp4_status_t ufp4_sf_atoms_layout(int64_t rows, int64_t k, const ufp4_quant_cfg_t *cfg, int64_t *atoms_k,
                                   size_t *bytes);

/* Size of the optional per-lane factor tiles (sf_lanes) of an E1M2 operand
 * with E4M3 x fp32 scales: bytes = ceil(rows / 128) * ceil(kpad / 128) * 4096.
 * Errors: INVALID_ARG (rows < 0, k < 0, bad cfg, bytes NULL), UNSUPPORTED
 * (another grid or scale format: no tiles). */
ufp4_status_t ufp4_sf_lanes_layout(int64_t rows, int64_t k, const ufp4_quant_cfg_t *cfg, size_t *bytes);

/* Absolute maximum of the rotated operand, max |H_n D x| over all elements
 * (the tensor amax that the two-level scale S is derived from; [PL] §2
 * "Random Hadamard transforms").  Input x_dev: bf16 [rows][ld] row-major,
 * 16-byte aligned, ld and (for ALONG_COLS) cols multiples of 8.  Writes one
 * fp32 to amax_dev (device).  Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED
 * (hadamard_n not in {0,16,32,64}), CUDA. */
ufp4_status_t ufp4_rht_amax(const void *x_dev, int64_t rows, int64_t cols, int64_t ld,
                            int32_t axis, int32_t hadamard_n, uint64_t rht_sign_mask,
                            float *amax_dev, void *stream);

/* Unfused RHT, the baseline of [GS] "Efficiëntie" (kernel fusion: the
 * pages time RHT fused into the FP4 quantizer against a separate RHT pass
 * followed by quantization).  y = bf16_RN(H_n D x) along the contiguous
 * dimension, per n-block of each row, with the quantizer's fp32 butterflies
 * (stages h = 1 .. n/2) and sign mask convention; n = 0 copies x.
 *   x_dev  bf16 [rows][ld], 16-byte aligned, ld % 8 == 0, cols % 64 == 0.
 *   y_dev  bf16 [rows][ldy] (caller-owned, 16-byte aligned, ldy % 8 == 0,
 *          ldy >= cols); may not overlap x.
 * Quantizing y with hadamard_n = 0 approximates ufp4_rht_quantize(x, n): the
 * rotated values pass through bf16 in between, so codes may differ where that
 * rounding moves a value across a decision boundary.
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED (n not in {0,16,32,64}, cols
 * not a multiple of 64), CUDA. */
ufp4_status_t ufp4_rht_bf16(const void *x_dev, int64_t rows, int64_t cols, int64_t ld, int32_t hadamard_n,
                            uint64_t rht_sign_mask, void *y_dev, int64_t ldy, void *stream);

/* Fused RHT + block absmax + scale + 4-bit rounding + packing ([PL] §2
 * "Blockwise quantization", "Rounding rules", "Random Hadamard transforms";
 * [PL] §5 and [GS] "Efficiëntie": RHT fused into the quantizer).
 *   x_dev       bf16 [rows][ld], row-major, 16-byte aligned, ld % 8 == 0;
 *               cols % 8 == 0 for ALONG_COLS, rows % 8 == 0 not required.
 *   axis        ufp4_axis_t, the reduction dimension of the consuming GEMM.
 *   tensor_amax_dev  device fp32 rotated amax (two-level scale only; from
 *               ufp4_rht_amax or the caller), else NULL.
 *   out         descriptor filled by the caller: codes/scales buffers sized by
 *               ufp4_qtensor_layout, rows = output rows (rows for ALONG_COLS,
 *               cols for ALONG_ROWS), k = the other dimension, kpad,
 *               scale_ld, cfg; tensor_scale (two-level) receives S.
 * SR draws are a pure function of (sr_seed, sr_stream, output row, column):
 * the same call gives the same bits on any launch configuration.
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED, CUDA. */
ufp4_status_t ufp4_rht_quantize(const void *x_dev, int64_t rows, int64_t cols, int64_t ld,
                                int32_t axis, const float *tensor_amax_dev,
                                ufp4_qtensor_t *out, void *stream);

/* Dual-output quantizer: both quantizations of one tensor from a single read
 * of it.  Every operand of the recipe feeds two GEMMs along different axes
 * (X: FPROP along cols, WGRAD along rows; W: FPROP along cols, DGRAD along
 * rows; dY: DGRAD along cols, WGRAD along rows), so reading the bf16 tile
 * once and writing both results extends the fusion of RHT into the quantizer
 * that [GS] "Efficiëntie" (kernel fusion) describes.  No counterpart call on
 * the pages: the results are bit-identical to
 *   ufp4_rht_quantize(x, ..., UFP4_ALONG_COLS, tensor_amax_cols_dev, out_cols)
 *   ufp4_rht_quantize(x, ..., UFP4_ALONG_ROWS, tensor_amax_rows_dev, out_rows)
 * (SR draws included: they depend on seed, stream, output row and column only).
 *   x_dev       bf16 [rows][ld], the constraints of ufp4_rht_quantize.
 *   out_cols    the ALONG_COLS result (rows = rows, k = cols).
 *   out_rows    the ALONG_ROWS result (rows = cols, k = rows).
 *   tensor_amax_cols_dev / tensor_amax_rows_dev  rotated amaxes along each
 *               axis (two-level scale only, from ufp4_rht_amax_dual), else NULL.
 * The two cfgs must agree on everything but sr_stream (grid, rounding,
 * sr_seed, hadamard_n and the first hadamard_n sign bits, block, scale_fmt),
 * else UFP4_ERR_UNSUPPORTED: call ufp4_rht_quantize twice instead.
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED, CUDA. */
ufp4_status_t ufp4_rht_quantize_dual(const void *x_dev, int64_t rows, int64_t cols, int64_t ld,
                                     const float *tensor_amax_cols_dev,
                                     const float *tensor_amax_rows_dev, ufp4_qtensor_t *out_cols,
                                     ufp4_qtensor_t *out_rows, void *stream);

/* Both rotated amaxes of one tensor from a single read: amax_cols_dev
 * receives ufp4_rht_amax(..., UFP4_ALONG_COLS, ...) and amax_rows_dev
 * ufp4_rht_amax(..., UFP4_ALONG_ROWS, ...) (bit-identical).  Input
 * constraints and errors as ufp4_rht_amax. */
ufp4_status_t ufp4_rht_amax_dual(const void *x_dev, int64_t rows, int64_t cols, int64_t ld,
                                 int32_t hadamard_n, uint64_t rht_sign_mask, float *amax_cols_dev,
                                 float *amax_rows_dev, void *stream);

/* FPROP, fwd_y:  Y[M][N] = X W^T.  xq: X quantized ALONG_COLS ([M][K]);
 * wq: W quantized ALONG_COLS ([N][K]).  y_dev fp32 [M][ldy], ldy >= N,
 * 4-byte aligned (rows that are 16-byte aligned get vector stores).
 * ([PL] §2: rotation along input channels.)
 * Errors: INVALID_ARG, ALIGNMENT, OPERAND_MISMATCH (grid, block, scale format,
 * hadamard_n, sign mask or kpad differ), UNSUPPORTED, CUDA. */
ufp4_status_t ufp4_gemm_fprop(const ufp4_qtensor_t *xq, const ufp4_qtensor_t *wq,
                              float *y_dev, int64_t ldy, void *stream);

/* DGRAD, bwd_dx:  dX[M][K] = dY W.  dyq: dY [M][N] quantized ALONG_COLS
 * (usually SR); wtq: W [N][K] quantized ALONG_ROWS, i.e. W^T [K][N] K-major.
 * dx_dev fp32 [M][lddx].  ([PL] §2: rotation along output channels.) */
ufp4_status_t ufp4_gemm_dgrad(const ufp4_qtensor_t *dyq, const ufp4_qtensor_t *wtq,
                              float *dx_dev, int64_t lddx, void *stream);

/* WGRAD, bwd_dw:  dW[N][K] = dY^T X.  dytq: dY [M][N] quantized ALONG_ROWS
 * (dY^T [N][M]); xtq: X [M][K] quantized ALONG_ROWS (X^T [K][M]).
 * dw_dev fp32 [N][lddw].  ([PL] §2: rotation along batch tokens.) */
ufp4_status_t ufp4_gemm_wgrad(const ufp4_qtensor_t *dytq, const ufp4_qtensor_t *xtq,
                              float *dw_dev, int64_t lddw, void *stream);

/* Grouped contraction for mixture-of-experts layers (the recipe is trained
 * on MoE 7.9B / 124B models, [PL] §5 Q2-Q3).  groups_dev: device array of
 * num_groups ufp4_group_t, read by the kernel (the tile schedule is derived on
 * the device, so the table may be written by earlier kernels on the same
 * stream without a host round trip).  Each group contracts its own window of
 * the shared quantized operands a and b: rows [a_row, a_row+m) x columns
 * [a_col, a_col+k) of a and the same for b, so a and b must agree on grid,
 * block, scale format, hadamard_n and sign mask but not on k.  Typical uses:
 * per-expert token segments of a routed activation (FPROP / DGRAD, ragged m),
 * per-expert K windows of a stacked weight quantized ALONG_ROWS (DGRAD), and
 * per-expert token windows along K (WGRAD, segments zero-padded to 64).
 * Requirements checked on the device: k, a_col, b_col multiples of 64; a_row,
 * b_row multiples of 16; a group that violates them is skipped and writes
 * nothing.  Factor atoms (sf_atoms) are not read here: the grouped kernels
 * build the factors from the block-major scales.  Reads outside an operand
 * return zeros.  The caller guarantees that
 * every group's output window lies inside c_dev [..][ldc] and that groups do
 * not overlap.  Errors: INVALID_ARG, ALIGNMENT, OPERAND_MISMATCH, CUDA. */
ufp4_status_t ufp4_grouped_gemm(const ufp4_qtensor_t *a, const ufp4_qtensor_t *b,
                                const ufp4_group_t *groups_dev, int32_t num_groups,
                                float *c_dev, int64_t ldc, void *stream);

/* Kernel family for GEMMs whose operands carry two-level (E4M3 x fp32)
 * scales.  Both families run the block-scaled FP4 MMA (kind::mxf4nvf4, UE4M3
 * factors per 16 elements), with E1M2 codes split exactly into two E2M1
 * planes (four MMAs per K step), and compute the same contraction:
 *   UFP4_GEMM_PATH_NATIVE_FP4 one CTA per 128 x 192 tile, two accumulators
 *                             (the epilogue overlaps the next tile);
 *   UFP4_GEMM_PATH_NATIVE_FP4_PAIR256  CTA pairs (cta_group::2) with 256 x 256
 *                             tiles (half the operand bytes per flop of one
 *                             CTA); needs E2M1 operands, or E1M2 operands whose
 *                             correction planes follow their codes in one
 *                             allocation (else the one-CTA path);
 *   UFP4_GEMM_PATH_AUTO       the library's choice (default; currently the
 *                             256 x 256 CTA-pair path where it applies, else
 *                             the one-CTA path).
 * Values 1, 2 and 4 named kernel families that are no longer built.  The
 * setting is process-wide and read at each GEMM call; fp32 and UE8M0 block
 * scales are unaffected (fp32-scale kernel, or the MX path).  Errors:
 * INVALID_ARG for any other value. */
typedef enum {
    UFP4_GEMM_PATH_AUTO = 0,
    UFP4_GEMM_PATH_NATIVE_FP4 = 3,
    UFP4_GEMM_PATH_NATIVE_FP4_PAIR256 = 5
} ufp4_gemm_path_t;
ufp4_status_t ufp4_set_two_level_gemm_path(int32_t path);
int32_t ufp4_get_two_level_gemm_path(void);

/* ---------------------------------------------------------------------------
 * Quantization diagnostics ([PL] §5 "Q1: Grid geometry and RHT" and Appendix A
 * "RHT-Induced SQNR Changes in Tensors and GEMM Outputs"; [GS] "Kwantisatie en
 * GEMM Diagnostiek": tensor and GEMM-output SQNR, their change under the RHT,
 * bucket use, and the signed level error of §3.1 "Shrinkage Bias").  The
 * pages print no formulas; the definitions below are this library's.
 *
 * Sums and counts over the logical columns [0, k) of every output row of a
 * quantized operand, u the rotated value the quantizer rounded (recomputed
 * from x with the operand's cfg) and sigma its block step (s, or e_b * S):
 *   signal          sum u^2
 *   noise           sum (u - deq)^2, deq = +-lvl(code) * sigma
 *   level_err[k]    sum over elements of magnitude code k in blocks with
 *                   sigma > 0 of lvl(k) - |u| / sigma (grid units; < 0 means
 *                   the level sits below the values it stands for)
 *   level_n[k]      the number of those elements
 *   code_count[c]   elements per 4-bit code c (0x8 never occurs)
 *   nonzero         elements with u != 0;  underflow: of those, coded 0
 * The floating-point sums are accumulated in fp32 over each 64-element
 * segment of a row and in fp64 across segments (relative error well below
 * 1e-5); the order of the fp64 additions is not fixed (atomics). */
typedef struct {
    double signal;
    double noise;
    double level_err[8];
    uint64_t level_n[8];
    uint64_t code_count[16];
    uint64_t nonzero;
    uint64_t underflow;
} ufp4_qstats_t;

/* Fills *stats_dev (device memory, zeroed by the call) for the operand q
 * quantized from x_dev along axis (the arguments of the ufp4_rht_quantize
 * call that produced q).  Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED, CUDA. */
ufp4_status_t ufp4_quant_stats(const void *x_dev, int64_t rows, int64_t cols, int64_t ld,
                               int32_t axis, const ufp4_qtensor_t *q, ufp4_qstats_t *stats_dev,
                               void *stream);

/* Derived figures of a host copy of the sums (plain host arithmetic):
 *   sqnr_db          10 log10(signal / noise) (+inf when noise = 0)
 *   bucket_ratio     share of the grid's codes (15; 9 for the restricted
 *                    E2M1 grid) holding more than 1/(15*16) of the elements
 *   underflow_ratio  underflow / nonzero (0 when nonzero = 0)
 *   level_mean_err   level_err[k] / level_n[k] (NaN when level_n[k] = 0)
 * Errors: INVALID_ARG (NULL pointer, unknown grid). */
typedef struct {
    double sqnr_db;
    double bucket_ratio;
    double underflow_ratio;
    double level_mean_err[8];
} ufp4_qstats_summary_t;
ufp4_status_t ufp4_qstats_summarize(const ufp4_qstats_t *stats_host, int32_t grid,
                                    ufp4_qstats_summary_t *out);

/* GEMM-output SQNR sums: sums_dev[0] = sum ref^2, sums_dev[1] = sum (test -
 * ref)^2 over a rows x cols fp32 region (row pitches ld_ref, ld_test >= cols),
 * accumulated in fp64 (device memory, zeroed by the call).  SQNR =
 * 10 log10(sums[0] / sums[1]).  Errors: INVALID_ARG, CUDA. */
ufp4_status_t ufp4_sqnr_sums(const float *ref_dev, int64_t ld_ref, const float *test_dev,
                             int64_t ld_test, int64_t rows, int64_t cols, double *sums_dev,
                             void *stream);

/* Reads and clears the device-side error word that kernels set when a
 * bounded pipeline wait gives up (synchronises the current device).
 * Returns UFP4_OK or UFP4_ERR_DEVICE_TIMEOUT (or UFP4_ERR_CUDA). */
ufp4_status_t ufp4_check_device_status(void);

/* Test support (no counterpart in the pages): sets the time limit of the
 * quantizer's producer-side wait for a free pipeline stage, in ns, for the
 * current device; 0 restores the default (2 s).  A limit far below one
 * stage's compute time makes that wait give up during a call: the kernel
 * stops issuing loads, lets every issued load land (the drain keeps its
 * normal bound), unwinds, and the next ufp4_check_device_status() reports
 * UFP4_ERR_DEVICE_TIMEOUT once.  Outputs of such a call are incomplete.
 * Synchronous; not for concurrent use with quantize calls.  Errors: CUDA. */
ufp4_status_t ufp4_test_set_quantize_wait_limit(uint64_t limit_ns);

/* Human-readable name of a status code (static string). */
const char *ufp4_status_string(ufp4_status_t status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t ufp4_version(void);

#ifdef __cplusplus
}
#endif
#endif /* UFP4_H */
