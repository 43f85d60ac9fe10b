/*
 * ufp4_oracle.h -- plain CPU oracle for the UFP4 quantize + GEMM hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this code: only tests/, __graft_entry__.smoke() and the cpu_baseline /
 * reference legs of bench.py use it.  It shares no source with the CUDA
 * library (no headers, tables or helpers in common).
 *
 * Sources (web pages on arXiv 2606.20381, "Rethinking Shrinkage Bias in LLM
 * FP4 Pretraining: Geometric Origin, Systemic Impact, and UFP4 Recipe"):
 *   [PL]  paperlayer.ai per-section summary of the paper
 *   [GS]  gist.science technical summary ("Technische Samenvatting")
 *   [DW]  dreamwings.cn author blog post on the paper
 * Each function names the section it follows.  Where the pages leave a step
 * open the adopted reading is stated at the function.
 *
 * Logical (unpacked) layouts used here:
 *   codes  int8  [rows_out][kpad]   nibble value 0..15: bit3 = sign, bits0..2 = k
 *   scales float [rows_out][kpad/B] (fp32 mode)
 *   escale uint8 [rows_out][kpad/B] (two-level mode: E4M3 bytes) + one fp32 S
 */
#ifndef UFP4_ORACLE_H
#define UFP4_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { UO_GRID_E1M2 = 0, UO_GRID_E2M1 = 1, UO_GRID_E2M1_MAX2 = 2 };
enum { UO_ROUND_RTNE = 0, UO_ROUND_SR = 1 };
enum { UO_SCALE_FP32 = 0, UO_SCALE_E4M3_X_FP32 = 1, UO_SCALE_UE8M0 = 2 };
enum { UO_ALONG_COLS = 0, UO_ALONG_ROWS = 1 };

typedef struct {
    int grid;            /* UO_GRID_*                                   */
    int rounding;        /* UO_ROUND_*                                  */
    uint64_t sr_seed;    /* Philox key for stochastic rounding          */
    uint32_t sr_stream;  /* Philox counter word 2                       */
    int hadamard_n;      /* 0 (off), 16, 32, 64                         */
    uint64_t sign_mask;  /* bit i set => D_ii = -1 (i < hadamard_n)     */
    int block;           /* scale block: 16 or 32                       */
    int scale_fmt;       /* UO_SCALE_*                                  */
} uo_cfg_t;

/* grids */
double uo_level(int grid, int k);
double uo_gmax(int grid);
/* MX-style power-of-two block scale: byte X + 127 of the smallest X with
 * amax <= gmax * 2^X (clamped to [-127, 127]; 0 when amax = 0), and its value */
uint8_t uo_ue8m0_scale(int grid, float amax);
double uo_ue8m0_value(uint8_t e);
int uo_top_code(int grid);   /* largest magnitude code the grid uses */

/* bf16 bit pattern -> float (exact) */
float uo_bf16_to_f32(uint16_t b);

/* in-place fp32 Walsh-Hadamard butterflies, stages h = 1, 2, ..., n/2 */
void uo_fwht_f32(float *v, int n);
/* the same transform in fp64 (used by the pins only) */
void uo_fwht_f64(double *v, int n);

/* OCP OFP8 E4M3: round-to-nearest-even with saturation to 448 (x >= 0) */
uint8_t uo_e4m3_rne_satfinite(float x);
double uo_e4m3_value(uint8_t b);

/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11) */
void uo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);
/* 16-bit uniform that stochastic rounding uses for logical element L */
uint32_t uo_sr_u16(uint64_t seed, uint32_t stream, uint64_t L);

/* rounding decisions on the exact quotient |u| / s (s > 0), return k in 0..7 */
int uo_round_rtne(int grid, double au, double s);
int uo_round_sr(int grid, double au, double s, uint32_t r16);

/* two-level scale hierarchy helpers */
float uo_tensor_scale(int grid, float amax_t);     /* S */
float uo_block_decode_base(int grid, float S);     /* G = RN(gmax*S) */

int64_t uo_kpad(int64_t k);

/* rotated-domain absolute maximum of a whole operand */
float uo_rht_amax(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int axis,
                  int hadamard_n, uint64_t sign_mask);

/*
 * Quantize output rows [r0, r0+nr) of the operand's K-major view.
 *   axis = UO_ALONG_COLS: output row r is input row r, K = cols.
 *   axis = UO_ALONG_ROWS: output row r is input column r, K = rows.
 * Outputs are written for the nr requested rows, packed from index 0.
 * u_out (optional, may be NULL): the rotated fp32 values [nr][kpad].
 * Returns 0 on success.
 */
int uo_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int axis,
                const uo_cfg_t *cfg, float tensor_amax, int64_t r0, int64_t nr,
                int8_t *codes, float *scales, uint8_t *escales, float *S_out,
                float *u_out);

/* dequantized rotated values s*lvl(c) (without 1/sqrt(n)), fp64 [nr][kpad] */
void uo_dequantize(const int8_t *codes, const float *scales, const uint8_t *escales,
                   float S, int64_t nr, int64_t kpad, int grid, int block,
                   int scale_fmt, double *out);

/* C[i][j] = inv_n * sum_k A[i][k] * B[j][k] in fp64 (TN contraction) */
void uo_gemm_tn_f64(const double *A, const double *B, int64_t M, int64_t N, int64_t K,
                    double inv_n, double *C, int64_t ldc);
/* same for a list of (i, j) entries */
void uo_gemm_tn_f64_entries(const double *A, const double *B, int64_t K, double inv_n,
                            const int64_t *ii, const int64_t *jj, int64_t count,
                            double *out);

int uo_num_threads(void);

/* array forms of the scalar routines (used by the pins) */
void uo_e4m3_rne_satfinite_array(const float *x, int64_t n, uint8_t *out);
void uo_sr_u16_array(uint64_t seed, uint32_t stream, const uint64_t *L, int64_t n,
                     uint32_t *out);
void uo_sr_u16_seeds(const uint64_t *seeds, int64_t n, uint32_t stream, uint64_t L,
                     uint32_t *out);
void uo_round_rtne_array(int grid, const double *au, double s, int64_t n, int32_t *out);
void uo_round_sr_array(int grid, const double *au, double s, const uint32_t *r16,
                       int64_t n, int32_t *out);

#ifdef __cplusplus
}
#endif
#endif
