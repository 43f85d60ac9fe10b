/*
 * ufp4_oracle.c -- plain, slow, step-by-step CPU oracle of the UFP4 hot path.
 *
 * TEST INFRASTRUCTURE ONLY (see ufp4_oracle.h).  Built with
 *   gcc -O2 -ffp-contract=off -fno-fast-math [-fopenmp]
 * so every float operation below is one IEEE binary32/binary64 operation in
 * the order written.  Decisions that pick a 4-bit code are made by exact
 * comparisons in binary64 (every product compared there is exact).
 */
#include "ufp4_oracle.h"

#include <math.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Grids.  [PL] §2 Preliminaries "FP4 formats": one sign bit plus exponent and
 * mantissa fields; the study's codebooks are E2M1, E1M2 and INT4.
 * E2M1 magnitudes follow the OCP FP4 encoding (the range-restricted set
 * {0, 0.5, 1, 1.5, 2} of [PL] §5 Q4 is its prefix).  E1M2: the pages give no
 * level list; reading: IEEE-style field layout with exponent bias 1, so the
 * magnitudes are k/4, k = 0..7 -- a uniform grid, identical up to a power of
 * two to sign-magnitude INT4 ("E1M2/INT4-style uniform grid", [PL] §4). */
static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double uo_level(int grid, int k)
{
    if (k < 0 || k > 7) return 0.0;
    if (grid == UO_GRID_E2M1 || grid == UO_GRID_E2M1_MAX2) return kE2M1[k];
    return (double)k / 4.0;
}

/* The largest magnitude code a grid uses.  The range-restricted E2M1 variant
 * ([PL] §5 Q4, max_fpx = 2.0) keeps the E2M1 code points but stops at code 4
 * (magnitude 2.0): block scales map the block maximum to 2.0 and larger
 * quotients saturate there.  Reading: "max_fpx" is the grid maximum that the
 * scale targets, the level set being the printed {0, 0.5, 1, 1.5, 2}. */
int uo_top_code(int grid) { return grid == UO_GRID_E2M1_MAX2 ? 4 : 7; }

double uo_gmax(int grid) { return uo_level(grid, uo_top_code(grid)); }

float uo_bf16_to_f32(uint16_t b)
{
    uint32_t w = (uint32_t)b << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return f;
}

int64_t uo_kpad(int64_t k) { return (k + 63) / 64 * 64; }

int uo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Random Hadamard transform, [PL] §2 "Random Hadamard transforms": a random
 * sign diagonal D first, then a Sylvester Hadamard matrix, applied along the
 * GEMM's reduction dimension.  Unnormalised butterflies in natural (Sylvester)
 * order: for h = 1, 2, 4, ..., n/2, every pair (j, j+h) with bit h of j clear
 * becomes (a+b, a-b).  The result is u = H_n D x with
 * H_n[i][j] = (-1)^popcount(i & j).  The fp32 version rounds after every
 * add exactly as written; the stage order is part of the contract. */
void uo_fwht_f32(float *v, int n)
{
    for (int h = 1; h < n; h <<= 1) {
        for (int j = 0; j < n; j++) {
            if (j & h) continue;
            float a = v[j];
            float b = v[j + h];
            v[j] = a + b;
            v[j + h] = a - b;
        }
    }
}

void uo_fwht_f64(double *v, int n)
{
    for (int h = 1; h < n; h <<= 1) {
        for (int j = 0; j < n; j++) {
            if (j & h) continue;
            double a = v[j];
            double b = v[j + h];
            v[j] = a + b;
            v[j + h] = a - b;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* OCP OFP8 E4M3 ("E4M3FN"): bias 7, 3 mantissa bits, subnormals m/8 * 2^-6,
 * largest finite 0x7E = 1.75 * 2^8 = 448, no infinities.  Conversion from a
 * non-negative binary32 value: round to nearest, ties to even mantissa,
 * saturating to 448 ("satfinite"). */
uint8_t uo_e4m3_rne_satfinite(float x)
{
    double xd = (double)x;
    if (!(xd > 0.0)) return 0;           /* zero (and any negative input) */
    if (xd >= 448.0) return 0x7E;
    if (xd < ldexp(1.0, -6)) {           /* subnormal range, step 2^-9 */
        double m = nearbyint(xd * 512.0);
        if (m >= 8.0) return 0x08;       /* rounds up to 2^-6 */
        return (uint8_t)m;
    }
    int E;
    double f = frexp(xd, &E);            /* xd = f * 2^E, f in [0.5, 1) */
    double q = 2.0 * f;                  /* [1, 2) */
    int eu = E - 1;
    double m = nearbyint((q - 1.0) * 8.0);
    if (m >= 8.0) { m = 0.0; eu += 1; }
    int eb = eu + 7;
    if (eb > 15 || (eb == 15 && m > 6.0)) return 0x7E;
    return (uint8_t)((eb << 3) | (int)m);
}

double uo_e4m3_value(uint8_t b)
{
    int e = (b >> 3) & 15, m = b & 7;
    if (e == 0) return ldexp((double)m, -9);
    return ldexp(1.0 + (double)m / 8.0, e - 7);
}

/* ------------------------------------------------------------------------ */
/* Philox4x32-10, from the round function of Salmon et al., "Parallel Random
 * Numbers: As Easy as 1, 2, 3" (SC'11): two 32x32->64 multiplications per
 * round with multipliers 0xD2511F53 and 0xCD9E8D57, the key bumped by the
 * Weyl constants 0x9E3779B9 / 0xBB67AE85 between rounds, ten rounds. */
static void philox_round(uint32_t c[4], const uint32_t k[2])
{
    uint64_t p0 = (uint64_t)0xD2511F53u * c[0];
    uint64_t p1 = (uint64_t)0xCD9E8D57u * c[2];
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c[1] ^ k[0];
    uint32_t n2 = hi0 ^ c[3] ^ k[1];
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
}

void uo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
    uint32_t k[2] = {key[0], key[1]};
    for (int r = 0; r < 10; r++) {
        if (r > 0) {
            k[0] += 0x9E3779B9u;
            k[1] += 0xBB67AE85u;
        }
        philox_round(c, k);
    }
    memcpy(out, c, sizeof c);
}

/* Reading of "stochastic rounding on dY" ([PL] §2 "Rounding rules", §4): the
 * pages fix no generator.  One Philox call yields eight 16-bit uniforms for
 * eight consecutive logical elements L = row * kpad + col of the K-major
 * output operand: counter (g lo, g hi, stream, 0) with g = L >> 3, key
 * (seed lo, seed hi), word (L >> 1) & 3, low half for even L. */
uint32_t uo_sr_u16(uint64_t seed, uint32_t stream, uint64_t L)
{
    uint64_t g = L >> 3;
    uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), stream, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    uo_philox4x32_10(ctr, key, out);
    uint32_t w = out[(L >> 1) & 3];
    return (L & 1) ? (w >> 16) : (w & 0xFFFFu);
}

/* ------------------------------------------------------------------------ */
/* Rounding rules, [PL] §2 "Rounding rules".
 * RTNE: the nearest codebook level, ties to the even magnitude index (which
 * is the even mantissa for both grids), decided on the exact quotient |u|/s:
 * |u| is compared with (level midpoint) * s, a product exact in binary64.
 * Magnitudes beyond gmax saturate to gmax ("no clipping", [PL] limitations). */
int uo_round_rtne(int grid, double au, double s)
{
    const int top = uo_top_code(grid);
    for (int j = 0; j < top; j++) {
        double mid = (uo_level(grid, j) + uo_level(grid, j + 1)) / 2.0;
        double t = mid * s;
        if (au < t) return j;
        if (au == t) return (j % 2 == 0) ? j : j + 1;
    }
    return top;
}

/* SR: between the adjacent levels lo <= |u|/s < hi, round up iff
 * |u| > (lo + r16 * 2^-16 * (hi - lo)) * s, so P(up) is the fractional
 * position within the bin (to 2^-16) and values on a level never move. */
int uo_round_sr(int grid, double au, double s, uint32_t r16)
{
    const int top = uo_top_code(grid);
    int lo = top;
    while (lo > 0 && uo_level(grid, lo) * s > au) lo--;
    if (lo == top) return top;
    double L0 = uo_level(grid, lo), L1 = uo_level(grid, lo + 1);
    double c = L0 + (L1 - L0) * ((double)r16 / 65536.0);
    return (au > c * s) ? lo + 1 : lo;
}

/* ------------------------------------------------------------------------ */
/* Two-level scales.  [PL] §6 names NVFP4's "smaller blocks and a two-level
 * scale hierarchy"; [DW] says UFP4 reproduces the NVFP4 recipe with the grid
 * swapped.  Reading: an fp32 tensor scale S = RN(amax_T / (gmax * 448)) from
 * the rotated tensor's absolute maximum (S = 1 when amax_T = 0), G = RN(gmax*S),
 * and per block e_b = E4M3(RN(amax_b / G)).  The block's dequantisation step
 * is the exact product e_b * S. */
float uo_tensor_scale(int grid, float amax_t)
{
    if (!(amax_t > 0.0f)) return 1.0f;
    float denom = (float)(uo_gmax(grid) * 448.0);
    return amax_t / denom;
}

float uo_block_decode_base(int grid, float S)
{
    float gm = (float)uo_gmax(grid);
    return gm * S;
}

/* MX-style block scale.  [PL] §6 places the study in the lineage of MXFP4,
 * whose block scaling is coarser than NVFP4's: OCP MX formats give a block of
 * 32 elements one shared scale that is a power of two, stored as an 8-bit
 * biased exponent (UE8M0).  Reading: the scale 2^X is the smallest power of
 * two that keeps the block maximum on the grid (amax <= gmax * 2^X, the "no
 * clipping" rule of the other formats), X clamped to the byte's range
 * [-127, 127]; an all-zero block stores 0.  Found by plain search over X. */
uint8_t uo_ue8m0_scale(int grid, float amax)
{
    if (!(amax > 0.0f)) return 0;
    const double gm = uo_gmax(grid);
    int X = -127;
    while (X < 127 && ldexp(gm, X) < (double)amax) X++;
    return (uint8_t)(X + 127);
}

double uo_ue8m0_value(uint8_t e) { return ldexp(1.0, (int)e - 127); }

/* ------------------------------------------------------------------------ */
/* Load logical row r of the K-major view, zero padded to kpad, apply D then
 * H_n per n-block.  [PL] §2: for the three training GEMMs the rotation acts
 * along the shared reduction dimension (input channels for fwd_y, output
 * channels for bwd_dx, tokens for bwd_dw). */
static void rotated_row(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                        int axis, int64_t r, int64_t K, int64_t kpad, int n,
                        uint64_t mask, float *v)
{
    for (int64_t t = 0; t < kpad; t++) {
        float f = 0.0f;
        if (t < K) {
            uint16_t b = (axis == UO_ALONG_COLS) ? x[r * ld + t] : x[t * ld + r];
            f = uo_bf16_to_f32(b);
        }
        v[t] = f;
    }
    (void)rows; (void)cols;
    if (n <= 0) return;
    for (int64_t b0 = 0; b0 < kpad; b0 += n) {
        for (int i = 0; i < n; i++)
            if ((mask >> i) & 1u) v[b0 + i] = -v[b0 + i];
        uo_fwht_f32(v + b0, n);
    }
}

float uo_rht_amax(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int axis,
                  int hadamard_n, uint64_t sign_mask)
{
    int64_t K = (axis == UO_ALONG_COLS) ? cols : rows;
    int64_t nout = (axis == UO_ALONG_COLS) ? rows : cols;
    int64_t kpad = uo_kpad(K);
    float amax = 0.0f;
#pragma omp parallel
    {
        float *v = (float *)malloc(sizeof(float) * (size_t)kpad);
        float local = 0.0f;
#pragma omp for schedule(static)
        for (int64_t r = 0; r < nout; r++) {
            rotated_row(x, rows, cols, ld, axis, r, K, kpad, hadamard_n, sign_mask, v);
            for (int64_t t = 0; t < kpad; t++) {
                float a = fabsf(v[t]);
                if (a > local) local = a;
            }
        }
#pragma omp critical
        if (local > amax) amax = local;
        free(v);
    }
    return amax;
}

/* Block-wise quantisation, [PL] §2 "Blockwise quantization": contiguous
 * blocks along K share one scale; the normalised codebook's largest
 * magnitude is gmax and the rounding rule rho_G maps |u|/s to a level. */
int uo_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int axis,
                const uo_cfg_t *cfg, float tensor_amax, int64_t r0, int64_t nr,
                int8_t *codes, float *scales, uint8_t *escales, float *S_out,
                float *u_out)
{
    const int n = cfg->hadamard_n, B = cfg->block, grid = cfg->grid;
    if (!(n == 0 || n == 16 || n == 32 || n == 64)) return 1;
    if (!(B == 16 || B == 32)) return 2;
    if (cfg->scale_fmt == UO_SCALE_UE8M0 && B != 32) return 3;   /* MX blocks are 32 long */
    const int64_t K = (axis == UO_ALONG_COLS) ? cols : rows;
    const int64_t kpad = uo_kpad(K);
    const int64_t nb = kpad / B;
    const double gmax = uo_gmax(grid);
    float S = 1.0f, G = 0.0f;
    if (cfg->scale_fmt == UO_SCALE_E4M3_X_FP32) {
        S = uo_tensor_scale(grid, tensor_amax);
        G = uo_block_decode_base(grid, S);
        if (S_out) *S_out = S;
    }
    int err = 0;
#pragma omp parallel
    {
        float *v = (float *)malloc(sizeof(float) * (size_t)kpad);
#pragma omp for schedule(static)
        for (int64_t i = 0; i < nr; i++) {
            const int64_t r = r0 + i;
            rotated_row(x, rows, cols, ld, axis, r, K, kpad, n, cfg->sign_mask, v);
            if (u_out) memcpy(u_out + i * kpad, v, sizeof(float) * (size_t)kpad);
            for (int64_t b = 0; b < nb; b++) {
                float amax = 0.0f;
                for (int t = 0; t < B; t++) {
                    float a = fabsf(v[b * B + t]);
                    if (a > amax) amax = a;
                }
                double s;
                if (cfg->scale_fmt == UO_SCALE_FP32) {
                    float sf = amax / (float)gmax;
                    scales[i * nb + b] = sf;
                    s = (double)sf;
                } else if (cfg->scale_fmt == UO_SCALE_UE8M0) {
                    uint8_t e = uo_ue8m0_scale(grid, amax);
                    escales[i * nb + b] = e;
                    s = uo_ue8m0_value(e);
                } else {
                    float q = amax / G;
                    uint8_t e = uo_e4m3_rne_satfinite(q);
                    escales[i * nb + b] = e;
                    s = uo_e4m3_value(e) * (double)S;
                }
                for (int t = 0; t < B; t++) {
                    const int64_t col = b * B + t;
                    const float u = v[col];
                    const double au = fabs((double)u);
                    int k = 0;
                    if (s > 0.0) {
                        if (cfg->rounding == UO_ROUND_RTNE) {
                            k = uo_round_rtne(grid, au, s);
                        } else {
                            uint64_t L = (uint64_t)r * (uint64_t)kpad + (uint64_t)col;
                            k = uo_round_sr(grid, au, s, uo_sr_u16(cfg->sr_seed, cfg->sr_stream, L));
                        }
                    }
                    int8_t c = (int8_t)k;
                    if (k != 0 && u < 0.0f) c = (int8_t)(k | 8);
                    codes[i * kpad + col] = c;
                }
            }
        }
        free(v);
    }
    return err;
}

void uo_dequantize(const int8_t *codes, const float *scales, const uint8_t *escales,
                   float S, int64_t nr, int64_t kpad, int grid, int block,
                   int scale_fmt, double *out)
{
    const int64_t nb = kpad / block;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nr; i++) {
        for (int64_t t = 0; t < kpad; t++) {
            int c = codes[i * kpad + t];
            double lv = uo_level(grid, c & 7);
            if (c & 8) lv = -lv;
            int64_t b = t / block;
            double s = (scale_fmt == UO_SCALE_FP32)    ? (double)scales[i * nb + b]
                       : (scale_fmt == UO_SCALE_UE8M0) ? uo_ue8m0_value(escales[i * nb + b])
                                                       : uo_e4m3_value(escales[i * nb + b]) * (double)S;
            out[i * kpad + t] = s * lv;
        }
    }
}

/* GEMM definition, [PL] §2 / §4: the low-precision GEMM contracts the two
 * rotated, quantised operands along the shared reduction dimension; with the
 * same D and H_n on both sides the rotation cancels up to the factor n
 * ((A D H)(B D H)^T = n A B^T), applied here as inv_n.  fp64 accumulation in
 * ascending k. */
void uo_gemm_tn_f64(const double *A, const double *B, int64_t M, int64_t N, int64_t K,
                    double inv_n, double *C, int64_t ldc)
{
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t i = 0; i < M; i++) {
        const double *a = A + i * K;
        for (int64_t j = 0; j < N; j++) {
            const double *b = B + j * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++) acc += a[k] * b[k];
            C[i * ldc + j] = acc * inv_n;
        }
    }
}

void uo_gemm_tn_f64_entries(const double *A, const double *B, int64_t K, double inv_n,
                            const int64_t *ii, const int64_t *jj, int64_t count,
                            double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t e = 0; e < count; e++) {
        const double *a = A + ii[e] * K;
        const double *b = B + jj[e] * K;
        double acc = 0.0;
        for (int64_t k = 0; k < K; k++) acc += a[k] * b[k];
        out[e] = acc * inv_n;
    }
}

/* ------------------------------------------------------------------------ */
/* Array forms of the scalar routines above, for the pins (no new arithmetic). */
void uo_e4m3_rne_satfinite_array(const float *x, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; i++) out[i] = uo_e4m3_rne_satfinite(x[i]);
}

void uo_sr_u16_array(uint64_t seed, uint32_t stream, const uint64_t *L, int64_t n,
                     uint32_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) out[i] = uo_sr_u16(seed, stream, L[i]);
}

void uo_sr_u16_seeds(const uint64_t *seeds, int64_t n, uint32_t stream, uint64_t L,
                     uint32_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) out[i] = uo_sr_u16(seeds[i], stream, L);
}

void uo_round_rtne_array(int grid, const double *au, double s, int64_t n, int32_t *out)
{
    for (int64_t i = 0; i < n; i++) out[i] = uo_round_rtne(grid, au[i], s);
}

void uo_round_sr_array(int grid, const double *au, double s, const uint32_t *r16,
                       int64_t n, int32_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) out[i] = uo_round_sr(grid, au[i], s, r16[i]);
}
