/*
 * IntLoRA integer low-rank merge: CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY. The tests, the smoke check and the CPU-baseline
 * leg of the benchmark load this file's library; the CUDA library never does,
 * and the two share no code, header, table or constant generator.
 *
 * Everything here is plain fp64 C written from the method's definition, one
 * step at a time in the order the method states it, with no blocking, fusion
 * or reordering. Sources cited below:
 *
 *   [IntLoRA notes]  "IntLoRA: Integral Low-rank Adaptation of Quantized
 *                    Diffusion Models", Paper-Notes page (ICML2025), section
 *                    "方法详解" (method), subsections 1 (AQS), 2 (MLA),
 *                    3 (VMC) and "两种实现版本" (the MUL and SHIFT variants).
 *   [IntLoRA summary] atlas.scime.ai summary of the same paper, sections
 *                    "Approach" and "Measured effects" (Laplace beats
 *                    Gaussian, Cauchy and Student-t as the auxiliary law).
 *   [Philox]         Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
 *                    easy as 1, 2, 3", SC'11: the Philox4x32 round, its two
 *                    multipliers and its two Weyl key increments.
 *   [Affine quant]   Jacob et al., CVPR 2018: asymmetric uniform quantizer
 *                    whose range contains real 0, integer zero-point.
 *
 * Readings the pages leave open (all listed in the design notes):
 *   - sigma is the population standard deviation (mean removed, divide by N);
 *   - "s * I" in the MLA equation is the per-row scale broadcast along the row;
 *   - where W_round - z = 0 the quotient term of U is taken as 0;
 *   - the quantizer range always contains 0; a row whose range is {0} gets
 *     scale 1 and zero-point 0;
 *   - rounding is to nearest, ties to even (C nearbyint in the default mode);
 *   - SHIFT: V = U / max_j |U_ij|, shift = nearest integer to -log2|V|,
 *     clamped to [0, 2^b - 1], and ">>" is an arithmetic (floor) shift;
 *   - the STE backward is the plain pair dA = G B^T, dB = A^T G;
 *   - the integer inference GEMM takes int8 activations with a per-token
 *     scale and the merged integer weights with their per-row scale s_bar.
 *
 * Parity pins: every exported function is pinned by a test that does not
 * retype its formula (brute-force enumeration, closed forms, exact rational
 * identities, an independent Philox implementation, numpy matmul).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 [Philox]. Counter (c0,c1,c2,c3), key (k0,k1).               */
/* ------------------------------------------------------------------------ */

#define PHILOX_MUL_0 0xD2511F53u
#define PHILOX_MUL_1 0xCD9E8D57u
#define PHILOX_WEYL_0 0x9E3779B9u
#define PHILOX_WEYL_1 0xBB67AE85u

/* One Philox4x32 round: two 32x32->64 products, then the S-box style
 * recombination of the high halves with the other two words and the key. */
static void philox_round(uint32_t c[4], const uint32_t k[2]) {
    uint64_t prod0 = (uint64_t)PHILOX_MUL_0 * (uint64_t)c[0];
    uint64_t prod1 = (uint64_t)PHILOX_MUL_1 * (uint64_t)c[2];
    uint32_t hi0 = (uint32_t)(prod0 >> 32), lo0 = (uint32_t)prod0;
    uint32_t hi1 = (uint32_t)(prod1 >> 32), lo1 = (uint32_t)prod1;
    uint32_t out0 = hi1 ^ c[1] ^ k[0];
    uint32_t out2 = hi0 ^ c[3] ^ k[1];
    c[0] = out0;
    c[1] = lo1;
    c[2] = out2;
    c[3] = lo0;
}

/* Ten rounds; the key is bumped by the Weyl constants between rounds. */
void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
    uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
    uint32_t k[2] = {key[0], key[1]};
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k[0] += PHILOX_WEYL_0;
            k[1] += PHILOX_WEYL_1;
        }
        philox_round(c, k);
    }
    memcpy(out, c, sizeof c);
}

/* The random word of flat element e = i*n + j of the auxiliary matrix:
 * block e/4 of the Philox stream (key = seed, counter = (e/4 low, e/4 high,
 * stream_id, 0)), word e mod 4. "R is regenerated online from a fixed seed,
 * with no storage" [IntLoRA notes, AQS]. */
uint32_t orc_aux_word(uint64_t seed, uint32_t stream_id, int64_t e) {
    uint64_t block = (uint64_t)e >> 2;
    uint32_t ctr[4] = {(uint32_t)block, (uint32_t)(block >> 32), stream_id, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    orc_philox4x32_10(ctr, key, out);
    return out[e & 3];
}

/* ------------------------------------------------------------------------ */
/* Laplace(0, 1) sample from one 32-bit word by the inverse CDF              */
/* [IntLoRA summary, Measured effects: Laplace auxiliary law].               */
/* u = (2*(x >> 9) + 1) * 2^-24 lies strictly inside (0, 1);                 */
/* v = u - 1/2 is never 0; R = -sign(v) * ln(1 - 2|v|).                      */
/* ------------------------------------------------------------------------ */
double orc_laplace_from_word(uint32_t x) {
    double u = (2.0 * (double)(x >> 9) + 1.0) * 0x1p-24;
    double v = u - 0.5;
    double sign_v = (v > 0.0) ? 1.0 : -1.0;
    return -sign_v * log(1.0 - 2.0 * fabs(v));
}

/* ------------------------------------------------------------------------ */
/* The auxiliary laws the ablation compares with Laplace [IntLoRA summary,   */
/* Measured effects: Gaussian, Cauchy and Student-t auxiliary matrices].     */
/* Each maps the same Philox words through u = (2 (x >> 9) + 1) 2^-24:      */
/*   Gaussian N(0,1): Box-Muller on the word pair (2p, 2p + 1) of a block,  */
/*     rho = sqrt(-2 ln u_2p); word 2p gets rho cos(2 pi u_2p+1), word 2p+1 */
/*     gets rho sin(2 pi u_2p+1);                                            */
/*   Cauchy(0,1): tan(pi (u - 1/2)) (inverse CDF);                           */
/*   Student-t with 2 degrees of freedom: (2u - 1) / sqrt(2 u (1 - u))       */
/*     (inverse CDF; the pages give no degrees of freedom: reading taken).   */
/* ------------------------------------------------------------------------ */
#define PI_F64 3.14159265358979323846264338327950288
#define DIST_LAPLACE 0
#define DIST_GAUSSIAN 1
#define DIST_CAUCHY 2
#define DIST_STUDENT_T2 3

static double unit_from_word(uint32_t x) { return (2.0 * (double)(x >> 9) + 1.0) * 0x1p-24; }

double orc_aux_value(uint64_t seed, uint32_t stream_id, int64_t e, int dist) {
    if (dist == DIST_LAPLACE) return orc_laplace_from_word(orc_aux_word(seed, stream_id, e));
    uint64_t block = (uint64_t)e >> 2;
    uint32_t ctr[4] = {(uint32_t)block, (uint32_t)(block >> 32), stream_id, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t w[4];
    orc_philox4x32_10(ctr, key, w);
    int c = (int)(e & 3);
    double u = unit_from_word(w[c]);
    if (dist == DIST_GAUSSIAN) {
        int p = c & ~1;
        double rho = sqrt(-2.0 * log(unit_from_word(w[p])));
        double theta = 2.0 * PI_F64 * unit_from_word(w[p + 1]);
        return (c & 1) ? rho * sin(theta) : rho * cos(theta);
    }
    if (dist == DIST_CAUCHY) return tan(PI_F64 * (u - 0.5));
    if (dist == DIST_STUDENT_T2) return (2.0 * u - 1.0) / sqrt(2.0 * u * (1.0 - u));
    return NAN;
}

/* R for count consecutive flat indices starting at e0. */
void orc_aux_block(uint64_t seed, uint32_t stream_id, int64_t e0, int64_t count, double* out,
                   int dist) {
    for (int64_t t = 0; t < count; ++t) out[t] = orc_aux_value(seed, stream_id, e0 + t, dist);
}

/* ------------------------------------------------------------------------ */
/* Population standard deviation, two passes (mean, then squared deviations) */
/* [IntLoRA notes, VMC: sigma_W and sigma_R].                                */
/* ------------------------------------------------------------------------ */
double orc_population_std(const double* x, int64_t count) {
    double sum = 0.0;
    for (int64_t t = 0; t < count; ++t) sum += x[t];
    double mean = sum / (double)count;
    double ssd = 0.0;
    for (int64_t t = 0; t < count; ++t) ssd += (x[t] - mean) * (x[t] - mean);
    return sqrt(ssd / (double)count);
}

/* sigma of an fp32 tensor of d rows of n values (row-major, dense). Each row
 * is summed in order; the row sums are then added in row order, so the value
 * does not depend on the number of threads. */
double orc_std_f32(const float* x, int64_t d, int64_t n) {
    double* row_acc = (double*)malloc(sizeof(double) * (size_t)d);
    double total = 0.0;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int64_t j = 0; j < n; ++j) acc += (double)x[i * n + j];
        row_acc[i] = acc;
    }
    for (int64_t i = 0; i < d; ++i) total += row_acc[i];
    double mean = total / ((double)d * (double)n);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            double dev = (double)x[i * n + j] - mean;
            acc += dev * dev;
        }
        row_acc[i] = acc;
    }
    double ssd = 0.0;
    for (int64_t i = 0; i < d; ++i) ssd += row_acc[i];
    free(row_acc);
    return sqrt(ssd / ((double)d * (double)n));
}

/* sigma_R of the regenerated d x n auxiliary matrix (two passes, each one
 * regenerating R; nothing is stored). */
double orc_sigma_r(int64_t d, int64_t n, uint64_t seed, uint32_t stream_id, int dist) {
    double* row_acc = (double*)malloc(sizeof(double) * (size_t)d);
    double total = 0.0;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int64_t j = 0; j < n; ++j)
            acc += orc_aux_value(seed, stream_id, i * n + j, dist);
        row_acc[i] = acc;
    }
    for (int64_t i = 0; i < d; ++i) total += row_acc[i];
    double mean = total / ((double)d * (double)n);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            double dev = orc_aux_value(seed, stream_id, i * n + j, dist) - mean;
            acc += dev * dev;
        }
        row_acc[i] = acc;
    }
    double ssd = 0.0;
    for (int64_t i = 0; i < d; ++i) ssd += row_acc[i];
    free(row_acc);
    return sqrt(ssd / ((double)d * (double)n));
}

/* VMC [IntLoRA notes, VMC]: R* = r^alpha * R with r = sigma_W / sigma_R. */
double orc_vmc_scale(double sigma_w, double sigma_r, double alpha) {
    return pow(sigma_w / sigma_r, alpha);
}

/* ------------------------------------------------------------------------ */
/* Asymmetric per-row uniform quantizer [Affine quant], used for W_round     */
/* (AQS: Q[W - sg(R)]) and for U_round (IntLoRA_MUL) [IntLoRA notes].        */
/* The range is [min(0, min x), max(0, max x)]; scale = range / (2^b - 1);   */
/* zero-point z = clamp(rne(-x_min / scale), 0, 2^b - 1);                    */
/* code = clamp(rne(x / scale) + z, 0, 2^b - 1).                             */
/* pre[j] receives x/scale and *zpre receives -x_min/scale (the values that  */
/* the rounding decides); either may be NULL.                                */
/* ------------------------------------------------------------------------ */
void orc_affine_quantize_row(const double* x, int64_t n, int bits, double* scale_out,
                             int32_t* zero_out, int32_t* codes, double* pre, double* zpre) {
    double qmax = ldexp(1.0, bits) - 1.0;
    double x_min = 0.0, x_max = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        if (x[j] < x_min) x_min = x[j];
        if (x[j] > x_max) x_max = x[j];
    }
    double scale = (x_max - x_min) / qmax;
    double zero;
    if (scale == 0.0) {
        scale = 1.0;
        zero = 0.0;
        if (zpre) *zpre = 0.0;
    } else {
        double zp = -x_min / scale;
        if (zpre) *zpre = zp;
        zero = nearbyint(zp);
        if (zero < 0.0) zero = 0.0;
        if (zero > qmax) zero = qmax;
    }
    for (int64_t j = 0; j < n; ++j) {
        double p = x[j] / scale;
        if (pre) pre[j] = p;
        double q = nearbyint(p) + zero;
        if (q < 0.0) q = 0.0;
        if (q > qmax) q = qmax;
        codes[j] = (int32_t)q;
    }
    *scale_out = scale;
    *zero_out = (int32_t)zero;
}

/* ------------------------------------------------------------------------ */
/* Layer preparation (AQS + VMC) [IntLoRA notes, AQS and VMC]:               */
/*   sigma_W = std(W), sigma_R = std(R), c = (sigma_W / sigma_R)^alpha,      */
/*   R* = c R, and W_round, s, z quantize X = W - R* row by row.             */
/* Only rows [row_begin, row_begin + row_count) are quantized; outputs are   */
/* for those rows (row-major, row_count x n). sigma values cover the whole   */
/* d x n layer.                                                              */
/* ------------------------------------------------------------------------ */
/* One row i of the base quantization: X_j = W_ij - c R_ij (flat index
 * e = i n + j), then the affine quantizer of the row. */
static void quantize_row(const float* W_row, int64_t n, uint64_t seed, uint32_t stream_id, double c,
                         int w_bits, int64_t i, double* r_star_row, int32_t* codes_row,
                         double* s_out, int32_t* z_out, double* pre_row, double* zpre, int dist) {
    double* x = (double*)malloc(sizeof(double) * (size_t)n);
    for (int64_t j = 0; j < n; ++j) {
        double r_star = c * orc_aux_value(seed, stream_id, i * n + j, dist);
        if (r_star_row) r_star_row[j] = r_star;
        x[j] = (double)W_row[j] - r_star;
    }
    orc_affine_quantize_row(x, n, w_bits, s_out, z_out, codes_row, pre_row, zpre);
    free(x);
}

void orc_gen_aux(const float* W, int64_t d, int64_t n, uint64_t seed, uint32_t stream_id,
                 double alpha, int w_bits, int64_t row_begin, int64_t row_count,
                 double* sigma_w_out, double* sigma_r_out, double* c_out,
                 double* r_star_out, int32_t* codes, double* s_out, int32_t* z_out,
                 double* pre, double* zpre, int dist) {
    double sigma_w = orc_std_f32(W, d, n);
    double sigma_r = orc_sigma_r(d, n, seed, stream_id, dist);
    double c = orc_vmc_scale(sigma_w, sigma_r, alpha);
    *sigma_w_out = sigma_w;
    *sigma_r_out = sigma_r;
    *c_out = c;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < row_count; ++t)
        quantize_row(&W[(row_begin + t) * n], n, seed, stream_id, c, w_bits, row_begin + t,
                     r_star_out ? &r_star_out[t * n] : NULL, &codes[t * n], &s_out[t], &z_out[t],
                     pre ? &pre[t * n] : NULL, zpre ? &zpre[t] : NULL, dist);
}

/* The same row quantization for rows whose W is given alone (W_rows holds
 * rows [row_begin, row_begin + row_count) of the layer) and whose VMC factor
 * c is given: layers too large to hold or reduce on the host. */
void orc_quantize_rows(const float* W_rows, int64_t n, uint64_t seed, uint32_t stream_id, double c,
                       int w_bits, int64_t row_begin, int64_t row_count, int32_t* codes,
                       double* s_out, int32_t* z_out, double* pre, double* zpre, int dist) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < row_count; ++t)
        quantize_row(&W_rows[t * n], n, seed, stream_id, c, w_bits, row_begin + t, NULL,
                     &codes[t * n], &s_out[t], &z_out[t], pre ? &pre[t * n] : NULL,
                     zpre ? &zpre[t] : NULL, dist);
}

/* ------------------------------------------------------------------------ */
/* Adaptation term of MLA [IntLoRA notes, MLA]:                              */
/*   U = s + (R* + A B) / (W_round - z),                                     */
/* with the quotient taken as 0 where W_round - z = 0. Computes U and the    */
/* integer term D = W_round - z for one row i.                               */
/* ------------------------------------------------------------------------ */
static void adaptation_row(const int32_t* codes_row, float s_i32, int32_t z_i, const float* A_row,
                           const float* B, int64_t n, int r, uint64_t seed, uint32_t stream_id,
                           double c, int64_t i, double* U, int64_t* D, int dist) {
    double s_i = (double)s_i32;
    for (int64_t j = 0; j < n; ++j) {
        double r_star = c * orc_aux_value(seed, stream_id, i * n + j, dist);
        double ab = 0.0;
        for (int k = 0; k < r; ++k) ab += (double)A_row[k] * (double)B[(int64_t)k * n + j];
        int64_t dij = (int64_t)codes_row[j] - (int64_t)z_i;
        D[j] = dij;
        U[j] = (dij != 0) ? s_i + (r_star + ab) / (double)dij : s_i;
    }
}

/* Pre-quantization MLA weight U * D for rows [row_begin, +row_count): the
 * value the MUL and SHIFT merges quantize. */
void orc_mla_rows(const int32_t* codes, int64_t ld_codes, const float* s, const int32_t* z,
                  const float* A, const float* B, int64_t d, int64_t n, int r, uint64_t seed,
                  uint32_t stream_id, double sigma_w, double sigma_r, double alpha,
                  int64_t row_begin, int64_t row_count, double* U_out, int64_t* D_out, int dist) {
    (void)d;
    double c = orc_vmc_scale(sigma_w, sigma_r, alpha);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < row_count; ++t)
        adaptation_row(&codes[(row_begin + t) * ld_codes], s[row_begin + t], z[row_begin + t],
                       &A[(row_begin + t) * r], B, n, r, seed, stream_id, c, row_begin + t,
                       &U_out[t * n], &D_out[t * n], dist);
}

/* ------------------------------------------------------------------------ */
/* IntLoRA_MUL [IntLoRA notes, 两种实现版本]:                                 */
/*   U is quantized per row by the affine quantizer (scale s_bar, zero-point */
/*   z_bar, codes U_round); the merged weight is                             */
/*   W' = s_bar * (U_round - z_bar) * (W_round - z), kept as the integer     */
/*   product P = (U_round - z_bar) * D and the per-row scale s_bar.          */
/* ------------------------------------------------------------------------ */
void orc_merge_mul_rows(const int32_t* codes_rows, int64_t ld_codes, const float* s_rows,
                        const int32_t* z_rows, const float* A_rows, const float* B, int64_t n,
                        int r, uint64_t seed, uint32_t stream_id, double c, int u_bits,
                        int64_t row_begin, int64_t row_count, int32_t* u_round, double* sbar,
                        int32_t* zbar, int64_t* P, double* pre, double* zpre, int dist);

void orc_merge_mul(const int32_t* codes, int64_t ld_codes, const float* s, const int32_t* z,
                   const float* A, const float* B, int64_t d, int64_t n, int r, uint64_t seed,
                   uint32_t stream_id, double sigma_w, double sigma_r, double alpha, int u_bits,
                   int64_t row_begin, int64_t row_count, double* U_out, int32_t* u_round,
                   double* sbar, int32_t* zbar, int64_t* P, double* pre, double* zpre, int dist) {
    (void)d;
    double c = orc_vmc_scale(sigma_w, sigma_r, alpha);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < row_count; ++t) {
        int64_t i = row_begin + t;
        double* U = (double*)malloc(sizeof(double) * (size_t)n);
        int64_t* D = (int64_t*)malloc(sizeof(int64_t) * (size_t)n);
        adaptation_row(&codes[i * ld_codes], s[i], z[i], &A[i * r], B, n, r, seed, stream_id, c, i,
                       U, D, dist);
        orc_affine_quantize_row(U, n, u_bits, &sbar[t], &zbar[t], &u_round[t * n],
                                pre ? &pre[t * n] : NULL, zpre ? &zpre[t] : NULL);
        for (int64_t j = 0; j < n; ++j) {
            if (U_out) U_out[t * n + j] = U[j];
            P[t * n + j] = ((int64_t)u_round[t * n + j] - (int64_t)zbar[t]) * D[j];
        }
        free(U);
        free(D);
    }
}

/* The MUL merge of rows whose inputs are given alone (codes_rows, s_rows,
 * z_rows, A_rows hold rows [row_begin, row_begin + row_count) of the layer)
 * and whose VMC factor c is given: layers too large for the host. */
void orc_merge_mul_rows(const int32_t* codes_rows, int64_t ld_codes, const float* s_rows,
                        const int32_t* z_rows, const float* A_rows, const float* B, int64_t n,
                        int r, uint64_t seed, uint32_t stream_id, double c, int u_bits,
                        int64_t row_begin, int64_t row_count, int32_t* u_round, double* sbar,
                        int32_t* zbar, int64_t* P, double* pre, double* zpre, int dist) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < row_count; ++t) {
        double* U = (double*)malloc(sizeof(double) * (size_t)n);
        int64_t* D = (int64_t*)malloc(sizeof(int64_t) * (size_t)n);
        adaptation_row(&codes_rows[t * ld_codes], s_rows[t], z_rows[t], &A_rows[t * r], B, n, r,
                       seed, stream_id, c, row_begin + t, U, D, dist);
        orc_affine_quantize_row(U, n, u_bits, &sbar[t], &zbar[t], &u_round[t * n],
                                pre ? &pre[t * n] : NULL, zpre ? &zpre[t] : NULL);
        for (int64_t j = 0; j < n; ++j)
            P[t * n + j] = ((int64_t)u_round[t * n + j] - (int64_t)zbar[t]) * D[j];
        free(U);
        free(D);
    }
}

/* ------------------------------------------------------------------------ */
/* IntLoRA_SHIFT [IntLoRA notes, 两种实现版本]:                               */
/*   W' = sign(V) * [(W_round - z) >> shift], a log2 quantizer of the        */
/*   adaptation term. V = U / s_bar with s_bar = max_j |U_ij| (so |V| <= 1);  */
/*   shift = clamp(nearest integer of -log2|V|, 0, 2^b - 1); ">>" is floor   */
/*   division by 2^shift. The merged weight is s_bar * M with                 */
/*   M = sign(V) * (D >> shift). pre[j] receives -log2|V| (+inf where V = 0). */
/* ------------------------------------------------------------------------ */
/* The SHIFT quantizer of one row: given U and D, writes s_bar, the shift
 * codes and M. pre[j] (nullable) receives -log2|V_j| (+inf where V_j = 0). */
void orc_shift_quantize_row(const double* U, const int64_t* D, int64_t n, int shift_bits,
                            double* sbar_out, int32_t* shift, int64_t* M, double* pre) {
    double shift_max = ldexp(1.0, shift_bits) - 1.0;
    double umax = 0.0;
    for (int64_t j = 0; j < n; ++j)
        if (fabs(U[j]) > umax) umax = fabs(U[j]);
    if (umax == 0.0) umax = 1.0;
    *sbar_out = umax;
    for (int64_t j = 0; j < n; ++j) {
        double v = U[j] / umax;
        double sign_v = (v > 0.0) ? 1.0 : ((v < 0.0) ? -1.0 : 0.0);
        double tlog = (v != 0.0) ? -log2(fabs(v)) : INFINITY;
        if (pre) pre[j] = tlog;
        double k = (v != 0.0) ? nearbyint(tlog) : shift_max;
        if (k < 0.0) k = 0.0;
        if (k > shift_max) k = shift_max;
        double shifted = floor((double)D[j] / ldexp(1.0, (int)k));
        shift[j] = (int32_t)k;
        M[j] = (int64_t)(sign_v * shifted);
    }
}

void orc_merge_shift(const int32_t* codes, int64_t ld_codes, const float* s, const int32_t* z,
                     const float* A, const float* B, int64_t d, int64_t n, int r, uint64_t seed,
                     uint32_t stream_id, double sigma_w, double sigma_r, double alpha,
                     int shift_bits, int64_t row_begin, int64_t row_count, double* U_out,
                     double* sbar, int32_t* shift, int64_t* M, double* pre, int dist) {
    (void)d;
    double c = orc_vmc_scale(sigma_w, sigma_r, alpha);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < row_count; ++t) {
        int64_t i = row_begin + t;
        double* U = (double*)malloc(sizeof(double) * (size_t)n);
        int64_t* D = (int64_t*)malloc(sizeof(int64_t) * (size_t)n);
        adaptation_row(&codes[i * ld_codes], s[i], z[i], &A[i * r], B, n, r, seed, stream_id, c, i,
                       U, D, dist);
        orc_shift_quantize_row(U, D, n, shift_bits, &sbar[t], &shift[t * n], &M[t * n],
                               pre ? &pre[t * n] : NULL);
        if (U_out)
            for (int64_t j = 0; j < n; ++j) U_out[t * n + j] = U[j];
        free(U);
        free(D);
    }
}

/* ------------------------------------------------------------------------ */
/* STE backward [IntLoRA notes, "训练时使用 STE"]: the straight-through        */
/* estimator passes the upstream gradient G on W' to A B unchanged, so       */
/*   dA = G B^T  (d x r),   dB = A^T G  (r x n).                             */
/* Inputs are fp64 copies of the bf16 tensors.                               */
/* ------------------------------------------------------------------------ */
void orc_ste_backward(const double* G, const double* A, const double* B, int64_t d, int64_t n,
                      int r, double* dA, double* dB) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d; ++i)
        for (int k = 0; k < r; ++k) {
            double acc = 0.0;
            for (int64_t j = 0; j < n; ++j) acc += G[i * n + j] * B[(int64_t)k * n + j];
            dA[i * r + k] = acc;
        }
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j)
        for (int k = 0; k < r; ++k) {
            double acc = 0.0;
            for (int64_t i = 0; i < d; ++i) acc += A[i * r + k] * G[i * n + j];
            dB[(int64_t)k * n + j] = acc;
        }
}

/* Sampled STE outputs for full-size layers: rows of dA and columns of dB.
 * G is bf16 stored as uint16 (upper half of the fp32 pattern); A, B too. */
static double bf16_value(uint16_t h) {
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

void orc_ste_sampled(const uint16_t* G, const uint16_t* A, const uint16_t* B, int64_t d, int64_t n,
                     int r, const int64_t* rows, int64_t n_rows, const int64_t* cols,
                     int64_t n_cols, double* dA_rows, double* dB_cols) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < n_rows; ++t) {
        int64_t i = rows[t];
        for (int k = 0; k < r; ++k) {
            double acc = 0.0;
            for (int64_t j = 0; j < n; ++j)
                acc += bf16_value(G[i * n + j]) * bf16_value(B[(int64_t)k * n + j]);
            dA_rows[t * r + k] = acc;
        }
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < n_cols; ++t) {
        int64_t j = cols[t];
        for (int k = 0; k < r; ++k) {
            double acc = 0.0;
            for (int64_t i = 0; i < d; ++i)
                acc += bf16_value(A[i * r + k]) * bf16_value(G[i * n + j]);
            dB_cols[t * r + k] = acc;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Integer inference on the merged weights [IntLoRA notes, "两种实现版本" and */
/* the efficiency table: the merged weight s_bar_i Q_ij is already integer,   */
/* so a layer runs as an integer GEMM with no post-training quantization].    */
/* ------------------------------------------------------------------------ */

/* Digits of an integer weight in base 128 for an 8-bit integer MMA: with P
 * planes, digit k < P-1 is (w >> 7k) & 127 and the top digit is w >> 7(P-1)
 * (arithmetic shift), so w = sum_k 128^k digit_k. Layout [d][P][n]. Returns
 * the number of weights whose top digit leaves [-128, 127] (stored truncated). */
int64_t orc_int_digits(const int64_t* w, int64_t d, int64_t n, int planes, int8_t* out) {
    int64_t bad = 0;
    for (int64_t i = 0; i < d; ++i)
        for (int64_t j = 0; j < n; ++j) {
            int64_t v = w[i * n + j];
            for (int k = 0; k < planes; ++k) {
                int64_t digit = k < planes - 1 ? (v >> (7 * k)) & 127 : v >> (7 * k);
                if (k == planes - 1 && (digit < -128 || digit > 127)) ++bad;
                out[(i * planes + k) * n + j] = (int8_t)digit;
            }
        }
    return bad;
}

/* Y[t][i] = x_scale[t] * w_scale[i] * sum_j X[t][j] W[i][j] for the listed
 * token rows: the integer sum is exact (int64), the scaling is fp64. */
void orc_int_gemm_rows(const int8_t* X, const double* x_scale, const int64_t* W,
                       const double* w_scale, int64_t tokens, int64_t d, int64_t n,
                       const int64_t* rows, int64_t n_rows, double* Y) {
    (void)tokens;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t q = 0; q < n_rows * d; ++q) {
        int64_t t = rows[q / d], i = q % d;
        int64_t acc = 0;
        for (int64_t j = 0; j < n; ++j) acc += (int64_t)X[t * n + j] * W[i * n + j];
        Y[q] = (double)acc * x_scale[t] * w_scale[i];
    }
}

/* ------------------------------------------------------------------------ */
/* Training forward on the merged weights [IntLoRA notes, 两种实现版本 and    */
/* the efficiency table]: the merged weight enters the layer GEMM as bf16.   */
/* ------------------------------------------------------------------------ */

/* bf16 of an fp32 value: round to nearest with ties to even on the upper 16
 * bits of the pattern (finite values). */
static uint16_t bf16_rne(float f) {
    uint32_t b;
    memcpy(&b, &f, sizeof b);
    b += 0x7FFFu + ((b >> 16) & 1u);
    return (uint16_t)(b >> 16);
}

/* W'_bf16[i][j] = bf16(fp32(s_bar_i * Q_ij)): the fp32 product, then bf16. */
void orc_fakequant_bf16(const int64_t* Q, const float* sbar, int64_t d, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < d; ++i)
        for (int64_t j = 0; j < n; ++j) {
            float w = sbar[i] * (float)Q[i * n + j];
            out[i * n + j] = bf16_rne(w);
        }
}

static double bf16_to_f64(uint16_t h) {
    uint32_t b = (uint32_t)h << 16;
    float f;
    memcpy(&f, &b, sizeof f);
    return (double)f;
}

/* Y[t][i] = sum_j X[t][j] W[i][j] in fp64 for the listed token rows (X, W
 * bf16 patterns). */
void orc_linear_rows(const uint16_t* X, const uint16_t* W, int64_t tokens, int64_t d, int64_t n,
                     const int64_t* rows, int64_t n_rows, double* Y) {
    (void)tokens;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t q = 0; q < n_rows * d; ++q) {
        int64_t t = rows[q / d], i = q % d;
        double acc = 0.0;
        for (int64_t j = 0; j < n; ++j) acc += bf16_to_f64(X[t * n + j]) * bf16_to_f64(W[i * n + j]);
        Y[q] = acc;
    }
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads of the calling thread's later parallel regions (n >= 1); the
 * benchmark's single-core figure uses it. No arithmetic depends on it: every
 * parallel loop above writes disjoint outputs, each computed in one thread. */
void orc_set_num_threads(int n) {
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
