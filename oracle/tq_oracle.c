/*
 * tq_oracle.c -- plain, slow CPU oracle for the TQ4_1S weight codec and its
 * dequant-GEMV.  TEST INFRASTRUCTURE ONLY: nothing in the product path may link,
 * load or call this file.  It shares no code, header, table or constant
 * generator with the CUDA library; only the seeded input generators are common.
 *
 * Citations name web pages by title.  "TQ page" is the page titled
 * "企业官网建设流程全解析" (hotelren.com/news/5458160), whose body describes the
 * TQ4_1S codec; its relevant parts are the paragraph "格式原理" (items 1-3 and the
 * paragraph after them) and the section "解码速度：分硬件汇总".
 *
 * Arithmetic contract: every float (fp32) operation below is one IEEE-754
 * binary32 operation rounded to nearest-even (compile with -ffp-contract=off,
 * no -ffast-math, no FTZ/DAZ).  fp64 is used where the codec does not fix
 * the precision (codebook construction, dequantisation, matrix products).
 *
 * Readings of points the pages leave open (each is also listed in the design
 * notes of the repository):
 *   - sign pattern: golden-ratio (Fibonacci) multiplicative hash of the global
 *     column index, followed by one MurmurHash3-style mixing round, bit 31;
 *   - Hadamard matrix: unnormalised Sylvester H (H H^T = 32 I), inverse = H/32;
 *   - half-block scale: fp16(RMS of the 16 rotated coordinates), rounded
 *     to nearest-even;
 *   - code: 1 sign bit (bit 3, 1 = negative) + 3-bit magnitude rank,
 *     magnitude = number of thresholds strictly exceeded (ties go down);
 *   - packing: superblocks of four 32-element blocks (64 code bytes + 4x2
 *     fp16 scales); byte order inside a superblock chosen for 128-bit loads.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define TQO_BLOCK 32
#define TQO_HALF 16
#define TQO_SB_BLOCKS 4

/* ------------------------------------------------------------------------ */
/* Standard normal density / tail helpers (fp64, libm erfc).                 */
/* ------------------------------------------------------------------------ */
static double tqo_phi(double x) {
    if (isinf(x)) return 0.0;
    return exp(-0.5 * x * x) / sqrt(2.0 * M_PI);
}

/* Upper tail Q(x) = P(Z > x). */
static double tqo_q(double x) { return 0.5 * erfc(x / sqrt(2.0)); }

/* P(a < Z < b), evaluated on the side that avoids cancellation. */
static double tqo_cell_prob(double a, double b) {
    if (a >= 0.0) return tqo_q(a) - tqo_q(b);
    if (b <= 0.0) return tqo_q(-b) - tqo_q(-a);
    return 1.0 - tqo_q(b) - tqo_q(-a);
}

static double tqo_xphi(double x) { return isinf(x) ? 0.0 : x * tqo_phi(x); }

/*
 * Lloyd-Max scalar quantiser for N(0,1) with L levels (TQ page, 格式原理 item 2:
 * each rotated coordinate goes to the nearest optimal centroid of N(0,1); the
 * paragraph after the items says the codebook is built with Lloyd's algorithm).
 *
 * Lloyd's two alternating conditions: thresholds are midpoints of neighbouring
 * centroids; each centroid is the conditional mean of its cell, which for the
 * Gaussian is (phi(a) - phi(b)) / (Phi(b) - Phi(a)).  Start: L evenly spaced
 * points on [-3, 3].  Stop when no centroid moves by more than 1e-15.
 *
 * Output: centroids (ascending), the mean squared error of the quantiser
 * (closed form: per cell  P + a phi(a) - b phi(b) - 2c (phi(a)-phi(b)) + c^2 P),
 * and the iteration count.  Returns 0 on convergence, 1 if max_iter is hit.
 */
int tqo_lloyd(int L, int max_iter, double *centroids, double *mse_out, int *iters_out) {
    if (L < 1 || L > 256) return 2;
    double c[256], t[257];
    for (int i = 0; i < L; ++i) c[i] = -3.0 + 6.0 * (i + 0.5) / L;
    int it = 0, converged = 0;
    for (it = 0; it < max_iter; ++it) {
        t[0] = -INFINITY;
        t[L] = INFINITY;
        for (int i = 1; i < L; ++i) t[i] = 0.5 * (c[i - 1] + c[i]);
        double delta = 0.0;
        for (int i = 0; i < L; ++i) {
            double p = tqo_cell_prob(t[i], t[i + 1]);
            double next = (tqo_phi(t[i]) - tqo_phi(t[i + 1])) / p;
            double d = fabs(next - c[i]);
            if (d > delta) delta = d;
            c[i] = next;
        }
        if (delta < 1e-15) { converged = 1; ++it; break; }
    }
    /* thresholds consistent with the final centroids */
    t[0] = -INFINITY;
    t[L] = INFINITY;
    for (int i = 1; i < L; ++i) t[i] = 0.5 * (c[i - 1] + c[i]);
    double mse = 0.0;
    for (int i = 0; i < L; ++i) {
        double a = t[i], b = t[i + 1], p = tqo_cell_prob(a, b);
        mse += p + tqo_xphi(a) - tqo_xphi(b) - 2.0 * c[i] * (tqo_phi(a) - tqo_phi(b)) + c[i] * c[i] * p;
    }
    for (int i = 0; i < L; ++i) centroids[i] = c[i];
    if (mse_out) *mse_out = mse;
    if (iters_out) *iters_out = it;
    return converged ? 0 : 1;
}

/*
 * The TQ4_1S codebook (TQ page, paragraph after 格式原理: 16 optimal centroids,
 * no correction term).  The 16-level table is symmetric, so it is kept as
 * eight magnitudes M[0..7] (ascending) with the sign carried separately.
 *   M32[j] = fp32(M64[j])                        (round to nearest-even)
 *   B32[j] = fp32((M64[j] + M64[j+1]) / 2), j=0..6 (decision thresholds)
 */
int tqo_codebook(float *M32, float *B32, double *M64) {
    /* computed once per process; the iteration is deterministic */
    static int ready = 0, rc = 0;
    static double c[16];
    if (!ready) {
        rc = tqo_lloyd(16, 1000000, c, NULL, NULL);
        ready = 1;
    }
    for (int j = 0; j < 8; ++j) {
        M64[j] = c[8 + j];
        M32[j] = (float)c[8 + j];
    }
    for (int j = 0; j < 7; ++j) B32[j] = (float)(0.5 * (c[8 + j] + c[9 + j]));
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Sign pattern (TQ page, 格式原理 item 1: randomised Hadamard transform with  */
/* golden-ratio sign flips).  Depends on the global column index only, so one */
/* pre-rotated activation serves every output row.                            */
/* ------------------------------------------------------------------------ */
uint32_t tqo_sign_hash(uint32_t k) {
    uint32_t h = k * 0x9E3779B9u; /* floor(2^32 / golden ratio) */
    h ^= h >> 16;
    h *= 0x85EBCA6Bu;
    h ^= h >> 13;
    return h;
}

/* -1 if bit 31 of the hash is set, else +1 */
int tqo_sign(uint32_t k) { return (tqo_sign_hash(k) >> 31) ? -1 : 1; }

/* ------------------------------------------------------------------------ */
/* 32-point fast Walsh-Hadamard transform, unnormalised Sylvester order.      */
/* Stages h = 1, 2, 4, 8, 16; in each stage every pair (i, i+h) with          */
/* (i & h) == 0 becomes (a + b, a - b).  (TQ page, paragraph after 格式原理:  */
/* fast structured rotation, O(d log d).)                                     */
/* ------------------------------------------------------------------------ */
void tqo_fwht32_f32(float *v) {
    for (int h = 1; h < TQO_BLOCK; h <<= 1)
        for (int i = 0; i < TQO_BLOCK; ++i)
            if ((i & h) == 0) {
                float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
}

void tqo_fwht32_f64(double *v) {
    for (int h = 1; h < TQO_BLOCK; h <<= 1)
        for (int i = 0; i < TQO_BLOCK; ++i)
            if ((i & h) == 0) {
                double a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
}

/* ------------------------------------------------------------------------ */
/* IEEE binary16 conversions, written out from the format definition.         */
/* ------------------------------------------------------------------------ */
uint16_t tqo_f32_to_f16(float x) {
    uint32_t u;
    memcpy(&u, &x, 4);
    uint32_t sign = (u >> 16) & 0x8000u;
    uint32_t a = u & 0x7FFFFFFFu;
    if (a > 0x7F800000u) return (uint16_t)(sign | 0x7E00u); /* NaN */
    if (a >= 0x477FF000u) return (uint16_t)(sign | 0x7C00u); /* >= 65520 rounds to inf */
    if (a >= 0x38800000u) {                                  /* normal half: >= 2^-14 */
        uint32_t e = (a >> 23) - 127 + 15;
        uint32_t mant = a & 0x7FFFFFu;
        uint32_t r = (e << 10) | (mant >> 13);
        uint32_t rem = mant & 0x1FFFu;
        if (rem > 0x1000u || (rem == 0x1000u && (r & 1u))) r += 1; /* carry into exponent is correct */
        return (uint16_t)(sign | r);
    }
    if (a < 0x00800000u) return (uint16_t)sign; /* fp32 zero/subnormal: far below half's range */
    /* half subnormal: result = round(x * 2^24) in units of 2^-24 */
    int e = (int)(a >> 23) - 127;       /* x = sig * 2^(e-23), sig in [2^23, 2^24) */
    uint32_t sig = (a & 0x7FFFFFu) | 0x800000u;
    int s = -(e + 1);                    /* x * 2^24 = sig >> s */
    if (s >= 25) return (uint16_t)sign;  /* < 0.5 unit: rounds to zero */
    uint32_t q = sig >> s, rem = sig & ((1u << s) - 1u), half = 1u << (s - 1);
    if (rem > half || (rem == half && (q & 1u))) q += 1;
    return (uint16_t)(sign | q);
}

float tqo_f16_to_f32(uint16_t h) {
    uint32_t sign = ((uint32_t)h & 0x8000u) << 16;
    uint32_t e = (h >> 10) & 0x1Fu, m = h & 0x3FFu;
    float mag;
    if (e == 0) mag = ldexpf((float)m, -24);
    else if (e == 31) mag = m ? NAN : INFINITY;
    else mag = ldexpf((float)(m | 0x400u), (int)e - 25);
    uint32_t u;
    memcpy(&u, &mag, 4);
    u |= sign;
    float out;
    memcpy(&out, &u, 4);
    return out;
}

/* ------------------------------------------------------------------------ */
/* Quantise one 32-element block.  w: the 32 source weights (fp32), k0: the   */
/* global column of w[0].  Output: logical codes code[e] (e = element index)  */
/* and the two fp16 scale bit patterns d[0] (elements 0-15), d[1] (16-31).    */
/*   1. u_e = s(k0+e) * w_e                       (TQ page 格式原理 item 1)    */
/*   2. y = H u  (fwht32_f32)                     (item 1)                     */
/*   3. d_h = fp16(sqrt(S_h * 0.0625)), S_h = pairwise sum of y_e^2 over the   */
/*      half, adjacent order ((q0+q1)+(q2+q3))+...  (item 3: dual half scales) */
/*   4. t_j = B32[j] * D_h, D_h = float(d_h); mag = #{j : |y_e| > t_j};        */
/*      code = 8*(y_e < 0) + mag                  (item 2: nearest centroid)  */
/* ------------------------------------------------------------------------ */
void tqo_quantize_block(const float *w, uint32_t k0, const float *B32, uint8_t *code, uint16_t *d) {
    float y[TQO_BLOCK];
    for (int e = 0; e < TQO_BLOCK; ++e) y[e] = tqo_sign(k0 + (uint32_t)e) < 0 ? -w[e] : w[e];
    tqo_fwht32_f32(y);
    for (int h = 0; h < 2; ++h) {
        float s[TQO_HALF];
        for (int e = 0; e < TQO_HALF; ++e) s[e] = y[h * TQO_HALF + e] * y[h * TQO_HALF + e];
        for (int step = 1; step < TQO_HALF; step <<= 1)
            for (int i = 0; i < TQO_HALF; i += 2 * step) s[i] = s[i] + s[i + step];
        float ms = s[0] * 0.0625f;
        d[h] = tqo_f32_to_f16(sqrtf(ms));
    }
    for (int e = 0; e < TQO_BLOCK; ++e) {
        float D = tqo_f16_to_f32(d[e / TQO_HALF]);
        float ay = fabsf(y[e]);
        int mag = 0;
        for (int j = 0; j < 7; ++j) {
            float t = B32[j] * D;
            if (ay > t) ++mag;
        }
        code[e] = (uint8_t)((y[e] < 0.0f ? 8 : 0) + mag);
    }
}

/* ------------------------------------------------------------------------ */
/* Packed layout (the repository's stated format; the pages fix only "16     */
/* optimal centroids + clean nibble packing + no correction term", TQ page).  */
/*   Rows are grouped in tiles of 16 (T = ceil(N/16)); each row has           */
/*   NSB = ceil(K/128) superblocks of four blocks.  A unit = (tile, sb) is     */
/*   stored contiguously, units in tile-major order:                           */
/*     codes  [T][NSB][16 rows][64 B]   scales [T][NSB][16 rows][4 blocks][2]  */
/*   Inside a row's 64-byte superblock, logical byte L (0..15) of block j is   */
/*   code[2L] | code[2L+1] << 4 and sits at byte 16*(L % 4) + 4*j + L / 4.     */
/*   Blocks past K/32 and rows past N are zero codes with zero scales.        */
/* ------------------------------------------------------------------------ */
int64_t tqo_superblocks(int64_t k) { return (k / TQO_BLOCK + TQO_SB_BLOCKS - 1) / TQO_SB_BLOCKS; }

int64_t tqo_tiles(int64_t n) { return (n + 15) / 16; }

static int64_t tqo_unit_row(int64_t nsb, int64_t row, int64_t blk) {
    int64_t sb = blk / TQO_SB_BLOCKS;
    return ((row / 16) * nsb + sb) * 16 + row % 16; /* index of the row's 64-byte slot */
}

static int64_t tqo_code_offset(int64_t nsb, int64_t row, int64_t blk, int L) {
    int64_t j = blk % TQO_SB_BLOCKS;
    return tqo_unit_row(nsb, row, blk) * 64 + 16 * (L % 4) + 4 * j + L / 4;
}

static int64_t tqo_scale_offset(int64_t nsb, int64_t row, int64_t blk, int h) {
    int64_t j = blk % TQO_SB_BLOCKS;
    return tqo_unit_row(nsb, row, blk) * 8 + 2 * j + h;
}

/* W: fp32, n x k, leading dimension ldw (elements).  codes: T*NSB*1024 bytes,
 * scales: T*NSB*128 uint16.  Returns 0, or 1 if k % 32 != 0. */
int tqo_quantize(const float *W, int64_t n, int64_t k, int64_t ldw, uint8_t *codes, uint16_t *scales) {
    if (k % TQO_BLOCK != 0 || n < 0) return 1;
    float M32[8], B32[7];
    double M64[8];
    tqo_codebook(M32, B32, M64);
    int64_t nsb = tqo_superblocks(k), nb = k / TQO_BLOCK;
    memset(codes, 0, (size_t)(tqo_tiles(n) * nsb * 1024));
    memset(scales, 0, (size_t)(tqo_tiles(n) * nsb * 128) * sizeof(uint16_t));
    for (int64_t r = 0; r < n; ++r)
        for (int64_t b = 0; b < nb; ++b) {
            uint8_t code[TQO_BLOCK];
            uint16_t d[2];
            tqo_quantize_block(W + r * ldw + b * TQO_BLOCK, (uint32_t)(b * TQO_BLOCK), B32, code, d);
            for (int L = 0; L < 16; ++L)
                codes[tqo_code_offset(nsb, r, b, L)] = (uint8_t)(code[2 * L] | (code[2 * L + 1] << 4));
            scales[tqo_scale_offset(nsb, r, b, 0)] = d[0];
            scales[tqo_scale_offset(nsb, r, b, 1)] = d[1];
        }
    return 0;
}

/* Inverse of the packing: logical codes [n][k] (one code per element) and
 * logical scales [n][k/32][2]. */
void tqo_unpack(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, uint8_t *code_out,
                uint16_t *d_out) {
    int64_t nsb = tqo_superblocks(k), nb = k / TQO_BLOCK;
    for (int64_t r = 0; r < n; ++r)
        for (int64_t b = 0; b < nb; ++b) {
            for (int L = 0; L < 16; ++L) {
                uint8_t byte = codes[tqo_code_offset(nsb, r, b, L)];
                code_out[r * k + b * TQO_BLOCK + 2 * L] = byte & 15;
                code_out[r * k + b * TQO_BLOCK + 2 * L + 1] = byte >> 4;
            }
            d_out[(r * nb + b) * 2] = scales[tqo_scale_offset(nsb, r, b, 0)];
            d_out[(r * nb + b) * 2 + 1] = scales[tqo_scale_offset(nsb, r, b, 1)];
        }
}

/*
 * Dequantise (TQ page, paragraph after 格式原理: the reference dequantiser
 * inverse-rotates and rescales).  In fp64, exactly:
 *   c_e = (code_e & 8 ? -1 : 1) * M32[code_e & 7] * D_h(e)
 *   w~  = s (.) (H c) / 32
 * W: fp64, n x k, leading dimension ldw.
 */
void tqo_dequantize(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, double *W, int64_t ldw) {
    float M32[8], B32[7];
    double M64[8];
    tqo_codebook(M32, B32, M64);
    int64_t nsb = tqo_superblocks(k), nb = k / TQO_BLOCK;
    for (int64_t r = 0; r < n; ++r)
        for (int64_t b = 0; b < nb; ++b) {
            double v[TQO_BLOCK];
            for (int L = 0; L < 16; ++L) {
                uint8_t byte = codes[tqo_code_offset(nsb, r, b, L)];
                for (int q = 0; q < 2; ++q) {
                    int e = 2 * L + q;
                    int code = q ? (byte >> 4) : (byte & 15);
                    double D = (double)tqo_f16_to_f32(scales[tqo_scale_offset(nsb, r, b, e / TQO_HALF)]);
                    double c = (double)M32[code & 7] * D;
                    v[e] = (code & 8) ? -c : c;
                }
            }
            tqo_fwht32_f64(v);
            for (int e = 0; e < TQO_BLOCK; ++e) {
                double w = v[e] / 32.0;
                W[r * ldw + b * TQO_BLOCK + e] = tqo_sign((uint32_t)(b * TQO_BLOCK + e)) < 0 ? -w : w;
            }
        }
}

/*
 * Reference matrix product over the dequantised weights, in fp64:
 *   Y[m][r] = sum_k  w~[r][k] * X[m][k]       (r = output row of W)
 * X: fp64 [m][ldx], Y: fp64 [m][ldy].  This is the plain definition of what
 * the fused kernel computes; the pre-rotation in the TQ page's 解码速度 section
 * is an algebraic rearrangement of the same sum.
 */
void tqo_gemm(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const double *X, int64_t m,
              int64_t ldx, double *Y, int64_t ldy) {
    double *w = (double *)malloc((size_t)(k > 0 ? k : 1) * sizeof(double));
    double *tile = (double *)malloc((size_t)16 * (size_t)(k > 0 ? k : 1) * sizeof(double));
    int64_t nsb = tqo_superblocks(k);
    for (int64_t r = 0; r < n; ++r) {
        /* dequantise the row's 16-row tile, keep row r */
        if (r % 16 == 0) tqo_dequantize(codes + (r / 16) * nsb * 1024, scales + (r / 16) * nsb * 128, 16, k, tile, k);
        memcpy(w, tile + (r % 16) * k, (size_t)k * sizeof(double));
        for (int64_t i = 0; i < m; ++i) {
            double acc = 0.0;
            for (int64_t c = 0; c < k; ++c) acc += w[c] * X[i * ldx + c];
            Y[i * ldy + r] = acc;
        }
    }
    free(w);
    free(tile);
}

/* ======================================================================== */
/* NVFP4 comparison codec (the llm-compressor and llama.cpp-quantizer pages */
/* name NVFP4 checkpoints and "weight and input tensor scales"; the pages   */
/* give no bit recipe, so this is the plainest reading of the format):      */
/*   g   = amax|W| / (6 * 448)                      per-tensor fp32 scale    */
/*   s_b = e4m3_rne_satfinite(amax_b / (6 * g))      per 16-element block     */
/*   q   = e2m1_rne_satfinite(w / (s_b * g))         per element (0 if s_b=0) */
/*   w~  = q * s_b * g                                                       */
/* Every quotient / product is one IEEE fp32 operation in that order.       */
/* ======================================================================== */

/* E4M3 (bias 7, no infinities, max 448): value of an 8-bit code. */
float tqo_e4m3_to_f32(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    float v;
    if (e == 15 && m == 7) v = NAN;
    else if (e == 0) v = ldexpf((float)m, -9);
    else v = ldexpf((float)(8 + m), e - 10);
    return s ? -v : v;
}

/* Nearest E4M3 code, ties to the even code, finite values above 448 saturate. */
uint8_t tqo_e4m3_from_f32(float x) {
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    float a = fabsf(x);
    if (a >= 448.0f) return sign | 0x7E;
    /* scan the 127 finite magnitudes in increasing order */
    uint8_t best = 0;
    for (int c = 1; c <= 0x7E; ++c) {
        float v = tqo_e4m3_to_f32((uint8_t)c);
        if (v <= a) best = (uint8_t)c;
    }
    if (best == 0x7E) return sign | best;
    float lo = tqo_e4m3_to_f32(best), hi = tqo_e4m3_to_f32((uint8_t)(best + 1));
    double dl = (double)a - lo, dh = (double)hi - a;
    uint8_t r = best;
    if (dh < dl || (dh == dl && (best & 1))) r = (uint8_t)(best + 1);
    return sign | r;
}

/* E2M1 magnitudes by 3-bit code: 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
float tqo_e2m1_to_f32(uint8_t c) {
    static const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
    float v = mag[c & 7];
    return (c & 8) ? -v : v;
}

/* Nearest E2M1 code (bit 3 = sign), ties to the even code, saturating at 6.
 * -0 and +0 both map to code 0 (a zero carries no sign). */
uint8_t tqo_e2m1_from_f32(float x) {
    uint8_t sign = (x < 0.0f) ? 8 : 0;
    float a = fabsf(x);
    if (a >= 6.0f) return sign | 7;
    uint8_t best = 0;
    for (int c = 1; c <= 7; ++c)
        if (tqo_e2m1_to_f32((uint8_t)c) <= a) best = (uint8_t)c;
    uint8_t r = best;
    if (best < 7) {
        float lo = tqo_e2m1_to_f32(best), hi = tqo_e2m1_to_f32((uint8_t)(best + 1));
        float dl = a - lo, dh = hi - a; /* exact: all operands are short binary fractions */
        if (dh < dl || (dh == dl && (best & 1))) r = (uint8_t)(best + 1);
    }
    return r == 0 ? 0 : (uint8_t)(sign | r);
}

/* Packed NVFP4 layout (this repository's): the same tile-major units as
 * TQ4_1S -- codes [T][NSB][16 rows][64 B] with the same byte order inside a
 * row's 64 bytes (a pair of 16-element blocks plays the role of one 32-element
 * block), scales E4M3 [T][NSB][16 rows][8 blocks], plus one fp32 tensor scale.
 * k must be a multiple of 32.  4.5 bits per weight. */
static int64_t tqo_nv_scale_offset(int64_t nsb, int64_t row, int64_t blk16) {
    int64_t sb = blk16 / 8;
    return (((row / 16) * nsb + sb) * 16 + row % 16) * 8 + blk16 % 8;
}

int tqo_nvfp4_quantize(const float *W, int64_t n, int64_t k, int64_t ldw, uint8_t *codes, uint8_t *scales,
                       float *g_out) {
    if (k % TQO_BLOCK != 0 || n < 0) return 1;
    int64_t nsb = tqo_superblocks(k), nb16 = k / 16;
    memset(codes, 0, (size_t)(tqo_tiles(n) * nsb * 1024));
    memset(scales, 0, (size_t)(tqo_tiles(n) * nsb * 128));
    float amax = 0.0f;
    for (int64_t r = 0; r < n; ++r)
        for (int64_t c = 0; c < k; ++c) {
            float a = fabsf(W[r * ldw + c]);
            if (a > amax) amax = a;
        }
    float g = amax / (6.0f * 448.0f);
    *g_out = g;
    float denom = 6.0f * g;
    for (int64_t r = 0; r < n; ++r)
        for (int64_t b = 0; b < nb16; ++b) {
            const float *w = W + r * ldw + b * 16;
            float am = 0.0f;
            for (int e = 0; e < 16; ++e)
                if (fabsf(w[e]) > am) am = fabsf(w[e]);
            uint8_t s = (denom > 0.0f) ? tqo_e4m3_from_f32(am / denom) : 0;
            float scale = tqo_e4m3_to_f32(s) * g;
            scales[tqo_nv_scale_offset(nsb, r, b)] = s;
            for (int e = 0; e < 16; ++e) {
                uint8_t q = (scale > 0.0f) ? tqo_e2m1_from_f32(w[e] / scale) : 0;
                int64_t blk32 = b / 2;
                int el = (int)(b % 2) * 16 + e; /* element index inside the 32-column pair */
                int L = el / 2;
                int64_t off = tqo_code_offset(nsb, r, blk32, L);
                codes[off] |= (uint8_t)((el & 1) ? (q << 4) : q);
            }
        }
    return 0;
}

void tqo_nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales, float g, int64_t n, int64_t k, double *W,
                          int64_t ldw) {
    int64_t nsb = tqo_superblocks(k), nb16 = k / 16;
    for (int64_t r = 0; r < n; ++r)
        for (int64_t b = 0; b < nb16; ++b) {
            double s = (double)tqo_e4m3_to_f32(scales[tqo_nv_scale_offset(nsb, r, b)]) * (double)g;
            for (int e = 0; e < 16; ++e) {
                int el = (int)(b % 2) * 16 + e;
                uint8_t byte = codes[tqo_code_offset(nsb, r, b / 2, el / 2)];
                uint8_t q = (el & 1) ? (byte >> 4) : (byte & 15);
                W[r * ldw + b * 16 + e] = (double)tqo_e2m1_to_f32(q) * s;
            }
        }
}

/* Y[m][r] = sum_k w~[r][k] X[m][k] over the NVFP4 reconstruction, fp64. */
void tqo_nvfp4_gemm(const uint8_t *codes, const uint8_t *scales, float g, int64_t n, int64_t k, const double *X,
                    int64_t m, int64_t ldx, double *Y, int64_t ldy) {
    double *tile = (double *)malloc((size_t)16 * (size_t)(k > 0 ? k : 1) * sizeof(double));
    int64_t nsb = tqo_superblocks(k);
    for (int64_t r = 0; r < n; ++r) {
        if (r % 16 == 0) tqo_nvfp4_dequantize(codes + (r / 16) * nsb * 1024, scales + (r / 16) * nsb * 128, g, 16, k,
                                              tile, k);
        for (int64_t i = 0; i < m; ++i) {
            double acc = 0.0;
            for (int64_t c = 0; c < k; ++c) acc += tile[(r % 16) * k + c] * X[i * ldx + c];
            Y[i * ldy + r] = acc;
        }
    }
    free(tile);
}
