/*
 * nq_oracle.c -- plain CPU fp64 oracle for the low-rank binary factorised linear.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and its
 * Python binding) includes, links or calls this file; only the tests, the smoke check
 * and the CPU-baseline leg of the benchmark do.  It shares no code, header, table or
 * helper with the CUDA sources: its own bit reader, its own bf16/fp16 decoders.
 *
 * What it computes, and where that is defined:
 *
 *  - The weight of a factorised linear layer is a product of +1/-1 matrices and
 *    diagonal scaling vectors (hardwired.dev, "NanoQuant jednoduse: 70B model na herni
 *    grafice", section "Jak NanoQuant funguje"; rapidrecap.app "Nanoquant: Efficient
 *    Sub-1-Bit Quantization of Large Language Models", section "Quantization Technique":
 *    U and V binary matrices plus scaling factors).  Read here as
 *        W = diag(s1) . U . V^T . diag(s2),   U in {+1,-1}^{m x r},  V in {+1,-1}^{n x r},
 *    s1 (m) and s2 (n) fp16, and the layer output
 *        y = s1 (.) ( U . ( V^T . ( s2 (.) x ) ) ).
 *  - The sign matrices are stored one bit per entry (same section of hardwired.dev:
 *    r*(m+n) binary values plus the scales).  Storage bit 1 stands for +1, bit 0 for -1;
 *    32 entries per uint32, least significant bit first, words contiguous along the
 *    reduction dimension:  bit b of word w of a row = column 32*w + b.
 *    U is stored as its m rows (reduction over r), V as the r rows of V^T (reduction
 *    over n).  A row of `cols` entries takes ceil(cols/32) words; unused high bits of
 *    the last word are zero.
 *  - sign(0) is taken as +1 (the sign projection of the ADMM step, hardwired.dev section
 *    "Krok 2", does not say; this is the reading used throughout).
 *  - Bits per weight = (r*(m+n) + 16*(m+n)) / (m*n): r(m+n) one-bit entries plus two
 *    fp16 scale vectors (hardwired.dev sections "Jak NanoQuant funguje" and
 *    "Co znamena sub-1-bit").
 *
 * Arithmetic: every input is decoded exactly into double; x' = s2*x is exact in double
 * (8-bit by 11-bit significands); sums run in increasing index order in double.  The
 * optional OpenMP pragma only spreads independent output rows over threads; it does not
 * change any sum.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG (-1)
#define ORC_ERR_VALUE (-5)

/* ---- exact decoders, written from the IEEE 754 binary16 / bfloat16 bit layouts ---- */

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits.  It is the upper
 * half of an IEEE binary32, so the value is that binary32 with 16 zero bits appended.
 * Decoded here from the fields, without type punning, so it is checkable by eye. */
double orc_bf16_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int expo = (h >> 7) & 0xFF;
    int frac = h & 0x7F;
    double v;
    if (expo == 0xFF) {
        v = frac ? NAN : INFINITY;
    } else if (expo == 0) {
        v = ldexp((double)frac, -126 - 7);           /* subnormal: 0.frac * 2^-126 */
    } else {
        v = ldexp((double)(frac | 0x80), expo - 127 - 7); /* 1.frac * 2^(e-127) */
    }
    return sign ? -v : v;
}

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double orc_f16_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1F;
    int frac = h & 0x3FF;
    double v;
    if (expo == 0x1F) {
        v = frac ? NAN : INFINITY;
    } else if (expo == 0) {
        v = ldexp((double)frac, -14 - 10);            /* subnormal: 0.frac * 2^-14 */
    } else {
        v = ldexp((double)(frac | 0x400), expo - 15 - 10);
    }
    return sign ? -v : v;
}

/* ---- storage of the sign matrices ---- */

static int64_t words_per_row(int64_t cols) { return (cols + 31) / 32; }

/* The entry (row, col) of a packed sign matrix, as +1 or -1. */
static int orc_sign_at(const uint32_t *packed, int64_t wpr, int64_t row, int64_t col) {
    uint32_t word = packed[row * wpr + col / 32];
    return ((word >> (col % 32)) & 1u) ? +1 : -1;
}

/* Pack a rows x cols matrix of int8 signs (row-major) into rows x ceil(cols/32) words.
 * Entries must be -1, 0 or +1; 0 packs as +1.  Any other value: ORC_ERR_VALUE and the
 * output is left untouched. */
int orc_pack_signs(const int8_t *signs, int64_t rows, int64_t cols, uint32_t *out) {
    if (rows < 0 || cols < 0 || (rows * cols > 0 && (!signs || !out))) return ORC_ERR_ARG;
    for (int64_t i = 0; i < rows * cols; ++i)
        if (signs[i] < -1 || signs[i] > 1) return ORC_ERR_VALUE;
    int64_t wpr = words_per_row(cols);
    for (int64_t row = 0; row < rows; ++row) {
        for (int64_t w = 0; w < wpr; ++w) {
            uint32_t word = 0;
            for (int b = 0; b < 32; ++b) {
                int64_t col = 32 * w + b;
                if (col < cols && signs[row * cols + col] >= 0) word |= (1u << b);
            }
            out[row * wpr + w] = word;
        }
    }
    return ORC_OK;
}

/* Inverse of orc_pack_signs: rows x cols int8 in {-1, +1}. */
int orc_unpack_signs(const uint32_t *packed, int64_t rows, int64_t cols, int8_t *out) {
    if (rows < 0 || cols < 0 || (rows * cols > 0 && (!packed || !out))) return ORC_ERR_ARG;
    int64_t wpr = words_per_row(cols);
    for (int64_t row = 0; row < rows; ++row)
        for (int64_t col = 0; col < cols; ++col)
            out[row * cols + col] = (int8_t)orc_sign_at(packed, wpr, row, col);
    return ORC_OK;
}

/* ---- the forward pass ----
 *
 * x   : batch x n bfloat16 bit patterns, row-major (one token per row)
 * Upk : m rows of ceil(r/32) words   (row i holds U[i][0..r))
 * Vpk : r rows of ceil(n/32) words   (row k holds V^T[k][0..n) = V[0..n)[k])
 * s1  : m fp16 bit patterns;  s2 : n fp16 bit patterns
 * y   : batch x m doubles (written)
 */
int orc_lowrank_linear_fwd(const uint16_t *x, const uint32_t *Upk, const uint32_t *Vpk,
                           const uint16_t *s1, const uint16_t *s2, int64_t m, int64_t n,
                           int64_t r, int64_t batch, double *y) {
    if (m <= 0 || n <= 0 || r <= 0 || batch < 0) return ORC_ERR_ARG;
    if (batch == 0) return ORC_OK;
    if (!x || !Upk || !Vpk || !s1 || !s2 || !y) return ORC_ERR_ARG;
    const int64_t wpr_u = words_per_row(r), wpr_v = words_per_row(n);
    double *xs = (double *)malloc(sizeof(double) * (size_t)(n * batch));
    double *t = (double *)malloc(sizeof(double) * (size_t)(r * batch));
    if (!xs || !t) { free(xs); free(t); return ORC_ERR_ARG; }

    /* step 1: x' = s2 (.) x, exact in double */
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t j = 0; j < n; ++j)
            xs[b * n + j] = orc_f16_to_double(s2[j]) * orc_bf16_to_double(x[b * n + j]);

    /* step 2: t_k = sum_j V[j][k] * x'_j, increasing j */
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < r; ++k) {
        for (int64_t b = 0; b < batch; ++b) {
            double acc = 0.0;
            for (int64_t j = 0; j < n; ++j)
                acc += orc_sign_at(Vpk, wpr_v, k, j) * xs[b * n + j];
            t[b * r + k] = acc;
        }
    }

    /* step 3: y_i = s1_i * sum_k U[i][k] * t_k, increasing k */
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < m; ++i) {
        double si = orc_f16_to_double(s1[i]);
        for (int64_t b = 0; b < batch; ++b) {
            double acc = 0.0;
            for (int64_t k = 0; k < r; ++k)
                acc += orc_sign_at(Upk, wpr_u, i, k) * t[b * r + k];
            y[b * m + i] = si * acc;
        }
    }
    free(xs);
    free(t);
    return ORC_OK;
}

/* ---- the rank-l envelope variant of the forward pass ----
 *
 * MDBF ("Multi-Envelope DBF", hardwired.dev section "Kontext: co existuje kolem") replaces
 * the simple scaling of the binary factorisation with a rank-l envelope; the same section
 * notes that under the simple scaling all rank components share one magnitude profile.
 * Read here as the weight
 *     W = E (.) (U V^T),   E = sum_{q<l} a_q b_q^T   (a_q: m fp16, b_q: n fp16),
 * whose l = 1 case is diag(s1) U V^T diag(s2) with s1 = a_0, s2 = b_0.  Since
 * (a b^T) (.) (U V^T) = diag(a) U V^T diag(b), the output is
 *     y = sum_{q<l} a_q (.) ( U . ( V^T . ( b_q (.) x ) ) ),
 * each term the forward pass above with (s1, s2) = (a_q, b_q), added in increasing q.
 *
 * a : l rows of m fp16 bit patterns;  b : l rows of n fp16 bit patterns;  l >= 1.
 * y : batch x m doubles (written).  Other arguments as orc_lowrank_linear_fwd.
 */
int orc_lowrank_linear_fwd_envelope(const uint16_t *x, const uint32_t *Upk, const uint32_t *Vpk,
                                    const uint16_t *a, const uint16_t *b, int64_t l, int64_t m,
                                    int64_t n, int64_t r, int64_t batch, double *y) {
    if (l <= 0 || m <= 0 || n <= 0 || r <= 0 || batch < 0) return ORC_ERR_ARG;
    if (batch == 0) return ORC_OK;
    if (!a || !b) return ORC_ERR_ARG;
    /* the first term straight into y (so that l = 1 is the forward pass bit for bit) */
    int st = orc_lowrank_linear_fwd(x, Upk, Vpk, a, b, m, n, r, batch, y);
    if (st != ORC_OK || l == 1) return st;
    double *term = (double *)malloc(sizeof(double) * (size_t)(m * batch));
    if (!term) return ORC_ERR_ARG;
    for (int64_t q = 1; q < l && st == ORC_OK; ++q) {
        st = orc_lowrank_linear_fwd(x, Upk, Vpk, a + q * m, b + q * n, m, n, r, batch, term);
        for (int64_t e = 0; e < m * batch && st == ORC_OK; ++e) y[e] += term[e];
    }
    free(term);
    return st;
}

/* Bits per weight of the envelope variant: r(m+n) sign bits plus l pairs of fp16 vectors,
 * (r*(m+n) + 16*l*(m+n)) / (m*n); -1 for a non-positive argument. */
double orc_bits_per_weight_envelope(int64_t m, int64_t n, int64_t r, int64_t l) {
    if (m <= 0 || n <= 0 || r <= 0 || l <= 0) return -1.0;
    return ((double)r * (double)(m + n) + 16.0 * (double)l * (double)(m + n)) / ((double)m * (double)n);
}

/* ---- the input gradient ----
 *
 * The refinement step fine-tunes the factorised components with straight-through
 * estimators (hardwired.dev, section "Krok 3": the gradient of the sign function is taken
 * as the identity on the backward pass), so every step back-propagates through the layer.
 * With the signs and scales held fixed the layer is the linear map W x, and the gradient
 * with respect to its input is the transpose applied to the output gradient:
 *     dx = W^T dy = s2 (.) ( V . ( U^T . ( s1 (.) dy ) ) ).
 *
 * dy  : batch x m bfloat16 bit patterns, row-major (one token per row)
 * Upk, Vpk, s1, s2 : exactly as in the forward pass (this routine reads the same packings)
 * dx  : batch x n doubles (written)
 */
int orc_lowrank_linear_bwd_input(const uint16_t *dy, const uint32_t *Upk, const uint32_t *Vpk,
                                 const uint16_t *s1, const uint16_t *s2, int64_t m, int64_t n,
                                 int64_t r, int64_t batch, double *dx) {
    if (m <= 0 || n <= 0 || r <= 0 || batch < 0) return ORC_ERR_ARG;
    if (batch == 0) return ORC_OK;
    if (!dy || !Upk || !Vpk || !s1 || !s2 || !dx) return ORC_ERR_ARG;
    const int64_t wpr_u = words_per_row(r), wpr_v = words_per_row(n);
    double *g = (double *)malloc(sizeof(double) * (size_t)(m * batch));
    double *u = (double *)malloc(sizeof(double) * (size_t)(r * batch));
    if (!g || !u) { free(g); free(u); return ORC_ERR_ARG; }

    /* step 1: g = s1 (.) dy, exact in double */
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t i = 0; i < m; ++i)
            g[b * m + i] = orc_f16_to_double(s1[i]) * orc_bf16_to_double(dy[b * m + i]);

    /* step 2: u_k = sum_i U[i][k] * g_i, increasing i */
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < r; ++k) {
        for (int64_t b = 0; b < batch; ++b) {
            double acc = 0.0;
            for (int64_t i = 0; i < m; ++i)
                acc += orc_sign_at(Upk, wpr_u, i, k) * g[b * m + i];
            u[b * r + k] = acc;
        }
    }

    /* step 3: dx_j = s2_j * sum_k V[j][k] * u_k, increasing k (V[j][k] is entry (k, j) of V^T) */
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        double sj = orc_f16_to_double(s2[j]);
        for (int64_t b = 0; b < batch; ++b) {
            double acc = 0.0;
            for (int64_t k = 0; k < r; ++k)
                acc += orc_sign_at(Vpk, wpr_v, k, j) * u[b * r + k];
            dx[b * n + j] = sj * acc;
        }
    }
    free(g);
    free(u);
    return ORC_OK;
}

/* The two rank-r vectors of the backward pass, per token: t = V^T (s2 (.) x) and
 * u = U^T (s1 (.) dy) (batch x r doubles each), sums in increasing index. */
static void orc_rank_vectors(const uint16_t *x, const uint16_t *dy, const uint32_t *Upk,
                             const uint32_t *Vpk, const uint16_t *s1, const uint16_t *s2, int64_t m,
                             int64_t n, int64_t r, int64_t batch, double *t, double *u) {
    const int64_t wpr_u = words_per_row(r), wpr_v = words_per_row(n);
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t k = 0; k < r; ++k) {
            double at = 0.0, au = 0.0;
            for (int64_t j = 0; j < n; ++j)
                at += orc_sign_at(Vpk, wpr_v, k, j) * (orc_f16_to_double(s2[j]) * orc_bf16_to_double(x[b * n + j]));
            for (int64_t i = 0; i < m; ++i)
                au += orc_sign_at(Upk, wpr_u, i, k) * (orc_f16_to_double(s1[i]) * orc_bf16_to_double(dy[b * m + i]));
            t[b * r + k] = at;
            u[b * r + k] = au;
        }
}

/* ---- the scale gradients ----
 *
 * The refinement step tunes the scaling factors together with the binary factors
 * (hardwired.dev, section "Krok 3").  For a loss with output gradient dy, y is linear in
 * each scale vector, so
 *     ds1_i = sum_b dy[b][i] * z[b][i],   z = U (V^T (s2 (.) x))      (y = s1 (.) z)
 *     ds2_j = sum_b x[b][j]  * w[b][j],   w = V (U^T (s1 (.) dy))     (dx = s2 (.) w)
 * x: batch x n and dy: batch x m bfloat16 bit patterns; Upk, Vpk, s1, s2 as in the
 * forward pass; ds1 (m) and ds2 (n) doubles (written).  The sums over b run in increasing
 * b after z and w are complete.
 */
int orc_lowrank_linear_bwd_scales(const uint16_t *x, const uint16_t *dy, const uint32_t *Upk,
                                  const uint32_t *Vpk, const uint16_t *s1, const uint16_t *s2,
                                  int64_t m, int64_t n, int64_t r, int64_t batch, double *ds1,
                                  double *ds2) {
    if (m <= 0 || n <= 0 || r <= 0 || batch < 0) return ORC_ERR_ARG;
    if (!ds1 || !ds2) return ORC_ERR_ARG;
    for (int64_t i = 0; i < m; ++i) ds1[i] = 0.0;
    for (int64_t j = 0; j < n; ++j) ds2[j] = 0.0;
    if (batch == 0) return ORC_OK;
    if (!x || !dy || !Upk || !Vpk || !s1 || !s2) return ORC_ERR_ARG;
    const int64_t wpr_u = words_per_row(r), wpr_v = words_per_row(n);
    double *t = (double *)malloc(sizeof(double) * (size_t)(r * batch));
    double *u = (double *)malloc(sizeof(double) * (size_t)(r * batch));
    if (!t || !u) { free(t); free(u); return ORC_ERR_ARG; }
    orc_rank_vectors(x, dy, Upk, Vpk, s1, s2, m, n, r, batch, t, u);
    /* ds1_i = sum_b dy_bi * (U t_b)_i ;  ds2_j = sum_b x_bj * (V u_b)_j */
    for (int64_t i = 0; i < m; ++i)
        for (int64_t b = 0; b < batch; ++b) {
            double z = 0.0;
            for (int64_t k = 0; k < r; ++k) z += orc_sign_at(Upk, wpr_u, i, k) * t[b * r + k];
            ds1[i] += orc_bf16_to_double(dy[b * m + i]) * z;
        }
    for (int64_t j = 0; j < n; ++j)
        for (int64_t b = 0; b < batch; ++b) {
            double w = 0.0;
            for (int64_t k = 0; k < r; ++k) w += orc_sign_at(Vpk, wpr_v, k, j) * u[b * r + k];
            ds2[j] += orc_bf16_to_double(x[b * n + j]) * w;
        }
    free(t);
    free(u);
    return ORC_OK;
}

/* ---- the gradients of the factors ----
 *
 * The straight-through estimator of the refinement step (hardwired.dev, section "Krok 3")
 * passes the gradient of the sign function as the identity, so the gradient with respect
 * to the latent factors is the gradient with respect to the +1/-1 factors themselves:
 *     dU[i][k] = s1_i * sum_b dy[b][i] * t[b][k],   t = V^T (s2 (.) x)
 *     dV[j][k] = s2_j * sum_b x[b][j]  * u[b][k],   u = U^T (s1 (.) dy)
 * x: batch x n, dy: batch x m bfloat16 bit patterns; Upk, Vpk, s1, s2 as in the forward
 * pass; dU (m x r) and dV (n x r) doubles, row-major (written).  Sums over b in increasing b.
 */
int orc_lowrank_linear_bwd_factors(const uint16_t *x, const uint16_t *dy, const uint32_t *Upk,
                                   const uint32_t *Vpk, const uint16_t *s1, const uint16_t *s2,
                                   int64_t m, int64_t n, int64_t r, int64_t batch, double *dU,
                                   double *dV) {
    if (m <= 0 || n <= 0 || r <= 0 || batch < 0) return ORC_ERR_ARG;
    if (!dU || !dV) return ORC_ERR_ARG;
    for (int64_t q = 0; q < m * r; ++q) dU[q] = 0.0;
    for (int64_t q = 0; q < n * r; ++q) dV[q] = 0.0;
    if (batch == 0) return ORC_OK;
    if (!x || !dy || !Upk || !Vpk || !s1 || !s2) return ORC_ERR_ARG;
    double *t = (double *)malloc(sizeof(double) * (size_t)(r * batch));
    double *u = (double *)malloc(sizeof(double) * (size_t)(r * batch));
    if (!t || !u) { free(t); free(u); return ORC_ERR_ARG; }
    orc_rank_vectors(x, dy, Upk, Vpk, s1, s2, m, n, r, batch, t, u);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < m; ++i) {
        const double si = orc_f16_to_double(s1[i]);
        for (int64_t k = 0; k < r; ++k) {
            double acc = 0.0;
            for (int64_t b = 0; b < batch; ++b) acc += orc_bf16_to_double(dy[b * m + i]) * t[b * r + k];
            dU[i * r + k] = si * acc;
        }
    }
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        const double s2j = orc_f16_to_double(s2[j]);
        for (int64_t k = 0; k < r; ++k) {
            double acc = 0.0;
            for (int64_t b = 0; b < batch; ++b) acc += orc_bf16_to_double(x[b * n + j]) * u[b * r + k];
            dV[j * r + k] = s2j * acc;
        }
    }
    free(t);
    free(u);
    return ORC_OK;
}

/* Transpose of a packed sign matrix: `in` holds rows x cols entries in rows x ceil(cols/32)
 * words, `out` receives the cols x rows transpose in cols x ceil(rows/32) words (same bit
 * convention, unused high bits zero). */
int orc_transpose_signs(const uint32_t *in, int64_t rows, int64_t cols, uint32_t *out) {
    if (rows < 0 || cols < 0) return ORC_ERR_ARG;
    if (rows == 0 || cols == 0) return ORC_OK;
    if (!in || !out) return ORC_ERR_ARG;
    const int64_t wpr_in = words_per_row(cols), wpr_out = words_per_row(rows);
    memset(out, 0, sizeof(uint32_t) * (size_t)(cols * wpr_out));
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t j = 0; j < cols; ++j)
            if (orc_sign_at(in, wpr_in, i, j) > 0) out[j * wpr_out + i / 32] |= 1u << (i % 32);
    return ORC_OK;
}

/* The intermediate t = V^T (s2 (.) x) alone (batch x r doubles), for tests that look
 * at the rank bottleneck. */
int orc_stage1(const uint16_t *x, const uint32_t *Vpk, const uint16_t *s2, int64_t n,
               int64_t r, int64_t batch, double *t) {
    if (n <= 0 || r <= 0 || batch < 0) return ORC_ERR_ARG;
    if (batch == 0) return ORC_OK;
    if (!x || !Vpk || !s2 || !t) return ORC_ERR_ARG;
    const int64_t wpr_v = words_per_row(n);
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t k = 0; k < r; ++k) {
            double acc = 0.0;
            for (int64_t j = 0; j < n; ++j)
                acc += orc_sign_at(Vpk, wpr_v, k, j) *
                       (orc_f16_to_double(s2[j]) * orc_bf16_to_double(x[b * n + j]));
            t[b * r + k] = acc;
        }
    return ORC_OK;
}

/* Storage accounting: (r(m+n) + 16(m+n)) / (mn); -1.0 if any argument is <= 0. */
double orc_bits_per_weight(int64_t m, int64_t n, int64_t r) {
    if (m <= 0 || n <= 0 || r <= 0) return -1.0;
    double num = (double)r * (double)(m + n) + 16.0 * (double)(m + n);
    return num / ((double)m * (double)n);
}

/* Number of threads the parallel loops above use (1 without OpenMP). */
int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---- helpers of the decode chain ----
 *
 * A decode step runs a decoder's linear layers one after the other (hardwired.dev,
 * section "Cisla", reports decode tokens/s of a whole quantised 70B model).  The pages
 * print neither the layers between the linears nor any normalisation, so the chain used
 * here is a reading: each block's input h is a bfloat16 vector of unit root-mean-square;
 * q, k, v, gate and up read h; o reads bf16(v's output); down reads bf16(up's output);
 * the next block's h is bf16(down's output / rms(down's output)).  The two helpers
 * below are that rounding and that normalisation. */

/* Nearest bfloat16 of v, ties to even (the IEEE 754 default rounding), written from the
 * bfloat16 layout: 1 sign, 8 exponent (bias 127) and 7 fraction bits; normal numbers
 * 1.f x 2^E with -126 <= E <= 127, subnormals 0.f x 2^-126.  Overflow gives infinity,
 * NaN the quiet NaN 0x7FC0. */
uint16_t orc_round_to_bf16(double v) {
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7F80;
    int e;
    frexp(a, &e);                      /* a = f * 2^e with 0.5 <= f < 1: a = 1.x * 2^(e-1) */
    int E = e - 1;
    if (E < -126) E = -126;            /* below the normal range the quantum stays 2^-133 */
    double q = rint(ldexp(a, 7 - E));  /* a in units of the quantum 2^(E-7), ties to even */
    if (q >= 256.0) {                  /* rounded up into the next binade */
        E += 1;
        q = 128.0;
    }
    if (E > 127) return sign | 0x7F80;
    if (q < 128.0) return sign | (uint16_t)q;  /* subnormal: exponent field 0 */
    return sign | (uint16_t)(((uint32_t)(E + 127) << 7) | ((uint32_t)q - 128u));
}

int orc_round_array_bf16(const double *v, int64_t count, uint16_t *out) {
    if (count < 0 || (count > 0 && (!v || !out))) return ORC_ERR_ARG;
    for (int64_t i = 0; i < count; ++i) out[i] = orc_round_to_bf16(v[i]);
    return ORC_OK;
}

/* out[row][j] = bf16( y[row][j] / sqrt( (1/cols) * sum_j y[row][j]^2 ) ), the sum in
 * increasing j in double.  A row whose sum of squares is 0 is copied as bf16(y) (signed
 * zeros): there is nothing to normalise. */
int orc_rms_normalize_bf16(const double *y, int64_t rows, int64_t cols, uint16_t *out) {
    if (rows < 0 || cols <= 0 || (rows > 0 && (!y || !out))) return ORC_ERR_ARG;
    for (int64_t row = 0; row < rows; ++row) {
        const double *yr = y + row * cols;
        double acc = 0.0;
        for (int64_t j = 0; j < cols; ++j) acc += yr[j] * yr[j];
        double rms = sqrt(acc / (double)cols);
        for (int64_t j = 0; j < cols; ++j)
            out[row * cols + j] = orc_round_to_bf16(rms > 0.0 ? yr[j] / rms : yr[j]);
    }
    return ORC_OK;
}
