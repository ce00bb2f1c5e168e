/*
 * convrot_oracle.c -- plain, slow CPU oracle for the ConvRot W8A8 INT8 linear.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline leg use it.  It shares no code, header, table or constant with
 * the CUDA library under w8a8_int8_quantized_block_b200/csrc.
 *
 * What it computes, and the passage each step follows:
 *
 *  rotation    "180 linear layers quantized to INT8 behind a block-diagonal
 *              Hadamard rotation" -- lehuy.net, "Nen mo hinh video khuech tan
 *              31B xuong 14B chi voi 6 buoc", section "Cach nen hoat dong".
 *              Each run of b consecutive channels of a token is multiplied by
 *              the Sylvester Hadamard matrix H_b, H[i][j] = (-1)^popcount(i&j)
 *              (unnormalised; the 1/b that makes H/sqrt(b) orthonormal on both
 *              operands is applied once in the dequantisation).  The pages say
 *              the rotation is undone exactly ("HyperFlow H3 Flash MLX",
 *              section "How to run": weights dequantized and "their Hadamard
 *              rotation undone (exact)").
 *              Computed as the textbook in-place fast Walsh-Hadamard transform
 *              in fp32, stages h = 1, 2, 4, ..., b/2 in that order, each
 *              butterfly (u, v) -> (u + v, u - v) rounded to nearest-even.
 *              The pages fix no order; this one is the reading both sides use.
 *  regular     the "DC-balanced regular orthogonal Hadamard matrix
 *              H_256 = H_4^(x)4" of "MiniMax-H3-Rung-Omega" README, section
 *              "Technical Architecture Overview", item 1 (there for another
 *              weight format; here an alternative rotation of orders 16, 64,
 *              256).  H_4 is read as J - 2I: every row sums to +2, so the
 *              Kronecker power of order b = 4^k has every row sum sqrt(b) and
 *              maps a constant block to a constant block.  Entry (i, j) is the
 *              product over the k base-4 digits of -1 where the digits agree
 *              and +1 where they differ.  Computed in fp32 as k radix-4
 *              stages, digit strides 1, 4, 16, 64 in that order; each group
 *              (x0, x1, x2, x3) of a stage becomes t - 2 x_i with
 *              t = (x0 + x1) + (x2 + x3), every operation rounded to
 *              nearest-even (2 x_i is exact, so each output rounds once more).
 *              Again the order is this reading's, shared by both sides.
 *  act quant   rowwise symmetric int8 ("SwiGLU + ConvRot64 + Rowwise INT8
 *              Quantize" -- MiniMax-H3-Rung-Omega README, "Technical
 *              Architecture Overview", item 2, Floor 1):
 *              amax = max_k |z_k|;  s = amax / 127 (f32);
 *              q_k = clamp(rne(z_k * (127 / amax)), -127, 127); amax = 0 gives
 *              s = 0 and q = 0.
 *  weights     same rotation along K, then per-output-channel scales
 *              ("preserves ConvRot metadata and per-output F32 scales" --
 *              "MiniMax H3 - pruned INT8 ConvRot - input-major", section
 *              "Input-major checkpoint"); storage [output, input].
 *  GEMM        acc[m][n] = sum_k qx[m][k] * qw[n][k], exact in int64
 *              ("W8A8 INT8" -- HyperFlow H3 Flash card, "Choose a Weight
 *              Format").
 *  activation  the down projection's input, "SwiGLU + ConvRot64 + Rowwise
 *  prologue    INT8 Quantize" fused in MLP.fc2 (MiniMax-H3-Rung-Omega README,
 *              "Technical Architecture Overview", item 2, Floor 1): from the
 *              up projection's bf16 output h, x = silu(g) * u with
 *              silu(g) = g / (1 + exp(-g)) and [g | u] the two halves of h's
 *              row (gate first), or x = gelu(h) = h Phi(h) = 0.5 h erfc(-h/sqrt 2);
 *              computed in fp64 and rounded once to f32, the precision the
 *              rotation and the quantiser then work in.
 *  dequant     y = acc * s_x[m] * s_w[n] * alpha + bias[n] in fp64, where
 *              alpha = 1/b for a rotated pair (b = 0 or 1: alpha = 1);
 *              optional exact-erf GELU.
 *
 * Pins (tests/test_oracle_pins.py): H*H^T = b*I in exact integers for both
 * kinds; the Sylvester entries equal the doubling recursion and the regular
 * ones numpy's Kronecker powers of J - 2I, with every row sum sqrt(b); both
 * transforms equal the explicit matrix product on integer inputs and are
 * involutions up to b; constant and spike blocks give closed-form codes;
 * rounding ties match an exact rational arbiter; the product is rounded to
 * f32 before the integer; sign and power-of-two scale invariances; the int64
 * GEMM equals a pure-Python brute force.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* H_b[i][j] from its definition: (-1)^(number of common one bits of i, j). */
int oracle_hadamard_entry(int64_t i, int64_t j) {
    return (__builtin_popcountll((unsigned long long)(i & j)) & 1) ? -1 : 1;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* In-place FWHT of one block of b floats, stages h = 1, 2, ..., b/2. */
static void fwht_block_f32(float *v, int b) {
    for (int h = 1; h < b; h <<= 1) {
        for (int i = 0; i < b; i += 2 * h) {
            for (int j = i; j < i + h; ++j) {
                float u = v[j];
                float w = v[j + h];
                v[j] = u + w;
                v[j + h] = u - w;
            }
        }
    }
}

/* Apply the block-diagonal transform to a vector of n floats (n % b == 0). */
void oracle_fwht_f32(float *v, int64_t n, int b) {
    if (b <= 1) return;
    for (int64_t o = 0; o < n; o += b) fwht_block_f32(v + o, b);
}

/* Regular H_4^(x)k, b = 4^k: entry from its definition, digit by digit. */
int oracle_regular_entry(int64_t i, int64_t j, int b) {
    int sign = 1;
    for (int st = 1; st < b; st *= 4) {
        if ((i / st) % 4 == (j / st) % 4) sign = -sign; /* H_4 = J - 2I: -1 on the diagonal */
    }
    return sign;
}

/* In-place regular transform of one block of b = 4^k floats: stages with
 * digit strides 1, 4, ..., b/4; each group (x0, x1, x2, x3) -> t - 2 x_i,
 * t = (x0 + x1) + (x2 + x3). */
static void rfwht_block_f32(float *v, int b) {
    for (int st = 1; st < b; st *= 4) {
        for (int i = 0; i < b; i += 4 * st) {
            for (int j = i; j < i + st; ++j) {
                float x0 = v[j], x1 = v[j + st], x2 = v[j + 2 * st], x3 = v[j + 3 * st];
                float t = (x0 + x1) + (x2 + x3);
                v[j] = t - 2.0f * x0;
                v[j + st] = t - 2.0f * x1;
                v[j + 2 * st] = t - 2.0f * x2;
                v[j + 3 * st] = t - 2.0f * x3;
            }
        }
    }
}

/* The rotation of a vector of n floats: Sylvester blocks, or regular ones. */
void oracle_rotate_f32(float *v, int64_t n, int b, int regular) {
    if (b <= 1) return;
    for (int64_t o = 0; o < n; o += b) {
        if (regular) rfwht_block_f32(v + o, b);
        else fwht_block_f32(v + o, b);
    }
}

/* Rowwise symmetric quantisation of one row of K rotated values. */
static void quantize_row(const float *z, int64_t K, int8_t *q, float *s) {
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(z[k]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        *s = 0.0f;
        memset(q, 0, (size_t)K);
        return;
    }
    float inv = 127.0f / amax;
    *s = amax / 127.0f;
    for (int64_t k = 0; k < K; ++k) {
        float v = z[k] * inv;
        float r = rintf(v); /* default rounding mode: nearest, ties to even */
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        q[k] = (int8_t)r;
    }
}

/* Quantise f32 rows that are already rotated (or need no rotation). */
void oracle_quantize_rows_f32(const float *z, int64_t M, int64_t K, int64_t ldz,
                              int8_t *q, int64_t ldq, float *s) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) quantize_row(z + m * ldz, K, q + m * ldq, s + m);
}

static float bf16_bits_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Activations: bf16 rows (raw bits) -> rotate per block of b -> int8 + scale. */
void oracle_quantize_act_bf16(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                              int b, int regular, int8_t *q, int64_t ldq, float *s) {
#pragma omp parallel
    {
        float *row = (float *)malloc((size_t)K * sizeof(float));
#pragma omp for schedule(static)
        for (int64_t m = 0; m < M; ++m) {
            for (int64_t k = 0; k < K; ++k) row[k] = bf16_bits_to_f32(x[m * ldx + k]);
            oracle_rotate_f32(row, K, b, regular);
            quantize_row(row, K, q + m * ldq, s + m);
        }
        free(row);
    }
}

/* gelu(y) = y * Phi(y), Phi the standard normal CDF, written as
 * 0.5 * erfc(-y / sqrt 2): the same function as 0.5 * (1 + erf(y / sqrt 2))
 * without the cancellation that form suffers for negative y. */
static double gelu_f64(double y) { return 0.5 * y * erfc(-y / sqrt(2.0)); }
static double silu_f64(double g) { return g / (1.0 + exp(-g)); }

/* The activation of one row: act 0 = none (x = h), 1 = GELU (x = gelu(h),
 * h has K columns), 2 = SwiGLU (x = silu(g) * u, g = h[0..K), u = h[K..2K)).
 * Each x is the fp64 value rounded once to f32. */
static void act_row_f32(const uint16_t *h, int64_t K, int act, float *x) {
    for (int64_t k = 0; k < K; ++k) {
        double v = (double)bf16_bits_to_f32(h[k]);
        if (act == 1) v = gelu_f64(v);
        else if (act == 2) v = silu_f64(v) * (double)bf16_bits_to_f32(h[K + k]);
        x[k] = (float)v;
    }
}

/* The activation alone, for the pins: x [M][K] f32. */
void oracle_act_f32(const uint16_t *h, int64_t M, int64_t K, int64_t ldh, int act, float *x) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) act_row_f32(h + m * ldh, K, act, x + m * K);
}

/* Activation prologue + rotation + rowwise quantisation (the down
 * projection's input): h bf16 rows of K (GELU) or 2K (SwiGLU) columns. */
void oracle_act_quantize_bf16(const uint16_t *h, int64_t M, int64_t K, int64_t ldh, int act,
                              int b, int regular, int8_t *q, int64_t ldq, float *s) {
#pragma omp parallel
    {
        float *row = (float *)malloc((size_t)K * sizeof(float));
#pragma omp for schedule(static)
        for (int64_t m = 0; m < M; ++m) {
            act_row_f32(h + m * ldh, K, act, row);
            oracle_rotate_f32(row, K, b, regular);
            quantize_row(row, K, q + m * ldq, s + m);
        }
        free(row);
    }
}

/* Weights: f32 [N, K] rows -> same rotation along K -> int8 + per-row scale. */
void oracle_pack_weight_f32(const float *w, int64_t N, int64_t K, int b, int regular,
                            int8_t *q, float *s) {
#pragma omp parallel
    {
        float *row = (float *)malloc((size_t)K * sizeof(float));
#pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            memcpy(row, w + n * K, (size_t)K * sizeof(float));
            oracle_rotate_f32(row, K, b, regular);
            quantize_row(row, K, q + n * K, s + n);
        }
        free(row);
    }
}

/* acc[m][n] = sum_k A[m][k] * B[n][k], exact int64 (both operands K-major). */
void oracle_igemm_s64(const int8_t *A, int64_t lda, const int8_t *B, int64_t ldb,
                      int64_t M, int64_t N, int64_t K, int64_t *C, int64_t ldc) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const int8_t *a = A + m * lda;
        for (int64_t n = 0; n < N; ++n) {
            const int8_t *bb = B + n * ldb;
            int64_t acc = 0;
            for (int64_t k = 0; k < K; ++k) acc += (int64_t)a[k] * (int64_t)bb[k];
            C[m * ldc + n] = acc;
        }
    }
}

/* The same dot products for an explicit list of (row, column) pairs. */
void oracle_igemm_s64_pairs(const int8_t *A, int64_t lda, const int8_t *B, int64_t ldb,
                            int64_t K, const int64_t *mi, const int64_t *ni,
                            int64_t count, int64_t *out) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < count; ++t) {
        const int8_t *a = A + mi[t] * lda;
        const int8_t *bb = B + ni[t] * ldb;
        int64_t acc = 0;
        for (int64_t k = 0; k < K; ++k) acc += (int64_t)a[k] * (int64_t)bb[k];
        out[t] = acc;
    }
}


/* y = acc * s_a[m] * s_b[n] * alpha + bias[n] (bias may be NULL), in fp64. */
void oracle_dequant_f64(const int64_t *acc, int64_t M, int64_t N,
                        const float *s_a, const float *s_b, const float *bias,
                        double alpha, int gelu, double *y) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double v = (double)acc[m * N + n] * (double)s_a[m] * (double)s_b[n] * alpha;
            if (bias) v += (double)bias[n];
            if (gelu) v = gelu_f64(v);
            y[m * N + n] = v;
        }
    }
}

/* Dequantise an explicit list of (row, column) accumulators. */
void oracle_dequant_pairs_f64(const int64_t *acc, const int64_t *mi, const int64_t *ni,
                              int64_t count, const float *s_a, const float *s_b,
                              const float *bias, double alpha, int gelu, double *y) {
    for (int64_t t = 0; t < count; ++t) {
        double v = (double)acc[t] * (double)s_a[mi[t]] * (double)s_b[ni[t]] * alpha;
        if (bias) v += (double)bias[ni[t]];
        if (gelu) v = gelu_f64(v);
        y[t] = v;
    }
}

/*
 * Exact-arithmetic companion of the rotation: z = blockdiag(H_b) x (Sylvester
 * or regular H_b) by the explicit matrix, accumulated in fp64 (exact for bf16
 * inputs whose block spans fewer than ~45 binades).  Used only to measure how
 * far a quantiser input sits from a rounding boundary.
 */
void oracle_rotate_explicit_f64(const float *x, int64_t M, int64_t K, int b, int regular, double *z) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const float *xr = x + m * K;
        double *zr = z + m * K;
        if (b <= 1) {
            for (int64_t k = 0; k < K; ++k) zr[k] = (double)xr[k];
            continue;
        }
        for (int64_t o = 0; o < K; o += b) {
            for (int i = 0; i < b; ++i) {
                double acc = 0.0;
                for (int j = 0; j < b; ++j) {
                    int e = regular ? oracle_regular_entry(i, j, b) : oracle_hadamard_entry(i, j);
                    acc += (double)e * (double)xr[o + j];
                }
                zr[o + i] = acc;
            }
        }
    }
}
