/*
 * tern_oracle.c -- plain, slow, fp64 CPU oracle for the ternary linear layer
 * of "1.58-bit FLUX" (arXiv 2412.18653).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or constant
 * with the CUDA library; the two are written independently from the same
 * definitions so that one can check the other.
 *
 * What it follows (page "1.58-bit FLUX", arXiv HTML v1):
 *   - Abstract and Section 1: linear-layer weights are restricted to the
 *     three values {-1, 0, +1} and are stored as 2-bit signed integers,
 *     compressed from 16-bit precision.
 *   - Section 1 and Section 2: the quantiser is "akin to BitNet b1.58".
 *     The pages give no formula; the plainest reading, which the rest of
 *     the pages support, is BitNet b1.58's absmean rule per output channel:
 *         gamma_n = mean_k |W[n,k]|,   s_n = gamma_n + eps,
 *         T[n,k]  = RoundClip(W[n,k] / s_n, -1, +1),
 *     with RoundClip(v, a, b) = max(a, min(b, round(v))) and round() to
 *     nearest, ties to even.  The dequantised weight is T[n,k] * s_n.
 *   - Section 4 (limitations): activations are not quantised, so x, b and y
 *     stay 16-bit (bf16 here) and the layer is
 *         y[m,n] = s_n * sum_k x[m,k] * T[n,k] + b_n.
 *
 * Arithmetic: every bf16 input is widened exactly to double; all sums and
 * products are in IEEE double (no -ffast-math, no reassociation beyond the
 * natural k order).
 *
 * Two packed layouts are implemented, both from their written definitions:
 *   canonical: row-major [N][K/4] bytes; element k of row n sits in byte
 *              n*K/4 + k/4 at bit 2*(k%4);
 *   tiled    : N%128 == 0, K%64 == 0; 16-byte groups, one per (row n,
 *              64-wide k chunk c = k/64), the group at byte offset
 *                ((n/128)*(K/64) + c)*2048 + (n%128)*16;
 *              inside the group, little-endian 32-bit word w = (k%64)/16;
 *              inside the word, with j = (k%16)/2 and h = k%2, the code sits
 *              at bits 16*h + 2*j and 16*h + 2*j + 1.
 * A code is the 2-bit two's-complement integer: +1 -> 01, 0 -> 00,
 * -1 -> 11; the pattern 10 (-2) is never written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Exact widening of a bf16 bit pattern (the upper half of an IEEE single). */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* absmean scale per output channel: s_n = mean_k |W[n,k]| + eps. */
void oracle_absmean_scales(const uint16_t *W, int64_t N, int64_t K, double eps,
                           double *s) {
    for (int64_t n = 0; n < N; ++n) {
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) acc += fabs(bf16_to_double(W[n * K + k]));
        double gamma = acc / (double)K;
        s[n] = gamma + eps;
    }
}

/* RoundClip(w / s, -1, +1) with round-to-nearest-even.  A scale of zero only
 * arises for an all-zero row with eps = 0; every element is then 0. */
static int8_t round_clip(double w, double s) {
    if (s == 0.0) return 0;
    double r = nearbyint(w / s); /* default rounding mode: nearest, ties even */
    if (r > 1.0) r = 1.0;
    if (r < -1.0) r = -1.0;
    return (int8_t)r;
}

/* Ternarise W with the given per-row scales (the oracle's own, or another
 * implementation's, to compare codes "given the scales"). */
void oracle_ternarize(const uint16_t *W, int64_t N, int64_t K, const double *s,
                      int8_t *T) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            T[n * K + k] = round_clip(bf16_to_double(W[n * K + k]), s[n]);
}

/* Marks elements whose |w|/s lies within `band` of the 0.5 rounding
 * threshold; returns how many there are. */
int64_t oracle_near_threshold(const uint16_t *W, int64_t N, int64_t K,
                              const double *s, double band, uint8_t *mask) {
    int64_t count = 0;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t near = 0;
            if (s[n] > 0.0) {
                double r = fabs(bf16_to_double(W[n * K + k])) / s[n];
                near = fabs(r - 0.5) < band;
            }
            mask[n * K + k] = near;
            count += near;
        }
    return count;
}

/* Full quantiser: scales, then codes. */
void oracle_quantize(const uint16_t *W, int64_t N, int64_t K, double eps,
                     int8_t *T, double *s) {
    oracle_absmean_scales(W, N, K, eps, s);
    oracle_ternarize(W, N, K, s, T);
}

static unsigned code_of(int8_t t) { return (unsigned)t & 3u; } /* 2-bit two's complement */

/* Returns 0 for a valid code, else marks it invalid. */
static int8_t value_of(unsigned code, int *bad) {
    switch (code & 3u) {
    case 0u: return 0;
    case 1u: return 1;
    case 3u: return -1;
    default: *bad += 1; return 0;
    }
}

void oracle_pack_canonical(const int8_t *T, int64_t N, int64_t K, uint8_t *P) {
    memset(P, 0, (size_t)(N * K / 4));
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            P[n * (K / 4) + k / 4] |= (uint8_t)(code_of(T[n * K + k]) << (2 * (k % 4)));
}

/* Returns the number of invalid (10) codes met. */
int oracle_unpack_canonical(const uint8_t *P, int64_t N, int64_t K, int8_t *T) {
    int bad = 0;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            T[n * K + k] = value_of(P[n * (K / 4) + k / 4] >> (2 * (k % 4)), &bad);
    return bad;
}

/* Byte index and bit shift of element (n, k) in the tiled layout. */
static void tiled_position(int64_t n, int64_t k, int64_t K, int64_t *byte, int *shift) {
    int64_t group = ((n / 128) * (K / 64) + k / 64) * 2048 + (n % 128) * 16;
    int64_t word = (k % 64) / 16;
    int j = (int)((k % 16) / 2);
    int h = (int)(k % 2);
    int bit = 16 * h + 2 * j; /* bit inside the little-endian 32-bit word */
    *byte = group + 4 * word + bit / 8;
    *shift = bit % 8;
}

/* Bytes of the tiled layout: whole slabs of 128 channels, so N rounds up to
 * a multiple of 128 and the rows past N hold zero codes. */
int64_t oracle_tiled_bytes(int64_t N, int64_t K) {
    return ((N + 127) / 128) * 128 * K / 4;
}

/* Returns -1 if the shape does not tile (N%16 or K%64 nonzero), else 0.  P
 * holds oracle_tiled_bytes(N, K) bytes; the padding rows are written as 0. */
int oracle_pack_tiled(const int8_t *T, int64_t N, int64_t K, uint8_t *P) {
    if (N <= 0 || N % 16 != 0 || K % 64 != 0) return -1;
    memset(P, 0, (size_t)oracle_tiled_bytes(N, K));
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int64_t byte;
            int shift;
            tiled_position(n, k, K, &byte, &shift);
            P[byte] |= (uint8_t)(code_of(T[n * K + k]) << shift);
        }
    return 0;
}

/* Returns -1 for a shape that does not tile, else the number of invalid codes. */
int oracle_unpack_tiled(const uint8_t *P, int64_t N, int64_t K, int8_t *T) {
    if (N <= 0 || N % 16 != 0 || K % 64 != 0) return -1;
    int bad = 0;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int64_t byte;
            int shift;
            tiled_position(n, k, K, &byte, &shift);
            T[n * K + k] = value_of((unsigned)P[byte] >> shift, &bad);
        }
    return bad;
}

/* y[m,n] = s_n * sum_k x[m,k] * T[n,k] + b_n, all in double.  bias may be
 * NULL (no bias).  Rows of y are independent, so they are shared out over
 * OpenMP threads; each y element is still one plain k-ordered sum. */
void oracle_linear(const uint16_t *x, int64_t M, int64_t K, const int8_t *T,
                   const double *s, const uint16_t *bias, int64_t N, double *y) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        double *xm = (double *)malloc((size_t)K * sizeof(double));
        for (int64_t k = 0; k < K; ++k) xm[k] = bf16_to_double(x[m * K + k]);
        for (int64_t n = 0; n < N; ++n) {
            const int8_t *tn = T + n * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += xm[k] * (double)tn[k];
            double b = bias ? bf16_to_double(bias[n]) : 0.0;
            y[m * N + n] = s[n] * acc + b;
        }
        free(xm);
    }
}

/* The tanh form of GELU, applied in place to columns [col0, N) of y [M, N]:
 *     g(v) = 0.5 * v * (1 + tanh(sqrt(2/pi) * (v + 0.044715 * v^3))).
 * The pages quantise the linears of FLUX's transformer blocks (Section 3.1)
 * but do not describe the operations around them; FLUX.1's MLP applies this
 * activation to the output of its first linear, which is what a fused
 * epilogue of that linear computes.  Written from the definition, in double. */
void oracle_gelu_tanh(double *y, int64_t M, int64_t N, int64_t col0) {
    const double c = sqrt(2.0 / 3.14159265358979323846);
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = col0; n < N; ++n) {
            const double v = y[m * N + n];
            y[m * N + n] = 0.5 * v * (1.0 + tanh(c * (v + 0.044715 * v * v * v)));
        }
}

/* Number of OpenMP threads a parallel region would use (1 without OpenMP). */
int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
