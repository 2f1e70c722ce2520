/*
 * aria_oracle.c -- plain, slow CPU oracle for the quantized linear layers of
 * "A Quantized Native Runtime for On-Device Semantic Audio Generation"
 * (aria project page: "What aria is" -- quantization that replaces the fp16
 * footprint; "Results" -- the fp16 / q8 / W8A8 / q4 precision table and the
 * note that W8A8 runs 8-bit arithmetic on integer tensor cores; "Steering is
 * real" -- a direction vector added at one block, removable at alpha = 0).
 *
 * TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's
 * CPU-baseline leg may load this library. The CUDA product path never does,
 * and this file shares no code, header, table or helper with it.
 *
 * The pages name the precisions but print none of the arithmetic. The
 * formats written out here are the ones the project fixes for this library:
 *   q8   : per output channel n, s[n] = absmax_k |W[n,k]| / 127 (fp32),
 *          q = clamp(round_half_even(W / s), -127, 127), int8 [N,K].
 *   q4   : per output channel n and group j of 32 consecutive k,
 *          s16 = fp16_rn(absmax / 7), q = clamp(rhe(W / float(s16)), -7, 7),
 *          stored offset-binary q+8, even k in the low nibble, [N,K/2] bytes,
 *          scales fp16 [N,K/32].
 *   A8   : per token row m, exactly the q8 rule along K (scale fp32 [M]).
 *   W8A8 : acc = sum_k Xq[m,k]*Wq[n,k] in exact integer arithmetic, then
 *          y = fp16_rn(acc*s_x[m]*s_w[n] + bias[n] + alpha*v[n]) in fp64.
 *   weight-only (q8, q4): y_ref = sum_k X[m,k]*q[n,k]*s + bias[n] + alpha*v[n]
 *          in fp64, NOT rounded (the fp16 output is compared with tolerance).
 *   fp16 : the unquantised rung of the "Results" precision table,
 *          y_ref = sum_k X[m,k]*W[n,k] + bias[n] + alpha*v[n] in fp64, NOT
 *          rounded (compared with the same tolerance as weight-only).
 * Every division is the IEEE fp32 quotient, rounded once; every rounding to
 * an integer is round-half-even (nearbyint under the default rounding mode).
 * An all-zero row / group / token gets scale 0 and codes 0.
 * Steering is skipped entirely (not "+ 0*v") when v is NULL or alpha == 0.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC.
 * Single-threaded on purpose: plain loops a reader can check by eye.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>

/* ---------------------------------------------------------------- fp16 --- */

/* IEEE binary16 bit pattern -> double, exact. */
double orc_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* zero / subnormal */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);     /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

static float h2f(uint16_t h) { return (float)orc_half_to_double(h); } /* exact */

/* double -> IEEE binary16, round to nearest, ties to even, one rounding. */
uint16_t orc_double_to_half(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double ax = fabs(x);
    if (isnan(x))
        return (uint16_t)(sign | 0x7e00);
    /* 65520 is halfway between 65504 (odd significand) and 2^16: ties go up. */
    if (ax >= 65520.0)
        return (uint16_t)(sign | 0x7c00);
    if (ax < ldexp(1.0, -14)) {
        /* subnormal range: units of 2^-24; scaling by a power of two is exact */
        double r = nearbyint(ax * ldexp(1.0, 24));
        return (uint16_t)(sign | (uint16_t)r);     /* r == 1024 is the smallest normal */
    }
    int E;
    (void)frexp(ax, &E);                           /* ax in [2^(E-1), 2^E) */
    double r = nearbyint(ldexp(ax, 11 - E));       /* significand in [1024, 2048] */
    int ef = E - 1 + 15;
    if (r >= 2048.0) {
        r = 1024.0;
        ef += 1;
    }
    if (ef >= 31)
        return (uint16_t)(sign | 0x7c00);
    return (uint16_t)(sign | (uint16_t)(ef << 10) | (uint16_t)(r - 1024.0));
}

uint16_t orc_float_to_half(float x) { return orc_double_to_half((double)x); }

/* bulk helpers for the Python side */
void orc_half_to_double_n(const uint16_t *h, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_half_to_double(h[i]);
}

void orc_double_to_half_n(const double *x, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_double_to_half(x[i]);
}

void orc_float_to_half_n(const float *x, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_float_to_half(x[i]);
}

/* ------------------------------------------------- symmetric int8 rows --- */

/* One row of R x K fp16 values -> int8 codes + fp32 scale (the q8 rule).
 * Used for weight rows (q8 pack) and for token rows (per-token activation
 * quantisation): both are "per row, symmetric, absmax / 127". */
static void quant_row_i8(const uint16_t *x, int64_t K, int8_t *q, float *scale)
{
    float a = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float v = fabsf(h2f(x[k]));
        if (v > a)
            a = v;
    }
    float s = a / 127.0f;
    *scale = s;
    for (int64_t k = 0; k < K; ++k) {
        if (a == 0.0f) {
            q[k] = 0;
            continue;
        }
        float quot = h2f(x[k]) / s;                /* IEEE fp32 quotient */
        float r = nearbyintf(quot);                /* ties to even */
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        q[k] = (int8_t)r;
    }
}

/* q8 pack: W fp16 [N,K] -> Wq int8 [N,K], s_w fp32 [N]. */
void orc_pack_q8(const uint16_t *W, int64_t N, int64_t K, int8_t *Wq, float *sw)
{
    for (int64_t n = 0; n < N; ++n)
        quant_row_i8(W + n * K, K, Wq + n * K, sw + n);
}

/* per-token activation quantisation: X fp16 [M,K] -> Xq int8 [M,K], s_x fp32 [M]. */
void orc_act_quant(const uint16_t *X, int64_t M, int64_t K, int8_t *Xq, float *sx)
{
    for (int64_t m = 0; m < M; ++m)
        quant_row_i8(X + m * K, K, Xq + m * K, sx + m);
}

/* ------------------------------------------------------- q4 group-32 --- */

/* q4 pack: W fp16 [N,K] (K % 32 == 0) -> P uint8 [N,K/2], S fp16 bits [N,K/32]. */
void orc_pack_q4(const uint16_t *W, int64_t N, int64_t K, uint8_t *P, uint16_t *S)
{
    const int64_t G = K / 32;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < G; ++j) {
            const uint16_t *w = W + n * K + j * 32;
            float a = 0.0f;
            for (int i = 0; i < 32; ++i) {
                float v = fabsf(h2f(w[i]));
                if (v > a)
                    a = v;
            }
            uint16_t s16 = orc_float_to_half(a / 7.0f);
            float sf = h2f(s16);
            S[n * G + j] = s16;
            for (int i = 0; i < 32; ++i) {
                int q = 0;
                if (sf != 0.0f) {
                    float r = nearbyintf(h2f(w[i]) / sf);
                    if (r > 7.0f) r = 7.0f;
                    if (r < -7.0f) r = -7.0f;
                    q = (int)r;
                }
                int64_t k = j * 32 + i;
                uint8_t nib = (uint8_t)(q + 8);
                uint8_t *byte = P + n * (K / 2) + k / 2;
                if ((k & 1) == 0)
                    *byte = (uint8_t)((*byte & 0xf0) | nib);
                else
                    *byte = (uint8_t)((*byte & 0x0f) | (nib << 4));
            }
        }
    }
}

/* dequantised weights in fp64, for tests: q8 -> q*s, q4 -> (nib-8)*float(s16) */
void orc_dequant_q8(const int8_t *Wq, const float *sw, int64_t N, int64_t K, double *out)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            out[n * K + k] = (double)Wq[n * K + k] * (double)sw[n];
}

void orc_dequant_q4(const uint8_t *P, const uint16_t *S, int64_t N, int64_t K, double *out)
{
    const int64_t G = K / 32;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = P[n * (K / 2) + k / 2];
            int nib = (k & 1) ? (byte >> 4) : (byte & 0x0f);
            out[n * K + k] = (double)(nib - 8) * orc_half_to_double(S[n * G + k / 32]);
        }
}

/* ------------------------------------------------------------- GEMMs --- */

/* Row selection: rows == NULL means all M rows; otherwise n_rows row indices
 * into X, and output row i corresponds to X row rows[i]. */
static int64_t pick(const int64_t *rows, int64_t i) { return rows ? rows[i] : i; }

/* exact integer GEMM: C[i,n] = sum_k Xq[rows[i],k] * Wq[n,k]. Accumulates in
 * int64; returns 1 if any result leaves the int32 range (C then unspecified). */
int orc_gemm_s32(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                 const int64_t *rows, int64_t n_rows, int32_t *C)
{
    int overflow = 0;
    int64_t R = rows ? n_rows : M;
    for (int64_t i = 0; i < R; ++i) {
        const int8_t *x = Xq + pick(rows, i) * K;
        for (int64_t n = 0; n < N; ++n) {
            const int8_t *w = Wq + n * K;
            int64_t acc = 0;
            for (int64_t k = 0; k < K; ++k)
                acc += (int64_t)x[k] * (int64_t)w[k];
            if (acc > INT32_MAX || acc < INT32_MIN)
                overflow = 1;
            C[i * N + n] = (int32_t)acc;
        }
    }
    return overflow;
}

/* fused epilogue terms for column n, in fp64 (bias and steering optional) */
static double epi_terms(int64_t n, const uint16_t *bias, const float *v, float alpha, double y)
{
    if (bias)
        y += orc_half_to_double(bias[n]);
    if (v && alpha != 0.0f)
        y += (double)alpha * (double)v[n];
    return y;
}

/* W8A8 output: Y[i,n] = fp16_rn(acc*s_x*s_w + bias + alpha*v), fp64 arithmetic.
 * acc is the exact int32 result from orc_gemm_s32 for the same rows. */
void orc_w8a8_out(const int32_t *C, const float *sx, const float *sw, int64_t M, int64_t N,
                  const int64_t *rows, int64_t n_rows, const uint16_t *bias, const float *v,
                  float alpha, uint16_t *Y)
{
    int64_t R = rows ? n_rows : M;
    for (int64_t i = 0; i < R; ++i) {
        double smx = (double)sx[pick(rows, i)];
        for (int64_t n = 0; n < N; ++n) {
            double y = (double)C[i * N + n] * smx * (double)sw[n];
            Y[i * N + n] = orc_double_to_half(epi_terms(n, bias, v, alpha, y));
        }
    }
}

/* q8 weight-only reference, fp64 and unrounded:
 * Yref[i,n] = sum_k X[rows[i],k] * Wq[n,k] * s_w[n] + bias[n] + alpha*v[n]. */
void orc_wo_q8_ref(const uint16_t *X, const int8_t *Wq, const float *sw, int64_t M, int64_t N,
                   int64_t K, const int64_t *rows, int64_t n_rows, const uint16_t *bias,
                   const float *v, float alpha, double *Yref)
{
    int64_t R = rows ? n_rows : M;
    for (int64_t i = 0; i < R; ++i) {
        const uint16_t *x = X + pick(rows, i) * K;
        for (int64_t n = 0; n < N; ++n) {
            double s = (double)sw[n];
            double y = 0.0;
            for (int64_t k = 0; k < K; ++k)
                y += orc_half_to_double(x[k]) * ((double)Wq[n * K + k] * s);
            Yref[i * N + n] = epi_terms(n, bias, v, alpha, y);
        }
    }
}

/* q4 weight-only reference, fp64 and unrounded:
 * Yref[i,n] = sum_k X[rows[i],k] * (nib[n,k]-8) * s16[n,k/32] + bias[n] + alpha*v[n]. */
void orc_wo_q4_ref(const uint16_t *X, const uint8_t *P, const uint16_t *S, int64_t M, int64_t N,
                   int64_t K, const int64_t *rows, int64_t n_rows, const uint16_t *bias,
                   const float *v, float alpha, double *Yref)
{
    const int64_t G = K / 32;
    int64_t R = rows ? n_rows : M;
    for (int64_t i = 0; i < R; ++i) {
        const uint16_t *x = X + pick(rows, i) * K;
        for (int64_t n = 0; n < N; ++n) {
            double y = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                uint8_t byte = P[n * (K / 2) + k / 2];
                int nib = (k & 1) ? (byte >> 4) : (byte & 0x0f);
                double w = (double)(nib - 8) * orc_half_to_double(S[n * G + k / 32]);
                y += orc_half_to_double(x[k]) * w;
            }
            Yref[i * N + n] = epi_terms(n, bias, v, alpha, y);
        }
    }
}

/* fp16 (unquantised) reference, fp64 and unrounded (the fp16 column of the
 * "Results" precision table):
 * Yref[i,n] = sum_k X[rows[i],k] * W[n,k] + bias[n] + alpha*v[n]. */
void orc_f16_ref(const uint16_t *X, const uint16_t *W, int64_t M, int64_t N, int64_t K,
                 const int64_t *rows, int64_t n_rows, const uint16_t *bias, const float *v,
                 float alpha, double *Yref)
{
    int64_t R = rows ? n_rows : M;
    for (int64_t i = 0; i < R; ++i) {
        const uint16_t *x = X + pick(rows, i) * K;
        for (int64_t n = 0; n < N; ++n) {
            const uint16_t *w = W + n * K;
            double y = 0.0;
            for (int64_t k = 0; k < K; ++k)
                y += orc_half_to_double(x[k]) * orc_half_to_double(w[k]);
            Yref[i * N + n] = epi_terms(n, bias, v, alpha, y);
        }
    }
}
