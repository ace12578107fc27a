/*
 * zq_oracle.c — plain, slow, obviously-correct CPU oracle for the weight-only
 * quantized linear layer.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may load or call this code. It shares no code, header, table
 * or constant with the CUDA library; the library never loads it.
 *
 * Sources (cited by page title and section):
 *   [wiki]  "ZSE - open-source движок для запуска LLM локально на GPU - 2026"
 *           (wiki.iphoster.net), section "Формат модели .zse": per group of 128
 *           weights scale = (max - min)/15, zero = min,
 *           q = clamp(round((w - zero)/scale), 0, 15); two INT4 codes per byte,
 *           low nibble first; scales and zeros stored as float16.
 *   [lavx]  "ZSE: A Memory-Efficient LLM Inference Engine with Smart Resource
 *           Orchestration", section "Technical Architecture" (zQuantize:
 *           per-tensor INT2-8 mixed precision).
 *
 * Readings where the pages leave a step open (all listed in the design notes):
 *   - b-bit codes use L = 2^b - 1 in place of 15 (b in {2,3,4,8}).
 *   - q is computed from the STORED fp16 scale and zero (s16, z16).
 *   - "round" is round-half-to-even; all arithmetic is IEEE fp64 with one
 *     rounding to fp16 for the stored scale and zero.
 *   - scale == 0 (constant group or fp16 underflow): every q is 0, so the
 *     dequantized value is z16.
 *   - codes of a row form one little-endian bitstream: bit t of the stream is
 *     bit (t mod 32) of word t/32; code i occupies bits [i*b, i*b+b). At b=4
 *     this is exactly "two codes per byte, low nibble first".
 *   - dequant: w_hat = q*s16 + z16 (zero is the float minimum, not an integer
 *     zero point), computed exactly in fp64.
 *   - linear: y[m][n] = sum_k x[m][k]*w_hat[n][k] in fp64 (W is N x K, the
 *     PyTorch Linear convention y = x W^T); bound = sum_k |x||w_hat|.
 *   - group sizes: 128 (the pages' figure) and also 32 and 64 (the encoding
 *     variants: the same quantizer on shorter groups, scale/zero per group).
 *   - fp16 passthrough (the .zse format keeps some tensors unquantized):
 *     bits = 16 means the weights are fp16 values used as they are.
 *   - bf16 activations: x given as bfloat16 (the top 16 bits of a binary32),
 *     decoded exactly.
 *   - symmetric quantization (listed by [wiki] for INT8 without a formula):
 *     Q = 2^(b-1) - 1, scale = fp16(max|w| / Q), q = clamp(round(w/scale),
 *     -Q, Q); stored as code = q + 2^(b-1), zero = -2^(b-1)*scale (exact), so
 *     the same dequant gives q*scale.  A zero below -65504 is rejected.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -fopenmp -ffp-contract=off
 *        (no -ffast-math: the fp64 steps must be plain IEEE operations).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ZO_OK 0
#define ZO_INVALID 1
#define ZO_UNSUPPORTED 2
#define ZO_NONFINITE 3

/* bfloat16, written from its definition: the upper half of an IEEE binary32 */
/*   1 sign bit, 8 exponent bits (bias 127), 7 fraction bits;               */
/*   e in 1..254: 2^(e-127) * (1 + f/128); e == 0: 2^-126 * f/128;          */
/*   e == 255: infinity (f == 0) or NaN.                                    */
double zo_bf16_to_f64(uint16_t b)
{
    int sign = (b >> 15) & 1;
    int e = (b >> 7) & 0xFF;
    int f = b & 0x7F;
    double v;
    if (e == 0)
        v = ldexp((double)f, -133);              /* f * 2^-126 / 128 */
    else if (e == 255)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + f), e - 134);   /* (128+f) * 2^(e-127-7) */
    return sign ? -v : v;
}

/* Round-to-nearest, ties-to-even conversion of an fp64 value to bfloat16
 * (the largest finite value is (2 - 2^-7) * 2^127; the midpoint above it
 * overflows to infinity). */
uint16_t zo_f64_to_bf16(double v)
{
    if (isnan(v))
        return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a >= ldexp(255.5, 120))                  /* (2 - 2^-8) * 2^127 */
        return sign | 0x7F80;
    if (a < ldexp(1.0, -126)) {
        double m = rint(ldexp(a, 133));          /* multiples of 2^-133: 0 .. 128 */
        return sign | (uint16_t)m;               /* m == 128 encodes 2^-126 */
    }
    int ex;
    (void)frexp(a, &ex);
    int E = ex - 1;                              /* 2^E <= a < 2^(E+1) */
    double m = rint(ldexp(a, 7 - E));            /* 128 .. 256 */
    if (m == 256.0) {
        m = 128.0;
        E += 1;
    }
    if (E > 127)
        return sign | 0x7F80;
    return sign | (uint16_t)((E + 127) << 7) | (uint16_t)(m - 128.0);
}

/* ------------------------------------------------------------------------ */
/* IEEE-754 binary16, written from the format's definition:                 */
/*   1 sign bit, 5 exponent bits (bias 15), 10 fraction bits;               */
/*   e in 1..30: value 2^(e-15) * (1 + f/1024); e == 0: 2^-14 * f/1024;     */
/*   e == 31: infinity (f == 0) or NaN.                                     */
/* ------------------------------------------------------------------------ */

double zo_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int f = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);               /* subnormal: f * 2^-24 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);   /* (1024+f) * 2^(e-15-10) */
    return sign ? -v : v;
}

/* Round-to-nearest, ties-to-even conversion of an fp64 value to binary16.
 * Relies on rint() under the default rounding mode (nearest-even). */
uint16_t zo_f64_to_f16(double v)
{
    if (isnan(v))
        return 0x7E00;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    /* 65504 is the largest finite half; the next step would be 65536, and the
     * midpoint 65520 rounds to the even neighbour, i.e. overflows. */
    if (a >= 65520.0)
        return sign | 0x7C00;
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: representable values are multiples of 2^-24 */
        double m = rint(ldexp(a, 24));           /* 0 .. 1024 */
        return sign | (uint16_t)m;               /* m == 1024 encodes 2^-14 */
    }
    int ex;
    (void)frexp(a, &ex);                         /* 2^(ex-1) <= a < 2^ex */
    int E = ex - 1;
    double m = rint(ldexp(a, 10 - E));           /* 1024 .. 2048 */
    if (m == 2048.0) {                           /* carried into next binade */
        m = 1024.0;
        E += 1;
    }
    return sign | (uint16_t)((E + 15) << 10) | (uint16_t)(m - 1024.0);
}

/* ------------------------------------------------------------------------ */
/* Quantizer: one group, [wiki] "Формат модели .zse", L = 2^b - 1.          */
/* ------------------------------------------------------------------------ */

int zo_quantize_group(const float *w, int n, int L,
                      uint16_t *s16_out, uint16_t *z16_out, uint8_t *q)
{
    for (int i = 0; i < n; ++i)
        if (!isfinite(w[i]) || fabs((double)w[i]) > 65504.0)
            return ZO_NONFINITE;
    double mn = w[0], mx = w[0];
    for (int i = 1; i < n; ++i) {
        if (w[i] < mn) mn = w[i];
        if (w[i] > mx) mx = w[i];
    }
    uint16_t z16 = zo_f64_to_f16(mn);                     /* zero = min   */
    uint16_t s16 = zo_f64_to_f16((mx - mn) / (double)L);  /* scale        */
    double s = zo_f16_to_f64(s16);
    double z = zo_f16_to_f64(z16);
    for (int i = 0; i < n; ++i) {
        if (s == 0.0) {
            q[i] = 0;
            continue;
        }
        double t = rint(((double)w[i] - z) / s);          /* round half even */
        if (t < 0.0) t = 0.0;
        if (t > (double)L) t = (double)L;
        q[i] = (uint8_t)t;
    }
    *s16_out = s16;
    *z16_out = z16;
    return ZO_OK;
}

/* ------------------------------------------------------------------------ */
/* Symmetric quantizer: one group.  [wiki] "Формат модели .zse" lists       */
/* symmetric INT8 quantization (reserved) beside the asymmetric INT4 one,   */
/* without a formula.  Reading: Q = 2^(b-1) - 1 (127 at b = 8),             */
/* scale = max|w| / Q, q = clamp(round(w / scale), -Q, Q), w_hat = q*scale, */
/* with the same fp64 steps and fp16 rounding as the asymmetric quantizer.  */
/* Stored in the asymmetric format: code = q + 2^(b-1), zero = -2^(b-1) *   */
/* s16 (exact, a power-of-two multiple), so code*s16 + zero = q*s16.        */
/* ------------------------------------------------------------------------ */

int zo_quantize_group_symmetric(const float *w, int n, int bits,
                                uint16_t *s16_out, uint16_t *z16_out, uint8_t *codes)
{
    for (int i = 0; i < n; ++i)
        if (!isfinite(w[i]) || fabs((double)w[i]) > 65504.0)
            return ZO_NONFINITE;
    double half = (double)(1 << (bits - 1));          /* code offset 2^(b-1) */
    double Q = half - 1.0;                            /* largest |q|         */
    double amax = 0.0;
    for (int i = 0; i < n; ++i)
        if (fabs((double)w[i]) > amax) amax = fabs((double)w[i]);
    uint16_t s16 = zo_f64_to_f16(amax / Q);           /* scale               */
    double s = zo_f16_to_f64(s16);
    double z = -half * s;                             /* zero, exact in fp64 */
    if (z < -65504.0)
        return ZO_NONFINITE;                          /* zero not storable   */
    for (int i = 0; i < n; ++i) {
        double t = 0.0;
        if (s != 0.0) {
            t = rint((double)w[i] / s);               /* round half even     */
            if (t < -Q) t = -Q;
            if (t > Q) t = Q;
        }
        codes[i] = (uint8_t)(t + half);
    }
    *s16_out = s16;
    *z16_out = zo_f64_to_f16(z);
    return ZO_OK;
}

/* ------------------------------------------------------------------------ */
/* Bitstream packing of one row: code i -> stream bits [i*b, i*b+b);        */
/* stream bit t -> bit (t % 32) of word t / 32. Done bit by bit on purpose. */
/* ------------------------------------------------------------------------ */

void zo_pack_row(const uint8_t *codes, int K, int bits, uint32_t *words)
{
    int nw = K * bits / 32;
    memset(words, 0, (size_t)nw * sizeof(uint32_t));
    for (int i = 0; i < K; ++i)
        for (int j = 0; j < bits; ++j) {
            long t = (long)i * bits + j;
            if ((codes[i] >> j) & 1u)
                words[t / 32] |= 1u << (t % 32);
        }
}

void zo_unpack_row(const uint32_t *words, int K, int bits, uint8_t *codes)
{
    for (int i = 0; i < K; ++i) {
        unsigned c = 0;
        for (int j = 0; j < bits; ++j) {
            long t = (long)i * bits + j;
            c |= ((words[t / 32] >> (t % 32)) & 1u) << j;
        }
        codes[i] = (uint8_t)c;
    }
}

static int zo_check_format(int N, int K, int bits, int group)
{
    if (!(bits == 2 || bits == 3 || bits == 4 || bits == 8) ||
        !(group == 32 || group == 64 || group == 128))
        return ZO_UNSUPPORTED;
    if (N <= 0 || K <= 0 || K % group != 0)
        return ZO_INVALID;
    return ZO_OK;
}

/* Whole tensor: W is N x K fp32 row-major. packed is N x (K*bits/32) uint32,
 * scales and zeros are N x (K/group) fp16 bit patterns. */
int zo_quantize_pack(const float *w, int N, int K, int bits, int group,
                     uint32_t *packed, uint16_t *scales, uint16_t *zeros)
{
    int st = zo_check_format(N, K, bits, group);
    if (st != ZO_OK)
        return st;
    int L = (1 << bits) - 1;
    int G = K / group;
    int wpr = K * bits / 32;
    int status = ZO_OK;
#pragma omp parallel for schedule(dynamic, 16)
    for (int n = 0; n < N; ++n) {
        uint8_t *codes = (uint8_t *)malloc((size_t)K);
        for (int g = 0; g < G; ++g) {
            int r = zo_quantize_group(w + (size_t)n * K + (size_t)g * group, group, L,
                                      &scales[(size_t)n * G + g],
                                      &zeros[(size_t)n * G + g],
                                      codes + (size_t)g * group);
            if (r != ZO_OK) {
#pragma omp atomic write
                status = r;
            }
        }
        zo_pack_row(codes, K, bits, packed + (size_t)n * wpr);
        free(codes);
    }
    return status;
}

/* Whole tensor, symmetric quantizer; output layout as zo_quantize_pack. */
int zo_quantize_pack_symmetric(const float *w, int N, int K, int bits, int group,
                               uint32_t *packed, uint16_t *scales, uint16_t *zeros)
{
    int st = zo_check_format(N, K, bits, group);
    if (st != ZO_OK)
        return st;
    int G = K / group;
    int wpr = K * bits / 32;
    int status = ZO_OK;
#pragma omp parallel for schedule(dynamic, 16)
    for (int n = 0; n < N; ++n) {
        uint8_t *codes = (uint8_t *)malloc((size_t)K);
        for (int g = 0; g < G; ++g) {
            int r = zo_quantize_group_symmetric(w + (size_t)n * K + (size_t)g * group, group, bits,
                                                &scales[(size_t)n * G + g],
                                                &zeros[(size_t)n * G + g],
                                                codes + (size_t)g * group);
            if (r != ZO_OK) {
#pragma omp atomic write
                status = r;
            }
        }
        zo_pack_row(codes, K, bits, packed + (size_t)n * wpr);
        free(codes);
    }
    return status;
}

int zo_unpack(const uint32_t *packed, int N, int K, int bits, uint8_t *codes)
{
    int st = zo_check_format(N, K, bits, 32);  /* rows of whole words: K a multiple of 32 */
    if (st != ZO_OK)
        return st;
    int wpr = K * bits / 32;
    for (int n = 0; n < N; ++n)
        zo_unpack_row(packed + (size_t)n * wpr, K, bits, codes + (size_t)n * K);
    return ZO_OK;
}

/* w_hat[n][k] = q * s16 + z16 in fp64 (exact: q has <= 8 significant bits and
 * s16 has 11, so q*s16 and the sum with z16 fit in 53 bits). */
int zo_dequant(const uint32_t *packed, const uint16_t *scales, const uint16_t *zeros,
               int bits, int group, int N, int K, double *w_hat)
{
    int st = zo_check_format(N, K, bits, group);
    if (st != ZO_OK)
        return st;
    int G = K / group;
    int wpr = K * bits / 32;
#pragma omp parallel for schedule(dynamic, 16)
    for (int n = 0; n < N; ++n) {
        uint8_t *codes = (uint8_t *)malloc((size_t)K);
        zo_unpack_row(packed + (size_t)n * wpr, K, bits, codes);
        for (int k = 0; k < K; ++k) {
            int g = k / group;
            double s = zo_f16_to_f64(scales[(size_t)n * G + g]);
            double z = zo_f16_to_f64(zeros[(size_t)n * G + g]);
            w_hat[(size_t)n * K + k] = (double)codes[k] * s + z;
        }
        free(codes);
    }
    return ZO_OK;
}

/* Linear on a subset of output columns: for each listed row r of W (output
 * feature), y[m][i] = sum_k x[m][k] * w_hat[r][k] and
 * bound[m][i] = sum_k |x[m][k]| * |w_hat[r][k]|, both fp64. x is M x K fp16
 * (xfmt 0) or bf16 (xfmt 1) bit patterns; y and bound are M x nrows. Pass
 * rows == NULL for all N rows.  bits == 16: `packed` holds the weights as
 * fp16 bit patterns, N x K (read as uint16), w_hat is their value, and
 * scales/zeros are not read. */
int zo_linear_rows_ex(const uint16_t *x, int xfmt, int M, int K,
                      const uint32_t *packed, const uint16_t *scales, const uint16_t *zeros,
                      int bits, int group, int N, const int64_t *rows, int nrows,
                      double *y, double *bound)
{
    int st = bits == 16 ? ((N <= 0 || K <= 0) ? ZO_INVALID : ZO_OK) : zo_check_format(N, K, bits, group);
    if (st != ZO_OK)
        return st;
    if (xfmt != 0 && xfmt != 1)
        return ZO_UNSUPPORTED;
    if (M <= 0)
        return ZO_INVALID;
    if (rows == NULL)
        nrows = N;
    for (int i = 0; i < nrows; ++i) {
        long r = rows ? (long)rows[i] : i;
        if (r < 0 || r >= N)
            return ZO_INVALID;
    }
    int G = bits == 16 ? 0 : K / group;
    int wpr = bits == 16 ? 0 : K * bits / 32;
    double *xd = (double *)malloc((size_t)M * K * sizeof(double));
    for (size_t i = 0; i < (size_t)M * K; ++i)
        xd[i] = xfmt == 1 ? zo_bf16_to_f64(x[i]) : zo_f16_to_f64(x[i]);
#pragma omp parallel for schedule(dynamic, 4)
    for (int i = 0; i < nrows; ++i) {
        long r = rows ? (long)rows[i] : i;
        uint8_t *codes = (uint8_t *)malloc((size_t)K);
        double *wh = (double *)malloc((size_t)K * sizeof(double));
        if (bits == 16) {
            const uint16_t *w16 = (const uint16_t *)packed + (size_t)r * K;
            for (int k = 0; k < K; ++k)
                wh[k] = zo_f16_to_f64(w16[k]);
        } else {
            zo_unpack_row(packed + (size_t)r * wpr, K, bits, codes);
            for (int k = 0; k < K; ++k) {
                int g = k / group;
                double s = zo_f16_to_f64(scales[(size_t)r * G + g]);
                double z = zo_f16_to_f64(zeros[(size_t)r * G + g]);
                wh[k] = (double)codes[k] * s + z;
            }
        }
        for (int m = 0; m < M; ++m) {
            double acc = 0.0, bnd = 0.0;
            const double *xr = xd + (size_t)m * K;
            for (int k = 0; k < K; ++k) {
                acc += xr[k] * wh[k];
                bnd += fabs(xr[k]) * fabs(wh[k]);
            }
            y[(size_t)m * nrows + i] = acc;
            bound[(size_t)m * nrows + i] = bnd;
        }
        free(wh);
        free(codes);
    }
    free(xd);
    return ZO_OK;
}

/* fp16 activations; see zo_linear_rows_ex. */
int zo_linear_rows(const uint16_t *x, int M, int K,
                   const uint32_t *packed, const uint16_t *scales, const uint16_t *zeros,
                   int bits, int group, int N, const int64_t *rows, int nrows,
                   double *y, double *bound)
{
    return zo_linear_rows_ex(x, 0, M, K, packed, scales, zeros, bits, group, N, rows, nrows, y, bound);
}

/* Thread control for timing the oracle on the host cores. */
void zo_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int zo_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
