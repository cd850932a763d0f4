/*
 * wq_oracle.c -- plain, slow CPU oracle for group-wise weight quantisation
 * and the dequant-then-matmul that reads it.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this code.  It shares nothing with
 * the CUDA library (no headers, helpers, tables or constants) and the CUDA
 * library never calls it.
 *
 * Sources (web pages; cited by title and section):
 *  [P2] "Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF --
 *       the model's accounting zoom" (blog.lo0.es), section "The minimum
 *       maths: scale and zero-point" (scale, zero-point, encode and decode
 *       equations) and section "Numerical example" (8-weight table, storage).
 *  [P3] "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and
 *       KV-Cache Quantization" (cruxly.in), section "What quantisation does:
 *       scale, round, and the outlier that ruins a group" (symmetric absmax
 *       INT8, granularity: per tensor / per output channel / per group).
 *  [P1C] "Test-time quantization: quantising on the fly with no calibration
 *       dataset" (blog.lo0.es), section "The error of quantising an outlier
 *       with the wrong scale" (rounding error bounded by half a scale).
 *
 * Arithmetic rules (the pages do not fix them; these readings are listed
 * with the rest in the design notes):
 *  - Quantisation runs in IEEE binary32 with round-to-nearest-even for every
 *    operation; "round" is round-half-to-even (nearbyintf in the default
 *    rounding mode).  Build with -ffp-contract=off and no fast-math.
 *  - mode WQ_ORACLE_STORED (the library's format): the scale and the
 *    zero-point are rounded to bf16 (round-to-nearest-even) and the codes are
 *    chosen against those stored values, so the decode the codes were chosen
 *    for is exactly the decode that runs.
 *  - mode WQ_ORACLE_EXACT: s and z stay binary32, no bf16 rounding; used to
 *    check the pages' own numbers and the half-a-scale error bound.
 *  - Degenerate group (the pages are silent): if the scale comes out 0 (all
 *    values equal, or a range too small to represent), the scale becomes
 *    max(|min|, |max|) for INT4; if that is also 0 the scale is 1.  A group of
 *    equal values c then decodes to c (when c is representable in the scale's
 *    precision) and an all-zero group decodes to 0.
 *  - Dequantisation and the matmul run in binary64.  s*(q - z) with a bf16 or
 *    binary32 s and small integers q, z is exact in binary64.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define WQ_ORACLE_EXACT 0
#define WQ_ORACLE_STORED 1

/* ---------------------------------------------------------------------- */
/* bf16 <-> binary32.  bf16 is the top 16 bits of a binary32.              */
/* ---------------------------------------------------------------------- */

static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float bits_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* Round a binary32 to the nearest bf16, ties to even (the 16 dropped bits
 * decide; an exact half rounds towards the even kept value).  Inputs are
 * finite by contract; a NaN is returned as a quiet NaN. */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u = f32_bits(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xffffu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept += 1u;
    return (uint16_t)kept;
}

float oracle_bf16_to_f32(uint16_t h) { return bits_f32((uint32_t)h << 16); }

void oracle_f32_to_bf16_array(const float *src, int64_t n, uint16_t *dst)
{
    for (int64_t i = 0; i < n; ++i) dst[i] = oracle_f32_to_bf16(src[i]);
}

/* Apply the storage rounding of the chosen mode to a parameter. */
static float store_param(float v, int mode)
{
    return mode == WQ_ORACLE_STORED ? oracle_bf16_to_f32(oracle_f32_to_bf16(v)) : v;
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------------- */
/* Asymmetric INT4, one (s, z) per group of g consecutive weights of a row. */
/* [P2] "The minimum maths": s = (max - min)/(2^b - 1), z = round(-min/s),  */
/*      q = clip(round(w/s + z), 0, 2^b - 1), w_hat = s*(q - z).            */
/* ---------------------------------------------------------------------- */

/*
 * w      : [N][ldw] binary32 (bf16 inputs are widened exactly by the caller)
 * codes  : [N][K] output codes 0..15, one per byte (unpacked)
 * s_out  : [N][K/g] scale as used for encoding (binary32 value)
 * z_out  : [N][K/g] zero-point as used for encoding (binary32 value)
 * Returns 0, or -1 if g does not divide K or a size is not positive.
 */
int oracle_quantize_int4(const float *w, int64_t N, int64_t K, int64_t ldw, int64_t g, int mode,
                         uint8_t *codes, float *s_out, float *z_out)
{
    if (N <= 0 || K <= 0 || g <= 0 || K % g != 0 || ldw < K) return -1;
    const int64_t G = K / g;
    int64_t n;
#pragma omp parallel for schedule(static)
    for (n = 0; n < N; ++n) {
        for (int64_t gi = 0; gi < G; ++gi) {
            const float *wg = w + n * ldw + gi * g;
            /* min and max over the group (exact). */
            float mn = wg[0], mx = wg[0];
            for (int64_t i = 1; i < g; ++i) {
                if (wg[i] < mn) mn = wg[i];
                if (wg[i] > mx) mx = wg[i];
            }
            /* s = (max - min) / 15 : one binary32 subtraction, one division. */
            float s = store_param((mx - mn) / 15.0f, mode);
            if (s == 0.0f) {
                /* degenerate group: no range to spread over 16 levels. */
                float amax = fabsf(mn) > fabsf(mx) ? fabsf(mn) : fabsf(mx);
                s = store_param(amax, mode);
                if (s == 0.0f) s = 1.0f;
            }
            /* z = round(-min / s); adding +0 turns a -0 into +0. */
            float z = store_param(nearbyintf(-mn / s) + 0.0f, mode);
            s_out[n * G + gi] = s;
            z_out[n * G + gi] = z;
            /* q = clip(round(w/s + z), 0, 15). */
            for (int64_t i = 0; i < g; ++i) {
                float t = nearbyintf(wg[i] / s + z);
                if (t < 0.0f) t = 0.0f;
                if (t > 15.0f) t = 15.0f;
                codes[n * K + gi * g + i] = (uint8_t)t;
            }
        }
    }
    return 0;
}

/* Two 4-bit codes per byte: byte j of a row holds code 2j in bits 0-3 and
 * code 2j+1 in bits 4-7 ([P2] "Numerical example": 8 codes x 4 bits = 4 B). */
int oracle_pack_int4(const uint8_t *codes, int64_t N, int64_t K, uint8_t *packed)
{
    if (N <= 0 || K <= 0 || K % 2 != 0) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K / 2; ++j)
            packed[n * (K / 2) + j] =
                (uint8_t)((codes[n * K + 2 * j] & 0xf) | ((codes[n * K + 2 * j + 1] & 0xf) << 4));
    return 0;
}

int oracle_unpack_int4(const uint8_t *packed, int64_t N, int64_t K, uint8_t *codes)
{
    if (N <= 0 || K <= 0 || K % 2 != 0) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K / 2; ++j) {
            codes[n * K + 2 * j] = packed[n * (K / 2) + j] & 0xf;
            codes[n * K + 2 * j + 1] = packed[n * (K / 2) + j] >> 4;
        }
    return 0;
}

/* ---------------------------------------------------------------------- */
/* Symmetric INT4, one s per group, levels -7..7.                           */
/* [P1C] "The error of quantising an outlier with the wrong scale": a       */
/*      b-bit symmetric range covering a largest magnitude M has            */
/*      s = M / (2^(b-1) - 1), M/7 at 4 bits.  [P3] "The methods compared"  */
/*      (the AWQ example): symmetric int4 with codes -7 to 7.               */
/*      q = clip(round(w/s), -7, 7), w_hat = q*s; max|w| = 0 gives s = 1.   */
/*      The code is stored as q + 8 (1..15) in the INT4 nibble layout, so   */
/*      the asymmetric decode s*(code - z) with z = 8 reads it as q*s.      */
/* ---------------------------------------------------------------------- */

/*
 * codes  : [N][K] output codes q + 8, one per byte (unpacked)
 * s_out  : [N][K/g] scale as used for encoding
 */
int oracle_quantize_int4_sym(const float *w, int64_t N, int64_t K, int64_t ldw, int64_t g, int mode,
                             uint8_t *codes, float *s_out)
{
    if (N <= 0 || K <= 0 || g <= 0 || K % g != 0 || ldw < K) return -1;
    const int64_t G = K / g;
    int64_t n;
#pragma omp parallel for schedule(static)
    for (n = 0; n < N; ++n) {
        for (int64_t gi = 0; gi < G; ++gi) {
            const float *wg = w + n * ldw + gi * g;
            float amax = 0.0f;  /* largest magnitude of the group */
            for (int64_t i = 0; i < g; ++i) {
                const float a = fabsf(wg[i]);
                if (a > amax) amax = a;
            }
            float s = store_param(amax / 7.0f, mode);
            if (s == 0.0f) s = 1.0f;
            s_out[n * G + gi] = s;
            for (int64_t i = 0; i < g; ++i) {
                float q = nearbyintf(wg[i] / s);
                if (q < -7.0f) q = -7.0f;
                if (q > 7.0f) q = 7.0f;
                codes[n * K + gi * g + i] = (uint8_t)((int)q + 8);
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------- */
/* Symmetric absmax INT8, one s per group (g = K: one per output channel).  */
/* [P3] "What quantisation does": s = max|w| / 127, q = round(w/s),        */
/*      w_hat = q*s.  q is clipped to [-127, 127] because the stored bf16   */
/*      s may be slightly below max|w|/127 (the page gives no clip).        */
/* ---------------------------------------------------------------------- */

int oracle_quantize_int8(const float *w, int64_t N, int64_t K, int64_t ldw, int64_t g, int mode,
                         int8_t *codes, float *s_out)
{
    if (N <= 0 || K <= 0 || g <= 0 || K % g != 0 || ldw < K) return -1;
    const int64_t G = K / g;
    int64_t n;
#pragma omp parallel for schedule(static)
    for (n = 0; n < N; ++n) {
        for (int64_t gi = 0; gi < G; ++gi) {
            const float *wg = w + n * ldw + gi * g;
            float amax = 0.0f;
            for (int64_t i = 0; i < g; ++i)
                if (fabsf(wg[i]) > amax) amax = fabsf(wg[i]);
            float s = store_param(amax / 127.0f, mode);
            if (s == 0.0f) s = 1.0f;
            s_out[n * G + gi] = s;
            for (int64_t i = 0; i < g; ++i) {
                float t = nearbyintf(wg[i] / s);
                if (t < -127.0f) t = -127.0f;
                if (t > 127.0f) t = 127.0f;
                codes[n * K + gi * g + i] = (int8_t)t;
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------- */
/* Dequantisation in binary64 (exact for these operands).                   */
/* ---------------------------------------------------------------------- */

/* [P2] decode equation: w_hat = s * (q - z). */
int oracle_dequant_int4(const uint8_t *codes, const float *s, const float *z, int64_t N, int64_t K,
                        int64_t g, double *w_hat)
{
    if (N <= 0 || K <= 0 || g <= 0 || K % g != 0) return -1;
    const int64_t G = K / g;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            w_hat[n * K + k] =
                (double)s[n * G + k / g] * ((double)codes[n * K + k] - (double)z[n * G + k / g]);
    return 0;
}

/* [P3] dequantised value = q * s. */
int oracle_dequant_int8(const int8_t *codes, const float *s, int64_t N, int64_t K, int64_t g,
                        double *w_hat)
{
    if (N <= 0 || K <= 0 || g <= 0 || K % g != 0) return -1;
    const int64_t G = K / g;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            w_hat[n * K + k] = (double)s[n * G + k / g] * (double)codes[n * K + k];
    return 0;
}

/* ---------------------------------------------------------------------- */
/* The weight-only matmul, y[m][n] = sum_k x[m][k] * w_hat[n][k], binary64. */
/* Also a[m][n] = sum_k |x[m][k] * w_hat[n][k]|, the scale of the rounding   */
/* error any finite-precision evaluation of y may make.                      */
/* ---------------------------------------------------------------------- */

int oracle_matmul(const double *x, const double *w_hat, int64_t M, int64_t N, int64_t K,
                  double *y, double *a)
{
    if (M <= 0 || N <= 0 || K <= 0) return -1;
    int64_t mn;
#pragma omp parallel for schedule(static)
    for (mn = 0; mn < M * N; ++mn) {
        const int64_t m = mn / N, n = mn % N;
        double acc = 0.0, aacc = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const double p = x[m * K + k] * w_hat[n * K + k];
            acc += p;
            aacc += fabs(p);
        }
        y[m * N + n] = acc;
        if (a) a[m * N + n] = aacc;
    }
    return 0;
}

/* ---------------------------------------------------------------------- */
/* FP8 (groundwork for the FP8 W8A8 row).                                   */
/* "Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF",        */
/* section "FP8: the Hopper/Blackwell datacenter format": E4M3 has 4        */
/* exponent and 3 mantissa bits, range +-448; E5M2 has 5 and 2, range       */
/* +-57,344.  Reading: binary formats with exponent bias 2^(e-1) - 1 and    */
/* subnormals.  E4M3 keeps finite values in its all-ones exponent (448 is   */
/* 1.75 * 2^8) and only the all-ones pattern is NaN; E5M2 keeps the         */
/* all-ones exponent for infinities and NaN (57,344 = 1.75 * 2^15).         */
/* Encoding rounds to the nearest value, ties to the even code, and         */
/* saturates finite values beyond the range to +-max.                       */
/* fmt 0 = E4M3, fmt 1 = E5M2.                                              */
/* ---------------------------------------------------------------------- */

/* The value of an FP8 code; NaN for NaN codes, +-inf for E5M2 infinities. */
double oracle_fp8_decode(uint8_t code, int fmt)
{
    const int ebits = fmt == 0 ? 4 : 5, mbits = fmt == 0 ? 3 : 2;
    const int bias = (1 << (ebits - 1)) - 1;
    const int sign = code >> 7;
    const int e = (code >> mbits) & ((1 << ebits) - 1);
    const int m = code & ((1 << mbits) - 1);
    double v;
    if (fmt == 0 && e == 15 && m == 7) return NAN;
    if (fmt == 1 && e == 31) v = m == 0 ? INFINITY : NAN;
    else if (e == 0) v = ldexp((double)m, 1 - bias - mbits);
    else v = ldexp(1.0 + (double)m / (double)(1 << mbits), e - bias);
    return sign ? -v : v;
}

/* Largest finite value of the format. */
double oracle_fp8_max(int fmt) { return fmt == 0 ? 448.0 : 57344.0; }

/* Nearest finite FP8 code to v (ties to the even code), saturating beyond +-max; NaN for non-finite v.
 * Plain exhaustive search over the codes of v's sign. */
uint8_t oracle_fp8_encode(float v, int fmt)
{
    const uint8_t nan_code = fmt == 0 ? 0x7f : 0x7f;
    if (!isfinite(v)) return nan_code;
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a > oracle_fp8_max(fmt)) a = oracle_fp8_max(fmt);
    int best = -1;
    double best_d = 0.0;
    for (int c = 0; c < 128; ++c) {
        const double cv = oracle_fp8_decode((uint8_t)c, fmt);
        if (!isfinite(cv)) continue;
        const double d = fabs(cv - a);
        if (best < 0 || d < best_d || (d == best_d && (c & 1) == 0)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)(sign | best);
}

/* FP8 quantisation, one binary32 scale per row (per output channel):
 * s = max|w| / max_fmt (1 when the row is all zero), code = encode(w / s). */
int oracle_quantize_fp8_rows(const float *w, int64_t N, int64_t K, int64_t ldw, int fmt, uint8_t *codes,
                             float *s_out)
{
    if (N <= 0 || K <= 0 || ldw < K || (fmt != 0 && fmt != 1)) return -1;
    int64_t n;
#pragma omp parallel for schedule(static)
    for (n = 0; n < N; ++n) {
        const float *row = w + n * ldw;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k)
            if (fabsf(row[k]) > amax) amax = fabsf(row[k]);
        float s = amax / (float)oracle_fp8_max(fmt);
        if (s == 0.0f) s = 1.0f;
        s_out[n] = s;
        for (int64_t k = 0; k < K; ++k) codes[n * K + k] = oracle_fp8_encode(row[k] / s, fmt);
    }
    return 0;
}

/* w_hat[n][k] = s[n] * value(code) in binary64. */
int oracle_dequant_fp8_rows(const uint8_t *codes, const float *s, int64_t N, int64_t K, int fmt, double *out)
{
    if (N <= 0 || K <= 0) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            out[n * K + k] = (double)s[n] * oracle_fp8_decode(codes[n * K + k], fmt);
    return 0;
}

/* ---------------------------------------------------------------------- */
/* NVFP4 (groundwork for the NVFP4 row).                                    */
/* "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache   */
/* Quantization", section "Hardware, formats and the roofline": NVFP4 holds */
/* 4-bit values with one 8-bit (E4M3) scale per 16 values plus an fp32      */
/* tensor scale, 4.5 bits per weight; "Quantization for LLM inference ...", */
/* section "Microscaling: NVFP4 and MXFP4": small blocks (16 or 32 values)  */
/* with an FP8 scale.  Readings (the pages do not define the 4-bit values   */
/* or how the scales are chosen): the 4-bit values are E2M1 (sign, 2        */
/* exponent bits with bias 1, 1 mantissa bit: 0, 0.5, 1, 1.5, 2, 3, 4, 6);  */
/* the tensor scale is max|w| / (6 * 448), so block scales fit E4M3; a      */
/* block's scale is the E4M3 code of (block max|w| / 6) / tensor scale;     */
/* values are the nearest E2M1 of w / (block scale * tensor scale), ties to */
/* the even code, saturating at +-6.                                        */
/* ---------------------------------------------------------------------- */

double oracle_e2m1_decode(uint8_t code)
{
    const int sign = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    const double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return sign ? -v : v;
}

/* Nearest E2M1 code to v (ties to the even code), saturating at +-6; exhaustive over the 8 magnitudes. */
uint8_t oracle_e2m1_encode(float v)
{
    const uint8_t sign = signbit(v) ? 8 : 0;
    double a = fabs((double)v);
    if (!(a <= 6.0)) a = 6.0;  /* also maps NaN to the largest magnitude */
    int best = 0;
    double best_d = fabs(oracle_e2m1_decode(0) - a);
    for (int c = 1; c < 8; ++c) {
        const double d = fabs(oracle_e2m1_decode((uint8_t)c) - a);
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)(sign | best);
}

/*
 * codes       : [N][K] E2M1 codes, one per byte
 * block_codes : [N][K/16] E4M3 codes of the block scales
 * tensor_scale: the binary32 tensor scale
 */
int oracle_quantize_nvfp4(const float *w, int64_t N, int64_t K, int64_t ldw, uint8_t *codes,
                          uint8_t *block_codes, float *tensor_scale)
{
    if (N <= 0 || K <= 0 || K % 16 != 0 || ldw < K) return -1;
    float amax = 0.0f;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            if (fabsf(w[n * ldw + k]) > amax) amax = fabsf(w[n * ldw + k]);
    float st = amax / (6.0f * 448.0f);
    if (st == 0.0f) st = 1.0f;
    *tensor_scale = st;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t b = 0; b < K / 16; ++b) {
            const float *wb = w + n * ldw + b * 16;
            float bmax = 0.0f;
            for (int i = 0; i < 16; ++i)
                if (fabsf(wb[i]) > bmax) bmax = fabsf(wb[i]);
            const uint8_t sc = oracle_fp8_encode((bmax / 6.0f) / st, 0);
            block_codes[n * (K / 16) + b] = sc;
            const float S = (float)oracle_fp8_decode(sc, 0) * st;
            for (int i = 0; i < 16; ++i)
                codes[n * K + b * 16 + i] = S == 0.0f ? 0 : oracle_e2m1_encode(wb[i] / S);
        }
    return 0;
}

/* w_hat = e2m1(code) * e4m3(block code) * tensor scale, binary64. */
int oracle_dequant_nvfp4(const uint8_t *codes, const uint8_t *block_codes, float tensor_scale, int64_t N,
                         int64_t K, double *out)
{
    if (N <= 0 || K <= 0 || K % 16 != 0) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            out[n * K + k] = oracle_e2m1_decode(codes[n * K + k]) *
                             oracle_fp8_decode(block_codes[n * (K / 16) + k / 16], 0) * (double)tensor_scale;
    return 0;
}
