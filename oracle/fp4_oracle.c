/*
 * fp4_oracle.c -- plain, slow CPU oracle for FP4 (ExMy) weight quantization
 * and the W4A16 matrix multiply.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes
 * or calls this file; only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark load it.  It shares no code, header, table or helper
 * with the CUDA library: every formula here is written out again from the
 * method's description.
 *
 * Sources followed (page title, then section):
 *  - "首个支持4-bit浮点量化的LLM来了" (LLM-FP4 summary), paragraph on the
 *    floating-point number formula: sign s, exponent field p in [0, 2^e-1]
 *    selecting the binade, mantissa bits d_i, integer bias b.
 *  - same page, "scale and clip": clip to +-Qmax with a full-precision
 *    scaling factor kept outside the low-bit product; the bias derived from
 *    the tensor's range can act as a real-valued scale (eq. (2)-(4)).
 *  - same page, "compare and quantize" (eq. (5)): each scaled value goes to
 *    the quantization interval it falls in, i.e. the nearest grid value.
 *  - same page, efficient matrix multiplication: the scale factors are taken
 *    out of the low-bit product.
 *  - same page, search over exponent/mantissa split and quantization range.
 *  - same page, pre-shifted exponent bias: per-channel activation maximum
 *    from calibration data, split into one per-tensor real factor times a
 *    per-channel power of two that is folded into the weights.
 *  - "为什么我们需要4-bit浮点量化" tutorial, section 2.2: two 4-bit values
 *    packed per byte.
 *
 * Readings where the pages' formulas were lost in extraction (each is also
 * listed in the design notes):
 *  R1 value of code (s,p,d):  p == 0 : (-1)^s * 2^(1-b) * (0.d1..dm)_2
 *                             p  > 0 : (-1)^s * 2^(p-b) * (1.d1..dm)_2
 *     no Inf/NaN codes; default bias b = 2^(e-1) - 1, which makes E2M1 the
 *     set {0, .5, 1, 1.5, 2, 3, 4, 6}.  Code = s<<3 | p<<m | d.
 *  R2 bias candidates act as a real scale: clip range = absmax * c_j with
 *     c_j = fl32(2^(-j/8)), j = 0..7 (j = 0 is plain absmax).
 *  R3 scale s = R_store(fl32(fl32(A * c_j) / Qmax)); the STORED scale (fp32,
 *     or fp16 by round-to-nearest-even) is what quantizes and dequantizes.
 *  R4 q = fl32(x / s); magnitude index = nearest grid magnitude, ties to the
 *     even index, |q| >= Qmax saturates to index 7, s == 0 gives index 0;
 *     sign bit = signbit(x) (so -0 and small negatives give code 0x8).
 *  R5 search: SSE = sum (W' - v*s)^2 in fp64 over the whole tensor; the first
 *     strict minimum over formats (E1M2, E2M1, E3M0) x j ascending wins.
 *  R6 pre-shift: c_k = max_m |X[m,k]|, rho = max_k c_k (1 if all zero),
 *     e_k = ceil(log2(c_k / rho)) clamped to [-126, 0] (0 when c_k == 0);
 *     W' = W * 2^e_k;  X~ = bf16(fl32(fl32(X * 2^-e_k) / rho));  Y *= rho.
 *  R10 4-bit activations with the pre-shifted bias: the activation of
 *     channel k is clipped to rho * 2^e_k (the calibration's per-tensor
 *     real factor times the channel's power of two).  The power of two goes
 *     into the weights (R6), so what is quantized is X' = fl32(X * 2^-e_k)
 *     with ONE per-tensor scale s_a = fl32(fl32(rho * c_j) / Qmax) kept in
 *     fp32 (R3 with A = rho); codes by R4 from q = fl32(X' / s_a).  The
 *     product takes both scales out of the low-bit sum:
 *       Y[m,n] = s_a * sum_k v_a(a[m,k]) * v(w[n,k]) * s[n, k/g].
 *  R11 granularity: the absmax A of R3 is taken over a block, either g
 *     consecutive elements of a row (group), a whole row (output channel),
 *     or N/heads consecutive rows (an attention head); the block's scale is
 *     stored in every group slot it covers.  Per-block search: each block
 *     takes the bias index j minimising its own SSE (fp64, first strict
 *     minimum, j ascending); the format stays per tensor.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC.
 * float arithmetic below is IEEE binary32 with round-to-nearest-even
 * (x86-64 SSE, FLT_EVAL_METHOD == 0); contraction into FMA is disabled.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#include "fp4_oracle.h"

/* ---------------------------------------------------------------- formats */

/* (e, m, b) of E1M2, E2M1, E3M0 with the IEEE-style default bias 2^(e-1)-1 */
static const int ORC_E[3] = {1, 2, 3};
static const int ORC_M[3] = {2, 1, 0};

int orc_format_bias(int fmt) { return (1 << (ORC_E[fmt] - 1)) - 1; }

/* Reading R1: value of a 4-bit code in format fmt. */
double orc_code_value(int fmt, int code)
{
    int e = ORC_E[fmt], m = ORC_M[fmt], b = orc_format_bias(fmt);
    int s = (code >> 3) & 1;
    int p = (code >> m) & ((1 << e) - 1);
    int d = code & ((1 << m) - 1);
    double frac = (double)d / (double)(1 << m); /* (0.d1..dm)_2 */
    double v;
    if (p == 0)
        v = ldexp(frac, 1 - b);
    else
        v = ldexp(1.0 + frac, p - b);
    return s ? -v : v;
}

void orc_format_table(int fmt, double mags[8], double *qmax)
{
    for (int i = 0; i < 8; ++i) mags[i] = orc_code_value(fmt, i);
    *qmax = mags[7];
}

/* Reading R2: real-valued bias factor c_j = fl32(2^(-j/8)). */
float orc_bias_factor(int j) { return (float)exp2l(-(long double)j / 8.0L); }

/* ------------------------------------------------------- float rounding */

static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* binary32 -> bfloat16 bits, round to nearest even (NaN kept quiet). */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u = f2u(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

float orc_bf16_to_f32(uint16_t h) { return u2f((uint32_t)h << 16); }

/* binary32 -> binary16 bits, round to nearest even, overflow -> Inf,
 * gradual underflow to subnormals. Written from the binary16 definition:
 * value = the representable binary16 number nearest to f. */
uint16_t orc_f32_to_f16(float f)
{
    uint32_t u = f2u(f);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t a = u & 0x7fffffffu;
    if (a > 0x7f800000u) return (uint16_t)(sign | 0x7e00u);      /* NaN */
    if (a == 0x7f800000u) return (uint16_t)(sign | 0x7c00u);     /* Inf */
    double x = (double)u2f(a);                                    /* exact */
    /* binary16 grid spacing: 2^(E-10) for normal binade 2^E, E >= -14;
     * 2^-24 below 2^-14. */
    int E;
    frexp(x, &E);            /* x = f * 2^E, f in [0.5, 1) -> binade 2^(E-1) */
    int binade = E - 1;
    if (binade < -14) binade = -14;
    double ulp = ldexp(1.0, binade - 10);
    double q = x / ulp;       /* exact: power-of-two division */
    double r = floor(q);
    double rem = q - r;
    if (rem > 0.5 || (rem == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    double y = r * ulp;
    if (y > 65504.0) return (uint16_t)(sign | 0x7c00u);
    /* encode y exactly */
    if (y == 0.0) return sign;
    int Ey;
    frexp(y, &Ey);
    int by = Ey - 1;
    if (by < -14) { /* subnormal: y = k * 2^-24 */
        uint16_t k = (uint16_t)ldexp(y, 24);
        return (uint16_t)(sign | k);
    }
    uint16_t expf = (uint16_t)(by + 15);
    uint16_t mant = (uint16_t)(ldexp(y, -by) * 1024.0 - 1024.0);
    return (uint16_t)(sign | (expf << 10) | mant);
}

float orc_f16_to_f32(uint16_t h)
{
    int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp(1.0 + m / 1024.0, e - 15);
    return (float)(s ? -v : v);
}

/* ------------------------------------------------------------- quantize */

/* Reading R4: nearest magnitude index of |q| among mags[0..7], ties to the
 * even index, saturating at Qmax.  Exhaustive search, distances in fp64
 * (exact: q is a float, the grid values are short dyadic rationals). */
int orc_nearest_index(double a, const double mags[8])
{
    if (a >= mags[7]) return 7;
    int best = 0;
    double bd = fabs(a - mags[0]);
    for (int i = 1; i < 8; ++i) {
        double d = fabs(a - mags[i]);
        if (d < bd) { bd = d; best = i; }
        else if (d == bd && (i % 2) == 0) { best = i; }
    }
    return best;
}

static float pow2f(int e) { return ldexpf(1.0f, e); }

/* Scale of one group (reading R3).  Returns 0 on success, -1 if the stored
 * scale is not finite. */
static int group_scale(float A, float cj, float qmax, int sdt, float *s_out, uint32_t *raw)
{
    float t = A * cj;            /* fl32 */
    float s32 = t / qmax;        /* fl32 IEEE division */
    if (sdt == ORC_SCALE_F16) {
        uint16_t h = orc_f32_to_f16(s32);
        if ((h & 0x7c00u) == 0x7c00u) return -1;
        *raw = h;
        *s_out = orc_f16_to_f32(h);
    } else {
        if (!isfinite(s32)) return -1;
        *raw = f2u(s32);
        *s_out = s32;
    }
    return 0;
}

/* One row of the fixed-choice quantizer.  Writes packed codes and scales
 * when the pointers are not NULL, returns the row's SSE in *sse_row.
 * Returns 0, or an ORC_ERR_* code. */
static int quantize_row(const float *Wrow, int K, int g, int fmt, int j, const int8_t *shift,
                        int sdt, uint8_t *prow, void *srow, double *sse_row)
{
    double mags[8], qmax_d;
    orc_format_table(fmt, mags, &qmax_d);
    float qmax = (float)qmax_d; /* exact */
    float cj = orc_bias_factor(j);
    double sse = 0.0;
    int G = K / g;
    float *wp = (float *)malloc(sizeof(float) * (size_t)g);
    if (!wp) return ORC_ERR_ALLOC;
    for (int gi = 0; gi < G; ++gi) {
        /* fold of the pre-shifted exponent bias (reading R6): W' = W * 2^e */
        float A = 0.0f;
        for (int t = 0; t < g; ++t) {
            int k = gi * g + t;
            float w = Wrow[k];
            if (shift) w = w * pow2f(shift[k]);
            if (!isfinite(w)) { free(wp); return ORC_ERR_NONFINITE; }
            wp[t] = w;
            float a = fabsf(w);
            if (a > A) A = a;
        }
        float s;
        uint32_t raw;
        if (group_scale(A, cj, qmax, sdt, &s, &raw) != 0) { free(wp); return ORC_ERR_SCALE; }
        if (srow) {
            if (sdt == ORC_SCALE_F16) ((uint16_t *)srow)[gi] = (uint16_t)raw;
            else ((uint32_t *)srow)[gi] = raw;
        }
        for (int t = 0; t < g; ++t) {
            float w = wp[t];
            int idx = 0;
            if (s != 0.0f) {
                float q = w / s; /* fl32, IEEE round to nearest */
                idx = orc_nearest_index(fabs((double)q), mags);
            }
            int sign = signbit(w) ? 1 : 0;
            int code = (sign << 3) | idx;
            double v = sign ? -mags[idx] : mags[idx];
            double diff = (double)w - v * (double)s;
            sse += diff * diff;
            if (prow) {
                int k = gi * g + t;
                uint8_t *byte = &prow[k >> 1];
                if ((k & 1) == 0) *byte = (uint8_t)((*byte & 0xf0u) | code);
                else *byte = (uint8_t)((*byte & 0x0fu) | (code << 4));
            }
        }
    }
    free(wp);
    *sse_row = sse;
    return 0;
}

static int check_args(int N, int K, int g)
{
    if (N < 0 || K < 0 || g <= 0 || (g % 2) != 0 || (K % g) != 0) return ORC_ERR_ARG;
    return 0;
}

int orc_quantize_fixed(const float *W, int N, int K, int g, int fmt, int j, const int8_t *shift,
                       int sdt, uint8_t *packed, void *scales, double *sse_out)
{
    int rc = check_args(N, K, g);
    if (rc) return rc;
    if (fmt < 0 || fmt > 2 || j < 0 || j > 7) return ORC_ERR_ARG;
    int G = K / g;
    size_t ssz = (sdt == ORC_SCALE_F16) ? 2 : 4;
    double *rows = (double *)calloc((size_t)(N > 0 ? N : 1), sizeof(double));
    if (!rows) return ORC_ERR_ALLOC;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 16)
    for (int n = 0; n < N; ++n) {
        int e = quantize_row(W + (size_t)n * K, K, g, fmt, j, shift, sdt,
                             packed ? packed + (size_t)n * (K / 2) : NULL,
                             scales ? (char *)scales + (size_t)n * G * ssz : NULL, &rows[n]);
        if (e) {
#pragma omp atomic write
            err = e;
        }
    }
    /* row partials summed in row order: independent of the thread count */
    double sse = 0.0;
    for (int n = 0; n < N; ++n) sse += rows[n];
    free(rows);
    if (err) return err;
    if (sse_out) *sse_out = sse;
    return 0;
}

int orc_quantize(const float *W, int N, int K, int g, int fmt_mode, int bias_search,
                 const int8_t *shift, int sdt, uint8_t *packed, void *scales, int32_t choice[2],
                 double sse24[24])
{
    int rc = check_args(N, K, g);
    if (rc) return rc;
    if (fmt_mode < -1 || fmt_mode > 2) return ORC_ERR_ARG;
    int f0 = fmt_mode < 0 ? 0 : fmt_mode, f1 = fmt_mode < 0 ? 2 : fmt_mode;
    int j1 = bias_search ? 7 : 0;
    for (int c = 0; c < 24; ++c) sse24[c] = NAN;
    int bf = f0, bj = 0;
    double best = INFINITY;
    int single = (f0 == f1 && j1 == 0);
    if (!single) {
        for (int f = f0; f <= f1; ++f)
            for (int j = 0; j <= j1; ++j) {
                double s;
                int e = orc_quantize_fixed(W, N, K, g, f, j, shift, sdt, NULL, NULL, &s);
                if (e) return e;
                sse24[f * 8 + j] = s;
                if (s < best) { best = s; bf = f; bj = j; } /* first strict minimum */
            }
    }
    double s;
    int e = orc_quantize_fixed(W, N, K, g, bf, bj, shift, sdt, packed, scales, &s);
    if (e) return e;
    if (single) sse24[bf * 8 + bj] = s;
    choice[0] = bf;
    choice[1] = bj;
    return 0;
}

/* ----------------------------------------------------------- dequantize */

static double code_times_scale(int fmt, int code, double s) { return orc_code_value(fmt, code) * s; }

static float load_scale(const void *scales, int sdt, size_t idx)
{
    if (sdt == ORC_SCALE_F16) return orc_f16_to_f32(((const uint16_t *)scales)[idx]);
    return ((const float *)scales)[idx];
}

int orc_dequantize(const uint8_t *packed, const void *scales, int sdt, int fmt, int N, int K, int g,
                   double *W_hat)
{
    int rc = check_args(N, K, g);
    if (rc) return rc;
    int G = K / g;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            uint8_t b = packed[(size_t)n * (K / 2) + (k >> 1)];
            int code = (k & 1) ? (b >> 4) : (b & 15);
            double s = load_scale(scales, sdt, (size_t)n * G + k / g);
            W_hat[(size_t)n * K + k] = code_times_scale(fmt, code, s);
        }
    return 0;
}

/* ----------------------------------------------------------------- GEMM */

/* Y[m,n] = rho * sum_k X[m,k] * v(code[n,k]) * s[n, k/g], all in fp64, in
 * increasing k.  The plain definition of the W4A16 product with the scale
 * factored per group. */
static double gemm_one(const uint16_t *X, const uint8_t *packed, const void *scales, int sdt,
                       int fmt, int K, int g, double rho, int m, int n)
{
    int G = K / g;
    double acc = 0.0;
    const uint16_t *xr = X + (size_t)m * K;
    const uint8_t *pr = packed + (size_t)n * (K / 2);
    for (int k = 0; k < K; ++k) {
        int code = (k & 1) ? (pr[k >> 1] >> 4) : (pr[k >> 1] & 15);
        double w = code_times_scale(fmt, code, (double)load_scale(scales, sdt, (size_t)n * G + k / g));
        acc += (double)orc_bf16_to_f32(xr[k]) * w;
    }
    return rho * acc;
}

int orc_gemm(const uint16_t *X, const uint8_t *packed, const void *scales, int sdt, int fmt, int M,
             int N, int K, int g, float rho, double *Y)
{
    if (M < 0) return ORC_ERR_ARG;
    int rc = check_args(N, K, g);
    if (rc) return rc;
#pragma omp parallel for collapse(2) schedule(static)
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n)
            Y[(size_t)m * N + n] = gemm_one(X, packed, scales, sdt, fmt, K, g, (double)rho, m, n);
    return 0;
}

int orc_gemm_sampled(const uint16_t *X, const uint8_t *packed, const void *scales, int sdt, int fmt,
                     int M, int N, int K, int g, float rho, int count, const int32_t *ms,
                     const int32_t *ns, double *out)
{
    int rc = check_args(N, K, g);
    if (rc) return rc;
    for (int i = 0; i < count; ++i)
        if (ms[i] < 0 || ms[i] >= M || ns[i] < 0 || ns[i] >= N) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int i = 0; i < count; ++i)
        out[i] = gemm_one(X, packed, scales, sdt, fmt, K, g, (double)rho, ms[i], ns[i]);
    return 0;
}

/* ---------------------------------------------------- granularity (R11) */

int orc_block_count(int N, int K, int g, int gran, int heads)
{
    if (gran == ORC_GRAN_GROUP) return g > 0 ? N * (K / g) : 0;
    if (gran == ORC_GRAN_CHANNEL) return N;
    if (gran == ORC_GRAN_HEAD) return heads;
    return 0;
}

/* Rows [r0, r1) x columns [k0, k1) of block b. */
static void block_extent(int b, int N, int K, int g, int gran, int heads, int *r0, int *r1, int *k0,
                         int *k1)
{
    if (gran == ORC_GRAN_GROUP) {
        int G = K / g;
        *r0 = b / G;
        *r1 = *r0 + 1;
        *k0 = (b % G) * g;
        *k1 = *k0 + g;
    } else if (gran == ORC_GRAN_CHANNEL) {
        *r0 = b;
        *r1 = b + 1;
        *k0 = 0;
        *k1 = K;
    } else {
        int R = N / heads;
        *r0 = b * R;
        *r1 = *r0 + R;
        *k0 = 0;
        *k1 = K;
    }
}

/* W'[r,k] = W[r,k] * 2^shift[k] (reading R6). */
static float folded(const float *W, int K, const int8_t *shift, int r, int k)
{
    float w = W[(size_t)r * K + k];
    return shift ? w * pow2f(shift[k]) : w;
}

/* One block with bias index j: its scale, and its SSE (elements in
 * row-major order); codes written when packed != NULL. */
static int block_pass(const float *W, int K, const int8_t *shift, int r0, int r1, int k0, int k1,
                      float A, int fmt, int j, int sdt, uint8_t *packed, float *s_out, uint32_t *raw,
                      double *sse_out)
{
    double mags[8], qmax_d;
    orc_format_table(fmt, mags, &qmax_d);
    float s;
    if (group_scale(A, orc_bias_factor(j), (float)qmax_d, sdt, &s, raw) != 0) return ORC_ERR_SCALE;
    double sse = 0.0;
    for (int r = r0; r < r1; ++r)
        for (int k = k0; k < k1; ++k) {
            float w = folded(W, K, shift, r, k);
            int idx = 0;
            if (s != 0.0f) {
                float q = w / s;
                idx = orc_nearest_index(fabs((double)q), mags);
            }
            int sign = signbit(w) ? 1 : 0;
            double v = sign ? -mags[idx] : mags[idx];
            double diff = (double)w - v * (double)s;
            sse += diff * diff;
            if (packed) {
                uint8_t *byte = &packed[(size_t)r * (K / 2) + (k >> 1)];
                int code = (sign << 3) | idx;
                if ((k & 1) == 0) *byte = (uint8_t)((*byte & 0xf0u) | code);
                else *byte = (uint8_t)((*byte & 0x0fu) | (code << 4));
            }
        }
    *s_out = s;
    *sse_out = sse;
    return 0;
}

int orc_quantize_blocks(const float *W, int N, int K, int g, int gran, int heads, int fmt, int j,
                        const int8_t *jforce, const int8_t *shift, int sdt, uint8_t *packed,
                        void *scales, int8_t *jmap, double *sse_out)
{
    int rc = check_args(N, K, g);
    if (rc) return rc;
    if (fmt < 0 || fmt > 2 || j < -1 || j > 7) return ORC_ERR_ARG;
    if (gran < ORC_GRAN_GROUP || gran > ORC_GRAN_HEAD) return ORC_ERR_ARG;
    if (gran == ORC_GRAN_HEAD && (heads <= 0 || N % heads != 0)) return ORC_ERR_ARG;
    int nb = orc_block_count(N, K, g, gran, heads);
    int G = K / g;
    double *bsse = (double *)calloc((size_t)(nb > 0 ? nb : 1), sizeof(double));
    if (!bsse) return ORC_ERR_ALLOC;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < nb; ++b) {
        int r0, r1, k0, k1;
        block_extent(b, N, K, g, gran, heads, &r0, &r1, &k0, &k1);
        /* the block's absmax of W' */
        float A = 0.0f;
        int e = 0;
        for (int r = r0; r < r1 && !e; ++r)
            for (int k = k0; k < k1; ++k) {
                float w = folded(W, K, shift, r, k);
                if (!isfinite(w)) { e = ORC_ERR_NONFINITE; break; }
                if (fabsf(w) > A) A = fabsf(w);
            }
        int jb = j;
        float s;
        uint32_t raw;
        double sse;
        if (!e && jforce) jb = jforce[b];
        else if (!e && j < 0) {
            /* per-block search: first strict minimum, j ascending */
            double best = INFINITY;
            jb = 0;
            for (int jj = 0; jj < 8 && !e; ++jj) {
                e = block_pass(W, K, shift, r0, r1, k0, k1, A, fmt, jj, sdt, NULL, &s, &raw, &sse);
                if (!e && sse < best) { best = sse; jb = jj; }
            }
        }
        if (!e && (jb < 0 || jb > 7)) e = ORC_ERR_ARG;
        if (!e) e = block_pass(W, K, shift, r0, r1, k0, k1, A, fmt, jb, sdt, packed, &s, &raw, &sse);
        if (e) {
#pragma omp atomic write
            err = e;
            continue;
        }
        bsse[b] = sse;
        if (jmap) jmap[b] = (int8_t)jb;
        if (scales)
            for (int r = r0; r < r1; ++r)
                for (int gi = k0 / g; gi < k1 / g; ++gi) {
                    if (sdt == ORC_SCALE_F16) ((uint16_t *)scales)[(size_t)r * G + gi] = (uint16_t)raw;
                    else ((uint32_t *)scales)[(size_t)r * G + gi] = raw;
                }
    }
    double tot = 0.0;
    for (int b = 0; b < nb; ++b) tot += bsse[b];
    free(bsse);
    if (err) return err;
    if (sse_out) *sse_out = tot;
    return 0;
}

/* ------------------------------------------------- 4-bit activations (R10) */

int orc_act_quantize(const uint16_t *X, int M, int K, const int8_t *shift, float rho, int fmt, int j,
                     uint8_t *packed, float *s_out)
{
    if (M < 0 || K < 0 || (K % 2) != 0 || fmt < 0 || fmt > 2 || j < 0 || j > 7) return ORC_ERR_ARG;
    if (!(rho > 0.0f) || !isfinite(rho)) return ORC_ERR_ARG;
    double mags[8], qmax_d;
    orc_format_table(fmt, mags, &qmax_d);
    float s;
    uint32_t raw;
    if (group_scale(rho, orc_bias_factor(j), (float)qmax_d, ORC_SCALE_F32, &s, &raw) != 0) return ORC_ERR_SCALE;
    for (size_t i = 0; i < (size_t)M * K; ++i)
        if (!isfinite(orc_bf16_to_f32(X[i]))) return ORC_ERR_NONFINITE;
    for (int m = 0; m < M; ++m)
        for (int k = 0; k < K; ++k) {
            float x = orc_bf16_to_f32(X[(size_t)m * K + k]);
            float xs = shift ? x * pow2f(-shift[k]) : x; /* exact unless it overflows */
            int idx = 0;
            if (s != 0.0f) {
                float q = xs / s; /* fl32 */
                idx = orc_nearest_index(fabs((double)q), mags);
            }
            int code = ((signbit(xs) ? 1 : 0) << 3) | idx;
            uint8_t *byte = &packed[(size_t)m * (K / 2) + (k >> 1)];
            if ((k & 1) == 0) *byte = (uint8_t)((*byte & 0xf0u) | code);
            else *byte = (uint8_t)((*byte & 0x0fu) | (code << 4));
        }
    *s_out = s;
    return 0;
}

/* Y[m,n] = s_a * sum_k v_a(a[m,k]) * v(w[n,k]) * s[n, k/g], fp64, k
 * increasing: both scale factors outside the low-bit product. */
static double w4a4_one(const uint8_t *apacked, int afmt, double s_a, const uint8_t *packed,
                       const void *scales, int sdt, int fmt, int K, int g, int m, int n)
{
    int G = K / g;
    double acc = 0.0;
    const uint8_t *ar = apacked + (size_t)m * (K / 2);
    const uint8_t *pr = packed + (size_t)n * (K / 2);
    for (int k = 0; k < K; ++k) {
        int ac = (k & 1) ? (ar[k >> 1] >> 4) : (ar[k >> 1] & 15);
        int wc = (k & 1) ? (pr[k >> 1] >> 4) : (pr[k >> 1] & 15);
        double w = code_times_scale(fmt, wc, (double)load_scale(scales, sdt, (size_t)n * G + k / g));
        acc += orc_code_value(afmt, ac) * w;
    }
    return s_a * acc;
}

int orc_gemm_w4a4(const uint8_t *apacked, int afmt, float s_a, const uint8_t *packed,
                  const void *scales, int sdt, int fmt, int M, int N, int K, int g, double *Y)
{
    if (M < 0 || afmt < 0 || afmt > 2) return ORC_ERR_ARG;
    int rc = check_args(N, K, g);
    if (rc) return rc;
#pragma omp parallel for collapse(2) schedule(static)
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n)
            Y[(size_t)m * N + n] = w4a4_one(apacked, afmt, (double)s_a, packed, scales, sdt, fmt, K, g, m, n);
    return 0;
}

int orc_gemm_w4a4_sampled(const uint8_t *apacked, int afmt, float s_a, const uint8_t *packed,
                          const void *scales, int sdt, int fmt, int M, int N, int K, int g,
                          int count, const int32_t *ms, const int32_t *ns, double *out)
{
    if (afmt < 0 || afmt > 2) return ORC_ERR_ARG;
    int rc = check_args(N, K, g);
    if (rc) return rc;
    for (int i = 0; i < count; ++i)
        if (ms[i] < 0 || ms[i] >= M || ns[i] < 0 || ns[i] >= N) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int i = 0; i < count; ++i)
        out[i] = w4a4_one(apacked, afmt, (double)s_a, packed, scales, sdt, fmt, K, g, ms[i], ns[i]);
    return 0;
}

/* ------------------------------------------------------------ pre-shift */

/* Reading R6, calibration.  e = ceil(log2(c / rho)) computed exactly from
 * the binary exponents: c = f1 * 2^q1, rho = f2 * 2^q2 with f in [0.5, 1),
 * so c/rho = (f1/f2) * 2^(q1-q2) and f1/f2 in (0.5, 2). */
int orc_preshift_calibrate(const uint16_t *X, int M, int K, int8_t *shift, float *rho_out)
{
    if (M < 0 || K < 0) return ORC_ERR_ARG;
    float *c = (float *)calloc((size_t)(K > 0 ? K : 1), sizeof(float));
    if (!c) return ORC_ERR_ALLOC;
    for (int m = 0; m < M; ++m)
        for (int k = 0; k < K; ++k) {
            float x = orc_bf16_to_f32(X[(size_t)m * K + k]);
            if (!isfinite(x)) { free(c); return ORC_ERR_NONFINITE; }
            float a = fabsf(x);
            if (a > c[k]) c[k] = a;
        }
    float rho = 0.0f;
    for (int k = 0; k < K; ++k)
        if (c[k] > rho) rho = c[k];
    if (rho == 0.0f) rho = 1.0f;
    int q2;
    float f2 = frexpf(rho, &q2);
    for (int k = 0; k < K; ++k) {
        int e = 0;
        if (c[k] > 0.0f) {
            int q1;
            float f1 = frexpf(c[k], &q1);
            e = q1 - q2 + (f1 > f2 ? 1 : 0);
            if (e < -126) e = -126;
            if (e > 0) e = 0;
        }
        shift[k] = (int8_t)e;
    }
    free(c);
    *rho_out = rho;
    return 0;
}

int orc_preshift_apply(const uint16_t *X, int M, int K, const int8_t *shift, float rho, uint16_t *Xt)
{
    if (M < 0 || K < 0) return ORC_ERR_ARG;
    for (int m = 0; m < M; ++m)
        for (int k = 0; k < K; ++k) {
            float x = orc_bf16_to_f32(X[(size_t)m * K + k]);
            float y = x * pow2f(-shift[k]); /* exact power-of-two scaling */
            float z = y / rho;              /* fl32 */
            Xt[(size_t)m * K + k] = orc_f32_to_bf16(z);
        }
    return 0;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
