/*
 * OPQ oracle: plain, slow, fp64 CPU restatement of Optimal Power Quantization.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may call this file:
 * only the tests, the package's smoke check and the benchmark's CPU-baseline
 * leg load it. It shares no code, table or helper with the CUDA library.
 *
 * Source: "OPQ INT4 Z-Image" model card (huggingpeers mirror), section
 * "OPQ principle" (normalise u = |w| / max|w|, power v = u^alpha, quantize
 * q = round(15 v) to 16 levels, inverse w' = sign(w) (q/15)^(1/alpha) max|w|),
 * section "Technical details / storage format" (4-bit magnitudes packed 8 per
 * uint32, 1-bit signs packed 32 per uint32, one scale) and "inference
 * decoding" (w = sign * (q/15)^(1/alpha) * max).
 *
 * Readings where the page is silent or is overridden by the task contract:
 *   - max|w| is taken per output row (row n of W[N,K]) and stored as fp32
 *     (the per-row format); the page's own per-group float16 max is the
 *     group-wise variant further down, with its readings there.
 *   - round() is round-half-to-even on the exact real value, here evaluated
 *     with nearbyint() under the default rounding mode.
 *   - for alpha == 1 the power is the identity and v*15 is evaluated as
 *     (15|w|)/max: 15|w| is exact in fp64, so the single rounding of the
 *     division can never move an exact .5 tie (ties are common at alpha = 1).
 *   - sign bit = 1 iff w < 0 (so -0.0 stores sign 0); a row whose max is 0
 *     quantizes to all-zero codes.
 *   - bit order: element 8j+i of a row is nibble i (bits 4i..4i+3) of code
 *     word j; element 32j+i is bit i of sign word j.
 *   - near-tie flag: |v15 - (floor(v15) + 1/2)| <= 1e-6.
 *
 * Build: plain C99, -O2, no fast-math (IEEE semantics are relied on).
 */
#define _DEFAULT_SOURCE
#include <fenv.h>
#include <math.h>
#include <stdlib.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OPQ_LEVELS 15

/* bf16 bit pattern -> exact double */
static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* exact double -> bf16 bit pattern, round to nearest even, computed from the
 * definition: keep 8 significant bits at the value's binade, with the binade
 * floored at the bf16 subnormal quantum 2^-133 and overflow to infinity. */
static uint16_t double_to_bf16_rne(double x)
{
    if (isnan(x))
        return 0x7FC0;
    int neg = signbit(x) ? 1 : 0;
    double a = fabs(x);
    uint16_t out;
    if (a == 0.0) {
        out = 0;
    } else if (isinf(a)) {
        out = 0x7F80;
    } else {
        int e;
        (void)frexp(a, &e);          /* a = m * 2^e, m in [0.5, 1) */
        int qexp = e - 8;            /* quantum of an 8-significant-bit value */
        if (qexp < -133)
            qexp = -133;
        double r = nearbyint(ldexp(a, -qexp));   /* integer number of quanta, RNE */
        double v = ldexp(r, qexp);
        /* largest finite bf16 is (2 - 2^-7) * 2^127 */
        if (v > ldexp(255.0, 120)) {
            out = 0x7F80;
        } else {
            float f = (float)v;                  /* exact: v has <= 8 significant bits */
            uint32_t u;
            memcpy(&u, &f, sizeof u);
            out = (uint16_t)(u >> 16);
        }
    }
    return (uint16_t)(out | (neg ? 0x8000 : 0));
}

int oracle_rounding_mode_ok(void) { return fegetround() == FE_TONEAREST; }

/* threads the OpenMP loops use (1 when built without OpenMP); reported beside timings */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

uint16_t oracle_double_to_bf16(double x) { return double_to_bf16_rne(x); }

/* ------------------------------------------------------------------------ */
/* quantize: W bf16 [N, ldw] (first K columns used) -> codes, signs, scales   */
/* near_tie (optional, may be NULL): one byte per element, 1 = |v15 - (floor + .5)| <= 1e-6 */
/* v15_out (optional): the oracle's 15 * u^alpha per element                  */
/* ------------------------------------------------------------------------ */
/* max |w| over row[k0 .. k1) */
static double max_abs(const uint16_t *row, int64_t k0, int64_t k1)
{
    double mx = 0.0;
    for (int64_t k = k0; k < k1; ++k) {
        double a = fabs(bf16_value(row[k]));
        if (a > mx)
            mx = a;
    }
    return mx;
}

/* steps 2-4 for element k of row n against the max mx: code and sign into the packed planes
 * (cw code words and sw sign words per row, both zeroed beforehand), the near-tie flag and
 * 15 u^alpha */
static void quantize_element(double wk, double mx, double alpha, int bits, int64_t n, int64_t k, int64_t K,
                             int64_t cw, int64_t sw, uint32_t *codes, uint32_t *signs,
                             uint8_t *near_tie, double *v15_out)
{
    const double levels = (double)((1 << bits) - 1);   /* 15 for the card's 4 bits */
    double a = fabs(wk);
    double v15;
    if (mx == 0.0)
        v15 = 0.0;
    else if (alpha == 1.0)
        v15 = (levels * a) / mx;                 /* u^1 = u */
    else
        v15 = levels * pow(a / mx, alpha);       /* L * u^alpha */
    double qd = nearbyint(v15);                  /* ties to even */
    if (qd < 0.0) qd = 0.0;
    if (qd > levels) qd = levels;
    uint32_t q = (uint32_t)qd;
    uint32_t s = (wk < 0.0) ? 1u : 0u;
    /* the codes of a row as one little-endian bit stream: element k at bits k*bits .. of the
     * row's words (for 4 bits: nibble k % 8 of word k / 8) */
    const int64_t bit = k * bits;
    codes[n * cw + bit / 32] |= q << (bit % 32);
    if (bit % 32 + bits > 32)
        codes[n * cw + bit / 32 + 1] |= q >> (32 - bit % 32);
    signs[n * sw + k / 32] |= s << (k % 32);
    if (near_tie)
        near_tie[n * K + k] = (fabs(v15 - (floor(v15) + 0.5)) <= 1e-6) ? 1 : 0;
    if (v15_out)
        v15_out[n * K + k] = v15;
}

void oracle_quantize(const uint16_t *w, int64_t N, int64_t K, int64_t ldw, double alpha,
                     uint32_t *codes, uint32_t *signs, float *scales,
                     uint8_t *near_tie, double *v15_out)
{
    const int64_t cw = K / 8, sw = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const uint16_t *row = w + n * ldw;
        /* step 1: max |w| over the row */
        double mx = max_abs(row, 0, K);
        scales[n] = (float)mx;  /* exact: mx is a bf16 value */
        for (int64_t j = 0; j < cw; ++j)
            codes[n * cw + j] = 0;
        for (int64_t j = 0; j < sw; ++j)
            signs[n * sw + j] = 0;
        for (int64_t k = 0; k < K; ++k)
            quantize_element(bf16_value(row[k]), mx, alpha, 4, n, k, K, cw, sw, codes, signs, near_tie, v15_out);
    }
}

/* the same per-row quantization with `bits` bits per magnitude (3, 4, 5 or 6; the card's
 * "OPQ configuration" lists them, its storage section describes 4): 2^bits - 1 levels, the
 * codes of a row packed as one little-endian bit stream of K * bits / 32 words */
void oracle_quantize_bits(const uint16_t *w, int64_t N, int64_t K, int64_t ldw, int bits, double alpha,
                          uint32_t *codes, uint32_t *signs, float *scales, uint8_t *near_tie, double *vl_out)
{
    const int64_t cw = K * bits / 32, sw = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const uint16_t *row = w + n * ldw;
        double mx = max_abs(row, 0, K);
        scales[n] = (float)mx;
        for (int64_t j = 0; j < cw; ++j)
            codes[n * cw + j] = 0;
        for (int64_t j = 0; j < sw; ++j)
            signs[n * sw + j] = 0;
        for (int64_t k = 0; k < K; ++k)
            quantize_element(bf16_value(row[k]), mx, alpha, bits, n, k, K, cw, sw, codes, signs, near_tie, vl_out);
    }
}

/* magnitude code and sign of element (n, k) from the packed planes */
static uint32_t code_at(const uint32_t *codes, int64_t K, int64_t n, int64_t k)
{
    return (codes[n * (K / 8) + k / 8] >> (4 * (k % 8))) & 0xFu;
}

static uint32_t sign_at(const uint32_t *signs, int64_t K, int64_t n, int64_t k)
{
    return (signs[n * (K / 32) + k / 32] >> (k % 32)) & 1u;
}

/* w' = sign * (q/15)^(1/alpha) * max, unrounded fp64 */
static double dequant_value_levels(uint32_t q, uint32_t s, double alpha, double mx, double levels)
{
    double mag = pow((double)q / levels, 1.0 / alpha) * mx;
    return s ? -mag : mag;
}

static double dequant_value(uint32_t q, uint32_t s, double alpha, double mx)
{
    return dequant_value_levels(q, s, alpha, mx, 15.0);
}

/* code of element (n, k) of a `bits`-bit stream plane */
static uint32_t code_at_bits(const uint32_t *codes, int64_t K, int bits, int64_t n, int64_t k)
{
    const int64_t cw = K * bits / 32, bit = k * bits;
    uint64_t two = codes[n * cw + bit / 32];
    if (bit % 32 + bits > 32)
        two |= (uint64_t)codes[n * cw + bit / 32 + 1] << 32;
    return (uint32_t)(two >> (bit % 32)) & ((1u << bits) - 1u);
}

/* dequantize to fp64 (unrounded) */
void oracle_dequantize_f64(const uint32_t *codes, const uint32_t *signs, const float *scales,
                           int64_t N, int64_t K, double alpha, double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            out[n * K + k] = dequant_value(code_at(codes, K, n, k), sign_at(signs, K, n, k),
                                           alpha, (double)scales[n]);
}

/* dequantize, rounded once to bf16 (round to nearest even) */
void oracle_dequantize_bf16(const uint32_t *codes, const uint32_t *signs, const float *scales,
                            int64_t N, int64_t K, double alpha, uint16_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            out[n * K + k] = double_to_bf16_rne(dequant_value(code_at(codes, K, n, k),
                                                              sign_at(signs, K, n, k),
                                                              alpha, (double)scales[n]));
}

void oracle_dequantize_bits_f64(const uint32_t *codes, const uint32_t *signs, const float *scales, int64_t N,
                                int64_t K, int bits, double alpha, double *out)
{
    const double levels = (double)((1 << bits) - 1);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            out[n * K + k] = dequant_value_levels(code_at_bits(codes, K, bits, n, k), sign_at(signs, K, n, k), alpha,
                                                  (double)scales[n], levels);
}

void oracle_dequantize_bits_bf16(const uint32_t *codes, const uint32_t *signs, const float *scales, int64_t N,
                                 int64_t K, int bits, double alpha, uint16_t *out)
{
    const double levels = (double)((1 << bits) - 1);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            out[n * K + k] = double_to_bf16_rne(dequant_value_levels(code_at_bits(codes, K, bits, n, k),
                                                                     sign_at(signs, K, n, k), alpha,
                                                                     (double)scales[n], levels));
}

/* ------------------------------------------------------------------------ */
/* linear: y[m, n] = sum_k x[m, k] * w'[n, k] (fp64, unrounded w'),          */
/* bound[m, n] = sum_k |x[m, k]| * |w'[n, k]|                                */
/* ------------------------------------------------------------------------ */
/* where w'[n, k] comes from: one scale per row, or one float16 max per group */
typedef struct {
    const uint32_t *codes, *signs;
    const float *scales;     /* per row, or NULL */
    const uint16_t *gmax;    /* per group (float16 bits), or NULL */
    int64_t K, GS;
    double alpha;
} planes_t;

static double group_max_at(const uint16_t *gmax, int64_t K, int64_t GS, int64_t n, int64_t k);

static double wprime(const planes_t *p, int64_t n, int64_t k)
{
    double mx = p->scales ? (double)p->scales[n] : group_max_at(p->gmax, p->K, p->GS, n, k);
    return dequant_value(code_at(p->codes, p->K, n, k), sign_at(p->signs, p->K, n, k), p->alpha, mx);
}

static void linear_rows(const uint16_t *x, int64_t M, int64_t K, const planes_t *p, int64_t N,
                        double *y, double *bound)
{
#pragma omp parallel
    {
        /* w'[n, :] is evaluated once per row and reused for every m */
        double *wrow = (double *)malloc((size_t)K * sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t n = 0; n < N; ++n) {
            for (int64_t k = 0; k < K; ++k)
                wrow[k] = wprime(p, n, k);
            for (int64_t m = 0; m < M; ++m) {
                double acc = 0.0, b = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    double xv = bf16_value(x[m * K + k]);
                    acc += xv * wrow[k];
                    b += fabs(xv) * fabs(wrow[k]);
                }
                y[m * N + n] = acc;
                if (bound)
                    bound[m * N + n] = b;
            }
        }
        free(wrow);
    }
}

/* the same sum for an explicit list of (m, n) output positions */
static void linear_list(const uint16_t *x, int64_t K, const planes_t *p, int64_t count,
                        const int64_t *ms, const int64_t *ns, double *y, double *bound)
{
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = ms[i], n = ns[i];
        double acc = 0.0, b = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double wv = wprime(p, n, k);
            double xv = bf16_value(x[m * K + k]);
            acc += xv * wv;
            b += fabs(xv) * fabs(wv);
        }
        y[i] = acc;
        if (bound)
            bound[i] = b;
    }
}

void oracle_linear(const uint16_t *x, int64_t M, int64_t K,
                   const uint32_t *codes, const uint32_t *signs, const float *scales,
                   int64_t N, double alpha, double *y, double *bound)
{
    planes_t p = {codes, signs, scales, NULL, K, K, alpha};
    linear_rows(x, M, K, &p, N, y, bound);
}

void oracle_linear_pairs(const uint16_t *x, int64_t M, int64_t K,
                         const uint32_t *codes, const uint32_t *signs, const float *scales,
                         int64_t N, double alpha, int64_t count, const int64_t *ms,
                         const int64_t *ns, double *y, double *bound)
{
    (void)M;
    (void)N;
    planes_t p = {codes, signs, scales, NULL, K, K, alpha};
    linear_list(x, K, &p, count, ms, ns, y, bound);
}

/* ------------------------------------------------------------------------ */
/* Group-wise variant: the model card's own storage format ("Technical        */
/* details / storage format": one float16 group max shared by every 128       */
/* weights; its "OPQ configuration" lists group sizes 32, 64, 128 and 256).   */
/* A group is GS consecutive weights of one row (K % GS == 0). Readings:      */
/*   - the group max is max|w| over the group, stored as IEEE binary16,       */
/*     rounded to nearest even; a max beyond the largest finite float16       */
/*     (65504) saturates to it instead of becoming infinity;                  */
/*   - quantization and decoding both use the stored float16 max, so that     */
/*     they agree (for a max in float16's normal range the conversion is      */
/*     exact: a bf16 value has 8 significant bits, float16 has 11);           */
/*   - |w| above a max that rounded down (float16's subnormal range) gives    */
/*     u > 1 and a code clamped to 15; a group whose stored max is 0          */
/*     quantizes to all-zero codes; the rest as for the per-row format.       */
/* ------------------------------------------------------------------------ */

/* float16 bit pattern -> exact double, from the binary16 definition */
static double fp16_value(uint16_t bits)
{
    int s = (bits >> 15) & 1, e = (bits >> 10) & 0x1F, m = bits & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                    /* subnormal: m * 2^-24 */
    else if (e == 0x1F)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);         /* (1 + m/1024) * 2^(e-15) */
    return s ? -v : v;
}

/* non-negative double -> float16 bit pattern: 11 significant bits at the value's binade
 * (binade floored at the subnormal quantum 2^-24), round to nearest even, saturating at
 * 65504 */
static uint16_t nonneg_to_fp16_rne_sat(double a)
{
    if (!(a > 0.0))
        return 0;
    int e;
    (void)frexp(a, &e);                 /* a = m * 2^e, m in [0.5, 1) */
    int qexp = e - 11;
    if (qexp < -24)
        qexp = -24;
    double v = ldexp(nearbyint(ldexp(a, -qexp)), qexp);
    if (v > 65504.0)
        v = 65504.0;
    if (v < ldexp(1.0, -14))            /* subnormal (or zero): v / 2^-24 quanta */
        return (uint16_t)ldexp(v, 24);
    (void)frexp(v, &e);                 /* v = m * 2^e, m in [0.5, 1) */
    int field = e - 1 + 15;
    uint16_t mant = (uint16_t)(ldexp(v, 11 - e) - 1024.0);   /* exact: v has <= 11 bits */
    return (uint16_t)((field << 10) | mant);
}

double oracle_fp16_value(uint16_t bits) { return fp16_value(bits); }
uint16_t oracle_fp16_from_nonneg(double a) { return nonneg_to_fp16_rne_sat(a); }

/* gmax: uint16 float16 bits [N, K / GS] */
void oracle_quantize_grouped(const uint16_t *w, int64_t N, int64_t K, int64_t ldw, int64_t GS,
                             double alpha, uint32_t *codes, uint32_t *signs, uint16_t *gmax,
                             uint8_t *near_tie, double *v15_out)
{
    const int64_t cw = K / 8, sw = K / 32, ng = K / GS;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const uint16_t *row = w + n * ldw;
        for (int64_t j = 0; j < cw; ++j)
            codes[n * cw + j] = 0;
        for (int64_t j = 0; j < sw; ++j)
            signs[n * sw + j] = 0;
        for (int64_t g = 0; g < ng; ++g) {
            /* step 1: max |w| over the group, kept as float16 */
            uint16_t gb = nonneg_to_fp16_rne_sat(max_abs(row, g * GS, (g + 1) * GS));
            gmax[n * ng + g] = gb;
            /* steps 2-4 per weight, against the stored max */
            for (int64_t k = g * GS; k < (g + 1) * GS; ++k)
                quantize_element(bf16_value(row[k]), fp16_value(gb), alpha, 4, n, k, K, cw, sw, codes, signs,
                                 near_tie, v15_out);
        }
    }
}

static double group_max_at(const uint16_t *gmax, int64_t K, int64_t GS, int64_t n, int64_t k)
{
    return fp16_value(gmax[n * (K / GS) + k / GS]);
}

void oracle_dequantize_grouped_f64(const uint32_t *codes, const uint32_t *signs, const uint16_t *gmax,
                                   int64_t N, int64_t K, int64_t GS, double alpha, double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            out[n * K + k] = dequant_value(code_at(codes, K, n, k), sign_at(signs, K, n, k), alpha,
                                           group_max_at(gmax, K, GS, n, k));
}

void oracle_dequantize_grouped_bf16(const uint32_t *codes, const uint32_t *signs, const uint16_t *gmax,
                                    int64_t N, int64_t K, int64_t GS, double alpha, uint16_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            out[n * K + k] = double_to_bf16_rne(dequant_value(code_at(codes, K, n, k), sign_at(signs, K, n, k),
                                                              alpha, group_max_at(gmax, K, GS, n, k)));
}

void oracle_linear_grouped(const uint16_t *x, int64_t M, int64_t K, const uint32_t *codes,
                           const uint32_t *signs, const uint16_t *gmax, int64_t N, int64_t GS,
                           double alpha, double *y, double *bound)
{
    planes_t p = {codes, signs, NULL, gmax, K, GS, alpha};
    linear_rows(x, M, K, &p, N, y, bound);
}

void oracle_linear_grouped_pairs(const uint16_t *x, int64_t M, int64_t K, const uint32_t *codes,
                                 const uint32_t *signs, const uint16_t *gmax, int64_t N, int64_t GS,
                                 double alpha, int64_t count, const int64_t *ms, const int64_t *ns,
                                 double *y, double *bound)
{
    (void)M;
    (void)N;
    planes_t p = {codes, signs, NULL, gmax, K, GS, alpha};
    linear_list(x, K, &p, count, ms, ns, y, bound);
}

/* ------------------------------------------------------------------------ */
/* fused epilogue of the linear: the OPQLinear layers replace nn.Linear       */
/* modules (y = x W^T + b); in the feed-forward blocks an activation follows. */
/* In place on y[M, N]: y = act(y + bias[n]), fp64. act 0 none, 1 SiLU        */
/* v / (1 + e^-v), 2 GELU's tanh form 0.5 v (1 + tanh(sqrt(2/pi) (v +        */
/* 0.044715 v^3))). bias: bf16 bits [N] or NULL.                              */
/* ------------------------------------------------------------------------ */
void oracle_apply_epilogue(double *y, int64_t M, int64_t N, const uint16_t *bias, int act)
{
    const double c = sqrt(2.0 / M_PI);
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double v = y[m * N + n] + (bias ? bf16_value(bias[n]) : 0.0);
            if (act == 1)
                v = v / (1.0 + exp(-v));
            else if (act == 2)
                v = 0.5 * v * (1.0 + tanh(c * (v + 0.044715 * v * v * v)));
            y[m * N + n] = v;
        }
}

/* ------------------------------------------------------------------------ */
/* quality context: SNR in dB of a reconstruction against the bf16 weights   */
/* ------------------------------------------------------------------------ */
double oracle_snr_db(const uint16_t *w, const double *w_rec, int64_t count)
{
    double sig = 0.0, err = 0.0;
    for (int64_t i = 0; i < count; ++i) {
        double a = bf16_value(w[i]);
        double d = a - w_rec[i];
        sig += a * a;
        err += d * d;
    }
    if (err == 0.0)
        return INFINITY;
    return 10.0 * log10(sig / err);
}

/* symmetric per-row uniform INT4 baseline: q = clip(RNE(w / (max/7)), -7, 7),
 * reconstruction q * max / 7 (the page's "uniform quantization q = round(w/delta)"
 * with delta = max/7, the reading used for the SNR comparison) */
void oracle_uniform_int4(const uint16_t *w, int64_t N, int64_t K, double *w_rec)
{
    for (int64_t n = 0; n < N; ++n) {
        double mx = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double a = fabs(bf16_value(w[n * K + k]));
            if (a > mx)
                mx = a;
        }
        for (int64_t k = 0; k < K; ++k) {
            double v = bf16_value(w[n * K + k]);
            double q = (mx == 0.0) ? 0.0 : nearbyint(v / (mx / 7.0));
            if (q > 7.0) q = 7.0;
            if (q < -7.0) q = -7.0;
            w_rec[n * K + k] = q * mx / 7.0;
        }
    }
}
