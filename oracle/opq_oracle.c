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
 *   - max|w| is taken per output row (row n of W[N,K]) and stored as fp32;
 *     the page uses a per-128 group max in fp16.
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
void oracle_quantize(const uint16_t *w, int64_t N, int64_t K, int64_t ldw, double alpha,
                     uint32_t *codes, uint32_t *signs, float *scales,
                     uint8_t *near_tie, double *v15_out)
{
    const int64_t cw = K / 8, sw = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const uint16_t *row = w + n * ldw;
        /* step 1: max |w| over the row */
        double mx = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double a = fabs(bf16_value(row[k]));
            if (a > mx)
                mx = a;
        }
        scales[n] = (float)mx;  /* exact: mx is a bf16 value */
        for (int64_t j = 0; j < cw; ++j)
            codes[n * cw + j] = 0;
        for (int64_t j = 0; j < sw; ++j)
            signs[n * sw + j] = 0;
        for (int64_t k = 0; k < K; ++k) {
            double wk = bf16_value(row[k]);
            double a = fabs(wk);
            double v15;
            if (mx == 0.0)
                v15 = 0.0;
            else if (alpha == 1.0)
                v15 = (15.0 * a) / mx;                 /* u^1 = u */
            else
                v15 = 15.0 * pow(a / mx, alpha);       /* 15 * u^alpha */
            double qd = nearbyint(v15);                /* ties to even */
            if (qd < 0.0) qd = 0.0;
            if (qd > OPQ_LEVELS) qd = OPQ_LEVELS;
            uint32_t q = (uint32_t)qd;
            uint32_t s = (wk < 0.0) ? 1u : 0u;
            codes[n * cw + k / 8] |= q << (4 * (k % 8));
            signs[n * sw + k / 32] |= s << (k % 32);
            if (near_tie)
                near_tie[n * K + k] = (fabs(v15 - (floor(v15) + 0.5)) <= 1e-6) ? 1 : 0;
            if (v15_out)
                v15_out[n * K + k] = v15;
        }
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
static double dequant_value(uint32_t q, uint32_t s, double alpha, double mx)
{
    double mag = pow((double)q / 15.0, 1.0 / alpha) * mx;
    return s ? -mag : mag;
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

/* ------------------------------------------------------------------------ */
/* linear: y[m, n] = sum_k x[m, k] * w'[n, k] (fp64, unrounded w'),          */
/* bound[m, n] = sum_k |x[m, k]| * |w'[n, k]|                                */
/* ------------------------------------------------------------------------ */
void oracle_linear(const uint16_t *x, int64_t M, int64_t K,
                   const uint32_t *codes, const uint32_t *signs, const float *scales,
                   int64_t N, double alpha, double *y, double *bound)
{
#pragma omp parallel
    {
        /* w'[n, :] is evaluated once per row and reused for every m */
        double *wrow = (double *)malloc((size_t)K * sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t n = 0; n < N; ++n) {
            for (int64_t k = 0; k < K; ++k)
                wrow[k] = dequant_value(code_at(codes, K, n, k), sign_at(signs, K, n, k),
                                        alpha, (double)scales[n]);
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
void oracle_linear_pairs(const uint16_t *x, int64_t M, int64_t K,
                         const uint32_t *codes, const uint32_t *signs, const float *scales,
                         int64_t N, double alpha, int64_t count, const int64_t *ms,
                         const int64_t *ns, double *y, double *bound)
{
    (void)M;
    (void)N;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = ms[i], n = ns[i];
        double acc = 0.0, b = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double wv = dequant_value(code_at(codes, K, n, k), sign_at(signs, K, n, k),
                                      alpha, (double)scales[n]);
            double xv = bf16_value(x[m * K + k]);
            acc += xv * wv;
            b += fabs(xv) * fabs(wv);
        }
        y[i] = acc;
        if (bound)
            bound[i] = b;
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
