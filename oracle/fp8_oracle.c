/*
 * fp8_oracle.c -- plain, slow, obviously-correct CPU oracle for the FP8
 * mixed-precision training hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is loaded by the tests, by the smoke
 * check and by the benchmark's CPU-baseline leg, and by nothing else.  It
 * shares no code, header, table or helper with the CUDA library; the two only
 * ever see the same seeded input bytes.  Arithmetic is float64 throughout.
 *
 * Sources (cited by page title and section):
 *   [FP8-LM]   "FP8-LM: Training FP8 Large Language Models" (paper memo),
 *              sections 提案手法 (O1 with Eq. 3, O2) and アブレーション研究.
 *   [FP8-AMAX] "Training and inference of large language models using 8-bit
 *              floating point" (paper review), sections ABSTRACT and 제안 방법.
 *   [OFP8]     OCP 8-bit Floating Point Specification: bit layouts of E4M3
 *              and E5M2 (the pages name the formats but print no layout).
 *
 * Readings of the pages that are not printed there are marked "reading:".
 * Parity unpinned: the NaN code chosen by the encoder (no workload has NaN).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_E4M3 0
#define ORC_E5M2 1
#define ORC_F16 2

#define ORC_DT_F32 0
#define ORC_DT_BF16 1
#define ORC_DT_F16 2

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_NONFINITE 6

/* ------------------------------------------------------------------------
 * Formats.  [FP8-AMAX] 제안 방법: E4M3 ("FP8_E4") for weights and
 * activations, E5M2 ("FP8_E5") for gradients.  [FP8-LM] 提案手法 O2: FP16
 * for the second moment and for the master weights.  Bit layouts per [OFP8]
 * and IEEE 754 binary16.
 * ---------------------------------------------------------------------- */

/* Decode one 8-bit code straight from its bit fields. */
double orc_fp8_decode(int fmt, unsigned code)
{
    int ebits = (fmt == ORC_E4M3) ? 4 : 5;
    int mbits = 7 - ebits;
    int bias = (fmt == ORC_E4M3) ? 7 : 15;
    int neg = (code >> 7) & 1;
    int E = (int)((code >> mbits) & ((1u << ebits) - 1u));
    int Mt = (int)(code & ((1u << mbits) - 1u));
    double v;
    if (fmt == ORC_E4M3 && E == 15 && Mt == 7)
        return NAN; /* E4M3 has no infinities; S.1111.111 is NaN */
    if (fmt == ORC_E5M2 && E == 31)
        v = (Mt == 0) ? INFINITY : NAN;
    else if (E == 0)
        v = ldexp((double)Mt, 1 - bias - mbits); /* subnormal: 0.M x 2^(1-bias) */
    else
        v = ldexp((double)((1 << mbits) + Mt), E - bias - mbits); /* 1.M x 2^(E-bias) */
    return neg ? -v : v;
}

/* Decode an IEEE binary16 bit pattern. */
double orc_f16_decode(unsigned h)
{
    int neg = (h >> 15) & 1;
    int E = (h >> 10) & 31;
    int Mt = h & 1023;
    double v;
    if (E == 31)
        v = (Mt == 0) ? INFINITY : NAN;
    else if (E == 0)
        v = ldexp((double)Mt, -24);
    else
        v = ldexp((double)(1024 + Mt), E - 25);
    return neg ? -v : v;
}

/* bfloat16 is the top half of an IEEE binary32. */
static double bf16_decode(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double load_elem(const void *x, int dtype, size_t i)
{
    if (dtype == ORC_DT_F32)
        return (double)((const float *)x)[i];
    if (dtype == ORC_DT_BF16)
        return bf16_decode(((const uint16_t *)x)[i]);
    return orc_f16_decode(((const uint16_t *)x)[i]);
}

/* Largest finite positive code of each storage format. */
static unsigned top_code(int fmt)
{
    if (fmt == ORC_E4M3)
        return 0x7E; /* 448 */
    if (fmt == ORC_E5M2)
        return 0x7B; /* 57344 */
    return 0x7BFF;   /* 65504 */
}

double orc_fmt_max(int fmt)
{
    return fmt == ORC_F16 ? orc_f16_decode(top_code(fmt)) : orc_fp8_decode(fmt, top_code(fmt));
}

static double code_value(int fmt, unsigned c)
{
    return fmt == ORC_F16 ? orc_f16_decode(c) : orc_fp8_decode(fmt, c);
}

/*
 * Round |y| to the nearest value in the sorted table of non-negative finite
 * codes 0..top, ties to the code whose last mantissa bit is 0 (the code's
 * lowest bit is the mantissa's lowest bit).  Binary search for the bracket,
 * then compare against the exact midpoint of the bracket.
 */
static unsigned nearest_code(int fmt, double a)
{
    unsigned lo = 0, hi = top_code(fmt);
    while (hi - lo > 1) {
        unsigned mid = (lo + hi) / 2;
        if (code_value(fmt, mid) <= a)
            lo = mid;
        else
            hi = mid;
    }
    double vlo = code_value(fmt, lo), vhi = code_value(fmt, hi);
    if (a <= vlo)
        return lo;
    if (a >= vhi)
        return hi;
    double midpoint = 0.5 * (vlo + vhi); /* exact: both have few significant bits */
    if (a < midpoint)
        return lo;
    if (a > midpoint)
        return hi;
    return (lo & 1u) ? hi : lo;
}

/*
 * Encode a real number as E4M3 / E5M2: round to nearest, ties to even,
 * saturating at +-max ("scale before the cast", [FP8-AMAX] 제안 방법).
 * readings: +-inf saturates to +-max as well; NaN becomes the positive NaN
 * code 0x7F whatever its sign bit (a NaN's sign carries no meaning, and the
 * scaling multiply before the cast does not keep it) -- parity unpinned.
 */
unsigned orc_fp8_encode(int fmt, double y)
{
    if (isnan(y))
        return 0x7Fu;
    unsigned sign = signbit(y) ? 0x80u : 0u;
    double a = fabs(y);
    unsigned top = top_code(fmt);
    if (a >= code_value(fmt, top))
        return sign | top;
    return sign | nearest_code(fmt, a);
}

/* IEEE binary16 round-to-nearest-even; overflow past 65520 gives inf.
 * reading: NaN becomes the positive all-ones NaN 0x7FFF (see orc_fp8_encode). */
unsigned orc_f16_encode(double y)
{
    if (isnan(y))
        return 0x7FFFu;
    unsigned sign = signbit(y) ? 0x8000u : 0u;
    double a = fabs(y);
    if (a >= 65520.0)
        return sign | 0x7C00u;
    if (a >= 65504.0)
        return sign | 0x7BFFu;
    return sign | nearest_code(ORC_F16, a);
}

/* ------------------------------------------------------------------------
 * amax.  [FP8-AMAX] 제안 방법 / ABSTRACT: per-tensor maximum absolute value
 * of each weight, activation and gradient tensor.
 * reading: any NaN makes the result NaN; otherwise any inf makes it +inf.
 * ---------------------------------------------------------------------- */
double orc_amax(const void *x, int dtype, size_t n)
{
    double m = 0.0;
    int saw_nan = 0;
    for (size_t i = 0; i < n; i++) {
        double v = load_elem(x, dtype, i);
        if (isnan(v))
            saw_nan = 1;
        else if (fabs(v) > m)
            m = fabs(v);
    }
    return saw_nan ? NAN : m;
}

/* ------------------------------------------------------------------------
 * Scale rule.  [FP8-AMAX] 제안 방법 (compute_bias): the scaling exponent is
 * the log2 of fmt_max / amax, with a configurable margin:
 *     s = 2^(floor(log2(fmt_max / amax)) - margin).
 * floor(log2(fmt_max / amax)) is the largest integer e with
 * amax * 2^e <= fmt_max; it is computed exactly from frexp() so that no
 * rounded log2 or division decides the floor.
 * readings: amax == 0 gives s = 1; a non-finite amax is an error and gives
 * s = 1; e - margin is clamped to [-126, 126] so that s and 1/s are normal
 * binary32 numbers.
 * ---------------------------------------------------------------------- */
int orc_floor_log2_ratio(double amax, double fmt_max)
{
    int p, r;
    double a = frexp(amax, &p);   /* amax    = a * 2^p, a in [0.5, 1) */
    double f = frexp(fmt_max, &r); /* fmt_max = f * 2^r, f in [0.5, 1) */
    return (a <= f) ? (r - p) : (r - p - 1);
}

int orc_compute_scale(double amax, int fmt, int margin, double *scale)
{
    if (!isfinite(amax)) {
        *scale = 1.0;
        return ORC_ERR_NONFINITE;
    }
    if (amax == 0.0) {
        *scale = 1.0;
        return ORC_OK;
    }
    int k = orc_floor_log2_ratio(amax, orc_fmt_max(fmt)) - margin;
    if (k < -126)
        k = -126;
    if (k > 126)
        k = 126;
    *scale = ldexp(1.0, k);
    return ORC_OK;
}

/*
 * Gradient auto-scaling.  [FP8-LM] 提案手法 O1, Eq. 3: g' = mu * g before
 * the FP8 cast.  The scale is taken from amax(g') = mu * amax(g) and the cast
 * multiplies g by mu * s_g; the descale is 1 / (mu * s_g).
 */
int orc_compute_scale_mu(double amax, int fmt, int margin, double mu, double *total_scale)
{
    double s_g;
    int rc = orc_compute_scale(mu * amax, fmt, margin, &s_g);
    /* reading: the combined multiplier is itself kept a normal binary32 */
    double t = mu * s_g;
    if (t < ldexp(1.0, -126))
        t = ldexp(1.0, -126);
    if (t > ldexp(1.0, 126))
        t = ldexp(1.0, 126);
    *total_scale = t;
    return rc;
}

/* ------------------------------------------------------------------------
 * Cast.  [FP8-AMAX] 제안 방법: scale the input before casting to FP8.
 * q_i = enc(x_i * s); x_i * s is exact in float64.  fmt ORC_F16 stores a
 * scaled IEEE half (the tensor-scaled FP16 of [FP8-LM] 提案手法 O2).
 * ---------------------------------------------------------------------- */
void orc_cast(const void *x, int dtype, size_t n, int fmt, double scale, void *q)
{
    long long i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < (long long)n; i++) {
        double y = load_elem(x, dtype, (size_t)i) * scale;
        if (fmt == ORC_F16)
            ((uint16_t *)q)[i] = (uint16_t)orc_f16_encode(y);
        else
            ((uint8_t *)q)[i] = (uint8_t)orc_fp8_encode(fmt, y);
    }
}

/* ------------------------------------------------------------------------
 * Underflow / overflow counters.  [FP8-LM] アブレーション研究 compares the
 * gradient scaling variants by their underflow and overflow rates; [FP8-AMAX]
 * 실험 결과 (research question RQ3) asks which scaling keeps weights,
 * activations and gradients clear of both.  reading: an element underflows when it is a non-zero number and
 * its code is zero; it overflows when |x * s| exceeds the format's largest
 * finite value (the cast saturates it; inf included, NaN in neither).
 * counts[0] += underflows, counts[1] += overflows.
 * ---------------------------------------------------------------------- */
void orc_cast_counts(const void *x, int dtype, size_t n, int fmt, double scale, void *q,
                     unsigned long long *counts)
{
    orc_cast(x, dtype, n, fmt, scale, q);
    double fmax = orc_fmt_max(fmt);
    unsigned long long under = 0, over = 0;
    for (size_t i = 0; i < n; i++) {
        double v = load_elem(x, dtype, i);
        unsigned c = fmt == ORC_F16 ? ((const uint16_t *)q)[i] : ((const uint8_t *)q)[i];
        if (!isnan(v) && v != 0.0 && code_value(fmt, c) == 0.0)
            under++;
        if (fabs(v * scale) > fmax)
            over++;
    }
    counts[0] += under;
    counts[1] += over;
}

/*
 * Shared payload scale of the FP8 gradient all-reduce ([FP8-LM] 提案手法 O1,
 * Eq. 3).  reading: every rank casts its gradient with one scale taken from
 * the amax over all ranks' gradients before auto-scaling, times mu:
 *     S = mu * 2^(floor(log2(fmt_max / amax)) - margin),
 * so that mu < 1 leaves headroom for the sum of the ranks' payloads.  The
 * exponent rule, its clamps and amax == 0 / non-finite as in
 * orc_compute_scale; mu is a power of two and S is clamped to
 * [2^-126, 2^126].
 */
int orc_grad_scale(double amax, int fmt, int margin, double mu, double *scale)
{
    double s;
    int rc = orc_compute_scale(amax, fmt, margin, &s);
    double t = mu * s;
    if (t < ldexp(1.0, -126))
        t = ldexp(1.0, -126);
    if (t > ldexp(1.0, 126))
        t = ldexp(1.0, 126);
    *scale = t;
    return rc;
}

/*
 * Reduction of the ranks' FP8 payloads ([FP8-LM] 提案手法 O1: gradients
 * all-reduced in FP8).  in holds nranks rows of ld codes, all cast with the
 * same scale; out_i = enc(sum_r dec(in[r * ld + i])): the exact sum (every
 * FP8 value is a multiple of the format's smallest subnormal, so float64 adds
 * them without rounding), re-encoded once in the same format and scale.
 * readings: the sum starts at +0, so a zero sum is code 0x00; a NaN sum (a
 * NaN code, or +inf and -inf) gives code 0x7F.
 * counts as in orc_cast_counts, on the sums: [0] non-zero sums with a zero
 * code, [1] sums beyond fmt_max (saturated).
 */
void orc_sum_codes(const uint8_t *in, int nranks, size_t ld, size_t n, int fmt, uint8_t *out,
                   unsigned long long *counts)
{
    double fmax = orc_fmt_max(fmt);
    for (size_t i = 0; i < n; i++) {
        double sum = 0.0;
        for (int r = 0; r < nranks; r++)
            sum += orc_fp8_decode(fmt, in[(size_t)r * ld + i]);
        unsigned c = isnan(sum) ? 0x7Fu : orc_fp8_encode(fmt, sum);
        out[i] = (uint8_t)c;
        if (!isnan(sum) && sum != 0.0 && orc_fp8_decode(fmt, c) == 0.0)
            counts[0]++;
        if (fabs(sum) > fmax)
            counts[1]++;
    }
}

/*
 * Auto-scaling update of mu between steps ([FP8-LM] 提案手法 O1: mu changes
 * dynamically).  The pages give no rule; this one is the build's own, in the
 * manner of dynamic loss scaling: when more than theta * n of the n reduced
 * gradient elements overflowed, mu halves (not below mu_min) and the count
 * of clean steps restarts; otherwise the count grows, and after `interval`
 * clean steps in a row mu doubles (not above mu_max) and the count restarts.
 */
void orc_mu_update(double *mu, int *clean, unsigned long long overflows, unsigned long long n,
                   double theta, int interval, double mu_min, double mu_max)
{
    if ((double)overflows > theta * (double)n) {
        *mu = (*mu * 0.5 < mu_min) ? mu_min : *mu * 0.5;
        *clean = 0;
        return;
    }
    *clean += 1;
    if (*clean >= interval) {
        *mu = (*mu * 2.0 > mu_max) ? mu_max : *mu * 2.0;
        *clean = 0;
    }
}

/* amax over all cores: the same definition as orc_amax, split into ranges. */
double orc_amax_parallel(const void *x, int dtype, size_t n)
{
    int nt = 1;
#ifdef _OPENMP
    nt = omp_get_max_threads();
#endif
    double part[1024];
    int saw[1024];
    if (nt > 1024)
        nt = 1024;
    long long t;
#pragma omp parallel for num_threads(nt) schedule(static)
    for (t = 0; t < nt; t++) {
        size_t b = n * (size_t)t / (size_t)nt, e = n * (size_t)(t + 1) / (size_t)nt;
        double m = orc_amax((const char *)x + b * (dtype == ORC_DT_F32 ? 4 : 2), dtype, e - b);
        saw[t] = isnan(m);
        part[t] = isnan(m) ? 0.0 : m;
    }
    double m = 0.0;
    for (int i = 0; i < nt; i++) {
        if (saw[i])
            return NAN;
        if (part[i] > m)
            m = part[i];
    }
    return m;
}

/* ------------------------------------------------------------------------
 * FP8 GEMM.  [FP8-AMAX] 제안 방법: after the FP8 matrix multiplication the
 * scaling is undone.  C(i,j) = sum_k a(i,k) b(j,k) / (s_a s_b) with a, b the
 * decoded codes; a(i,k) = A[i*a_si + k*a_sk], b(j,k) = B[j*b_sj + k*b_sk].
 * Also returns sum_k |a(i,k) b(j,k)| / (s_a s_b), the scale of the error
 * bound.  Bias (optional, length N) is added in float64.
 * ---------------------------------------------------------------------- */
static double gemm_entry(const uint8_t *A, int fa, long long a_si, long long a_sk,
                         const uint8_t *B, int fb, long long b_sj, long long b_sk,
                         int K, int i, int j, double *abs_sum)
{
    double s = 0.0, sa = 0.0;
    for (int k = 0; k < K; k++) {
        double p = orc_fp8_decode(fa, A[i * a_si + k * a_sk]) * orc_fp8_decode(fb, B[j * b_sj + k * b_sk]);
        s += p;
        sa += fabs(p);
    }
    *abs_sum = sa;
    return s;
}

void orc_gemm(const uint8_t *A, int fa, long long a_si, long long a_sk, double inv_sa,
              const uint8_t *B, int fb, long long b_sj, long long b_sk, double inv_sb,
              const double *bias, int M, int N, int K, double *C, double *C_abs)
{
    long long ij;
#pragma omp parallel for schedule(static)
    for (ij = 0; ij < (long long)M * N; ij++) {
        int i = (int)(ij / N), j = (int)(ij % N);
        double sa;
        double s = gemm_entry(A, fa, a_si, a_sk, B, fb, b_sj, b_sk, K, i, j, &sa);
        C[ij] = s * inv_sa * inv_sb + (bias ? bias[j] : 0.0);
        if (C_abs)
            C_abs[ij] = sa * inv_sa * inv_sb;
    }
}

/* The same entries, only at the listed (row, col) positions. */
void orc_gemm_sampled(const uint8_t *A, int fa, long long a_si, long long a_sk, double inv_sa,
                      const uint8_t *B, int fb, long long b_sj, long long b_sk, double inv_sb,
                      const double *bias, int K, const int *rows, const int *cols, long long nsamp,
                      double *C, double *C_abs)
{
    long long t;
#pragma omp parallel for schedule(dynamic, 16)
    for (t = 0; t < nsamp; t++) {
        double sa;
        double s = gemm_entry(A, fa, a_si, a_sk, B, fb, b_sj, b_sk, K, rows[t], cols[t], &sa);
        C[t] = s * inv_sa * inv_sb + (bias ? bias[cols[t]] : 0.0);
        if (C_abs)
            C_abs[t] = sa * inv_sa * inv_sb;
    }
}

/* ------------------------------------------------------------------------
 * Precision-decoupled Adam.  [FP8-LM] 提案手法 O2: FP8 first moment, FP16
 * second moment, FP16 master weights with tensor scaling; the gradient
 * arrives as FP8 (O1).  [FP8-LM] アブレーション研究 fixes FP16 (not FP8) for
 * the master and the second moment.
 * readings: Kingma-Ba Adam with bias correction and eps outside the square
 * root, no weight decay; the update uses the unquantised new moments; every
 * stored tensor gets a just-in-time power-of-two scale from its new amax
 * (same scale rule and margin as the linear layer; fmt_max 448 for the
 * E4M3 moment, 65504 for the FP16 moment and master).
 * ---------------------------------------------------------------------- */

/* Step 2-3 of the update in float64 on decoded values. */
void orc_adam_update_f64(size_t n, const double *g, const double *m0, const double *v0,
                         const double *w0, double lr, double beta1, double beta2, double eps,
                         int t, double *m, double *v, double *w)
{
    double bc1 = 1.0 - pow(beta1, (double)t);
    double bc2 = 1.0 - pow(beta2, (double)t);
    long long i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < (long long)n; i++) {
        m[i] = beta1 * m0[i] + (1.0 - beta1) * g[i];
        v[i] = beta2 * v0[i] + (1.0 - beta2) * g[i] * g[i];
        double mhat = m[i] / bc1;
        double vhat = v[i] / bc2;
        w[i] = w0[i] - lr * mhat / (sqrt(vhat) + eps);
    }
}

static double max_abs(const double *x, size_t n)
{
    double r = 0.0;
    for (size_t i = 0; i < n; i++) {
        if (isnan(x[i]))
            return NAN;
        if (fabs(x[i]) > r)
            r = fabs(x[i]);
    }
    return r;
}

/*
 * One Adam step over one tensor, in place on its stored form:
 *   gq (E5M2, descale g_inv = 1/(s_g mu)), mq (E4M3, scale *s_m),
 *   vh (FP16, scale *s_v), wh (FP16, scale *s_w).
 * Scratch: 7 arrays of n doubles supplied by the caller (work).
 * amax_out[0..2] receives amax|m|, amax v, amax|w| of the new float64 values.
 * amax_in: NULL, or the three amaxes the new scales are taken from instead
 * (those of the whole tensor when this call updates one slice of it, as in
 * the element-sharded optimizer of "FP8-LM", 提案手法 O3).
 * Returns ORC_ERR_NONFINITE if any amax the scales come from is not finite.
 */
int orc_adam_step_amax(size_t n, const uint8_t *gq, double g_inv, uint8_t *mq, double *s_m,
                       uint16_t *vh, double *s_v, uint16_t *wh, double *s_w, double lr, double beta1,
                       double beta2, double eps, int t, int margin, double *work,
                       const double *amax_in, double *amax_out)
{
    double *g = work, *m0 = work + n, *v0 = work + 2 * n, *w0 = work + 3 * n;
    double *m = work + 4 * n, *v = work + 5 * n, *w = work + 6 * n;
    long long i;
    /* 1. decode the stored state */
#pragma omp parallel for schedule(static)
    for (i = 0; i < (long long)n; i++) {
        g[i] = orc_fp8_decode(ORC_E5M2, gq[i]) * g_inv;
        m0[i] = orc_fp8_decode(ORC_E4M3, mq[i]) / *s_m;
        v0[i] = orc_f16_decode(vh[i]) / *s_v;
        w0[i] = orc_f16_decode(wh[i]) / *s_w;
    }
    /* 2-3. the update */
    orc_adam_update_f64(n, g, m0, v0, w0, lr, beta1, beta2, eps, t, m, v, w);
    /* 4. just-in-time scales from the new values */
    double am = max_abs(m, n), av = max_abs(v, n), aw = max_abs(w, n);
    amax_out[0] = am;
    amax_out[1] = av;
    amax_out[2] = aw;
    if (amax_in) {
        am = amax_in[0];
        av = amax_in[1];
        aw = amax_in[2];
    }
    int rc = ORC_OK;
    rc |= orc_compute_scale(am, ORC_E4M3, margin, s_m);
    rc |= orc_compute_scale(av, ORC_F16, margin, s_v);
    rc |= orc_compute_scale(aw, ORC_F16, margin, s_w);
    /* 5. requantise */
    double sm = *s_m, sv = *s_v, sw = *s_w;
#pragma omp parallel for schedule(static)
    for (i = 0; i < (long long)n; i++) {
        mq[i] = (uint8_t)orc_fp8_encode(ORC_E4M3, m[i] * sm);
        vh[i] = (uint16_t)orc_f16_encode(v[i] * sv);
        wh[i] = (uint16_t)orc_f16_encode(w[i] * sw);
    }
    return rc ? ORC_ERR_NONFINITE : ORC_OK;
}

int orc_adam_step(size_t n, const uint8_t *gq, double g_inv, uint8_t *mq, double *s_m,
                  uint16_t *vh, double *s_v, uint16_t *wh, double *s_w, double lr, double beta1,
                  double beta2, double eps, int t, int margin, double *work, double *amax_out)
{
    return orc_adam_step_amax(n, gq, g_inv, mq, s_m, vh, s_v, wh, s_w, lr, beta1, beta2, eps, t,
                              margin, work, NULL, amax_out);
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_num_threads(int nt)
{
#ifdef _OPENMP
    if (nt > 0)
        omp_set_num_threads(nt);
#else
    (void)nt;
#endif
}
