/*
 * echo_oracle.c - plain, slow, single-threaded CPU oracle for Echo's
 * error-compensated 4-bit all-reduce.
 *
 * TEST INFRASTRUCTURE ONLY: the CUDA library never calls this code and
 * shares nothing with it. The method, its sources and the readings this file
 * fixes are listed in echo_oracle.h.
 *
 * The steps follow the order the pages describe them
 * [rit.work "Echo 4-bit GPU communication", section "How Echo returns the
 *  error to later calls"]:
 *   1. each rank takes its partial sum; the owner of a segment adds the stored
 *      correction to its own partial;
 *   2. every rank rounds its partial to 4-bit integers per group (rounding #1);
 *   3. each segment owner restores the P incoming segments and adds them in
 *      high precision (binary32, rank 0 first);
 *   4. the owner rounds the total to 4-bit integers again (rounding #2), the
 *      value every rank receives;
 *   5. the owner measures the error that rounding #2 injected, from the
 *      high-precision total, and folds it into two smoothed estimates (fast and
 *      slow) that form the correction of the next call.
 *
 * Arithmetic: binary32 where the method computes (the sum, the correction, the
 * estimates), binary64 only where it is exact (scaling by powers of two,
 * comparing against 7 * 2^e). Compiled with -ffp-contract=off so that no
 * product is fused into a following add.
 */
#include "echo_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

static float bf16_bits_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float v;
    memcpy(&v, &u, sizeof v);
    return v;
}

/* A bf16 is the upper half of a binary32. The values written here are q*2^e
 * with |q| <= 7, so the lower half must be zero: anything else means the
 * output would need a third rounding, which the method excludes. */
static int float_to_bf16_bits_exact(float v, uint16_t *h)
{
    uint32_t u;
    memcpy(&u, &v, sizeof u);
    if ((u & 0xFFFFu) != 0)
        return -2;
    *h = (uint16_t)(u >> 16);
    return 0;
}

/* Smallest e >= -127 with A <= 7 * 2^e. */
static int choose_exponent(double A)
{
    int e = -127;
    while (!(A <= ldexp(7.0, e))) {
        e = e + 1;
        if (e > 126)
            return 1000; /* past the domain */
    }
    return e;
}

/* Largest magnitude of a group, exact in binary64; -1 for a non-finite value. */
static double group_absmax(const float *v, int G)
{
    double A = 0.0;
    for (int k = 0; k < G; k++) {
        if (!isfinite(v[k]))
            return -1.0;
        double a = fabs((double)v[k]);
        if (a > A)
            A = a;
    }
    return A;
}

int echo_oracle_quantize_group(const float *v, int G, int8_t *q)
{
    double A = group_absmax(v, G);
    if (A < 0)
        return -1;
    int e = choose_exponent(A);
    if (e > 126)
        return -2;
    for (int k = 0; k < G; k++) {
        /* v / 2^e is exact in binary64; nearbyint in the default rounding mode
         * rounds halves to even. */
        double t = nearbyint(ldexp((double)v[k], -e));
        if (t > 7.0 || t < -7.0)
            return -2; /* cannot happen when A <= 7 * 2^e */
        q[k] = (int8_t)t;
    }
    return e + 127;
}

float echo_oracle_dequant(int q, int b)
{
    return (float)ldexp((double)q, b - 127);
}

/* ---- binary16-scale variant ------------------------------------------- */

/* Value of a binary16 bit pattern (finite values only), exact in binary64:
 * sign, 5 exponent bits (bias 15), 10 fraction bits; exponent 0 holds the
 * subnormals frac * 2^-24. */
double echo_oracle_half_value(uint16_t h)
{
    int ex = (h >> 10) & 0x1F;
    int frac = h & 0x3FF;
    double v = ex == 0 ? ldexp((double)frac, -24) : ldexp((double)(frac | 0x400), ex - 25);
    return (h & 0x8000u) ? -v : v;
}

/* Smallest positive finite binary16 s with 7*s >= A (7*s is exact in
 * binary64); 0 when A == 0; the largest finite binary16, 65504, when no
 * binary16 is large enough (the codes then saturate at +-7). Positive
 * binary16 values grow with their bit patterns, so a bisection over the
 * patterns 0x0001..0x7BFF finds it. */
static uint16_t choose_half_scale(double A)
{
    if (A == 0.0)
        return 0;
    uint16_t lo = 1, hi = 0x7BFF;
    if (7.0 * echo_oracle_half_value(hi) < A)
        return hi;
    while (lo < hi) {
        uint16_t mid = (uint16_t)(lo + (hi - lo) / 2);
        if (7.0 * echo_oracle_half_value(mid) >= A)
            hi = mid;
        else
            lo = (uint16_t)(mid + 1);
    }
    return lo;
}

/* The code in [-7, 7] nearest to v/s, a tie going to the even code. |v| is
 * compared with the midpoints (k + 1/2)*s, which binary64 holds exactly
 * (at most 15 significant bits), so no quotient is rounded. */
static int nearest_code(double v, double s)
{
    double a = fabs(v);
    int k = 0;
    while (k < 7 && a > (k + 0.5) * s)
        k = k + 1;
    if (k < 7 && a == (k + 0.5) * s && (k % 2) == 1)
        k = k + 1;
    return v < 0 ? -k : k;
}

int echo_oracle_quantize_group_f16(const float *v, int G, int8_t *q, uint16_t *scale)
{
    double A = group_absmax(v, G);
    if (A < 0)
        return -1;
    uint16_t h = choose_half_scale(A);
    double sv = echo_oracle_half_value(h);
    for (int k = 0; k < G; k++)
        q[k] = (int8_t)nearest_code((double)v[k], sv);
    *scale = h;
    return 0;
}

float echo_oracle_dequant_f16(int q, uint16_t h)
{
    return (float)((double)q * echo_oracle_half_value(h)); /* <= 14 significant bits: exact */
}

/* v rounded to the nearest bf16 (8 significant bits), a tie going to the
 * even last bit; v is finite with |v| < 2^127. */
float echo_oracle_round_bf16(float v)
{
    double a = fabs((double)v);
    if (a == 0.0)
        return v;
    int e;
    frexp(a, &e);                             /* 2^(e-1) <= a < 2^e */
    double step = ldexp(1.0, (e - 8 < -133) ? -133 : e - 8);
    double lo = floor(a / step) * step;       /* power-of-two scaling: exact */
    double hi = lo + step;
    double r;
    if (a - lo < hi - a)
        r = lo;
    else if (a - lo > hi - a)
        r = hi;
    else
        r = (fmod(lo / step, 2.0) == 0.0) ? lo : hi;
    return (float)(v < 0 ? -r : r);
}

void echo_oracle_pack(const int8_t *q, size_t count, uint8_t *out)
{
    for (size_t j = 0; j < count / 2; j++) {
        unsigned lo = (unsigned)q[2 * j] & 0xFu;
        unsigned hi = (unsigned)q[2 * j + 1] & 0xFu;
        out[j] = (uint8_t)(lo | (hi << 4));
    }
}

static int nibble_value(unsigned u)
{
    return (u & 0x8u) ? (int)u - 16 : (int)u;
}

void echo_oracle_unpack(const uint8_t *in, size_t count, int8_t *q)
{
    for (size_t j = 0; j < count / 2; j++) {
        q[2 * j] = (int8_t)nibble_value(in[j] & 0xFu);
        q[2 * j + 1] = (int8_t)nibble_value(in[j] >> 4);
    }
}

static float load_input(const void *x, int dtype, size_t idx)
{
    if (dtype == ECHO_ORACLE_BF16)
        return bf16_bits_to_float(((const uint16_t *)x)[idx]);
    return ((const float *)x)[idx];
}

static int store_output(void *out, int dtype, size_t idx, float v)
{
    if (dtype == ECHO_ORACLE_BF16)
        return float_to_bf16_bits_exact(v, &((uint16_t *)out)[idx]);
    ((float *)out)[idx] = v;
    return 0;
}

/* Restored value of code q under a scale byte (power of two) or a binary16
 * scale pattern. */
static float restore(int q, int scale, int half_scale)
{
    return half_scale ? echo_oracle_dequant_f16(q, (uint16_t)scale) : echo_oracle_dequant(q, scale);
}

static void put_scale(uint8_t *out, size_t t, int scale, int half_scale)
{
    if (half_scale) {
        out[2 * t] = (uint8_t)(scale & 0xFF);
        out[2 * t + 1] = (uint8_t)((scale >> 8) & 0xFF);
    } else {
        out[t] = (uint8_t)scale;
    }
}

int echo_oracle_allreduce_groups_ex(int P, int G, size_t ngroups,
                                    const int32_t *owner, int dtype,
                                    const void *x, void *out, float *f, float *s,
                                    float *eps, float lambda, float beta_f,
                                    float beta_s, int enable, int variant,
                                    uint8_t *codes1, uint8_t *scales1,
                                    uint8_t *qcodes, uint8_t *qscales,
                                    float *c_out, float *err_out)
{
    const int owner_sum = (variant & ECHO_ORACLE_OWNER_SUM) != 0;
    const int sender_ef = (variant & ECHO_ORACLE_SENDER_EF) != 0;
    const int half_scale = (variant & ECHO_ORACLE_FP16_SCALE) != 0;
    if (P < 2 || P > 16 || G < 2 || (G % 2) != 0 || ngroups == 0)
        return -1;
    if (dtype != ECHO_ORACLE_BF16 && dtype != ECHO_ORACLE_FP32)
        return -1;
    if (variant & ~(ECHO_ORACLE_OWNER_SUM | ECHO_ORACLE_SENDER_EF | ECHO_ORACLE_FP16_SCALE))
        return -1;
    if (!owner || !x || !out || (enable && (!f || !s)) || (sender_ef && !eps))
        return -1;
    for (size_t g = 0; g < ngroups; g++)
        if (owner[g] < 0 || owner[g] >= P)
            return -1;

    const size_t m = ngroups * (size_t)G;
    int rc = 0;
    float *c = (float *)calloc(m, sizeof(float));
    float *v = (float *)malloc((size_t)G * sizeof(float));
    int8_t *q1 = (int8_t *)malloc((size_t)P * m);
    int *b1 = (int *)malloc((size_t)P * ngroups * sizeof(int));
    float *S = (float *)malloc((size_t)G * sizeof(float));
    int8_t *Q = (int8_t *)malloc(m);
    int *bQ = (int *)malloc(ngroups * sizeof(int));
    if (!c || !v || !q1 || !b1 || !S || !Q || !bQ) {
        rc = -1;
        goto done;
    }

    const float one_minus_lambda = 1.0f - lambda;
    const float one_minus_beta_f = 1.0f - beta_f;
    const float one_minus_beta_s = 1.0f - beta_s;

    /* Step 1: the correction each owner adds, from the stored estimates. */
    if (enable) {
        for (size_t i = 0; i < m; i++) {
            float from_fast = lambda * f[i];
            float from_slow = one_minus_lambda * s[i];
            c[i] = from_fast + from_slow;
        }
    }

    /* Steps 1-2: every rank forms its value (the owner with the correction)
     * and rounds it to 4-bit codes per group: rounding #1. */
    for (int r = 0; r < P; r++) {
        for (size_t g = 0; g < ngroups; g++) {
            for (int k = 0; k < G; k++) {
                size_t i = g * (size_t)G + (size_t)k;
                float xi = load_input(x, dtype, (size_t)r * m + i);
                if (!isfinite(xi)) {
                    rc = -1;
                    goto done;
                }
                /* Variant: the rank first adds back its own rounding-#1 error
                 * of its previous call. */
                float u = xi;
                if (sender_ef)
                    u = xi + eps[(size_t)r * m + i];
                if (enable && !owner_sum && owner[g] == r)
                    v[k] = u + c[i];
                else
                    v[k] = u;
            }
            int b;
            if (half_scale) {
                uint16_t h = 0;
                b = echo_oracle_quantize_group_f16(v, G, q1 + (size_t)r * m + g * (size_t)G, &h);
                if (b == 0)
                    b = h;
            } else {
                b = echo_oracle_quantize_group(v, G, q1 + (size_t)r * m + g * (size_t)G);
            }
            if (b < 0) {
                rc = b;
                goto done;
            }
            b1[(size_t)r * ngroups + g] = b;
            /* Variant: keep this rounding's error for the rank's next call
             * (exact in binary32, as for rounding #2, unless a binary16
             * scale saturated). */
            if (sender_ef)
                for (int k = 0; k < G; k++) {
                    size_t i = g * (size_t)G + (size_t)k;
                    float restored = restore(q1[(size_t)r * m + i], b, half_scale);
                    eps[(size_t)r * m + i] = v[k] - restored;
                }
        }
    }

    /* Steps 3-5, per group at its owner. */
    for (size_t g = 0; g < ngroups; g++) {
        /* Step 3: restore the P segments and add them in binary32, rank 0
         * first. Each restored value is exact. */
        for (int k = 0; k < G; k++) {
            size_t i = g * (size_t)G + (size_t)k;
            float sum = 0.0f;
            for (int r = 0; r < P; r++) {
                float d = restore(q1[(size_t)r * m + i], b1[(size_t)r * ngroups + g], half_scale);
                sum = sum + d;
            }
            /* Variant: the owner folds the correction into its sum, after
             * the P ranks, instead of the sender adding it to its partial. */
            if (enable && owner_sum)
                sum = sum + c[i];
            S[k] = sum;
        }
        /* Step 4: rounding #2 of the total. */
        int bq;
        if (half_scale) {
            uint16_t h = 0;
            bq = echo_oracle_quantize_group_f16(S, G, Q + g * (size_t)G, &h);
            if (bq == 0)
                bq = h;
        } else {
            bq = echo_oracle_quantize_group(S, G, Q + g * (size_t)G);
        }
        if (bq < 0) {
            rc = bq;
            goto done;
        }
        bQ[g] = bq;
        for (int k = 0; k < G; k++) {
            size_t i = g * (size_t)G + (size_t)k;
            float Y = restore(Q[i], bq, half_scale);
            /* Variant: a binary16 scale makes Y a 14-bit value, which a bf16
             * output rounds once more; every rank receives that value. */
            if (half_scale && dtype == ECHO_ORACLE_BF16)
                Y = echo_oracle_round_bf16(Y);
            /* Step 5: the error injected into what the ranks receive (exact
             * in binary32). */
            float err = S[k] - Y;
            if (enable) {
                float f_keep = beta_f * f[i];
                float f_new = one_minus_beta_f * err;
                f[i] = f_keep + f_new;
                float s_keep = beta_s * s[i];
                float s_new = one_minus_beta_s * err;
                s[i] = s_keep + s_new;
            }
            if (err_out)
                err_out[i] = err;
            if (c_out)
                c_out[i] = c[i];
            int so = store_output(out, dtype, i, Y);
            if (so != 0) {
                rc = so;
                goto done;
            }
        }
    }

    if (codes1)
        for (int r = 0; r < P; r++)
            echo_oracle_pack(q1 + (size_t)r * m, m, codes1 + (size_t)r * (m / 2));
    /* Scale bytes: one per group, or a little-endian binary16 (two bytes)
     * per group under the binary16-scale variant. */
    if (scales1)
        for (size_t t = 0; t < (size_t)P * ngroups; t++)
            put_scale(scales1, t, b1[t], half_scale);
    if (qcodes)
        echo_oracle_pack(Q, m, qcodes);
    if (qscales)
        for (size_t g = 0; g < ngroups; g++)
            put_scale(qscales, g, bQ[g], half_scale);

done:
    free(c);
    free(v);
    free(q1);
    free(b1);
    free(S);
    free(Q);
    free(bQ);
    return rc;
}

int echo_oracle_allreduce_groups(int P, int G, size_t ngroups,
                                 const int32_t *owner, int dtype,
                                 const void *x, void *out, float *f, float *s,
                                 float lambda, float beta_f, float beta_s,
                                 int enable, uint8_t *codes1, uint8_t *scales1,
                                 uint8_t *qcodes, uint8_t *qscales,
                                 float *c_out, float *err_out)
{
    return echo_oracle_allreduce_groups_ex(P, G, ngroups, owner, dtype, x, out, f, s, NULL,
                                           lambda, beta_f, beta_s, enable, 0, codes1,
                                           scales1, qcodes, qscales, c_out, err_out);
}

int echo_oracle_allreduce_ex(int P, size_t n, int G, int dtype, const void *x,
                             void *out, float *f, float *s, float *eps, float lambda,
                             float beta_f, float beta_s, int enable, int variant,
                             uint8_t *codes1, uint8_t *scales1, uint8_t *qcodes,
                             uint8_t *qscales, float *c_out, float *err_out)
{
    if (P < 2 || G < 2 || n == 0 || n % ((size_t)P * (size_t)G) != 0)
        return -1;
    size_t ngroups = n / (size_t)G;
    size_t seg = n / (size_t)P;
    int32_t *owner = (int32_t *)malloc(ngroups * sizeof(int32_t));
    if (!owner)
        return -1;
    for (size_t g = 0; g < ngroups; g++)
        owner[g] = (int32_t)((g * (size_t)G) / seg);
    int rc = echo_oracle_allreduce_groups_ex(P, G, ngroups, owner, dtype, x, out, f, s, eps,
                                             lambda, beta_f, beta_s, enable, variant, codes1,
                                             scales1, qcodes, qscales, c_out, err_out);
    free(owner);
    return rc;
}

int echo_oracle_allreduce(int P, size_t n, int G, int dtype, const void *x,
                          void *out, float *f, float *s, float lambda,
                          float beta_f, float beta_s, int enable,
                          uint8_t *codes1, uint8_t *scales1, uint8_t *qcodes,
                          uint8_t *qscales, float *c_out, float *err_out)
{
    return echo_oracle_allreduce_ex(P, n, G, dtype, x, out, f, s, NULL, lambda, beta_f,
                                    beta_s, enable, 0, codes1, scales1, qcodes, qscales,
                                    c_out, err_out);
}
