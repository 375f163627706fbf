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

int echo_oracle_quantize_group(const float *v, int G, int8_t *q)
{
    double A = 0.0;
    for (int k = 0; k < G; k++) {
        if (!isfinite(v[k]))
            return -1;
        double a = fabs((double)v[k]);
        if (a > A)
            A = a;
    }
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
    if (P < 2 || P > 16 || G < 2 || (G % 2) != 0 || ngroups == 0)
        return -1;
    if (dtype != ECHO_ORACLE_BF16 && dtype != ECHO_ORACLE_FP32)
        return -1;
    if (variant & ~(ECHO_ORACLE_OWNER_SUM | ECHO_ORACLE_SENDER_EF))
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
            int b = echo_oracle_quantize_group(v, G, q1 + (size_t)r * m + g * (size_t)G);
            if (b < 0) {
                rc = b;
                goto done;
            }
            b1[(size_t)r * ngroups + g] = b;
            /* Variant: keep this rounding's error for the rank's next call
             * (exact in binary32, as for rounding #2). */
            if (sender_ef)
                for (int k = 0; k < G; k++) {
                    size_t i = g * (size_t)G + (size_t)k;
                    float restored = echo_oracle_dequant(q1[(size_t)r * m + i], b);
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
                float d = echo_oracle_dequant(q1[(size_t)r * m + i], b1[(size_t)r * ngroups + g]);
                sum = sum + d;
            }
            /* Variant: the owner folds the correction into its sum, after
             * the P ranks, instead of the sender adding it to its partial. */
            if (enable && owner_sum)
                sum = sum + c[i];
            S[k] = sum;
        }
        /* Step 4: rounding #2 of the total. */
        int bq = echo_oracle_quantize_group(S, G, Q + g * (size_t)G);
        if (bq < 0) {
            rc = bq;
            goto done;
        }
        bQ[g] = bq;
        for (int k = 0; k < G; k++) {
            size_t i = g * (size_t)G + (size_t)k;
            float Y = echo_oracle_dequant(Q[i], bq);
            /* Step 5: the error rounding #2 injected (exact in binary32). */
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
    if (scales1)
        for (size_t t = 0; t < (size_t)P * ngroups; t++)
            scales1[t] = (uint8_t)b1[t];
    if (qcodes)
        echo_oracle_pack(Q, m, qcodes);
    if (qscales)
        for (size_t g = 0; g < ngroups; g++)
            qscales[g] = (uint8_t)bQ[g];

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
