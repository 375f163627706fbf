/*
 * echo_oracle.h - CPU oracle for Echo's error-compensated 4-bit all-reduce.
 *
 * TEST INFRASTRUCTURE. This library exists to check the CUDA library against
 * a plain restatement of the method. Only the test suite, the package's
 * smoke check and the benchmark's CPU-baseline leg load it. It shares no
 * code, header, table or helper with the CUDA library, and neither side
 * includes or links the other.
 *
 * Sources restated (both pages are digests of the preprint "Echo:
 * Error-Compensated 4-Bit Tensor-Parallel Communication for LLM Training and
 * Inference"):
 *   [rit.work "Echo 4-bit GPU communication", section "How Echo returns the
 *    error to later calls"]: segments travel as 4-bit integers; the segment
 *    owner restores and adds them in high precision; the compressed total goes
 *    back to every rank; each element is rounded at most twice whatever the
 *    group size; the error of the last rounding is measured from the
 *    high-precision sum, stored, and added back in later calls; two smoothed
 *    estimates (fast, slow) are kept; forward and backward keep separate state.
 *   [heraldofai.com "Come Echo permette ai modelli AI...", section "Come Echo
 *    evita che gli errori si accumulino"]: the same mechanism.
 *
 * The pages give no group size, scale format, rounding mode, EMA coefficients
 * or combining rule. The readings fixed here (all are also the CUDA
 * library's contract):
 *   - group G of consecutive elements (32 in the product; any even G >= 2 here);
 *   - power-of-two scale 2^e stored as the byte e+127, e the smallest integer
 *     >= -127 with max|v| <= 7 * 2^e (no code ever saturates);
 *   - codes q = round-half-to-even(v / 2^e) in [-7, 7], two per byte, element
 *     2j in the low nibble, element 2j+1 in the high nibble, two's complement;
 *   - the owner of element i is the rank whose contiguous segment holds it;
 *   - only the owner adds the correction c to its own partial, before its
 *     rounding #1;
 *   - the owner sums the P dequantised values in binary32, rank 0 first;
 *   - the captured error is err = S - Y with Y the requantised total;
 *   - f <- beta_f*f + (1-beta_f)*err, s <- beta_s*s + (1-beta_s)*err and
 *     c = lambda*f + (1-lambda)*s, every product and sum rounded to binary32
 *     on its own (no fused multiply-add), 1-lambda and 1-beta themselves
 *     formed in binary32, subnormals kept; with sender feedback the owner's
 *     value is (x + eps) + c, rounded after each add. The tests pin this order
 *     with hand-worked cases where a fused or regrouped form gives another
 *     binary32 value (tests/golden/rounding_order_p3_g32.json).
 *
 * Status codes: 0 on success, -1 on an invalid argument or a non-finite
 * value, -2 when a value leaves the domain (output not exactly
 * representable in bf16, scale search past e = 126).
 */
#ifndef ECHO_ORACLE_H
#define ECHO_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ECHO_ORACLE_BF16 0
#define ECHO_ORACLE_FP32 1

/* Variants (bits of `variant` in the _ex calls; 0 is the method above):
 *   ECHO_ORACLE_OWNER_SUM  the owner adds the correction c to its binary32
 *                          sum, after the P restored values, instead of the
 *                          sender adding it to its partial before rounding #1;
 *   ECHO_ORACLE_SENDER_EF  every rank keeps its own rounding-#1 error
 *                          eps = v - q*2^e per element (exact) and adds it to
 *                          its partial in its next call, before the owner's
 *                          correction: v = RN(RN(x + eps) + c). */
#define ECHO_ORACLE_OWNER_SUM 1
#define ECHO_ORACLE_SENDER_EF 2
/*   ECHO_ORACLE_FP16_SCALE every group (both roundings) takes a binary16
 *                          scale s instead of a power of two: s is the
 *                          smallest positive finite binary16 with
 *                          7*s >= max|v| (0 for an all-zero group; 65504,
 *                          with saturated codes, past 7*65504); each code is
 *                          the integer in [-7, 7] nearest to v/s, ties to
 *                          even. Restored values q*s are exact in binary32;
 *                          bf16 outputs are q*s rounded to the nearest bf16
 *                          (ties to even), and the captured error is taken
 *                          against that received value. Wire scales are
 *                          little-endian binary16, two bytes per group. */
#define ECHO_ORACLE_FP16_SCALE 4

/* Scale choice and rounding of one group (rounding #1 at a sender, #2 at the
 * owner). v: G binary32 values. Writes G codes to q. Returns the scale byte
 * e+127 (0..253), or -1 for a non-finite value, -2 past the domain. */
int echo_oracle_quantize_group(const float *v, int G, int8_t *q);

/* Value of code q under scale byte b: q * 2^(b-127), exact in binary32. */
float echo_oracle_dequant(int q, int b);

/* Binary16-scale codec (variant ECHO_ORACLE_FP16_SCALE): scale pattern and
 * codes of one group (returns 0, or -1 for a non-finite value); the value of
 * code q under scale pattern h; the value of a binary16 pattern; a binary32
 * rounded to the nearest bf16, ties to even. */
int echo_oracle_quantize_group_f16(const float *v, int G, int8_t *q, uint16_t *scale);
float echo_oracle_dequant_f16(int q, uint16_t h);
double echo_oracle_half_value(uint16_t h);
float echo_oracle_round_bf16(float v);

/* Pack count codes (count even) two per byte; unpack the reverse. */
void echo_oracle_pack(const int8_t *q, size_t count, uint8_t *out);
void echo_oracle_unpack(const uint8_t *in, size_t count, int8_t *q);

/*
 * One all-reduce call over ngroups groups of G elements.
 *
 * x        P rank partials, rank-major: x[r*m + i], m = ngroups*G elements
 *          each; uint16 bf16 bit patterns (dtype 0) or binary32 (dtype 1).
 * owner    owner rank of each group (0..P-1).
 * f, s     the phase's compensator state, m binary32 each, read and updated
 *          in place (untouched when enable == 0).
 * out      m elements of dtype: the value every rank receives.
 * codes1   optional [P][m/2] stage-1 packed codes, scales1 [P][ngroups]
 *          (bytes; [P][2*ngroups] under ECHO_ORACLE_FP16_SCALE).
 * qcodes   optional [m/2] requantised codes, qscales [ngroups] (bytes;
 *          [2*ngroups] under ECHO_ORACLE_FP16_SCALE).
 * c_out    optional [m] correction the owner added (0 when off).
 * err_out  optional [m] captured error S - Y.
 */
int echo_oracle_allreduce_groups(int P, int G, size_t ngroups,
                                 const int32_t *owner, int dtype,
                                 const void *x, void *out, float *f, float *s,
                                 float lambda, float beta_f, float beta_s,
                                 int enable, uint8_t *codes1, uint8_t *scales1,
                                 uint8_t *qcodes, uint8_t *qscales,
                                 float *c_out, float *err_out);

/* The same with a variant (see above); eps [P][m] is every rank's
 * rounding-#1 error state, read and updated when ECHO_ORACLE_SENDER_EF. */
int echo_oracle_allreduce_groups_ex(int P, int G, size_t ngroups,
                                    const int32_t *owner, int dtype,
                                    const void *x, void *out, float *f, float *s,
                                    float *eps, float lambda, float beta_f,
                                    float beta_s, int enable, int variant,
                                    uint8_t *codes1, uint8_t *scales1,
                                    uint8_t *qcodes, uint8_t *qscales,
                                    float *c_out, float *err_out);

/* Same call over n elements per rank with contiguous segments: rank r owns
 * elements [r*n/P, (r+1)*n/P). Requires n % (P*G) == 0. */
int echo_oracle_allreduce(int P, size_t n, int G, int dtype, const void *x,
                          void *out, float *f, float *s, float lambda,
                          float beta_f, float beta_s, int enable,
                          uint8_t *codes1, uint8_t *scales1, uint8_t *qcodes,
                          uint8_t *qscales, float *c_out, float *err_out);

int echo_oracle_allreduce_ex(int P, size_t n, int G, int dtype, const void *x,
                             void *out, float *f, float *s, float *eps, float lambda,
                             float beta_f, float beta_s, int enable, int variant,
                             uint8_t *codes1, uint8_t *scales1, uint8_t *qcodes,
                             uint8_t *qscales, float *c_out, float *err_out);

#ifdef __cplusplus
}
#endif
#endif
