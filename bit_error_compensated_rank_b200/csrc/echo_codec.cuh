// echo_codec.cuh - device-side 4-bit codec of the Echo all-reduce.
//
// Format (fixed readings of the 4-bit segments on [rit.work "Echo 4-bit GPU
// communication", section "How Echo returns the error to later calls"]):
// groups of G consecutive elements (32 by default; 16, 64 and 128 are the
// group-size variants) share a power-of-two scale 2^e, stored
// as the byte e+127, e the smallest integer >= -127 with max|v| <= 7*2^e;
// codes are round(v/2^e), halves to even, in [-7, 7]; two codes per byte,
// element 2j in the low nibble, two's complement.
//
// Every helper here is exact integer or power-of-two arithmetic; the only
// rounding is the choice of the nearest code (code_bits), which rounds halves
// to even.
//
// Binary16-scale variant: the scale is the smallest positive finite binary16
// s with 7*s >= max|v| (0 for an all-zero group, 65504 with saturated codes
// beyond 7*65504), stored as its two-byte pattern; codes are the integers in
// [-7, 7] nearest to v/s, ties to even (code_bits_near). Restored values q*s
// have at most 14 significant bits and are exact in binary32.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace echo {

constexpr int kChunk = 8;           // elements per thread (one 32-bit code word)
constexpr int kMinGroup = 16;       // elements per scale: 16, 32, 64 or 128 (2, 4, 8 or 16 lanes)
constexpr int kMaxRanks = 16;

struct RankPtrs {
    const void *p[kMaxRanks];
};
struct RankOutPtrs {
    void *p[kMaxRanks];
};

// Scale byte e+127 of a group from its absolute maximum A (finite, >= 0).
// With A = (1 + M/2^23) * 2^(E-127) (E the exponent field, M the mantissa
// field), A <= 7*2^e holds for e = E-129 exactly when the leading factor is
// at most 7/4, i.e. M <= 0x600000; otherwise e = E-128. Zero and subnormal A
// (E = 0) and every A <= 7*2^-127 land on the floor e = -127 (byte 0).
__device__ __forceinline__ uint32_t scale_byte(float A)
{
    const uint32_t u = __float_as_uint(A);
    const int E = static_cast<int>(u >> 23);
    const int b = E - 2 + ((u & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    return b < 0 ? 0u : static_cast<uint32_t>(b);
}

// 2^(byte-127) as a binary32; byte 0 is the subnormal 2^-127.
__device__ __forceinline__ float step_of(uint32_t byte)
{
    return __uint_as_float(byte ? (byte << 23) : 0x00400000u);
}

// 2^(127-byte), byte in [0, 253]: always a normal binary32.
__device__ __forceinline__ float inv_step_of(uint32_t byte)
{
    return __uint_as_float((254u - byte) << 23);
}

// ---- rounding to a code ---------------------------------------------------
// kRound = 1.5 * 2^23. For |t| <= 7, RN(t + kRound) lands in [2^23, 2^24),
// where the spacing of binary32 is exactly 1, so the addition rounds t to the
// nearest integer k, halves to the even one (kRound is even, so the last
// significand bit is the parity of k), and the bit pattern of the result is
// 0x4B400000 + k: its low byte is k as a two's-complement int8.
// fma(v, inv, kRound) computes RN(v*inv + kRound) from the exact product
// v*inv (inv is a power of two and |v*inv| <= 7 by the scale rule), so it is
// round-half-even(v / 2^e) with no intermediate rounding, subnormals included.
constexpr float kRound = 12582912.0f;      // 1.5 * 2^23, bits 0x4B400000
constexpr uint32_t kRoundBits = 0x4B400000u;
constexpr float kRoundPlus8 = 12582920.0f; // kRound + 8

// Bit pattern kRoundBits + q of the nearest code q of v at step 1/inv.
__device__ __forceinline__ uint32_t code_bits(float v, float inv)
{
    return __float_as_uint(__fmaf_rn(v, inv, kRound));
}

// Code q (as a float) from its rounded bit pattern (exact subtraction).
__device__ __forceinline__ float code_value(uint32_t bits)
{
    return __fsub_rn(__uint_as_float(bits), kRound);
}

// ---- binary16 scales --------------------------------------------------------
// Value of a binary16 scale pattern (exact conversion).
__device__ __forceinline__ float half_step(uint32_t h)
{
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h)));
}

// Smallest positive finite binary16 s with 7*s >= A (A finite, >= 0), as its
// pattern; 0 for A == 0; 0x7BFF (65504) when 7*65504 < A. The estimate
// u = A * RU(1/7), rounded up, is at least A/7 and within a relative 2^-22
// of it; rounded up to binary16 it is therefore never below the answer and
// at most one binary16 step above it (the binary16 spacing is 2^-10
// relative). One exact test on the step below settles it: 7*s has at most
// 14 significant bits, so the binary32 product is exact.
__device__ __forceinline__ uint32_t half_scale_bits(float A)
{
    const float u = __fmul_ru(A, __uint_as_float(0x3E124925u)); // RU(1/7) = 0.14285715
    const uint32_t h = min(static_cast<uint32_t>(__half_as_ushort(__float2half_ru(u))), 0x7BFFu);
    const bool down = h > 1u && __fmul_rn(7.f, half_step(h - 1u)) >= A;
    return h - (down ? 1u : 0u);
}

// Bit pattern kRoundBits + q of the code q in [-7, 7] nearest to v/step, a
// tie going to the even code, for any step >= 0 (inv an estimate of 1/step,
// 0 when step is 0; half = step/2, exact). The estimate k = nearest integer
// to v*inv can only miss by one, next to a midpoint; the remainder
// r = v - k*step is exact there (|r| <= step/2 needs at most 24 significant
// bits), so comparing |r| with half moves k to the nearest code, or off an
// odd code on a tie. The pattern kRound + k has k's parity in its last bit
// and moves by one per code. A saturated group (v/step beyond 7.5) ends at
// +-7 after the clamp.
__device__ __forceinline__ uint32_t code_bits_near(float v, float step, float inv, float half)
{
    const float y = fminf(fmaxf(__fmul_rn(v, inv), -8.f), 8.f);
    const float t = __fadd_rn(y, kRound);
    const float r = __fmaf_rn(-__fsub_rn(t, kRound), step, v);
    const float ar = fabsf(r);
    int bits = __float_as_int(t);
    if (ar > half || (ar == half && (bits & 1)))
        bits += r < 0.f ? -1 : 1;
    bits = min(max(bits, static_cast<int>(kRoundBits) - 7), static_cast<int>(kRoundBits) + 7);
    return static_cast<uint32_t>(bits);
}

// True when a group with maximum A gets the saturated scale 65504 and codes
// clamped at +-7.
__device__ __forceinline__ bool half_scale_saturates(float A)
{
    return A > 458528.f; // 7 * 65504
}

// The 8 codes of one lane under a binary16 step (the results of
// code_bits_near), in z-form: the bit pattern z of the binary32
// RN(v*inv + kZ), kZ = 192 + 1/2 + 2*2^-16. In a group whose scale did not
// saturate, |v/step| <= 7, so z stays in the binade [128, 256), where the
// spacing is 2^-16 and z = 0x43400000 + Z with the integer
// Z = RN(2^16*(v*inv + 1/2) + 2). Then z >> 16 = 0x4340 + floor(Z / 2^16),
// and byte 2 of z holds that code as 0x40 + q (its low nibble is q in two's
// complement). inv has a relative error of at most about 2^-23 (half_inv),
// so Z lies within 0.56 of 2^16*(v/step + 1/2) + 2. When the low 16 bits of
// Z are at least 3, 2^16*(v/step + 1/2) is then strictly between two
// multiples of 2^16 and floor(Z / 2^16) is the nearest code to v/step, not a
// tie. The lane takes the minimum of its 8 low halves two at a time (a 16x2
// minimum); if one is below 3, or the group saturated, the lane takes the exact path for all 8
// values: one branch per lane, taken rarely.
//
// Values of 8 significant bits (bf16 partials that carry no correction)
// need no exact path. With v = a*2^p (|a| < 2^8) and the step s = b*2^q
// (b < 2^11, any binary16), a non-zero distance from v/s to a midpoint,
// |v/s - (j + 1/2)| = |2a*2^p - (2j+1)*b*2^q| / (2b*2^q), is at least
// 2^(min(p,q)-q) / (2b): more than 2^-12 when p >= q; when p < q, a |v|
// that reaches a midpoint (>= s/2) has 2^(p-q) >= b/(2|a|), so more than
// 2^-10. That is at least 16 units of 2^-16 against the estimate's 0.06, so
// floor(Z / 2^16) is the nearest code unless v/s is exactly a midpoint. An
// exact midpoint lands on a fraction of exactly 2 and floor(Z / 2^16) is the
// code above it; the tie goes to the even code, so an odd code moves down
// by one. A fraction below kZTie flags those values: no 8-bit value reaches
// [0, kZTie) otherwise.
constexpr float kZ = 192.500030517578125f; // 192 + 1/2 + 2*2^-16, bits 0x43408002
constexpr uint32_t kZMargin = 3;
constexpr uint32_t kZTie = 4;

__device__ __forceinline__ uint32_t min_u16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("min.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// z-form of the rounded pattern kRoundBits + q (for the exact path).
__device__ __forceinline__ uint32_t zcode_of_bits(uint32_t bits)
{
    return ((bits - kRoundBits) << 16) + 0x43408000u;
}

// The rounded pattern kRoundBits + q of a z-form code (code_value, pack8_bits).
__device__ __forceinline__ uint32_t zcode_bits(uint32_t z)
{
    return (z >> 16) + (kRoundBits - 0x4340u);
}

// Whether either 16-bit half of x is below bound (<= 0x8000): such a half
// borrows into its own top bit, which was clear.
__device__ __forceinline__ bool half_below(uint32_t x, uint32_t bound)
{
    return ((x - bound * 0x00010001u) & ~x & 0x80008000u) != 0;
}

// short_vals: every v[k] has at most 8 significant bits (see kZTie).
// The z-form products go two at a time through sm_100's packed f32x2 FMA,
// which rounds each component exactly as the scalar __fmaf_rn does. One
// test sends a lane off the common path: a saturated scale, or a fraction
// below the margin (below kZTie for short values); there a saturated or
// long-valued lane takes the exact path and a short-valued one settles its
// exact midpoints.
__device__ __forceinline__ void codes8_half(const float (&v)[kChunk], float step, float inv, float half, bool sat,
                                            bool short_vals, uint32_t (&z)[kChunk])
{
#pragma unroll
    for (int j = 0; j < kChunk / 2; j++) {
        const float2 p = __ffma2_rn(make_float2(v[2 * j], v[2 * j + 1]), make_float2(inv, inv), make_float2(kZ, kZ));
        z[2 * j] = __float_as_uint(p.x);
        z[2 * j + 1] = __float_as_uint(p.y);
    }
    const uint32_t lo = min_u16x2(min_u16x2(__byte_perm(z[0], z[1], 0x5410), __byte_perm(z[2], z[3], 0x5410)),
                                  min_u16x2(__byte_perm(z[4], z[5], 0x5410), __byte_perm(z[6], z[7], 0x5410)));
    if (sat || half_below(lo, short_vals ? kZTie : kZMargin)) {
        if (sat || !short_vals) {
#pragma unroll
            for (int k = 0; k < kChunk; k++)
                z[k] = zcode_of_bits(code_bits_near(v[k], step, inv, half));
        } else {
            // exact midpoints: an odd code (bit 16, the parity of byte 2) moves down
#pragma unroll
            for (int k = 0; k < kChunk; k++)
                if ((z[k] & 0x1FFFFu) - 0x10000u < kZTie)
                    z[k] -= 0x10000u;
        }
    }
}

// Reciprocal estimate used by code_bits_near and codes8_half (0 for a zero
// step): the hardware approximation (rcp.approx, at most 1 ulp off, so a
// relative error of at most 2^-23; steps are normal binary32 values). Both
// users settle every code exactly, so the estimate only has to be close.
__device__ __forceinline__ float half_inv(float step)
{
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(step));
    return step > 0.f ? r : 0.f;
}

// Nearest bf16 to a binary32 (ties to even), as the upper half of a binary32:
// the value every rank receives under binary16 scales with bf16 outputs.
__device__ __forceinline__ float round_bf16(float y)
{
    return __bfloat162float(__float2bfloat16_rn(y));
}

// Pack the codes of 8 rounded bit patterns (element k = low byte of b[k])
// into one word, element 2j in the low nibble of byte j and 2j+1 in its high
// nibble. prmt gathers the low bytes of the even and the odd elements; one
// shift and one masked merge interleave them.
__device__ __forceinline__ uint32_t pack8_bits(const uint32_t (&b)[kChunk])
{
    const uint32_t even = __byte_perm(__byte_perm(b[0], b[2], 0x0040), __byte_perm(b[4], b[6], 0x0040), 0x5410);
    const uint32_t odd = __byte_perm(__byte_perm(b[1], b[3], 0x0040), __byte_perm(b[5], b[7], 0x0040), 0x5410);
    return (even & 0x0F0F0F0Fu) | ((odd << 4) & 0xF0F0F0F0u);
}

// pack8_bits for z-form codes: the same interleave from byte 2 of each.
__device__ __forceinline__ uint32_t pack8_zcodes(const uint32_t (&z)[kChunk])
{
    const uint32_t even = __byte_perm(__byte_perm(z[0], z[2], 0x0062), __byte_perm(z[4], z[6], 0x0062), 0x5410);
    const uint32_t odd = __byte_perm(__byte_perm(z[1], z[3], 0x0062), __byte_perm(z[5], z[7], 0x0062), 0x5410);
    return (even & 0x0F0F0F0Fu) | ((odd << 4) & 0xF0F0F0F0u);
}

// ---- restoring codes --------------------------------------------------------
// A packed word holds 8 two's-complement nibbles. Flipping bit 3 of each
// nibble turns q in [-8, 7] into q + 8 in [0, 15]; placing that byte in the
// low byte of kRoundBits gives the binary32 kRound + q + 8, so subtracting
// kRound + 8 yields q exactly.
struct Unpacked {
    uint32_t even; // bytes j: q_{2j} + 8
    uint32_t odd;  // bytes j: q_{2j+1} + 8
};

__device__ __forceinline__ Unpacked unpack8(uint32_t w)
{
    return Unpacked{(w & 0x0F0F0F0Fu) ^ 0x08080808u, ((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u};
}

// Code of element k (0..7) as a float; k is a constant after unrolling.
__device__ __forceinline__ float code_at(const Unpacked &u, int k)
{
    const uint32_t src = (k & 1) ? u.odd : u.even;
    const uint32_t bits = __byte_perm(src, kRoundBits, 0x7650 + (k >> 1));
    return __fsub_rn(__uint_as_float(bits), kRoundPlus8);
}

// max(|a|, |b|, |c|): the three-input maximum of absolute values that sm_100
// adds to PTX (max.abs.f32 with three sources); exact, like every maximum.
__device__ __forceinline__ float max3_abs(float a, float b, float c)
{
    float r;
    asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Absolute maximum of one lane's 8 values (finite), as a tree.
__device__ __forceinline__ float absmax8(const float (&v)[kChunk])
{
    return fmaxf(max3_abs(v[0], v[1], v[2]), max3_abs(v[3], v[4], max3_abs(v[5], v[6], v[7])));
}

// The same over 16 values in two rows of 8 (8 three-input maxima).
__device__ __forceinline__ float absmax16(const float (&a)[kChunk], const float (&b)[kChunk])
{
    const float m0 = max3_abs(a[0], a[1], a[2]), m1 = max3_abs(a[3], a[4], a[5]), m2 = max3_abs(a[6], a[7], b[0]);
    const float m3 = max3_abs(b[1], b[2], b[3]), m4 = max3_abs(b[4], b[5], b[6]);
    return fmaxf(max3_abs(m0, m1, m2), max3_abs(m3, m4, b[7]));
}

// Codes of elements 2j and 2j+1 as a pair of floats, by one packed
// subtraction (sm_100's f32x2 forms round each component exactly as the
// scalar __fadd_rn, __fmul_rn and __fmaf_rn do); j is a constant after
// unrolling.
__device__ __forceinline__ float2 code_pair(const Unpacked &u, int j)
{
    const float a = __uint_as_float(__byte_perm(u.even, kRoundBits, 0x7650 + j));
    const float b = __uint_as_float(__byte_perm(u.odd, kRoundBits, 0x7650 + j));
    return __fadd2_rn(make_float2(a, b), make_float2(-kRoundPlus8, -kRoundPlus8));
}

// Absolute maximum over the 2^lanes_log2 consecutive lanes (8 elements each)
// that form a group. Every lane of the warp calls it with the same
// lanes_log2.
__device__ __forceinline__ float group_absmax(float a, uint32_t lanes_log2)
{
    for (uint32_t d = 1; d < (1u << lanes_log2); d <<= 1)
        a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, d));
    return a;
}

// bf16 <-> binary32: a bf16 is the upper half of a binary32.
__device__ __forceinline__ void bf16x8_to_f32(const uint4 &raw, float (&v)[kChunk])
{
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int j = 0; j < 4; j++) {
        v[2 * j] = __uint_as_float(w[j] << 16);
        v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
}

// Values q*2^e with |q| <= 7 have zero low halves, so keeping the upper
// halves (one prmt per pair) is exact.
__device__ __forceinline__ uint4 f32x8_to_bf16_exact(const float (&y)[kChunk])
{
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; j++)
        w[j] = __byte_perm(__float_as_uint(y[2 * j]), __float_as_uint(y[2 * j + 1]), 0x7632);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

} // namespace echo
