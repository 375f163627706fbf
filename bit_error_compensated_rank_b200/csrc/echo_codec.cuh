// echo_codec.cuh - device-side 4-bit codec of the Echo all-reduce.
//
// Format (fixed readings of the 4-bit segments on [rit.work "Echo 4-bit GPU
// communication", section "How Echo returns the error to later calls"]):
// groups of 32 consecutive elements share a power-of-two scale 2^e, stored
// as the byte e+127, e the smallest integer >= -127 with max|v| <= 7*2^e;
// codes are round(v/2^e), halves to even, in [-7, 7]; two codes per byte,
// element 2j in the low nibble, two's complement.
//
// Every helper here is exact integer or power-of-two arithmetic; the only
// rounding is the conversion to the nearest code (cvt.rni), which rounds
// halves to even.
#pragma once

#include <cstdint>

namespace echo {

constexpr int kGroup = 32;          // elements per scale
constexpr int kChunk = 8;           // elements per thread (one 32-bit code word)
constexpr int kLanesPerGroup = kGroup / kChunk;
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

// Nearest code of v at scale 1/inv (v*inv is exact whenever it is normal; a
// subnormal product is below 1/2 and rounds to 0 either way).
__device__ __forceinline__ int code_of(float v, float inv)
{
    int q = __float2int_rn(__fmul_rn(v, inv));
    q = q > 7 ? 7 : q;
    return q < -7 ? -7 : q;
}

// Pack 8 codes (element k in nibble k) into one word.
__device__ __forceinline__ uint32_t pack8(const int (&q)[kChunk])
{
    uint32_t w = 0;
#pragma unroll
    for (int k = 0; k < kChunk; k++)
        w |= (static_cast<uint32_t>(q[k]) & 0xFu) << (4 * k);
    return w;
}

// Signed code in nibble k of w.
__device__ __forceinline__ int nibble(uint32_t w, int k)
{
    return static_cast<int>(w << (28 - 4 * k)) >> 28;
}

// Absolute maximum over the 4 lanes (32 elements) of a group. The lanes of a
// group are 4 consecutive lanes of the warp; every lane of the warp calls it.
__device__ __forceinline__ float group_absmax(float a)
{
    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 2));
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

// Values q*2^e with |q| <= 7 have zero low halves, so truncation is exact.
__device__ __forceinline__ uint4 f32x8_to_bf16_exact(const float (&y)[kChunk])
{
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; j++)
        w[j] = (__float_as_uint(y[2 * j]) >> 16) | (__float_as_uint(y[2 * j + 1]) & 0xFFFF0000u);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

} // namespace echo
