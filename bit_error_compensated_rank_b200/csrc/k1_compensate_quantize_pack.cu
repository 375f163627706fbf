// k1_compensate_quantize_pack.cu - kernel 1 of the Echo all-reduce.
//
// Every rank rounds its partial to 4-bit codes per group of 32 (rounding #1);
// on its own segment the owner first adds the correction
// c = lambda*f + (1-lambda)*s built from the two smoothed error estimates
// [rit.work "Echo 4-bit GPU communication", section "How Echo returns the
// error to later calls": the stored error is added back in later calls].
//
// Layout: the rank partials are P separate buffers of n elements; the output
// is the stage-1 wire, codes [P][n/2] (two per byte) and scale bytes
// [P][n/32]. A lane owns 8 consecutive elements (one 128-bit bf16 load, one
// 32-bit code word); 4 lanes form a group and find its maximum with two
// shuffles. One warp step covers 256 elements of every rank, so per step a
// warp issues P x 512 B of coalesced partial loads, 1 KB of state loads
// (compensation on) and P x 128 B of code stores.
//
// Algorithmic HBM bytes per element of n: P*b (partials) + 8 (f, s; each
// element is corrected by exactly one rank) read, P*17/32 written.
#include "echo_kernels.h"

#include <cuda_runtime.h>

namespace echo {
namespace {

constexpr int kThreads = 256;

template <bool BF16>
struct Raw;
template <>
struct Raw<true> {
    uint4 a;
};
template <>
struct Raw<false> {
    uint4 a, b;
};

// Partials are read once: stream them past L1 with an evict-first hint.
template <bool BF16>
__device__ __forceinline__ Raw<BF16> load_raw(const void *base, uint32_t chunk);
template <>
__device__ __forceinline__ Raw<true> load_raw<true>(const void *base, uint32_t chunk)
{
    return Raw<true>{__ldcs(reinterpret_cast<const uint4 *>(base) + chunk)};
}
template <>
__device__ __forceinline__ Raw<false> load_raw<false>(const void *base, uint32_t chunk)
{
    const uint4 *p = reinterpret_cast<const uint4 *>(base) + 2 * static_cast<size_t>(chunk);
    return Raw<false>{__ldcs(p), __ldcs(p + 1)};
}

__device__ __forceinline__ void to_f32(const Raw<true> &r, float (&v)[kChunk])
{
    bf16x8_to_f32(r.a, v);
}
__device__ __forceinline__ void to_f32(const Raw<false> &r, float (&v)[kChunk])
{
    v[0] = __uint_as_float(r.a.x);
    v[1] = __uint_as_float(r.a.y);
    v[2] = __uint_as_float(r.a.z);
    v[3] = __uint_as_float(r.a.w);
    v[4] = __uint_as_float(r.b.x);
    v[5] = __uint_as_float(r.b.y);
    v[6] = __uint_as_float(r.b.z);
    v[7] = __uint_as_float(r.b.w);
}

template <int P, bool BF16, bool COMP>
__global__ void __launch_bounds__(kThreads)
    k1_compensate_quantize_pack(const K1Args a)
{
    // Ranks whose partials are loaded together before any is processed: all
    // of them for bf16 (4 registers each), eight at a time for binary32.
    constexpr int kBatch = BF16 ? P : (P < 8 ? P : 8);
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = (blockIdx.x * kThreads + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * kThreads) >> 5;
    const uint32_t ntiles = (a.chunk_end - a.chunk_begin + 31u) >> 5;
    const size_t code_words = a.n / kChunk;   // 32-bit code words per rank
    const size_t scale_bytes = a.n / kGroup;  // scale bytes per rank

    for (uint32_t t = warp; t < ntiles; t += nwarps) {
        const uint32_t chunk = a.chunk_begin + t * 32u + lane;
        const bool active = chunk < a.chunk_end;
        const uint32_t g = chunk / kLanesPerGroup;

        float c[kChunk];
        uint32_t owner = 0xFFFFFFFFu;
        if (COMP) {
            owner = g / a.groups_per_seg;
            float4 f0 = make_float4(0.f, 0.f, 0.f, 0.f), f1 = f0, s0 = f0, s1 = f0;
            if (active) {
                const float4 *fp = reinterpret_cast<const float4 *>(a.f) + 2 * static_cast<size_t>(chunk);
                const float4 *sp = reinterpret_cast<const float4 *>(a.s) + 2 * static_cast<size_t>(chunk);
                f0 = fp[0];
                f1 = fp[1];
                s0 = sp[0];
                s1 = sp[1];
            }
            const float fv[kChunk] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
            const float sv[kChunk] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
            for (int k = 0; k < kChunk; k++)
                c[k] = __fadd_rn(__fmul_rn(a.lambda, fv[k]), __fmul_rn(a.one_minus_lambda, sv[k]));
        }

#pragma unroll
        for (int r0 = 0; r0 < P; r0 += kBatch) {
            Raw<BF16> raw[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; j++) {
                if (r0 + j < P) {
                    if (active)
                        raw[j] = load_raw<BF16>(a.x.p[r0 + j], chunk);
                    else
                        raw[j] = Raw<BF16>{};
                }
            }
#pragma unroll
            for (int j = 0; j < kBatch; j++) {
                const int r = r0 + j;
                if (r >= P)
                    continue;
                float v[kChunk];
                to_f32(raw[j], v);
                if (COMP && owner == static_cast<uint32_t>(r)) {
#pragma unroll
                    for (int k = 0; k < kChunk; k++)
                        v[k] = __fadd_rn(v[k], c[k]);
                }
                float amax = 0.f;
#pragma unroll
                for (int k = 0; k < kChunk; k++)
                    amax = fmaxf(amax, fabsf(v[k]));
                amax = group_absmax(amax);
                const uint32_t byte = scale_byte(amax);
                const float inv = inv_step_of(byte);
                int q[kChunk];
#pragma unroll
                for (int k = 0; k < kChunk; k++)
                    q[k] = code_of(v[k], inv);
                if (active) {
                    reinterpret_cast<uint32_t *>(a.codes)[static_cast<size_t>(r) * code_words + chunk] = pack8(q);
                    if ((lane & 3u) == 0)
                        a.scales[static_cast<size_t>(r) * scale_bytes + g] = static_cast<uint8_t>(byte);
                }
            }
        }
    }
}

template <int P, bool BF16, bool COMP>
cudaError_t launch_p(const K1Args &a, cudaStream_t st, int max_ctas)
{
    static int resident = 0;
    auto kern = k1_compensate_quantize_pack<P, BF16, COMP>;
    if (resident == 0) {
        int r = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&r, kern, kThreads, 0);
        if (e != cudaSuccess)
            return e;
        resident = r > 0 ? r : 1;
    }
    const uint32_t tiles = (a.chunk_end - a.chunk_begin + 31u) >> 5;
    const int grid = grid_for(tiles, resident, max_ctas);
    kern<<<grid, kThreads, 0, st>>>(a);
    return cudaGetLastError();
}

template <int P>
cudaError_t dispatch_flags(const K1Args &a, cudaStream_t st, int max_ctas)
{
    if (a.bf16)
        return a.enable ? launch_p<P, true, true>(a, st, max_ctas) : launch_p<P, true, false>(a, st, max_ctas);
    return a.enable ? launch_p<P, false, true>(a, st, max_ctas) : launch_p<P, false, false>(a, st, max_ctas);
}

} // namespace

cudaError_t launch_k1_compensate_quantize_pack(const K1Args &a, cudaStream_t st, int max_ctas)
{
    if (a.chunk_end <= a.chunk_begin)
        return cudaSuccess;
    switch (a.P) {
    case 2: return dispatch_flags<2>(a, st, max_ctas);
    case 3: return dispatch_flags<3>(a, st, max_ctas);
    case 4: return dispatch_flags<4>(a, st, max_ctas);
    case 5: return dispatch_flags<5>(a, st, max_ctas);
    case 6: return dispatch_flags<6>(a, st, max_ctas);
    case 7: return dispatch_flags<7>(a, st, max_ctas);
    case 8: return dispatch_flags<8>(a, st, max_ctas);
    case 9: return dispatch_flags<9>(a, st, max_ctas);
    case 10: return dispatch_flags<10>(a, st, max_ctas);
    case 11: return dispatch_flags<11>(a, st, max_ctas);
    case 12: return dispatch_flags<12>(a, st, max_ctas);
    case 13: return dispatch_flags<13>(a, st, max_ctas);
    case 14: return dispatch_flags<14>(a, st, max_ctas);
    case 15: return dispatch_flags<15>(a, st, max_ctas);
    case 16: return dispatch_flags<16>(a, st, max_ctas);
    default: return cudaErrorInvalidValue;
    }
}

} // namespace echo
