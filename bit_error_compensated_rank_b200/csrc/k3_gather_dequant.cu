// k3_gather_dequant.cu - kernel 3 of the Echo all-reduce.
//
// Every rank receives the owner's requantised total and restores it
// [rit.work "Echo 4-bit GPU communication", section "How Echo returns the
// error to later calls": the compressed total is sent back to every rank].
// Y = Q*2^E has at most three significant bits, so it is exact in bf16 and
// in binary32: the restore adds no third rounding.
//
// On one GPU all P ranks read the same requantised buffer; a lane restores
// 8 elements once (one 32-bit code word and one scale byte) and writes them
// to all P rank outputs (one 128-bit store per rank for bf16). Per element
// of n the kernel writes P*b bytes; the requantised wire (17/32 bytes) is
// read from HBM once and reused from registers for the P ranks.
#include "echo_kernels.h"

#include <cuda_runtime.h>

namespace echo {
namespace {

constexpr int kThreads = 256;

template <int P, bool BF16>
__global__ void __launch_bounds__(kThreads)
    k3_gather_dequant(const K3Args a)
{
    const uint32_t stride = gridDim.x * kThreads;
    const uint32_t *qcodes = reinterpret_cast<const uint32_t *>(a.qcodes);
    for (uint32_t chunk = a.chunk_begin + blockIdx.x * kThreads + threadIdx.x; chunk < a.chunk_end;
         chunk += stride) {
        const uint32_t w = __ldcs(qcodes + chunk);
        const float st = step_of(static_cast<uint32_t>(__ldcs(a.qscales + chunk / kLanesPerGroup)));
        float y[kChunk];
#pragma unroll
        for (int k = 0; k < kChunk; k++)
            y[k] = __fmul_rn(static_cast<float>(nibble(w, k)), st);
        if (BF16) {
            const uint4 o = f32x8_to_bf16_exact(y);
#pragma unroll
            for (int r = 0; r < P; r++)
                __stcs(reinterpret_cast<uint4 *>(a.out.p[r]) + chunk, o);
        } else {
            const float4 o0 = make_float4(y[0], y[1], y[2], y[3]);
            const float4 o1 = make_float4(y[4], y[5], y[6], y[7]);
#pragma unroll
            for (int r = 0; r < P; r++) {
                float4 *dst = reinterpret_cast<float4 *>(a.out.p[r]) + 2 * static_cast<size_t>(chunk);
                __stcs(dst, o0);
                __stcs(dst + 1, o1);
            }
        }
    }
}

template <int P, bool BF16>
cudaError_t launch_p(const K3Args &a, cudaStream_t st, int max_ctas)
{
    static int resident = 0;
    auto kern = k3_gather_dequant<P, BF16>;
    if (resident == 0) {
        int r = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&r, kern, kThreads, 0);
        if (e != cudaSuccess)
            return e;
        resident = r > 0 ? r : 1;
    }
    const uint32_t tiles = (a.chunk_end - a.chunk_begin + 31u) >> 5;
    kern<<<grid_for(tiles, resident, max_ctas), kThreads, 0, st>>>(a);
    return cudaGetLastError();
}

template <int P>
cudaError_t dispatch_flags(const K3Args &a, cudaStream_t st, int max_ctas)
{
    return a.bf16 ? launch_p<P, true>(a, st, max_ctas) : launch_p<P, false>(a, st, max_ctas);
}

} // namespace

cudaError_t launch_k3_gather_dequant(const K3Args &a, cudaStream_t st, int max_ctas)
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
