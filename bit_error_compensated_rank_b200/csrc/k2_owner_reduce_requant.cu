// k2_owner_reduce_requant.cu - kernel 2 of the Echo all-reduce.
//
// Each segment owner restores the P incoming 4-bit segments, adds them in
// binary32 in the fixed order rank 0, 1, ..., P-1, rounds the total to 4 bits
// again (rounding #2), measures the error that rounding injected from the
// high-precision total, err = S - Y, and folds it into the phase's fast and
// slow estimates [rit.work "Echo 4-bit GPU communication", section "How Echo
// returns the error to later calls": segments restored and added with high
// precision at the owner, the rounding error computed from that sum, kept in
// two smoothed estimates, separately for forward and backward].
//
// Every restored value q*2^e is exact, so the only roundings are the P-1
// binary32 additions, rounding #2, and the two estimates' products and sums
// (each rounded on its own: __fmul_rn / __fadd_rn are never contracted).
// err is exact: S and Y = Q*2^E differ by at most 2^(E-1) and both are
// multiples of ulp(S).
//
// On one GPU the P owners' segments are contiguous slices of one index
// space, so a launch simply covers the whole of it: lane = 8 elements, warp
// step = 256 elements. Per element of n it reads P*17/32 bytes of wire and
// 8 bytes of state, and writes 17/32 bytes of wire and 8 bytes of state.
#include "echo_kernels.h"

#include <cuda_runtime.h>

namespace echo {
namespace {

constexpr int kThreads = 256;

template <int P, bool COMP>
__global__ void __launch_bounds__(kThreads)
    k2_owner_reduce_requant(const K2Args a)
{
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = (blockIdx.x * kThreads + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * kThreads) >> 5;
    const uint32_t ntiles = (a.chunk_end - a.chunk_begin + 31u) >> 5;
    const size_t code_words = a.n / kChunk;
    const size_t scale_bytes = a.n / kGroup;
    const uint32_t *codes = reinterpret_cast<const uint32_t *>(a.codes);

    for (uint32_t t = warp; t < ntiles; t += nwarps) {
        const uint32_t chunk = a.chunk_begin + t * 32u + lane;
        const bool active = chunk < a.chunk_end;
        const uint32_t g = chunk / kLanesPerGroup;

        uint32_t w[P];
        uint32_t b[P];
#pragma unroll
        for (int r = 0; r < P; r++) {
            w[r] = active ? __ldcs(codes + static_cast<size_t>(r) * code_words + chunk) : 0u;
            b[r] = active ? static_cast<uint32_t>(__ldcs(a.scales + static_cast<size_t>(r) * scale_bytes + g)) : 0u;
        }
        float4 f0 = make_float4(0.f, 0.f, 0.f, 0.f), f1 = f0, s0 = f0, s1 = f0;
        float4 *fp = reinterpret_cast<float4 *>(a.f) + 2 * static_cast<size_t>(chunk);
        float4 *sp = reinterpret_cast<float4 *>(a.s) + 2 * static_cast<size_t>(chunk);
        if (COMP && active) {
            f0 = fp[0];
            f1 = fp[1];
            s0 = sp[0];
            s1 = sp[1];
        }

        // Restore and add, rank 0 first.
        float S[kChunk];
#pragma unroll
        for (int k = 0; k < kChunk; k++)
            S[k] = 0.f;
#pragma unroll
        for (int r = 0; r < P; r++) {
            const float st = step_of(b[r]);
#pragma unroll
            for (int k = 0; k < kChunk; k++)
                S[k] = __fadd_rn(S[k], __fmul_rn(static_cast<float>(nibble(w[r], k)), st));
        }

        // Rounding #2.
        float amax = 0.f;
#pragma unroll
        for (int k = 0; k < kChunk; k++)
            amax = fmaxf(amax, fabsf(S[k]));
        amax = group_absmax(amax);
        const uint32_t byte = scale_byte(amax);
        const float inv = inv_step_of(byte);
        const float st = step_of(byte);
        int q[kChunk];
        float err[kChunk];
#pragma unroll
        for (int k = 0; k < kChunk; k++) {
            q[k] = code_of(S[k], inv);
            err[k] = __fsub_rn(S[k], __fmul_rn(static_cast<float>(q[k]), st));
        }

        if (!active)
            continue;
        reinterpret_cast<uint32_t *>(a.qcodes)[chunk] = pack8(q);
        if ((lane & 3u) == 0)
            a.qscales[g] = static_cast<uint8_t>(byte);

        if (COMP) {
            float fv[kChunk] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
            float sv[kChunk] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
            for (int k = 0; k < kChunk; k++) {
                fv[k] = __fadd_rn(__fmul_rn(a.beta_f, fv[k]), __fmul_rn(a.one_minus_beta_f, err[k]));
                sv[k] = __fadd_rn(__fmul_rn(a.beta_s, sv[k]), __fmul_rn(a.one_minus_beta_s, err[k]));
            }
            fp[0] = make_float4(fv[0], fv[1], fv[2], fv[3]);
            fp[1] = make_float4(fv[4], fv[5], fv[6], fv[7]);
            sp[0] = make_float4(sv[0], sv[1], sv[2], sv[3]);
            sp[1] = make_float4(sv[4], sv[5], sv[6], sv[7]);
        }
    }
}

template <int P, bool COMP>
cudaError_t launch_p(const K2Args &a, cudaStream_t st, int max_ctas)
{
    static int resident = 0;
    auto kern = k2_owner_reduce_requant<P, COMP>;
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
cudaError_t dispatch_flags(const K2Args &a, cudaStream_t st, int max_ctas)
{
    return a.enable ? launch_p<P, true>(a, st, max_ctas) : launch_p<P, false>(a, st, max_ctas);
}

} // namespace

cudaError_t launch_k2_owner_reduce_requant(const K2Args &a, cudaStream_t st, int max_ctas)
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
