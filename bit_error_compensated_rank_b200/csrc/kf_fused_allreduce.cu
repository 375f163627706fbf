// kf_fused_allreduce.cu - the Echo all-reduce as one kernel, for small messages.
//
// Every step of the three pipelined kernels works on one group of G elements
// at a time [rit.work "Echo 4-bit GPU communication", section "How Echo
// returns the error to later calls"]:
//   - kernel 1 gives a rank's group its correction (owner) and its 4-bit codes;
//   - kernel 2 has the owner restore and add the P ranks' codes of the group,
//     round the total to 4 bits again and fold the error into the state;
//   - kernel 3 has every rank restore the group's requantised total.
// So one lane can take its chunk of 8 elements through all three steps, with
// no other CTA involved, and a call is one launch. Up to about 2 MiB per
// rank the three dependent launches, not the bytes, set the time of a call:
// there this kernel takes their place.
//
// It computes exactly what the three kernels compute, in the same operation
// order, and writes the same buffers: both wires (every rank's stage-1 codes
// and scales, the requantised total), the sender errors, the state and the P
// outputs. The owner's restore uses the codes the lane has just produced, not
// the wire bytes it wrote; on one GPU both hold the same codes. That shortcut
// needs every rank's partial on this GPU: ranks on separate GPUs (the
// per-rank entry points) must read the wire at the receiver, and keep the
// three stages.
//
// A warp takes 32 consecutive chunks (256 elements). Each lane first copies
// its P partial chunks (and its P sender errors) into its own slots in shared
// memory with cp.async and waits for them once. The P loads are then in flight
// together: plain loads could not be hoisted above the wire stores of the
// ranks before them, which the compiler must assume may alias. No lane reads
// another lane's slots; the kernel has no barrier and no spin-wait.
//
// HBM bytes per element of n: P*b partials + 8 state read, P*17/32 + 17/32
// wire + 8 state + P*b outputs written; sender feedback adds 4P read and 4P
// written. The stage-1 wire is not read back.
#include "echo_bulk.cuh"
#include "echo_kernels.h"

#include <cuda_runtime.h>

#include <atomic>

namespace echo {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;

// 16 bytes global -> shared, completed by cp_async_wait_all in the same thread.
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Shared memory of one warp: P partial chunks per lane, then P error chunks
// per lane with sender feedback.
__host__ __device__ constexpr uint32_t kf_warp_bytes(int P, bool bf16, bool ef)
{
    return static_cast<uint32_t>(P) * 32u * (bf16 ? 16u : 32u) + (ef ? static_cast<uint32_t>(P) * 32u * 32u : 0u);
}

__device__ __forceinline__ void load8(const float *p, float (&v)[kChunk])
{
    const float4 a = reinterpret_cast<const float4 *>(p)[0];
    const float4 b = reinterpret_cast<const float4 *>(p)[1];
    v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w;
    v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
}

__device__ __forceinline__ void store8(float *p, const float (&v)[kChunk])
{
    reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// Rounded bit patterns kRoundBits + q of the codes of v under its group's
// scale, as kernel 1 and kernel 2 compute them; returns the scale (byte or
// binary16 pattern) and its step.
template <bool F16>
__device__ __forceinline__ uint32_t quantise8(const float (&v)[kChunk], float amax, bool short_vals,
                                              uint32_t (&qb)[kChunk], float &st)
{
    if (F16) {
        const uint32_t scale = half_scale_bits(amax);
        st = half_step(scale);
        codes8_half(v, st, half_inv(st), __fmul_rn(0.5f, st), half_scale_saturates(amax), short_vals, qb);
#pragma unroll
        for (int k = 0; k < kChunk; k++)
            qb[k] = zcode_bits(qb[k]);
        return scale;
    }
    const uint32_t scale = scale_byte(amax);
    st = step_of(scale);
    const float inv = inv_step_of(scale);
#pragma unroll
    for (int k = 0; k < kChunk; k++)
        qb[k] = code_bits(v[k], inv);
    return scale;
}

template <int P, bool BF16, bool F16>
__global__ void __launch_bounds__(kThreads) kf_fused_allreduce(const KFArgs a)
{
    constexpr uint32_t kEB = BF16 ? 2u : 4u;
    constexpr uint32_t kXB = kChunk * kEB; // bytes of one partial chunk
    extern __shared__ __align__(128) uint8_t smem[];
    wait_for_predecessor(); // nothing above touches global memory
    allow_successor();

    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = threadIdx.x >> 5;
    const bool ef = a.sender_ef;
    uint8_t *wbase = smem + warp * kf_warp_bytes(P, BF16, ef);
    uint8_t *xs = wbase + lane * kXB;                   // rank r's chunk at xs + r * 32 * kXB
    float *es = reinterpret_cast<float *>(wbase + P * 32u * kXB) + lane * kChunk; // at es + r * 256
    const uint32_t lanes_log2 = a.lanes_log2;
    const uint32_t code_words = static_cast<uint32_t>(a.n / kChunk);
    const uint32_t items = (a.chunk_end - a.chunk_begin + 31u) >> 5;
    const bool comp = a.enable && !a.owner_sum; // the owner corrects its partial
    const bool first = (lane & ((1u << lanes_log2) - 1u)) == 0; // the group's first lane

    for (uint32_t item = blockIdx.x * kWarps + warp; item < items; item += gridDim.x * kWarps) {
        const uint32_t chunk = a.chunk_begin + (item << 5) + lane;
        const uint32_t g = chunk >> lanes_log2;
        const size_t e = static_cast<size_t>(chunk) * kChunk;
        // Groups lie wholly inside or outside the range, so the lanes past its
        // end only feed shuffles of their own groups; they load and store nothing.
        const bool ok = chunk < a.chunk_end &&
                        in_bounds(chunk < code_words && (g + 1) * (F16 ? 2u : 1u) <= a.scale_stride, a.ctl.status);
        if (ok) {
#pragma unroll
            for (int r = 0; r < P; r++) {
                const uint8_t *src = static_cast<const uint8_t *>(a.x.p[r]) + e * kEB;
#pragma unroll
                for (uint32_t h = 0; h < kXB; h += 16)
                    cp_async16(xs + r * 32u * kXB + h, src + h);
                if (ef) {
                    cp_async16(es + r * 256, a.eps + static_cast<size_t>(r) * a.n + e);
                    cp_async16(es + r * 256 + 4, a.eps + static_cast<size_t>(r) * a.n + e + 4);
                }
            }
        }
        float fv[kChunk], sv[kChunk];
        if (a.enable && ok) {
            load8(a.f + e, fv);
            load8(a.s + e, sv);
        } else {
#pragma unroll
            for (int k = 0; k < kChunk; k++)
                fv[k] = sv[k] = 0.f;
        }
        cp_async_wait_all();

        // Kernel 1 for each rank, and kernel 2's restore-and-add, rank 0 first.
        float S_[kChunk];
#pragma unroll
        for (int k = 0; k < kChunk; k++)
            S_[k] = 0.f;
#pragma unroll
        for (int r = 0; r < P; r++) {
            float v[kChunk];
            if (BF16)
                bf16x8_to_f32(*reinterpret_cast<const uint4 *>(xs + r * 32u * kXB), v);
            else
                load8(reinterpret_cast<const float *>(xs + r * 32u * kXB), v);
            bool short_vals = BF16 && !ef; // bf16 partials keep 8 significant bits unless something is added
            if (ef) {
                float ev[kChunk];
                load8(es + r * 256, ev);
#pragma unroll
                for (int k = 0; k < kChunk; k++)
                    v[k] = __fadd_rn(v[k], ev[k]);
            }
            if (comp && g / a.groups_per_seg == static_cast<uint32_t>(r)) {
                short_vals = false;
#pragma unroll
                for (int k = 0; k < kChunk; k++)
                    v[k] = __fadd_rn(v[k], __fadd_rn(__fmul_rn(a.lambda, fv[k]), __fmul_rn(a.one_minus_lambda, sv[k])));
            }
            uint32_t qb[kChunk];
            float st;
            const uint32_t scale = quantise8<F16>(v, group_absmax(absmax8(v), lanes_log2), short_vals, qb, st);
            if (ok) {
                reinterpret_cast<uint32_t *>(a.codes)[static_cast<size_t>(r) * code_words + chunk] = pack8_bits(qb);
                if (first) {
                    uint8_t *row = a.scales + static_cast<size_t>(r) * a.scale_stride;
                    if (F16)
                        reinterpret_cast<uint16_t *>(row)[g] = static_cast<uint16_t>(scale);
                    else
                        row[g] = static_cast<uint8_t>(scale);
                }
            }
            if (ef && ok) { // the new error v - q*step (exact unless a binary16 scale saturated)
                float en[kChunk];
#pragma unroll
                for (int k = 0; k < kChunk; k++)
                    en[k] = __fmaf_rn(-code_value(qb[k]), st, v[k]);
                store8(a.eps + static_cast<size_t>(r) * a.n + e, en);
            }
            // q*step is exact, so fma(q, step, S) = RN(S + q*step)
#pragma unroll
            for (int k = 0; k < kChunk; k++)
                S_[k] = __fmaf_rn(code_value(qb[k]), st, S_[k]);
        }
        if (a.enable && a.owner_sum) { // variant: the correction enters the owner's sum
#pragma unroll
            for (int k = 0; k < kChunk; k++)
                S_[k] = __fadd_rn(S_[k], __fadd_rn(__fmul_rn(a.lambda, fv[k]), __fmul_rn(a.one_minus_lambda, sv[k])));
        }

        // Kernel 2: rounding #2, the error it injects, the estimates.
        uint32_t qb[kChunk];
        float st;
        const uint32_t scale = quantise8<F16>(S_, group_absmax(absmax8(S_), lanes_log2), false, qb, st);
        float y[kChunk]; // the value every rank receives, before its bf16 rounding
#pragma unroll
        for (int k = 0; k < kChunk; k++)
            y[k] = __fmul_rn(code_value(qb[k]), st); // exact
        if (ok) {
            reinterpret_cast<uint32_t *>(a.qcodes)[chunk] = pack8_bits(qb);
            if (first) {
                if (F16)
                    reinterpret_cast<uint16_t *>(a.qscales)[g] = static_cast<uint16_t>(scale);
                else
                    a.qscales[g] = static_cast<uint8_t>(scale);
            }
            if (a.enable) {
#pragma unroll
                for (int k = 0; k < kChunk; k++) {
                    // err = S - Y, exact; under binary16 scales with bf16 outputs
                    // Y is the bf16 value the ranks receive
                    const float err = F16 ? __fsub_rn(S_[k], a.bf16 ? round_bf16(y[k]) : y[k])
                                          : __fmaf_rn(-code_value(qb[k]), st, S_[k]);
                    fv[k] = __fadd_rn(__fmul_rn(a.beta_f, fv[k]), __fmul_rn(a.one_minus_beta_f, err));
                    sv[k] = __fadd_rn(__fmul_rn(a.beta_s, sv[k]), __fmul_rn(a.one_minus_beta_s, err));
                }
                store8(a.f + e, fv);
                store8(a.s + e, sv);
            }

            // Kernel 3: every rank's output.
            if (BF16) {
                uint4 w;
                if (F16) { // round to the nearest bf16
                    uint32_t h[4];
#pragma unroll
                    for (int j = 0; j < 4; j++)
                        h[j] = __float_as_uint(round_bf16(y[2 * j])) >> 16 |
                               (__float_as_uint(round_bf16(y[2 * j + 1])) & 0xFFFF0000u);
                    w = make_uint4(h[0], h[1], h[2], h[3]);
                } else {
                    w = f32x8_to_bf16_exact(y);
                }
#pragma unroll
                for (int p = 0; p < P; p++)
                    reinterpret_cast<uint4 *>(a.out.p[p])[chunk] = w;
            } else {
#pragma unroll
                for (int p = 0; p < P; p++)
                    store8(static_cast<float *>(a.out.p[p]) + e, y);
            }
        }
    }
}

template <int P, bool BF16, bool F16>
cudaError_t launch_p(const KFArgs &a, cudaStream_t st)
{
    // The shared-memory limit of this instantiation is set once, for its
    // largest use (sender feedback); its CTAs per SM are found once for each
    // of its two shared-memory sizes. Threads that race here compute the
    // same values.
    static std::atomic<int> cached[2] = {{0}, {0}};
    auto kern = kf_fused_allreduce<P, BF16, F16>;
    const int ef = a.sender_ef ? 1 : 0;
    const int smem = static_cast<int>(kWarps * kf_warp_bytes(P, BF16, ef != 0));
    int resident = cached[ef].load(std::memory_order_relaxed);
    if (resident == 0) {
        int unused = 0;
        cudaError_t e = prepare_kernel(reinterpret_cast<const void *>(kern), kThreads,
                                       kWarps * kf_warp_bytes(P, BF16, true), &unused);
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, reinterpret_cast<const void *>(kern),
                                                              kThreads, smem);
        if (e != cudaSuccess)
            return e;
        resident = resident > 0 ? resident : 1;
        cached[ef].store(resident, std::memory_order_relaxed);
    }
    const uint32_t items = (a.chunk_end - a.chunk_begin + 31u) >> 5;
    const int grid = persistent_grid((items + kWarps - 1) / kWarps, resident);
    return launch_chained(kern, grid, kThreads, smem, st, a);
}

template <int P>
cudaError_t dispatch_types(const KFArgs &a, cudaStream_t st)
{
    if (a.bf16)
        return a.fp16_scale ? launch_p<P, true, true>(a, st) : launch_p<P, true, false>(a, st);
    return a.fp16_scale ? launch_p<P, false, true>(a, st) : launch_p<P, false, false>(a, st);
}

} // namespace

cudaError_t launch_kf_fused_allreduce(const KFArgs &a, cudaStream_t st)
{
    if (a.chunk_end <= a.chunk_begin)
        return cudaSuccess;
    switch (a.P) {
    case 2: return dispatch_types<2>(a, st);
    case 3: return dispatch_types<3>(a, st);
    case 4: return dispatch_types<4>(a, st);
    case 5: return dispatch_types<5>(a, st);
    case 6: return dispatch_types<6>(a, st);
    case 7: return dispatch_types<7>(a, st);
    case 8: return dispatch_types<8>(a, st);
    case 9: return dispatch_types<9>(a, st);
    case 10: return dispatch_types<10>(a, st);
    case 11: return dispatch_types<11>(a, st);
    case 12: return dispatch_types<12>(a, st);
    case 13: return dispatch_types<13>(a, st);
    case 14: return dispatch_types<14>(a, st);
    case 15: return dispatch_types<15>(a, st);
    case 16: return dispatch_types<16>(a, st);
    default: return cudaErrorInvalidValue;
    }
}

} // namespace echo
