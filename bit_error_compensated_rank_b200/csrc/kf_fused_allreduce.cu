// kf_fused_allreduce.cu - the whole all-reduce in one launch, for small
// messages.
//
// Below a few MiB per call the three pipelined kernels cost mostly launch and
// pipeline latency. This kernel runs the same three steps in one cooperative
// launch, with a grid-wide barrier between them:
//   A. every rank's compensated partial is rounded to 4-bit codes and written
//      to the stage-1 wire (kernel 1's step);
//   B. each owner restores the P segments from the wire, sums them in
//      binary32 in rank order, rounds the total again, captures the error and
//      updates the two estimates (kernel 2's step);
//   C. every rank restores the requantised total from the wire (kernel 3's
//      step).
// The wire still goes through global memory, so the data flow is that of the
// pipelined kernels; every operation and its rounding is the same, so the
// results are bit for bit theirs (and the CPU oracle's). Plain 128-bit loads
// and stores replace the bulk copies: at these sizes the data sit in L2.
//
// Every variant of the pipelined path is supported (feedback variants, group
// sizes, binary16 scales); they are run-time flags here, since the kernel is
// bound by latency, not by instruction issue.
//
// The barrier is a counter and a generation word in device memory. Each
// CTA's thread 0 reads the generation, arrives on the counter, and waits
// (bounded by clock64) for the generation to move; the last CTA to arrive
// resets the counter and moves the generation. So the words return to their
// rest state after every barrier, and graph replays need no reset. A wait
// that runs out sets kStatusTimeoutFused; while that bit is set the kernel
// does nothing, until the host clears the status word (which also resets the
// barrier words). The launch is cooperative, so every CTA is resident.
#include "echo_bulk.cuh"
#include "echo_kernels.h"

#include <cuda_runtime.h>

namespace echo {
namespace {

constexpr int kThreads = 512;
constexpr int kCtasPerSm = 2; // few CTAs at the barrier, enough threads for one item each up to 2^21 elements

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(uint32_t *p, uint32_t v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Grid-wide barrier (see the file comment). Returns false, for every thread
// of the CTA, when the wait ran out. With `stall` (the ECHO_FAULT=stall test
// injection) the last CTA to arrive does not release the others: their waits
// run out, and it reports the same failure.
__device__ bool grid_barrier(uint32_t *bar, long long limit, bool stall, int *status)
{
    __shared__ int ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        ok = 1;
        const uint32_t gen = ld_acquire(bar + 1);
        __threadfence(); // this CTA's writes before its arrival
        const bool last = atomicAdd(bar, 1u) == gridDim.x - 1;
        if (last && !stall) {
            atomicExch(bar, 0u);
            __threadfence();
            st_release(bar + 1, gen + 1u);
        } else if (last) {
            atomicOr(status, kStatusTimeoutFused);
            ok = 0;
        } else {
            const long long t0 = clock64();
            while (ld_acquire(bar + 1) == gen) {
                if (clock64() - t0 > limit) {
                    atomicOr(status, kStatusTimeoutFused);
                    ok = 0;
                    break;
                }
            }
        }
    }
    __syncthreads();
    return ok != 0;
}

__device__ __forceinline__ void load8(const void *base, size_t chunk, bool bf16, float (&v)[kChunk])
{
    if (bf16) {
        bf16x8_to_f32(reinterpret_cast<const uint4 *>(base)[chunk], v);
    } else {
        const float4 a = reinterpret_cast<const float4 *>(base)[2 * chunk];
        const float4 b = reinterpret_cast<const float4 *>(base)[2 * chunk + 1];
        v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w;
        v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
    }
}

__device__ __forceinline__ void load8_f32(const float *base, size_t chunk, float (&v)[kChunk])
{
    const float4 a = reinterpret_cast<const float4 *>(base)[2 * chunk];
    const float4 b = reinterpret_cast<const float4 *>(base)[2 * chunk + 1];
    v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w;
    v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
}

// The same, through L2 only (data written by other CTAs in this launch).
__device__ __forceinline__ uint32_t ldcg_u32(const uint8_t *p, size_t word)
{
    return __ldcg(reinterpret_cast<const unsigned int *>(p) + word);
}

__device__ __forceinline__ void store8_f32(float *base, size_t chunk, const float (&v)[kChunk])
{
    reinterpret_cast<float4 *>(base)[2 * chunk] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4 *>(base)[2 * chunk + 1] = make_float4(v[4], v[5], v[6], v[7]);
}

// Scale of a group from its maximum in the launch's format, the step it
// restores with, and the 8 codes of one lane.
__device__ __forceinline__ uint32_t quantise8(const float (&v)[kChunk], float amax, bool f16, float &st,
                                              uint32_t (&qb)[kChunk])
{
    if (f16) {
        const uint32_t h = half_scale_bits(amax);
        st = half_step(h);
        const float inv = half_inv(st);
        const float half = __fmul_rn(0.5f, st);
        codes8_half(v, st, inv, half, half_scale_saturates(amax), qb);
        return h;
    }
    const uint32_t byte = scale_byte(amax);
    st = step_of(byte);
    const float inv = inv_step_of(byte);
#pragma unroll
    for (int k = 0; k < kChunk; k++)
        qb[k] = code_bits(v[k], inv);
    return byte;
}

__device__ __forceinline__ float absmax8(const float (&v)[kChunk])
{
    const float m01 = fmaxf(fabsf(v[0]), fabsf(v[1])), m23 = fmaxf(fabsf(v[2]), fabsf(v[3]));
    const float m45 = fmaxf(fabsf(v[4]), fabsf(v[5])), m67 = fmaxf(fabsf(v[6]), fabsf(v[7]));
    return fmaxf(fmaxf(m01, m23), fmaxf(m45, m67));
}

__device__ __forceinline__ float scale_at(const uint8_t *row, size_t g, bool f16, bool through_l2)
{
    if (f16) {
        const unsigned short *r16 = reinterpret_cast<const unsigned short *>(row);
        return half_step(through_l2 ? __ldcg(r16 + g) : r16[g]);
    }
    return step_of(through_l2 ? __ldcg(row + g) : row[g]);
}

__device__ __forceinline__ void store_scale(uint8_t *row, size_t g, bool f16, uint32_t scale)
{
    if (f16)
        reinterpret_cast<uint16_t *>(row)[g] = static_cast<uint16_t>(scale);
    else
        row[g] = static_cast<uint8_t>(scale);
}

__global__ void __launch_bounds__(kThreads) kf_fused_allreduce(const FusedArgs a)
{
    wait_for_predecessor(); // launched early (programmatic launch): wait for the previous call's writes
    allow_successor();
    if (__ldcg(a.ctl.status) & kStatusTimeoutFused)
        return; // an earlier launch lost its barrier: do nothing until the host clears the word
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp_first = blockIdx.x * kThreads + (threadIdx.x & ~31u); // first item of this warp
    const uint32_t stride = gridDim.x * kThreads;
    const uint32_t lanes_log2 = a.lanes_log2;
    const uint32_t nct = a.chunk_end - a.chunk_begin; // chunks in the range, per rank
    const size_t code_words = a.n / kChunk;
    const int P = a.P;
    const bool f16 = a.fp16_scale;
    const uint32_t first_lane_mask = (1u << lanes_log2) - 1u;

    // ---- A: compensate, round #1, pack (every rank) --------------------------
    const uint32_t items_a = static_cast<uint32_t>(P) * nct;
    for (uint32_t base = warp_first; base < items_a; base += stride) {
        const uint32_t i = base + lane;
        const bool active = i < items_a; // whole groups are active or not
        const uint32_t r = active ? i / nct : 0u;
        const uint32_t chunk = a.chunk_begin + (active ? i - r * nct : 0u);
        const uint32_t g = chunk >> lanes_log2;
        float v[kChunk] = {};
        if (active) {
            load8(a.x.p[r], chunk, a.bf16, v);
            if (a.sender_ef) {
                float e[kChunk];
                load8_f32(a.eps + static_cast<size_t>(r) * a.n, chunk, e);
#pragma unroll
                for (int k = 0; k < kChunk; k++)
                    v[k] = __fadd_rn(v[k], e[k]);
            }
            if (a.enable && !a.owner_sum && g - r * a.groups_per_seg < a.groups_per_seg) {
                float fv[kChunk], sv[kChunk];
                load8_f32(a.f, chunk, fv);
                load8_f32(a.s, chunk, sv);
#pragma unroll
                for (int k = 0; k < kChunk; k++)
                    v[k] = __fadd_rn(v[k], __fadd_rn(__fmul_rn(a.lambda, fv[k]), __fmul_rn(a.one_minus_lambda, sv[k])));
            }
        }
        const float amax = group_absmax(absmax8(v), lanes_log2);
        float st;
        uint32_t qb[kChunk];
        const uint32_t scale = quantise8(v, amax, f16, st, qb);
        if (active && in_bounds(chunk < code_words && (g + 1) * (f16 ? 2u : 1u) <= a.scale_stride, a.ctl.status)) {
            reinterpret_cast<uint32_t *>(a.codes1)[static_cast<size_t>(r) * code_words + chunk] = pack8_bits(qb);
            if ((lane & first_lane_mask) == 0)
                store_scale(a.scales1 + static_cast<size_t>(r) * a.scale_stride, g, f16, scale);
            if (a.sender_ef) {
                float e[kChunk];
#pragma unroll
                for (int k = 0; k < kChunk; k++)
                    e[k] = __fmaf_rn(-code_value(qb[k]), st, v[k]);
                store8_f32(a.eps + static_cast<size_t>(r) * a.n, chunk, e);
            }
        }
    }
    if (!grid_barrier(a.barrier, a.ctl.wait_cycles, a.ctl.stall, a.ctl.status))
        return;

    // ---- B: restore, sum in rank order, round #2, capture, update (owners) ---
    for (uint32_t base = warp_first; base < nct; base += stride) {
        const uint32_t i = base + lane;
        const bool active = i < nct;
        const uint32_t chunk = a.chunk_begin + (active ? i : 0u);
        const uint32_t g = chunk >> lanes_log2;
        float S_[kChunk] = {};
        float fv[kChunk] = {}, sv[kChunk] = {};
        if (active) {
            for (int r = 0; r < P; r++) {
                const uint32_t w = ldcg_u32(a.codes1, static_cast<size_t>(r) * code_words + chunk);
                const float st = scale_at(a.scales1 + static_cast<size_t>(r) * a.scale_stride, g, f16, true);
                const Unpacked u = unpack8(w);
#pragma unroll
                for (int k = 0; k < kChunk; k++)
                    S_[k] = __fmaf_rn(code_at(u, k), st, S_[k]);
            }
            if (a.enable) {
                load8_f32(a.f, chunk, fv);
                load8_f32(a.s, chunk, sv);
            }
            if (a.enable && a.owner_sum) {
#pragma unroll
                for (int k = 0; k < kChunk; k++)
                    S_[k] = __fadd_rn(S_[k], __fadd_rn(__fmul_rn(a.lambda, fv[k]), __fmul_rn(a.one_minus_lambda, sv[k])));
            }
        }
        const float amax = group_absmax(absmax8(S_), lanes_log2);
        float st;
        uint32_t qb[kChunk];
        const uint32_t scale = quantise8(S_, amax, f16, st, qb);
        float err[kChunk];
#pragma unroll
        for (int k = 0; k < kChunk; k++) {
            if (f16) {
                const float y = __fmul_rn(code_value(qb[k]), st); // exact
                err[k] = __fsub_rn(S_[k], a.bf16 ? round_bf16(y) : y);
            } else {
                err[k] = __fmaf_rn(-code_value(qb[k]), st, S_[k]); // exact
            }
        }
        if (active && in_bounds(chunk < code_words && (g + 1) * (f16 ? 2u : 1u) <= a.scale_stride, a.ctl.status)) {
            reinterpret_cast<uint32_t *>(a.qcodes)[chunk] = pack8_bits(qb);
            if ((lane & first_lane_mask) == 0)
                store_scale(a.qscales, g, f16, scale);
            if (a.enable) {
#pragma unroll
                for (int k = 0; k < kChunk; k++) {
                    fv[k] = __fadd_rn(__fmul_rn(a.beta_f, fv[k]), __fmul_rn(a.one_minus_beta_f, err[k]));
                    sv[k] = __fadd_rn(__fmul_rn(a.beta_s, sv[k]), __fmul_rn(a.one_minus_beta_s, err[k]));
                }
                store8_f32(a.f, chunk, fv);
                store8_f32(a.s, chunk, sv);
            }
        }
    }
    if (!grid_barrier(a.barrier, a.ctl.wait_cycles, a.ctl.stall, a.ctl.status))
        return;

    // ---- C: every rank restores the requantised total ------------------------
    for (uint32_t i = blockIdx.x * kThreads + threadIdx.x; i < nct; i += stride) {
        const uint32_t chunk = a.chunk_begin + i;
        if (!in_bounds(chunk < code_words, a.ctl.status))
            continue;
        const uint32_t w = ldcg_u32(a.qcodes, chunk);
        const float st = scale_at(a.qscales, chunk >> lanes_log2, f16, true);
        const Unpacked u = unpack8(w);
        float y[kChunk];
#pragma unroll
        for (int k = 0; k < kChunk; k++)
            y[k] = __fmul_rn(code_at(u, k), st);
        if (a.bf16) {
            uint4 word;
            if (f16) {
                uint32_t w2[4];
#pragma unroll
                for (int j = 0; j < 4; j++)
                    w2[j] = __float_as_uint(round_bf16(y[2 * j])) >> 16 |
                            (__float_as_uint(round_bf16(y[2 * j + 1])) & 0xFFFF0000u);
                word = make_uint4(w2[0], w2[1], w2[2], w2[3]);
            } else {
                word = f32x8_to_bf16_exact(y);
            }
            for (int r = 0; r < P; r++)
                reinterpret_cast<uint4 *>(a.out.p[r])[chunk] = word;
        } else {
            for (int r = 0; r < P; r++)
                store8_f32(static_cast<float *>(a.out.p[r]), chunk, y);
        }
    }
}

} // namespace

int fused_max_grid()
{
    static int grid = 0;
    if (grid == 0) {
        int per_sm = 0, dev = 0, sms = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kf_fused_allreduce, kThreads, 0) != cudaSuccess ||
            cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return 0;
        grid = (per_sm < kCtasPerSm ? per_sm : kCtasPerSm) * sms;
    }
    return grid;
}

cudaError_t launch_kf_fused_allreduce(const FusedArgs &a, cudaStream_t st)
{
    if (a.chunk_end <= a.chunk_begin)
        return cudaSuccess;
    const int max_grid = fused_max_grid();
    if (max_grid <= 0)
        return cudaErrorInvalidConfiguration;
    // enough CTAs for one item per thread in the widest step (A), at most
    // what the GPU holds at once (a cooperative launch needs every CTA resident)
    const size_t items = static_cast<size_t>(a.P) * (a.chunk_end - a.chunk_begin);
    const int grid = static_cast<int>(items / kThreads + 1 < static_cast<size_t>(max_grid) ? items / kThreads + 1
                                                                                             : static_cast<size_t>(max_grid));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    // cooperative (every CTA resident, for the barrier) and, where the driver
    // takes both, programmatic (launched while the previous call drains)
    static bool programmatic = true;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = programmatic ? 2 : 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kf_fused_allreduce, a);
    if (e != cudaSuccess && programmatic) {
        cudaGetLastError();
        programmatic = false;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kf_fused_allreduce, a);
    }
    return e;
}

} // namespace echo
