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
// [P][scale_stride].
//
// Pipeline (warp-specialised, persistent): a CTA takes tiles of kTile
// consecutive elements. One producer warp bulk-copies the P partial tiles and
// the f, s tiles of a tile into one stage of a kStages ring in shared memory
// (mbarrier full[s] counts the bytes); eight consumer warps compute from
// shared memory and release the stage on mbarrier empty[s]. A lane owns 8
// consecutive elements of one rank; 4 lanes form a group and find its
// maximum with two shuffles; codes leave as one coalesced 32-bit store per
// lane.
//
// Algorithmic HBM bytes per element of n: P*b (partials) + 8 (f, s; each
// element is corrected by exactly one rank) read, P*17/32 written.
#include "echo_bulk.cuh"
#include "echo_kernels.h"

#include <cuda_runtime.h>

namespace echo {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32; // + one producer warp

template <int P, bool BF16, bool COMP>
struct K1Shape {
    static constexpr int kEB = BF16 ? 2 : 4;
    // Tile length keeps one stage near 12-24 KB whatever P and the dtype.
    static constexpr int kTile = (P * kEB <= 16) ? ECHO_K1_TILE : (P * kEB <= 32 ? ECHO_K1_TILE / 2 : ECHO_K1_TILE / 4);
    static constexpr int kStages = ECHO_K1_STAGES;
    static constexpr int kXBytes = kTile * kEB; // one rank's partial tile
    static constexpr int kStageBytes = P * kXBytes + (COMP ? 2 * kTile * 4 : 0);
    static constexpr int kSmem = kStages * kStageBytes + 2 * kStages * 8;
    static_assert(kSmem <= ECHO_SMEM_BUDGET, "kernel 1 stages exceed shared memory");
    static constexpr int kChunksPerTile = kTile / kChunk; // a multiple of 32
};

template <bool BF16>
__device__ __forceinline__ void load_chunk(const uint8_t *p, float (&v)[kChunk])
{
    if (BF16) {
        bf16x8_to_f32(*reinterpret_cast<const uint4 *>(p), v);
    } else {
        const float4 a = reinterpret_cast<const float4 *>(p)[0];
        const float4 b = reinterpret_cast<const float4 *>(p)[1];
        v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w;
        v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
    }
}

template <int P, bool BF16, bool COMP>
__global__ void __launch_bounds__(kThreads)
    k1_compensate_quantize_pack(const K1Args a)
{
    using Sh = K1Shape<P, BF16, COMP>;
    constexpr int S = Sh::kStages;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + S * Sh::kStageBytes);
    uint64_t *empty = full + S;

    const uint32_t tid = threadIdx.x;
    const uint32_t warp = tid >> 5;
    const uint32_t lane = tid & 31u;
    const size_t e0 = static_cast<size_t>(a.chunk_begin) * kChunk;
    const size_t e1 = static_cast<size_t>(a.chunk_end) * kChunk;
    const uint32_t ntiles = static_cast<uint32_t>((e1 - e0 + Sh::kTile - 1) / Sh::kTile);
    const uint32_t mine = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (tid == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        mbar_init_fence();
    }
    __syncthreads();

    if (warp == kConsumerWarps) { // producer
        if (lane == 0)
            produce_tiles<S>(full, empty, mine, a.ctl.stall, a.ctl.wait_cycles, a.ctl.status, kStatusTimeoutK1,
                             [&](uint32_t i) {
                                 const size_t el0 = e0 + static_cast<size_t>(blockIdx.x + i * gridDim.x) * Sh::kTile;
                                 const uint32_t cnt = static_cast<uint32_t>(
                                     e1 - el0 < size_t(Sh::kTile) ? e1 - el0 : Sh::kTile);
                                 uint8_t *stage = smem + (i % S) * Sh::kStageBytes;
                                 uint64_t *bar = &full[i % S];
                                 mbar_arrive_expect_tx(bar, P * cnt * Sh::kEB + (COMP ? 2 * cnt * 4 : 0));
#pragma unroll
                                 for (int r = 0; r < P; r++)
                                     bulk_load(stage + r * Sh::kXBytes,
                                               static_cast<const uint8_t *>(a.x.p[r]) + el0 * Sh::kEB,
                                               cnt * Sh::kEB, bar);
                                 if (COMP) {
                                     bulk_load(stage + P * Sh::kXBytes, a.f + el0, cnt * 4, bar);
                                     bulk_load(stage + P * Sh::kXBytes + Sh::kTile * 4, a.s + el0, cnt * 4, bar);
                                 }
                             });
        return;
    }

    const uint32_t code_words = static_cast<uint32_t>(a.n / kChunk); // 32-bit code words per rank
    for (uint32_t i = 0; i < mine; i++) {
        const uint32_t s = i % S;
        if (!warp_wait(&full[s], (i / S) & 1u, a.ctl.wait_cycles, a.ctl.status, kStatusTimeoutK1))
            return;
        const uint32_t tile_chunk0 = static_cast<uint32_t>(e0 / kChunk) + (blockIdx.x + i * gridDim.x) * (Sh::kTile / kChunk);
        const uint32_t cnt_chunks = min(static_cast<uint32_t>(Sh::kChunksPerTile), a.chunk_end - tile_chunk0);
        const uint8_t *stage = smem + s * Sh::kStageBytes;
        const float *fs = reinterpret_cast<const float *>(stage + P * Sh::kXBytes);

#pragma unroll 2
        for (uint32_t it = tid; it < static_cast<uint32_t>(P * Sh::kChunksPerTile); it += kConsumers) {
            const uint32_t r = it / Sh::kChunksPerTile; // warp-uniform
            const uint32_t c = it % Sh::kChunksPerTile;
            const bool active = c < cnt_chunks;
            const uint32_t chunk = tile_chunk0 + c;
            const uint32_t g = chunk / kLanesPerGroup;

            float v[kChunk];
            load_chunk<BF16>(stage + r * Sh::kXBytes + c * (kChunk * Sh::kEB), v);
            // rank r owns groups [r*gps, (r+1)*gps): one unsigned range test
            if (COMP && g - r * a.groups_per_seg < a.groups_per_seg) {
                const float4 f0 = reinterpret_cast<const float4 *>(fs)[2 * c];
                const float4 f1 = reinterpret_cast<const float4 *>(fs)[2 * c + 1];
                const float4 s0 = reinterpret_cast<const float4 *>(fs + Sh::kTile)[2 * c];
                const float4 s1 = reinterpret_cast<const float4 *>(fs + Sh::kTile)[2 * c + 1];
                const float fv[kChunk] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
                const float sv[kChunk] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
                for (int k = 0; k < kChunk; k++)
                    v[k] = __fadd_rn(v[k], __fadd_rn(__fmul_rn(a.lambda, fv[k]),
                                                     __fmul_rn(a.one_minus_lambda, sv[k])));
            }
            // max |v| as a tree (fmax is exact, so the order is free)
            const float m01 = fmaxf(fabsf(v[0]), fabsf(v[1])), m23 = fmaxf(fabsf(v[2]), fabsf(v[3]));
            const float m45 = fmaxf(fabsf(v[4]), fabsf(v[5])), m67 = fmaxf(fabsf(v[6]), fabsf(v[7]));
            const float amax = group_absmax(fmaxf(fmaxf(m01, m23), fmaxf(m45, m67)));
            const uint32_t byte = scale_byte(amax);
            const float inv = inv_step_of(byte);
            uint32_t qb[kChunk];
#pragma unroll
            for (int k = 0; k < kChunk; k++)
                qb[k] = code_bits(v[k], inv);
            const uint32_t word = pack8_bits(qb);
            if (active) {
                reinterpret_cast<uint32_t *>(a.codes)[static_cast<size_t>(r) * code_words + chunk] = word;
                if ((lane & 3u) == 0)
                    a.scales[static_cast<size_t>(r) * a.scale_stride + g] = static_cast<uint8_t>(byte);
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[s]); // this warp is done reading stage s
    }
}

template <int P, bool BF16, bool COMP>
cudaError_t launch_p(const K1Args &a, cudaStream_t st)
{
    using Sh = K1Shape<P, BF16, COMP>;
    static int resident = 0;
    auto kern = k1_compensate_quantize_pack<P, BF16, COMP>;
    if (resident == 0) {
        cudaError_t e = prepare_kernel(reinterpret_cast<const void *>(kern), kThreads, Sh::kSmem, &resident);
        if (e != cudaSuccess)
            return e;
    }
    const size_t elems = static_cast<size_t>(a.chunk_end - a.chunk_begin) * kChunk;
    const uint32_t tiles = static_cast<uint32_t>((elems + Sh::kTile - 1) / Sh::kTile);
    kern<<<persistent_grid(tiles, resident), kThreads, Sh::kSmem, st>>>(a);
    return cudaGetLastError();
}

template <int P>
cudaError_t dispatch_flags(const K1Args &a, cudaStream_t st)
{
    if (a.bf16)
        return a.enable ? launch_p<P, true, true>(a, st) : launch_p<P, true, false>(a, st);
    return a.enable ? launch_p<P, false, true>(a, st) : launch_p<P, false, false>(a, st);
}

} // namespace

cudaError_t launch_k1_compensate_quantize_pack(const K1Args &a, cudaStream_t st)
{
    if (a.chunk_end <= a.chunk_begin)
        return cudaSuccess;
    switch (a.P) {
    case 2: return dispatch_flags<2>(a, st);
    case 3: return dispatch_flags<3>(a, st);
    case 4: return dispatch_flags<4>(a, st);
    case 5: return dispatch_flags<5>(a, st);
    case 6: return dispatch_flags<6>(a, st);
    case 7: return dispatch_flags<7>(a, st);
    case 8: return dispatch_flags<8>(a, st);
    case 9: return dispatch_flags<9>(a, st);
    case 10: return dispatch_flags<10>(a, st);
    case 11: return dispatch_flags<11>(a, st);
    case 12: return dispatch_flags<12>(a, st);
    case 13: return dispatch_flags<13>(a, st);
    case 14: return dispatch_flags<14>(a, st);
    case 15: return dispatch_flags<15>(a, st);
    case 16: return dispatch_flags<16>(a, st);
    default: return cudaErrorInvalidValue;
    }
}

} // namespace echo
