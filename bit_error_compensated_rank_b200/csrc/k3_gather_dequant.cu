// k3_gather_dequant.cu - kernel 3 of the Echo all-reduce.
//
// Every rank receives the owner's requantised total and restores it
// [rit.work "Echo 4-bit GPU communication", section "How Echo returns the
// error to later calls": the compressed total is sent back to every rank].
// Y = Q*2^E has at most three significant bits, so it is exact in bf16 and
// in binary32: the restore adds no third rounding. Under the binary16-scale
// variant (F16) Y = Q*s has up to 14 significant bits: exact in binary32,
// rounded to the nearest bf16 (ties to even) for bf16 outputs, the value
// kernel 2 measured its error against.
//
// Pipeline (warp-specialised, persistent): a CTA takes tiles of kTile
// elements. A load warp bulk-copies the tile's codes and scale bytes into a
// kInStages ring (mbarriers in_full / in_empty); eight consumer warps restore
// the tile once into one of kOutBufs output buffers in shared memory
// (mbarriers out_full / out_empty); a store warp bulk-stores each finished
// buffer to all P rank outputs, so the TMA engine, not the load/store units,
// moves the P-fold write stream, and hands the buffer back once the engine
// has read it. On one GPU the P ranks share one requantised buffer, which is
// read from HBM once. Per element of n: P*b bytes written, 17/32 bytes read.
#include "echo_bulk.cuh"
#include "echo_kernels.h"

#include <cuda_runtime.h>

#include <atomic>

namespace echo {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kLoadWarp = kConsumerWarps;
constexpr int kStoreWarp = kConsumerWarps + 1;
constexpr int kThreads = kConsumers + 64;

template <bool BF16, bool F16>
struct K3Shape {
    static constexpr int kEB = BF16 ? 2 : 4;
    static constexpr int kTile = BF16 ? ECHO_K3_TILE : ECHO_K3_TILE / 2;
    static constexpr int kInStages = ECHO_K3_IN_STAGES;
    static constexpr int kOutBufs = ECHO_K3_OUT_BUFS;
    static constexpr int kCodeBytes = kTile / 2;
    static constexpr int kScaleBytes = kTile / kMinGroup * (F16 ? 2 : 1); // room for the tile's scales
    static constexpr int kInBytes = kCodeBytes + kScaleBytes;
    static constexpr int kOutBytes = kTile * kEB;
    static constexpr int kOutOff = kInStages * kInBytes;
    static constexpr int kBarOff = kOutOff + kOutBufs * kOutBytes;
    static constexpr int kSmem = kBarOff + (2 * kInStages + 2 * kOutBufs) * 8;
    static_assert(kSmem <= ECHO_SMEM_BUDGET, "kernel 3 buffers exceed shared memory");
};

__device__ __forceinline__ uint32_t round16(uint32_t x) { return (x + 15u) & ~15u; }

template <int P, bool BF16, bool F16>
__global__ void __launch_bounds__(kThreads)
    k3_gather_dequant(const K3Args a)
{
    using Sh = K3Shape<BF16, F16>;
    constexpr uint32_t kScaleLog2 = F16 ? 1u : 0u; // log2 of the bytes per scale
    constexpr int S = Sh::kInStages;
    constexpr int B = Sh::kOutBufs;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *in_full = reinterpret_cast<uint64_t *>(smem + Sh::kBarOff);
    uint64_t *in_empty = in_full + S;
    uint64_t *out_full = in_empty + S;
    uint64_t *out_empty = out_full + B;

    const uint32_t tid = threadIdx.x;
    const uint32_t warp = tid >> 5;
    const uint32_t lane = tid & 31u;
    const size_t e0 = static_cast<size_t>(a.chunk_begin) * kChunk;
    const size_t e1 = static_cast<size_t>(a.chunk_end) * kChunk;
    // the tile length of this launch: a power of two <= Sh::kTile (smem strides keep Sh::kTile)
    const uint32_t tile = a.tile;
    const uint32_t ntiles = static_cast<uint32_t>((e1 - e0 + tile - 1) >> a.tile_log2);
    const uint32_t mine = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    auto tile_start = [&](uint32_t i) { return e0 + static_cast<size_t>(blockIdx.x + i * gridDim.x) * tile; };
    auto tile_count = [&](size_t el0) {
        return static_cast<uint32_t>(e1 - el0 < size_t(tile) ? e1 - el0 : tile);
    };

    if (tid == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&in_full[s], 1);
            mbar_init(&in_empty[s], kConsumerWarps);
        }
        for (int b = 0; b < B; b++) {
            mbar_init(&out_full[b], kConsumerWarps);
            mbar_init(&out_empty[b], 1);
        }
        mbar_init_fence();
    }
    __syncthreads();
    wait_for_predecessor(); // nothing above touches global memory
    allow_successor();

    if (warp == kLoadWarp) {
        // scale rows are padded to 16 bytes, so a ragged tile's scale copy may
        // round up to 16 bytes without leaving the row
        if (lane == 0)
            produce_tiles<S>(in_full, in_empty, mine, a.ctl.stall, a.ctl.wait_cycles, a.ctl.status,
                             kStatusTimeoutK3, [&](uint32_t i) {
                                 const size_t el0 = tile_start(i);
                                 const uint32_t cnt = tile_count(el0);
                                 const uint32_t sc_bytes = round16((cnt >> (a.lanes_log2 + 3)) << kScaleLog2);
                                 uint8_t *stage = smem + (i % S) * Sh::kInBytes;
                                 uint64_t *bar = &in_full[i % S];
                                 // the requantised scales have room for 2n/G bytes
                                 const bool ok = in_bounds(el0 + cnt <= a.n && cnt <= Sh::kTile &&
                                                               sc_bytes <= Sh::kScaleBytes &&
                                                               ((el0 >> (a.lanes_log2 + 3)) << kScaleLog2) +
                                                                       sc_bytes <= a.scale_stride,
                                                           a.ctl.status);
                                 mbar_arrive_expect_tx(bar, ok ? cnt / 2 + sc_bytes : 0u);
                                 if (!ok)
                                     return;
                                 bulk_load(stage, a.qcodes + el0 / 2, cnt / 2, bar);
                                 bulk_load(stage + Sh::kCodeBytes,
                                           a.qscales + ((el0 >> (a.lanes_log2 + 3)) << kScaleLog2), sc_bytes, bar);
                             });
        return;
    }

    if (warp == kStoreWarp) {
        if (lane == 0) {
            // the outputs are written once and not read again in the call:
            // their lines are the first that L2 evicts (measured 0.3 to 0.6 %
            // faster than the default policy)
            const uint64_t policy = l2_evict_first_policy();
            for (uint32_t i = 0; i < mine; i++) {
                const uint32_t b = i % B;
                if (!mbar_wait_bounded(&out_full[b], (i / B) & 1u, a.ctl.wait_cycles)) {
                    atomicOr(a.ctl.status, kStatusTimeoutK3);
                    break;
                }
                const size_t el0 = tile_start(i);
                const uint32_t bytes = tile_count(el0) * Sh::kEB;
                const uint8_t *buf = smem + Sh::kOutOff + b * Sh::kOutBytes;
                if (in_bounds(el0 + tile_count(el0) <= a.n, a.ctl.status)) {
#pragma unroll
                    for (int r = 0; r < P; r++)
                        bulk_store_hint(static_cast<uint8_t *>(a.out.p[r]) + el0 * Sh::kEB, buf, bytes, policy);
                }
                bulk_commit();
                // at most B-1 younger groups still read: tile i-(B-1) is done
                bulk_wait_read<B - 1>();
                if (i >= static_cast<uint32_t>(B - 1))
                    mbar_arrive(&out_empty[(i - (B - 1)) % B]);
            }
            bulk_wait_all();
        }
        return;
    }

    for (uint32_t i = 0; i < mine; i++) {
        const uint32_t s = i % S;
        const uint32_t b = i % B;
        if (!warp_wait(&in_full[s], (i / S) & 1u, a.ctl.wait_cycles, a.ctl.status, kStatusTimeoutK3))
            return;
        if (i >= static_cast<uint32_t>(B) &&
            !warp_wait(&out_empty[b], ((i / B) - 1) & 1u, a.ctl.wait_cycles, a.ctl.status, kStatusTimeoutK3))
            return;
        const uint8_t *stage = smem + s * Sh::kInBytes;
        uint8_t *out = smem + Sh::kOutOff + b * Sh::kOutBytes;
#pragma unroll 2
        for (uint32_t j = 0; j < tile / (kChunk * kConsumers); j++) {
            const uint32_t c = tid + j * kConsumers;
            const uint32_t w = reinterpret_cast<const uint32_t *>(stage)[c];
            const float st =
                F16 ? half_step(reinterpret_cast<const uint16_t *>(stage + Sh::kCodeBytes)[c >> a.lanes_log2])
                    : step_of(stage[Sh::kCodeBytes + (c >> a.lanes_log2)]);
            const Unpacked u = unpack8(w);
            float y[kChunk];
#pragma unroll
            for (int k = 0; k < kChunk; k++)
                y[k] = __fmul_rn(code_at(u, k), st);
            if (BF16 && F16) { // round to the nearest bf16
                uint32_t w2[4];
#pragma unroll
                for (int j = 0; j < 4; j++)
                    w2[j] = __float_as_uint(round_bf16(y[2 * j])) >> 16 |
                            (__float_as_uint(round_bf16(y[2 * j + 1])) & 0xFFFF0000u);
                reinterpret_cast<uint4 *>(out)[c] = make_uint4(w2[0], w2[1], w2[2], w2[3]);
            } else if (BF16) {
                reinterpret_cast<uint4 *>(out)[c] = f32x8_to_bf16_exact(y);
            } else {
                reinterpret_cast<float4 *>(out)[2 * c] = make_float4(y[0], y[1], y[2], y[3]);
                reinterpret_cast<float4 *>(out)[2 * c + 1] = make_float4(y[4], y[5], y[6], y[7]);
            }
        }
        fence_proxy_async_smem(); // the restored tile is read next by the bulk stores
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&in_empty[s]);
            mbar_arrive(&out_full[b]);
        }
    }
}

template <int P, bool BF16, bool F16>
cudaError_t launch_p(const K3Args &a, cudaStream_t st)
{
    using Sh = K3Shape<BF16, F16>;
    // CTAs per SM of this instantiation, found once (threads that race here
    // compute the same value)
    static std::atomic<int> cached{0};
    int resident = cached.load(std::memory_order_relaxed);
    auto kern = k3_gather_dequant<P, BF16, F16>;
    if (resident == 0) {
        cudaError_t e = prepare_kernel(reinterpret_cast<const void *>(kern), kThreads, Sh::kSmem, &resident);
        if (e != cudaSuccess)
            return e;
        cached.store(resident, std::memory_order_relaxed);
    }
    const size_t elems = static_cast<size_t>(a.chunk_end - a.chunk_begin) * kChunk;
    K3Args b = a;
    b.tile_log2 = pick_tile_log2(elems, Sh::kTile, kConsumers * kChunk, resident);
    b.tile = 1u << b.tile_log2;
    const uint32_t tiles = static_cast<uint32_t>((elems + b.tile - 1) >> b.tile_log2);
    return launch_chained(kern, persistent_grid(tiles, resident), kThreads, Sh::kSmem, st, b);
}

template <int P>
cudaError_t dispatch_flags(const K3Args &a, cudaStream_t st)
{
    if (a.fp16_scale)
        return a.bf16 ? launch_p<P, true, true>(a, st) : launch_p<P, false, true>(a, st);
    return a.bf16 ? launch_p<P, true, false>(a, st) : launch_p<P, false, false>(a, st);
}

} // namespace

cudaError_t launch_k3_gather_dequant(const K3Args &a, cudaStream_t st)
{
    if (a.chunk_end <= a.chunk_begin)
        return cudaSuccess;
    switch (a.P) {
    case 1: return dispatch_flags<1>(a, st); // one output per process
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
