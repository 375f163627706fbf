// k3_gather_dequant.cu - kernel 3 of the Echo all-reduce.
//
// Every rank receives the owner's requantised total and restores it
// [rit.work "Echo 4-bit GPU communication", section "How Echo returns the
// error to later calls": the compressed total is sent back to every rank].
// Y = Q*2^E has at most three significant bits, so it is exact in bf16 and
// in binary32: the restore adds no third rounding.
//
// Pipeline: a persistent CTA takes tiles of kTile elements. Thread 0
// bulk-copies the tile's codes and scale bytes into a kInStages ring; the CTA
// restores the tile once into one of kOutBufs output buffers in shared
// memory; thread 0 then bulk-stores that buffer to all P rank outputs, so the
// TMA engine, not the load/store units, moves the P-fold write stream. On one
// GPU the P ranks share one requantised buffer, which is read from HBM once.
// Per element of n: P*b bytes written, 17/32 bytes read.
#include "echo_bulk.cuh"
#include "echo_kernels.h"

#include <cuda_runtime.h>

namespace echo {
namespace {

constexpr int kThreads = 256;

template <bool BF16>
struct K3Shape {
    static constexpr int kEB = BF16 ? 2 : 4;
    static constexpr int kTile = BF16 ? 4096 : 2048;
    static constexpr int kInStages = 4;
    static constexpr int kOutBufs = 2;
    static constexpr int kCodeBytes = kTile / 2;
    static constexpr int kScaleBytes = kTile / kGroup;
    static constexpr int kInBytes = kCodeBytes + kScaleBytes;
    static constexpr int kOutBytes = kTile * kEB;
    static constexpr int kOutOff = kInStages * kInBytes;
    static constexpr int kSmem = kOutOff + kOutBufs * kOutBytes + kInStages * 8;
    static constexpr int kChunksPerTile = kTile / kChunk;
};

__device__ __forceinline__ uint32_t round16(uint32_t x) { return (x + 15u) & ~15u; }

template <int P, bool BF16>
__global__ void __launch_bounds__(kThreads)
    k3_gather_dequant(const K3Args a)
{
    using Sh = K3Shape<BF16>;
    constexpr int S = Sh::kInStages;
    constexpr int B = Sh::kOutBufs;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Sh::kOutOff + B * Sh::kOutBytes);

    const uint32_t tid = threadIdx.x;
    const size_t e0 = static_cast<size_t>(a.chunk_begin) * kChunk;
    const size_t e1 = static_cast<size_t>(a.chunk_end) * kChunk;
    const uint32_t ntiles = static_cast<uint32_t>((e1 - e0 + Sh::kTile - 1) / Sh::kTile);
    const uint32_t mine = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (tid == 0) {
        for (int s = 0; s < S; s++)
            mbar_init(&full[s], 1);
        mbar_init_fence();
    }
    __syncthreads();

    auto issue = [&](uint32_t i) {
        const size_t el0 = e0 + static_cast<size_t>(blockIdx.x + i * gridDim.x) * Sh::kTile;
        const uint32_t cnt = static_cast<uint32_t>(e1 - el0 < size_t(Sh::kTile) ? e1 - el0 : Sh::kTile);
        const uint32_t sc_bytes = round16(cnt / kGroup); // scale rows are padded to 16 bytes
        uint8_t *stage = smem + (i % S) * Sh::kInBytes;
        uint64_t *bar = &full[i % S];
        mbar_arrive_expect_tx(bar, cnt / 2 + sc_bytes);
        bulk_load(stage, a.qcodes + el0 / 2, cnt / 2, bar);
        bulk_load(stage + Sh::kCodeBytes, a.qscales + el0 / kGroup, sc_bytes, bar);
    };

    uint32_t issued = 0; // meaningful on thread 0 only
    if (tid == 0 && !a.ctl.stall)
        for (; issued < mine && issued < static_cast<uint32_t>(S); issued++)
            issue(issued);

    for (uint32_t i = 0; i < mine; i++) {
        // Output buffer i % B was last stored for tile i - B: make sure that
        // store has finished reading it (at most B-1 younger groups pending).
        if (tid == 0)
            bulk_wait_read<B - 1>();
        if (!wait_tile(&full[i % S], (i / S) & 1u, a.ctl.wait_cycles, a.ctl.status, kStatusTimeoutK3)) {
            drain_loads(full, S, i, issued, a.ctl.wait_cycles);
            if (tid == 0)
                bulk_wait_all();
            return;
        }
        if (tid == 0 && i >= 1 && i - 1 + S < mine) {
            issue(i - 1 + S);
            issued++;
        }

        const size_t el0 = e0 + static_cast<size_t>(blockIdx.x + i * gridDim.x) * Sh::kTile;
        const uint32_t cnt = static_cast<uint32_t>(e1 - el0 < size_t(Sh::kTile) ? e1 - el0 : Sh::kTile);
        const uint8_t *stage = smem + (i % S) * Sh::kInBytes;
        uint8_t *out = smem + Sh::kOutOff + (i % B) * Sh::kOutBytes;

#pragma unroll
        for (int j = 0; j < Sh::kChunksPerTile / kThreads; j++) {
            const uint32_t c = tid + j * kThreads;
            const uint32_t w = reinterpret_cast<const uint32_t *>(stage)[c];
            const float st = step_of(stage[Sh::kCodeBytes + c / kLanesPerGroup]);
            const Unpacked u = unpack8(w);
            float y[kChunk];
#pragma unroll
            for (int k = 0; k < kChunk; k++)
                y[k] = __fmul_rn(code_at(u, k), st);
            if (BF16) {
                reinterpret_cast<uint4 *>(out)[c] = f32x8_to_bf16_exact(y);
            } else {
                reinterpret_cast<float4 *>(out)[2 * c] = make_float4(y[0], y[1], y[2], y[3]);
                reinterpret_cast<float4 *>(out)[2 * c + 1] = make_float4(y[4], y[5], y[6], y[7]);
            }
        }
        fence_proxy_async_smem(); // the restored tile is read next by the bulk stores
        __syncthreads();
        if (tid == 0) {
#pragma unroll
            for (int r = 0; r < P; r++)
                bulk_store(static_cast<uint8_t *>(a.out.p[r]) + el0 * Sh::kEB, out, cnt * Sh::kEB);
            bulk_commit();
        }
    }
    if (tid == 0)
        bulk_wait_all();
}

template <int P, bool BF16>
cudaError_t launch_p(const K3Args &a, cudaStream_t st)
{
    using Sh = K3Shape<BF16>;
    static int resident = 0;
    auto kern = k3_gather_dequant<P, BF16>;
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
cudaError_t dispatch_flags(const K3Args &a, cudaStream_t st)
{
    return a.bf16 ? launch_p<P, true>(a, st) : launch_p<P, false>(a, st);
}

} // namespace

cudaError_t launch_k3_gather_dequant(const K3Args &a, cudaStream_t st)
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
