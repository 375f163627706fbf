// echo_bulk.cuh - bulk-copy (TMA engine) pipeline helpers for sm_100a.
//
// The three kernels stream tiles between HBM and shared memory with the
// untiled bulk copy (cp.async.bulk): one elected thread of a producer warp
// issues whole-tile copies, completion is tracked by an mbarrier's
// transaction count ("full"), consumer warps compute from shared memory and
// hand each stage back on a second mbarrier ("empty"). No copy uses cluster
// multicast, and every bulk load reads this GPU's memory only; the only bulk
// stores into another rank's memory are kernel 1's code words with one handle
// per rank and sender feedback (a peer's receive block, on several GPUs).
//
// Every wait is bounded in time: a warp that does not see its barrier phase
// complete within the limit records the failure in the device status word
// and leaves its loop (warp_wait, produce_tiles), so a fault in the pipeline
// can never hang the GPU.
#pragma once

#include <cstdint>

namespace echo {

// Device status word bits (the host reads them with echo_device_status).
constexpr int kStatusTimeoutK1 = 1;
constexpr int kStatusTimeoutK2 = 2;
constexpr int kStatusTimeoutK3 = 4;
constexpr int kStatusBounds = 8;  // debug build: an access would leave its buffer
constexpr int kStatusCanary = 16; // debug build: a guard byte around a buffer changed

#ifndef ECHO_DEBUG
#define ECHO_DEBUG 0
#endif

// In the debug build (ECHO_DEBUG=1), a failed check of an index or a copy
// range against its buffer records kStatusBounds and returns false, so the
// caller skips the access; the release build checks nothing and returns true.
__device__ __forceinline__ bool in_bounds(bool ok, int *status)
{
#if ECHO_DEBUG
    if (!ok) {
        atomicOr(status, kStatusBounds);
        return false;
    }
#else
    (void)ok;
    (void)status;
#endif
    return true;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async proxy before first use.
__device__ __forceinline__ void mbar_init_fence()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t done;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(done)
                 : "r"(smem_u32(bar)), "r"(parity)
                 : "memory");
    return done != 0;
}

// Poll the barrier's phase with parity `parity` for at most `limit` SM
// clock cycles (a real-time bound, whatever try_wait's own suspend window is).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, long long limit)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > limit)
            return false;
    return true;
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses
// 16-byte aligned), completing `bytes` transactions on `bar`.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gmem_src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(smem_dst)),
                 "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Shared -> global bulk copy, tracked by the issuing thread's bulk groups.
__device__ __forceinline__ void bulk_store(void *gmem_dst, const void *smem_src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gmem_dst),
                 "r"(smem_u32(smem_src)), "r"(bytes)
                 : "memory");
}

// An L2 policy that makes the lines it touches the first to be evicted.
__device__ __forceinline__ uint64_t l2_evict_first_policy()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// bulk_store with an L2 cache policy (l2_evict_first_policy).
__device__ __forceinline__ void bulk_store_hint(void *gmem_dst, const void *smem_src, uint32_t bytes, uint64_t policy)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;" ::"l"(gmem_dst),
                 "r"(smem_u32(smem_src)), "r"(bytes), "l"(policy)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N committed store groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until every committed store group has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Order this thread's generic-proxy writes to shared memory before later
// async-proxy (bulk copy) reads of it.
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Programmatic dependent launch. Each kernel is launched allowed to start
// before its predecessor in the stream has finished; it sets up its own
// barriers, then waits here until every prerequisite grid has completed and
// its memory is visible, before it touches any global memory. Right after,
// it lets its own successor start launching (that successor waits the same
// way). Without the launch attribute both are no-ops.
__device__ __forceinline__ void wait_for_predecessor()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void allow_successor()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Every lane of the calling warp waits (bounded) for the phase with parity
// `parity`; the outcome is made warp-uniform, so the warp goes on or leaves
// as a whole. On a timeout lane 0 records `status_bit`.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, long long limit, int *status,
                                          int status_bit)
{
    const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(bar, parity, limit));
    if (!ok && (threadIdx.x & 31u) == 0)
        atomicOr(status, status_bit);
    return ok;
}

// Producer side of an S-stage ring of tiles (one elected thread). issue(i)
// must arm full[i % S] with the byte count and start the copies of local tile
// i. Stage s is reused only after every consumer warp has released it on
// empty[s]. Before returning, the producer waits (bounded) until the loads of
// the last S tiles it issued have landed, so no copy is in flight when the CTA
// leaves, also after a timeout.
template <int S, typename Issue>
__device__ __forceinline__ void produce_tiles(uint64_t *full, uint64_t *empty, uint32_t tiles, bool stall,
                                              long long limit, int *status, int status_bit, Issue issue)
{
    uint32_t i = 0;
    if (!stall) {
        for (; i < tiles; i++) {
            const uint32_t s = i % S;
            if (i >= static_cast<uint32_t>(S) && !mbar_wait_bounded(&empty[s], ((i / S) - 1) & 1u, limit)) {
                atomicOr(status, status_bit);
                break;
            }
            issue(i);
        }
    }
    for (uint32_t t = i > static_cast<uint32_t>(S) ? i - S : 0; t < i; t++)
        mbar_wait_bounded(&full[t % S], (t / S) & 1u, limit);
}

// produce_tiles with a write-back: the consumers leave results in a stage
// (written to shared memory, then fence.proxy.async, then their release on
// empty[s]), and writeback(t) bulk-stores them for local tile t. A stage is
// refilled only after the stores of its previous tile have read it. After
// the last tile the producer waits (bounded) for the consumers to release
// each tile not yet written back, writes it back, and waits until every store
// has completed before returning. If a consumer wait runs out, the remaining
// tiles are not written back (the status bit says why) and the producer only
// waits for their loads to land.
template <int S, typename Issue, typename WriteBack>
__device__ __forceinline__ void produce_tiles_writeback(uint64_t *full, uint64_t *empty, uint32_t tiles, bool stall,
                                                        long long limit, int *status, int status_bit, Issue issue,
                                                        WriteBack writeback)
{
    uint32_t i = 0;
    bool ok = true;
    if (!stall) {
        for (; i < tiles; i++) {
            const uint32_t s = i % S;
            if (i >= static_cast<uint32_t>(S)) {
                if (!mbar_wait_bounded(&empty[s], ((i / S) - 1) & 1u, limit)) {
                    atomicOr(status, status_bit);
                    ok = false;
                    break;
                }
                writeback(i - S);
                bulk_commit();
                bulk_wait_read<0>(); // the stores have read the stage: it may be refilled
            }
            issue(i);
        }
    }
    for (uint32_t t = i > static_cast<uint32_t>(S) ? i - S : 0; t < i; t++) {
        if (ok && mbar_wait_bounded(&empty[t % S], (t / S) & 1u, limit)) {
            writeback(t);
            bulk_commit();
        } else {
            if (ok)
                atomicOr(status, status_bit);
            ok = false;
            mbar_wait_bounded(&full[t % S], (t / S) & 1u, limit);
        }
    }
    bulk_wait_all();
}

// The same ring fed by the whole producer warp: for local tile i, lane 0
// arms full[i % S] (arm(i): arrive with the tile's byte count), then the
// tile's ncopies bulk copies are issued by the 32 lanes in parallel
// (copy(i, k) for k = lane, lane + 32, ...), so a tile made of many small
// copies does not wait on one thread issuing them in turn. Every lane of the
// warp must call it. The stage waits and the final drain are as in
// produce_tiles, and bounded the same way.
template <int S, typename Arm, typename Copy>
__device__ __forceinline__ void produce_tiles_warp(uint64_t *full, uint64_t *empty, uint32_t tiles, bool stall,
                                                   long long limit, int *status, int status_bit, uint32_t ncopies,
                                                   Arm arm, Copy copy)
{
    const uint32_t lane = threadIdx.x & 31u;
    uint32_t i = 0;
    if (!stall) {
        for (; i < tiles; i++) {
            const uint32_t s = i % S;
            if (i >= static_cast<uint32_t>(S) &&
                !__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&empty[s], ((i / S) - 1) & 1u, limit))) {
                if (lane == 0)
                    atomicOr(status, status_bit);
                break;
            }
            if (lane == 0)
                arm(i);
            __syncwarp();
            for (uint32_t k = lane; k < ncopies; k += 32)
                copy(i, k);
        }
    }
    if (lane == 0)
        for (uint32_t t = i > static_cast<uint32_t>(S) ? i - S : 0; t < i; t++)
            mbar_wait_bounded(&full[t % S], (t / S) & 1u, limit);
    __syncwarp();
}

} // namespace echo
