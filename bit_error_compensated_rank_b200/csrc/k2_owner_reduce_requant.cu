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
// In the owner-sum variant the correction c = lambda*f + (1-lambda)*s is
// added to the binary32 sum after the P restored values (one more rounding),
// instead of being added by the owner to its partial in kernel 1.
//
// Every restored value q*2^e is exact, so the only roundings are the P-1
// binary32 additions, rounding #2, and the two estimates' products and sums
// (each rounded on its own: __fmul_rn / __fadd_rn are never contracted).
// err is exact: S and Y = Q*2^E differ by at most 2^(E-1) and both are
// multiples of ulp(S).
//
// Binary16-scale variant (F16): scales are binary16 patterns (two bytes per
// group), restored values q*s are still exact, and with bf16 outputs the
// value every rank receives is q*s rounded to bf16; err is measured against
// that received value (still exact in binary32: it is a multiple of ulp(S)
// below 2^(exponent of S)).
//
// Pipeline (warp-specialised, persistent): a CTA takes tiles of kTile
// elements; one producer warp bulk-copies the P code tiles, the P scale tiles
// and the f, s tiles of a tile into one stage of a kStages ring (mbarrier
// full[s]); each lane of the eight consumer warps then restores one chunk of
// 8 elements across all P ranks, and each warp releases the stage on
// mbarrier empty[s]. On one GPU the P owners' segments are
// contiguous slices of one index space, so a launch covers all of them.
// Per element of n: P*17/32 bytes of wire and 8 bytes of state read, 17/32
// bytes of wire and 8 bytes of state written.
#include "echo_bulk.cuh"
#include "echo_kernels.h"

#include <cuda_runtime.h>

#include <atomic>

namespace echo {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32; // + one producer warp

// Bytes of one stage for `chunks` chunks per consumer thread: P code tiles,
// P scale tiles (1 or 2 bytes per group of at least kMinGroup), and the f, s
// tiles.
constexpr int k2_stage_bytes(int P, bool comp, bool f16, int chunks)
{
    return P * (kConsumers * kChunk * chunks / 2 + kConsumers * kChunk * chunks / kMinGroup * (f16 ? 2 : 1)) +
           (comp ? 2 * kConsumers * kChunk * chunks * 4 : 0);
}

// The largest of ECHO_K2_CHUNKS, /2, /4 whose stages fit the budget.
constexpr int k2_chunks(int P, bool comp, bool f16)
{
    int c = ECHO_K2_CHUNKS;
    while (c > 1 && ECHO_K2_STAGES * k2_stage_bytes(P, comp, f16, c) + 64 > ECHO_SMEM_BUDGET)
        c /= 2;
    return c;
}

// Stages of the ring: ECHO_K2_STAGES, or, when the tile had to shrink, as
// many of the smaller stages as fit, up to ECHO_K2_MAX_STAGES.
constexpr int k2_stages(int P, bool comp, bool f16)
{
    const int c = k2_chunks(P, comp, f16);
    int s = ECHO_K2_STAGES;
    if (c < ECHO_K2_CHUNKS)
        while (s < ECHO_K2_MAX_STAGES && (s + 1) * (k2_stage_bytes(P, comp, f16, c) + 16) <= ECHO_SMEM_BUDGET)
            s++;
    return s;
}

template <int P, bool COMP, bool F16>
struct K2Shape {
    static constexpr int kChunks = k2_chunks(P, COMP, F16); // chunks per consumer thread
    static constexpr int kTile = kConsumers * kChunk * kChunks;
    static constexpr int kStages = k2_stages(P, COMP, F16);
    static constexpr int kCodeBytes = kTile / 2;          // one rank's code tile
    static constexpr int kScaleBytes = kTile / kMinGroup * (F16 ? 2 : 1); // room for one rank's scale tile
    static constexpr int kStateOff = P * (kCodeBytes + kScaleBytes);
    static constexpr int kStageBytes = kStateOff + (COMP ? 2 * kTile * 4 : 0);
    static constexpr int kSmem = kStages * kStageBytes + 2 * kStages * 8;
    static_assert(kSmem <= ECHO_SMEM_BUDGET, "kernel 2 stages exceed shared memory");
};

__device__ __forceinline__ uint32_t round16(uint32_t x) { return (x + 15u) & ~15u; }

template <int P, bool COMP, bool SUM, bool F16>
__global__ void __launch_bounds__(kThreads)
    k2_owner_reduce_requant(const K2Args a)
{
    using Sh = K2Shape<P, COMP, F16>;
    constexpr uint32_t kScaleLog2 = F16 ? 1u : 0u; // log2 of the bytes per scale
    // From P = 11 on the kernel issues more instructions than its bytes
    // hide, so the restore-and-add and the codes of rounding #2 use sm_100's
    // packed f32x2 FMA (two elements per instruction, each rounded as the
    // scalar __fmaf_rn). At P <= 8 the scalar form measured faster. No
    // product feeds a separate addition here, so nothing can be contracted.
    constexpr bool kPacked = P >= 11;
    constexpr int S = Sh::kStages;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + S * Sh::kStageBytes);
    uint64_t *empty = full + S;

    const uint32_t tid = threadIdx.x;
    const uint32_t warp = tid >> 5;
    const uint32_t lane = tid & 31u;
    const size_t e0 = static_cast<size_t>(a.chunk_begin) * kChunk;
    const size_t e1 = static_cast<size_t>(a.chunk_end) * kChunk;
    // the tile length of this launch: a power of two <= Sh::kTile (smem strides keep Sh::kTile)
    const uint32_t tile = a.tile;
    const uint32_t ntiles = static_cast<uint32_t>((e1 - e0 + tile - 1) >> a.tile_log2);
    const uint32_t mine = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (tid == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        mbar_init_fence();
    }
    __syncthreads();
    wait_for_predecessor(); // nothing above touches global memory
    allow_successor();

    if (warp == kConsumerWarps) { // producer
        // The scale tile of a ragged last tile is rounded up to 16 bytes;
        // scale rows are padded to 16 bytes, so the extra bytes stay inside
        // the row and are never used.
        // A tile is 2P + 2 copies (P code slices, P scale slices, f, s),
        // issued by the warp's lanes in parallel.
        struct Tile {
            size_t el0;
            uint32_t cnt, sc_bytes;
            bool ok;
        };
        auto tile_of = [&](uint32_t i) {
            Tile t;
            t.el0 = e0 + static_cast<size_t>(blockIdx.x + i * gridDim.x) * tile;
            t.cnt = static_cast<uint32_t>(e1 - t.el0 < size_t(tile) ? e1 - t.el0 : tile);
            t.sc_bytes = round16((t.cnt >> (a.lanes_log2 + 3)) << kScaleLog2);
            // code, state and scale copies against their rows
            t.ok = in_bounds(t.el0 + t.cnt <= a.n && t.cnt <= Sh::kTile && t.sc_bytes <= Sh::kScaleBytes &&
                                 ((t.el0 >> (a.lanes_log2 + 3)) << kScaleLog2) + t.sc_bytes <= a.scale_stride,
                             a.ctl.status);
            return t;
        };
        produce_tiles_warp<S>(
            full, empty, mine, a.ctl.stall, a.ctl.wait_cycles, a.ctl.status, kStatusTimeoutK2,
            2 * P + (COMP ? 2 : 0),
            [&](uint32_t i) {
                const Tile t = tile_of(i);
                mbar_arrive_expect_tx(&full[i % S],
                                      t.ok ? P * (t.cnt / 2 + t.sc_bytes) + (COMP ? 2 * t.cnt * 4 : 0) : 0u);
            },
            [&](uint32_t i, uint32_t k) {
                const Tile t = tile_of(i);
                if (!t.ok)
                    return;
                uint8_t *stage = smem + (i % S) * Sh::kStageBytes;
                uint64_t *bar = &full[i % S];
                if (k < static_cast<uint32_t>(P)) {
                    bulk_load(stage + k * Sh::kCodeBytes, a.codes + k * (a.n / 2) + t.el0 / 2, t.cnt / 2, bar);
                } else if (k < 2u * P) {
                    const uint32_t r = k - P;
                    bulk_load(stage + P * Sh::kCodeBytes + r * Sh::kScaleBytes,
                              a.scales + r * a.scale_stride + ((t.el0 >> (a.lanes_log2 + 3)) << kScaleLog2),
                              t.sc_bytes, bar);
                } else if (COMP) {
                    const uint32_t j = k - 2 * P; // 0: f, 1: s
                    bulk_load(stage + Sh::kStateOff + j * Sh::kTile * 4, (j ? a.s : a.f) + t.el0, t.cnt * 4, bar);
                }
            });
        return;
    }

    for (uint32_t i = 0; i < mine; i++) {
        const uint32_t sidx = i % S;
        if (!warp_wait(&full[sidx], (i / S) & 1u, a.ctl.wait_cycles, a.ctl.status, kStatusTimeoutK2))
            return;
        const uint32_t tile_chunk0 = static_cast<uint32_t>(e0 / kChunk) + (blockIdx.x + i * gridDim.x) * (tile / kChunk);
        const uint8_t *stage = smem + sidx * Sh::kStageBytes;
#pragma unroll 1
        for (uint32_t j = 0; j < tile / (kChunk * kConsumers); j++) {
            const uint32_t c = tid + j * kConsumers; // chunk within the tile
            const uint32_t chunk = tile_chunk0 + c;
            const bool active = chunk < a.chunk_end;
            const uint32_t g = chunk >> a.lanes_log2;

            float fv[kChunk], sv[kChunk];
            if (COMP) {
                const float *fs = reinterpret_cast<const float *>(stage + Sh::kStateOff);
                const float4 f0 = reinterpret_cast<const float4 *>(fs)[2 * c];
                const float4 f1 = reinterpret_cast<const float4 *>(fs)[2 * c + 1];
                const float4 s0 = reinterpret_cast<const float4 *>(fs + Sh::kTile)[2 * c];
                const float4 s1 = reinterpret_cast<const float4 *>(fs + Sh::kTile)[2 * c + 1];
                fv[0] = f0.x, fv[1] = f0.y, fv[2] = f0.z, fv[3] = f0.w;
                fv[4] = f1.x, fv[5] = f1.y, fv[6] = f1.z, fv[7] = f1.w;
                sv[0] = s0.x, sv[1] = s0.y, sv[2] = s0.z, sv[3] = s0.w;
                sv[4] = s1.x, sv[5] = s1.y, sv[6] = s1.z, sv[7] = s1.w;
            }

            // Restore and add, rank 0 first. The product q*step is exact, so
            // fma(q, step, S) = RN(S + q*step): one rounding per addition.
            float S_[kChunk];
#pragma unroll
            for (int k = 0; k < kChunk; k++)
                S_[k] = 0.f;
#pragma unroll
            for (int r = 0; r < P; r++) {
                const uint32_t w = reinterpret_cast<const uint32_t *>(stage + r * Sh::kCodeBytes)[c];
                const uint8_t *srow = stage + P * Sh::kCodeBytes + r * Sh::kScaleBytes;
                const float st = F16 ? half_step(reinterpret_cast<const uint16_t *>(srow)[c >> a.lanes_log2])
                                     : step_of(srow[c >> a.lanes_log2]);
                const Unpacked u = unpack8(w);
                if (kPacked) {
                    const float2 st2 = make_float2(st, st);
#pragma unroll
                    for (int j = 0; j < kChunk / 2; j++) { // two elements per packed FMA
                        const float2 acc =
                            __ffma2_rn(code_pair(u, j), st2, make_float2(S_[2 * j], S_[2 * j + 1]));
                        S_[2 * j] = acc.x, S_[2 * j + 1] = acc.y;
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < kChunk; k++)
                        S_[k] = __fmaf_rn(code_at(u, k), st, S_[k]);
                }
            }
            if (SUM) { // variant: the correction enters the owner's sum, after the P ranks
#pragma unroll
                for (int k = 0; k < kChunk; k++)
                    S_[k] = __fadd_rn(S_[k], __fadd_rn(__fmul_rn(a.lambda, fv[k]),
                                                       __fmul_rn(a.one_minus_lambda, sv[k])));
            }

            // Rounding #2 and the error it injects.
            const float amax = group_absmax(absmax8(S_), a.lanes_log2);
            uint32_t qb[kChunk];
            float err[kChunk];
            uint32_t scale;
            if (F16) {
                scale = half_scale_bits(amax);
                const float st = half_step(scale);
                const float inv = half_inv(st);
                const float half = __fmul_rn(0.5f, st);
                codes8_half(S_, st, inv, half, half_scale_saturates(amax), false, qb);
#pragma unroll
                for (int k = 0; k < kChunk; k++) {
                    qb[k] = zcode_bits(qb[k]);
                    const float y = __fmul_rn(code_value(qb[k]), st); // exact
                    err[k] = __fsub_rn(S_[k], a.bf16 ? round_bf16(y) : y);
                }
            } else {
                scale = scale_byte(amax);
                const float inv = inv_step_of(scale);
                const float st = step_of(scale);
                if (kPacked) {
#pragma unroll
                    for (int j = 0; j < kChunk / 2; j++) {
                        const float2 S2 = make_float2(S_[2 * j], S_[2 * j + 1]);
                        const float2 t = __ffma2_rn(S2, make_float2(inv, inv), make_float2(kRound, kRound));
                        qb[2 * j] = __float_as_uint(t.x), qb[2 * j + 1] = __float_as_uint(t.y);
                        // S - Q*2^E, exact: Q = t - kRound, then Q*(-2^E) + S
                        const float2 e2 =
                            __ffma2_rn(__fadd2_rn(t, make_float2(-kRound, -kRound)), make_float2(-st, -st), S2);
                        err[2 * j] = e2.x, err[2 * j + 1] = e2.y;
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < kChunk; k++) {
                        qb[k] = code_bits(S_[k], inv);
                        err[k] = __fmaf_rn(-code_value(qb[k]), st, S_[k]); // S - Q*2^E, exact
                    }
                }
            }

            if (active && a.to_ranks &&
                in_bounds(chunk < a.n / kChunk && (size_t(a.q_chunk0) + chunk + 1) * 4u <= a.q_scales_off &&
                              (size_t(a.q_group0) + g + 1) * (F16 ? 2u : 1u) <= a.q_scale_bytes,
                          a.ctl.status)) {
                // one handle per rank: the owned segment straight into every rank's gathered buffer
                const uint32_t word = pack8_bits(qb);
                const bool first = (lane & ((1u << a.lanes_log2) - 1u)) == 0;
#pragma unroll
                for (int p = 0; p < P; p++) {
                    uint8_t *blk = static_cast<uint8_t *>(a.ranks.p[p]);
                    reinterpret_cast<uint32_t *>(blk)[a.q_chunk0 + chunk] = word;
                    if (first) {
                        if (F16)
                            reinterpret_cast<uint16_t *>(blk + a.q_scales_off)[a.q_group0 + g] =
                                static_cast<uint16_t>(scale);
                        else
                            blk[a.q_scales_off + a.q_group0 + g] = static_cast<uint8_t>(scale);
                    }
                }
            }
            if (active && in_bounds(chunk < a.n / kChunk && (g + 1) * (F16 ? 2u : 1u) <= a.scale_stride,
                                    a.ctl.status)) {
                if (!a.to_ranks) {
                    reinterpret_cast<uint32_t *>(a.qcodes)[chunk] = pack8_bits(qb);
                    if ((lane & ((1u << a.lanes_log2) - 1u)) == 0) { // the group's first lane
                        if (F16)
                            reinterpret_cast<uint16_t *>(a.qscales)[g] = static_cast<uint16_t>(scale);
                        else
                            a.qscales[g] = static_cast<uint8_t>(scale);
                    }
                }
                if (COMP) {
                    // Scalar on purpose: packed f32x2 multiplies followed by a
                    // packed add did not match the oracle on B200 (one element
                    // of the slow estimate in millions, as if fused into one
                    // FMA), so the estimates keep the scalar roundings.
#pragma unroll
                    for (int k = 0; k < kChunk; k++) {
                        fv[k] = __fadd_rn(__fmul_rn(a.beta_f, fv[k]), __fmul_rn(a.one_minus_beta_f, err[k]));
                        sv[k] = __fadd_rn(__fmul_rn(a.beta_s, sv[k]), __fmul_rn(a.one_minus_beta_s, err[k]));
                    }
                    float4 *fo = reinterpret_cast<float4 *>(a.f) + 2 * static_cast<size_t>(chunk);
                    float4 *so = reinterpret_cast<float4 *>(a.s) + 2 * static_cast<size_t>(chunk);
                    fo[0] = make_float4(fv[0], fv[1], fv[2], fv[3]);
                    fo[1] = make_float4(fv[4], fv[5], fv[6], fv[7]);
                    so[0] = make_float4(sv[0], sv[1], sv[2], sv[3]);
                    so[1] = make_float4(sv[4], sv[5], sv[6], sv[7]);
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[sidx]); // this warp is done reading the stage
    }
}

template <int P, bool COMP, bool SUM, bool F16>
cudaError_t launch_p(const K2Args &a, cudaStream_t st)
{
    using Sh = K2Shape<P, COMP, F16>;
    // CTAs per SM of this instantiation, found once (threads that race here
    // compute the same value)
    static std::atomic<int> cached{0};
    int resident = cached.load(std::memory_order_relaxed);
    auto kern = k2_owner_reduce_requant<P, COMP, SUM, F16>;
    if (resident == 0) {
        cudaError_t e = prepare_kernel(reinterpret_cast<const void *>(kern), kThreads, Sh::kSmem, &resident);
        if (e != cudaSuccess)
            return e;
        cached.store(resident, std::memory_order_relaxed);
    }
    const size_t elems = static_cast<size_t>(a.chunk_end - a.chunk_begin) * kChunk;
    K2Args b = a;
    b.tile_log2 = pick_tile_log2(elems, Sh::kTile, kConsumers * kChunk, resident);
    b.tile = 1u << b.tile_log2;
    const uint32_t tiles = static_cast<uint32_t>((elems + b.tile - 1) >> b.tile_log2);
    return launch_chained(kern, persistent_grid(tiles, resident), kThreads, Sh::kSmem, st, b);
}

template <int P, bool F16>
cudaError_t dispatch_state(const K2Args &a, cudaStream_t st)
{
    if (!a.enable)
        return launch_p<P, false, false, F16>(a, st);
    return a.owner_sum ? launch_p<P, true, true, F16>(a, st) : launch_p<P, true, false, F16>(a, st);
}

template <int P>
cudaError_t dispatch_flags(const K2Args &a, cudaStream_t st)
{
    return a.fp16_scale ? dispatch_state<P, true>(a, st) : dispatch_state<P, false>(a, st);
}

} // namespace

cudaError_t launch_k2_owner_reduce_requant(const K2Args &a, cudaStream_t st)
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
