// k1_compensate_quantize_pack.cuh - kernel 1 of the Echo all-reduce (body).
//
// Every rank rounds its partial to 4-bit codes per group of 32 (rounding #1);
// on its own segment the owner first adds the correction
// c = lambda*f + (1-lambda)*s built from the two smoothed error estimates
// [rit.work "Echo 4-bit GPU communication", section "How Echo returns the
// error to later calls": the stored error is added back in later calls].
// With sender feedback (a variant), every rank first adds back its own
// rounding-#1 error of its previous call and stores the new one, exact:
// v = RN(RN(x + eps) + c), eps <- v - q*2^e.
//
// Layout: the rank partials are P separate buffers of n elements; the output
// is the stage-1 wire, codes [P][n/2] (two per byte) and scales
// [P][scale_stride] (n/G bytes per rank, or n/G binary16 patterns under the
// binary16-scale variant); the sender errors are [P][n] binary32.
//
// Two builds of the kernel: the default one (groups of 32, power-of-two
// scales) and a general one for the variants, which selects once per launch
// a consumer body compiled for the launch's group size and scale format.
//
// Pipeline (warp-specialised, persistent): a CTA takes tiles of kTile
// consecutive elements. One producer warp bulk-copies the P partial tiles
// (and the f, s tiles, and the P error tiles, when used) of a tile into one
// stage of a kStages ring in shared memory (mbarrier full[s] counts the
// bytes); consumer warps (8 in the default build, 16 in the variants' builds
// and with sender feedback, whose longer dependency chains want more warps to
// hide them) compute from shared memory and release the stage on mbarrier
// empty[s]. A lane owns 8 consecutive
// elements of one rank; G/8 lanes form a group and find its maximum with
// log2(G/8) shuffles; codes leave as one coalesced 32-bit store per lane.
// The binary16-scale body for bf16 partials without sender feedback, bound
// by instruction issue, gives a lane 16 elements instead (k1_consume_wide).
// With sender feedback each lane writes its 8 new errors over the old ones
// in the stage, and the producer bulk-stores the P error tiles once every
// consumer warp has released the stage, before it refills it: the TMA engine,
// not the load/store units, carries that 4P bytes per element of writes. A
// one-rank launch (one handle per rank) with sender feedback sends its code
// words to the owners the same way.
//
// Algorithmic HBM bytes per element of n: P*b (partials) + 8 (f, s; each
// element is corrected by exactly one rank) read, P*17/32 written; sender
// feedback adds 4P read and 4P written. A one-rank launch (one handle per
// rank) reads the state of its own segment only: 8/P bytes per element.
#pragma once

#include "echo_bulk.cuh"
#include "echo_kernels.h"

#include <cuda_runtime.h>

#include <atomic>

// Included by k1_compensate_quantize_pack.cu (the default build) and by the
// k1_variants_*.cu files (the general build, split by element type and
// feedback setting so that they compile in parallel). Everything here has
// internal linkage in each of them.
namespace echo {
namespace {

// The kernel's three builds: the default one (groups of 32, power-of-two
// scales) and the general one, split into its power-of-two group sizes and
// its binary16-scale bodies, which get their own count of consumer warps.
enum K1Build { kDefaultBuild = 0, kGroupsBuild = 1, kHalfScaleBuild = 2 };

// Whether a build runs the wide binary16 body (k1_consume_wide).
__host__ __device__ constexpr bool k1_wide(int B, bool bf16, bool ef) { return B == kHalfScaleBuild && bf16 && !ef; }

template <int B, bool BF16, bool EF>
struct K1Warps {
    static constexpr int kConsumerWarps = k1_wide(B, BF16, EF) ? ECHO_K1_WARPS_HALF_WIDE
                                          : B == kHalfScaleBuild ? ECHO_K1_WARPS_HALF_SCALE
                                          : B == kGroupsBuild    ? ECHO_K1_WARPS_GROUPS
                                          : EF                   ? ECHO_K1_WARPS_SENDER_EF
                                                                 : ECHO_K1_WARPS;
    static constexpr int kConsumers = kConsumerWarps * 32;
    static constexpr int kThreads = kConsumers + 32; // + one producer warp
};

// Bytes one stage holds per element of the tile.
constexpr int k1_bytes_per_elem(int P, bool bf16, bool comp, bool ef)
{
    return P * (bf16 ? 2 : 4) + (comp ? 8 : 0) + (ef ? 4 * P : 0);
}

// The largest tile whose stages fit the CTA's budget (ECHO_K1_CTA_BUDGET;
// ECHO_K1_EF_BUDGET with sender feedback, whose stages are written back
// before they are refilled), from ECHO_K1_TILE (times 16 / (P * element
// bytes) when the P partials of an element take fewer than 16 bytes, so that
// a tile holds about as many partial bytes at small P) down to 256 elements.
constexpr int k1_tile(int P, bool bf16, bool comp, bool ef)
{
    const int xb = P * (bf16 ? 2 : 4);
    const int budget = ef ? ECHO_K1_EF_BUDGET : ECHO_K1_CTA_BUDGET;
    int t = xb < 16 ? ECHO_K1_TILE * (16 / xb) : ECHO_K1_TILE;
    // a one-rank tile with sender feedback also holds its code words (half a
    // byte per element)
    while (t > 256 && ECHO_K1_STAGES * (t * k1_bytes_per_elem(P, bf16, comp, ef) + (P == 1 && ef ? t / 2 : 0)) >
                          budget)
        t /= 2;
    return t;
}

template <int P, bool BF16, bool COMP, bool EF>
struct K1Shape {
    static constexpr int kEB = BF16 ? 2 : 4;
    static constexpr int kTile = k1_tile(P, BF16, COMP, EF);
    static constexpr int kStages = ECHO_K1_STAGES;
    static constexpr int kXBytes = kTile * kEB;             // one rank's partial tile
    static constexpr int kStateOff = P * kXBytes;           // f tile, then s tile
    static constexpr int kEpsOff = kStateOff + (COMP ? 2 * kTile * 4 : 0); // P error tiles
    static constexpr int kCodeOff = kEpsOff + (EF ? P * kTile * 4 : 0); // one rank, feedback: code words
    static constexpr int kStageBytes = kCodeOff + (P == 1 && EF ? kTile / 2 : 0);
    static constexpr int kSmem = kStages * kStageBytes + 2 * kStages * 8;
    static_assert(kSmem <= ECHO_SMEM_BUDGET, "kernel 1 stages exceed shared memory");
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

__device__ __forceinline__ void load_f32x8(const float *p, float (&v)[kChunk])
{
    const float4 a = reinterpret_cast<const float4 *>(p)[0];
    const float4 b = reinterpret_cast<const float4 *>(p)[1];
    v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w;
    v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
}

// The consumer warps' part of kernel 1 for a group of 8 << LANES elements and
// one scale format (F16: binary16 scales), both fixed at compile time, run by
// NC consumer threads.
template <int P, bool BF16, bool COMP, bool EF, uint32_t LANES, bool F16, int NC>
__device__ __forceinline__ void k1_consume(const K1Args &a, const uint8_t *smem, uint64_t *full, uint64_t *empty,
                                           uint32_t mine, uint32_t cpt_log2, size_t e0)
{
    using Sh = K1Shape<P, BF16, COMP, EF>;
    constexpr int S = Sh::kStages;
    constexpr uint32_t lanes_log2 = LANES;
    constexpr bool f16 = F16;
    const uint32_t tid = threadIdx.x;
    const uint32_t lane = tid & 31u;
    const uint32_t code_words = static_cast<uint32_t>(a.n / kChunk); // 32-bit code words per rank
    for (uint32_t i = 0; i < mine; i++) {
        const uint32_t s = i % S;
        if (!warp_wait(&full[s], (i / S) & 1u, a.ctl.wait_cycles, a.ctl.status, kStatusTimeoutK1))
            return;
        const uint32_t tile_chunk0 = static_cast<uint32_t>(e0 / kChunk) + ((blockIdx.x + i * gridDim.x) << cpt_log2);
        const uint32_t cnt_chunks = min(1u << cpt_log2, a.chunk_end - tile_chunk0);
        const uint8_t *stage = smem + s * Sh::kStageBytes;
        const float *fs = reinterpret_cast<const float *>(stage + Sh::kStateOff);
        // the error tiles: read, then overwritten in place with the new errors,
        // which the producer bulk-stores once the stage is released
        float *es = reinterpret_cast<float *>(const_cast<uint8_t *>(stage) + Sh::kEpsOff);

#pragma unroll 2
        for (uint32_t it = tid; it < (static_cast<uint32_t>(P) << cpt_log2); it += NC) {
            const uint32_t r = it >> cpt_log2; // warp-uniform (a tile has >= 32 chunks)
            const uint32_t c = it & ((1u << cpt_log2) - 1u);
            const bool active = c < cnt_chunks;
            const uint32_t chunk = tile_chunk0 + c;
            const uint32_t g = chunk >> lanes_log2;

            float v[kChunk];
            load_chunk<BF16>(stage + r * Sh::kXBytes + c * (kChunk * Sh::kEB), v);
            if (EF) { // add back this rank's own rounding-#1 error
                float e[kChunk];
                load_f32x8(es + r * Sh::kTile + c * kChunk, e);
#pragma unroll
                for (int k = 0; k < kChunk; k++)
                    v[k] = __fadd_rn(v[k], e[k]);
            }
            // bf16 partials keep 8 significant bits unless something is added
            bool short_vals = BF16 && !EF;
            // rank r owns groups [r*gps, (r+1)*gps): one unsigned range test
            if (COMP && g - (r + a.rank_base) * a.groups_per_seg < a.groups_per_seg) {
                short_vals = false;
                float fv[kChunk], sv[kChunk];
                load_f32x8(fs + c * kChunk, fv);
                load_f32x8(fs + Sh::kTile + c * kChunk, sv);
#pragma unroll
                for (int k = 0; k < kChunk; k++)
                    v[k] = __fadd_rn(v[k], __fadd_rn(__fmul_rn(a.lambda, fv[k]),
                                                     __fmul_rn(a.one_minus_lambda, sv[k])));
            }
            // max |v| as a tree (fmax is exact, so the order is free)
            const float amax = group_absmax(absmax8(v), lanes_log2);
            uint32_t qb[kChunk];
            uint32_t scale; // scale byte, or binary16 pattern
            float st;       // the step q is restored with
            if (f16) {
                scale = half_scale_bits(amax);
                st = half_step(scale);
                const float inv = half_inv(st);
                const float half = __fmul_rn(0.5f, st);
                codes8_half(v, st, inv, half, half_scale_saturates(amax), short_vals, qb);
            } else {
                scale = scale_byte(amax);
                st = step_of(scale);
                const float inv = inv_step_of(scale);
#pragma unroll
                for (int k = 0; k < kChunk; k++)
                    qb[k] = code_bits(v[k], inv);
            }
            const uint32_t word = f16 ? pack8_zcodes(qb) : pack8_bits(qb); // binary16: z-form codes
            if (P == 1 && a.to_owners) {
                // one handle per rank: into the owner's receive block. With
                // sender feedback the producer already bulk-stores the error
                // tiles from the released stage, so the code words go that way
                // too; otherwise each lane stores its own (a stage waiting for
                // its stores measured slower there).
                const uint32_t owner = g / a.groups_per_seg;
                const uint32_t gl = g - owner * a.groups_per_seg;               // group in the segment
                const uint32_t cl = chunk - ((owner * a.groups_per_seg) << lanes_log2); // chunk in the segment
                if (EF && active)
                    reinterpret_cast<uint32_t *>(const_cast<uint8_t *>(stage) + Sh::kCodeOff)[c] = word;
                if (active && in_bounds(owner < kMaxRanks && (size_t(gl) + 1) * (f16 ? 2u : 1u) <= a.seg_scale_stride &&
                                            (size_t(cl) + 1) * 4u <= a.seg_code_bytes,
                                        a.ctl.status)) {
                    uint8_t *blk = static_cast<uint8_t *>(a.owners.p[owner]);
                    if (!EF)
                        reinterpret_cast<uint32_t *>(blk + a.rank_base * a.seg_code_bytes)[cl] = word;
                    if ((lane & ((1u << lanes_log2) - 1u)) == 0) { // the group's first lane
                        uint8_t *row = blk + a.recv_scales_off + a.rank_base * a.seg_scale_stride;
                        if (f16)
                            reinterpret_cast<uint16_t *>(row)[gl] = static_cast<uint16_t>(scale);
                        else
                            row[gl] = static_cast<uint8_t>(scale);
                    }
                }
            } else if (active && in_bounds(chunk < code_words && (g + 1) * (f16 ? 2u : 1u) <= a.scale_stride,
                                           a.ctl.status)) {
                reinterpret_cast<uint32_t *>(a.codes)[static_cast<size_t>(r) * code_words + chunk] = word;
                if ((lane & ((1u << lanes_log2) - 1u)) == 0) { // the group's first lane
                    uint8_t *row = a.scales + static_cast<size_t>(r) * a.scale_stride;
                    if (f16)
                        reinterpret_cast<uint16_t *>(row)[g] = static_cast<uint16_t>(scale);
                    else
                        row[g] = static_cast<uint8_t>(scale);
                }
            }
            if (EF && active) {
                // the new error v - q*step (exact unless a binary16 scale saturated),
                // over the old one in the stage
                float en[kChunk];
#pragma unroll
                for (int k = 0; k < kChunk; k++)
                    en[k] = __fmaf_rn(-code_value(f16 ? zcode_bits(qb[k]) : qb[k]), st, v[k]);
                float4 *eo = reinterpret_cast<float4 *>(es + r * Sh::kTile + c * kChunk);
                eo[0] = make_float4(en[0], en[1], en[2], en[3]);
                eo[1] = make_float4(en[4], en[5], en[6], en[7]);
            }
        }
        if (EF)
            fence_proxy_async_smem(); // read next by the producer's bulk stores
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[s]); // this warp is done with stage s
    }
}

// The consumer body for binary16 scales with bf16 partials and no sender
// feedback. That body is bound by instruction issue, not by HBM, so here a
// lane owns 16 consecutive elements (two code words) of one rank, and the
// work a lane does once per unit (its indices, the group maximum's shuffles,
// the scale with its step and reciprocal, the stores) is spent once per 16
// elements instead of once per 8. A group of 8 << LANES elements spans
// 2^LANES / 2 lanes. The lane reads its 32 bytes of partials as two 16-byte
// halves, half sw = (lane >> 2) & 1 first, so the 8 lanes of each
// shared-memory phase cover the 32 banks once; row 0 of its values (and of
// the state it adds) is chunk c + sw of the unit, row 1 the other chunk, and
// the two code words are put back in element order for one 8-byte store.
template <int P, bool COMP, uint32_t LANES, int NC>
__device__ __forceinline__ void k1_consume_wide(const K1Args &a, const uint8_t *smem, uint64_t *full,
                                                uint64_t *empty, uint32_t mine, uint32_t cpt_log2, size_t e0)
{
    using Sh = K1Shape<P, true, COMP, false>;
    constexpr int S = Sh::kStages;
    constexpr uint32_t lanes_log2 = LANES;     // log2(G / 8)
    constexpr uint32_t glanes = (1u << LANES) / 2; // lanes per group
    const uint32_t tid = threadIdx.x;
    const uint32_t lane = tid & 31u;
    const uint32_t sw = (lane >> 2) & 1u;
    const uint32_t upt_log2 = cpt_log2 - 1; // 16-element units per tile = 2^upt_log2
    const uint32_t code_words = static_cast<uint32_t>(a.n / kChunk);
    for (uint32_t i = 0; i < mine; i++) {
        const uint32_t s = i % S;
        if (!warp_wait(&full[s], (i / S) & 1u, a.ctl.wait_cycles, a.ctl.status, kStatusTimeoutK1))
            return;
        const uint32_t tile_chunk0 = static_cast<uint32_t>(e0 / kChunk) + ((blockIdx.x + i * gridDim.x) << cpt_log2);
        const uint32_t cnt_chunks = min(1u << cpt_log2, a.chunk_end - tile_chunk0); // even
        const uint8_t *stage = smem + s * Sh::kStageBytes;
        const float *fs = reinterpret_cast<const float *>(stage + Sh::kStateOff);

#pragma unroll 1 // an item is 16 elements: unrolling by 2 measured the same
        for (uint32_t it = tid; it < (static_cast<uint32_t>(P) << upt_log2); it += NC) {
            const uint32_t r = it >> upt_log2; // warp-uniform (a tile has >= 32 units)
            const uint32_t c = (it & ((1u << upt_log2) - 1u)) << 1; // the unit's first chunk
            const bool active = c < cnt_chunks;
            const uint32_t chunk = tile_chunk0 + c;
            const uint32_t g = chunk >> lanes_log2;

            const uint8_t *xp = stage + r * Sh::kXBytes + c * (kChunk * 2);
            float v[2][kChunk];
            bf16x8_to_f32(*reinterpret_cast<const uint4 *>(xp + 16u * sw), v[0]);
            bf16x8_to_f32(*reinterpret_cast<const uint4 *>(xp + 16u * (sw ^ 1u)), v[1]);
            bool short_vals = true; // bf16 partials keep 8 significant bits unless corrected
            if (COMP && g - (r + a.rank_base) * a.groups_per_seg < a.groups_per_seg) {
                short_vals = false;
#pragma unroll
                for (uint32_t h = 0; h < 2; h++) {
                    float fv[kChunk], sv[kChunk];
                    load_f32x8(fs + (c + (sw ^ h)) * kChunk, fv);
                    load_f32x8(fs + Sh::kTile + (c + (sw ^ h)) * kChunk, sv);
#pragma unroll
                    for (int k = 0; k < kChunk; k++)
                        v[h][k] = __fadd_rn(v[h][k], __fadd_rn(__fmul_rn(a.lambda, fv[k]),
                                                               __fmul_rn(a.one_minus_lambda, sv[k])));
                }
            }
            const float amax = group_absmax(absmax16(v[0], v[1]), lanes_log2 - 1);
            const uint32_t scale = half_scale_bits(amax);
            const float st = half_step(scale);
            const float inv = half_inv(st);
            const float half = __fmul_rn(0.5f, st);
            const bool sat = half_scale_saturates(amax);
            uint32_t z[kChunk];
            codes8_half(v[0], st, inv, half, sat, short_vals, z);
            const uint32_t w0 = pack8_zcodes(z);
            codes8_half(v[1], st, inv, half, sat, short_vals, z);
            const uint32_t w1 = pack8_zcodes(z);
            const uint2 words = sw ? make_uint2(w1, w0) : make_uint2(w0, w1); // chunks c, c + 1
            const bool first = (lane & (glanes - 1u)) == 0; // the group's first lane
            if (P == 1 && a.to_owners) {
                // one handle per rank: into the owner's receive block
                const uint32_t owner = g / a.groups_per_seg;
                const uint32_t gl = g - owner * a.groups_per_seg;               // group in the segment
                const uint32_t cl = chunk - ((owner * a.groups_per_seg) << lanes_log2); // chunk in the segment
                if (active && in_bounds(owner < kMaxRanks && (size_t(gl) + 1) * 2u <= a.seg_scale_stride &&
                                            (size_t(cl) + 2) * 4u <= a.seg_code_bytes,
                                        a.ctl.status)) {
                    uint8_t *blk = static_cast<uint8_t *>(a.owners.p[owner]);
                    reinterpret_cast<uint2 *>(blk + a.rank_base * a.seg_code_bytes)[cl / 2] = words;
                    if (first)
                        reinterpret_cast<uint16_t *>(blk + a.recv_scales_off +
                                                     a.rank_base * a.seg_scale_stride)[gl] =
                            static_cast<uint16_t>(scale);
                }
            } else if (active && in_bounds(chunk + 2 <= code_words && (g + 1) * 2u <= a.scale_stride, a.ctl.status)) {
                reinterpret_cast<uint2 *>(a.codes)[(static_cast<size_t>(r) * code_words + chunk) / 2] = words;
                if (first)
                    reinterpret_cast<uint16_t *>(a.scales + static_cast<size_t>(r) * a.scale_stride)[g] =
                        static_cast<uint16_t>(scale);
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[s]); // this warp is done with stage s
    }
}

template <int P, bool BF16, bool COMP, bool EF, int B>
__global__ void __launch_bounds__(K1Warps<B, BF16, EF>::kThreads, 2)
    k1_compensate_quantize_pack(const K1Args a)
{
    using Sh = K1Shape<P, BF16, COMP, EF>;
    constexpr int kConsumerWarps = K1Warps<B, BF16, EF>::kConsumerWarps;
    constexpr int NC = K1Warps<B, BF16, EF>::kConsumers;
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
    const uint32_t cpt_log2 = a.tile_log2 - 3; // chunks per tile = 2^cpt_log2
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
        // The state holds the elements this launch's ranks own, [state_lo,
        // state_lo + P*seg): all n for P simulated ranks, one segment for a
        // one-rank launch. Only the part of a tile inside it is loaded.
        const size_t seg = static_cast<size_t>(a.groups_per_seg) << (a.lanes_log2 + 3);
        const size_t state_lo = static_cast<size_t>(a.rank_base) * seg;
        const size_t state_hi = state_lo + static_cast<size_t>(P) * seg;
        auto issue = [&](uint32_t i) {
            const size_t el0 = e0 + static_cast<size_t>(blockIdx.x + i * gridDim.x) * tile;
            const uint32_t cnt = static_cast<uint32_t>(e1 - el0 < size_t(tile) ? e1 - el0 : tile);
            uint8_t *stage = smem + (i % S) * Sh::kStageBytes;
            uint64_t *bar = &full[i % S];
            // the partial and error copies cover elements [el0, el0 + cnt) of an
            // n-element row; the state copies [lo, hi), its part inside the state
            const size_t lo = el0 > state_lo ? el0 : state_lo;
            const size_t hi = el0 + cnt < state_hi ? el0 + cnt : state_hi;
            const uint32_t sn = COMP && hi > lo ? static_cast<uint32_t>(hi - lo) : 0u;
            const bool ok = in_bounds(el0 + cnt <= a.n && cnt <= Sh::kTile, a.ctl.status);
            mbar_arrive_expect_tx(
                bar, ok ? cnt * (P * Sh::kEB + (EF ? 4u * P : 0u)) + 8u * sn : 0u);
            if (!ok)
                return;
#pragma unroll
            for (int r = 0; r < P; r++)
                bulk_load(stage + r * Sh::kXBytes,
                          static_cast<const uint8_t *>(a.x.p[r]) + el0 * Sh::kEB,
                          cnt * Sh::kEB, bar);
            if (COMP && sn) {
                const size_t off = (lo - el0) * 4;
                bulk_load(stage + Sh::kStateOff + off, a.f + (lo - state_lo), sn * 4, bar);
                bulk_load(stage + Sh::kStateOff + Sh::kTile * 4 + off, a.s + (lo - state_lo),
                          sn * 4, bar);
            }
            if (EF) {
#pragma unroll
                for (int r = 0; r < P; r++)
                    bulk_load(stage + Sh::kEpsOff + r * Sh::kTile * 4,
                              a.eps + static_cast<size_t>(r) * a.n + el0, cnt * 4, bar);
            }
        };
        // With sender feedback, what the consumers leave in a released stage
        // goes out by bulk stores: the new errors, and with one handle per
        // rank the code words, into each owner's receive block for the part of
        // the tile in its segment (segment bounds are multiples of 32
        // elements, so every piece starts on 16 bytes).
        auto writeback = [&](uint32_t t) {
            const size_t el0 = e0 + static_cast<size_t>(blockIdx.x + t * gridDim.x) * tile;
            const uint32_t cnt = static_cast<uint32_t>(e1 - el0 < size_t(tile) ? e1 - el0 : tile);
            const uint8_t *stage = smem + (t % S) * Sh::kStageBytes;
            if (!in_bounds(el0 + cnt <= a.n && cnt <= Sh::kTile, a.ctl.status))
                return;
            if constexpr (EF) {
#pragma unroll
                for (int r = 0; r < P; r++)
                    bulk_store(a.eps + static_cast<size_t>(r) * a.n + el0, stage + Sh::kEpsOff + r * Sh::kTile * 4,
                               cnt * 4);
            }
            if constexpr (P == 1 && EF) {
                if (a.to_owners) {
                    for (size_t lo = el0; lo < el0 + cnt;) {
                        const size_t owner = lo / seg;
                        const size_t hi = el0 + cnt < (owner + 1) * seg ? el0 + cnt : (owner + 1) * seg;
                        if (in_bounds(owner < kMaxRanks && (lo - owner * seg + (hi - lo)) / 2 <= a.seg_code_bytes,
                                      a.ctl.status))
                            bulk_store(static_cast<uint8_t *>(a.owners.p[owner]) + a.rank_base * a.seg_code_bytes +
                                           (lo - owner * seg) / 2,
                                       stage + Sh::kCodeOff + (lo - el0) / 2, static_cast<uint32_t>(hi - lo) / 2);
                        lo = hi;
                    }
                }
            }
        };
        if (lane == 0) {
            if constexpr (EF)
                produce_tiles_writeback<S>(full, empty, mine, a.ctl.stall, a.ctl.wait_cycles, a.ctl.status,
                                           kStatusTimeoutK1, issue, writeback);
            else
                produce_tiles<S>(full, empty, mine, a.ctl.stall, a.ctl.wait_cycles, a.ctl.status, kStatusTimeoutK1,
                                 issue);
        }
        return;
    }

    if constexpr (B == kDefaultBuild) {
        k1_consume<P, BF16, COMP, EF, 2u, false, NC>(a, smem, full, empty, mine, cpt_log2, e0);
    } else if constexpr (B == kGroupsBuild) {
        // one switch per launch selects the compile-time group size (8 << lanes_log2)
        switch (a.lanes_log2) {
        case 1u: k1_consume<P, BF16, COMP, EF, 1u, false, NC>(a, smem, full, empty, mine, cpt_log2, e0); break;
        case 3u: k1_consume<P, BF16, COMP, EF, 3u, false, NC>(a, smem, full, empty, mine, cpt_log2, e0); break;
        case 4u: k1_consume<P, BF16, COMP, EF, 4u, false, NC>(a, smem, full, empty, mine, cpt_log2, e0); break;
        default: break; // the host accepts no other group size
        }
    } else if constexpr (k1_wide(B, BF16, EF)) {
        switch (a.lanes_log2) {
        case 1u: k1_consume_wide<P, COMP, 1u, NC>(a, smem, full, empty, mine, cpt_log2, e0); break;
        case 2u: k1_consume_wide<P, COMP, 2u, NC>(a, smem, full, empty, mine, cpt_log2, e0); break;
        case 3u: k1_consume_wide<P, COMP, 3u, NC>(a, smem, full, empty, mine, cpt_log2, e0); break;
        case 4u: k1_consume_wide<P, COMP, 4u, NC>(a, smem, full, empty, mine, cpt_log2, e0); break;
        default: break;
        }
    } else {
        switch (a.lanes_log2) {
        case 1u: k1_consume<P, BF16, COMP, EF, 1u, true, NC>(a, smem, full, empty, mine, cpt_log2, e0); break;
        case 2u: k1_consume<P, BF16, COMP, EF, 2u, true, NC>(a, smem, full, empty, mine, cpt_log2, e0); break;
        case 3u: k1_consume<P, BF16, COMP, EF, 3u, true, NC>(a, smem, full, empty, mine, cpt_log2, e0); break;
        case 4u: k1_consume<P, BF16, COMP, EF, 4u, true, NC>(a, smem, full, empty, mine, cpt_log2, e0); break;
        default: break;
        }
    }
}

template <int P, bool BF16, bool COMP, bool EF, int B>
cudaError_t launch_p(const K1Args &a, cudaStream_t st)
{
    using Sh = K1Shape<P, BF16, COMP, EF>;
    constexpr int kThreads = K1Warps<B, BF16, EF>::kThreads;
    // Every consumer loop runs over a whole warp's items or none, so that the
    // group shuffles see all 32 lanes: a tile holds at least 32 items of each
    // rank (chunks of 8 elements; units of 16 in the wide binary16 body).
    constexpr int kMinTile = k1_wide(B, BF16, EF) ? 512 : 256;
    static_assert(Sh::kTile >= kMinTile, "kernel 1 tile below a warp's items");
    // CTAs per SM of this instantiation, found once (threads that race here
    // compute the same value)
    static std::atomic<int> cached{0};
    int resident = cached.load(std::memory_order_relaxed);
    auto kern = k1_compensate_quantize_pack<P, BF16, COMP, EF, B>;
    if (resident == 0) {
        cudaError_t e = prepare_kernel(reinterpret_cast<const void *>(kern), kThreads, Sh::kSmem, &resident);
        if (e != cudaSuccess)
            return e;
        cached.store(resident, std::memory_order_relaxed);
    }
    const size_t elems = static_cast<size_t>(a.chunk_end - a.chunk_begin) * kChunk;
    K1Args b = a;
    b.tile_log2 = pick_tile_log2(elems, Sh::kTile, kMinTile, resident);
    b.tile = 1u << b.tile_log2;
    const uint32_t tiles = static_cast<uint32_t>((elems + b.tile - 1) >> b.tile_log2);
    return launch_chained(kern, persistent_grid(tiles, resident), kThreads, Sh::kSmem, st, b);
}

template <int P, bool BF16, bool EF, int B>
cudaError_t dispatch_state(const K1Args &a, cudaStream_t st)
{
    return a.enable ? launch_p<P, BF16, true, EF, B>(a, st) : launch_p<P, BF16, false, EF, B>(a, st);
}

// One element type, feedback setting and build of the kernel, over P.
template <bool BF16, bool EF, int B>
cudaError_t dispatch_ranks(const K1Args &a, cudaStream_t st)
{
    switch (a.P) {
    case 1: return dispatch_state<1, BF16, EF, B>(a, st); // one rank per process
    case 2: return dispatch_state<2, BF16, EF, B>(a, st);
    case 3: return dispatch_state<3, BF16, EF, B>(a, st);
    case 4: return dispatch_state<4, BF16, EF, B>(a, st);
    case 5: return dispatch_state<5, BF16, EF, B>(a, st);
    case 6: return dispatch_state<6, BF16, EF, B>(a, st);
    case 7: return dispatch_state<7, BF16, EF, B>(a, st);
    case 8: return dispatch_state<8, BF16, EF, B>(a, st);
    case 9: return dispatch_state<9, BF16, EF, B>(a, st);
    case 10: return dispatch_state<10, BF16, EF, B>(a, st);
    case 11: return dispatch_state<11, BF16, EF, B>(a, st);
    case 12: return dispatch_state<12, BF16, EF, B>(a, st);
    case 13: return dispatch_state<13, BF16, EF, B>(a, st);
    case 14: return dispatch_state<14, BF16, EF, B>(a, st);
    case 15: return dispatch_state<15, BF16, EF, B>(a, st);
    case 16: return dispatch_state<16, BF16, EF, B>(a, st);
    default: return cudaErrorInvalidValue;
    }
}

// The general build: the power-of-two group sizes or the binary16 bodies.
template <bool BF16, bool EF>
cudaError_t dispatch_variant(const K1Args &a, cudaStream_t st)
{
    return a.fp16_scale ? dispatch_ranks<BF16, EF, kHalfScaleBuild>(a, st)
                        : dispatch_ranks<BF16, EF, kGroupsBuild>(a, st);
}

} // namespace
} // namespace echo
