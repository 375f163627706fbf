// echo_kernels.h - launchers of the three kernels of the Echo all-reduce.
//
// A launch covers elements [8*chunk_begin, 8*chunk_end) of the n elements
// (the whole tensor, or one slice of it when host transfers are pipelined);
// both bounds are multiples of 32, so no group is split. Each kernel is a
// persistent grid of CTAs that take tiles of consecutive elements in turn;
// tiles move between HBM and shared memory with bulk copies (echo_bulk.cuh).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "echo_codec.cuh"

// Pipeline shapes, chosen by sweeping on B200 at P = 8, 1 GiB per rank
// (larger bulk copies win as long as two CTAs fit on an SM).
// ECHO_K1_TILE is kernel 1's tile length in elements when the P partials of
// an element take 16 bytes (longer below, shorter beyond, within the CTA's
// shared-memory budget).
// ECHO_K2_CHUNKS is kernel 2's chunks of 8 elements per consumer thread per
// tile, reduced for large P so that ECHO_K2_STAGES stages fit in shared
// memory; a reduced tile then takes as many stages as fit, up to
// ECHO_K2_MAX_STAGES. ECHO_K3_TILE is kernel 3's bf16 tile (halved for binary32).
#ifndef ECHO_K1_TILE
#define ECHO_K1_TILE 2048
#endif
#ifndef ECHO_K1_STAGES
#define ECHO_K1_STAGES 2
#endif
// Kernel 1's consumer warps: the default build (bound by HBM; 16 warps
// measured 1 to 7 % slower), the power-of-two group-size variants, the
// binary16-scale variants, and the default group with sender feedback. The
// last three have longer chains per item (more shuffles for large groups; the
// binary16 scale, reciprocal and code settling; the error tiles' loads and
// stores) and want more warps per SM to hide them. The binary16 body for bf16
// partials without sender feedback (16 elements per lane) has twice the work
// per item, and 8 warps measured as fast as 12 and faster than 16.
#ifndef ECHO_K1_WARPS
#define ECHO_K1_WARPS 8
#endif
#ifndef ECHO_K1_WARPS_GROUPS
#define ECHO_K1_WARPS_GROUPS 16
#endif
#ifndef ECHO_K1_WARPS_SENDER_EF
#define ECHO_K1_WARPS_SENDER_EF 16
#endif
#ifndef ECHO_K1_WARPS_HALF_SCALE
#define ECHO_K1_WARPS_HALF_SCALE 16
#endif
#ifndef ECHO_K1_WARPS_HALF_WIDE
#define ECHO_K1_WARPS_HALF_WIDE 8
#endif
#ifndef ECHO_K2_STAGES
#define ECHO_K2_STAGES 2
#endif
#ifndef ECHO_K2_CHUNKS
#define ECHO_K2_CHUNKS 4
#endif
#ifndef ECHO_K2_MAX_STAGES
#define ECHO_K2_MAX_STAGES 3
#endif
#ifndef ECHO_K3_TILE
#define ECHO_K3_TILE 16384
#endif
#ifndef ECHO_K3_IN_STAGES
#define ECHO_K3_IN_STAGES 4
#endif
#ifndef ECHO_K3_OUT_BUFS
#define ECHO_K3_OUT_BUFS 2
#endif
// Largest n per rank whose calls run as one kernel (kf_fused_allreduce) by
// default; larger calls run the three pipelined kernels. At P = 8, bf16, the
// one kernel took 4.1 to 9.4 us per call up to 2^20 elements per rank, against
// 6.6 to 18.2 us, where the three launches set the pipelined kernels' time.
// Past that the one kernel's lead comes mostly from skipping the wire
// read-back that one GPU allows and P GPUs do not, so the pipelined kernels
// keep the larger calls.
#ifndef ECHO_FUSED_LIMIT
#define ECHO_FUSED_LIMIT (static_cast<size_t>(1) << 20)
#endif
// Shared memory one CTA may use (the B200 limit is 227 KB), and kernel 1's
// budget per CTA so that two CTAs share an SM.
#define ECHO_SMEM_BUDGET (225 * 1024)
#ifndef ECHO_K1_CTA_BUDGET
#define ECHO_K1_CTA_BUDGET (100 * 1024)
#endif
// With sender feedback a stage is written back before it is refilled, and
// stages of at most 32 KB measured best: both feedbacks at P = 8 took 7.12
// against 7.42 ms with 512- instead of 1024-element tiles (48 KB stages),
// sender feedback alone at P = 2 to 8 kept its time.
#ifndef ECHO_K1_EF_BUDGET
#define ECHO_K1_EF_BUDGET (64 * 1024)
#endif

namespace echo {

// Pipeline controls shared by the three kernels.
struct PipeCtl {
    int *status;           // device status word (kStatusTimeout* bits)
    long long wait_cycles; // bound of every wait, in SM clock cycles
    bool stall;            // test hook: issue no loads, so every wait runs out
};

struct K1Args {
    RankPtrs x;              // P rank partials (bf16 or binary32), n elements each
    const float *f;          // phase state, fast estimate, of the elements the launch's ranks
    const float *s;          // own, from rank_base's segment on: [n] for P ranks, [n/P] for one
    uint8_t *codes;          // stage-1 wire codes [P][n/2]
    uint8_t *scales;         // stage-1 wire scales [P][scale_stride]: n/G bytes or binary16s per rank
    size_t n;
    size_t scale_stride;     // bytes between ranks' scale rows (2n/G rounded up to 16)
    uint32_t chunk_begin, chunk_end;
    uint32_t tile, tile_log2; // set by the launcher: this launch's tile length
    uint32_t lanes_log2;     // log2(G / 8): lanes per group
    uint32_t groups_per_seg; // n / P / G: owner of group g is g / groups_per_seg
    uint32_t rank_base;      // global rank of partial 0 (a one-rank launch of a process
                             // that holds one rank of a larger group; 0 otherwise)
    // One handle per rank (P == 1 launches only): the stage-1 row goes
    // straight to the owners. Segment s lands in owner s's receive block
    // owners.p[s], in the slot of rank rank_base: codes at
    // rank_base * seg_code_bytes, scales at recv_scales_off + rank_base *
    // seg_scale_stride.
    bool to_owners;
    RankOutPtrs owners;
    size_t seg_code_bytes, recv_scales_off, seg_scale_stride;
    float lambda, one_minus_lambda;
    float *eps;              // sender feedback: every rank's rounding-#1 error [P][n]
    int P;
    bool bf16;
    bool enable;             // the owner adds the correction to its partial
    bool sender_ef;          // every rank adds back and renews its own error
    bool fp16_scale;         // binary16 scales (rounded up) instead of powers of two
    PipeCtl ctl;
};

struct K2Args {
    const uint8_t *codes;    // stage-1 wire [P][n/2]
    const uint8_t *scales;   // [P][scale_stride]
    uint8_t *qcodes;         // requantised total [n/2]
    uint8_t *qscales;        // [scale_stride]
    float *f, *s;            // phase state, updated in place
    size_t n;
    size_t scale_stride;
    uint32_t chunk_begin, chunk_end;
    uint32_t tile, tile_log2; // set by the launcher: this launch's tile length
    uint32_t lanes_log2;     // log2(G / 8): lanes per group
    float beta_f, one_minus_beta_f, beta_s, one_minus_beta_s;
    float lambda, one_minus_lambda;
    int P;
    bool enable;             // read the state, capture the error, update the state
    bool owner_sum;          // add the correction to the owner's sum
    bool fp16_scale;         // binary16 scales
    bool bf16;               // bf16 outputs: under binary16 scales the error is
                             // taken against the bf16-rounded value ranks receive
    // One handle per rank: the requantised segment goes straight to every
    // rank's gathered buffer ranks.p[r] (codes from word q_chunk0, scales at
    // q_scales_off + q_group0 scales), instead of qcodes / qscales.
    bool to_ranks;
    RankOutPtrs ranks;
    uint32_t q_chunk0, q_group0;
    size_t q_scales_off, q_scale_bytes; // where the scales start, and their room
    PipeCtl ctl;
};

struct K3Args {
    const uint8_t *qcodes;
    const uint8_t *qscales;  // [scale_stride]
    RankOutPtrs out;         // P rank outputs (bf16 or binary32)
    size_t n;
    size_t scale_stride;
    uint32_t chunk_begin, chunk_end;
    uint32_t tile, tile_log2; // set by the launcher: this launch's tile length
    uint32_t lanes_log2;     // log2(G / 8): lanes per group
    int P;
    bool bf16;
    bool fp16_scale;         // binary16 scales: outputs q*s rounded to bf16 when bf16
    PipeCtl ctl;
};

// The whole call as one kernel (small messages): every argument of the three
// kernels' simulated-rank launches, over one element range.
struct KFArgs {
    RankPtrs x;              // P rank partials (bf16 or binary32), n elements each
    RankOutPtrs out;         // P rank outputs (may equal x: in place)
    float *f, *s;            // phase state [n], read and updated in place
    float *eps;              // sender feedback: every rank's rounding-#1 error [P][n]
    uint8_t *codes;          // stage-1 wire codes [P][n/2]
    uint8_t *scales;         // stage-1 wire scales [P][scale_stride]
    uint8_t *qcodes;         // requantised total [n/2]
    uint8_t *qscales;        // [scale_stride]
    size_t n;
    size_t scale_stride;
    uint32_t chunk_begin, chunk_end;
    uint32_t lanes_log2;     // log2(G / 8): lanes per group
    uint32_t groups_per_seg; // n / P / G: owner of group g is g / groups_per_seg
    float lambda, one_minus_lambda;
    float beta_f, one_minus_beta_f, beta_s, one_minus_beta_s;
    int P;
    bool bf16;
    bool enable;             // compensation: state read, error captured, state updated
    bool owner_sum;          // the correction enters the owner's sum (else the owner's partial)
    bool sender_ef;          // every rank adds back and renews its own rounding-#1 error
    bool fp16_scale;         // binary16 scales
    PipeCtl ctl;
};

// Guard bytes around the library's device buffers (debug build only).
constexpr size_t kGuardBytes = 256;
constexpr uint8_t kGuardByte = 0xA5;
constexpr int kMaxGuards = 16;
struct GuardList {
    const uint8_t *region[kMaxGuards]; // kGuardBytes each
    int count;
};
cudaError_t launch_check_guards(const GuardList &g, int *status, cudaStream_t st);

// Each returns the launch's cudaError_t (cudaSuccess when enqueued).
cudaError_t launch_k1_compensate_quantize_pack(const K1Args &a, cudaStream_t st);
// The general build of kernel 1 (group size and scale format at run time),
// one function per element type and sender-feedback setting; called by
// launch_k1_compensate_quantize_pack for the variants.
cudaError_t launch_k1_variant_bf16(const K1Args &a, cudaStream_t st);
cudaError_t launch_k1_variant_bf16_ef(const K1Args &a, cudaStream_t st);
cudaError_t launch_k1_variant_fp32(const K1Args &a, cudaStream_t st);
cudaError_t launch_k1_variant_fp32_ef(const K1Args &a, cudaStream_t st);
cudaError_t launch_k2_owner_reduce_requant(const K2Args &a, cudaStream_t st);
cudaError_t launch_k3_gather_dequant(const K3Args &a, cudaStream_t st);
cudaError_t launch_kf_fused_allreduce(const KFArgs &a, cudaStream_t st);

// Persistent grid: one CTA per tile up to (SMs x resident CTAs per SM).
int persistent_grid(uint32_t tiles, int resident_per_sm);

// log2 of a launch's tile length: the largest power of two in
// [min_tile, max_tile] that still gives every CTA of a full persistent grid
// about four tiles, so mid-sized tensors keep the pipelines fed and balanced.
uint32_t pick_tile_log2(size_t elems, int max_tile, int min_tile, int resident_per_sm);

// Set a kernel's dynamic shared memory and return its resident CTAs per SM
// (cached by the caller per instantiation).
cudaError_t prepare_kernel(const void *kernel, int threads, int smem_bytes, int *resident);

// Record `message` as this thread's last error (echo_last_error /
// echo_last_status) and return `code`.
int record_error(int code, const char *message);

// Launch `kern` with programmatic stream serialisation: it may begin (set up
// its barriers) while the previous kernel in the stream finishes; the kernel
// itself waits (wait_for_predecessor) before touching global memory.
template <typename Arg>
cudaError_t launch_chained(void (*kern)(Arg), int grid, int threads, int smem, cudaStream_t st, const Arg &a)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

} // namespace echo
