/*
 * echo.h - C ABI of libecho.so: Echo's error-compensated 4-bit all-reduce on
 * one B200 (sm_100a).
 *
 * The method [rit.work "Echo 4-bit GPU communication", section "How Echo
 * returns the error to later calls"; heraldofai.com "Come Echo permette ai
 * modelli AI...", section "Come Echo evita che gli errori si accumulino"]:
 * tensor-parallel ranks hold partial sums of one tensor; each rank sends its
 * segments as 4-bit integers to the segment's owner; the owner restores them,
 * adds them in high precision, requantises the total to 4 bits and sends it
 * back to every rank, so each element is rounded at most twice whatever the
 * number of ranks. The owner measures the error of its rounding from the
 * high-precision sum and folds it into two smoothed estimates (fast, slow),
 * kept separately for the forward and the backward pass, that correct later
 * calls.
 *
 * On one GPU the P ranks are P device buffers in the same HBM and the "wire"
 * is the packed 4-bit buffers the ranks write and read; the bytes that would
 * cross a link are counted (echo_stats), not sent.
 *
 * Fixed readings of what the pages leave open (every entry point follows
 * them; echo_create's group and echo_set_variant select the variants listed
 * there): group of G = 32 consecutive elements; scale 2^e stored as the byte
 * e+127, e the smallest integer >= -127 with max|v| <= 7*2^e; codes
 * round(v/2^e) with halves to even, in [-7, 7], two per byte (element 2j in
 * the low nibble); rank s owns the contiguous segment [s*n/P, (s+1)*n/P) and
 * only it adds the correction c = lambda*f + (1-lambda)*s_est to its partial
 * before rounding #1; the owner sums in binary32, rank 0 first; the captured
 * error is err = S - Y; f <- beta_f*f + (1-beta_f)*err and
 * s_est <- beta_s*s_est + (1-beta_s)*err; every product and sum rounded to
 * binary32 on its own, subnormals kept. Defaults: lambda = 1/2, beta_f = 1/2,
 * beta_s = 7/8, compensation on. Inputs must be finite with |x| < 2^120.
 *
 * Conventions for every entry point:
 *   - "stream" is a cudaStream_t passed as void* (NULL: the legacy default
 *     stream). Work is enqueued on it; calls on one handle must be ordered on
 *     streams by the caller (they share the handle's state and wire).
 *   - Device pointers are CUDA device addresses on the current device; host
 *     pointers are ordinary (preferably page-locked) host memory.
 *   - Return: ECHO_OK (0) or a negative ECHO_ERR_* code; on error nothing is
 *     enqueued and no state changes, and echo_last_error() describes it.
 *     No entry point aborts or traps.
 */
#ifndef ECHO_H
#define ECHO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#ifndef ECHO_API
#define ECHO_API __attribute__((visibility("default")))
#endif

typedef struct echo_handle echo_handle; /* opaque, owned by the library */

typedef enum { ECHO_BF16 = 0, ECHO_FP32 = 1 } echo_dtype;
typedef enum { ECHO_FWD = 0, ECHO_BWD = 1 } echo_phase;

enum {
    ECHO_OK = 0,
    ECHO_ERR_INVALID = -1,     /* bad argument: nothing enqueued */
    ECHO_ERR_UNSUPPORTED = -2, /* valid but not built (group not 16/32/64/128, n too large) */
    ECHO_ERR_CUDA = -3,        /* a CUDA runtime call failed; message has its string */
    ECHO_ERR_OOM = -4          /* device allocation failed */
};

#define ECHO_MAX_RANKS 16
#define ECHO_GROUP 32

/*
 * echo_create - a handle for all-reduces of P ranks x n elements of dtype.
 * Defined by [rit.work "Echo 4-bit GPU communication", section "How Echo
 * returns the error to later calls"]: P tensor-parallel ranks each hold a
 * partial sum of the same tensor, cut into P segments with one owner each;
 * the handle holds the wire those ranks exchange and the compensator state.
 *   P      number of simulated tensor-parallel ranks, 2..16.
 *   n      elements per rank; n % (P*group) == 0 and n <= 2^34; also
 *          n % 32 == 0 (16-byte code rows), which only group 16 with an
 *          odd P can miss (ECHO_ERR_UNSUPPORTED).
 *   group  elements per scale: 32 (the default reading) or, as group-size
 *          variants, 16, 64 or 128; anything else ECHO_ERR_UNSUPPORTED. The
 *          wire then costs 1/2 + 1/group bytes per element.
 *   dtype  ECHO_BF16 or ECHO_FP32: the element type of the rank buffers.
 * Allocates on the current device: stage-1 wire (P x n/2 code bytes and
 * P x 2n/group scale bytes, room for binary16 scales), the requantised wire
 * (n/2 + 2n/group bytes) and the compensator state (2 phases x 2 estimates x
 * n binary32, zeroed).
 * Returns NULL on any error (see echo_last_error). The handle is bound to the
 * device that was current at creation.
 */
ECHO_API echo_handle *echo_create(int P, size_t n, int group, int dtype);

/*
 * echo_allreduce - in-place Echo all-reduce of P rank buffers.
 * Defined by [rit.work "Echo 4-bit GPU communication", section "How Echo
 * returns the error to later calls"]: every rank rounds its partial to 4-bit
 * integers (the owner of a segment first adds the correction to its own part
 * of it), each owner restores and adds the P segments in high precision,
 * rounds the total to 4 bits once more and sends it back to every rank, so
 * each element is rounded at most twice; the owner's rounding error updates
 * the fast and slow estimates of the call's phase.
 *   rank_ptrs  P device pointers, each n elements of the handle's dtype,
 *              16-byte aligned, pairwise non-overlapping. Caller-owned.
 *   phase      ECHO_FWD or ECHO_BWD: which compensator state is read and
 *              updated (the two never mix).
 * Enqueues three kernels (compensate+quantise+pack, owner reduce+requantise,
 * gather+dequantise) and returns. When the stream reaches the end, every
 * rank_ptrs[r] holds the same value Y = Q*2^E, exactly representable in the
 * dtype (Q*s under ECHO_VARIANT_FP16_SCALE, rounded to the nearest bf16 for
 * bf16 buffers), and the phase's state holds the updated estimates.
 */
ECHO_API int echo_allreduce(echo_handle *h, void *const rank_ptrs[], int phase, void *stream);

/*
 * echo_allreduce_out - the same all-reduce out of place: reads send_ptrs[r],
 * writes recv_ptrs[r]. Each send buffer may equal its own recv buffer; no
 * other overlap is allowed. Same alignment and size rules.
 */
ECHO_API int echo_allreduce_out(echo_handle *h, const void *const send_ptrs[],
                       void *const recv_ptrs[], int phase, void *stream);

/*
 * echo_allreduce_host - end to end from host memory: copies the P host
 * partials host_send[r] (n elements each) to library-owned device buffers,
 * runs the all-reduce, and copies the result (identical on every rank, n
 * elements) back to host_recv. Copies and kernels are enqueued on stream in
 * chunks so transfers overlap compute; the call returns after the result is
 * in host_recv (it synchronises the stream). The device staging buffers
 * (P x n elements) are allocated on first use and kept until echo_destroy.
 */
ECHO_API int echo_allreduce_host(echo_handle *h, const void *const host_send[], void *host_recv,
                        int phase, void *stream);

/*
 * echo_allreduce_static - the in-place all-reduce of echo_allreduce for
 * callers that cannot allocate device memory (the paper has no counterpart:
 * this is a deployment variant of the same computation). Typical callers are
 * a serving process that reserved all of HBM for its own pool at start-up, a
 * plugin running inside a host application that owns every allocation, and a
 * latency-critical path where a cudaMalloc, which can synchronise the device,
 * is not acceptable. It allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library call.
 *   rank_ptrs  P device pointers, n elements of dtype each, as for
 *              echo_allreduce (read, then overwritten with the result).
 *   f, s       the caller's compensator state for this phase: n binary32 each,
 *              device memory, read and updated in place (ignored, and may be
 *              NULL, when enable == 0). Zero them before the first call.
 *   beta_fast, beta_slow, lambda, enable   as for echo_set_params.
 * The wire buffers the kernels exchange live in one array compiled into the
 * library, ECHO_STATIC_SCRATCH_BYTES (32 MiB) per GPU, kept until the process
 * exits. A call needs about (P+1)*17/32 bytes per element of n (at P = 8, n
 * up to about 7 million elements); larger sizes, and n > 2^34, are rejected
 * with ECHO_ERR_UNSUPPORTED and nothing is enqueued. Argument errors (P, n,
 * dtype, parameters, NULL, misaligned, non-device, other-device or
 * overlapping pointers, state overlapping a rank buffer) return
 * ECHO_ERR_INVALID with nothing enqueued.
 * Set-up: the first call of echo_allreduce_static or echo_static_status on a
 * device, with that device current, looks up the array's device address
 * (cudaGetSymbolAddress) and zeroes its status word, synchronously. Under
 * CUDA's lazy module loading that is also when the 32 MiB are taken from the
 * device. So make one such call (echo_static_status is the cheap one) at
 * start-up: before reserving the rest of HBM for a memory pool, and before
 * any stream capture.
 * All calls share the array and it keeps the last call's contents; calls
 * whose work overlaps on the GPU (other streams or threads at once) race on
 * it. Calls with n <= 2^20 run as one kernel, as echo_allreduce does by
 * default (echo_set_fused_limit); larger ones run the three kernels.
 */
#define ECHO_STATIC_SCRATCH_BYTES (32u * 1024u * 1024u)
ECHO_API int echo_allreduce_static(int P, size_t n, int dtype, void *const rank_ptrs[], float *f, float *s,
                                   float beta_fast, float beta_slow, float lambda, int enable, void *stream);

/*
 * echo_static_status - the static path's device status word on the current
 * device (synchronous: waits for the device first), with the bits of
 * echo_device_status. Every echo_allreduce_static call on the device ORs
 * into the same word, so it gathers the timeouts of all calls since it was
 * last cleared; clear != 0 zeroes it after reading. The first use on a
 * device sets up the static array (see echo_allreduce_static) and allocates
 * nothing else.
 */
ECHO_API int echo_static_status(int *status, int clear);

/* echo_reset - zero the compensator state (and the sender errors, if
 * allocated) of the phases in phase_mask (bit 0 forward, bit 1 backward);
 * waits for the device first and completes before return. The forward and
 * the backward pass keep separate estimates [rit.work "Echo 4-bit GPU
 * communication", end of section "How Echo returns the error to later
 * calls"]. */
ECHO_API int echo_reset(echo_handle *h, int phase_mask);

/* echo_destroy - free everything the handle owns (synchronises the device
 * first). NULL is a no-op. The handle must not be used afterwards. */
ECHO_API int echo_destroy(echo_handle *h);

/* echo_last_error - message of the last failed call on this thread
 * ("" if none). The string stays valid until the thread's next failing call.
 * echo_last_status - that call's ECHO_ERR_* code (ECHO_OK if none); the way
 * to tell why echo_create returned NULL. */
ECHO_API const char *echo_last_error(void);
ECHO_API int echo_last_status(void);

/*
 * echo_set_params - compensator settings for later calls: beta_fast and
 * beta_slow in [0, 1), lambda in [0, 1], enable 0 (no correction, state
 * neither read nor written) or 1. Out-of-range values: ECHO_ERR_INVALID.
 */
ECHO_API int echo_set_params(echo_handle *h, float beta_fast, float beta_slow, float lambda,
                    int enable);

/*
 * echo_set_variant - variants of where the rounding errors are fed back, for
 * later calls (bits; 0 is the method described above):
 *   ECHO_VARIANT_OWNER_SUM  the owner adds c = lambda*f + (1-lambda)*s to its
 *       binary32 sum after the P restored values, instead of adding it to its
 *       own partial before rounding #1. The correction then passes no 4-bit
 *       rounding, and kernel 1 reads no state (8 bytes less per element).
 *   ECHO_VARIANT_SENDER_EF  every rank also feeds back its own rounding-#1
 *       error: v = RN(RN(x + eps_r) + c), eps_r <- v - q*2^e (exact), one
 *       binary32 per element per rank and phase (zeroed when first switched
 *       on; allocated then, ECHO_ERR_OOM if that fails). With both roundings
 *       fed back the running sum of all injected error stays bounded.
 *   ECHO_VARIANT_FP16_SCALE  a scale format variant for both roundings: each
 *       group's scale is the smallest positive finite binary16 s with
 *       7*s >= max|v| (0 for an all-zero group; 65504 past 7*65504, where
 *       codes saturate at +-7), stored as two little-endian bytes; each code
 *       is the integer in [-7, 7] nearest to v/s, ties to even. Restored
 *       values q*s are exact in binary32; bf16 outputs are q*s rounded to the
 *       nearest bf16 (ties to even), and the owner's captured error is taken
 *       against that received value. The wire costs 1/2 + 2/group bytes per
 *       element; steps follow max|v| within 2^-10 instead of a factor of 2.
 * The pages say the error a rounding injects is stored and added back in later
 * calls [rit.work "Echo 4-bit GPU communication", section "How Echo returns
 * the error to later calls"] and that the high-precision sum reveals every
 * injected error [heraldofai.com, section "Come Echo evita che gli errori si
 * accumulino"]; these variants are readings of where that happens.
 */
#define ECHO_VARIANT_OWNER_SUM 1
#define ECHO_VARIANT_SENDER_EF 2
#define ECHO_VARIANT_FP16_SCALE 4
ECHO_API int echo_set_variant(echo_handle *h, int variant);

/*
 * echo_set_fused_limit - calls of this handle with n <= max_n (elements per
 * rank) run as one kernel instead of the three: every step of the method
 * works on one group of G elements at a time [rit.work "Echo 4-bit GPU
 * communication", section "How Echo returns the error to later calls": a
 * rank's segment rounded, the owner's high-precision sum rounded again, the
 * total sent back], so one lane can take its 8 elements through all three
 * steps. Up to about 2 MiB per rank the three dependent launches, not the
 * bytes, set the time of a call. The fused call computes the same results bit
 * for bit and writes the same buffers (both wires, state, sender errors,
 * outputs); it does not read the stage-1 wire back. Every variant and group
 * size runs fused. 0 turns it off; the default is 2^20. It applies to
 * echo_allreduce, echo_allreduce_out and echo_allreduce_host. The static
 * entry point makes the same choice with the default limit; the per-rank
 * entry points (echo_dist_*) always run their three stages. echo_stats still
 * counts the three kernels' model bytes. echo_get_fused_limit reads the setting (max_n non-NULL, else
 * ECHO_ERR_INVALID).
 */
ECHO_API int echo_set_fused_limit(echo_handle *h, size_t max_n);
ECHO_API int echo_get_fused_limit(echo_handle *h, size_t *max_n);

/* Synchronous copies of rank `rank`'s sender errors for `phase` (elements
 * [offset, offset+count) to host; all n from host). ECHO_ERR_INVALID if sender
 * feedback was never switched on. */
ECHO_API int echo_get_sender_state(echo_handle *h, int phase, int rank, size_t offset, size_t count,
                                   float *host);
ECHO_API int echo_set_sender_state(echo_handle *h, int phase, int rank, const float *host);

/* echo_get_state / echo_set_state - synchronous copies of a phase's two
 * estimates (n binary32 each) to / from host memory. A checkpoint is the pair
 * for both phases. The two smoothed estimates, one fast and one slow, per
 * phase: [rit.work "Echo 4-bit GPU communication", end of section "How Echo
 * returns the error to later calls"]. */
ECHO_API int echo_get_state(echo_handle *h, int phase, float *f_host, float *s_host);
ECHO_API int echo_set_state(echo_handle *h, int phase, const float *f_host, const float *s_host);

/* Range variants: elements [offset, offset+count). */
ECHO_API int echo_get_state_range(echo_handle *h, int phase, size_t offset, size_t count,
                         float *f_host, float *s_host);

/*
 * echo_get_wire - synchronous copy of the wire left by the last call: the
 * 4-bit segments every rank sends to the owners, and the 4-bit total the
 * owners send back [rit.work "Echo 4-bit GPU communication", section "How
 * Echo returns the error to later calls"].
 *   stage 1: rank's packed codes (n/2 bytes) and scales (n/group bytes, or
 *            n/group little-endian binary16 patterns under
 *            ECHO_VARIANT_FP16_SCALE: 2n/group bytes);
 *   stage 2: the requantised total (rank ignored).
 * Either output pointer may be NULL to skip it.
 */
ECHO_API int echo_get_wire(echo_handle *h, int stage, int rank, uint8_t *codes_host,
                  uint8_t *scales_host);

/* Range variant over groups [group_offset, group_offset+ngroups):
 * group/2 * ngroups code bytes and ngroups scales (1 or 2 bytes each). */
ECHO_API int echo_get_wire_range(echo_handle *h, int stage, int rank, size_t group_offset,
                        size_t ngroups, uint8_t *codes_host, uint8_t *scales_host);

/*
 * echo_stats - counters since creation (the exchanged volume is the pages'
 * point: 4-bit words make it almost four times smaller than 16-bit ones,
 * [rit.work "Echo 4-bit GPU communication", section "Why plain 4-bit
 * summation damages the model"]): bytes that would cross links
 * (reduce-scatter + all-gather, 2(P-1) * n * w per call, with w the wire
 * bytes per element: 17/32 at the default group of 32), modelled HBM
 * bytes (sum of the three kernels' algorithmic bytes), and calls made through
 * the API (replays of a captured CUDA graph are not counted). Any output
 * pointer may be NULL.
 */
ECHO_API int echo_stats(echo_handle *h, uint64_t *link_bytes, uint64_t *model_hbm_bytes,
               uint64_t *calls);

/*
 * echo_model_bytes - algorithmic bytes of one call, host-only arithmetic:
 *   out[0..2]  HBM bytes read + written by kernels 1, 2, 3
 *              (P*b + 8 + P*w, P*w + 16 + w, P*w + P*b per element, w = 17/32
 *               at group 32, b = element bytes; the 8/16 state terms vanish
 *               with compensation off),
 *   out[3]     link bytes of one call, 2(P-1) * n * w.
 * Same argument rules as echo_create.
 */
ECHO_API int echo_model_bytes(int P, size_t n, int dtype, int enable, uint64_t out[4]);

/* The same for any group size and variant: the wire is 1/2 + 1/group bytes
 * per element (1/2 + 2/group with FP16_SCALE); OWNER_SUM drops kernel 1's 8
 * state bytes; SENDER_EF adds 8P bytes (each rank's error read and written)
 * to kernel 1. */
ECHO_API int echo_model_bytes_ex(int P, size_t n, int group, int dtype, int enable, int variant,
                                 uint64_t out[4]);

/*
 * Kernel timing. echo_set_timing(h, 1) starts a measurement: every later
 * echo_allreduce / echo_allreduce_out call records CUDA events around each of
 * its three kernels on its own stream (no host wait inside the calls).
 * echo_last_kernel_ms returns the three durations of the last call (waiting
 * for it); echo_kernel_ms_total returns their sums over every timed call since
 * the measurement started, and how many calls that was (waiting for the last).
 * echo_set_timing(h, 0) stops recording; the totals stay readable.
 */
ECHO_API int echo_set_timing(echo_handle *h, int enable);
ECHO_API int echo_last_kernel_ms(echo_handle *h, float ms[3]);
/* (A call that ran as one kernel, see echo_set_fused_limit, reports its whole
 * time as kernel 1's and 0 for kernels 2 and 3.) */
ECHO_API int echo_kernel_ms_total(echo_handle *h, double ms[3], uint64_t *timed_calls);

/*
 * echo_device_status - the handle's device status word (synchronous): 0, or
 * bits 1/2/4 (ECHO_STATUS_TIMEOUT_K1..K3) when a wait inside kernel 1/2/3 ran
 * out of its time bound (about a second). The kernels never spin without
 * bound; a CTA whose tile did not arrive in time records the bit and returns,
 * leaving that call's outputs incomplete. The debug build adds
 * ECHO_STATUS_BOUNDS (an index or copy range would have left its buffer; the
 * access was skipped) and ECHO_STATUS_CANARY (a guard byte around one of the
 * library's buffers changed). clear != 0 resets the word after reading it.
 */
#define ECHO_STATUS_TIMEOUT_K1 1
#define ECHO_STATUS_TIMEOUT_K2 2
#define ECHO_STATUS_TIMEOUT_K3 4
#define ECHO_STATUS_BOUNDS 8
#define ECHO_STATUS_CANARY 16
ECHO_API int echo_device_status(echo_handle *h, int *status, int clear);

/*
 * Debug build (libecho_debug.so, compiled with ECHO_DEBUG=1): every kernel
 * checks each computed index and bulk-copy range against its buffer, and
 * every device buffer the library allocates carries 256 guard bytes on each
 * side, checked after each call. echo_debug_build returns 1 in that build and
 * 0 in the release build. echo_debug_touch_guard overwrites one guard byte
 * (the first after the stage-1 code buffer) so that a test can see the next
 * call report ECHO_STATUS_CANARY; it returns ECHO_ERR_UNSUPPORTED in the
 * release build.
 */
ECHO_API int echo_debug_build(void);
ECHO_API int echo_debug_touch_guard(echo_handle *h);

/*
 * One rank per handle (echo_dist_*): the same all-reduce when each of the
 * world ranks holds only its own partial, as on a real tensor-parallel
 * group [rit.work "Echo 4-bit GPU communication", sections "How Echo returns
 * the error to later calls" (segments go to their owner, the owner's 4-bit
 * total goes back to every rank) and "When the gain changes the
 * infrastructure plan" (the exchange crosses NVLink, PCIe or the network)].
 * Ranks may be separate processes (one per GPU, or several sharing a GPU) or
 * several handles in one process. Every rank keeps the compensator state of
 * the segment it owns, [rank*n/world, (rank+1)*n/world), and exports a block
 * that the others write into: a receive slot per rank for the owned segment's
 * stage-1 wire, and the gathered requantised tensor. A call runs in three
 * stages:
 *   stage 1  kernel 1 rounds this rank's partial x and stores each segment's
 *            codes and scales straight into its owner's receive slot;
 *   stage 2  kernel 2 sums the owned segment from the receive slots,
 *            requantises it, updates the owned state, and stores the
 *            requantised segment into every rank's gathered tensor;
 *   stage 3  kernel 3 writes the result (n elements, identical on every rank)
 *            from the local gathered tensor to out.
 * The wire moves as plain stores into the other ranks' blocks (on several
 * GPUs, peer stores over NVLink); the kernels read local memory only, and no
 * kernel waits on another rank or spins on a flag.
 * Ordering: every rank records an event after each of its stages (CUDA IPC
 * events across processes), and each stage first makes its stream wait for
 * the events it depends on, on every rank (stage 1 on the stage-2 events of
 * the previous call, stage 2 on the stage-1 and the previous call's stage-3
 * events, stage 3 on the stage-2 events). A wait takes an event's latest
 * record when it is enqueued, so the caller puts a host barrier over all
 * ranks after every rank has enqueued stage 1, and again after stage 2,
 * of every call. Nothing waits for the GPU: the stream of each rank carries
 * the ordering. The results are bit for bit those of echo_allreduce on the
 * same partials.
 *
 * echo_dist_create(world, rank, n, group, dtype): world in [2, 16], rank in
 *   [0, world), n a positive multiple of world x max(group, 32) (segments of
 *   whole groups whose code rows start on 16 bytes), group and dtype as for
 *   echo_create. Allocates on the current device, NULL on error.
 * echo_dist_export: writes ECHO_DIST_HANDLE_BYTES bytes that describe this
 *   rank to the others: the CUDA IPC handles of its block and of its three
 *   stage events, its process, its rank, world, n, group and dtype.
 * echo_dist_connect: handles = world such blobs in rank order (this rank's
 *   own entry is ignored). Blobs from this process are used directly (their
 *   handles must stay alive while this one is used); the others are opened
 *   through CUDA IPC. A blob whose rank, world, n, group or dtype does not
 *   match is rejected with ECHO_ERR_INVALID. Once per handle.
 * echo_dist_stage(d, stage, x, out, phase, stream): x (stage 1) and out
 *   (stage 3) are device pointers to n elements of dtype, 16-byte aligned
 *   (unused in the other stages; out may equal x). The three stages of a
 *   rank's call go on one stream, or on streams the caller orders.
 * echo_dist_set_params / echo_dist_set_variant: as echo_set_params and
 *   echo_set_variant, for this rank (every rank must use the same settings).
 * echo_dist_get_state: the owned segment's two estimates (n/world binary32
 *   each) of a phase, synchronous.
 * echo_dist_device_status: as echo_device_status.
 * echo_dist_destroy: closes the peers' buffers and events and frees this
 *   rank's (call on every rank after its stream is idle and after a final
 *   barrier).
 */
#define ECHO_DIST_HANDLE_BYTES 320
typedef struct echo_dist echo_dist; /* opaque */
ECHO_API echo_dist *echo_dist_create(int world, int rank, size_t n, int group, int dtype);
ECHO_API int echo_dist_export(echo_dist *d, uint8_t handle[ECHO_DIST_HANDLE_BYTES]);
ECHO_API int echo_dist_connect(echo_dist *d, const uint8_t *handles);
ECHO_API int echo_dist_stage(echo_dist *d, int stage, const void *x, void *out, int phase, void *stream);
ECHO_API int echo_dist_set_params(echo_dist *d, float beta_fast, float beta_slow, float lambda, int enable);
ECHO_API int echo_dist_set_variant(echo_dist *d, int variant);
ECHO_API int echo_dist_get_state(echo_dist *d, int phase, float *f_host, float *s_host);
ECHO_API int echo_dist_device_status(echo_dist *d, int *status, int clear);
ECHO_API int echo_dist_destroy(echo_dist *d);

#ifdef __cplusplus
}
#endif
#endif /* ECHO_H */
