// echo_api.cu - host side of libecho.so: the C ABI declared in include/echo.h.
//
// Owns the handle (wire buffers, compensator state, counters, events),
// validates every argument before anything is enqueued, and enqueues the
// three kernels of one all-reduce call in order on the caller's stream:
//   K1 compensate + quantise + pack   (every rank -> stage-1 wire)
//   K2 owner reduce + requantise      (stage-1 wire -> requantised wire, state)
//   K3 gather + dequantise            (requantised wire -> every rank)
// Stream order is the only synchronisation between them; no kernel waits on
// another.
#include "echo.h"
#include "echo_kernels.h"

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <set>
#include <string>

namespace {

thread_local std::string g_err;
thread_local int g_status = ECHO_OK;

int set_error(int code, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    g_status = code;
    return code;
}

int cuda_error(cudaError_t e, const char *what)
{
    return set_error(ECHO_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

// Fault injection for tests: ECHO_FAULT=alloc makes echo_create fail as if
// the device were out of memory and ECHO_FAULT=launch makes the all-reduce
// entry points fail as if the launch had failed (nothing reaches the GPU);
// ECHO_FAULT=stall launches the kernels with no loads issued and a short
// wait bound, so every CTA's first wait runs out and the kernels record a
// timeout in the device status word and return.
bool fault_injected(const char *what)
{
    const char *e = std::getenv("ECHO_FAULT");
    return e && std::strcmp(e, what) == 0;
}

std::mutex g_mu;
std::set<const echo_handle *> g_live; // handles created and not destroyed

constexpr size_t kMaxN = size_t(1) << 34;  // chunk indices stay 32-bit
// Bound of every kernel wait: about a second at B200 clocks (a tile normally
// lands in microseconds); the injected stall uses about half a millisecond.
constexpr long long kWaitCycles = 1LL << 31;
constexpr long long kStallWaitCycles = 1LL << 20;
// Host-path pieces: 2^25 elements per rank measured best at 1 GiB (159 ms per
// step, against 168 at 2^22, whose 1024 copies per step each cost set-up,
// and 161 at 2^26, whose first and last pieces take longer to fill and drain).
#ifndef ECHO_HOST_PIECE_LOG2
#define ECHO_HOST_PIECE_LOG2 25
#endif
constexpr size_t kHostPiece = size_t(1) << ECHO_HOST_PIECE_LOG2; // elements per pipelined host transfer
constexpr int kVariantBits = ECHO_VARIANT_OWNER_SUM | ECHO_VARIANT_SENDER_EF | ECHO_VARIANT_FP16_SCALE;
constexpr int kTimingRing = 32;                 // event sets of timed calls in flight

size_t elem_bytes(int dtype) { return dtype == ECHO_BF16 ? 2 : 4; }

int check_shape(int P, size_t n, int group, int dtype)
{
    if (P < 2 || P > ECHO_MAX_RANKS)
        return set_error(ECHO_ERR_INVALID, "P = %d is outside [2, %d]", P, ECHO_MAX_RANKS);
    if (dtype != ECHO_BF16 && dtype != ECHO_FP32)
        return set_error(ECHO_ERR_INVALID, "unknown dtype %d", dtype);
    if (group <= 0)
        return set_error(ECHO_ERR_INVALID, "group = %d must be positive", group);
    if (n == 0 || n % (static_cast<size_t>(P) * static_cast<size_t>(group)) != 0)
        return set_error(ECHO_ERR_INVALID, "n = %zu must be a positive multiple of P*group = %d", n,
                         P * group);
    if (group != 16 && group != 32 && group != 64 && group != 128)
        return set_error(ECHO_ERR_UNSUPPORTED, "group = %d: the built group sizes are 16, 32, 64 and 128", group);
    // Every rank's code row (n/2 bytes) must start on a 16-byte boundary for
    // the bulk copies; only group 16 with an odd P can miss it.
    if (n % 32 != 0)
        return set_error(ECHO_ERR_UNSUPPORTED, "n = %zu: code rows need n to be a multiple of 32", n);
    if (n > kMaxN)
        return set_error(ECHO_ERR_UNSUPPORTED, "n = %zu exceeds the supported maximum %zu", n, kMaxN);
    return ECHO_OK;
}

void model_bytes(int P, size_t n, int group, int dtype, bool enable, int variant, uint64_t out[4])
{
    const uint64_t b = elem_bytes(dtype);
    // n * (1/2 + 1/G) bytes, or n * (1/2 + 2/G) with binary16 scales
    const uint64_t scale_bytes = (variant & ECHO_VARIANT_FP16_SCALE) ? 2 : 1;
    const uint64_t wire = static_cast<uint64_t>(n) / 2 + scale_bytes * static_cast<uint64_t>(n) / group;
    const uint64_t state = enable ? 8 * static_cast<uint64_t>(n) : 0;
    // the owner-sum variant reads f, s in kernel 2 only
    const uint64_t k1_state = (variant & ECHO_VARIANT_OWNER_SUM) ? 0 : state;
    // sender feedback: every rank reads and writes its own error (4 + 4 bytes)
    const uint64_t eps = (variant & ECHO_VARIANT_SENDER_EF) ? 8 * static_cast<uint64_t>(P) * n : 0;
    out[0] = P * b * n + k1_state + P * wire + eps;  // K1
    out[1] = P * wire + 2 * state + wire;            // K2
    out[2] = P * wire + P * b * n;                   // K3
    out[3] = 2 * static_cast<uint64_t>(P - 1) * wire; // link bytes
}

} // namespace

struct echo_handle {
    int P = 0;
    size_t n = 0;
    int dtype = ECHO_BF16;
    int group = ECHO_GROUP;     // elements per scale
    uint32_t lanes_log2 = 2;    // log2(group / 8)
    int device = 0;
    uint8_t *codes1 = nullptr;  // [P][n/2]
    uint8_t *scales1 = nullptr; // [P][scale_stride], n/group bytes used per rank
    uint8_t *qcodes = nullptr;  // [n/2]
    uint8_t *qscales = nullptr; // [scale_stride]
    size_t scale_stride = 0;    // 2n/group rounded up to 16 bytes (bulk-copy alignment)
    int *dstatus = nullptr;     // device status word written by timed-out waits
    float *state = nullptr;     // [phase][f|s][n]
    float beta_f = 0.5f, beta_s = 0.875f, lambda = 0.5f;
    bool enable = true;
    int variant = 0;            // ECHO_VARIANT_* bits
    float *eps = nullptr;       // [phase][P][n]: sender errors (allocated with the variant)
    size_t fused_limit = ECHO_FUSED_LIMIT; // calls with n <= this run as one kernel
    uint64_t link_bytes = 0, hbm_bytes = 0, calls = 0;
    // Kernel timing: each timed call records 4 events (before K1, after K1,
    // K2, K3) into slot (call index mod kTimingRing); a slot's durations are
    // folded into the totals before the slot is reused or when queried, so a
    // timed loop of calls never waits on the device.
    bool timing = false;
    cudaEvent_t ring[kTimingRing][4] = {};
    bool ring_fused[kTimingRing] = {}; // the slot's call ran as one kernel: events 0 and 1 only
    uint64_t ring_calls = 0; // timed calls since timing was switched on
    uint64_t folded = 0;     // timed calls already added to total_ms
    double total_ms[3] = {};
    int last_slot = -1;      // slot of the last call if it was timed
    // end-to-end host path
    uint8_t *staging = nullptr; // [P][n] elements
    cudaStream_t s_in = nullptr, s_comp = nullptr, s_out = nullptr;
    cudaEvent_t e_start = nullptr, e_in = nullptr, e_comp = nullptr, e_done = nullptr;
    // pointers that already passed the device-memory check
    const void *checked[2 * ECHO_MAX_RANKS] = {};
    bool checked_valid = false;
    // debug build: the guard regions around every buffer above
    echo::GuardList guards = {};
};

namespace {

#ifndef ECHO_DEBUG
#define ECHO_DEBUG 0
#endif

// Device allocation of every library buffer. The debug build puts
// kGuardBytes of kGuardByte on both sides of each buffer and records the two
// regions in the handle; the release build allocates exactly `bytes`.
cudaError_t dev_alloc(echo_handle *h, void **p, size_t bytes)
{
    if (!ECHO_DEBUG)
        return cudaMalloc(p, bytes);
    if (h->guards.count + 2 > echo::kMaxGuards)
        return cudaErrorInvalidValue;
    uint8_t *base = nullptr;
    cudaError_t e = cudaMalloc(reinterpret_cast<void **>(&base), bytes + 2 * echo::kGuardBytes);
    if (e != cudaSuccess)
        return e;
    e = cudaMemset(base, echo::kGuardByte, echo::kGuardBytes);
    if (e == cudaSuccess)
        e = cudaMemset(base + echo::kGuardBytes + bytes, echo::kGuardByte, echo::kGuardBytes);
    if (e != cudaSuccess) {
        cudaFree(base);
        return e;
    }
    h->guards.region[h->guards.count++] = base;
    h->guards.region[h->guards.count++] = base + echo::kGuardBytes + bytes;
    *p = base + echo::kGuardBytes;
    return cudaSuccess;
}

void dev_free(void *p)
{
    if (p)
        cudaFree(ECHO_DEBUG ? static_cast<uint8_t *>(p) - echo::kGuardBytes : p);
}

int check_handle(const echo_handle *h)
{
    if (!h)
        return set_error(ECHO_ERR_INVALID, "handle is NULL");
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_live.count(h))
        return set_error(ECHO_ERR_INVALID, "handle %p is unknown or destroyed", static_cast<const void *>(h));
    return ECHO_OK;
}

int check_device(const echo_handle *h)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return cuda_error(e, "cudaGetDevice");
    if (dev != h->device)
        return set_error(ECHO_ERR_INVALID, "handle lives on device %d but device %d is current", h->device, dev);
    return ECHO_OK;
}

int check_phase(int phase)
{
    if (phase != ECHO_FWD && phase != ECHO_BWD)
        return set_error(ECHO_ERR_INVALID, "phase %d is neither ECHO_FWD (0) nor ECHO_BWD (1)", phase);
    return ECHO_OK;
}

// P send and P recv buffers of n elements: non-NULL, 16-byte aligned, on the
// handle's device, and pairwise disjoint except send[r] == recv[r].
int check_buffers(echo_handle *h, const void *const send[], void *const recv[])
{
    if (!send || !recv)
        return set_error(ECHO_ERR_INVALID, "rank pointer array is NULL");
    const int P = h->P;
    const size_t bytes = h->n * elem_bytes(h->dtype);
    const void *all[2 * ECHO_MAX_RANKS];
    for (int r = 0; r < P; r++) {
        all[r] = send[r];
        all[P + r] = recv[r];
    }
    for (int i = 0; i < 2 * P; i++) {
        if (!all[i])
            return set_error(ECHO_ERR_INVALID, "%s pointer of rank %d is NULL", i < P ? "send" : "recv", i % P);
        if (reinterpret_cast<uintptr_t>(all[i]) % 16 != 0)
            return set_error(ECHO_ERR_INVALID, "%s pointer of rank %d is not 16-byte aligned",
                             i < P ? "send" : "recv", i % P);
    }
    for (int i = 0; i < 2 * P; i++) {
        for (int j = i + 1; j < 2 * P; j++) {
            if (j == i + P && all[i] == all[j])
                continue; // in place for rank i
            const uintptr_t a = reinterpret_cast<uintptr_t>(all[i]);
            const uintptr_t b = reinterpret_cast<uintptr_t>(all[j]);
            if (a < b + bytes && b < a + bytes)
                return set_error(ECHO_ERR_INVALID, "rank buffers %d and %d overlap", i, j);
        }
    }
    bool same = h->checked_valid;
    for (int i = 0; i < 2 * P && same; i++)
        same = h->checked[i] == all[i];
    if (same)
        return ECHO_OK;
    for (int i = 0; i < 2 * P; i++) {
        cudaPointerAttributes attr;
        cudaError_t e = cudaPointerGetAttributes(&attr, all[i]);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return set_error(ECHO_ERR_INVALID, "rank pointer %d is not CUDA memory (%s)", i, cudaGetErrorString(e));
        }
        if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
            return set_error(ECHO_ERR_INVALID, "rank pointer %d is not device memory", i);
        if (attr.device != h->device)
            return set_error(ECHO_ERR_INVALID, "rank pointer %d is on device %d, handle on %d", i, attr.device,
                             h->device);
    }
    for (int i = 0; i < 2 * P; i++)
        h->checked[i] = all[i];
    h->checked_valid = true;
    return ECHO_OK;
}

// Add the kernel durations of timed calls [h->folded, upto) to the totals.
// The three kernel durations of timing slot `slot` (waiting for its events).
// A call that ran as one kernel recorded events 0 and 1 only: its whole time
// is kernel 1's, and kernels 2 and 3 are 0.
cudaError_t slot_ms(const echo_handle *h, int slot, float ms[3])
{
    const cudaEvent_t *ev = h->ring[slot];
    const int kernels = h->ring_fused[slot] ? 1 : 3;
    cudaError_t e = cudaEventSynchronize(ev[kernels]);
    for (int k = 0; k < 3 && e == cudaSuccess; k++) {
        ms[k] = 0.f;
        if (k < kernels)
            e = cudaEventElapsedTime(&ms[k], ev[k], ev[k + 1]);
    }
    return e;
}

int fold_timings(echo_handle *h, uint64_t upto)
{
    for (; h->folded < upto; h->folded++) {
        float ms[3];
        cudaError_t e = slot_ms(h, static_cast<int>(h->folded % kTimingRing), ms);
        if (e != cudaSuccess)
            return cuda_error(e, "kernel timing events");
        for (int k = 0; k < 3; k++)
            h->total_ms[k] += ms[k];
    }
    return ECHO_OK;
}

struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

// Enqueue K1, K2, K3 over chunks [cb, ce) (multiples of 4) of the tensor.
// With record_events the call takes the next timing slot.
int enqueue_call(echo_handle *h, const void *const send[], void *const recv[], int phase, cudaStream_t st,
                 uint32_t cb, uint32_t ce, bool record_events)
{
    // The range starts at a multiple of 16 groups, so every bulk copy
    // (partials, codes, 16-byte scale rows, state) is 16-byte aligned.
    if ((static_cast<size_t>(cb) * echo::kChunk) % (16 * static_cast<size_t>(h->group)) != 0 || ce < cb)
        return set_error(ECHO_ERR_INVALID, "internal: element range must start at a multiple of 16 groups");
    // Every wait in the kernels is bounded; ECHO_FAULT=stall (tests) issues no
    // loads at all and shortens the bound, so each wait runs out quickly.
    const bool stall = fault_injected("stall");
    // Small calls run as one kernel (the injected stall exercises the three
    // kernels' bounded waits, so it always runs them).
    const bool fused = !stall && h->n <= h->fused_limit;
    cudaEvent_t *ev = nullptr;
    if (record_events) {
        if (h->ring_calls >= static_cast<uint64_t>(kTimingRing)) {
            int rc = fold_timings(h, h->ring_calls - kTimingRing + 1);
            if (rc != ECHO_OK)
                return rc;
        }
        h->last_slot = static_cast<int>(h->ring_calls % kTimingRing);
        ev = h->ring[h->last_slot];
        h->ring_fused[h->last_slot] = fused;
        h->ring_calls += 1;
    } else {
        h->last_slot = -1;
    }
    float *f = h->state + static_cast<size_t>(phase) * 2 * h->n;
    float *s = f + h->n;
    echo::K1Args a1{};
    echo::K2Args a2{};
    echo::K3Args a3{};
    for (int r = 0; r < h->P; r++) {
        a1.x.p[r] = send[r];
        a3.out.p[r] = recv[r];
    }
    a1.f = f;
    a1.s = s;
    a1.codes = h->codes1;
    a1.scales = h->scales1;
    a1.n = h->n;
    a1.chunk_begin = cb;
    a1.chunk_end = ce;
    a1.groups_per_seg = static_cast<uint32_t>(h->n / h->P / h->group);
    a1.lanes_log2 = a2.lanes_log2 = a3.lanes_log2 = h->lanes_log2;
    a1.lambda = h->lambda;
    a1.one_minus_lambda = 1.0f - h->lambda;
    a1.P = h->P;
    a1.bf16 = h->dtype == ECHO_BF16;
    a1.enable = h->enable && !(h->variant & ECHO_VARIANT_OWNER_SUM);
    a1.sender_ef = (h->variant & ECHO_VARIANT_SENDER_EF) != 0;
    a1.fp16_scale = a2.fp16_scale = a3.fp16_scale = (h->variant & ECHO_VARIANT_FP16_SCALE) != 0;
    a2.bf16 = h->dtype == ECHO_BF16;
    a1.eps = a1.sender_ef ? h->eps + static_cast<size_t>(phase) * h->P * h->n : nullptr;

    a2.codes = h->codes1;
    a2.scales = h->scales1;
    a2.qcodes = h->qcodes;
    a2.qscales = h->qscales;
    a2.f = f;
    a2.s = s;
    a2.n = h->n;
    a2.chunk_begin = cb;
    a2.chunk_end = ce;
    a2.beta_f = h->beta_f;
    a2.one_minus_beta_f = 1.0f - h->beta_f;
    a2.beta_s = h->beta_s;
    a2.one_minus_beta_s = 1.0f - h->beta_s;
    a2.lambda = h->lambda;
    a2.one_minus_lambda = 1.0f - h->lambda;
    a2.P = h->P;
    a2.enable = h->enable;
    a2.owner_sum = h->enable && (h->variant & ECHO_VARIANT_OWNER_SUM);

    a3.qcodes = h->qcodes;
    a3.qscales = h->qscales;
    a3.n = h->n;
    a3.chunk_begin = cb;
    a3.chunk_end = ce;
    a3.P = h->P;
    a3.bf16 = h->dtype == ECHO_BF16;

    const echo::PipeCtl ctl{h->dstatus, stall ? kStallWaitCycles : kWaitCycles, stall};
    a1.ctl = a2.ctl = a3.ctl = ctl;
    a1.scale_stride = a2.scale_stride = a3.scale_stride = h->scale_stride;

    // NVTX ranges (no-ops unless a profiler is attached) mark the call and
    // each kernel's enqueue, so a timeline tool can attribute the launches.
    NvtxRange call_range("echo_allreduce");
    cudaError_t e = cudaSuccess;
    const char *what = "cudaEventRecord";
    if (ev)
        e = cudaEventRecord(ev[0], st);
    if (e == cudaSuccess && fused) {
        echo::KFArgs af{};
        for (int r = 0; r < h->P; r++) {
            af.x.p[r] = send[r];
            af.out.p[r] = recv[r];
        }
        af.f = f;
        af.s = s;
        af.eps = a1.eps;
        af.codes = h->codes1;
        af.scales = h->scales1;
        af.qcodes = h->qcodes;
        af.qscales = h->qscales;
        af.n = h->n;
        af.scale_stride = h->scale_stride;
        af.chunk_begin = cb;
        af.chunk_end = ce;
        af.lanes_log2 = h->lanes_log2;
        af.groups_per_seg = a1.groups_per_seg;
        af.lambda = a1.lambda;
        af.one_minus_lambda = a1.one_minus_lambda;
        af.beta_f = a2.beta_f;
        af.one_minus_beta_f = a2.one_minus_beta_f;
        af.beta_s = a2.beta_s;
        af.one_minus_beta_s = a2.one_minus_beta_s;
        af.P = h->P;
        af.bf16 = h->dtype == ECHO_BF16;
        af.enable = h->enable;
        af.owner_sum = a2.owner_sum;
        af.sender_ef = a1.sender_ef;
        af.fp16_scale = a1.fp16_scale;
        af.ctl = ctl;
        NvtxRange r("kf_fused_allreduce");
        if ((e = echo::launch_kf_fused_allreduce(af, st)) != cudaSuccess)
            what = "launch kf_fused_allreduce";
        if (e == cudaSuccess && ev) // the whole call counts as kernel 1's time
            e = cudaEventRecord(ev[1], st);
    }
    if (e == cudaSuccess && !fused) {
        NvtxRange r("k1_compensate_quantize_pack");
        if ((e = echo::launch_k1_compensate_quantize_pack(a1, st)) != cudaSuccess)
            what = "launch k1_compensate_quantize_pack";
    }
    if (e == cudaSuccess && !fused && ev)
        e = cudaEventRecord(ev[1], st);
    if (e == cudaSuccess && !fused) {
        NvtxRange r("k2_owner_reduce_requant");
        if ((e = echo::launch_k2_owner_reduce_requant(a2, st)) != cudaSuccess)
            what = "launch k2_owner_reduce_requant";
    }
    if (e == cudaSuccess && !fused && ev)
        e = cudaEventRecord(ev[2], st);
    if (e == cudaSuccess && !fused) {
        NvtxRange r("k3_gather_dequant");
        if ((e = echo::launch_k3_gather_dequant(a3, st)) != cudaSuccess)
            what = "launch k3_gather_dequant";
    }
    if (e == cudaSuccess && !fused && ev)
        e = cudaEventRecord(ev[3], st);
    if (ECHO_DEBUG && e == cudaSuccess && (e = echo::launch_check_guards(h->guards, h->dstatus, st)) != cudaSuccess)
        what = "launch check_guards";
    if (e != cudaSuccess) {
        if (ev) { // the slot was not fully recorded: give it back
            h->ring_calls -= 1;
            h->last_slot = -1;
        }
        return cuda_error(e, what);
    }
    return ECHO_OK;
}

void count_call(echo_handle *h)
{
    uint64_t mb[4];
    model_bytes(h->P, h->n, h->group, h->dtype, h->enable, h->variant, mb);
    h->hbm_bytes += mb[0] + mb[1] + mb[2];
    h->link_bytes += mb[3];
    h->calls += 1;
}

int allreduce_impl(echo_handle *h, const void *const send[], void *const recv[], int phase, void *stream)
{
    int rc;
    if ((rc = check_handle(h)) != ECHO_OK || (rc = check_phase(phase)) != ECHO_OK ||
        (rc = check_device(h)) != ECHO_OK || (rc = check_buffers(h, send, recv)) != ECHO_OK)
        return rc;
    if (fault_injected("launch"))
        return set_error(ECHO_ERR_CUDA, "injected launch failure (ECHO_FAULT=launch)");
    const uint32_t chunks = static_cast<uint32_t>(h->n / echo::kChunk);
    rc = enqueue_call(h, send, recv, phase, static_cast<cudaStream_t>(stream), 0, chunks, h->timing);
    if (rc != ECHO_OK)
        return rc;
    count_call(h);
    return ECHO_OK;
}

void free_handle(echo_handle *h)
{
    dev_free(h->codes1);
    dev_free(h->scales1);
    dev_free(h->qcodes);
    dev_free(h->qscales);
    dev_free(h->state);
    dev_free(h->dstatus);
    dev_free(h->eps);
    dev_free(h->staging);
    for (auto &slot : h->ring)
        for (cudaEvent_t e : slot)
            if (e)
                cudaEventDestroy(e);
    for (cudaEvent_t e : {h->e_start, h->e_in, h->e_comp, h->e_done})
        if (e)
            cudaEventDestroy(e);
    for (cudaStream_t s : {h->s_in, h->s_comp, h->s_out})
        if (s)
            cudaStreamDestroy(s);
    delete h;
}

} // namespace

namespace echo {

static int sm_count()
{
    static std::atomic<int> cached{0}; // threads that race here compute the same value
    int sms = cached.load(std::memory_order_relaxed);
    if (sms == 0) {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
            sms = v;
        else
            sms = 148;
        cached.store(sms, std::memory_order_relaxed);
    }
    return sms;
}

int persistent_grid(uint32_t tiles, int resident_per_sm)
{
    const long full = static_cast<long>(sm_count()) * (resident_per_sm > 0 ? resident_per_sm : 1);
    const long g = static_cast<long>(tiles) < full ? static_cast<long>(tiles) : full;
    return g < 1 ? 1 : static_cast<int>(g);
}

int record_error(int code, const char *message) { return set_error(code, "%s", message); }

uint32_t pick_tile_log2(size_t elems, int max_tile, int min_tile, int resident_per_sm)
{
    const size_t ctas = static_cast<size_t>(sm_count()) * (resident_per_sm > 0 ? resident_per_sm : 1);
    size_t t = static_cast<size_t>(max_tile);
    while (t > static_cast<size_t>(min_tile) && elems / t < 4 * ctas)
        t /= 2;
    uint32_t lg = 0;
    while ((size_t(1) << lg) < t)
        lg++;
    return lg;
}

cudaError_t prepare_kernel(const void *kernel, int threads, int smem_bytes, int *resident)
{
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e != cudaSuccess)
        return e;
    int r = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&r, kernel, threads, smem_bytes);
    if (e != cudaSuccess)
        return e;
    *resident = r > 0 ? r : 1;
    return cudaSuccess;
}

} // namespace echo

extern "C" {

const char *echo_last_error(void) { return g_err.c_str(); }

int echo_last_status(void) { return g_status; }

int echo_model_bytes(int P, size_t n, int dtype, int enable, uint64_t out[4])
{
    int rc = check_shape(P, n, ECHO_GROUP, dtype);
    if (rc != ECHO_OK)
        return rc;
    if (!out)
        return set_error(ECHO_ERR_INVALID, "out is NULL");
    model_bytes(P, n, ECHO_GROUP, dtype, enable != 0, 0, out);
    return ECHO_OK;
}

int echo_model_bytes_ex(int P, size_t n, int group, int dtype, int enable, int variant, uint64_t out[4])
{
    int rc = check_shape(P, n, group, dtype);
    if (rc != ECHO_OK)
        return rc;
    if (!out)
        return set_error(ECHO_ERR_INVALID, "out is NULL");
    if (variant & ~kVariantBits)
        return set_error(ECHO_ERR_INVALID, "unknown variant bits 0x%x", variant);
    model_bytes(P, n, group, dtype, enable != 0, variant, out);
    return ECHO_OK;
}

int echo_set_variant(echo_handle *h, int variant)
{
    int rc;
    if ((rc = check_handle(h)) != ECHO_OK || (rc = check_device(h)) != ECHO_OK)
        return rc;
    if (variant & ~kVariantBits)
        return set_error(ECHO_ERR_INVALID, "unknown variant bits 0x%x", variant);
    if ((variant & ECHO_VARIANT_SENDER_EF) && !h->eps) {
        const size_t bytes = 2 * static_cast<size_t>(h->P) * h->n * sizeof(float);
        cudaError_t e = cudaDeviceSynchronize();
        if (e == cudaSuccess)
            e = dev_alloc(h, reinterpret_cast<void **>(&h->eps), bytes);
        if (e != cudaSuccess) {
            h->eps = nullptr;
            cudaGetLastError();
            return set_error(ECHO_ERR_OOM, "sender-error state of %zu bytes: %s", bytes, cudaGetErrorString(e));
        }
        e = cudaMemset(h->eps, 0, bytes);
        if (e == cudaSuccess)
            e = cudaDeviceSynchronize();
        if (e != cudaSuccess)
            return cuda_error(e, "echo_set_variant");
    }
    h->variant = variant;
    return ECHO_OK;
}

int echo_get_sender_state(echo_handle *h, int phase, int rank, size_t offset, size_t count, float *host)
{
    int rc;
    if ((rc = check_handle(h)) != ECHO_OK || (rc = check_phase(phase)) != ECHO_OK ||
        (rc = check_device(h)) != ECHO_OK)
        return rc;
    if (!h->eps)
        return set_error(ECHO_ERR_INVALID, "sender feedback was never switched on (echo_set_variant)");
    if (rank < 0 || rank >= h->P || !host || offset > h->n || count > h->n - offset)
        return set_error(ECHO_ERR_INVALID, "bad rank, range or NULL output");
    const float *src = h->eps + (static_cast<size_t>(phase) * h->P + rank) * h->n + offset;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess)
        e = cudaMemcpy(host, src, count * sizeof(float), cudaMemcpyDeviceToHost);
    return e == cudaSuccess ? ECHO_OK : cuda_error(e, "echo_get_sender_state");
}

int echo_set_sender_state(echo_handle *h, int phase, int rank, const float *host)
{
    int rc;
    if ((rc = check_handle(h)) != ECHO_OK || (rc = check_phase(phase)) != ECHO_OK ||
        (rc = check_device(h)) != ECHO_OK)
        return rc;
    if (!h->eps)
        return set_error(ECHO_ERR_INVALID, "sender feedback was never switched on (echo_set_variant)");
    if (rank < 0 || rank >= h->P || !host)
        return set_error(ECHO_ERR_INVALID, "bad rank or NULL input");
    float *dst = h->eps + (static_cast<size_t>(phase) * h->P + rank) * h->n;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess)
        e = cudaMemcpy(dst, host, h->n * sizeof(float), cudaMemcpyHostToDevice);
    return e == cudaSuccess ? ECHO_OK : cuda_error(e, "echo_set_sender_state");
}

echo_handle *echo_create(int P, size_t n, int group, int dtype)
{
    if (check_shape(P, n, group, dtype) != ECHO_OK)
        return nullptr;
    if (fault_injected("alloc")) {
        set_error(ECHO_ERR_OOM, "injected allocation failure (ECHO_FAULT=alloc)");
        return nullptr;
    }
    echo_handle *h = new (std::nothrow) echo_handle();
    if (!h) {
        set_error(ECHO_ERR_OOM, "host allocation of the handle failed");
        return nullptr;
    }
    h->P = P;
    h->n = n;
    h->dtype = dtype;
    h->group = group;
    h->lanes_log2 = 0; // group = 8 << lanes_log2 (a power of two in [16, 128])
    while ((8u << h->lanes_log2) != static_cast<uint32_t>(group))
        h->lanes_log2++;
    h->scale_stride = (2 * (n / group) + 15) / 16 * 16; // room for binary16 scales
    cudaError_t e = cudaGetDevice(&h->device);
    if (e != cudaSuccess) {
        cuda_error(e, "cudaGetDevice");
        delete h;
        return nullptr;
    }
    struct {
        void **p;
        size_t bytes;
    } allocs[] = {
        {reinterpret_cast<void **>(&h->codes1), static_cast<size_t>(P) * (n / 2)},
        {reinterpret_cast<void **>(&h->scales1), static_cast<size_t>(P) * h->scale_stride},
        {reinterpret_cast<void **>(&h->qcodes), n / 2},
        {reinterpret_cast<void **>(&h->qscales), h->scale_stride},
        {reinterpret_cast<void **>(&h->state), 4 * n * sizeof(float)},
        {reinterpret_cast<void **>(&h->dstatus), sizeof(int)},
    };
    for (auto &a : allocs) {
        e = dev_alloc(h, a.p, a.bytes);
        if (e != cudaSuccess) {
            if (e == cudaErrorMemoryAllocation)
                set_error(ECHO_ERR_OOM, "cudaMalloc of %zu bytes failed: %s", a.bytes, cudaGetErrorString(e));
            else
                cuda_error(e, "cudaMalloc");
            cudaGetLastError();
            free_handle(h);
            return nullptr;
        }
    }
    e = cudaMemset(h->state, 0, 4 * n * sizeof(float));
    if (e == cudaSuccess)
        e = cudaMemset(h->dstatus, 0, sizeof(int));
    if (e == cudaSuccess)
        e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        cuda_error(e, "echo_create");
        free_handle(h);
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    g_live.insert(h);
    return h;
}

int echo_destroy(echo_handle *h)
{
    if (!h)
        return ECHO_OK;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_live.erase(h))
            return set_error(ECHO_ERR_INVALID, "handle %p is unknown or destroyed", static_cast<void *>(h));
    }
    cudaDeviceSynchronize();
    free_handle(h);
    return ECHO_OK;
}

int echo_allreduce(echo_handle *h, void *const rank_ptrs[], int phase, void *stream)
{
    return allreduce_impl(h, const_cast<const void *const *>(rank_ptrs), rank_ptrs, phase, stream);
}

int echo_allreduce_out(echo_handle *h, const void *const send_ptrs[], void *const recv_ptrs[], int phase,
                       void *stream)
{
    return allreduce_impl(h, send_ptrs, recv_ptrs, phase, stream);
}

int echo_allreduce_host(echo_handle *h, const void *const host_send[], void *host_recv, int phase, void *stream)
{
    int rc;
    if ((rc = check_handle(h)) != ECHO_OK || (rc = check_phase(phase)) != ECHO_OK ||
        (rc = check_device(h)) != ECHO_OK)
        return rc;
    if (!host_send || !host_recv)
        return set_error(ECHO_ERR_INVALID, "host buffer pointer is NULL");
    for (int r = 0; r < h->P; r++)
        if (!host_send[r])
            return set_error(ECHO_ERR_INVALID, "host send pointer of rank %d is NULL", r);
    if (fault_injected("launch"))
        return set_error(ECHO_ERR_CUDA, "injected launch failure (ECHO_FAULT=launch)");
    const size_t eb = elem_bytes(h->dtype);
    cudaError_t e;
    if (!h->staging) {
        if ((e = dev_alloc(h, reinterpret_cast<void **>(&h->staging), static_cast<size_t>(h->P) * h->n * eb)) !=
            cudaSuccess) {
            h->staging = nullptr;
            cudaGetLastError();
            return set_error(ECHO_ERR_OOM, "staging allocation failed: %s", cudaGetErrorString(e));
        }
        for (cudaStream_t *s : {&h->s_in, &h->s_comp, &h->s_out})
            if ((e = cudaStreamCreateWithFlags(s, cudaStreamNonBlocking)) != cudaSuccess)
                return cuda_error(e, "cudaStreamCreate");
        for (cudaEvent_t *ev : {&h->e_start, &h->e_in, &h->e_comp, &h->e_done})
            if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess)
                return cuda_error(e, "cudaEventCreate");
    }
    const void *dsend[ECHO_MAX_RANKS];
    void *drecv[ECHO_MAX_RANKS];
    for (int r = 0; r < h->P; r++) {
        drecv[r] = h->staging + static_cast<size_t>(r) * h->n * eb;
        dsend[r] = drecv[r];
    }
    cudaStream_t user = static_cast<cudaStream_t>(stream);
    // The three internal streams start after the caller's prior work.
    if ((e = cudaEventRecord(h->e_start, user)) != cudaSuccess)
        return cuda_error(e, "cudaEventRecord");
    for (cudaStream_t s : {h->s_in, h->s_comp, h->s_out})
        if ((e = cudaStreamWaitEvent(s, h->e_start, 0)) != cudaSuccess)
            return cuda_error(e, "cudaStreamWaitEvent");
    // Pieces of kHostPiece elements: copy in (s_in) -> K1..K3 (s_comp) ->
    // copy the result out (s_out), so transfers of one piece overlap the
    // kernels of the previous one.
    for (size_t a = 0; a < h->n; a += kHostPiece) {
        const size_t b = a + kHostPiece < h->n ? a + kHostPiece : h->n;
        for (int r = 0; r < h->P; r++) {
            e = cudaMemcpyAsync(static_cast<uint8_t *>(drecv[r]) + a * eb,
                                static_cast<const uint8_t *>(host_send[r]) + a * eb, (b - a) * eb,
                                cudaMemcpyHostToDevice, h->s_in);
            if (e != cudaSuccess)
                return cuda_error(e, "cudaMemcpyAsync H2D");
        }
        if ((e = cudaEventRecord(h->e_in, h->s_in)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(h->s_comp, h->e_in, 0)) != cudaSuccess)
            return cuda_error(e, "event ordering");
        rc = enqueue_call(h, dsend, drecv, phase, h->s_comp, static_cast<uint32_t>(a / echo::kChunk),
                          static_cast<uint32_t>(b / echo::kChunk), false);
        if (rc != ECHO_OK)
            return rc;
        if ((e = cudaEventRecord(h->e_comp, h->s_comp)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(h->s_out, h->e_comp, 0)) != cudaSuccess)
            return cuda_error(e, "event ordering");
        e = cudaMemcpyAsync(static_cast<uint8_t *>(host_recv) + a * eb, static_cast<uint8_t *>(drecv[0]) + a * eb,
                            (b - a) * eb, cudaMemcpyDeviceToHost, h->s_out);
        if (e != cudaSuccess)
            return cuda_error(e, "cudaMemcpyAsync D2H");
    }
    if ((e = cudaEventRecord(h->e_done, h->s_out)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(user, h->e_done, 0)) != cudaSuccess ||
        (e = cudaStreamSynchronize(user)) != cudaSuccess)
        return cuda_error(e, "echo_allreduce_host completion");
    count_call(h);
    return ECHO_OK;
}

int echo_reset(echo_handle *h, int phase_mask)
{
    int rc;
    if ((rc = check_handle(h)) != ECHO_OK || (rc = check_device(h)) != ECHO_OK)
        return rc;
    if (phase_mask < 0 || phase_mask > 3)
        return set_error(ECHO_ERR_INVALID, "phase_mask %d: only bits 0 (fwd) and 1 (bwd) exist", phase_mask);
    cudaError_t e = cudaDeviceSynchronize();
    for (int p = 0; p < 2 && e == cudaSuccess; p++) {
        if (!(phase_mask & (1 << p)))
            continue;
        e = cudaMemset(h->state + static_cast<size_t>(p) * 2 * h->n, 0, 2 * h->n * sizeof(float));
        if (e == cudaSuccess && h->eps)
            e = cudaMemset(h->eps + static_cast<size_t>(p) * h->P * h->n, 0,
                           static_cast<size_t>(h->P) * h->n * sizeof(float));
    }
    if (e == cudaSuccess)
        e = cudaDeviceSynchronize();
    return e == cudaSuccess ? ECHO_OK : cuda_error(e, "echo_reset");
}

int echo_set_params(echo_handle *h, float beta_fast, float beta_slow, float lambda, int enable)
{
    int rc = check_handle(h);
    if (rc != ECHO_OK)
        return rc;
    if (!(beta_fast >= 0.f && beta_fast < 1.f) || !(beta_slow >= 0.f && beta_slow < 1.f) ||
        !(lambda >= 0.f && lambda <= 1.f) || (enable != 0 && enable != 1))
        return set_error(ECHO_ERR_INVALID,
                         "parameters out of range: beta_fast %g, beta_slow %g in [0,1), lambda %g in [0,1], "
                         "enable %d in {0,1}",
                         beta_fast, beta_slow, lambda, enable);
    h->beta_f = beta_fast;
    h->beta_s = beta_slow;
    h->lambda = lambda;
    h->enable = enable != 0;
    return ECHO_OK;
}

int echo_get_state_range(echo_handle *h, int phase, size_t offset, size_t count, float *f_host, float *s_host)
{
    int rc;
    if ((rc = check_handle(h)) != ECHO_OK || (rc = check_phase(phase)) != ECHO_OK ||
        (rc = check_device(h)) != ECHO_OK)
        return rc;
    if (offset > h->n || count > h->n - offset)
        return set_error(ECHO_ERR_INVALID, "range [%zu, %zu+%zu) exceeds n = %zu", offset, offset, count, h->n);
    const float *f = h->state + static_cast<size_t>(phase) * 2 * h->n;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess && f_host)
        e = cudaMemcpy(f_host, f + offset, count * sizeof(float), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && s_host)
        e = cudaMemcpy(s_host, f + h->n + offset, count * sizeof(float), cudaMemcpyDeviceToHost);
    return e == cudaSuccess ? ECHO_OK : cuda_error(e, "echo_get_state");
}

int echo_get_state(echo_handle *h, int phase, float *f_host, float *s_host)
{
    int rc = check_handle(h);
    if (rc != ECHO_OK)
        return rc;
    return echo_get_state_range(h, phase, 0, h->n, f_host, s_host);
}

int echo_set_state(echo_handle *h, int phase, const float *f_host, const float *s_host)
{
    int rc;
    if ((rc = check_handle(h)) != ECHO_OK || (rc = check_phase(phase)) != ECHO_OK ||
        (rc = check_device(h)) != ECHO_OK)
        return rc;
    if (!f_host || !s_host)
        return set_error(ECHO_ERR_INVALID, "state pointer is NULL");
    float *f = h->state + static_cast<size_t>(phase) * 2 * h->n;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess)
        e = cudaMemcpy(f, f_host, h->n * sizeof(float), cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
        e = cudaMemcpy(f + h->n, s_host, h->n * sizeof(float), cudaMemcpyHostToDevice);
    return e == cudaSuccess ? ECHO_OK : cuda_error(e, "echo_set_state");
}

int echo_get_wire_range(echo_handle *h, int stage, int rank, size_t group_offset, size_t ngroups,
                        uint8_t *codes_host, uint8_t *scales_host)
{
    int rc;
    if ((rc = check_handle(h)) != ECHO_OK || (rc = check_device(h)) != ECHO_OK)
        return rc;
    const size_t groups = h->n / h->group;
    if (stage != 1 && stage != 2)
        return set_error(ECHO_ERR_INVALID, "stage %d is neither 1 (per-rank wire) nor 2 (requantised)", stage);
    if (stage == 1 && (rank < 0 || rank >= h->P))
        return set_error(ECHO_ERR_INVALID, "rank %d outside [0, %d)", rank, h->P);
    if (group_offset > groups || ngroups > groups - group_offset)
        return set_error(ECHO_ERR_INVALID, "group range exceeds %zu groups", groups);
    const uint8_t *codes = stage == 1 ? h->codes1 + static_cast<size_t>(rank) * (h->n / 2) : h->qcodes;
    const uint8_t *scales = stage == 1 ? h->scales1 + static_cast<size_t>(rank) * h->scale_stride : h->qscales;
    const size_t sb = (h->variant & ECHO_VARIANT_FP16_SCALE) ? 2 : 1; // bytes per scale
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess && codes_host)
        e = cudaMemcpy(codes_host, codes + group_offset * (h->group / 2), ngroups * (h->group / 2),
                       cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && scales_host)
        e = cudaMemcpy(scales_host, scales + sb * group_offset, sb * ngroups, cudaMemcpyDeviceToHost);
    return e == cudaSuccess ? ECHO_OK : cuda_error(e, "echo_get_wire");
}

int echo_get_wire(echo_handle *h, int stage, int rank, uint8_t *codes_host, uint8_t *scales_host)
{
    int rc = check_handle(h);
    if (rc != ECHO_OK)
        return rc;
    return echo_get_wire_range(h, stage, rank, 0, h->n / h->group, codes_host, scales_host);
}

int echo_stats(echo_handle *h, uint64_t *link_bytes, uint64_t *model_hbm_bytes, uint64_t *calls)
{
    int rc = check_handle(h);
    if (rc != ECHO_OK)
        return rc;
    if (link_bytes)
        *link_bytes = h->link_bytes;
    if (model_hbm_bytes)
        *model_hbm_bytes = h->hbm_bytes;
    if (calls)
        *calls = h->calls;
    return ECHO_OK;
}

int echo_set_fused_limit(echo_handle *h, size_t max_n)
{
    int rc = check_handle(h);
    if (rc != ECHO_OK)
        return rc;
    h->fused_limit = max_n;
    return ECHO_OK;
}

int echo_get_fused_limit(echo_handle *h, size_t *max_n)
{
    int rc = check_handle(h);
    if (rc != ECHO_OK)
        return rc;
    if (!max_n)
        return set_error(ECHO_ERR_INVALID, "max_n is NULL");
    *max_n = h->fused_limit;
    return ECHO_OK;
}

int echo_set_timing(echo_handle *h, int enable)
{
    int rc = check_handle(h);
    if (rc != ECHO_OK)
        return rc;
    if (enable && !h->ring[0][0]) {
        if ((rc = check_device(h)) != ECHO_OK)
            return rc;
        for (auto &slot : h->ring)
            for (cudaEvent_t &e : slot) {
                cudaError_t err = cudaEventCreate(&e);
                if (err != cudaSuccess)
                    return cuda_error(err, "cudaEventCreate");
            }
    }
    if (enable) {
        // Start a new measurement: drain the slots still in flight first.
        if ((rc = fold_timings(h, h->ring_calls)) != ECHO_OK)
            return rc;
        h->ring_calls = h->folded = 0;
        h->total_ms[0] = h->total_ms[1] = h->total_ms[2] = 0.0;
    }
    h->timing = enable != 0;
    return ECHO_OK;
}

int echo_last_kernel_ms(echo_handle *h, float ms[3])
{
    int rc = check_handle(h);
    if (rc != ECHO_OK)
        return rc;
    if (!ms)
        return set_error(ECHO_ERR_INVALID, "ms is NULL");
    if (h->last_slot < 0)
        return set_error(ECHO_ERR_INVALID, "the last call was not timed (echo_set_timing)");
    cudaError_t e = slot_ms(h, h->last_slot, ms);
    return e == cudaSuccess ? ECHO_OK : cuda_error(e, "echo_last_kernel_ms");
}

int echo_device_status(echo_handle *h, int *status, int clear)
{
    int rc;
    if ((rc = check_handle(h)) != ECHO_OK || (rc = check_device(h)) != ECHO_OK)
        return rc;
    if (!status)
        return set_error(ECHO_ERR_INVALID, "status is NULL");
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess)
        e = cudaMemcpy(status, h->dstatus, sizeof(int), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && clear)
        e = cudaMemset(h->dstatus, 0, sizeof(int));
    if (e == cudaSuccess && clear)
        e = cudaDeviceSynchronize();
    return e == cudaSuccess ? ECHO_OK : cuda_error(e, "echo_device_status");
}

int echo_debug_build(void) { return ECHO_DEBUG ? 1 : 0; }

int echo_debug_touch_guard(echo_handle *h)
{
    int rc;
    if ((rc = check_handle(h)) != ECHO_OK || (rc = check_device(h)) != ECHO_OK)
        return rc;
    if (!ECHO_DEBUG || h->guards.count < 2)
        return set_error(ECHO_ERR_UNSUPPORTED, "guard bytes exist only in the debug build");
    // the first byte after the stage-1 code buffer (the first buffer allocated)
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess)
        e = cudaMemset(const_cast<uint8_t *>(h->guards.region[1]), 0, 1);
    if (e == cudaSuccess)
        e = cudaDeviceSynchronize();
    return e == cudaSuccess ? ECHO_OK : cuda_error(e, "echo_debug_touch_guard");
}

int echo_kernel_ms_total(echo_handle *h, double ms[3], uint64_t *timed_calls)
{
    int rc = check_handle(h);
    if (rc != ECHO_OK)
        return rc;
    if (!ms)
        return set_error(ECHO_ERR_INVALID, "ms is NULL");
    if ((rc = fold_timings(h, h->ring_calls)) != ECHO_OK)
        return rc;
    for (int k = 0; k < 3; k++)
        ms[k] = h->total_ms[k];
    if (timed_calls)
        *timed_calls = h->folded;
    return ECHO_OK;
}

} // extern "C"
