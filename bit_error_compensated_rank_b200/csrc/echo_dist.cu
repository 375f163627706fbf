// echo_dist.cu - the all-reduce with one handle per rank (echo_dist_* in
// include/echo.h).
//
// Each rank (a process, or one of several handles in a process) holds its own
// partial, the compensator state of the segment it owns, and an exported
// block that the other ranks write into (through CUDA IPC across processes):
// a receive slot per rank for the owned segment's stage-1 wire, and the
// gathered requantised tensor. The three kernels run as three stages, and the
// wire moves inside them as plain stores into the other ranks' blocks [rit.work "Echo 4-bit GPU communication", section "How
// Echo returns the error to later calls": segments go to their owner, the
// owner's compressed total goes back to every rank]:
//   stage 1  kernel 1 on this rank's partial (one rank, owner mapping of the
//            whole group) stores each segment's codes and scales straight
//            into its owner's receive slot for this rank;
//   stage 2  kernel 2 reduces and requantises the owned segment from the
//            local receive slots, updates its state, and stores the
//            requantised segment into every rank's gathered tensor;
//   stage 3  kernel 3 restores the local gathered tensor into this rank's
//            output.
// On several GPUs the stores cross NVLink as peer stores; the kernels read
// local memory only. No kernel waits on another process or spins on a flag.
// The stages are ordered on the GPU by events: every rank records one
// interprocess event after each of its stages, and before a stage each rank's
// stream waits for the events of the stages it depends on on every rank:
//   stage 1 (call k) writes the owners' receive slots, which stage 2 of call
//            k-1 read: it waits for every rank's stage-2 event;
//   stage 2 reads the receive slots every rank's stage 1 wrote, and writes
//            the gathered tensors that stage 3 of call k-1 read: it waits for
//            every rank's stage-1 and stage-3 events;
//   stage 3 reads the gathered tensor every rank's stage 2 wrote: it waits
//            for every rank's stage-2 event.
// A wait takes the event's latest record at the time it is enqueued, so the
// caller puts a host barrier over all ranks after stage 1 and after stage 2
// of every call (each rank has enqueued its record before any rank enqueues
// the waits that need it). The host never waits for the GPU, and the next
// record of each event comes only after the following barrier. Ranks in one
// process use each other's buffers and events directly; ranks in other
// processes through CUDA IPC. Every operation is the single-process path's,
// so the results are bit for bit the same.
#include "echo.h"
#include "echo_kernels.h"

#include <cuda_runtime.h>

#include <unistd.h>

#include <chrono>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <set>

struct echo_dist {
    int world = 0, rank = 0;
    size_t n = 0, seg = 0;
    int group = ECHO_GROUP;
    uint32_t lanes_log2 = 2;
    int dtype = ECHO_BF16;
    int device = 0;
    int variant = 0;
    float beta_f = 0.5f, beta_s = 0.875f, lambda = 0.5f;
    bool enable = true;
    // exported block: receive slots [world][seg/2] codes and [world][seg scale
    // stride] scales for the owned segment, then the gathered requantised
    // tensor ([n/2] codes, [2n/G rounded up] scales)
    uint8_t *xbuf = nullptr;
    size_t off_recv_scales = 0, off_q_codes = 0, off_q_scales = 0;
    size_t row_scale_stride = 0, seg_scale_stride = 0; // 2n/G and 2seg/G rounded up to 16
    float *state = nullptr; // [phase][f|s][seg]: the owned segment's estimates
    float *eps = nullptr;   // [phase][n], sender feedback
    int *dstatus = nullptr;
    const uint8_t *peer[ECHO_MAX_RANKS] = {}; // every rank's exported block (own included)
    bool peer_ipc[ECHO_MAX_RANKS] = {};       // opened through CUDA IPC (closed at destroy)
    cudaEvent_t done[3] = {};                 // recorded after this rank's stage 1, 2, 3
    cudaEvent_t peer_done[ECHO_MAX_RANKS][3] = {}; // every rank's (own included)
    bool connected = false;
    uint64_t calls = 0;
};

namespace {

std::mutex g_mu;
std::set<const echo_dist *> g_live;

constexpr long long kWaitCycles = 1LL << 31;

// Layout of the blob echo_dist_export writes (ECHO_DIST_HANDLE_BYTES):
//   [0, 64)     CUDA IPC handle of the exported block
//   [64, 256)   CUDA IPC handles of the three stage events
//   [256, 264)  token of the exporting process
//   [264, 272)  the exporting handle (used only inside that process)
//   [272, 280)  n;  [280, 284) world;  [284, 288) rank;  [288, 292) group;
//   [292, 296)  dtype;  the rest zero
struct Blob {
    cudaIpcMemHandle_t mem;
    cudaIpcEventHandle_t ev[3];
    uint64_t token;
    uint64_t self;
    uint64_t n;
    int32_t world, rank, group, dtype;
};
static_assert(sizeof(cudaIpcMemHandle_t) == 64 && sizeof(cudaIpcEventHandle_t) == 64, "CUDA IPC handle size");
static_assert(sizeof(Blob) <= ECHO_DIST_HANDLE_BYTES, "exported blob size");

// Identifies this process in exported blobs: the pid and the start time.
uint64_t process_token()
{
    static const uint64_t token =
        (static_cast<uint64_t>(getpid()) << 32) ^
        static_cast<uint64_t>(std::chrono::steady_clock::now().time_since_epoch().count());
    return token;
}

int fail(int code, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    return echo::record_error(code, buf);
}

int cuda_fail(cudaError_t e, const char *what)
{
    return fail(ECHO_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

size_t round16(size_t x) { return (x + 15) / 16 * 16; }
size_t round256(size_t x) { return (x + 255) / 256 * 256; }

int check(const echo_dist *d)
{
    if (!d)
        return fail(ECHO_ERR_INVALID, "handle is NULL");
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_live.count(d))
            return fail(ECHO_ERR_INVALID, "distributed handle %p is unknown or destroyed",
                        static_cast<const void *>(d));
    }
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaGetDevice");
    if (dev != d->device)
        return fail(ECHO_ERR_INVALID, "the handle belongs to device %d, the current device is %d", d->device, dev);
    return ECHO_OK;
}

int check_user_buffer(const void *p, int device, const char *what)
{
    if (!p)
        return fail(ECHO_ERR_INVALID, "%s is NULL", what);
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0)
        return fail(ECHO_ERR_INVALID, "%s is not 16-byte aligned", what);
    cudaPointerAttributes attr;
    cudaError_t e = cudaPointerGetAttributes(&attr, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(ECHO_ERR_INVALID, "%s is not CUDA memory (%s)", what, cudaGetErrorString(e));
    }
    if ((attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) || attr.device != device)
        return fail(ECHO_ERR_INVALID, "%s is not memory of device %d", what, device);
    return ECHO_OK;
}

void free_dist(echo_dist *d)
{
    for (int p = 0; p < d->world; p++) {
        if (!d->peer_ipc[p])
            continue;
        if (d->peer[p])
            cudaIpcCloseMemHandle(const_cast<uint8_t *>(d->peer[p]));
        for (int k = 0; k < 3; k++)
            if (d->peer_done[p][k])
                cudaEventDestroy(d->peer_done[p][k]);
    }
    for (int k = 0; k < 3; k++)
        if (d->done[k])
            cudaEventDestroy(d->done[k]);
    for (void *p : {static_cast<void *>(d->xbuf), static_cast<void *>(d->state), static_cast<void *>(d->eps),
                    static_cast<void *>(d->dstatus)})
        if (p)
            cudaFree(p);
    delete d;
}

echo::PipeCtl ctl_of(const echo_dist *d) { return echo::PipeCtl{d->dstatus, kWaitCycles, false}; }

int stage1(echo_dist *d, const void *x, int phase, cudaStream_t st)
{
    echo::K1Args a{};
    a.x.p[0] = x;
    a.f = d->state + static_cast<size_t>(phase) * 2 * d->seg; // the owned segment's estimates
    a.s = a.f + d->seg;
    a.to_owners = true;
    for (int p = 0; p < d->world; p++)
        a.owners.p[p] = const_cast<uint8_t *>(d->peer[p]);
    a.seg_code_bytes = d->seg / 2;
    a.recv_scales_off = d->off_recv_scales;
    a.seg_scale_stride = d->seg_scale_stride;
    a.n = d->n;
    a.scale_stride = d->row_scale_stride;
    a.chunk_begin = 0;
    a.chunk_end = static_cast<uint32_t>(d->n / echo::kChunk);
    a.lanes_log2 = d->lanes_log2;
    a.groups_per_seg = static_cast<uint32_t>(d->seg / d->group);
    a.rank_base = static_cast<uint32_t>(d->rank);
    a.lambda = d->lambda;
    a.one_minus_lambda = 1.0f - d->lambda;
    a.eps = (d->variant & ECHO_VARIANT_SENDER_EF) ? d->eps + static_cast<size_t>(phase) * d->n : nullptr;
    a.P = 1;
    a.bf16 = d->dtype == ECHO_BF16;
    a.enable = d->enable && !(d->variant & ECHO_VARIANT_OWNER_SUM);
    a.sender_ef = (d->variant & ECHO_VARIANT_SENDER_EF) != 0;
    a.fp16_scale = (d->variant & ECHO_VARIANT_FP16_SCALE) != 0;
    a.ctl = ctl_of(d);
    // Only the owned segment carries the correction: with compensation on,
    // one launch covers it with the state, and the rest of the row goes in
    // launches that stage no state (their tiles hold partials only, so they
    // are long enough to keep HBM busy).
    const uint32_t s0 = static_cast<uint32_t>(d->rank * (d->seg / echo::kChunk));
    const uint32_t s1 = s0 + static_cast<uint32_t>(d->seg / echo::kChunk);
    struct Range {
        uint32_t begin, end;
        bool comp;
    } ranges[3] = {{s0, s1, true}, {0, s0, false}, {s1, a.chunk_end, false}};
    const int nranges = a.enable ? 3 : 1;
    if (!a.enable)
        ranges[0] = {0, a.chunk_end, false};
    for (int i = 0; i < nranges; i++) {
        if (ranges[i].end <= ranges[i].begin)
            continue;
        echo::K1Args b = a;
        b.chunk_begin = ranges[i].begin;
        b.chunk_end = ranges[i].end;
        b.enable = a.enable && ranges[i].comp;
        cudaError_t e = echo::launch_k1_compensate_quantize_pack(b, st);
        if (e != cudaSuccess)
            return cuda_fail(e, "launch k1_compensate_quantize_pack");
    }
    return ECHO_OK;
}

int stage2(echo_dist *d, int phase, cudaStream_t st)
{
    float *f = d->state + static_cast<size_t>(phase) * 2 * d->seg;
    echo::K2Args a{};
    a.codes = d->xbuf; // the receive slots, one per rank
    a.scales = d->xbuf + d->off_recv_scales;
    a.f = f;
    a.s = f + d->seg;
    a.n = d->seg;
    a.scale_stride = d->seg_scale_stride;
    a.chunk_begin = 0;
    a.chunk_end = static_cast<uint32_t>(d->seg / echo::kChunk);
    a.lanes_log2 = d->lanes_log2;
    a.beta_f = d->beta_f;
    a.one_minus_beta_f = 1.0f - d->beta_f;
    a.beta_s = d->beta_s;
    a.one_minus_beta_s = 1.0f - d->beta_s;
    a.lambda = d->lambda;
    a.one_minus_lambda = 1.0f - d->lambda;
    a.P = d->world;
    a.enable = d->enable;
    a.owner_sum = d->enable && (d->variant & ECHO_VARIANT_OWNER_SUM);
    a.fp16_scale = (d->variant & ECHO_VARIANT_FP16_SCALE) != 0;
    a.bf16 = d->dtype == ECHO_BF16;
    a.to_ranks = true;
    for (int p = 0; p < d->world; p++)
        a.ranks.p[p] = const_cast<uint8_t *>(d->peer[p]) + d->off_q_codes;
    a.q_chunk0 = static_cast<uint32_t>(d->rank * (d->seg / echo::kChunk));
    a.q_group0 = static_cast<uint32_t>(d->rank * (d->seg / d->group));
    a.q_scales_off = d->off_q_scales - d->off_q_codes;
    a.q_scale_bytes = d->row_scale_stride;
    a.ctl = ctl_of(d);
    cudaError_t e = echo::launch_k2_owner_reduce_requant(a, st);
    return e == cudaSuccess ? ECHO_OK : cuda_fail(e, "launch k2_owner_reduce_requant");
}

int stage3(echo_dist *d, void *out, cudaStream_t st)
{
    echo::K3Args a{};
    a.qcodes = d->xbuf + d->off_q_codes; // written by every owner in stage 2
    a.qscales = d->xbuf + d->off_q_scales;
    a.out.p[0] = out;
    a.n = d->n;
    a.scale_stride = d->row_scale_stride;
    a.chunk_begin = 0;
    a.chunk_end = static_cast<uint32_t>(d->n / echo::kChunk);
    a.lanes_log2 = d->lanes_log2;
    a.P = 1;
    a.bf16 = d->dtype == ECHO_BF16;
    a.fp16_scale = (d->variant & ECHO_VARIANT_FP16_SCALE) != 0;
    a.ctl = ctl_of(d);
    cudaError_t e = echo::launch_k3_gather_dequant(a, st);
    return e == cudaSuccess ? ECHO_OK : cuda_fail(e, "launch k3_gather_dequant");
}

} // namespace

extern "C" {

echo_dist *echo_dist_create(int world, int rank, size_t n, int group, int dtype)
{
    if (world < 2 || world > ECHO_MAX_RANKS) {
        fail(ECHO_ERR_INVALID, "world = %d is outside [2, %d]", world, ECHO_MAX_RANKS);
        return nullptr;
    }
    if (rank < 0 || rank >= world) {
        fail(ECHO_ERR_INVALID, "rank %d outside [0, %d)", rank, world);
        return nullptr;
    }
    if (dtype != ECHO_BF16 && dtype != ECHO_FP32) {
        fail(ECHO_ERR_INVALID, "unknown dtype %d", dtype);
        return nullptr;
    }
    if (group != 16 && group != 32 && group != 64 && group != 128) {
        fail(ECHO_ERR_UNSUPPORTED, "group = %d: the built group sizes are 16, 32, 64 and 128", group);
        return nullptr;
    }
    // segments of whole groups whose code rows start on 16 bytes
    const size_t unit = static_cast<size_t>(world) * (group > 32 ? group : 32);
    if (n == 0 || n % unit != 0) {
        fail(ECHO_ERR_INVALID, "n = %zu must be a positive multiple of %zu (world x max(group, 32))", n, unit);
        return nullptr;
    }
    if (n > (size_t(1) << 34)) {
        fail(ECHO_ERR_UNSUPPORTED, "n = %zu exceeds the supported maximum 2^34", n);
        return nullptr;
    }
    echo_dist *d = new (std::nothrow) echo_dist();
    if (!d) {
        fail(ECHO_ERR_OOM, "host allocation of the handle failed");
        return nullptr;
    }
    d->world = world;
    d->rank = rank;
    d->n = n;
    d->seg = n / world;
    d->group = group;
    d->lanes_log2 = 0; // group = 8 << lanes_log2
    while ((8u << d->lanes_log2) != static_cast<uint32_t>(group))
        d->lanes_log2++;
    d->dtype = dtype;
    d->row_scale_stride = round16(2 * (n / group));
    d->seg_scale_stride = round16(2 * (d->seg / group));
    d->off_recv_scales = round256(static_cast<size_t>(world) * (d->seg / 2));
    d->off_q_codes = d->off_recv_scales + round256(static_cast<size_t>(world) * d->seg_scale_stride);
    d->off_q_scales = d->off_q_codes + round256(n / 2);
    const size_t xbytes = d->off_q_scales + round256(d->row_scale_stride);
    cudaError_t e = cudaGetDevice(&d->device);
    struct {
        void **p;
        size_t bytes;
    } allocs[] = {
        {reinterpret_cast<void **>(&d->xbuf), xbytes},
        {reinterpret_cast<void **>(&d->state), 4 * d->seg * sizeof(float)},
        {reinterpret_cast<void **>(&d->dstatus), sizeof(int)},
    };
    for (auto &a : allocs) {
        if (e == cudaSuccess)
            e = cudaMalloc(a.p, a.bytes);
    }
    for (int k = 0; k < 3 && e == cudaSuccess; k++)
        e = cudaEventCreateWithFlags(&d->done[k], cudaEventDisableTiming | cudaEventInterprocess);
    if (e == cudaSuccess)
        e = cudaMemset(d->state, 0, 4 * d->seg * sizeof(float));
    if (e == cudaSuccess)
        e = cudaMemset(d->dstatus, 0, sizeof(int));
    if (e == cudaSuccess)
        e = cudaMemset(d->xbuf, 0, xbytes);
    if (e == cudaSuccess)
        e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        if (e == cudaErrorMemoryAllocation)
            fail(ECHO_ERR_OOM, "device allocation failed: %s", cudaGetErrorString(e));
        else
            cuda_fail(e, "echo_dist_create");
        cudaGetLastError();
        free_dist(d);
        return nullptr;
    }
    d->peer[rank] = d->xbuf;
    for (int k = 0; k < 3; k++)
        d->peer_done[rank][k] = d->done[k];
    std::lock_guard<std::mutex> lock(g_mu);
    g_live.insert(d);
    return d;
}

int echo_dist_export(echo_dist *d, uint8_t handle[ECHO_DIST_HANDLE_BYTES])
{
    int rc = check(d);
    if (rc != ECHO_OK)
        return rc;
    if (!handle)
        return fail(ECHO_ERR_INVALID, "handle buffer is NULL");
    Blob b;
    std::memset(&b, 0, sizeof b);
    cudaError_t e = cudaIpcGetMemHandle(&b.mem, d->xbuf);
    for (int k = 0; k < 3 && e == cudaSuccess; k++)
        e = cudaIpcGetEventHandle(&b.ev[k], d->done[k]);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaIpcGetMemHandle / cudaIpcGetEventHandle");
    b.token = process_token();
    b.self = reinterpret_cast<uintptr_t>(d);
    b.n = d->n;
    b.world = d->world;
    b.rank = d->rank;
    b.group = d->group;
    b.dtype = d->dtype;
    std::memset(handle, 0, ECHO_DIST_HANDLE_BYTES);
    std::memcpy(handle, &b, sizeof b);
    return ECHO_OK;
}

namespace {

void disconnect(echo_dist *d)
{
    for (int q = 0; q < d->world; q++) {
        if (q == d->rank)
            continue;
        if (d->peer_ipc[q]) {
            if (d->peer[q])
                cudaIpcCloseMemHandle(const_cast<uint8_t *>(d->peer[q]));
            for (int k = 0; k < 3; k++)
                if (d->peer_done[q][k])
                    cudaEventDestroy(d->peer_done[q][k]);
        }
        d->peer[q] = nullptr;
        d->peer_ipc[q] = false;
        for (int k = 0; k < 3; k++)
            d->peer_done[q][k] = nullptr;
    }
}

} // namespace

int echo_dist_connect(echo_dist *d, const uint8_t *handles)
{
    int rc = check(d);
    if (rc != ECHO_OK)
        return rc;
    if (!handles)
        return fail(ECHO_ERR_INVALID, "handles is NULL");
    if (d->connected)
        return fail(ECHO_ERR_INVALID, "already connected");
    Blob b[ECHO_MAX_RANKS];
    for (int p = 0; p < d->world; p++) {
        std::memcpy(&b[p], handles + static_cast<size_t>(p) * ECHO_DIST_HANDLE_BYTES, sizeof(Blob));
        if (b[p].world != d->world || b[p].rank != p || b[p].n != d->n || b[p].group != d->group ||
            b[p].dtype != d->dtype)
            return fail(ECHO_ERR_INVALID,
                        "handle %d is from rank %d of world %d (n = %llu, group %d, dtype %d); expected rank %d of "
                        "world %d (n = %zu, group %d, dtype %d)",
                        p, b[p].rank, b[p].world, static_cast<unsigned long long>(b[p].n), b[p].group, b[p].dtype, p,
                        d->world, d->n, d->group, d->dtype);
    }
    const uint64_t me = process_token();
    for (int p = 0; p < d->world; p++) {
        if (p == d->rank)
            continue;
        cudaError_t e = cudaSuccess;
        if (b[p].token == me) {
            // a rank of this process: its buffers and events directly
            echo_dist *o = reinterpret_cast<echo_dist *>(static_cast<uintptr_t>(b[p].self));
            bool live;
            {
                std::lock_guard<std::mutex> lock(g_mu);
                live = g_live.count(o) != 0;
            }
            if (!live) {
                disconnect(d);
                return fail(ECHO_ERR_INVALID, "handle %d names a rank of this process that no longer exists", p);
            }
            if (o->device != d->device) {
                e = cudaDeviceEnablePeerAccess(o->device, 0);
                if (e == cudaErrorPeerAccessAlreadyEnabled) {
                    cudaGetLastError();
                    e = cudaSuccess;
                }
                if (e != cudaSuccess) {
                    cudaGetLastError();
                    disconnect(d);
                    return cuda_fail(e, "cudaDeviceEnablePeerAccess");
                }
            }
            d->peer[p] = o->xbuf;
            for (int k = 0; k < 3; k++)
                d->peer_done[p][k] = o->done[k];
            continue;
        }
        void *ptr = nullptr;
        e = cudaIpcOpenMemHandle(&ptr, b[p].mem, cudaIpcMemLazyEnablePeerAccess);
        if (e == cudaSuccess) {
            d->peer[p] = static_cast<const uint8_t *>(ptr);
            d->peer_ipc[p] = true;
            for (int k = 0; k < 3 && e == cudaSuccess; k++)
                e = cudaIpcOpenEventHandle(&d->peer_done[p][k], b[p].ev[k]);
        }
        if (e != cudaSuccess) {
            cudaGetLastError();
            if (ptr && !d->peer_ipc[p])
                cudaIpcCloseMemHandle(ptr);
            disconnect(d);
            return cuda_fail(e, "cudaIpcOpenMemHandle / cudaIpcOpenEventHandle");
        }
    }
    d->connected = true;
    return ECHO_OK;
}

int echo_dist_stage(echo_dist *d, int stage, const void *x, void *out, int phase, void *stream)
{
    int rc = check(d);
    if (rc != ECHO_OK)
        return rc;
    if (!d->connected)
        return fail(ECHO_ERR_INVALID, "not connected (echo_dist_connect)");
    if (phase != ECHO_FWD && phase != ECHO_BWD)
        return fail(ECHO_ERR_INVALID, "phase %d is neither ECHO_FWD (0) nor ECHO_BWD (1)", phase);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (stage < 1 || stage > 3)
        return fail(ECHO_ERR_INVALID, "stage %d is not 1, 2 or 3", stage);
    if (stage == 1 && (rc = check_user_buffer(x, d->device, "x")) != ECHO_OK)
        return rc;
    if (stage == 3 && (rc = check_user_buffer(out, d->device, "out")) != ECHO_OK)
        return rc;
    // the events of the stages this one depends on, on every rank
    const int deps[3][2] = {{2, 0}, {1, 3}, {2, 0}}; // stage numbers, 0 = none
    for (int j = 0; j < 2; j++) {
        const int dep = deps[stage - 1][j];
        if (!dep)
            continue;
        for (int p = 0; p < d->world; p++) {
            cudaError_t e = cudaStreamWaitEvent(st, d->peer_done[p][dep - 1], 0);
            if (e != cudaSuccess)
                return cuda_fail(e, "cudaStreamWaitEvent");
        }
    }
    rc = stage == 1 ? stage1(d, x, phase, st) : stage == 2 ? stage2(d, phase, st) : stage3(d, out, st);
    if (rc != ECHO_OK)
        return rc;
    cudaError_t e = cudaEventRecord(d->done[stage - 1], st);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaEventRecord");
    if (stage == 3)
        d->calls += 1;
    return ECHO_OK;
}

int echo_dist_set_params(echo_dist *d, float beta_fast, float beta_slow, float lambda, int enable)
{
    int rc = check(d);
    if (rc != ECHO_OK)
        return rc;
    if (!(beta_fast >= 0.f && beta_fast < 1.f) || !(beta_slow >= 0.f && beta_slow < 1.f) ||
        !(lambda >= 0.f && lambda <= 1.f) || (enable != 0 && enable != 1))
        return fail(ECHO_ERR_INVALID, "parameters out of range (beta in [0,1), lambda in [0,1], enable 0/1)");
    d->beta_f = beta_fast;
    d->beta_s = beta_slow;
    d->lambda = lambda;
    d->enable = enable != 0;
    return ECHO_OK;
}

int echo_dist_set_variant(echo_dist *d, int variant)
{
    int rc = check(d);
    if (rc != ECHO_OK)
        return rc;
    if (variant & ~(ECHO_VARIANT_OWNER_SUM | ECHO_VARIANT_SENDER_EF | ECHO_VARIANT_FP16_SCALE))
        return fail(ECHO_ERR_INVALID, "unknown variant bits 0x%x", variant);
    if ((variant & ECHO_VARIANT_SENDER_EF) && !d->eps) {
        const size_t bytes = 2 * d->n * sizeof(float);
        cudaError_t e = cudaMalloc(&d->eps, bytes);
        if (e == cudaSuccess)
            e = cudaMemset(d->eps, 0, bytes);
        if (e == cudaSuccess)
            e = cudaDeviceSynchronize();
        if (e != cudaSuccess) {
            cudaGetLastError();
            if (d->eps)
                cudaFree(d->eps);
            d->eps = nullptr;
            return fail(ECHO_ERR_OOM, "sender-error state of %zu bytes: %s", bytes, cudaGetErrorString(e));
        }
    }
    d->variant = variant;
    return ECHO_OK;
}

int echo_dist_get_state(echo_dist *d, int phase, float *f_host, float *s_host)
{
    int rc = check(d);
    if (rc != ECHO_OK)
        return rc;
    if (phase != ECHO_FWD && phase != ECHO_BWD)
        return fail(ECHO_ERR_INVALID, "phase %d is neither ECHO_FWD (0) nor ECHO_BWD (1)", phase);
    const float *f = d->state + static_cast<size_t>(phase) * 2 * d->seg;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess && f_host)
        e = cudaMemcpy(f_host, f, d->seg * sizeof(float), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && s_host)
        e = cudaMemcpy(s_host, f + d->seg, d->seg * sizeof(float), cudaMemcpyDeviceToHost);
    return e == cudaSuccess ? ECHO_OK : cuda_fail(e, "echo_dist_get_state");
}

int echo_dist_device_status(echo_dist *d, int *status, int clear)
{
    int rc = check(d);
    if (rc != ECHO_OK)
        return rc;
    if (!status)
        return fail(ECHO_ERR_INVALID, "status is NULL");
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess)
        e = cudaMemcpy(status, d->dstatus, sizeof(int), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && clear)
        e = cudaMemset(d->dstatus, 0, sizeof(int));
    if (e == cudaSuccess && clear)
        e = cudaDeviceSynchronize();
    return e == cudaSuccess ? ECHO_OK : cuda_fail(e, "echo_dist_device_status");
}

int echo_dist_destroy(echo_dist *d)
{
    if (!d)
        return ECHO_OK;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_live.erase(d))
            return fail(ECHO_ERR_INVALID, "distributed handle %p is unknown or destroyed",
                        static_cast<const void *>(d));
    }
    cudaDeviceSynchronize();
    free_dist(d);
    return ECHO_OK;
}

} // extern "C"
