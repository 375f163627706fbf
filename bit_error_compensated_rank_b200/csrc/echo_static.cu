// echo_static.cu - the all-reduce without any device allocation.
//
// Some callers cannot allocate device memory when they want to reduce: a
// serving process that reserved all of HBM for its own pool or KV cache at
// start-up, a plugin that runs inside a host application which owns every
// allocation, or a latency-critical path where a cudaMalloc (which can
// synchronise the device) is not acceptable. echo_allreduce_static serves
// them: the caller passes its rank buffers and the compensator state, and the
// wire buffers the three kernels exchange live in a fixed scratch array
// compiled into the library (ECHO_STATIC_SCRATCH_BYTES, 32 MiB, held on every
// GPU where it has been set up until the process exits).
//
// In host code the array's name is only a host-side stand-in, not a device
// address, so the device address is looked up with cudaGetSymbolAddress, once
// per device, by the first call of echo_allreduce_static or
// echo_static_status made with that device current. Under CUDA's lazy module
// loading that lookup is also when the 32 MiB are taken from the device, so a
// caller that reserves the rest of HBM for its own pool, or captures streams
// into graphs, makes one such call first. The set-up also zeroes the device
// status word at the start of the array. The kernels only ever OR bits into
// that word (bounded waits that ran out), so it keeps them across calls until
// echo_static_status clears it. Every call shares the one array and leaves
// its contents behind; calls whose work overlaps on the GPU (two streams, or
// two host threads, at once) race on the array.
#include "echo.h"
#include "echo_bulk.cuh"
#include "echo_kernels.h"

#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

namespace {

static __device__ __align__(256) uint8_t g_static_scratch[ECHO_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
constexpr size_t kMaxN = size_t(1) << 34;          // as echo_create: chunk indices stay 32-bit
constexpr long long kWaitCycles = 1LL << 31;      // about a second at B200 clocks
constexpr long long kStallWaitCycles = 1LL << 20; // the injected stall (tests)

std::mutex g_addr_mu;
uint8_t *g_addr[kMaxDevices] = {}; // device address of the array, per device

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

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

bool disjoint(const void *a, size_t abytes, const void *b, size_t bbytes)
{
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x + abytes <= y || y + bbytes <= x;
}

int check_device_pointer(const void *p, int device, const char *what, int index)
{
    if (!p)
        return fail(ECHO_ERR_INVALID, "%s %d is NULL", what, index);
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0)
        return fail(ECHO_ERR_INVALID, "%s %d is not 16-byte aligned", what, index);
    cudaPointerAttributes attr;
    cudaError_t e = cudaPointerGetAttributes(&attr, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(ECHO_ERR_INVALID, "%s %d is not CUDA memory (%s)", what, index, cudaGetErrorString(e));
    }
    if ((attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) || attr.device != device)
        return fail(ECHO_ERR_INVALID, "%s %d is not memory of the current device %d", what, index, device);
    return ECHO_OK;
}

// Test hook shared with the handle path: ECHO_FAULT=stall launches the
// kernels with no loads issued and a short wait bound, so every CTA's first
// wait runs out and records its bit in the status word.
bool stall_injected()
{
    const char *e = std::getenv("ECHO_FAULT");
    return e && std::strcmp(e, "stall") == 0;
}

// The array's device address on the current device. The first lookup on a
// device also zeroes the status word (synchronously).
int static_base(uint8_t **base)
{
    int device = -1;
    cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess)
        return fail(ECHO_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (device < 0 || device >= kMaxDevices)
        return fail(ECHO_ERR_UNSUPPORTED, "device %d is beyond the %d devices this entry point tracks", device,
                    kMaxDevices);
    std::lock_guard<std::mutex> lock(g_addr_mu);
    if (!g_addr[device]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess)
            return fail(ECHO_ERR_CUDA, "cudaGetSymbolAddress of the static scratch: %s", cudaGetErrorString(e));
        e = cudaMemset(p, 0, sizeof(int));
        if (e == cudaSuccess)
            e = cudaDeviceSynchronize();
        if (e != cudaSuccess)
            return fail(ECHO_ERR_CUDA, "clearing the static status word: %s", cudaGetErrorString(e));
        g_addr[device] = static_cast<uint8_t *>(p);
    }
    *base = g_addr[device];
    return ECHO_OK;
}

} // namespace

extern "C" int echo_static_status(int *status, int clear)
{
    if (!status)
        return fail(ECHO_ERR_INVALID, "status is NULL");
    uint8_t *base = nullptr;
    int rc = static_base(&base);
    if (rc != ECHO_OK)
        return rc;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess)
        e = cudaMemcpy(status, base, sizeof(int), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && clear)
        e = cudaMemset(base, 0, sizeof(int));
    if (e == cudaSuccess && clear)
        e = cudaDeviceSynchronize();
    if (e != cudaSuccess)
        return fail(ECHO_ERR_CUDA, "echo_static_status: %s", cudaGetErrorString(e));
    return ECHO_OK;
}

extern "C" int echo_allreduce_static(int P, size_t n, int dtype, void *const rank_ptrs[], float *f, float *s,
                                     float beta_fast, float beta_slow, float lambda, int enable, void *stream)
{
    // ---- arguments (nothing is enqueued on any error) ----
    if (P < 2 || P > ECHO_MAX_RANKS)
        return fail(ECHO_ERR_INVALID, "P = %d is outside [2, %d]", P, ECHO_MAX_RANKS);
    if (dtype != ECHO_BF16 && dtype != ECHO_FP32)
        return fail(ECHO_ERR_INVALID, "unknown dtype %d", dtype);
    if (n == 0 || n % (static_cast<size_t>(P) * ECHO_GROUP) != 0)
        return fail(ECHO_ERR_INVALID, "n = %zu must be a positive multiple of P*32 = %d", n, P * ECHO_GROUP);
    // Before any size arithmetic, so that nothing below can wrap around.
    if (n > kMaxN)
        return fail(ECHO_ERR_UNSUPPORTED, "n = %zu exceeds the supported maximum %zu", n, kMaxN);
    if (!(beta_fast >= 0.f && beta_fast < 1.f) || !(beta_slow >= 0.f && beta_slow < 1.f) ||
        !(lambda >= 0.f && lambda <= 1.f) || (enable != 0 && enable != 1))
        return fail(ECHO_ERR_INVALID, "parameters out of range (beta in [0,1), lambda in [0,1], enable 0/1)");
    const size_t scale_stride = (n / ECHO_GROUP + 15) / 16 * 16;
    const size_t off_codes1 = 256; // bytes [0, 256): device status word
    const size_t off_scales1 = off_codes1 + round256(static_cast<size_t>(P) * (n / 2));
    const size_t off_qcodes = off_scales1 + round256(static_cast<size_t>(P) * scale_stride);
    const size_t off_qscales = off_qcodes + round256(n / 2);
    const size_t need = off_qscales + round256(scale_stride);
    if (need > static_cast<size_t>(ECHO_STATIC_SCRATCH_BYTES))
        return fail(ECHO_ERR_UNSUPPORTED,
                    "P = %d, n = %zu needs %zu bytes of scratch; the static scratch holds %zu bytes "
                    "(ECHO_STATIC_SCRATCH_BYTES): use echo_create / echo_allreduce for this size",
                    P, n, need, static_cast<size_t>(ECHO_STATIC_SCRATCH_BYTES));
    int device = -1;
    cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess)
        return fail(ECHO_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (!rank_ptrs)
        return fail(ECHO_ERR_INVALID, "rank pointer array is NULL");
    const size_t bytes = n * (dtype == ECHO_BF16 ? 2 : 4);
    int rc;
    for (int r = 0; r < P; r++)
        if ((rc = check_device_pointer(rank_ptrs[r], device, "rank pointer", r)) != ECHO_OK)
            return rc;
    for (int i = 0; i < P; i++)
        for (int j = i + 1; j < P; j++)
            if (!disjoint(rank_ptrs[i], bytes, rank_ptrs[j], bytes))
                return fail(ECHO_ERR_INVALID, "rank buffers %d and %d overlap", i, j);
    if (enable) {
        if ((rc = check_device_pointer(f, device, "state pointer", 0)) != ECHO_OK ||
            (rc = check_device_pointer(s, device, "state pointer", 1)) != ECHO_OK)
            return rc;
        const size_t sb = n * sizeof(float);
        if (!disjoint(f, sb, s, sb))
            return fail(ECHO_ERR_INVALID, "the two state arrays overlap");
        for (int r = 0; r < P; r++)
            if (!disjoint(f, sb, rank_ptrs[r], bytes) || !disjoint(s, sb, rank_ptrs[r], bytes))
                return fail(ECHO_ERR_INVALID, "a state array overlaps rank buffer %d", r);
    }

    // ---- the array's device address on this device (looked up once) ----
    uint8_t *base = nullptr;
    if ((rc = static_base(&base)) != ECHO_OK)
        return rc;

    // ---- the kernels, as echo_allreduce enqueues them with its default
    // path choice: one kernel up to ECHO_FUSED_LIMIT elements per rank (the
    // injected stall, which exercises the bounded waits, always runs three) ----
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int *status = reinterpret_cast<int *>(base);
    uint8_t *codes1 = base + off_codes1, *scales1 = base + off_scales1;
    uint8_t *qcodes = base + off_qcodes, *qscales = base + off_qscales;
    const uint32_t chunks = static_cast<uint32_t>(n / echo::kChunk);
    const bool stall = stall_injected();
    const echo::PipeCtl ctl{status, stall ? kStallWaitCycles : kWaitCycles, stall};

    if (!stall && n <= ECHO_FUSED_LIMIT) {
        echo::KFArgs af{};
        for (int r = 0; r < P; r++) {
            af.x.p[r] = rank_ptrs[r];
            af.out.p[r] = rank_ptrs[r];
        }
        af.f = f;
        af.s = s;
        af.codes = codes1;
        af.scales = scales1;
        af.qcodes = qcodes;
        af.qscales = qscales;
        af.n = n;
        af.scale_stride = scale_stride;
        af.chunk_begin = 0;
        af.chunk_end = chunks;
        af.lanes_log2 = 2; // groups of 32: 4 lanes
        af.groups_per_seg = static_cast<uint32_t>(n / P / ECHO_GROUP);
        af.lambda = lambda;
        af.one_minus_lambda = 1.0f - lambda;
        af.beta_f = beta_fast;
        af.one_minus_beta_f = 1.0f - beta_fast;
        af.beta_s = beta_slow;
        af.one_minus_beta_s = 1.0f - beta_slow;
        af.P = P;
        af.bf16 = dtype == ECHO_BF16;
        af.enable = enable != 0;
        af.ctl = ctl;
        if ((e = echo::launch_kf_fused_allreduce(af, st)) != cudaSuccess)
            return fail(ECHO_ERR_CUDA, "launch kf_fused_allreduce: %s", cudaGetErrorString(e));
        return ECHO_OK;
    }

    echo::K1Args a1{};
    echo::K2Args a2{};
    echo::K3Args a3{};
    for (int r = 0; r < P; r++) {
        a1.x.p[r] = rank_ptrs[r];
        a3.out.p[r] = rank_ptrs[r];
    }
    a1.f = f;
    a1.s = s;
    a1.codes = codes1;
    a1.scales = scales1;
    a1.n = n;
    a1.scale_stride = scale_stride;
    a1.chunk_begin = 0;
    a1.chunk_end = chunks;
    a1.groups_per_seg = static_cast<uint32_t>(n / P / ECHO_GROUP);
    a1.lanes_log2 = a2.lanes_log2 = a3.lanes_log2 = 2; // groups of 32: 4 lanes
    a1.lambda = lambda;
    a1.one_minus_lambda = 1.0f - lambda;
    a1.P = P;
    a1.bf16 = dtype == ECHO_BF16;
    a1.enable = enable != 0;
    a1.ctl = ctl;

    a2.codes = codes1;
    a2.scales = scales1;
    a2.qcodes = qcodes;
    a2.qscales = qscales;
    a2.f = f;
    a2.s = s;
    a2.n = n;
    a2.scale_stride = scale_stride;
    a2.chunk_begin = 0;
    a2.chunk_end = chunks;
    a2.beta_f = beta_fast;
    a2.one_minus_beta_f = 1.0f - beta_fast;
    a2.beta_s = beta_slow;
    a2.one_minus_beta_s = 1.0f - beta_slow;
    a2.P = P;
    a2.enable = enable != 0;
    a2.ctl = ctl;

    a3.qcodes = qcodes;
    a3.qscales = qscales;
    a3.n = n;
    a3.scale_stride = scale_stride;
    a3.chunk_begin = 0;
    a3.chunk_end = chunks;
    a3.P = P;
    a3.bf16 = dtype == ECHO_BF16;
    a3.ctl = ctl;

    const char *what = "launch k1_compensate_quantize_pack";
    e = echo::launch_k1_compensate_quantize_pack(a1, st);
    if (e == cudaSuccess && (e = echo::launch_k2_owner_reduce_requant(a2, st)) != cudaSuccess)
        what = "launch k2_owner_reduce_requant";
    if (e == cudaSuccess && (e = echo::launch_k3_gather_dequant(a3, st)) != cudaSuccess)
        what = "launch k3_gather_dequant";
    if (e != cudaSuccess)
        return fail(ECHO_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return ECHO_OK;
}
