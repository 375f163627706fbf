// echo_guards.cu - the guard-byte check of the debug build.
//
// In the debug build every device buffer the library allocates carries
// kGuardBytes of kGuardByte before and after it. After each call one block
// per guard region reads the region back; any changed byte sets
// kStatusCanary in the handle's device status word. A write that strays past
// a buffer therefore shows up in echo_device_status instead of silently
// corrupting a neighbour.
#include "echo_bulk.cuh"
#include "echo_kernels.h"

#include <cuda_runtime.h>

namespace echo {
namespace {

__global__ void check_guards(const GuardList g, int *status)
{
    const uint8_t *p = g.region[blockIdx.x];
    bool bad = false;
    for (uint32_t i = threadIdx.x; i < kGuardBytes; i += blockDim.x)
        bad |= p[i] != kGuardByte;
    if (__syncthreads_or(bad) && threadIdx.x == 0)
        atomicOr(status, kStatusCanary);
}

} // namespace

cudaError_t launch_check_guards(const GuardList &g, int *status, cudaStream_t st)
{
    if (g.count <= 0)
        return cudaSuccess;
    check_guards<<<g.count, 128, 0, st>>>(g, status);
    return cudaGetLastError();
}

} // namespace echo
