// echo_kernels.h - launchers of the three kernels of the Echo all-reduce.
//
// Work is split in chunks of 8 consecutive elements (one 32-bit code word);
// a warp covers 32 chunks = 256 elements = 8 groups per step. A launch covers
// chunks [chunk_begin, chunk_end) of the n elements (the whole tensor, or one
// slice of it when host transfers are pipelined); both bounds are multiples
// of 4, so no group is split.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "echo_codec.cuh"

namespace echo {

struct K1Args {
    RankPtrs x;             // P rank partials (bf16 or binary32), n elements each
    const float *f;         // phase state, fast estimate [n]
    const float *s;         // phase state, slow estimate [n]
    uint8_t *codes;         // stage-1 wire codes [P][n/2]
    uint8_t *scales;        // stage-1 wire scale bytes [P][n/32]
    size_t n;
    uint32_t chunk_begin, chunk_end;
    uint32_t groups_per_seg; // n / P / 32: owner of group g is g / groups_per_seg
    float lambda, one_minus_lambda;
    int P;
    bool bf16;
    bool enable;
};

struct K2Args {
    const uint8_t *codes;   // stage-1 wire [P][n/2]
    const uint8_t *scales;  // [P][n/32]
    uint8_t *qcodes;        // requantised total [n/2]
    uint8_t *qscales;       // [n/32]
    float *f, *s;           // phase state, updated in place
    size_t n;
    uint32_t chunk_begin, chunk_end;
    float beta_f, one_minus_beta_f, beta_s, one_minus_beta_s;
    int P;
    bool enable;
};

struct K3Args {
    const uint8_t *qcodes;
    const uint8_t *qscales;
    RankOutPtrs out;        // P rank outputs (bf16 or binary32)
    size_t n;
    uint32_t chunk_begin, chunk_end;
    int P;
    bool bf16;
};

// Each returns the launch's cudaError_t (cudaSuccess when enqueued).
// max_ctas caps the grid (0: one full wave of resident CTAs).
cudaError_t launch_k1_compensate_quantize_pack(const K1Args &a, cudaStream_t st, int max_ctas);
cudaError_t launch_k2_owner_reduce_requant(const K2Args &a, cudaStream_t st, int max_ctas);
cudaError_t launch_k3_gather_dequant(const K3Args &a, cudaStream_t st, int max_ctas);

// Number of CTAs for a launch of `warp_tiles` warp steps of a kernel with
// `resident` CTAs per SM (256 threads each).
int grid_for(uint32_t warp_tiles, int resident_per_sm, int max_ctas);

} // namespace echo
