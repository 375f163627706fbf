// k1_compensate_quantize_pack.cu - kernel 1 of the Echo all-reduce: the
// default build (groups of 32, power-of-two scales) and the entry point. The
// kernel body, its pipeline and its byte counts are described in
// k1_compensate_quantize_pack.cuh.
#include "k1_compensate_quantize_pack.cuh"

namespace echo {

cudaError_t launch_k1_compensate_quantize_pack(const K1Args &a, cudaStream_t st)
{
    if (a.chunk_end <= a.chunk_begin)
        return cudaSuccess;
    if (a.P < 1 || a.P > kMaxRanks)
        return cudaErrorInvalidValue;
    if (a.lanes_log2 != 2u || a.fp16_scale) { // a group-size or scale-format variant
        if (a.bf16)
            return a.sender_ef ? launch_k1_variant_bf16_ef(a, st) : launch_k1_variant_bf16(a, st);
        return a.sender_ef ? launch_k1_variant_fp32_ef(a, st) : launch_k1_variant_fp32(a, st);
    }
    if (a.bf16)
        return a.sender_ef ? dispatch_ranks<true, true, kDefaultBuild>(a, st)
                         : dispatch_ranks<true, false, kDefaultBuild>(a, st);
    return a.sender_ef ? dispatch_ranks<false, true, kDefaultBuild>(a, st)
                     : dispatch_ranks<false, false, kDefaultBuild>(a, st);
}

} // namespace echo
