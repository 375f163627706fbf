// k1_variants_bf16.cu - the general build of kernel 1 (group size and scale
// format chosen at run time) for bf16 partials.
#include "k1_compensate_quantize_pack.cuh"

namespace echo {

cudaError_t launch_k1_variant_bf16(const K1Args &a, cudaStream_t st)
{
    return dispatch_variant<true, false>(a, st);
}

} // namespace echo
