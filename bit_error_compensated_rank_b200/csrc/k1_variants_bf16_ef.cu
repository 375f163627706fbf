// k1_variants_bf16_ef.cu - the general build of kernel 1 (group size and scale
// format chosen at run time) for bf16 partials, with sender feedback.
#include "k1_compensate_quantize_pack.cuh"

namespace echo {

cudaError_t launch_k1_variant_bf16_ef(const K1Args &a, cudaStream_t st)
{
    return dispatch_variant<true, true>(a, st);
}

} // namespace echo
