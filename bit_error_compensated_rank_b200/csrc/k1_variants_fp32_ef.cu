// k1_variants_fp32_ef.cu - the general build of kernel 1 (group size and scale
// format chosen at run time) for binary32 partials, with sender feedback.
#include "k1_compensate_quantize_pack.cuh"

namespace echo {

cudaError_t launch_k1_variant_fp32_ef(const K1Args &a, cudaStream_t st)
{
    return dispatch_variant<false, true>(a, st);
}

} // namespace echo
