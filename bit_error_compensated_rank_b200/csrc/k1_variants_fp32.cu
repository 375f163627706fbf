// k1_variants_fp32.cu - the general build of kernel 1 (group size and scale
// format chosen at run time) for binary32 partials.
#include "k1_compensate_quantize_pack.cuh"

namespace echo {

cudaError_t launch_k1_variant_fp32(const K1Args &a, cudaStream_t st)
{
    return dispatch_variant<false, false>(a, st);
}

} // namespace echo
