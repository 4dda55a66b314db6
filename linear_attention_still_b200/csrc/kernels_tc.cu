// kernels_tc.cu -- tcgen05 / TMEM / TMA kernels for sm_100a (bf16): the hybrid merge and the
// banded saliency.  (Filled in below as they land; until then the generic kernels serve.)
#include "common.cuh"
#include "still_internal.h"

namespace still {

bool tc_merge_supported(const Dims &) { return false; }
cudaError_t launch_merge_tc(const Dims &, const void *, const void *, const void *, const void *, const void *,
                            const void *, const float *, const float *, void *, unsigned *, cudaStream_t) {
    return cudaErrorNotSupported;
}
bool tc_saliency_supported(const Dims &) { return false; }
cudaError_t launch_saliency_tc(const Dims &, const void *, const void *, float *, float *, unsigned *, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace still
