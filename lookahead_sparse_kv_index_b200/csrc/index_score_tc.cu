// Tensor-core (tcgen05) index scan -- placeholder until the kernel lands:
// every shape falls through to the CUDA-core path.
#include "lsa_internal.cuh"

namespace lsa {

lsa_status launch_index_score_tc(const void *, const float *, const void *, lsa_dtype, const float *,
                                 const int64_t *, int64_t, int32_t, int32_t, int32_t, float *, float *,
                                 cudaStream_t, bool *handled) {
    *handled = false;
    return LSA_OK;
}

}  // namespace lsa
