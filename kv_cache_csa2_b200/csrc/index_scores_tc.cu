// Tensor-core (tcgen05) indexer-score kernel.  Not built yet: every shape
// goes to the CUDA-core kernel of index_scores.cu.
#include "common.cuh"

namespace csa2 {
csa2_status launch_index_scores_tc(const void*, const float*, const void*, int, int, int, int,
                                   int64_t, const int32_t*, const int32_t*, int, csa2_index_act,
                                   float*, cudaStream_t) {
  return CSA2_ERR_UNSUPPORTED;
}
}  // namespace csa2
