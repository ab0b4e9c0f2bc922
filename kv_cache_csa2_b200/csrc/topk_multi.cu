// Multi-CTA top-k selection.  Not built yet: every row goes to the one-CTA
// kernel of topk.cu.
#include "common.cuh"

namespace csa2 {
size_t select_topk_multi_workspace(int64_t, int64_t, int) { return 0; }
csa2_status launch_select_topk_multi(const float*, int64_t, int64_t, int, const int32_t*, int32_t*,
                                     void*, size_t, cudaStream_t) {
  return CSA2_ERR_UNSUPPORTED;
}
}  // namespace csa2
