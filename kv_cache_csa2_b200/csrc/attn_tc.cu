// Tensor-core (tcgen05) sparse-attention kernel.  Not built yet: every shape
// goes to the CUDA-core kernel of attn.cu.
#include "common.cuh"

namespace csa2 {
size_t sparse_attn_tc_workspace(int, int, int, int, int, csa2_kv_fmt) { return 0; }
csa2_status launch_sparse_attn_tc(const void*, const csa2_kv&, const int32_t*, int, int, int, int,
                                  float, void*, float*, void*, size_t, cudaStream_t) {
  return CSA2_ERR_UNSUPPORTED;
}
}  // namespace csa2
