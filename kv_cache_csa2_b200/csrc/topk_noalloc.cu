// Top-k selection whose scratch is a device array of this library instead of
// a caller workspace.  A convenience of this library: the pages describe no
// such call.  The selection itself is csa2_select_topk's (same launcher, same
// kernels, same result bit for bit); only the scratch comes from elsewhere.
#include <mutex>

#include "common.cuh"
#include "launchers.h"

namespace csa2 {
namespace {

// One copy per device: a module-scope __device__ array exists in every
// context that loads this library.  Zero-initialised at load; the launcher
// clears the part the kernels need at zero before each use.
static __device__ __align__(256) unsigned char g_select_scratch[CSA2_SELECT_TOPK_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices];

// Device address of g_select_scratch on the current device, looked up once
// per device while that device is current.
csa2_status scratch_address(void** addr) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(CSA2_ERR_CUDA, "csa2_select_topk_noalloc: cudaGetDevice failed: %s", cudaGetErrorString(e));
  }
  if (dev < 0 || dev >= kMaxDevices)
    return fail(CSA2_ERR_UNSUPPORTED, "csa2_select_topk_noalloc: device ordinal %d >= %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* a = nullptr;
    e = cudaGetSymbolAddress(&a, g_select_scratch);
    if (e != cudaSuccess || a == nullptr) {
      cudaGetLastError();
      return fail(CSA2_ERR_CUDA, "csa2_select_topk_noalloc: scratch address on device %d: %s", dev,
                  cudaGetErrorString(e));
    }
    g_scratch_addr[dev] = a;
  }
  *addr = g_scratch_addr[dev];
  return CSA2_OK;
}

}  // namespace
}  // namespace csa2

extern "C" csa2_status csa2_select_topk_noalloc(const float* scores, int64_t rows, int64_t L,
                                                int count, const int32_t* ids, int32_t* out,
                                                csa2_stream stream) {
  using namespace csa2;
  CSA2_TRY(fault_gate());
  if (rows < 0 || L < 0 || count < 0)
    return fail(CSA2_ERR_INVALID, "csa2_select_topk_noalloc: negative size");
  if (L > 0x7fffffffLL) return fail(CSA2_ERR_INVALID, "csa2_select_topk_noalloc: L too large");
  if (rows == 0 || count == 0) return CSA2_OK;
  if (out == nullptr || (L > 0 && scores == nullptr))
    return fail(CSA2_ERR_INVALID, "csa2_select_topk_noalloc: null pointer");
  // the scratch of the kernel that will run (0 for the kernels that keep
  // their state in shared memory), not csa2_select_topk_workspace's bound
  const size_t need = select_topk_scratch_bytes(rows, L, count);
  const size_t cap = CSA2_SELECT_TOPK_NOALLOC_SCRATCH_BYTES;
  if (need > cap)
    return fail(CSA2_ERR_OOM,
                "csa2_select_topk_noalloc: rows=%lld, L=%lld need %zu bytes of scratch, more than the "
                "%zu-byte static scratch; call csa2_select_topk with a workspace instead",
                static_cast<long long>(rows), static_cast<long long>(L), need, cap);
  void* scratch = nullptr;
  if (need > 0) CSA2_TRY(scratch_address(&scratch));
  return launch_select_topk(scores, rows, L, count, ids, out, scratch, need > 0 ? cap : 0,
                            reinterpret_cast<cudaStream_t>(stream));
}
