// Host side of TMA: encoding tensor maps through the driver entry point
// (resolved once through the runtime, so the library needs no -lcuda).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace csa2 {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

csa2_status make_tensor_map_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows,
                                    uint64_t cols, uint64_t row_pitch_bytes, uint32_t box_cols,
                                    uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(CSA2_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  if ((reinterpret_cast<uintptr_t>(base) & 15u) || (row_pitch_bytes & 15u) || box_cols * 2 > 128 ||
      box_rows > 256 || (box_cols * 2) % 16)
    return fail(CSA2_ERR_INVALID, "tensor map: base, pitch or box not valid for a 128-byte swizzle");
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_pitch_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSA2_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return CSA2_OK;
}

}  // namespace csa2
