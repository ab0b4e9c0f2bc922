// Top-k selection over score rows.
// Source: "读完这篇，你就搞懂 DeepSeek v4 了", 闪电索引机制: keep the k entries
// with the highest relevance; the hierarchical-indexer pool ("Recall之王",
// Hierarchical Sparse Indexer; V4.1 Flash transcript) is the same selection
// with a larger count.
//
// Exact radix select on an order-preserving 32-bit key of each f32 score:
// three histogram passes (11 + 11 + 10 bits) find the key T of the count-th
// best score and how many scores equal to T must be taken; a final pass walks
// the row in position order and writes every key > T plus the lowest-position
// keys == T, so ties go to the lower position and the output lists positions
// in ascending order.  Integer histograms and ordered scans make the result
// bit-for-bit deterministic and independent of how many rows run together.
//
// Kernel shape: one 1024-thread CTA per row (this file); rows longer than a
// few thousand entries with few rows use the multi-CTA kernel of
// topk_multi.cu when it applies.
#include "common.cuh"
#include "launchers.h"

namespace csa2 {

// multi-CTA selection (topk_multi.cu); CSA2_ERR_UNSUPPORTED when not applicable
size_t select_topk_multi_workspace(int64_t rows, int64_t L, int count);
csa2_status launch_select_topk_multi(const float* scores, int64_t rows, int64_t L, int count,
                                     const int32_t* ids, int32_t* out, void* ws, size_t ws_bytes,
                                     cudaStream_t stream);

namespace {

constexpr int kT = 1024;

// Order-preserving key: larger score -> larger key.  -inf and NaN map to 0,
// which no selectable score has (the smallest valid key is 0x00800000).
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (f != f || u == 0xff800000u) return 0u;
  if (u == 0x80000000u) u = 0u;                    // -0 ranks as +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive prefix sum of one int per thread, in thread order.
__device__ __forceinline__ int block_excl_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int s = warp_sums[lane];
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    warp_sums[lane] = incl - s;        // exclusive prefix of the warp totals
    if (lane == 31) warp_sums[32] = incl;
  }
  __syncthreads();
  const int res = warp_sums[wid] + x - v;
  *total = warp_sums[32];
  __syncthreads();
  return res;
}

__global__ void __launch_bounds__(kT) topk_row_kernel(const float* __restrict__ scores, int64_t L,
                                                      int count, const int32_t* __restrict__ ids,
                                                      int32_t* __restrict__ out) {
  __shared__ int hist[2048];
  __shared__ int warp_sums[33];
  __shared__ int sh_bin, sh_above;
  const int64_t r = blockIdx.x;
  const float* s = scores + r * L;
  int32_t* o = out + r * static_cast<int64_t>(count);
  const int tid = threadIdx.x;

  uint32_t prefix = 0, mask = 0;
  int kk = count;
  bool take_all = false;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass];
    const int bins = 1 << widths[pass];
    for (int i = tid; i < bins; i += kT) hist[i] = 0;
    __syncthreads();
    for (int64_t i = tid; i < L; i += kT) {
      const uint32_t key = score_key(s[i]);
      if (key != 0u && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (bins - 1)], 1);
    }
    __syncthreads();
    // bins owned by this thread: [tid*per, tid*per + per), scanned from the top
    const int per = bins / kT;
    int local = 0;
    for (int u = 0; u < per; ++u) local += hist[tid * per + u];
    // suffix sum over threads = prefix sum in reversed thread order
    int total;
    // reverse: thread tid contributes at position kT-1-tid
    // (computed with a second scan on the mirrored value set)
    __shared__ int mirror[kT];
    mirror[kT - 1 - tid] = local;
    __syncthreads();
    const int mine = mirror[tid];
    const int excl_m = block_excl_scan(mine, warp_sums, &total);
    // excl_m = sum of bins above the bins of thread (kT-1-tid)
    mirror[tid] = excl_m;
    __syncthreads();
    const int above0 = mirror[kT - 1 - tid];   // sum of all bins above this thread's bins
    if (pass == 0 && total <= count) take_all = true;  // fewer selectable than count
    if (!take_all) {
      int above = above0;
      for (int u = per - 1; u >= 0; --u) {
        const int bin = tid * per + u;
        const int h = hist[bin];
        if (above < kk && above + h >= kk) {
          sh_bin = bin;
          sh_above = above;
        }
        above += h;
      }
    }
    __syncthreads();
    if (take_all) break;
    prefix |= static_cast<uint32_t>(sh_bin) << shift;
    mask |= static_cast<uint32_t>(bins - 1) << shift;
    kk -= sh_above;
    __syncthreads();
  }
  // threshold key T and the number of keys equal to T to take (lowest positions first)
  const uint32_t T = take_all ? 0u : prefix;
  const int need_eq = take_all ? 0 : kk;

  int base_sel = 0, base_eq = 0;
  for (int64_t c0 = 0; c0 < L && base_sel < count; c0 += kT) {
    const int64_t i = c0 + tid;
    const uint32_t key = i < L ? score_key(s[i]) : 0u;
    const int gt = key != 0u && key > T;
    const int eq = key != 0u && key == T;
    int tot_eq, tot_sel;
    const int eq_rank = base_eq + block_excl_scan(eq, warp_sums, &tot_eq);
    const int sel = gt || (eq && eq_rank < need_eq);
    const int pos = base_sel + block_excl_scan(sel, warp_sums, &tot_sel);
    if (sel && pos < count) o[pos] = ids ? ids[r * L + i] : static_cast<int32_t>(i);
    base_eq += tot_eq;
    base_sel += tot_sel;
  }
  for (int p = base_sel + tid; p < count; p += kT) o[p] = -1;
}

}  // namespace

size_t select_topk_workspace(int64_t rows, int64_t L, int count) {
  return select_topk_multi_workspace(rows, L, count);
}

csa2_status launch_select_topk(const float* scores, int64_t rows, int64_t L, int count,
                               const int32_t* ids, int32_t* out, void* ws, size_t ws_bytes,
                               cudaStream_t stream) {
  if (rows == 0 || count == 0) return CSA2_OK;
  csa2_status s = launch_select_topk_multi(scores, rows, L, count, ids, out, ws, ws_bytes, stream);
  if (s != CSA2_ERR_UNSUPPORTED) return s;
  if (rows > 0x7fffffff) return fail(CSA2_ERR_UNSUPPORTED, "select_topk: too many rows");
  begin_launch(stream);
  topk_row_kernel<<<static_cast<unsigned>(rows), kT, 0, stream>>>(scores, L, count, ids, out);
  note_launch(LK_TOPK, 1, stream);
  return check_launch("select_topk");
}

}  // namespace csa2
