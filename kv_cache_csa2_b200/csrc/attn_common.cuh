// Arithmetic shared by the two tensor-core attention kernels (attn_tc.cu:
// a query's tiles on several CTAs; attn_seq.cu: a query's tiles in sequence
// on one CTA).  Source: "读完这篇，你就搞懂 DeepSeek v4 了", 注意力计算 (eq. 9)
// and 批无关性 (batch invariance).
//
// A query's rows are cut into tiles of 128 rows.  For tile t both kernels
// compute, with the same instructions in the same order:
//   S_t  = KV_t q^T on the tensor cores (f32), x = scale * S_t (masked rows -inf)
//   m_t  = per-head max of x over the tile's rows
//   P_t  = bf16(exp(x - m_t)),  l_t = per-head sum of P_t (one fixed tree)
//   O_t  = P_t^T KV_t on the tensor cores (f32)
// and then combine the tiles in tile order with a running max:
//   M_t = max(M_{t-1}, m_t),  a_t = exp(M_{t-1} - M_t),  b_t = exp(m_t - M_t)
//   L_t = L_{t-1} a_t + l_t b_t,  acc_t = acc_{t-1} a_t + O_t b_t
//   out = acc_T / L_T (bf16),  lse = M_T + log L_T.
// Every step is written with explicit round-to-nearest intrinsics, so the
// compiler cannot fuse a multiply into a neighbouring add differently in the
// two kernels: a query's result is the same bits whichever kernel runs it,
// and whatever else is in the batch.
#pragma once

#include <cstdint>

#include "common.cuh"

namespace csa2 {
namespace attn {

constexpr int HA = 64;                        // heads
constexpr int DV = 512;                       // entry width
constexpr int kRows = 128;                    // rows per tile (MMA M of S^T)
constexpr int kKB = DV / 64;                  // 8 K-blocks of 64 dims
constexpr int kKBBytes = kRows * 128;         // 16 KiB: one K-block of a tile
constexpr int kMaxTiles = 64;                 // k <= 8192

// Row of its source that row r of tile `tile` of query qi reads, or -1 for
// an empty slot: a selected entry (tile < T_sel: the selection list, or the
// slot itself when dense), or a window row (tile == T_sel).  An index
// outside its source is recorded and treated as empty.  P is either
// kernel's parameter block (the same field names).
template <class P>
__device__ __forceinline__ int tile_row(const P& p, int64_t qi, int tile, int r) {
  if (tile < p.T_sel) {
    const int64_t pos = static_cast<int64_t>(tile) * kRows + r;
    if (pos >= p.k) return -1;
    if (!p.topk) {
      const int64_t vis = p.n_vis ? p.n_vis[qi] : p.k;
      return pos < vis ? static_cast<int>(pos) : -1;
    }
    const int id = p.topk[qi * p.k + pos];
    if (id >= p.n || id < -1) {
      raise_dev_error(p.err, DEVERR_BOUNDS);
      return -1;
    }
    return id;
  }
  const int e = p.win_end[qi];
  if (e < 0 || e > p.win_rows) {
    raise_dev_error(p.err, DEVERR_BOUNDS);
    return -1;
  }
  const int row = e - p.W + r;
  return (r < p.W && row >= 0) ? row : -1;
}

// x of one score: scale * s, or -inf for an empty row
__device__ __forceinline__ float scaled_score(bool valid, float scale, uint32_t s_bits) {
  return valid ? __fmul_rn(scale, __uint_as_float(s_bits)) : -INFINITY;
}

// exp(x - m) (0 for an empty row); rounded to bf16 by the caller
__device__ __forceinline__ float p_value(float x, float m) {
  return x == -INFINITY ? 0.0f : __expf(__fsub_rn(x, m));
}

// Max of one float over the 32 lanes of a warp (every lane gets it).
__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// Sums (or maxes) N per-lane values over the 32 lanes of a warp: five
// exchange steps (partner lanes 16, 8, 4, 2, 1 apart), each halving the
// values a lane keeps.  On return v[0 .. N/32) hold values
// (N/32) * lane + i.  For a given value the additions form the same tree
// (pairs by lane bit 4, then 3, 2, 1, 0) whatever N is, so N = 64 and N = 32
// give the same bits.
template <int N, bool MAX>
__device__ __forceinline__ void warp_transpose_reduce(float (&v)[N], int lane) {
  static_assert(N == 32 || N == 64, "values per lane");
#pragma unroll
  for (int step = 0; step < 5; ++step) {
    const int half = (N / 2) >> step;      // values kept after this step
    const int ofs = 16 >> step;            // partner lane distance
    const bool upper = lane & ofs;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float keep = upper ? v[i + half] : v[i];
      const float give = upper ? v[i] : v[i + half];
      const float got = __shfl_xor_sync(0xffffffffu, give, ofs);
      v[i] = MAX ? fmaxf(keep, got) : __fadd_rn(keep, got);
    }
  }
}

// l_t of one head from the four lane quarters' sums, slot j holding quarter
// (j + 2) & 3 (the order both kernels fill them in)
__device__ __forceinline__ float quad_sum(float s0, float s1, float s2, float s3) {
  return __fadd_rn(__fadd_rn(s0, s1), __fadd_rn(s2, s3));
}

// weight of a partial with max m in a sum whose max is M (0 when either is -inf)
__device__ __forceinline__ float rescale(float m, float M) {
  return (m == -INFINITY || M == -INFINITY) ? 0.0f : __expf(__fsub_rn(m, M));
}

// One step of the tile-order combine for one head: updates the running max M
// and sum L with tile j's (m_j, l_j); returns the factors (a, b) that the
// output accumulator takes for this tile.
__device__ __forceinline__ float2 combine_step(float& M, float& L, float mj, float lj) {
  const float Mn = fmaxf(M, mj);
  const float a = rescale(M, Mn), b = rescale(mj, Mn);
  L = __fmaf_rn(lj, b, __fmul_rn(L, a));
  M = Mn;
  return make_float2(a, b);
}

// acc * a + o * b
__device__ __forceinline__ float combine_acc(float acc, float o, float a, float b) {
  return __fmaf_rn(o, b, __fmul_rn(acc, a));
}

// 1 / L, or 0 when nothing was visible
__device__ __forceinline__ float inv_sum(float L) { return L > 0.0f ? __frcp_rn(L) : 0.0f; }

__device__ __forceinline__ float lse_of(float M, float L) {
  return L > 0.0f ? __fadd_rn(M, logf(L)) : -INFINITY;
}

}  // namespace attn
}  // namespace csa2
