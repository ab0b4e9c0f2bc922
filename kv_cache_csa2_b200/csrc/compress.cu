// Token -> entry compression.
// Source: "读完这篇，你就搞懂 DeepSeek v4 了", CSA compression (the recorder
// attends to two consecutive meetings) and eq. (11) (weights S = softmax of
// the projected logits Z plus the learned bias B).  Entry j is the per-channel
// softmax-weighted sum of the token values of blocks j-1 and j.
//
// One thread owns 8 channels of one entry: it reads the 2m window rows of z
// (2 x 16 B), bias (2 x 16 B) and c (16 B), takes the window max, then the
// exp-weighted sums, all in f32, and writes 8 bf16 (16 B).  Consecutive
// threads own consecutive channel groups, so every row access of a warp is
// one contiguous 512 B (c) / 1 KiB (z) segment.  Windows of neighbouring
// entries overlap by one block; the repeat read is served by L1/L2.
#include "common.cuh"
#include "launchers.h"

namespace csa2 {
namespace {

__device__ __forceinline__ void load8f(const float* p, float* v) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__global__ void __launch_bounds__(256) compress_kernel(
    const uint16_t* __restrict__ c, const float* __restrict__ z, const float* __restrict__ bias,
    int N, int D, int m, int halo, int64_t t_in, uint16_t* __restrict__ out, int64_t out_bstride) {
  const int groups = D / 8;
  const int64_t gid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int b = blockIdx.y;
  if (gid >= static_cast<int64_t>(N) * groups) return;
  const int j = static_cast<int>(gid / groups);
  const int g = static_cast<int>(gid % groups);
  const int ch0 = g * 8;

  // array row of window position 0; positions before the first row are absent
  const int64_t first = static_cast<int64_t>(j - 1) * m + halo;
  const int w0 = first >= 0 ? 0 : m;
  const int64_t seq = static_cast<int64_t>(b) * t_in * D;

  float mx[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) mx[u] = -INFINITY;
  for (int w = w0; w < 2 * m; ++w) {
    float zz[8], bb[8];
    load8f(z + seq + (first + w) * D + ch0, zz);
    load8f(bias + static_cast<int64_t>(w) * D + ch0, bb);
#pragma unroll
    for (int u = 0; u < 8; ++u) mx[u] = fmaxf(mx[u], zz[u] + bb[u]);
  }
  float den[8], num[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) { den[u] = 0.0f; num[u] = 0.0f; }
  for (int w = w0; w < 2 * m; ++w) {
    float zz[8], bb[8];
    load8f(z + seq + (first + w) * D + ch0, zz);
    load8f(bias + static_cast<int64_t>(w) * D + ch0, bb);
    const uint4 cv = __ldg(reinterpret_cast<const uint4*>(c + seq + (first + w) * D + ch0));
    const float cc[8] = {bf16_lo(cv.x), bf16_hi(cv.x), bf16_lo(cv.y), bf16_hi(cv.y),
                         bf16_lo(cv.z), bf16_hi(cv.z), bf16_lo(cv.w), bf16_hi(cv.w)};
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float p = expf((zz[u] + bb[u]) - mx[u]);
      den[u] += p;
      num[u] = fmaf(p, cc[u], num[u]);
    }
  }
  uint4 o;
  o.x = pack_bf16x2(num[0] / den[0], num[1] / den[1]);
  o.y = pack_bf16x2(num[2] / den[2], num[3] / den[3]);
  o.z = pack_bf16x2(num[4] / den[4], num[5] / den[5]);
  o.w = pack_bf16x2(num[6] / den[6], num[7] / den[7]);
  *reinterpret_cast<uint4*>(out + static_cast<int64_t>(b) * out_bstride +
                            static_cast<int64_t>(j) * D + ch0) = o;
}

// HCA compression ("读完这篇，你就搞懂 DeepSeek v4 了", HCA 压缩机制, eq. 10 and
// 11): entry j is the per-channel softmax-weighted sum of the m tokens of
// block j alone (no overlap with the block before), bias [m, D] indexed by the
// position in the block.  Blocks are long (m up to 1024), so the block's rows
// are split over kHcaSplit lanes of a warp (lane s takes rows s, s + 8, ..),
// each lane runs one pass with a running max (its sums rescaled when the max
// grows), and the lanes' (max, sum, weighted sum) merge by shuffles in a fixed
// order.  A warp covers 4 channel groups (128 bytes of z) of 8 rows at a time.
constexpr int kHcaSplit = 8;

__device__ __forceinline__ void merge_softmax(float& mx, float& den, float& num, float mx2, float den2,
                                              float num2) {
  const float M = fmaxf(mx, mx2);
  const float a = mx == -INFINITY ? 0.0f : expf(mx - M);
  const float b = mx2 == -INFINITY ? 0.0f : expf(mx2 - M);
  den = den * a + den2 * b;
  num = num * a + num2 * b;
  mx = M;
}

__global__ void __launch_bounds__(256) compress_hca_kernel(
    const uint16_t* __restrict__ c, const float* __restrict__ z, const float* __restrict__ bias,
    int N, int D, int m, int64_t t_in, uint16_t* __restrict__ out, int64_t out_bstride) {
  const int groups = D / 8;
  const int64_t tid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int lane = threadIdx.x & 31;
  const int s = lane / 4;                          // this lane's share of the rows: s, s + 8, ...
  // (entry, channel group) of the lane: 4 per warp, consecutive channel groups
  const int64_t gid = (tid / 32) * 4 + (lane & 3);
  const int b = blockIdx.y;
  const bool live = gid < static_cast<int64_t>(N) * groups;
  const int j = live ? static_cast<int>(gid / groups) : 0;
  const int ch0 = live ? static_cast<int>(gid % groups) * 8 : 0;
  const int64_t seq = static_cast<int64_t>(b) * t_in * D;
  const int64_t first = static_cast<int64_t>(j) * m;

  float mx[8], den[8], num[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) { mx[u] = -INFINITY; den[u] = 0.0f; num[u] = 0.0f; }
#pragma unroll 2
  for (int w = s; w < (live ? m : 0); w += kHcaSplit) {
    float zz[8], bb[8];
    load8f(z + seq + (first + w) * D + ch0, zz);
    load8f(bias + static_cast<int64_t>(w) * D + ch0, bb);
    const uint4 cv = __ldg(reinterpret_cast<const uint4*>(c + seq + (first + w) * D + ch0));
    const float cc[8] = {bf16_lo(cv.x), bf16_hi(cv.x), bf16_lo(cv.y), bf16_hi(cv.y),
                         bf16_lo(cv.z), bf16_hi(cv.z), bf16_lo(cv.w), bf16_hi(cv.w)};
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float x = zz[u] + bb[u];
      if (x > mx[u]) {                       // a new max: rescale what is summed so far
        const float s = expf(mx[u] - x);     // 0 while nothing is summed (mx = -inf)
        den[u] *= s;
        num[u] *= s;
        mx[u] = x;
      }
      const float p = x == -INFINITY ? 0.0f : expf(x - mx[u]);
      den[u] += p;
      num[u] = fmaf(p, cc[u], num[u]);
    }
  }
  // the 8 lanes of one (entry, channel group) sit 4 apart: merge them
#pragma unroll
  for (int ofs = 16; ofs >= 4; ofs >>= 1) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float mx2 = __shfl_xor_sync(0xffffffffu, mx[u], ofs);
      const float den2 = __shfl_xor_sync(0xffffffffu, den[u], ofs);
      const float num2 = __shfl_xor_sync(0xffffffffu, num[u], ofs);
      merge_softmax(mx[u], den[u], num[u], mx2, den2, num2);
    }
  }
  if (!live || s != 0) return;
  uint4 o;
  o.x = pack_bf16x2(num[0] / den[0], num[1] / den[1]);
  o.y = pack_bf16x2(num[2] / den[2], num[3] / den[3]);
  o.z = pack_bf16x2(num[4] / den[4], num[5] / den[5]);
  o.w = pack_bf16x2(num[6] / den[6], num[7] / den[7]);
  *reinterpret_cast<uint4*>(out + static_cast<int64_t>(b) * out_bstride +
                            static_cast<int64_t>(j) * D + ch0) = o;
}

}  // namespace

csa2_status launch_compress_hca(const void* c, const float* z, const float* bias, int B, int64_t T,
                                int D, int m, void* out, int64_t out_bstride, cudaStream_t stream) {
  const int64_t N = T / m;
  if (N == 0 || B == 0) return CSA2_OK;
  const int64_t work = N * (D / 8);                  // (entry, channel group) pairs, 4 per warp
  const int64_t lanes = (work + 3) / 4 * 32;
  const int threads = 256;
  dim3 grid(static_cast<unsigned>((lanes + threads - 1) / threads), static_cast<unsigned>(B));
  begin_launch(stream);
  compress_hca_kernel<<<grid, threads, 0, stream>>>(static_cast<const uint16_t*>(c), z, bias,
                                                    static_cast<int>(N), D, m, T,
                                                    static_cast<uint16_t*>(out), out_bstride);
  note_launch(LK_COMPRESS, 1, stream);
  return check_launch("compress_hca");
}

csa2_status launch_compress(const void* c, const float* z, const float* bias, int B, int64_t T,
                            int D, int m, int halo, void* out, int64_t out_bstride,
                            cudaStream_t stream) {
  const int64_t N = T / m;
  if (N == 0 || B == 0) return CSA2_OK;
  const int64_t t_in = T + (halo ? m : 0);
  const int64_t work = N * (D / 8);
  const int threads = 256;
  dim3 grid(static_cast<unsigned>((work + threads - 1) / threads), static_cast<unsigned>(B));
  begin_launch(stream);
  compress_kernel<<<grid, threads, 0, stream>>>(
      static_cast<const uint16_t*>(c), z, bias, static_cast<int>(N), D, m, halo ? m : 0, t_in,
      static_cast<uint16_t*>(out), out_bstride);
  note_launch(LK_COMPRESS, 1, stream);
  return check_launch("compress");
}

}  // namespace csa2
