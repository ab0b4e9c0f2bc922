// Lightning-indexer scores.
// Source: "读完这篇，你就搞懂 DeepSeek v4 了", 闪电索引机制 (eq. 8): every
// query scores every compressed entry; each indexer head's score is weighted
// by the query's per-head weight and summed (DSA form, ReLU per head).
//
// This file holds the CUDA-core kernel: one thread per scored entry, the
// query's heads (f32) and weights in shared memory, the entry's indexer key
// in registers.  It serves every shape; the tensor-core kernel in
// index_scores_tc.cu takes the shapes it supports.
#include "common.cuh"
#include "launchers.h"

namespace csa2 {

// tensor-core path (index_scores_tc.cu); returns CSA2_ERR_UNSUPPORTED when the
// shape is not one it handles
csa2_status launch_index_scores_tc(const void* q, const float* w, const void* k, int B, int Q,
                                   int H, int d, int64_t N, const int32_t* n_visible,
                                   const int32_t* pool, int P, csa2_index_act act, float* scores,
                                   cudaStream_t stream, ClearOnLaunch* clear);

namespace {

constexpr int kThreads = 256;

template <int DD>
__global__ void __launch_bounds__(kThreads) index_scores_simt(
    const uint16_t* __restrict__ q, const float* __restrict__ w, const uint16_t* __restrict__ k,
    int Q, int H, int d_rt, int64_t N, const int32_t* __restrict__ n_visible,
    const int32_t* __restrict__ pool, int P, int relu, float* __restrict__ scores, int* err) {
  const int d = DD > 0 ? DD : d_rt;
  extern __shared__ float smem[];
  float* q_s = smem;              // [H][d]
  float* w_s = smem + H * d;      // [H]
  const int b = blockIdx.z, t = blockIdx.y;
  const int64_t bq = static_cast<int64_t>(b) * Q + t;
  const uint16_t* qg = q + bq * H * d;
  for (int i = threadIdx.x; i < H * d; i += kThreads) q_s[i] = __uint_as_float(uint32_t(qg[i]) << 16);
  for (int i = threadIdx.x; i < H; i += kThreads) w_s[i] = w[bq * H + i];
  __syncthreads();

  const int64_t L = pool ? P : N;
  const int64_t j = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  if (j >= L) return;
  int64_t e;
  bool valid;
  if (pool) {
    e = pool[bq * P + j];
    valid = e >= 0;
    if (e >= N || e < -1) {
      raise_dev_error(err, DEVERR_BOUNDS);
      valid = false;
    }
  } else {
    e = j;
    const int64_t nv = n_visible ? n_visible[bq] : N;
    valid = e < nv;
  }
  float s = -INFINITY;
  if (valid) {
    constexpr int KW = (DD > 0 ? DD : 256) / 2;   // 32-bit words of the key row
    uint32_t kr[KW];
    const uint4* krow = reinterpret_cast<const uint4*>(k + (static_cast<int64_t>(b) * N + e) * d);
#pragma unroll
    for (int i = 0; i < KW / 4; ++i) {
      if (DD > 0 || i < d / 8) {
        const uint4 v = __ldg(krow + i);
        kr[4 * i] = v.x; kr[4 * i + 1] = v.y; kr[4 * i + 2] = v.z; kr[4 * i + 3] = v.w;
      }
    }
    s = 0.0f;
    for (int h = 0; h < H; ++h) {
      const float2* qh = reinterpret_cast<const float2*>(q_s + h * d);
      float dot = 0.0f;
#pragma unroll
      for (int i = 0; i < KW; ++i) {
        if (DD > 0 || i < d / 2) {
          const float2 qq = qh[i];
          dot = fmaf(qq.x, bf16_lo(kr[i]), dot);
          dot = fmaf(qq.y, bf16_hi(kr[i]), dot);
        }
      }
      if (relu) dot = fmaxf(dot, 0.0f);
      s = fmaf(w_s[h], dot, s);
    }
  }
  scores[bq * L + j] = s;
}

template <int DD>
csa2_status run_simt(const void* q, const float* w, const void* k, int B, int Q, int H, int d,
                     int64_t N, const int32_t* n_visible, const int32_t* pool, int P,
                     csa2_index_act act, float* scores, cudaStream_t stream) {
  const int64_t L = pool ? P : N;
  const size_t smem = (static_cast<size_t>(H) * d + H) * sizeof(float);
  auto kern = index_scores_simt<DD>;
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return check_launch("index_scores: shared-memory opt-in");
  }
  dim3 grid(static_cast<unsigned>((L + kThreads - 1) / kThreads), static_cast<unsigned>(Q),
            static_cast<unsigned>(B));
  begin_launch(stream);
  kern<<<grid, kThreads, smem, stream>>>(
      static_cast<const uint16_t*>(q), w, static_cast<const uint16_t*>(k), Q, H, d, N, n_visible,
      pool, P, act == CSA2_ACT_RELU ? 1 : 0, scores, device_error_word());
  note_launch(pool ? LK_INDEX_POOL : LK_INDEX, 1, stream);
  return check_launch("index_scores");
}

}  // namespace

csa2_status launch_index_scores_simt(const void* q, const float* w, const void* k, int B, int Q,
                                     int H, int d, int64_t N, const int32_t* n_visible,
                                     const int32_t* pool, int P, csa2_index_act act,
                                     float* scores, cudaStream_t stream) {
  if (static_cast<int64_t>(H) * d > 16384)
    return fail(CSA2_ERR_UNSUPPORTED, "index_scores: H*d = %d exceeds 16384", H * d);
  if (d == 64)
    return run_simt<64>(q, w, k, B, Q, H, d, N, n_visible, pool, P, act, scores, stream);
  if (d == 128)
    return run_simt<128>(q, w, k, B, Q, H, d, N, n_visible, pool, P, act, scores, stream);
  return run_simt<0>(q, w, k, B, Q, H, d, N, n_visible, pool, P, act, scores, stream);
}

csa2_status launch_index_scores(const void* q, const float* w, const void* k, int B, int Q, int H,
                                int d, int64_t N, const int32_t* n_visible, const int32_t* pool,
                                int P, csa2_index_act act, float* scores, cudaStream_t stream,
                                ClearOnLaunch* clear) {
  const int64_t L = pool ? P : N;
  if (L == 0 || B == 0 || Q == 0) return CSA2_OK;
  csa2_status s = launch_index_scores_tc(q, w, k, B, Q, H, d, N, n_visible, pool, P, act, scores,
                                         stream, clear);
  if (s != CSA2_ERR_UNSUPPORTED) return s;
  return launch_index_scores_simt(q, w, k, B, Q, H, d, N, n_visible, pool, P, act, scores, stream);
}

}  // namespace csa2
