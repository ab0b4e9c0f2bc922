// Shared-KV sparse attention on the 5th-generation tensor cores (tcgen05),
// one thread-block cluster per query.
// Source: "读完这篇，你就搞懂 DeepSeek v4 了", 注意力计算 (eq. 9): standard
// softmax attention in which all query heads share the selected compressed
// entries as keys and values; 批无关性 (batch invariance): the per-query
// reduction order is fixed.
//
// Shapes: 64 heads, entries of width 512, bf16.  A query's k selected rows
// are split over the CS CTAs of its cluster, T tiles of 128 rows per CTA.
// Per CTA:
//   warp 0     gathers a tile's 128 rows (1 KiB each) with cp.async into a
//              128-byte-swizzled tile (zero rows for empty slots); the
//              query's 64 x 512 heads arrive by TMA;
//   warp 1     allocates TMEM and issues the MMAs:
//                S^T[row, head] = KV[row, :] . q[head, :]    (M=128, N=64, K=512)
//                O^T[dim, head] += KV[row, dim] * P[row, head] (M=128 dims x4, N=64, K=128)
//              both operands of the second product read the same tiles
//              through MN-major descriptors (no transposes);
//   warps 2-5  softmax and reduction.  Pass A: per-head max of
//              scale * S over the CTA's rows, pushed to every CTA of the
//              cluster through distributed shared memory; after a cluster
//              barrier every CTA knows the query's global per-head max M, so
//              P = exp(scale*S - M) needs no later rescaling.  Pass B: P in
//              bf16 into shared memory for the PV product, row sums l in f32.
//              Then each CTA sends its f32 partial O^T slice for dims owned by
//              CTA r (512/CS dims each) and its l to CTA r; every owner adds
//              the CS partials in rank order, divides by L = sum of l and
//              writes its dims of out (bf16) -- rank 0 also writes lse.
// Tiles of one CTA that no longer fit in shared memory are gathered again for
// the PV product (their rows are then in L2).  Four cluster barriers; every
// other wait is bounded (2 s) and a CTA that gives up still takes part in
// every cluster barrier, so a cluster never waits for a CTA that left.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "launchers.h"
#include "sm100.cuh"

namespace csa2 {
namespace {
using namespace sm100;

constexpr int HA = 64;
constexpr int DV = 512;
constexpr int kRows = 128;                    // rows per tile (MMA M of S^T)
constexpr int kThreads = 6 * 32;
constexpr int kKB = DV / 64;                  // 8 K-blocks of 64 dims
constexpr int kKBBytes = kRows * 128;         // 16 KiB
constexpr int kMaxCS = 16;
constexpr int kRecvStride = HA + 4;           // floats per received (src, dim) row: 272 B

constexpr int OFF_KV = 0;                              // 128 KiB: KV tile
constexpr int OFF_P = OFF_KV + kKB * kKBBytes;         // 16 KiB: P tile
constexpr int OFF_Q = OFF_P + kRows * 128;             // 64 KiB: q (8 K-blocks x 64 rows)
constexpr int OFF_MAX = OFF_Q + kKB * HA * 128;        // [kMaxCS][HA] f32, written by peers
constexpr int OFF_L = OFF_MAX + kMaxCS * HA * 4;       // [kMaxCS][HA] f32, written by peers
constexpr int OFF_RED = OFF_L + kMaxCS * HA * 4;       // [4 warps][HA] f32
constexpr int OFF_M = OFF_RED + 4 * HA * 4;            // [HA] f32 global max, [HA] f32 L
constexpr int OFF_BAR = OFF_M + 2 * HA * 4;
constexpr int NBAR = 16;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
static_assert(DV * kRecvStride * 4 <= OFF_Q, "partials received into the KV + P region");
static_assert(SMEM_BYTES <= 232448, "shared memory");

struct Params {
  const uint16_t* kv;      // [B, n, 512]
  const int32_t* topk;     // [B*Q, k]
  uint16_t* out;           // [B*Q, 64, 512]
  float* lse;              // [B*Q, 64] or null
  int* err;
  int64_t n;
  int Q, k, cs;
  float scale;
};

// Reduce 64 per-thread values over the 32 lanes of a warp (max or sum): five
// exchange steps, each halving the values a lane keeps; on return v[0], v[1]
// hold heads base, base+1 with base = the lane's bit pattern (as below).
template <bool MAX>
__device__ __forceinline__ void warp_transpose_reduce(float (&v)[64], int lane) {
#pragma unroll
  for (int step = 0; step < 5; ++step) {
    const int half = 32 >> step;           // values kept after this step
    const int ofs = 16 >> step;            // partner lane distance
    const bool upper = lane & ofs;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float keep = upper ? v[i + half] : v[i];
      const float give = upper ? v[i] : v[i + half];
      const float got = __shfl_xor_sync(0xffffffffu, give, ofs);
      v[i] = MAX ? fmaxf(keep, got) : keep + got;
    }
  }
}
__device__ __forceinline__ int reduced_head_base(int lane) {
  return ((lane >> 4) & 1) * 32 + ((lane >> 3) & 1) * 16 + ((lane >> 2) & 1) * 8 +
         ((lane >> 1) & 1) * 4 + (lane & 1) * 2;
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int T>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKV = smem + OFF_KV;
  uint8_t* sP = smem + OFF_P;
  uint8_t* sQ = smem + OFF_Q;
  float* sMax = reinterpret_cast<float*>(smem + OFF_MAX);
  float* sL = reinterpret_cast<float*>(smem + OFF_L);
  float* sRed = reinterpret_cast<float*>(smem + OFF_RED);
  float* sM = reinterpret_cast<float*>(smem + OFF_M);
  float* sLt = sM + HA;
  float* sRecv = reinterpret_cast<float*>(smem + OFF_KV);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bar + 0;
  uint64_t* kv_full = bar + 1;
  uint64_t* kv_free = bar + 2;
  uint64_t* p_full = bar + 3;
  uint64_t* p_free = bar + 4;
  uint64_t* o_full = bar + 5;
  uint64_t* s_full = bar + 6;                  // [T]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cs = p.cs;
  const uint32_t me = cluster_rank();
  const int64_t qi = blockIdx.x / cs;                 // flat (b, q)
  const int64_t b = qi / p.Q;
  const uint16_t* kv_b = p.kv + b * p.n * DV;
  const int32_t* ids = p.topk + qi * p.k;
  constexpr uint32_t S_COL = 0;                       // S_j at columns [64 j, 64 j + 64)
  constexpr uint32_t O_COL = 256;                     // O^T chunk mc at [256 + 64 mc, ...)

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(kv_full, 32);
    mbar_init(kv_free, 1);
    mbar_init(p_full, 4);
    mbar_init(p_free, 1);
    mbar_init(o_full, 1);
    for (int j = 0; j < T; ++j) mbar_init(&s_full[j], 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensor_map(&qmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  cluster_sync_all();          // barrier 0: every CTA of the cluster is running before peers write to it

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, HA * DV * 2);
#pragma unroll
      for (int kb = 0; kb < kKB; ++kb)
        tma_load_2d(sQ + kb * HA * 128, &qmap, q_full, kb * 64, static_cast<int32_t>(qi * HA));
    }
    // load order: tiles 0..T-1 (pass A), then T-2..0 again (pass B)
    bool ok = true;
    for (int li = 0; li < 2 * T - 1; ++li) {
      const int j = li < T ? li : 2 * T - 2 - li;
      if (li == T) {                                   // barrier 1 sits between the passes
        __syncwarp();
        cluster_sync_all();
      }
      if (!ok) continue;
      if (li >= 1 && !mbar_wait(kv_free, (li - 1) & 1, abort_flag, p.err)) { ok = false; continue; }
      const int64_t base = (static_cast<int64_t>(me) * T + j) * kRows;
      for (int i = lane; i < kRows * 64; i += 32) {
        const int r = i >> 6, cc = i & 63;
        const int64_t pos = base + r;
        int64_t id = pos < p.k ? ids[pos] : -1;
        if (id >= p.n || id < -1) {
          if (cc == 0) raise_dev_error(p.err, DEVERR_BOUNDS);
          id = -1;
        }
        const uint16_t* src = kv_b + (id >= 0 ? id : 0) * DV + cc * 8;
        cp_async_16(sKV + (cc >> 3) * kKBBytes + sw128_offset(r, cc & 7), src, id >= 0 ? 16u : 0u);
      }
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(kv_full);
    }
    __syncwarp();
    if (T == 1) cluster_sync_all();                    // barrier 1 (no pass-B loads)
    cluster_sync_all();                                // barrier 2
    cluster_sync_all();                                // barrier 3
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = true;
    if (lane == 0) ok = mbar_wait(q_full, 0, abort_flag, p.err);
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, HA, false, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, HA, true, true);
    const uint32_t kv0 = smem_u32(sKV), q0 = smem_u32(sQ), p0 = smem_u32(sP);
    for (int j = 0; j < T; ++j) {                      // pass A
      if (lane == 0 && ok) {
        ok = mbar_wait(kv_full, j & 1, abort_flag, p.err);
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int kb = 0; kb < kKB; ++kb)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16(tmem + S_COL + 64 * j, desc_kmajor_sw128(kv0 + kb * kKBBytes + kk * 32),
                       desc_kmajor_sw128(q0 + kb * HA * 128 + kk * 32), idesc_s, (kb | kk) != 0);
          mma_commit(&s_full[j]);
          if (j < T - 1) mma_commit(kv_free);
        }
      }
      __syncwarp();
    }
    cluster_sync_all();                                // barrier 1
    for (int jj = 0; jj < T; ++jj) {                   // pass B: tiles T-1 .. 0
      if (lane == 0 && ok) {
        if (jj >= 1) ok = mbar_wait(kv_full, (T - 1 + jj) & 1, abort_flag, p.err);
        if (ok) ok = mbar_wait(p_full, jj & 1, abort_flag, p.err);
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int mc = 0; mc < 4; ++mc)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_bf16(tmem + O_COL + 64 * mc,
                       desc_mnmajor_sw128(kv0 + 2 * mc * kKBBytes + kk * 2048, kKBBytes, 1024),
                       desc_mnmajor_sw128(p0 + kk * 2048, 8192, 1024), idesc_o, (jj | kk) != 0);
          mma_commit(p_free);
          mma_commit(kv_free);
        }
      }
      __syncwarp();
    }
    if (lane == 0 && ok) mma_commit(o_full);
    __syncwarp();
    cluster_sync_all();                                // barrier 2
    cluster_sync_all();                                // barrier 3
  } else {
    // ------------------------------------------------------------ softmax + reduction
    const int quad = warp & 3;
    const int ew = warp - 2;                           // epilogue warp 0..3
    const int row = quad * 32 + lane;                  // TMEM lane = tile row
    const int et = ew * 32 + lane;                     // epilogue thread 0..127
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    bool ok = true;
    float mx[HA];
#pragma unroll
    for (int h = 0; h < HA; ++h) mx[h] = -INFINITY;
    bool valid[T];
    for (int j = 0; j < T; ++j) {                      // pass A: per-head max
      const int64_t pos = (static_cast<int64_t>(me) * T + j) * kRows + row;
      const int64_t id = pos < p.k ? ids[pos] : -1;
      valid[j] = id >= 0 && id < p.n;
      if (!ok || !mbar_wait(&s_full[j], 0, abort_flag, p.err)) { ok = false; continue; }
      tc_fence_after();
      uint32_t v[32];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        tmem_ld32(tmem + lane_off + S_COL + 64 * j + 32 * half, v);
        tmem_wait_ld();
        if (valid[j]) {
#pragma unroll
          for (int h = 0; h < 32; ++h) mx[32 * half + h] = fmaxf(mx[32 * half + h], p.scale * __uint_as_float(v[h]));
        }
      }
    }
    warp_transpose_reduce<true>(mx, lane);
    const int hb = reduced_head_base(lane);
    sRed[ew * HA + hb] = mx[0];
    sRed[ew * HA + hb + 1] = mx[1];
    epi_bar();
    for (int i = et; i < cs * HA; i += 128) {          // push the CTA max to every CTA
      const int h = i % HA, dst = i / HA;
      const float m = fmaxf(fmaxf(sRed[h], sRed[HA + h]), fmaxf(sRed[2 * HA + h], sRed[3 * HA + h]));
      st_cluster_f32(map_to_rank(smem_u32(&sMax[me * HA + h]), dst), m);
    }
    __syncwarp();
    cluster_sync_all();                                // barrier 1
    if (et < HA) {
      float m = -INFINITY;
      for (int c = 0; c < cs; ++c) m = fmaxf(m, sMax[c * HA + et]);
      sM[et] = m;
    }
    epi_bar();
    float lsum[HA];
#pragma unroll
    for (int h = 0; h < HA; ++h) lsum[h] = 0.0f;
    for (int jj = 0; jj < T; ++jj) {                   // pass B: P = exp(scale*S - M)
      const int j = T - 1 - jj;
      if (!ok) continue;
      if (jj >= 1 && !mbar_wait(p_free, (jj - 1) & 1, abort_flag, p.err)) { ok = false; continue; }
      tc_fence_after();
      uint32_t v[32];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        tmem_ld32(tmem + lane_off + S_COL + 64 * j + 32 * half, v);
        tmem_wait_ld();
        uint32_t packed[16];
#pragma unroll
        for (int h2 = 0; h2 < 16; ++h2) {
          float e[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int h = 32 * half + 2 * h2 + u;
            const float m = sM[h];
            const float x = p.scale * __uint_as_float(v[2 * h2 + u]);
            e[u] = (valid[j] && m != -INFINITY) ? __expf(x - m) : 0.0f;
          }
          packed[h2] = pack_bf16x2(e[0], e[1]);
          lsum[32 * half + 2 * h2] += bf16_lo(packed[h2]);
          lsum[32 * half + 2 * h2 + 1] += bf16_hi(packed[h2]);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(sP + sw128_offset(row, 4 * half + c)) =
              make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
      }
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    warp_transpose_reduce<false>(lsum, lane);
    epi_bar();
    sRed[ew * HA + hb] = lsum[0];
    sRed[ew * HA + hb + 1] = lsum[1];
    epi_bar();
    for (int i = et; i < cs * HA; i += 128) {          // push the CTA row sums to every owner
      const int h = i % HA, dst = i / HA;
      const float l = (sRed[h] + sRed[HA + h]) + (sRed[2 * HA + h] + sRed[3 * HA + h]);
      st_cluster_f32(map_to_rank(smem_u32(&sL[me * HA + h]), dst), l);
    }
    if (ok) ok = mbar_wait(o_full, 0, abort_flag, p.err);
    __syncwarp();
    cluster_sync_all();                                // barrier 2: every CTA's KV/P region is free
    const int dpo = DV / cs;                           // dims per owner
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int mc = 0; mc < 4; ++mc) {
        const int dim = mc * 128 + row;
        const int owner = dim / dpo, dl = dim % dpo;
        const uint32_t dst = map_to_rank(
            smem_u32(sRecv + (static_cast<int64_t>(me) * dpo + dl) * kRecvStride), owner);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + O_COL + 64 * mc + 32 * half, v);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_cluster_v4(dst + (32 * half + 4 * c) * 4, __uint_as_float(v[4 * c]),
                          __uint_as_float(v[4 * c + 1]), __uint_as_float(v[4 * c + 2]),
                          __uint_as_float(v[4 * c + 3]));
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    cluster_sync_all();                                // barrier 3: partials delivered
    if (et < HA) {
      float L = 0.0f;
      for (int c = 0; c < cs; ++c) L += sL[c * HA + et];
      sLt[et] = L;
      if (me == 0 && p.lse) p.lse[qi * HA + et] = L > 0.0f ? sM[et] + logf(L) : -INFINITY;
    }
    epi_bar();
    uint16_t* out_q = p.out + qi * HA * DV;
    for (int i = et; i < dpo * (HA / 4); i += 128) {
      const int dl = i % dpo, h4 = i / dpo;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int c = 0; c < cs; ++c) {
        const float4 x = *reinterpret_cast<const float4*>(sRecv + (static_cast<int64_t>(c) * dpo + dl) * kRecvStride + 4 * h4);
        acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
      }
      const int dim = static_cast<int>(me) * dpo + dl;
      const float a[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int h = 4 * h4 + u;
        const float L = sLt[h];
        const __nv_bfloat16 o = __float2bfloat16_rn(L > 0.0f ? a[u] / L : 0.0f);
        out_q[h * DV + dim] = *reinterpret_cast<const uint16_t*>(&o);
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  if (threadIdx.x == 32) {
    // the query tile's TMA may still be landing if the MMA warp gave up early
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(q_full, 0) && globaltimer_ns() - t0 < 100000000ull) {
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

int max_cluster_size() {
  static std::once_flag once;
  static int best = 8;
  std::call_once(once, [] {
    auto kern = attn_tc_kernel<1>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
      cudaGetLastError();
      return;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(16 * 64);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 16;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n >= 4) best = 16;
    cudaGetLastError();
  });
  return best;
}

template <int T>
csa2_status run_attn(const CUtensorMap& qmap, const Params& p, int64_t n_queries, cudaStream_t stream) {
  auto kern = attn_tc_kernel<T>;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [&] {
    attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (attr == cudaSuccess)
      attr = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  });
  if (attr != cudaSuccess) return fail(CSA2_ERR_CUDA, "sparse_attn_tc: function attributes");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(n_queries * p.cs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = p.cs;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  begin_launch(stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, qmap, p);
  note_launch(LK_ATTN, 1, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(CSA2_ERR_CUDA, "sparse_attn_tc: launch failed: %s", cudaGetErrorString(e));
  }
  return check_launch("sparse_attn_tc");
}

}  // namespace

size_t sparse_attn_tc_workspace(int, int, int, int, int, csa2_kv_fmt) { return 0; }

csa2_status launch_sparse_attn_tc(const void* q, const csa2_kv& kv, const int32_t* topk, int B,
                                  int Q, int Ha, int k, float scale, void* out, float* lse,
                                  void*, size_t, cudaStream_t stream) {
  if (getenv("CSA2_ATTN_SIMT")) return CSA2_ERR_UNSUPPORTED;      // force the CUDA-core kernel
  if (kv.fmt != CSA2_KV_BF16 || kv.dim != DV || Ha != HA || k <= 0) return CSA2_ERR_UNSUPPORTED;
  const int64_t n_queries = static_cast<int64_t>(B) * Q;
  if (n_queries * HA > 0x7fffffffLL) return CSA2_ERR_UNSUPPORTED;
  const int tiles = (k + kRows - 1) / kRows;
  int max_cs = max_cluster_size();
  if (const char* e = getenv("CSA2_ATTN_MAX_CLUSTER")) {   // tests: smaller clusters
    const int v = atoi(e);
    if (v == 1 || v == 2 || v == 4 || v == 8 || v == 16) max_cs = std::min(max_cs, v);
  }
  int cs = 1;
  while (cs < tiles && cs < max_cs) cs *= 2;
  const int T = (tiles + cs - 1) / cs;
  if (T > 3) return CSA2_ERR_UNSUPPORTED;
  CUtensorMap qmap;
  memset(&qmap, 0, sizeof(qmap));
  CSA2_TRY(make_tensor_map_bf16_2d(&qmap, q, static_cast<uint64_t>(n_queries) * HA, DV, DV * 2, 64, HA));
  Params p;
  p.kv = static_cast<const uint16_t*>(kv.data);
  p.topk = topk;
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.err = device_error_word();
  p.n = kv.n;
  p.Q = Q;
  p.k = k;
  p.cs = cs;
  p.scale = scale;
  if (T == 1) return run_attn<1>(qmap, p, n_queries, stream);
  if (T == 2) return run_attn<2>(qmap, p, n_queries, stream);
  return run_attn<3>(qmap, p, n_queries, stream);
}

}  // namespace csa2
