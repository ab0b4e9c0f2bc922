// Shared-KV sparse attention on the 5th-generation tensor cores (tcgen05).
// Source: "读完这篇，你就搞懂 DeepSeek v4 了", 注意力计算 (eq. 9): standard
// softmax attention in which all query heads share the selected compressed
// entries as keys and values; 批无关性 (batch invariance): the per-query
// reduction order is fixed and does not depend on the batch.
//
// Shapes: 64 heads, entries of width 512, bf16.  A query's k selected rows are
// cut into tiles of 128 rows, one tile per CTA; the tiles of a query are
// spread over NCL thread-block clusters of CS CTAs (CS = 4, or 2 when k
// fits two tiles; NCL = tiles/CS <= 16; both fixed by k alone).  Per CTA:
//   warp 0     loads the query's 64 x 512 heads (TMA) and gathers the tile's
//              128 selected rows with TMA row gathers (4 rows x 128 bytes per
//              instruction, issued by all 32 lanes, one barrier per 64-column
//              block so the first MMAs start early) into a 128-byte-swizzled
//              tile; empty slots gather a real row and are masked out;
//   warp 1     allocates TMEM and issues the MMAs:
//                S^T[row, head] = KV[row, :] . q[head, :]    (M=128, N=64, K=512)
//                O^T[dim, head] += KV[row, dim] * P[row, head] (M=128 dims x4, N=64, K=128)
//              both products read the same tile through K-major and MN-major
//              descriptors (no transposes);
//   warps 2-5  softmax with the tile's own per-head max m (P in bf16 for the
//              PV product, row sums l in f32), then the reductions.
// Cluster reduction: every CTA pushes (m, l) to its peers over distributed
// shared memory and stages its partial O^T in its own shared memory; after a
// cluster barrier the CTA that owns dims [r*512/CS, (r+1)*512/CS) reads that
// slice from every peer and adds them in rank order, each weighted by
// exp(m_c - M) with M the cluster's max.  With one cluster per query the owner
// divides by L and writes out (bf16) and lse.  With several, each owner writes
// its (O, M, L) slice to a global workspace and takes a ticket; the owner that
// arrives last merges the NCL slices in cluster order (same weighting) and
// writes out -- no CTA waits for another cluster.  Three cluster barriers;
// every other wait is bounded (2 s), and a CTA that gives up still takes part
// in every cluster barrier.
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
constexpr int kMinCS = 2;                     // an owner's slice must fit the q region
constexpr int kMaxCS = 8;
constexpr int kDefaultCS = 4;
constexpr int kMaxNCL = 2 * kMaxCS;           // clusters per query: weights live in the (m, l) region
constexpr int kStageStride = HA + 4;          // floats per staged dim row: 272 B

constexpr int OFF_KV = 0;                              // 128 KiB: KV tile
constexpr int OFF_P = OFF_KV + kKB * kKBBytes;         // 16 KiB: P tile
constexpr int OFF_Q = OFF_P + kRows * 128;             // 64 KiB: q (8 K-blocks x 64 rows)
constexpr int OFF_ML = OFF_Q + kKB * HA * 128;         // [kMaxCS][2][HA] f32 (m, l), written by peers
constexpr int OFF_RED = OFF_ML + kMaxCS * 2 * HA * 4;  // [4 warps][HA] f32
constexpr int OFF_W = OFF_RED + 4 * HA * 4;            // [kMaxCS][HA] f32 weights, [HA] M, [HA] L
constexpr int OFF_BAR = OFF_W + (kMaxCS + 2) * HA * 4;
constexpr int NBAR = 16;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
static_assert(DV * kStageStride * 4 <= OFF_Q, "partial O^T staged in the KV + P region");
static_assert(HA * (DV / kMinCS) * 4 <= kKB * HA * 128, "an owner's slice fits the q region");
static_assert(SMEM_BYTES <= 232448, "shared memory");
static_assert(kMaxNCL * HA <= kMaxCS * 2 * HA, "per-cluster weights fit the (m, l) region");

struct Params {
  const int32_t* topk;     // [B*Q, k]
  uint16_t* out;           // [B*Q, 64, 512]
  float* lse;              // [B*Q, 64] or null
  float* part;             // [B*Q][ncl][cs][dpo*64 + 2*64] cross-cluster slices (ncl > 1)
  unsigned* ticket;        // [B*Q][cs], zero before the launch (ncl > 1)
  int* err;
  int64_t n;
  int Q, k, cs, ncl;
  float scale;
};

// Reduce 64 per-thread values over the 32 lanes of a warp (max or sum): five
// exchange steps, each halving the values a lane keeps; on return v[0], v[1]
// hold heads base, base+1 with base = reduced_head_base(lane).
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

// weight of a partial with max m in a sum whose max is M (0 for empty partials)
__device__ __forceinline__ float rescale(float m, float M) {
  return (m == -INFINITY || M == -INFINITY) ? 0.0f : __expf(m - M);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kvmap,
                   const Params p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ unsigned sh_ticket;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKV = smem + OFF_KV;
  uint8_t* sP = smem + OFF_P;
  uint8_t* sQ = smem + OFF_Q;
  float* sML = reinterpret_cast<float*>(smem + OFF_ML);     // [c][0][h] = m_c, [c][1][h] = l_c
  float* sRed = reinterpret_cast<float*>(smem + OFF_RED);
  float* sWt = reinterpret_cast<float*>(smem + OFF_W);      // [c][h] weights exp(m_c - M)
  float* sMcl = sWt + kMaxCS * HA;                          // [h] max M
  float* sLcl = sMcl + HA;                                  // [h] sum L
  float* sStage = reinterpret_cast<float*>(smem + OFF_KV);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bar + 0;
  uint64_t* p_full = bar + 1;
  uint64_t* o_full = bar + 2;
  uint64_t* s_full = bar + 3;
  uint64_t* kv_full = bar + 8;                 // [8]: one per 64-column block of the tile
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cs = p.cs;
  const uint32_t me = cluster_rank();
  const int64_t per_query = static_cast<int64_t>(cs) * p.ncl;
  const int64_t qi = blockIdx.x / per_query;                      // flat (b, q)
  const int cl = static_cast<int>((blockIdx.x % per_query) / cs); // cluster index within the query
  const int tile = cl * cs + static_cast<int>(me);
  const int64_t b = qi / p.Q;
  const int32_t* ids = p.topk + qi * p.k;
  constexpr uint32_t S_COL = 0;                       // S at columns [0, 64)
  constexpr uint32_t O_COL = 256;                     // O^T chunk mc at [256 + 64 mc, ...)

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(p_full, 4);
    mbar_init(o_full, 1);
    mbar_init(s_full, 1);
    for (int kb = 0; kb < kKB; ++kb) mbar_init(&kv_full[kb], 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensor_map(&qmap);
    prefetch_tensor_map(&kvmap);
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
    // lane g gathers rows 4g .. 4g+3 of the tile, one 64-column block at a time
    const int32_t seq_row0 = static_cast<int32_t>(b * p.n);
    const int64_t pos0 = static_cast<int64_t>(tile) * kRows + 4 * lane;
    int32_t row[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      int id = pos0 + u < p.k ? ids[pos0 + u] : -1;
      if (id >= p.n || id < -1) {
        raise_dev_error(p.err, DEVERR_BOUNDS);
        id = -1;
      }
      row[u] = seq_row0 + (id >= 0 ? id : 0);          // empty slot: masked later
    }
#pragma unroll
    for (int kb = 0; kb < kKB; ++kb) {
      if (lane == 0) mbar_arrive_expect_tx(&kv_full[kb], kRows * 128);
      __syncwarp();
      tma_gather4(sKV + kb * kKBBytes + 4 * lane * 128, &kvmap, &kv_full[kb], kb * 64, row[0], row[1],
                  row[2], row[3]);
    }
    __syncwarp();
    cluster_sync_all();                                // barrier 1
    cluster_sync_all();                                // barrier 2
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, HA, false, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, HA, true, true);
    const uint32_t kv0 = smem_u32(sKV), q0 = smem_u32(sQ), p0 = smem_u32(sP);
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, abort_flag, p.err);
#pragma unroll 1
      for (int kb = 0; kb < kKB && ok; ++kb) {
        ok = mbar_wait(&kv_full[kb], 0, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + S_COL, desc_kmajor_sw128(kv0 + kb * kKBBytes + kk * 32),
                   desc_kmajor_sw128(q0 + kb * HA * 128 + kk * 32), idesc_s, (kb | kk) != 0);
      }
      if (ok) mma_commit(s_full);
      if (ok) ok = mbar_wait(p_full, 0, abort_flag, p.err);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int mc = 0; mc < 4; ++mc)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16(tmem + O_COL + 64 * mc,
                     desc_mnmajor_sw128(kv0 + 2 * mc * kKBBytes + kk * 2048, kKBBytes, 1024),
                     desc_mnmajor_sw128(p0 + kk * 2048, 8192, 1024), idesc_o, kk != 0);
        mma_commit(o_full);
      }
    }
    __syncwarp();
    cluster_sync_all();                                // barrier 1
    cluster_sync_all();                                // barrier 2
  } else {
    // ------------------------------------------------------------ softmax + reductions
    const int quad = warp & 3;
    const int ew = warp - 2;                           // epilogue warp 0..3
    const int row = quad * 32 + lane;                  // TMEM lane = tile row
    const int et = ew * 32 + lane;                     // epilogue thread 0..127
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int64_t pos = static_cast<int64_t>(tile) * kRows + row;
    const int64_t id = pos < p.k ? ids[pos] : -1;
    const bool valid = id >= 0 && id < p.n;
    const int hb = reduced_head_base(lane);
    bool ok = mbar_wait(s_full, 0, abort_flag, p.err);
    float x[HA];
    if (ok) {
      tc_fence_after();
      uint32_t v[32];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        tmem_ld32(tmem + lane_off + S_COL + 32 * half, v);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 32; ++h) x[32 * half + h] = valid ? p.scale * __uint_as_float(v[h]) : -INFINITY;
      }
    } else {
#pragma unroll
      for (int h = 0; h < HA; ++h) x[h] = -INFINITY;
    }
    // the tile's per-head max m
    float red[HA];
#pragma unroll
    for (int h = 0; h < HA; ++h) red[h] = x[h];
    warp_transpose_reduce<true>(red, lane);
    sRed[ew * HA + hb] = red[0];
    sRed[ew * HA + hb + 1] = red[1];
    epi_bar();
    float* mine = sML + me * 2 * HA;                   // this CTA's (m, l) slot (also in every peer)
    if (et < HA)
      mine[et] = fmaxf(fmaxf(sRed[et], sRed[HA + et]), fmaxf(sRed[2 * HA + et], sRed[3 * HA + et]));
    epi_bar();
    // P = exp(x - m) in bf16, and its row sums
    float lsum[HA];
    {
      uint32_t packed[32];
#pragma unroll
      for (int h2 = 0; h2 < 32; ++h2) {
        float e[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int h = 2 * h2 + u;
          e[u] = (x[h] == -INFINITY) ? 0.0f : __expf(x[h] - mine[h]);
        }
        packed[h2] = pack_bf16x2(e[0], e[1]);
        lsum[2 * h2] = bf16_lo(packed[h2]);
        lsum[2 * h2 + 1] = bf16_hi(packed[h2]);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(sP + sw128_offset(row, c)) =
            make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(p_full);
    warp_transpose_reduce<false>(lsum, lane);
    sRed[ew * HA + hb] = lsum[0];
    sRed[ew * HA + hb + 1] = lsum[1];
    epi_bar();
    if (et < HA) mine[HA + et] = (sRed[et] + sRed[HA + et]) + (sRed[2 * HA + et] + sRed[3 * HA + et]);
    epi_bar();
    // push (m, l) to every peer
    for (int i = et; i < cs * 2 * HA; i += 128) {
      const int dst = i / (2 * HA), j = i % (2 * HA);
      if (dst != static_cast<int>(me)) st_cluster_f32(map_to_rank(smem_u32(&mine[j]), dst), mine[j]);
    }
    // stage the partial O^T [dim][head] in this CTA's own KV + P region
    if (ok) ok = mbar_wait(o_full, 0, abort_flag, p.err);
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int mc = 0; mc < 4; ++mc) {
        float* dst = sStage + (mc * 128 + row) * kStageStride;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + O_COL + 64 * mc + 32 * half, v);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<float4*>(dst + 32 * half + 4 * c) =
                make_float4(__uint_as_float(v[4 * c]), __uint_as_float(v[4 * c + 1]),
                            __uint_as_float(v[4 * c + 2]), __uint_as_float(v[4 * c + 3]));
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    cluster_sync_all();                                // barrier 1: every partial and (m, l) is in place
    // cluster max M, per-peer weights, cluster sum L
    if (et < HA) {
      float M = -INFINITY;
      for (int c = 0; c < cs; ++c) M = fmaxf(M, sML[c * 2 * HA + et]);
      float L = 0.0f;
      for (int c = 0; c < cs; ++c) {
        const float wgt = rescale(sML[c * 2 * HA + et], M);
        sWt[c * HA + et] = wgt;
        L += sML[c * 2 * HA + HA + et] * wgt;
      }
      sMcl[et] = M;
      sLcl[et] = L;
    }
    epi_bar();
    // pull this CTA's dims from every peer (16-byte chunks, consecutive threads
    // read consecutive chunks of a staged row) and add them in rank order
    const int dpo = DV / cs;                           // dims per owner
    float* sOwn = reinterpret_cast<float*>(sQ);        // [HA][dpo] f32 (q is no longer needed)
    const uint32_t stage0 = smem_u32(sStage);
#pragma unroll 2
    for (int ci = et; ci < dpo * (HA / 4); ci += 128) {
      const int dl = ci / (HA / 4), h4 = ci % (HA / 4);
      const uint32_t off = ((static_cast<uint32_t>(me) * dpo + dl) * kStageStride + 4 * h4) * 4;
      float4 part[kMaxCS];
#pragma unroll
      for (int c = 0; c < kMaxCS; ++c)
        if (c < cs) part[c] = ld_cluster_v4(map_to_rank(stage0 + off, c));
      float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < kMaxCS; ++c) {
        if (c < cs) {
          a[0] += part[c].x * sWt[c * HA + 4 * h4];
          a[1] += part[c].y * sWt[c * HA + 4 * h4 + 1];
          a[2] += part[c].z * sWt[c * HA + 4 * h4 + 2];
          a[3] += part[c].w * sWt[c * HA + 4 * h4 + 3];
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) sOwn[(4 * h4 + u) * dpo + dl] = a[u];
    }
    __syncwarp();
    cluster_sync_all();                                // barrier 2: peers are done reading this CTA
    // this owner's slice: [HA][dpo] f32 in sOwn, with (M, L) per head
    const int64_t out_base = qi * HA * DV + static_cast<int64_t>(me) * dpo;
    bool finish = p.ncl == 1;
    if (p.ncl > 1) {
      // publish the slice; the owner whose cluster arrives last merges them all
      const int64_t slice = static_cast<int64_t>(dpo) * HA + 2 * HA;
      float* g = p.part + ((qi * p.ncl + cl) * cs + me) * slice;
      for (int i = et; i < dpo * HA / 4; i += 128)
        reinterpret_cast<float4*>(g)[i] = reinterpret_cast<const float4*>(sOwn)[i];
      if (et < HA) {
        g[dpo * HA + et] = sMcl[et];
        g[dpo * HA + HA + et] = sLcl[et];
      }
      __threadfence();
      epi_bar();
      if (et == 0) sh_ticket = atomicAdd(&p.ticket[qi * cs + me], 1u);
      epi_bar();
      finish = sh_ticket == static_cast<unsigned>(p.ncl - 1);
      if (finish) {
        __threadfence();
        const float* g0 = p.part + (qi * p.ncl * cs + me) * slice;   // cluster c2 at + c2*cs*slice
        float* sWc = sML;                              // [ncl][HA] per-cluster weights ((m, l) exchange is over)
        if (et < HA) {
          float M = -INFINITY;
          for (int c2 = 0; c2 < p.ncl; ++c2) M = fmaxf(M, __ldcg(g0 + c2 * cs * slice + dpo * HA + et));
          float L = 0.0f;
          for (int c2 = 0; c2 < p.ncl; ++c2) {
            const float* gc = g0 + c2 * cs * slice;
            const float wgt = rescale(__ldcg(gc + dpo * HA + et), M);
            sWc[c2 * HA + et] = wgt;
            L += __ldcg(gc + dpo * HA + HA + et) * wgt;
          }
          sMcl[et] = M;
          sLcl[et] = L;
        }
        epi_bar();
        // 8 float4 chunks per thread and pass, two clusters per step: 16 loads in flight
        const int nchunk = dpo * HA / 4;
        for (int i0 = et; i0 < nchunk; i0 += 8 * 128) {
          float4 acc[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
          for (int c2 = 0; c2 < p.ncl; ++c2) {
            const float4* gc = reinterpret_cast<const float4*>(g0 + c2 * cs * slice);
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int i = i0 + u * 128;
              v[u] = i < nchunk ? __ldcg(gc + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int h = min((4 * (i0 + u * 128)) / dpo, HA - 1);
              const float w = sWc[c2 * HA + h];
              acc[u].x += v[u].x * w;
              acc[u].y += v[u].y * w;
              acc[u].z += v[u].z * w;
              acc[u].w += v[u].w * w;
            }
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * 128;
            if (i < nchunk) reinterpret_cast<float4*>(sOwn)[i] = acc[u];
          }
        }
        if (et == 0) p.ticket[qi * cs + me] = 0u;     // ready for the next call
        epi_bar();
      }
    }
    if (finish) {
      // normalise, bf16, coalesced 16-byte stores of the owned [64 heads x dpo dims] block
      const int pieces = dpo / 8;
      for (int i = et; i < HA * pieces; i += 128) {
        const int h = i / pieces, pc = i % pieces;
        const float L = sLcl[h];
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        const float* a = sOwn + h * dpo + pc * 8;
        uint4 o;
        o.x = pack_bf16x2(a[0] * inv, a[1] * inv);
        o.y = pack_bf16x2(a[2] * inv, a[3] * inv);
        o.z = pack_bf16x2(a[4] * inv, a[5] * inv);
        o.w = pack_bf16x2(a[6] * inv, a[7] * inv);
        *reinterpret_cast<uint4*>(p.out + out_base + static_cast<int64_t>(h) * DV + pc * 8) = o;
      }
      if (me == 0 && p.lse && et < HA)
        p.lse[qi * HA + et] = sLcl[et] > 0.0f ? sMcl[et] + logf(sLcl[et]) : -INFINITY;
    }
  }

  // ---------------------------------------------------------------- teardown
  if (threadIdx.x == 32) {
    // loads may still be landing if a wait gave up early (bounded: 0.1 s)
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(q_full, 0) && globaltimer_ns() - t0 < 100000000ull) {
    }
    for (int kb = 0; kb < kKB; ++kb)
      while (!mbar_try_wait(&kv_full[kb], 0) && globaltimer_ns() - t0 < 100000000ull) {
      }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

struct Shape {
  int cs, ncl;
};

// Cluster size and clusters per query for k selected rows (depends on k only).
Shape shape_for(int k) {
  const int tiles = (k + kRows - 1) / kRows;
  // Clusters of 4 leave every cluster of a batch-8 decode co-resident; of 8,
  // fewer fit at once than 148 SMs would suggest (whole GPCs are needed).
  int max_cs = kDefaultCS;
  if (const char* e = getenv("CSA2_ATTN_MAX_CLUSTER")) {   // tests: other cluster sizes
    const int v = atoi(e);
    if (v == 2 || v == 4 || v == 8) max_cs = v;
    if (v == 1) max_cs = kMinCS;
  }
  int cs = kMinCS;
  while (cs < tiles && cs < max_cs) cs *= 2;
  return {cs, (tiles + cs - 1) / cs};
}

size_t part_bytes(int64_t n_queries, Shape s) {
  if (s.ncl <= 1) return 0;
  const int64_t slice = static_cast<int64_t>(DV / s.cs) * HA + 2 * HA;
  return static_cast<size_t>(n_queries * s.ncl * s.cs * slice * 4);
}

size_t ticket_bytes(int64_t n_queries, Shape s) {
  return s.ncl <= 1 ? 0 : static_cast<size_t>(n_queries * s.cs * 4);
}

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

size_t sparse_attn_tc_workspace(int B, int Q, int Ha, int D, int k, csa2_kv_fmt fmt) {
  if (fmt != CSA2_KV_BF16 || Ha != HA || D != DV || k <= 0) return 0;
  const Shape s = shape_for(k);
  const int64_t nq = static_cast<int64_t>(B) * Q;
  if (s.ncl <= 1 || s.ncl > kMaxNCL) return 0;
  return a256(part_bytes(nq, s)) + a256(ticket_bytes(nq, s));
}

csa2_status launch_sparse_attn_tc(const void* q, const csa2_kv& kv, const int32_t* topk, int B,
                                  int Q, int Ha, int k, float scale, void* out, float* lse,
                                  void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (getenv("CSA2_ATTN_SIMT")) return CSA2_ERR_UNSUPPORTED;      // force the CUDA-core kernel
  if (kv.fmt != CSA2_KV_BF16 || kv.dim != DV || Ha != HA || k <= 0) return CSA2_ERR_UNSUPPORTED;
  const int64_t n_queries = static_cast<int64_t>(B) * Q;
  if (n_queries * HA > 0x7fffffffLL || static_cast<int64_t>(B) * kv.n > 0x7fffffffLL)
    return CSA2_ERR_UNSUPPORTED;
  const Shape s = shape_for(k);
  if (s.ncl > kMaxNCL || n_queries * s.cs * s.ncl > 0x7fffffffLL) return CSA2_ERR_UNSUPPORTED;
  const size_t need = sparse_attn_tc_workspace(B, Q, Ha, kv.dim, k, kv.fmt);
  if (need > 0 && (!ws || ws_bytes < need)) return CSA2_ERR_UNSUPPORTED;
  CUtensorMap qmap, kvmap;
  memset(&qmap, 0, sizeof(qmap));
  memset(&kvmap, 0, sizeof(kvmap));
  CSA2_TRY(make_tensor_map_bf16_2d(&qmap, q, static_cast<uint64_t>(n_queries) * HA, DV, DV * 2, 64, HA));
  CSA2_TRY(make_tensor_map_bf16_2d(&kvmap, kv.data, static_cast<uint64_t>(B) * kv.n, DV, DV * 2, 64, 1));
  Params p;
  p.topk = topk;
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.part = nullptr;
  p.ticket = nullptr;
  if (s.ncl > 1) {
    p.part = static_cast<float*>(ws);
    p.ticket = reinterpret_cast<unsigned*>(static_cast<char*>(ws) + a256(part_bytes(n_queries, s)));
    begin_launch(stream);
    if (cudaMemsetAsync(p.ticket, 0, ticket_bytes(n_queries, s), stream) != cudaSuccess)
      return check_launch("sparse_attn_tc: clear tickets");
    note_launch(LK_OTHER, 1, stream);
  }
  p.err = device_error_word();
  p.n = kv.n;
  p.Q = Q;
  p.k = k;
  p.cs = s.cs;
  p.ncl = s.ncl;
  p.scale = scale;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  });
  if (attr != cudaSuccess) return fail(CSA2_ERR_CUDA, "sparse_attn_tc: function attributes");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(n_queries * s.cs * s.ncl));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = s.cs;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  begin_launch(stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, attn_tc_kernel, qmap, kvmap, p);
  note_launch(LK_ATTN, 1, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(CSA2_ERR_CUDA, "sparse_attn_tc: launch failed: %s", cudaGetErrorString(e));
  }
  return check_launch("sparse_attn_tc");
}

}  // namespace csa2
