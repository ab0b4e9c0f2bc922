// Shared-KV sparse attention on the 5th-generation tensor cores (tcgen05).
// Source: "读完这篇，你就搞懂 DeepSeek v4 了", 注意力计算 (eq. 9): standard
// softmax attention in which all query heads share the selected compressed
// entries as keys and values; 批无关性 (batch invariance): the per-query
// reduction order is fixed and does not depend on the batch.
//
// Shapes: 64 heads, entries of width 512, bf16.  A query's k selected rows are
// cut into T = ceil(k / 128) tiles of 128 rows and each (query, tile) unit runs
// on one CTA.  The CTA computes its tile's partial result with the tile's own
// per-head max m (P = exp(s - m) rounded to bf16, l = sum of P, O = P^T KV in
// f32), writes (O, m, l) to a global workspace and raises its flag (a count
// of the partials it has written).  CTA t then reduces output dims
// [t * dpc, (t + 1) * dpc) over the T partials in tile order -- partial j is
// fetched as soon as tile j's flag shows it --, each weighted by
// exp(m_j - M) with M = max_j m_j, divides by L = sum_j l_j exp(m_j - M) and
// writes bf16 out (tile 0 also lse = M + log L).  The launch is cooperative:
// the whole grid is resident, so every flag wait ends.  A grid holds
// the units of G queries and loops over the batch in waves of G queries.  The
// split and the reduction order depend on k only, so results are
// deterministic and batch-invariant.
//
// Per CTA (6 warps):
//   warp 0     TMA load of the query's 64 x 512 heads, once per wave;
//   warp 1     TMEM allocation and MMA issue:
//                S^T[row, head]  = KV[row, :] . q[head, :]      (M=128, N=64, K=512)
//                O^T[dim, head] += KV[row, dim] * P[row, head]  (M=128 x4, N=64, K=128)
//              both read the same tile through K-major and MN-major descriptors;
//   warps 2-5  gather of the tile's 128 rows (16-byte cp.async copies straight
//              into the 128-byte-swizzled layout, 64 per thread in flight; the
//              next wave's gather is issued as soon as this wave's products are
//              done), softmax, partial write, flag waits, reduction, output.
// Every wait is bounded (mbarriers 2 s, the flags 1 s or the host-set bound);
// a CTA that gives up records CSA2_ERR_TIMEOUT and still takes every later
// step, so no other CTA waits for it in vain, and before it exits it waits
// (bounded) for its own copies and products in flight.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "launchers.h"
#include "attn_common.cuh"
#include "sm100.cuh"

namespace csa2 {
namespace {
using namespace sm100;
using namespace attn;

constexpr int kThreads = 6 * 32;
constexpr int kPartFloats = DV * HA;          // partial O^T [dim][head], 128 KiB
constexpr int kSlotFloats = kPartFloats + 2 * HA;   // + the tile's m[HA], l[HA]

constexpr int OFF_KV = 0;                              // 128 KiB: KV tile
constexpr int OFF_P = OFF_KV + kKB * kKBBytes;         // 16 KiB: P tile
constexpr int OFF_Q = OFF_P + kRows * 128;             // 64 KiB: q; after the products, the reduction's scratch
constexpr int OFF_RED = OFF_Q + kKB * HA * 128;        // [4 warps][HA] f32
constexpr int OFF_ML = OFF_RED + 4 * HA * 4;           // this tile's m[HA], l[HA]
constexpr int OFF_ML2 = OFF_ML + 2 * HA * 4;           // the query's M[HA], L[HA]
constexpr int OFF_BAR = OFF_ML2 + 2 * HA * 4;
constexpr int NBAR = 20;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
// reduction scratch inside the q region: output staging [HA][kStageStride]
// f32 for up to kStageDims dims, then per-tile weights and row sums [T][HA] f32
constexpr int kStageDims = 64;
constexpr int kStageStride = kStageDims + 1;
constexpr int kWeightsOff = HA * kStageStride * 4;
static_assert(kWeightsOff % 16 == 0 && kWeightsOff + 2 * kMaxTiles * HA * 4 <= kKB * HA * 128,
              "staging, weights and row sums fit the q region");
static_assert(SMEM_BYTES <= 232448, "shared memory");

struct Params {
  const int32_t* topk;             // [B*Q, k], or null: slot j is entry j (dense)
  const int32_t* n_vis;            // dense: [B*Q] visible entries, or null (all k)
  const uint16_t* win;             // window rows [B, win_rows, 512], or null (no window tile)
  const int32_t* win_end;          // [B*Q] one past the query's last window row
  int64_t win_rows;
  int W;                           // window length
  int T_sel;                       // tiles of selected rows; tile T_sel is the window tile
  const uint16_t* kv;              // [B, n, 512]
  uint16_t* out;                   // [B*Q, 64, 512]
  float* lse;                      // [B*Q, 64] or null
  float* part;                     // [2][grid][kSlotFloats]
  unsigned* flag;                  // [grid] partials written per CTA (equal across a query's CTAs between waves)
  int* err;
  int64_t n, n_queries;
  int Q, k, T, G, dpc;
  int bulk;                        // a CTA's dims of all T partials fit the KV region, their (m, l) the P region
  float scale;
  unsigned long long wait_ns;      // bound of the wait for another tile's partial
  unsigned wait_offset;            // added to the awaited count (0, or unreachable for tests)
};

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Drops a 128-byte line from L2 without writing it back (its content becomes
// undefined); used on workspace lines that no one reads again.
__device__ __forceinline__ void discard_l2_line(const void* p) {
  asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ unsigned sh_gen;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKV = smem + OFF_KV;
  uint8_t* sP = smem + OFF_P;
  uint8_t* sQ = smem + OFF_Q;
  float* sRed = reinterpret_cast<float*>(smem + OFF_RED);
  float* sML = reinterpret_cast<float*>(smem + OFF_ML);      // m[HA], l[HA] of this tile
  float* sML2 = reinterpret_cast<float*>(smem + OFF_ML2);    // M[HA], L[HA] of the query
  float* sStage = reinterpret_cast<float*>(sQ);              // [HA][kStageStride]
  float* sW = reinterpret_cast<float*>(sQ + kWeightsOff);    // [T][HA] combine factors a_j
  float* sLv = sW + kMaxTiles * HA;                          // [T][HA] combine factors b_j
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bar + 0;
  uint64_t* s_full = bar + 1;
  uint64_t* p_full = bar + 2;
  uint64_t* o_full = bar + 16;                 // [4]: one per 128-dim chunk of O^T
  uint64_t* m_done = bar + 4;                  // the reduction no longer needs the q region
  uint64_t* r_full = bar + 5;                  // this CTA's dims of every partial are in the KV region
  uint64_t* kv_full = bar + 8;                 // [8]: one per 64-column block of the tile
  uint64_t* mma_fin = bar + 3;                 // every MMA of this CTA has completed (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = static_cast<int>(blockIdx.x % p.T);
  const int slot = static_cast<int>(blockIdx.x / p.T);        // query slot: queries slot, slot+G, ...
  const int64_t n_waves = (p.n_queries - slot + p.G - 1) / p.G;
  constexpr uint32_t S_COL = 0;                       // S at columns [0, 64)
  constexpr uint32_t O_COL = 256;                     // O^T chunk mc at [256 + 64 mc, ...)
  // gather mapping (warps 2-5): thread et copies 16-byte chunk c16 of rows
  // grow0 + 16 i (i < 8) in every 64-column block; eight consecutive threads
  // cover one 128-byte row segment
  const int et = (warp - 2) * 32 + lane;
  const int c16 = et & 7, grow0 = et >> 3;
  // (grow0 + 16 i) & 7 == grow0 & 7: one swizzle per thread
  const uint32_t swz = static_cast<uint32_t>((c16 ^ (grow0 & 7)) << 4);
  auto issue_gather = [&](int64_t qi) {
    const bool win_tile = tile >= p.T_sel;
    const uint16_t* base = (win_tile ? p.win + (qi / p.Q) * p.win_rows * DV
                                     : p.kv + (qi / p.Q) * p.n * DV) + c16 * 8;
    int64_t off[8];
    uint32_t nbytes[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int id = tile_row(p, qi, tile, grow0 + 16 * i);
      off[i] = static_cast<int64_t>(id >= 0 ? id : 0) * DV;
      nbytes[i] = id >= 0 ? 16u : 0u;            // empty slot: zero fill, nothing read
    }
#pragma unroll 1
    for (int kb = 0; kb < kKB; ++kb) {          // not unrolled: one short body, re-executed
#pragma unroll
      for (int i = 0; i < 8; ++i)
        cp_async_16(sKV + kb * kKBBytes + (grow0 + 16 * i) * 128 + swz, base + off[i] + kb * 64,
                    nbytes[i]);
      cp_async_commit();
    }
  };
  // the first wave's rows are requested before the barriers and TMEM are set
  // up (the copies need neither; they are published after the set-up)
  pdl_wait();                                  // the selection comes from the kernel before
  if (warp >= 2 && n_waves > 0) issue_gather(slot);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 4);
    for (int mc = 0; mc < 4; ++mc) mbar_init(&o_full[mc], 1);
    mbar_init(m_done, 1);
    mbar_init(r_full, 1);
    mbar_init(mma_fin, 1);
    for (int kb = 0; kb < kKB; ++kb) mbar_init(&kv_full[kb], 128);
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

  if (warp == 0) {
    // ------------------------------------------------------------ q loader
    if (lane == 0) {
      int64_t issued = 0;
      for (int64_t w = 0; w < n_waves; ++w) {
        if (w > 0 && !mbar_wait(m_done, static_cast<uint32_t>((w - 1) & 1), abort_flag, p.err)) break;
        const int64_t qi = slot + w * p.G;
        mbar_arrive_expect_tx(q_full, HA * DV * 2);
#pragma unroll
        for (int kb = 0; kb < kKB; ++kb)
          tma_load_2d(sQ + kb * HA * 128, &qmap, q_full, kb * 64, static_cast<int32_t>(qi * HA));
        issued = w + 1;
      }
      // the last load has landed before the CTA may exit (bounded: 0.1 s)
      if (issued > 0) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(q_full, static_cast<uint32_t>((issued - 1) & 1)) &&
               globaltimer_ns() - t0 < 100000000ull) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, HA, false, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, HA, true, true);
    const uint32_t kv0 = smem_u32(sKV), q0 = smem_u32(sQ), p0 = smem_u32(sP);
    if (lane == 0) {
      for (int64_t w = 0; w < n_waves; ++w) {
        const uint32_t par = static_cast<uint32_t>(w & 1);
        bool ok = mbar_wait(q_full, par, abort_flag, p.err);
#pragma unroll 1
        for (int kb = 0; kb < kKB && ok; ++kb) {
          ok = mbar_wait(&kv_full[kb], par, abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + S_COL, desc_kmajor_sw128(kv0 + kb * kKBBytes + kk * 32),
                     desc_kmajor_sw128(q0 + kb * HA * 128 + kk * 32), idesc_s, (kb | kk) != 0);
        }
        if (!ok) break;
        mma_commit(s_full);
        if (!mbar_wait(p_full, par, abort_flag, p.err)) break;
        tc_fence_after();
#pragma unroll
        for (int mc = 0; mc < 4; ++mc) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16(tmem + O_COL + 64 * mc,
                     desc_mnmajor_sw128(kv0 + 2 * mc * kKBBytes + kk * 2048, kKBBytes, 1024),
                     desc_mnmajor_sw128(p0 + kk * 2048, 8192, 1024), idesc_o, kk != 0);
          mma_commit(&o_full[mc]);                 // chunk mc can be read while mc+1 computes
        }
      }
      // before TMEM is freed, every product issued above has completed, also
      // when a wait gave up on the way (bounded: 0.1 s)
      mma_commit(mma_fin);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(mma_fin, 0) && globaltimer_ns() - t0 < 100000000ull) {
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ gather, softmax, reduction
    const int quad = warp & 3;
    const int ew = warp - 2;                           // epilogue warp 0..3
    const int row = quad * 32 + lane;                  // TMEM lane = tile row
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int hb = 2 * lane;                         // the heads lane reduces last
    // each 64-column block is published once this thread's copies into it landed
    auto publish_gather = [&]() {
#define CSA2_PUBLISH(KB)            \
  cp_async_wait<kKB - 1 - (KB)>();  \
  fence_proxy_async_smem();         \
  mbar_arrive(&kv_full[KB]);
      CSA2_PUBLISH(0) CSA2_PUBLISH(1) CSA2_PUBLISH(2) CSA2_PUBLISH(3)
      CSA2_PUBLISH(4) CSA2_PUBLISH(5) CSA2_PUBLISH(6) CSA2_PUBLISH(7)
#undef CSA2_PUBLISH
    };
    if (n_waves > 0) publish_gather();
    bool ok = true;
    for (int64_t w = 0; w < n_waves; ++w) {
      const int64_t qi = slot + w * p.G;
      const uint32_t par = static_cast<uint32_t>(w & 1);
      const bool valid = tile_row(p, qi, tile, row) >= 0;
      ok = ok && mbar_wait(s_full, par, abort_flag, p.err);
      float x[HA];
      if (ok) {
        tc_fence_after();
        uint32_t v0[32], v1[32];
        tmem_ld32(tmem + lane_off + S_COL, v0);
        tmem_ld32(tmem + lane_off + S_COL + 32, v1);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 32; ++h) {
          x[h] = scaled_score(valid, p.scale, v0[h]);
          x[32 + h] = scaled_score(valid, p.scale, v1[h]);
        }
      } else {
#pragma unroll
        for (int h = 0; h < HA; ++h) x[h] = -INFINITY;
      }
      // the tile's per-head max m: one warp-wide max per head, then over the 4 warps
#pragma unroll
      for (int h = 0; h < HA; ++h) {
        const float mh = warp_max_f32(x[h]);
        if (lane == 0) sRed[ew * HA + h] = mh;
      }
      epi_bar();
      if (et < HA)
        sML[et] = fmaxf(fmaxf(sRed[et], sRed[HA + et]), fmaxf(sRed[2 * HA + et], sRed[3 * HA + et]));
      epi_bar();
      // P = exp(x - m) in bf16, and its row sums
      float lsum[HA];
      {
        const uint32_t ml0 = smem_u32(sML), p0 = smem_u32(sP);
        uint32_t packed[32];
#pragma unroll
        for (int h4 = 0; h4 < HA / 4; ++h4) {
          const float4 m4 = lds_v4f(ml0 + 16 * h4);
          const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int h = 4 * h4 + 2 * u;
            const float e0 = p_value(x[h], mm[2 * u]);
            const float e1 = p_value(x[h + 1], mm[2 * u + 1]);
            const uint32_t pk = pack_bf16x2(e0, e1);
            packed[2 * h4 + u] = pk;
            lsum[h] = bf16_lo(pk);
            lsum[h + 1] = bf16_hi(pk);
          }
        }
#pragma unroll
        for (int c = 0; c < 8; ++c)
          sts_v4u(p0 + sw128_offset(row, c), packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      warp_transpose_reduce<HA, false>(lsum, lane);
      sRed[ew * HA + hb] = lsum[0];
      sRed[ew * HA + hb + 1] = lsum[1];
      epi_bar();
      if (et < HA) sML[HA + et] = quad_sum(sRed[et], sRed[HA + et], sRed[2 * HA + et], sRed[3 * HA + et]);
      // partial (O^T, m, l) of this tile to workspace slot (buffer w & 1, CTA).
      // O^T is staged in the KV region as [dim][16 chunks of 4 heads] with
      // chunk h4 at position h4 ^ (dim & 7) (conflict-free) and written with
      // (m, l) by two bulk stores; the slot keeps that layout.
      const bool more = w + 1 < n_waves;
      const int64_t buf = (w & 1) * static_cast<int64_t>(gridDim.x);
      const uint32_t kv0 = smem_u32(sKV);
      float* my_slot = p.part + (buf + blockIdx.x) * kSlotFloats;
#pragma unroll 1
      for (int mc = 0; mc < 4; ++mc) {
        const int dim = mc * 128 + row;
        const uint32_t srow = kv0 + dim * (HA * 4);
        // chunk mc's products are done; its staging rows are the KV blocks
        // 2mc, 2mc+1, which only chunk mc's products read
        ok = ok && mbar_wait(&o_full[mc], par, abort_flag, p.err);
        tc_fence_after();
        if (ok) {
          uint32_t v0[32], v1[32];
          tmem_ld32(tmem + lane_off + O_COL + 64 * mc, v0);
          tmem_ld32(tmem + lane_off + O_COL + 64 * mc + 32, v1);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            sts_v4u(srow + ((c ^ (dim & 7)) << 4), v0[4 * c], v0[4 * c + 1], v0[4 * c + 2], v0[4 * c + 3]);
            sts_v4u(srow + (((8 + c) ^ (dim & 7)) << 4), v1[4 * c], v1[4 * c + 1], v1[4 * c + 2], v1[4 * c + 3]);
          }
        }
        fence_proxy_async_smem();
        epi_bar();                                     // chunk mc staged (and, at mc = 3, l is in sML)
        if (et == 0) {
          bulk_store(my_slot + mc * 128 * HA, sKV + mc * 128 * HA * 4, 128 * HA * 4);
          if (mc == 3) bulk_store(my_slot + kPartFloats, sML, 2 * HA * 4);
          bulk_commit();
        }
      }
      tc_fence_before();
      const int64_t base = buf + (blockIdx.x - tile);  // workspace slot of tile 0
      const float* pb = p.part + base * kSlotFloats;   // slot j at pb + j * kSlotFloats
      const int d0 = min(DV, tile * p.dpc), d1 = min(DV, d0 + p.dpc);
      const uint32_t slice_bytes = static_cast<uint32_t>(d1 - d0) * HA * 4;
      if (et == 0) {
        bulk_wait_all();
        fence_proxy_async_global();
        __threadfence();
        // publish: this CTA's flag counts the partials it has written
        sh_gen = atomicAdd(&p.flag[blockIdx.x], 1u) + 1u;
        if (p.bulk) mbar_arrive_expect_tx(r_full, (slice_bytes + 2 * HA * 4) * p.T);
      }
      epi_bar();
      // thread j waits for tile j's partial of this wave (every CTA of the grid
      // is resident: the launch is cooperative) and, on the bulk path, loads
      // this CTA's dims of it and its (m, l) at once
      if (et < p.T) {
        const unsigned gen = sh_gen + p.wait_offset;
        const unsigned* fj = p.flag + (blockIdx.x - tile) + et;
        const uint64_t t0 = globaltimer_ns();
        while (static_cast<int>(ld_acquire_u32(fj) - gen) < 0) {
          if (globaltimer_ns() - t0 > p.wait_ns) {
            raise_dev_error(p.err, DEVERR_TIMEOUT);
            *abort_flag = 1;
            break;
          }
        }
        fence_proxy_async_global();
        if (p.bulk) {
          const float* sj = pb + static_cast<int64_t>(et) * kSlotFloats;
          if (slice_bytes > 0) bulk_load(sKV + et * slice_bytes, sj + d0 * HA, slice_bytes, r_full);
          bulk_load(sP + et * 2 * HA * 4, sj + kPartFloats, 2 * HA * 4, r_full);
        }
      }
      epi_bar();
      // the tile-order combine factors (a_j, b_j) of every head, the query's M and L
      {
        if (p.bulk) {
          // the copies read memory that exists whatever the flags said, so they
          // all land: wait for them also after a give-up (bounded: 0.1 s), so
          // that no copy is in flight when the region is reused or the CTA exits
          const uint64_t t0 = globaltimer_ns();
          bool landed;
          while (!(landed = mbar_try_wait(r_full, par)) && globaltimer_ns() - t0 < 100000000ull) {
          }
          ok = ok && landed;
        } else {
          // (m_j, l_j) of every tile into sW (m) and sLv (l)
          float* dstv = et < HA ? sW : sLv;
#pragma unroll 8
          for (int j = 0; j < p.T; ++j)
            dstv[j * HA + (et & (HA - 1))] = __ldcg(pb + static_cast<int64_t>(j) * kSlotFloats + kPartFloats + et);
          epi_bar();
        }
        if (et < HA) {
          // m_j, l_j: on the bulk path in the P region (tile j at j * 512 bytes:
          // m then l), else in sW / sLv; a_j over m_j in sW, b_j over l_j in sLv
          const uint32_t mlb = smem_u32(sP) + et * 4;
          float M = -INFINITY, L = 0.0f;
          for (int j = 0; j < p.T; ++j) {
            const float mj = p.bulk ? lds_f32(mlb + j * 2 * HA * 4) : sW[j * HA + et];
            const float lj = p.bulk ? lds_f32(mlb + j * 2 * HA * 4 + HA * 4) : sLv[j * HA + et];
            const float2 ab = combine_step(M, L, mj, lj);
            sW[j * HA + et] = ab.x;
            sLv[j * HA + et] = ab.y;
          }
          sML2[et] = M;
          sML2[HA + et] = L;
        }
      }
      epi_bar();
      // this CTA's output dims: sum over the partials in tile order
      const uint32_t w0 = smem_u32(sW), l0 = smem_u32(sLv);
      for (int ds = d0; ds < d1; ds += kStageDims) {
        const int nd = min(kStageDims, d1 - ds);
        const int nch = nd * (HA / 4);                 // float4 chunks (dim, 4 heads)
        for (int c0 = et; c0 < nch; c0 += 4 * 128) {
          const int h4 = c0 & 15;                      // the same for every u below
          uint32_t off[4];                             // byte offset of chunk u within a slice
          bool in[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int c = c0 + u * 128;
            const int dim = ds + (c >> 4);
            in[u] = c < nch;
            off[u] = static_cast<uint32_t>((dim - d0) * (HA * 4) + ((h4 ^ (dim & 7)) << 4));
          }
          float4 acc[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (p.bulk) {
#pragma unroll 2
            for (int j = 0; j < p.T; ++j) {
              float4 v[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) v[u] = lds_v4f(kv0 + j * slice_bytes + (in[u] ? off[u] : 0));
              const float4 aj = lds_v4f(w0 + (j * HA + 4 * h4) * 4);
              const float4 bj = lds_v4f(l0 + (j * HA + 4 * h4) * 4);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                acc[u].x = combine_acc(acc[u].x, v[u].x, aj.x, bj.x);
                acc[u].y = combine_acc(acc[u].y, v[u].y, aj.y, bj.y);
                acc[u].z = combine_acc(acc[u].z, v[u].z, aj.z, bj.z);
                acc[u].w = combine_acc(acc[u].w, v[u].w, aj.w, bj.w);
              }
            }
          } else {
#pragma unroll 4
            for (int j = 0; j < p.T; ++j) {
              const uint8_t* sj = reinterpret_cast<const uint8_t*>(pb + static_cast<int64_t>(j) * kSlotFloats + d0 * HA);
              float4 v[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) v[u] = __ldcg(reinterpret_cast<const float4*>(sj + (in[u] ? off[u] : 0)));
              const float4 aj = *reinterpret_cast<const float4*>(sW + j * HA + 4 * h4);
              const float4 bj = *reinterpret_cast<const float4*>(sLv + j * HA + 4 * h4);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                acc[u].x = combine_acc(acc[u].x, v[u].x, aj.x, bj.x);
                acc[u].y = combine_acc(acc[u].y, v[u].y, aj.y, bj.y);
                acc[u].z = combine_acc(acc[u].z, v[u].z, aj.z, bj.z);
                acc[u].w = combine_acc(acc[u].w, v[u].w, aj.w, bj.w);
              }
            }
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (in[u]) {
              const int dl = (c0 + u * 128) >> 4, h0 = 4 * h4;
              sStage[(h0 + 0) * kStageStride + dl] = acc[u].x;
              sStage[(h0 + 1) * kStageStride + dl] = acc[u].y;
              sStage[(h0 + 2) * kStageStride + dl] = acc[u].z;
              sStage[(h0 + 3) * kStageStride + dl] = acc[u].w;
            }
          }
        }
        epi_bar();
        if (more && ds + kStageDims >= d1) issue_gather(qi + p.G);   // the KV region is free again
        // normalise, bf16, 8-byte stores of 4 dims
        const int pieces = nd / 4;
        for (int i = et; i < HA * pieces; i += 128) {
          const int h = i / pieces, pc = i % pieces;
          const float inv = inv_sum(sML2[HA + h]);
          const float* a = sStage + h * kStageStride + 4 * pc;
          uint2 o;
          o.x = pack_bf16x2(__fmul_rn(a[0], inv), __fmul_rn(a[1], inv));
          o.y = pack_bf16x2(__fmul_rn(a[2], inv), __fmul_rn(a[3], inv));
          *reinterpret_cast<uint2*>(p.out + (qi * HA + h) * DV + ds + 4 * pc) = o;
        }
        epi_bar();
      }
      if (more && d1 <= d0) issue_gather(qi + p.G);
      if (tile == 0 && p.lse && et < HA)
        p.lse[qi * HA + et] = lse_of(sML2[et], sML2[HA + et]);
      // this CTA alone reads its dims of every partial: drop those lines from L2
      if (d1 > d0) {
        const int lines = static_cast<int>(slice_bytes / 128);
        for (int i = et; i < p.T * lines; i += 128) {
          const int j = i / lines, ln = i % lines;
          discard_l2_line(pb + static_cast<int64_t>(j) * kSlotFloats + d0 * HA + ln * 32);
        }
      }
      epi_bar();
      if (et == 0) mbar_arrive(m_done);
      if (more) publish_gather();
    }
    cp_async_wait<0>();
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

struct Shape {
  int T_sel, T, dpc;
};

// T_sel tiles of selected rows (k slots), plus one window tile when `win`.
Shape shape_for(int k, bool win) {
  const int T_sel = (k + kRows - 1) / kRows;
  const int T = T_sel + (win ? 1 : 0);
  const int per = (DV + T - 1) / T;
  return {T_sel, T, (per + 3) / 4 * 4};
}

// CTAs of this kernel that fit on the device at once (cached), capped by the
// environment variable CSA2_ATTN_MAX_CTAS (tests: several waves per launch).
int resident_ctas() {
  static PerDevice<int> cache;
  int c = cache.get([] {
    int per_sm = 0;
    if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attn_tc_kernel, kThreads, SMEM_BYTES) !=
            cudaSuccess) {
      cudaGetLastError();
      per_sm = 0;
    }
    return std::min(per_sm * sm_count(), kAttnMaxGrid);
  });
  if (const char* e = getenv("CSA2_ATTN_MAX_CTAS")) {
    const int v = atoi(e);
    if (v > 0) c = std::min(c, v);
  }
  return c;
}

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace sized for the largest grid the kernel can get on any device
// (kAttnMaxGrid CTAs), so that its size does not depend on the device.
struct WsLayout {
  size_t part, sync, total;
};
WsLayout ws_layout(int64_t n_queries, Shape s) {
  const int64_t g = std::min<int64_t>(n_queries, kAttnMaxGrid / s.T);
  const int64_t ctas = g * s.T;
  WsLayout l;
  l.part = a256(static_cast<size_t>(2 * ctas) * kSlotFloats * 4);
  l.sync = a256(static_cast<size_t>(ctas) * 4);
  l.total = l.part + l.sync;
  return l;
}

bool applies(int Ha, int D, int k, csa2_kv_fmt fmt, bool win) {
  if (fmt != CSA2_KV_BF16 || Ha != HA || D != DV || k < 0) return false;
  const Shape s = shape_for(k, win);
  return s.T >= 1 && s.T <= kMaxTiles && s.T <= kAttnMaxGrid;
}

}  // namespace

size_t sparse_attn_tc_workspace(int B, int Q, int Ha, int D, int k, csa2_kv_fmt fmt, bool win) {
  if (!applies(Ha, D, k, fmt, win)) return 0;
  return ws_layout(static_cast<int64_t>(B) * Q, shape_for(k, win)).total;
}

csa2_status launch_sparse_attn_tc(const void* q, const csa2_kv& kv, const int32_t* topk, int B,
                                  int Q, int Ha, int k, float scale, void* out, float* lse,
                                  void* ws, size_t ws_bytes, unsigned long long* sync_zeroed,
                                  cudaStream_t stream, const AttnRows& rows) {
  if (getenv("CSA2_ATTN_SIMT")) return CSA2_ERR_UNSUPPORTED;      // force the CUDA-core kernel
  const bool win = rows.win != nullptr;
  if (!applies(Ha, kv.dim, k, kv.fmt, win)) return CSA2_ERR_UNSUPPORTED;
  const int64_t n_queries = static_cast<int64_t>(B) * Q;
  if (n_queries * HA > 0x7fffffffLL) return CSA2_ERR_UNSUPPORTED;
  if (sparse_attn_seq_applies(n_queries, k, win))       // many queries: one CTA per query
    return launch_sparse_attn_seq(q, kv, topk, B, Q, k, scale, out, lse, stream, rows);
  const Shape s = shape_for(k, win);
  const int cap = resident_ctas();
  if (cap < s.T) return CSA2_ERR_UNSUPPORTED;
  const WsLayout lay = ws_layout(n_queries, s);
  if (!ws || ws_bytes < lay.total) return CSA2_ERR_UNSUPPORTED;
  const int64_t G = std::min<int64_t>(n_queries, cap / s.T);
  CUtensorMap qmap;
  memset(&qmap, 0, sizeof(qmap));
  CSA2_TRY(make_tensor_map_bf16_2d(&qmap, q, static_cast<uint64_t>(n_queries) * HA, DV, DV * 2, 64, HA));
  Params p;
  p.topk = topk;
  p.n_vis = rows.n_visible;
  p.win = static_cast<const uint16_t*>(rows.win);
  p.win_end = rows.win_end;
  p.win_rows = rows.win_rows;
  p.W = rows.W;
  p.T_sel = s.T_sel;
  p.kv = static_cast<const uint16_t*>(kv.data);
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.part = static_cast<float*>(ws);
  p.flag = sync_zeroed ? reinterpret_cast<unsigned*>(sync_zeroed)
                       : reinterpret_cast<unsigned*>(static_cast<char*>(ws) + lay.part);
  p.err = device_error_word();
  p.n = kv.n;
  p.n_queries = n_queries;
  p.Q = Q;
  p.k = k;
  p.T = s.T;
  p.G = static_cast<int>(G);
  p.dpc = s.dpc;
  p.bulk = static_cast<int64_t>(s.T) * s.dpc * HA * 4 <= kKB * kKBBytes && s.T * 2 * HA * 4 <= kRows * 128;
  p.scale = scale;
  p.wait_ns = cross_cta_wait_ns();
  p.wait_offset = cross_cta_wait_offset();
  if (!sync_zeroed) {          // a caller workspace: flags start at zero
    begin_launch(stream);
    if (cudaMemsetAsync(p.flag, 0, static_cast<size_t>(G) * s.T * 4, stream) != cudaSuccess)
      return check_launch("sparse_attn_tc: clear flags");
    note_launch(LK_OTHER, 1, stream);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(G * s.T));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  at[1] = pdl_attribute();
  cfg.attrs = at;
  cfg.numAttrs = 2;
  begin_launch(stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, attn_tc_kernel, qmap, p);
  note_launch(LK_ATTN, 1, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(CSA2_ERR_CUDA, "sparse_attn_tc: launch failed: %s", cudaGetErrorString(e));
  }
  return check_launch("sparse_attn_tc");
}

}  // namespace csa2
