// Shared-KV sparse attention on the tensor cores for narrow entries (width
// 128; 16, 32 or 64 heads; bf16 or FP4 rows).  Sources: "读完这篇，你就搞懂
// DeepSeek v4 了", 注意力计算 (eq. 9): every head attends the same selected
// entries as keys and values; "Recall之王 祭出Reuse", FP4 主KV缓存: E2M1 values
// with one E4M3 scale per 16 channels (each dequantised value is exact in
// bf16, so the FP4 rows enter the products exactly).
//
// A query's slots are cut into T tiles of 128 rows (the selected slots, then
// one tile of window rows when the layer has that branch); each (query, tile)
// unit runs on one CTA:
//   warps 2-5  gather the tile's rows into the 128-byte-swizzled layout
//              (bf16 rows by 16-byte cp.async; FP4 rows loaded, dequantised to
//              bf16 and stored), q likewise, then the softmax of the tile;
//   warp 1     TMEM allocation and the two products:
//                S^T[row, head] = KV[row, :] . q[head, :]     (M=128, N=HA, K=128)
//                O^T[dim, head] = KV[row, dim] * P[row, head] (M=128, N=HA, K=128)
//              (P is stored transposed, [head][row], so both B operands are
//              K-major; KV^T is read through an MN-major descriptor).
// The tile's result (O with the tile's own max m and row sum l) is final when
// T = 1; otherwise it goes to a workspace slot and the query's last CTA to
// finish combines the T partials in tile order with the running-max combine
// of attn_common.cuh.  The split and the order depend on k and the window
// only: a query's result does not depend on the batch.  Every wait is bounded.
#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "attn_common.cuh"
#include "common.cuh"
#include "launchers.h"
#include "sm100.cuh"

namespace csa2 {
namespace {
using namespace sm100;
using attn::combine_acc;
using attn::combine_step;
using attn::inv_sum;
using attn::lse_of;
using attn::p_value;
using attn::scaled_score;
using attn::tile_row;
using attn::warp_max_f32;

constexpr int DN = 128;                       // entry width
constexpr int kRows = 128;                    // rows per tile
constexpr int kKBBytes = kRows * 128;         // one 64-column block of the tile (16 KiB)
constexpr int kThreads = 6 * 32;
constexpr int kMaxTilesN = 64;

template <int HA>
struct Lay {
  static constexpr int QKB = HA * 128;                  // one 64-dim block of q (or P^T)
  static constexpr int OFF_KV = 0;                      // 32 KiB
  static constexpr int OFF_Q = OFF_KV + 2 * kKBBytes;   // 2 blocks of [HA][64] bf16
  static constexpr int OFF_P = OFF_Q + 2 * QKB;         // P^T: 2 blocks of [HA][64 rows] bf16
  static constexpr int OFF_RED = OFF_P + 2 * QKB;       // [4 warps][HA] f32
  static constexpr int OFF_ML = OFF_RED + 4 * HA * 4;   // m[HA], l[HA] of the tile
  static constexpr int OFF_AB = OFF_ML + 2 * HA * 4;    // combine factors [T][2][HA]
  static constexpr int OFF_BAR = OFF_AB + kMaxTilesN * 2 * HA * 4;
  static constexpr int OFF_MISC = OFF_BAR + 4 * 8;
  static constexpr int BYTES = OFF_MISC + 16 + 1024;
  static_assert(OFF_Q % 1024 == 0 && OFF_P % 1024 == 0 && OFF_BAR % 8 == 0, "alignment");
};

struct Params {
  const int32_t* topk;             // [B*Q, k], or null: slot j is entry j (dense)
  const int32_t* n_vis;            // dense: [B*Q] visible entries, or null (all k)
  const uint16_t* win;             // window rows [B, win_rows, 128] bf16, or null
  const int32_t* win_end;          // [B*Q]
  int64_t win_rows;
  int W;
  int T_sel;                       // tiles of selected rows; tile T_sel is the window tile
  const void* kv;                  // [B, n, 128] bf16, or FP4 codes [B, n, 64]
  const uint8_t* kv_scales;        // FP4: [B, n, 8] E4M3 scales, else null
  const uint16_t* q;               // [B*Q, HA, 128]
  uint16_t* out;                   // [B*Q, HA, 128]
  float* lse;                      // [B*Q, HA] or null
  float* part;                     // [queries of the launch][T][128 * HA + 2 * HA]
  unsigned* counters;              // [queries of the launch]: zero before, left zero after
  int* err;
  int64_t n, q_base;
  int Q, k, T;
  float scale;
};

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// byte offset of 16-byte chunk c of row r in a 128-byte-swizzled block
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

// E2M1 code (4 bits) times an E4M3 scale, exact in f32 (and in bf16)
__device__ __forceinline__ float e2m1_times(uint32_t code, float s) {
  const uint32_t e = (code >> 1) & 3u, mt = code & 1u;
  const float mag = (e == 0) ? 0.5f * static_cast<float>(mt)
                             : (1.0f + 0.5f * static_cast<float>(mt)) * static_cast<float>(1u << (e - 1));
  return ((code & 8u) ? -mag : mag) * s;
}
__device__ __forceinline__ float e4m3_value(uint32_t sc) {
  const uint32_t se = (sc >> 3) & 15u, sm = sc & 7u;
  float s = (se == 0) ? static_cast<float>(sm) * 0x1p-9f : __uint_as_float(((se + 120u) << 23) | (sm << 20));
  return (sc & 128u) ? -s : s;
}

template <int HA, bool FP4>
__global__ void __launch_bounds__(kThreads) attn_narrow_kernel(const Params p) {
  using L = Lay<HA>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int last_s;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKV = smem + L::OFF_KV;
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sP = smem + L::OFF_P;
  float* sRed = reinterpret_cast<float*>(smem + L::OFF_RED);
  float* sML = reinterpret_cast<float*>(smem + L::OFF_ML);
  float* sAB = reinterpret_cast<float*>(smem + L::OFF_AB);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* kv_full = bar + 0;                 // rows and q in place (128 epilogue threads)
  uint64_t* s_full = bar + 1;
  uint64_t* p_full = bar + 2;                  // P^T in place (4 epilogue warps)
  uint64_t* o_full = bar + 3;                  // also: every product has completed (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ql = blockIdx.x / p.T;                  // query within the launch
  const int tile = static_cast<int>(blockIdx.x % p.T);
  const int64_t qi = p.q_base + ql;                     // flat (b, q)
  const int64_t seq = qi / p.Q;
  constexpr uint32_t S_COL = 0, O_COL = 64;             // S^T and O^T: HA columns each

  pdl_wait();                                           // the selection comes from the kernel before
  // q and the tile's rows are requested before the barriers and TMEM are set
  // up (warps 2-5; thread et takes row et); they land in shared memory after
  const int et = (warp - 2) * 32 + lane;                // 0..127 in warps 2-5
  const bool win_tile = tile >= p.T_sel;
  constexpr int QPT = HA * 16 / 128;                    // 16-byte chunks of q per thread
  uint4 qv[QPT];
  uint4 codes[4] = {};
  uint2 scl = make_uint2(0, 0);
  int id = -1;
  if (warp >= 2) {
    const uint4* qg = reinterpret_cast<const uint4*>(p.q + qi * HA * DN);
#pragma unroll
    for (int j = 0; j < QPT; ++j) qv[j] = __ldg(qg + et + 128 * j);
    id = tile_row(p, qi, tile, et);
    if (!FP4 || win_tile) {
      const uint16_t* src = win_tile ? p.win + (seq * p.win_rows + (id >= 0 ? id : 0)) * DN
                                     : static_cast<const uint16_t*>(p.kv) + (seq * p.n + (id >= 0 ? id : 0)) * DN;
#pragma unroll
      for (int c = 0; c < 16; ++c)
        cp_async_16(sKV + (c >> 3) * kKBBytes + swz(et, c & 7), src + c * 8, id >= 0 ? 16u : 0u);
      cp_async_commit();
    } else if (id >= 0) {
      const int64_t r = seq * p.n + id;
      const uint4* cg = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.kv) + r * (DN / 2));
#pragma unroll
      for (int j = 0; j < 4; ++j) codes[j] = __ldg(cg + j);
      scl = __ldg(reinterpret_cast<const uint2*>(p.kv_scales + r * (DN / 16)));
    }
  }
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 128);
    mbar_init(s_full, 1);
    mbar_init(p_full, 4);
    mbar_init(o_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, HA, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, HA, true, false);
      const uint32_t kv0 = smem_u32(sKV), q0 = smem_u32(sQ), p0 = smem_u32(sP);
      bool ok = mbar_wait(kv_full, 0, abort_flag, p.err);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + S_COL, desc_kmajor_sw128(kv0 + kb * kKBBytes + kk * 32),
                     desc_kmajor_sw128(q0 + kb * L::QKB + kk * 32), idesc_s, (kb | kk) != 0);
        mma_commit(s_full);
        ok = mbar_wait(p_full, 0, abort_flag, p.err);
      }
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)            // 16 rows per product
          mma_bf16(tmem + O_COL, desc_mnmajor_sw128(kv0 + kk * 2048, kKBBytes, 1024),
                   desc_kmajor_sw128(p0 + (kk >> 2) * L::QKB + (kk & 3) * 32), idesc_o, kk != 0);
      }
      // o_full completes once every product issued above has completed, also
      // when a wait gave up on the way
      mma_commit(o_full);
    }
    __syncwarp();
  } else if (warp >= 2) {
    // ------------------------------------------------------------ gather, softmax, output
    const int quad = warp & 3;
    const int ew = warp - 2;                            // 0..3
    const int row = quad * 32 + lane;                   // TMEM lane = tile row (and O^T dim)
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    // q: [HA heads][128 dims] in two 64-dim blocks of 16-byte chunks
#pragma unroll
    for (int j = 0; j < QPT; ++j) {
      const int i = et + 128 * j, h = i >> 4, c = i & 15;
      *reinterpret_cast<uint4*>(sQ + (c >> 3) * L::QKB + swz(h, c & 7)) = qv[j];
    }
    if (!FP4 || win_tile) {
      cp_async_wait<0>();
    } else {
      // chunk c holds channels 8c .. 8c+7: 4 code bytes of block c / 2
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint4 cw4 = codes[c >> 2];
        const uint32_t cw = (c & 3) == 0 ? cw4.x : (c & 3) == 1 ? cw4.y : (c & 3) == 2 ? cw4.z : cw4.w;
        const uint32_t sb = ((c >> 1) < 4 ? scl.x >> (8 * (c >> 1)) : scl.y >> (8 * ((c >> 1) - 4))) & 255u;
        const float s = e4m3_value(sb);
        uint32_t w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          w[u] = pack_bf16x2(e2m1_times((cw >> (8 * u)) & 15u, s), e2m1_times((cw >> (8 * u + 4)) & 15u, s));
        *reinterpret_cast<uint4*>(sKV + (c >> 3) * kKBBytes + swz(et, c & 7)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    fence_proxy_async_smem();
    mbar_arrive(kv_full);
    // S^T of this tile: the per-head max over the rows, P^T in bf16, row sums
    const bool valid = tile_row(p, qi, tile, row) >= 0;
    bool ok = mbar_wait(s_full, 0, abort_flag, p.err);
    float x[HA];
    if (ok) {
      tc_fence_after();
      uint32_t v[16];
#pragma unroll
      for (int h0 = 0; h0 < HA; h0 += 16) {
        tmem_ld16(tmem + lane_off + S_COL + h0, v);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 16; ++h) x[h0 + h] = scaled_score(valid, p.scale, v[h]);
      }
    } else {
#pragma unroll
      for (int h = 0; h < HA; ++h) x[h] = -INFINITY;
    }
#pragma unroll
    for (int h = 0; h < HA; ++h) {
      const float mh = warp_max_f32(x[h]);
      if (lane == 0) sRed[ew * HA + h] = mh;
    }
    epi_bar();
    if (et < HA) sML[et] = fmaxf(fmaxf(sRed[et], sRed[HA + et]), fmaxf(sRed[2 * HA + et], sRed[3 * HA + et]));
    epi_bar();
    float lsum[HA];
    {
      // P^T[head][row]: row `row` is element row % 8 of chunk (row % 64) / 8 of
      // block row / 64 in head h's 128-byte line
      uint8_t* pb = sP + (row >> 6) * L::QKB;
      const int c = (row & 63) >> 3, e = row & 7;
#pragma unroll
      for (int h = 0; h < HA; h += 2) {
        const uint32_t pk = pack_bf16x2(p_value(x[h], sML[h]), p_value(x[h + 1], sML[h + 1]));
        lsum[h] = bf16_lo(pk);
        lsum[h + 1] = bf16_hi(pk);
        *reinterpret_cast<uint16_t*>(pb + swz(h, c) + 2 * e) = static_cast<uint16_t>(pk & 0xffffu);
        *reinterpret_cast<uint16_t*>(pb + swz(h + 1, c) + 2 * e) = static_cast<uint16_t>(pk >> 16);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(p_full);
    // l per head: a warp sum over the quarter's rows, then over the quarters
#pragma unroll
    for (int h = 0; h < HA; ++h) {
      float v = lsum[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) sRed[ew * HA + h] = v;
    }
    epi_bar();
    if (et < HA) sML[HA + et] = (sRed[et] + sRed[HA + et]) + (sRed[2 * HA + et] + sRed[3 * HA + et]);
    epi_bar();
    // O^T of this tile: dim `row`, every head
    float o[HA];
    {
      const uint64_t t0 = globaltimer_ns();
      bool landed;
      while (!(landed = mbar_try_wait(o_full, 0)) && globaltimer_ns() - t0 < 2000000000ull) {
      }
      if (!landed) {
        raise_dev_error(p.err, DEVERR_TIMEOUT);
        ok = false;
      }
      ok = ok && !*abort_flag;
      tc_fence_after();
      uint32_t v[16];
#pragma unroll
      for (int h0 = 0; h0 < HA; h0 += 16) {
        if (ok) {
          tmem_ld16(tmem + lane_off + O_COL + h0, v);
          tmem_wait_ld();
        }
#pragma unroll
        for (int h = 0; h < 16; ++h) o[h0 + h] = ok ? __uint_as_float(v[h]) : 0.0f;
      }
    }
    const int dim = row;
    if (p.T == 1) {
#pragma unroll
      for (int h = 0; h < HA; ++h) {
        const float inv = inv_sum(sML[HA + h]);
        p.out[(qi * HA + h) * DN + dim] = static_cast<uint16_t>(pack_bf16x2(__fmul_rn(o[h], inv), 0.0f) & 0xffffu);
      }
      if (p.lse && et < HA) p.lse[qi * HA + et] = lse_of(sML[et], sML[HA + et]);
    } else {
      // the tile's partial: O^T[dim][HA], then m[HA], l[HA]
      constexpr int kSlot = DN * HA + 2 * HA;
      float* slot = p.part + (ql * p.T + tile) * kSlot;
#pragma unroll
      for (int h = 0; h < HA; h += 4)
        __stcg(reinterpret_cast<float4*>(slot + dim * HA + h), make_float4(o[h], o[h + 1], o[h + 2], o[h + 3]));
      if (et < 2 * HA) __stcg(slot + DN * HA + et, sML[et]);
      __threadfence();
      epi_bar();
      if (et == 0) last_s = atomicAdd(p.counters + ql, 1u) == static_cast<unsigned>(p.T - 1);
      epi_bar();
      if (last_s) {
        // the query's last tile to finish combines the T partials in tile order
        __threadfence();
        const float* pq = p.part + ql * p.T * kSlot;
        if (et < HA) {
          float M = -INFINITY, Ls = 0.0f;
          for (int j = 0; j < p.T; ++j) {
            const float2 ab = combine_step(M, Ls, __ldcg(pq + j * kSlot + DN * HA + et),
                                           __ldcg(pq + j * kSlot + DN * HA + HA + et));
            sAB[(2 * j) * HA + et] = ab.x;
            sAB[(2 * j + 1) * HA + et] = ab.y;
          }
          sML[et] = M;
          sML[HA + et] = Ls;
        }
        epi_bar();
        float acc[HA];
#pragma unroll
        for (int h = 0; h < HA; ++h) acc[h] = 0.0f;
#pragma unroll 1
        for (int j = 0; j < p.T; ++j) {
          float vj[HA];
#pragma unroll
          for (int h = 0; h < HA; h += 4) {
            const float4 t4 = __ldcg(reinterpret_cast<const float4*>(pq + j * kSlot + dim * HA + h));
            vj[h] = t4.x; vj[h + 1] = t4.y; vj[h + 2] = t4.z; vj[h + 3] = t4.w;
          }
#pragma unroll
          for (int h = 0; h < HA; ++h)
            acc[h] = combine_acc(acc[h], vj[h], sAB[(2 * j) * HA + h], sAB[(2 * j + 1) * HA + h]);
        }
#pragma unroll
        for (int h = 0; h < HA; ++h) {
          const float inv = inv_sum(sML[HA + h]);
          p.out[(qi * HA + h) * DN + dim] = static_cast<uint16_t>(pack_bf16x2(__fmul_rn(acc[h], inv), 0.0f) & 0xffffu);
        }
        if (p.lse && et < HA) p.lse[qi * HA + et] = lse_of(sML[et], sML[HA + et]);
        if (et == 0) p.counters[ql] = 0u;               // ready for the next launch
      }
    }
  } else {
    __syncwarp();
  }

  // ---------------------------------------------------------------- teardown
  // every product has completed before TMEM is freed (bounded: 0.1 s)
  if (warp == 1 && lane == 0) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(o_full, 0) && globaltimer_ns() - t0 < 100000000ull) {
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 128);
}

int tiles_narrow(int k, bool win) { return (k + kRows - 1) / kRows + (win ? 1 : 0); }

size_t slot_bytes(int Ha, int T) { return static_cast<size_t>(T) * (DN * Ha + 2 * Ha) * 4; }
constexpr size_t kNarrowWsCap = size_t(64) << 20;   // partials of one launch

// queries per launch whose partials fit the cap (all of them when T == 1)
int64_t per_launch(int64_t n_queries, int Ha, int T) {
  if (T <= 1) return n_queries;
  return std::max<int64_t>(1, std::min<int64_t>(n_queries, static_cast<int64_t>(kNarrowWsCap / slot_bytes(Ha, T))));
}

template <int HA, bool FP4>
csa2_status run_narrow(const void* q, const csa2_kv& kv, const int32_t* topk, int B, int Q, int k,
                       float scale, void* out, float* lse, void* ws, size_t ws_bytes,
                       unsigned long long* sync_zeroed, cudaStream_t stream, const AttnRows& rows) {
  using Ly = Lay<HA>;
  static PerDevice<cudaError_t> opt_in;
  const cudaError_t attr = opt_in.get([] {
    const cudaError_t e = cudaFuncSetAttribute(attn_narrow_kernel<HA, FP4>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::BYTES);
    if (e != cudaSuccess) cudaGetLastError();
    return e;
  });
  if (attr != cudaSuccess) return fail(CSA2_ERR_CUDA, "sparse_attn_narrow: shared-memory opt-in failed");
  const bool win = rows.win != nullptr;
  const int64_t n_queries = static_cast<int64_t>(B) * Q;
  const int T = tiles_narrow(k, win);
  const int64_t per = per_launch(n_queries, HA, T);
  const size_t part_bytes = (static_cast<size_t>(per) * slot_bytes(HA, T) + 255) & ~size_t(255);
  // the counters: a layer group's (zeroed once, left zero by every launch), or the workspace's
  const bool own_counters = !(sync_zeroed && per <= 2 * kAttnMaxGrid);
  if (T > 1 && (!ws || ws_bytes < part_bytes + (own_counters ? static_cast<size_t>(per) * 4 : 0)))
    return fail(CSA2_ERR_INVALID, "sparse_attn: workspace too small");
  Params p;
  p.topk = topk;
  p.n_vis = rows.n_visible;
  p.win = static_cast<const uint16_t*>(rows.win);
  p.win_end = rows.win_end;
  p.win_rows = rows.win_rows;
  p.W = rows.W;
  p.T_sel = (k + kRows - 1) / kRows;
  p.kv = kv.data;
  p.kv_scales = kv.scales;
  p.q = static_cast<const uint16_t*>(q);
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.part = static_cast<float*>(ws);
  p.counters = own_counters ? reinterpret_cast<unsigned*>(static_cast<char*>(ws) + part_bytes)
                            : reinterpret_cast<unsigned*>(sync_zeroed);
  p.err = device_error_word();
  p.n = kv.n;
  p.Q = Q;
  p.k = k;
  p.T = T;
  p.scale = scale;
  for (int64_t q0 = 0; q0 < n_queries; q0 += per) {
    const int64_t nq = std::min<int64_t>(per, n_queries - q0);
    p.q_base = q0;
    if (T > 1 && own_counters) {
      begin_launch(stream);
      if (cudaMemsetAsync(p.counters, 0, static_cast<size_t>(nq) * 4, stream) != cudaSuccess)
        return check_launch("sparse_attn_narrow: clear counters");
      note_launch(LK_OTHER, 1, stream);
    }
    const int64_t grid = nq * T;
    if (grid > 0x7fffffffLL) return fail(CSA2_ERR_UNSUPPORTED, "sparse_attn_narrow: too many CTAs");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = Ly::BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0] = pdl_attribute();
    cfg.attrs = at;
    cfg.numAttrs = 1;
    begin_launch(stream);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, attn_narrow_kernel<HA, FP4>, p);
    note_launch(LK_ATTN, 1, stream);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(CSA2_ERR_CUDA, "sparse_attn_narrow: launch failed: %s", cudaGetErrorString(e));
    }
    CSA2_TRY(check_launch("sparse_attn_narrow"));
  }
  return CSA2_OK;
}

}  // namespace

bool sparse_attn_narrow_applies(int Ha, int D, int k, bool win) {
  if (getenv("CSA2_ATTN_SIMT")) return false;          // force the CUDA-core kernel
  if (D != DN || (Ha != 16 && Ha != 32 && Ha != 64) || k < 0) return false;
  const int T = tiles_narrow(k, win);
  return T >= 1 && T <= kMaxTilesN;
}

size_t sparse_attn_narrow_workspace(int B, int Q, int Ha, int k, bool win) {
  const int T = tiles_narrow(k, win);
  if (T <= 1) return 0;
  const int64_t per = per_launch(static_cast<int64_t>(B) * Q, Ha, T);
  return ((static_cast<size_t>(per) * slot_bytes(Ha, T) + 255) & ~size_t(255)) + static_cast<size_t>(per) * 4;
}

csa2_status launch_sparse_attn_narrow(const void* q, const csa2_kv& kv, const int32_t* topk, int B,
                                      int Q, int Ha, int k, float scale, void* out, float* lse,
                                      void* ws, size_t ws_bytes, unsigned long long* sync_zeroed,
                                      cudaStream_t stream, const AttnRows& rows) {
  const bool fp4 = kv.fmt == CSA2_KV_FP4;
  if (rows.win && rows.W > kRows) return CSA2_ERR_UNSUPPORTED;
#define CSA2_NARROW(HA_)                                                                       \
  if (Ha == HA_)                                                                               \
    return fp4 ? run_narrow<HA_, true>(q, kv, topk, B, Q, k, scale, out, lse, ws, ws_bytes,    \
                                       sync_zeroed, stream, rows)                              \
               : run_narrow<HA_, false>(q, kv, topk, B, Q, k, scale, out, lse, ws, ws_bytes,   \
                                        sync_zeroed, stream, rows);
  CSA2_NARROW(16) CSA2_NARROW(32) CSA2_NARROW(64)
#undef CSA2_NARROW
  return CSA2_ERR_UNSUPPORTED;
}

}  // namespace csa2
