// Shared-KV sparse attention for large batches: one CTA per query, the
// query's tiles in sequence.  Source: "读完这篇，你就搞懂 DeepSeek v4 了",
// 注意力计算 (eq. 9) and 批无关性 (batch invariance).
//
// attn_tc.cu spreads a query's T tiles of 128 rows over T CTAs and combines
// their partial results through L2: the right shape when a few queries must
// fill the GPU (decode), but with many queries (prefill) every wave of the
// grid pays the whole latency chain and the exchange moves as many bytes as
// the gather.  Here a persistent CTA takes whole queries (c, c + grid, ...)
// and runs their tiles one after another, with no exchange: tile t's partial
// O_t stays in TMEM and joins the query's f32 accumulator, also in TMEM, at
// once.  Each
// tile's arithmetic, and the tile-order combine, are those of attn_tc.cu,
// instruction for instruction (attn_common.cuh): a query's output and lse
// are the same bits whichever kernel runs it.
//
// Per CTA (10 warps):
//   warp 0     TMA load of each query's 64 x 512 heads (the next query's as
//              soon as the last product of the current one has read q);
//   warp 1     TMEM allocation and MMA issue, per tile:
//                S^T[row, head]  = KV[row, :] . q[head, :]      (M=128, N=64, K=512)
//                O^T[dim, head]  = KV[row, dim] * P[row, head]  (M=128 x4, N=64, K=128)
//   warps 2-9  two warps per TMEM lane quarter, each with 32 of the 64 heads:
//              the gather of the next tile's rows (16-byte cp.async copies into
//              the 128-byte-swizzled layout, K-blocks 2mc and 2mc+1 as soon as
//              the current tile's product chunk mc no longer reads them), the
//              softmax of the tile (the decode kernel's per-head max, bf16 P
//              and row sums), the running combine, and the output.
// Every wait is bounded (mbarriers 2 s); a wait that gives up records
// CSA2_ERR_TIMEOUT and the CTA winds down, letting its copies land and its
// products finish before it frees TMEM.
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
using namespace attn;

constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = (2 + kEpiWarps) * 32;

constexpr int OFF_KV = 0;                              // 128 KiB: KV tile
constexpr int OFF_Q = OFF_KV + kKB * kKBBytes;         // 64 KiB: q
constexpr int OFF_P = OFF_Q + kKB * HA * 128;          // 16 KiB: P tile
constexpr int OFF_RED = OFF_P + kRows * 128;           // [4 quarters][HA] f32
constexpr int OFF_ML = OFF_RED + 4 * HA * 4;           // m_t[HA]
constexpr int OFF_AB = OFF_ML + HA * 4;                // a_t[HA], b_t[HA]
constexpr int OFF_ML2 = OFF_AB + 2 * HA * 4;           // the query's M[HA], L[HA]
constexpr int OFF_BAR = OFF_ML2 + 2 * HA * 4;
constexpr int NBAR = 21;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
static_assert(OFF_RED % 16 == 0 && OFF_BAR % 8 == 0, "alignment");
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
  int* err;
  int64_t n, n_queries;
  int Q, k, T;
  float scale;
};

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
    attn_seq_kernel(const __grid_constant__ CUtensorMap qmap, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKV = smem + OFF_KV;
  uint8_t* sP = smem + OFF_P;
  uint8_t* sQ = smem + OFF_Q;
  float* sRed = reinterpret_cast<float*>(smem + OFF_RED);
  float* sML = reinterpret_cast<float*>(smem + OFF_ML);
  float* sAB = reinterpret_cast<float*>(smem + OFF_AB);
  float* sML2 = reinterpret_cast<float*>(smem + OFF_ML2);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bar + 0;
  uint64_t* q_empty = bar + 1;                 // the last product of a query has read q
  uint64_t* s_full = bar + 2;
  uint64_t* p_full = bar + 3;
  uint64_t* o_full = bar + 4;                  // [4]: one per 128-dim chunk of O^T
  uint64_t* o_empty = bar + 8;                 // [4]: chunk mc read by every epilogue warp
  uint64_t* kv_full = bar + 12;                // [8]: one per 64-column block of the tile
  uint64_t* mma_fin = bar + 20;                // every MMA of this CTA has completed (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_mine = p.n_queries > blockIdx.x ? (p.n_queries - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int64_t n_units = n_mine * p.T;        // (query, tile) units of this CTA, in order
  auto unit_query = [&](int64_t u) { return blockIdx.x + (u / p.T) * gridDim.x; };
  // TMEM columns: O_t^T chunk mc at [64 mc, 64 mc + 64); S^T shares chunk 3's
  // columns (read before chunk 3 is written; the next S waits until chunk 3
  // was read); the accumulator's chunk mc at [256 + 64 mc, ...)
  constexpr uint32_t O_COL = 0, S_COL = 192, ACC_COL = 256;

  // gather mapping (warps 2-9): thread et copies 16-byte chunk c16 of rows
  // grow0 + 32 i (i < 4) in each 64-column block
  const int et = (warp - 2) * 32 + lane;
  const int c16 = et & 7, grow0 = et >> 3;
  const uint32_t swz = static_cast<uint32_t>((c16 ^ (grow0 & 7)) << 4);   // (grow0 + 32 i) & 7 == grow0 & 7
  int32_t ids[4];                              // rows of the unit being gathered
  auto load_ids = [&](int64_t u) {
    const int64_t qi = unit_query(u);
    const int tile = static_cast<int>(u % p.T);
#pragma unroll
    for (int i = 0; i < 4; ++i) ids[i] = tile_row(p, qi, tile, grow0 + 32 * i);
  };
  // copies of K-blocks kb0, kb0 + 1 of unit u, one commit group
  auto issue_pair = [&](int64_t u, int kb0) {
    const int64_t qi = unit_query(u);
    const bool win_tile = static_cast<int>(u % p.T) >= p.T_sel;
    const uint16_t* base = (win_tile ? p.win + (qi / p.Q) * p.win_rows * DV
                                     : p.kv + (qi / p.Q) * p.n * DV) + c16 * 8;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      const int kb = kb0 + kk;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int id = ids[i];
        cp_async_16(sKV + kb * kKBBytes + (grow0 + 32 * i) * 128 + swz,
                    base + static_cast<int64_t>(id >= 0 ? id : 0) * DV + kb * 64, id >= 0 ? 16u : 0u);
      }
    }
    cp_async_commit();
  };
  // each 64-column block is published once this thread's copies into it landed
  auto publish = [&]() {
#define CSA2_PUBLISH(N, KB)                 \
  cp_async_wait<N>();                       \
  fence_proxy_async_smem();                 \
  mbar_arrive(&kv_full[KB]);                \
  mbar_arrive(&kv_full[KB + 1]);
    CSA2_PUBLISH(3, 0) CSA2_PUBLISH(2, 2) CSA2_PUBLISH(1, 4) CSA2_PUBLISH(0, 6)
#undef CSA2_PUBLISH
  };

  pdl_wait();                                  // the selection comes from the kernel before
  if (warp >= 2 && n_units > 0) {              // the first tile's rows, before the set-up
    load_ids(0);
    for (int kb = 0; kb < kKB; kb += 2) issue_pair(0, kb);
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, kEpiWarps);
    for (int mc = 0; mc < 4; ++mc) {
      mbar_init(&o_full[mc], 1);
      mbar_init(&o_empty[mc], kEpiWarps);
    }
    for (int kb = 0; kb < kKB; ++kb) mbar_init(&kv_full[kb], kEpiThreads);
    mbar_init(mma_fin, 1);
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
      for (int64_t j = 0; j < n_mine; ++j) {
        if (j > 0 && !mbar_wait(q_empty, static_cast<uint32_t>((j - 1) & 1), abort_flag, p.err)) break;
        const int64_t qi = blockIdx.x + j * gridDim.x;
        mbar_arrive_expect_tx(q_full, HA * DV * 2);
#pragma unroll
        for (int kb = 0; kb < kKB; ++kb)
          tma_load_2d(sQ + kb * HA * 128, &qmap, q_full, kb * 64, static_cast<int32_t>(qi * HA));
        issued = j + 1;
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
      for (int64_t u = 0; u < n_units; ++u) {
        const uint32_t par = static_cast<uint32_t>(u & 1);
        const int tile = static_cast<int>(u % p.T);
        bool ok = true;
        if (tile == 0) ok = mbar_wait(q_full, static_cast<uint32_t>((u / p.T) & 1), abort_flag, p.err);
        // S^T lands on chunk 3's columns: the previous tile's chunk 3 was read
        if (ok && u > 0) ok = mbar_wait(&o_empty[3], static_cast<uint32_t>((u - 1) & 1), abort_flag, p.err);
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
        if (tile == p.T - 1) mma_commit(q_empty);        // q may be replaced
        if (!mbar_wait(p_full, par, abort_flag, p.err)) break;
        tc_fence_after();
#pragma unroll 1
        for (int mc = 0; mc < 4 && ok; ++mc) {
          // the epilogue has read the previous tile's chunk mc
          if (u > 0) ok = mbar_wait(&o_empty[mc], static_cast<uint32_t>((u - 1) & 1), abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16(tmem + O_COL + 64 * mc,
                     desc_mnmajor_sw128(kv0 + 2 * mc * kKBBytes + kk * 2048, kKBBytes, 1024),
                     desc_mnmajor_sw128(p0 + kk * 2048, 8192, 1024), idesc_o, kk != 0);
          mma_commit(&o_full[mc]);
        }
        if (!ok) break;
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
    // ------------------------------------------------------------ gather, softmax, combine, output
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;                  // heads [32 half, 32 half + 32)
    const int slot = (quad + 2) & 3;                   // this quarter's slot in sRed (as in attn_tc)
    const int row = quad * 32 + lane;                  // TMEM lane = tile row
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int h0 = 32 * half;
    float Mh = -INFINITY, Lh = 0.0f;                   // running max and sum of head et (et < HA)
    bool ok = true;
    if (n_units > 0) publish();
    for (int64_t u = 0; u < n_units; ++u) {
      const int64_t qi = unit_query(u);
      const int tile = static_cast<int>(u % p.T);
      const uint32_t par = static_cast<uint32_t>(u & 1);
      const bool next = u + 1 < n_units;
      const bool valid = tile_row(p, qi, tile, row) >= 0;
      if (next) load_ids(u + 1);                       // the next tile's rows, ahead of their copies
      ok = ok && mbar_wait(s_full, par, abort_flag, p.err);
      float x[32];
      if (ok) {
        tc_fence_after();
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + S_COL + h0, v);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 32; ++h) x[h] = scaled_score(valid, p.scale, v[h]);
      } else {
#pragma unroll
        for (int h = 0; h < 32; ++h) x[h] = -INFINITY;
      }
      // the tile's per-head max m_t over its rows
#pragma unroll
      for (int h = 0; h < 32; ++h) {
        const float mh = warp_max_f32(x[h]);
        if (lane == 0) sRed[slot * HA + h0 + h] = mh;
      }
      epi_bar();
      if (et < HA)
        sML[et] = fmaxf(fmaxf(sRed[et], sRed[HA + et]), fmaxf(sRed[2 * HA + et], sRed[3 * HA + et]));
      epi_bar();
      // P = exp(x - m_t) in bf16, and its row sums
      float lsum[32];
      {
        const uint32_t ml0 = smem_u32(sML) + h0 * 4, p0 = smem_u32(sP);
        uint32_t packed[16];
#pragma unroll
        for (int h4 = 0; h4 < 8; ++h4) {
          const float4 m4 = lds_v4f(ml0 + 16 * h4);
          const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
          for (int w2 = 0; w2 < 2; ++w2) {
            const int h = 4 * h4 + 2 * w2;
            const uint32_t pk = pack_bf16x2(p_value(x[h], mm[2 * w2]), p_value(x[h + 1], mm[2 * w2 + 1]));
            packed[2 * h4 + w2] = pk;
            lsum[h] = bf16_lo(pk);
            lsum[h + 1] = bf16_hi(pk);
          }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
          sts_v4u(p0 + sw128_offset(row, 4 * half + c), packed[4 * c], packed[4 * c + 1], packed[4 * c + 2],
                  packed[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      warp_transpose_reduce<32, false>(lsum, lane);    // lane holds head h0 + lane
      sRed[slot * HA + h0 + lane] = lsum[0];
      epi_bar();
      if (et < HA) {
        const float lt = quad_sum(sRed[et], sRed[HA + et], sRed[2 * HA + et], sRed[3 * HA + et]);
        const float2 ab = combine_step(Mh, Lh, sML[et], lt);
        sAB[et] = ab.x;
        sAB[HA + et] = ab.y;
        if (tile == p.T - 1) {
          sML2[et] = Mh;
          sML2[HA + et] = Lh;
        }
      }
      epi_bar();
      // O_t chunk by chunk into the accumulator; the K-blocks a chunk's
      // product read take the next tile's rows at once
      const uint32_t ab0 = smem_u32(sAB) + h0 * 4;
      const bool first = tile == 0, last = tile == p.T - 1;
      const uint32_t ml2 = smem_u32(sML2);
#pragma unroll 1
      for (int mc = 0; mc < 4; ++mc) {
        ok = ok && mbar_wait(&o_full[mc], par, abort_flag, p.err);
        if (next) issue_pair(u + 1, 2 * mc);
        uint32_t o[32], c[32];
        if (ok) {
          tc_fence_after();
          tmem_ld32(tmem + lane_off + O_COL + 64 * mc + h0, o);
          if (!first) tmem_ld32(tmem + lane_off + ACC_COL + 64 * mc + h0, c);
          tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_empty[mc]);
        if (!ok) continue;
#pragma unroll
        for (int h4 = 0; h4 < 8; ++h4) {
          const float4 a4 = lds_v4f(ab0 + 16 * h4), b4 = lds_v4f(ab0 + HA * 4 + 16 * h4);
          const float av[4] = {a4.x, a4.y, a4.z, a4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int h = 4 * h4 + i;
            const float prev = first ? 0.0f : __uint_as_float(c[h]);
            c[h] = __float_as_uint(combine_acc(prev, __uint_as_float(o[h]), av[i], bv[i]));
          }
        }
        if (!last) {
          tmem_st32(tmem + lane_off + ACC_COL + 64 * mc + h0, c);
        } else {
          // the query's output: dim mc * 128 + row of heads h0 .. h0 + 31
#pragma unroll
          for (int h = 0; h < 32; ++h) {
            const float inv = inv_sum(lds_f32(ml2 + (HA + h0 + h) * 4));
            const uint32_t pk = pack_bf16x2(__fmul_rn(__uint_as_float(c[h]), inv), 0.0f);
            p.out[(qi * HA + h0 + h) * DV + mc * 128 + row] = static_cast<uint16_t>(pk & 0xffffu);
          }
        }
      }
      tmem_wait_st();                                  // the accumulator is in place for the next tile
      if (next) publish();
      if (last) {
        if (p.lse && et < HA) p.lse[qi * HA + et] = lse_of(Mh, Lh);
        Mh = -INFINITY;
        Lh = 0.0f;
      }
    }
    cp_async_wait<0>();
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// the shape attn_tc.cu uses for k selected slots (and a window tile)
int tiles_for(int k, bool win) { return (k + kRows - 1) / kRows + (win ? 1 : 0); }

}  // namespace

bool sparse_attn_seq_applies(int64_t n_queries, int k, bool win) {
  if (const char* e = getenv("CSA2_ATTN_SEQ")) return atoi(e) != 0 && n_queries > 0;
  const int T = tiles_for(k, win);
  if (T < 1 || T > kMaxTiles) return false;
  // measured on B200 (64 heads x 512, k = 2048): the split kernel runs
  // floor(SMs / T) queries per wave of about 24 us; one query per CTA takes
  // about 10 us per tile (the tile's rows are gathered while nothing else of
  // the CTA's runs)
  const int64_t per_wave = std::max(1, sm_count() / T);
  const int64_t waves_split = (n_queries + per_wave - 1) / per_wave;
  const int64_t rounds_seq = (n_queries + sm_count() - 1) / sm_count();
  return rounds_seq * T * 10 < waves_split * 24;
}

csa2_status launch_sparse_attn_seq(const void* q, const csa2_kv& kv, const int32_t* topk, int B,
                                   int Q, int k, float scale, void* out, float* lse,
                                   cudaStream_t stream, const AttnRows& rows) {
  const bool win = rows.win != nullptr;
  const int64_t n_queries = static_cast<int64_t>(B) * Q;
  const int T = tiles_for(k, win);
  if (T < 1 || T > kMaxTiles || n_queries * HA > 0x7fffffffLL) return CSA2_ERR_UNSUPPORTED;
  static PerDevice<cudaError_t> opt_in;
  const cudaError_t attr = opt_in.get([] {
    const cudaError_t e = cudaFuncSetAttribute(attn_seq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) cudaGetLastError();
    return e;
  });
  if (attr != cudaSuccess) return fail(CSA2_ERR_CUDA, "sparse_attn_seq: shared-memory opt-in failed");
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
  p.T_sel = (k + kRows - 1) / kRows;
  p.kv = static_cast<const uint16_t*>(kv.data);
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.err = device_error_word();
  p.n = kv.n;
  p.n_queries = n_queries;
  p.Q = Q;
  p.k = k;
  p.T = T;
  p.scale = scale;
  const int64_t grid = std::min<int64_t>(n_queries, sm_count());
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0] = pdl_attribute();
  cfg.attrs = at;
  cfg.numAttrs = 1;
  begin_launch(stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, attn_seq_kernel, qmap, p);
  note_launch(LK_ATTN, 1, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(CSA2_ERR_CUDA, "sparse_attn_seq: launch failed: %s", cudaGetErrorString(e));
  }
  return check_launch("sparse_attn_seq");
}

}  // namespace csa2
