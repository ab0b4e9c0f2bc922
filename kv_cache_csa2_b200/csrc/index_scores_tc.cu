// Lightning-indexer scores on the 5th-generation tensor cores (tcgen05).
// Source: "读完这篇，你就搞懂 DeepSeek v4 了", 闪电索引机制 (eq. 8): the score
// of entry j for a query is sum_h w_h * ReLU(q_h . k_j).
//
// The contraction is entries x (queries * heads) x d: one tile is 128 entries
// (MMA M, one TMEM lane each) by NQ queries of HP heads (MMA N = NQ*HP,
// padded heads are zero) by d (MMA K, 16 per instruction).  Per CTA
// (persistent, one per SM):
//   warp 0     producer: per tile, the 128 key rows into a shared-memory ring
//              (dense: one TMA tiled load per 64-column K-block; pool: a
//              cp.async gather of the rows the pool names by warps 0 and 6..12,
//              zero-filled for empty slots); per query group, the queries
//              (TMA when a group is one query of unpadded heads, else swizzled
//              by the lanes) and head weights into one of two slots;
//   warp 1     allocates TMEM; one lane issues the MMAs of a tile into one of
//              two accumulators and commits them to the ring slot and the
//              accumulator barriers;
//   warps 2-5  epilogue: TMEM -> registers, s = sum_h w_h * ReLU(acc_h) per
//              query, causal / pool mask, coalesced f32 stores.
// The epilogue of tile i overlaps the loads and MMAs of tiles i+1 and i+2.
// Every wait is bounded (2 s); a wait that runs out records CSA2_ERR_TIMEOUT
// and the CTA winds down, frees its TMEM and exits.
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

constexpr int kWarps = 6;
constexpr int kThreads = kWarps * 32;
// pool scoring gathers rows with cp.async from eight producer warps (0, 6..12)
constexpr int kPoolProducers = 8 * 32;
constexpr int kPoolThreads = 13 * 32;
constexpr int kPoolRows = 128 * 8 / kPoolProducers;   // rows per producer thread and tile
constexpr int kTileRows = 128;
constexpr int kKBlockBytes = kTileRows * 128;  // 128 rows x 64 bf16
constexpr int kLag = 4;                        // pool gathers: stages of copies kept in flight

struct Params {
  const uint16_t* q;
  const float* w;
  const uint16_t* k;
  const int32_t* n_visible;
  const int32_t* pool;
  float* scores;
  int* err;
  int Q, H, P;
  int64_t N;
  int relu;
  int q_tma;          // queries by TMA (one query per group, no padded heads)
  uint32_t* clear;    // words CTA 0 zeroes at start for the next kernel, or null
  int clear_words;
  int n_qgroups, n_tiles;
  int64_t n_units;
};

template <int DK, int NQ, int HP, bool POOL>
struct Cfg {
  static constexpr int KB = DK / 64;                       // K-blocks of 64 bf16
  static constexpr int NCOL = NQ * HP;                     // MMA N, TMEM columns per accumulator
  static constexpr int STAGES = (NQ * HP >= 256) ? 2 : (DK == 128 ? 5 : 8);
  static constexpr int TILE_A = KB * kKBlockBytes;         // bytes of one key tile
  static constexpr int QROWS = NQ * HP;
  static constexpr int QKB = QROWS * 128;                  // bytes of one q K-block
  static constexpr int QBYTES = KB * QKB;
  static constexpr int TMEM_COLS = (2 * NCOL <= 32) ? 32 : (2 * NCOL <= 64) ? 64
                                   : (2 * NCOL <= 128) ? 128 : (2 * NCOL <= 256) ? 256 : 512;
  // shared memory map (offsets from a 1024-aligned base)
  static constexpr int OFF_A = 0;
  static constexpr int OFF_Q = OFF_A + STAGES * TILE_A;
  static constexpr int OFF_W = OFF_Q + 2 * QBYTES;
  static constexpr int OFF_BAR = OFF_W + 2 * QROWS * 4;
  static constexpr int NBAR = 2 * STAGES + 8;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16 + 1024;       // + alignment slack
  static_assert(NCOL % 16 == 0 && NCOL <= 256, "MMA N");
  static_assert(QKB % 1024 == 0 && TILE_A % 1024 == 0, "swizzle atoms must stay 1 KiB aligned");
  static_assert(BYTES <= 232448, "shared memory");
  static_assert(!POOL || kLag < STAGES, "pool gathers keep fewer stages in flight than the ring holds");
};

template <int DK, int NQ, int HP, bool POOL>
__global__ void __launch_bounds__(POOL ? kPoolThreads : kThreads, 1)
    index_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                    const Params p) {
  using C = Cfg<DK, NQ, HP, POOL>;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + C::OFF_A;
  uint8_t* sQ = smem + C::OFF_Q;
  float* sW = reinterpret_cast<float*>(smem + C::OFF_W);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bar;
  uint64_t* empty = bar + S;
  uint64_t* tfull = bar + 2 * S;
  uint64_t* tempty = tfull + 2;
  uint64_t* qfull = tfull + 4;
  uint64_t* qempty = tfull + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t L = POOL ? p.P : p.N;
  pdl_release();                               // the selection kernel may start launching
  if (blockIdx.x == 0 && p.clear)              // the selection's counters (read after this kernel)
    for (int i = threadIdx.x; i < p.clear_words; i += blockDim.x) p.clear[i] = 0u;

  // balanced contiguous range of units for this CTA
  const int64_t u0 = p.n_units * blockIdx.x / gridDim.x;
  const int64_t u1 = p.n_units * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], POOL ? kPoolProducers : 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
      mbar_init(&qfull[i], 1);
      mbar_init(&qempty[i], 1 + 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
    if (!POOL) prefetch_tensor_map(&kmap);
    if (p.q_tma) prefetch_tensor_map(&qmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 || (POOL && warp >= 6)) {
    // ---------------------------------------------------------------- producer
    const int ptid = warp == 0 ? lane : 32 + (warp - 6) * 32 + lane;   // pool: producer thread index
    int64_t prev_bg = -1;
    int qi = -1;
    int64_t it = 0;
    bool ok = true;
    // pool gather: thread ptid copies 16-byte chunk c16 of rows rg + RS i
    // (i < kPoolRows) in every K-block, so eight consecutive lanes read one
    // 128-byte segment; the ids of the next unit are loaded during the current one
    constexpr int RS = kPoolProducers / 8;          // row stride between a thread's rows
    const int c16 = ptid & 7, rg = ptid >> 3;
    auto pool_ids = [&](int64_t v, int32_t (&ids)[kPoolRows]) {
      const int64_t bgv = v / p.n_tiles;
      const int64_t qrow = (bgv / p.n_qgroups) * p.Q + bgv % p.n_qgroups;
#pragma unroll
      for (int i = 0; i < kPoolRows; ++i) {
        const int64_t slot_i = (v % p.n_tiles) * kTileRows + rg + RS * i;
        ids[i] = slot_i < L ? p.pool[qrow * p.P + slot_i] : -1;
      }
    };
    int32_t next_ids[kPoolRows];
    if (POOL && u0 < u1) pool_ids(u0, next_ids);
    for (int64_t u = u0; u < u1 && ok; ++u, ++it) {
      const int64_t bg = u / p.n_tiles;
      const int t = static_cast<int>(u % p.n_tiles);
      const int b = static_cast<int>(bg / p.n_qgroups);
      const int g = static_cast<int>(bg % p.n_qgroups);
      if (bg != prev_bg && warp != 0) {
        ++qi;
        prev_bg = bg;
      } else if (bg != prev_bg) {
        ++qi;
        const int slot = qi & 1;
        if (qi >= 2 && !mbar_wait(&qempty[slot], ((qi >> 1) - 1) & 1, abort_flag, p.err)) { ok = false; break; }
        uint8_t* qs = sQ + slot * C::QBYTES;
        if (p.q_tma) {
          // head weights by the lanes, then the query's HP x DK heads by TMA
          for (int r = lane; r < C::QROWS; r += 32)
            sW[slot * C::QROWS + r] = p.w[(static_cast<int64_t>(b) * p.Q + g) * p.H + r];
          __syncwarp();
          if (lane == 0) {
            mbar_arrive_expect_tx(&qfull[slot], C::QBYTES);
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb)
              tma_load_2d(qs + kb * C::QKB, &qmap, &qfull[slot], kb * 64,
                          static_cast<int32_t>((static_cast<int64_t>(b) * p.Q + g) * p.H));
          }
          prev_bg = bg;
        } else {
        // rows r = qq * HP + h; 16-byte chunks c = kb * 8 + cc; 8 loads per
        // lane in flight before any is stored
        constexpr int NCH = C::QROWS * (DK / 8);
        for (int i0 = lane; i0 < NCH; i0 += 32 * 8) {
          uint4 v[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = i0 + 32 * u;
            const int r = i / (DK / 8), c = i % (DK / 8);
            const int qq = r / HP, h = r % HP;
            const int query = g * NQ + qq;
            v[u] = make_uint4(0, 0, 0, 0);
            if (i < NCH && h < p.H && query < p.Q)
              v[u] = __ldg(reinterpret_cast<const uint4*>(p.q + ((static_cast<int64_t>(b) * p.Q + query) * p.H + h) * DK + c * 8));
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = i0 + 32 * u;
            const int r = i / (DK / 8), c = i % (DK / 8);
            if (i < NCH) *reinterpret_cast<uint4*>(qs + (c / 8) * C::QKB + sw128_offset(r, c % 8)) = v[u];
          }
        }
        for (int r = lane; r < C::QROWS; r += 32) {
          const int qq = r / HP, h = r % HP;
          const int query = g * NQ + qq;
          sW[slot * C::QROWS + r] =
              (h < p.H && query < p.Q) ? p.w[(static_cast<int64_t>(b) * p.Q + query) * p.H + h] : 0.0f;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&qfull[slot]);
        prev_bg = bg;
        }
      }
      const int stage = static_cast<int>(it % S);
      if (it >= S && !mbar_wait(&empty[stage], ((it / S) - 1) & 1, abort_flag, p.err)) { ok = false; break; }
      uint8_t* dst = sA + stage * C::TILE_A;
      if (!POOL) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[stage], C::TILE_A);
          const int32_t row = static_cast<int32_t>(static_cast<int64_t>(b) * p.N + static_cast<int64_t>(t) * kTileRows);
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb) tma_load_2d(dst + kb * kKBlockBytes, &kmap, &full[stage], kb * 64, row);
        }
      } else {
        {
          int32_t ids[kPoolRows];
#pragma unroll
          for (int i = 0; i < kPoolRows; ++i) ids[i] = next_ids[i];
          if (u + 1 < u1) pool_ids(u + 1, next_ids);             // in flight during this unit
#pragma unroll
          for (int i = 0; i < kPoolRows; ++i) {
            const bool valid = ids[i] >= 0 && ids[i] < p.N;
            const uint16_t* src = p.k + (static_cast<int64_t>(b) * p.N + (valid ? ids[i] : 0)) * DK + c16 * 8;
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb)
              cp_async_16(dst + kb * kKBlockBytes + sw128_offset(rg + RS * i, c16), src + kb * 64, valid ? 16u : 0u);
          }
        }
        cp_async_commit();
        // keep kLag stages of copies in flight; stage it-kLag is complete now
        if (it >= kLag) {
          cp_async_wait<kLag>();
          fence_proxy_async_smem();
          mbar_arrive(&full[(it - kLag) % S]);
        }
      }
    }
    if (POOL) {
      cp_async_wait<0>();
      fence_proxy_async_smem();
      for (int64_t j = (it > kLag ? it - kLag : 0); j < it; ++j) mbar_arrive(&full[j % S]);
    }
    if (!ok && !POOL && lane == 0) {
      // let TMA loads still in flight land before the CTA's shared memory goes
      // away (bounded: at most 0.1 s per stage)
      const int64_t n_issued = it;
      for (int64_t j = (n_issued > S ? n_issued - S : 0); j < n_issued; ++j) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&full[j % S], (j / S) & 1) && globaltimer_ns() - t0 < 100000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, C::NCOL, false, false);
      int64_t prev_bg = -1;
      int qi = -1;
      int64_t it = 0;
      for (int64_t u = u0; u < u1; ++u, ++it) {
        const int64_t bg = u / p.n_tiles;
        if (bg != prev_bg) {
          if (qi >= 0) mma_commit(&qempty[qi & 1]);
          ++qi;
          if (!mbar_wait(&qfull[qi & 1], (qi >> 1) & 1, abort_flag, p.err)) break;
          prev_bg = bg;
        }
        const int stage = static_cast<int>(it % S);
        const int acc = static_cast<int>(it & 1);
        if (!mbar_wait(&full[stage], (it / S) & 1, abort_flag, p.err)) break;
        if (it >= 2 && !mbar_wait(&tempty[acc], ((it >> 1) - 1) & 1, abort_flag, p.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * C::NCOL;
        const uint32_t a0 = smem_u32(sA + stage * C::TILE_A);
        const uint32_t b0 = smem_u32(sQ + (qi & 1) * C::QBYTES);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = desc_kmajor_sw128(a0 + kb * kKBlockBytes + kk * 32);
            const uint64_t bd = desc_kmajor_sw128(b0 + kb * C::QKB + kk * 32);
            mma_bf16(d_tmem, ad, bd, idesc, (kb | kk) != 0);
          }
        }
        mma_commit(&empty[stage]);
        mma_commit(&tfull[acc]);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;                 // TMEM lanes this warp may access
    const int row = quad * 32 + lane;
    int64_t prev_bg = -1;
    int qi = -1;
    int64_t it = 0;
    for (int64_t u = u0; u < u1; ++u, ++it) {
      const int64_t bg = u / p.n_tiles;
      const int t = static_cast<int>(u % p.n_tiles);
      const int b = static_cast<int>(bg / p.n_qgroups);
      const int g = static_cast<int>(bg % p.n_qgroups);
      if (bg != prev_bg) {
        if (qi >= 0 && lane == 0) mbar_arrive(&qempty[qi & 1]);
        ++qi;
        if (!mbar_wait(&qfull[qi & 1], (qi >> 1) & 1, abort_flag, p.err)) break;
        prev_bg = bg;
      }
      const int acc = static_cast<int>(it & 1);
      const int64_t e = static_cast<int64_t>(t) * kTileRows + row;   // entry or pool slot
      // pool: this row's entry id, loaded while the products are computed
      const int64_t pid = POOL && e < L ? p.pool[(static_cast<int64_t>(b) * p.Q + g) * p.P + e] : -1;
      if (!mbar_wait(&tfull[acc], (it >> 1) & 1, abort_flag, p.err)) break;
      tc_fence_after();
      const float* w = sW + (qi & 1) * C::QROWS;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * C::NCOL;
      float s[NQ];
#pragma unroll
      for (int qq = 0; qq < NQ; ++qq) {
        float a = 0.0f;
#pragma unroll
        for (int h0 = 0; h0 < HP; h0 += 16) {
          uint32_t v[16];
          tmem_ld16(taddr + qq * HP + h0, v);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            float x = __uint_as_float(v[h]);
            if (p.relu) x = fmaxf(x, 0.0f);
            a = fmaf(w[qq * HP + h0 + h], x, a);
          }
        }
        s[qq] = a;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (e < L) {
        bool valid = true;
        if (POOL) {
          if (pid >= p.N || pid < -1) raise_dev_error(p.err, DEVERR_BOUNDS);
          valid = pid >= 0 && pid < p.N;
        }
#pragma unroll
        for (int qq = 0; qq < NQ; ++qq) {
          const int query = g * NQ + qq;
          if (query >= p.Q) break;
          const int64_t qr = static_cast<int64_t>(b) * p.Q + query;
          bool vis = valid;
          if (!POOL && p.n_visible) vis = e < p.n_visible[qr];
          p.scores[qr * L + e] = vis ? s[qq] : -INFINITY;
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

template <int DK, int NQ, int HP, bool POOL>
csa2_status run_tc(const void* q, const float* w, const void* k, int B, int Q, int H, int64_t N,
                   const int32_t* n_visible, const int32_t* pool, int P, csa2_index_act act,
                   float* scores, cudaStream_t stream, ClearOnLaunch* clear) {
  using C = Cfg<DK, NQ, HP, POOL>;
  CUtensorMap map;
  memset(&map, 0, sizeof(map));
  if (!POOL) {
    CSA2_TRY(make_tensor_map_bf16_2d(&map, k, static_cast<uint64_t>(B) * N, DK, DK * 2, 64, kTileRows));
  }
  CUtensorMap qmap;
  memset(&qmap, 0, sizeof(qmap));
  const bool q_tma = NQ == 1 && H == HP && (reinterpret_cast<uintptr_t>(q) & 15u) == 0;
  if (q_tma)
    CSA2_TRY(make_tensor_map_bf16_2d(&qmap, q, static_cast<uint64_t>(B) * Q * H, DK, DK * 2, 64, HP));
  Params p;
  p.q = static_cast<const uint16_t*>(q);
  p.w = w;
  p.k = static_cast<const uint16_t*>(k);
  p.n_visible = n_visible;
  p.pool = pool;
  p.scores = scores;
  p.err = device_error_word();
  p.Q = Q;
  p.H = H;
  p.P = P;
  p.N = N;
  p.relu = act == CSA2_ACT_RELU ? 1 : 0;
  p.q_tma = q_tma ? 1 : 0;
  p.clear = clear ? clear->ptr : nullptr;
  p.clear_words = clear ? clear->words : 0;
  p.n_qgroups = (Q + NQ - 1) / NQ;
  const int64_t L = POOL ? P : N;
  p.n_tiles = static_cast<int>((L + kTileRows - 1) / kTileRows);
  p.n_units = static_cast<int64_t>(B) * p.n_qgroups * p.n_tiles;
  auto kern = index_tc_kernel<DK, NQ, HP, POOL>;
  static PerDevice<cudaError_t> opt_in;
  const cudaError_t attr_err = opt_in.get([] {
    const cudaError_t e = cudaFuncSetAttribute(index_tc_kernel<DK, NQ, HP, POOL>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, C::BYTES);
    if (e != cudaSuccess) cudaGetLastError();
    return e;
  });
  if (attr_err != cudaSuccess) return fail(CSA2_ERR_CUDA, "index_scores_tc: smem opt-in failed");
  const int64_t grid = std::min<int64_t>(sm_count(), p.n_units);
  begin_launch(stream);
  kern<<<static_cast<unsigned>(grid), POOL ? kPoolThreads : kThreads, C::BYTES, stream>>>(map, qmap, p);
  note_launch(POOL ? LK_INDEX_POOL : LK_INDEX, 1, stream);
  const csa2_status st = check_launch("index_scores_tc");
  if (st == CSA2_OK && clear) clear->done = true;
  return st;
}

}  // namespace

csa2_status launch_index_scores_tc(const void* q, const float* w, const void* k, int B, int Q,
                                   int H, int d, int64_t N, const int32_t* n_visible,
                                   const int32_t* pool, int P, csa2_index_act act, float* scores,
                                   cudaStream_t stream, ClearOnLaunch* clear) {
  if (getenv("CSA2_INDEX_SIMT")) return CSA2_ERR_UNSUPPORTED;   // force the CUDA-core kernel
  if ((d != 64 && d != 128) || H > 64) return CSA2_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * N > 0x7fffffffLL) return CSA2_ERR_UNSUPPORTED;
  const bool small = H <= 16;
  if (pool) {
    if (d == 64)
      return small ? run_tc<64, 1, 16, true>(q, w, k, B, Q, H, N, n_visible, pool, P, act, scores, stream, clear)
                   : run_tc<64, 1, 64, true>(q, w, k, B, Q, H, N, n_visible, pool, P, act, scores, stream, clear);
    return small ? run_tc<128, 1, 16, true>(q, w, k, B, Q, H, N, n_visible, pool, P, act, scores, stream, clear)
                 : run_tc<128, 1, 64, true>(q, w, k, B, Q, H, N, n_visible, pool, P, act, scores, stream, clear);
  }
  const bool many = Q >= 4;
  if (d == 64) {
    if (small)
      return many ? run_tc<64, 16, 16, false>(q, w, k, B, Q, H, N, n_visible, nullptr, 0, act, scores, stream, clear)
                  : run_tc<64, 1, 16, false>(q, w, k, B, Q, H, N, n_visible, nullptr, 0, act, scores, stream, clear);
    return many ? run_tc<64, 4, 64, false>(q, w, k, B, Q, H, N, n_visible, nullptr, 0, act, scores, stream, clear)
                : run_tc<64, 1, 64, false>(q, w, k, B, Q, H, N, n_visible, nullptr, 0, act, scores, stream, clear);
  }
  if (small)
    return many ? run_tc<128, 16, 16, false>(q, w, k, B, Q, H, N, n_visible, nullptr, 0, act, scores, stream, clear)
                : run_tc<128, 1, 16, false>(q, w, k, B, Q, H, N, n_visible, nullptr, 0, act, scores, stream, clear);
  return many ? run_tc<128, 4, 64, false>(q, w, k, B, Q, H, N, n_visible, nullptr, 0, act, scores, stream, clear)
              : run_tc<128, 1, 64, false>(q, w, k, B, Q, H, N, n_visible, nullptr, 0, act, scores, stream, clear);
}

}  // namespace csa2
