// A Full layer's lightning indexer fused with a streaming top-k, for many
// queries (prefill): the scores never leave the SM.  Sources:
// "读完这篇，你就搞懂 DeepSeek v4 了", 闪电索引机制 (eq. 8: s_j = sum_h w_h *
// ReLU(q_h . k_j); keep the k best entries) -- the order is score
// descending, ties to the lower entry index, -inf / NaN never chosen.
//
// Each CTA (persistent, one per SM) owns whole groups of NQ = 4 queries and
// runs every key tile of 128 entries for them in entry order: the scores are
// the bf16 tensor-core contraction of index_scores_tc.cu (M = 128 entries,
// N = 4 queries x HP heads, K = d; producer / MMA / epilogue warps).  The
// epilogue keeps, per query, a candidate list in shared memory (order-
// preserving 32-bit score keys and entry indices) and a threshold tau: an
// entry is appended when its key is above tau, in entry order (one ballot and
// one barrier per tile place a tile's entries after the earlier ones).  When
// a list could overflow, it is compacted to its k best -- a radix select of
// the k-th key T (four 8-bit digits) and a stable compaction that keeps the
// keys above T and the first keys equal to T -- and tau becomes T.  That is
// exact: every entry not kept is outranked by k kept ones, and a later entry
// with key T has a higher index than every kept one, so it can only enter
// with a key above T.  After the group's last tile the lists are compacted to
// k once more and written (ascending entry indices, -1 padded).
// Every wait is bounded; a wait that runs out records CSA2_ERR_TIMEOUT and
// the CTA winds down, letting its copies land and its MMAs finish.
#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "launchers.h"
#include "sm100.cuh"

namespace csa2 {
namespace {
using namespace sm100;

constexpr int kTileRows = 128;
constexpr int kKBlockBytes = kTileRows * 128;  // 128 rows x 64 bf16
constexpr int kEpiWarps = 8;                   // epilogue: two warps per TMEM lane quarter
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = (2 + kEpiWarps) * 32;
constexpr int NQ = 4;                          // queries per group
constexpr int kCap = 3000;                     // candidates per query
constexpr int QPW = NQ / 2;                    // queries per epilogue warp
constexpr int kSeg = (kCap + kEpiThreads - 1) / kEpiThreads;   // list entries per epilogue thread in a compaction

struct Params {
  const uint16_t* q;         // [B, Q, H, d]
  const float* w;            // [B, Q, H]
  const int32_t* n_visible;  // [B, Q] or null
  int32_t* topk;             // [B, Q, k]
  int* err;
  int Q, H, k;
  int64_t N;
  int relu;
  int n_qgroups, n_tiles;
  int64_t n_groups;          // B * n_qgroups
};

template <int DK, int HP>
struct Cfg {
  static constexpr int KB = DK / 64;
  static constexpr int NCOL = NQ * HP;                     // MMA N, TMEM columns per accumulator
  static constexpr int STAGES = 2;
  static constexpr int TILE_A = KB * kKBlockBytes;
  static constexpr int QROWS = NQ * HP;
  static constexpr int QKB = QROWS * 128;
  static constexpr int QBYTES = KB * QKB;
  static constexpr int TMEM_COLS = (2 * NCOL <= 128) ? 128 : (2 * NCOL <= 256) ? 256 : 512;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_Q = OFF_A + STAGES * TILE_A;
  static constexpr int OFF_W = OFF_Q + QBYTES;                  // one query-group slot
  static constexpr int OFF_CK = OFF_W + QROWS * 4;              // candidate keys [NQ][kCap]
  static constexpr int OFF_CI = OFF_CK + NQ * kCap * 4;         // candidate entries [NQ][kCap]
  static constexpr int OFF_HIST = OFF_CI + NQ * kCap * 4;       // radix histogram [256]
  static constexpr int OFF_WC = OFF_HIST + 256 * 4;             // per-warp append counts [2][4][NQ]
  static constexpr int OFF_SC = OFF_WC + 2 * 4 * NQ * 4;        // scan scratch [kEpiWarps], bin, count
  static constexpr int OFF_BAR = OFF_SC + 16 * 4;
  static constexpr int NBAR = 2 * STAGES + 7;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16 + 1024;
  static_assert(NCOL % 16 == 0 && NCOL <= 256, "MMA N");
  static_assert(QKB % 1024 == 0 && TILE_A % 1024 == 0, "swizzle atoms must stay 1 KiB aligned");
  static_assert(OFF_BAR % 8 == 0, "barriers");
  static_assert(BYTES <= 232448, "shared memory");
};

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (f != f || u == 0xff800000u) return 0u;        // NaN and -inf: never selected
  if (u == 0x80000000u) u = 0u;                      // -0 ranks as +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// exclusive prefix sum over the epilogue threads in thread order (et);
// *total = the sum.  Uses sc[0 .. kEpiWarps).
__device__ __forceinline__ int epi_scan(int v, int et, int* sc, int* total) {
  const int lane = et & 31, wq = et >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sc[wq] = x;
  epi_bar();
  int before = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < kEpiWarps; ++i) {
    before += i < wq ? sc[i] : 0;
    tot += sc[i];
  }
  *total = tot;
  epi_bar();
  return before + x - v;
}

// Compacts list qq (n entries, in entry order) to its k best: the k-th key T
// by four 8-bit radix passes, then a stable compaction keeping the keys
// above T and the first keys equal to T.  Returns T.  All epilogue
// threads call it with the same arguments.
__device__ uint32_t compact_list(uint32_t* ck, int32_t* ci, int n, int k, int et, int* hist, int* sc,
                                 int* sh) {
  const int lo = min(n, et * kSeg), hi = min(n, lo + kSeg);
  uint32_t key[kSeg];
  int32_t idx[kSeg];
#pragma unroll
  for (int i = 0; i < kSeg; ++i) {
    key[i] = lo + i < hi ? ck[lo + i] : 0u;
    idx[i] = lo + i < hi ? ci[lo + i] : -1;
  }
  uint32_t prefix = 0, mask = 0;
  int kk = k;
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = et; i < 256; i += kEpiThreads) hist[i] = 0;
    epi_bar();
#pragma unroll
    for (int i = 0; i < kSeg; ++i)
      if (lo + i < hi && (key[i] & mask) == prefix) atomicAdd(&hist[(key[i] >> shift) & 255], 1);
    epi_bar();
    if (et < 32) {
      // lane l owns bins 255 - 8l .. 248 - 8l (from the top); find the bin
      // where the count from the top reaches kk
      int c[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[255 - 8 * et - i];
        sum += c[i];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (et >= o) incl += y;
      }
      int above = incl - sum;                       // keys in bins above this lane's
      if (above < kk && incl >= kk) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (above < kk && above + c[i] >= kk) {
            sh[0] = 255 - 8 * et - i;
            sh[1] = above;
          }
          above += c[i];
        }
      }
    }
    epi_bar();
    prefix |= static_cast<uint32_t>(sh[0]) << shift;
    mask |= 255u << shift;
    kk -= sh[1];
    epi_bar();
  }
  const uint32_t T = prefix;
  int gt = 0, eq = 0;
#pragma unroll
  for (int i = 0; i < kSeg; ++i) {
    gt += (lo + i < hi && key[i] > T) ? 1 : 0;
    eq += (lo + i < hi && key[i] == T) ? 1 : 0;
  }
  int tot;
  const int packed_before = epi_scan(gt | (eq << 16), et, sc, &tot);   // counts < 2^16
  const int gt_before = packed_before & 0xffff, eq_before = packed_before >> 16;
  int pos = gt_before + min(eq_before, kk), eq_seen = eq_before;
#pragma unroll
  for (int i = 0; i < kSeg; ++i) {
    if (lo + i >= hi) break;
    bool keep = key[i] > T;
    if (key[i] == T) {
      keep = eq_seen < kk;
      ++eq_seen;
    }
    if (keep) {
      ck[pos] = key[i];
      ci[pos] = idx[i];
      ++pos;
    }
  }
  epi_bar();
  return T;
}

template <int DK, int HP>
__global__ void __launch_bounds__(kThreads, 1)
    index_topk_fused_kernel(const __grid_constant__ CUtensorMap kmap, const Params p) {
  using C = Cfg<DK, HP>;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + C::OFF_A;
  uint8_t* sQ = smem + C::OFF_Q;
  float* sW = reinterpret_cast<float*>(smem + C::OFF_W);
  uint32_t* sCK = reinterpret_cast<uint32_t*>(smem + C::OFF_CK);
  int32_t* sCI = reinterpret_cast<int32_t*>(smem + C::OFF_CI);
  int* sHist = reinterpret_cast<int*>(smem + C::OFF_HIST);
  int* sWC = reinterpret_cast<int*>(smem + C::OFF_WC);
  int* sSC = reinterpret_cast<int*>(smem + C::OFF_SC);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bar;
  uint64_t* empty = bar + S;
  uint64_t* tfull = bar + 2 * S;
  uint64_t* tempty = tfull + 2;
  uint64_t* qfull = tfull + 4;
  uint64_t* qempty = tfull + 5;
  uint64_t* mma_fin = tfull + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_release();
  // whole query groups per CTA, then every tile of each
  const int64_t g0 = p.n_groups * blockIdx.x / gridDim.x;
  const int64_t g1 = p.n_groups * (blockIdx.x + 1) / gridDim.x;
  const int64_t u0 = g0 * p.n_tiles, u1 = g1 * p.n_tiles;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kEpiWarps);
    }
    mbar_init(qfull, 1);
    mbar_init(qempty, 1 + kEpiWarps);
    mbar_init(mma_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensor_map(&kmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    int64_t prev_bg = -1;
    int qi = -1;
    int64_t it = 0;
    bool ok = true;
    for (int64_t u = u0; u < u1 && ok; ++u, ++it) {
      const int64_t bg = u / p.n_tiles;
      const int t = static_cast<int>(u % p.n_tiles);
      const int b = static_cast<int>(bg / p.n_qgroups);
      const int g = static_cast<int>(bg % p.n_qgroups);
      if (bg != prev_bg) {
        ++qi;
        prev_bg = bg;
        if (qi >= 1 && !mbar_wait(qempty, (qi - 1) & 1, abort_flag, p.err)) { ok = false; break; }
        // rows r = qq * HP + h; 16-byte chunks c = kb * 8 + cc; 8 loads per lane in flight
        constexpr int NCH = C::QROWS * (DK / 8);
        for (int i0 = lane; i0 < NCH; i0 += 32 * 8) {
          uint4 v[8];
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const int i = i0 + 32 * x;
            const int r = i / (DK / 8), c = i % (DK / 8);
            const int qq = r / HP, h = r % HP;
            const int query = g * NQ + qq;
            v[x] = make_uint4(0, 0, 0, 0);
            if (i < NCH && h < p.H && query < p.Q)
              v[x] = __ldg(reinterpret_cast<const uint4*>(p.q + ((static_cast<int64_t>(b) * p.Q + query) * p.H + h) * DK + c * 8));
          }
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const int i = i0 + 32 * x;
            const int r = i / (DK / 8), c = i % (DK / 8);
            if (i < NCH) *reinterpret_cast<uint4*>(sQ + (c / 8) * C::QKB + sw128_offset(r, c % 8)) = v[x];
          }
        }
        for (int r = lane; r < C::QROWS; r += 32) {
          const int qq = r / HP, h = r % HP;
          const int query = g * NQ + qq;
          sW[r] = (h < p.H && query < p.Q) ? p.w[(static_cast<int64_t>(b) * p.Q + query) * p.H + h] : 0.0f;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(qfull);
      }
      const int stage = static_cast<int>(it % S);
      if (it >= S && !mbar_wait(&empty[stage], ((it / S) - 1) & 1, abort_flag, p.err)) { ok = false; break; }
      if (lane == 0) {
        uint8_t* dst = sA + stage * C::TILE_A;
        mbar_arrive_expect_tx(&full[stage], C::TILE_A);
        const int32_t row = static_cast<int32_t>(static_cast<int64_t>(b) * p.N + static_cast<int64_t>(t) * kTileRows);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) tma_load_2d(dst + kb * kKBlockBytes, &kmap, &full[stage], kb * 64, row);
      }
      __syncwarp();
    }
    if (lane == 0) {
      // the TMA loads still in flight land before the CTA's shared memory goes away
      for (int64_t j = (it > S ? it - S : 0); j < it; ++j) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&full[j % S], (j / S) & 1) && globaltimer_ns() - t0 < 100000000ull) {
        }
      }
    }
    __syncwarp();
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
          if (qi >= 0) mma_commit(qempty);
          ++qi;
          if (!mbar_wait(qfull, qi & 1, abort_flag, p.err)) break;
          prev_bg = bg;
        }
        const int stage = static_cast<int>(it % S);
        const int acc = static_cast<int>(it & 1);
        if (!mbar_wait(&full[stage], (it / S) & 1, abort_flag, p.err)) break;
        if (it >= 2 && !mbar_wait(&tempty[acc], ((it >> 1) - 1) & 1, abort_flag, p.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * C::NCOL;
        const uint32_t a0 = smem_u32(sA + stage * C::TILE_A);
        const uint32_t b0 = smem_u32(sQ);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(d_tmem, desc_kmajor_sw128(a0 + kb * kKBlockBytes + kk * 32),
                     desc_kmajor_sw128(b0 + kb * C::QKB + kk * 32), idesc, (kb | kk) != 0);
        }
        mma_commit(&empty[stage]);
        mma_commit(&tfull[acc]);
      }
      mma_commit(mma_fin);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(mma_fin, 0) && globaltimer_ns() - t0 < 100000000ull) {
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue + streaming top-k
    // 8 warps: two per TMEM lane quarter (rows quad*32 ..), each scoring QPW
    // of the group's queries for its rows
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    const int et = (warp - 2) * 32 + lane;     // 0..255: list-work index
    const unsigned lt_mask = (1u << lane) - 1u;
    int64_t prev_bg = -1;
    int qi = -1;
    int64_t it = 0;
    int cnt[NQ];
    uint32_t tau[NQ];
    int64_t nvis[NQ];
    int64_t qrow0 = 0;                         // b * Q + g * NQ of the current group
    auto finish_group = [&]() {
      for (int qq = 0; qq < NQ; ++qq) {
        if (cnt[qq] > p.k) {
          compact_list(sCK + qq * kCap, sCI + qq * kCap, cnt[qq], p.k, et, sHist, sSC, sSC + kEpiWarps);
          cnt[qq] = p.k;
        }
      }
      const int b = static_cast<int>(qrow0 / p.Q);
      const int q0 = static_cast<int>(qrow0 % p.Q);
      for (int qq = 0; qq < NQ; ++qq) {
        if (q0 + qq >= p.Q) break;
        int32_t* o = p.topk + (static_cast<int64_t>(b) * p.Q + q0 + qq) * p.k;
        for (int i = et; i < p.k; i += kEpiThreads) o[i] = i < cnt[qq] ? sCI[qq * kCap + i] : -1;
      }
      epi_bar();
    };
    for (int64_t u = u0; u < u1; ++u, ++it) {
      const int64_t bg = u / p.n_tiles;
      const int t = static_cast<int>(u % p.n_tiles);
      if (bg != prev_bg) {
        if (qi >= 0) {
          if (lane == 0) mbar_arrive(qempty);   // q and weights of the group no longer read
          finish_group();
        }
        ++qi;
        // a wait that gives up leaves the CTA winding down: the epilogue still
        // runs every tile (on whatever TMEM holds), so every epilogue thread
        // takes the same named barriers and none waits for another in vain
        mbar_wait(qfull, qi & 1, abort_flag, p.err);
        prev_bg = bg;
        const int b = static_cast<int>(bg / p.n_qgroups);
        qrow0 = static_cast<int64_t>(b) * p.Q + (bg % p.n_qgroups) * NQ;
#pragma unroll
        for (int qq = 0; qq < NQ; ++qq) {
          cnt[qq] = 0;
          tau[qq] = 0u;
          // entries [0, nvis) are visible to query qq of the group (none past
          // the sequence's last query)
          const bool real = (qrow0 % p.Q) + qq < p.Q;
          nvis[qq] = !real ? 0 : p.n_visible ? std::min<int64_t>(p.n_visible[qrow0 + qq], p.N) : p.N;
        }
      }
      const int acc = static_cast<int>(it & 1);
      const int64_t e = static_cast<int64_t>(t) * kTileRows + row;   // this row's entry
      mbar_wait(&tfull[acc], (it >> 1) & 1, abort_flag, p.err);
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * C::NCOL;
      // this warp's QPW queries, HP columns each, read in chunks of kChunk
      // columns one chunk ahead of the arithmetic (a wait covers every load
      // issued before it, so chunk c + 1 is requested after chunk c landed)
      constexpr int kChunk = HP % 32 == 0 ? 32 : 16;
      constexpr int kPerQ = HP / kChunk;
      constexpr int kChunks = QPW * kPerQ;
      const uint32_t tq = taddr + static_cast<uint32_t>(half * QPW * HP);
      uint32_t v[2][kChunk];
      auto load_chunk = [&](int c, uint32_t (&dst)[kChunk]) {
        const uint32_t col = static_cast<uint32_t>((c / kPerQ) * HP + (c % kPerQ) * kChunk);
        if constexpr (kChunk == 32) tmem_ld32(tq + col, dst);
        else tmem_ld16(tq + col, dst);
      };
      float a[QPW];
#pragma unroll
      for (int j = 0; j < QPW; ++j) a[j] = 0.0f;
      const float* wq = sW + half * QPW * HP;
      load_chunk(0, v[0]);
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        tmem_wait_ld();
        if (c + 1 < kChunks) load_chunk(c + 1, v[(c + 1) & 1]);
        const int j = c / kPerQ, h0 = (c % kPerQ) * kChunk;
#pragma unroll
        for (int h = 0; h < kChunk; ++h) {
          float x = __uint_as_float(v[c & 1][h]);
          if (p.relu) x = fmaxf(x, 0.0f);
          a[j] = fmaf(wq[j * HP + h0 + h], x, a[j]);
        }
      }
      // (arrays over all NQ queries keep compile-time indices; the branch on
      // the warp's half is uniform over the warp)
      float s[NQ];
#pragma unroll
      for (int qq = 0; qq < NQ; ++qq) s[qq] = qq / QPW == half ? a[qq % QPW] : 0.0f;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      // append, in entry order, the rows whose key beats each query's threshold
      uint32_t key[NQ];
      unsigned bal[NQ];
      int* wc = sWC + (it & 1) * 4 * NQ;
#pragma unroll
      for (int qq = 0; qq < NQ; ++qq) {
        key[qq] = 0u;
        bal[qq] = 0u;
        if (qq / QPW != half) continue;
        key[qq] = e < nvis[qq] ? score_key(s[qq]) : 0u;
        bal[qq] = __ballot_sync(0xffffffffu, key[qq] > tau[qq]);
        if (lane == 0) wc[quad * NQ + qq] = __popc(bal[qq]);
      }
      epi_bar();
#pragma unroll
      for (int qq = 0; qq < NQ; ++qq) {
        int before = cnt[qq], total = 0;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int c = wc[x * NQ + qq];
          before += x < quad ? c : 0;
          total += c;
        }
        if (qq / QPW == half && key[qq] > tau[qq]) {
          const int pos = before + __popc(bal[qq] & lt_mask);
          sCK[qq * kCap + pos] = key[qq];
          sCI[qq * kCap + pos] = static_cast<int32_t>(e);
        }
        cnt[qq] += total;
      }
      // a list that the next tile could overflow is compacted to its k best now
#pragma unroll 1
      for (int qq = 0; qq < NQ; ++qq) {
        if (cnt[qq] + kTileRows > kCap) {
          epi_bar();                            // the appends above are in place
          tau[qq] = compact_list(sCK + qq * kCap, sCI + qq * kCap, cnt[qq], p.k, et, sHist, sSC, sSC + kEpiWarps);
          cnt[qq] = p.k;
        }
      }
    }
    if (qi >= 0) {
      epi_bar();
      finish_group();
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

template <int DK, int HP>
csa2_status run_fused(const void* q, const float* w, const void* k, int B, int Q, int H, int64_t N,
                      const int32_t* n_visible, int k_top, csa2_index_act act, int32_t* topk,
                      cudaStream_t stream) {
  using C = Cfg<DK, HP>;
  CUtensorMap map;
  memset(&map, 0, sizeof(map));
  CSA2_TRY(make_tensor_map_bf16_2d(&map, k, static_cast<uint64_t>(B) * N, DK, DK * 2, 64, kTileRows));
  Params p;
  p.q = static_cast<const uint16_t*>(q);
  p.w = w;
  p.n_visible = n_visible;
  p.topk = topk;
  p.err = device_error_word();
  p.Q = Q;
  p.H = H;
  p.k = k_top;
  p.N = N;
  p.relu = act == CSA2_ACT_RELU ? 1 : 0;
  p.n_qgroups = (Q + NQ - 1) / NQ;
  p.n_tiles = static_cast<int>((N + kTileRows - 1) / kTileRows);
  p.n_groups = static_cast<int64_t>(B) * p.n_qgroups;
  static PerDevice<cudaError_t> opt_in;
  const cudaError_t attr_err = opt_in.get([] {
    const cudaError_t e = cudaFuncSetAttribute(index_topk_fused_kernel<DK, HP>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, C::BYTES);
    if (e != cudaSuccess) cudaGetLastError();
    return e;
  });
  if (attr_err != cudaSuccess) return fail(CSA2_ERR_CUDA, "index_topk_fused: smem opt-in failed");
  const int64_t grid = std::min<int64_t>(sm_count(), p.n_groups);
  begin_launch(stream);
  index_topk_fused_kernel<DK, HP><<<static_cast<unsigned>(grid), kThreads, C::BYTES, stream>>>(map, p);
  note_launch(LK_INDEX, 1, stream);
  return check_launch("index_topk_fused");
}

}  // namespace

bool index_topk_fused_applies(int B, int Q, int H, int d, int64_t N, int k_top) {
  if (getenv("CSA2_NO_FUSED_TOPK")) return false;
  if ((d != 64 && d != 128) || H > 64 || k_top <= 0 || k_top > kMaxFusedTopk) return false;
  if (static_cast<int64_t>(B) * N > 0x7fffffffLL || N <= 0) return false;
  // enough query groups to give every SM whole groups of work
  return static_cast<int64_t>(B) * ((Q + NQ - 1) / NQ) >= sm_count();
}

csa2_status launch_index_topk_fused(const void* q, const float* w, const void* k, int B, int Q,
                                    int H, int d, int64_t N, const int32_t* n_visible, int k_top,
                                    csa2_index_act act, int32_t* topk, cudaStream_t stream) {
  if (d == 64)
    return H <= 16 ? run_fused<64, 16>(q, w, k, B, Q, H, N, n_visible, k_top, act, topk, stream)
                   : run_fused<64, 64>(q, w, k, B, Q, H, N, n_visible, k_top, act, topk, stream);
  return H <= 16 ? run_fused<128, 16>(q, w, k, B, Q, H, N, n_visible, k_top, act, topk, stream)
                 : run_fused<128, 64>(q, w, k, B, Q, H, N, n_visible, k_top, act, topk, stream);
}

}  // namespace csa2
