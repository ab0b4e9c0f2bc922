// Top-k selection with a cluster of 8 CTAs per row, for batches too small to
// fill the GPU with one CTA per row: the hierarchical indexer's pool in a
// Reindex layer (8 rows of 16384) and a Full layer's pool and top-k (8 rows
// of 262144).  Two variants: 512 threads and up to 4096 keys per CTA (rows of
// up to 32768), 1024 threads and up to 32768 keys per CTA (rows of up to
// 262144).  Sources: "读完这篇，你就搞懂 DeepSeek v4 了", 闪电索引机制
// (keep the k best entries); "Recall之王", Hierarchical Sparse Indexer (the
// Full layer's pool and its top-k; the Reindex layer's top-k inside the pool).
//
// Same result as the one-CTA kernel: score descending, ties to the lower
// position, -inf and NaN never chosen, -0 ranks as +0; selected positions
// are written in position order, padded with -1.  CTA c of a row's cluster
// holds positions [c * chunk, (c + 1) * chunk) as order-preserving keys in
// its shared memory.  Data moves between the CTAs by stores into the other
// CTAs' shared memory followed by one cluster barrier (a remote load costs a
// round trip; a store does not wait):
//   1. each CTA's smallest / largest selectable key and count go to every CTA;
//   2. radix passes of 8-bit digits below the bits all selectable keys share:
//      each warp counts its keys into its own histogram, the CTA's sum is
//      stored into every CTA, so every CTA sums the same eight histograms and
//      takes the same bin;
//   3. once the threshold bin holds at most kMaxCand keys, each CTA compacts
//      its keys in or above the bin (the survivors, in position order, with
//      their positions; the per-warp histograms give each warp its offset),
//      lists the bin's keys, and every CTA copies the eight lists (in CTA
//      order); the remaining passes (9-bit digits) run over the candidates;
//   4. each CTA's output offset follows from the counts it has: the keys above
//      the threshold bins in the CTAs before it (sent with the lists) and the
//      candidates before its own in the copied list; the ordered write runs
//      over the survivors.  A CTA with more survivors than its buffer holds
//      sweeps its whole chunk instead, and only a row whose threshold bin
//      never fits the list needs one more exchange of counts.
// Integer counts only: the result is deterministic.
#include <cooperative_groups.h>

#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "launchers.h"

namespace csa2 {
namespace {
namespace cg = cooperative_groups;

constexpr int kC = 8;                      // CTAs per row (one cluster)
constexpr int kDigit = 8;
constexpr int kBins = 1 << kDigit;         // one warp finds the bin: 8 bins per lane
constexpr int kLocalDigit = 9;             // passes over the gathered candidates
constexpr int kLocalBins = 1 << kLocalDigit;   // 16 bins per lane
constexpr int kMaxCand = 4096;
constexpr int kHistStores = kC * (kBins / 4);   // 16-byte histogram stores per CTA and pass

struct ClParams {
  const float* scores;
  int64_t L;
  int chunk;                               // keys per CTA, multiple of 4 * warps
  int seg;                                 // keys per warp = chunk / warps
  int count;
  const int32_t* ids;
  int32_t* out;
  // when set, key i of row r is scores[r * src_stride + gather[r * L + i]]
  // (a negative entry: not selectable)
  const int32_t* gather;
  int64_t src_stride;
};

template <int NT, int MAXCHUNK, int SURV>
struct Smem {
  static constexpr int NW = NT / 32;
  uint32_t keys[MAXCHUNK];                 // this CTA's keys (0 = not selectable)
  uint32_t lcand[kMaxCand];                // this CTA's keys in the threshold bin
  union {
    int inbox[2][kC][kBins];               // histograms stored by each CTA (pass parity)
    uint32_t cand[kMaxCand];               // after the passes: every CTA's list, in CTA order
  } x;
  union {
    int whist[NW][kBins];                  // each warp's histogram of the pass
    struct {                               // after the passes: keys in or above the
      uint32_t key[SURV];                  // threshold bin, in position order, with
      uint16_t pos[SURV];                  // their positions in the chunk
    } surv;
  } w;
  int hist[2][kLocalBins];                 // the CTA's histogram; the local passes' (parity)
  int gsum[kBins];                         // the cluster's histogram
  uint32_t x_min[kC], x_max[kC];           // stored by each CTA: its selectable keys
  int x_n[kC];
  int x_nl[kC], x_above[kC];               // stored by each CTA with its list
  int x_g[kC], x_e[kC];                    // stored by each CTA: keys above / equal to T
  int wg[NW], we[NW], wg_off[NW], we_off[NW];
  uint32_t kmin, kmax;
  int nsel, nl, cnt_g, cnt_e;
  int bin, above, bin_cnt;
};
static_assert(sizeof(uint32_t) * kMaxCand <= sizeof(int) * 2 * kC * kBins, "list fits the inboxes");

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (f != f || u == 0xff800000u) return 0u;       // NaN, -inf: never chosen
  if (u == 0x80000000u) u = 0u;                    // -0 ranks as +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Warp 0 only: the bin of h[0..nb) (nb <= 32 * PER) holding the kk-th largest
// key; sets S.bin, S.above (keys in higher bins) and S.bin_cnt.
template <int PER, class SM>
__device__ __forceinline__ void warp_find_bin(const int* h, int nb, int kk, SM& S) {
  const int lane = threadIdx.x & 31;
  int v[PER];
  int mine = 0;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    v[u] = PER * lane + u < nb ? h[PER * lane + u] : 0;
    mine += v[u];
  }
  int x = mine;                              // inclusive suffix sum over the lanes
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_down_sync(0xffffffffu, x, o);
    if (lane + o < 32) x += y;
  }
  int above = x - mine;
#pragma unroll
  for (int u = PER - 1; u >= 0; --u) {
    if (above < kk && above + v[u] >= kk) {
      S.bin = PER * lane + u;
      S.above = above;
      S.bin_cnt = v[u];
    }
    above += v[u];
  }
}

template <class SM>
__device__ __forceinline__ uint4 keys4(const SM& S, int i, int lo, int w_hi) {
  return i < w_hi ? *reinterpret_cast<const uint4*>(&S.keys[i - lo]) : make_uint4(0u, 0u, 0u, 0u);
}

__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Exclusive prefix over the warps of per-warp counts (g, e) in S.wg / S.we
// (warp 0 computes it into S.wg_off / S.we_off and returns the CTA totals).
template <class SM, int NW>
__device__ __forceinline__ void warp_offsets(SM& S, int* g_tot, int* e_tot) {
  const int lane = threadIdx.x & 31;
  const int g = lane < NW ? S.wg[lane] : 0, e = lane < NW ? S.we[lane] : 0;
  int gi = g, ei = e;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int yg = __shfl_up_sync(0xffffffffu, gi, o), ye = __shfl_up_sync(0xffffffffu, ei, o);
    if (lane >= o) {
      gi += yg;
      ei += ye;
    }
  }
  if (lane < NW) {
    S.wg_off[lane] = gi - g;
    S.we_off[lane] = ei - e;
  }
  *g_tot = __shfl_sync(0xffffffffu, gi, 31);
  *e_tot = __shfl_sync(0xffffffffu, ei, 31);
}

template <int NT, int MAXCHUNK, int SURV>
__global__ void __cluster_dims__(kC, 1, 1) __launch_bounds__(NT, 1)
    topk_cluster_kernel(ClParams p) {
  using SM = Smem<NT, MAXCHUNK, SURV>;
  constexpr int NW = SM::NW;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SM& S = *reinterpret_cast<SM*>(smem_raw);
  cg::cluster_group cl = cg::this_cluster();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cta = static_cast<int>(cl.block_rank());
  const int64_t r = blockIdx.x / kC;
  const int L = static_cast<int>(p.L);
  const float* s = p.scores + r * p.L;
  const int lo = min(L, cta * p.chunk), hi = min(L, lo + p.chunk);
  const int w_lo = lo + warp * p.seg, w_hi = min(hi, w_lo + p.seg);   // empty when w_lo >= hi
  const unsigned lt = (1u << lane) - 1u;
  pdl_wait();                                // the scores come from the kernel before
  pdl_release();

  if (tid == 0) {
    S.kmin = 0xffffffffu;
    S.kmax = 0u;
    S.nsel = 0;
    S.nl = 0;
    S.cnt_g = 0;
    S.cnt_e = 0;
  }
  for (int i = tid; i < NW * kBins; i += NT) (&S.w.whist[0][0])[i] = 0;
  for (int i = tid; i < 2 * kLocalBins; i += NT) (&S.hist[0][0])[i] = 0;
  __syncthreads();

  // ---- this warp's keys; the CTA's smallest / largest selectable key
  {
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    int nsel = 0;
    const bool vec = (reinterpret_cast<uintptr_t>(s) & 15u) == 0;   // lo, w_lo, i: multiples of 4
    const int32_t* gidx = p.gather ? p.gather + r * p.L : nullptr;
    const float* src = p.scores + r * p.src_stride;
    // four groups of 128 keys per step: each lane has its loads in flight
    // before it converts any of them
    for (int b0 = w_lo; b0 < w_hi; b0 += 4 * 128) {
      float f[4][4];
      if (gidx) {
        int g[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = b0 + q * 128 + 4 * lane + u;
            g[q][u] = i < w_hi ? __ldg(gidx + i) : -1;
          }
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int u = 0; u < 4; ++u)
            f[q][u] = g[q][u] >= 0 && g[q][u] < p.src_stride ? __ldg(src + g[q][u]) : __int_as_float(0xff800000);
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = b0 + q * 128 + 4 * lane;
          if (vec && i + 3 < w_hi) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(s + i));
            f[q][0] = v.x; f[q][1] = v.y; f[q][2] = v.z; f[q][3] = v.w;
          } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) f[q][u] = i + u < w_hi ? __ldg(s + i + u) : __int_as_float(0xff800000);
          }
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = b0 + q * 128 + 4 * lane;
        if (i >= w_hi) break;                // (i - lo) stays inside the CTA's chunk
        uint32_t k4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          k4[u] = score_key(f[q][u]);
          if (k4[u]) {
            kmin = min(kmin, k4[u]);
            kmax = max(kmax, k4[u]);
            ++nsel;
          }
        }
        *reinterpret_cast<uint4*>(&S.keys[i - lo]) = make_uint4(k4[0], k4[1], k4[2], k4[3]);
      }
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    nsel = __reduce_add_sync(0xffffffffu, nsel);
    if (lane == 0) {
      atomicMin(&S.kmin, kmin);
      atomicMax(&S.kmax, kmax);
      atomicAdd(&S.nsel, nsel);
    }
  }
  __syncthreads();
  if (tid < kC) {
    SM* R = cl.map_shared_rank(&S, tid);
    R->x_min[cta] = S.kmin;
    R->x_max[cta] = S.kmax;
    R->x_n[cta] = S.nsel;
  }
  cl.sync();                                 // every CTA's min / max / count is here
  uint32_t rmin = 0xffffffffu, rmax = 0u;
  int total_sel = 0, nsel_before = 0;
#pragma unroll
  for (int c = 0; c < kC; ++c) {
    rmin = min(rmin, S.x_min[c]);
    rmax = max(rmax, S.x_max[c]);
    total_sel += S.x_n[c];
    nsel_before += c < cta ? S.x_n[c] : 0;
  }
  const bool all = total_sel <= p.count;     // every selectable key is chosen

  // ---- threshold key T, how many keys equal to T to take (take), how many
  // there are (eqcnt); keys above / equal to T in the CTAs before this one
  uint32_t T = 0u;
  int take = 0, eqcnt = 0, cgb = 0, ceb = 0;
  bool exchange = false;                     // the counts still need an exchange
  bool fast = false;                         // the output runs over the survivors
  int nsurv = 0;
  if (all) {
    cgb = nsel_before;
    cluster_arrive();
  } else if (rmin == rmax) {                 // one distinct key, more of it than wanted
    T = rmin;
    take = p.count;
    eqcnt = total_sel;
    ceb = nsel_before;
    cluster_arrive();
  } else {
    const int common = __clz(rmin ^ rmax);
    const uint32_t cmask = common == 0 ? 0u : ~0u << (32 - common);
    uint32_t prefix = rmin & cmask, mask = cmask;
    int kk = p.count;
    int lowbit = 32 - common;                // key bits [lowbit-1 : 0] still undecided
    int par = 0;
    int w_above = 0, w_inbin = 0;            // this warp's keys above / in the threshold bins
    bool gathered = false;
    int ncand = 0, my_off = 0;
    int* wh = S.w.whist[warp];
    while (lowbit > 0 && !gathered) {
      const int width = lowbit >= kDigit ? kDigit : lowbit;
      const int shift = lowbit - width;
      const uint32_t dmask = (1u << width) - 1u;
      const int nb = 1 << width;
      for (int b0 = w_lo; b0 < w_hi; b0 += 128) {
        const int i = b0 + 4 * lane;
        const uint4 k4 = keys4(S, i, lo, w_hi);
        const uint32_t kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (kv[u] && i + u < w_hi && (kv[u] & mask) == prefix) atomicAdd(&wh[(kv[u] >> shift) & dmask], 1);
      }
      __syncthreads();
      for (int b = tid; b < nb; b += NT) {   // the CTA's histogram: the warps' sum
        int v = 0;
#pragma unroll 8
        for (int w = 0; w < NW; ++w) v += S.w.whist[w][b];
        S.hist[0][b] = v;
      }
      __syncthreads();
      if (tid < kHistStores) {
        const int d = tid / (kBins / 4), q4 = 4 * (tid % (kBins / 4));
        SM* R = cl.map_shared_rank(&S, d);
        *reinterpret_cast<int4*>(&R->x.inbox[par][cta][q4]) = *reinterpret_cast<const int4*>(&S.hist[0][q4]);
      }
      cl.sync();                             // every CTA's histogram is here
      if (tid < nb) {
        int v = 0;
#pragma unroll
        for (int c = 0; c < kC; ++c) v += S.x.inbox[par][c][tid];
        S.gsum[tid] = v;
      }
      __syncthreads();
      if (warp == 0) warp_find_bin<kBins / 32>(S.gsum, nb, kk, S);
      __syncthreads();
      const int b = S.bin;
      kk -= S.above;
      eqcnt = S.bin_cnt;
      prefix |= static_cast<uint32_t>(b) << shift;
      mask |= dmask << shift;
      lowbit = shift;
      par ^= 1;
      {                                      // this warp's keys above / in the bin; its histogram back to zero
        int wa = 0, wb = 0;
        for (int d = lane; d < nb; d += 32) {
          const int v = wh[d];
          wa += d > b ? v : 0;
          wb += d == b ? v : 0;
          wh[d] = 0;
        }
        w_above += __reduce_add_sync(0xffffffffu, wa);
        w_inbin = __reduce_add_sync(0xffffffffu, wb);
      }
      if (lowbit > 0 && eqcnt <= kMaxCand) {
        // survivors: this CTA's keys in the bin or above it (key >= prefix)
        if (lane == 0) {
          S.wg[warp] = w_above + w_inbin;
          S.we[warp] = w_above;
        }
        __syncthreads();                     // every warp is done with its histogram
        int base, tot, above_cta, cand_before;
        {                                    // every warp: scan over the warps' counts
          const int sv = lane < NW ? S.wg[lane] : 0, av = lane < NW ? S.we[lane] : 0;
          int si = sv, ci = sv - av;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int ys = __shfl_up_sync(0xffffffffu, si, o), yc = __shfl_up_sync(0xffffffffu, ci, o);
            if (lane >= o) {
              si += ys;
              ci += yc;
            }
          }
          base = __shfl_sync(0xffffffffu, si - sv, warp);
          cand_before = __shfl_sync(0xffffffffu, ci - (sv - av), warp);
          tot = __shfl_sync(0xffffffffu, si, 31);
          above_cta = __reduce_add_sync(0xffffffffu, av);
        }
        nsurv = tot;
        fast = tot <= SURV;                  // the same in every thread of the CTA
        if (fast) {
          // the survivors in position order, then the bin's keys among them
          if (w_above + w_inbin) {
            for (int b0 = w_lo; b0 < w_hi; b0 += 128) {
              const int i = b0 + 4 * lane;
              const uint4 k4 = keys4(S, i, lo, w_hi);
              const uint32_t kv[4] = {k4.x, k4.y, k4.z, k4.w};
              int m4 = 0;
#pragma unroll
              for (int u = 0; u < 4; ++u) m4 |= (kv[u] && i + u < w_hi && kv[u] >= prefix) << u;
              // position order is lane-major: lower lanes' keys, then this
              // lane's earlier keys, come first
              int lower = 0, total = 0;
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const unsigned bal = __ballot_sync(0xffffffffu, (m4 >> u) & 1);
                lower += __popc(bal & lt);
                total += __popc(bal);
              }
              int j = base + lower;
#pragma unroll
              for (int u = 0; u < 4; ++u)
                if ((m4 >> u) & 1) {
                  S.w.surv.key[j] = kv[u];
                  S.w.surv.pos[j] = static_cast<uint16_t>(i + u - lo);
                  ++j;
                }
              base += total;
            }
          }
          __syncthreads();
          for (int j0 = warp * 32; j0 < tot; j0 += NT) {
            const int j = j0 + lane;
            const uint32_t key = j < tot ? S.w.surv.key[j] : 0u;
            const bool m = j < tot && (key & mask) == prefix;
            const unsigned bal = __ballot_sync(0xffffffffu, m);
            int at = 0;
            if (lane == 0 && bal) at = atomicAdd(&S.nl, __popc(bal));
            at = __shfl_sync(0xffffffffu, at, 0);
            if (m) S.lcand[at + __popc(bal & lt)] = key;
          }
        } else {
          // too many for the survivor buffer: the bin's keys from the whole chunk
          int wbase = cand_before;
          if (w_inbin) {
            for (int b0 = w_lo; b0 < w_hi; b0 += 128) {
              const int i = b0 + 4 * lane;
              const uint4 k4 = keys4(S, i, lo, w_hi);
              const uint32_t kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const bool m = kv[u] && i + u < w_hi && (kv[u] & mask) == prefix;
                const unsigned bal = __ballot_sync(0xffffffffu, m);
                if (m) S.lcand[wbase + __popc(bal & lt)] = kv[u];
                wbase += __popc(bal);
              }
            }
          }
          if (tid == 0) S.nl = tot - above_cta;
        }
        __syncthreads();
        if (tid < kC) {
          SM* R = cl.map_shared_rank(&S, tid);
          R->x_nl[cta] = S.nl;
          R->x_above[cta] = above_cta;
        }
        for (int i = tid; i < 2 * kLocalBins; i += NT) (&S.hist[0][0])[i] = 0;   // for the local passes
        cl.sync();                           // every CTA's list and count is here
        int off[kC];
        int acc = 0;
#pragma unroll
        for (int c = 0; c < kC; ++c) {
          off[c] = acc;
          if (c == cta) my_off = acc;
          acc += S.x_nl[c];
          cgb += c < cta ? S.x_above[c] : 0;
        }
        ncand = acc;                         // == eqcnt
        for (int j = tid; j < ncand; j += NT) {
          int c = 0, cbase = 0;              // the last CTA whose list starts at or before j
#pragma unroll
          for (int u = 1; u < kC; ++u)
            if (j >= off[u]) {
              c = u;
              cbase = off[u];
            }
          S.x.cand[j] = cl.map_shared_rank(S.lcand, c)[j - cbase];
        }
        gathered = true;
        __syncthreads();
        cluster_arrive();                    // this CTA reads no other CTA's memory from here on
      }
    }
    if (gathered) {
      // further passes over the candidates alone (both histograms are zero)
      int lp = 0;
      while (lowbit > 0) {
        const int width = lowbit >= kLocalDigit ? kLocalDigit : lowbit;
        const int shift = lowbit - width;
        const uint32_t dmask = (1u << width) - 1u;
        for (int j = tid; j < ncand; j += NT) {
          const uint32_t key = S.x.cand[j];
          if ((key & mask) == prefix) atomicAdd(&S.hist[lp][(key >> shift) & dmask], 1);
        }
        __syncthreads();
        if (warp == 0) warp_find_bin<kLocalBins / 32>(S.hist[lp], 1 << width, kk, S);
        __syncthreads();
        prefix |= static_cast<uint32_t>(S.bin) << shift;
        mask |= dmask << shift;
        kk -= S.above;
        eqcnt = S.bin_cnt;
        lowbit = shift;
        // zero for the pass after next, whose counts start after the next
        // pass's first barrier
        for (int i = tid; i < kLocalBins; i += NT) S.hist[lp][i] = 0;
        lp ^= 1;
      }
      T = prefix;
      take = kk;
      // candidates above / equal to T listed before this CTA's own
      int g = 0, e = 0;
      for (int j = tid; j < my_off; j += NT) {
        const uint32_t key = S.x.cand[j];
        g += key > T;
        e += key == T;
      }
      g = __reduce_add_sync(0xffffffffu, g);
      e = __reduce_add_sync(0xffffffffu, e);
      if (lane == 0 && (g | e)) {
        atomicAdd(&S.cnt_g, g);
        atomicAdd(&S.cnt_e, e);
      }
      __syncthreads();
      cgb += S.cnt_g;
      ceb = S.cnt_e;
    } else {
      // the bin never fit the list: every key bit is decided, counts follow below
      T = prefix;
      take = kk;
      exchange = true;
    }
  }

  int32_t* o = p.out + r * static_cast<int64_t>(p.count);
  const bool simple = all || take >= eqcnt;
  if (fast) {
    // ---- ordered write over the survivors: warp w takes a run of them
    const int per = (nsurv + NW * 32 - 1) / (NW * 32) * 32;
    const int j_lo = min(nsurv, warp * per), j_hi = min(nsurv, j_lo + per);
    int g = 0, e = 0;
    for (int j0 = j_lo; j0 < j_hi; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t key = j < j_hi ? S.w.surv.key[j] : 0u;
      g += key > T ? 1 : 0;
      e += key == T ? 1 : 0;
    }
    g = __reduce_add_sync(0xffffffffu, g);
    e = __reduce_add_sync(0xffffffffu, e);
    if (lane == 0) {
      S.wg[warp] = g;
      S.we[warp] = e;
    }
    __syncthreads();
    if (warp == 0) {
      int gt, et;
      warp_offsets<SM, NW>(S, &gt, &et);
    }
    __syncthreads();
    int run_eq = ceb + S.we_off[warp];
    int run_sel = cgb + S.wg_off[warp] + min(run_eq, take);
    for (int j0 = j_lo; j0 < j_hi; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t key = j < j_hi ? S.w.surv.key[j] : 0u;
      const bool eq = key == T && j < j_hi;
      const unsigned eb = __ballot_sync(0xffffffffu, eq);
      bool sel = key > T;
      if (eq) sel = run_eq + __popc(eb & lt) < take;
      const unsigned sb = __ballot_sync(0xffffffffu, sel);
      if (sel) {
        const int q = run_sel + __popc(sb & lt);
        const int posn = lo + S.w.surv.pos[j];
        if (q < p.count) o[q] = p.ids ? p.ids[r * p.L + posn] : posn;
      }
      run_sel += __popc(sb);
      run_eq += __popc(eb);
    }
  } else {
    // ---- per warp: keys above / equal to T over the whole chunk.  All keys
    // equal to T taken (the usual case): one sweep compacts each warp's
    // picks, in order, into its own part of the key buffer (never past the
    // keys it has read).
    const uint32_t thr = all ? 1u : T;
    {
      int g = 0, e = 0;
      if (simple) {
        for (int b0 = w_lo; b0 < w_hi; b0 += 128) {
          const int i = b0 + 4 * lane;
          const uint4 k4 = keys4(S, i, lo, w_hi);
          const uint32_t kv[4] = {k4.x, k4.y, k4.z, k4.w};
          int sel_m = 0;
#pragma unroll
          for (int u = 0; u < 4; ++u) sel_m |= (kv[u] >= thr && i + u < w_hi) << u;
          if (!__any_sync(0xffffffffu, sel_m)) continue;
          int lower = 0, total = 0;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const unsigned sb = __ballot_sync(0xffffffffu, (sel_m >> u) & 1);
            lower += __popc(sb & lt);
            total += __popc(sb);
          }
          int q = g + lower;
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if ((sel_m >> u) & 1) S.keys[w_lo - lo + q++] = static_cast<uint32_t>(i + u);
          g += total;
        }
      } else {
        for (int b0 = w_lo; b0 < w_hi; b0 += 128) {
          const int i = b0 + 4 * lane;
          const uint4 k4 = keys4(S, i, lo, w_hi);
          const uint32_t kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const bool valid = kv[u] != 0u && i + u < w_hi;
            g += (valid && kv[u] > T) ? 1 : 0;
            e += (valid && kv[u] == T) ? 1 : 0;
          }
        }
        g = __reduce_add_sync(0xffffffffu, g);
        e = __reduce_add_sync(0xffffffffu, e);
      }
      if (lane == 0) {
        S.wg[warp] = g;
        S.we[warp] = e;
      }
    }
    __syncthreads();
    if (warp == 0) {
      int gt, et;
      warp_offsets<SM, NW>(S, &gt, &et);
      if (exchange && lane < kC) {           // this CTA's totals to every CTA
        SM* R = cl.map_shared_rank(&S, lane);
        R->x_g[cta] = gt;
        R->x_e[cta] = et;
      }
    }
    if (exchange) {
      cl.sync();                             // every CTA's counts are here
#pragma unroll
      for (int c = 0; c < kC; ++c) {
        cgb += c < cta ? S.x_g[c] : 0;
        ceb += c < cta ? S.x_e[c] : 0;
      }
      cluster_arrive();
    } else {
      __syncthreads();
    }
    const int g_before = cgb + S.wg_off[warp];
    const int e_before = ceb + S.we_off[warp];
    if (simple) {
      const int sel_start = g_before + min(e_before, take);
      for (int j = lane; j < S.wg[warp]; j += 32) {
        const int q = sel_start + j;
        const int posn = static_cast<int>(S.keys[w_lo - lo + j]);
        if (q < p.count) o[q] = p.ids ? p.ids[r * p.L + posn] : posn;
      }
    } else {
      int run_sel = g_before + min(e_before, take), run_eq = e_before;
      for (int b0 = w_lo; b0 < w_hi; b0 += 128) {
        const int i = b0 + 4 * lane;
        const uint4 k4 = keys4(S, i, lo, w_hi);
        const uint32_t kv[4] = {k4.x, k4.y, k4.z, k4.w};
        int sel_m = 0, eq_m = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const bool valid = kv[u] != 0u && i + u < w_hi;
          sel_m |= (valid && kv[u] > T) << u;
          eq_m |= (valid && kv[u] == T) << u;
        }
        // position order is lane-major: lower lanes' keys, then this lane's
        // earlier keys, come first
        int eq_lower = 0, warp_eq = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const unsigned eb = __ballot_sync(0xffffffffu, (eq_m >> u) & 1);
          eq_lower += __popc(eb & lt);
          warp_eq += __popc(eb);
        }
        int rank = run_eq + eq_lower;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if ((eq_m >> u) & 1) {
            if (rank < take) sel_m |= 1 << u;
            ++rank;
          }
        int sel_lower = 0, warp_sel = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const unsigned sb = __ballot_sync(0xffffffffu, (sel_m >> u) & 1);
          sel_lower += __popc(sb & lt);
          warp_sel += __popc(sb);
        }
        int pos = run_sel + sel_lower;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if ((sel_m >> u) & 1) {
            if (pos < p.count) o[pos] = p.ids ? p.ids[r * p.L + i + u] : i + u;
            ++pos;
          }
        run_sel += warp_sel;
        run_eq += warp_eq;
      }
    }
  }
  // padding: positions beyond the selectable keys
  const int n_out = all ? total_sel : p.count;
  for (int q = n_out + cta * NT + tid; q < p.count; q += kC * NT) o[q] = -1;
  // no CTA leaves while another may still read its shared memory
  cluster_wait();
}

constexpr int kSmallThreads = 512, kSmallChunk = 4096, kSmallSurv = 2048;
constexpr int kLargeThreads = 1024, kLargeChunk = 32768, kLargeSurv = 4096;
static_assert(kHistStores <= kSmallThreads, "one 16-byte histogram store per thread");

template <int NT, int MAXCHUNK, int SURV>
csa2_status launch_variant(ClParams p, int64_t rows, cudaStream_t stream) {
  constexpr int NW = NT / 32;
  const int64_t per = (p.L + kC - 1) / kC;
  p.chunk = static_cast<int>((per + 4 * NW - 1) / (4 * NW) * (4 * NW));
  p.seg = p.chunk / NW;
  if (p.chunk > MAXCHUNK) return CSA2_ERR_UNSUPPORTED;
  using SM = Smem<NT, MAXCHUNK, SURV>;
  static PerDevice<cudaError_t> opt_in;
  const cudaError_t attr = opt_in.get([] {
    const cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel<NT, MAXCHUNK, SURV>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(sizeof(SM)));
    if (e != cudaSuccess) cudaGetLastError();
    return e;
  });
  if (attr != cudaSuccess) return fail(CSA2_ERR_CUDA, "select_topk_cluster: shared-memory opt-in failed");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(rows * kC));
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = sizeof(SM);
  cfg.stream = stream;
  cudaLaunchAttribute at[1] = {pdl_attribute()};
  cfg.attrs = at;
  cfg.numAttrs = 1;
  begin_launch(stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel<NT, MAXCHUNK, SURV>, p);
  note_launch(LK_TOPK, 1, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(CSA2_ERR_CUDA, "select_topk_cluster: launch failed: %s", cudaGetErrorString(e));
  }
  return check_launch("select_topk_cluster");
}

}  // namespace

// Clusters of 8 CTAs win while they all run at once (a few rows; measured
// on B200: 8 rows of 16384 keys in about 12 us, against 16 us on one CTA per
// row).  With more rows they run in waves, and rows of at most
// kSelectCtaMaxL keys go to one CTA each instead (32 rows of 16384: 35 ->
// 18 us; 64 rows of 32768: 55 -> 22 us).
constexpr int64_t kClusterMaxRows = 16;

bool select_topk_cluster_applies(int64_t rows, int64_t L, int count0, int count1) {
  return count1 <= 0 && count0 > 0 && rows > 0 && rows < sm_count() && L > 0 &&
         (rows <= kClusterMaxRows || L > kSelectCtaMaxL) &&
         L <= static_cast<int64_t>(kC) * kLargeChunk && !getenv("CSA2_TOPK_NO_CLUSTER");
}

csa2_status launch_select_topk_cluster(const float* scores, int64_t rows, int64_t L, int count,
                                       const int32_t* ids, int32_t* out, cudaStream_t stream,
                                       const int32_t* gather, int64_t src_stride) {
  if (!select_topk_cluster_applies(rows, L, count, 0)) return CSA2_ERR_UNSUPPORTED;
  ClParams p;
  p.scores = scores;
  p.L = L;
  p.count = count;
  p.ids = ids;
  p.out = out;
  p.gather = gather;
  p.src_stride = gather ? src_stride : L;
  if (L <= static_cast<int64_t>(kC) * kSmallChunk)
    return launch_variant<kSmallThreads, kSmallChunk, kSmallSurv>(p, rows, stream);
  return launch_variant<kLargeThreads, kLargeChunk, kLargeSurv>(p, rows, stream);
}

}  // namespace csa2
