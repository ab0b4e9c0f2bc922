// Top-k selection with several CTAs per row (few long rows, e.g. decode over
// a 1M-token context), and two selections of one row in the same passes (the
// hierarchical-indexer pool and the layer's own top-k, which is a subset of
// the pool: "Recall之王", Hierarchical Sparse Indexer; V4.1 Flash transcript,
// hierarchical sparse indexer paragraph; "读完这篇，你就搞懂 DeepSeek v4 了",
// 闪电索引机制 for the top-k itself).
//
// A row of L scores is split into C chunks, one CTA each; a CTA keeps its
// chunk as order-preserving 32-bit keys in shared memory, so the scores are
// read from memory once.  The row's smallest and largest selectable keys are
// found first; the radix digits (12 bits each) start right below the bits
// they share, so the first digit spreads the keys over its bins even when the
// scores lie in a narrow range (typically two passes).  Each CTA adds its
// histogram into the row's global histogram, the row's CTAs meet at a barrier
// (a counter in global memory, bounded wait), and every CTA then derives the
// same next key prefix from the global histogram; a row held by one CTA needs
// neither.  When, after the first pass, few keys share each selection's
// threshold bin (at most kCandCap), the CTAs copy those keys and positions to
// a per-row candidate list with their counts of keys above the bin, meet once
// more, and each CTA finishes alone from the list: the remaining digits, its
// output offset and its share of the keys equal to T.  Otherwise, after the
// last pass, the threshold key T and the number
// of keys equal to T to take are known; the CTAs exchange per-chunk counts
// (one more barrier) and each writes its selected positions, in position
// order, at the offset the lower chunks leave -- ties at T go to the lowest
// positions.  Integer histograms and ordered writes make the result
// deterministic and equal to the one-CTA kernel's.
//
// The launch is cooperative (all CTAs resident); CTA groups loop over rows,
// each row having its own counter, histogram and count slots in the
// workspace; the counters and ranges are cleared before the launch, the
// histograms by the kernel itself.
#include <algorithm>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "launchers.h"
#include "sm100.cuh"

namespace csa2 {
namespace {

constexpr int kT = 512;
constexpr int kDigit = 12;                 // radix digit bits
constexpr int kBins = 1 << kDigit;
constexpr int kPasses = 3;                 // 32 bits need at most three 12-bit digits
constexpr int kTracks = 2;
constexpr int kMaxRowsMulti = 1024;
constexpr int kMaxC = 64;
constexpr int kCandCap = 4096;            // candidate keys per row and selection
static_assert(kCandCap % 512 == 0 && kCandCap < (1 << 15), "candidates per thread; packed counts");

struct SelParams {
  const float* scores;
  int64_t rows, L;
  int C, chunk, ntracks;
  int count[kTracks];
  const int32_t* ids;
  int32_t* out[kTracks];
  int* hist;          // [rows][kPasses][kTracks][kBins], cleared by the kernel
  int* cnt;           // [rows][C][kTracks][2]
  unsigned* minmax;   // [rows][2]: max of ~key (so the min), max key; zero at launch
  unsigned* bar;      // [rows], zero at launch
  uint32_t* ckey;     // [rows][kTracks][kCandCap] keys of the threshold bin after pass 0
  int32_t* cpos;      // [rows][kTracks][kCandCap] their positions
  int* ccnt;          // [rows][kTracks]
  int* err;
  unsigned long long wait_ns;   // bound of a row-barrier wait
  unsigned wait_offset;         // added to every barrier target (0, or unreachable for tests)
};

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (f != f || u == 0xff800000u) return 0u;
  if (u == 0x80000000u) u = 0u;                    // -0 ranks as +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// exclusive block-wide prefix sum (thread order) of one int; *total = sum
__device__ __forceinline__ int block_scan(int v, int* ws, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) ws[wid] = x;
  __syncthreads();
  if (wid == 0) {
    const int s = lane < kT / 32 ? ws[lane] : 0;
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane < kT / 32) ws[lane] = incl - s;
    if (lane == 31) ws[32] = incl;
  }
  __syncthreads();
  const int res = ws[wid] + x - v;
  *total = ws[32];
  __syncthreads();
  return res;
}

// Barrier of the C CTAs working on one row: arrive on the row's counter, wait
// (bounded by p.wait_ns, 1 s by default) until all have arrived `target`
// times in total.  A CTA that gave up arrives at no later barrier and takes
// no step that needs the other CTAs; they give up at their next barrier.
__device__ __forceinline__ bool row_barrier(const SelParams& p, unsigned* ctr, unsigned target,
                                            int* abort_s) {
  __syncthreads();
  if (threadIdx.x == 0 && !*abort_s) {
    __threadfence();
    atomicAdd(ctr, 1u);
    const uint64_t t0 = sm100::globaltimer_ns();
    target += p.wait_offset;
    while (*reinterpret_cast<volatile unsigned*>(ctr) < target) {
      if (sm100::globaltimer_ns() - t0 > p.wait_ns) {
        raise_dev_error(p.err, DEVERR_TIMEOUT);
        *abort_s = 1;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
  }
  __syncthreads();
  return !*abort_s;
}

__global__ void __launch_bounds__(kT, 2) topk_multi_kernel(SelParams p) {
  extern __shared__ uint32_t keys[];
  __shared__ int hist_s[kTracks][kBins];
  __shared__ int ws[33];
  __shared__ uint32_t sh_min, sh_max;
  __shared__ int sh_bin[kTracks], sh_above[kTracks], sh_total[kTracks];
  __shared__ int sh_off[kTracks], sh_take[kTracks], sh_all_sel[kTracks], sh_eqin[kTracks];
  __shared__ int seg_gt[kTracks][kT / 32], seg_eq[kTracks][kT / 32];
  __shared__ int abort_s;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int C = p.C;
  const int c = blockIdx.x % C;
  const int64_t groups = gridDim.x / C;
  if (tid == 0) abort_s = 0;
  pdl_wait();                               // the scores come from the kernel before
  pdl_release();
  __syncthreads();

  for (int64_t r = blockIdx.x / C; r < p.rows; r += groups) {
    const int64_t lo = static_cast<int64_t>(c) * p.chunk;
    const int n = static_cast<int>(std::max<int64_t>(0, std::min<int64_t>(p.L - lo, p.chunk)));
    const float* s = p.scores + r * p.L + lo;
    unsigned* ctr = p.bar + r;
    int* gh = p.hist + r * kPasses * kTracks * kBins;
    unsigned* gmm = p.minmax + r * 2;
    unsigned epoch = 0;
    bool ok = true;

    // keys, and the smallest / largest selectable key of the chunk
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    auto take_key = [&](int i, float f) {
      const uint32_t key = score_key(f);
      keys[i] = key;
      if (key != 0u) {
        kmin = min(kmin, key);
        kmax = max(kmax, key);
      }
    };
    int n_vec = 0;
    if ((reinterpret_cast<uintptr_t>(s) & 15u) == 0) {
      // 16-byte loads, four per thread in flight before any is used
      const int n4 = n >> 2;
      const float4* s4 = reinterpret_cast<const float4*>(s);
      for (int i = tid; i < n4; i += 4 * kT) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = i + u * kT;
          v[u] = j < n4 ? __ldg(s4 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = i + u * kT;
          if (j < n4) {
            take_key(4 * j, v[u].x);
            take_key(4 * j + 1, v[u].y);
            take_key(4 * j + 2, v[u].z);
            take_key(4 * j + 3, v[u].w);
          }
        }
      }
      n_vec = n4 * 4;
    }
    for (int i0 = n_vec; i0 < n; i0 += 4 * kT) {
      float v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + tid + u * kT;
        v[u] = i < n ? __ldg(s + i) : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + tid + u * kT;
        if (i < n) take_key(i, v[u]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
      kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if (tid == 0) {
      sh_min = 0xffffffffu;
      sh_max = 0u;
    }
    __syncthreads();
    if (lane == 0) {
      atomicMin(&sh_min, kmin);
      atomicMax(&sh_max, kmax);
    }
    __syncthreads();
    if (C > 1) {      // the row's range over all chunks
      // this CTA's share of the row's histograms (and, for chunk 0, the
      // candidate counters) start at zero; the barrier below publishes it
      {
        const int words = kPasses * kTracks * kBins;
        const int per = (words + C - 1) / C;
        for (int i = c * per + tid; i < min(words, (c + 1) * per); i += kT) gh[i] = 0;
        if (c == 0 && tid < kTracks) p.ccnt[r * kTracks + tid] = 0;
      }
      if (tid == 0) {
        atomicMax(&gmm[0], ~sh_min);
        atomicMax(&gmm[1], sh_max);
      }
      ok = row_barrier(p, ctr, C * (++epoch), &abort_s);
      if (tid == 0) {
        sh_min = ~__ldcg(&gmm[0]);
        sh_max = __ldcg(&gmm[1]);
      }
      __syncthreads();
    }
    const uint32_t rmin = sh_min, rmax = sh_max;
    // radix digits start right below the bits every selectable key shares
    const int common = (rmax >= rmin) ? __clz(rmin ^ rmax) : 32;   // 32: one distinct key (or none)
    uint32_t prefix[kTracks], mask[kTracks];
    int kk[kTracks] = {p.count[0], p.count[1]};
    bool all[kTracks] = {false, false};
    const uint32_t cmask = common >= 32 ? 0xffffffffu : (common == 0 ? 0u : ~0u << (32 - common));
#pragma unroll
    for (int t = 0; t < kTracks; ++t) {
      prefix[t] = rmin & cmask;
      mask[t] = cmask;
    }
    int lowbit = 32 - common;               // bits [lowbit-1 : 0] still undecided
    bool use_cand = false;
    for (int pass = 0; pass < kPasses && lowbit > 0 && ok; ++pass) {
      const int width = lowbit >= kDigit ? kDigit : lowbit;
      const int shift = lowbit - width;
      const int bins = 1 << width;
      for (int i = tid; i < kTracks * kBins; i += kT) (&hist_s[0][0])[i] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += kT) {
        const uint32_t key = keys[i];
        if (key == 0u) continue;
#pragma unroll
        for (int t = 0; t < kTracks; ++t)
          if (t < p.ntracks && !all[t] && (key & mask[t]) == prefix[t])
            atomicAdd(&hist_s[t][(key >> shift) & (bins - 1)], 1);
      }
      __syncthreads();
      int* ghp = gh + pass * kTracks * kBins;
      if (C > 1) {      // merge into the row's histogram, then meet the row's other CTAs
        for (int i = tid; i < p.ntracks * bins; i += kT) {
          const int t = i / bins, bin = i % bins;
          const int v = hist_s[t][bin];
          if (v) atomicAdd(&ghp[t * kBins + bin], v);
        }
        ok = row_barrier(p, ctr, C * (++epoch), &abort_s);
        if (!ok) break;
      }
      // every CTA derives the same next prefix from the row's histogram
      for (int t = 0; t < p.ntracks; ++t) {
        if (all[t]) continue;
        const int per = (bins + kT - 1) / kT;      // bins per thread (bins owned in order)
        int h[kBins / kT];
        int local = 0;
#pragma unroll
        for (int u = 0; u < kBins / kT; ++u) {
          const int bin = tid * per + u;
          h[u] = (u < per && bin < bins) ? (C > 1 ? __ldcg(&ghp[t * kBins + bin]) : hist_s[t][bin]) : 0;
          local += h[u];
        }
        int total;
        const int before = block_scan(local, ws, &total);   // sum over lower threads
        if (tid == 0) sh_total[t] = total;
        int above = total - before - local;                 // sum over higher threads
#pragma unroll
        for (int u = kBins / kT - 1; u >= 0; --u) {
          if (u < per && above < kk[t] && above + h[u] >= kk[t]) {
            sh_bin[t] = tid * per + u;
            sh_above[t] = above;
          }
          above += h[u];
        }
        __syncthreads();
        if (pass == 0 && sh_total[t] <= p.count[t]) {
          all[t] = true;
          continue;
        }
        prefix[t] |= static_cast<uint32_t>(sh_bin[t]) << shift;
        mask[t] |= static_cast<uint32_t>(bins - 1) << shift;
        kk[t] -= sh_above[t];
        __syncthreads();
      }
      lowbit = shift;
      if (pass == 0 && C > 1) {
        // few keys share the threshold bin of every selection: finish on those
        // candidates instead of more passes over the row (the same decision in
        // every CTA of the row: it reads the row's histogram)
        bool fits = true;
        for (int t = 0; t < p.ntracks; ++t)
          if (!all[t] && __ldcg(&ghp[t * kBins + sh_bin[t]]) > kCandCap) fits = false;
        if (fits) {
          use_cand = true;
          break;
        }
      }
    }
    int* cr = p.cnt + r * C * kTracks * 2;
    if (use_cand && ok) {
      // (1) candidates: keys of each selection's threshold bin, with their
      // positions; and this chunk's keys above that bin
      uint32_t* ck = p.ckey + r * kTracks * kCandCap;
      int32_t* cp = p.cpos + r * kTracks * kCandCap;
      int* cc = p.ccnt + r * kTracks;
      {
        uint32_t bin_max[kTracks];
#pragma unroll
        for (int t = 0; t < kTracks; ++t) bin_max[t] = prefix[t] | ~mask[t];
        int above[kTracks] = {0, 0};
        for (int i0 = 0; i0 < n; i0 += kT) {                 // one sweep serves both selections
          const int i = i0 + tid;
          const uint32_t key = i < n ? keys[i] : 0u;
#pragma unroll
          for (int t = 0; t < kTracks; ++t) {
            if (t >= p.ntracks) break;
            above[t] += (key != 0u && (all[t] || key > bin_max[t])) ? 1 : 0;
            const bool in_bin = key != 0u && !all[t] && (key & mask[t]) == prefix[t];
            const unsigned bal = __ballot_sync(0xffffffffu, in_bin);
            if (bal) {                                       // rare: the threshold bin is small
              int base = 0;
              if (lane == 0) base = atomicAdd(&cc[t], __popc(bal));
              base = __shfl_sync(0xffffffffu, base, 0);
              if (in_bin) {
                const int idx = base + __popc(bal & ((1u << lane) - 1u));
                ck[t * kCandCap + idx] = key;
                cp[t * kCandCap + idx] = static_cast<int32_t>(lo + i);
              }
            }
          }
        }
        for (int t = 0; t < p.ntracks; ++t) {
          int tot;
          block_scan(above[t], ws, &tot);
          if (tid == 0) cr[(c * kTracks + t) * 2] = tot;
        }
      }
      ok = row_barrier(p, ctr, C * (++epoch), &abort_s);
      // (2) every CTA refines the threshold over the candidates (same result)
      for (int t = 0; t < p.ntracks && ok; ++t) {
        if (all[t]) continue;
        const int nc = __ldcg(&cc[t]);
        // this thread's candidates (nc <= kCandCap = 8 per thread), loaded once
        constexpr int kPer = kCandCap / kT;
        uint32_t ckr[kPer];
        int32_t cpr[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
          const int i = tid + u * kT;
          ckr[u] = i < nc ? __ldcg(&ck[t * kCandCap + i]) : 0u;
          cpr[u] = i < nc ? __ldcg(&cp[t * kCandCap + i]) : -1;
        }
        int lb = lowbit;
        while (lb > 0) {
          const int width = lb >= kDigit ? kDigit : lb;
          const int shift = lb - width;
          const int bins = 1 << width;
          for (int i = tid; i < kBins; i += kT) hist_s[t][i] = 0;
          __syncthreads();
#pragma unroll
          for (int u = 0; u < kPer; ++u)
            if (cpr[u] >= 0 && (ckr[u] & mask[t]) == prefix[t])
              atomicAdd(&hist_s[t][(ckr[u] >> shift) & (bins - 1)], 1);
          __syncthreads();
          const int per = (bins + kT - 1) / kT;
          int h[kBins / kT];
          int local = 0;
#pragma unroll
          for (int u = 0; u < kBins / kT; ++u) {
            const int bin = tid * per + u;
            h[u] = (u < per && bin < bins) ? hist_s[t][bin] : 0;
            local += h[u];
          }
          int total;
          const int before = block_scan(local, ws, &total);
          int ab = total - before - local;
#pragma unroll
          for (int u = kBins / kT - 1; u >= 0; --u) {
            if (u < per && ab < kk[t] && ab + h[u] >= kk[t]) {
              sh_bin[t] = tid * per + u;
              sh_above[t] = ab;
            }
            ab += h[u];
          }
          __syncthreads();
          prefix[t] |= static_cast<uint32_t>(sh_bin[t]) << shift;
          mask[t] |= static_cast<uint32_t>(bins - 1) << shift;
          kk[t] -= sh_above[t];
          __syncthreads();
          lb = shift;
        }
        // (3) this chunk's offset and its share of the keys equal to T: from
        // the lower chunks' counts above the bin and the candidates' positions
        const uint32_t Tt = prefix[t];
        int gt_b = 0, eq_b = 0, eq_in = 0;
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
          const int64_t pos = cpr[u];
          if (pos < 0) continue;
          if (pos < lo) {
            gt_b += ckr[u] > Tt ? 1 : 0;
            eq_b += ckr[u] == Tt ? 1 : 0;
          } else if (pos < lo + n) {
            eq_in += ckr[u] == Tt ? 1 : 0;
          }
        }
        for (int cc2 = tid; cc2 < c; cc2 += kT) gt_b += __ldcg(&cr[(cc2 * kTracks + t) * 2]);
        int tg, tp;
        block_scan(gt_b, ws, &tg);
        block_scan(eq_b | (eq_in << 16), ws, &tp);          // both counts <= kCandCap < 2^16
        const int te = tp & 0xffff, ti = tp >> 16;
        if (tid == 0) {
          sh_off[t] = tg + min(te, kk[t]);
          sh_take[t] = max(0, min(kk[t] - te, ti));
          sh_eqin[t] = ti;
          sh_all_sel[t] = p.count[t];
        }
      }
      if (ok) {
        for (int t = 0; t < p.ntracks; ++t) {
          if (!all[t]) continue;          // every selectable key: offsets from the counts alone
          int before = 0, tot_all = 0;
          for (int cc2 = tid; cc2 < C; cc2 += kT) {
            const int v = __ldcg(&cr[(cc2 * kTracks + t) * 2]);
            if (cc2 < c) before += v;
            tot_all += v;
          }
          int tb, ta;
          block_scan(before, ws, &tb);
          block_scan(tot_all, ws, &ta);
          if (tid == 0) {
            sh_off[t] = tb;
            sh_take[t] = 0;
            sh_all_sel[t] = ta;
          }
        }
      }
      __syncthreads();
    }
    if (common >= 32 && ok) {               // every selectable key is the same value
#pragma unroll
      for (int t = 0; t < kTracks; ++t) {
        prefix[t] = rmin;
        if (rmax < rmin) all[t] = true;     // nothing selectable at all
      }
    }

    // Candidate path, every selection taking all of this chunk's keys equal to
    // its T: one sweep per selection compacts the picks, in order, into the
    // (now free) histogram space, then per-warp offsets and coalesced copies.
    bool simple = use_cand && ok;
    for (int t = 0; t < p.ntracks; ++t)
      if (!all[t] && sh_take[t] != sh_eqin[t]) simple = false;
    if (simple) {
      const unsigned ltm = (1u << lane) - 1u;
      const int sseg = (((n + kT / 32 - 1) / (kT / 32)) + 31) & ~31;
      const int s_lo = std::min(n, warp * sseg), s_hi = std::min(n, s_lo + sseg);
      int* stage = &hist_s[0][0];                 // kTracks * kBins >= n ints
      for (int t = 0; t < p.ntracks; ++t) {
        const uint32_t thr = all[t] ? 1u : prefix[t];
        int cnt = 0;
        for (int i0 = s_lo; i0 < s_hi; i0 += 32) {
          const int i = i0 + lane;
          const uint32_t key = i < s_hi ? keys[i] : 0u;
          const bool sel = key >= thr;
          const unsigned sb = __ballot_sync(0xffffffffu, sel);
          if (sel) stage[s_lo + cnt + __popc(sb & ltm)] = static_cast<int>(lo + i);
          cnt += __popc(sb);
        }
        if (lane == 0) seg_gt[t][warp] = cnt;
        __syncthreads();
        int before = 0;
        for (int w2 = 0; w2 < warp; ++w2) before += seg_gt[t][w2];
        int32_t* o = p.out[t] + r * static_cast<int64_t>(p.count[t]);
        for (int j = lane; j < cnt; j += 32) {
          const int q = sh_off[t] + before + j;
          const int posn = stage[s_lo + j];
          if (q < p.count[t]) o[q] = p.ids ? p.ids[r * p.L + posn] : posn;
        }
        if (c == C - 1)
          for (int q = sh_all_sel[t] + tid; q < p.count[t]; q += kT) o[q] = -1;
        __syncthreads();
      }
    } else {
    // per-chunk counts of keys above / equal to each threshold, per warp
    // segment (16 contiguous segments of the chunk, one per warp)
    const unsigned lt_mask = (1u << lane) - 1u;
    const int seg = (((n + kT / 32 - 1) / (kT / 32)) + 31) & ~31;
    const int w_lo = std::min(n, warp * seg), w_hi = std::min(n, w_lo + seg);
    uint32_t T[kTracks];
    int need_eq[kTracks];
    for (int t = 0; t < kTracks; ++t) {
      T[t] = all[t] ? 0u : prefix[t];
      need_eq[t] = all[t] ? 0 : kk[t];
      int g = 0, e = 0;
      if (t < p.ntracks)
        for (int i0 = w_lo; i0 < w_hi; i0 += 32) {
          const int i = i0 + lane;
          const uint32_t key = i < w_hi ? keys[i] : 0u;
          g += __popc(__ballot_sync(0xffffffffu, key != 0u && key > T[t]));
          e += __popc(__ballot_sync(0xffffffffu, key != 0u && key == T[t]));
        }
      if (lane == 0) {
        seg_gt[t][warp] = g;
        seg_eq[t][warp] = e;
      }
    }
    __syncthreads();
    if (!use_cand && tid < kTracks) {
      int g = 0, e = 0;
      for (int w = 0; w < kT / 32; ++w) {
        g += seg_gt[tid][w];
        e += seg_eq[tid][w];
      }
      cr[(c * kTracks + tid) * 2] = g;
      cr[(c * kTracks + tid) * 2 + 1] = e;
    }
    if (ok && C > 1 && !use_cand) ok = row_barrier(p, ctr, C * (++epoch), &abort_s);
    __syncthreads();
    if (tid < p.ntracks && ok && !use_cand) {
      int off = 0, eq_left = need_eq[tid], take = 0, all_sel = 0;
      for (int cc = 0; cc < C; ++cc) {
        const int g = __ldcg(&cr[(cc * kTracks + tid) * 2]);
        const int e = __ldcg(&cr[(cc * kTracks + tid) * 2 + 1]);
        const int tk = std::min(e, std::max(eq_left, 0));
        if (cc == c) {
          sh_off[tid] = off;
          take = tk;
        }
        off += g + tk;
        eq_left -= tk;
        all_sel = off;
      }
      sh_take[tid] = take;
      sh_all_sel[tid] = all_sel;
    }
    __syncthreads();
    if (ok) {
      for (int t = 0; t < p.ntracks; ++t) {
        int32_t* o = p.out[t] + r * static_cast<int64_t>(p.count[t]);
        const int take = sh_take[t];
        // this warp's place among the chunk's selected keys (lower warps first)
        int eq_before = 0, sel_before = 0;
        for (int w = 0; w < warp; ++w) {
          const int tk = std::min(seg_eq[t][w], std::max(take - eq_before, 0));
          sel_before += seg_gt[t][w] + tk;
          eq_before += seg_eq[t][w];
        }
        int run_eq = eq_before, run_sel = sh_off[t] + sel_before;
        for (int i0 = w_lo; i0 < w_hi; i0 += 32) {
          const int i = i0 + lane;
          const uint32_t key = i < w_hi ? keys[i] : 0u;
          const bool gt = key != 0u && key > T[t];
          const bool eq = key != 0u && key == T[t];
          const unsigned eb = __ballot_sync(0xffffffffu, eq);
          const bool sel = gt || (eq && run_eq + __popc(eb & lt_mask) < take);
          const unsigned sb = __ballot_sync(0xffffffffu, sel);
          const int pos = run_sel + __popc(sb & lt_mask);
          if (sel && pos < p.count[t])
            o[pos] = p.ids ? p.ids[r * p.L + lo + i] : static_cast<int32_t>(lo + i);
          run_eq += __popc(eb);
          run_sel += __popc(sb);
        }
        if (c == C - 1)
          for (int q = sh_all_sel[t] + tid; q < p.count[t]; q += kT) o[q] = -1;
      }
    }
    }  // not simple
    __syncthreads();
  }
}

// Rows up to kOneCtaKeys keys are selected by one CTA (no cross-CTA
// barriers); longer rows are split into chunks of kChunkKeys.
constexpr int kOneCtaKeys = 32768;
constexpr int kChunkKeys = 8192;
int chunk_for(int64_t L) { return L <= kOneCtaKeys ? static_cast<int>(L) : kChunkKeys; }

int max_resident_ctas(size_t smem) {
  struct PerSm {
    int small_chunk, one_cta_row;
  };
  static PerDevice<PerSm> cache;
  const PerSm per_sm = cache.get([] {
    PerSm r{0, 0};
    if (cudaFuncSetAttribute(topk_multi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kOneCtaKeys * 4) != cudaSuccess) {
      cudaGetLastError();
      return r;
    }
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&r.small_chunk, topk_multi_kernel, kT,
                                                      kChunkKeys * 4) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&r.one_cta_row, topk_multi_kernel, kT,
                                                      kOneCtaKeys * 4) != cudaSuccess) {
      cudaGetLastError();
      r = PerSm{0, 0};
    }
    return r;
  });
  return (smem > kChunkKeys * 4 ? per_sm.one_cta_row : per_sm.small_chunk) * sm_count();
}

// The one-CTA kernel of topk_cta.cu takes rows of up to kSelectCtaMaxL keys
// unless CSA2_TOPK_NO_CTA is set (tests: this kernel's one-chunk path).
bool cta_kernel_takes(int64_t rows, int64_t L) {
  return select_topk_cta_applies(rows, L) && !getenv("CSA2_TOPK_NO_CTA");
}

bool multi_applies(int64_t rows, int64_t L) {
  if (getenv("CSA2_TOPK_ONE_CTA") || cta_kernel_takes(rows, L)) return false;
  if (rows <= 0 || rows > kMaxRowsMulti || L < 2048) return false;
  const int64_t C = (L + chunk_for(L) - 1) / chunk_for(L);
  return C <= kMaxC;
}

// Workspace: [minmax | bar] (cleared before each launch), then [hist | ccnt]
// (cleared by the kernel itself before its first barrier), [cnt] and the
// candidate lists [ckey | cpos] (written before being read).
size_t ws_cleared_bytes(int64_t rows) {
  return (static_cast<size_t>(rows) * 3 * 4 + 255) & ~size_t(255);
}

size_t ws_bytes_for(int64_t rows, int64_t L) {
  const int64_t C = (L + chunk_for(L) - 1) / chunk_for(L);
  const size_t words = static_cast<size_t>(rows) * (kPasses * kTracks * kBins + kTracks + C * kTracks * 2);
  return ws_cleared_bytes(rows) + ((words * 4 + 255) & ~size_t(255)) +
         static_cast<size_t>(rows) * kTracks * kCandCap * 8 + 256;
}

}  // namespace

size_t select_topk_multi_workspace(int64_t rows, int64_t L, int) {
  return multi_applies(rows, L) ? ws_bytes_for(rows, L) : 0;
}

size_t select_topk_scratch_bytes(int64_t rows, int64_t L, int count) {
  if (rows <= 0 || count <= 0 || select_topk_cluster_applies(rows, L, count, 0)) return 0;
  return multi_applies(rows, L) ? ws_bytes_for(rows, L) : 0;
}

// Up to two selections of the same rows (count1 may be 0 for one).
csa2_status launch_select_topk2(const float* scores, int64_t rows, int64_t L, int count0,
                                const int32_t* ids, int32_t* out0, int count1, int32_t* out1,
                                void* ws, size_t ws_bytes, cudaStream_t stream, bool ws_cleared) {
  if (select_topk_cluster_applies(rows, L, count0, count1))
    return launch_select_topk_cluster(scores, rows, L, count0, ids, out0, stream);
  if (count0 > 0 && count1 > 0 && !ids &&
      select_topk_cluster_applies(rows, L, std::max(count0, count1), 0)) {
    // The smaller selection lies inside the larger one (same order, same tie
    // rule), so it runs over the larger one's positions: pool, then top-k.
    const bool first_big = count0 >= count1;
    const int big = first_big ? count0 : count1, small = first_big ? count1 : count0;
    int32_t* out_big = first_big ? out0 : out1;
    int32_t* out_small = first_big ? out1 : out0;
    CSA2_TRY(launch_select_topk_cluster(scores, rows, L, big, nullptr, out_big, stream));
    return launch_select_topk_cluster(scores, rows, big, small, out_big, out_small, stream, out_big, L);
  }
  if (cta_kernel_takes(rows, L))
    return launch_select_topk_cta(scores, rows, L, count0, ids, out0, count1, out1, stream);
  if (!multi_applies(rows, L)) return CSA2_ERR_UNSUPPORTED;
  const int chunk = chunk_for(L);
  const int C = static_cast<int>((L + chunk - 1) / chunk);
  const size_t need = ws_bytes_for(rows, L);
  if (!ws || ws_bytes < need) return CSA2_ERR_UNSUPPORTED;
  const int cap = max_resident_ctas(static_cast<size_t>(chunk) * 4);
  if (cap < C) return CSA2_ERR_UNSUPPORTED;
  const int64_t groups = std::min<int64_t>(rows, cap / C);
  SelParams p;
  p.scores = scores;
  p.rows = rows;
  p.L = L;
  p.C = C;
  p.chunk = chunk;
  p.ntracks = count1 > 0 ? 2 : 1;
  p.count[0] = count0;
  p.count[1] = count1;
  p.ids = ids;
  p.out[0] = out0;
  p.out[1] = out1;
  const size_t cleared = ws_cleared_bytes(rows);
  p.minmax = static_cast<unsigned*>(ws);
  p.bar = p.minmax + rows * 2;
  p.hist = reinterpret_cast<int*>(static_cast<char*>(ws) + cleared);
  p.ccnt = p.hist + rows * kPasses * kTracks * kBins;
  p.cnt = p.ccnt + rows * kTracks;
  const size_t words = static_cast<size_t>(rows) * (kPasses * kTracks * kBins + kTracks + C * kTracks * 2);
  p.ckey = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + cleared + ((words * 4 + 255) & ~size_t(255)));
  p.cpos = reinterpret_cast<int32_t*>(p.ckey + rows * kTracks * kCandCap);
  p.err = device_error_word();
  p.wait_ns = cross_cta_wait_ns();
  p.wait_offset = cross_cta_wait_offset();
  if (C > 1 && !ws_cleared) {          // row ranges and barrier counters start at zero
    begin_launch(stream);
    if (cudaMemsetAsync(ws, 0, cleared, stream) != cudaSuccess) return check_launch("select_topk: clear");
    note_launch(LK_OTHER, 1, stream);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(groups * C));
  cfg.blockDim = dim3(kT);
  cfg.dynamicSmemBytes = static_cast<size_t>(chunk) * 4;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  at[1] = pdl_attribute();
  cfg.attrs = at;
  cfg.numAttrs = 2;
  begin_launch(stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, topk_multi_kernel, p);
  note_launch(LK_TOPK, 1, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(CSA2_ERR_CUDA, "select_topk: cooperative launch failed: %s", cudaGetErrorString(e));
  }
  return check_launch("select_topk_multi");
}

ClearOnLaunch select_topk_clear_region(int64_t rows, int64_t L, void* ws, size_t ws_bytes) {
  ClearOnLaunch c;
  if (cta_kernel_takes(rows, L) || !multi_applies(rows, L) || !ws || ws_bytes < ws_bytes_for(rows, L))
    return c;
  if ((L + chunk_for(L) - 1) / chunk_for(L) <= 1) return c;
  c.ptr = static_cast<uint32_t*>(ws);
  c.words = static_cast<int>(ws_cleared_bytes(rows) / 4);
  return c;
}

csa2_status select_topk_clear(int64_t rows, int64_t L, void* ws, size_t ws_bytes,
                              cudaStream_t stream) {
  if (cta_kernel_takes(rows, L) || !multi_applies(rows, L) || !ws || ws_bytes < ws_bytes_for(rows, L))
    return CSA2_OK;
  const int64_t C = (L + chunk_for(L) - 1) / chunk_for(L);
  if (C <= 1) return CSA2_OK;
  begin_launch(stream);
  if (cudaMemsetAsync(ws, 0, ws_cleared_bytes(rows), stream) != cudaSuccess)
    return check_launch("select_topk: clear");
  note_launch(LK_OTHER, 1, stream);
  return CSA2_OK;
}

csa2_status launch_select_topk_multi(const float* scores, int64_t rows, int64_t L, int count,
                                     const int32_t* ids, int32_t* out, void* ws, size_t ws_bytes,
                                     cudaStream_t stream) {
  return launch_select_topk2(scores, rows, L, count, ids, out, 0, nullptr, ws, ws_bytes, stream);
}

}  // namespace csa2
