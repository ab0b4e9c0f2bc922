// Top-k selection with one CTA of 1024 threads per row, for rows of up to
// 32768 scores (the hierarchical indexer's pool in a Reindex layer, decode
// rows of short contexts).  Sources: "读完这篇，你就搞懂 DeepSeek v4 了",
// 闪电索引机制 (keep the k best entries); "Recall之王", Hierarchical Sparse
// Indexer, and the V4.1 Flash transcript's hierarchical-indexer paragraph (a
// Full layer's pool and its own top-k, selected from the same scores).
//
// Order: score descending, ties to the lower position; -inf and NaN are never
// chosen; -0 and +0 are the same score.  The row's scores become
// order-preserving 32-bit keys in shared memory (read from memory once; key 0
// = not selectable).  Pass 0 histograms the 11 bits right below the bits that
// every selectable key shares.  For each selection ("track": a launch can
// select the pool and the top-k of the same row) the bin holding its
// count-th largest key is found and that bin's keys are copied to a short
// candidate list; further 11-bit passes over the candidates fix the threshold
// key T and how many keys equal to T are taken (the lowest positions first).
// A bin too large for the list is refined over the whole row instead.  Each
// warp then walks its 1/32 of the row in position order and writes the
// selected positions at offsets from one scan over the warps.  Integer counts
// only: the result is deterministic and independent of the other rows.
#include <cstdint>
#include <mutex>

#include "common.cuh"
#include "launchers.h"

namespace csa2 {
namespace {

constexpr int NT = 1024;
constexpr int NW = NT / 32;
constexpr int kDigit = 11;
constexpr int kBins = 1 << kDigit;         // 2 bins per thread
constexpr int kMaxCand = 4096;             // candidate keys per track
constexpr int kTracks = 2;

struct CtaParams {
  const float* scores;
  int64_t L;
  int seg;                                 // keys per warp segment (multiple of 128)
  int ntracks;
  int count[kTracks];
  const int32_t* ids;
  int32_t* out[kTracks];
};

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (f != f || u == 0xff800000u) return 0u;       // NaN, -inf: never chosen
  if (u == 0x80000000u) u = 0u;                    // -0 ranks as +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Smem {
  int hist[kTracks][kBins];
  uint32_t cand[kTracks][kMaxCand];
  int ws[NW + 1];
  int seg_gt[kTracks][NW], seg_eq[kTracks][NW];
  int off_sel[kTracks][NW], off_eq[kTracks][NW];
  uint32_t kmin, kmax;
  int nsel;                                // selectable keys in the row
  int ncand[kTracks];
  int bin[kTracks], above[kTracks];
};

// Exclusive block-wide prefix sum (thread order) of one int; *total = sum.
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
    const int s = ws[lane];
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    ws[lane] = incl - s;
    if (lane == 31) ws[NW] = incl;
  }
  __syncthreads();
  const int res = ws[wid] + x - v;
  *total = ws[NW];
  __syncthreads();
  return res;
}

// Finds, in hist[0..bins) (bins <= kBins), the bin holding the kk-th largest
// key: sets *bin and *above (keys in higher bins).  Every thread calls it.
__device__ __forceinline__ void find_bin(const int* hist, int bins, int kk, int* ws, int* bin_out,
                                         int* above_out) {
  const int b0 = 2 * threadIdx.x;
  const int h0 = b0 < bins ? hist[b0] : 0, h1 = b0 + 1 < bins ? hist[b0 + 1] : 0;
  int total;
  const int before = block_scan(h0 + h1, ws, &total);
  int above = total - before - h0 - h1;             // keys in bins of higher threads
  if (above < kk && above + h1 >= kk) {
    *bin_out = b0 + 1;
    *above_out = above;
  }
  above += h1;
  if (above < kk && above + h0 >= kk) {
    *bin_out = b0;
    *above_out = above;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(NT, 1) topk_cta_kernel(CtaParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + ((sizeof(Smem) + 15) & ~size_t(15)));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t r = blockIdx.x;
  const int L = static_cast<int>(p.L);
  const float* s = p.scores + r * p.L;
  const int w_lo = warp * p.seg, w_hi = min(L, w_lo + p.seg);
  pdl_wait();                                // the scores come from the kernel before
  pdl_release();

  if (tid == 0) {
    S.kmin = 0xffffffffu;
    S.kmax = 0u;
    S.nsel = 0;
  }
  for (int i = tid; i < kTracks * kBins; i += NT) (&S.hist[0][0])[i] = 0;
  __syncthreads();

  // ---- keys of this warp's segment; the row's smallest / largest selectable key
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  int nsel = 0;
  const bool vec = (reinterpret_cast<uintptr_t>(s) & 15u) == 0;
  // four groups of 128 scores per step: each lane has its four loads in flight
  for (int b0 = w_lo; b0 < w_hi; b0 += 4 * 128) {
    float f[4][4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const int i = b0 + g * 128 + 4 * lane;
      if (vec && i + 3 < w_hi) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(s + i));
        f[g][0] = v.x; f[g][1] = v.y; f[g][2] = v.z; f[g][3] = v.w;
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) f[g][u] = i + u < w_hi ? __ldg(s + i + u) : __int_as_float(0xff800000);
      }
    }
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const int i = b0 + g * 128 + 4 * lane;
      if (i >= w_lo + p.seg) break;                 // past this warp's part of the buffer
      uint32_t k4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        k4[u] = score_key(f[g][u]);
        if (k4[u]) {
          kmin = min(kmin, k4[u]);
          kmax = max(kmax, k4[u]);
          ++nsel;
        }
      }
      *reinterpret_cast<uint4*>(keys + i) = make_uint4(k4[0], k4[1], k4[2], k4[3]);
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
  __syncthreads();
  const uint32_t rmin = S.kmin, rmax = S.kmax;
  const int total_sel = S.nsel;

  // ---- per track: threshold key T[t], and how many keys equal to T[t] to take
  uint32_t T[kTracks] = {0u, 0u};
  int take[kTracks] = {0, 0};
  int eqcnt[kTracks] = {0, 0};             // keys equal to T[t] in the row
  bool all[kTracks] = {true, true};        // every selectable key is chosen
  int kk[kTracks];
  uint32_t prefix[kTracks], mask[kTracks];
  bool in_cand[kTracks] = {false, false};
  const int common = rmax >= rmin ? __clz(rmin ^ rmax) : 32;   // 32: at most one distinct key
  const uint32_t cmask = common >= 32 ? 0xffffffffu : (common == 0 ? 0u : ~0u << (32 - common));
  bool any = false;
#pragma unroll
  for (int t = 0; t < kTracks; ++t) {
    kk[t] = p.count[t];
    prefix[t] = rmin & cmask;
    mask[t] = cmask;
    if (t < p.ntracks && total_sel > p.count[t]) {
      all[t] = false;
      any = true;
    }
  }
  int lowbit = 32 - common;                // key bits [lowbit-1 : 0] still undecided
  if (any && lowbit == 0) {                // one distinct key, more of it than wanted
#pragma unroll
    for (int t = 0; t < kTracks; ++t) T[t] = rmin, take[t] = kk[t], eqcnt[t] = total_sel;
  } else if (any) {
    // pass 0 over the whole row (one histogram serves both tracks)
    int width = lowbit >= kDigit ? kDigit : lowbit;
    int shift = lowbit - width;
    for (int b0 = w_lo; b0 < w_hi; b0 += 128) {
      const int i = b0 + 4 * lane;
      const uint4 k4 = *reinterpret_cast<const uint4*>(keys + i);
      const uint32_t kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (kv[u] && i + u < w_hi) atomicAdd(&S.hist[0][(kv[u] >> shift) & ((1u << width) - 1)], 1);
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < kTracks; ++t)
      if (!all[t]) find_bin(S.hist[0], 1 << width, kk[t], S.ws, &S.bin[t], &S.above[t]);
#pragma unroll
    for (int t = 0; t < kTracks; ++t) {
      if (all[t]) continue;
      const int b = S.bin[t];
      prefix[t] |= static_cast<uint32_t>(b) << shift;
      mask[t] |= ((1u << width) - 1) << shift;
      kk[t] -= S.above[t];
      in_cand[t] = S.hist[0][b] <= kMaxCand;
      eqcnt[t] = S.hist[0][b];
    }
    __syncthreads();
    if (tid < kTracks) S.ncand[tid] = 0;
    __syncthreads();
    // candidate lists: the keys of each track's bin
    if (shift > 0 && (in_cand[0] || in_cand[1])) {
      for (int b0 = w_lo; b0 < w_hi; b0 += 128) {
        const int i = b0 + 4 * lane;
        const uint4 k4 = *reinterpret_cast<const uint4*>(keys + i);
        const uint32_t kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int t = 0; t < kTracks; ++t) {
          if (!in_cand[t]) continue;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const bool m = kv[u] && i + u < w_hi && (kv[u] & mask[t]) == prefix[t];
            const unsigned bal = __ballot_sync(0xffffffffu, m);
            int base = 0;
            if (lane == 0 && bal) base = atomicAdd(&S.ncand[t], __popc(bal));
            base = __shfl_sync(0xffffffffu, base, 0);
            if (m) S.cand[t][base + __popc(bal & ((1u << lane) - 1u))] = kv[u];
          }
        }
      }
      __syncthreads();
    }
    lowbit = shift;
    // refinement passes over the candidates (or the whole row)
    while (lowbit > 0) {
      width = lowbit >= kDigit ? kDigit : lowbit;
      shift = lowbit - width;
      for (int i = tid; i < kTracks * kBins; i += NT) (&S.hist[0][0])[i] = 0;
      __syncthreads();
#pragma unroll
      for (int t = 0; t < kTracks; ++t) {
        if (all[t]) continue;
        const uint32_t* src = in_cand[t] ? S.cand[t] : keys;
        const int n = in_cand[t] ? S.ncand[t] : L;
        for (int i = tid; i < n; i += NT) {
          const uint32_t key = src[i];
          if (key && (key & mask[t]) == prefix[t])
            atomicAdd(&S.hist[t][(key >> shift) & ((1u << width) - 1)], 1);
        }
      }
      __syncthreads();
#pragma unroll
      for (int t = 0; t < kTracks; ++t)
        if (!all[t]) find_bin(S.hist[t], 1 << width, kk[t], S.ws, &S.bin[t], &S.above[t]);
#pragma unroll
      for (int t = 0; t < kTracks; ++t) {
        if (all[t]) continue;
        prefix[t] |= static_cast<uint32_t>(S.bin[t]) << shift;
        mask[t] |= ((1u << width) - 1) << shift;
        kk[t] -= S.above[t];
        eqcnt[t] = S.hist[t][S.bin[t]];
      }
      __syncthreads();
      lowbit = shift;
    }
#pragma unroll
    for (int t = 0; t < kTracks; ++t) T[t] = prefix[t], take[t] = kk[t];
  }

  // ---- ordered write.  One selection whose keys equal to T are all taken (the
  // usual case): one sweep compacts each warp's picks, in order, into its own
  // part of the key buffer (never past the keys it has read), then offsets
  // over the warps and coalesced copies.  Otherwise: per-warp counts of keys
  // above / equal to T, offsets, and a sweep that ranks the equal keys.
#pragma unroll
  for (int t = 0; t < kTracks; ++t) {
    if (t >= p.ntracks) break;
    const bool simple = p.ntracks == 1 && (all[t] || take[t] >= eqcnt[t]);
    const uint32_t thr = all[t] ? 1u : T[t];
    int g = 0, e = 0;
    if (simple) {
      const unsigned lt = (1u << lane) - 1u;
      for (int b0 = w_lo; b0 < w_hi; b0 += 128) {
        const int i = b0 + 4 * lane;
        const uint4 k4 = *reinterpret_cast<const uint4*>(keys + i);
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
          if ((sel_m >> u) & 1) keys[w_lo + q++] = static_cast<uint32_t>(i + u);
        g += total;
      }
    } else {
      for (int b0 = w_lo; b0 < w_hi; b0 += 128) {
        const int i = b0 + 4 * lane;
        const uint4 k4 = *reinterpret_cast<const uint4*>(keys + i);
        const uint32_t kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const bool valid = kv[u] != 0u && i + u < w_hi;
          g += (valid && (all[t] || kv[u] > T[t])) ? 1 : 0;
          e += (valid && !all[t] && kv[u] == T[t]) ? 1 : 0;
        }
      }
      g = __reduce_add_sync(0xffffffffu, g);
      e = __reduce_add_sync(0xffffffffu, e);
    }
    if (lane == 0) {
      S.seg_gt[t][warp] = g;
      S.seg_eq[t][warp] = e;
    }
  }
  __syncthreads();
  if (warp < p.ntracks) {
    const int t = warp;
    int g = S.seg_gt[t][lane], e = S.seg_eq[t][lane];
    int gi = g, ei = e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yg = __shfl_up_sync(0xffffffffu, gi, o), ye = __shfl_up_sync(0xffffffffu, ei, o);
      if (lane >= o) {
        gi += yg;
        ei += ye;
      }
    }
    const int g_before = gi - g, e_before = ei - e;
    S.off_eq[t][lane] = e_before;
    S.off_sel[t][lane] = g_before + min(e_before, take[t]);
  }
  __syncthreads();
#pragma unroll
  for (int t = 0; t < kTracks; ++t) {
    if (t >= p.ntracks) break;
    int32_t* o = p.out[t] + r * static_cast<int64_t>(p.count[t]);
    const int sel_start = S.off_sel[t][warp];
    const bool simple = p.ntracks == 1 && (all[t] || take[t] >= eqcnt[t]);
    if (simple) {
      for (int j = lane; j < S.seg_gt[t][warp]; j += 32) {
        const int q = sel_start + j;
        const int posn = static_cast<int>(keys[w_lo + j]);
        if (q < p.count[t]) o[q] = p.ids ? p.ids[r * p.L + posn] : posn;
      }
      continue;
    }
    int run_sel = sel_start, run_eq = S.off_eq[t][warp];
    const unsigned lt = (1u << lane) - 1u;
    for (int b0 = w_lo; b0 < w_hi; b0 += 128) {
      const int i = b0 + 4 * lane;
      const uint4 k4 = *reinterpret_cast<const uint4*>(keys + i);
      const uint32_t kv[4] = {k4.x, k4.y, k4.z, k4.w};
      int sel_m = 0, eq_m = 0;                 // bit u: key u is above / equal to T
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool valid = kv[u] != 0u && i + u < w_hi;
        sel_m |= (valid && (all[t] || kv[u] > T[t])) << u;
        eq_m |= (valid && !all[t] && kv[u] == T[t]) << u;
      }
      // position order is lane-major: the keys of lower lanes, then this
      // lane's earlier keys, come first
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
          if (rank < take[t]) sel_m |= 1 << u;
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
          if (pos < p.count[t]) o[pos] = p.ids ? p.ids[r * p.L + i + u] : i + u;
          ++pos;
        }
      run_sel += warp_sel;
      run_eq += warp_eq;
    }
  }
  // padding: positions beyond the selectable keys
  __syncthreads();
#pragma unroll
  for (int t = 0; t < kTracks; ++t) {
    if (t >= p.ntracks) break;
    const int n_out = all[t] ? total_sel : p.count[t];
    int32_t* o = p.out[t] + r * static_cast<int64_t>(p.count[t]);
    for (int q = n_out + tid; q < p.count[t]; q += NT) o[q] = -1;
  }
}

size_t smem_bytes(int64_t L, int seg) {
  const size_t keys = static_cast<size_t>(NW) * seg * 4;
  (void)L;
  return ((sizeof(Smem) + 15) & ~size_t(15)) + keys;
}

}  // namespace

bool select_topk_cta_applies(int64_t rows, int64_t L) {
  return rows > 0 && rows <= 0x7fffffffLL && L > 0 && L <= kSelectCtaMaxL;
}

csa2_status launch_select_topk_cta(const float* scores, int64_t rows, int64_t L, int count0,
                                   const int32_t* ids, int32_t* out0, int count1, int32_t* out1,
                                   cudaStream_t stream) {
  if (!select_topk_cta_applies(rows, L)) return CSA2_ERR_UNSUPPORTED;
  CtaParams p;
  p.scores = scores;
  p.L = L;
  p.seg = static_cast<int>(((L + NW - 1) / NW + 127) / 128 * 128);
  p.ntracks = count1 > 0 ? 2 : 1;
  p.count[0] = count0;
  p.count[1] = count1 > 0 ? count1 : 0;
  p.ids = ids;
  p.out[0] = out0;
  p.out[1] = out1;
  const size_t smem = smem_bytes(L, p.seg);
  static PerDevice<cudaError_t> opt_in;
  const cudaError_t attr = opt_in.get([] {
    const cudaError_t e = cudaFuncSetAttribute(topk_cta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem_bytes(kSelectCtaMaxL, kSelectCtaMaxL / NW)));
    if (e != cudaSuccess) cudaGetLastError();
    return e;
  });
  if (attr != cudaSuccess) return fail(CSA2_ERR_CUDA, "select_topk_cta: shared-memory opt-in failed");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(rows));
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[1] = {pdl_attribute()};
  cfg.attrs = at;
  cfg.numAttrs = 1;
  begin_launch(stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, topk_cta_kernel, p);
  note_launch(LK_TOPK, 1, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(CSA2_ERR_CUDA, "select_topk_cta: launch failed: %s", cudaGetErrorString(e));
  }
  return check_launch("select_topk_cta");
}

}  // namespace csa2
