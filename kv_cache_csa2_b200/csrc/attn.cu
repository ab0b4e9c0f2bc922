// Shared-KV sparse attention over the selected entries.
// Source: "读完这篇，你就搞懂 DeepSeek v4 了", 注意力计算 (eq. 9): standard
// attention in which every query head uses the same compressed entries as
// keys and values, restricted to the indexer's top-k; FP4 rows ("Recall之王",
// FP4 主KV缓存) are dequantised in the kernel.
//
// This file holds the CUDA-core kernel: one CTA per query, the query's heads
// in shared memory, the selected rows staged 16 at a time (f32, padded
// stride), an online softmax per head and the per-head outputs in registers.
// It serves every shape; the tensor-core kernels take the shapes they
// support first (attn_tc.cu / attn_seq.cu: 64 heads x 512 bf16;
// attn_narrow.cu: entries of width 128), so this kernel runs the rest (width
// 512 with 16 or 32 heads, FP4 at 64 x 512).  The reduction order per query
// is fixed (rows in list order, 16 at a time), so a query's result does not
// depend on B or Q.
#include <algorithm>

#include "common.cuh"
#include "launchers.h"

namespace csa2 {

csa2_status launch_sparse_attn_tc(const void* q, const csa2_kv& kv, const int32_t* topk, int B,
                                  int Q, int Ha, int k, float scale, void* out, float* lse,
                                  void* ws, size_t ws_bytes, unsigned long long* sync_zeroed,
                                  cudaStream_t stream, const AttnRows& rows);
size_t sparse_attn_tc_workspace(int B, int Q, int Ha, int D, int k, csa2_kv_fmt fmt, bool win);

namespace {

constexpr int kT = 256;
constexpr int kR = 16;  // rows staged per step

template <int HA, int DD>
struct AttnSmem {
  static constexpr int RS = DD + 1;  // padded f32 row stride: conflict-free column reads
  static constexpr size_t q_words = HA * DD / 2;
  static constexpr size_t bytes = q_words * 4 + size_t(kR) * RS * 4 + size_t(HA) * (kR + 1) * 4 +
                                  3 * HA * 4 + 2 * kR * 4;
};

// The row sources of launch_sparse_attn (AttnRows) as the kernel takes them,
// and the split of a query's rows over CTAs.
struct SimtRows {
  const int32_t* n_visible;
  const uint16_t* win;
  int64_t win_rows;
  const int32_t* win_end;
  int W;
  int Q;              // queries per sequence
  int64_t q_base;     // first query (flat b * Q + q) of this launch
  int n_chunks;       // CTAs per query; 1: one CTA takes every row and writes the output
  int chunk_rows;     // rows (slots) per CTA, a multiple of kR
  float* part;        // [queries of the launch][n_chunks][HA * DD + 2 HA]: sums, max, row sum
  unsigned* counters; // [queries of the launch], zero before the launch, left zero after it
};

// weight of a partial with max m in a sum whose max is M (0 for empty partials)
__device__ __forceinline__ float rescale_part(float m, float M) {
  return (m == -INFINITY || M == -INFINITY) ? 0.0f : expf(m - M);
}

template <int HA, int DD, bool FP4>
__global__ void __launch_bounds__(kT) attn_simt_kernel(
    const uint16_t* __restrict__ q, const void* __restrict__ kv_data,
    const uint8_t* __restrict__ kv_scales, int64_t n, const int32_t* __restrict__ topk, int k,
    float scale, uint16_t* __restrict__ out, float* __restrict__ lse, int* err, SimtRows rs) {
  using S = AttnSmem<HA, DD>;
  constexpr int TPH = kT / HA;      // threads per head in the accumulation
  constexpr int OPT = DD / TPH;     // outputs per thread
  constexpr int PAIRS = HA * kR / kT;
  static_assert(kT % HA == 0 && DD % TPH == 0 && (HA * kR) % kT == 0, "shape");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint32_t* q_s = reinterpret_cast<uint32_t*>(smem_raw);
  float* rows_s = reinterpret_cast<float*>(q_s + S::q_words);
  float* p_s = rows_s + kR * S::RS;           // [HA][kR+1]
  float* m_s = p_s + HA * (kR + 1);
  float* l_s = m_s + HA;
  float* a_s = l_s + HA;
  int* id_s = reinterpret_cast<int*>(a_s + HA);   // [kR] row ids; [kR] their source (1 = window)
  int* src_s = id_s + kR;

  __shared__ int last_s;
  const int tid = threadIdx.x;
  const int64_t ql = blockIdx.x / rs.n_chunks;                      // query within the launch
  const int chunk = static_cast<int>(blockIdx.x % rs.n_chunks);
  const int64_t qi = rs.q_base + ql;                                // flat (b, q)
  const int64_t seq = qi / rs.Q;                                    // sequence b
  const uint32_t* qg = reinterpret_cast<const uint32_t*>(q + qi * HA * DD);
  for (int i = tid; i < HA * DD / 2; i += kT) q_s[i] = qg[i];
  for (int h = tid; h < HA; h += kT) { m_s[h] = -INFINITY; l_s[h] = 0.0f; }
  const int h_o = tid / TPH, d_o = tid % TPH;
  float acc[OPT];
#pragma unroll
  for (int i = 0; i < OPT; ++i) acc[i] = 0.0f;
  // slots: k selected (topk, or dense: slot j is entry j while j < n_visible),
  // then W window rows
  const int64_t vis = (!topk && rs.n_visible) ? rs.n_visible[qi] : k;
  int w_end = 0;
  if (rs.win) {
    w_end = rs.win_end[qi];
    if (w_end < 0 || w_end > rs.win_rows) {
      if (tid == 0) raise_dev_error(err, DEVERR_BOUNDS);
      w_end = 0;
    }
  }
  // this CTA's slots: [chunk * chunk_rows, +chunk_rows) of the query's
  // k selected and W window slots
  const int slots = min(k + (rs.win ? rs.W : 0), (chunk + 1) * rs.chunk_rows);

  for (int c0 = chunk * rs.chunk_rows; c0 < slots; c0 += kR) {
    __syncthreads();   // previous step done with rows_s / p_s / id_s
    if (tid < kR) {
      const int s = c0 + tid;
      int id = -1, src = 0;
      if (s >= slots) {
        // past this CTA's slots
      } else if (s < k) {
        if (topk) {
          id = topk[qi * k + s];
          if (id >= n || id < -1) { raise_dev_error(err, DEVERR_BOUNDS); id = -1; }
        } else {
          id = s < vis ? s : -1;
        }
      } else {
        const int row = w_end - rs.W + (s - k);
        id = row >= 0 ? row : -1;
        src = 1;
      }
      id_s[tid] = id;
      src_s[tid] = src;
    }
    __syncthreads();
    // stage rows as f32 (zeros for empty slots)
    if (!FP4) {
      constexpr int V = DD / 8;   // uint4 per row
      for (int i = tid; i < kR * V; i += kT) {
        const int r = i / V, c = i % V;
        const int id = id_s[r];
        uint4 v = make_uint4(0, 0, 0, 0);
        if (id >= 0) {
          const uint16_t* base = src_s[r] ? rs.win + (seq * rs.win_rows + id) * DD
                                          : static_cast<const uint16_t*>(kv_data) + (seq * n + id) * DD;
          v = __ldg(reinterpret_cast<const uint4*>(base) + c);
        }
        float* dst = rows_s + r * S::RS + c * 8;
        dst[0] = bf16_lo(v.x); dst[1] = bf16_hi(v.x); dst[2] = bf16_lo(v.y); dst[3] = bf16_hi(v.y);
        dst[4] = bf16_lo(v.z); dst[5] = bf16_hi(v.z); dst[6] = bf16_lo(v.w); dst[7] = bf16_hi(v.w);
      }
    } else {
      constexpr int NB = DD / 16;  // 16-channel blocks per row
      for (int i = tid; i < kR * NB; i += kT) {
        const int r = i / NB, blk = i % NB;
        const int id = id_s[r];
        float* dst = rows_s + r * S::RS + blk * 16;
        if (id < 0) {
#pragma unroll
          for (int u = 0; u < 16; ++u) dst[u] = 0.0f;
          continue;
        }
        if (src_s[r]) {            // window rows are uncompressed bf16
          const uint4* wp = reinterpret_cast<const uint4*>(rs.win + (seq * rs.win_rows + id) * DD + blk * 16);
          const uint4 a = __ldg(wp), b = __ldg(wp + 1);
          const uint32_t wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            dst[2 * u] = bf16_lo(wv[u]);
            dst[2 * u + 1] = bf16_hi(wv[u]);
          }
          continue;
        }
        const int64_t row = seq * n + id;
        const uint2 cw = __ldg(reinterpret_cast<const uint2*>(
                                   static_cast<const uint8_t*>(kv_data) + row * (DD / 2)) + blk);
        const uint32_t sc = __ldg(kv_scales + row * NB + blk);
        const uint32_t se = (sc >> 3) & 15u, sm = sc & 7u;
        float s = (se == 0) ? static_cast<float>(sm) * 0x1p-9f
                            : __uint_as_float(((se + 120u) << 23) | (sm << 20));
        if (sc & 128u) s = -s;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const uint32_t c = ((u < 8 ? cw.x : cw.y) >> (4 * (u & 7))) & 15u;
          const uint32_t e = (c >> 1) & 3u, mt = c & 1u;
          float mag = (e == 0) ? 0.5f * mt : (1.0f + 0.5f * mt) * static_cast<float>(1u << (e - 1));
          dst[u] = ((c & 8u) ? -mag : mag) * s;
        }
      }
    }
    __syncthreads();
    // logits for (head, row) pairs
#pragma unroll
    for (int pi = 0; pi < PAIRS; ++pi) {
      const int r = tid % kR;
      const int h = tid / kR + (kT / kR) * pi;
      float dot = 0.0f;
      const float* row = rows_s + r * S::RS;
      const uint32_t* qh = q_s + h * (DD / 2);
#pragma unroll 8
      for (int i = 0; i < DD / 2; ++i) {
        const uint32_t qq = qh[i];
        dot = fmaf(bf16_lo(qq), row[2 * i], dot);
        dot = fmaf(bf16_hi(qq), row[2 * i + 1], dot);
      }
      p_s[h * (kR + 1) + r] = (id_s[r] >= 0) ? scale * dot : -INFINITY;
    }
    __syncthreads();
    // online softmax update, one thread per head
    for (int h = tid; h < HA; h += kT) {
      float* ph = p_s + h * (kR + 1);
      float mx = m_s[h];
#pragma unroll
      for (int r = 0; r < kR; ++r) mx = fmaxf(mx, ph[r]);
      float alpha = 1.0f, l = l_s[h];
      if (mx != -INFINITY) {
        alpha = (m_s[h] == -INFINITY) ? 0.0f : expf(m_s[h] - mx);
        l *= alpha;
#pragma unroll
        for (int r = 0; r < kR; ++r) {
          const float p = (ph[r] == -INFINITY) ? 0.0f : expf(ph[r] - mx);
          ph[r] = p;
          l += p;
        }
      } else {
#pragma unroll
        for (int r = 0; r < kR; ++r) ph[r] = 0.0f;
      }
      m_s[h] = mx;
      l_s[h] = l;
      a_s[h] = alpha;
    }
    __syncthreads();
    const float alpha = a_s[h_o];
    const float* ph = p_s + h_o * (kR + 1);
#pragma unroll
    for (int i = 0; i < OPT; ++i) acc[i] *= alpha;
#pragma unroll
    for (int r = 0; r < kR; ++r) {
      const float p = ph[r];
      const float* row = rows_s + r * S::RS + d_o;
#pragma unroll
      for (int i = 0; i < OPT; ++i) acc[i] = fmaf(p, row[i * TPH], acc[i]);
    }
  }
  __syncthreads();
  uint16_t* og = out + (qi * HA + h_o) * DD + d_o;
  if (rs.n_chunks <= 1) {
    const float l = l_s[h_o];
    const float inv = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll
    for (int i = 0; i < OPT; ++i) {
      __nv_bfloat16 v = __float2bfloat16_rn(acc[i] * inv);
      og[i * TPH] = *reinterpret_cast<uint16_t*>(&v);
    }
    if (lse && d_o == 0) lse[qi * HA + h_o] = l > 0.0f ? m_s[h_o] + logf(l) : -INFINITY;
    return;
  }
  // this chunk's partial: unnormalised sums, the running max and row sum per head
  constexpr int kStride = HA * DD + 2 * HA;
  float* pp = rs.part + (ql * rs.n_chunks + chunk) * kStride;
#pragma unroll
  for (int i = 0; i < OPT; ++i) __stcg(pp + h_o * DD + d_o + i * TPH, acc[i]);
  for (int h = tid; h < HA; h += kT) {
    __stcg(pp + HA * DD + h, m_s[h]);
    __stcg(pp + HA * DD + HA + h, l_s[h]);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) last_s = atomicAdd(rs.counters + ql, 1u) == static_cast<unsigned>(rs.n_chunks - 1);
  __syncthreads();
  if (!last_s) return;
  // the query's last chunk to finish combines the partials, in chunk order
  __threadfence();
  const float* pq = rs.part + ql * rs.n_chunks * kStride;
  float M = -INFINITY;
  for (int c = 0; c < rs.n_chunks; ++c) M = fmaxf(M, __ldcg(pq + c * kStride + HA * DD + h_o));
  float L = 0.0f, o[OPT];
#pragma unroll
  for (int i = 0; i < OPT; ++i) o[i] = 0.0f;
  for (int c = 0; c < rs.n_chunks; ++c) {
    const float* pc = pq + c * kStride;
    const float wc = rescale_part(__ldcg(pc + HA * DD + h_o), M);
    L += __ldcg(pc + HA * DD + HA + h_o) * wc;
#pragma unroll
    for (int i = 0; i < OPT; ++i) o[i] += __ldcg(pc + h_o * DD + d_o + i * TPH) * wc;
  }
  const float inv = L > 0.0f ? 1.0f / L : 0.0f;
#pragma unroll
  for (int i = 0; i < OPT; ++i) {
    __nv_bfloat16 v = __float2bfloat16_rn(o[i] * inv);
    og[i * TPH] = *reinterpret_cast<uint16_t*>(&v);
  }
  if (lse && d_o == 0) lse[qi * HA + h_o] = L > 0.0f ? M + logf(L) : -INFINITY;
  if (tid == 0) rs.counters[ql] = 0u;            // ready for the next launch
}

// The split of a query's slots over CTAs: it depends on the slots alone (k and
// the window), so a query's result does not depend on the batch.  Up to
// kMaxChunks CTAs of at least kR rows each.
constexpr int kMaxChunks = 16;
constexpr size_t kSimtWsCap = size_t(64) << 20;   // partials of one launch
struct Split {
  int n_chunks, chunk_rows;
  int64_t per_launch;                             // queries per launch (partials in the workspace)
  size_t bytes;                                   // workspace: partials, then counters
};

Split split_for(int64_t n_queries, int Ha, int D, int k, bool win, int W) {
  Split s;
  const int slots = k + (win ? W : 0);
  s.n_chunks = slots <= kR ? 1 : std::min(kMaxChunks, (slots + kR - 1) / kR);
  const int per = (slots + s.n_chunks - 1) / s.n_chunks;
  s.chunk_rows = std::max(kR, (per + kR - 1) / kR * kR);
  s.n_chunks = std::max(1, (slots + s.chunk_rows - 1) / s.chunk_rows);
  if (s.n_chunks == 1) {
    s.per_launch = n_queries;
    s.bytes = 0;
    return s;
  }
  const size_t per_query = static_cast<size_t>(s.n_chunks) * (static_cast<size_t>(Ha) * D + 2 * Ha) * 4;
  s.per_launch = std::max<int64_t>(1, std::min<int64_t>(n_queries, static_cast<int64_t>(kSimtWsCap / per_query)));
  s.bytes = ((static_cast<size_t>(s.per_launch) * per_query + 255) & ~size_t(255)) +
            ((static_cast<size_t>(s.per_launch) * 4 + 255) & ~size_t(255));
  return s;
}

template <int HA, int DD>
csa2_status run_simt(const void* q, const csa2_kv& kv, const int32_t* topk, int B, int Q, int k,
                     float scale, void* out, float* lse, void* ws, size_t ws_bytes,
                     unsigned long long* sync_zeroed, cudaStream_t stream, const AttnRows& rows) {
  const size_t smem = AttnSmem<HA, DD>::bytes;
  auto kern = kv.fmt == CSA2_KV_FP4 ? attn_simt_kernel<HA, DD, true> : attn_simt_kernel<HA, DD, false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return check_launch("sparse_attn: shared-memory opt-in");
  const int64_t n_queries = static_cast<int64_t>(B) * Q;
  Split sp = split_for(n_queries, HA, DD, k, rows.win != nullptr, rows.W);
  if (sp.n_chunks > 1 && (!ws || ws_bytes < sp.bytes)) {     // no room for partials: one CTA per query
    sp.n_chunks = 1;
    sp.chunk_rows = k + (rows.win ? rows.W : 0);
    sp.per_launch = n_queries;
  }
  SimtRows rs{rows.n_visible, static_cast<const uint16_t*>(rows.win), rows.win_rows, rows.win_end,
              rows.win ? rows.W : 0, Q, 0, sp.n_chunks, std::max(sp.chunk_rows, 1), nullptr, nullptr};
  // the counters: a layer group's (zeroed once, left zero by every launch)
  // when they are enough, else the workspace's, cleared before each launch
  const bool own_counters = !(sync_zeroed && sp.per_launch <= 2 * kAttnMaxGrid);
  if (sp.n_chunks > 1) {
    const size_t part_bytes = sp.bytes - ((static_cast<size_t>(sp.per_launch) * 4 + 255) & ~size_t(255));
    rs.part = static_cast<float*>(ws);
    rs.counters = own_counters ? reinterpret_cast<unsigned*>(static_cast<char*>(ws) + part_bytes)
                               : reinterpret_cast<unsigned*>(sync_zeroed);
  }
  for (int64_t q0 = 0; q0 < n_queries; q0 += sp.per_launch) {
    const int64_t nq = std::min<int64_t>(sp.per_launch, n_queries - q0);
    const int64_t grid = nq * sp.n_chunks;
    if (grid > 0x7fffffffLL) return fail(CSA2_ERR_UNSUPPORTED, "sparse_attn: too many CTAs");
    rs.q_base = q0;
    if (sp.n_chunks > 1 && own_counters) {
      begin_launch(stream);
      if (cudaMemsetAsync(rs.counters, 0, static_cast<size_t>(nq) * 4, stream) != cudaSuccess)
        return check_launch("sparse_attn: clear counters");
      note_launch(LK_OTHER, 1, stream);
    }
    begin_launch(stream);
    kern<<<static_cast<unsigned>(grid), kT, smem, stream>>>(
        static_cast<const uint16_t*>(q), kv.data, kv.scales, kv.n, topk, k, scale,
        static_cast<uint16_t*>(out), lse, device_error_word(), rs);
    note_launch(LK_ATTN, 1, stream);
    CSA2_TRY(check_launch("sparse_attn"));
  }
  return CSA2_OK;
}

}  // namespace

size_t sparse_attn_workspace(int B, int Q, int Ha, int D, int k, csa2_kv_fmt fmt, bool window) {
  const size_t tc = sparse_attn_tc_workspace(B, Q, Ha, D, k, fmt, window);
  if (tc > 0) return tc;
  const size_t simt = split_for(static_cast<int64_t>(B) * Q, Ha, D, k, window, kMaxWindow).bytes;
  if (sparse_attn_narrow_applies(Ha, D, k, window))
    return std::max(simt, sparse_attn_narrow_workspace(B, Q, Ha, k, window));
  return simt;
}

csa2_status launch_sparse_attn(const void* q, const csa2_kv& kv, const int32_t* topk, int B,
                               int Q, int Ha, int k, float scale, void* out, float* lse, void* ws,
                               size_t ws_bytes, unsigned long long* sync_zeroed,
                               cudaStream_t stream, const AttnRows& rows) {
  if (B == 0 || Q == 0) return CSA2_OK;
  csa2_status s = launch_sparse_attn_tc(q, kv, topk, B, Q, Ha, k, scale, out, lse, ws, ws_bytes,
                                        sync_zeroed, stream, rows);
  if (s != CSA2_ERR_UNSUPPORTED) return s;
  const int D = kv.dim;
  if (sparse_attn_narrow_applies(Ha, D, k, rows.win != nullptr)) {
    s = launch_sparse_attn_narrow(q, kv, topk, B, Q, Ha, k, scale, out, lse, ws, ws_bytes, sync_zeroed,
                                  stream, rows);
    if (s != CSA2_ERR_UNSUPPORTED) return s;
  }
#define CSA2_SIMT(HA_, D_)                                                                       \
  if (Ha == HA_ && D == D_)                                                                      \
    return run_simt<HA_, D_>(q, kv, topk, B, Q, k, scale, out, lse, ws, ws_bytes, sync_zeroed, stream, rows);
  CSA2_SIMT(64, 512) CSA2_SIMT(16, 128) CSA2_SIMT(16, 512) CSA2_SIMT(64, 128) CSA2_SIMT(32, 128)
  CSA2_SIMT(32, 512)
#undef CSA2_SIMT
  return fail(CSA2_ERR_UNSUPPORTED, "sparse_attn: (Ha=%d, D=%d) not instantiated", Ha, D);
}

}  // namespace csa2
