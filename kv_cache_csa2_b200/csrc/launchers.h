// Internal launchers, one per kernel family.  Arguments are already validated
// by the C-ABI layer (api.cu); each launcher picks the kernel instance and
// enqueues it on `stream`.
#pragma once

#include "common.cuh"

namespace csa2 {

csa2_status launch_compress(const void* c, const float* z, const float* bias, int B, int64_t T,
                            int D, int m, int halo, void* out, int64_t out_bstride,
                            cudaStream_t stream);
// HCA compression: entry j is the softmax-weighted sum of block j alone.
constexpr int kMaxHcaBlock = 1024;
csa2_status launch_compress_hca(const void* c, const float* z, const float* bias, int B, int64_t T,
                                int D, int m, void* out, int64_t out_bstride, cudaStream_t stream);

// Words of device memory that the scoring kernel clears at its start for the
// selection launched after it, so that no separate memset sits between the
// two; `done` tells whether the kernel that ran took it on.
struct ClearOnLaunch {
  uint32_t* ptr = nullptr;
  int words = 0;
  bool done = false;
};
csa2_status launch_index_scores(const void* q, const float* w, const void* k, int B, int Q, int H,
                                int d, int64_t N, const int32_t* n_visible, const int32_t* pool,
                                int P, csa2_index_act act, float* scores, cudaStream_t stream,
                                ClearOnLaunch* clear = nullptr);

// A Full layer's indexer fused with a streaming top-k (no score round trip):
// many queries (at least one group of 4 per SM), k_top <= kMaxFusedTopk.
// Same scores and the same exact selection as scoring then selecting.
constexpr int kMaxFusedTopk = 2048;
bool index_topk_fused_applies(int B, int Q, int H, int d, int64_t N, int k_top);
csa2_status launch_index_topk_fused(const void* q, const float* w, const void* k, int B, int Q,
                                    int H, int d, int64_t N, const int32_t* n_visible, int k_top,
                                    csa2_index_act act, int32_t* topk, cudaStream_t stream);

// FP4 indexer (q and K in the main-KV FP4 format, bf16 scores): scores
// rounded to bf16, stored as bf16 (out_bf16) or as f32 holding the bf16 value.
struct Fp4IndexArgs {
  const uint8_t* q_codes;    // [B, Q, H, d/2]
  const uint8_t* q_scales;   // [B, Q, H, d/16]
  const float* w;            // [B, Q, H]
  const uint8_t* k_codes;    // [B, N, d/2]
  const uint8_t* k_scales;   // [B, N, d/16]
  int B, Q, H, d;
  int64_t N;
  const int32_t* n_visible;  // [B, Q] or null
  const int32_t* pool;       // [B, Q, P] or null
  int P;
  csa2_index_act act;
  void* scores;              // [B, Q, N or P]
};
csa2_status launch_index_scores_fp4(const Fp4IndexArgs& a, bool out_bf16, cudaStream_t stream);

size_t select_topk_workspace(int64_t rows, int64_t L, int count);
// The workspace one selection (launch_select_topk) will actually use on the
// current device: 0 when the cluster, one-CTA or fallback kernel takes the
// rows (select_topk_workspace is an upper bound over devices and paths).
size_t select_topk_scratch_bytes(int64_t rows, int64_t L, int count);
// Two selections of the same rows in one pass set (multi-CTA kernel); returns
// CSA2_ERR_UNSUPPORTED when that kernel does not apply to the shape.
// ws_cleared: select_topk_clear() already ran on this workspace on `stream`
// (lets the caller clear it before the kernel that writes the scores, so the
// selection follows that kernel directly).
csa2_status launch_select_topk2(const float* scores, int64_t rows, int64_t L, int count0,
                                const int32_t* ids, int32_t* out0, int count1, int32_t* out1,
                                void* ws, size_t ws_bytes, cudaStream_t stream,
                                bool ws_cleared = false);
csa2_status select_topk_clear(int64_t rows, int64_t L, void* ws, size_t ws_bytes,
                              cudaStream_t stream);
// The words select_topk_clear() would clear (ptr = NULL when there are none).
ClearOnLaunch select_topk_clear_region(int64_t rows, int64_t L, void* ws, size_t ws_bytes);
// One CTA per row, no workspace: rows of up to kSelectCtaMaxL scores.
constexpr int64_t kSelectCtaMaxL = 32768;
bool select_topk_cta_applies(int64_t rows, int64_t L);
csa2_status launch_select_topk_cta(const float* scores, int64_t rows, int64_t L, int count0,
                                   const int32_t* ids, int32_t* out0, int count1, int32_t* out1,
                                   cudaStream_t stream);
// A cluster of 8 CTAs per row, no workspace: one selection (count1 <= 0) of
// rows of up to 262144 scores when there are fewer rows than SMs.  With
// `gather`, key i of row r is scores[r * src_stride + gather[r * L + i]]
// (negative entries are not selectable).
bool select_topk_cluster_applies(int64_t rows, int64_t L, int count0, int count1);
csa2_status launch_select_topk_cluster(const float* scores, int64_t rows, int64_t L, int count,
                                       const int32_t* ids, int32_t* out, cudaStream_t stream,
                                       const int32_t* gather = nullptr, int64_t src_stride = 0);
csa2_status launch_select_topk(const float* scores, int64_t rows, int64_t L, int count,
                               const int32_t* ids, int32_t* out, void* ws, size_t ws_bytes,
                               cudaStream_t stream);

// Largest grid of the tensor-core attention kernel on any device (>= the
// CTAs that fit at once); sizes its workspace and its arrival counters.
constexpr int kAttnMaxGrid = 160;

// Rows an attention launch takes besides a selection list.
//  - topk == NULL (dense): slot j of a query is entry j, visible while
//    j < n_visible[query] (all k = kv.n slots when n_visible is NULL).
//  - win != NULL: one more tile of rows per query, from a sliding window of
//    uncompressed rows (bf16 [B, win_rows, D]): query qi takes rows
//    [max(0, e - W), e) with e = win_end[qi] (0 <= e <= win_rows), in the same
//    softmax as its other rows.
struct AttnRows {
  const int32_t* n_visible = nullptr;
  const void* win = nullptr;
  int64_t win_rows = 0;
  const int32_t* win_end = nullptr;
  int W = 0;
};
constexpr int kMaxWindow = 128;

// The tensor-core attention for 64 heads x 512 in two schedules with the same
// arithmetic per query (bit for bit): a query's tiles on several CTAs
// (attn_tc.cu, few queries) or in sequence on one CTA (attn_seq.cu, many
// queries; no workspace).  CSA2_ATTN_SEQ=0 / 1 forces the choice.
// Entries of width 128 (16, 32 or 64 heads, bf16 or FP4 rows) on the tensor
// cores (attn_narrow.cu); CSA2_ATTN_SIMT forces the CUDA-core kernel.
bool sparse_attn_narrow_applies(int Ha, int D, int k, bool win);
size_t sparse_attn_narrow_workspace(int B, int Q, int Ha, int k, bool win);
csa2_status launch_sparse_attn_narrow(const void* q, const csa2_kv& kv, const int32_t* topk, int B,
                                      int Q, int Ha, int k, float scale, void* out, float* lse,
                                      void* ws, size_t ws_bytes, unsigned long long* sync_zeroed,
                                      cudaStream_t stream, const AttnRows& rows);
bool sparse_attn_seq_applies(int64_t n_queries, int k, bool win);
csa2_status launch_sparse_attn_seq(const void* q, const csa2_kv& kv, const int32_t* topk, int B,
                                   int Q, int k, float scale, void* out, float* lse,
                                   cudaStream_t stream, const AttnRows& rows);

size_t sparse_attn_workspace(int B, int Q, int Ha, int D, int k, csa2_kv_fmt fmt, bool window = false);
// sync_zeroed: kAttnMaxGrid * 8 bytes of per-CTA flags that were zero before
// their first use and are left consistent by every launch (a layer group's),
// or NULL to take them from the workspace and clear them on the stream.
csa2_status launch_sparse_attn(const void* q, const csa2_kv& kv, const int32_t* topk, int B,
                               int Q, int Ha, int k, float scale, void* out, float* lse, void* ws,
                               size_t ws_bytes, unsigned long long* sync_zeroed,
                               cudaStream_t stream, const AttnRows& rows = AttnRows());
// csa2_sparse_attn's argument checks, then launch_sparse_attn.
csa2_status sparse_attn_checked(csa2_mode mode, const void* q, const csa2_kv* kv,
                                const int32_t* topk, int B, int Q, int Ha, int k, float scale,
                                void* out, float* lse, void* workspace, size_t workspace_bytes,
                                unsigned long long* sync_zeroed, cudaStream_t stream,
                                const AttnRows& rows = AttnRows());

csa2_status launch_fp4_pack(const void* x, int64_t rows, int D, uint8_t* codes, uint8_t* scales,
                            cudaStream_t stream);
csa2_status launch_fp4_unpack(const uint8_t* codes, const uint8_t* scales, int64_t rows, int D,
                              void* x, cudaStream_t stream);

}  // namespace csa2
