/*
 * csa2.h -- C ABI of libcsa2.so, the CSA2 compressed-sparse-attention hot path
 * for NVIDIA B200 (sm_100a).
 *
 * Sources (the pages' formulas were lost in extraction; readings are stated
 * per call):
 *   [V4]   "读完这篇，你就搞懂 DeepSeek v4 了" (DeepSeek V4 explainer): CSA
 *          compression ("meeting recorder" over two consecutive meetings;
 *          eq. 11 weight matrix S from logits Z plus bias B), 闪电索引机制
 *          (lightning indexer, eq. 8), 注意力计算 (shared-KV attention, eq. 9),
 *          批无关性 (batch invariance).
 *   [V41]  DeepSeek V4.1 Flash video transcript: the CSA2 paragraph (Full /
 *          Reindex / Reuse layer modes) and the hierarchical sparse indexer
 *          paragraph (a Full layer builds a candidate pool of about 16,384
 *          positions; later Reindex layers search only inside it).
 *   [R]    "Recall之王 祭出Reuse": CSA2 bullets -- Hierarchical Sparse Indexer,
 *          FP4 main-KV cache (E2M1 values, one E4M3 scale per 16 channels).
 *
 * Conventions for every call
 *   - Tensor pointers are DEVICE pointers on the current CUDA device, owned by
 *     the caller.  The library never frees caller memory and never keeps a
 *     pointer past the call, except a layer group (below), which keeps
 *     non-owning references to the KV and indexer K registered by its last
 *     Full layer.
 *   - bf16 = IEEE bfloat16 stored as 16-bit words; f32 = float.  Shapes are
 *     row-major, innermost dimension last, densely packed unless a stride
 *     argument says otherwise.  Every tensor must start on a 16-byte boundary.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously.  The return value reports argument,
 *     mode and launch errors found on the host.  Errors found by the kernels
 *     (an index out of range, a bounded wait that ran out) are recorded in a
 *     per-device error word read by csa2_device_error().
 *   - On any non-OK status nothing was enqueued (except CSA2_ERR_CUDA, raised
 *     when a launch itself fails) and csa2_last_error() describes the problem
 *     (thread-local string).
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* csa2_stream; /* a cudaStream_t */

typedef enum {
  CSA2_OK = 0,
  CSA2_ERR_INVALID = 1,     /* bad argument: null pointer, size, alignment       */
  CSA2_ERR_MODE = 2,        /* call not allowed in this layer mode / mode order  */
  CSA2_ERR_UNSUPPORTED = 3, /* valid but not implemented shape                   */
  CSA2_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed              */
  CSA2_ERR_TIMEOUT = 5,     /* a bounded device-side wait gave up                */
  CSA2_ERR_OOM = 6,         /* allocation (layer group only) or workspace too small */
  CSA2_ERR_BOUNDS = 7       /* a kernel met an entry index outside [0, n)        */
} csa2_status;

/* [V41] CSA2 paragraph: the three per-layer modes. */
typedef enum { CSA2_FULL = 0, CSA2_REINDEX = 1, CSA2_REUSE = 2 } csa2_mode;

/* Main-KV storage.  [R] FP4 主KV缓存: E2M1 codes + one E4M3 scale / 16 channels. */
typedef enum { CSA2_KV_BF16 = 0, CSA2_KV_FP4 = 1 } csa2_kv_fmt;

/* Per-head activation of the indexer score: ReLU (the DSA form [V4] eq. 8 is
 * tied to) or none. */
typedef enum { CSA2_ACT_RELU = 0, CSA2_ACT_IDENTITY = 1 } csa2_index_act;

/* A main-KV buffer holding B sequences of n entries of width dim.
 *   BF16: data = bf16 [B, n, dim]; scales = NULL.
 *   FP4 : data = uint8 codes [B, n, dim/2] (channel 2i in the low nibble of
 *         byte i, 2i+1 in the high nibble); scales = uint8 E4M3 [B, n, dim/16].
 */
typedef struct {
  csa2_kv_fmt fmt;
  const void* data;
  const uint8_t* scales;
  int64_t n;
  int dim;
} csa2_kv;

/* ------------------------------------------------------------------------ */
/* (a1) Token -> entry compression.  [V4] CSA compression and eq. (11).
 *
 * e[b, j, ch] = sum_{t in W_j} softmax_t(z[b,t,ch] + bias[t - (j-1)m, ch]) * c[b,t,ch]
 * with W_j = tokens [(j-1)m, (j+1)m) (blocks j-1 and j; the softmax runs per
 * channel over the window).  Tokens before the chunk are absent unless
 * has_left_halo = 1, in which case the first m rows of c and z are the block
 * that precedes the chunk.  The last partial block forms no entry.
 * Arithmetic in f32, result rounded once to bf16 (nearest, ties to even).
 *
 *   c     bf16 [B, T + halo, D]     value projections (halo = has_left_halo ? m : 0)
 *   z     f32  [B, T + halo, D]     logits
 *   bias  f32  [2m, D]              learned positional bias, row = position in window
 *   out   bf16 entries: row j of sequence b at out + b*out_batch_stride + j*D,
 *         j in [0, T/m).  out_batch_stride (elements) = 0 means (T/m)*D.  Passing
 *         a pointer into a larger KV buffer appends the new entries to it.
 * Requires D % 8 == 0, 1 <= m <= 16, T >= 0.  Errors: CSA2_ERR_INVALID.
 */
csa2_status csa2_compress(const void* c, const float* z, const float* bias, int B, int64_t T,
                          int D, int m, int has_left_halo, void* out, int64_t out_batch_stride,
                          csa2_stream stream);

/* HCA (heavily compressed attention) compression.  [V4] HCA 压缩机制, eq. (10)
 * with the weights of eq. (11): blocks of m tokens (m >> the CSA block), and
 * unlike csa2_compress an entry does not join two consecutive blocks:
 *   e[b, j, ch] = sum_{t in [jm, (j+1)m)} softmax_t(z[b,t,ch] + bias[t - jm, ch]) * c[b,t,ch]
 * f32 arithmetic (one pass with a running max), rounded once to bf16.
 *   c bf16 [B, T, D]    z f32 [B, T, D]    bias f32 [m, D]
 *   out bf16 entries j in [0, T/m) at out + b*out_batch_stride + j*D (stride 0 = (T/m)*D).
 * Requires D % 8 == 0, 1 <= m <= 1024.  Errors: CSA2_ERR_INVALID. */
csa2_status csa2_compress_hca(const void* c, const float* z, const float* bias, int B, int64_t T,
                              int D, int m, void* out, int64_t out_batch_stride,
                              csa2_stream stream);

/* ------------------------------------------------------------------------ */
/* (a2) Lightning-indexer scores.  [V4] 闪电索引机制, eq. (8):
 *   s[b,q,j] = sum_h w[b,q,h] * act(q[b,q,h,:] . k[b,e,:])
 * where e = j (no pool) or e = pool[b,q,j] (pool given: hierarchical indexer,
 * [V41] / [R]).  Unscored slots get -inf: entries e >= n_visible[b,q] (no
 * pool; n_visible = NULL means all N visible) and pool slots holding -1.
 * Dot products accumulate in f32 from exact bf16 products.
 *
 *   q         bf16 [B, Q, H, d]       w  f32 [B, Q, H]       k  bf16 [B, N, d]
 *   n_visible int32 [B, Q] or NULL    pool int32 [B, Q, P] or NULL
 *   scores    f32 [B, Q, N] (no pool) or [B, Q, P]
 * Requires d % 8 == 0, d <= 256, H <= 128.  A pool entry outside [0, N) other
 * than -1 is recorded as CSA2_ERR_BOUNDS in the device error word and scored
 * -inf.
 */
csa2_status csa2_index_scores(const void* q, const float* w, const void* k, int B, int Q, int H,
                              int d, int64_t N, const int32_t* n_visible, const int32_t* pool,
                              int P, csa2_index_act act, float* scores, csa2_stream stream);

/* (a3) Top-k selection over score rows.  [V4] 闪电索引机制: keep the k most
 * relevant entries.  Order: score descending, ties to the lower position; -inf
 * and NaN are never chosen.  Row r's result lists the chosen positions in
 * ascending order, padded with -1 when fewer than `count` are selectable.  If
 * ids != NULL the positions are replaced by ids[r, pos] (mapping pool slots
 * back to entry indices; ids must then be ascending in the selectable slots so
 * that position order is index order, as every pool this library writes is).
 * The result is bit-for-bit deterministic and does not depend on how many rows
 * are selected together.
 *
 *   scores f32 [rows, L]    ids int32 [rows, L] or NULL    out int32 [rows, count]
 *   workspace: csa2_select_topk_workspace(rows, L, count) bytes of device memory
 *   (an upper bound: with fewer rows than the GPU has SMs and L <= 262144 the
 *   selection runs on clusters of CTAs and uses none of it).
 */
size_t csa2_select_topk_workspace(int64_t rows, int64_t L, int count);
csa2_status csa2_select_topk(const float* scores, int64_t rows, int64_t L, int count,
                             const int32_t* ids, int32_t* out, void* workspace,
                             size_t workspace_bytes, csa2_stream stream);

/* csa2_select_topk without a workspace argument.  The pages have no
 * counterpart to this call: it is a convenience of this library for callers
 * that cannot hand out device memory.  Arguments, result and errors are those
 * of csa2_select_topk (same kernels, bit-identical output); the scratch is a
 * static device array of CSA2_SELECT_TOPK_NOALLOC_SCRATCH_BYTES per device
 * inside the library, so the call allocates nothing.
 *   - Only the kernel with several cooperating CTAs per row uses scratch
 *     (rows of more than 262144 keys, or at least as many rows as the GPU has
 *     SMs with more than 32768 keys); it needs about 164 KiB per row, so at
 *     most 25 rows fit.  A call on that path that needs more than the array
 *     returns CSA2_ERR_OOM with nothing enqueued.  The paths that keep their
 *     state in shared memory (fewer rows than SMs and L <= 262144; L <= 32768)
 *     need no scratch and have no such limit.
 *   - The part of the scratch that must start at zero is cleared on `stream`
 *     before every launch (an asynchronous memset, no allocation).
 *   - The scratch is shared: calls that overlap on one device (other streams,
 *     other host threads) race on it and give wrong results.  Serialise them.
 *   - The first call on each device looks up the scratch's address and the
 *     kernel's occupancy on the host; make one call on a device before
 *     capturing a stream that contains this call. */
#define CSA2_SELECT_TOPK_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
csa2_status csa2_select_topk_noalloc(const float* scores, int64_t rows, int64_t L, int count,
                                     const int32_t* ids, int32_t* out, csa2_stream stream);

/* (a2 + a3) Indexer scores followed by top-k, per layer mode ([V41] CSA2
 * paragraph, hierarchical indexer paragraph; [R] Hierarchical Sparse Indexer):
 *   CSA2_FULL    : pool_in must be NULL.  Scores every visible entry, writes
 *                  topk_out [B,Q,k_top] and, if pool_out != NULL, the pool of
 *                  the P_out best entries pool_out [B,Q,P_out] (top-k is a
 *                  subset of the pool: both use the same order).
 *   CSA2_REINDEX : pool_out must be NULL.  With pool_in [B,Q,P_in] scores only
 *                  the pool's entries, else every visible entry; writes topk_out.
 *   CSA2_REUSE   : runs no indexer -> CSA2_ERR_MODE.
 * Outputs are entry indices, ascending per query, -1 padded.
 * workspace: csa2_index_topk_workspace(...) bytes (scores plus selection state).
 */
size_t csa2_index_topk_workspace(int B, int Q, int64_t N, int P_in, int k_top, int P_out);
csa2_status csa2_index_topk(csa2_mode mode, const void* q, const float* w, const void* k, int B,
                            int Q, int H, int d, int64_t N, const int32_t* n_visible,
                            const int32_t* pool_in, int P_in, int k_top, int32_t* topk_out,
                            int32_t* pool_out, int P_out, csa2_index_act act, void* workspace,
                            size_t workspace_bytes, csa2_stream stream);

/* (a2 + a3, FP4 variant) The lightning indexer with FP4 queries and keys and
 * BF16 scores.  [V4] FP4量化感知训练: the indexer's q and K are kept in FP4,
 * its scores in BF16.  q and K use the FP4 format of csa2_fp4_pack (E2M1
 * codes, channel 2i in the low nibble, one E4M3 scale per 16 channels along
 * d).  Each score is eq. (8) over the dequantised values (exact products, f32
 * accumulation) rounded once to bf16 (nearest even); unscored slots are -inf.
 *   q_codes uint8 [B, Q, H, d/2]   q_scales uint8 [B, Q, H, d/16]   w f32 [B, Q, H]
 *   k_codes uint8 [B, N, d/2]      k_scales uint8 [B, N, d/16]
 *   n_visible, pool, P, act: as csa2_index_scores
 *   scores  bf16 [B, Q, N] (no pool) or [B, Q, P]
 * Requires d in {64, 128}, H <= 64; k_codes 16-byte aligned, q_codes 8-byte
 * aligned, k_scales d/16-byte aligned.  Pool entries outside [0, N) other
 * than -1 are recorded as CSA2_ERR_BOUNDS and scored -inf. */
csa2_status csa2_index_scores_fp4(const uint8_t* q_codes, const uint8_t* q_scales, const float* w,
                                  const uint8_t* k_codes, const uint8_t* k_scales, int B, int Q,
                                  int H, int d, int64_t N, const int32_t* n_visible,
                                  const int32_t* pool, int P, csa2_index_act act, void* scores,
                                  csa2_stream stream);
/* csa2_index_topk with the FP4 indexer: the same modes, outputs, order and
 * errors, the selection taken over the bf16 scores (ties to the lower
 * position).  workspace: csa2_index_topk_workspace(...) bytes. */
csa2_status csa2_index_topk_fp4(csa2_mode mode, const uint8_t* q_codes, const uint8_t* q_scales,
                                const float* w, const uint8_t* k_codes, const uint8_t* k_scales,
                                int B, int Q, int H, int d, int64_t N, const int32_t* n_visible,
                                const int32_t* pool_in, int P_in, int k_top, int32_t* topk_out,
                                int32_t* pool_out, int P_out, csa2_index_act act, void* workspace,
                                size_t workspace_bytes, csa2_stream stream);

/* ------------------------------------------------------------------------ */
/* (a4) Shared-KV sparse attention.  [V4] 注意力计算, eq. (9): every query head
 * attends, with softmax(scale * q_h . e_j), over the selected entries e_j,
 * which serve as both keys and values:
 *   out[b,q,h,:] = sum_{j in topk[b,q]} p_hj * e_j      (bf16, rounded once)
 *   lse[b,q,h]   = log sum_j exp(scale * q_h . e_j)      (f32, natural log)
 * -1 slots of topk are skipped; an empty selection gives out = 0 and
 * lse = -inf.  FP4 KV ([R] FP4 主KV缓存) is dequantised inside the kernel;
 * the result equals bf16 attention over csa2_fp4_unpack(kv).  The mode only
 * labels the call (the arithmetic is the same in every mode; Reuse passes the
 * previous layer's topk).  The result for a query does not depend on B or Q
 * (fixed reduction order per query, [V4] 批无关性).
 *
 *   q     bf16 [B, Q, Ha, D]   kv  B sequences, kv->dim == D   topk int32 [B, Q, k]
 *   out   bf16 [B, Q, Ha, D]   lse f32 [B, Q, Ha] or NULL
 *   workspace: csa2_sparse_attn_workspace(...) bytes (may be 0 -> NULL allowed).
 * Errors: CSA2_ERR_INVALID; an index outside [0, kv->n) is recorded as
 * CSA2_ERR_BOUNDS in the device error word and skipped.
 */
size_t csa2_sparse_attn_workspace(int B, int Q, int Ha, int D, int k, csa2_kv_fmt fmt);
csa2_status csa2_sparse_attn(csa2_mode mode, const void* q, const csa2_kv* kv,
                             const int32_t* topk, int B, int Q, int Ha, int k, float scale,
                             void* out, float* lse, void* workspace, size_t workspace_bytes,
                             csa2_stream stream);

/* (a4 + SWA branch) Sparse attention together with the layer's sliding-window
 * branch.  [V41] layer layout: every CSA2 layer keeps a sliding-window
 * attention branch over its own uncompressed KV of the most recent 128 tokens
 * (layer-specific, never shared between layers).  Reading: the window rows
 * enter the same softmax as the selected entries (same heads, same scale,
 * shared K = V), which equals merging the two branches' normalised outputs by
 * their log-sum-exp: out = (e^lse_c out_c + e^lse_w out_w) / (e^lse_c + e^lse_w),
 * lse = log(e^lse_c + e^lse_w).  The kernel merges f32 partials, not rounded
 * branch outputs.
 *   win     bf16 [B, win_rows, D]: each sequence's uncompressed window rows
 *   win_end int32 [B, Q]: query (b, q) attends rows [max(0, e - W), e) of
 *           sequence b with e = win_end[b, q], 0 <= e <= win_rows (decode: the
 *           last W rows with e = win_rows; a prefill chunk: e = the query's
 *           own row + 1)
 *   W       window length, 1 <= W <= 128
 * Other arguments, outputs and errors are csa2_sparse_attn's; an e outside
 * [0, win_rows] is recorded as CSA2_ERR_BOUNDS and the window taken empty.
 * workspace: csa2_sparse_attn_swa_workspace(...) bytes. */
size_t csa2_sparse_attn_swa_workspace(int B, int Q, int Ha, int D, int k, csa2_kv_fmt fmt);
csa2_status csa2_sparse_attn_swa(csa2_mode mode, const void* q, const csa2_kv* kv,
                                 const int32_t* topk, int B, int Q, int Ha, int k, float scale,
                                 const void* win, int64_t win_rows, const int32_t* win_end, int W,
                                 void* out, float* lse, void* workspace, size_t workspace_bytes,
                                 csa2_stream stream);

/* HCA attention.  [V4] HCA 注意力计算: the queries attend, as in eq. (9) with
 * shared K = V, to every compressed entry (no indexer, no top-k).  Query
 * (b, q) takes entries [0, n_visible[b, q]) of sequence b (n_visible = NULL:
 * all kv->n).  Same kernels, outputs and errors as csa2_sparse_attn with the
 * selection j -> j.  workspace: csa2_dense_attn_workspace(B, Q, Ha, D, kv->n, fmt). */
size_t csa2_dense_attn_workspace(int B, int Q, int Ha, int D, int64_t N, csa2_kv_fmt fmt);
csa2_status csa2_dense_attn(const void* q, const csa2_kv* kv, const int32_t* n_visible, int B,
                            int Q, int Ha, float scale, void* out, float* lse, void* workspace,
                            size_t workspace_bytes, csa2_stream stream);

/* ------------------------------------------------------------------------ */
/* (a5) FP4 main-KV format.  [R] FP4 主KV缓存: E2M1 with one E4M3 scale per 16
 * channels.  Per 16-channel block: scale s = E4M3 value nearest absmax/6
 * (ties to even, saturating at 448; chosen without a division by comparing
 * absmax with 6x the E4M3 midpoints); code = E2M1 value nearest x/s (ties to
 * even code, saturating at +-6; sign bit = sign of x); absmax = 0 gives scale
 * 0x00 and zero magnitudes.  Unpack: x = e2m1(code) * e4m3(scale), exact in
 * bf16.  Both directions are bit-exact.
 *
 *   x      bf16 [rows, D]      codes uint8 [rows, D/2]     scales uint8 [rows, D/16]
 * Requires D % 16 == 0.
 */
csa2_status csa2_fp4_pack(const void* x, int64_t rows, int D, uint8_t* codes, uint8_t* scales,
                          csa2_stream stream);
csa2_status csa2_fp4_unpack(const uint8_t* codes, const uint8_t* scales, int64_t rows, int D,
                            void* x, csa2_stream stream);

/* ------------------------------------------------------------------------ */
/* (a6) Layer-mode driver.  [V41] CSA2 paragraph: Full builds its KV and
 * indexer K, runs the indexer and picks its own top-k; Reindex reuses the
 * previous main KV and indexer K but scores its own queries; Reuse reuses
 * everything including the top-k and runs attention only.  [V41]/[R]
 * hierarchical indexer: with P > 0 the Full layer also keeps a pool of the P
 * best entries and Reindex layers score only inside it.
 *
 * The group owns its workspace (scores, top-k, pool, selection state; device
 * memory allocated at create on the current device) and holds non-owning
 * references to the KV and indexer K of its last Full layer.  Layers may be
 * called in any order subject to: Reindex and Reuse need a Full layer before
 * them (CSA2_ERR_MODE otherwise).  Reuse attends with the most recent
 * selection.
 */
typedef struct csa2_group csa2_group;

typedef struct {
  int B, Q;           /* sequences, query tokens per sequence                  */
  int64_t N;          /* entries per sequence                                  */
  int D, Ha;          /* main-KV width, attention heads                        */
  int Hi, d;          /* indexer heads and width                               */
  int k, P;           /* selected entries; pool size (0 = no pool)             */
  float scale;        /* attention scale                                       */
  csa2_kv_fmt kv_fmt;
  csa2_index_act act;
  int n_layers;
  const csa2_mode* modes; /* [n_layers], copied at create                     */
} csa2_group_desc;

typedef struct {
  csa2_kv kv;                /* FULL: this layer's main KV (registered for later layers) */
  const void* index_k;       /* FULL: bf16 [B, N, d] (registered)                          */
  const int32_t* n_visible;  /* FULL, and REINDEX without pool: int32 [B, Q] or NULL      */
  const void* q_index;       /* FULL / REINDEX: bf16 [B, Q, Hi, d]                          */
  const float* w_index;      /* FULL / REINDEX: f32 [B, Q, Hi]                              */
  const void* q_attn;        /* all modes: bf16 [B, Q, Ha, D]                               */
  void* out;                 /* all modes: bf16 [B, Q, Ha, D]                               */
  float* lse;                /* all modes: f32 [B, Q, Ha] or NULL                           */
  /* Optional sliding-window branch of this layer (csa2_sparse_attn_swa):
   * NULL swa_kv = none.  Each layer passes its own window rows. */
  const void* swa_kv;        /* bf16 [B, swa_rows, D]                                        */
  int64_t swa_rows;
  const int32_t* swa_end;    /* int32 [B, Q]                                                 */
  int swa_window;            /* W, 1..128                                                    */
} csa2_layer_io;

csa2_status csa2_group_create(csa2_group** group, const csa2_group_desc* desc);
csa2_status csa2_group_layer(csa2_group* group, int layer, const csa2_layer_io* io,
                             csa2_stream stream);
/* Device pointers to the group's current selection (valid until destroy). */
csa2_status csa2_group_selection(const csa2_group* group, const int32_t** topk,
                                 const int32_t** pool);
/* Copies the current selection into caller buffers (device memory; either may
 * be NULL): topk int32 [B, Q, k], pool int32 [B, Q, P].  Enqueued on stream. */
csa2_status csa2_group_copy_selection(const csa2_group* group, int32_t* topk, int32_t* pool,
                                      csa2_stream stream);
void csa2_group_destroy(csa2_group* group);

/* ------------------------------------------------------------------------ */
/* Status, errors and instrumentation. */
const char* csa2_status_string(csa2_status s);
const char* csa2_last_error(void);
/* Synchronises `stream`, returns the first device-side error recorded on the
 * current device since the last call (CSA2_OK, CSA2_ERR_BOUNDS or
 * CSA2_ERR_TIMEOUT) and clears it. */
csa2_status csa2_device_error(csa2_stream stream);
/* Kernel launches issued by this library since the last reset, per kind:
 * 0 compress, 1 index scores (all entries), 2 top-k, 3 attention, 4 attention
 * combine, 5 fp4 pack, 6 fp4 unpack, 7 other (memsets), 8 index scores inside
 * a pool.  Returns the number of kinds. */
int csa2_launch_counts(int64_t* counts, int n);
void csa2_reset_launch_counts(void);
/* Per-kind device time of this library's kernels (instrumentation).  While
 * enabled, each launch is bracketed by two CUDA events recorded on its own
 * stream (not inside stream capture).  csa2_kernel_times() waits for the
 * recorded events and returns, for each kind (numbered as above), the summed
 * milliseconds and the number of timed launches since the last reset; it
 * returns the number of kinds. */
csa2_status csa2_timing_enable(int on);
int csa2_kernel_times(double* ms, int64_t* launches, int n);
void csa2_timing_reset(void);
/* Bound of the device waits in which one CTA waits for another: the row
 * barrier of the multi-CTA top-k and the attention kernel's wait for another
 * tile's partial.  Such a wait gives up after limit_ns nanoseconds (0 = the
 * default, one second), records CSA2_ERR_TIMEOUT in the device error word,
 * and the kernel then finishes its remaining steps without waiting again on
 * the CTA it gave up on, so it ends and leaves the context usable (its
 * results are then undefined).  With unreachable != 0 those waits target a
 * count that no CTA writes, so each one runs out: a test of the error path
 * without a fault.  Applies to launches enqueued after the call; process-wide. */
csa2_status csa2_set_device_wait(uint64_t limit_ns, int unreachable);
/* Host-side fault injection for tests: "alloc", "launch" or "" (off).  While
 * set, every call returns CSA2_ERR_OOM / CSA2_ERR_CUDA before touching the
 * device.  The environment variable CSA2_FAULT sets the initial value. */
csa2_status csa2_set_fault(const char* kind);
int csa2_version(void);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_H */
