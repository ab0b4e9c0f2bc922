// Layer-mode driver: carries the main KV, indexer K, top-k and pool across
// the Full / Reindex / Reuse layers of one CSA2 layer group.
// Source: DeepSeek V4.1 Flash video transcript, CSA2 paragraph (Full builds
// its own global KV and grouped indexer K, runs the sparse indexer and picks
// its own top-k; Reindex reuses the previous main KV and indexer K but makes
// its own queries and a fresh top-k; Reuse reuses everything including the
// top-k indices and runs no indexer) and the hierarchical sparse indexer
// paragraph (the first Full layer builds a candidate pool; Reindex layers
// score only inside it); "Recall之王", CSA2 bullets (Hierarchical Sparse
// Indexer).
//
// Host-only: each layer enqueues the kernels of its mode on the caller's
// stream.  A Reuse layer issues no indexer or selection launch.
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "common.cuh"
#include "launchers.h"

using namespace csa2;

struct csa2_group {
  csa2_group_desc desc;
  std::vector<csa2_mode> modes;
  int device = 0;
  int32_t* topk = nullptr;   // [B, Q, k]   current selection
  int32_t* pool = nullptr;   // [B, Q, P]   pool of the last Full layer (P > 0)
  void* ws = nullptr;        // scores + selection state, then attention workspace
  size_t ws_bytes = 0;
  // attention arrival counters, zeroed once: [0, kAttnMaxGrid) for layers
  // without a window branch, [kAttnMaxGrid, 2 kAttnMaxGrid) for layers with
  // one (each launch shape keeps its own counters consistent)
  unsigned long long* attn_sync = nullptr;
  bool have_full = false;
  csa2_kv kv{};              // registered by the last Full layer (not owned)
  const void* index_k = nullptr;
};

static size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

extern "C" {

csa2_status csa2_group_create(csa2_group** group, const csa2_group_desc* d) {
  CSA2_TRY(fault_gate());
  if (!group || !d) return fail(CSA2_ERR_INVALID, "csa2_group_create: null argument");
  *group = nullptr;
  if (d->B <= 0 || d->Q <= 0 || d->N <= 0 || d->k <= 0 || d->P < 0 || d->n_layers <= 0 ||
      !d->modes || d->Ha <= 0 || d->D <= 0 || d->D % 16 != 0 || d->Hi <= 0 || d->d <= 0)
    return fail(CSA2_ERR_INVALID, "csa2_group_create: bad descriptor");
  if (d->kv_fmt != CSA2_KV_BF16 && d->kv_fmt != CSA2_KV_FP4)
    return fail(CSA2_ERR_INVALID, "csa2_group_create: unknown kv format");
  for (int i = 0; i < d->n_layers; ++i)
    if (d->modes[i] != CSA2_FULL && d->modes[i] != CSA2_REINDEX && d->modes[i] != CSA2_REUSE)
      return fail(CSA2_ERR_INVALID, "csa2_group_create: layer %d has unknown mode %d", i,
                  int(d->modes[i]));
  csa2_group* g = new (std::nothrow) csa2_group();
  if (!g) return fail(CSA2_ERR_OOM, "csa2_group_create: host allocation failed");
  g->desc = *d;
  g->modes.assign(d->modes, d->modes + d->n_layers);
  g->desc.modes = g->modes.data();
  cudaGetDevice(&g->device);
  const size_t rows = static_cast<size_t>(d->B) * d->Q;
  // the largest index+top-k workspace over the modes this group runs
  size_t ws = csa2_index_topk_workspace(d->B, d->Q, d->N, 0, d->k, d->P);
  if (d->P > 0) {
    const size_t w2 = csa2_index_topk_workspace(d->B, d->Q, d->N, d->P, d->k, 0);
    if (w2 > ws) ws = w2;
  }
  size_t wa = csa2_sparse_attn_workspace(d->B, d->Q, d->Ha, d->D, d->k, d->kv_fmt);
  const size_t wa2 = csa2_sparse_attn_swa_workspace(d->B, d->Q, d->Ha, d->D, d->k, d->kv_fmt);
  if (wa2 > wa) wa = wa2;
  if (wa > ws) ws = wa;
  g->ws_bytes = a256(ws);
  cudaError_t e = cudaMalloc(&g->topk, a256(rows * d->k * sizeof(int32_t)));
  if (e == cudaSuccess && d->P > 0) e = cudaMalloc(&g->pool, a256(rows * d->P * sizeof(int32_t)));
  if (e == cudaSuccess) e = cudaMalloc(&g->ws, g->ws_bytes);
  if (e == cudaSuccess) e = cudaMalloc(&g->attn_sync, 2 * kAttnMaxGrid * sizeof(unsigned long long));
  if (e == cudaSuccess) e = cudaMemset(g->attn_sync, 0, 2 * kAttnMaxGrid * sizeof(unsigned long long));
  if (e != cudaSuccess) {
    cudaGetLastError();
    csa2_group_destroy(g);
    return fail(CSA2_ERR_OOM, "csa2_group_create: cudaMalloc failed: %s", cudaGetErrorString(e));
  }
  *group = g;
  return CSA2_OK;
}

void csa2_group_destroy(csa2_group* g) {
  if (!g) return;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(g->device);
  if (g->topk) cudaFree(g->topk);
  if (g->pool) cudaFree(g->pool);
  if (g->ws) cudaFree(g->ws);
  if (g->attn_sync) cudaFree(g->attn_sync);
  cudaSetDevice(prev);
  delete g;
}

csa2_status csa2_group_selection(const csa2_group* g, const int32_t** topk, const int32_t** pool) {
  if (!g) return fail(CSA2_ERR_INVALID, "csa2_group_selection: null group");
  if (topk) *topk = g->topk;
  if (pool) *pool = g->pool;
  return CSA2_OK;
}

csa2_status csa2_group_copy_selection(const csa2_group* g, int32_t* topk, int32_t* pool,
                                      csa2_stream stream) {
  CSA2_TRY(fault_gate());
  if (!g) return fail(CSA2_ERR_INVALID, "csa2_group_copy_selection: null group");
  if (pool && !g->pool) return fail(CSA2_ERR_MODE, "csa2_group_copy_selection: group has no pool");
  const size_t rows = static_cast<size_t>(g->desc.B) * g->desc.Q;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (topk && cudaMemcpyAsync(topk, g->topk, rows * g->desc.k * sizeof(int32_t),
                              cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return check_launch("csa2_group_copy_selection");
  if (pool && cudaMemcpyAsync(pool, g->pool, rows * g->desc.P * sizeof(int32_t),
                              cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return check_launch("csa2_group_copy_selection");
  return CSA2_OK;
}

csa2_status csa2_group_layer(csa2_group* g, int layer, const csa2_layer_io* io,
                             csa2_stream stream) {
  CSA2_TRY(fault_gate());
  if (!g || !io) return fail(CSA2_ERR_INVALID, "csa2_group_layer: null argument");
  if (layer < 0 || layer >= g->desc.n_layers)
    return fail(CSA2_ERR_INVALID, "csa2_group_layer: layer %d outside [0, %d)", layer,
                g->desc.n_layers);
  const csa2_group_desc& d = g->desc;
  const csa2_mode mode = g->modes[layer];
  if (mode != CSA2_FULL && !g->have_full)
    return fail(CSA2_ERR_MODE, "csa2_group_layer: layer %d (%s) needs a Full layer before it",
                layer, mode == CSA2_REINDEX ? "Reindex" : "Reuse");
  if (mode == CSA2_FULL) {
    if (!io->index_k || !io->kv.data)
      return fail(CSA2_ERR_INVALID, "csa2_group_layer: Full layer %d needs kv and index_k", layer);
    if (io->kv.fmt != d.kv_fmt || io->kv.dim != d.D || io->kv.n != d.N)
      return fail(CSA2_ERR_INVALID, "csa2_group_layer: kv does not match the group descriptor");
  }
  if (mode != CSA2_REUSE && (!io->q_index || !io->w_index))
    return fail(CSA2_ERR_INVALID, "csa2_group_layer: layer %d needs q_index and w_index", layer);
  csa2_status s;
  if (mode == CSA2_FULL) {
    s = csa2_index_topk(CSA2_FULL, io->q_index, io->w_index, io->index_k, d.B, d.Q, d.Hi, d.d, d.N,
                        io->n_visible, nullptr, 0, d.k, g->topk, d.P > 0 ? g->pool : nullptr, d.P,
                        d.act, g->ws, g->ws_bytes, stream);
    if (s != CSA2_OK) return s;
    g->kv = io->kv;
    g->index_k = io->index_k;
    g->have_full = true;
  } else if (mode == CSA2_REINDEX) {
    s = csa2_index_topk(CSA2_REINDEX, io->q_index, io->w_index, g->index_k, d.B, d.Q, d.Hi, d.d,
                        d.N, d.P > 0 ? nullptr : io->n_visible, d.P > 0 ? g->pool : nullptr,
                        d.P, d.k, g->topk, nullptr, 0, d.act, g->ws, g->ws_bytes, stream);
    if (s != CSA2_OK) return s;
  }
  AttnRows rows;
  if (io->swa_kv) {             // this layer's own sliding-window branch
    rows.win = io->swa_kv;
    rows.win_rows = io->swa_rows;
    rows.win_end = io->swa_end;
    rows.W = io->swa_window;
  }
  return sparse_attn_checked(mode, io->q_attn, &g->kv, g->topk, d.B, d.Q, d.Ha, d.k, d.scale,
                             io->out, io->lse, g->ws, g->ws_bytes,
                             g->attn_sync + (io->swa_kv ? kAttnMaxGrid : 0),
                             reinterpret_cast<cudaStream_t>(stream), rows);
}

}  // extern "C"
