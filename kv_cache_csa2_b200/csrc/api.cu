// The C ABI of libcsa2 (include/csa2.h): argument validation, status and
// error plumbing, the per-device error word, launch counters, host-side fault
// injection, and the composite index+top-k call.  The layer-group driver is in
// group.cu.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "launchers.h"

namespace csa2 {

// ------------------------------------------------------------------ status
static thread_local char t_msg[512] = "";

csa2_status fail(csa2_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_msg, sizeof(t_msg), fmt, ap);
  va_end(ap);
  return s;
}

csa2_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return CSA2_OK;
  return fail(CSA2_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ----------------------------------------------------------- fault injection
static std::atomic<int> g_fault{-1};  // -1: not yet read from the environment

static int parse_fault(const char* k) {
  if (!k || !*k) return 0;
  if (!strcmp(k, "alloc")) return 1;
  if (!strcmp(k, "launch")) return 2;
  return -2;
}

csa2_status fault_gate() {
  int f = g_fault.load();
  if (f == -1) {
    f = parse_fault(getenv("CSA2_FAULT"));
    if (f < 0) f = 0;
    g_fault.store(f);
  }
  if (f == 1) return fail(CSA2_ERR_OOM, "injected fault: alloc");
  if (f == 2) return fail(CSA2_ERR_CUDA, "injected fault: launch");
  return CSA2_OK;
}

// ---------------------------------------------------------- launch counters
static std::atomic<long long> g_launches[LK_NUM];

// -------------------------------------------------------- launch timing
struct TimedLaunch {
  int kind;
  cudaEvent_t start, stop;
};
static std::atomic<bool> g_timing{false};
static std::mutex g_tmu;
static std::vector<cudaEvent_t> g_event_pool;
static std::vector<TimedLaunch> g_timed;
static double g_ms[LK_NUM];
static long long g_timed_n[LK_NUM];
static thread_local cudaEvent_t t_start = nullptr;

static cudaEvent_t take_event() {
  std::lock_guard<std::mutex> lk(g_tmu);
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return e;
}

static bool capturing(cudaStream_t s) {
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &st) != cudaSuccess) {
    cudaGetLastError();
    return true;
  }
  return st != cudaStreamCaptureStatusNone;
}

void begin_launch(cudaStream_t s) {
  if (!g_timing.load(std::memory_order_relaxed) || capturing(s)) return;
  t_start = take_event();
  if (t_start) cudaEventRecord(t_start, s);
}

void note_launch(LaunchKind kind, int n, cudaStream_t s) {
  g_launches[kind] += n;
  if (!t_start) return;
  cudaEvent_t stop = take_event();
  if (stop) {
    cudaEventRecord(stop, s);
    std::lock_guard<std::mutex> lk(g_tmu);
    g_timed.push_back({static_cast<int>(kind), t_start, stop});
  }
  t_start = nullptr;
}

// ------------------------------------------------------- device error word
__device__ int g_dev_err;

static std::mutex g_dev_mu;
static int* g_err_ptr[kMaxDevices];
static int g_sms[kMaxDevices];

static int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  return dev < kMaxDevices ? dev : kMaxDevices - 1;
}

int current_device_or_none() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return dev >= 0 && dev < kMaxDevices ? dev : -1;
}

int* device_error_word() {
  const int dev = current_device();
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev_err) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_err_ptr[dev] = static_cast<int*>(p);
  }
  return g_err_ptr[dev];
}

bool pdl_enabled() {
  static const bool on = getenv("CSA2_NO_PDL") == nullptr;
  return on;
}

// ------------------------------------------------------ cross-CTA wait bound
static std::atomic<unsigned long long> g_wait_ns{0};     // 0: the default
static std::atomic<int> g_wait_unreachable{0};

unsigned long long cross_cta_wait_ns() {
  const unsigned long long v = g_wait_ns.load(std::memory_order_relaxed);
  return v ? v : kDefaultCrossCtaWaitNs;
}

unsigned cross_cta_wait_offset() {
  return g_wait_unreachable.load(std::memory_order_relaxed) ? kUnreachableWaitOffset : 0u;
}

int sm_count() {
  const int dev = current_device();
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_sms[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_sms[dev] = n > 0 ? n : 1;
  }
  return g_sms[dev];
}

}  // namespace csa2

using namespace csa2;

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

#define REQUIRE(cond, ...) \
  do {                     \
    if (!(cond)) return fail(CSA2_ERR_INVALID, __VA_ARGS__); \
  } while (0)
#define REQUIRE_PTR(p) REQUIRE((p) != nullptr && aligned16(p), "%s: pointer " #p " is null or not 16-byte aligned", __func__)

namespace csa2 {
csa2_status sparse_attn_checked(csa2_mode mode, const void* q, const csa2_kv* kv,
                                const int32_t* topk, int B, int Q, int Ha, int k, float scale,
                                void* out, float* lse, void* workspace, size_t workspace_bytes,
                                unsigned long long* sync_zeroed, cudaStream_t stream,
                                const AttnRows& rows) {
  CSA2_TRY(fault_gate());
  REQUIRE(mode == CSA2_FULL || mode == CSA2_REINDEX || mode == CSA2_REUSE,
          "csa2_sparse_attn: unknown mode %d", int(mode));
  REQUIRE(kv != nullptr, "csa2_sparse_attn: kv is null");
  REQUIRE(B >= 0 && Q >= 0 && k >= 0 && Ha > 0, "csa2_sparse_attn: bad size");
  REQUIRE(kv->fmt == CSA2_KV_BF16 || kv->fmt == CSA2_KV_FP4, "csa2_sparse_attn: unknown kv format");
  REQUIRE(kv->dim > 0 && kv->dim % 16 == 0, "csa2_sparse_attn: D=%d must be a multiple of 16", kv->dim);
  REQUIRE(kv->n >= 0 && kv->n <= 0x7fffffffLL, "csa2_sparse_attn: bad kv->n");
  if (B == 0 || Q == 0) return CSA2_OK;
  REQUIRE_PTR(q); REQUIRE_PTR(out); REQUIRE_PTR(kv->data);
  REQUIRE(kv->fmt == CSA2_KV_BF16 || kv->scales != nullptr, "csa2_sparse_attn: FP4 kv without scales");
  if (rows.win) {
    REQUIRE(aligned16(rows.win) && rows.win_end != nullptr && rows.win_rows >= 0 &&
                rows.win_rows <= 0x7fffffffLL && rows.W >= 1 && rows.W <= kMaxWindow,
            "csa2_sparse_attn: window rows need a 16-byte aligned buffer, win_end and 1 <= W <= %d",
            kMaxWindow);
  }
  const size_t need = sparse_attn_workspace(B, Q, Ha, kv->dim, k, kv->fmt, rows.win != nullptr);
  if (workspace_bytes < need || (need > 0 && !workspace))
    return fail(CSA2_ERR_OOM, "csa2_sparse_attn: workspace %zu < %zu bytes", workspace_bytes, need);
  return launch_sparse_attn(q, *kv, topk, B, Q, Ha, k, scale, out, lse, workspace, workspace_bytes,
                            sync_zeroed, stream, rows);
}
}  // namespace csa2


extern "C" {

const char* csa2_status_string(csa2_status s) {
  switch (s) {
    case CSA2_OK: return "CSA2_OK";
    case CSA2_ERR_INVALID: return "CSA2_ERR_INVALID";
    case CSA2_ERR_MODE: return "CSA2_ERR_MODE";
    case CSA2_ERR_UNSUPPORTED: return "CSA2_ERR_UNSUPPORTED";
    case CSA2_ERR_CUDA: return "CSA2_ERR_CUDA";
    case CSA2_ERR_TIMEOUT: return "CSA2_ERR_TIMEOUT";
    case CSA2_ERR_OOM: return "CSA2_ERR_OOM";
    case CSA2_ERR_BOUNDS: return "CSA2_ERR_BOUNDS";
  }
  return "CSA2_ERR_UNKNOWN";
}

const char* csa2_last_error(void) { return t_msg; }

int csa2_version(void) { return 2; }

csa2_status csa2_set_device_wait(uint64_t limit_ns, int unreachable) {
  g_wait_ns.store(limit_ns);
  g_wait_unreachable.store(unreachable ? 1 : 0);
  return CSA2_OK;
}

csa2_status csa2_set_fault(const char* kind) {
  const int f = parse_fault(kind);
  if (f < 0) return fail(CSA2_ERR_INVALID, "csa2_set_fault: unknown kind '%s'", kind);
  g_fault.store(f);
  return CSA2_OK;
}

int csa2_launch_counts(int64_t* counts, int n) {
  for (int i = 0; i < n && i < LK_NUM; ++i) counts[i] = g_launches[i].load();
  return LK_NUM;
}

void csa2_reset_launch_counts(void) {
  for (int i = 0; i < LK_NUM; ++i) g_launches[i] = 0;
}

csa2_status csa2_timing_enable(int on) {
  g_timing.store(on != 0);
  return CSA2_OK;
}

int csa2_kernel_times(double* ms, int64_t* launches, int n) {
  std::vector<TimedLaunch> pending;
  {
    std::lock_guard<std::mutex> lk(g_tmu);
    pending.swap(g_timed);
  }
  for (const TimedLaunch& t : pending) {
    float f = 0.0f;
    if (cudaEventSynchronize(t.stop) == cudaSuccess &&
        cudaEventElapsedTime(&f, t.start, t.stop) == cudaSuccess) {
      std::lock_guard<std::mutex> lk(g_tmu);
      g_ms[t.kind] += f;
      g_timed_n[t.kind] += 1;
    } else {
      cudaGetLastError();
    }
    std::lock_guard<std::mutex> lk(g_tmu);
    g_event_pool.push_back(t.start);
    g_event_pool.push_back(t.stop);
  }
  std::lock_guard<std::mutex> lk(g_tmu);
  for (int i = 0; i < n && i < LK_NUM; ++i) {
    if (ms) ms[i] = g_ms[i];
    if (launches) launches[i] = g_timed_n[i];
  }
  return LK_NUM;
}

void csa2_timing_reset(void) {
  csa2_kernel_times(nullptr, nullptr, 0);   // drain what is pending
  std::lock_guard<std::mutex> lk(g_tmu);
  for (int i = 0; i < LK_NUM; ++i) {
    g_ms[i] = 0.0;
    g_timed_n[i] = 0;
  }
}

csa2_status csa2_device_error(csa2_stream stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(CSA2_ERR_CUDA, "csa2_device_error: %s", cudaGetErrorString(e));
  int* w = device_error_word();
  if (!w) return fail(CSA2_ERR_CUDA, "csa2_device_error: no error word on this device");
  int v = 0;
  e = cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(CSA2_ERR_CUDA, "csa2_device_error: %s", cudaGetErrorString(e));
  if (v != 0) {
    const int zero = 0;
    cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice);
    return fail(static_cast<csa2_status>(v), "device-side error %s recorded by a kernel",
                csa2_status_string(static_cast<csa2_status>(v)));
  }
  return CSA2_OK;
}

// ------------------------------------------------------------- (a1)
csa2_status csa2_compress(const void* c, const float* z, const float* bias, int B, int64_t T,
                          int D, int m, int has_left_halo, void* out, int64_t out_batch_stride,
                          csa2_stream stream) {
  CSA2_TRY(fault_gate());
  REQUIRE(B >= 0 && T >= 0, "csa2_compress: negative size (B=%d, T=%lld)", B, (long long)T);
  REQUIRE(D > 0 && D % 8 == 0, "csa2_compress: D=%d must be a positive multiple of 8", D);
  REQUIRE(m >= 1 && m <= 16, "csa2_compress: m=%d outside [1, 16]", m);
  const int64_t N = T / m;
  if (B == 0 || N == 0) return CSA2_OK;
  REQUIRE_PTR(c); REQUIRE_PTR(z); REQUIRE_PTR(bias); REQUIRE_PTR(out);
  if (out_batch_stride == 0) out_batch_stride = N * D;
  REQUIRE(out_batch_stride >= N * D && out_batch_stride % 8 == 0,
          "csa2_compress: out_batch_stride=%lld must be >= (T/m)*D and a multiple of 8",
          (long long)out_batch_stride);
  return launch_compress(c, z, bias, B, T, D, m, has_left_halo ? 1 : 0, out, out_batch_stride,
                         reinterpret_cast<cudaStream_t>(stream));
}

csa2_status csa2_compress_hca(const void* c, const float* z, const float* bias, int B, int64_t T,
                              int D, int m, void* out, int64_t out_batch_stride,
                              csa2_stream stream) {
  CSA2_TRY(fault_gate());
  REQUIRE(B >= 0 && T >= 0, "csa2_compress_hca: negative size (B=%d, T=%lld)", B, (long long)T);
  REQUIRE(D > 0 && D % 8 == 0, "csa2_compress_hca: D=%d must be a positive multiple of 8", D);
  REQUIRE(m >= 1 && m <= kMaxHcaBlock, "csa2_compress_hca: m=%d outside [1, %d]", m, kMaxHcaBlock);
  const int64_t N = T / m;
  if (B == 0 || N == 0) return CSA2_OK;
  REQUIRE_PTR(c); REQUIRE_PTR(z); REQUIRE_PTR(bias); REQUIRE_PTR(out);
  if (out_batch_stride == 0) out_batch_stride = N * D;
  REQUIRE(out_batch_stride >= N * D && out_batch_stride % 8 == 0,
          "csa2_compress_hca: out_batch_stride=%lld must be >= (T/m)*D and a multiple of 8",
          (long long)out_batch_stride);
  return launch_compress_hca(c, z, bias, B, T, D, m, out, out_batch_stride,
                             reinterpret_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------- (a2)
static csa2_status check_index_args(const char* fn, const void* q, const float* w, const void* k,
                                    int B, int Q, int H, int d, int64_t N, const int32_t* pool,
                                    int P) {
  if (B < 0 || Q < 0 || N < 0) return fail(CSA2_ERR_INVALID, "%s: negative size", fn);
  if (H <= 0 || H > 128) return fail(CSA2_ERR_INVALID, "%s: H=%d outside [1, 128]", fn, H);
  if (d <= 0 || d % 8 != 0 || d > 256)
    return fail(CSA2_ERR_INVALID, "%s: d=%d must be a multiple of 8 in [8, 256]", fn, d);
  if (N > 0x7fffffffLL) return fail(CSA2_ERR_INVALID, "%s: N too large", fn);
  if (pool && P <= 0) return fail(CSA2_ERR_INVALID, "%s: pool given with P=%d", fn, P);
  if (B == 0 || Q == 0) return CSA2_OK;
  if (!q || !aligned16(q) || !w || !k || !aligned16(k))
    return fail(CSA2_ERR_INVALID, "%s: q/w/k null or q/k not 16-byte aligned", fn);
  return CSA2_OK;
}

csa2_status csa2_index_scores(const void* q, const float* w, const void* k, int B, int Q, int H,
                              int d, int64_t N, const int32_t* n_visible, const int32_t* pool,
                              int P, csa2_index_act act, float* scores, csa2_stream stream) {
  CSA2_TRY(fault_gate());
  CSA2_TRY(check_index_args(__func__, q, w, k, B, Q, H, d, N, pool, P));
  if (B == 0 || Q == 0) return CSA2_OK;
  REQUIRE(scores != nullptr, "csa2_index_scores: scores is null");
  return launch_index_scores(q, w, k, B, Q, H, d, N, n_visible, pool, pool ? P : 0, act, scores,
                             reinterpret_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------- (a3)
size_t csa2_select_topk_workspace(int64_t rows, int64_t L, int count) {
  return select_topk_workspace(rows, L, count);
}

csa2_status csa2_select_topk(const float* scores, int64_t rows, int64_t L, int count,
                             const int32_t* ids, int32_t* out, void* workspace,
                             size_t workspace_bytes, csa2_stream stream) {
  CSA2_TRY(fault_gate());
  REQUIRE(rows >= 0 && L >= 0 && count >= 0, "csa2_select_topk: negative size");
  REQUIRE(L <= 0x7fffffffLL, "csa2_select_topk: L too large");
  if (rows == 0 || count == 0) return CSA2_OK;
  REQUIRE(out != nullptr && (L == 0 || scores != nullptr), "csa2_select_topk: null pointer");
  const size_t need = select_topk_workspace(rows, L, count);
  if (workspace_bytes < need)
    return fail(CSA2_ERR_OOM, "csa2_select_topk: workspace %zu < %zu bytes", workspace_bytes, need);
  return launch_select_topk(scores, rows, L, count, ids, out, workspace, workspace_bytes,
                            reinterpret_cast<cudaStream_t>(stream));
}

size_t csa2_index_topk_workspace(int B, int Q, int64_t N, int P_in, int k_top, int P_out) {
  const int64_t L = P_in > 0 ? P_in : N;
  const int64_t rows = static_cast<int64_t>(B) * Q;
  size_t sel = select_topk_workspace(rows, L, k_top);
  if (P_out > 0) {
    const size_t s2 = select_topk_workspace(rows, L, P_out);
    if (s2 > sel) sel = s2;
  }
  return align256(static_cast<size_t>(rows) * L * sizeof(float)) + align256(sel);
}

csa2_status csa2_index_topk(csa2_mode mode, const void* q, const float* w, const void* k, int B,
                            int Q, int H, int d, int64_t N, const int32_t* n_visible,
                            const int32_t* pool_in, int P_in, int k_top, int32_t* topk_out,
                            int32_t* pool_out, int P_out, csa2_index_act act, void* workspace,
                            size_t workspace_bytes, csa2_stream stream) {
  CSA2_TRY(fault_gate());
  if (mode == CSA2_REUSE)
    return fail(CSA2_ERR_MODE, "csa2_index_topk: a Reuse layer runs no indexer");
  if (mode != CSA2_FULL && mode != CSA2_REINDEX)
    return fail(CSA2_ERR_INVALID, "csa2_index_topk: unknown mode %d", int(mode));
  if (mode == CSA2_FULL && pool_in)
    return fail(CSA2_ERR_MODE, "csa2_index_topk: a Full layer builds its pool, pool_in must be NULL");
  if (mode == CSA2_REINDEX && pool_out)
    return fail(CSA2_ERR_MODE, "csa2_index_topk: a Reindex layer keeps no pool, pool_out must be NULL");
  CSA2_TRY(check_index_args(__func__, q, w, k, B, Q, H, d, N, pool_in, P_in));
  REQUIRE(k_top > 0, "csa2_index_topk: k_top=%d must be positive", k_top);
  REQUIRE(!pool_out || P_out > 0, "csa2_index_topk: pool_out given with P_out=%d", P_out);
  if (B == 0 || Q == 0) return CSA2_OK;
  REQUIRE(topk_out != nullptr, "csa2_index_topk: topk_out is null");
  const int64_t L = pool_in ? P_in : N;
  const int64_t rows = static_cast<int64_t>(B) * Q;
  const size_t need = csa2_index_topk_workspace(B, Q, N, pool_in ? P_in : 0, k_top,
                                                pool_out ? P_out : 0);
  if (!workspace || workspace_bytes < need)
    return fail(CSA2_ERR_OOM, "csa2_index_topk: workspace %zu < %zu bytes", workspace_bytes, need);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // many queries and no pool: scoring and selection in one kernel, no score round trip
  if (!pool_in && !pool_out && index_topk_fused_applies(B, Q, H, d, N, k_top))
    return launch_index_topk_fused(q, w, k, B, Q, H, d, N, n_visible, k_top, act, topk_out, s);
  float* scores = static_cast<float*>(workspace);
  const size_t sbytes = align256(static_cast<size_t>(rows) * L * sizeof(float));
  void* sel_ws = static_cast<char*>(workspace) + sbytes;
  const size_t sel_bytes = workspace_bytes - sbytes;
  // the dual selection's counters are cleared by the scoring kernel (or else
  // just after it), so that the selection follows that kernel directly
  // (programmatic dependent launch)
  ClearOnLaunch clear;
  if (pool_out) clear = select_topk_clear_region(rows, L, sel_ws, sel_bytes);
  CSA2_TRY(launch_index_scores(q, w, k, B, Q, H, d, N, n_visible, pool_in, pool_in ? P_in : 0, act,
                               scores, s, clear.ptr ? &clear : nullptr));
  if (pool_out && clear.ptr && !clear.done) CSA2_TRY(select_topk_clear(rows, L, sel_ws, sel_bytes, s));
  if (pool_out) {
    // the pool and the top-k in the same selection passes when the kernel applies
    const csa2_status st = launch_select_topk2(scores, rows, L, k_top, nullptr, topk_out, P_out,
                                               pool_out, sel_ws, sel_bytes, s, true);
    if (st != CSA2_ERR_UNSUPPORTED) return st;
  }
  CSA2_TRY(launch_select_topk(scores, rows, L, k_top, pool_in, topk_out, sel_ws, sel_bytes, s));
  if (pool_out)
    CSA2_TRY(launch_select_topk(scores, rows, L, P_out, nullptr, pool_out, sel_ws, sel_bytes, s));
  return CSA2_OK;
}

// ------------------------------------------------------------- (a2, a3) FP4 indexer
static csa2_status check_fp4_index_args(const char* fn, const uint8_t* q_codes,
                                        const uint8_t* q_scales, const float* w,
                                        const uint8_t* k_codes, const uint8_t* k_scales, int B,
                                        int Q, int H, int d, int64_t N, const int32_t* pool, int P) {
  if (B < 0 || Q < 0 || N < 0) return fail(CSA2_ERR_INVALID, "%s: negative size", fn);
  if (H <= 0 || H > 64) return fail(CSA2_ERR_INVALID, "%s: H=%d outside [1, 64]", fn, H);
  if (d != 64 && d != 128) return fail(CSA2_ERR_INVALID, "%s: d=%d must be 64 or 128", fn, d);
  if (N > 0x7fffffffLL) return fail(CSA2_ERR_INVALID, "%s: N too large", fn);
  if (pool && P <= 0) return fail(CSA2_ERR_INVALID, "%s: pool given with P=%d", fn, P);
  if (B == 0 || Q == 0) return CSA2_OK;
  const uintptr_t sal = static_cast<uintptr_t>(d / 16) - 1;   // scale rows: 8 or 4 bytes
  if (!q_codes || !q_scales || !w || !k_codes || !k_scales || !aligned16(k_codes) ||
      (reinterpret_cast<uintptr_t>(q_codes) & 7) || (reinterpret_cast<uintptr_t>(k_scales) & sal))
    return fail(CSA2_ERR_INVALID,
                "%s: null pointer, or k_codes not 16-byte, q_codes not 8-byte, k_scales not %d-byte aligned",
                fn, d / 16);
  return CSA2_OK;
}

csa2_status csa2_index_scores_fp4(const uint8_t* q_codes, const uint8_t* q_scales, const float* w,
                                  const uint8_t* k_codes, const uint8_t* k_scales, int B, int Q,
                                  int H, int d, int64_t N, const int32_t* n_visible,
                                  const int32_t* pool, int P, csa2_index_act act, void* scores,
                                  csa2_stream stream) {
  CSA2_TRY(fault_gate());
  CSA2_TRY(check_fp4_index_args(__func__, q_codes, q_scales, w, k_codes, k_scales, B, Q, H, d, N, pool, P));
  if (B == 0 || Q == 0) return CSA2_OK;
  REQUIRE(scores != nullptr, "csa2_index_scores_fp4: scores is null");
  Fp4IndexArgs a{q_codes, q_scales, w, k_codes, k_scales, B, Q, H, d, N, n_visible, pool,
                 pool ? P : 0, act, scores};
  return launch_index_scores_fp4(a, true, reinterpret_cast<cudaStream_t>(stream));
}

csa2_status csa2_index_topk_fp4(csa2_mode mode, const uint8_t* q_codes, const uint8_t* q_scales,
                                const float* w, const uint8_t* k_codes, const uint8_t* k_scales,
                                int B, int Q, int H, int d, int64_t N, const int32_t* n_visible,
                                const int32_t* pool_in, int P_in, int k_top, int32_t* topk_out,
                                int32_t* pool_out, int P_out, csa2_index_act act, void* workspace,
                                size_t workspace_bytes, csa2_stream stream) {
  CSA2_TRY(fault_gate());
  if (mode == CSA2_REUSE)
    return fail(CSA2_ERR_MODE, "csa2_index_topk_fp4: a Reuse layer runs no indexer");
  if (mode != CSA2_FULL && mode != CSA2_REINDEX)
    return fail(CSA2_ERR_INVALID, "csa2_index_topk_fp4: unknown mode %d", int(mode));
  if (mode == CSA2_FULL && pool_in)
    return fail(CSA2_ERR_MODE, "csa2_index_topk_fp4: a Full layer builds its pool, pool_in must be NULL");
  if (mode == CSA2_REINDEX && pool_out)
    return fail(CSA2_ERR_MODE, "csa2_index_topk_fp4: a Reindex layer keeps no pool, pool_out must be NULL");
  CSA2_TRY(check_fp4_index_args(__func__, q_codes, q_scales, w, k_codes, k_scales, B, Q, H, d, N,
                                pool_in, P_in));
  REQUIRE(k_top > 0, "csa2_index_topk_fp4: k_top=%d must be positive", k_top);
  REQUIRE(!pool_out || P_out > 0, "csa2_index_topk_fp4: pool_out given with P_out=%d", P_out);
  if (B == 0 || Q == 0) return CSA2_OK;
  REQUIRE(topk_out != nullptr, "csa2_index_topk_fp4: topk_out is null");
  const int64_t L = pool_in ? P_in : N;
  const int64_t rows = static_cast<int64_t>(B) * Q;
  const size_t need = csa2_index_topk_workspace(B, Q, N, pool_in ? P_in : 0, k_top, pool_out ? P_out : 0);
  if (!workspace || workspace_bytes < need)
    return fail(CSA2_ERR_OOM, "csa2_index_topk_fp4: workspace %zu < %zu bytes", workspace_bytes, need);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* scores = static_cast<float*>(workspace);          // f32 holding bf16 values
  const size_t sbytes = align256(static_cast<size_t>(rows) * L * sizeof(float));
  void* sel_ws = static_cast<char*>(workspace) + sbytes;
  const size_t sel_bytes = workspace_bytes - sbytes;
  Fp4IndexArgs a{q_codes, q_scales, w, k_codes, k_scales, B, Q, H, d, N, n_visible, pool_in,
                 pool_in ? P_in : 0, act, scores};
  CSA2_TRY(launch_index_scores_fp4(a, false, s));
  if (pool_out) {
    CSA2_TRY(select_topk_clear(rows, L, sel_ws, sel_bytes, s));
    const csa2_status st = launch_select_topk2(scores, rows, L, k_top, nullptr, topk_out, P_out,
                                               pool_out, sel_ws, sel_bytes, s, true);
    if (st != CSA2_ERR_UNSUPPORTED) return st;
  }
  CSA2_TRY(launch_select_topk(scores, rows, L, k_top, pool_in, topk_out, sel_ws, sel_bytes, s));
  if (pool_out)
    CSA2_TRY(launch_select_topk(scores, rows, L, P_out, nullptr, pool_out, sel_ws, sel_bytes, s));
  return CSA2_OK;
}

// ------------------------------------------------------------- (a4)
size_t csa2_sparse_attn_workspace(int B, int Q, int Ha, int D, int k, csa2_kv_fmt fmt) {
  return sparse_attn_workspace(B, Q, Ha, D, k, fmt);
}

csa2_status csa2_sparse_attn(csa2_mode mode, const void* q, const csa2_kv* kv,
                             const int32_t* topk, int B, int Q, int Ha, int k, float scale,
                             void* out, float* lse, void* workspace, size_t workspace_bytes,
                             csa2_stream stream) {
  REQUIRE(k <= 0 || B <= 0 || Q <= 0 || topk != nullptr, "csa2_sparse_attn: topk is null");
  return sparse_attn_checked(mode, q, kv, topk, B, Q, Ha, k, scale, out, lse, workspace,
                             workspace_bytes, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

size_t csa2_sparse_attn_swa_workspace(int B, int Q, int Ha, int D, int k, csa2_kv_fmt fmt) {
  return sparse_attn_workspace(B, Q, Ha, D, k, fmt, true);
}

csa2_status csa2_sparse_attn_swa(csa2_mode mode, const void* q, const csa2_kv* kv,
                                 const int32_t* topk, int B, int Q, int Ha, int k, float scale,
                                 const void* win, int64_t win_rows, const int32_t* win_end, int W,
                                 void* out, float* lse, void* workspace, size_t workspace_bytes,
                                 csa2_stream stream) {
  REQUIRE(k <= 0 || B <= 0 || Q <= 0 || topk != nullptr, "csa2_sparse_attn_swa: topk is null");
  REQUIRE(win != nullptr, "csa2_sparse_attn_swa: window rows are null");
  AttnRows rows;
  rows.win = win;
  rows.win_rows = win_rows;
  rows.win_end = win_end;
  rows.W = W;
  return sparse_attn_checked(mode, q, kv, topk, B, Q, Ha, k, scale, out, lse, workspace,
                             workspace_bytes, nullptr, reinterpret_cast<cudaStream_t>(stream), rows);
}

size_t csa2_dense_attn_workspace(int B, int Q, int Ha, int D, int64_t N, csa2_kv_fmt fmt) {
  if (N < 0 || N > 0x7fffffffLL) return 0;
  return sparse_attn_workspace(B, Q, Ha, D, static_cast<int>(N), fmt, false);
}

csa2_status csa2_dense_attn(const void* q, const csa2_kv* kv, const int32_t* n_visible, int B,
                            int Q, int Ha, float scale, void* out, float* lse, void* workspace,
                            size_t workspace_bytes, csa2_stream stream) {
  REQUIRE(kv != nullptr, "csa2_dense_attn: kv is null");
  REQUIRE(kv->n >= 0 && kv->n <= 0x7fffffffLL, "csa2_dense_attn: bad kv->n");
  AttnRows rows;
  rows.n_visible = n_visible;
  return sparse_attn_checked(CSA2_FULL, q, kv, nullptr, B, Q, Ha, static_cast<int>(kv->n), scale,
                             out, lse, workspace, workspace_bytes, nullptr,
                             reinterpret_cast<cudaStream_t>(stream), rows);
}

// ------------------------------------------------------------- (a5)
csa2_status csa2_fp4_pack(const void* x, int64_t rows, int D, uint8_t* codes, uint8_t* scales,
                          csa2_stream stream) {
  CSA2_TRY(fault_gate());
  REQUIRE(rows >= 0 && D > 0 && D % 16 == 0, "csa2_fp4_pack: D=%d must be a multiple of 16", D);
  if (rows == 0) return CSA2_OK;
  REQUIRE_PTR(x);
  REQUIRE(codes && (reinterpret_cast<uintptr_t>(codes) & 7) == 0 && scales,
          "csa2_fp4_pack: codes null or not 8-byte aligned, or scales null");
  return launch_fp4_pack(x, rows, D, codes, scales, reinterpret_cast<cudaStream_t>(stream));
}

csa2_status csa2_fp4_unpack(const uint8_t* codes, const uint8_t* scales, int64_t rows, int D,
                            void* x, csa2_stream stream) {
  CSA2_TRY(fault_gate());
  REQUIRE(rows >= 0 && D > 0 && D % 16 == 0, "csa2_fp4_unpack: D=%d must be a multiple of 16", D);
  if (rows == 0) return CSA2_OK;
  REQUIRE_PTR(x);
  REQUIRE(codes && (reinterpret_cast<uintptr_t>(codes) & 7) == 0 && scales,
          "csa2_fp4_unpack: codes null or not 8-byte aligned, or scales null");
  return launch_fp4_unpack(codes, scales, rows, D, x, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
