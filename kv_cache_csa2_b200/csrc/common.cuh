// Shared internals of libcsa2: status plumbing, the per-device error word,
// launch counters and small device helpers.  Not part of the C ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "csa2.h"

namespace csa2 {

// ---------------------------------------------------------------- host side
enum LaunchKind {
  LK_COMPRESS = 0,
  LK_INDEX = 1,
  LK_TOPK = 2,
  LK_ATTN = 3,
  LK_COMBINE = 4,
  LK_PACK = 5,
  LK_UNPACK = 6,
  LK_OTHER = 7,
  LK_INDEX_POOL = 8,
  LK_NUM = 9
};
// Call begin_launch(stream) right before a kernel launch and
// note_launch(kind, n, stream) right after it: counts the launch and, when
// timing is enabled, brackets it with events on `stream`.
void begin_launch(cudaStream_t stream);
void note_launch(LaunchKind kind, int n = 1, cudaStream_t stream = nullptr);

// Sets the thread-local message and returns `s`.
csa2_status fail(csa2_status s, const char* fmt, ...);
// CSA2_OK, or CSA2_ERR_CUDA with the pending launch error as the message.
csa2_status check_launch(const char* what);
// Host-side fault injection: returns the injected status or CSA2_OK.
csa2_status fault_gate();
// Device address of the current device's error word (resolved once per device).
int* device_error_word();
// Number of SMs of the current device (cached per device).
int sm_count();
// Ordinal of the current device, or -1 when it cannot be read or is >= kMaxDevices.
constexpr int kMaxDevices = 64;
int current_device_or_none();

// A value computed once per device, with that device current (a kernel's
// shared-memory opt-in or its occupancy binds to the device current when it
// is made).  Devices past kMaxDevices recompute it on every call.
template <class T>
struct PerDevice {
  std::once_flag once[kMaxDevices];
  T value[kMaxDevices] = {};
  T get(T (*make)()) {
    const int dev = current_device_or_none();
    if (dev < 0) return make();
    std::call_once(once[dev], [this, dev, make] { value[dev] = make(); });
    return value[dev];
  }
};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Programmatic dependent launch.  A kernel launched with the attribute from
// pdl_attribute() may start while the kernel before it on the stream is still
// running, once every CTA of that kernel has called pdl_release() (or
// exited); it calls pdl_wait() before it reads anything that kernel wrote
// (the wait returns when that kernel has completed and its writes are
// visible).  Disabled when CSA2_NO_PDL is set.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
bool pdl_enabled();

// Bound of the waits in which one CTA waits for another (the multi-CTA top-k
// row barrier, the attention kernel's wait for another tile's partial):
// csa2_set_device_wait() sets it, by default one second.  A kernel adds
// cross_cta_wait_offset() to the count it waits for: 0, or, for a test of
// the error path, an offset no count ever reaches.
constexpr unsigned long long kDefaultCrossCtaWaitNs = 1000000000ull;
constexpr unsigned kUnreachableWaitOffset = 0x40000000u;
unsigned long long cross_cta_wait_ns();
unsigned cross_cta_wait_offset();
inline cudaLaunchAttribute pdl_attribute() {
  cudaLaunchAttribute a;
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  return a;
}

#define CSA2_TRY(expr)                          \
  do {                                          \
    csa2_status _s = (expr);                    \
    if (_s != CSA2_OK) return _s;               \
  } while (0)

// -------------------------------------------------------------- device side
enum : int { DEVERR_BOUNDS = CSA2_ERR_BOUNDS, DEVERR_TIMEOUT = CSA2_ERR_TIMEOUT };

__device__ __forceinline__ void raise_dev_error(int* word, int code) {
  if (word) atomicCAS(word, 0, code);
}

// bf16 halves of a 32-bit word -> f32 (exact)
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// f32 pair -> packed bf16x2, round to nearest even
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace csa2
