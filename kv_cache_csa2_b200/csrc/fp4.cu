// FP4 main-KV format: E2M1 codes with one E4M3 scale per 16 channels.
// Source: "Recall之王 祭出Reuse", CSA2 bullets, FP4 主KV缓存.
//
// One thread owns one 16-channel block: 32 bytes of bf16 in, 8 bytes of codes
// and 1 scale byte out (pack), or the reverse (unpack).  Both kernels are
// HBM-bound streaming passes with 16-byte loads; every decision is taken with
// exact f32 comparisons, so the result is bit-exact.
#include "common.cuh"
#include "launchers.h"

namespace csa2 {
namespace {

// E4M3 ("fn" variant, bias 7, no inf) code -> value, codes 0..126 only.
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = c >> 3, m = c & 7u;
  if (e == 0) return static_cast<float>(m) * 0x1p-9f;
  return __uint_as_float(((e + 120u) << 23) | (m << 20));  // (1 + m/8) * 2^(e-7)
}

// Scale code: the E4M3 value nearest amax/6, ties to the even code, saturating
// at 448 (code 126).  Division-free: binary search for the largest code whose
// 6x value is <= amax, then compare amax with 6x the midpoint to the next
// code.  6x an E4M3 value or midpoint has at most 7 significant bits, so every
// product and comparison is exact in f32.
__device__ __forceinline__ uint32_t scale_code_for(float amax) {
  uint32_t lo = 0, hi = 126;  // invariant: 6*v(lo) <= amax (v(0) = 0)
  while (lo < hi) {
    const uint32_t mid = (lo + hi + 1) >> 1;
    if (6.0f * e4m3_value(mid) <= amax) lo = mid; else hi = mid - 1;
  }
  if (lo == 126) return 126;
  const float six_mid = 3.0f * (e4m3_value(lo) + e4m3_value(lo + 1));
  if (amax > six_mid) return lo + 1;
  if (amax < six_mid) return lo;
  return (lo & 1u) ? lo + 1 : lo;  // tie: even code
}

// E2M1 magnitude code (0..7) nearest |x|/s with s > 0, ties to the even code,
// saturating at 6.  Thresholds are the grid midpoints times s (exact).
__device__ __forceinline__ uint32_t e2m1_code(float ax, float s) {
  const float mids[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};
  uint32_t c = 0;
#pragma unroll
  for (int i = 0; i < 7; ++i) {
    const float t = mids[i] * s;
    // passing threshold i moves from code i to i+1; at equality only if i+1 is even
    if (ax > t || (ax == t && ((i + 1) & 1) == 0)) c = i + 1;
  }
  return c;
}

__global__ void __launch_bounds__(256) fp4_pack_kernel(const uint4* __restrict__ x,
                                                       int64_t nblocks,
                                                       uint2* __restrict__ codes,
                                                       uint8_t* __restrict__ scales) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i >= nblocks) return;
  const uint4 a = __ldg(x + 2 * i), b = __ldg(x + 2 * i + 1);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t h[16];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    h[2 * j] = w[j] & 0xffffu;
    h[2 * j + 1] = w[j] >> 16;
  }
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) amax = fmaxf(amax, __uint_as_float((h[j] & 0x7fffu) << 16));
  const uint32_t sc = scale_code_for(amax);
  const float s = e4m3_value(sc);
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float ax = __uint_as_float((h[j] & 0x7fffu) << 16);
    uint32_t c = (s > 0.0f) ? e2m1_code(ax, s) : 0u;
    c |= (h[j] >> 12) & 8u;  // sign bit of the bf16 input
    if (j < 8) lo |= c << (4 * j); else hi |= c << (4 * (j - 8));
  }
  codes[i] = make_uint2(lo, hi);
  scales[i] = static_cast<uint8_t>(sc);
}

__global__ void __launch_bounds__(256) fp4_unpack_kernel(const uint2* __restrict__ codes,
                                                         const uint8_t* __restrict__ scales,
                                                         int64_t nblocks, uint4* __restrict__ x) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i >= nblocks) return;
  const uint2 cw = __ldg(codes + i);
  const uint32_t sc = __ldg(scales + i);
  const uint32_t se = (sc >> 3) & 15u, sm = sc & 7u;
  // E4M3 scale as f32 (NaN code 0x7f / 0xff gives NaN)
  float s = (se == 0) ? static_cast<float>(sm) * 0x1p-9f
                      : __uint_as_float(((se + 120u) << 23) | (sm << 20));
  if (se == 15 && sm == 7) s = __uint_as_float(0x7fc00000u);
  if (sc & 128u) s = -s;
  uint32_t out[8];
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    float v[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int ch = j + u;
      const uint32_t c = ((ch < 8 ? cw.x : cw.y) >> (4 * (ch & 7))) & 15u;
      const uint32_t e = (c >> 1) & 3u, mt = c & 1u;
      float mag = (e == 0) ? 0.5f * static_cast<float>(mt)
                           : (1.0f + 0.5f * static_cast<float>(mt)) * static_cast<float>(1u << (e - 1));
      if (c & 8u) mag = -mag;
      v[u] = mag * s;  // exact: at most 5 significant bits
    }
    out[j / 2] = pack_bf16x2(v[0], v[1]);
  }
  x[2 * i] = make_uint4(out[0], out[1], out[2], out[3]);
  x[2 * i + 1] = make_uint4(out[4], out[5], out[6], out[7]);
}

}  // namespace

csa2_status launch_fp4_pack(const void* x, int64_t rows, int D, uint8_t* codes, uint8_t* scales,
                            cudaStream_t stream) {
  const int64_t nb = rows * (D / 16);
  if (nb == 0) return CSA2_OK;
  const int threads = 256;
  const int64_t grid = (nb + threads - 1) / threads;
  begin_launch(stream);
  fp4_pack_kernel<<<static_cast<unsigned>(grid), threads, 0, stream>>>(
      static_cast<const uint4*>(x), nb, reinterpret_cast<uint2*>(codes), scales);
  note_launch(LK_PACK, 1, stream);
  return check_launch("fp4_pack");
}

csa2_status launch_fp4_unpack(const uint8_t* codes, const uint8_t* scales, int64_t rows, int D,
                              void* x, cudaStream_t stream) {
  const int64_t nb = rows * (D / 16);
  if (nb == 0) return CSA2_OK;
  const int threads = 256;
  const int64_t grid = (nb + threads - 1) / threads;
  begin_launch(stream);
  fp4_unpack_kernel<<<static_cast<unsigned>(grid), threads, 0, stream>>>(
      reinterpret_cast<const uint2*>(codes), scales, nb, static_cast<uint4*>(x));
  note_launch(LK_UNPACK, 1, stream);
  return check_launch("fp4_unpack");
}

}  // namespace csa2
