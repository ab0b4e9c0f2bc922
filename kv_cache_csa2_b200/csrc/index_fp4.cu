// Lightning-indexer scores with FP4 queries and keys and BF16 scores, on the
// 5th-generation tensor cores.  Source: "读完这篇，你就搞懂 DeepSeek v4 了",
// 闪电索引机制 (eq. 8: s_j = sum_h w_h * ReLU(q_h . k_j)) and FP4量化感知训练
// (the indexer's q and K are kept in FP4, its scores in BF16); the FP4 format
// is the main-KV one of "Recall之王" (E2M1 values, one E4M3 scale per 16
// channels).
//
// An E2M1 value times an E4M3 scale has at most 6 significant bits and lies
// in [2^-10, 2688], so every dequantised q and K value is exact in f16 (the
// hardware E2M1 -> f16 conversion, then one exact multiply by the scale) and
// every product q_i k_i is exact in f32: the contraction runs on the tensor
// cores (tcgen05 kind::f16 with f16 operands, f32 accumulation) on tiles
// dequantised in shared memory, and only the bytes read from memory shrink
// (72 instead of 256 per 128-wide key row).  Each score is rounded once to
// bf16.
//
// Per CTA (persistent, one per SM), units = (query, tile of 128 keys) in a
// contiguous range:
//   warp 0     the query's FP4 heads dequantised into one of two q slots
//              (K-major, 128-byte swizzle), with the head weights;
//   warp 1     TMEM allocation and MMA issue (M = 128 keys, N = heads padded
//              to HP, K = d), two accumulators;
//   warps 2-5  epilogue: s = sum_h w_h * act(acc_h), causal / pool mask,
//              round to bf16, store;
//   warps 6-9  key loaders: thread r copies row r of the tile (codes and
//              scales, cp.async, kLag tiles in flight into its own slots of a
//              raw ring), then dequantises that row into the bf16 stage once
//              the MMA has released it.
// Every wait is bounded; a wait that runs out records CSA2_ERR_TIMEOUT and
// the CTA winds down, letting its copies land and its MMAs finish before TMEM
// is freed.
#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "launchers.h"
#include "sm100.cuh"

namespace csa2 {
namespace {
using namespace sm100;

constexpr int kTileRows = 128;
constexpr int kKBlockBytes = kTileRows * 128;  // 128 rows x 64 bf16
constexpr int kLoadWarp = 6;
constexpr int kThreads = 10 * 32;
constexpr int kLag = 4;                        // key tiles of copies in flight per loader thread
// raw slots: a slot is refilled two tiles after its dequantisation began, so
// every loader has passed that tile's barrier (and finished reading it) by then
constexpr int kRaw = kLag + 2;

struct Params {
  const uint8_t* q_codes;    // [B, Q, H, d/2]
  const uint8_t* q_scales;   // [B, Q, H, d/16]
  const float* w;            // [B, Q, H]
  const uint8_t* k_codes;    // [B, N, d/2]
  const uint8_t* k_scales;   // [B, N, d/16]
  const int32_t* n_visible;  // [B, Q] or null
  const int32_t* pool;       // [B, Q, P] or null
  void* scores;              // bf16 or f32 [B, Q, N or P]
  int* err;
  int Q, H, P;
  int64_t N;
  int relu;
  int n_tiles;
  int64_t n_units;
};

template <int DK, int HP>
struct Cfg {
  static constexpr int KB = DK / 64;                       // K-blocks of 64 bf16
  static constexpr int STAGES = 4;
  static constexpr int TILE_A = KB * kKBlockBytes;         // bytes of one bf16 key tile
  static constexpr int QKB = HP * 128;                     // bytes of one q K-block
  static constexpr int QBYTES = KB * QKB;
  static constexpr int RAW_CODES = kTileRows * (DK / 2);   // a tile's codes, then its scales
  static constexpr int RAW_SLOT = RAW_CODES + kTileRows * (DK / 16);
  static constexpr int TMEM_COLS = (2 * HP <= 32) ? 32 : (2 * HP <= 64) ? 64 : 128;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_Q = OFF_A + STAGES * TILE_A;
  static constexpr int OFF_RAW = OFF_Q + 2 * QBYTES;
  static constexpr int OFF_W = OFF_RAW + kRaw * RAW_SLOT;

  static constexpr int OFF_BAR = OFF_W + 2 * HP * 4;
  static constexpr int NBAR = 2 * STAGES + 9;      // + the teardown barrier
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16 + 1024;
  static_assert(HP % 16 == 0 && HP <= 64, "MMA N");
  static_assert(QKB % 1024 == 0 && TILE_A % 1024 == 0 && RAW_SLOT % 16 == 0, "alignment");
  static_assert(OFF_BAR % 8 == 0, "barriers");
  static_assert(BYTES <= 232448, "shared memory");
};

// E4M3 scale code -> f32 (codes 0..126, the "fn" variant: bias 7, no inf).
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  const float mag = e == 0 ? static_cast<float>(m) * 0x1p-9f : __uint_as_float(((e + 120u) << 23) | (m << 20));
  return (c & 128u) ? -mag : mag;
}

// Two E2M1 codes (one byte: the lower channel in the low nibble) -> f16x2
// (lower channel in the low half), by the hardware conversion.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t r;
  const uint16_t b = static_cast<uint16_t>(byte);
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u16 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(r) : "h"(b));
  return r;
}

// One 16-channel block: 8 code bytes (channel 2i low nibble, 2i+1 high) and
// its E4M3 scale -> 8 words of two f16 each.  Exact: an E2M1 value times an
// E4M3 scale has at most 6 significant bits and lies in [2^-10, 2688].
__device__ __forceinline__ void fp4_block_to_f16(uint2 codes, uint32_t scale, uint32_t (&out)[8]) {
  const __half sh = __float2half_rn(e4m3_to_f32(scale));
  const __half2 s2 = __halves2half2(sh, sh);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t pr = e2m1x2_to_f16x2(((i < 4 ? codes.x : codes.y) >> (8 * (i & 3))) & 0xffu);
    const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&pr), s2);
    out[i] = *reinterpret_cast<const uint32_t*>(&v);
  }
}

template <int DK, int HP, bool POOL, bool OUT_BF16>
__global__ void __launch_bounds__(kThreads, 1) index_fp4_kernel(const Params p) {
  using C = Cfg<DK, HP>;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + C::OFF_A;
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sRaw = smem + C::OFF_RAW;
  float* sW = reinterpret_cast<float*>(smem + C::OFF_W);

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bar;                      // [S] a bf16 key tile is ready (128 loader arrivals)
  uint64_t* empty = bar + S;                 // [S] the MMAs of a tile are done
  uint64_t* tfull = bar + 2 * S;             // [2] accumulator ready
  uint64_t* tempty = tfull + 2;              // [2] accumulator read (4 epilogue warps)
  uint64_t* qfull = tfull + 4;               // [2] q slot ready
  uint64_t* qempty = tfull + 6;              // [2] q slot no longer read (MMA + 4 epilogue warps)
  uint64_t* mma_fin = tfull + 8;             // every MMA has completed (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t L = POOL ? p.P : p.N;
  pdl_release();
  const int64_t u0 = p.n_units * blockIdx.x / gridDim.x;
  const int64_t u1 = p.n_units * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 128);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
      mbar_init(&qfull[i], 1);
      mbar_init(&qempty[i], 1 + 4);
    }
    mbar_init(mma_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- q producer
    int64_t prev = -1;
    int qi = -1;
    for (int64_t u = u0; u < u1; ++u) {
      const int64_t qrow = u / p.n_tiles;              // b * Q + query
      if (qrow == prev) continue;
      prev = qrow;
      ++qi;
      const int slot = qi & 1;
      if (qi >= 2 && !mbar_wait(&qempty[slot], ((qi >> 1) - 1) & 1, abort_flag, p.err)) break;
      uint8_t* qs = sQ + slot * C::QBYTES;
      // items (head, 16-channel block): 8 bf16 words = two 16-byte chunks of a K-block row
      constexpr int NBLK = DK / 16;
      for (int i = lane; i < HP * NBLK; i += 32) {
        const int h = i / NBLK, blk = i % NBLK;
        uint32_t o[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (h < p.H) {
          const int64_t hr = qrow * p.H + h;
          const uint2 cw = __ldg(reinterpret_cast<const uint2*>(p.q_codes + hr * (DK / 2)) + blk);
          fp4_block_to_f16(cw, __ldg(p.q_scales + hr * NBLK + blk), o);
        }
        const int kb = blk / 4, c = (blk % 4) * 2;
        *reinterpret_cast<uint4*>(qs + kb * C::QKB + sw128_offset(h, c)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(qs + kb * C::QKB + sw128_offset(h, c + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
      for (int h = lane; h < HP; h += 32) sW[slot * HP + h] = h < p.H ? p.w[qrow * p.H + h] : 0.0f;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&qfull[slot]);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, HP, false, false);
      int64_t prev = -1;
      int qi = -1;
      int64_t it = 0;
      for (int64_t u = u0; u < u1; ++u, ++it) {
        const int64_t qrow = u / p.n_tiles;
        if (qrow != prev) {
          if (qi >= 0) mma_commit(&qempty[qi & 1]);
          ++qi;
          if (!mbar_wait(&qfull[qi & 1], (qi >> 1) & 1, abort_flag, p.err)) break;
          prev = qrow;
        }
        const int stage = static_cast<int>(it % S);
        const int acc = static_cast<int>(it & 1);
        if (!mbar_wait(&full[stage], (it / S) & 1, abort_flag, p.err)) break;
        if (it >= 2 && !mbar_wait(&tempty[acc], ((it >> 1) - 1) & 1, abort_flag, p.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * HP;
        const uint32_t a0 = smem_u32(sA + stage * C::TILE_A);
        const uint32_t b0 = smem_u32(sQ + (qi & 1) * C::QBYTES);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(d_tmem, desc_kmajor_sw128(a0 + kb * kKBlockBytes + kk * 32),
                     desc_kmajor_sw128(b0 + kb * C::QKB + kk * 32), idesc, (kb | kk) != 0);
        }
        mma_commit(&empty[stage]);
        mma_commit(&tfull[acc]);
      }
      // every product has completed before TMEM is freed (bounded: 0.1 s)
      mma_commit(mma_fin);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(mma_fin, 0) && globaltimer_ns() - t0 < 100000000ull) {
      }
    }
    __syncwarp();
  } else if (warp >= kLoadWarp) {
    // ---------------------------------------------------------------- key loaders
    const int r = static_cast<int>(threadIdx.x) - kLoadWarp * 32;   // tile row 0..127
    // raw slot: codes of row r at r * d/2, its scales at RAW_CODES + r * d/16
    bool ok = true;
    auto issue = [&](int64_t u, int slot) {
      const int64_t qrow = u / p.n_tiles;
      const int64_t b = qrow / p.Q;
      const int64_t e = (u % p.n_tiles) * kTileRows + r;
      int64_t id = e < L ? e : -1;
      if (POOL && id >= 0) {
        id = p.pool[qrow * p.P + e];
        if (id >= p.N || id < -1) id = -1;               // recorded by the epilogue
      }
      const uint32_t nb = id >= 0 ? 16u : 0u;
      const int64_t row = b * p.N + (id >= 0 ? id : 0);
      uint8_t* dst = sRaw + slot * C::RAW_SLOT;
#pragma unroll
      for (int c = 0; c < DK / 32; ++c)
        cp_async_16(dst + r * (DK / 2) + 16 * c, p.k_codes + row * (DK / 2) + 16 * c, nb);
      // scales: DK/16 bytes (8 for d = 128, 4 for d = 64)
      uint8_t* sdst = dst + C::RAW_CODES + r * (DK / 16);
      if (DK / 16 == 8)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_u32(sdst)),
                     "l"(p.k_scales + row * (DK / 16)), "r"(id >= 0 ? 8u : 0u) : "memory");
      else
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(sdst)),
                     "l"(p.k_scales + row * (DK / 16)), "r"(id >= 0 ? 4u : 0u) : "memory");
      cp_async_commit();
    };
    // the 128 loader threads dequantise a tile together, once each has seen its
    // own copies land (named barrier 3): thread r takes 16-channel blocks
    // r + 128 u, so eight threads read one row's codes contiguously
    auto load_bar = [] { asm volatile("bar.sync 3, 128;" ::: "memory"); };
    auto convert = [&](int64_t it_c) {
      const int stage = static_cast<int>(it_c % S);
      // (a wait that gives up leaves the CTA winding down; every loader still
      // takes every barrier, so none waits for another in vain)
      if (it_c >= S) mbar_wait(&empty[stage], ((it_c / S) - 1) & 1, abort_flag, p.err);
      load_bar();
      const uint8_t* src = sRaw + (it_c % kRaw) * C::RAW_SLOT;
      uint8_t* dst = sA + stage * C::TILE_A;
      constexpr int NBLK = DK / 16;
#pragma unroll
      for (int u = 0; u < NBLK; ++u) {
        const int i = r + 128 * u, row = i / NBLK, blk = i % NBLK;
        const uint2 cw = *reinterpret_cast<const uint2*>(src + row * (DK / 2) + 8 * blk);
        uint32_t o[8];
        fp4_block_to_f16(cw, src[C::RAW_CODES + row * NBLK + blk], o);
        const int kb = blk / 4, c = (blk % 4) * 2;
        *reinterpret_cast<uint4*>(dst + kb * kKBlockBytes + sw128_offset(row, c)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(dst + kb * kKBlockBytes + sw128_offset(row, c + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&full[stage]);
    };
    int64_t it = 0;
    for (int64_t u = u0; u < u1; ++u, ++it) {
      issue(u, static_cast<int>(it % kRaw));
      if (it >= kLag) {                      // tile it - kLag has landed: dequantise it
        cp_async_wait<kLag>();
        convert(it - kLag);
      }
    }
    cp_async_wait<0>();
    for (int64_t j = (it > kLag ? it - kLag : 0); j < it; ++j) convert(j);
    (void)ok;
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;                 // TMEM lanes this warp may access
    const int row = quad * 32 + lane;
    int64_t prev = -1;
    int qi = -1;
    int64_t it = 0;
    for (int64_t u = u0; u < u1; ++u, ++it) {
      const int64_t qrow = u / p.n_tiles;
      if (qrow != prev) {
        if (qi >= 0 && lane == 0) mbar_arrive(&qempty[qi & 1]);
        ++qi;
        if (!mbar_wait(&qfull[qi & 1], (qi >> 1) & 1, abort_flag, p.err)) break;
        prev = qrow;
      }
      const int acc = static_cast<int>(it & 1);
      const int64_t e = (u % p.n_tiles) * kTileRows + row;     // entry or pool slot
      const int64_t pid = POOL && e < L ? p.pool[qrow * p.P + e] : -1;
      if (!mbar_wait(&tfull[acc], (it >> 1) & 1, abort_flag, p.err)) break;
      tc_fence_after();
      const float* w = sW + (qi & 1) * HP;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * HP;
      float a = 0.0f;
#pragma unroll
      for (int h0 = 0; h0 < HP; h0 += 16) {
        uint32_t v[16];
        tmem_ld16(taddr + h0, v);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          float x = __uint_as_float(v[h]);
          if (p.relu) x = fmaxf(x, 0.0f);
          a = fmaf(w[h0 + h], x, a);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (e < L) {
        bool vis = true;
        if (POOL) {
          if (pid >= p.N || pid < -1) raise_dev_error(p.err, DEVERR_BOUNDS);
          vis = pid >= 0 && pid < p.N;
        } else if (p.n_visible) {
          vis = e < p.n_visible[qrow];
        }
        const float s = vis ? __bfloat162float(__float2bfloat16_rn(a)) : -INFINITY;
        if (OUT_BF16) {
          const __nv_bfloat16 hb = __float2bfloat16_rn(s);
          static_cast<uint16_t*>(p.scores)[qrow * L + e] = *reinterpret_cast<const uint16_t*>(&hb);
        } else {
          static_cast<float*>(p.scores)[qrow * L + e] = s;
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

template <int DK, int HP, bool POOL, bool OUT_BF16>
csa2_status run_fp4(const Fp4IndexArgs& a, cudaStream_t stream) {
  using C = Cfg<DK, HP>;
  Params p;
  p.q_codes = a.q_codes;
  p.q_scales = a.q_scales;
  p.w = a.w;
  p.k_codes = a.k_codes;
  p.k_scales = a.k_scales;
  p.n_visible = a.n_visible;
  p.pool = a.pool;
  p.scores = a.scores;
  p.err = device_error_word();
  p.Q = a.Q;
  p.H = a.H;
  p.P = a.P;
  p.N = a.N;
  p.relu = a.act == CSA2_ACT_RELU ? 1 : 0;
  const int64_t L = POOL ? a.P : a.N;
  p.n_tiles = static_cast<int>((L + kTileRows - 1) / kTileRows);
  p.n_units = static_cast<int64_t>(a.B) * a.Q * p.n_tiles;
  static PerDevice<cudaError_t> opt_in;
  const cudaError_t attr_err = opt_in.get([] {
    const cudaError_t e = cudaFuncSetAttribute(index_fp4_kernel<DK, HP, POOL, OUT_BF16>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, C::BYTES);
    if (e != cudaSuccess) cudaGetLastError();
    return e;
  });
  if (attr_err != cudaSuccess) return fail(CSA2_ERR_CUDA, "index_fp4: smem opt-in failed");
  const int64_t grid = std::min<int64_t>(sm_count(), p.n_units);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute at[1] = {pdl_attribute()};
  cfg.attrs = at;
  cfg.numAttrs = 1;
  begin_launch(stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, index_fp4_kernel<DK, HP, POOL, OUT_BF16>, p);
  note_launch(POOL ? LK_INDEX_POOL : LK_INDEX, 1, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(CSA2_ERR_CUDA, "index_fp4: launch failed: %s", cudaGetErrorString(e));
  }
  return check_launch("index_fp4");
}

template <int DK, bool POOL, bool OUT_BF16>
csa2_status run_fp4_heads(const Fp4IndexArgs& a, cudaStream_t stream) {
  return a.H <= 16 ? run_fp4<DK, 16, POOL, OUT_BF16>(a, stream) : run_fp4<DK, 64, POOL, OUT_BF16>(a, stream);
}

template <bool POOL, bool OUT_BF16>
csa2_status run_fp4_dims(const Fp4IndexArgs& a, cudaStream_t stream) {
  return a.d == 64 ? run_fp4_heads<64, POOL, OUT_BF16>(a, stream) : run_fp4_heads<128, POOL, OUT_BF16>(a, stream);
}

}  // namespace

csa2_status launch_index_scores_fp4(const Fp4IndexArgs& a, bool out_bf16, cudaStream_t stream) {
  const int64_t L = a.pool ? a.P : a.N;
  if (L == 0 || a.B == 0 || a.Q == 0) return CSA2_OK;
  if ((a.d != 64 && a.d != 128) || a.H > 64)
    return fail(CSA2_ERR_UNSUPPORTED, "index_scores_fp4: d=%d, H=%d (supported: d 64 or 128, H <= 64)", a.d, a.H);
  if (a.pool) return out_bf16 ? run_fp4_dims<true, true>(a, stream) : run_fp4_dims<true, false>(a, stream);
  return out_bf16 ? run_fp4_dims<false, true>(a, stream) : run_fp4_dims<false, false>(a, stream);
}

}  // namespace csa2
