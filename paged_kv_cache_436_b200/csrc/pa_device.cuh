// Device helpers for libpa: element decoders, the sticky device error word,
// mbarrier + 1-D bulk-copy (TMA engine, no tensor map, no multicast) wrappers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

constexpr int kPartitionTokens = 512;      // split-K partition length of the v2-style decode
constexpr unsigned kFull = 0xffffffffu;
constexpr int kSelftestKernelId = 0x7E57;   // kernel id the wait self-test records

// ---------------------------------------------------------------------------
// sticky device error word: [code, info0, info1, info2]; the first error wins
// ---------------------------------------------------------------------------
// defined once: the library's device code is a single translation unit
__device__ int g_pa_error[4];

__device__ __forceinline__ void record_error(int code, int a, int b, int c) {
  if (atomicCAS(&g_pa_error[0], 0, code) == 0) {
    g_pa_error[1] = a;
    g_pa_error[2] = b;
    g_pa_error[3] = c;
  }
}

// ---------------------------------------------------------------------------
// element formats of the cache
// ---------------------------------------------------------------------------
template <int KV>
struct Kv;

template <>
struct Kv<PA_F16> {
  static constexpr int kBytes = 2;
  static constexpr int kPer16B = 8;
  __device__ __forceinline__ static void decode(const uint4& raw, float* f) {
    const __half2* h = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = __half22float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
};

template <>
struct Kv<PA_BF16> {
  static constexpr int kBytes = 2;
  static constexpr int kPer16B = 8;
  // bfloat16 is the upper half of a binary32: widening is a shift / mask
  __device__ __forceinline__ static void decode(const uint4& raw, float* f) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

template <>
struct Kv<PA_E4M3> {
  static constexpr int kBytes = 1;
  static constexpr int kPer16B = 16;
  // hardware e4m3x2 -> f16x2 conversion, then f16 -> f32 (both exact)
  __device__ __forceinline__ static void decode(const uint4& raw, float* f) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>(w[i] & 0xffffu), __NV_E4M3);
      const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>(w[i] >> 16), __NV_E4M3);
      const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
      const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
      f[4 * i + 0] = a.x;
      f[4 * i + 1] = a.y;
      f[4 * i + 2] = b.x;
      f[4 * i + 3] = b.y;
    }
  }
};

// query / output element types
template <int QD>
struct Q;
template <>
struct Q<PA_F16> {
  using T = __half;
  __device__ __forceinline__ static float to_float(T x) { return __half2float(x); }
  __device__ __forceinline__ static T from_float(float x) { return __float2half_rn(x); }
};
template <>
struct Q<PA_BF16> {
  using T = __nv_bfloat16;
  __device__ __forceinline__ static float to_float(T x) { return __bfloat162float(x); }
  __device__ __forceinline__ static T from_float(float x) { return __float2bfloat16_rn(x); }
};

// ---------------------------------------------------------------------------
// mbarrier + bulk copy
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait: gives up after `limit_ns` of wall time and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t limit_ns = 2000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
}

// One-dimensional bulk copy global -> shared through the TMA engine; completion is
// signalled on `bar` as transaction bytes. dst/src 16-byte aligned, bytes % 16 == 0.
// The L2 policy marks the streamed KV bytes evict-first: each is read once per step.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 2-D tiled TMA load (box given by the tensor map) signalling `bar` with its bytes.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

// Programmatic dependent launch (no-ops when the kernel was launched normally).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dependency_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace pa
