// KV-cache write (reshape_and_cache), block copy (copy-on-write) and the device
// mirror of block-table updates, for sm_100a.
//
// Slot addressing: page 1 «突破GPU内存瓶颈：vLLM与PagedAttention技术深度解析», section
// "2. PagedAttention的革命性设计" -- a block table maps a sequence's logical blocks to
// physical ones; slot = block * BS + offset. Block sharing and the copy a writer
// needs before it appends into a shared block: page 3
// «内存优化：KV Cache管理、PagedAttention原理与内存池配置», section "PagedAttention原理"
// (reference-counted sharing); page 1, section "5. 高级应用场景" (parallel sampling,
// beam search). FP8 cache: page 2, section "4.2 混合精度策略" ("KV缓存 FP8").
//
// All three kernels are pure data movement: 16-byte vector loads and stores,
// coalesced along head_dim; the write path of an E4M3 cache converts in registers.
#include <cuda_runtime.h>

#include <cmath>

#include "pa.h"
#include "pa_device.cuh"

namespace pa {

// Eight 16-bit values (one 16-byte vector) stored into an E4M3 cache: x / scale in
// binary32 (round to nearest), then E4M3 round-to-nearest-even, saturating to +-448.
template <int IN>
__device__ __forceinline__ uint2 encode_e4m3x8(const uint4& raw, float scale) {
  using IT = typename Q<IN>::T;
  const IT* e = reinterpret_cast<const IT*>(&raw);
  uint32_t packed[2];
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    uint32_t word = 0;
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const float a = __fdiv_rn(Q<IN>::to_float(e[4 * w + 2 * pr]), scale);
      const float b = __fdiv_rn(Q<IN>::to_float(e[4 * w + 2 * pr + 1]), scale);
      const __nv_fp8x2_storage_t two = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
      word |= uint32_t(two) << (16 * pr);
    }
    packed[w] = word;
  }
  return make_uint2(packed[0], packed[1]);
}

// grid (tokens, 2, chunks): y = 0 writes K, y = 1 writes V; each thread moves one
// vector of 8 input elements (16 bytes) of the token's Hkv * D row.
template <int KV, int IN>
__global__ void __launch_bounds__(128) reshape_kernel(const uint8_t* __restrict__ k,
                                                      const uint8_t* __restrict__ v,
                                                      int64_t k_stride_bytes, int64_t v_stride_bytes,
                                                      const int64_t* __restrict__ slots,
                                                      uint8_t* __restrict__ kc, uint8_t* __restrict__ vc,
                                                      int Hkv, int BS, int D, int num_blocks,
                                                      float k_scale, float v_scale) {
  const int t = blockIdx.x, which = blockIdx.y;
  const int i = blockIdx.z * blockDim.x + threadIdx.x;
  const int nvec = Hkv * D / 8;
  if (i >= nvec) return;
  const int64_t slot = slots[t];
  if (slot < 0) return;
  const int64_t limit = int64_t(num_blocks) * BS;
  if (slot >= limit) {
    if (i == 0 && which == 0)
      record_error(PA_DEV_BAD_SLOT, t, int(slot > 0x7fffffff ? 0x7fffffff : slot),
                   int(limit > 0x7fffffff ? 0x7fffffff : limit));
    return;
  }
  const int64_t blk = slot / BS;
  const int off = int(slot - blk * BS);
  constexpr int EB = Kv<KV>::kBytes;
  const uint8_t* src = (which ? v : k) + int64_t(t) * (which ? v_stride_bytes : k_stride_bytes);
  uint8_t* dst_base = which ? vc : kc;
  const int e0 = i * 8;
  const int h = e0 / D, d = e0 - h * D;
  const uint4 raw = *reinterpret_cast<const uint4*>(src + size_t(e0) * 2);
  uint8_t* dst = dst_base + (((size_t(blk) * Hkv + h) * BS + off) * D + d) * EB;
  if constexpr (KV != PA_E4M3) {
    *reinterpret_cast<uint4*>(dst) = raw;
  } else {
    *reinterpret_cast<uint2*>(dst) = encode_e4m3x8<IN>(raw, which ? v_scale : k_scale);
  }
}

// grid (pairs, 2): y = 0 copies K, y = 1 copies V; 16-byte vectors over the block.
// Pairs run concurrently, so a pair is copied only if no other pair of the batch writes
// its source or its destination, or reads its destination (the relation is symmetric:
// both pairs of a clash are skipped and one of them is recorded). Every pair that is
// copied then reads the cache as it was before the call.
__global__ void __launch_bounds__(256) copy_blocks_kernel(const int64_t* __restrict__ pairs, int num_pairs,
                                                          uint8_t* kc, uint8_t* vc,
                                                          int64_t block_bytes, int num_blocks) {
  const int i = blockIdx.x;
  const int64_t src = pairs[2 * i], dst = pairs[2 * i + 1];
  auto clamp32 = [](int64_t x) { return int(x < INT32_MIN ? INT32_MIN : (x > INT32_MAX ? INT32_MAX : x)); };
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) record_error(PA_DEV_BAD_COPY_PAIR, i, clamp32(src), clamp32(dst));
    return;
  }
  int clash = 0;
  for (int j = threadIdx.x; j < num_pairs; j += blockDim.x) {
    if (j == i) continue;
    const int64_t sj = pairs[2 * j], dj = pairs[2 * j + 1];
    clash |= (dj == src) | (dj == dst) | (sj == dst);
  }
  if (__syncthreads_or(clash)) {
    if (threadIdx.x == 0 && blockIdx.y == 0) record_error(PA_DEV_BAD_COPY_PAIR, i, clamp32(src), clamp32(dst));
    return;
  }
  uint8_t* base = blockIdx.y ? vc : kc;
  const uint4* s = reinterpret_cast<const uint4*>(base + src * block_bytes);
  uint4* d = reinterpret_cast<uint4*>(base + dst * block_bytes);
  const int64_t n = block_bytes / 16;
  for (int64_t e = threadIdx.x; e < n; e += blockDim.x) d[e] = s[e];
}

__global__ void table_update_kernel(const int32_t* __restrict__ upd, int n, int32_t* bt, int num_seqs,
                                    int max_blocks) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int s = upd[3 * i], col = upd[3 * i + 1], b = upd[3 * i + 2];
  if (s < 0 || s >= num_seqs || col < 0 || col >= max_blocks) {
    record_error(PA_DEV_BAD_TABLE_UPDATE, i, s, col);
    return;
  }
  bt[size_t(s) * max_blocks + col] = b;
}

pa_status validate_cache(const pa_cache_desc* c);

inline bool aligned16_(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace pa

namespace pa {

// One thread waits on an mbarrier that nothing arrives at, through the bounded wait every
// kernel of the library uses; when the limit runs out it records the timeout in the device
// error word and returns, leaving the context usable.
__global__ void __launch_bounds__(32) selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  const uint64_t t0 = global_timer_ns();
  if (!mbar_wait_bounded(&bar, 0, limit_ns))
    record_error(PA_DEV_WAIT_TIMEOUT, kSelftestKernelId, int((global_timer_ns() - t0) / 1000), 0);
}

}  // namespace pa

extern "C" {

pa_status pa_reshape_and_cache(const void* k, const void* v, int32_t in_dtype, int32_t num_tokens,
                               int64_t k_token_stride, int64_t v_token_stride,
                               const int64_t* slot_mapping, const pa_cache_desc* c, void* stream) {
  pa_status st = pa::validate_cache(c);
  if (st != PA_OK) return st;
  if (num_tokens < 0) return PA_ERR_ARG;
  if (in_dtype != PA_F16 && in_dtype != PA_BF16) return PA_ERR_ARG;
  if (c->kv_dtype != PA_E4M3 && in_dtype != c->kv_dtype) return PA_ERR_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !slot_mapping) return PA_ERR_ARG;
  const int64_t row = int64_t(c->num_kv_heads) * c->head_dim;
  if (k_token_stride < row || v_token_stride < row) return PA_ERR_ARG;
  if (!pa::aligned16_(k) || !pa::aligned16_(v) || (k_token_stride * 2) % 16 || (v_token_stride * 2) % 16)
    return PA_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto* kc = static_cast<uint8_t*>(c->k_cache);
  auto* vc = static_cast<uint8_t*>(c->v_cache);
  const auto* kb = static_cast<const uint8_t*>(k);
  const auto* vb = static_cast<const uint8_t*>(v);
  const int64_t ks = k_token_stride * 2, vs = v_token_stride * 2;
  const int nvec = c->num_kv_heads * c->head_dim / 8;
  const dim3 grid(num_tokens, 2, (nvec + 127) / 128), block(128);
  if (c->kv_dtype == PA_F16)
    pa::reshape_kernel<PA_F16, PA_F16><<<grid, block, 0, s>>>(kb, vb, ks, vs, slot_mapping, kc, vc, c->num_kv_heads,
                                                              c->block_size, c->head_dim, c->num_blocks, 1.f, 1.f);
  else if (c->kv_dtype == PA_BF16)
    pa::reshape_kernel<PA_BF16, PA_BF16><<<grid, block, 0, s>>>(kb, vb, ks, vs, slot_mapping, kc, vc, c->num_kv_heads,
                                                                c->block_size, c->head_dim, c->num_blocks, 1.f, 1.f);
  else if (in_dtype == PA_F16)
    pa::reshape_kernel<PA_E4M3, PA_F16><<<grid, block, 0, s>>>(kb, vb, ks, vs, slot_mapping, kc, vc, c->num_kv_heads,
                                                               c->block_size, c->head_dim, c->num_blocks,
                                                               c->k_scale, c->v_scale);
  else
    pa::reshape_kernel<PA_E4M3, PA_BF16><<<grid, block, 0, s>>>(kb, vb, ks, vs, slot_mapping, kc, vc, c->num_kv_heads,
                                                                c->block_size, c->head_dim, c->num_blocks,
                                                                c->k_scale, c->v_scale);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_copy_blocks(const int64_t* pairs, int32_t num_pairs, const pa_cache_desc* c, void* stream) {
  pa_status st = pa::validate_cache(c);
  if (st != PA_OK) return st;
  if (num_pairs < 0) return PA_ERR_ARG;
  if (num_pairs == 0) return PA_OK;
  if (!pairs) return PA_ERR_ARG;
  const int eb = c->kv_dtype == PA_E4M3 ? 1 : 2;
  const int64_t block_bytes = int64_t(c->num_kv_heads) * c->block_size * c->head_dim * eb;
  pa::copy_blocks_kernel<<<dim3(num_pairs, 2), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      pairs, num_pairs, static_cast<uint8_t*>(c->k_cache), static_cast<uint8_t*>(c->v_cache), block_bytes, c->num_blocks);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_block_table_update(const int32_t* updates, int32_t num_updates, int32_t* block_tables,
                                int32_t num_seqs, int32_t max_blocks_per_seq, void* stream) {
  if (num_updates < 0 || num_seqs < 0 || max_blocks_per_seq <= 0) return PA_ERR_ARG;
  if (num_updates == 0) return PA_OK;
  if (!updates || !block_tables) return PA_ERR_ARG;
  pa::table_update_kernel<<<(num_updates + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      updates, num_updates, block_tables, num_seqs, max_blocks_per_seq);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_selftest_wait_timeout(uint32_t limit_us, void* stream) {
  if (limit_us == 0 || limit_us > 2000000) return PA_ERR_ARG;
  pa::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(uint64_t(limit_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // extern "C"
