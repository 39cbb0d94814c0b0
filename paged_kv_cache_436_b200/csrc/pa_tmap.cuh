// Host side: TMA tensor maps over the paged cache. cuTensorMapEncodeTiled is reached
// through the runtime's driver entry point, so the library does not link libcuda.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "pa.h"

namespace pa {

typedef CUresult (*TmapEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The encoder, or null when the driver does not provide it.
inline TmapEncodeFn tmap_encoder() {
  static std::once_flag once;
  static TmapEncodeFn fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<TmapEncodeFn>(f);
  });
  return fn;
}

// A 16-bit cache viewed as [blocks * kv heads * block_size rows][head_dim]; box = 64 dims x
// one cache block of one kv head, 128B swizzle (16-byte chunk c of a 128-byte row r lands
// at chunk c ^ (r % 8)). Base 16-byte aligned, rows head_dim * 2 bytes.
inline bool cache_tmap(TmapEncodeFn enc, CUtensorMap* m, const void* base, int qd, long long rows, int BS, int D) {
  const cuuint64_t dims[2] = {cuuint64_t(D), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(D) * 2};
  const cuuint32_t box[2] = {64, cuuint32_t(BS)};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, qd == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
             const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace pa
