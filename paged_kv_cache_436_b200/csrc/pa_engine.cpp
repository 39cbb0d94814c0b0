// Native decode-step driver: one call per step runs the host bookkeeping of every
// sequence and enqueues the step's device work, so no interpreter sits between the
// pool and the kernels.
//
// Step order (page 3 «内存优化：KV Cache管理、PagedAttention原理与内存池配置», section
// "PagedAttention原理": blocks taken on demand and shared by reference count; page 2,
// untitled, first section "1. 为什么vLLM能实现24倍推理加速", section "2.2 关键数据结构剖析":
// block tables and context lengths travel to the kernels as attention metadata):
//   1. pa_batch_append on the host: slots, copy-on-write pairs, table updates;
//   2. one cudaMemcpyAsync of the packed metadata from pinned host memory;
//   3. pa_block_table_update, pa_copy_blocks, pa_reshape_and_cache, pa_decode.
#include <cuda_runtime.h>

#include <cstring>
#include <new>

#include "pa.h"

namespace {

constexpr size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

struct MetaLayout {
  size_t slots, cows, lens, upd, total;
  explicit MetaLayout(int32_t S) {
    slots = 0;
    cows = align16(slots + size_t(S) * 8);
    lens = align16(cows + size_t(S) * 16);
    upd = align16(lens + size_t(S) * 4);
    total = align16(upd + size_t(S) * 12);
  }
};

}  // namespace

struct pa_engine {
  pa_engine_config cfg;
  MetaLayout meta{0};
  cudaEvent_t meta_done[2] = {nullptr, nullptr};
  bool meta_used[2] = {false, false};
  int flip = 0;
  int32_t last_cow = 0, last_updates = 0, last_launches = 0;
};

extern "C" {

size_t pa_engine_meta_bytes(int32_t num_seqs) { return num_seqs < 0 ? 0 : MetaLayout(num_seqs).total; }

pa_status pa_engine_create(const pa_engine_config* c, pa_engine** out) {
  if (!out || !c) return PA_ERR_ARG;
  *out = nullptr;
  if (!c->pool || !c->block_tables_host || !c->context_lens_host || !c->block_tables_dev ||
      !c->meta_host[0] || !c->meta_host[1] || !c->meta_dev || !c->workspace)
    return PA_ERR_ARG;
  if (c->num_seqs <= 0 || c->num_q_heads <= 0 || c->max_blocks_per_seq <= 0 || c->max_context_len < 0)
    return PA_ERR_ARG;
  if (c->meta_bytes < pa_engine_meta_bytes(c->num_seqs)) return PA_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(c->meta_dev) & 15) != 0) return PA_ERR_ARG;
  if (c->workspace_bytes < pa_decode_workspace_size(c->num_seqs, c->num_q_heads, c->cache.head_dim,
                                                    c->max_context_len))
    return PA_ERR_ARG;
  pa_engine* e = new (std::nothrow) pa_engine;
  if (!e) return PA_ERR_OOM;
  e->cfg = *c;
  e->meta = MetaLayout(c->num_seqs);
  for (int i = 0; i < 2; ++i) {
    if (cudaEventCreateWithFlags(&e->meta_done[i], cudaEventDisableTiming) != cudaSuccess) {
      pa_engine_destroy(e);
      return PA_ERR_CUDA;
    }
  }
  *out = e;
  return PA_OK;
}

void pa_engine_destroy(pa_engine* e) {
  if (!e) return;
  for (int i = 0; i < 2; ++i)
    if (e->meta_done[i]) cudaEventDestroy(e->meta_done[i]);
  delete e;
}

pa_status pa_engine_step(pa_engine* e, const void* q, const void* k_new, const void* v_new, void* out,
                         void* stream, void* ev_partition_begin, void* ev_partition_end) {
  if (!e || !q || !k_new || !v_new || !out) return PA_ERR_ARG;
  const pa_engine_config& c = e->cfg;
  const int32_t S = c.num_seqs;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // 1. host bookkeeping into the pinned buffer the copy of two steps ago has released
  const int i = e->flip;
  e->flip ^= 1;
  if (e->meta_used[i] && cudaEventSynchronize(e->meta_done[i]) != cudaSuccess) return PA_ERR_CUDA;
  uint8_t* h = static_cast<uint8_t*>(c.meta_host[i]);
  auto* slots = reinterpret_cast<int64_t*>(h + e->meta.slots);
  auto* cows = reinterpret_cast<int64_t*>(h + e->meta.cows);
  auto* lens = reinterpret_cast<int32_t*>(h + e->meta.lens);
  auto* upd = reinterpret_cast<int32_t*>(h + e->meta.upd);
  int32_t ncow = 0, nupd = 0, done = 0;
  pa_status st = pa_batch_append(c.pool, c.block_tables_host, S, c.max_blocks_per_seq, c.context_lens_host,
                                 c.cache.block_size, slots, cows, &ncow, upd, &nupd, &done);
  // the sequences appended so far hold one more token, even when a later one failed
  for (int32_t k = 0; k < done; ++k) ++c.context_lens_host[k];
  if (st != PA_OK) return st;
  std::memcpy(lens, c.context_lens_host, size_t(S) * 4);

  // 2. one upload of the step's metadata
  uint8_t* d = static_cast<uint8_t*>(c.meta_dev);
  if (cudaMemcpyAsync(d, h, e->meta.total, cudaMemcpyHostToDevice, s) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaEventRecord(e->meta_done[i], s) != cudaSuccess) return PA_ERR_CUDA;
  e->meta_used[i] = true;

  // 3. device work
  int launches = 0;
  if (nupd) {
    st = pa_block_table_update(reinterpret_cast<const int32_t*>(d + e->meta.upd), nupd, c.block_tables_dev, S,
                               c.max_blocks_per_seq, stream);
    if (st != PA_OK) return st;
    ++launches;
  }
  if (ncow) {
    st = pa_copy_blocks(reinterpret_cast<const int64_t*>(d + e->meta.cows), ncow, &c.cache, stream);
    if (st != PA_OK) return st;
    ++launches;
  }
  const int64_t row = int64_t(c.cache.num_kv_heads) * c.cache.head_dim;
  st = pa_reshape_and_cache(k_new, v_new, c.q_dtype, S, row, row, reinterpret_cast<const int64_t*>(d + e->meta.slots),
                            &c.cache, stream);
  if (st != PA_OK) return st;
  ++launches;
  const int32_t* dlens = reinterpret_cast<const int32_t*>(d + e->meta.lens);
  for (int stage = 0; stage < 3; ++stage) {
    if (stage == 1 && ev_partition_begin &&
        cudaEventRecord(static_cast<cudaEvent_t>(ev_partition_begin), s) != cudaSuccess)
      return PA_ERR_CUDA;
    st = pa_decode_stage(stage, q, c.q_dtype, S, c.num_q_heads, &c.cache, c.block_tables_dev, c.max_blocks_per_seq,
                         dlens, c.max_context_len, c.scale, out, c.workspace, c.workspace_bytes, stream);
    if (st != PA_OK) return st;
    if (stage == 1 && ev_partition_end &&
        cudaEventRecord(static_cast<cudaEvent_t>(ev_partition_end), s) != cudaSuccess)
      return PA_ERR_CUDA;
  }
  launches += c.max_context_len > 512 ? 3 : 2;
  e->last_cow = ncow;
  e->last_updates = nupd;
  e->last_launches = launches;
  return PA_OK;
}

pa_status pa_engine_last_step(const pa_engine* e, int32_t* num_cow, int32_t* num_updates, int32_t* launches) {
  if (!e) return PA_ERR_ARG;
  if (num_cow) *num_cow = e->last_cow;
  if (num_updates) *num_updates = e->last_updates;
  if (launches) *launches = e->last_launches;
  return PA_OK;
}

}  // extern "C"
