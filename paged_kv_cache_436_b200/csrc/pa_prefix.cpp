// Prefix cache: a host index from the content of a prompt's full KV blocks to the
// physical blocks that already hold them.
//
// Page 3 «内存优化：KV Cache管理、PagedAttention原理与内存池配置», section "案例与场景":
// the KV blocks of a common prefix get a global hash index; a request whose prefix
// matches reuses those physical blocks and allocates only for its new tokens. Section
// "误区与复盘" (误区3): it works only for exactly equal prefixes, and the table costs
// host memory.
//
// Key of full block k of a prompt: FNV-1a (64-bit) over the key of block k-1 and the
// block's BS token ids, so equal keys stand for equal whole prefixes. Every entry keeps
// its parent key and its tokens, and a lookup accepts an entry only when both match:
// a hit is an exact prefix match even if two prefixes ever hashed alike (such a
// collision can only cost a missed reuse). The index holds one reference on each block
// it lists.
#include <cstring>
#include <deque>
#include <new>
#include <unordered_map>
#include <vector>

#include "pa.h"

namespace {

constexpr uint64_t kFnvOffset = 14695981039346656037ull;
constexpr uint64_t kFnvPrime = 1099511628211ull;

inline uint64_t fnv1a(uint64_t h, const void* data, size_t n) {
  const unsigned char* p = static_cast<const unsigned char*>(data);
  for (size_t i = 0; i < n; ++i) {
    h ^= p[i];
    h *= kFnvPrime;
  }
  return h;
}

inline uint64_t block_key(uint64_t parent, const int32_t* tokens, int32_t bs) {
  uint64_t h = fnv1a(kFnvOffset, &parent, sizeof(parent));
  return fnv1a(h, tokens, size_t(bs) * sizeof(int32_t));
}

struct Entry {
  uint64_t parent;
  int32_t block;
  std::vector<int32_t> tokens;
};

}  // namespace

struct pa_prefix_cache {
  int32_t bs;
  std::unordered_map<uint64_t, Entry> map;
  std::deque<uint64_t> order;     // keys in insertion order (eviction walks it)
};

extern "C" {

pa_status pa_prefix_cache_create(int32_t block_size, pa_prefix_cache** out) {
  if (!out || block_size <= 0) return PA_ERR_ARG;
  *out = new (std::nothrow) pa_prefix_cache;
  if (!*out) return PA_ERR_OOM;
  (*out)->bs = block_size;
  return PA_OK;
}

void pa_prefix_cache_destroy(pa_prefix_cache* c) { delete c; }

int32_t pa_prefix_cache_size(const pa_prefix_cache* c) { return c ? int32_t(c->map.size()) : -1; }

pa_status pa_prefix_cache_match(pa_prefix_cache* c, pa_pool* pool, const int32_t* tokens, int32_t n_tokens,
                                int32_t* block_table_row, int32_t max_blocks, int32_t* n_matched) {
  if (n_matched) *n_matched = 0;
  if (!c || !pool || (!tokens && n_tokens > 0) || !block_table_row || !n_matched || n_tokens < 0)
    return PA_ERR_ARG;
  const int32_t bs = c->bs, full = n_tokens / bs;
  uint64_t parent = 0;
  int32_t n = 0;
  for (int32_t k = 0; k < full && k < max_blocks; ++k) {
    const int32_t* tk = tokens + size_t(k) * bs;
    const uint64_t key = block_key(parent, tk, bs);
    auto it = c->map.find(key);
    if (it == c->map.end() || it->second.parent != parent ||
        std::memcmp(it->second.tokens.data(), tk, size_t(bs) * sizeof(int32_t)) != 0)
      break;
    const pa_status st = pa_pool_incref(pool, it->second.block);
    if (st != PA_OK) {   // the references taken so far stand and are reported
      *n_matched = n;
      return st;
    }
    block_table_row[k] = it->second.block;
    parent = key;
    ++n;
  }
  *n_matched = n;
  return PA_OK;
}

pa_status pa_prefix_cache_insert(pa_prefix_cache* c, pa_pool* pool, const int32_t* tokens, int32_t n_tokens,
                                 const int32_t* block_table_row, int32_t* n_inserted) {
  if (n_inserted) *n_inserted = 0;
  if (!c || !pool || (!tokens && n_tokens > 0) || !block_table_row || n_tokens < 0) return PA_ERR_ARG;
  const int32_t bs = c->bs, full = n_tokens / bs;
  uint64_t parent = 0;
  int32_t added = 0;
  for (int32_t k = 0; k < full; ++k) {
    const int32_t* tk = tokens + size_t(k) * bs;
    const uint64_t key = block_key(parent, tk, bs);
    if (c->map.find(key) == c->map.end()) {
      const pa_status st = pa_pool_incref(pool, block_table_row[k]);
      if (st != PA_OK) {   // the entries added so far stand and are reported
        if (n_inserted) *n_inserted = added;
        return st;
      }
      Entry e;
      e.parent = parent;
      e.block = block_table_row[k];
      e.tokens.assign(tk, tk + bs);
      c->map.emplace(key, std::move(e));
      c->order.push_back(key);
      ++added;
    }
    parent = key;
  }
  if (n_inserted) *n_inserted = added;
  return PA_OK;
}

pa_status pa_prefix_cache_evict(pa_prefix_cache* c, pa_pool* pool, int32_t max_blocks, int32_t* n_evicted) {
  if (n_evicted) *n_evicted = 0;
  if (!c || !pool || max_blocks < 0) return PA_ERR_ARG;
  int32_t n = 0;
  pa_status st = PA_OK;
  std::deque<uint64_t> keep;
  for (const uint64_t key : c->order) {
    auto it = c->map.find(key);
    if (st == PA_OK && n < max_blocks && pa_pool_refcount(pool, it->second.block) == 1) {
      st = pa_pool_decref(pool, it->second.block);
      if (st == PA_OK) {
        c->map.erase(it);
        ++n;
        continue;
      }
    }
    keep.push_back(key);   // also every entry from a failed release on: order and map stay in step
  }
  c->order.swap(keep);
  if (n_evicted) *n_evicted = n;
  return st;
}

pa_status pa_prefix_cache_clear(pa_prefix_cache* c, pa_pool* pool, int32_t* n_released) {
  if (n_released) *n_released = 0;
  if (!c || !pool) return PA_ERR_ARG;
  int32_t n = 0;
  while (!c->order.empty()) {   // entries leave the index as their reference is returned
    const uint64_t key = c->order.front();
    auto it = c->map.find(key);
    const pa_status st = pa_pool_decref(pool, it->second.block);
    if (st != PA_OK) {
      if (n_released) *n_released = n;
      return st;
    }
    c->map.erase(it);
    c->order.pop_front();
    ++n;
  }
  if (n_released) *n_released = n;
  return PA_OK;
}

}  // extern "C"
