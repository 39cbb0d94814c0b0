// Host block pool: a LIFO free list threaded through an array, plus reference
// counts. Page 3 «内存优化：KV Cache管理、PagedAttention原理与内存池配置», section
// "PagedAttention原理": free blocks kept as a linked list so that alloc and free
// are O(1); blocks shared between sequences through reference counts; blocks taken
// only as a sequence grows. Every operation here is O(1) per block and touches no
// device memory.
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "pa.h"

struct pa_pool {
  int32_t num_blocks;
  int32_t head;             // next block to hand out, -1 when empty
  int32_t num_free;
  std::vector<int32_t> next;     // free-list link of each free block
  std::vector<int32_t> refcnt;   // 0 = free
};

namespace {

inline bool in_range(const pa_pool* p, int32_t b) { return b >= 0 && b < p->num_blocks; }

inline int32_t pop(pa_pool* p) {
  int32_t b = p->head;
  p->head = p->next[b];
  p->next[b] = -1;
  p->refcnt[b] = 1;
  --p->num_free;
  return b;
}

inline void push(pa_pool* p, int32_t b) {
  p->next[b] = p->head;
  p->head = b;
  ++p->num_free;
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace

extern "C" {

pa_status pa_pool_create(int32_t num_blocks, const int32_t* initial_order, pa_pool** out) {
  if (!out || num_blocks <= 0) return PA_ERR_ARG;
  *out = nullptr;
  pa_pool* p = new (std::nothrow) pa_pool;
  if (!p) return PA_ERR_OOM;
  p->num_blocks = num_blocks;
  p->next.assign(num_blocks, -1);
  p->refcnt.assign(num_blocks, 0);
  std::vector<char> seen(num_blocks, 0);
  for (int32_t i = 0; i < num_blocks; ++i) {
    int32_t b = initial_order ? initial_order[i] : i;
    if (b < 0 || b >= num_blocks || seen[b]) {
      delete p;
      return PA_ERR_ARG;
    }
    seen[b] = 1;
  }
  // thread the list so that pops return initial_order[0], [1], ...
  p->head = -1;
  p->num_free = 0;
  for (int32_t i = num_blocks - 1; i >= 0; --i) push(p, initial_order ? initial_order[i] : i);
  *out = p;
  return PA_OK;
}

void pa_pool_destroy(pa_pool* pool) { delete pool; }

pa_status pa_pool_alloc(pa_pool* pool, int32_t* block) {
  if (!pool || !block) return PA_ERR_ARG;
  if (pool->head < 0) return PA_ERR_OOM;
  *block = pop(pool);
  return PA_OK;
}

pa_status pa_pool_incref(pa_pool* pool, int32_t block) {
  if (!pool || !in_range(pool, block)) return PA_ERR_ARG;
  if (pool->refcnt[block] == 0) return PA_ERR_STATE;
  ++pool->refcnt[block];
  return PA_OK;
}

pa_status pa_pool_decref(pa_pool* pool, int32_t block) {
  if (!pool || !in_range(pool, block)) return PA_ERR_ARG;
  if (pool->refcnt[block] == 0) return PA_ERR_STATE;
  if (--pool->refcnt[block] == 0) push(pool, block);
  return PA_OK;
}

int32_t pa_pool_refcount(const pa_pool* pool, int32_t block) {
  if (!pool || !in_range(pool, block)) return -1;
  return pool->refcnt[block];
}

int32_t pa_pool_num_free(const pa_pool* pool) { return pool ? pool->num_free : -1; }

int32_t pa_pool_num_blocks(const pa_pool* pool) { return pool ? pool->num_blocks : -1; }

int32_t pa_pool_free_list(const pa_pool* pool, int32_t* blocks, int32_t capacity) {
  if (!pool || (!blocks && capacity > 0)) return 0;
  int32_t n = 0;
  for (int32_t b = pool->head; b >= 0 && n < capacity; b = pool->next[b]) blocks[n++] = b;
  return n;
}

pa_status pa_seq_append(pa_pool* pool, int32_t* row, int32_t max_blocks, int32_t pos,
                        int32_t block_size, int64_t* slot, int32_t* cow_src, int32_t* cow_dst) {
  if (!pool || !row || !slot || !cow_src || !cow_dst || pos < 0 || block_size <= 0)
    return PA_ERR_ARG;
  const int32_t lb = pos / block_size, off = pos % block_size;
  if (lb >= max_blocks) return PA_ERR_ARG;
  *cow_src = *cow_dst = -1;
  if (off == 0) {
    if (pool->head < 0) return PA_ERR_OOM;
    row[lb] = pop(pool);
  } else {
    const int32_t old = row[lb];
    if (!in_range(pool, old) || pool->refcnt[old] == 0) return PA_ERR_STATE;
    if (pool->refcnt[old] > 1) {
      if (pool->head < 0) return PA_ERR_OOM;
      const int32_t fresh = pop(pool);
      --pool->refcnt[old];   // > 1 before: never frees here
      row[lb] = fresh;
      *cow_src = old;
      *cow_dst = fresh;
    }
  }
  *slot = int64_t(row[lb]) * block_size + off;
  return PA_OK;
}

pa_status pa_seq_extend(pa_pool* pool, int32_t* row, int32_t max_blocks, int32_t start_pos,
                        int32_t n_tokens, int32_t block_size, int64_t* slots, int32_t* cow_src,
                        int32_t* cow_dst, int32_t* n_done) {
  if (n_done) *n_done = 0;
  if (!pool || !row || !cow_src || !cow_dst || n_tokens < 0 || start_pos < 0 || block_size <= 0)
    return PA_ERR_ARG;
  if (n_tokens > 0 && ceil_div(int64_t(start_pos) + n_tokens, block_size) > max_blocks) return PA_ERR_ARG;
  if (int64_t(start_pos) + n_tokens > INT32_MAX) return PA_ERR_ARG;
  *cow_src = *cow_dst = -1;
  for (int32_t i = 0; i < n_tokens; ++i) {
    int64_t slot;
    int32_t cs, cd;
    pa_status st = pa_seq_append(pool, row, max_blocks, start_pos + i, block_size, &slot, &cs, &cd);
    if (st != PA_OK) return st;
    if (cs >= 0) {
      *cow_src = cs;
      *cow_dst = cd;
    }
    if (slots) slots[i] = slot;
    if (n_done) *n_done = i + 1;
  }
  return PA_OK;
}

pa_status pa_seq_fork(pa_pool* pool, const int32_t* row, int32_t n_blocks) {
  if (!pool || (!row && n_blocks > 0) || n_blocks < 0) return PA_ERR_ARG;
  for (int32_t i = 0; i < n_blocks; ++i) {
    if (!in_range(pool, row[i])) return PA_ERR_ARG;
    if (pool->refcnt[row[i]] == 0) return PA_ERR_STATE;
  }
  for (int32_t i = 0; i < n_blocks; ++i) ++pool->refcnt[row[i]];
  return PA_OK;
}

pa_status pa_seq_free(pa_pool* pool, const int32_t* row, int32_t n_blocks) {
  if (!pool || (!row && n_blocks > 0) || n_blocks < 0) return PA_ERR_ARG;
  for (int32_t i = 0; i < n_blocks; ++i) {   // checked first: a refused call drops nothing
    if (!in_range(pool, row[i])) return PA_ERR_ARG;
    if (pool->refcnt[row[i]] == 0) return PA_ERR_STATE;
  }
  for (int32_t i = 0; i < n_blocks; ++i) {
    pa_status st = pa_pool_decref(pool, row[i]);
    if (st != PA_OK) return st;   // only if a block is listed more often than it is held
  }
  return PA_OK;
}

pa_status pa_batch_append(pa_pool* pool, int32_t* block_tables, int32_t num_seqs, int32_t max_blocks,
                          const int32_t* positions, int32_t block_size, int64_t* slots,
                          int64_t* cow_pairs, int32_t* num_cow, int32_t* updates,
                          int32_t* num_updates, int32_t* n_done) {
  if (n_done) *n_done = 0;
  if (num_cow) *num_cow = 0;
  if (num_updates) *num_updates = 0;
  if (!pool || !block_tables || !positions || !slots || !cow_pairs || !num_cow || !updates ||
      !num_updates || num_seqs < 0 || max_blocks <= 0 || block_size <= 0)
    return PA_ERR_ARG;
  for (int32_t s = 0; s < num_seqs; ++s) {
    int32_t* row = block_tables + int64_t(s) * max_blocks;
    const int32_t pos = positions[s];
    int32_t cs, cd;
    pa_status st = pa_seq_append(pool, row, max_blocks, pos, block_size, &slots[s], &cs, &cd);
    if (st != PA_OK) return st;
    if (cs >= 0) {
      cow_pairs[2 * *num_cow] = cs;
      cow_pairs[2 * *num_cow + 1] = cd;
      ++*num_cow;
    }
    if (pos % block_size == 0 || cs >= 0) {
      int32_t* u = updates + 3 * *num_updates;
      u[0] = s;
      u[1] = pos / block_size;
      u[2] = row[pos / block_size];
      ++*num_updates;
    }
    if (n_done) *n_done = s + 1;
  }
  return PA_OK;
}

pa_status pa_batch_reorder(pa_pool* pool, int32_t* block_tables, int32_t* context_lens, int32_t num_seqs,
                           int32_t max_blocks, int32_t block_size, const int32_t* parents) {
  if (!pool || !block_tables || !context_lens || !parents || num_seqs < 0 || max_blocks <= 0 || block_size <= 0)
    return PA_ERR_ARG;
  for (int32_t i = 0; i < num_seqs; ++i) {
    if (parents[i] < 0 || parents[i] >= num_seqs) return PA_ERR_ARG;
    if (context_lens[i] < 0 || ceil_div(context_lens[i], block_size) > max_blocks) return PA_ERR_ARG;
  }
  const size_t n = size_t(num_seqs) * max_blocks;
  std::vector<int32_t> old_tables(block_tables, block_tables + n);
  std::vector<int32_t> old_lens(context_lens, context_lens + num_seqs);
  // every old row's blocks (not only the parents'): each of them loses a reference below
  for (int32_t i = 0; i < num_seqs; ++i) {
    const int32_t nb = int32_t(ceil_div(old_lens[i], block_size));
    for (int32_t k = 0; k < nb; ++k)
      if (!in_range(pool, old_tables[size_t(i) * max_blocks + k]) ||
          pool->refcnt[old_tables[size_t(i) * max_blocks + k]] == 0)
        return PA_ERR_STATE;
  }
  // every new row takes its references before any old row drops its own
  for (int32_t i = 0; i < num_seqs; ++i) {
    const int32_t p = parents[i];
    const int32_t nb = int32_t(ceil_div(old_lens[p], block_size));
    std::memcpy(block_tables + size_t(i) * max_blocks, old_tables.data() + size_t(p) * max_blocks,
                size_t(max_blocks) * sizeof(int32_t));
    context_lens[i] = old_lens[p];
    for (int32_t k = 0; k < nb; ++k) ++pool->refcnt[old_tables[size_t(p) * max_blocks + k]];
  }
  for (int32_t i = 0; i < num_seqs; ++i) {
    const int32_t nb = int32_t(ceil_div(old_lens[i], block_size));
    for (int32_t k = 0; k < nb; ++k) {
      const int32_t b = old_tables[size_t(i) * max_blocks + k];
      if (--pool->refcnt[b] == 0) push(pool, b);
    }
  }
  return PA_OK;
}

}  // extern "C"
