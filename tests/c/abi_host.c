/* A plain C11 consumer of include/pa.h: the host calls of the C ABI (block pool,
 * copy-on-write bookkeeping, beam re-selection, prefix cache) driven from C with no GPU.
 * Exit status 0 when every expectation holds; the first failed one is printed. */
#include <stdint.h>
#include <stdio.h>

#include "pa.h"

#define EXPECT(c)                                                   \
  do {                                                              \
    if (!(c)) {                                                     \
      fprintf(stderr, "%s:%d: expectation failed: %s\n", __FILE__, __LINE__, #c); \
      return 1;                                                     \
    }                                                               \
  } while (0)

int main(void) {
  /* page 1's block tables: seq_1 = [0, 1, 3], seq_2 = [2, 1, 4] with block 1 shared */
  pa_pool* pool = NULL;
  EXPECT(pa_pool_create(8, NULL, &pool) == PA_OK && pool);
  int32_t s1[4] = {0}, s2[4] = {0}, b = -1;
  EXPECT(pa_pool_alloc(pool, &b) == PA_OK && b == 0); s1[0] = b;
  EXPECT(pa_pool_alloc(pool, &b) == PA_OK && b == 1); s1[1] = b;
  EXPECT(pa_pool_alloc(pool, &b) == PA_OK && b == 2); s2[0] = b;
  EXPECT(pa_pool_incref(pool, 1) == PA_OK); s2[1] = 1;
  EXPECT(pa_pool_alloc(pool, &b) == PA_OK && b == 3); s1[2] = b;
  EXPECT(pa_pool_alloc(pool, &b) == PA_OK && b == 4); s2[2] = b;
  EXPECT(pa_pool_refcount(pool, 1) == 2 && pa_pool_num_free(pool) == 3);
  EXPECT(s1[0] == 0 && s1[1] == 1 && s1[2] == 3 && s2[0] == 2 && s2[1] == 1 && s2[2] == 4);

  /* copy-on-write: a forked sequence appends into the shared partial block */
  pa_pool* p2 = NULL;
  EXPECT(pa_pool_create(10, NULL, &p2) == PA_OK);
  int32_t a[4] = {0}, f[4] = {0}, cs = 0, cd = 0, done = 0;
  int64_t slots[20], slot = 0;
  EXPECT(pa_seq_extend(p2, a, 4, 0, 20, 16, slots, &cs, &cd, &done) == PA_OK && done == 20);
  EXPECT(cs == -1 && slots[19] == (int64_t)a[1] * 16 + 3);
  EXPECT(pa_seq_fork(p2, a, 2) == PA_OK);
  f[0] = a[0]; f[1] = a[1];
  EXPECT(pa_seq_append(p2, f, 4, 20, 16, &slot, &cs, &cd) == PA_OK);
  EXPECT(cs == a[1] && cd != a[1] && f[1] == cd && slot == (int64_t)cd * 16 + 4);
  EXPECT(pa_pool_refcount(p2, a[1]) == 1 && pa_pool_refcount(p2, a[0]) == 2);

  /* beam re-selection: both rows continue row 0; row 1's private block is freed */
  int32_t tables[2][4] = {{a[0], a[1], 0, 0}, {f[0], f[1], 0, 0}};
  int32_t lens[2] = {20, 21}, parents[2] = {0, 0};
  const int32_t nfree = pa_pool_num_free(p2);
  EXPECT(pa_batch_reorder(p2, &tables[0][0], lens, 2, 4, 16, parents) == PA_OK);
  EXPECT(tables[1][0] == a[0] && tables[1][1] == a[1] && lens[1] == 20);
  EXPECT(pa_pool_refcount(p2, a[1]) == 2 && pa_pool_num_free(p2) == nfree + 1);

  /* prefix cache: a second request with the same 8-token prompt reuses both blocks */
  pa_prefix_cache* pc = NULL;
  EXPECT(pa_prefix_cache_create(4, &pc) == PA_OK);
  pa_pool* p3 = NULL;
  EXPECT(pa_pool_create(6, NULL, &p3) == PA_OK);
  const int32_t toks[8] = {1, 2, 3, 4, 5, 6, 7, 8};
  int32_t r1[2] = {0}, r2[2] = {-1, -1}, n = -1;
  EXPECT(pa_seq_extend(p3, r1, 2, 0, 8, 4, NULL, &cs, &cd, &done) == PA_OK);
  EXPECT(pa_prefix_cache_insert(pc, p3, toks, 8, r1, &n) == PA_OK && n == 2);
  EXPECT(pa_prefix_cache_match(pc, p3, toks, 8, r2, 2, &n) == PA_OK && n == 2);
  EXPECT(r2[0] == r1[0] && r2[1] == r1[1] && pa_pool_refcount(p3, r1[0]) == 3);
  EXPECT(pa_prefix_cache_clear(pc, p3, &n) == PA_OK && n == 2 && pa_prefix_cache_size(pc) == 0);

  /* errors: out of blocks, a reference on a free block, a bad argument */
  int32_t x;
  pa_pool* p4 = NULL;
  EXPECT(pa_pool_create(1, NULL, &p4) == PA_OK && pa_pool_alloc(p4, &x) == PA_OK);
  EXPECT(pa_pool_alloc(p4, &x) == PA_ERR_OOM);
  EXPECT(pa_pool_decref(p4, 0) == PA_OK && pa_pool_decref(p4, 0) == PA_ERR_STATE);
  EXPECT(pa_pool_create(0, NULL, &p4) == PA_ERR_ARG);

  pa_prefix_cache_destroy(pc);
  pa_pool_destroy(pool);
  pa_pool_destroy(p2);
  pa_pool_destroy(p3);
  printf("c abi ok: %s\n", pa_version());
  return 0;
}
