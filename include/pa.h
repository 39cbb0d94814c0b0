/*
 * pa.h -- C ABI of libpa for NVIDIA B200 (sm_100a): paged KV-cache decode attention,
 * the cache write and block copy it needs, the host block pool, and on the same cache
 * multi-query (extend) and whole-prompt (prefill) attention, a prefix-cache index and
 * beam re-selection.
 *
 * The method (PagedAttention as three web pages describe it):
 *   page 1 "突破GPU内存瓶颈：vLLM与PagedAttention技术深度解析", section
 *          "2. PagedAttention的革命性设计" -- fixed-size blocks, a per-sequence block
 *          table mapping logical to physical blocks, blocks shared between sequences;
 *          section "5. 高级应用场景" -- parallel sampling and beam search share blocks;
 *   page 2 (untitled; first section "1. 为什么vLLM能实现24倍推理加速"), section
 *          "1.1 PagedAttention的内存管理革命" -- the op
 *          paged_attention(queries, key_cache, value_cache, block_tables); section
 *          "2.1 核心组件交互流程" -- prefill, decode and extend modes; section
 *          "2.2 关键数据结构剖析" -- the metadata (block_tables, context_lens,
 *          query lengths, num_heads, head_size); section "3.3 常见问题排查" -- the v2
 *          kernel for long text; section "4.2 混合精度策略" -- an FP8 KV cache;
 *   page 3 "内存优化：KV Cache管理、PagedAttention原理与内存池配置", section
 *          "PagedAttention原理" -- blocks of 16 or 32 tokens, refcounted sharing, a free
 *          list with O(1) alloc/free and no device allocation per request; section
 *          "案例与场景" -- a hash index over the blocks of common prefixes.
 *
 * Conventions for every call below.
 *   - Device pointers are plain CUDA device addresses owned by the caller; the
 *     library never allocates or frees device memory. The only device memory it
 *     holds is part of its own device image: the sticky device error word (below)
 *     and the fixed scratch array of pa_decode_no_alloc. Host pointers are plain
 *     host memory owned by the caller.
 *   - The library keeps per-device state for the life of the process: kernel
 *     attributes set on first use, occupancy figures, and the device address of the
 *     pa_decode_no_alloc array. All of it belongs to the device's primary context.
 *     cudaDeviceReset destroys that context (the array may then sit at another
 *     address), so do not call the library on a device after resetting it.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream). GPU calls only enqueue work and return; results are ready when the
 *     stream reaches them.
 *   - Argument checks that need no device data (null pointers, shapes, dtype
 *     combinations, 16-byte alignment, supported head_dim / block_size / group
 *     size) run on the host before anything is enqueued and return PA_ERR_ARG;
 *     nothing is launched then.
 *   - Checks of device data (block ids in [0, num_blocks), context lengths within
 *     the block table and the declared maximum, slots and copy pairs in range)
 *     run inside the kernels. A violation never touches memory out of range: the
 *     offending item is skipped (or its length clamped), and a sticky device error
 *     word records the first violation; read it with pa_last_device_error().
 *   - A CUDA launch error returns PA_ERR_CUDA.
 *
 * Cache layout (both K and V): [num_blocks][num_kv_heads][block_size][head_dim],
 * row-major, contiguous. Token position j of a sequence s lives at
 *   cache[block_tables[s][j / block_size]][h][j % block_size][:].
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_ARG = -1,          /* invalid argument (host-side check); nothing enqueued */
  PA_ERR_OOM = -2,          /* block pool has no free block */
  PA_ERR_STATE = -3,        /* refcount of a free block taken or dropped */
  PA_ERR_CUDA = -4,         /* a CUDA runtime call failed */
  PA_ERR_DEVICE_CHECK = -5  /* a kernel found invalid device data (see pa_last_device_error) */
} pa_status;

typedef enum { PA_F16 = 0, PA_BF16 = 1, PA_E4M3 = 2 } pa_dtype;

/* Device error codes recorded by the kernels (first one wins until read). */
enum {
  PA_DEV_OK = 0,
  PA_DEV_BAD_BLOCK_ID = 1,     /* info: seq, logical block, value */
  PA_DEV_BAD_CONTEXT_LEN = 2,  /* info: seq, value, limit */
  PA_DEV_BAD_SLOT = 3,         /* info: token, value, limit */
  PA_DEV_BAD_COPY_PAIR = 4,    /* info: pair, src, dst */
  PA_DEV_BAD_TABLE_UPDATE = 5, /* info: update, seq, col */
  PA_DEV_WAIT_TIMEOUT = 6      /* info: kernel id, unit, stage */
};

/*
 * One KV cache (K and V of one attention layer).
 *   num_blocks    physical blocks in the pool
 *   num_kv_heads  kv heads (Hkv)
 *   block_size    tokens per block: 8, 16 or 32 (page 3, section "内存池配置": 8..32;
 *                 16 the default, 32 for sequences beyond 4K tokens)
 *   head_dim      64 or 128
 *   kv_dtype      PA_F16, PA_BF16 or PA_E4M3 (OCP E4M3, saturating, one scale per tensor)
 *   k_scale, v_scale  per-tensor dequantisation scales: stored code c means c * scale.
 *                 Must be 1.0 for 16-bit caches.
 *   k_cache, v_cache  device pointers, 16-byte aligned.
 */
typedef struct {
  int32_t num_blocks;
  int32_t num_kv_heads;
  int32_t block_size;
  int32_t head_dim;
  int32_t kv_dtype;
  float k_scale;
  float v_scale;
  void* k_cache;
  void* v_cache;
} pa_cache_desc;

/* ------------------------------------------------------------------------- */
/* KV-cache write                                                             */
/* ------------------------------------------------------------------------- */
/*
 * pa_reshape_and_cache -- write each new token's K and V rows into its slot.
 * The slot of logical position j of a sequence is block_table[j / BS] * BS + j % BS
 * (page 1, section "2. PagedAttention的革命性设计", the block table).
 *   k, v          device [num_tokens][num_kv_heads][head_dim] of in_dtype; consecutive
 *                 tokens are k_token_stride (v_token_stride) elements apart, heads and
 *                 dims contiguous inside a token; 16-byte aligned rows.
 *   in_dtype      PA_F16 or PA_BF16. For 16-bit caches it must equal kv_dtype and the
 *                 codes are copied bit for bit. For an E4M3 cache each value x is stored
 *                 as e4m3_rne_satfinite(x / scale), the division in binary32.
 *   slot_mapping  device int64 [num_tokens]; a negative slot skips the token; a slot
 *                 >= num_blocks * block_size is skipped and recorded (PA_DEV_BAD_SLOT).
 * Two tokens with the same slot race; callers give distinct slots.
 */
pa_status pa_reshape_and_cache(const void* k, const void* v, int32_t in_dtype, int32_t num_tokens,
                               int64_t k_token_stride, int64_t v_token_stride,
                               const int64_t* slot_mapping, const pa_cache_desc* cache,
                               void* stream);

/* ------------------------------------------------------------------------- */
/* Block copy (copy-on-write)                                                 */
/* ------------------------------------------------------------------------- */
/*
 * pa_copy_blocks -- for each pair (src, dst): block dst of K and of V becomes a bit
 * copy of block src (all kv heads, all slots). This is the copy that copy-on-write
 * needs when a sequence appends into a block it shares (page 3, section
 * "PagedAttention原理": blocks shared between requests through reference counts;
 * page 1, section "5. 高级应用场景": parallel sampling and beam search).
 *   src_dst_pairs device int64 [num_pairs][2].
 * Pairs are copied concurrently, so a batch must not chain copies: no block may be
 * the destination of one pair and the source or destination of another (two pairs
 * may share a source). The kernel checks this: a pair that clashes with another in
 * this way is not copied, and neither is the other one; a clash, like an out-of-range
 * id, skips the pair and is recorded (PA_DEV_BAD_COPY_PAIR, info = pair index, src,
 * dst). Every pair that is copied reads the cache as it was before the call. The
 * check costs each pair a scan of the batch (num_pairs * 16 bytes, from L2).
 * num_pairs == 0 enqueues nothing.
 */
pa_status pa_copy_blocks(const int64_t* src_dst_pairs, int32_t num_pairs,
                         const pa_cache_desc* cache, void* stream);

/* ------------------------------------------------------------------------- */
/* Decode attention                                                           */
/* ------------------------------------------------------------------------- */
/*
 * pa_decode -- one query token per sequence attends over its whole paged context:
 *   out[s,h,:] = sum_j softmax_j(scale * <q[s,h,:], K_s[j]>) * V_s[j],  j < context_lens[s]
 * with K_s[j] = k_scale * cache_k[block_tables[s][j / BS]][h / G][j % BS][:] (V likewise),
 * G = num_q_heads / num_kv_heads (query head h reads kv head h / G).
 * Page 2, section "1.1 PagedAttention的内存管理革命" (the paged op beside
 * matmul(q, k^T)/sqrt(d)); page 3, section "核心原理" (one query against all cached keys).
 * Long contexts are split into partitions of 512 tokens whose partial results
 * (running max, sum of exponentials, unnormalised output) are merged by a second,
 * log-sum-exp kernel (page 2, section "3.3 常见问题排查": the v2 kernel for long text).
 * All softmax and accumulation arithmetic is binary32.
 *   q              device [num_seqs][num_q_heads][head_dim] of q_dtype (PA_F16 / PA_BF16);
 *                  for 16-bit caches q_dtype must equal kv_dtype.
 *   block_tables   device int32 [num_seqs][max_blocks_per_seq].
 *   context_lens   device int32 [num_seqs]; 0 gives an all-zero output row.
 *   max_context_len host upper bound of context_lens (sizes the partition grid);
 *                  at most 6,291,456 (12288 partitions).
 *   scale          softmax scale (e.g. 1/sqrt(head_dim)).
 *   out            device [num_seqs][num_q_heads][head_dim] of q_dtype, rounded to
 *                  nearest even from binary32.
 *   workspace      device scratch of at least pa_decode_workspace_size() bytes,
 *                  256-byte aligned; owned by the caller; contents need not be
 *                  initialised and are undefined afterwards. Two pa_decode calls that
 *                  run at the same time need separate workspaces.
 * Supported: head_dim 64 or 128; block_size 8, 16, 32; G in {1, 2, 4, 8}.
 */
pa_status pa_decode(const void* q, int32_t q_dtype, int32_t num_seqs, int32_t num_q_heads,
                    const pa_cache_desc* cache, const int32_t* block_tables,
                    int32_t max_blocks_per_seq, const int32_t* context_lens,
                    int32_t max_context_len, float scale, void* out, void* workspace,
                    size_t workspace_bytes, void* stream);

/* Bytes of workspace pa_decode needs for these sizes: 0 for a negative sequence count or
 * context length and for a non-positive head count or head_dim. A size is returned for any
 * max_context_len >= 0; pa_decode itself refuses one above 6,291,456 (PA_ERR_ARG). */
size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                int32_t max_context_len);

/*
 * pa_decode_stage -- run one of pa_decode's three launches alone, with the same
 * arguments: stage 0 plans the partitions (and zeroes rows of empty sequences),
 * stage 1 runs the partition kernel, stage 2 merges partitions. Running 0, 1, 2 in
 * order on one stream is exactly pa_decode. For timing one kernel in isolation.
 */
pa_status pa_decode_stage(int32_t stage, const void* q, int32_t q_dtype, int32_t num_seqs,
                          int32_t num_q_heads, const pa_cache_desc* cache,
                          const int32_t* block_tables, int32_t max_blocks_per_seq,
                          const int32_t* context_lens, int32_t max_context_len, float scale,
                          void* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * pa_decode_no_alloc -- pa_decode for callers that may not allocate device memory.
 * The source pages have no counterpart; this entry point exists for integration.
 * Who needs it: code that is not allowed to call cudaMalloc/cudaFree, e.g. a plugin
 * inside a host framework that owns all device memory through its own caching
 * allocator (raw allocations would escape its accounting, and cudaFree synchronises
 * the device), or a serving loop that forbids allocation calls because they can
 * stall other streams. Same arguments and results as pa_decode, minus the
 * workspace: the split-K scratch is a fixed array of PA_NO_ALLOC_WORKSPACE_BYTES
 * (16 MiB) inside the library's device image, present on every GPU that loads the
 * library until the process exits. The call allocates nothing.
 *   - Sizes whose pa_decode_workspace_size() exceeds PA_NO_ALLOC_WORKSPACE_BYTES are
 *     rejected with PA_ERR_ARG before anything is enqueued (e.g. 8 sequences x 32 q
 *     heads x 32K tokens x head_dim 128 fit; 256 x 40 heads x 8K do not).
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current, through cudaGetSymbolAddress) and keeps it
 *     for the life of the process; make that first call before any stream capture.
 *     The address is that of the device's primary context: after cudaDeviceReset it
 *     is stale (see the conventions above).
 *   - Every call on a device shares the one array and leaves its contents behind;
 *     nothing in it needs to start at zero. Calls that may overlap on the GPU (on
 *     different streams, or from different host threads) race on it: serialise them.
 */
#define PA_NO_ALLOC_WORKSPACE_BYTES ((size_t)16 << 20)
pa_status pa_decode_no_alloc(const void* q, int32_t q_dtype, int32_t num_seqs, int32_t num_q_heads,
                             const pa_cache_desc* cache, const int32_t* block_tables,
                             int32_t max_blocks_per_seq, const int32_t* context_lens,
                             int32_t max_context_len, float scale, void* out, void* stream);

/*
 * pa_extend -- several new tokens per sequence attend causally over the paged context
 * (speculative verification, chunked prefill). Page 2, section "2.1 核心组件交互流程":
 * the engine runs prefill, decode and extend modes; section "2.2 关键数据结构剖析": the
 * metadata carries query lengths beside the context lengths.
 *   query_start    device int32 [num_seqs + 1]: sequence s owns query rows
 *                  query_start[s] .. query_start[s+1]-1 (Q_s rows), query_start[0] = 0
 *   num_tokens     host: query_start[num_seqs] (rows of q and out)
 *   context_lens   device int32 [num_seqs]: L_s, including the Q_s new tokens, whose K/V
 *                  are already in the cache (pa_reshape_and_cache)
 *   q, out         device [num_tokens][num_q_heads][head_dim] of q_dtype
 * Query i of sequence s sits at position L_s - Q_s + i and attends to tokens
 * 0 .. L_s - Q_s + i; out = softmax(scale * q K^T) V over them. Q_s > L_s, or a range
 * outside [0, num_tokens], is recorded (PA_DEV_BAD_CONTEXT_LEN) and its rows are zero.
 * Runs on the tensor cores (16-bit inputs, binary32 accumulation): mma.sync for short
 * query runs, tcgen05 with TMEM accumulators for long ones (16-bit caches, head_dim 128,
 * scale > 0); context chunks (multiples of 512 tokens) merged by a log-sum-exp kernel as
 * in pa_decode. P enters P V in the products' 16-bit type; for bf16 its rounded remainder
 * p - bf16(p) enters as a second product (always on mma.sync; on tcgen05 for every
 * 128-token tile in which some row has a weight above 1/8 of its running sum), so every
 * weight is carried to within 2^-16 of its value where that matters. Cache bytes past a
 * context never affect the output.
 * E4M3 caches: each cache block is converted to f16 in shared memory (exact) and the
 * products run in f16 with P in f16; a bf16 q is read as f16 after a 2^-8 scaling (exact
 * for |q| in [2^-6, 1.6e7], saturating above); k_scale and v_scale multiply the scores
 * and the output. These take the mma.sync path for runs of any length.
 * Supported: 16-bit caches with q_dtype == kv_dtype, or E4M3 caches with q_dtype PA_F16
 * or PA_BF16; head_dim 64 or 128, block_size 16 or 32, G in {1, 2, 4, 8}.
 * workspace >= pa_extend_workspace_size(...), 256-byte aligned. A call with num_seqs or
 * num_tokens 0 checks its arguments and launches nothing.
 */
pa_status pa_extend(const void* q, int32_t q_dtype, int32_t num_seqs, int32_t num_q_heads,
                    const int32_t* query_start, int32_t num_tokens, const pa_cache_desc* cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                    int32_t max_context_len, float scale, void* out, void* workspace, size_t workspace_bytes,
                    void* stream);
/* Bytes of workspace pa_extend and pa_prefill need: 0 for negative counts or lengths and for a
 * non-positive head count or head_dim; the same length limit as pa_decode applies to the calls. */
size_t pa_extend_workspace_size(int32_t num_seqs, int32_t num_tokens, int32_t num_q_heads, int32_t head_dim,
                                int32_t max_context_len);

/*
 * pa_prefill -- causal attention of whole prompts over themselves, writing the prompts'
 * K / V into the paged cache in the same pass. Page 2, section "2.1 核心组件交互流程":
 * the engine's prefill mode processes the prompt and fills the KV cache that decode then
 * reads (paged layout of page 3, section "PagedAttention原理").
 *   q              device [num_tokens][num_q_heads][head_dim], dtype
 *   k, v           device [num_tokens][num_kv_heads][head_dim], dtype: the prompts' keys
 *                  and values, rows in query order (as pa_reshape_and_cache takes them)
 *   query_start    device int32 [num_seqs + 1]: sequence s owns rows query_start[s] ..
 *                  query_start[s+1]-1 (its prompt of Q_s tokens), query_start[0] = 0
 *   context_lens   device int32 [num_seqs]: must equal Q_s (a prompt attends to itself);
 *                  otherwise the sequence is recorded (PA_DEV_BAD_CONTEXT_LEN) and its rows
 *                  are zero
 *   block_tables   device int32 [num_seqs][max_blocks_per_seq]: blocks that belong to the
 *                  sequence alone (freshly allocated), covering its Q_s tokens
 *   out            device [num_tokens][num_q_heads][head_dim], dtype
 * Afterwards cache slot bt[s][i / BS] * BS + i % BS holds k / v of prompt token i (bit for
 * bit for a 16-bit cache; for an E4M3 cache encoded as pa_reshape_and_cache encodes it,
 * e4m3_rne_satfinite(x / scale)), for every i < Q_s; the slots past Q_s in a prompt's last
 * block hold unspecified values. out is as pa_extend computes it with those cache contents
 * (for an E4M3 cache: over the quantised K / V).
 * 16-bit caches: one tcgen05 kernel loads each K / V tile from the prompt rows, writes it
 * into the cache and attends to it in the same pass. E4M3 caches: one launch quantises the
 * prompts into the cache, then pa_extend's E4M3 kernel reads them back.
 * Supported: dtype = the cache's kv_dtype = PA_F16 or PA_BF16 with head_dim 128 and
 * scale > 0 (the tcgen05 path), or an E4M3 cache with dtype PA_F16 or PA_BF16 and head_dim
 * 64 or 128; block_size 16 or 32, G in {1, 2, 4, 8}; PA_ERR_ARG otherwise. workspace >=
 * pa_extend_workspace_size(...), 256-byte aligned; k, v, q and out 16-byte aligned.
 */
pa_status pa_prefill(const void* q, const void* k, const void* v, int32_t dtype, int32_t num_seqs,
                     int32_t num_q_heads, const int32_t* query_start, int32_t num_tokens, const pa_cache_desc* cache,
                     const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                     int32_t max_context_len, float scale, void* out, void* workspace, size_t workspace_bytes,
                     void* stream);

/*
 * pa_selftest_wait_timeout -- failure-detection self-test (the pages have no counterpart:
 * it exercises this library's own guard). Enqueues one CTA on `stream` whose thread
 * waits, through the same bounded mbarrier wait every kernel here uses, on a barrier that
 * nothing ever arrives at. After limit_us microseconds the wait gives up, records
 * PA_DEV_WAIT_TIMEOUT with info = {0x7E57, elapsed microseconds, 0} and the kernel
 * returns: nothing faults, nothing hangs, the context stays usable. Read the result with
 * pa_last_device_error. limit_us in 1 .. 2000000, else PA_ERR_ARG.
 */
pa_status pa_selftest_wait_timeout(uint32_t limit_us, void* stream);

/*
 * pa_last_device_error -- synchronise `stream`, then read and clear the device error
 * word of the current device. *code receives a PA_DEV_* value; info (may be NULL)
 * receives 3 int32 details. Returns PA_ERR_DEVICE_CHECK when *code != 0.
 */
pa_status pa_last_device_error(void* stream, int32_t* code, int32_t* info);

/* ------------------------------------------------------------------------- */
/* Device mirror of the block tables                                          */
/* ------------------------------------------------------------------------- */
/*
 * pa_block_table_update -- apply table entries produced by the host bookkeeping
 * (pa_batch_append's updates) to the device copy of the block tables:
 *   block_tables[u.seq * max_blocks_per_seq + u.col] = u.block for every update u.
 *   updates  device int32 [num_updates][3] = (seq, col, block).
 * Out-of-range (seq, col) skips the update and is recorded (PA_DEV_BAD_TABLE_UPDATE).
 */
pa_status pa_block_table_update(const int32_t* updates, int32_t num_updates, int32_t* block_tables,
                                int32_t num_seqs, int32_t max_blocks_per_seq, void* stream);

/* ------------------------------------------------------------------------- */
/* Host block pool: O(1) free list + reference counts                         */
/* ------------------------------------------------------------------------- */
/*
 * Page 3, section "PagedAttention原理": free blocks form a linked list, alloc and free
 * are O(1), blocks are shared through reference counts; a sequence takes a block
 * only when it grows into one and returns all of them when it finishes; waste is
 * confined to a sequence's last block (page 1, section "2. PagedAttention的革命性设计").
 * The free list is a LIFO stack threaded through an array; initial_order seeds it
 * so that successive allocations return initial_order[0], [1], ...; a block whose
 * count reaches zero is pushed on top. Not thread-safe: one pool per engine thread.
 */
typedef struct pa_pool pa_pool;

/* initial_order: host int32 permutation of 0..num_blocks-1, or NULL for 0..N-1. */
pa_status pa_pool_create(int32_t num_blocks, const int32_t* initial_order, pa_pool** out);
void pa_pool_destroy(pa_pool* pool);
pa_status pa_pool_alloc(pa_pool* pool, int32_t* block);      /* refcount := 1; PA_ERR_OOM if empty */
pa_status pa_pool_incref(pa_pool* pool, int32_t block);      /* PA_ERR_STATE if block is free */
pa_status pa_pool_decref(pa_pool* pool, int32_t block);      /* at 0 the block is freed;
                                                                PA_ERR_STATE if already free */
int32_t pa_pool_refcount(const pa_pool* pool, int32_t block); /* -1 if out of range */
int32_t pa_pool_num_free(const pa_pool* pool);
int32_t pa_pool_num_blocks(const pa_pool* pool);
/* The free list in allocation order (first = next to be handed out); writes
 * min(capacity, num_free) ids and returns how many it wrote. */
int32_t pa_pool_free_list(const pa_pool* pool, int32_t* blocks, int32_t capacity);

/*
 * pa_seq_append -- host bookkeeping for appending logical position `pos` to one
 * sequence. block_table_row (host, max_blocks entries) holds ceil(pos / BS) valid
 * entries before the call. If pos % BS == 0 a new block is allocated into entry
 * pos / BS. Otherwise, if the last block is shared (refcount > 1), a fresh block is
 * allocated, (old, new) is reported through *cow_src / *cow_dst for pa_copy_blocks,
 * the old block loses one reference and the entry is replaced (copy-on-write).
 * *slot = row[pos / BS] * BS + pos % BS. *cow_src = *cow_dst = -1 when no copy.
 * On PA_ERR_OOM nothing has changed.
 */
pa_status pa_seq_append(pa_pool* pool, int32_t* block_table_row, int32_t max_blocks, int32_t pos,
                        int32_t block_size, int64_t* slot, int32_t* cow_src, int32_t* cow_dst);

/*
 * pa_seq_extend -- append positions start_pos .. start_pos + n_tokens - 1 (a prompt).
 * slots (host int64 [n_tokens]) may be NULL. At most the first position can need a
 * copy; it is reported through *cow_src / *cow_dst (-1 when none). On PA_ERR_OOM the
 * positions before the failing one have been appended; *n_done (may be NULL) says
 * how many.
 */
pa_status pa_seq_extend(pa_pool* pool, int32_t* block_table_row, int32_t max_blocks,
                        int32_t start_pos, int32_t n_tokens, int32_t block_size, int64_t* slots,
                        int32_t* cow_src, int32_t* cow_dst, int32_t* n_done);

/* pa_seq_fork -- a sequence sharing the first n_blocks blocks of row: each gets one
 * more reference; the caller copies the row. */
pa_status pa_seq_fork(pa_pool* pool, const int32_t* block_table_row, int32_t n_blocks);

/* pa_seq_free -- a finished sequence drops one reference of each of its n_blocks blocks.
 * The blocks are checked first: one out of range (PA_ERR_ARG) or already free
 * (PA_ERR_STATE) drops nothing. */
pa_status pa_seq_free(pa_pool* pool, const int32_t* block_table_row, int32_t n_blocks);

/*
 * pa_batch_append -- one decode step's bookkeeping for a batch: pa_seq_append for
 * sequences 0..num_seqs-1 in order, at positions[s].
 *   block_tables  host int32 [num_seqs][max_blocks] (updated in place)
 *   slots         host int64 [num_seqs] out
 *   cow_pairs     host int64 [num_seqs][2] out; *num_cow pairs written
 *   updates       host int32 [num_seqs][3] out; (seq, col, block) for every table
 *                 entry written, *num_updates of them (for pa_block_table_update)
 *   n_done        sequences fully processed (== num_seqs on success)
 * On an error the sequences before *n_done have been appended and reported.
 */
pa_status pa_batch_append(pa_pool* pool, int32_t* block_tables, int32_t num_seqs, int32_t max_blocks,
                          const int32_t* positions, int32_t block_size, int64_t* slots,
                          int64_t* cow_pairs, int32_t* num_cow, int32_t* updates,
                          int32_t* num_updates, int32_t* n_done);

/* ------------------------------------------------------------------------- */
/* Prefix cache (host)                                                        */
/* ------------------------------------------------------------------------- */
/*
 * A host index from the token content of full KV blocks to the physical blocks that
 * hold them (page 3, section "案例与场景": a global hash index over the KV blocks of a
 * common prefix; a matching request reuses those blocks and allocates only for its
 * new tokens; section "误区与复盘" (误区3): only exactly equal prefixes hit).
 * Full block k of a prompt is reusable iff the prompt's tokens [0, (k+1)*BS) equal
 * those of the sequence that filled the cached block. Keys chain a 64-bit FNV-1a hash
 * over the previous block's key and the block's token ids; every hit is verified
 * against the stored parent key and tokens, so a reuse is always exact. The index
 * holds one pool reference on every block it lists. Not thread-safe.
 */
typedef struct pa_prefix_cache pa_prefix_cache;
pa_status pa_prefix_cache_create(int32_t block_size, pa_prefix_cache** out);
/* Frees the index only; call pa_prefix_cache_clear first to return its references. */
void pa_prefix_cache_destroy(pa_prefix_cache* cache);
int32_t pa_prefix_cache_size(const pa_prefix_cache* cache);
/* Walks the prompt's full blocks in order; each hit takes a reference and is written
 * to block_table_row[k]; stops at the first miss. *n_matched = blocks reused. If a
 * reference is refused (PA_ERR_STATE: a listed block was freed behind the index's back)
 * the hits before it stand and *n_matched counts them. */
pa_status pa_prefix_cache_match(pa_prefix_cache* cache, pa_pool* pool, const int32_t* tokens, int32_t n_tokens,
                                int32_t* block_table_row, int32_t max_blocks, int32_t* n_matched);
/* Lists every full block of a sequence (tokens from position 0, blocks in
 * block_table_row, one entry per full block) that the index does not hold yet, taking
 * a reference on each. On an error the entries added before it stand (*n_inserted). */
pa_status pa_prefix_cache_insert(pa_prefix_cache* cache, pa_pool* pool, const int32_t* tokens, int32_t n_tokens,
                                 const int32_t* block_table_row, int32_t* n_inserted);
/* Drops, oldest insertion first, up to max_blocks entries whose block only the index
 * holds (refcount 1); those blocks return to the free list. */
pa_status pa_prefix_cache_evict(pa_prefix_cache* cache, pa_pool* pool, int32_t max_blocks, int32_t* n_evicted);
/* Drops every entry and its reference. On an error the entries released before it
 * have left the index (*n_released); the rest remain listed. */
pa_status pa_prefix_cache_clear(pa_prefix_cache* cache, pa_pool* pool, int32_t* n_released);

/* ------------------------------------------------------------------------- */
/* Native decode step                                                         */
/* ------------------------------------------------------------------------- */
/*
 * pa_engine -- one call per decode step: host bookkeeping for every sequence and
 * the step's device work, with no interpreter in between (page 3, section
 * "PagedAttention原理": blocks taken on demand, shared by reference count; page 2,
 * section "2.2 关键数据结构剖析": block tables and context lengths reach the kernels as
 * attention metadata). The engine owns two CUDA events and nothing else; every
 * buffer below is the caller's and must outlive the engine.
 *   pool                  the block pool (borrowed; not thread-safe, see above)
 *   block_tables_host     host int32 [num_seqs][max_blocks_per_seq], the pool's tables
 *   context_lens_host     host int32 [num_seqs]: tokens each sequence holds; a step
 *                         appends one token to every sequence and increments them
 *   block_tables_dev      device int32 [num_seqs][max_blocks_per_seq], the mirror the
 *                         kernels read (patched every step with the updates)
 *   meta_host[2]          two pinned host buffers of meta_bytes (double-buffered)
 *   meta_dev              device buffer of meta_bytes, 16-byte aligned
 *   meta_bytes            >= pa_engine_meta_bytes(num_seqs)
 *   workspace             device scratch for pa_decode (>= pa_decode_workspace_size)
 *   cache, q_dtype, num_q_heads, max_context_len, scale   as for pa_decode
 */
typedef struct {
  pa_pool* pool;
  int32_t num_seqs;
  int32_t num_q_heads;
  int32_t max_blocks_per_seq;
  int32_t max_context_len;
  int32_t q_dtype;
  float scale;
  pa_cache_desc cache;
  int32_t* block_tables_host;
  int32_t* context_lens_host;
  int32_t* block_tables_dev;
  void* meta_host[2];
  void* meta_dev;
  size_t meta_bytes;
  void* workspace;
  size_t workspace_bytes;
} pa_engine_config;

typedef struct pa_engine pa_engine;

/* Bytes of one metadata buffer for num_seqs sequences (slots, copy pairs, lengths,
 * table updates, each 16-byte aligned). */
size_t pa_engine_meta_bytes(int32_t num_seqs);
pa_status pa_engine_create(const pa_engine_config* config, pa_engine** out);
void pa_engine_destroy(pa_engine* engine);

/*
 * pa_engine_step -- append one token to every sequence and decode:
 *   1. pa_batch_append on the host (slots, copy-on-write pairs, table updates);
 *   2. one cudaMemcpyAsync of the packed metadata (waits first, on the host, for the
 *      copy of two steps ago that read the same pinned buffer);
 *   3. pa_block_table_update, pa_copy_blocks (only when there are updates / pairs),
 *      pa_reshape_and_cache of k_new / v_new, pa_decode.
 *   q, out        device [num_seqs][num_q_heads][head_dim] of q_dtype
 *   k_new, v_new  device [num_seqs][num_kv_heads][head_dim] of q_dtype, contiguous
 *   ev_partition_begin / _end  optional cudaEvent_t (NULL = none), recorded on the
 *                 stream right before and after the partition kernel (for timing it)
 * On PA_ERR_OOM the sequences before the failing one have been appended (their
 * context_lens_host entries incremented) and nothing has been enqueued.
 */
pa_status pa_engine_step(pa_engine* engine, const void* q, const void* k_new, const void* v_new, void* out,
                         void* stream, void* ev_partition_begin, void* ev_partition_end);

/* Copy pairs, table updates and kernel launches of the last step. */
pa_status pa_engine_last_step(const pa_engine* engine, int32_t* num_cow, int32_t* num_updates,
                              int32_t* launches);

/*
 * pa_batch_reorder -- beam re-selection: new sequence i continues old sequence
 * parents[i] (page 1, section "5. 高级应用场景": beams share their common blocks).
 * Row i of block_tables (host int32 [num_seqs][max_blocks]) becomes a copy of old row
 * parents[i] and context_lens[i] (host, tokens held) its length; every new row takes
 * one reference per block before any old row drops its references, so a beam chosen
 * k times holds its blocks k times and a beam chosen 0 times frees its private
 * blocks. The next pa_seq_append / pa_batch_append into a shared partial block then
 * reports the copy-on-write pair. O(total blocks). The caller refreshes the device
 * mirror of the tables (e.g. a full upload). Every old row's blocks are checked first
 * (in range and held); PA_ERR_ARG / PA_ERR_STATE leave everything unchanged.
 */
pa_status pa_batch_reorder(pa_pool* pool, int32_t* block_tables, int32_t* context_lens, int32_t num_seqs,
                           int32_t max_blocks, int32_t block_size, const int32_t* parents);

/* Library version string and the device architecture it was built for. */
const char* pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
