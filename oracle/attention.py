"""Paged single-query decode attention in float64 (oracle; test infrastructure only).

What is computed (page 2, section "1.1 PagedAttention的内存管理革命", where the
paged op ``paged_attention(queries, key_cache, value_cache, block_tables)`` is
set beside the dense ``matmul(query, key^T) / sqrt(dim)``; page 3, section
"核心原理", where each decode step scores the current token's query against the
keys and values of every earlier token): paging changes *where* K and V live,
not the arithmetic. For sequence s with context length L_s and query head h:

    K_s[j] = dec(k_cache[bt[s][j // BS], g, j % BS, :]) * k_scale     j < L_s
    V_s[j] = dec(v_cache[bt[s][j // BS], g, j % BS, :]) * v_scale
    x_j    = scale * <dec(q[s, h, :]), K_s[j]>
    out[s, h, :] = sum_j softmax(x)_j * V_s[j]

The address mapping -- logical block j // BS of a sequence looked up in its
block table, offset j % BS inside the physical block -- is the block table of
page 1, section "2. PagedAttention的革命性设计" (``seq_1: [0, 1, 3]``) and the
logical-to-physical figure of page 3 ("传统静态分配 vs vLLM PagedAttention 显存管理").

Readings where the pages are silent:

* grouped query heads: q head h reads kv head g = h // (Hq / Hkv);
* L_s = 0 gives an all-zero output row;
* the softmax is evaluated with the maximum subtracted (exact in real
  arithmetic; it only keeps exp() finite).

No partitioning, blocking or reordering: one (s, h) at a time, the whole
context at once.
"""

from __future__ import annotations

import numpy as np

from . import codecs


def gather_sequence(cache: np.ndarray, block_table_row, context_len: int,
                    kv_head: int) -> np.ndarray:
    """Rows 0..L-1 of one sequence for one kv head, in logical order.

    ``cache`` is a cache of shape [NB, Hkv, BS, D] (decoded values or raw codes).
    Token j lives in physical block ``block_table_row[j // BS]`` at offset ``j % BS``.
    """
    bs = cache.shape[2]
    rows = []
    for j in range(context_len):
        phys = int(block_table_row[j // bs])
        rows.append(cache[phys, kv_head, j % bs, :])
    if not rows:
        return np.zeros((0, cache.shape[3]), dtype=cache.dtype)
    return np.stack(rows)


def softmax_weighted_sum(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * K q) . V for one query row, in float64, max-subtracted."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    x = scale * (K @ q)
    w = np.exp(x - np.max(x))
    return (w @ V) / np.sum(w)


def paged_decode_f64(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                     block_tables: np.ndarray, context_lens, scale: float,
                     heads=None) -> np.ndarray:
    """Decode attention on already-decoded float64 arrays.

    q: [S, Hq, D]; k_cache, v_cache: [NB, Hkv, BS, D] (scales already applied);
    block_tables: [S, MB] int; context_lens: [S]. ``heads`` optionally restricts
    the work to a list of (s, h) pairs; the other output rows stay zero.
    Returns out: [S, Hq, D] float64.
    """
    S, Hq, D = q.shape
    Hkv = k_cache.shape[1]
    assert Hq % Hkv == 0
    G = Hq // Hkv
    out = np.zeros((S, Hq, D), dtype=np.float64)
    pairs = heads if heads is not None else [(s, h) for s in range(S) for h in range(Hq)]
    for s, h in pairs:
        g = h // G
        L = int(context_lens[s])
        K = gather_sequence(k_cache, block_tables[s], L, g)
        V = gather_sequence(v_cache, block_tables[s], L, g)
        out[s, h] = softmax_weighted_sum(q[s, h].astype(np.float64), K, V, scale)
    return out


def paged_decode(q_codes: np.ndarray, q_dtype: str, k_codes: np.ndarray, v_codes: np.ndarray,
                 kv_dtype: str, k_scale: float, v_scale: float, block_tables: np.ndarray,
                 context_lens, scale: float, heads=None) -> np.ndarray:
    """Decode attention from raw element codes (what the device buffers hold).

    For each (s, h): gathers the sequence's K and V codes of kv head h // G through
    its block table, decodes them with the oracle's own bit-level codecs,
    multiplies by the per-tensor scales (1.0 for 16-bit caches) and evaluates
    :func:`softmax_weighted_sum`. Decoding is elementwise, so gathering first
    gives the same values as decoding the whole cache first.
    """
    q = codecs.decode(q_codes, q_dtype)
    S, Hq, D = q.shape
    Hkv = k_codes.shape[1]
    assert Hq % Hkv == 0
    G = Hq // Hkv
    out = np.zeros((S, Hq, D), dtype=np.float64)
    pairs = heads if heads is not None else [(s, h) for s in range(S) for h in range(Hq)]
    for s, h in pairs:
        g = h // G
        L = int(context_lens[s])
        K = codecs.decode(gather_sequence(k_codes, block_tables[s], L, g), kv_dtype) * float(k_scale)
        V = codecs.decode(gather_sequence(v_codes, block_tables[s], L, g), kv_dtype) * float(v_scale)
        out[s, h] = softmax_weighted_sum(q[s, h], K, V, scale)
    return out


def _nblocks(context_len: int, block_size: int) -> int:
    return -(-context_len // block_size)


def paged_extend(q_codes: np.ndarray, q_dtype: str, k_codes: np.ndarray, v_codes: np.ndarray,
                 kv_dtype: str, k_scale: float, v_scale: float, block_tables: np.ndarray,
                 context_lens, query_start, scale: float, rows=None) -> np.ndarray:
    """Several new tokens per sequence attend causally over the paged context.

    Page 2 (untitled; first section "1. 为什么vLLM能实现24倍推理加速"), section
    "2.1 核心组件交互流程": the execution engine runs prefill, decode and "extend"
    (long-context extension) modes; section "2.2 关键数据结构剖析": the attention
    metadata carries per-sequence query lengths beside the context lengths.

    Reading: sequence s owns query rows query_start[s] .. query_start[s+1]-1 (Q_s of
    them); its context_lens[s] = L_s tokens include the Q_s new ones, whose K/V are
    already in the cache. Query i of s sits at position L_s - Q_s + i and attends to
    tokens 0 .. L_s - Q_s + i (itself and everything before it). With Q_s = 1 this is
    :func:`paged_decode`. ``rows`` optionally restricts the work to (query row, q head)
    pairs. Returns out [T, Hq, D] float64.
    """
    q = codecs.decode(q_codes, q_dtype)
    T, Hq, D = q.shape
    Hkv = k_codes.shape[1]
    G = Hq // Hkv
    out = np.zeros((T, Hq, D), dtype=np.float64)
    owner = {}
    for s in range(len(context_lens)):
        for t in range(int(query_start[s]), int(query_start[s + 1])):
            owner[t] = s
    pairs = rows if rows is not None else [(t, h) for t in range(T) for h in range(Hq)]
    for t, h in pairs:
        s = owner[t]
        L = int(context_lens[s])
        Qs = int(query_start[s + 1]) - int(query_start[s])
        pos = L - Qs + (t - int(query_start[s]))
        g = h // G
        K = codecs.decode(gather_sequence(k_codes, block_tables[s], pos + 1, g), kv_dtype) * float(k_scale)
        V = codecs.decode(gather_sequence(v_codes, block_tables[s], pos + 1, g), kv_dtype) * float(v_scale)
        out[t, h] = softmax_weighted_sum(q[t, h], K, V, scale)
    return out
