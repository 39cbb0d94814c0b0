"""KV-cache byte accounting (oracle; test infrastructure only).

* ``kv_cache_bytes``: the closed form of page 3, section "核心原理" ("关键参数速览"):
  2 (K and V) x layers x heads x head_dim x seq_len x batch x bytes per element;
  the page's example is a 7B model, 32 layers x 32 heads x 128, fp16, 1024
  tokens -> 536,870,912 bytes ("约 536MB").
* ``paged_cache_bytes``: the same quantity counted the way a paged cache holds
  it -- whole blocks of [Hkv, BS, D] for K and for V.
* ``static_reservation``: the figure of page 3 ("传统静态分配 vs vLLM PagedAttention
  显存管理"): a static allocator reserves max_seq_len tokens per request.
* ``decode_bytes``: the bytes one decode step must move at minimum -- every
  context token's K and V row once per kv head, q in, out back, the block-table
  entries the step reads and the context lengths.
"""

from __future__ import annotations


def kv_cache_bytes(num_layers, num_heads, head_dim, seq_len, batch, dtype_bytes) -> int:
    return 2 * num_layers * num_heads * head_dim * seq_len * batch * dtype_bytes


def paged_cache_bytes(num_blocks, num_kv_heads, block_size, head_dim, dtype_bytes, num_layers=1) -> int:
    return 2 * num_layers * num_blocks * num_kv_heads * block_size * head_dim * dtype_bytes


def static_reservation(used_tokens, max_seq_len):
    """(reserved, used, wasted) tokens when every request reserves max_seq_len."""
    reserved = max_seq_len * len(used_tokens)
    used = sum(used_tokens)
    return reserved, used, reserved - used


def paged_waste(used_tokens, block_size):
    """Unused slots per sequence when each holds ceil(L / BS) blocks."""
    return [-(-L // block_size) * block_size - L for L in used_tokens]


def decode_bytes(context_lens, num_kv_heads, num_q_heads, head_dim, kv_bytes, q_bytes, block_size) -> int:
    kv = sum(2 * int(L) * num_kv_heads * head_dim * kv_bytes for L in context_lens)
    S = len(context_lens)
    q = S * num_q_heads * head_dim * q_bytes
    out = S * num_q_heads * head_dim * q_bytes
    tables = sum(4 * (-(-int(L) // block_size)) for L in context_lens)
    lens = 4 * S
    return kv + q + out + tables + lens
