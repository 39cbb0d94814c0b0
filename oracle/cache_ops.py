"""KV-cache slot write and block copy as plain array operations (oracle; test infrastructure only).

* ``reshape_and_cache``: token t's K and V rows ([Hkv, D]) go to slot
  ``slot_mapping[t]``, i.e. physical block ``slot // BS`` at offset ``slot % BS``
  of a cache laid out [NB, Hkv, BS, D]. The slot of logical position j of a
  sequence is ``block_table[j // BS] * BS + j % BS`` (page 1, section
  "2. PagedAttention的革命性设计": the block table maps logical to physical
  blocks; page 3, section "PagedAttention原理": blocks of 16 or 32 tokens).
  Readings: a negative slot is padding and writes nothing; for 16-bit caches
  the element codes are copied bit for bit; for an E4M3 cache each value is
  divided by the tensor's scale in binary32 and rounded to E4M3 by
  round-to-nearest-even with saturation (page 2, section "4.2 混合精度策略",
  "KV缓存 FP8").
* ``copy_blocks``: for every (src, dst) pair the whole physical block -- all kv
  heads, all slots -- of K and of V is copied, bit for bit. This is the copy
  that copy-on-write of a shared block needs (page 3, section
  "PagedAttention原理": several requests share physical blocks by reference
  count; page 1, section "5. 高级应用场景": parallel sampling and beam search).
  Reading: all pairs read the cache as it was before the call.
"""

from __future__ import annotations

import numpy as np

from . import codecs


def encode_for_cache(values_codes: np.ndarray, in_dtype: str, kv_dtype: str, scale: float) -> np.ndarray:
    """Codes to store for input codes of ``in_dtype`` in a cache of ``kv_dtype``."""
    if kv_dtype in ("f16", "bf16"):
        assert in_dtype == kv_dtype, "16-bit caches store the input codes unchanged"
        return np.asarray(values_codes).copy()
    x32 = codecs.decode(values_codes, in_dtype).astype(np.float32)   # exact: 16-bit floats embed in binary32
    return codecs.encode_e4m3(codecs.f32_div(x32, scale))


def reshape_and_cache(k_codes: np.ndarray, v_codes: np.ndarray, in_dtype: str,
                      slot_mapping, k_cache: np.ndarray, v_cache: np.ndarray,
                      kv_dtype: str, k_scale: float = 1.0, v_scale: float = 1.0):
    """Return new (k_cache, v_cache) code arrays with tokens written to their slots.

    k_codes, v_codes: [T, Hkv, D] input codes; caches: [NB, Hkv, BS, D] codes.
    """
    kc = k_cache.copy()
    vc = v_cache.copy()
    bs = kc.shape[2]
    for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        blk, off = slot // bs, slot % bs
        kc[blk, :, off, :] = encode_for_cache(k_codes[t], in_dtype, kv_dtype, k_scale)
        vc[blk, :, off, :] = encode_for_cache(v_codes[t], in_dtype, kv_dtype, v_scale)
    return kc, vc


def copy_blocks(k_cache: np.ndarray, v_cache: np.ndarray, pairs):
    """Return new (k_cache, v_cache) with block dst := block src for each pair."""
    kc = k_cache.copy()
    vc = v_cache.copy()
    for src, dst in np.asarray(pairs).reshape(-1, 2).tolist():
        kc[dst] = k_cache[src]
        vc[dst] = v_cache[src]
    return kc, vc
