"""One decode step of the paged-KV-cache path, end to end, on one GPU.

A step, for a batch of S sequences that each append one token:

1. host bookkeeping (C++ ``pa_batch_append``): the slot of each new token, a
   new block when a sequence crosses a block boundary, a copy-on-write pair when
   it appends into a shared block (page 3 «内存优化：KV Cache管理、PagedAttention原理与
   内存池配置», section "PagedAttention原理");
2. one host->device copy of the step's metadata (slots, copy pairs, block-table
   updates) from a pinned buffer; the block-table mirror is patched on the device
   (``pa_block_table_update``) -- page 2 (untitled, first section "1. 为什么vLLM能
   实现24倍推理加速"), section "2.2 关键数据结构剖析": block tables and context lengths
   travel with the attention metadata;
3. ``pa_copy_blocks`` for the copy-on-write pairs;
4. ``pa_reshape_and_cache`` of the new tokens' K and V;
5. ``pa_decode``.

Every computation happens in libpa; this class only owns buffers and orders calls.
"""

from __future__ import annotations

import numpy as np
import torch

from . import (KVCache, Pool, block_table_update, copy_blocks, decode, decode_workspace_size,
               reshape_and_cache)

_TORCH = {"f16": torch.float16, "bf16": torch.bfloat16}


class DecodeEngine:
    def __init__(self, *, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, kv_dtype,
                 q_dtype, num_blocks, initial_order, max_blocks_per_seq, max_context_len,
                 k_scale=1.0, v_scale=1.0, device="cuda", k_cache=None, v_cache=None):
        self.S, self.Hq, self.Hkv, self.D = num_seqs, num_q_heads, num_kv_heads, head_dim
        self.BS, self.kv_dtype, self.q_dtype = block_size, kv_dtype, q_dtype
        self.MB = max_blocks_per_seq
        self.device = torch.device(device)
        self.pool = Pool(num_blocks, initial_order)
        cache_t = torch.uint8 if kv_dtype == "e4m3" else _TORCH[kv_dtype]
        shape = (num_blocks, num_kv_heads, block_size, head_dim)
        self.k_cache = k_cache if k_cache is not None else torch.empty(shape, dtype=cache_t, device=self.device)
        self.v_cache = v_cache if v_cache is not None else torch.empty(shape, dtype=cache_t, device=self.device)
        self.cache = KVCache(self.k_cache, self.v_cache, kv_dtype, k_scale, v_scale)
        self.bt_host = np.zeros((num_seqs, max_blocks_per_seq), dtype=np.int32)
        self.lens = np.zeros(num_seqs, dtype=np.int32)          # tokens each sequence holds
        self.bt_dev = torch.zeros((num_seqs, max_blocks_per_seq), dtype=torch.int32, device=self.device)
        self.lens_dev = torch.zeros(num_seqs, dtype=torch.int32, device=self.device)
        self.max_context_len = int(max_context_len)
        self.ws = torch.empty(decode_workspace_size(num_seqs, num_q_heads, head_dim, self.max_context_len),
                              dtype=torch.uint8, device=self.device)
        # packed per-step metadata: slots (int64 S) | cow pairs (int64 2S) | lens (int32 S) | updates (int32 3S)
        self._off_cow = 8 * num_seqs
        self._off_lens = self._off_cow + 16 * num_seqs
        self._off_upd = self._off_lens + 4 * num_seqs
        self._meta_bytes = self._off_upd + 12 * num_seqs
        self._meta_host = [torch.empty(self._meta_bytes, dtype=torch.uint8).pin_memory() for _ in range(2)]
        self._meta_event = [None, None]
        self._meta_dev = torch.empty(self._meta_bytes, dtype=torch.uint8, device=self.device)
        self._flip = 0
        self.last_num_cow = 0
        self.last_num_updates = 0

    # ------------------------------------------------------------------ set-up
    def extend(self, s: int, n_tokens: int, slots: np.ndarray | None = None):
        """Host bookkeeping for n_tokens more tokens of sequence s (e.g. a prompt)."""
        row = self.bt_host[s]
        cs, cd = self.pool.seq_extend(row, int(self.lens[s]), n_tokens, self.BS, slots)
        self.lens[s] += n_tokens
        return cs, cd

    def fork(self, parent: int, child: int):
        """Sequence `child` shares every block of `parent` (prefix sharing / beams)."""
        nb = -(-int(self.lens[parent]) // self.BS)
        self.pool.seq_fork(self.bt_host[parent], nb)
        self.bt_host[child] = self.bt_host[parent]
        self.lens[child] = self.lens[parent]

    def upload_tables(self):
        """Copy the whole host block table and lengths to the device (set-up only)."""
        self.bt_dev.copy_(torch.from_numpy(self.bt_host))
        self.lens_dev.copy_(torch.from_numpy(self.lens))

    # ------------------------------------------------------------------ step
    def bookkeeping(self, stream=None):
        """Step parts 1-2: host bookkeeping for one token per sequence and the
        metadata upload. Returns device views (slots, cow_pairs, updates)."""
        i = self._flip
        self._flip ^= 1
        if self._meta_event[i] is not None:
            self._meta_event[i].synchronize()      # the copy that last read this buffer is done
        host = self._meta_host[i]
        S = self.S
        slots = host[:self._off_cow].view(torch.int64).numpy()
        cows = host[self._off_cow:self._off_lens].view(torch.int64).numpy().reshape(S, 2)
        lens = host[self._off_lens:self._off_upd].view(torch.int32).numpy()
        upd = host[self._off_upd:].view(torch.int32).numpy().reshape(S, 3)
        positions = self.lens.copy()
        ncow, nupd = self.pool.batch_append(self.bt_host, positions, self.BS, slots, cows, upd)
        self.lens += 1
        lens[:] = self.lens
        self.last_num_cow, self.last_num_updates = ncow, nupd
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        with torch.cuda.stream(s):
            self._meta_dev.copy_(host, non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(s)
        self._meta_event[i] = ev
        d = self._meta_dev
        return (d[:self._off_cow].view(torch.int64),
                d[self._off_cow:self._off_lens].view(torch.int64).view(S, 2)[:ncow],
                d[self._off_lens:self._off_upd].view(torch.int32),
                d[self._off_upd:].view(torch.int32).view(S, 3)[:nupd])

    def step(self, q, k_new, v_new, out, scale: float, stream=None):
        """One full decode step: bookkeeping, table patch, CoW copies, cache write, decode."""
        slots, cows, lens, upd = self.bookkeeping(stream)
        if upd.shape[0]:
            block_table_update(upd, self.bt_dev, stream)
        if cows.shape[0]:
            copy_blocks(cows, self.cache, stream)
        reshape_and_cache(k_new, v_new, slots, self.cache, stream)
        self.lens_dev = lens
        decode(q, self.cache, self.bt_dev, lens, self.max_context_len, scale, out, self.ws, stream)
        return out

    def run_decode(self, q, out, scale: float, stream=None, stage=None):
        """pa_decode alone over the current device tables and lengths."""
        decode(q, self.cache, self.bt_dev, self.lens_dev, self.max_context_len, scale, out, self.ws,
               stream, stage=stage)


class HostPipeline:
    """Decode steps whose inputs and outputs live in pinned host memory.

    Each step copies its q and new K/V rows host->device and its output
    device->host, every step. The copies run on their own streams (one per
    direction) into double-buffered device tensors, ordered by events, so the
    copies of step i+1 / i-1 overlap the kernels of step i. The caller must not
    modify a step's host inputs, or read its host output, before ``sync()``.
    """

    def __init__(self, engine: DecodeEngine, scale: float):
        self.eng, self.scale = engine, scale
        dev = engine.device
        S, Hq, Hkv, D = engine.S, engine.Hq, engine.Hkv, engine.D
        qt = _TORCH[engine.q_dtype]
        self.dq = [torch.empty((S, Hq, D), dtype=qt, device=dev) for _ in range(2)]
        self.dk = [torch.empty((S, Hkv, D), dtype=qt, device=dev) for _ in range(2)]
        self.dv = [torch.empty((S, Hkv, D), dtype=qt, device=dev) for _ in range(2)]
        self.dout = [torch.empty((S, Hq, D), dtype=qt, device=dev) for _ in range(2)]
        self.compute = torch.cuda.current_stream(dev)
        self.h2d = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)
        self.free_in = [None, None]     # step that last read buffer b has finished
        self.free_out = [None, None]    # the output copy that last read dout[b] has finished
        self.n = 0

    def submit(self, hq, hk, hv, hout):
        b = self.n & 1
        self.n += 1
        with torch.cuda.stream(self.h2d):
            if self.free_in[b] is not None:
                self.h2d.wait_event(self.free_in[b])
            self.dq[b].copy_(hq, non_blocking=True)
            self.dk[b].copy_(hk, non_blocking=True)
            self.dv[b].copy_(hv, non_blocking=True)
            landed = torch.cuda.Event()
            landed.record(self.h2d)
        self.compute.wait_event(landed)
        if self.free_out[b] is not None:
            self.compute.wait_event(self.free_out[b])
        self.eng.step(self.dq[b], self.dk[b], self.dv[b], self.dout[b], self.scale, stream=self.compute)
        done = torch.cuda.Event()
        done.record(self.compute)
        self.free_in[b] = done
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(done)
            hout.copy_(self.dout[b], non_blocking=True)
            copied = torch.cuda.Event()
            copied.record(self.d2h)
        self.free_out[b] = copied
        return copied

    def sync(self):
        self.d2h.synchronize()
        self.compute.synchronize()
