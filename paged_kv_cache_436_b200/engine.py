"""One decode step of the paged-KV-cache path, end to end, on one GPU.

A step appends one token to every sequence of the batch and decodes:

1. host bookkeeping (C++ ``pa_batch_append``): the slot of each new token, a
   new block when a sequence crosses a block boundary, a copy-on-write pair when
   it appends into a shared block (page 3 «内存优化：KV Cache管理、PagedAttention原理与
   内存池配置», section "PagedAttention原理");
2. one host->device copy of the step's metadata from a pinned buffer (page 2,
   untitled, first section "1. 为什么vLLM能实现24倍推理加速", section "2.2 关键数据结构
   剖析": block tables and context lengths travel with the attention metadata);
3. ``pa_block_table_update``, ``pa_copy_blocks``, ``pa_reshape_and_cache``,
   ``pa_decode``.

All of it runs in one native call (``pa_engine_step``); this class owns the
buffers the native engine borrows and the set-up helpers.
"""

from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import (EngineConfig, KVCache, Pool, _check, _dev, _stream, decode, decode_workspace_size, dtype_code, lib)

_TORCH = {"f16": torch.float16, "bf16": torch.bfloat16}


class DecodeEngine:
    def __init__(self, *, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, kv_dtype,
                 q_dtype, num_blocks, initial_order, max_blocks_per_seq, max_context_len, scale=None,
                 k_scale=1.0, v_scale=1.0, device="cuda", k_cache=None, v_cache=None):
        self.S, self.Hq, self.Hkv, self.D = num_seqs, num_q_heads, num_kv_heads, head_dim
        self.BS, self.kv_dtype, self.q_dtype = block_size, kv_dtype, q_dtype
        self.MB = max_blocks_per_seq
        self.scale = float(scale) if scale is not None else 1.0 / float(np.sqrt(head_dim))
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
        self.meta_bytes = int(lib().pa_engine_meta_bytes(num_seqs))
        self._meta_host = [torch.empty(self.meta_bytes, dtype=torch.uint8).pin_memory() for _ in range(2)]
        self._meta_dev = torch.empty(self.meta_bytes, dtype=torch.uint8, device=self.device)
        self._native = None
        self._native_key = None
        self._stage = [(torch.empty((num_seqs, max_blocks_per_seq), dtype=torch.int32).pin_memory(),
                        torch.empty(num_seqs, dtype=torch.int32).pin_memory()) for _ in range(2)]
        self._stage_event = [None, None]
        self._stage_flip = 0

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

    def reorder(self, parents, stream=None):
        """Beam re-selection: sequence i continues old sequence parents[i] (host
        bookkeeping in C++), then the device mirror of the tables and lengths is
        refreshed from a pinned staging buffer (double-buffered, asynchronous)."""
        self.pool.batch_reorder(self.bt_host, self.lens, self.BS, parents)
        i = self._stage_flip
        self._stage_flip ^= 1
        if self._stage_event[i] is not None:
            self._stage_event[i].synchronize()      # the copy that last read this buffer is done
        bt_h, lens_h = self._stage[i]
        bt_h.numpy()[:] = self.bt_host
        lens_h.numpy()[:] = self.lens
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        with torch.cuda.stream(s):
            self.bt_dev.copy_(bt_h, non_blocking=True)
            self.lens_dev.copy_(lens_h, non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(s)
        self._stage_event[i] = ev

    def upload_tables(self):
        """Copy the whole host block table and lengths to the device (set-up only)."""
        self.bt_dev.copy_(torch.from_numpy(self.bt_host))
        self.lens_dev.copy_(torch.from_numpy(self.lens))

    # ------------------------------------------------------------------ step
    def _engine(self):
        d = self.cache.desc
        key = (self.scale, d.k_scale, d.v_scale)
        if self._native is not None and self._native_key == key:
            return self._native
        self.close()
        cfg = EngineConfig()
        cfg.pool = self.pool._h
        cfg.num_seqs, cfg.num_q_heads, cfg.max_blocks_per_seq = self.S, self.Hq, self.MB
        cfg.max_context_len, cfg.q_dtype, cfg.scale = self.max_context_len, dtype_code(
            torch.empty(0, dtype=_TORCH[self.q_dtype])), self.scale
        cfg.cache = d
        cfg.block_tables_host = self.bt_host.ctypes.data
        cfg.context_lens_host = self.lens.ctypes.data
        cfg.block_tables_dev = self.bt_dev.data_ptr()
        cfg.meta_host[0], cfg.meta_host[1] = self._meta_host[0].data_ptr(), self._meta_host[1].data_ptr()
        cfg.meta_dev, cfg.meta_bytes = self._meta_dev.data_ptr(), self.meta_bytes
        cfg.workspace, cfg.workspace_bytes = self.ws.data_ptr(), self.ws.numel()
        h = ctypes.c_void_p()
        _check(lib().pa_engine_create(ctypes.byref(cfg), ctypes.byref(h)), "pa_engine_create")
        self._native, self._native_key = h, key
        return h

    def close(self):
        if self._native is not None:
            lib().pa_engine_destroy(self._native)
            self._native = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def step(self, q, k_new, v_new, out, scale=None, stream=None, events=None):
        """One full decode step (native): bookkeeping, metadata upload, table patch,
        copy-on-write copies, cache write of k_new / v_new, decode into out.
        `events` = (begin, end) torch.cuda.Events recorded around the partition kernel
        (they must exist already: torch creates an event at its first record)."""
        if scale is not None and float(scale) != self.scale:
            raise ValueError("the softmax scale is fixed when the engine is created")
        qt = _TORCH[self.q_dtype]
        for name, t, shape in (("q", q, (self.S, self.Hq, self.D)), ("k_new", k_new, (self.S, self.Hkv, self.D)),
                               ("v_new", v_new, (self.S, self.Hkv, self.D)), ("out", out, (self.S, self.Hq, self.D))):
            _dev(t, name, qt, 3)
            if tuple(t.shape) != shape:
                raise ValueError(f"{name} shape {tuple(t.shape)} is not {list(shape)}")
        h = self._engine()
        e0 = ctypes.c_void_p(events[0].cuda_event) if events else None
        e1 = ctypes.c_void_p(events[1].cuda_event) if events else None
        st = lib().pa_engine_step(h, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k_new.data_ptr()),
                                  ctypes.c_void_p(v_new.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                  _stream(stream), e0, e1)
        _check(st, "pa_engine_step")
        return out

    def last_step(self):
        """(copy pairs, table updates, kernel launches) of the last step."""
        a, b, c = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib().pa_engine_last_step(self._native, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
               "pa_engine_last_step")
        return a.value, b.value, c.value

    def run_decode(self, q, out, scale=None, stream=None, stage=None):
        """pa_decode alone over the current device tables and `lens_dev`."""
        decode(q, self.cache, self.bt_dev, self.lens_dev, self.max_context_len,
               self.scale if scale is None else scale, out, self.ws, stream, stage=stage)


class HostPipeline:
    """Decode steps whose inputs and outputs live in pinned host memory.

    Each step copies its q and new K/V rows host->device and its output
    device->host, every step. The copies run on their own streams (one per
    direction) into double-buffered device tensors, ordered by events, so the
    copies of step i+1 / i-1 overlap the kernels of step i. The caller must not
    modify a step's host inputs, or read its host output, before ``sync()``.
    """

    def __init__(self, engine: DecodeEngine, scale=None):
        self.eng = engine
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
        # the previous step's attention kernel has started: its small metadata copy is done,
        # so the next inputs' large copy cannot delay it on the copy engine
        self.started = None
        self._ev = [(torch.cuda.Event(), torch.cuda.Event()) for _ in range(2)]
        for a, b in self._ev:            # torch creates the CUDA events at their first record
            a.record(self.compute)
            b.record(self.compute)
        self.n = 0

    def submit(self, hq, hk, hv, hout):
        b = self.n & 1
        self.n += 1
        with torch.cuda.stream(self.h2d):
            if self.free_in[b] is not None:
                self.h2d.wait_event(self.free_in[b])
            if self.started is not None:
                self.h2d.wait_event(self.started)
            self.dq[b].copy_(hq, non_blocking=True)
            self.dk[b].copy_(hk, non_blocking=True)
            self.dv[b].copy_(hv, non_blocking=True)
            landed = torch.cuda.Event()
            landed.record(self.h2d)
        self.compute.wait_event(landed)
        if self.free_out[b] is not None:
            self.compute.wait_event(self.free_out[b])
        ev = self._ev[b]
        self.eng.step(self.dq[b], self.dk[b], self.dv[b], self.dout[b], stream=self.compute, events=ev)
        self.started = ev[0]
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
