"""Python binding of libpa: paged KV-cache attention for B200 (sm_100a).

Argument marshalling only. Every step of the path -- the block bookkeeping, the
KV-cache write, the block copy, decode attention, multi-query (extend / prefill)
attention, the prefix-cache index and beam re-selection -- runs inside libpa (C++
on the host, CUDA kernels on the device). Host buffers are checked for element type,
contiguity and the extent the C header states before their pointers are passed. PyTorch provides device memory and
streams; this module passes ``tensor.data_ptr()`` and the current stream.

There is no fallback: if ``lib/libpa.so`` is missing or cannot be loaded every
call raises :class:`LibraryMissing`.
"""

from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libpa.so")

PA_OK, PA_ERR_ARG, PA_ERR_OOM, PA_ERR_STATE, PA_ERR_CUDA, PA_ERR_DEVICE_CHECK = 0, -1, -2, -3, -4, -5
PA_F16, PA_BF16, PA_E4M3 = 0, 1, 2
DTYPES = {"f16": PA_F16, "bf16": PA_BF16, "e4m3": PA_E4M3}
DEVICE_ERRORS = {0: "ok", 1: "bad block id", 2: "bad context length", 3: "bad slot",
                 4: "bad copy pair", 5: "bad table update", 6: "wait timeout"}
STATUS = {PA_OK: "ok", PA_ERR_ARG: "invalid argument", PA_ERR_OOM: "out of blocks",
          PA_ERR_STATE: "refcount state", PA_ERR_CUDA: "CUDA error", PA_ERR_DEVICE_CHECK: "device check"}


class LibraryMissing(RuntimeError):
    pass


class PaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)} ({status})")
        self.status = status


class CacheDesc(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("kv_dtype", ctypes.c_int32), ("k_scale", ctypes.c_float),
                ("v_scale", ctypes.c_float), ("k_cache", ctypes.c_void_p),
                ("v_cache", ctypes.c_void_p)]


class EngineConfig(ctypes.Structure):
    _fields_ = [("pool", ctypes.c_void_p), ("num_seqs", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("max_blocks_per_seq", ctypes.c_int32), ("max_context_len", ctypes.c_int32),
                ("q_dtype", ctypes.c_int32), ("scale", ctypes.c_float), ("cache", CacheDesc),
                ("block_tables_host", ctypes.c_void_p), ("context_lens_host", ctypes.c_void_p),
                ("block_tables_dev", ctypes.c_void_p), ("meta_host", ctypes.c_void_p * 2),
                ("meta_dev", ctypes.c_void_p), ("meta_bytes", ctypes.c_size_t),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t)]


_lib = None

_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_PI32 = ctypes.POINTER(ctypes.c_int32)
_PI64 = ctypes.POINTER(ctypes.c_int64)
_PDESC = ctypes.POINTER(CacheDesc)

_SIGNATURES = {
    "pa_reshape_and_cache": (_I32, [_P, _P, _I32, _I32, _I64, _I64, _P, _PDESC, _P]),
    "pa_copy_blocks": (_I32, [_P, _I32, _PDESC, _P]),
    "pa_decode": (_I32, [_P, _I32, _I32, _I32, _PDESC, _P, _I32, _P, _I32, ctypes.c_float, _P, _P,
                         ctypes.c_size_t, _P]),
    "pa_decode_stage": (_I32, [_I32, _P, _I32, _I32, _I32, _PDESC, _P, _I32, _P, _I32, ctypes.c_float,
                               _P, _P, ctypes.c_size_t, _P]),
    "pa_decode_workspace_size": (ctypes.c_size_t, [_I32, _I32, _I32, _I32]),
    "pa_decode_no_alloc": (_I32, [_P, _I32, _I32, _I32, _PDESC, _P, _I32, _P, _I32, ctypes.c_float, _P, _P]),
    "pa_last_device_error": (_I32, [_P, _PI32, _PI32]),
    "pa_block_table_update": (_I32, [_P, _I32, _P, _I32, _I32, _P]),
    "pa_pool_create": (_I32, [_I32, _PI32, ctypes.POINTER(_P)]),
    "pa_pool_destroy": (None, [_P]),
    "pa_pool_alloc": (_I32, [_P, _PI32]),
    "pa_pool_incref": (_I32, [_P, _I32]),
    "pa_pool_decref": (_I32, [_P, _I32]),
    "pa_pool_refcount": (_I32, [_P, _I32]),
    "pa_pool_num_free": (_I32, [_P]),
    "pa_pool_num_blocks": (_I32, [_P]),
    "pa_pool_free_list": (_I32, [_P, _PI32, _I32]),
    "pa_seq_append": (_I32, [_P, _PI32, _I32, _I32, _I32, _PI64, _PI32, _PI32]),
    "pa_seq_extend": (_I32, [_P, _PI32, _I32, _I32, _I32, _I32, _PI64, _PI32, _PI32, _PI32]),
    "pa_seq_fork": (_I32, [_P, _PI32, _I32]),
    "pa_seq_free": (_I32, [_P, _PI32, _I32]),
    "pa_batch_append": (_I32, [_P, _PI32, _I32, _I32, _PI32, _I32, _PI64, _PI64, _PI32, _PI32, _PI32,
                               _PI32]),
    "pa_engine_meta_bytes": (ctypes.c_size_t, [_I32]),
    "pa_engine_create": (_I32, [ctypes.POINTER(EngineConfig), ctypes.POINTER(_P)]),
    "pa_engine_destroy": (None, [_P]),
    "pa_engine_step": (_I32, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "pa_engine_last_step": (_I32, [_P, _PI32, _PI32, _PI32]),
    "pa_prefix_cache_create": (_I32, [_I32, ctypes.POINTER(_P)]),
    "pa_prefix_cache_destroy": (None, [_P]),
    "pa_prefix_cache_size": (_I32, [_P]),
    "pa_prefix_cache_match": (_I32, [_P, _P, _PI32, _I32, _PI32, _I32, _PI32]),
    "pa_prefix_cache_insert": (_I32, [_P, _P, _PI32, _I32, _PI32, _PI32]),
    "pa_prefix_cache_evict": (_I32, [_P, _P, _I32, _PI32]),
    "pa_prefix_cache_clear": (_I32, [_P, _P, _PI32]),
    "pa_batch_reorder": (_I32, [_P, _PI32, _PI32, _I32, _I32, _I32, _PI32]),
    "pa_extend": (_I32, [_P, _I32, _I32, _I32, _P, _I32, _PDESC, _P, _I32, _P, _I32, ctypes.c_float, _P, _P,
                         ctypes.c_size_t, _P]),
    "pa_extend_workspace_size": (ctypes.c_size_t, [_I32, _I32, _I32, _I32, _I32]),
    "pa_selftest_wait_timeout": (_I32, [ctypes.c_uint32, _P]),
    "pa_prefill": (_I32, [_P, _P, _P, _I32, _I32, _I32, _P, _I32, _PDESC, _P, _I32, _P, _I32, ctypes.c_float, _P,
                          _P, ctypes.c_size_t, _P]),
    "pa_version": (ctypes.c_char_p, []),
}


def lib():
    """The loaded libpa (raises LibraryMissing when it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise LibraryMissing(f"{LIB_PATH} not built: run `python -m paged_kv_cache_436_b200.build`")
        try:
            L = ctypes.CDLL(LIB_PATH)
        except OSError as e:
            raise LibraryMissing(f"cannot load {LIB_PATH}: {e}") from e
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != PA_OK:
        raise PaError(status, what)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _host_ptr(a, bits: int, min_size: int, ptr_type):
    """Pointer to a contiguous host buffer of `bits`-bit integers (numpy array or CPU
    tensor) with at least `min_size` elements. The native calls trust the extent the
    header states, so any other buffer is refused here."""
    if hasattr(a, "ctypes"):                                   # numpy
        import numpy as np
        if a.dtype != np.dtype(f"int{bits}") or not a.flags.c_contiguous:
            raise TypeError(f"expected a C-contiguous int{bits} array, got {a.dtype} "
                            f"(contiguous={a.flags.c_contiguous})")
        n, p = a.size, a.ctypes.data_as(ptr_type)
    else:                                                      # torch
        import torch
        want = torch.int32 if bits == 32 else torch.int64
        if a.dtype != want or a.device.type != "cpu" or not a.is_contiguous():
            raise TypeError(f"expected a contiguous host {want} tensor, got {a.dtype} on {a.device}")
        n, p = a.numel(), ctypes.cast(a.data_ptr(), ptr_type)
    if n < min_size:
        raise ValueError(f"host buffer of {n} elements, {min_size} needed")
    return p


def _i32p(a, min_size: int = 0):
    """Pointer into a contiguous host int32 buffer (numpy array or CPU tensor)."""
    return _host_ptr(a, 32, min_size, _PI32)


def _i64p(a, min_size: int = 0):
    """Pointer into a contiguous host int64 buffer (numpy array or CPU tensor)."""
    return _host_ptr(a, 64, min_size, _PI64)


# ---------------------------------------------------------------------------
# device ops
# ---------------------------------------------------------------------------

def _dev(t, what: str, dtype=None, ndim=None, min_numel=0, contiguous=True):
    """Refuse, before its pointer reaches a kernel, a tensor that is not on a CUDA device
    or does not have the element type, rank, layout or size the header states (a host
    pointer or a short buffer would be read out of bounds on the device)."""
    if t is None or not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{what}: dtype {t.dtype}, expected {dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{what}: {t.dim()}-D, expected {ndim}-D")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if t.numel() < min_numel:
        raise ValueError(f"{what}: {t.numel()} elements, at least {min_numel} needed")


def _qk_types():
    import torch
    return (torch.float16, torch.bfloat16)


def _check_cache(cache: "KVCache"):
    _dev(cache.k_cache, "k_cache")
    _dev(cache.v_cache, "v_cache")


def _check_attention(q, out, cache: "KVCache", block_tables, context_lens, num_seqs: int):
    """q / out [rows, Hq, D] of one 16-bit type with D the cache's head_dim; int32 block
    tables with a row per sequence and an int32 length per sequence."""
    import torch
    _dev(q, "q", _qk_types(), 3)
    if q.shape[2] != cache.desc.head_dim:
        raise ValueError(f"q head_dim {q.shape[2]} != cache head_dim {cache.desc.head_dim}")
    _dev(out, "out", q.dtype, 3)
    if out.shape != q.shape:
        raise ValueError(f"out shape {tuple(out.shape)} != q shape {tuple(q.shape)}")
    _check_cache(cache)
    _dev(block_tables, "block_tables", torch.int32, 2)
    if block_tables.shape[0] < num_seqs:
        raise ValueError(f"block_tables has {block_tables.shape[0]} rows for {num_seqs} sequences")
    _dev(context_lens, "context_lens", torch.int32, None, num_seqs)

def dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float16:
        return PA_F16
    if t.dtype == torch.bfloat16:
        return PA_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return PA_E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


class KVCache:
    """K and V caches [num_blocks, num_kv_heads, block_size, head_dim] plus their scales."""

    def __init__(self, k_cache, v_cache, kv_dtype: str, k_scale: float = 1.0, v_scale: float = 1.0):
        if kv_dtype not in DTYPES:
            raise ValueError(f"kv_dtype must be one of {sorted(DTYPES)}, got {kv_dtype!r}")
        if k_cache.shape != v_cache.shape or k_cache.dim() != 4:
            raise ValueError(f"K and V caches must share one 4-D shape, got {tuple(k_cache.shape)} "
                             f"and {tuple(v_cache.shape)}")
        if not (k_cache.is_contiguous() and v_cache.is_contiguous()):
            raise ValueError("K and V caches must be contiguous")
        if dtype_code(k_cache) != DTYPES[kv_dtype] or dtype_code(v_cache) != DTYPES[kv_dtype]:
            raise TypeError(f"cache tensors of {k_cache.dtype} / {v_cache.dtype} do not hold {kv_dtype}")
        self.k_cache, self.v_cache = k_cache, v_cache
        self.kv_dtype = kv_dtype
        nb, hkv, bs, d = k_cache.shape
        self.desc = CacheDesc(nb, hkv, bs, d, DTYPES[kv_dtype], float(k_scale), float(v_scale),
                              k_cache.data_ptr(), v_cache.data_ptr())

    @property
    def num_blocks(self):
        return self.desc.num_blocks

    @property
    def block_size(self):
        return self.desc.block_size


def reshape_and_cache(k, v, slot_mapping, cache: KVCache, stream=None) -> None:
    """Write each token's K/V rows ([T, Hkv, D], fp16/bf16) into its slot (int64 [T])."""
    import torch
    T = k.shape[0]
    for name, x in (("k", k), ("v", v)):
        _dev(x, name, _qk_types(), 3, contiguous=False)
        if tuple(x.shape[1:]) != (cache.desc.num_kv_heads, cache.desc.head_dim) or x.shape[0] != T:
            raise ValueError(f"{name} shape {tuple(x.shape)} is not [{T}, {cache.desc.num_kv_heads}, "
                             f"{cache.desc.head_dim}]")
        if x.stride(2) != 1 or x.stride(1) != cache.desc.head_dim:
            raise ValueError(f"{name}: heads and dims must be contiguous inside a token")
    if v.dtype != k.dtype:
        raise TypeError("k and v differ in dtype")
    _check_cache(cache)
    _dev(slot_mapping, "slot_mapping", torch.int64, None, T)
    st = lib().pa_reshape_and_cache(_ptr(k), _ptr(v), dtype_code(k), T, k.stride(0), v.stride(0),
                                    _ptr(slot_mapping), ctypes.byref(cache.desc), _stream(stream))
    _check(st, "pa_reshape_and_cache")


def copy_blocks(pairs, cache: KVCache, stream=None) -> None:
    """Copy whole blocks src -> dst for each row of the device int64 [n, 2] ``pairs``."""
    import torch
    n = 0 if pairs is None else pairs.shape[0]
    if n:
        _dev(pairs, "pairs", torch.int64, 2)
        if pairs.shape[1] != 2:
            raise ValueError(f"pairs shape {tuple(pairs.shape)} is not [n, 2]")
        _check_cache(cache)
    st = lib().pa_copy_blocks(_ptr(pairs), n, ctypes.byref(cache.desc), _stream(stream))
    _check(st, "pa_copy_blocks")


def decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len) -> int:
    return int(lib().pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len))


def decode(q, cache: KVCache, block_tables, context_lens, max_context_len: int, scale: float, out,
           workspace, stream=None, stage=None) -> None:
    """Paged decode attention: out[s, h] = softmax(scale q K^T) V over each context.

    q, out: [S, Hq, D] fp16/bf16; block_tables int32 [S, MB]; context_lens int32 [S];
    workspace: uint8 device buffer of at least decode_workspace_size(...) bytes.
    ``stage`` (0, 1 or 2) runs one of the three launches alone.
    """
    S, Hq, _ = q.shape
    _check_attention(q, out, cache, block_tables, context_lens, S)
    _dev(workspace, "workspace")
    args = (_ptr(q), dtype_code(q), S, Hq, ctypes.byref(cache.desc), _ptr(block_tables),
            block_tables.shape[1], _ptr(context_lens), int(max_context_len), float(scale), _ptr(out),
            _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if stage is None:
        _check(lib().pa_decode(*args), "pa_decode")
    else:
        _check(lib().pa_decode_stage(int(stage), *args), f"pa_decode_stage({stage})")


def extend_workspace_size(num_seqs, num_tokens, num_q_heads, head_dim, max_context_len) -> int:
    return int(lib().pa_extend_workspace_size(num_seqs, num_tokens, num_q_heads, head_dim, max_context_len))


def extend(q, cache: KVCache, query_start, block_tables, context_lens, max_context_len: int, scale: float, out,
           workspace, stream=None) -> None:
    """Multi-query causal attention: q, out [T, Hq, D]; query_start int32 [S + 1] (device)."""
    import torch
    T, Hq, _ = q.shape
    _dev(query_start, "query_start", torch.int32, 1, 1)
    S = query_start.shape[0] - 1
    _check_attention(q, out, cache, block_tables, context_lens, S)
    _dev(workspace, "workspace")
    st = lib().pa_extend(_ptr(q), dtype_code(q), S, Hq, _ptr(query_start), T, ctypes.byref(cache.desc),
                         _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), int(max_context_len),
                         float(scale), _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                         _stream(stream))
    _check(st, "pa_extend")


def prefill(q, k, v, cache: KVCache, query_start, block_tables, context_lens, max_context_len: int, scale: float,
            out, workspace, stream=None) -> None:
    """Whole prompts: q, out [T, Hq, D]; k, v [T, Hkv, D] (the prompts' keys and values, written
    into the cache by the same kernel); query_start int32 [S + 1]; context_lens = prompt lengths."""
    import torch
    T, Hq, _ = q.shape
    _dev(query_start, "query_start", torch.int32, 1, 1)
    S = query_start.shape[0] - 1
    _check_attention(q, out, cache, block_tables, context_lens, S)
    for name, x in (("k", k), ("v", v)):
        _dev(x, name, q.dtype, 3)
        if tuple(x.shape) != (T, cache.desc.num_kv_heads, cache.desc.head_dim):
            raise ValueError(f"{name} shape {tuple(x.shape)} is not [{T}, {cache.desc.num_kv_heads}, "
                             f"{cache.desc.head_dim}]")
    _dev(workspace, "workspace")
    st = lib().pa_prefill(_ptr(q), _ptr(k), _ptr(v), dtype_code(q), S, Hq, _ptr(query_start), T,
                          ctypes.byref(cache.desc), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
                          int(max_context_len), float(scale), _ptr(out), _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "pa_prefill")


def selftest_wait_timeout(limit_us: int, stream=None) -> None:
    """Enqueue the bounded-wait self-test (a wait on a barrier nothing arrives at); read the
    recorded timeout with last_device_error()."""
    _check(lib().pa_selftest_wait_timeout(int(limit_us), _stream(stream)), "pa_selftest_wait_timeout")


NO_ALLOC_WORKSPACE_BYTES = 16 << 20


def decode_no_alloc(q, cache: KVCache, block_tables, context_lens, max_context_len: int, scale: float, out,
                    stream=None) -> None:
    """pa_decode without a caller workspace: for callers that may not allocate device
    memory. The split-K scratch is a fixed 16 MiB array inside the library, shared by
    every call on a device (serialise calls that could overlap); sizes needing more
    raise PaError(PA_ERR_ARG)."""
    S, Hq, _ = q.shape
    _check_attention(q, out, cache, block_tables, context_lens, S)
    st = lib().pa_decode_no_alloc(_ptr(q), dtype_code(q), S, Hq, ctypes.byref(cache.desc), _ptr(block_tables),
                                  block_tables.shape[1], _ptr(context_lens), int(max_context_len), float(scale),
                                  _ptr(out), _stream(stream))
    _check(st, "pa_decode_no_alloc")


def block_table_update(updates, block_tables, stream=None) -> None:
    """Apply (seq, col, block) int32 [n, 3] device updates to the device block tables."""
    import torch
    n = 0 if updates is None else updates.shape[0]
    _dev(block_tables, "block_tables", torch.int32, 2)
    if n:
        _dev(updates, "updates", torch.int32, 2)
        if updates.shape[1] != 3:
            raise ValueError(f"updates shape {tuple(updates.shape)} is not [n, 3]")
    st = lib().pa_block_table_update(_ptr(updates), n, _ptr(block_tables), block_tables.shape[0],
                                     block_tables.shape[1], _stream(stream))
    _check(st, "pa_block_table_update")


def last_device_error(stream=None):
    """(code, info) of the sticky device error word, cleared by the read (synchronises)."""
    code = ctypes.c_int32(0)
    info = (ctypes.c_int32 * 3)()
    st = lib().pa_last_device_error(_stream(stream), ctypes.byref(code), info)
    if st not in (PA_OK, PA_ERR_DEVICE_CHECK):
        raise PaError(st, "pa_last_device_error")
    return code.value, tuple(info)


# ---------------------------------------------------------------------------
# host block pool
# ---------------------------------------------------------------------------

class Pool:
    """O(1) free-list block pool with reference counts (host memory only)."""

    def __init__(self, num_blocks: int, initial_order=None):
        import numpy as np
        self._h = ctypes.c_void_p()
        order = None
        if initial_order is not None:
            self._order = np.ascontiguousarray(np.asarray(initial_order, dtype=np.int32))
            order = _i32p(self._order)
        _check(lib().pa_pool_create(int(num_blocks), order, ctypes.byref(self._h)), "pa_pool_create")

    def close(self):
        if self._h:
            lib().pa_pool_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def alloc(self) -> int:
        b = ctypes.c_int32()
        _check(lib().pa_pool_alloc(self._h, ctypes.byref(b)), "pa_pool_alloc")
        return b.value

    def incref(self, b: int):
        _check(lib().pa_pool_incref(self._h, int(b)), "pa_pool_incref")

    def decref(self, b: int):
        _check(lib().pa_pool_decref(self._h, int(b)), "pa_pool_decref")

    def refcount(self, b: int) -> int:
        return lib().pa_pool_refcount(self._h, int(b))

    def num_free(self) -> int:
        return lib().pa_pool_num_free(self._h)

    def num_blocks(self) -> int:
        return lib().pa_pool_num_blocks(self._h)

    def free_list(self):
        import numpy as np
        n = self.num_free()
        buf = np.zeros(max(n, 1), dtype=np.int32)
        got = lib().pa_pool_free_list(self._h, _i32p(buf), n)
        return buf[:got].tolist()

    def seq_append(self, row, pos: int, block_size: int):
        """row: host int32 array (numpy), updated in place. Returns (slot, cow_src, cow_dst)."""
        slot = ctypes.c_int64()
        cs, cd = ctypes.c_int32(), ctypes.c_int32()
        _check(lib().pa_seq_append(self._h, _i32p(row), row.shape[-1], int(pos), int(block_size),
                                   ctypes.byref(slot), ctypes.byref(cs), ctypes.byref(cd)), "pa_seq_append")
        return slot.value, cs.value, cd.value

    def seq_extend(self, row, start_pos: int, n_tokens: int, block_size: int, slots=None):
        cs, cd, done = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        st = lib().pa_seq_extend(self._h, _i32p(row), row.shape[-1], int(start_pos), int(n_tokens),
                                 int(block_size), _i64p(slots, int(n_tokens)) if slots is not None else None,
                                 ctypes.byref(cs), ctypes.byref(cd), ctypes.byref(done))
        _check(st, "pa_seq_extend")
        return cs.value, cd.value

    def seq_fork(self, row, n_blocks: int):
        _check(lib().pa_seq_fork(self._h, _i32p(row, int(n_blocks)), int(n_blocks)), "pa_seq_fork")

    def seq_free(self, row, n_blocks: int):
        _check(lib().pa_seq_free(self._h, _i32p(row, int(n_blocks)), int(n_blocks)), "pa_seq_free")

    def batch_reorder(self, block_tables, context_lens, block_size: int, parents):
        """Beam re-selection in place: row i continues old row parents[i] (host int32 arrays)."""
        import numpy as np
        par = np.ascontiguousarray(parents, dtype=np.int32)
        S, MB = block_tables.shape
        _check(lib().pa_batch_reorder(self._h, _i32p(block_tables), _i32p(context_lens, S), S, MB, int(block_size),
                                      _i32p(par, S)), "pa_batch_reorder")

    def batch_append(self, block_tables, positions, block_size: int, slots, cow_pairs, updates):
        """One step's bookkeeping. All buffers are contiguous host arrays; returns (n_cow, n_updates)."""
        ncow, nupd, done = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        S, MB = block_tables.shape
        st = lib().pa_batch_append(self._h, _i32p(block_tables), S, MB, _i32p(positions, S), int(block_size),
                                   _i64p(slots, S), _i64p(cow_pairs, 2 * S), ctypes.byref(ncow),
                                   _i32p(updates, 3 * S), ctypes.byref(nupd), ctypes.byref(done))
        _check(st, "pa_batch_append")
        return ncow.value, nupd.value


class PrefixCache:
    """Host index from the content of full KV blocks to cached physical blocks."""

    def __init__(self, block_size: int):
        self._h = ctypes.c_void_p()
        self.block_size = int(block_size)
        _check(lib().pa_prefix_cache_create(int(block_size), ctypes.byref(self._h)), "pa_prefix_cache_create")

    def __len__(self):
        return lib().pa_prefix_cache_size(self._h)

    def __del__(self):
        try:
            if self._h:
                lib().pa_prefix_cache_destroy(self._h)
        except Exception:
            pass

    def match(self, pool: Pool, tokens, row) -> int:
        """Reuse the leading cached full blocks of `tokens` into `row` (host int32)."""
        import numpy as np
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        n = ctypes.c_int32()
        _check(lib().pa_prefix_cache_match(self._h, pool._h, _i32p(t), t.size, _i32p(row), row.shape[-1],
                                           ctypes.byref(n)), "pa_prefix_cache_match")
        return n.value

    def insert(self, pool: Pool, tokens, row) -> int:
        import numpy as np
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        n = ctypes.c_int32()
        rp = _i32p(row, t.size // self.block_size if self.block_size > 0 else 0)   # one entry per full block
        _check(lib().pa_prefix_cache_insert(self._h, pool._h, _i32p(t), t.size, rp, ctypes.byref(n)),
               "pa_prefix_cache_insert")
        return n.value

    def evict(self, pool: Pool, max_blocks: int) -> int:
        n = ctypes.c_int32()
        _check(lib().pa_prefix_cache_evict(self._h, pool._h, int(max_blocks), ctypes.byref(n)),
               "pa_prefix_cache_evict")
        return n.value

    def clear(self, pool: Pool) -> int:
        n = ctypes.c_int32()
        _check(lib().pa_prefix_cache_clear(self._h, pool._h, ctypes.byref(n)), "pa_prefix_cache_clear")
        return n.value


def version() -> str:
    return lib().pa_version().decode()
