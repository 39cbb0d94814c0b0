"""CPU tests of the C-ABI library: it loads, exports every symbol the header
declares, and its host block pool matches the oracle's pool model bit for bit.
No GPU call is made here."""

import ctypes
import os
import re
import time

import numpy as np
import pytest

import paged_kv_cache_436_b200 as pa
from oracle.pool import BlockPool, PoolError
from paged_kv_cache_436_b200 import build as pa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_library():
    if pa_build.stale():
        pa_build.build()
    return pa.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "pa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = header_functions()
    assert len(names) >= 20
    L = ctypes.CDLL(pa.LIB_PATH)
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    assert set(names) == set(pa._SIGNATURES), "binding and header disagree"


def test_version_and_sizes():
    assert "sm_100a" in pa.version()
    # plan (S+1 ints) + (m, l) + acc per (seq, q head, partition), each 256-byte aligned; the
    # grouped-head tensor-core decode adds its unit records (32 bytes per sequence and
    # partition), the work counter and the chunk count per row
    S, Hq, D, P = 8, 32, 128, 64
    partials = 256 + S * Hq * P * 2 * 4 + S * Hq * P * D * 4
    assert pa.decode_workspace_size(S, Hq, D, 512 * P) == partials + S * P * 32 + 256 + 256
    assert pa.decode_workspace_size(-1, 32, 128, 10) == 0


def test_host_argument_checks_launch_nothing():
    L = pa.lib()
    desc = pa.CacheDesc(16, 2, 16, 128, pa.PA_BF16, 1.0, 1.0, 0, 0)      # null cache pointers
    assert L.pa_copy_blocks(None, 1, ctypes.byref(desc), None) == pa.PA_ERR_ARG
    desc = pa.CacheDesc(16, 2, 16, 96, pa.PA_BF16, 1.0, 1.0, 256, 256)  # unsupported head_dim
    assert L.pa_reshape_and_cache(None, None, pa.PA_BF16, 1, 256, 256, None, ctypes.byref(desc), None) == pa.PA_ERR_ARG
    desc = pa.CacheDesc(16, 2, 16, 128, pa.PA_BF16, 2.0, 1.0, 256, 256)  # scale on a 16-bit cache
    assert L.pa_copy_blocks(None, 0, ctypes.byref(desc), None) == pa.PA_ERR_ARG
    desc = pa.CacheDesc(16, 2, 12, 128, pa.PA_BF16, 1.0, 1.0, 256, 256)  # block size 12
    assert L.pa_copy_blocks(None, 0, ctypes.byref(desc), None) == pa.PA_ERR_ARG
    desc = pa.CacheDesc(16, 2, 16, 128, pa.PA_BF16, 1.0, 1.0, 256, 256)
    # 6 q heads over 2 kv heads: G = 3 is not supported
    assert L.pa_decode(256, pa.PA_BF16, 1, 6, ctypes.byref(desc), 256, 1, 256, 16, 1.0, 256, 256, 1 << 20,
                       None) == pa.PA_ERR_ARG
    # q dtype must match a 16-bit cache
    assert L.pa_decode(256, pa.PA_F16, 1, 2, ctypes.byref(desc), 256, 1, 256, 16, 1.0, 256, 256, 1 << 20,
                       None) == pa.PA_ERR_ARG
    # workspace too small
    assert L.pa_decode(256, pa.PA_BF16, 4, 2, ctypes.byref(desc), 256, 4, 256, 2048, 1.0, 256, 256, 64,
                       None) == pa.PA_ERR_ARG
    # no sequences: nothing to do
    assert L.pa_decode(None, pa.PA_BF16, 0, 2, ctypes.byref(desc), None, 1, None, 0, 1.0, None, None, 0,
                       None) == pa.PA_OK


def test_extend_and_prefill_argument_checks_launch_nothing():
    L = pa.lib()
    bf = pa.CacheDesc(64, 2, 16, 128, pa.PA_BF16, 1.0, 1.0, 256, 256)
    fp8 = pa.CacheDesc(64, 2, 16, 128, pa.PA_E4M3, 0.05, 0.05, 256, 256)
    d64 = pa.CacheDesc(64, 2, 16, 64, pa.PA_BF16, 1.0, 1.0, 256, 256)
    ws = pa.extend_workspace_size(2, 8, 4, 128, 64)
    assert ws > 0

    def extend(desc, q_dtype=pa.PA_BF16, Hq=4, q=256, scale=0.1, wsb=ws):
        return L.pa_extend(q, q_dtype, 2, Hq, 256, 8, ctypes.byref(desc), 256, 4, 256, 64, scale, 256, 256, wsb,
                           None)

    assert extend(fp8, q_dtype=pa.PA_E4M3) == pa.PA_ERR_ARG  # q is f16 or bf16, also over an E4M3 cache
    fp8_bs8 = pa.CacheDesc(64, 2, 8, 128, pa.PA_E4M3, 0.05, 0.05, 256, 256)
    assert extend(fp8_bs8) == pa.PA_ERR_ARG                  # extend reads blocks of 16 or 32 tokens
    assert extend(bf, q_dtype=pa.PA_F16) == pa.PA_ERR_ARG    # q dtype must equal the cache's
    assert extend(bf, Hq=6) == pa.PA_ERR_ARG                 # G = 3
    assert extend(bf, scale=float("nan")) == pa.PA_ERR_ARG
    assert extend(bf, q=258) == pa.PA_ERR_ARG                # q not 16-byte aligned
    assert extend(bf, wsb=64) == pa.PA_ERR_ARG               # workspace too small
    assert L.pa_extend(None, pa.PA_BF16, 0, 4, None, 0, ctypes.byref(bf), None, 4, None, 0, 0.1, None, None, 0,
                       None) == pa.PA_OK                      # nothing to do

    def prefill(desc, scale=0.1, k=256):
        return L.pa_prefill(256, k, k, pa.PA_BF16, 2, 4, 256, 8, ctypes.byref(desc), 256, 4, 256, 64, scale, 256,
                            256, ws, None)

    assert prefill(d64) == pa.PA_ERR_ARG                      # head_dim 64: no tcgen05 path
    assert prefill(bf, scale=-0.1) == pa.PA_ERR_ARG           # the tcgen05 path needs scale > 0
    assert prefill(fp8, k=None) == pa.PA_ERR_ARG              # an E4M3 prefill needs the prompts' K / V
    assert prefill(fp8, k=264) == pa.PA_ERR_ARG               # ... 16-byte aligned
    # the self-test refuses limits out of range before launching anything
    assert L.pa_selftest_wait_timeout(0, None) == pa.PA_ERR_ARG
    assert L.pa_selftest_wait_timeout(3000000, None) == pa.PA_ERR_ARG


def test_extend_workspace_size_bounds():
    size = pa.extend_workspace_size
    assert size(-1, 8, 4, 128, 64) == 0 and size(2, 8, 0, 128, 64) == 0
    a, b = size(4, 64, 8, 128, 1024), size(4, 64, 8, 128, 4096)
    assert 0 < a < b                                          # grows with the partitions a row can span
    assert size(4, 128, 8, 128, 1024) > a                     # and with the query rows
    assert a % 256 == 0


def _oracle_equal(native: pa.Pool, model: BlockPool):
    assert native.num_free() == model.num_free()
    assert native.free_list() == model.free_list()
    for b in range(model.num_blocks):
        assert native.refcount(b) == model.refcnt[b]


def test_native_pool_fixtures_match_oracle():
    order = [0, 1, 2, 4, 3, 7, 8, 9, 5, 6, 10, 11]
    native, model = pa.Pool(12, order), BlockPool(12, order)
    rows_n = {r: np.zeros(4, np.int32) for r in "ABC"}
    rows_m = {r: [] for r in "ABC"}
    lens = {"A": 3, "B": 3, "C": 2}
    for lb in range(3):
        for r in "ABC":
            if lb < lens[r]:
                sn = native.seq_append(rows_n[r], lb * 16, 16)
                sm = model.seq_append(rows_m[r], lb * 16, 16)
                assert sn == sm
    assert {r: rows_n[r][:lens[r]].tolist() for r in "ABC"} == {"A": [0, 4, 8], "B": [1, 3, 9], "C": [2, 7]}
    _oracle_equal(native, model)


def test_native_pool_errors():
    p = pa.Pool(2)
    assert [p.alloc(), p.alloc()] == [0, 1]
    with pytest.raises(pa.PaError) as e:
        p.alloc()
    assert e.value.status == pa.PA_ERR_OOM
    p.decref(1)
    with pytest.raises(pa.PaError) as e:
        p.decref(1)
    assert e.value.status == pa.PA_ERR_STATE
    with pytest.raises(pa.PaError) as e:
        p.incref(1)
    assert e.value.status == pa.PA_ERR_STATE
    with pytest.raises(pa.PaError) as e:
        pa.Pool(3, [0, 2, 2])
    assert e.value.status == pa.PA_ERR_ARG
    row = np.zeros(1, np.int32)
    with pytest.raises(pa.PaError):
        p.seq_append(row, 16, 16)          # logical block 1 is beyond the 1-entry row


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_native_pool_random_ops_match_oracle(seed):
    rng = np.random.default_rng(100 + seed)
    NB, BS, MB = 96, 8, 64
    order = rng.permutation(NB)
    native, model = pa.Pool(NB, order), BlockPool(NB, order)
    seqs = []    # [native row, model row, length]
    for _ in range(1500):
        op = int(rng.integers(0, 5))
        if op == 0 or not seqs:
            n = int(rng.integers(1, 40))
            rn, rm = np.zeros(MB, np.int32), []
            slots_n = np.zeros(n, np.int64)
            try:
                model.seq_extend(rm, 0, n, BS)
                ok_m = True
            except PoolError:
                ok_m = False
            try:
                native.seq_extend(rn, 0, n, BS, slots_n)
                ok_n = True
            except pa.PaError as e:
                assert e.status == pa.PA_ERR_OOM
                ok_n = False
            assert ok_m == ok_n
            if ok_m:
                seqs.append([rn, rm, n])
            else:
                # both stranded the same partial allocation; keep the pools comparable
                pass
        elif op == 1:
            i = int(rng.integers(len(seqs)))
            rn, rm, n = seqs[i]
            try:
                a = model.seq_append(rm, n, BS)
            except PoolError:
                a = None
            try:
                b = native.seq_append(rn, n, BS)
            except pa.PaError:
                b = None
            assert a == b
            if a is not None:
                seqs[i][2] = n + 1
        elif op == 2:
            i = int(rng.integers(len(seqs)))
            rn, rm, n = seqs[i]
            nb = -(-n // BS)
            native.seq_fork(rn, nb)
            seqs.append([rn.copy(), model.fork(rm), n])
        elif op == 3:
            i = int(rng.integers(len(seqs)))
            rn, rm, n = seqs.pop(i)
            native.seq_free(rn, -(-n // BS))
            model.free_seq(rm)
        else:
            # a batched decode step over all live sequences
            if not seqs:
                continue
            S = len(seqs)
            bt = np.zeros((S, MB), np.int32)
            for s, (rn, _, _) in enumerate(seqs):
                bt[s] = rn
            pos = np.array([n for _, _, n in seqs], np.int32)
            snap = (model.free_list(), list(model.refcnt), [list(r) for _, r, _ in seqs])
            try:
                slots_m, cows_m, upd_m = model.batch_append([r for _, r, _ in seqs], list(pos), BS)
                ok = True
            except PoolError:
                ok = False
            slots = np.zeros(S, np.int64)
            cows = np.zeros((S, 2), np.int64)
            upd = np.zeros((S, 3), np.int32)
            try:
                ncow, nupd = native.batch_append(bt, pos, BS, slots, cows, upd)
                ok_n = True
            except pa.PaError:
                ok_n = False
            assert ok == ok_n
            if not ok:
                # partial batch on both sides: rebuild the comparison from scratch
                return
            assert slots.tolist() == slots_m
            assert [tuple(x) for x in cows[:ncow].tolist()] == cows_m
            assert [tuple(x) for x in upd[:nupd].tolist()] == upd_m
            for s in range(S):
                seqs[s][0] = bt[s].copy()
                seqs[s][2] += 1
        for rn, rm, n in seqs:
            assert rn[:len(rm)].tolist() == rm
        _oracle_equal(native, model)


def test_alloc_free_cost_is_flat_in_pool_size():
    """O(1) alloc/free: the time per operation does not grow with the pool (page 3,
    section "PagedAttention原理")."""
    L = pa.lib()

    def per_op(nb):
        p = pa.Pool(nb)
        row = np.zeros(4096, np.int32)
        cs, cd, done = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        t0 = time.perf_counter()
        for _ in range(20):
            assert L.pa_seq_extend(p._h, pa._i32p(row), 4096, 0, 4096 * 16, 16, None,
                                   ctypes.byref(cs), ctypes.byref(cd), ctypes.byref(done)) == 0
            assert L.pa_seq_free(p._h, pa._i32p(row), 4096) == 0
        return (time.perf_counter() - t0) / (20 * 4096 * 16)

    small = min(per_op(4096) for _ in range(3))
    big = min(per_op(1 << 22) for _ in range(3))
    assert big < 4 * small + 2e-8, (small, big)


def test_binding_refuses_host_buffers_it_cannot_pass_safely():
    """The native calls trust the extents the header states; the binding checks element
    type, contiguity and size first and leaves the pool untouched when it refuses."""
    import torch
    p = pa.Pool(8)
    with pytest.raises(TypeError):
        p.seq_append(np.zeros(4, np.int64), 0, 16)                     # int64 row read as int32 pairs
    with pytest.raises(TypeError):
        p.seq_append(np.zeros((4, 2), np.int32)[:, 0], 0, 16)          # strided view
    with pytest.raises(TypeError):
        p.seq_append(torch.zeros(4, dtype=torch.int64), 0, 16)
    with pytest.raises(ValueError):
        p.seq_extend(np.zeros(4, np.int32), 0, 20, 16, np.zeros(19, np.int64))   # slots for 19 of 20 tokens
    with pytest.raises(ValueError):
        p.seq_free(np.zeros(2, np.int32), 3)
    S, MB = 3, 4
    bt = np.zeros((S, MB), np.int32)
    with pytest.raises(ValueError):
        p.batch_append(bt, np.zeros(S, np.int32), 16, np.zeros(S, np.int64), np.zeros(2 * S - 1, np.int64),
                       np.zeros(3 * S, np.int32))
    with pytest.raises(ValueError):
        p.batch_reorder(bt, np.zeros(S - 1, np.int32), 16, [0, 0, 0])
    assert p.num_free() == 8 and p.free_list() == list(range(8))
    # the same calls with the right buffers go through
    row = np.zeros(4, np.int32)
    slots = np.zeros(20, np.int64)
    assert p.seq_extend(row, 0, 20, 16, slots) == (-1, -1) and slots[19] == row[1] * 16 + 3
    c = pa.PrefixCache(4)
    with pytest.raises(ValueError):
        c.insert(p, list(range(12)), np.zeros(2, np.int32))            # 3 full blocks, 2 entries
    assert len(c) == 0


def test_kv_cache_descriptor_checks_its_tensors():
    import torch
    f16 = torch.zeros((2, 1, 16, 64), dtype=torch.float16)
    assert pa.KVCache(f16, f16.clone(), "f16").desc.head_dim == 64
    with pytest.raises(ValueError):
        pa.KVCache(f16, torch.zeros((2, 1, 16, 32), dtype=torch.float16), "f16")
    with pytest.raises(ValueError):
        pa.KVCache(f16.transpose(2, 3), f16.transpose(2, 3), "f16")
    with pytest.raises(TypeError):
        pa.KVCache(f16, f16.clone(), "bf16")
    with pytest.raises(TypeError):
        pa.KVCache(f16, f16.clone(), "e4m3")
    with pytest.raises(ValueError):
        pa.KVCache(f16, f16.clone(), "fp8")
    u8 = torch.zeros((2, 1, 16, 64), dtype=torch.uint8)
    assert pa.KVCache(u8, u8.clone(), "e4m3", 0.5, 0.25).desc.k_scale == 0.5


def test_refused_pool_calls_change_nothing():
    """seq_free and batch_reorder check every block before touching a count; seq_extend
    refuses positions whose end does not fit in int32."""
    p = pa.Pool(8, np.arange(8))
    row = np.zeros(4, np.int32)
    p.seq_extend(row, 0, 40, 16)                          # blocks 0, 1, 2
    p.decref(1)                                           # block 1 freed behind the row's back
    with pytest.raises(pa.PaError) as e:
        p.seq_free(row, 3)
    assert e.value.status == pa.PA_ERR_STATE
    assert [p.refcount(b) for b in range(3)] == [1, 0, 1] and p.num_free() == 6
    # beam reorder: row 1 is dropped (nobody continues it) and lists an out-of-range id
    bt = np.array([[0, 2, 0, 0], [7, 99, 0, 0]], np.int32)
    lens = np.array([20, 20], np.int32)
    p2 = pa.Pool(8, np.arange(8))
    for _ in range(3):
        p2.alloc()                                        # blocks 0, 1, 2 held once
    with pytest.raises(pa.PaError) as e:
        p2.batch_reorder(bt, lens, 16, [0, 0])
    assert e.value.status == pa.PA_ERR_STATE
    assert bt.tolist() == [[0, 2, 0, 0], [7, 99, 0, 0]] and lens.tolist() == [20, 20]
    assert [p2.refcount(b) for b in range(8)] == [1, 1, 1, 0, 0, 0, 0, 0]
    big = np.zeros(4, np.int32)
    with pytest.raises(pa.PaError) as e:
        p.seq_extend(big, 2**31 - 10, 20, 16)
    assert e.value.status == pa.PA_ERR_ARG and p.num_free() == 6


def test_engine_metadata_buffer_holds_every_region():
    """pa_engine_meta_bytes: slots (8 B), copy pairs (16 B), lengths (4 B) and table updates
    (12 B) per sequence, each region 16-byte aligned; 0 for a negative count."""
    L = pa.lib()
    for S in (1, 2, 3, 7, 20, 255, 256, 1000):
        n = L.pa_engine_meta_bytes(S)
        regions = [8 * S, 16 * S, 4 * S, 12 * S]
        want = 0
        for r in regions:
            want = (want + 15) // 16 * 16 + r
        assert n % 16 == 0 and n == (want + 15) // 16 * 16, (S, n)
    assert L.pa_engine_meta_bytes(-1) == 0


def test_engine_create_checks_its_configuration_before_any_cuda_call():
    """Every refusal here comes from a host check made before the engine creates its
    CUDA events; the pointers are placeholders and are never dereferenced."""
    L = pa.lib()
    pool = pa.Pool(64)
    S, Hq, MB, maxlen = 4, 8, 8, 128
    meta = L.pa_engine_meta_bytes(S)
    ws = L.pa_decode_workspace_size(S, Hq, 128, maxlen)

    def cfg(**kw):
        c = pa.EngineConfig()
        c.pool, c.num_seqs, c.num_q_heads, c.max_blocks_per_seq = pool._h, S, Hq, MB
        c.max_context_len, c.q_dtype, c.scale = maxlen, pa.PA_BF16, 0.125
        c.cache = pa.CacheDesc(64, 2, 16, 128, pa.PA_BF16, 1.0, 1.0, 256, 256)
        c.block_tables_host = c.context_lens_host = c.block_tables_dev = 4096
        c.meta_host[0], c.meta_host[1] = 4096, 8192
        c.meta_dev, c.meta_bytes, c.workspace, c.workspace_bytes = 4096, meta, 4096, ws
        for k, v in kw.items():
            setattr(c, k, v)
        return c

    out = ctypes.c_void_p()
    assert L.pa_engine_create(None, ctypes.byref(out)) == pa.PA_ERR_ARG
    for bad in (dict(pool=None), dict(num_seqs=0), dict(num_q_heads=0), dict(max_blocks_per_seq=0),
                dict(max_context_len=-1), dict(meta_bytes=meta - 1), dict(meta_dev=4096 + 8),
                dict(workspace_bytes=ws - 1), dict(workspace=None), dict(block_tables_dev=None)):
        assert L.pa_engine_create(ctypes.byref(cfg(**bad)), ctypes.byref(out)) == pa.PA_ERR_ARG, bad
        assert not out.value
    assert L.pa_engine_step(None, 256, 256, 256, 256, None, None, None) == pa.PA_ERR_ARG


def test_no_alloc_decode_refuses_oversized_work_before_any_cuda_call():
    L = pa.lib()
    desc = pa.CacheDesc(64, 40, 16, 128, pa.PA_BF16, 1.0, 1.0, 256, 256)
    big = 8192 + 512                                   # 256 seqs x 40 heads x 17 partitions
    assert L.pa_decode_workspace_size(256, 40, 128, big) > pa.NO_ALLOC_WORKSPACE_BYTES
    assert L.pa_decode_no_alloc(256, pa.PA_BF16, 256, 40, ctypes.byref(desc), 256, 1024, 256, big, 0.1,
                                256, None) == pa.PA_ERR_ARG
    assert L.pa_decode_no_alloc(256, pa.PA_BF16, 256, 40, None, 256, 1024, 256, 16, 0.1, 256, None) == pa.PA_ERR_ARG
    assert L.pa_decode_no_alloc(256, pa.PA_BF16, -1, 40, ctypes.byref(desc), 256, 1024, 256, 16, 0.1,
                                256, None) == pa.PA_ERR_ARG


def test_pool_size_and_usage():
    """The pool's size and free count give the cache-usage fraction (blocks in use / total)."""
    p = pa.Pool(12)
    assert p.num_blocks() == 12 and p.num_free() == 12
    taken = [p.alloc() for _ in range(5)]
    assert p.num_blocks() == 12 and (p.num_blocks() - p.num_free()) / p.num_blocks() == 5 / 12
    for b in taken:
        p.decref(b)
    assert p.num_free() == 12
    assert pa.lib().pa_pool_num_blocks(None) == -1 and pa.lib().pa_pool_num_free(None) == -1


def test_workspace_sizes_at_the_length_limit():
    """Sizes grow by one partition's partials at 512-token steps up to the 6,291,456-token
    limit; invalid counts give 0; calls beyond the limit are refused by the calls."""
    L = pa.lib()
    for f in (lambda m: L.pa_decode_workspace_size(8, 32, 128, m),
              lambda m: L.pa_extend_workspace_size(8, 8, 32, 128, m)):
        assert f(0) == f(1) == f(512) < f(513)
        assert f(6291456) > f(6291456 - 512) > 0
    assert L.pa_decode_workspace_size(-1, 32, 128, 16) == 0 and L.pa_decode_workspace_size(1, 0, 128, 16) == 0
    assert L.pa_extend_workspace_size(1, -1, 32, 128, 16) == 0 and L.pa_extend_workspace_size(1, 1, 32, 0, 16) == 0
    desc = pa.CacheDesc(64, 32, 16, 128, pa.PA_BF16, 1.0, 1.0, 256, 256)
    big = 6291456 + 1
    ws = L.pa_decode_workspace_size(8, 32, 128, big)
    assert L.pa_decode(256, pa.PA_BF16, 8, 32, ctypes.byref(desc), 256, 1 << 20, 256, big, 0.1, 256, 256, ws,
                       None) == pa.PA_ERR_ARG
