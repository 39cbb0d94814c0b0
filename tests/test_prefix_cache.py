"""Prefix cache: the oracle pinned by the pages' case and by its definition, and the
native index (C ABI) checked against the oracle bit for bit. CPU only."""

import numpy as np
import pytest

import paged_kv_cache_436_b200 as pa
from oracle.pool import BlockPool
from oracle.prefix_cache import PrefixCache
from paged_kv_cache_436_b200 import build as pa_build


@pytest.fixture(scope="module", autouse=True)
def built_library():
    if pa_build.stale():
        pa_build.build()
    return pa.lib()


def _serve(pool, cache, prompt, bs):
    """Admit one request: reuse cached full blocks, allocate the rest, cache its full blocks."""
    row = []
    n = cache.match(pool, prompt, row)
    pool.seq_extend(row, n * bs, len(prompt) - n * bs, bs)
    cache.insert(pool, prompt, row)
    return row, n


def test_page3_shared_history_case():
    """64 requests carrying the same 1000-token history (page 3, "案例与场景"): the first
    fills 62 full blocks and a partial one; each later request reuses the 62 full
    blocks and allocates only its partial block."""
    bs, hist = 16, list(range(1000))
    pool = BlockPool(5000)
    cache = PrefixCache(bs)
    rows = []
    for r in range(64):
        row, n = _serve(pool, cache, hist, bs)
        assert n == (0 if r == 0 else 62)
        rows.append(row)
    used_with = 5000 - pool.num_free()
    assert used_with == 62 + 64                       # 62 shared + one partial block each
    assert all(row[:62] == rows[0][:62] for row in rows)
    assert pool.refcount(rows[0][0]) == 64 + 1        # 64 sequences + the index
    # without the index every request holds its own 63 blocks
    pool2 = BlockPool(5000)
    for r in range(64):
        pool2.seq_extend([], 0, 1000, bs)
    assert 5000 - pool2.num_free() == 64 * 63


def test_dynamic_content_defeats_the_cache():
    """误区3: a differing token (a timestamp) stops reuse at its block."""
    bs = 16
    pool = BlockPool(100)
    cache = PrefixCache(bs)
    base = list(range(160))                          # 10 full blocks
    _serve(pool, cache, base, bs)
    early = list(base)
    early[3] = 9999                                  # differs inside block 0
    _, n = _serve(pool, cache, early, bs)
    assert n == 0
    late = list(base)
    late[5 * bs + 2] = 9999                          # differs inside block 5
    _, n = _serve(pool, cache, late, bs)
    assert n == 5


def test_key_is_the_whole_prefix():
    """Same tokens in block 1 after a different block 0: no reuse of block 1."""
    bs = 4
    pool = BlockPool(20)
    cache = PrefixCache(bs)
    _serve(pool, cache, [1, 2, 3, 4, 5, 6, 7, 8], bs)
    _, n = _serve(pool, cache, [9, 9, 9, 9, 5, 6, 7, 8], bs)
    assert n == 0
    _, n = _serve(pool, cache, [1, 2, 3, 4, 5, 6, 7, 8, 0], bs)
    assert n == 2


def test_a_block_repeated_at_another_position_is_not_reused():
    """Block 0's tokens again as block 1: its KV was computed at positions 0..3 with no
    context, so only block 0 is reused (a key of the block's own tokens would reuse it
    for block 1 as well)."""
    bs = 4
    pool = BlockPool(20)
    cache = PrefixCache(bs)
    first, _ = _serve(pool, cache, [1, 2, 3, 4, 5, 6, 7, 8], bs)
    row, n = _serve(pool, cache, [1, 2, 3, 4, 1, 2, 3, 4], bs)
    assert n == 1 and row[0] == first[0] and row[1] not in first


def test_evict_and_clear_release_only_unshared_blocks():
    bs = 4
    pool = BlockPool(20)
    cache = PrefixCache(bs)
    a, _ = _serve(pool, cache, list(range(8)), bs)         # 2 cached blocks
    b, _ = _serve(pool, cache, list(range(100, 112)), bs)  # 3 cached blocks
    pool.free_seq(b)                                     # b's blocks now held by the index only
    assert cache.evict(pool, 10) == 3 and len(cache) == 2  # a's blocks are still in use
    assert pool.num_free() == 20 - 2
    pool.free_seq(a)
    assert cache.clear(pool) == 2 and pool.num_free() == 20


def _native_serve(pool, cache, prompt, bs, mb):
    row = np.zeros(mb, np.int32)
    n = cache.match(pool, prompt, row)
    pool.seq_extend(row, n * bs, len(prompt) - n * bs, bs)
    cache.insert(pool, prompt, row)
    return row, n


def test_native_index_does_not_reuse_a_block_at_another_position():
    bs, NB, MB = 4, 20, 4
    npool = pa.Pool(NB, np.arange(NB))
    ncache = pa.PrefixCache(bs)
    first, _ = _native_serve(npool, ncache, [1, 2, 3, 4, 5, 6, 7, 8], bs, MB)
    row, n = _native_serve(npool, ncache, [1, 2, 3, 4, 1, 2, 3, 4], bs, MB)
    assert n == 1 and row[0] == first[0] and row[1] not in first[:2]
    _, n = _native_serve(npool, ncache, [1, 2, 3, 4, 1, 2, 3, 4, 9], bs, MB)
    assert n == 2                                      # now cached under its own prefix


def test_native_index_reports_partial_progress_and_stays_consistent():
    """A block freed behind the index's back: match keeps and reports the hits before
    it; clear releases what it can and keeps listing the rest, so a second clear
    neither crashes nor drops a reference twice."""
    import ctypes
    bs = 4
    p = pa.Pool(8, np.arange(8))
    c = pa.PrefixCache(bs)
    toks = np.arange(8, dtype=np.int32)
    row = np.zeros(4, np.int32)
    p.seq_extend(row, 0, 8, bs)                              # blocks 0, 1
    assert c.insert(p, toks, row) == 2
    p.seq_free(row, 2)                                       # the index holds them alone
    p.decref(1)                                              # ... until block 1 is freed anyway
    L, n = pa.lib(), ctypes.c_int32(-1)
    row2 = np.full(4, -1, np.int32)
    st = L.pa_prefix_cache_match(c._h, p._h, pa._i32p(toks), 8, pa._i32p(row2), 4, ctypes.byref(n))
    assert st == pa.PA_ERR_STATE and n.value == 1 and row2[0] == 0 and p.refcount(0) == 2
    assert c.evict(p, 10) == 0 and len(c) == 2               # block 0 is in use, block 1 is not 1-held
    st = L.pa_prefix_cache_clear(c._h, p._h, ctypes.byref(n))
    assert st == pa.PA_ERR_STATE and n.value == 1 and len(c) == 1 and p.refcount(0) == 1
    st = L.pa_prefix_cache_clear(c._h, p._h, ctypes.byref(n))
    assert st == pa.PA_ERR_STATE and n.value == 0 and len(c) == 1 and p.refcount(0) == 1


@pytest.mark.parametrize("seed", [0, 1])
def test_native_prefix_cache_matches_oracle(seed):
    rng = np.random.default_rng(200 + seed)
    bs, NB, MB = 8, 600, 40
    order = rng.permutation(NB)
    npool, opool = pa.Pool(NB, order), BlockPool(NB, order)
    ncache, ocache = pa.PrefixCache(bs), PrefixCache(bs)
    systems = [rng.integers(0, 50, size=int(rng.integers(8, 120))).tolist() for _ in range(4)]
    live = []
    for _ in range(300):
        op = rng.integers(0, 10)
        if op < 6:
            prompt = systems[int(rng.integers(4))] + rng.integers(0, 50, size=int(rng.integers(0, 60))).tolist()
            if rng.random() < 0.2 and len(prompt) > 3:
                prompt[int(rng.integers(len(prompt)))] = 777     # a "timestamp"
            if -(-len(prompt) // bs) > MB or opool.num_free() < MB + 2:
                continue
            orow, on = _serve(opool, ocache, prompt, bs)
            nrow, nn = _native_serve(npool, ncache, prompt, bs, MB)
            assert nn == on and nrow[:len(orow)].tolist() == orow
            live.append((orow, nrow, len(prompt)))
        elif op < 9 and live:
            orow, nrow, L = live.pop(int(rng.integers(len(live))))
            opool.free_seq(orow)
            npool.seq_free(nrow, -(-L // bs))
        else:
            k = int(rng.integers(0, 20))
            assert ncache.evict(npool, k) == ocache.evict(opool, k)
        assert len(ncache) == len(ocache)
        assert npool.num_free() == opool.num_free() and npool.free_list() == opool.free_list()
    for b in range(NB):
        assert npool.refcount(b) == opool.refcnt[b]
    assert ncache.clear(npool) == ocache.clear(opool)
