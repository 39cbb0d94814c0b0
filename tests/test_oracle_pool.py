"""Pins for the oracle's block pool, cache ops and byte accounting."""

import json
import os

import numpy as np
import pytest

from oracle import accounting, cache_ops, codecs
from oracle.pool import BlockPool, PoolError
from tests.conftest import GOLDEN


def _load(name):
    return json.load(open(os.path.join(GOLDEN, name)))


def test_page1_block_tables_and_shared_refcount():
    fx = _load("block_table_example.json")
    p = BlockPool(8)
    s1 = [p.alloc(), p.alloc()]            # 0, 1
    s2 = [p.alloc()]                       # 2
    p.incref(s1[1])                        # seq_2 shares physical block 1
    s2.append(s1[1])
    s1.append(p.alloc())                   # 3
    s2.append(p.alloc())                   # 4
    assert s1 == fx["tables"]["seq_1"] and s2 == fx["tables"]["seq_2"]
    assert p.refcount(1) == 2 and all(p.refcount(b) == 1 for b in (0, 2, 3, 4))
    assert p.num_free() == 3


def test_page3_twelve_block_diagram():
    fx = _load("pool_diagram_12_blocks.json")
    # requests take one block each in turn A, B, C, A, B, C, A, B
    order = [0, 1, 2, 4, 3, 7, 8, 9, 5, 6, 10, 11]
    p = BlockPool(fx["num_blocks"], order)
    rows = {"A": [], "B": [], "C": []}
    lens = {"A": 3, "B": 3, "C": 2}
    for lb in range(3):
        for r in "ABC":
            if lb < lens[r]:
                p.seq_append(rows[r], lb * 16, 16)
    assert rows == fx["tables"]
    assert sorted(p.free_list()) == fx["free"] and p.num_free() == 4


def test_static_reservation_and_paged_waste():
    fx = _load("static_reservation.json")
    reserved, used, wasted = accounting.static_reservation(fx["used_tokens"], fx["max_seq_len"])
    assert (reserved, used) == (fx["reserved"], fx["used"]) and wasted == 3072 - 896
    assert accounting.paged_waste(fx["used_tokens"], 16) == [0, 0, 0]
    assert all(0 <= w < 16 for w in accounting.paged_waste([1, 17, 50, 100, 255], 16))


def test_kv_size_closed_form():
    fx = _load("kv_size_closed_form.json")
    got = accounting.kv_cache_bytes(fx["num_layers"], fx["num_heads"], fx["head_dim"],
                                    fx["seq_len"], fx["batch"], fx["dtype_bytes"])
    assert got == fx["bytes"] == 536870912
    # the same bytes held as whole blocks of a paged cache: 1024 tokens = 64 blocks of 16
    assert accounting.paged_cache_bytes(64, 32, 16, 128, 2, num_layers=32) == got
    # the per-step count reads exactly K and V of every context token once
    kv_only = accounting.decode_bytes([1024], 32, 32, 128, 2, 2, 16) - (2 * 32 * 128 * 2 + 4 * 64 + 4)
    assert kv_only * 32 == got


def test_lifo_order_and_errors():
    p = BlockPool(4, [2, 0, 3, 1])
    assert [p.alloc() for _ in range(4)] == [2, 0, 3, 1]
    with pytest.raises(PoolError) as e:
        p.alloc()
    assert e.value.kind == "OOM"
    p.decref(3)
    p.decref(0)
    assert p.free_list() == [0, 3]          # last freed is handed out first
    with pytest.raises(PoolError) as e:
        p.decref(0)
    assert e.value.kind == "STATE"
    with pytest.raises(PoolError) as e:
        p.incref(3)
    assert e.value.kind == "STATE"
    with pytest.raises(PoolError):
        BlockPool(3, [0, 0, 1])


def test_copy_on_write_of_shared_partial_block():
    p = BlockPool(10)
    a = []
    p.seq_extend(a, 0, 20, 16)              # blocks 0 (full) and 1 (4 tokens)
    b = p.fork(a)
    assert p.refcount(0) == p.refcount(1) == 2
    slot, cs, cd = p.seq_append(b, 20, 16)  # b writes into the shared partial block
    assert (cs, cd) == (1, 2) and b == [0, 2] and slot == 2 * 16 + 4
    assert p.refcount(1) == 1 and p.refcount(0) == 2
    slot, cs, cd = p.seq_append(a, 20, 16)  # a is now the sole owner: in place
    assert (cs, cd) == (-1, -1) and slot == 1 * 16 + 4
    p.free_seq(b)
    p.free_seq(a)
    assert p.num_free() == 10


def test_prefix_sharing_cow_count_is_sharers_minus_one():
    p = BlockPool(200)
    owner = []
    p.seq_extend(owner, 0, 1000, 16)        # 62 full blocks + 8 tokens
    rows = [owner] + [p.fork(owner) for _ in range(63)]
    last = owner[-1]
    assert p.refcount(last) == 64
    cows = []
    for r in rows:
        _, cs, cd = p.seq_append(r, 1000, 16)
        if cs >= 0:
            cows.append((cs, cd))
    assert len(cows) == 63 and all(cs == last for cs, _ in cows)
    assert rows[63][-1] == last and p.refcount(last) == 1


def test_random_ops_keep_invariants():
    rng = np.random.default_rng(11)
    NB, BS = 64, 8
    p = BlockPool(NB, rng.permutation(NB))
    seqs = []                               # (row, length)
    for _ in range(3000):
        op = rng.integers(0, 4)
        try:
            if op == 0 or not seqs:
                row = []
                n = int(rng.integers(1, 30))
                p.seq_extend(row, 0, n, BS)
                seqs.append([row, n])
            elif op == 1:
                i = int(rng.integers(len(seqs)))
                row, n = seqs[i]
                p.seq_append(row, n, BS)
                seqs[i][1] = n + 1
            elif op == 2:
                i = int(rng.integers(len(seqs)))
                seqs.append([p.fork(seqs[i][0]), seqs[i][1]])
            else:
                i = int(rng.integers(len(seqs)))
                p.free_seq(seqs.pop(i)[0])
        except PoolError as e:
            # an OOM inside seq_extend strands the blocks it already took (the
            # new row is never recorded); seq_append fails before changing anything
            assert e.kind == "OOM"
        live = {}
        for row, n in seqs:
            assert len(row) == -(-n // BS)              # waste only in the last block
            for b in row:
                live[b] = live.get(b, 0) + 1
        # every reference in a table is counted; nothing else holds blocks, except
        # blocks stranded by an aborted append (still counted, owned by no table)
        for b, c in live.items():
            assert p.refcount(b) >= c
        assert p.num_free() + sum(1 for b in range(NB) if p.refcount(b) > 0) == NB
        assert len(set(p.free_list())) == p.num_free()


def test_batch_append_reports_slots_copies_and_table_updates():
    p = BlockPool(20, list(range(19, -1, -1)))
    a, b = [], []
    p.seq_extend(a, 0, 16, 4)               # 4 full blocks
    p.seq_extend(b, 0, 6, 4)
    c = p.fork(b)
    slots, cows, updates = p.batch_append([a, b, c], [16, 6, 6], 4)
    assert slots[0] == a[4] * 4 and updates[0] == (0, 4, a[4])
    assert cows == [(c[1], b[1])]
    assert updates[1] == (1, 1, b[1]) and len(updates) == 2


def test_cache_ops_reshape_and_copy():
    rng = np.random.default_rng(12)
    NB, H, BS, D = 6, 2, 4, 8
    kc = rng.integers(0, 1 << 16, size=(NB, H, BS, D)).astype(np.uint16)
    vc = rng.integers(0, 1 << 16, size=(NB, H, BS, D)).astype(np.uint16)
    k = rng.integers(0, 1 << 16, size=(3, H, D)).astype(np.uint16)
    v = rng.integers(0, 1 << 16, size=(3, H, D)).astype(np.uint16)
    nk, nv = cache_ops.reshape_and_cache(k, v, "bf16", [9, -1, 23], kc, vc, "bf16")
    assert np.array_equal(nk[2, :, 1], k[0]) and np.array_equal(nv[5, :, 3], v[2])
    changed = (nk != kc).any(axis=3)
    assert set(zip(*np.nonzero(changed))) <= {(2, h, 1) for h in range(H)} | {(5, h, 3) for h in range(H)}
    ck, cv = cache_ops.copy_blocks(kc, vc, [[0, 3], [4, 1]])
    assert np.array_equal(ck[3], kc[0]) and np.array_equal(cv[1], vc[4])
    assert np.array_equal(ck[[0, 2, 4, 5]], kc[[0, 2, 4, 5]])
    # all pairs read the state before the call
    ck, _ = cache_ops.copy_blocks(kc, vc, [[0, 1], [1, 2]])
    assert np.array_equal(ck[2], kc[1])


def test_cache_ops_fp8_encode_is_divide_then_round():
    x = np.array([[[1.0, -2.5, 0.0, 1000.0]]], dtype=np.float32)
    codes = x.view(np.uint32) >> 16                           # bf16 codes of exactly representable values
    codes = codes.astype(np.uint16)
    kc = np.zeros((1, 1, 2, 4), dtype=np.uint8)
    nk, _ = cache_ops.reshape_and_cache(codes, codes, "bf16", [1], kc, kc.copy(), "e4m3", 0.5, 0.5)
    assert codecs.decode_e4m3(nk[0, 0, 1]).tolist() == [2.0, -5.0, 0.0, 448.0]
