"""Beam re-selection (page 1, section "5. 高级应用场景"): the native pool against the
oracle under random beam steps, and the memory the sharing saves. CPU only."""

import numpy as np
import pytest

import paged_kv_cache_436_b200 as pa
import synthetic
from oracle import pool as opool_mod
from oracle.pool import BlockPool
from paged_kv_cache_436_b200 import build as pa_build


@pytest.fixture(scope="module", autouse=True)
def built_library():
    if pa_build.stale():
        pa_build.build()
    return pa.lib()


def test_reorder_keeps_chosen_beams_and_frees_dropped_ones():
    pool = BlockPool(20)
    rows = [[], []]
    pool.seq_extend(rows[0], 0, 10, 4)       # 3 blocks
    pool.seq_extend(rows[1], 0, 6, 4)        # 2 blocks
    rows2, lens2 = opool_mod.reorder(pool, rows, [10, 6], [0, 0])
    assert rows2 == [rows[0], rows[0]] and lens2 == [10, 10]
    assert all(pool.refcount(b) == 2 for b in rows[0]) and pool.num_free() == 20 - 3
    slot, cs, cd = pool.seq_append(rows2[1], 10, 4)      # shared partial block: copy on write
    assert cs == rows[0][2] and cd not in rows[0]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_native_beam_steps_match_oracle(seed):
    R, W, BS, MB = 3, 5, 8, 40
    w = synthetic.beam_workload(num_requests=R, width=W, prompt=40, num_heads=2, head_dim=64, block_size=BS,
                                growth=60, seed=300 + seed)
    npool, opool = pa.Pool(w.num_blocks, w.initial_order), BlockPool(w.num_blocks, w.initial_order)
    S = R * W
    bt = np.zeros((S, MB), np.int32)
    lens = np.zeros(S, np.int32)
    orows, olens = [[] for _ in range(S)], [0] * S
    for r in range(R):
        L = w.context_lens[r * W]
        npool.seq_extend(bt[r * W], 0, L, BS)
        opool.seq_extend(orows[r * W], 0, L, BS)
        for j in range(1, W):
            npool.seq_fork(bt[r * W], -(-L // BS))
            bt[r * W + j] = bt[r * W]
            orows[r * W + j] = opool.fork(orows[r * W])
        lens[r * W:(r + 1) * W] = L
        olens[r * W:(r + 1) * W] = [L] * W
    total_cows = 0
    for step in range(50):
        parents = synthetic.beam_parents(R, W, step, w.seed)
        npool.batch_reorder(bt, lens, BS, parents)
        orows, olens = opool_mod.reorder(opool, orows, olens, parents)
        slots, cows, upd = np.zeros(S, np.int64), np.zeros((S, 2), np.int64), np.zeros((S, 3), np.int32)
        ncow, nupd = npool.batch_append(bt, lens, BS, slots, cows, upd)
        oslots, ocows, oupd = opool.batch_append(orows, olens, BS)
        lens += 1
        olens = [L + 1 for L in olens]
        assert slots.tolist() == oslots and [tuple(c) for c in cows[:ncow].tolist()] == ocows
        assert [tuple(u) for u in upd[:nupd].tolist()] == oupd
        total_cows += ncow
        for s in range(S):
            assert bt[s, :len(orows[s])].tolist() == orows[s]
        assert npool.free_list() == opool.free_list()
    assert total_cows > 0
    for b in range(w.num_blocks):
        assert npool.refcount(b) == opool.refcnt[b]


def test_beam_sharing_saves_memory():
    """Width-5 beams over a 1024-token prompt hold the prompt once (page 1, section
    "5. 高级应用场景": 8.2 GB -> 3.7 GB for width 5)."""
    R, W, BS = 4, 5, 16
    w = synthetic.beam_workload(num_requests=R, width=W, prompt=1024, num_heads=2, head_dim=64, growth=64)
    pool = BlockPool(w.num_blocks, w.initial_order)
    rows = [[] for _ in range(R * W)]
    lens = [0] * (R * W)
    for r in range(R):
        L = w.context_lens[r * W]
        pool.seq_extend(rows[r * W], 0, L, BS)
        for j in range(1, W):
            rows[r * W + j] = pool.fork(rows[r * W])
        lens[r * W:(r + 1) * W] = [L] * W
    for step in range(64):
        rows, lens = opool_mod.reorder(pool, rows, lens, synthetic.beam_parents(R, W, step, w.seed))
        pool.batch_append(rows, lens, BS)
        lens = [L + 1 for L in lens]
    shared = w.num_blocks - pool.num_free()
    unshared = sum(-(-L // BS) for L in lens)
    assert unshared > 4 * shared
