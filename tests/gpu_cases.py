"""Shared set-up for the GPU parity tests: a workload is built twice, once through
the CUDA library (engine, C++ pool, kernels) and once through the oracle (its own
pool model, its own cache ops, float64 attention); the inputs come only from the
seeded generators in ``synthetic``."""

from __future__ import annotations

import numpy as np
import torch

import synthetic
from oracle import attention as oatt
from oracle import cache_ops as oops
from oracle.pool import BlockPool
import paged_kv_cache_436_b200 as pa
from paged_kv_cache_436_b200.engine import DecodeEngine

# parity tolerances of the decode output: |err| <= atol + rtol * |ref|
TOL = {"f16": (2e-3, 1e-2), "bf16": (2e-3, 1e-2), "e4m3": (3e-2, 3e-2)}


def codes_np(t):
    """Raw element codes of a tensor as an unsigned numpy array."""
    t = t.detach().cpu().contiguous()
    if t.element_size() == 1:
        return t.view(torch.uint8).numpy()
    return t.view(torch.int16).numpy().view(np.uint16)


def assert_close(got, ref, kv_dtype, what=""):
    atol, rtol = TOL[kv_dtype]
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance; "
                           f"max err {err.max():.3e}, worst ratio {(err / bound).max():.2f}")
    return float(err.max())


def make_engine(w, device="cuda", growth=0, k_scale=1.0, v_scale=1.0):
    """Engine sized for the workload's context lengths plus `growth` more tokens each."""
    MB = w.max_blocks_per_seq(growth)
    return DecodeEngine(num_seqs=w.num_seqs, num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads,
                        head_dim=w.head_dim, block_size=w.block_size, kv_dtype=w.kv_dtype,
                        q_dtype=w.q_dtype, num_blocks=w.num_blocks, initial_order=w.initial_order,
                        max_blocks_per_seq=MB, max_context_len=w.max_context_len + growth, scale=w.scale,
                        k_scale=k_scale, v_scale=v_scale, device=device)


def fill_cache(w, eng):
    """Seeded N(0,1) cache contents, drawn on the engine's device."""
    if w.kv_dtype == "e4m3":
        kc, ks = synthetic.normal_e4m3_codes(tuple(eng.k_cache.shape), w.seed * 10 + 1, eng.device)
        vc, vs = synthetic.normal_e4m3_codes(tuple(eng.v_cache.shape), w.seed * 10 + 2, eng.device)
        eng.k_cache.copy_(kc)
        eng.v_cache.copy_(vc)
        del kc, vc
        eng.cache.desc.k_scale = ks
        eng.cache.desc.v_scale = vs
    else:
        synthetic.fill_normal_(eng.k_cache, w.kv_dtype, w.seed * 10 + 1)
        synthetic.fill_normal_(eng.v_cache, w.kv_dtype, w.seed * 10 + 2)


class OracleMirror:
    """The oracle's own view of the same workload: pool model, tables, cache codes
    of the blocks it needs, and float64 attention."""

    def __init__(self, w):
        self.w = w
        self.pool = BlockPool(w.num_blocks, w.initial_order)
        self.rows = [[] for _ in range(w.num_seqs)]
        self.lens = [0] * w.num_seqs

    def extend(self, s, n):
        slots, cows = self.pool.seq_extend(self.rows[s], self.lens[s], n, self.w.block_size)
        self.lens[s] += n
        return slots, cows

    def fork(self, parent, child):
        self.rows[child] = self.pool.fork(self.rows[parent])
        self.lens[child] = self.lens[parent]

    def step_bookkeeping(self):
        pos = list(self.lens)
        slots, cows, upd = self.pool.batch_append(self.rows, pos, self.w.block_size)
        self.lens = [L + 1 for L in self.lens]
        return slots, cows, upd

    def table(self, MB):
        bt = np.zeros((self.w.num_seqs, MB), dtype=np.int32)
        for s, r in enumerate(self.rows):
            bt[s, :len(r)] = r
        return bt


def check_tables(eng, mirror):
    """Host block tables, lengths and reference counts of the C++ pool equal the oracle's."""
    w = mirror.w
    for s in range(w.num_seqs):
        n = len(mirror.rows[s])
        assert eng.bt_host[s, :n].tolist() == mirror.rows[s], f"block table of seq {s}"
        assert int(eng.lens[s]) == mirror.lens[s]
    assert eng.pool.num_free() == mirror.pool.num_free()
    assert eng.pool.free_list() == mirror.pool.free_list()
    for b in range(w.num_blocks):
        assert eng.pool.refcount(b) == mirror.pool.refcnt[b]


def run_decode_step(w, sample_heads=None, sample_seqs=None, growth=0, device="cuda", nan_tails=False):
    """History of L-1 tokens per sequence, then one full step that appends the
    last token and decodes over L (with nan_tails, every cache byte past the contexts
    is NaN before the step). Returns (max error, engine)."""
    eng = make_engine(w, device, growth=growth)
    fill_cache(w, eng)
    mir = OracleMirror(w)
    for s, L in enumerate(w.context_lens):
        eng.extend(s, L - 1)
        mir.extend(s, L - 1)
    check_tables(eng, mir)
    eng.upload_tables()
    if nan_tails:
        nan_past_contexts_(w, eng)
    slots_o, cows_o, _ = mir.step_bookkeeping()
    assert cows_o == []
    seqs = range(w.num_seqs) if sample_seqs is None else sample_seqs
    blocks = sorted({b for s in seqs for b in mir.rows[s]})
    idx = torch.tensor(blocks, dtype=torch.int64, device=device)
    k0 = codes_np(eng.k_cache.index_select(0, idx))          # the oracle's copy, before the step
    v0 = codes_np(eng.v_cache.index_select(0, idx))
    q, k, v = synthetic.step_inputs(w, 0)
    qd, kd, vd = q.to(device), k.to(device), v.to(device)
    out = torch.full_like(qd, float("nan"))
    eng.step(qd, kd, vd, out, w.scale)
    torch.cuda.synchronize()
    assert pa.last_device_error()[0] == 0
    check_tables(eng, mir)
    # the oracle writes the new tokens into its copy (slots remapped to the copied blocks)
    remap = {b: i for i, b in enumerate(blocks)}
    BS = w.block_size
    sl = np.array([remap[s_ // BS] * BS + s_ % BS if (s_ // BS) in remap else -1 for s_ in slots_o])
    ks, vs = eng.cache.desc.k_scale, eng.cache.desc.v_scale
    ek, ev = oops.reshape_and_cache(codes_np(k), codes_np(v), w.q_dtype, sl, k0, v0, w.kv_dtype, ks, vs)
    assert np.array_equal(codes_np(eng.k_cache.index_select(0, idx)), ek), "K cache after the step"
    assert np.array_equal(codes_np(eng.v_cache.index_select(0, idx)), ev), "V cache after the step"
    bt = np.zeros((w.num_seqs, eng.MB), np.int64)
    for s in seqs:
        bt[s, :len(mir.rows[s])] = [remap[b] for b in mir.rows[s]]
    heads = [(s, h) for s in seqs for h in (range(w.num_q_heads) if sample_heads is None else sample_heads)]
    ref = oatt.paged_decode(codes_np(q), w.q_dtype, ek, ev, w.kv_dtype, ks, vs, bt, mir.lens, w.scale,
                            heads=heads)
    got = out.double().cpu().numpy()
    hs = tuple(np.array(heads).T)
    return assert_close(got[hs], ref[hs], w.kv_dtype, w.name), eng


def run_prefill_case(lens, Hq, Hkv, BS, dt, seed, nrows, device="cuda"):
    """pa_prefill of whole prompts into a NaN-filled cache: every prompt slot bit-exact
    against the oracle's reshape_and_cache, sampled outputs against its paged_extend."""
    D = 128
    w = synthetic.custom(len(lens), Hq, Hkv, D, BS, dt, dt, lens, seed)
    eng = make_engine(w, device)
    eng.k_cache.fill_(float("nan"))
    eng.v_cache.fill_(float("nan"))
    k0, v0 = codes_np(eng.k_cache), codes_np(eng.v_cache)
    for s, L in enumerate(lens):
        eng.extend(s, L)
    eng.upload_tables()
    qs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(qs[-1])
    q = synthetic.normal_values((T, Hq, D), dt, seed + 7).to(device)
    k = synthetic.normal_values((T, Hkv, D), dt, seed + 8).to(device)
    v = synthetic.normal_values((T, Hkv, D), dt, seed + 9).to(device)
    out = torch.full_like(q, float("nan"))
    ws = torch.empty(pa.extend_workspace_size(w.num_seqs, T, Hq, D, eng.max_context_len), dtype=torch.uint8,
                     device=device)
    pa.prefill(q, k, v, eng.cache, torch.from_numpy(qs).to(device), eng.bt_dev, eng.lens_dev, eng.max_context_len,
               w.scale, out, ws)
    torch.cuda.synchronize()
    assert pa.last_device_error()[0] == 0

    # the oracle's cache: the same prompt tokens written through its reshape_and_cache
    bt = eng.bt_host.astype(np.int64)
    slots = np.concatenate([bt[s, np.arange(L) // BS] * BS + np.arange(L) % BS for s, L in enumerate(lens)])
    kc, vc = oops.reshape_and_cache(codes_np(k), codes_np(v), dt, slots, k0, v0, dt)
    gk, gv = codes_np(eng.k_cache), codes_np(eng.v_cache)
    blk, off = slots // BS, slots % BS
    assert np.array_equal(gk[blk, :, off, :], kc[blk, :, off, :]), "k slots"
    assert np.array_equal(gv[blk, :, off, :], vc[blk, :, off, :]), "v slots"

    rng = np.random.default_rng(seed)
    rows = {(int(t), int(h)) for t, h in zip(rng.integers(0, T, nrows), rng.integers(0, Hq, nrows))}
    for s in range(len(lens)):
        for t in (int(qs[s]), int(qs[s + 1]) - 1):
            rows.update((t, h) for h in range(Hq))
    rows = sorted(rows)
    ref = oatt.paged_extend(codes_np(q), dt, kc, vc, dt, 1.0, 1.0, bt, list(lens), qs, w.scale, rows=rows)
    idx = tuple(np.array(rows).T)
    got = out.double().cpu().numpy()
    assert np.isfinite(got[idx]).all()
    err = assert_close(got[idx], ref[idx], dt, f"prefill {dt} BS{BS} G{Hq // Hkv}")
    # the first token of every prompt sees itself only: its output is its V row exactly
    for s in range(len(lens)):
        t = int(qs[s])
        for h in range(Hq):
            assert torch.equal(out[t, h], v[t, h // (Hq // Hkv)])
    return err


# ---------------------------------------------------------------------------
# every output row at full size: the oracle on all host cores
# ---------------------------------------------------------------------------
# Large caches go to the oracle through shared memory, and the oracle runs in a pool of
# spawned processes (one per host core, one BLAS thread each) over whole sequences;
# spawn is safe after CUDA is initialised in this process (a fork is not).

def _shared_codes(shape, itemsize):
    """A zeroed shared-memory block holding an unsigned code array of `shape`."""
    from multiprocessing import shared_memory
    n = int(np.prod(shape)) * itemsize
    shm = shared_memory.SharedMemory(create=True, size=max(n, 1))
    arr = np.ndarray(shape, dtype=np.uint8 if itemsize == 1 else np.uint16, buffer=shm.buf)
    return shm, arr


def _device_to_shared(t):
    """Copy a device tensor's codes into shared memory (no intermediate host copy)."""
    shm, arr = _shared_codes(tuple(t.shape), t.element_size())
    dst = torch.from_numpy(arr.view(np.uint8) if t.element_size() == 1 else arr.view(np.int16))
    src = t.view(torch.uint8) if t.element_size() == 1 else t.view(torch.int16)
    step = max(1, (1 << 28) // max(1, src[0].numel() * t.element_size()))
    for i in range(0, t.shape[0], step):
        dst[i:i + step].copy_(src[i:i + step])
    return shm, arr


def _oracle_worker(task):
    """One process of the pool: the oracle rows of some sequences, caches read from
    shared memory. task = (kind, shm names, shapes, itemsize, args, rows)."""
    import os
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"
    from multiprocessing import shared_memory
    from threadpoolctl import threadpool_limits
    from oracle import attention as oatt_w
    kind, names, shape, itemsize, args, rows = task
    dt = np.uint8 if itemsize == 1 else np.uint16
    shms = [shared_memory.SharedMemory(name=n) for n in names]
    try:
        kc, vc = (np.ndarray(shape, dtype=dt, buffer=s.buf) for s in shms)
        with threadpool_limits(limits=1):
            if kind == "decode":
                q, qd, kvd, ks, vs, bt, lens, scale = args
                out = oatt_w.paged_decode(q, qd, kc, vc, kvd, ks, vs, bt, lens, scale, heads=rows)
            else:
                q, qd, kvd, ks, vs, bt, lens, qs, scale = args
                out = oatt_w.paged_extend(q, qd, kc, vc, kvd, ks, vs, bt, lens, qs, scale, rows=rows)
        idx = tuple(np.array(rows).T)
        return rows, out[idx]
    finally:
        for s in shms:
            s.close()


def oracle_rows_parallel(kind, shm_k, shm_v, shape, itemsize, args, groups):
    """The oracle's rows for every group of (row, head) pairs, one group per task, on
    one spawned process per host core. Returns {(row, head): float64 vector}."""
    import multiprocessing as mp
    import os
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    tasks = [(kind, (shm_k.name, shm_v.name), shape, itemsize, args, g) for g in groups if g]
    res = {}
    with mp.get_context("spawn").Pool(processes=max(1, min(cores, len(tasks)))) as pool:
        for rows, vals in pool.imap_unordered(_oracle_worker, tasks):
            for r, v in zip(rows, vals):
                res[tuple(r)] = v
    return res


def nan_code(kv_dtype):
    """The code of a NaN in the cache's format (E4M3: S.1111.111)."""
    return 0x7F if kv_dtype == "e4m3" else 0x7FC0 if kv_dtype == "bf16" else 0x7E00


def fill_nan_(t, kv_dtype):
    """Set every element of a cache slice to NaN."""
    if t.element_size() == 1:
        t.view(torch.uint8).fill_(nan_code(kv_dtype))
    else:
        t.view(torch.int16).fill_(nan_code(kv_dtype))


def nan_past_contexts_(w, eng):
    """Before a step: the cache bytes past every sequence's context (the rest of its last
    block) and every block no sequence holds (the step may take one) become NaN. Memory
    the pool handed out but nothing wrote may hold anything; no output may depend on it."""
    BS = w.block_size
    held = np.zeros(w.num_blocks, bool)
    for s in range(w.num_seqs):
        n = int(eng.lens[s])
        held[eng.bt_host[s, :-(-n // BS)]] = True
        if n % BS:
            b = int(eng.bt_host[s, (n - 1) // BS])
            fill_nan_(eng.k_cache[b, :, n % BS:, :], w.kv_dtype)
            fill_nan_(eng.v_cache[b, :, n % BS:, :], w.kv_dtype)
    free = torch.from_numpy(np.nonzero(~held)[0]).to(eng.device)
    if free.numel():
        for c in (eng.k_cache, eng.v_cache):
            sub = c.index_select(0, free)
            fill_nan_(sub, w.kv_dtype)
            c.index_copy_(0, free, sub)


def run_decode_step_all_rows(w, device="cuda", nan_tails=True):
    """One full decode step of the workload (history of L-1 tokens, then the step that
    appends the last token and decodes over L) with EVERY (sequence, q head) output row
    compared against the oracle, which runs on all host cores. Cache bytes past every
    context (the rest of each last block, and every free block the step may take) are
    NaN first. The whole cache after the step is compared bit for bit with the oracle's
    (the pre-step cache plus the oracle's own writes of the new tokens)."""
    eng = make_engine(w, device)
    fill_cache(w, eng)
    mir = OracleMirror(w)
    for s, L in enumerate(w.context_lens):
        eng.extend(s, L - 1)
        mir.extend(s, L - 1)
    check_tables(eng, mir)
    eng.upload_tables()
    BS = w.block_size
    if nan_tails:
        nan_past_contexts_(w, eng)
    torch.cuda.synchronize()
    # the oracle's copy of the whole cache before the step, in shared memory
    shm_k, ek = _device_to_shared(eng.k_cache)
    shm_v, ev = _device_to_shared(eng.v_cache)
    try:
        slots_o, cows_o, _ = mir.step_bookkeeping()
        assert cows_o == []
        q, k, v = synthetic.step_inputs(w, 0)
        out = torch.full((w.num_seqs, w.num_q_heads, w.head_dim), float("nan"), dtype=q.dtype, device=device)
        eng.step(q.to(device), k.to(device), v.to(device), out, w.scale)
        torch.cuda.synchronize()
        assert pa.last_device_error()[0] == 0
        check_tables(eng, mir)
        ks, vs = eng.cache.desc.k_scale, eng.cache.desc.v_scale
        # the oracle writes the new tokens into its copy, one block at a time
        kn, vn = codes_np(k), codes_np(v)
        for t, slot in enumerate(slots_o):
            b, off = slot // BS, slot % BS
            nk, nv = oops.reshape_and_cache(kn[t:t + 1], vn[t:t + 1], w.q_dtype, [off], ek[b:b + 1], ev[b:b + 1],
                                            w.kv_dtype, ks, vs)
            ek[b], ev[b] = nk[0], nv[0]
        # the device cache after the step equals the oracle's, bit for bit
        step = max(1, (1 << 28) // (ek[0].size * ek.itemsize))
        for c, e in ((eng.k_cache, ek), (eng.v_cache, ev)):
            for i in range(0, w.num_blocks, step):
                assert np.array_equal(codes_np(c[i:i + step]), e[i:i + step]), f"cache blocks {i}.. after the step"
        bt = mir.table(eng.MB).astype(np.int64)
        args = (codes_np(q), w.q_dtype, w.kv_dtype, ks, vs, bt, list(mir.lens), w.scale)
        # one task per sequence (all its heads), longest first
        order = sorted(range(w.num_seqs), key=lambda s: -mir.lens[s])
        groups = [[(s, h) for h in range(w.num_q_heads)] for s in order]
        ref = oracle_rows_parallel("decode", shm_k, shm_v, ek.shape, ek.itemsize, args, groups)
    finally:
        for shm in (shm_k, shm_v):
            shm.close()
            shm.unlink()
    got = out.double().cpu().numpy()
    keys = sorted(ref)
    want = np.stack([ref[r] for r in keys])
    idx = tuple(np.array(keys).T)
    assert len(keys) == w.num_seqs * w.num_q_heads
    return assert_close(got[idx], want, w.kv_dtype, f"{w.name}: every row"), eng
