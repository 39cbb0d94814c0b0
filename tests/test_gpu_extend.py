"""GPU parity of pa_extend (several new tokens per sequence, causal over the paged
context) against the float64 oracle: |err| <= 2e-3 + 1e-2 |ref| for 16-bit caches."""

import zlib

import numpy as np
import pytest
import torch

import paged_kv_cache_436_b200 as pa
import synthetic
from oracle import attention as oatt
from tests.gpu_cases import assert_close, codes_np, fill_cache, make_engine

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _setup(lens, qlens, Hq, Hkv, D, BS, dt, seed):
    w = synthetic.custom(len(lens), Hq, Hkv, D, BS, dt, dt, lens, seed)
    eng = make_engine(w, DEV)
    fill_cache(w, eng)
    for s, L in enumerate(lens):
        eng.extend(s, L)
    eng.upload_tables()
    qs = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    T = int(qs[-1])
    q = synthetic.normal_values((T, Hq, D), dt, seed + 7).to(DEV)
    return w, eng, torch.from_numpy(qs).to(DEV), q, qs


def _run(w, eng, qs_dev, q, qs_host):
    T, Hq, D = q.shape
    out = torch.full_like(q, float("nan"))
    ws = torch.empty(pa.extend_workspace_size(w.num_seqs, T, Hq, D, eng.max_context_len), dtype=torch.uint8,
                     device=DEV)
    pa.extend(q, eng.cache, qs_dev, eng.bt_dev, eng.lens_dev, eng.max_context_len, w.scale, out, ws)
    torch.cuda.synchronize()
    return out


def _ref(w, eng, q, qs_host, rows=None):
    bt = eng.bt_host.astype(np.int64)
    return oatt.paged_extend(codes_np(q), w.q_dtype, codes_np(eng.k_cache), codes_np(eng.v_cache), w.kv_dtype,
                             1.0, 1.0, bt, list(eng.lens), qs_host, w.scale, rows=rows)


@pytest.mark.parametrize("dt,D,BS,G", [("bf16", 128, 16, 1), ("f16", 128, 16, 1), ("bf16", 128, 32, 4),
                                       ("f16", 64, 16, 2), ("bf16", 64, 32, 8), ("bf16", 128, 16, 8)])
def test_extend_matches_oracle(dt, D, BS, G):
    lens = [1, 5, 17, 511, 512, 513, 530, 1030, 1600]
    qlens = [1, 5, 3, 8, 2, 7, 1, 16, 13]
    seed = zlib.crc32(repr((dt, D, BS, G)).encode()) % 10000
    w, eng, qs_dev, q, qs = _setup(lens, qlens, 2 * G, 2, D, BS, dt, seed)
    out = _run(w, eng, qs_dev, q, qs)
    assert pa.last_device_error()[0] == 0
    ref = _ref(w, eng, q, qs)
    assert_close(out.double().cpu().numpy(), ref, dt, f"extend {dt} D{D} BS{BS} G{G}")


def test_chunked_prefill_matches_oracle():
    """A whole 700-token prompt as queries (prefill), and a 150-token chunk over a
    1300-token context (chunked prefill), with GQA."""
    lens, qlens = [700, 1300], [700, 150]
    w, eng, qs_dev, q, qs = _setup(lens, qlens, 8, 2, 128, 16, "bf16", 31)
    out = _run(w, eng, qs_dev, q, qs)
    assert pa.last_device_error()[0] == 0
    rng = np.random.default_rng(5)
    rows = [(int(t), int(h)) for t in rng.choice(850, size=120, replace=False) for h in (0, 3, 7)]
    rows += [(0, h) for h in range(8)] + [(699, 1), (700, 2), (849, 5)]
    ref = _ref(w, eng, q, qs, rows=rows)
    got = out.double().cpu().numpy()
    idx = tuple(np.array(rows).T)
    assert_close(got[idx], ref[idx], "bf16", "chunked prefill")
    # query 0 of the prompt sees token 0 only: out = that V row, rounded once
    v0 = eng.v_cache[int(eng.bt_host[0, 0]), :, 0, :].float().cpu()
    for h in range(8):
        assert torch.equal(out[0, h].float().cpu(), v0[h // 4])


def test_single_query_extend_agrees_with_decode():
    lens = [40, 600, 1500, 3]
    w, eng, qs_dev, q, qs = _setup(lens, [1, 1, 1, 1], 8, 2, 128, 16, "bf16", 41)
    ext = _run(w, eng, qs_dev, q, qs)
    dec = torch.empty_like(q)
    eng.run_decode(q, dec)
    torch.cuda.synchronize()
    a, b = ext.double().cpu().numpy(), dec.double().cpu().numpy()
    assert np.all(np.abs(a - b) <= 2e-3 + 1e-2 * np.abs(b))


def test_more_queries_than_context_is_recorded_and_zero():
    lens, qlens = [10, 20], [3, 4]
    w, eng, qs_dev, q, qs = _setup(lens, qlens, 4, 4, 64, 16, "f16", 51)
    eng.lens_dev.copy_(torch.tensor([2, 20], dtype=torch.int32))     # sequence 0: 3 queries, 2 tokens
    out = _run(w, eng, qs_dev, q, qs)
    code, info = pa.last_device_error()
    assert code == 2 and info[0] == 0
    assert torch.count_nonzero(out[:3]) == 0 and torch.isfinite(out[3:].float()).all()


def _nan_tails(w, eng):
    """Cache bytes past each context in its last block set to NaN (the E4M3 NaN code for an
    E4M3 cache): memory that was never written may hold anything, and no output may
    depend on it."""
    from tests.gpu_cases import fill_nan_
    BS = w.block_size
    for s, L in enumerate(eng.lens):
        if L % BS:
            b = int(eng.bt_host[s, (L - 1) // BS])
            fill_nan_(eng.k_cache[b, :, L % BS:, :], w.kv_dtype)
            fill_nan_(eng.v_cache[b, :, L % BS:, :], w.kv_dtype)


def _sample_rows(qs, Hq, n, seed):
    """Random (token, head) rows plus the first and last query of every sequence."""
    T = int(qs[-1])
    rng = np.random.default_rng(seed)
    rows = {(int(t), int(h)) for t, h in zip(rng.integers(0, T, n), rng.integers(0, Hq, n))}
    for s in range(len(qs) - 1):
        if qs[s + 1] > qs[s]:
            for t in (int(qs[s]), int(qs[s + 1]) - 1):
                rows.update((t, h) for h in range(Hq))
    return sorted(rows)


def _check_rows(w, eng, q, qs, out, rows, what):
    ref = _ref(w, eng, q, qs, rows=rows)
    idx = tuple(np.array(rows).T)
    got = out.double().cpu().numpy()
    assert np.isfinite(got[idx]).all(), what
    assert_close(got[idx], ref[idx], w.kv_dtype, what)


@pytest.mark.parametrize("dt,BS,G", [("bf16", 16, 1), ("f16", 16, 2), ("bf16", 32, 4), ("f16", 32, 8),
                                     ("bf16", 16, 8), ("f16", 16, 1)])
def test_long_runs_split_context(dt, BS, G):
    """Long query runs (the 128-row tensor-core path): whole prompts, a chunk over a
    longer context, a single query and a two-token draft in one batch; few units, so
    the context is split into chunks merged by log-sum-exp. NaN past every context."""
    lens = [130, 700, 1025, 257, 1, 1500]
    qlens = [130, 700, 300, 257, 1, 2]
    seed = zlib.crc32(repr(("long", dt, BS, G)).encode()) % 10000
    w, eng, qs_dev, q, qs = _setup(lens, qlens, 2 * G, 2, 128, BS, dt, seed)
    _nan_tails(w, eng)
    out = _run(w, eng, qs_dev, q, qs)
    assert pa.last_device_error()[0] == 0
    _check_rows(w, eng, q, qs, out, _sample_rows(qs, 2 * G, 160, seed), f"long runs {dt} BS{BS} G{G}")


def test_long_runs_whole_context_per_unit():
    """Enough 128-row tiles to fill the GPU: every unit covers its rows' whole context
    and writes the output directly (no merge pass)."""
    lens = [1200, 1100, 1000, 1200]
    w, eng, qs_dev, q, qs = _setup(lens, lens, 8, 8, 128, 16, "bf16", 77)
    _nan_tails(w, eng)
    out = _run(w, eng, qs_dev, q, qs)
    assert pa.last_device_error()[0] == 0
    _check_rows(w, eng, q, qs, out, _sample_rows(qs, 8, 200, 77), "whole-context units")
    # query 0 of each prompt sees its token 0 only: the output is that V row exactly
    for s in range(len(lens)):
        v0 = eng.v_cache[int(eng.bt_host[s, 0]), :, 0, :]
        assert torch.equal(out[int(qs[s])], v0)


def test_prefill_8x2k_sampled():
    """The benchmarked prefill shapes (8 prompts of 2048 tokens, 32 heads, head_dim 128,
    bf16, 16-token blocks), checked on sampled rows."""
    w, eng, qs_dev, q, qs = _setup([2048] * 8, [2048] * 8, 32, 32, 128, 16, "bf16", 4371)
    out = _run(w, eng, qs_dev, q, qs)
    assert pa.last_device_error()[0] == 0
    _check_rows(w, eng, q, qs, out, _sample_rows(qs, 32, 120, 4371), "prefill 8x2k")


def test_short_runs_ignore_bytes_past_the_context():
    """The 16- and 64-row kernels never let cache bytes past the context reach P V."""
    lens, qlens = [37, 530, 1031], [3, 5, 2]                 # 16-row warp kernel
    w, eng, qs_dev, q, qs = _setup(lens, qlens, 4, 2, 128, 16, "bf16", 91)
    _nan_tails(w, eng)
    out = _run(w, eng, qs_dev, q, qs)
    assert pa.last_device_error()[0] == 0
    _check_rows(w, eng, q, qs, out, _sample_rows(qs, 4, 0, 91) + [(1, 1), (6, 3)], "warp kernel tails")
    lens, qlens = [300, 77], [200, 60]                       # 64-row cooperative kernel (head_dim 64)
    w, eng, qs_dev, q, qs = _setup(lens, qlens, 4, 2, 64, 16, "f16", 92)
    _nan_tails(w, eng)
    out = _run(w, eng, qs_dev, q, qs)
    assert pa.last_device_error()[0] == 0
    _check_rows(w, eng, q, qs, out, _sample_rows(qs, 4, 80, 92), "cooperative kernel tails")


def _compact(eng, seqs, BS):
    """The oracle's copy of the blocks of `seqs` (host codes) and block tables remapped to it."""
    lens = list(eng.lens)
    blocks = sorted({int(b) for s in seqs for b in eng.bt_host[s, :-(-lens[s] // BS)]})
    idx = torch.tensor(blocks, dtype=torch.int64, device=DEV)
    kc, vc = codes_np(eng.k_cache.index_select(0, idx)), codes_np(eng.v_cache.index_select(0, idx))
    remap = {b: i for i, b in enumerate(blocks)}
    bt = np.zeros(eng.bt_host.shape, np.int64)
    for s in seqs:
        nb = -(-lens[s] // BS)
        bt[s, :nb] = [remap[int(b)] for b in eng.bt_host[s, :nb]]
    return kc, vc, bt, lens


def test_spec4_mix_every_row():
    """The benchmarked speculative-verification shapes: 4 draft tokens per sequence over the
    13B mixed-length contexts (256 sequences, 40/40 heads, bf16). EVERY (query, head) row
    against the oracle on all host cores; NaN past every context."""
    from tests.gpu_cases import _device_to_shared, nan_past_contexts_, oracle_rows_parallel
    w = synthetic.make("llama13b_mix")
    eng = make_engine(w, DEV)
    fill_cache(w, eng)
    for s, L in enumerate(w.context_lens):
        eng.extend(s, L)
    eng.upload_tables()
    nan_past_contexts_(w, eng)
    qlens = [min(4, L) for L in w.context_lens]
    qs = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = synthetic.normal_values((int(qs[-1]), w.num_q_heads, w.head_dim), w.q_dtype, w.seed + 11).to(DEV)
    out = _run(w, eng, torch.from_numpy(qs).to(DEV), q, qs)
    assert pa.last_device_error()[0] == 0
    shm_k, kc = _device_to_shared(eng.k_cache)
    shm_v, vc = _device_to_shared(eng.v_cache)
    try:
        args = (codes_np(q), w.q_dtype, w.kv_dtype, 1.0, 1.0, eng.bt_host.astype(np.int64), list(eng.lens), qs,
                w.scale)
        order = sorted(range(w.num_seqs), key=lambda s_: -int(eng.lens[s_]))
        groups = [[(t, h) for t in range(int(qs[s_]), int(qs[s_ + 1])) for h in range(w.num_q_heads)]
                  for s_ in order]
        ref = oracle_rows_parallel("extend", shm_k, shm_v, kc.shape, kc.itemsize, args, groups)
    finally:
        for shm in (shm_k, shm_v):
            shm.close()
            shm.unlink()
    keys = sorted(ref)
    assert len(keys) == int(qs[-1]) * w.num_q_heads
    idx = tuple(np.array(keys).T)
    want = np.stack([ref[r] for r in keys])
    assert_close(out.double().cpu().numpy()[idx], want, w.kv_dtype, "spec4 mix, every row")


@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
def test_repeated_calls_share_one_workspace(kv):
    """The short-run kernels' warps take their units from a counter in the workspace that the
    plan kernel zeroes on every call: three calls with one workspace (and a different draft
    count in between) give bit-identical outputs, each against the oracle."""
    lens = [3, 40, 511, 512, 900, 1500, 2100, 64]
    w = synthetic.custom(len(lens), 4, 4, 128, 16 if kv == "bf16" else 32, kv, "bf16", lens, 91)
    eng = make_engine(w, DEV)
    fill_cache(w, eng)   # E4M3: codes with per-tensor scales
    for s, L in enumerate(lens):
        eng.extend(s, L)
    eng.upload_tables()
    _nan_tails(w, eng)
    T_max = 4 * len(lens)
    ws = torch.empty(pa.extend_workspace_size(w.num_seqs, T_max, 4, 128, eng.max_context_len), dtype=torch.uint8,
                     device=DEV)

    def call(qlens, seed):
        qs = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
        q = synthetic.normal_values((int(qs[-1]), 4, 128), "bf16", seed).to(DEV)
        out = torch.full_like(q, float("nan"))
        pa.extend(q, eng.cache, torch.from_numpy(qs).to(DEV), eng.bt_dev, eng.lens_dev, eng.max_context_len, w.scale,
                  out, ws)
        torch.cuda.synchronize()
        assert pa.last_device_error()[0] == 0
        return q, qs, out

    qlens = [min(4, L) for L in lens]
    q, qs, first = call(qlens, 92)
    _, _, other = call([1] * len(lens), 93)
    _, _, again = call(qlens, 92)
    assert torch.equal(first, again)
    d = eng.cache.desc
    want = oatt.paged_extend(codes_np(q), "bf16", codes_np(eng.k_cache), codes_np(eng.v_cache), w.kv_dtype,
                             d.k_scale, d.v_scale, eng.bt_host.astype(np.int64), list(eng.lens), qs, w.scale)
    assert_close(again.double().cpu().numpy(), want, w.kv_dtype, f"repeated extend calls, {kv} cache")
    assert torch.isfinite(other).all()


def test_ragged_and_empty_batches():
    """Sequences with no new token between others (ragged query_start), and a call with no
    token at all: the others' rows match the oracle; the empty call is a no-op."""
    lens = [9, 600, 33, 1200, 2]
    qlens = [3, 0, 5, 0, 2]
    w, eng, qs_dev, q, qs = _setup(lens, qlens, 8, 2, 128, 16, "bf16", 95)
    out = _run(w, eng, qs_dev, q, qs)
    assert pa.last_device_error()[0] == 0
    assert_close(out.double().cpu().numpy(), _ref(w, eng, q, qs), "bf16", "ragged batch")
    empty_q, empty_out = q[:0], out[:0]   # views: the pointers stay valid
    qs0 = torch.zeros(len(lens) + 1, dtype=torch.int32, device=DEV)
    ws = torch.empty(pa.extend_workspace_size(w.num_seqs, 1, 8, 128, eng.max_context_len), dtype=torch.uint8,
                     device=DEV)
    pa.extend(empty_q, eng.cache, qs0, eng.bt_dev, eng.lens_dev, eng.max_context_len, w.scale, empty_out, ws)
    torch.cuda.synchronize()
    assert pa.last_device_error()[0] == 0


def test_long_context_many_chunks():
    """A 256-query chunk at the end of a 20000-token context, GQA 4: few units, so the
    context is cut into many chunks merged by log-sum-exp."""
    lens, qlens = [20000], [256]
    w, eng, qs_dev, q, qs = _setup(lens, qlens, 8, 2, 128, 16, "bf16", 97)
    _nan_tails(w, eng)
    out = _run(w, eng, qs_dev, q, qs)
    assert pa.last_device_error()[0] == 0
    _check_rows(w, eng, q, qs, out, _sample_rows(qs, 8, 60, 97), "20000-token context")


# ---------------------------------------------------------------------------
# E4M3 caches
# ---------------------------------------------------------------------------

def _ref_scaled(w, eng, q, qs_host, rows=None):
    d = eng.cache.desc
    bt = eng.bt_host.astype(np.int64)
    return oatt.paged_extend(codes_np(q), w.q_dtype, codes_np(eng.k_cache), codes_np(eng.v_cache), w.kv_dtype,
                             d.k_scale, d.v_scale, bt, list(eng.lens), qs_host, w.scale, rows=rows)


@pytest.mark.parametrize("qd,D,BS,G", [("bf16", 128, 32, 1), ("f16", 128, 16, 4), ("bf16", 64, 16, 2),
                                       ("f16", 64, 32, 8), ("bf16", 128, 16, 8)])
def test_extend_e4m3_cache_matches_oracle(qd, D, BS, G):
    """Draft runs of 1-16 tokens over an E4M3 cache (codes of N(0, 1) draws with a
    per-tensor scale), partition edges and NaN codes past every context: every element
    within 3e-2 + 3e-2 |ref|."""
    lens = [1, 5, 17, 511, 512, 513, 530, 1030, 1600]
    qlens = [1, 5, 3, 8, 2, 7, 1, 16, 13]
    seed = zlib.crc32(repr(("e4m3", qd, D, BS, G)).encode()) % 10000
    w = synthetic.custom(len(lens), 2 * G, 2, D, BS, "e4m3", qd, lens, seed)
    eng = make_engine(w, DEV)
    fill_cache(w, eng)
    for s, L in enumerate(lens):
        eng.extend(s, L)
    eng.upload_tables()
    _nan_tails(w, eng)
    qs = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = synthetic.normal_values((int(qs[-1]), 2 * G, D), qd, seed + 7).to(DEV)
    out = _run(w, eng, torch.from_numpy(qs).to(DEV), q, qs)
    assert pa.last_device_error()[0] == 0
    assert_close(out.double().cpu().numpy(), _ref_scaled(w, eng, q, qs), "e4m3", f"extend e4m3 {qd} D{D} BS{BS} G{G}")


def test_extend_e4m3_long_runs_and_chunks():
    """Long query runs over an E4M3 cache (a whole 700-token prompt, a 300-token chunk over
    1300 tokens, a 256-token chunk at the end of 6000 tokens): the same kernel, merged
    across 512-token partitions; sampled rows."""
    lens, qlens = [700, 1300, 6000], [700, 300, 256]
    w = synthetic.custom(3, 8, 2, 128, 32, "e4m3", "bf16", lens, 61)
    eng = make_engine(w, DEV)
    fill_cache(w, eng)
    for s, L in enumerate(lens):
        eng.extend(s, L)
    eng.upload_tables()
    _nan_tails(w, eng)
    qs = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = synthetic.normal_values((int(qs[-1]), 8, 128), "bf16", 68).to(DEV)
    out = _run(w, eng, torch.from_numpy(qs).to(DEV), q, qs)
    assert pa.last_device_error()[0] == 0
    rows = _sample_rows(qs, 8, 200, 61)
    ref = _ref_scaled(w, eng, q, qs, rows=rows)
    idx = tuple(np.array(rows).T)
    assert_close(out.double().cpu().numpy()[idx], ref[idx], "e4m3", "e4m3 long runs")


def test_extend_e4m3_single_query_agrees_with_decode():
    """One query per sequence over an E4M3 cache: pa_extend and pa_decode compute the same
    rows (within the E4M3 tolerance of each other)."""
    lens = [40, 600, 1500, 3]
    w = synthetic.custom(4, 8, 2, 128, 32, "e4m3", "bf16", lens, 63)
    eng = make_engine(w, DEV)
    fill_cache(w, eng)
    for s, L in enumerate(lens):
        eng.extend(s, L)
    eng.upload_tables()
    qs = np.arange(5, dtype=np.int32)
    q = synthetic.normal_values((4, 8, 128), "bf16", 64).to(DEV)
    ext = _run(w, eng, torch.from_numpy(qs).to(DEV), q, qs)
    dec = torch.empty_like(q)
    eng.run_decode(q, dec)
    torch.cuda.synchronize()
    a, b = ext.double().cpu().numpy(), dec.double().cpu().numpy()
    assert np.all(np.abs(a - b) <= 3e-2 + 3e-2 * np.abs(b))


def test_spec4_long_fp8_every_row():
    """The benchmarked speculative-verification shape over the 32K E4M3 cache: 4 draft tokens
    for each of 8 sequences of 32768 tokens (32/32 heads, 32-token blocks). EVERY (query,
    head) row against the oracle on all host cores, at the E4M3 tolerance."""
    from tests.gpu_cases import _device_to_shared, oracle_rows_parallel
    w = synthetic.make("long_fp8")
    eng = make_engine(w, DEV)
    fill_cache(w, eng)
    for s, L in enumerate(w.context_lens):
        eng.extend(s, L)
    eng.upload_tables()
    qlens = [4] * w.num_seqs
    qs = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = synthetic.normal_values((int(qs[-1]), w.num_q_heads, w.head_dim), w.q_dtype, w.seed + 11).to(DEV)
    out = _run(w, eng, torch.from_numpy(qs).to(DEV), q, qs)
    assert pa.last_device_error()[0] == 0
    d = eng.cache.desc
    shm_k, kc = _device_to_shared(eng.k_cache)
    shm_v, vc = _device_to_shared(eng.v_cache)
    try:
        args = (codes_np(q), w.q_dtype, w.kv_dtype, d.k_scale, d.v_scale, eng.bt_host.astype(np.int64),
                list(eng.lens), qs, w.scale)
        groups = [[(t, h)] for s_ in range(w.num_seqs) for t in range(int(qs[s_]), int(qs[s_ + 1]))
                  for h in range(0, w.num_q_heads, 1)]
        groups = [sum(groups[i:i + 8], []) for i in range(0, len(groups), 8)]
        ref = oracle_rows_parallel("extend", shm_k, shm_v, kc.shape, kc.itemsize, args, groups)
    finally:
        for shm in (shm_k, shm_v):
            shm.close()
            shm.unlink()
    keys = sorted(ref)
    assert len(keys) == int(qs[-1]) * w.num_q_heads
    idx = tuple(np.array(keys).T)
    want = np.stack([ref[r] for r in keys])
    assert_close(out.double().cpu().numpy()[idx], want, "e4m3", "spec4 long fp8, every row")
