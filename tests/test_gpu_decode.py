"""GPU parity of the decode step against the float64 oracle.

Each case builds the workload twice from the same seeded inputs -- through the
CUDA library (C++ pool, device tables, kernels) and through the oracle (its own
pool model, cache ops and attention) -- and compares block tables and cache
bytes exactly and attention outputs within the tolerance of the KV format:
|err| <= 2e-3 + 1e-2 |ref| for fp16/bf16 caches, 3e-2 + 3e-2 |ref| for E4M3.
"""

import zlib

import numpy as np
import pytest
import torch

import paged_kv_cache_436_b200 as pa
import synthetic
from oracle import attention as oatt
from oracle import cache_ops as oops
from tests.gpu_cases import (OracleMirror, assert_close, check_tables, codes_np, fill_cache, make_engine,
                              run_decode_step)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_tiny_config():
    w = synthetic.make("tiny")
    run_decode_step(w)


def test_tiny_extra_slots_into_free_blocks():
    """4 new tokens written into slots of blocks no sequence holds: rows exact, rest untouched."""
    w = synthetic.make("tiny")
    eng = make_engine(w, DEV)
    fill_cache(w, eng)
    for s, L in enumerate(w.context_lens):
        eng.extend(s, L)
    held = {int(b) for s in range(4) for b in eng.bt_host[s, :-(-w.context_lens[s] // 16)]}
    assert not held & {sl // 16 for sl in w.extra_slots}
    k0, v0 = codes_np(eng.k_cache), codes_np(eng.v_cache)
    _, k, v = synthetic.step_inputs(w, 5)
    slots = np.array(w.extra_slots, np.int64)
    pa.reshape_and_cache(k.to(DEV), v.to(DEV), torch.from_numpy(slots).to(DEV), eng.cache)
    ek, ev = oops.reshape_and_cache(codes_np(k), codes_np(v), "f16", slots, k0, v0, "f16")
    assert np.array_equal(codes_np(eng.k_cache), ek) and np.array_equal(codes_np(eng.v_cache), ev)


def test_llama7b_step_config():
    run_decode_step(synthetic.make("llama7b_step"))


def test_gqa_prefix_config():
    """1000-token prefix written once and shared by 64 sequences; 63 copy-on-write
    block copies; private tokens written; decode with 32 q / 8 kv heads."""
    w = synthetic.make("gqa_prefix")
    eng = make_engine(w, DEV)
    fill_cache(w, eng)
    mir = OracleMirror(w)
    P = w.prefix_len
    pre_slots = np.zeros(P, np.int64)
    eng.extend(0, P, pre_slots)
    sl_o, _ = mir.extend(0, P)
    assert pre_slots.tolist() == sl_o
    for s in range(1, w.num_seqs):
        eng.fork(0, s)
        mir.fork(0, s)
    pairs, priv_slots, pairs_o, priv_o = [], [], [], []
    for s, p in enumerate(w.private_lens):
        sl = np.zeros(p, np.int64)
        cs, cd = eng.extend(s, p, sl)
        if cs >= 0:
            pairs.append((cs, cd))
        priv_slots.append(sl)
        so, co = mir.extend(s, p)
        pairs_o += co
        priv_o += so
    assert pairs == pairs_o and len(pairs) == w.num_seqs - 1
    priv_slots = np.concatenate(priv_slots)
    assert priv_slots.tolist() == priv_o
    check_tables(eng, mir)
    eng.upload_tables()
    k0, v0 = codes_np(eng.k_cache), codes_np(eng.v_cache)
    n_priv = int(sum(w.private_lens))
    kp = synthetic.normal_values((P, w.num_kv_heads, w.head_dim), "bf16", w.seed + 101)
    vp = synthetic.normal_values((P, w.num_kv_heads, w.head_dim), "bf16", w.seed + 102)
    kq = synthetic.normal_values((n_priv, w.num_kv_heads, w.head_dim), "bf16", w.seed + 103)
    vq = synthetic.normal_values((n_priv, w.num_kv_heads, w.head_dim), "bf16", w.seed + 104)
    q = synthetic.normal_values((w.num_seqs, w.num_q_heads, w.head_dim), "bf16", w.seed + 105)
    pa.reshape_and_cache(kp.to(DEV), vp.to(DEV), torch.from_numpy(pre_slots).to(DEV), eng.cache)
    pa.copy_blocks(torch.tensor(pairs, dtype=torch.int64, device=DEV), eng.cache)
    pa.reshape_and_cache(kq.to(DEV), vq.to(DEV), torch.from_numpy(priv_slots).to(DEV), eng.cache)
    out = torch.full((w.num_seqs, w.num_q_heads, w.head_dim), float("nan"), dtype=torch.bfloat16, device=DEV)
    eng.run_decode(q.to(DEV), out, w.scale)
    torch.cuda.synchronize()
    assert pa.last_device_error()[0] == 0
    ek, ev = oops.reshape_and_cache(codes_np(kp), codes_np(vp), "bf16", pre_slots, k0, v0, "bf16")
    ek, ev = oops.copy_blocks(ek, ev, pairs_o)
    ek, ev = oops.reshape_and_cache(codes_np(kq), codes_np(vq), "bf16", priv_slots, ek, ev, "bf16")
    assert np.array_equal(codes_np(eng.k_cache), ek) and np.array_equal(codes_np(eng.v_cache), ev)
    ref = oatt.paged_decode(codes_np(q), "bf16", ek, ev, "bf16", 1.0, 1.0, mir.table(eng.MB), mir.lens, w.scale)
    assert_close(out.double().cpu().numpy(), ref, "bf16", "gqa_prefix")


# partition edges (512), block edges, and a long tail
EDGE_LENS = [1, 2, 15, 16, 17, 511, 512, 513, 1023, 1024, 1025, 1537, 2100]


@pytest.mark.parametrize("kv,q,D,BS,G", [
    ("bf16", "bf16", 128, 16, 1), ("f16", "f16", 128, 16, 1), ("bf16", "bf16", 128, 16, 4),
    ("f16", "f16", 64, 16, 2), ("bf16", "bf16", 64, 8, 8), ("f16", "f16", 128, 32, 4),
    ("bf16", "bf16", 128, 8, 2), ("e4m3", "bf16", 128, 32, 1), ("e4m3", "f16", 64, 16, 4),
    ("e4m3", "bf16", 128, 16, 8), ("e4m3", "bf16", 64, 8, 1), ("bf16", "bf16", 128, 32, 8)])
def test_fuzz_shapes_and_partition_edges(kv, q, D, BS, G):
    """Every output row; the cache bytes past each context (and every free block) are NaN
    before the step, and no output may depend on them."""
    Hkv = 2
    seed = zlib.crc32(repr((kv, q, D, BS, G)).encode()) % 100000
    w = synthetic.custom(len(EDGE_LENS), Hkv * G, Hkv, D, BS, kv, q, EDGE_LENS, seed)
    run_decode_step(w, nan_tails=True)


def test_single_token_context_returns_value_row():
    w = synthetic.custom(3, 4, 4, 128, 16, "bf16", "bf16", [1, 1, 1], 77)
    err, eng = run_decode_step(w)
    assert err == 0.0      # the softmax of one score is exactly 1: out = V row, rounded once


def test_empty_context_gives_zero_rows():
    w = synthetic.custom(3, 8, 2, 128, 16, "bf16", "bf16", [40, 1, 700], 78)
    eng = make_engine(w, DEV)
    fill_cache(w, eng)
    for s, L in enumerate(w.context_lens):
        eng.extend(s, L)
    eng.upload_tables()
    eng.lens_dev.copy_(torch.tensor([40, 0, 700], dtype=torch.int32))
    q = synthetic.normal_values((3, 8, 128), "bf16", 5).to(DEV)
    out = torch.full_like(q, float("nan"))
    eng.run_decode(q, out, w.scale)
    o = out.float().cpu()
    assert torch.all(o[1] == 0) and torch.isfinite(o).all()


def test_block_permutation_gives_identical_bits():
    """Moving every physical block (and its table entries) leaves the output bits unchanged."""
    w = synthetic.custom(4, 8, 8, 128, 16, "bf16", "bf16", [100, 600, 1300, 31], 79)
    eng = make_engine(w, DEV)
    fill_cache(w, eng)
    for s, L in enumerate(w.context_lens):
        eng.extend(s, L)
    eng.upload_tables()
    q = synthetic.normal_values((4, 8, 128), "bf16", 6).to(DEV)
    out1 = torch.empty_like(q)
    eng.run_decode(q, out1, w.scale)
    perm = torch.from_numpy(np.random.default_rng(9).permutation(w.num_blocks)).to(DEV)
    kc2, vc2 = torch.empty_like(eng.k_cache), torch.empty_like(eng.v_cache)
    kc2[perm] = eng.k_cache
    vc2[perm] = eng.v_cache
    cache2 = pa.KVCache(kc2, vc2, "bf16")
    bt2 = perm.to(torch.int32)[eng.bt_dev.long()]
    out2 = torch.empty_like(q)
    pa.decode(q, cache2, bt2, eng.lens_dev, eng.max_context_len, w.scale, out2, eng.ws)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_gqa_equals_mha_with_duplicated_kv_heads():
    """G query heads sharing a kv head give what MHA over G copies of it gives: with G = 4
    the grouped decode runs on the tensor cores and the copies on the CUDA cores, so the
    two agree within the bf16 parity tolerance (the grouping maps q head h to kv head
    h // G)."""
    w = synthetic.custom(3, 8, 2, 128, 16, "bf16", "bf16", [77, 530, 1200], 80)
    eng = make_engine(w, DEV)
    fill_cache(w, eng)
    for s, L in enumerate(w.context_lens):
        eng.extend(s, L)
    eng.upload_tables()
    q = synthetic.normal_values((3, 8, 128), "bf16", 7).to(DEV)
    out_g = torch.empty_like(q)
    eng.run_decode(q, out_g, w.scale)
    kc = eng.k_cache.repeat_interleave(4, dim=1).contiguous()
    vc = eng.v_cache.repeat_interleave(4, dim=1).contiguous()
    out_m = torch.empty_like(q)
    pa.decode(q, pa.KVCache(kc, vc, "bf16"), eng.bt_dev, eng.lens_dev, eng.max_context_len, w.scale,
              out_m, eng.ws)
    a, b = out_g.double().cpu().numpy(), out_m.double().cpu().numpy()
    assert np.all(np.abs(a - b) <= 2e-3 + 1e-2 * np.abs(b))


def test_binding_refuses_mismatched_device_arguments_before_any_launch():
    w = synthetic.custom(2, 4, 4, 128, 16, "bf16", "bf16", [40, 20], 81)
    eng = make_engine(w, DEV)
    pa.last_device_error()                      # start from a clear error word
    q = torch.zeros((2, 4, 128), dtype=torch.bfloat16, device=DEV)
    out = torch.empty_like(q)
    q64 = torch.zeros((2, 4, 64), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError):             # head_dim 64 against a 128 cache: q would be over-read
        pa.decode(q64, eng.cache, eng.bt_dev, eng.lens_dev, eng.max_context_len, w.scale, torch.empty_like(q64),
                  eng.ws)
    with pytest.raises(TypeError):
        pa.decode(q, eng.cache, eng.bt_dev.long(), eng.lens_dev, eng.max_context_len, w.scale, out, eng.ws)
    with pytest.raises(ValueError):
        pa.decode(q, eng.cache, eng.bt_dev[:1], eng.lens_dev, eng.max_context_len, w.scale, out, eng.ws)
    with pytest.raises(TypeError):
        pa.decode(q, eng.cache, eng.bt_dev, eng.lens_dev, eng.max_context_len, w.scale, out.float(), eng.ws)
    qs = torch.tensor([0, 1, 2], dtype=torch.int32, device=DEV)
    with pytest.raises(ValueError):             # extend / prefill check the same way
        pa.extend(q64, eng.cache, qs, eng.bt_dev, eng.lens_dev, eng.max_context_len, w.scale,
                  torch.empty_like(q64), eng.ws)
    kv_bad = torch.zeros((2, 2, 128), dtype=torch.bfloat16, device=DEV)      # 2 kv heads, the cache has 4
    with pytest.raises(ValueError):
        pa.prefill(q, kv_bad, kv_bad, eng.cache, qs, eng.bt_dev, eng.lens_dev, eng.max_context_len, w.scale,
                   out, eng.ws)
    torch.cuda.synchronize()
    assert pa.last_device_error()[0] == 0


def test_bad_block_id_is_recorded_not_faulting():
    w = synthetic.custom(2, 4, 4, 128, 16, "bf16", "bf16", [40, 20], 81)
    eng = make_engine(w, DEV)
    fill_cache(w, eng)
    for s, L in enumerate(w.context_lens):
        eng.extend(s, L)
    eng.bt_host[1, 1] = w.num_blocks + 7
    eng.upload_tables()
    q = synthetic.normal_values((2, 4, 128), "bf16", 8).to(DEV)
    out = torch.empty_like(q)
    eng.run_decode(q, out, w.scale)
    code, info = pa.last_device_error()
    assert code == 1 and info == (1, 1, w.num_blocks + 7)


def test_context_beyond_table_is_clamped_and_recorded():
    w = synthetic.custom(2, 4, 4, 128, 16, "bf16", "bf16", [40, 20], 82)
    eng = make_engine(w, DEV)
    fill_cache(w, eng)
    for s, L in enumerate(w.context_lens):
        eng.extend(s, L)
    eng.upload_tables()
    eng.lens_dev.copy_(torch.tensor([40, 10 ** 6], dtype=torch.int32))
    q = synthetic.normal_values((2, 4, 128), "bf16", 9).to(DEV)
    out = torch.empty_like(q)
    eng.run_decode(q, out, w.scale)
    code, info = pa.last_device_error()
    assert code == 2 and info[0] == 1 and info[1] == 10 ** 6


def test_host_pipeline_matches_device_steps():
    """Steps fed from pinned host buffers (copies overlapped on their own streams)
    give the same output bits as the same steps fed from device tensors."""
    from paged_kv_cache_436_b200.engine import HostPipeline
    w = synthetic.custom(6, 8, 2, 128, 16, "bf16", "bf16", [30, 511, 700, 1200, 64, 2000], 83)
    outs = []
    for mode in ("device", "host"):
        eng = make_engine(w, DEV, growth=8)
        fill_cache(w, eng)
        for s, L in enumerate(w.context_lens):
            eng.extend(s, L - 1)
        eng.upload_tables()
        res = []
        if mode == "device":
            for i in range(5):
                q, k, v = (t.to(DEV) for t in synthetic.step_inputs(w, i))
                out = torch.empty_like(q)
                eng.step(q, k, v, out, w.scale)
                res.append(out.cpu())
        else:
            pipe = HostPipeline(eng, w.scale)
            hosts = []
            for i in range(5):
                q, k, v = synthetic.step_inputs(w, i)
                hq, hk, hv = q.pin_memory(), k.pin_memory(), v.pin_memory()
                hout = torch.empty_like(q).pin_memory()
                hosts.append((hq, hk, hv, hout))
                pipe.submit(hq, hk, hv, hout)
            pipe.sync()
            res = [h[3] for h in hosts]
        torch.cuda.synchronize()
        assert pa.last_device_error()[0] == 0
        outs.append(res)
    for a, b in zip(*outs):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_engine_step_out_of_blocks_reports_and_keeps_state_consistent():
    """A step that runs out of blocks mid-batch returns PA_ERR_OOM; the sequences
    before the failing one hold their new token, nothing is enqueued."""
    w = synthetic.custom(3, 4, 4, 64, 16, "f16", "f16", [16, 16, 16], 84, pool_factor=1.0)
    eng = make_engine(w, DEV, growth=16)
    fill_cache(w, eng)
    for s in range(3):
        eng.extend(s, 16)                      # every sequence fills its block exactly
    while eng.pool.num_free() > 1:             # leave one free block: only sequence 0 can grow
        eng.pool.alloc()
    eng.upload_tables()
    q, k, v = (t.to(DEV) for t in synthetic.step_inputs(w, 0))
    out = torch.zeros_like(q)
    with pytest.raises(pa.PaError) as e:
        eng.step(q, k, v, out, w.scale)
    assert e.value.status == pa.PA_ERR_OOM
    assert eng.lens.tolist() == [17, 16, 16] and eng.pool.num_free() == 0
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0


def test_decode_over_prefix_cache_built_batch():
    """Requests sharing a 1000-token history, admitted through the prefix cache: the
    first writes the history's K/V, the others reuse its 62 full blocks and write only
    their unmatched tokens. Tables, cache bytes and outputs against the oracle running
    its own pool, prefix cache and cache ops."""
    from oracle.pool import BlockPool
    from oracle.prefix_cache import PrefixCache as OPrefix
    S, Hq, Hkv, D, BS, hist_len = 12, 32, 8, 128, 16, 1000
    rng = np.random.default_rng(91)
    priv = rng.integers(1, 60, size=S).tolist()
    lens = [hist_len + p for p in priv]
    w = synthetic.custom(S, Hq, Hkv, D, BS, "bf16", "bf16", lens, 92, pool_factor=0.3)
    w.num_blocks = 62 + sum(-(-L // BS) - 62 for L in lens) + 4
    w.initial_order = rng.permutation(w.num_blocks).tolist()
    hist = rng.integers(0, 32000, size=hist_len).tolist()
    prompts = [hist + rng.integers(0, 32000, size=p).tolist() for p in priv]
    # K/V of every (position, token): history rows are the same for every request
    kh = synthetic.normal_values((hist_len, Hkv, D), "bf16", 93)
    vh = synthetic.normal_values((hist_len, Hkv, D), "bf16", 94)
    eng = make_engine(w, DEV)
    fill_cache(w, eng)
    ncache = pa.PrefixCache(BS)
    opool, ocache = BlockPool(w.num_blocks, w.initial_order), OPrefix(BS)
    k0, v0 = codes_np(eng.k_cache), codes_np(eng.v_cache)
    ek, ev = k0, v0
    orows = []
    for s, prompt in enumerate(prompts):
        n = ncache.match(eng.pool, prompt, eng.bt_host[s])
        eng.lens[s] = n * BS
        start = n * BS
        slots = np.zeros(len(prompt) - start, np.int64)
        eng.extend(s, len(prompt) - start, slots)
        ncache.insert(eng.pool, prompt, eng.bt_host[s])
        orow = []
        on = ocache.match(opool, prompt, orow)
        opool.seq_extend(orow, on * BS, len(prompt) - on * BS, BS)
        ocache.insert(opool, prompt, orow)
        orows.append(orow)
        assert n == on == (0 if s == 0 else 62)
        assert eng.bt_host[s, :len(orow)].tolist() == orow
        # this request's unmatched tokens: history rows from the shared table, then private rows
        m = len(prompt) - start
        kp = synthetic.normal_values((len(prompt) - hist_len, Hkv, D), "bf16", 1000 + s)
        vp = synthetic.normal_values((len(prompt) - hist_len, Hkv, D), "bf16", 2000 + s)
        kt = torch.cat([kh[start:], kp])[-m:] if start < hist_len else kp[start - hist_len:]
        vt = torch.cat([vh[start:], vp])[-m:] if start < hist_len else vp[start - hist_len:]
        pa.reshape_and_cache(kt.to(DEV), vt.to(DEV), torch.from_numpy(slots).to(DEV), eng.cache)
        ek, ev = oops.reshape_and_cache(codes_np(kt), codes_np(vt), "bf16", slots, ek, ev, "bf16")
    assert eng.pool.num_free() == opool.num_free() and len(ncache) == len(ocache) >= 62
    eng.upload_tables()
    q = synthetic.normal_values((S, Hq, D), "bf16", 95).to(DEV)
    out = torch.full_like(q, float("nan"))
    eng.run_decode(q, out, w.scale)
    torch.cuda.synchronize()
    assert pa.last_device_error()[0] == 0
    assert np.array_equal(codes_np(eng.k_cache), ek) and np.array_equal(codes_np(eng.v_cache), ev)
    bt = np.zeros((S, eng.MB), np.int64)
    for s, r in enumerate(orows):
        bt[s, :len(r)] = r
    ref = oatt.paged_decode(codes_np(q), "bf16", ek, ev, "bf16", 1.0, 1.0, bt, lens, w.scale)
    assert_close(out.double().cpu().numpy(), ref, "bf16", "prefix-cache batch")


def test_beam_search_steps():
    """Width-5 beams: each step re-selects beams (fork/free), appends one token per beam
    (copy-on-write of shared partial blocks), writes the tokens and decodes. Tables,
    copy pairs, cache bytes and outputs against the oracle over several steps."""
    from oracle import pool as opool_mod
    from oracle.pool import BlockPool
    R, W = 3, 5
    w = synthetic.beam_workload(num_requests=R, width=W, prompt=90, num_heads=4, head_dim=128,
                                block_size=16, growth=40, seed=4242)
    S = R * W
    eng = make_engine(w, DEV, growth=40)
    fill_cache(w, eng)
    opool = BlockPool(w.num_blocks, w.initial_order)
    orows, olens = [[] for _ in range(S)], [0] * S
    for r in range(R):
        L = w.context_lens[r * W]
        eng.extend(r * W, L)
        opool.seq_extend(orows[r * W], 0, L, w.block_size)
        for j in range(1, W):
            eng.fork(r * W, r * W + j)
            orows[r * W + j] = opool.fork(orows[r * W])
        olens[r * W:(r + 1) * W] = [L] * W
    eng.upload_tables()
    ek, ev = codes_np(eng.k_cache), codes_np(eng.v_cache)
    cows_seen = 0
    for step in range(6):
        parents = synthetic.beam_parents(R, W, step, w.seed)
        eng.reorder(parents)
        orows, olens = opool_mod.reorder(opool, orows, olens, parents)
        q, k, v = synthetic.step_inputs(w, step)
        out = torch.full(q.shape, float("nan"), dtype=q.dtype, device=DEV)
        eng.step(q.to(DEV), k.to(DEV), v.to(DEV), out, w.scale)
        torch.cuda.synchronize()
        assert pa.last_device_error()[0] == 0
        oslots, ocows, _ = opool.batch_append(orows, olens, w.block_size)
        olens = [L + 1 for L in olens]
        assert eng.last_step()[0] == len(ocows)
        cows_seen += len(ocows)
        for s in range(S):
            assert eng.bt_host[s, :len(orows[s])].tolist() == orows[s]
        ek, ev = oops.copy_blocks(ek, ev, ocows)
        ek, ev = oops.reshape_and_cache(codes_np(k), codes_np(v), w.q_dtype, oslots, ek, ev, w.kv_dtype)
        assert np.array_equal(codes_np(eng.k_cache), ek) and np.array_equal(codes_np(eng.v_cache), ev)
        bt = np.zeros((S, eng.MB), np.int64)
        for s, r in enumerate(orows):
            bt[s, :len(r)] = r
        ref = oatt.paged_decode(codes_np(q), w.q_dtype, ek, ev, w.kv_dtype, 1.0, 1.0, bt, olens, w.scale)
        assert_close(out.double().cpu().numpy(), ref, w.kv_dtype, f"beam step {step}")
    assert cows_seen > 0
