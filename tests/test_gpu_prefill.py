"""GPU parity of pa_prefill (whole prompts; the prompts' K / V written into the paged cache
by the same kernel) against the float64 oracle: every prompt slot of the cache bit-exact
against the oracle's reshape_and_cache, the outputs within 2e-3 + 1e-2 |ref| against the
oracle's paged_extend over that cache. The cache starts as NaN everywhere."""

import zlib

import numpy as np
import pytest
import torch

import paged_kv_cache_436_b200 as pa
import synthetic
from tests.gpu_cases import make_engine, run_prefill_case

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dt,BS,G", [("bf16", 16, 1), ("f16", 32, 2), ("bf16", 32, 4), ("f16", 16, 8),
                                     ("bf16", 16, 8)])
def test_prefill_matches_oracle(dt, BS, G):
    """Ragged prompts (1 token, block- and tile-unaligned lengths, several 512-token
    chunks) with few units, so contexts are split into chunks and merged."""
    lens = [1, 17, 130, 700, 1025, 257]
    seed = zlib.crc32(repr(("prefill", dt, BS, G)).encode()) % 10000
    run_prefill_case(lens, 2 * G, 2, BS, dt, seed, 160)


def test_prefill_whole_context_units():
    """Enough row tiles that every unit holds its rows' whole context (no merge)."""
    run_prefill_case([1200, 1100, 1000, 1200], 8, 8, 16, "bf16", 81, 200)


def test_prefill_rejects_context_longer_than_prompt():
    lens = [40, 60]
    w = synthetic.custom(2, 4, 4, 128, 16, "bf16", "bf16", lens, 83)
    eng = make_engine(w, DEV)
    for s, L in enumerate(lens):
        eng.extend(s, L)
    eng.upload_tables()
    qs = np.array([0, 30, 90], dtype=np.int32)                # sequence 0: 30 queries, 40 tokens
    q = synthetic.normal_values((90, 4, 128), "bf16", 1).to(DEV)
    k = synthetic.normal_values((90, 4, 128), "bf16", 2).to(DEV)
    out = torch.full_like(q, float("nan"))
    ws = torch.empty(pa.extend_workspace_size(2, 90, 4, 128, eng.max_context_len), dtype=torch.uint8, device=DEV)
    pa.prefill(q, k, k, eng.cache, torch.from_numpy(qs).to(DEV), eng.bt_dev, eng.lens_dev, eng.max_context_len,
               w.scale, out, ws)
    code, info = pa.last_device_error()
    assert code == 2 and info[0] == 0
    assert torch.count_nonzero(out[:30]) == 0 and torch.isfinite(out[30:].float()).all()


def test_prefill_unsupported_shapes_are_refused():
    w = synthetic.custom(1, 2, 2, 64, 16, "bf16", "bf16", [10], 85)   # head_dim 64: no tcgen05 path
    eng = make_engine(w, DEV)
    eng.extend(0, 10)
    eng.upload_tables()
    q = torch.zeros((10, 2, 64), dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device=DEV)
    with pytest.raises(RuntimeError):
        pa.prefill(q, q, q, eng.cache, torch.tensor([0, 10], dtype=torch.int32, device=DEV), eng.bt_dev,
                   eng.lens_dev, eng.max_context_len, w.scale, torch.empty_like(q), ws)


def test_prefill_8x2k_full_size():
    """The benchmarked prefill shapes (8 prompts x 2048 tokens, 32/32 heads, bf16, 16-token
    blocks): every cache slot bit-exact, sampled output rows against the oracle."""
    run_prefill_case([2048] * 8, 32, 32, 16, "bf16", 4371, 120)


def test_prefill_gqa_8x2k_full_size():
    """The benchmarked GQA prefill shapes (Llama-3-8B attention: 32 q heads over 8 kv heads,
    8 prompts x 2048 tokens): every cache slot bit-exact, sampled rows against the oracle."""
    run_prefill_case([2048] * 8, 32, 8, 16, "bf16", 4372, 120)


@pytest.mark.parametrize("dt,BS,G", [("bf16", 32, 1), ("f16", 16, 4)])
def test_prefill_into_e4m3_cache(dt, BS, G):
    """Whole prompts into an E4M3 cache: every prompt slot holds the oracle's E4M3 encoding
    of the prompt's K / V (x / scale, round to nearest even, saturating; scales chosen so
    that the largest values saturate) and every output element matches the oracle's
    attention over that cache within 3e-2 + 3e-2 |ref|."""
    from oracle import attention as oatt
    from oracle import cache_ops as oops
    from tests.gpu_cases import assert_close, codes_np
    lens = [1, 17, 130, 700, 257]
    D, Hkv = 128, 2
    Hq = Hkv * G
    seed = zlib.crc32(repr(("prefill e4m3", dt, BS, G)).encode()) % 10000
    w = synthetic.custom(len(lens), Hq, Hkv, D, BS, "e4m3", dt, lens, seed)
    ks, vs = 3.5 / 448, 3.0 / 448
    eng = make_engine(w, DEV, k_scale=ks, v_scale=vs)
    eng.k_cache.fill_(0x7F)                     # NaN codes everywhere beforehand
    eng.v_cache.fill_(0x7F)
    k0, v0 = codes_np(eng.k_cache), codes_np(eng.v_cache)
    for s, L in enumerate(lens):
        eng.extend(s, L)
    eng.upload_tables()
    qs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(qs[-1])
    q = synthetic.normal_values((T, Hq, D), dt, seed + 7).to(DEV)
    k = synthetic.normal_values((T, Hkv, D), dt, seed + 8).to(DEV)
    v = synthetic.normal_values((T, Hkv, D), dt, seed + 9).to(DEV)
    out = torch.full_like(q, float("nan"))
    ws = torch.empty(pa.extend_workspace_size(w.num_seqs, T, Hq, D, eng.max_context_len), dtype=torch.uint8,
                     device=DEV)
    pa.prefill(q, k, v, eng.cache, torch.from_numpy(qs).to(DEV), eng.bt_dev, eng.lens_dev, eng.max_context_len,
               w.scale, out, ws)
    torch.cuda.synchronize()
    assert pa.last_device_error()[0] == 0
    bt = eng.bt_host.astype(np.int64)
    slots = np.concatenate([bt[s, np.arange(L) // BS] * BS + np.arange(L) % BS for s, L in enumerate(lens)])
    kc, vc = oops.reshape_and_cache(codes_np(k), codes_np(v), dt, slots, k0, v0, "e4m3", ks, vs)
    gk, gv = codes_np(eng.k_cache), codes_np(eng.v_cache)
    assert np.array_equal(gk[slots // BS, :, slots % BS, :], kc[slots // BS, :, slots % BS, :]), "k slots"
    assert np.array_equal(gv[slots // BS, :, slots % BS, :], vc[slots // BS, :, slots % BS, :]), "v slots"
    ref = oatt.paged_extend(codes_np(q), dt, kc, vc, "e4m3", ks, vs, bt, lens, qs, w.scale)
    assert_close(out.double().cpu().numpy(), ref, "e4m3", f"prefill e4m3 {dt} BS{BS} G{G}")
