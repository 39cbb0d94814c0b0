"""Every output element of extend / prefill rows whose precision depends on how P enters
the P V product, against the float64 oracle at |err| <= 2e-3 + 1e-2 |ref|.

P rounded to bf16 alone can leave that tolerance when a few weights dominate a row and
their V values cancel: rows that see only a few tokens, and rows whose scores are peaked.
The kernels carry the bf16 remainder p - bf16(p) as a second operand (always in the
mma.sync kernels, for the tiles that need it on tcgen05), so every element of such rows
must be inside the tolerance -- checked here for many 1-15-token prompts (tcgen05,
pa_prefill), many 1-15-token draft runs over longer contexts (16-row mma.sync kernel),
long query runs (tcgen05 through pa_extend, and the 64-row kernel at head_dim 64), for
bf16 and f16, several seeds, and score scales from flat (scale * sqrt(D) = 1) to peaked
(4 and 12: a handful of tokens carry most of the weight).
"""

import zlib

import numpy as np
import pytest
import torch

import paged_kv_cache_436_b200 as pa
import synthetic
from oracle import attention as oatt
from oracle import cache_ops as oops
from tests.gpu_cases import assert_close, codes_np, fill_cache, make_engine, nan_past_contexts_

pytestmark = pytest.mark.gpu
DEV = "cuda"
MULTS = [1.0, 4.0, 12.0]          # scale * sqrt(head_dim): flat, peaked, very peaked


def _extend_case(lens, qlens, Hq, Hkv, D, dt, mult, seed):
    """pa_extend of qlens[s] new tokens over contexts of lens[s]; every element checked."""
    w = synthetic.custom(len(lens), Hq, Hkv, D, 16, dt, dt, lens, seed, scale=mult / np.sqrt(D))
    eng = make_engine(w, DEV)
    fill_cache(w, eng)
    for s, L in enumerate(lens):
        eng.extend(s, L)
    eng.upload_tables()
    nan_past_contexts_(w, eng)
    qs = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    T = int(qs[-1])
    q = synthetic.normal_values((T, Hq, D), dt, seed + 7).to(DEV)
    out = torch.full_like(q, float("nan"))
    ws = torch.empty(pa.extend_workspace_size(w.num_seqs, T, Hq, D, eng.max_context_len), dtype=torch.uint8,
                     device=DEV)
    pa.extend(q, eng.cache, torch.from_numpy(qs).to(DEV), eng.bt_dev, eng.lens_dev, eng.max_context_len, w.scale,
              out, ws)
    torch.cuda.synchronize()
    assert pa.last_device_error()[0] == 0
    ref = oatt.paged_extend(codes_np(q), dt, codes_np(eng.k_cache), codes_np(eng.v_cache), dt, 1.0, 1.0,
                            eng.bt_host.astype(np.int64), list(eng.lens), qs, w.scale)
    return assert_close(out.double().cpu().numpy(), ref, dt, f"extend {dt} x{mult} seed {seed}")


def _prefill_case(lens, Hq, Hkv, dt, mult, seed):
    """pa_prefill of whole prompts into a NaN cache; every slot bit-exact, every element
    of the output checked."""
    D = 128
    w = synthetic.custom(len(lens), Hq, Hkv, D, 16, dt, dt, lens, seed, scale=mult / np.sqrt(D))
    eng = make_engine(w, DEV)
    eng.k_cache.fill_(float("nan"))
    eng.v_cache.fill_(float("nan"))
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
    slots = np.concatenate([bt[s, np.arange(L) // 16] * 16 + np.arange(L) % 16 for s, L in enumerate(lens)])
    kc, vc = oops.reshape_and_cache(codes_np(k), codes_np(v), dt, slots, k0, v0, dt)
    gk, gv = codes_np(eng.k_cache), codes_np(eng.v_cache)
    assert np.array_equal(gk[slots // 16, :, slots % 16, :], kc[slots // 16, :, slots % 16, :])
    assert np.array_equal(gv[slots // 16, :, slots % 16, :], vc[slots // 16, :, slots % 16, :])
    ref = oatt.paged_extend(codes_np(q), dt, kc, vc, dt, 1.0, 1.0, bt, list(lens), qs, w.scale)
    return assert_close(out.double().cpu().numpy(), ref, dt, f"prefill {dt} x{mult} seed {seed}")


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("mult", MULTS)
def test_prefill_of_short_prompts_every_element(dt, mult):
    """Many 1-15-token prompts (every row sees 1-15 tokens) plus two longer ones, whole
    prompts on the tcgen05 path, G = 1 and 4."""
    for seed in range(3):
        base = zlib.crc32(repr(("short prefill", dt, mult, seed)).encode()) % 10000
        rng = np.random.default_rng(base)
        lens = rng.integers(1, 16, size=40).tolist() + [130, 301]
        _prefill_case(lens, 4, 4 if seed % 2 == 0 else 1, dt, mult, base)


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("mult", MULTS)
def test_short_draft_runs_every_element(dt, mult):
    """1-15 draft tokens per sequence over contexts of 16-700 tokens: with one q head per
    kv head the 16-row mma.sync kernel, with four (up to 60 rows per sequence) the 64-row
    one, at head_dim 128 and 64."""
    for seed, (Hq, D) in enumerate(((2, 128), (8, 128), (8, 64))):
        base = zlib.crc32(repr(("drafts", dt, mult, seed)).encode()) % 10000
        rng = np.random.default_rng(base)
        n = 24
        lens = rng.integers(16, 700, size=n).tolist()
        qlens = rng.integers(1, 16, size=n).tolist()
        _extend_case(lens, qlens, Hq, 2, D, dt, mult, base)


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("mult", MULTS)
def test_long_runs_every_element(dt, mult):
    """Long query runs: whole 300-token prompts and a 200-token chunk over a 900-token
    context (tcgen05 through pa_extend, head_dim 128), and the same at head_dim 64 (the
    64-row kernel)."""
    base = zlib.crc32(repr(("long", dt, mult)).encode()) % 10000
    _extend_case([300, 900, 60], [300, 200, 60], 8, 2, 128, dt, mult, base)
    _extend_case([300, 900, 60], [300, 200, 60], 4, 2, 64, dt, mult, base + 1)
