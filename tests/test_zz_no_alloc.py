"""pa_decode_no_alloc: decode for callers that may not allocate device memory.

Such callers -- a plugin inside a framework that owns all device memory through its
own allocator, or a serving loop that forbids allocation calls because they can
stall other streams -- cannot provide pa_decode's workspace. The entry point uses a
fixed 16 MiB array inside the library instead. These tests call it through the C
ABI and check it against pa_decode with a caller workspace: the same kernels run on
the same scratch layout, so the outputs must be bit-identical, on two calls in a row
with different inputs. One call is also compared with the float64 oracle at the
decode parity tolerance, and the largest size the header says fits (8 sequences x
32 q heads x 32K tokens, E4M3 cache) runs through the array's upper end. Sizes
needing more scratch than the array holds are refused. This file is collected last
on purpose: it must pass both alone and after the other tests.
"""

import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_436_b200 as pa
import synthetic
from oracle import attention as oatt
from tests.gpu_cases import assert_close, codes_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _setup(lens, seed, Hq=8, Hkv=2, D=128, BS=16, kv="bf16"):
    w = synthetic.custom(len(lens), Hq, Hkv, D, BS, kv, "bf16", lens, seed)
    nb = w.num_blocks
    if kv == "e4m3":
        kc, ks = synthetic.normal_e4m3_codes((nb, Hkv, BS, D), seed + 1, DEV)
        vc, vs = synthetic.normal_e4m3_codes((nb, Hkv, BS, D), seed + 2, DEV)
    else:
        kc = synthetic.normal_values((nb, Hkv, BS, D), kv, seed + 1, DEV)
        vc = synthetic.normal_values((nb, Hkv, BS, D), kv, seed + 2, DEV)
        ks = vs = 1.0
    cache = pa.KVCache(kc, vc, kv, ks, vs)
    MB = -(-max(lens) // BS)
    rng = np.random.default_rng(seed)
    bt_host = rng.integers(0, nb, size=(len(lens), MB)).astype(np.int32)
    bt = torch.from_numpy(bt_host).to(DEV)
    ctx = torch.tensor(lens, dtype=torch.int32, device=DEV)
    q = synthetic.normal_values((len(lens), Hq, D), "bf16", seed + 3, DEV)
    return w, cache, bt, bt_host, ctx, q, max(lens)


def _no_alloc_call(q, cache, bt, ctx, max_len, scale, out):
    return pa.lib().pa_decode_no_alloc(ctypes.c_void_p(q.data_ptr()), pa.PA_BF16, q.shape[0], q.shape[1],
                                       ctypes.byref(cache.desc), ctypes.c_void_p(bt.data_ptr()), bt.shape[1],
                                       ctypes.c_void_p(ctx.data_ptr()), max_len, scale,
                                       ctypes.c_void_p(out.data_ptr()),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _with_workspace(q, cache, bt, ctx, max_len, scale):
    out = torch.empty_like(q)
    ws = torch.empty(pa.decode_workspace_size(q.shape[0], q.shape[1], q.shape[2], max_len),
                     dtype=torch.uint8, device=DEV)
    pa.decode(q, cache, bt, ctx, max_len, scale, out, ws)
    return out


def test_no_alloc_matches_caller_workspace_on_two_calls_in_a_row():
    # two different problems back to back: the second must not see the first's scratch
    cases = [_setup([1, 700, 2100, 513, 64], 11), _setup([3000, 17, 1025], 12, Hq=16, Hkv=4)]
    for i, (w, cache, bt, bt_host, ctx, q, max_len) in enumerate(cases):
        out = torch.full_like(q, float("nan"))
        assert _no_alloc_call(q, cache, bt, ctx, max_len, w.scale, out) == pa.PA_OK
        ref = _with_workspace(q, cache, bt, ctx, max_len, w.scale)
        torch.cuda.synchronize()
        assert pa.last_device_error()[0] == 0
        assert torch.equal(out, ref), "the fixed array and a caller workspace give different bits"
        if i == 0:   # and the first call against the float64 oracle
            want = oatt.paged_decode(codes_np(q), "bf16", codes_np(cache.k_cache), codes_np(cache.v_cache), "bf16",
                                     1.0, 1.0, bt_host.astype(np.int64), list(w.context_lens), w.scale)
            assert_close(out.double().cpu().numpy(), want, "bf16", "no-alloc decode")


def test_no_alloc_largest_stated_size_e4m3():
    """8 sequences x 32 q heads x 32768 tokens, head_dim 128, E4M3 cache, 32-token blocks:
    the largest shape the header says fits (64 partitions per row, about 8.4 MiB of the
    array). Bit-identical to a caller workspace; sampled rows against the oracle."""
    lens = [32768] * 8
    w, cache, bt, bt_host, ctx, q, max_len = _setup(lens, 15, Hq=32, Hkv=32, BS=32, kv="e4m3")
    assert pa.decode_workspace_size(8, 32, 128, 32768) <= pa.NO_ALLOC_WORKSPACE_BYTES
    out = torch.full_like(q, float("nan"))
    assert _no_alloc_call(q, cache, bt, ctx, max_len, w.scale, out) == pa.PA_OK
    ref = _with_workspace(q, cache, bt, ctx, max_len, w.scale)
    torch.cuda.synchronize()
    assert pa.last_device_error()[0] == 0
    assert torch.equal(out, ref)
    heads = [(0, 0), (3, 17), (7, 31)]
    blocks = sorted({int(b) for s, _ in heads for b in bt_host[s]})
    remap = {b: i for i, b in enumerate(blocks)}
    idx = torch.tensor(blocks, dtype=torch.int64, device=DEV)
    kc, vc = codes_np(cache.k_cache.index_select(0, idx)), codes_np(cache.v_cache.index_select(0, idx))
    btc = np.zeros(bt_host.shape, np.int64)
    for s, _ in heads:
        btc[s] = [remap[int(b)] for b in bt_host[s]]
    d = cache.desc
    want = oatt.paged_decode(codes_np(q), "bf16", kc, vc, "e4m3", d.k_scale, d.v_scale, btc, lens, w.scale,
                             heads=heads)
    hs = tuple(np.array(heads).T)
    assert_close(out.double().cpu().numpy()[hs], want[hs], "e4m3", "no-alloc decode, 32K E4M3")


def test_no_alloc_refuses_sizes_beyond_its_array():
    w, cache, bt, _, ctx, q, _ = _setup([40, 20], 13)
    need = pa.decode_workspace_size(256, 40, 128, 8192)
    assert need > pa.NO_ALLOC_WORKSPACE_BYTES
    out = torch.zeros_like(q)
    # a declared maximum length whose scratch exceeds the 16 MiB array is refused up front
    big = 64 * 512 * 40
    assert pa.decode_workspace_size(q.shape[0], q.shape[1], 128, big) > pa.NO_ALLOC_WORKSPACE_BYTES
    assert _no_alloc_call(q, cache, bt, ctx, big, w.scale, out) == pa.PA_ERR_ARG
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0          # nothing was enqueued
    with pytest.raises(pa.PaError):
        pa.decode_no_alloc(q, cache, bt, ctx, big, w.scale, out)
