"""pa_decode_no_alloc: decode for callers that may not allocate device memory.

Such callers -- a plugin inside a framework that owns all device memory through its
own allocator, or a serving loop that forbids allocation calls because they can
stall other streams -- cannot provide pa_decode's workspace. The entry point uses a
fixed 16 MiB array inside the library instead. These tests call it through the C
ABI and check it against pa_decode (caller workspace) within the parity tolerance
of the decode tests, on two calls in a row with different inputs, and check that
sizes needing more scratch than the array holds are refused. This file is
collected last on purpose: it must pass both alone and after the other tests.
"""

import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_436_b200 as pa
import synthetic

pytestmark = pytest.mark.gpu
DEV = "cuda"
ATOL, RTOL = 2e-3, 1e-2      # the bf16 decode parity tolerance


def _setup(lens, seed, Hq=8, Hkv=2, D=128, BS=16):
    w = synthetic.custom(len(lens), Hq, Hkv, D, BS, "bf16", "bf16", lens, seed)
    nb = w.num_blocks
    kc = synthetic.normal_values((nb, Hkv, BS, D), "bf16", seed + 1, DEV)
    vc = synthetic.normal_values((nb, Hkv, BS, D), "bf16", seed + 2, DEV)
    cache = pa.KVCache(kc, vc, "bf16")
    MB = -(-max(lens) // BS)
    rng = np.random.default_rng(seed)
    bt = torch.from_numpy(rng.integers(0, nb, size=(len(lens), MB)).astype(np.int32)).to(DEV)
    ctx = torch.tensor(lens, dtype=torch.int32, device=DEV)
    q = synthetic.normal_values((len(lens), Hq, D), "bf16", seed + 3, DEV)
    return w, cache, bt, ctx, q, max(lens)


def _no_alloc_call(q, cache, bt, ctx, max_len, scale, out):
    st = pa.lib().pa_decode_no_alloc(ctypes.c_void_p(q.data_ptr()), pa.PA_BF16, q.shape[0], q.shape[1],
                                     ctypes.byref(cache.desc), ctypes.c_void_p(bt.data_ptr()), bt.shape[1],
                                     ctypes.c_void_p(ctx.data_ptr()), max_len, scale,
                                     ctypes.c_void_p(out.data_ptr()),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def _reference(q, cache, bt, ctx, max_len, scale):
    out = torch.empty_like(q)
    ws = torch.empty(pa.decode_workspace_size(q.shape[0], q.shape[1], q.shape[2], max_len),
                     dtype=torch.uint8, device=DEV)
    pa.decode(q, cache, bt, ctx, max_len, scale, out, ws)
    return out


def test_no_alloc_matches_caller_workspace_on_two_calls_in_a_row():
    # two different problems back to back: the second must not see the first's scratch
    cases = [_setup([1, 700, 2100, 513, 64], 11), _setup([3000, 17, 1025], 12, Hq=16, Hkv=4)]
    for w, cache, bt, ctx, q, max_len in cases:
        out = torch.full_like(q, float("nan"))
        assert _no_alloc_call(q, cache, bt, ctx, max_len, w.scale, out) == pa.PA_OK
        ref = _reference(q, cache, bt, ctx, max_len, w.scale)
        torch.cuda.synchronize()
        assert pa.last_device_error()[0] == 0
        got, want = out.double().cpu().numpy(), ref.double().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.all(np.abs(got - want) <= ATOL + RTOL * np.abs(want))


def test_no_alloc_refuses_sizes_beyond_its_array():
    w, cache, bt, ctx, q, _ = _setup([40, 20], 13)
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
