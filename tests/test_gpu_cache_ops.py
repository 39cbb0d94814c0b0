"""GPU parity of the cache write, the block copy and the table patch: bit-exact
against the oracle on whole cache tensors (untouched bytes included)."""

import numpy as np
import pytest
import torch

import paged_kv_cache_436_b200 as pa
import synthetic
from oracle import cache_ops as oops
from oracle import codecs
from tests.gpu_cases import codes_np

pytestmark = pytest.mark.gpu

DEV = "cuda"
TD = {"f16": torch.float16, "bf16": torch.bfloat16}


def _random_cache(shape, kv, seed):
    g = torch.Generator().manual_seed(seed)
    if kv == "e4m3":
        c = torch.randint(0, 256, shape, generator=g, dtype=torch.int32).to(torch.uint8)
    else:
        c = torch.randint(-32768, 32768, shape, generator=g, dtype=torch.int32).to(torch.int16).view(TD[kv])
    return c


@pytest.mark.parametrize("kv,inp,D,BS,Hkv", [
    ("f16", "f16", 64, 16, 4), ("bf16", "bf16", 128, 16, 8), ("f16", "f16", 128, 8, 2),
    ("bf16", "bf16", 64, 32, 3), ("e4m3", "bf16", 128, 32, 4), ("e4m3", "f16", 64, 8, 2),
    ("e4m3", "bf16", 64, 16, 5)])
def test_reshape_and_cache_bit_exact(kv, inp, D, BS, Hkv):
    NB, T = 11, 37
    kc0 = _random_cache((NB, Hkv, BS, D), kv, 1)
    vc0 = _random_cache((NB, Hkv, BS, D), kv, 2)
    rng = np.random.default_rng(3)
    slots = rng.choice(NB * BS, size=T, replace=False).astype(np.int64)
    slots[[3, 17]] = -1                                      # padding tokens
    # token rows with a wider stride than Hkv * D (a slice of a fused qkv buffer)
    stride = Hkv * D + 24
    kbuf = synthetic.normal_values((T, stride), inp, 4) * 3
    vbuf = synthetic.normal_values((T, stride), inp, 5) * 3
    if kv == "e4m3":
        # exercise saturation, subnormals and exact ties of E4M3 rounding
        mids = (codecs.decode_e4m3(np.arange(0, 0x7E)) + codecs.decode_e4m3(np.arange(1, 0x7F))) / 2
        vals = np.concatenate([mids, -mids, [500.0, -1e4, 600.0, 2.0 ** -10, 3 * 2.0 ** -11]])
        flat = kbuf.view(-1)
        flat[:len(vals)] = torch.from_numpy(vals.astype(np.float32)).to(TD[inp])
    k = kbuf[:, :Hkv * D].view(T, Hkv, D)
    v = vbuf[:, :Hkv * D].view(T, Hkv, D)
    k_scale, v_scale = (1.0, 0.0371) if kv == "e4m3" else (1.0, 1.0)
    kc, vc = kc0.clone().to(DEV), vc0.clone().to(DEV)
    cache = pa.KVCache(kc, vc, kv, k_scale, v_scale)
    kd = kbuf.to(DEV)[:, :Hkv * D].view(T, Hkv, D)
    vd = vbuf.to(DEV)[:, :Hkv * D].view(T, Hkv, D)
    pa.reshape_and_cache(kd, vd, torch.from_numpy(slots).to(DEV), cache)
    torch.cuda.synchronize()
    assert pa.last_device_error()[0] == 0
    ek, ev = oops.reshape_and_cache(codes_np(k), codes_np(v), inp, slots, codes_np(kc0), codes_np(vc0),
                                    kv, k_scale, v_scale)
    assert np.array_equal(codes_np(kc), ek)
    assert np.array_equal(codes_np(vc), ev)


def test_reshape_bad_slot_is_recorded_and_skipped():
    NB, Hkv, BS, D = 4, 2, 16, 64
    kc0 = _random_cache((NB, Hkv, BS, D), "f16", 7)
    kc, vc = kc0.clone().to(DEV), kc0.clone().to(DEV)
    cache = pa.KVCache(kc, vc, "f16")
    k = synthetic.normal_values((2, Hkv, D), "f16", 8).to(DEV)
    slots = torch.tensor([NB * BS + 5, 3], dtype=torch.int64, device=DEV)
    pa.reshape_and_cache(k, k, slots, cache)
    code, info = pa.last_device_error()
    assert code == 3 and info[0] == 0 and info[1] == NB * BS + 5
    got = codes_np(kc)
    assert np.array_equal(got[0, :, 3], codes_np(k)[1])
    got[0, :, 3] = codes_np(kc0)[0, :, 3]
    assert np.array_equal(got, codes_np(kc0))
    assert pa.last_device_error()[0] == 0                   # reading clears the word


@pytest.mark.parametrize("kv,Hkv,BS,D", [("bf16", 8, 16, 128), ("e4m3", 4, 32, 128), ("f16", 3, 8, 64)])
def test_copy_blocks_bit_exact(kv, Hkv, BS, D):
    NB = 40
    kc0 = _random_cache((NB, Hkv, BS, D), kv, 11)
    vc0 = _random_cache((NB, Hkv, BS, D), kv, 12)
    rng = np.random.default_rng(13)
    perm = rng.permutation(NB)
    pairs = np.stack([perm[:9], perm[9:18]], axis=1).astype(np.int64)   # sources and destinations disjoint
    kc, vc = kc0.clone().to(DEV), vc0.clone().to(DEV)
    cache = pa.KVCache(kc, vc, kv, 0.5 if kv == "e4m3" else 1.0, 0.25 if kv == "e4m3" else 1.0)
    pa.copy_blocks(torch.from_numpy(pairs).to(DEV), cache)
    ek, ev = oops.copy_blocks(codes_np(kc0), codes_np(vc0), pairs)
    assert np.array_equal(codes_np(kc), ek) and np.array_equal(codes_np(vc), ev)
    assert pa.last_device_error()[0] == 0
    # an out-of-range pair is skipped and recorded; the valid one is still copied
    bad = torch.tensor([[NB, 0], [perm[20], perm[21]]], dtype=torch.int64, device=DEV)
    pa.copy_blocks(bad, cache)
    code, info = pa.last_device_error()
    assert code == 4 and info[:2] == (0, NB)
    assert np.array_equal(codes_np(kc)[perm[21]], codes_np(kc0)[perm[20]])


def test_copy_blocks_refuses_chained_pairs():
    """Pairs run concurrently, so a batch may not chain copies (a block that one pair
    writes is read or written by another). Such pairs are skipped and recorded; the
    other pairs of the batch are copied as the oracle copies them (every pair reads the
    cache as it was before the call); a source shared by two pairs is allowed."""
    NB, Hkv, BS, D = 30, 2, 16, 64
    kc0 = _random_cache((NB, Hkv, BS, D), "bf16", 21)
    vc0 = _random_cache((NB, Hkv, BS, D), "bf16", 22)
    kc, vc = kc0.clone().to(DEV), vc0.clone().to(DEV)
    cache = pa.KVCache(kc, vc, "bf16")
    pairs = np.array([[1, 2], [2, 3],          # chain: 2 is written by pair 0 and read by pair 1
                      [4, 5], [6, 5],          # two writers of block 5
                      [7, 8], [7, 9],          # a shared source: allowed
                      [10, 11], [12, 10],      # pair 1's destination is pair 0's source
                      [13, 14]], dtype=np.int64)
    pa.copy_blocks(torch.from_numpy(pairs).to(DEV), cache)
    code, info = pa.last_device_error()
    assert code == 4 and (info[1], info[2]) in {tuple(r) for r in pairs[[0, 1, 2, 3, 6, 7]].tolist()}
    ok = pairs[[4, 5, 8]]
    ek, ev = oops.copy_blocks(codes_np(kc0), codes_np(vc0), ok)
    assert np.array_equal(codes_np(kc), ek) and np.array_equal(codes_np(vc), ev)


def test_block_table_update():
    bt = torch.full((5, 7), -1, dtype=torch.int32, device=DEV)
    upd = torch.tensor([[0, 0, 11], [4, 6, 3], [2, 3, 9]], dtype=torch.int32, device=DEV)
    pa.block_table_update(upd, bt)
    want = np.full((5, 7), -1, np.int32)
    want[0, 0], want[4, 6], want[2, 3] = 11, 3, 9
    assert np.array_equal(bt.cpu().numpy(), want)
    pa.block_table_update(torch.tensor([[5, 0, 1]], dtype=torch.int32, device=DEV), bt)
    assert pa.last_device_error()[0] == 5
