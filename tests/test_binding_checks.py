"""The binding refuses arguments a kernel would read out of bounds -- host tensors,
wrong element types, short buffers -- before any pointer reaches the library. These
refusals need no GPU: each raises before a stream is even looked up."""

import pytest
import torch

import paged_kv_cache_436_b200 as pa
from paged_kv_cache_436_b200 import build as pa_build


@pytest.fixture(scope="module", autouse=True)
def built_library():
    if pa_build.stale():
        pa_build.build()
    return pa.lib()


def _cache(D=64):
    c = torch.zeros((4, 2, 16, D), dtype=torch.bfloat16)
    return pa.KVCache(c, c.clone(), "bf16")


def test_host_tensors_never_reach_a_kernel():
    cache = _cache()
    q = torch.zeros((3, 4, 64), dtype=torch.bfloat16)
    bt = torch.zeros((3, 2), dtype=torch.int32)
    lens = torch.ones(3, dtype=torch.int32)
    ws = torch.zeros(1 << 16, dtype=torch.uint8)
    qs = torch.tensor([0, 1, 2, 3], dtype=torch.int32)
    kv = torch.zeros((3, 2, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        pa.decode(q, cache, bt, lens, 32, 0.125, torch.empty_like(q), ws)
    with pytest.raises(ValueError, match="CUDA"):
        pa.decode_no_alloc(q, cache, bt, lens, 32, 0.125, torch.empty_like(q))
    with pytest.raises(ValueError, match="CUDA"):
        pa.extend(q, cache, qs, bt, lens, 32, 0.125, torch.empty_like(q), ws)
    with pytest.raises(ValueError, match="CUDA"):
        pa.prefill(q, kv, kv, cache, qs, bt, lens, 32, 0.125, torch.empty_like(q), ws)
    with pytest.raises(ValueError, match="CUDA"):
        pa.reshape_and_cache(kv, kv, torch.zeros(3, dtype=torch.int64), cache)
    with pytest.raises(ValueError, match="CUDA"):
        pa.copy_blocks(torch.zeros((1, 2), dtype=torch.int64), cache)
    with pytest.raises(ValueError, match="CUDA"):
        pa.block_table_update(torch.zeros((1, 3), dtype=torch.int32), bt)


def test_check_helper_rules():
    """The rules themselves, on a stand-in that reports itself as a CUDA tensor."""
    class Fake:
        def __init__(self, t, cuda=True):
            self.t, self.is_cuda = t, cuda
            self.dtype, self.shape = t.dtype, t.shape

        def dim(self):
            return self.t.dim()

        def is_contiguous(self):
            return self.t.is_contiguous()

        def numel(self):
            return self.t.numel()

    i32 = torch.zeros((4, 3), dtype=torch.int32)
    pa._dev(Fake(i32), "x", torch.int32, 2, 12)
    with pytest.raises(ValueError):
        pa._dev(Fake(i32, cuda=False), "x")
    with pytest.raises(TypeError):
        pa._dev(Fake(i32), "x", torch.int64)
    with pytest.raises(ValueError):
        pa._dev(Fake(i32), "x", torch.int32, 1)
    with pytest.raises(ValueError):
        pa._dev(Fake(i32.t()), "x", torch.int32, 2)                     # transposed view
    pa._dev(Fake(i32.t()), "x", torch.int32, 2, contiguous=False)
    with pytest.raises(ValueError):
        pa._dev(Fake(i32), "x", torch.int32, 2, 13)                     # one element short
    pa._dev(Fake(i32), "x", (torch.float16, torch.int32))


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No fallback: without libpa.so every entry point raises LibraryMissing."""
    monkeypatch.setattr(pa, "LIB_PATH", str(tmp_path / "libpa.so"))
    monkeypatch.setattr(pa, "_lib", None)
    with pytest.raises(pa.LibraryMissing):
        pa.lib()
    with pytest.raises(pa.LibraryMissing):
        pa.Pool(4)
    with pytest.raises(pa.LibraryMissing):
        pa.PrefixCache(16)
    with pytest.raises(pa.LibraryMissing):
        pa.decode_workspace_size(1, 1, 128, 16)
    (tmp_path / "libpa.so").write_bytes(b"not a shared object")
    with pytest.raises(pa.LibraryMissing):
        pa.lib()
