"""The plumbing the full-size GPU parity tests use to run the oracle on every host core
(caches in shared memory, one spawned process per core, rows grouped per sequence) gives
exactly the rows of a plain serial oracle call, for decode and for extend (CPU only)."""

import numpy as np
import torch

from oracle import attention as oatt
from tests.gpu_cases import _device_to_shared, oracle_rows_parallel


def _cache(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def test_pooled_oracle_equals_serial_oracle():
    NB, Hkv, BS, D, Hq = 12, 2, 16, 64, 4
    kc, vc = _cache((NB, Hkv, BS, D), 1), _cache((NB, Hkv, BS, D), 2)
    lens = [5, 40, 17]
    bt = np.array([[3, 0, 0], [1, 7, 9], [11, 2, 0]], np.int64)
    q = _cache((3, Hq, D), 3).view(torch.int16).numpy().view(np.uint16)
    shm_k, k = _device_to_shared(kc)
    shm_v, v = _device_to_shared(vc)
    try:
        assert np.array_equal(k, kc.view(torch.int16).numpy().view(np.uint16))
        groups = [[(s, h) for h in range(Hq)] for s in range(3)]
        got = oracle_rows_parallel("decode", shm_k, shm_v, k.shape, k.itemsize,
                                   (q, "bf16", "bf16", 1.0, 1.0, bt, lens, 0.125), groups)
        want = oatt.paged_decode(q, "bf16", k, v, "bf16", 1.0, 1.0, bt, lens, 0.125)
        assert len(got) == 3 * Hq and all(np.array_equal(got[r], want[r]) for r in got)
        qs = np.array([0, 2, 5, 6], np.int32)
        qe = _cache((6, Hq, D), 4).view(torch.int16).numpy().view(np.uint16)
        groups = [[(t, h) for t in range(qs[s], qs[s + 1]) for h in range(Hq)] for s in range(3)]
        got = oracle_rows_parallel("extend", shm_k, shm_v, k.shape, k.itemsize,
                                   (qe, "bf16", "bf16", 1.0, 1.0, bt, lens, qs, 0.125), groups)
        want = oatt.paged_extend(qe, "bf16", k, v, "bf16", 1.0, 1.0, bt, lens, qs, 0.125)
        assert len(got) == 6 * Hq and all(np.array_equal(got[r], want[r]) for r in got)
    finally:
        for shm in (shm_k, shm_v):
            shm.close()
            shm.unlink()
