"""Failure detection on the GPU without a fault: the bounded mbarrier wait that every kernel
of the library uses gives up on a barrier nothing arrives at, records PA_DEV_WAIT_TIMEOUT in
the device error word and returns; the host reads the status, and the context stays usable
(a decode step afterwards still matches the oracle, with a clean error word)."""

import time

import pytest
import torch

import paged_kv_cache_436_b200 as pa
import synthetic
from tests.gpu_cases import run_decode_step

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_is_reported():
    assert pa.last_device_error()[0] == 0
    t0 = time.perf_counter()
    pa.selftest_wait_timeout(20000)              # 20 ms on a barrier nothing arrives at
    code, info = pa.last_device_error()
    elapsed = time.perf_counter() - t0
    assert code == 6 and info[0] == 0x7E57
    assert 20000 <= info[1] < 2000000            # the wait ran out after its limit, not at once
    assert elapsed < 5.0
    assert pa.last_device_error()[0] == 0        # reading clears the word


def test_context_usable_after_a_timeout():
    pa.selftest_wait_timeout(5000)
    assert pa.last_device_error()[0] == 6
    run_decode_step(synthetic.make("tiny"))       # parity against the oracle inside
    assert pa.last_device_error()[0] == 0
    torch.cuda.synchronize()


def test_limit_out_of_range_is_refused():
    with pytest.raises(pa.PaError):
        pa.selftest_wait_timeout(0)
    with pytest.raises(pa.PaError):
        pa.selftest_wait_timeout(3000000)
