import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


import pytest  # noqa: E402


@pytest.fixture(autouse=True)
def _clear_device_error_word(request):
    """A GPU test starts with a clear device error word: a test that failed before reading
    an error it provoked must not fail the next one."""
    if request.node.get_closest_marker("gpu") is not None:
        import torch
        if torch.cuda.is_available():
            import paged_kv_cache_436_b200 as pa
            try:
                pa.last_device_error()
            except Exception:
                pass
    yield
