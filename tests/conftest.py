import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name):
    """Parse a `key = value` fixture; values with spaces become int lists."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = [s.strip() for s in line.split("=", 1)]
            parts = val.split()
            out[key] = [int(p) for p in parts] if len(parts) > 1 else int(parts[0])
    return out


@pytest.fixture(scope="session")
def golden():
    return read_golden


@pytest.fixture(autouse=True)
def _short_device_waits(request):
    """GPU tests run with a 200 ms bound on every device-side wait, so a
    broken pipeline shows up as SWA_ERR_TIMEOUT quickly instead of stalling."""
    if request.node.get_closest_marker("gpu") is None:
        yield
        return
    import decode_swa_prefill_b200 as swa
    swa.swa_set_wait_limit_ns(200_000_000)
    yield
    status = swa.swa_get_device_status()
    swa.swa_set_wait_limit_ns(2_000_000_000)
    assert status in (swa.SWA_OK,), "device status word set after test: %d" % status
