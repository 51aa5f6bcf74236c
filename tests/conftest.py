import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")


def read_golden(name):
    """Rows of a golden text fixture, comments stripped, split on whitespace."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


def golden_dict(name):
    return {r[0]: r[1] for r in read_golden(name)}


@pytest.fixture(autouse=True)
def _device_status_clean(request):
    """After every GPU test: the library's device status word is clean (a bounded wait that
    gave up inside any kernel of the test would otherwise go unnoticed)."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    import nvfp4_block_scaled_14_b200 as nv
    torch.cuda.synchronize()
    st = nv.sync_status()
    assert st == 0, f"device status {st} left by the test"
