import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

CHECKED_RUN = os.environ.get("CSKV_CHECK", "0") not in ("", "0")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workload (minutes)")
    config.addinivalue_line("markers",
                            "bounds_events: feeds out-of-range device indices on purpose "
                            "(checked build) and reads the events itself")


@pytest.fixture(autouse=True)
def _no_bounds_event_in_a_checked_run(request):
    """With the checked build loaded (CSKV_CHECK=1), every GPU test ends with
    a read of the device status word: a valid call must not have recorded an
    out-of-range index."""
    yield
    if not CHECKED_RUN or request.node.get_closest_marker("gpu") is None:
        return
    if request.node.get_closest_marker("bounds_events") is not None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    import compressed_sparse_kv_softmax_b200 as C
    ev = C.check_device_errors()
    assert not ev & C.DEV_BOUNDS, f"the checked build recorded an out-of-range index ({ev:#x})"
