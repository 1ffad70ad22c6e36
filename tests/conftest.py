import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "exhaustive: long exhaustive sweep, opt-in via FO_EXHAUSTIVE=1")


def pytest_collection_modifyitems(config, items):
    if os.environ.get("FO_EXHAUSTIVE") == "1":
        return
    skip = pytest.mark.skip(reason="exhaustive sweep; set FO_EXHAUSTIVE=1")
    for item in items:
        if "exhaustive" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(autouse=True)
def _no_wait_timeouts(request):
    """After every GPU test that used the library: no step kernel gave up a
    bounded wait for a staged copy (its chunks would be left unstepped, which
    a sampled comparison could miss)."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    from bit_states_b200 import fo

    if fo._lib is not None:
        fo.fo_check_errors()


@pytest.fixture(scope="session")
def orc():
    import oracle

    oracle.build()
    return oracle


def threads():
    return max(1, min(16, os.cpu_count() or 1))
