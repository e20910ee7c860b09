import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU test")


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle.default()


@pytest.fixture(scope="session")
def nf4():
    import synth
    return synth.codebook()


@pytest.fixture(autouse=True)
def _no_failed_index_check(request):
    """Under Q4_LIBRARY=debug (the bounds-checked library build), a GPU test
    also fails when any kernel it ran met an index outside its buffer."""
    yield
    if request.node.get_closest_marker("gpu") is None or os.environ.get("Q4_LIBRARY") != "debug":
        return
    import weight_only_bit_gemv_b200 as q4
    if q4._lib is None:
        return
    assert q4.bounds_checked(), "Q4_LIBRARY=debug but the loaded library is not the checked build"
    flags = q4.bounds_flags()
    assert flags == 0, f"failed index checks, bits {flags:#x} (one bit per kernel source file)"
