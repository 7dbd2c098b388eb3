import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the CUDA library")
    config.addinivalue_line("markers", "slow: full-size workloads")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(autouse=True)
def guard_bands(request):
    """For every GPU test: the binding allocates each output and workspace
    between canary bands (tests/gpu_util.GuardedAllocator), and the bands are
    checked when the test ends, so a write past either end of any output
    fails the test."""
    if request.node.get_closest_marker("gpu") is None:
        yield None
        return
    import nvfp4_block_scaled_sm_b200 as mxq
    from gpu_util import GuardedAllocator
    alloc = GuardedAllocator()
    prev = mxq.set_output_allocator(alloc)
    try:
        yield alloc
    finally:
        mxq.set_output_allocator(prev)
    alloc.check()
