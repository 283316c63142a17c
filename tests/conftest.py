import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(autouse=True)
def device_flags_stay_clear(request):
    """After every GPU test: no kernel gave up on a bounded wait and, in the
    bounds-checked build, none skipped an out-of-bounds access (tests that
    raise a flag on purpose read and clear it themselves)."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    mod = sys.modules.get("prng_seeded_decompress_b200.seedlm")
    if mod is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    torch.cuda.synchronize()
    assert mod.device_error() == 0, "a kernel raised the device error flag during this test"
