"""The bounds-checked build (-DSEEDLM_CHECK=1): every kernel compares each
global and shared memory index it computes with the extent its arguments (or
its launch's shared memory) give, skips the access and raises bit 1 of
seedlm_device_error if it falls outside.  The GPU parity, encoder and
failure-path suites run again against that build, in a child process; the
conftest fixture then checks after every test that no index fell outside."""
import os
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def sl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from prng_seeded_decompress_b200 import build
    build.build(check=os.environ.get("SEEDLM_CHECKED", "0") == "1")
    from prng_seeded_decompress_b200 import seedlm
    return seedlm


def test_the_check_reaches_the_flag(sl):
    # An index one past its extent (compared on the device, never used as an
    # address) raises bit 1 in the checked build; the normal build compiles
    # the comparison away.
    torch.cuda.synchronize()
    assert sl.device_error() == 0
    sl.selftest_bounds_check(3, 4)
    torch.cuda.synchronize()
    assert sl.device_error() == 0
    sl.selftest_bounds_check(4, 4)
    torch.cuda.synchronize()
    assert sl.device_error() == (2 if sl.checked_build() else 0)
    assert sl.device_error() == 0


def test_parity_suites_pass_in_the_checked_build(sl):
    if sl.CHECKED:
        pytest.skip("already running against the checked build")
    from prng_seeded_decompress_b200 import build
    build.build(check=True)
    env = dict(os.environ, SEEDLM_CHECKED="1")
    suites = ["tests/test_gpu_parity.py", "tests/test_encode.py", "tests/test_failure_gpu.py",
              "tests/test_checked_build_gpu.py"]
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu",
                          "-p", "no:cacheprovider", *suites],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=3000)
    assert res.returncode == 0, res.stdout[-4000:] + res.stderr[-2000:]
    assert " passed" in res.stdout and " failed" not in res.stdout
