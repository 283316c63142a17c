"""Failure handling on the GPU without a fault: a bounded wait that nothing
ends gives up, raises the library's device flag and leaves the context
usable (the same wait, give-up flag and TMEM handling as the tensor-core
GEMM)."""
import os

import numpy as np
import pytest

from prng_seeded_decompress_b200 import inputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from prng_seeded_decompress_b200 import build
    build.build()
    from prng_seeded_decompress_b200 import seedlm
    return seedlm


def test_timed_out_wait_raises_the_flag_and_the_context_survives(sl, oracle_mod):
    torch.cuda.synchronize()
    assert sl.device_error() == 0
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    sl.selftest_wait_timeout(2_000_000)        # 2 ms
    t1.record()
    torch.cuda.synchronize()
    assert t0.elapsed_time(t1) >= 1.9          # it really waited its limit ...
    assert sl.device_error() == 1              # ... gave up and said so
    assert sl.device_error() == 0              # reading clears the flag
    # The context is intact: a GEMM (TMEM again) still matches the oracle.
    L = inputs.make_layer(256, 1024, *inputs.FORMAT_4BIT, seed=5)
    Xb, Xv = inputs.make_activations((16, 1024), "bf16", 6)
    rec = torch.from_numpy(L["rec"].view(np.int32)).cuda()
    X = torch.from_numpy(Xb.view(np.int16)).cuda().view(torch.bfloat16)
    Y = torch.empty((16, 256), device="cuda")
    sl.gemm_smallM(L["fmt"], rec, None, X, Y)
    torch.cuda.synchronize()
    assert sl.device_error() == 0
    ref, refabs = oracle_mod.gemm(L["fmt"], L["rec"], None, Xv, threads=os.cpu_count() or 1)
    got = Y.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= 1e-5 * refabs + 1e-30)
