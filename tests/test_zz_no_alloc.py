"""seedlm_gemm_smallM_noalloc: the small-M GEMM for callers that cannot
allocate device memory (a library embedded in a host program that owns the
GPU's memory pool, or a path that must not pay cudaMalloc's implicit device
synchronisation), so cannot hand in a workspace.  Its workspace is an array
inside libseedlm.so.

These tests call the entry point through the C ABI (ctypes) on two calls in
a row -- the second call finds the scratch exactly as the first one left it
-- and check each result twice: bit for bit against seedlm_gemm_smallM with
a caller workspace (the same kernel with the same split, so the same bits),
and against the fp64 CPU oracle within the tolerance every GPU product test
uses.  The file is named so that pytest collects it last.
"""
import ctypes
import os

import numpy as np
import pytest

from prng_seeded_decompress_b200 import inputs

torch = pytest.importorskip("torch")

TOL = 1e-5
C8, C12 = inputs.FORMAT_4BIT, inputs.FORMAT_3BIT


@pytest.fixture(scope="module")
def sl():
    from prng_seeded_decompress_b200 import build
    build.build()
    from prng_seeded_decompress_b200 import seedlm
    return seedlm


def test_noalloc_rejects_bad_arguments_before_cuda(sl):
    f = sl.Format.from_dict(dict(C=8, P=3, K=16, rows=4, cols=64, nb=8, rec_pitch=8, e_pitch=0))
    call = sl.lib.seedlm_gemm_smallM_noalloc
    assert call(None, 0x1000, None, 0x2000, 0, 4, 0x3000, None) == -1
    assert call(ctypes.byref(f), 0x1008, None, 0x2000, 0, 4, 0x3000, None) == -1
    for M in (0, 65):
        assert call(ctypes.byref(f), 0x1000, None, 0x2000, 0, M, 0x3000, None) == -1
    bad = sl.Format.from_dict(dict(C=9, P=3, K=16, rows=4, cols=64, nb=8, rec_pitch=8,
                                   e_pitch=0))
    assert call(ctypes.byref(bad), 0x1000, None, 0x2000, 0, 4, 0x3000, None) == -2


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _act(bits, dtype):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
    return t.view(torch.float16 if dtype == "f16" else torch.bfloat16)


def _noalloc(sl, L, rec, ep, X, Y):
    f = sl.Format.from_dict(L["fmt"])
    dt = 1 if X.dtype == torch.bfloat16 else 0
    stream = torch.cuda.current_stream().cuda_stream
    rc = sl.lib.seedlm_gemm_smallM_noalloc(
        ctypes.byref(f), rec.data_ptr(), None if ep is None else ep.data_ptr(), X.data_ptr(), dt,
        int(X.shape[0]), Y.data_ptr(), stream)
    return rc


@pytest.mark.gpu
@pytest.mark.parametrize("cp,rows,cols,M,dtype", [
    (C8, 1000, 8192, 64, "bf16"),   # 8 row tiles x 32 column splits
    (C12, 300, 3000, 17, "bf16"),   # ragged tiles, 3-bit
    (C8, 129, 777, 5, "f16"),       # ragged everything, fp16
    (C8, 256, 4096, 1, "bf16"),     # M = 1 (the GEMV kernel)
])
def test_noalloc_matches_workspace_entry_on_two_calls(sl, oracle_mod, cp, rows, cols, M, dtype):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = inputs.make_layer(rows, cols, *cp, seed=rows + cols + M)
    Xb, Xv = inputs.make_activations((M, cols), dtype, 7 + M)
    rec = _dev(L["rec"].view(np.int32))
    ep = _dev(L["eplane"]) if cp[1] == 4 else None
    X = _act(Xb, dtype)
    Y_ws = torch.full((M, rows), float("nan"), device="cuda")
    sl.gemm_smallM(L["fmt"], rec, ep, X, Y_ws, workspace=sl.gemm_workspace(L["fmt"], M))
    torch.cuda.synchronize()
    ws_bits = Y_ws.cpu().numpy().view(np.uint32)
    ref, refabs = oracle_mod.gemm(L["fmt"], L["rec"], L["eplane"], Xv,
                                  threads=os.cpu_count() or 1)
    for call in range(2):
        Y = torch.full((M, rows), float("nan"), device="cuda")
        assert _noalloc(sl, L, rec, ep, X, Y) == 0
        torch.cuda.synchronize()
        assert sl.device_error() == 0
        got = Y.cpu().numpy()
        assert np.array_equal(got.view(np.uint32), ws_bits), f"call {call}: differs from the " \
            "workspace entry point"
        err = np.abs(got.astype(np.float64) - ref)
        assert np.all(err <= TOL * refabs + 1e-30), f"call {call}: max err {err.max()}"


@pytest.mark.gpu
def test_noalloc_rejects_problems_beyond_its_scratch(sl):
    # 57344 rows = 448 row tiles over 8192 columns (64 chunks each) at
    # M = 64: one CTA per SM takes about 194 of the 28,672 (tile, chunk)
    # units, so it touches up to four row tiles and keeps a 32 KiB partial
    # tile for each: 148 x 4 x 32 KiB is more than the 16 MiB + 64 KiB the library
    # holds, and the call must be refused before anything is launched.
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    rows, cols, M = 57344, 8192, 64
    fmt = inputs.make_format(rows, cols, *C8)
    need = sl.gemm_workspace_bytes(fmt, M)
    assert need > (16 << 20) + (64 << 10), need
    rec = torch.zeros((rows, fmt["rec_pitch"]), dtype=torch.int32, device="cuda")
    X = torch.zeros((M, cols), dtype=torch.bfloat16, device="cuda")
    Y = torch.full((M, rows), 7.0, device="cuda")
    L = dict(fmt=fmt)
    n0 = sl.launch_count()
    assert _noalloc(sl, L, rec, None, X, Y) == -2
    torch.cuda.synchronize()
    assert sl.launch_count() == n0
    assert bool((Y == 7.0).all())
