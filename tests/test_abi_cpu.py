"""The C-ABI library builds, loads without a GPU and exports what its header
declares; argument checks reject bad calls before any CUDA work (no GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "seedlm.h")


@pytest.fixture(scope="module")
def sl():
    from prng_seeded_decompress_b200 import build
    build.build()
    from prng_seeded_decompress_b200 import seedlm
    return seedlm


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(seedlm_[a-zA-Z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("seedlm_decompress", "seedlm_gemv", "seedlm_gemm_smallM", "seedlm_gemm",
              "seedlm_init", "seedlm_strerror", "seedlm_shutdown"):
        assert n in names


def test_library_exports_every_declared_symbol(sl):
    names = declared_functions()
    lib = ctypes.CDLL(sl.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(sl.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", sl.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (seedlm_\w+)", out))
    assert exported == set(names)


def test_checked_build_exports_the_same_symbols(sl):
    # The bounds-checked build (-DSEEDLM_CHECK=1) is the same boundary; only
    # seedlm_checked_build tells the two apart.
    from prng_seeded_decompress_b200 import build
    path = build.build(check=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True,
                         text=True, check=True).stdout
    assert set(re.findall(r"\bT (seedlm_\w+)", out)) == set(declared_functions())
    assert ctypes.CDLL(path).seedlm_checked_build() == 1
    assert sl.lib.seedlm_checked_build() == (1 if sl.CHECKED else 0)


def test_selftest_arguments_are_checked_before_cuda(sl):
    assert sl.lib.seedlm_selftest_bounds_check(-1, 4, None) == -1
    assert sl.lib.seedlm_selftest_bounds_check(0, -4, None) == -1


def test_strerror_and_counters(sl):
    assert sl.strerror(0) == "success"
    for c in (-1, -2, -3, 7):
        assert isinstance(sl.strerror(c), str) and sl.strerror(c)
    assert sl.last_cuda_error() == 0
    assert sl.launch_count() == 0


def _fmt(**kw):
    d = dict(C=8, P=3, K=16, rows=4, cols=64, nb=8, rec_pitch=8, e_pitch=0)
    d.update(kw)
    return d


def test_row_bytes(sl):
    assert sl.row_bytes(_fmt()) == (32, 32)
    f3 = dict(C=12, P=4, K=16, rows=1, cols=4096, nb=342, rec_pitch=344, e_pitch=176)
    assert sl.row_bytes(f3) == (342 * 36 // 8, 4 * 344 + 176)
    assert sl.row_bytes(_fmt(C=9)) == (-1, -1)


@pytest.mark.parametrize("kw,code", [
    (dict(C=9), -2), (dict(P=4), -2), (dict(K=12), -2),
    (dict(nb=7), -1), (dict(rec_pitch=6), -1), (dict(rec_pitch=10), -1),
    (dict(rows=-1), -1), (dict(cols=-8, nb=-1), -1),
])
def test_bad_formats_are_rejected_before_cuda(sl, kw, code):
    f = sl.Format.from_dict(_fmt(**kw))
    rc = sl.lib.seedlm_gemv(ctypes.byref(f), 0x1000, None, 0x2000, 0, 0x3000, None)
    assert rc == code
    rc = sl.lib.seedlm_decompress(ctypes.byref(f), 0x1000, None, 0x2000, 64, None)
    assert rc == code


def test_bad_pointers_are_rejected_before_cuda(sl):
    f = sl.Format.from_dict(_fmt())
    L = sl.lib
    assert L.seedlm_gemv(ctypes.byref(f), None, None, 0x2000, 0, 0x3000, None) == -1
    assert L.seedlm_gemv(ctypes.byref(f), 0x1008, None, 0x2000, 0, 0x3000, None) == -1
    assert L.seedlm_gemv(ctypes.byref(f), 0x1000, None, 0x2000, 5, 0x3000, None) == -1
    assert L.seedlm_gemv(ctypes.byref(f), 0x1000, None, 0x2001, 0, 0x3000, None) == -1
    assert L.seedlm_gemv(ctypes.byref(f), 0x1000, None, 0x2000, 0, 0x3002, None) == -1
    assert L.seedlm_gemv(None, 0x1000, None, 0x2000, 0, 0x3000, None) == -1
    f3 = sl.Format.from_dict(dict(C=12, P=4, K=16, rows=2, cols=24, nb=2, rec_pitch=4,
                                  e_pitch=16))
    assert L.seedlm_gemv(ctypes.byref(f3), 0x1000, None, 0x2000, 0, 0x3000, None) == -1
    f3b = sl.Format.from_dict(dict(C=12, P=4, K=16, rows=2, cols=24, nb=2, rec_pitch=4,
                                   e_pitch=0))
    assert L.seedlm_gemv(ctypes.byref(f3b), 0x1000, 0x4000, 0x2000, 0, 0x3000, None) == -1
    for M in (0, 65, -1):
        assert L.seedlm_gemm_smallM(ctypes.byref(f), 0x1000, None, 0x2000, 0, M, 0x3000,
                                    None, 0, None) == -1
        assert L.seedlm_gemm_smallM_workspace_bytes(ctypes.byref(f), M) == -1
    assert L.seedlm_gemm_smallM(ctypes.byref(f), 0x1000, None, 0x2000, 0, 4, 0x3000,
                                None, -1, None) == -1
    for M in (0, -1):
        assert L.seedlm_gemm(ctypes.byref(f), 0x1000, None, 0x2000, 0, M, 0x3000,
                             None, 0, None) == -1
        assert L.seedlm_gemm_workspace_bytes(ctypes.byref(f), M) == -1
    assert L.seedlm_gemm(ctypes.byref(f), 0x1000, None, 0x2000, 0, 300, 0x3000, None, -1, None) == -1
    assert L.seedlm_gemm(ctypes.byref(f), 0x1000, None, 0x2000, 7, 300, 0x3000, None, 0, None) == -1
    assert L.seedlm_gemm(ctypes.byref(f), 0x1000, None, 0x2001, 0, 300, 0x3000, None, 0, None) == -1
    assert L.seedlm_device_error(None) == -1
    for limit in (0, 999, 100000001):
        assert L.seedlm_selftest_wait_timeout(limit, None) == -1
    assert L.seedlm_decompress(ctypes.byref(f), 0x1000, None, 0x2000, 63, None) == -1
    assert L.seedlm_dense_gemv_f16(4, 64, 0x1008, 64, 0x2000, 0x3000, None) == -1
    assert L.seedlm_dense_gemv_f16(4, 64, 0x1000, 60, 0x2000, 0x3000, None) == -1
    # Empty work is accepted without touching a device.
    f0 = sl.Format.from_dict(_fmt(rows=0))
    assert L.seedlm_gemv(ctypes.byref(f0), None, None, None, 0, None, None) == 0
    assert L.seedlm_decompress(ctypes.byref(f0), None, None, None, 64, None) == 0
    assert sl.launch_count() == 0


def test_binding_refuses_to_run_without_the_library(tmp_path):
    # A fresh interpreter that cannot find libseedlm.so must fail loudly.
    code = (
        "import sys, os, shutil\n"
        f"sys.path.insert(0, {str(tmp_path)!r})\n"
        "import prng_seeded_decompress_b200.seedlm\n"
    )
    pkg = tmp_path / "prng_seeded_decompress_b200"
    pkg.mkdir()
    for f in ("__init__.py", "seedlm.py"):
        (pkg / f).write_text(open(os.path.join(ROOT, "prng_seeded_decompress_b200", f)).read())
    res = subprocess.run(["python", "-c", code], capture_output=True, text=True)
    assert res.returncode != 0 and "libseedlm.so is missing" in res.stderr


def test_binding_refuses_layouts_the_library_cannot_read(sl):
    # Row-major with unit column stride is what the library addresses; a
    # transposed or strided tensor is refused before any call (CPU tensors
    # stand in for device ones: only the layout is looked at).
    torch = pytest.importorskip("torch")
    W = torch.empty((6, 10))
    assert sl._row_major_ld(W, 10) == 10
    assert sl._row_major_ld(torch.empty((6, 16))[:, :10], 10) == 16
    assert sl._row_major_ld(torch.empty((1, 10)), 10) == 10
    with pytest.raises(ValueError, match="unit column stride"):
        sl._row_major_ld(W.t(), 6)
    with pytest.raises(ValueError, match="unit column stride"):
        sl._row_major_ld(torch.empty(10), 10)
    with pytest.raises(ValueError, match="contiguous"):
        sl._dense(torch.empty((4, 8))[:, ::2], "X")
    assert sl._dense(torch.empty(5), "x").numel() == 5
