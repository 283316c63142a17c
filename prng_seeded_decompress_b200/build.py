"""Build libseedlm.so in-tree with nvcc for sm_100a.

    python -m prng_seeded_decompress_b200.build [--force] [--verbose] [--check]

Every ``csrc/*.cu`` is compiled separately (in parallel) into ``_build/`` and
linked into ``prng_seeded_decompress_b200/libseedlm.so`` with the CUDA runtime
linked statically, so the library needs nothing but the NVIDIA driver at run time.

``--check`` builds ``libseedlm_check.so`` (objects in ``_build_check/``) with
-DSEEDLM_CHECK=1: every kernel compares each memory index it computes with
its buffer's extent and reports violations through seedlm_device_error.  The
binding loads it when SEEDLM_CHECKED=1.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OBJ = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libseedlm.so")
OBJ_CHECK = os.path.join(PKG, "_build_check")
LIB_CHECK = os.path.join(PKG, "libseedlm_check.so")
HEADERS = [os.path.join(ROOT, "include", "seedlm.h")]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
              "-Xcompiler", "-fvisibility=hidden"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: install the CUDA toolkit or set NVCC")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(CSRC, "*.h"))) + HEADERS


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def _compile(src: str, verbose: bool, check: bool = False) -> str:
    obj = os.path.join(OBJ_CHECK if check else OBJ, os.path.basename(src)[:-3] + ".o")
    # SEEDLM_NVCC_FLAGS: extra flags for experiments (e.g. -DNAME=VALUE).
    extra = os.environ.get("SEEDLM_NVCC_FLAGS", "").split()
    if check:
        extra = extra + ["-DSEEDLM_CHECK=1"]
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr)
    return obj


def build(force: bool = False, verbose: bool = False, check: bool = False) -> str:
    """Compile and link libseedlm.so (libseedlm_check.so with check=True) if
    any source changed; returns its path."""
    lib, obj_dir = (LIB_CHECK, OBJ_CHECK) if check else (LIB, OBJ)
    if not force and up_to_date(lib):
        return lib
    os.makedirs(obj_dir, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, check), sources()))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, lib)
    return lib


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/spill reports")
    ap.add_argument("--check", action="store_true", help="bounds-checked build (libseedlm_check.so)")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, check=a.check))


if __name__ == "__main__":
    main()
