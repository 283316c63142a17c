"""CPU oracle for SeedLM reconstruction and products -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (the CUDA library and its
Python binding) never imports it, and it never imports the product.

The arithmetic lives in plain C (``seedlm_oracle.c``, fp64, see its header for
the definitions it follows and the pages it cites); this module only marshals
NumPy arrays into it.  ``search.py`` adds the brute-force seed search used by
the planted-seed pin.
"""
from __future__ import annotations

import ctypes
import functools
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "seedlm_oracle.c")
_HDR = os.path.join(_HERE, "seedlm_oracle.h")
_LIB = os.path.join(_HERE, "liboracle_seedlm.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle_seedlm.so`` with gcc."""
    newest_src = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest_src:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
               "-pthread", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


class _Fmt(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("C", "P", "K", "rows", "cols", "nb", "rec_pitch", "e_pitch")]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.POINTER
            lib.oracle_lfsr_next.restype = ctypes.c_uint16
            lib.oracle_lfsr_next.argtypes = [ctypes.c_uint16]
            lib.oracle_lfsr_states.argtypes = [ctypes.c_uint16, ctypes.c_int, ctypes.c_void_p]
            lib.oracle_check_format.argtypes = [P(_Fmt)]
            lib.oracle_block_fields.argtypes = [P(_Fmt), ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_void_p]
            lib.oracle_block_basis.argtypes = [ctypes.c_uint16, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_void_p]
            lib.oracle_basis_all.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
            lib.oracle_reconstruct_block.argtypes = [P(_Fmt), ctypes.c_void_p, ctypes.c_void_p,
                                                     ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
            lib.oracle_decompress.argtypes = [P(_Fmt), ctypes.c_void_p, ctypes.c_void_p,
                                              ctypes.c_void_p]
            lib.oracle_gemv.argtypes = [P(_Fmt), ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_int]
            lib.oracle_gemm.argtypes = [P(_Fmt), ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_int]
            u32 = ctypes.c_uint32
            lib.oracle_lfsr_next_k.restype = u32
            lib.oracle_lfsr_next_k.argtypes = [u32, ctypes.c_int, u32]
            lib.oracle_lfsr_period_k.restype = ctypes.c_uint64
            lib.oracle_lfsr_period_k.argtypes = [ctypes.c_int, u32]
            lib.oracle_block_basis_k.argtypes = [u32, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                 u32, ctypes.c_void_p]
            lib.oracle_basis_all_k.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, u32,
                                               ctypes.c_void_p]
            _lib = lib
    return _lib


def _fmt(fmt: dict) -> _Fmt:
    f = _Fmt(*(int(fmt[k]) for k in ("C", "P", "K", "rows", "cols", "nb", "rec_pitch",
                                      "e_pitch")))
    if _load().oracle_check_format(ctypes.byref(f)) != 0:
        raise ValueError(f"oracle: invalid format {fmt}")
    return f


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _planes(fmt, rec, eplane):
    rec = np.ascontiguousarray(rec, dtype=np.uint32)
    if rec.size < fmt["rows"] * fmt["rec_pitch"]:
        raise ValueError("oracle: record array too small")
    if fmt["P"] == 4:
        eplane = np.ascontiguousarray(eplane, dtype=np.uint8)
        if eplane.size < fmt["rows"] * fmt["e_pitch"]:
            raise ValueError("oracle: exponent plane too small")
    else:
        eplane = None
    return rec, eplane


def lfsr_next(s: int) -> int:
    return int(_load().oracle_lfsr_next(s))


def lfsr_states(seed: int, n: int) -> np.ndarray:
    out = np.zeros(n, dtype=np.uint16)
    _load().oracle_lfsr_states(seed, n, _ptr(out))
    return out


def block_fields(fmt, rec, eplane, r, b):
    """(seed, q[P], e) of block b in row r, decoded from the record layout."""
    f = _fmt(fmt)
    rec, eplane = _planes(fmt, rec, eplane)
    seed = np.zeros(1, np.uint16)
    q = np.zeros(4, np.int32)
    e = np.zeros(1, np.int32)
    _load().oracle_block_fields(ctypes.byref(f), _ptr(rec), _ptr(eplane), r, b,
                                _ptr(seed), _ptr(q), _ptr(e))
    return int(seed[0]), q[: fmt["P"]].copy(), int(e[0])


def block_basis(seed: int, C: int, P: int) -> np.ndarray:
    """U(seed) as a (C, P) float64 array."""
    U = np.zeros((C, P), np.float64)
    _load().oracle_block_basis(seed, C, P, _ptr(U))
    return U


def basis_all(C: int, P: int) -> np.ndarray:
    """U(s) for s = 1..65535 as a (65535, C, P) float64 array."""
    U = np.zeros((65535, C, P), np.float64)
    _load().oracle_basis_all(C, P, _ptr(U))
    return U


# ------------------------------------------------------ design-space variants

#: Taps of the 16-bit register the workload specifies (bits 0, 2, 3, 5:
#: s ^ s>>2 ^ s>>3 ^ s>>5).
TAPS_K16 = 0x2D


def lfsr_next_k(s: int, K: int, taps: int) -> int:
    return int(_load().oracle_lfsr_next_k(s, K, taps))


def lfsr_period_k(K: int, taps: int) -> int:
    """Steps from state 1 back to 1 (0 if it never returns within 2^K)."""
    return int(_load().oracle_lfsr_period_k(K, taps))


@functools.lru_cache(maxsize=None)
def primitive_taps(K: int) -> int:
    """Taps of the K-bit register used for the design-space variants: the
    spec's taps for K = 16, otherwise the smallest odd tap mask whose register
    visits all 2^K - 1 nonzero states (found by brute force; the pages give
    no polynomial for any K)."""
    if K == 16:
        return TAPS_K16
    full = (1 << K) - 1
    for taps in range(1, 1 << K, 2):
        if lfsr_period_k(K, taps) == full:
            return taps
    raise ValueError(f"no maximal-length register for K = {K}")


def block_basis_k(seed: int, C: int, P: int, K: int, taps: int) -> np.ndarray:
    U = np.zeros((C, P), np.float64)
    _load().oracle_block_basis_k(seed, C, P, K, taps, _ptr(U))
    return U


def basis_all_k(C: int, P: int, K: int, taps: int) -> np.ndarray:
    """U(s) for s = 1 .. 2^K - 1 as a (2^K - 1, C, P) float64 array."""
    U = np.zeros(((1 << K) - 1, C, P), np.float64)
    _load().oracle_basis_all_k(C, P, K, taps, _ptr(U))
    return U


def reconstruct_block(fmt, rec, eplane, r, b) -> np.ndarray:
    f = _fmt(fmt)
    rec, eplane = _planes(fmt, rec, eplane)
    w = np.zeros(fmt["C"], np.float64)
    _load().oracle_reconstruct_block(ctypes.byref(f), _ptr(rec), _ptr(eplane), r, b, _ptr(w))
    return w


def decompress(fmt, rec, eplane=None) -> np.ndarray:
    """W as a (rows, cols) float64 array (every entry exact)."""
    f = _fmt(fmt)
    rec, eplane = _planes(fmt, rec, eplane)
    W = np.zeros((fmt["rows"], fmt["cols"]), np.float64)
    if _load().oracle_decompress(ctypes.byref(f), _ptr(rec), _ptr(eplane), _ptr(W)) != 0:
        raise ValueError("oracle_decompress failed")
    return W


def gemv(fmt, rec, eplane, x, threads: int = 1):
    """(y, yabs): y = W x and yabs = |W| |x|, both float64 of length rows."""
    f = _fmt(fmt)
    rec, eplane = _planes(fmt, rec, eplane)
    x = np.ascontiguousarray(x, dtype=np.float64)
    if x.shape != (fmt["cols"],):
        raise ValueError("oracle.gemv: x must have shape (cols,)")
    y = np.zeros(fmt["rows"], np.float64)
    ya = np.zeros(fmt["rows"], np.float64)
    if _load().oracle_gemv(ctypes.byref(f), _ptr(rec), _ptr(eplane), _ptr(x), _ptr(y),
                           _ptr(ya), threads) != 0:
        raise ValueError("oracle_gemv failed")
    return y, ya


def gemm(fmt, rec, eplane, X, threads: int = 1):
    """(Y, Yabs): Y[m] = W X[m], shapes (M, rows); X is (M, cols)."""
    f = _fmt(fmt)
    rec, eplane = _planes(fmt, rec, eplane)
    X = np.ascontiguousarray(X, dtype=np.float64)
    if X.ndim != 2 or X.shape[1] != fmt["cols"]:
        raise ValueError("oracle.gemm: X must have shape (M, cols)")
    M = X.shape[0]
    Y = np.zeros((M, fmt["rows"]), np.float64)
    Ya = np.zeros((M, fmt["rows"]), np.float64)
    if _load().oracle_gemm(ctypes.byref(f), _ptr(rec), _ptr(eplane), _ptr(X), M, _ptr(Y),
                           _ptr(Ya), threads) != 0:
        raise ValueError("oracle_gemm failed")
    return Y, Ya


def gemv_rows(fmt, rec, eplane, x, rows):
    """y and yabs for a subset of rows only (sampled checks at full size)."""
    rows = np.asarray(rows, dtype=np.int64)
    sub = dict(fmt)
    sub["rows"] = len(rows)
    rec = np.asarray(rec).reshape(fmt["rows"], fmt["rec_pitch"])[rows]
    ep = None
    if fmt["P"] == 4:
        ep = np.asarray(eplane).reshape(fmt["rows"], fmt["e_pitch"])[rows]
    return gemv(sub, rec, ep, x)


def gemm_rows(fmt, rec, eplane, X, rows):
    """Y and Yabs (M, len(rows)) for a subset of rows only."""
    rows = np.asarray(rows, dtype=np.int64)
    sub = dict(fmt)
    sub["rows"] = len(rows)
    rec = np.asarray(rec).reshape(fmt["rows"], fmt["rec_pitch"])[rows]
    ep = None
    if fmt["P"] == 4:
        ep = np.asarray(eplane).reshape(fmt["rows"], fmt["e_pitch"])[rows]
    return gemm(sub, rec, ep, X)
