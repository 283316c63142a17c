"""ctypes binding of libseedlm.so (see include/seedlm.h for the contract).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels.  Tensors are passed as raw device pointers; the stream defaults
to PyTorch's current stream on the tensors' device.  If the library has not
been built, importing this module raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
#: SEEDLM_CHECKED=1 loads the bounds-checked build (`build --check`) instead.
CHECKED = os.environ.get("SEEDLM_CHECKED", "0") == "1"
LIB_PATH = os.path.join(PKG, "libseedlm_check.so" if CHECKED else "libseedlm.so")

F16 = 0
BF16 = 1

#: Every symbol include/seedlm.h declares.
EXPORTS = (
    "seedlm_init", "seedlm_decompress", "seedlm_gemv", "seedlm_gemm_smallM",
    "seedlm_gemm_smallM_workspace_bytes", "seedlm_gemm_smallM_noalloc", "seedlm_gemm",
    "seedlm_gemm_workspace_bytes", "seedlm_device_error",
    "seedlm_dense_gemv_f16", "seedlm_row_bytes_ideal", "seedlm_row_bytes_stored",
    "seedlm_strerror", "seedlm_last_cuda_error", "seedlm_launch_count", "seedlm_shutdown",
    "seedlm_encode", "seedlm_selftest_wait_timeout", "seedlm_checked_build",
    "seedlm_selftest_bounds_check", "seedlm_search_blocks", "seedlm_lfsr_taps",
    "seedlm_gemv_batch",
)


class SeedLMError(RuntimeError):
    def __init__(self, fn: str, code: int, detail: str):
        super().__init__(f"{fn} failed with {code}: {detail}")
        self.code = code


class Format(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("C", "P", "K", "rows", "cols", "nb", "rec_pitch", "e_pitch")]

    @classmethod
    def from_dict(cls, d: dict) -> "Format":
        return cls(*(int(d[k]) for k in ("C", "P", "K", "rows", "cols", "nb", "rec_pitch",
                                         "e_pitch")))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m prng_seeded_decompress_b200.build"
            f"{' --check' if CHECKED else ''}` (the SeedLM kernels have no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    fmtp = ctypes.POINTER(Format)
    sig = {
        "seedlm_init": (ctypes.c_int, []),
        "seedlm_decompress": (ctypes.c_int, [fmtp, vp, vp, vp, i64, vp]),
        "seedlm_gemv": (ctypes.c_int, [fmtp, vp, vp, vp, ctypes.c_int, vp, vp]),
        "seedlm_gemm_smallM": (ctypes.c_int, [fmtp, vp, vp, vp, ctypes.c_int, ctypes.c_int, vp,
                                              vp, i64, vp]),
        "seedlm_gemm_smallM_workspace_bytes": (i64, [fmtp, ctypes.c_int]),
        "seedlm_gemm": (ctypes.c_int, [fmtp, vp, vp, vp, ctypes.c_int, ctypes.c_int, vp, vp, i64, vp]),
        "seedlm_gemm_workspace_bytes": (i64, [fmtp, ctypes.c_int]),
        "seedlm_gemm_smallM_noalloc": (ctypes.c_int, [fmtp, vp, vp, vp, ctypes.c_int,
                                                      ctypes.c_int, vp, vp]),
        "seedlm_device_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int)]),
        "seedlm_encode": (ctypes.c_int, [fmtp, vp, i64, vp, vp, vp, vp]),
        "seedlm_selftest_wait_timeout": (ctypes.c_int, [i64, vp]),
        "seedlm_dense_gemv_f16": (ctypes.c_int, [i32, i32, vp, i64, vp, vp, vp]),
        "seedlm_row_bytes_ideal": (i64, [fmtp]),
        "seedlm_row_bytes_stored": (i64, [fmtp]),
        "seedlm_strerror": (ctypes.c_char_p, [ctypes.c_int]),
        "seedlm_last_cuda_error": (ctypes.c_int, []),
        "seedlm_launch_count": (i64, []),
        "seedlm_shutdown": (None, []),
        "seedlm_checked_build": (ctypes.c_int, []),
        "seedlm_selftest_bounds_check": (ctypes.c_int, [i64, i64, vp]),
        "seedlm_search_blocks": (ctypes.c_int, [i32, i32, i32, vp, i64, vp, vp, vp, vp, vp]),
        "seedlm_lfsr_taps": (ctypes.c_uint32, [i32]),
        "seedlm_gemv_batch": (ctypes.c_int, [i32, vp, vp, vp, vp, ctypes.c_int, vp, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def strerror(code: int) -> str:
    return lib.seedlm_strerror(code).decode()


def last_cuda_error() -> int:
    return int(lib.seedlm_last_cuda_error())


def launch_count() -> int:
    return int(lib.seedlm_launch_count())


def _check(fn: str, rc: int):
    if rc != 0:
        detail = strerror(rc)
        if rc == -3:
            detail += f" (cudaError {last_cuda_error()})"
        raise SeedLMError(fn, rc, detail)


def _ptr(t) -> int | None:
    """Device (or host) address of a tensor, an int address, or None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream, like=None):
    if stream is None:
        import torch
        dev = like.device if (like is not None and hasattr(like, "device")) else None
        return torch.cuda.current_stream(dev).cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _act_dtype(t) -> int:
    import torch
    if t.dtype == torch.float16:
        return F16
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"activations must be float16 or bfloat16, got {t.dtype}")


def _fmt(fmt) -> Format:
    return fmt if isinstance(fmt, Format) else Format.from_dict(fmt)


def _row_major_ld(t, cols: int) -> int:
    """Leading dimension of a row-major matrix argument (unit column stride)."""
    if t.dim() != 2 or (t.shape[1] > 1 and t.stride(1) != 1):
        raise ValueError("expected a 2-D row-major tensor with unit column stride")
    return int(t.stride(0)) if t.shape[0] > 1 else max(int(t.stride(0)), cols)


def _dense(t, name: str):
    """Arguments the library reads or writes as one dense array."""
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def init():
    _check("seedlm_init", lib.seedlm_init())


def decompress(fmt, rec, eplane, W, ldw: int | None = None, stream=None):
    """W[:rows, :cols] = the rebuilt weights (fp32)."""
    f = _fmt(fmt)
    ld = ldw if ldw is not None else _row_major_ld(W, f.cols)
    _check("seedlm_decompress", lib.seedlm_decompress(
        ctypes.byref(f), _ptr(rec), _ptr(eplane), _ptr(W), ld, _stream(stream, W)))


def encode(fmt, W, rec, eplane=None, err=None, ldw: int | None = None, stream=None):
    """Search seeds, coefficients and exponents for every block of W (fp32,
    rows x cols, device) and write them into rec (int32/uint32, rows x
    rec_pitch) and, for C = 12, eplane (uint8, rows x e_pitch).  err, if
    given, is a float64 (rows x nb) tensor that receives each block's squared
    reconstruction error."""
    f = _fmt(fmt)
    ld = ldw if ldw is not None else _row_major_ld(W, f.cols)
    _check("seedlm_encode", lib.seedlm_encode(
        ctypes.byref(f), _ptr(W), ld, _ptr(rec), _ptr(eplane), _ptr(err), _stream(stream, W)))


def search_blocks(C: int, P: int, K: int, W, seed, q, e, err=None, stream=None):
    """Design-space search over the 2^K - 1 seeds of a K-bit register for
    every row of W (float32, nblocks x C, device): seed (int32/uint32,
    nblocks), q (int8, nblocks x P), e (uint8, nblocks) and optionally err
    (float64, nblocks) receive the best fit of each block."""
    _dense(W, "W")
    n = int(W.shape[0]) if W.dim() == 2 else int(W.numel()) // int(C)
    _check("seedlm_search_blocks", lib.seedlm_search_blocks(
        int(C), int(P), int(K), _ptr(W), n, _ptr(seed), _ptr(q), _ptr(e), _ptr(err),
        _stream(stream, W)))


def lfsr_taps(K: int) -> int:
    """Tap mask of the K-bit register the design-space search uses (0 if K is
    unsupported)."""
    return int(lib.seedlm_lfsr_taps(int(K)))


def gemv(fmt, rec, eplane, x, y, stream=None):
    """y = W x; x float16/bfloat16 (cols), y float32 (rows)."""
    f = _fmt(fmt)
    _dense(x, "x"), _dense(y, "y")
    _check("seedlm_gemv", lib.seedlm_gemv(
        ctypes.byref(f), _ptr(rec), _ptr(eplane), _ptr(x), _act_dtype(x), _ptr(y),
        _stream(stream, y)))


def gemv_batch(items, stream=None):
    """Several independent GEMVs in one launch: items is a list of
    (fmt, rec, eplane, x, y) tuples, all of one storage format and one
    activation type."""
    n = len(items)
    if n == 0:
        return
    fmts = (Format * n)(*[_fmt(it[0]) for it in items])
    ptrs = lambda vals: (ctypes.c_void_p * n)(*vals)  # noqa: E731
    for it in items:
        _dense(it[3], "x"), _dense(it[4], "y")
    recs = ptrs([_ptr(it[1]) for it in items])
    eps = ptrs([_ptr(it[2]) for it in items])
    xs = ptrs([_ptr(it[3]) for it in items])
    ys = ptrs([_ptr(it[4]) for it in items])
    _check("seedlm_gemv_batch", lib.seedlm_gemv_batch(
        n, fmts, recs, eps, xs, _act_dtype(items[0][3]), ys, _stream(stream, items[0][4])))


def gemm_workspace_bytes(fmt, M: int) -> int:
    n = int(lib.seedlm_gemm_smallM_workspace_bytes(ctypes.byref(_fmt(fmt)), int(M)))
    if n < 0:
        _check("seedlm_gemm_smallM_workspace_bytes", n)
    return n


def gemm_workspace(fmt, M: int, device=None):
    """A zero-filled device workspace for seedlm_gemm_smallM (torch uint8 tensor).

    It can be reused by every later call with the same or a smaller need;
    calls that share it must not run concurrently."""
    import torch
    n = gemm_workspace_bytes(fmt, M)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def gemm_smallM(fmt, rec, eplane, X, Y, workspace=None, stream=None):
    """Y = X W^T; X float16/bfloat16 (M, cols), Y float32 (M, rows).

    `workspace` comes from gemm_workspace(); if omitted a fresh one is made."""
    f = _fmt(fmt)
    _dense(X, "X"), _dense(Y, "Y")
    M = int(X.shape[0])
    if workspace is None:
        workspace = gemm_workspace(f, M, device=Y.device)
    nbytes = workspace.numel() * workspace.element_size()
    _check("seedlm_gemm_smallM", lib.seedlm_gemm_smallM(
        ctypes.byref(f), _ptr(rec), _ptr(eplane), _ptr(X), _act_dtype(X), M, _ptr(Y),
        _ptr(workspace), nbytes, _stream(stream, Y)))


def gemm_any_workspace_bytes(fmt, M: int) -> int:
    n = int(lib.seedlm_gemm_workspace_bytes(ctypes.byref(_fmt(fmt)), int(M)))
    if n < 0:
        _check("seedlm_gemm_workspace_bytes", n)
    return n


def gemm(fmt, rec, eplane, X, Y, workspace=None, stream=None):
    """Y = X W^T for any number of rows M of X (seedlm_gemm: passes of at most
    256 rows on the tensor cores; M = 1 runs the GEMV).  `workspace`: a
    zero-filled uint8 tensor of at least gemm_any_workspace_bytes(fmt, M)
    bytes; if omitted a fresh one is made."""
    import torch
    f = _fmt(fmt)
    _dense(X, "X"), _dense(Y, "Y")
    M = int(X.shape[0])
    if workspace is None:
        workspace = torch.zeros(max(gemm_any_workspace_bytes(f, M), 256), dtype=torch.uint8,
                                device=Y.device)
    nbytes = workspace.numel() * workspace.element_size()
    _check("seedlm_gemm", lib.seedlm_gemm(
        ctypes.byref(f), _ptr(rec), _ptr(eplane), _ptr(X), _act_dtype(X), M, _ptr(Y),
        _ptr(workspace), nbytes, _stream(stream, Y)))


def gemm_smallM_noalloc(fmt, rec, eplane, X, Y, stream=None):
    """Y = X W^T without a workspace: the workspace (counters, X slabs, partial
    tiles; 16 MiB + 64 KiB) is an array inside the library; calls sharing it
    must not overlap."""
    f = _fmt(fmt)
    _dense(X, "X"), _dense(Y, "Y")
    _check("seedlm_gemm_smallM_noalloc", lib.seedlm_gemm_smallM_noalloc(
        ctypes.byref(f), _ptr(rec), _ptr(eplane), _ptr(X), _act_dtype(X), int(X.shape[0]),
        _ptr(Y), _stream(stream, Y)))


def device_error() -> int:
    """Reads and clears the device error flags: bit 0 if a kernel gave up on
    one of its own bounded waits, bit 1 if a kernel of the checked build
    skipped an out-of-bounds access.  Synchronous."""
    flag = ctypes.c_int(0)
    _check("seedlm_device_error", lib.seedlm_device_error(ctypes.byref(flag)))
    return int(flag.value)


def checked_build() -> bool:
    """True if the loaded library is the bounds-checked build."""
    return bool(lib.seedlm_checked_build())


def selftest_bounds_check(index: int, extent: int, stream=None):
    """Evaluate one bounds check on the device (no memory access): in the
    checked build index >= extent raises bit 1 of device_error()."""
    _check("seedlm_selftest_bounds_check",
           lib.seedlm_selftest_bounds_check(int(index), int(extent), _stream(stream)))


def selftest_wait_timeout(limit_ns: int = 2_000_000, stream=None):
    """Launch the failure-path self test: a bounded wait that gives up after
    limit_ns, raising the flag device_error() reads."""
    _check("seedlm_selftest_wait_timeout",
           lib.seedlm_selftest_wait_timeout(int(limit_ns), _stream(stream)))


def dense_gemv_f16(W, x, y, stream=None):
    """y = W x with dense fp16 W (rows, cols) -- the reference point."""
    _dense(x, "x"), _dense(y, "y")
    _check("seedlm_dense_gemv_f16", lib.seedlm_dense_gemv_f16(
        int(W.shape[0]), int(W.shape[1]), _ptr(W), _row_major_ld(W, int(W.shape[1])), _ptr(x), _ptr(y),
        _stream(stream, y)))


def row_bytes(fmt) -> tuple[int, int]:
    """(ideal, stored) compressed bytes per row."""
    f = _fmt(fmt)
    return int(lib.seedlm_row_bytes_ideal(ctypes.byref(f))), \
        int(lib.seedlm_row_bytes_stored(ctypes.byref(f)))
