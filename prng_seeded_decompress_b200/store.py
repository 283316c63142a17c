"""Save and load compressed layers: the record planes as raw little-endian
binary files next to a JSON description.

A layer ``<prefix>`` is stored as

* ``<prefix>.rec.bin``    -- rows x rec_pitch uint32 records, row-major;
* ``<prefix>.eplane.bin`` -- rows x e_pitch exponent bytes (the 3-bit format
  only: P = 4 keeps e in a nibble plane);
* ``<prefix>.json``       -- ``{"version": 1, "format": {C, P, K, rows, cols,
  nb, rec_pitch, e_pitch}, "planes": {name: {"file", "dtype", "shape",
  "sha256"}}}``.

The record layout is the one ``include/seedlm.h`` describes for
``seedlm_format``; nothing is converted, so a loaded plane can be copied to
the device and passed to the kernels as it is.  Loading checks the format's
fields against each other, every plane's size against the format, and every
plane's SHA-256 against the description, and raises ``ValueError`` on any
mismatch.  This is host-side plumbing (no counterpart in the pages): the
encoder is an offline step, and its output is saved once and loaded at model
load time.
"""
from __future__ import annotations

import hashlib
import json
import os

import numpy as np

VERSION = 1
_FIELDS = ("C", "P", "K", "rows", "cols", "nb", "rec_pitch", "e_pitch")
_FORMATS = {(8, 3, 16), (12, 4, 16)}


def check_format(fmt: dict) -> dict:
    """The format's fields as ints, or ValueError if they are inconsistent
    (the same rules the library applies to ``seedlm_format``)."""
    try:
        f = {k: int(fmt[k]) for k in _FIELDS}
    except (KeyError, TypeError, ValueError) as exc:
        raise ValueError(f"bad format description: {exc}") from None
    if (f["C"], f["P"], f["K"]) not in _FORMATS:
        raise ValueError(f"unsupported (C, P, K) = {(f['C'], f['P'], f['K'])}")
    if f["rows"] < 0 or f["cols"] < 0:
        raise ValueError("negative shape")
    if f["nb"] != (f["cols"] + f["C"] - 1) // f["C"]:
        raise ValueError("nb is not ceil(cols / C)")
    if f["rec_pitch"] < f["nb"] or f["rec_pitch"] % 4:
        raise ValueError("rec_pitch must be >= nb and a multiple of 4")
    if f["P"] == 4 and f["e_pitch"] < (f["nb"] + 1) // 2:
        raise ValueError("e_pitch must be >= ceil(nb / 2)")
    return f


def _plane(a, dtype, shape, name) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype.itemsize != np.dtype(dtype).itemsize or a.dtype.kind not in "iu":
        raise ValueError(f"{name}: expected {np.dtype(dtype).name} data, got {a.dtype}")
    a = a.view(dtype)
    if a.size != shape[0] * shape[1]:
        raise ValueError(f"{name}: {a.size} elements, the format needs {shape[0]} x {shape[1]}")
    return a.reshape(shape)


def _sha256(b: bytes) -> str:
    return hashlib.sha256(b).hexdigest()


def save_layer(prefix: str, fmt: dict, rec, eplane=None) -> dict:
    """Write the layer; returns the JSON description.  ``rec`` (and for the
    3-bit format ``eplane``; for the 4-bit format None or an empty array) are
    host arrays in the library's layout."""
    f = check_format(fmt)
    planes = {"rec": (_plane(rec, np.uint32, (f["rows"], f["rec_pitch"]), "rec"), "<u4")}
    if f["P"] == 4:
        if eplane is None:
            raise ValueError("the 3-bit format needs its exponent plane")
        planes["eplane"] = (_plane(eplane, np.uint8, (f["rows"], f["e_pitch"]), "eplane"), "u1")
    elif eplane is not None and np.asarray(eplane).size:
        raise ValueError("the 4-bit format has no exponent plane")
    desc = {"version": VERSION, "format": f, "planes": {}}
    base = os.path.basename(prefix)
    for name, (arr, dt) in planes.items():
        data = arr.astype(dt, copy=False).tobytes()
        fname = f"{base}.{name}.bin"
        with open(f"{prefix}.{name}.bin", "wb") as fh:
            fh.write(data)
        desc["planes"][name] = {"file": fname, "dtype": dt, "shape": list(arr.shape),
                                "sha256": _sha256(data)}
    with open(f"{prefix}.json", "w") as fh:
        json.dump(desc, fh, indent=1)
    return desc


def load_layer(prefix: str):
    """(fmt, rec, eplane) of a saved layer; eplane is None for the 4-bit
    format.  Raises ValueError if anything does not match its description."""
    with open(f"{prefix}.json") as fh:
        desc = json.load(fh)
    if desc.get("version") != VERSION:
        raise ValueError(f"unsupported version {desc.get('version')!r}")
    f = check_format(desc.get("format", {}))
    want = {"rec": ("<u4", [f["rows"], f["rec_pitch"]])}
    if f["P"] == 4:
        want["eplane"] = ("u1", [f["rows"], f["e_pitch"]])
    planes = desc.get("planes", {})
    if set(planes) != set(want):
        raise ValueError(f"planes {sorted(planes)} do not match the format ({sorted(want)})")
    out = {}
    folder = os.path.dirname(os.path.abspath(f"{prefix}.json"))
    for name, (dt, shape) in want.items():
        p = planes[name]
        if p.get("dtype") != dt or list(p.get("shape", [])) != shape:
            raise ValueError(f"{name}: description says {p.get('dtype')} {p.get('shape')}, "
                             f"the format needs {dt} {shape}")
        if os.path.basename(p.get("file", "")) != p.get("file"):
            raise ValueError(f"{name}: the plane file must sit next to the description")
        with open(os.path.join(folder, p["file"]), "rb") as fh:
            data = fh.read()
        if len(data) != np.dtype(dt).itemsize * shape[0] * shape[1]:
            raise ValueError(f"{name}: {len(data)} bytes on disk, the format needs "
                             f"{np.dtype(dt).itemsize * shape[0] * shape[1]}")
        if _sha256(data) != p.get("sha256"):
            raise ValueError(f"{name}: SHA-256 does not match the description")
        # Little-endian on disk, native in memory.
        out[name] = np.frombuffer(data, dtype=dt).astype(np.dtype(dt).newbyteorder("="),
                                                         copy=True).reshape(shape)
    return f, out["rec"], out.get("eplane")
