"""Seeded synthetic inputs for the SeedLM hot path.

This module serves both the CUDA path (tests, bench) and the CPU oracle; it
holds none of the method's arithmetic -- no LFSR, no reconstruction, no
product.  It only draws the stored fields and the activations with NumPy's
PCG64 generator and packs the fields into the record layout that both sides
read:

* one uint32 record per block of C weights, blocks of a row in column order,
  row r at ``rec[r * rec_pitch]`` (``rec_pitch`` a multiple of 4, so every row
  starts on a 16-byte boundary);
* bits [16, 32): the 16-bit seed;
* bits [4p, 4p + 4): coefficient q_p, 4-bit two's complement, for p < P;
* P == 3: the exponent e in bits [12, 16);
* P == 4: e in a nibble plane, row r at ``eplane[r * e_pitch]`` (``e_pitch`` a
  multiple of 16), block b in byte b // 2, low nibble for even b.

Distributions (the workload specification): seed uniform on [1, 65535], q
uniform on [-8, 7], e uniform on [8, 12]; activations N(0, 1) rounded to fp16
or bf16.  Records past ``nb`` in a row (the pitch padding) are filled with
random words, so a kernel that reads them instead of ignoring them fails its
parity test.
"""
from __future__ import annotations

import numpy as np

#: (C, P) of the two storage formats: 4 bits/weight and 3 bits/weight.
FORMAT_4BIT = (8, 3)
FORMAT_3BIT = (12, 4)


def _round_up(v: int, m: int) -> int:
    return (v + m - 1) // m * m


def make_format(rows: int, cols: int, C: int, P: int) -> dict:
    nb = (cols + C - 1) // C
    rec_pitch = _round_up(max(nb, 1), 4)
    e_pitch = _round_up(max((nb + 1) // 2, 1), 16) if P == 4 else 0
    return dict(C=C, P=P, K=16, rows=rows, cols=cols, nb=nb,
                rec_pitch=rec_pitch, e_pitch=e_pitch)


def draw_fields(rng: np.random.Generator, rows: int, nb: int, P: int,
                e_range=(8, 12)):
    """seeds (rows, nb) uint16, q (rows, nb, P) int8, e (rows, nb) uint8."""
    seeds = rng.integers(1, 65535, size=(rows, nb), dtype=np.uint16, endpoint=True)
    q = rng.integers(-8, 7, size=(rows, nb, P), dtype=np.int8, endpoint=True)
    e = rng.integers(e_range[0], e_range[1], size=(rows, nb), dtype=np.uint8, endpoint=True)
    return seeds, q, e


def pack_records(fmt: dict, seeds, q, e, rng: np.random.Generator | None = None):
    """Pack the fields into (rec, eplane) in the layout described above."""
    rows, nb, P = fmt["rows"], fmt["nb"], fmt["P"]
    seeds = np.asarray(seeds, dtype=np.uint32).reshape(rows, nb)
    q = np.asarray(q).reshape(rows, nb, P)
    e = np.asarray(e, dtype=np.uint32).reshape(rows, nb)
    if np.any((q < -8) | (q > 7)) or np.any(e > 15):
        raise ValueError("fields out of range")
    word = seeds << np.uint32(16)
    for p in range(P):
        word |= (q[:, :, p].astype(np.int32).astype(np.uint32) & np.uint32(15)) << \
            np.uint32(4 * p)
    rec = np.zeros((rows, fmt["rec_pitch"]), np.uint32)
    if rng is not None and fmt["rec_pitch"] > nb:
        rec[:, nb:] = rng.integers(0, 2 ** 32, size=(rows, fmt["rec_pitch"] - nb),
                                   dtype=np.uint64).astype(np.uint32)
    eplane = np.zeros((rows, max(fmt["e_pitch"], 0)), np.uint8)
    if P <= 3:
        word |= (e & np.uint32(15)) << np.uint32(4 * P)
    else:
        if rng is not None:
            eplane[:] = rng.integers(0, 256, size=eplane.shape, dtype=np.int64)
        half = (nb + 1) // 2
        ep = np.zeros((rows, half), np.uint32)
        ep[:, :half] |= e[:, 0::2]
        ep[:, : nb // 2] |= e[:, 1::2] << np.uint32(4)
        if nb % 2 == 1:  # keep the unused high nibble of the last byte random
            ep[:, half - 1] |= eplane[:, half - 1].astype(np.uint32) & np.uint32(0xF0)
        eplane[:, :half] = ep.astype(np.uint8)
    rec[:, :nb] = word
    return rec, eplane


def make_layer(rows: int, cols: int, C: int, P: int, seed: int, e_range=(8, 12)) -> dict:
    """A synthetic compressed weight matrix: format, packed planes and fields."""
    rng = np.random.Generator(np.random.PCG64(seed))
    fmt = make_format(rows, cols, C, P)
    seeds, q, e = draw_fields(rng, rows, fmt["nb"], P, e_range)
    rec, eplane = pack_records(fmt, seeds, q, e, rng)
    return dict(fmt=fmt, rec=rec, eplane=eplane, seeds=seeds, q=q, e=e)


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f64(b) -> np.ndarray:
    u = (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16))
    return u.view(np.float32).astype(np.float64)


def make_activations(shape, dtype: str, seed: int):
    """(bits, values): N(0,1) activations rounded to 'f16' or 'bf16'.

    ``bits`` is a uint16 array holding the storage bits, ``values`` the same
    numbers widened exactly to float64.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    v = rng.standard_normal(size=shape).astype(np.float32)
    if dtype == "f16":
        h = v.astype(np.float16)
        return h.view(np.uint16).copy(), h.astype(np.float64)
    if dtype == "bf16":
        bits = f32_to_bf16_bits(v)
        return bits, bf16_bits_to_f64(bits)
    raise ValueError(f"unknown activation dtype {dtype!r}")
