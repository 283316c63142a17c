"""Brute-force seed and coefficient search for one block -- TEST INFRASTRUCTURE.

The encoder side of SeedLM (paperhub.cn review thread, authors' replies on the
cost of parameter optimisation): for every block, search the seeds for the one
whose pseudo-random matrix, combined with quantised coefficients, minimises the
reconstruction error; the pseudo-inverses of all seeds' matrices are computed
once and cached, and the search runs over seeds and blocks in parallel.

The pages give no exponent rule and no rounding rule.  The reading used here:
for each seed s, t* = pinv(U(s)) w; for each exponent e in 0..15,
q = clamp(round-half-even(t* 2^e), -8, 7) and the error is
||w - U(s) q 2^-e||^2.  The minimum wins; ties go to the smallest seed, then to
the largest exponent.  ``np.linalg.pinv`` and ``np.rint`` are the library
primitives; U(s) comes from the C oracle.
"""
from __future__ import annotations

import functools

import numpy as np

from . import basis_all, basis_all_k


@functools.lru_cache(maxsize=4)
def _tables(C: int, P: int):
    U = basis_all(C, P)                 # (65535, C, P)
    Upinv = np.linalg.pinv(U)           # (65535, P, C)
    return U, Upinv


@functools.lru_cache(maxsize=4)
def _tables_k(C: int, P: int, K: int, taps: int):
    U = basis_all_k(C, P, K, taps)      # (2^K - 1, C, P)
    Upinv = np.linalg.pinv(U)           # (2^K - 1, P, C)
    return U, Upinv


def seed_search(w, C: int, P: int):
    """Best (seed, q, e, err, w_hat) for the length-C block ``w``."""
    return _search(w, C, *_tables(C, P))


def seed_search_k(w, C: int, P: int, K: int, taps: int):
    """The same search over the 2^K - 1 seeds of a K-bit register with the
    given taps (design-space variants: other block sizes C, latent
    dimensions P and seed widths K)."""
    return _search(w, C, *_tables_k(C, P, K, taps))


def _search(w, C: int, U, Upinv):
    w = np.asarray(w, dtype=np.float64)
    assert w.shape == (C,)
    tstar = Upinv @ w                   # (65535, P)
    best = None
    for e in range(15, -1, -1):         # descending so that ties keep the largest e
        q = np.clip(np.rint(tstar * 2.0 ** e), -8, 7)
        what = np.einsum("scp,sp->sc", U, q) * 2.0 ** (-e)
        err = ((w[None, :] - what) ** 2).sum(axis=1)
        s = int(np.argmin(err))         # first minimum = smallest seed
        cand = (float(err[s]), s + 1, e, q[s].astype(np.int64), what[s])
        if best is None or (cand[0], cand[1]) < (best[0], best[1]):
            best = cand
    err, seed, e, q, what = best
    return seed, q, e, err, what
