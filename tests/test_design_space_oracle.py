"""Pins for the oracle's design-space variants (other seed widths K, block
sizes C and latent dimensions P), all on the CPU.

The pages discuss these parameters (paperhub.cn review thread, authors'
replies on compression time against seed bit-width, block size and latent
dimension) but give no LFSR polynomial for any K.  The reading: a K-bit
register shifting right with the parity of its tapped bits fed in at the top,
taps 0x2D for K = 16 (the workload's register) and otherwise the smallest odd
tap mask whose register visits all 2^K - 1 nonzero states.  What pins it:
the register's period by brute force, its agreement with the 16-bit register
for K = 16, a basis worked by hand from a hand-stepped register, and
planted-seed recovery through the generalised brute-force search.
"""
import numpy as np
import pytest

import oracle
from oracle.search import seed_search_k

KS = (8, 10, 12, 14, 16, 18, 20)


def _step(s, K, taps):
    # Written out bit by bit, independently of the oracle's C code.
    bit = 0
    for i in range(K):
        if (taps >> i) & 1:
            bit ^= (s >> i) & 1
    return (s >> 1) | (bit << (K - 1))


@pytest.mark.parametrize("K", KS)
def test_taps_give_a_maximal_register(K):
    taps = oracle.primitive_taps(K)
    assert taps & 1, "a register without tap 0 is not invertible"
    assert oracle.lfsr_period_k(K, taps) == (1 << K) - 1


@pytest.mark.parametrize("K", (8, 10, 12))
def test_register_visits_every_nonzero_state(K):
    # Enumerate the states directly (no period routine): all 2^K - 1 nonzero
    # states appear once before the register returns to its start, and 0 is
    # the fixed point.
    taps = oracle.primitive_taps(K)
    seen = set()
    s = 1
    for _ in range((1 << K) - 1):
        assert s not in seen and s != 0
        seen.add(s)
        s = _step(s, K, taps)
    assert s == 1 and len(seen) == (1 << K) - 1
    assert _step(0, K, taps) == 0
    # No smaller odd mask is maximal: each returns to 1 early (or never).
    for t in range(1, taps, 2):
        assert oracle.lfsr_period_k(K, t) != (1 << K) - 1


def test_k16_register_is_the_workload_register():
    for s in range(1 << 16):
        assert oracle.lfsr_next_k(s, 16, 0x2D) == oracle.lfsr_next(s)


def test_basis_k_by_hand():
    # K = 8 register with the oracle's taps, seed 0x5A, C = 3, P = 2:
    # U[c][p] = (state_{3p + c} - 128) / 128 from a hand-stepped register.
    K, taps = 8, oracle.primitive_taps(8)
    st = [0x5A]
    for _ in range(5):
        st.append(_step(st[-1], K, taps))
    U = oracle.block_basis_k(0x5A, 3, 2, K, taps)
    want = np.array([[(st[p * 3 + c] - 128) / 128 for p in range(2)] for c in range(3)])
    assert np.array_equal(U, want)
    # And the 16-bit case agrees with the workload basis for any C, P.
    assert np.array_equal(oracle.block_basis_k(12345, 12, 4, 16, 0x2D),
                          oracle.block_basis(12345, 12, 4))


@pytest.mark.parametrize("C,P,K", [(8, 3, 12), (12, 3, 10), (16, 2, 10)])
def test_planted_seed_recovery_k(C, P, K):
    # A block built from (seed, q, e) is recovered exactly (error 0): the
    # search compares every seed of the K-bit register.
    taps = oracle.primitive_taps(K)
    rng = np.random.default_rng(C * 100 + P * 10 + K)
    for _ in range(2):
        seed = int(rng.integers(1, 1 << K))
        q = rng.integers(-8, 8, size=P)
        q[0] = 5  # not all zero
        e = int(rng.integers(4, 12))
        w = oracle.block_basis_k(seed, C, P, K, taps) @ q * 2.0 ** (-e)
        s2, q2, e2, err, what = seed_search_k(w, C, P, K, taps)
        assert err == 0.0
        assert np.array_equal(what, w)
        assert np.array_equal(oracle.block_basis_k(s2, C, P, K, taps) @ q2 * 2.0 ** (-e2), w)
