"""The column-table form of a block's dot product with x, checked in fp64
against the oracle's reconstruction.  No GPU.

A block's weights are w = U(seed) q 2^-e with U[c][p] = (state_{pC+c} -
32768) / 32768, so its dot with x is linear in the LFSR's stream bits.  With
b_n = bit 0 of state n, state k holds the stream bits k .. k+15, and

  x . w = 2^-e (sum_p q_p S_p - (sum_p q_p) sum_c x_c),
  S_p = 2^-15 sum_c x_c state_{pC+c} = sum_m b_{pC+m} X~_m,
  X~_m = sum_c x_c 2^(m-c-15)  (0 <= m - c <= 15).

Cut into bytes, S_p is a sum of lookups T_j[byte at bit pC + 8j] with
T_j[v] = sum_k bit_k(v) X~_{8j+k}: the tables depend on x only.  The 3-bit
column-table GEMV computes exactly this (four byte tables, X~ built by the
recursion X~_m = 2 X~_{m-1} + 2^-15 x_m - 2 x_{m-16}); at 4 bits three
tables serve (the form measured and not built).  The test checks the
identity, the recursion and the byte cut against U(seed) from the oracle,
over random blocks and a few with extreme activations."""
import numpy as np
import pytest

import oracle

BITS8 = ((np.arange(256)[:, None] >> np.arange(8)[None, :]) & 1).astype(np.float64)


def x_tilde(x, C, n):
    """X~_m for m < n from its definition (fp64)."""
    return np.array([sum(x[c] * 2.0 ** (m - c - 15) for c in range(C) if 0 <= m - c <= 15)
                     for m in range(n)])


def x_tilde_recursive(x, C, n):
    """The same values by the kernel's recursion."""
    out = np.zeros(n)
    for m in range(n):
        v = 2.0 * out[m - 1] if m else 0.0
        if m < C:
            v += x[m] * 2.0 ** -15
        if 0 <= m - 16 < C:
            v -= 2.0 * x[m - 16]
        out[m] = v
    return out


def table_dot(seed, q, e, x, C, P):
    """x . w through the byte tables of x (fp64)."""
    span = C + 15                       # bits behind one S_p
    ntab = (span + 7) // 8
    Xt = np.zeros(8 * ntab)
    Xt[:span] = x_tilde(x, C, span)
    T = np.stack([BITS8 @ Xt[8 * j: 8 * j + 8] for j in range(ntab)])   # (ntab, 256)
    nbits = C * (P - 1) + 8 * ntab
    b = (oracle.lfsr_states(seed, nbits) & 1).astype(np.int64)
    S = np.zeros(P)
    for p in range(P):
        for j in range(ntab):
            byte = int(sum(int(b[p * C + 8 * j + k]) << k for k in range(8)))
            S[p] += T[j, byte]
    return 2.0 ** -e * (float(np.dot(q, S)) - float(np.sum(q)) * float(np.sum(x)))


def cases(C, P, n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        s = int(rng.integers(1, 65536))
        q = rng.integers(-8, 8, size=P)
        e = int(rng.integers(0, 16))
        x = rng.standard_normal(C) * (10.0 ** rng.choice([-30, 0, 0, 0, 30]))
        out.append((s, q, e, x))
    # Seeds at the ends of the range, all-negative and all-positive q.
    out.append((1, np.full(P, -8), 0, rng.standard_normal(C)))
    out.append((65535, np.full(P, 7), 15, rng.standard_normal(C)))
    return out


@pytest.mark.parametrize("C,P", [(12, 4), (8, 3)])
def test_table_form_equals_the_reconstructed_block(C, P):
    for s, q, e, x in cases(C, P, 150, 1000 + C):
        w = oracle.block_basis(s, C, P) @ (q * 2.0 ** -e)
        direct = float(np.dot(x, w))
        scale = float(np.sum(np.abs(x * w))) + 1e-300
        got = table_dot(s, q, e, x, C, P)
        assert abs(got - direct) <= 1e-12 * scale, (s, list(q), e, got, direct)


@pytest.mark.parametrize("C", [12, 8])
def test_x_tilde_recursion_equals_its_definition(C):
    rng = np.random.default_rng(7 + C)
    for _ in range(50):
        x = rng.standard_normal(C) * 10.0 ** rng.integers(-20, 21)
        n = C + 15
        ref = x_tilde(x, C, n)
        got = x_tilde_recursive(x, C, n)
        assert np.all(np.abs(got - ref) <= 1e-12 * np.sum(np.abs(x)))
        # A table entry (a sum of some X~_m) stays below 2 sum |x|: the
        # range the kernel relies on.
        assert np.sum(np.abs(ref)) <= 2.0 * np.sum(np.abs(x))


def test_a_planted_mistake_in_the_byte_cut_is_caught():
    # Reading each S_p's bytes one bit late must break the identity: the
    # test above would notice an off-by-one in the kernel's stream offsets.
    C, P = 12, 4
    s, q, e, x = cases(C, P, 1, 5)[0]
    w = oracle.block_basis(s, C, P) @ (q * 2.0 ** -e)
    direct = float(np.dot(x, w))
    shifted = table_dot(oracle.lfsr_next(s), q, e, x, C, P)
    assert abs(shifted - direct) > 1e-6 * (float(np.sum(np.abs(x * w))) + 1e-300)
