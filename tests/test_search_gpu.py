"""The design-space search (seedlm_search_blocks) against the oracle's
brute-force search, for block sizes, latent dimensions and seed widths other
than the two storage formats.

Planted blocks (built exactly from a seed, coefficients and an exponent) must
come back with error 0 and the canonical triple (ties: smallest seed, then
largest exponent) that the oracle finds.  Gaussian blocks must reach the
oracle's minimum error within 1e-9 relative, and the triple the GPU returns
must rebuild, through the oracle's basis, to the error it reports.
"""
import numpy as np
import pytest

import oracle
from oracle.search import seed_search_k
from prng_seeded_decompress_b200 import build

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sl():
    build.build()
    from prng_seeded_decompress_b200 import seedlm
    return seedlm


def test_library_taps_match_the_oracle(sl):
    # Both sides find the taps independently (the library in C++, the oracle
    # in C driven from Python); a host call, no GPU needed.
    for K in range(8, 21):
        assert sl.lfsr_taps(K) == oracle.primitive_taps(K), K
    assert sl.lfsr_taps(7) == 0 and sl.lfsr_taps(21) == 0


def _blocks(C, P, K, taps, n_planted, n_gauss, seed):
    rng = np.random.default_rng(seed)
    W = []
    while len(W) < n_planted:
        # The block must be exact in fp32 (the search's input type).
        s = int(rng.integers(1, 1 << K))
        q = rng.integers(-8, 8, size=P)
        q[0] = -7
        e = int(rng.integers(6, 13))
        w = oracle.block_basis_k(s, C, P, K, taps) @ q * 2.0 ** (-e)
        if np.array_equal(w.astype(np.float32).astype(np.float64), w):
            W.append(w)
    for _ in range(n_gauss):
        W.append(rng.standard_normal(C) * 0.02)
    return np.array(W, dtype=np.float32).astype(np.float64)


@pytest.mark.gpu
@pytest.mark.parametrize("C,P,K,n_gauss", [
    (8, 3, 16, 3), (8, 4, 16, 3), (12, 3, 16, 3), (12, 4, 16, 3), (16, 4, 16, 2),
    (16, 2, 16, 2), (8, 3, 12, 4), (8, 2, 10, 4), (8, 3, 20, 1),
])
def test_search_matches_oracle(sl, C, P, K, n_gauss):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    taps = oracle.primitive_taps(K)
    W = _blocks(C, P, K, taps, 2, n_gauss, C * 1000 + P * 100 + K)
    n = W.shape[0]
    Wd = torch.from_numpy(W.astype(np.float32)).cuda()
    seed = torch.zeros(n, dtype=torch.int32, device="cuda")
    q = torch.zeros((n, P), dtype=torch.int8, device="cuda")
    e = torch.zeros(n, dtype=torch.uint8, device="cuda")
    err = torch.zeros(n, dtype=torch.float64, device="cuda")
    sl.search_blocks(C, P, K, Wd, seed, q, e, err)
    torch.cuda.synchronize()
    assert sl.device_error() == 0
    seed, q, e, err = (seed.cpu().numpy().view(np.uint32), q.cpu().numpy(), e.cpu().numpy(),
                       err.cpu().numpy())
    for b in range(n):
        w = W[b]
        s_o, q_o, e_o, err_o, _ = seed_search_k(w, C, P, K, taps)
        U = oracle.block_basis_k(int(seed[b]), C, P, K, taps)
        got = U @ q[b].astype(np.float64) * 2.0 ** (-int(e[b]))
        direct = float(((w - got) ** 2).sum())
        scale = float((w ** 2).sum())
        assert abs(direct - err[b]) <= 1e-12 * scale, (b, direct, err[b])
        if b < 2:  # planted: exact fit, canonical triple
            assert err[b] == 0.0 and err_o == 0.0
            assert (int(seed[b]), int(e[b])) == (s_o, e_o), (b, seed[b], e[b], s_o, e_o)
            assert np.array_equal(q[b].astype(np.int64), q_o)
        else:
            assert abs(err[b] - err_o) <= 1e-9 * scale, (b, err[b], err_o)


@pytest.mark.gpu
def test_search_rejects_unsupported_shapes(sl):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    W = torch.zeros((4, 8), device="cuda")
    seed = torch.zeros(4, dtype=torch.int32, device="cuda")
    q = torch.zeros((4, 4), dtype=torch.int8, device="cuda")
    e = torch.zeros(4, dtype=torch.uint8, device="cuda")
    for C, P, K in ((8, 1, 16), (8, 5, 16), (9, 3, 16), (8, 3, 7), (8, 3, 21)):
        with pytest.raises(sl.SeedLMError) as exc:
            sl.search_blocks(C, P, K, W, seed, q, e)
        assert exc.value.code == -2
