"""seedlm_encode (the encoder: seed, coefficient and exponent search) against
the oracle's brute-force search, oracle/search.py.

What is unique is the minimum reconstruction error of each block; the seed
that reaches it is unique too unless two candidates tie to the last bit, so
the tests compare the error (within fp64 rounding of two different
summation orders) and check that the GPU's (seed, q, e) decode -- through the
oracle's decoder -- to exactly that error.  Planted blocks (weights that some
(seed, q, e) reproduce exactly) must come back as the oracle's canonical
triple (smallest seed, then largest e, among the exact fits) and decode
bit-exactly.
"""
import os

import numpy as np
import pytest

from prng_seeded_decompress_b200 import inputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

C8, C12 = inputs.FORMAT_4BIT, inputs.FORMAT_3BIT


@pytest.fixture(scope="module")
def sl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from prng_seeded_decompress_b200 import build
    build.build()
    from prng_seeded_decompress_b200 import seedlm
    return seedlm


def gpu_encode(sl, fmt, W):
    rows = fmt["rows"]
    rec = torch.zeros((rows, fmt["rec_pitch"]), dtype=torch.int32, device="cuda")
    ep = None
    if fmt["P"] == 4:
        ep = torch.zeros((rows, fmt["e_pitch"]), dtype=torch.uint8, device="cuda")
    err = torch.full((rows, fmt["nb"]), float("nan"), dtype=torch.float64, device="cuda")
    Wd = torch.from_numpy(np.ascontiguousarray(W, dtype=np.float32)).cuda()
    sl.encode(fmt, Wd, rec, ep, err)
    torch.cuda.synchronize()
    rec_h = rec.cpu().numpy().view(np.uint32)
    ep_h = None if ep is None else ep.cpu().numpy()
    return rec_h, ep_h, err.cpu().numpy()


def padded_block(W, r, b, C):
    w = np.zeros(C)
    seg = W[r, b * C:(b + 1) * C].astype(np.float64)
    w[:len(seg)] = seg
    return w


def check_against_oracle(oracle_mod, fmt, W, rec, ep, err, blocks):
    from oracle.search import seed_search
    C, P = fmt["C"], fmt["P"]
    for r, b in blocks:
        w = padded_block(W, r, b, C)
        s, q, e, e_err, _ = seed_search(w, C, P)
        gs, gq, ge = oracle_mod.block_fields(fmt, rec, ep, r, b)
        what = oracle_mod.reconstruct_block(fmt, rec, ep, r, b)
        g_err = float(((w - what) ** 2).sum())
        scale = float((w ** 2).sum()) + 1e-300
        # The GPU's choice decodes to the error it reports ...
        assert abs(g_err - err[r, b]) <= 1e-12 * scale, (r, b, g_err, err[r, b])
        # ... and that error is the minimum the oracle finds.
        assert abs(g_err - e_err) <= 1e-9 * scale, (r, b, g_err, e_err, (gs, ge), (s, e))
        if gs == s:
            assert ge == e and np.array_equal(np.asarray(gq), np.asarray(q)), (r, b)


@pytest.mark.parametrize("cp", [C8, C12])
def test_planted_blocks_come_back_exactly(sl, oracle_mod, cp):
    # Weights that a planted (seed, q, e) reproduces exactly.  The planted
    # triple is not always the canonical one: (q, e) and (2q, e + 1) rebuild
    # the same block, and when q's last (first) entry is 0 the seed whose bit
    # stream starts C steps earlier (later) rebuilds it too, with q shifted.
    # So the GPU must return the oracle's choice -- smallest seed, then
    # largest e, among the exact fits -- and rebuild every block bit-exactly.
    rows, cols = 3, 5 * cp[0]
    L = inputs.make_layer(rows, cols, *cp, seed=123 + cp[0])
    fmt = L["fmt"]
    W = oracle_mod.decompress(fmt, L["rec"], L["eplane"])       # exact in fp32
    assert np.array_equal(W.astype(np.float32).astype(np.float64), W)
    rec, ep, err = gpu_encode(sl, fmt, W)
    from oracle.search import seed_search
    for r in range(rows):
        for b in range(fmt["nb"]):
            gs, gq, ge = oracle_mod.block_fields(fmt, rec, ep, r, b)
            s, q, e, e_err, _ = seed_search(padded_block(W, r, b, cp[0]), *cp)
            assert e_err == 0.0
            assert (gs, ge) == (s, e) and np.array_equal(np.asarray(gq), np.asarray(q)), \
                (r, b, (gs, gq, ge), (s, q, e))
            assert err[r, b] == 0.0
    assert np.array_equal(oracle_mod.decompress(fmt, rec, ep), W)


def test_shifted_stream_seed_wins_a_tie(sl, oracle_mod):
    # Block 2 of this planted 3-bit layer has q = (3, 2, -1, 0) at e = 8 with
    # seed 62848; seed 3572's stream is seed 62848's started 12 steps earlier,
    # so U(3572)'s columns 1..3 are U(62848)'s columns 0..2 and (0, 6, 4, -2)
    # at e = 9 rebuilds the block exactly.  Smallest seed and largest e win.
    L = inputs.make_layer(3, 60, *C12, seed=135)
    fmt = L["fmt"]
    assert oracle_mod.block_fields(fmt, L["rec"], L["eplane"], 0, 2)[0] == 62848
    W = oracle_mod.decompress(fmt, L["rec"], L["eplane"])
    rec, ep, err = gpu_encode(sl, fmt, W)
    s, q, e = oracle_mod.block_fields(fmt, rec, ep, 0, 2)
    assert (s, e) == (3572, 9) and list(q) == [0, 6, 4, -2]
    assert err[0, 2] == 0.0


@pytest.mark.parametrize("cp,rows,cols", [(C8, 4, 50), (C12, 3, 61)])
def test_gaussian_blocks_reach_the_oracle_minimum(sl, oracle_mod, cp, rows, cols):
    # Gaussian weights as in the pages' synthetic study; cols leaves a tail
    # block (50 = 6*8 + 2, 61 = 5*12 + 1) and, for C = 12, an odd block count.
    rng = np.random.default_rng(7 + cp[0])
    W = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    fmt = inputs.make_format(rows, cols, *cp)
    rec, ep, err = gpu_encode(sl, fmt, W)
    blocks = [(r, b) for r in range(rows) for b in range(fmt["nb"])]
    check_against_oracle(oracle_mod, fmt, W.astype(np.float64), rec, ep, err, blocks)


def test_zero_and_extreme_blocks(sl, oracle_mod):
    # An all-zero block (every candidate ties at 0: seed 1, e = 15, q = 0), a
    # block of one large value, and one of tiny values.
    cols = 24
    W = np.zeros((3, cols), np.float32)
    W[1, 9] = 3.0
    W[2, 16:24] = np.float32(1e-6) * np.arange(1, 9, dtype=np.float32)
    fmt = inputs.make_format(3, cols, *C8)
    rec, ep, err = gpu_encode(sl, fmt, W)
    s, q, e = oracle_mod.block_fields(fmt, rec, ep, 0, 0)
    assert (s, e) == (1, 15) and not np.any(q)
    blocks = [(r, b) for r in range(3) for b in range(fmt["nb"])]
    check_against_oracle(oracle_mod, fmt, W.astype(np.float64), rec, ep, err, blocks)


def test_padding_is_left_untouched(sl):
    # Record slots past nb and exponent bytes past ceil(nb / 2) keep their
    # contents; odd nb gets a zero high nibble in its last exponent byte.
    fmt = inputs.make_format(2, 36, *C12)   # nb = 3
    rec = torch.full((2, fmt["rec_pitch"]), -1, dtype=torch.int32, device="cuda")
    ep = torch.full((2, fmt["e_pitch"]), 0xAB, dtype=torch.uint8, device="cuda")
    W = torch.randn((2, 36), device="cuda") * 0.02
    sl.encode(fmt, W, rec, ep)
    torch.cuda.synchronize()
    r, e = rec.cpu().numpy(), ep.cpu().numpy()
    assert np.all(r[:, 3:] == -1)
    assert np.all(e[:, 2:] == 0xAB)
    assert np.all((e[:, 1] >> 4) == 0)


def test_encode_decode_roundtrip_through_the_gemv(sl, oracle_mod):
    # Encode Gaussian weights, then the GPU GEMV on the records matches the
    # oracle GEMV on the same records (the encoder's output is a valid input).
    rng = np.random.default_rng(3)
    rows, cols = 64, 256
    W = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    fmt = inputs.make_format(rows, cols, *C8)
    rec, ep, err = gpu_encode(sl, fmt, W)
    xb, xv = inputs.make_activations((cols,), "f16", 4)
    y = torch.empty(rows, device="cuda")
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.float16)
    sl.gemv(fmt, torch.from_numpy(rec.view(np.int32)).cuda(), None, x, y)
    torch.cuda.synchronize()
    ref, refabs = oracle_mod.gemv(fmt, rec, ep, xv, threads=os.cpu_count() or 1)
    got = y.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= 1e-5 * refabs + 1e-30)
    # Reconstruction quality: relative error of a 4-bit block fit.
    what = oracle_mod.decompress(fmt, rec, ep)
    rel = np.linalg.norm(what - W) / np.linalg.norm(W)
    assert rel < 0.5, rel


@pytest.mark.parametrize("cp,rows,cols", [(C8, 2400, 8192), (C12, 96, 1000)])
def test_encode_then_gemv_on_one_stream(sl, oracle_mod, cp, rows, cols):
    # The encoder writes the records and the GEMV (programmatic dependent
    # launch) reads them right after it on the same stream, with no host
    # synchronisation in between: the GEMV must wait for the encoder's
    # writes before it reads a record.  Both the large-product kernel (2400
    # rows) and the small one are covered.  The records start as garbage so
    # that an early read would show.
    rng = np.random.default_rng(cols)
    W = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    fmt = inputs.make_format(rows, cols, *cp)
    rec = torch.randint(-2 ** 31, 2 ** 31 - 1, (rows, fmt["rec_pitch"]), dtype=torch.int32,
                        device="cuda")
    ep = None
    if fmt["P"] == 4:
        ep = torch.randint(0, 256, (rows, fmt["e_pitch"]), dtype=torch.uint8, device="cuda")
    xb, xv = inputs.make_activations((cols,), "f16", 5)
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.float16)
    y = torch.full((rows,), float("nan"), device="cuda")
    Wd = torch.from_numpy(W).cuda()
    torch.cuda.synchronize()
    sl.encode(fmt, Wd, rec, ep)
    sl.gemv(fmt, rec, ep, x, y)
    torch.cuda.synchronize()
    assert sl.device_error() == 0
    rec_h = rec.cpu().numpy().view(np.uint32)
    ep_h = None if ep is None else ep.cpu().numpy()
    sample = np.unique(np.concatenate([np.arange(8), np.arange(rows - 8, rows),
                                       rng.integers(0, rows, 48)]))
    ref, refabs = oracle_mod.gemv_rows(fmt, rec_h, ep_h, xv, sample)
    got = y.cpu().numpy().astype(np.float64)[sample]
    assert np.all(np.abs(got - ref) <= 1e-5 * refabs + 1e-30)


@pytest.mark.parametrize("cp,rows,cols", [(C8, 640, 512), (C12, 400, 576)])
def test_many_tiles_per_cta_sampled_blocks(sl, oracle_mod, cp, rows, cols):
    # More 128-block tiles than the grid has CTAs (4-bit: 320 tiles on two
    # CTAs per SM; 3-bit: 150 tiles on one per SM), so CTAs run several tiles
    # and reuse their tensor memory, queues and barrier phases.  Blocks
    # sampled across the matrix (first, last, tile edges, random) must reach
    # the oracle's minimum error.
    rng = np.random.default_rng(21 + cp[0])
    W = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    fmt = inputs.make_format(rows, cols, *cp)
    rec, ep, err = gpu_encode(sl, fmt, W)
    nb = fmt["nb"]
    flat = [0, 127, 128, rows * nb - 1, 64 * 296 * 2 - 1, 64 * 296 * 2]
    flat += [int(v) for v in rng.integers(0, rows * nb, 12)]
    blocks = sorted({(f // nb, f % nb) for f in flat if f < rows * nb})
    check_against_oracle(oracle_mod, fmt, W.astype(np.float64), rec, ep, err, blocks)
    assert np.all(np.isfinite(err)) and np.all(err >= 0)


@pytest.mark.parametrize("cp", [C8, C12])
def test_leading_dimension_gives_the_same_records(sl, cp):
    # W as a column slice of a wider matrix (ldw > cols, ragged tail block)
    # encodes exactly as its contiguous copy: same records, exponents, errors.
    C = cp[0]
    rows, cols, wide = 37, 5 * C + 3, 8 * C + 4
    g = torch.Generator(device="cuda").manual_seed(17)
    Wwide = torch.randn((rows, wide), device="cuda", generator=g) * 0.02
    fmt = inputs.make_format(rows, cols, *cp)
    outs = []
    for W in (Wwide[:, :cols], Wwide[:, :cols].contiguous()):
        rec = torch.zeros((rows, fmt["rec_pitch"]), dtype=torch.int32, device="cuda")
        ep = (torch.zeros((rows, fmt["e_pitch"]), dtype=torch.uint8, device="cuda")
              if cp[1] == 4 else None)
        err = torch.empty((rows, fmt["nb"]), dtype=torch.float64, device="cuda")
        sl.encode(fmt, W, rec, ep, err)
        torch.cuda.synchronize()
        outs.append((rec.cpu(), None if ep is None else ep.cpu(), err.cpu()))
    assert Wwide[:, :cols].stride(0) == wide
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][2], outs[1][2])
    if cp[1] == 4:
        assert torch.equal(outs[0][1], outs[1][1])


@pytest.mark.parametrize("cp,seed", [(C8, 48395), (C8, 38137), (C12, 62544), (C12, 1596)])
def test_planted_fit_on_the_worst_conditioned_seeds(sl, oracle_mod, cp, seed):
    # The seeds whose U is closest to rank-deficient (condition number of
    # U^T U about 1e11 at 4 bits, 3e9 at 3 bits, checked here on the CPU):
    # a block planted on one of them still comes back as an exact fit with
    # the oracle's canonical triple -- the exact scoring's G^-1 is accurate
    # enough to round t* 2^e to the planted q.
    C, P = cp
    U = oracle_mod.block_basis(seed, C, P)
    assert np.linalg.cond(U.T @ U) > 1e9
    q = np.array([5, -3, 7, -6][:P], dtype=np.int64)
    e = 10
    fmt = inputs.make_format(1, C, *cp)
    w = (U @ q) * 2.0 ** -e
    assert np.array_equal(w.astype(np.float32).astype(np.float64), w)
    rec, ep, err = gpu_encode(sl, fmt, w.reshape(1, C).astype(np.float32))
    from oracle.search import seed_search
    s, qo, eo, e_err, _ = seed_search(w, C, P)
    gs, gq, ge = oracle_mod.block_fields(fmt, rec, ep, 0, 0)
    assert e_err == 0.0 and err[0, 0] == 0.0
    assert (gs, ge) == (s, eo) and np.array_equal(np.asarray(gq), np.asarray(qo))
    assert np.array_equal(oracle_mod.reconstruct_block(fmt, rec, ep, 0, 0), w)


@pytest.mark.parametrize("cp", [C8, C12])
def test_encode_save_load_then_gemv(sl, oracle_mod, tmp_path, cp):
    # The offline workflow: encode on the GPU, save the planes, load them
    # back (format, sizes and SHA-256 checked), then the GEMV on the loaded
    # planes matches the oracle GEMV on the same planes.
    from prng_seeded_decompress_b200 import store
    rng = np.random.default_rng(31 + cp[0])
    rows, cols = 48, 200
    W = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    fmt = inputs.make_format(rows, cols, *cp)
    rec, ep, _ = gpu_encode(sl, fmt, W)
    store.save_layer(str(tmp_path / "layer"), fmt, rec, ep)
    fmt2, rec2, ep2 = store.load_layer(str(tmp_path / "layer"))
    assert fmt2 == fmt and np.array_equal(rec2, rec)
    xb, xv = inputs.make_activations((cols,), "f16", 5)
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.float16)
    y = torch.empty(rows, device="cuda")
    sl.gemv(fmt2, torch.from_numpy(rec2.view(np.int32)).cuda(),
            None if ep2 is None else torch.from_numpy(ep2).cuda(), x, y)
    torch.cuda.synchronize()
    ref, refabs = oracle_mod.gemv(fmt2, rec2, ep2, xv)
    assert np.all(np.abs(y.cpu().numpy().astype(np.float64) - ref) <= 1e-5 * refabs + 1e-30)
