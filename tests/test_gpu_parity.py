"""GPU parity: the CUDA path against the CPU oracle on the same seeded inputs.

Decompression must match bit for bit (every weight is a short dyadic
rational, exact in fp32).  Products must satisfy, per output,
|y - y_oracle| <= 1e-5 * sum_j |W_rj x_j| (the oracle accumulates in fp64).
All calls go through the C ABI (ctypes binding).
"""
import os

import numpy as np
import pytest

from prng_seeded_decompress_b200 import inputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 1e-5
C8, C12 = inputs.FORMAT_4BIT, inputs.FORMAT_3BIT


@pytest.fixture(scope="module")
def sl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from prng_seeded_decompress_b200 import build
    build.build()
    from prng_seeded_decompress_b200 import seedlm
    seedlm.init()
    return seedlm


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def act_tensor(bits, dtype):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
    return t.view(torch.float16 if dtype == "f16" else torch.bfloat16)


def planes(L):
    rec = dev(L["rec"].view(np.int32))
    ep = dev(L["eplane"]) if L["fmt"]["P"] == 4 else None
    return rec, ep


def gpu_gemv(sl, L, xbits, dtype="f16"):
    rec, ep = planes(L)
    x = act_tensor(xbits, dtype)
    y = torch.full((L["fmt"]["rows"],), float("nan"), device="cuda")
    sl.gemv(L["fmt"], rec, ep, x, y)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def assert_within(y, ref, refabs):
    err = np.abs(y - ref)
    bound = TOL * refabs + 1e-30
    bad = np.nonzero(err > bound)[0]
    assert bad.size == 0, f"{bad.size} outputs out of tolerance, e.g. row {bad[:5]}: " \
                          f"err {err[bad[:5]]} bound {bound[bad[:5]]}"


# ------------------------------------------------------------- decompress

DECOMP_SHAPES = [
    (C8, 512, 512), (C8, 37, 203), (C8, 1, 1), (C8, 3, 8), (C8, 130, 2048),
    # Whole 32-column chunks but rows that end inside a warp's 1024-column
    # item (bulk tensor stores clipped at the row's end).
    (C8, 9, 96), (C8, 33, 1056), (C8, 1, 32),
    (C12, 61, 4096), (C12, 17, 1000), (C12, 2, 12), (C12, 5, 13),
]


@pytest.mark.parametrize("cp,rows,cols", DECOMP_SHAPES)
def test_decompress_bit_exact(sl, oracle_mod, cp, rows, cols):
    L = inputs.make_layer(rows, cols, *cp, seed=1000 + rows + cols, e_range=(0, 15))
    rec, ep = planes(L)
    W = torch.full((rows, cols), float("nan"), device="cuda")
    sl.decompress(L["fmt"], rec, ep, W)
    torch.cuda.synchronize()
    ref = oracle_mod.decompress(L["fmt"], L["rec"], L["eplane"]).astype(np.float32)
    got = W.cpu().numpy()
    # Bit patterns, so that -0 and +0 would differ too.
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("cp,rows,cols", [(C8, 4096, 4096), (C12, 2048, 6000)])
def test_decompress_multi_item_loop_bit_exact(sl, oracle_mod, cp, rows, cols):
    # More warp items (one row's 128 consecutive blocks each) than the grid
    # has warps (4 CTAs x 8 warps per SM), so every warp walks several items
    # and takes the next-item prefetch and row/column relocation path.
    L = inputs.make_layer(rows, cols, *cp, seed=rows * 3 + cols, e_range=(0, 15))
    rec, ep = planes(L)
    W = torch.full((rows, cols), float("nan"), device="cuda")
    sl.decompress(L["fmt"], rec, ep, W)
    torch.cuda.synchronize()
    ref = oracle_mod.decompress(L["fmt"], L["rec"], L["eplane"]).astype(np.float32)
    assert np.array_equal(W.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_decompress_full_size_sampled_rows(sl, oracle_mod):
    # The 70B down projection (8192 x 28672, 4-bit), the shape the benchmark
    # decompresses: bit patterns of sampled rows (first and last rows plus a
    # random sample) against the oracle's decompression of those rows' records.
    rows, cols = 8192, 28672
    L = inputs.make_layer(rows, cols, *C8, seed=4242, e_range=(0, 15))
    rec, ep = planes(L)
    W = torch.full((rows, cols), float("nan"), device="cuda")
    sl.decompress(L["fmt"], rec, ep, W)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    sample = np.unique(np.concatenate([np.arange(4), np.arange(rows - 4, rows),
                                       rng.integers(0, rows, 24)]))
    sub = dict(L["fmt"], rows=int(sample.size))
    ref = oracle_mod.decompress(sub, np.ascontiguousarray(L["rec"][sample]), None)
    got = W[torch.from_numpy(sample).cuda()].cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.astype(np.float32).view(np.uint32))


def test_decompress_leading_dimension_and_seed_zero(sl, oracle_mod):
    fmt = inputs.make_format(3, 20, 8, 3)
    seeds = np.array([[0, 1, 65535], [0, 0, 0], [12345, 0, 7]])
    q = np.random.default_rng(3).integers(-8, 8, size=(3, 3, 3))
    e = np.array([[0, 15, 8], [3, 4, 5], [12, 12, 12]])
    rec_np, ep_np = inputs.pack_records(fmt, seeds, q, e)
    L = dict(fmt=fmt, rec=rec_np, eplane=ep_np)
    rec, ep = planes(L)
    W = torch.full((3, 27), -1.0, device="cuda")
    sl.decompress(fmt, rec, ep, W, ldw=27)
    torch.cuda.synchronize()
    ref = oracle_mod.decompress(fmt, rec_np, ep_np)
    got = W.cpu().numpy()
    assert np.array_equal(got[:, :20], ref.astype(np.float32))
    assert np.all(got[:, 20:] == -1.0)


# ------------------------------------------------------------------- gemv

GEMV_SHAPES = [
    (C8, 512, 512), (C8, 1024, 1024), (C8, 64, 2048), (C8, 37, 203), (C8, 1, 8),
    (C8, 5, 1), (C8, 333, 4096), (C8, 70, 9000),
    (C12, 96, 4096), (C12, 40, 14336), (C12, 17, 1000), (C12, 3, 12), (C12, 9, 25),
]


@pytest.mark.parametrize("cp,rows,cols", GEMV_SHAPES)
def test_gemv_matches_oracle(sl, oracle_mod, cp, rows, cols):
    L = inputs.make_layer(rows, cols, *cp, seed=2000 + rows + cols)
    xb, xv = inputs.make_activations((cols,), "f16", 3000 + cols)
    y = gpu_gemv(sl, L, xb)
    ref, refabs = oracle_mod.gemv(L["fmt"], L["rec"], L["eplane"], xv)
    assert_within(y, ref, refabs)


@pytest.mark.parametrize("cp", [C8, C12])
def test_gemv_bf16_activations(sl, oracle_mod, cp):
    L = inputs.make_layer(200, 3000, *cp, seed=11)
    xb, xv = inputs.make_activations((3000,), "bf16", 12)
    y = gpu_gemv(sl, L, xb, "bf16")
    ref, refabs = oracle_mod.gemv(L["fmt"], L["rec"], L["eplane"], xv)
    assert_within(y, ref, refabs)


@pytest.mark.parametrize("cp", [C8, C12])
def test_gemv_one_hot_is_bit_exact(sl, oracle_mod, cp):
    # One nonzero product per row: the fused kernel must return column j of W
    # exactly (closed-form special case).
    rows, cols = 77, 777
    L = inputs.make_layer(rows, cols, *cp, seed=21, e_range=(0, 15))
    W = oracle_mod.decompress(L["fmt"], L["rec"], L["eplane"])
    for j in (0, 5, cols - 1):
        xv = np.zeros(cols)
        xv[j] = 1.0
        xb = xv.astype(np.float16).view(np.uint16)
        y = gpu_gemv(sl, L, xb)
        assert np.array_equal(y, W[:, j])


def test_gemv_is_deterministic_and_needs_no_zeroed_output(sl):
    L = inputs.make_layer(1000, 8192, *C8, seed=31)
    xb, _ = inputs.make_activations((8192,), "f16", 32)
    y1 = gpu_gemv(sl, L, xb)
    y2 = gpu_gemv(sl, L, xb)
    assert np.array_equal(y1.view(np.uint64), y2.view(np.uint64))


def test_gemv_empty_shapes(sl):
    for rows, cols in ((0, 64), (5, 0)):
        L = inputs.make_layer(rows, cols, *C8, seed=1)
        xb = np.zeros(max(cols, 1), np.uint16)
        if rows:
            y = gpu_gemv(sl, L, xb)
            assert np.array_equal(y, np.zeros(rows))
        else:
            rec, ep = planes(L)
            y = torch.zeros(1, device="cuda")
            sl.gemv(L["fmt"], rec, ep, act_tensor(xb, "f16"), y)


def test_gemm_decompress_encode_empty_shapes(sl):
    # rows = 0: nothing is launched or written; cols = 0: Y is all zeros (an
    # empty sum), decompression and encoding have nothing to do.
    for rows, cols in ((0, 64), (5, 0)):
        L = inputs.make_layer(rows, cols, *C8, seed=2)
        rec, ep = planes(L)
        X = torch.zeros((3, max(cols, 1)), dtype=torch.bfloat16, device="cuda")
        Y = torch.full((3, max(rows, 1)), float("nan"), device="cuda")
        sl.gemm_smallM(L["fmt"], rec, ep, X, Y)
        Y2 = torch.full((300, max(rows, 1)), float("nan"), device="cuda")
        sl.gemm(L["fmt"], rec, ep, torch.zeros((300, max(cols, 1)), dtype=torch.bfloat16,
                                               device="cuda"), Y2)
        W = torch.full((max(rows, 1), max(cols, 1)), float("nan"), device="cuda")
        sl.decompress(L["fmt"], rec, ep, W, ldw=max(cols, 1))
        sl.encode(L["fmt"], W, rec, ep, ldw=max(cols, 1))
        torch.cuda.synchronize()
        if rows:
            assert torch.equal(Y, torch.zeros_like(Y)) and torch.equal(Y2, torch.zeros_like(Y2))
        else:
            assert torch.isnan(Y).all() and torch.isnan(Y2).all()
        assert torch.isnan(W).all()
    assert sl.device_error() == 0


@pytest.mark.parametrize("cp,rows,cols", [(C8, 8192, 28672), (C8, 10240, 8192),
                                          (C12, 28672, 4096), (C12, 4096, 14336)])
def test_gemv_full_size_sampled_rows(sl, oracle_mod, cp, rows, cols):
    # The layer shapes the benchmark times, checked on a sample of rows that
    # covers the first and last tiles.
    L = inputs.make_layer(rows, cols, *cp, seed=rows + 7 * cols)
    xb, xv = inputs.make_activations((cols,), "f16", 99)
    y = gpu_gemv(sl, L, xb)
    rng = np.random.default_rng(0)
    sample = np.unique(np.concatenate([np.arange(8), np.arange(rows - 8, rows),
                                       rng.integers(0, rows, 48)]))
    ref, refabs = oracle_mod.gemv_rows(L["fmt"], L["rec"], L["eplane"], xv, sample)
    assert_within(y[sample], ref, refabs)


@pytest.mark.parametrize("rows,cols,dtype", [(19000, 1000, "bf16"), (37888, 385, "f16"),
                                             (28672, 8192, "f16"), (18944, 7, "bf16"),
                                             (18796, 30, "f16"), (18797, 30, "f16"),
                                             (37889, 30, "bf16")])
def test_gemv_tall_3bit_column_tables(sl, oracle_mod, rows, cols, dtype):
    # Tall 3-bit matrices (128 to 256 rows per SM) take the column-table
    # kernel: columns not a multiple of C, a last strip of 32 column blocks
    # that is partly empty (1000 columns: 84 blocks; 385: 33), rows not a
    # multiple of the 16 warps, the most rows per CTA it takes (37888), the
    # fewest (18944) with one 7-column block per row, the 3-bit MLP shape on
    # sampled rows, and both sides of the kernel choice on 148 SMs (18796
    # rows: 127 per CTA, per-row kernel; 18797: 128; 37889: 257, per-row
    # kernel again).  Two calls give the same bits.
    L = inputs.make_layer(rows, cols, *C12, seed=rows + cols, e_range=(0, 15))
    xb, xv = inputs.make_activations((cols,), dtype, 18)
    y = gpu_gemv(sl, L, xb, dtype)
    again = gpu_gemv(sl, L, xb, dtype)
    assert np.array_equal(y.view(np.uint64), again.view(np.uint64))
    if cols <= 1000:
        ref, refabs = oracle_mod.gemv(L["fmt"], L["rec"], L["eplane"], xv, threads=os.cpu_count() or 1)
        assert_within(y, ref, refabs)
    else:
        rng = np.random.default_rng(4)
        sample = np.unique(np.concatenate([np.arange(8), np.arange(rows - 8, rows),
                                           rng.integers(0, rows, 48)]))
        ref, refabs = oracle_mod.gemv_rows(L["fmt"], L["rec"], L["eplane"], xv, sample)
        assert_within(y[sample], ref, refabs)


@pytest.mark.parametrize("cp,rows", [(C12, 18944), (C12, 300), (C8, 300)])
@pytest.mark.parametrize("scale", [1e34, 1e-30])
def test_gemv_extreme_activations(sl, oracle_mod, cp, rows, scale):
    # bf16 activations near the top of the range and far below 1.  The
    # column-table kernel (3 bits, 18944 rows) keeps x's partial sums scaled
    # by 2^-15, within the range of x itself (a 2^15 larger table entry
    # would overflow fp32); the per-row kernels multiply x by the weights
    # themselves (at most P * 8 in magnitude).
    cols = 300
    L = inputs.make_layer(rows, cols, *cp, seed=77, e_range=(0, 15))
    base = np.random.default_rng(78).standard_normal(cols).astype(np.float32)
    xb = inputs.f32_to_bf16_bits((base * np.float32(scale)).astype(np.float32))
    xv = inputs.bf16_bits_to_f64(xb)
    assert np.all(np.isfinite(xv))
    y = gpu_gemv(sl, L, xb, "bf16")
    ref, refabs = oracle_mod.gemv(L["fmt"], L["rec"], L["eplane"], xv, threads=os.cpu_count() or 1)
    assert np.all(np.isfinite(y))
    err = np.abs(y - ref)
    assert np.all(err <= TOL * refabs), float((err / (refabs + 1e-300)).max())


@pytest.mark.parametrize("cp,rows,cols", [(C8, 100000, 16), (C12, 100000, 24),
                                          (C8, 1800, 56320), (C12, 6000, 42240)])
def test_gemv_multi_pass_and_wide_x(sl, oracle_mod, cp, rows, cols):
    # 100,000 short rows give each CTA about 169 row groups, more than one
    # partial-sum pass holds (144 for 16 warps), so every CTA runs two
    # passes: the second re-zeroes the partials and reuses the staged x.
    # The wide shapes stage x in several column segments.  Checked on
    # sampled rows.
    L = inputs.make_layer(rows, cols, *cp, seed=rows + cols)
    xb, xv = inputs.make_activations((cols,), "f16", 17)
    y = gpu_gemv(sl, L, xb)
    rng = np.random.default_rng(1)
    sample = np.unique(np.concatenate([np.arange(16), np.arange(rows - 16, rows),
                                       rng.integers(0, rows, 96)]))
    ref, refabs = oracle_mod.gemv_rows(L["fmt"], L["rec"], L["eplane"], xv, sample)
    assert_within(y[sample], ref, refabs)


def test_decompress_then_dense_equals_fused(sl, oracle_mod):
    L = inputs.make_layer(300, 5000, *C8, seed=41)
    xb, xv = inputs.make_activations((5000,), "f16", 42)
    rec, ep = planes(L)
    W = torch.empty((300, 5000), device="cuda")
    sl.decompress(L["fmt"], rec, ep, W)
    y = gpu_gemv(sl, L, xb)
    Wd = W.cpu().numpy().astype(np.float64)
    ref = Wd @ xv
    assert_within(y, ref, np.abs(Wd) @ np.abs(xv))


# ------------------------------------------------------------ small-M GEMM

def gpu_gemm(sl, L, Xb, dtype="bf16", workspace=None):
    rec, ep = planes(L)
    M = Xb.shape[0]
    X = act_tensor(Xb, dtype)
    Y = torch.full((M, L["fmt"]["rows"]), float("nan"), device="cuda")
    sl.gemm_smallM(L["fmt"], rec, ep, X, Y, workspace=workspace)
    torch.cuda.synchronize()
    assert sl.device_error() == 0
    return Y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("cp", [C8, C12])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 16, 17, 33, 64])
def test_gemm_small_matches_oracle(sl, oracle_mod, cp, M):
    rows, cols = 300, 3000  # 3 row tiles (one ragged), ragged last stage, split-K
    L = inputs.make_layer(rows, cols, *cp, seed=50 + M)
    Xb, Xv = inputs.make_activations((M, cols), "bf16", 60 + M)
    got = gpu_gemm(sl, L, Xb)
    ref, refabs = oracle_mod.gemm(L["fmt"], L["rec"], L["eplane"], Xv)
    for m in range(M):
        assert_within(got[m], ref[m], refabs[m])


@pytest.mark.parametrize("cp", [C8, C12])
def test_gemm_small_fp16_and_odd_shapes(sl, oracle_mod, cp):
    for rows, cols, M in ((1, 12, 5), (129, 100, 16), (70, 1000, 40)):
        L = inputs.make_layer(rows, cols, *cp, seed=rows + cols + M)
        Xb, Xv = inputs.make_activations((M, cols), "f16", 5)
        got = gpu_gemm(sl, L, Xb, "f16")
        ref, refabs = oracle_mod.gemm(L["fmt"], L["rec"], L["eplane"], Xv)
        for m in range(M):
            assert_within(got[m], ref[m], refabs[m])


@pytest.mark.parametrize("cp,rows,cols,M", [(C8, 57344, 128, 16), (C12, 20000, 200, 33)])
def test_gemm_many_short_tiles_per_cta(sl, oracle_mod, cp, rows, cols, M):
    # Few K chunks per row tile and many tiles: each CTA's range covers several
    # whole tiles (written straight to Y) plus shared ones at its ends, and
    # reuses both TMEM accumulators more than once.
    L = inputs.make_layer(rows, cols, *cp, seed=rows + M)
    Xb, Xv = inputs.make_activations((M, cols), "bf16", 17)
    got = gpu_gemm(sl, L, Xb)
    ref, refabs = oracle_mod.gemm(L["fmt"], L["rec"], L["eplane"], Xv, threads=os.cpu_count() or 1)
    for m in range(M):
        assert_within(got[m], ref[m], refabs[m])


@pytest.mark.parametrize("cp", [C8, C12])
def test_gemm_bf16_rows_of_any_magnitude(sl, oracle_mod, cp):
    # bf16 activations reach the tensor cores as fp16 scaled by a power of two
    # per row, chosen from the row's largest finite magnitude: rows near the
    # top and the bottom of bf16's range (subnormal included), a zero row,
    # and a row spanning 2^40 between its largest and smallest elements.
    rows, cols = 300, 3000
    L = inputs.make_layer(rows, cols, *cp, seed=404)
    rng = np.random.default_rng(405)
    base = rng.standard_normal((6, cols)).astype(np.float32)
    scales = np.array([1e30, 1e-30, 0.0, 1.5e-39, 1.0, 1e34], dtype=np.float32)
    v = base * scales[:, None]
    v[4] = base[4] * np.float32(1e-6)
    v[4, 7] = np.float32(1e6)  # one element 2^40 above the rest
    Xb = inputs.f32_to_bf16_bits(v.astype(np.float32))
    Xv = inputs.bf16_bits_to_f64(Xb)
    assert np.all(np.isfinite(Xv)) and np.any(Xv[3] != 0) and np.all(np.abs(Xv[3]) < 2.0 ** -126)
    got = gpu_gemm(sl, L, Xb)
    ref, refabs = oracle_mod.gemm(L["fmt"], L["rec"], L["eplane"], Xv)
    assert np.array_equal(got[2], np.zeros(rows))
    for m in range(6):
        # No absolute floor: the bound scales with the row.
        err = np.abs(got[m] - ref[m])
        assert np.all(err <= TOL * refabs[m]), (m, float((err / (refabs[m] + 1e-300)).max()))


@pytest.mark.parametrize("M", [2, 3, 4])
def test_gemm_few_rows_on_cuda_cores_match_oracle(sl, oracle_mod, M):
    # 2 to 4 rows of X at 3 bits run on the CUDA cores: rows not a multiple
    # of the item height, columns not a multiple of C, x wider than one
    # shared-memory segment (12,000 columns), a single block, fp16 and bf16;
    # no workspace.
    cp = C12
    assert sl.gemm_workspace_bytes(inputs.make_format(300, 5000, *cp), M) == 0
    assert sl.gemm_any_workspace_bytes(inputs.make_format(300, 5000, *cp), M) == 0
    assert sl.gemm_workspace_bytes(inputs.make_format(300, 5000, *C8), M) > 0  # tensor cores
    for rows, cols, dt in ((301, 12000, "bf16"), (37, 100, "f16"), (5, 12, "bf16"), (2, 9, "f16")):
        L = inputs.make_layer(rows, cols, *cp, seed=900 + rows + M)
        Xb, Xv = inputs.make_activations((M, cols), dt, 901 + cols + M)
        rec, ep = planes(L)
        X = act_tensor(Xb, dt)
        Y = torch.full((M, rows), float("nan"), device="cuda")
        sl.gemm_smallM(L["fmt"], rec, ep, X, Y, workspace=torch.zeros(0, dtype=torch.uint8, device="cuda"))
        torch.cuda.synchronize()
        assert sl.device_error() == 0
        got = Y.cpu().numpy().astype(np.float64)
        ref, refabs = oracle_mod.gemm(L["fmt"], L["rec"], L["eplane"], Xv)
        for m in range(M):
            assert_within(got[m], ref[m], refabs[m])


@pytest.mark.parametrize("cp,rows,cols,M", [(C8, 28672, 8192, 4), (C8, 8192, 28672, 2),
                                            (C12, 28672, 8192, 3), (C12, 8192, 28672, 4)])
def test_gemm_few_rows_full_size_sampled_rows(sl, oracle_mod, cp, rows, cols, M):
    # Full 70B MLP shapes: several partial-sum passes per CTA (28672 rows)
    # and several x segments (28672 columns); the same call twice gives the
    # same bits (sums in a fixed order).
    L = inputs.make_layer(rows, cols, *cp, seed=rows + cols + 7 * M)
    Xb, Xv = inputs.make_activations((M, cols), "bf16", 93 + M)
    got = gpu_gemm(sl, L, Xb)
    again = gpu_gemm(sl, L, Xb)
    assert np.array_equal(got.view(np.uint64), again.view(np.uint64))
    rng = np.random.default_rng(3)
    sample = np.unique(np.concatenate([np.arange(4), np.arange(rows - 4, rows),
                                       rng.integers(0, rows, 12)]))
    ref, refabs = oracle_mod.gemm_rows(L["fmt"], L["rec"], L["eplane"], Xv, sample)
    for m in range(M):
        assert_within(got[m, sample], ref[m], refabs[m])


@pytest.mark.parametrize("cp", [C8, C12])
def test_gemm_bf16_wide_rows_share_their_maximum(sl, oracle_mod, cp):
    # Rows wide enough (28672 columns) that the staging kernel splits each
    # row over several CTAs which exchange their parts' maxima: the row's
    # largest element sits in the first, a middle or the last part, or the
    # row spans 2^40; every part must scale by the one row-wide power of two.
    rows, cols = 200, 28672
    L = inputs.make_layer(rows, cols, *cp, seed=406)
    rng = np.random.default_rng(407)
    v = (rng.standard_normal((6, cols)) * 1e-3).astype(np.float32)
    v[0, 5] = np.float32(3e4)             # maximum in the first part
    v[1, cols // 2 + 3] = np.float32(3e4)  # ... in a middle part
    v[2, cols - 2] = np.float32(3e4)       # ... in the last part
    v[3] *= np.float32(1e-33)              # the whole row far below 1
    v[3, cols - 9] = np.float32(2e-30)
    v[4] = 0.0
    v[5, cols - 1] = np.float32(1e9)       # 2^40 above the rest, last column
    Xb = inputs.f32_to_bf16_bits(v)
    Xv = inputs.bf16_bits_to_f64(Xb)
    got = gpu_gemm(sl, L, Xb)
    ref, refabs = oracle_mod.gemm(L["fmt"], L["rec"], L["eplane"], Xv, threads=os.cpu_count() or 1)
    assert np.array_equal(got[4], np.zeros(rows))
    for m in range(6):
        err = np.abs(got[m] - ref[m])
        assert np.all(err <= TOL * refabs[m]), (m, float((err / (refabs[m] + 1e-300)).max()))


def gpu_gemm_any(sl, L, Xb, dtype="bf16"):
    rec, ep = planes(L)
    M = Xb.shape[0]
    X = act_tensor(Xb, dtype)
    Y = torch.full((M, L["fmt"]["rows"]), float("nan"), device="cuda")
    sl.gemm(L["fmt"], rec, ep, X, Y)
    torch.cuda.synchronize()
    assert sl.device_error() == 0
    return Y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("cp", [C8, C12])
@pytest.mark.parametrize("M", [65, 128, 129, 256, 257, 600])
def test_gemm_large_batches_match_oracle(sl, oracle_mod, cp, M):
    # seedlm_gemm: one N = 128 pass (65-128 rows), one N = 256 pass with
    # half-width units (129-256), and several passes sharing one workspace
    # (257, 600: the last pass narrower than the others).
    rows, cols = 300, 3000  # 3 row tiles (one ragged), ragged last K chunk
    L = inputs.make_layer(rows, cols, *cp, seed=700 + M)
    Xb, Xv = inputs.make_activations((M, cols), "bf16", 701 + M)
    got = gpu_gemm_any(sl, L, Xb)
    ref, refabs = oracle_mod.gemm(L["fmt"], L["rec"], L["eplane"], Xv, threads=os.cpu_count() or 1)
    for m in range(M):
        assert_within(got[m], ref[m], refabs[m])


@pytest.mark.parametrize("cp", [C8, C12])
def test_gemm_large_batches_fp16_and_small_M_agreement(sl, oracle_mod, cp):
    L = inputs.make_layer(129, 1000, *cp, seed=711)
    Xb, Xv = inputs.make_activations((200, 1000), "f16", 712)
    got = gpu_gemm_any(sl, L, Xb, "f16")
    ref, refabs = oracle_mod.gemm(L["fmt"], L["rec"], L["eplane"], Xv, threads=os.cpu_count() or 1)
    for m in range(200):
        assert_within(got[m], ref[m], refabs[m])
    # Up to 64 rows seedlm_gemm is seedlm_gemm_smallM, bit for bit.
    Xs = Xb[:33]
    assert np.array_equal(gpu_gemm_any(sl, L, Xs, "f16").view(np.uint64),
                          gpu_gemm(sl, L, Xs, "f16").view(np.uint64))


def test_gemm_any_M_one_row_is_the_gemv_and_workspace_query(sl):
    L = inputs.make_layer(256, 4096, *C8, seed=73)
    xb, _ = inputs.make_activations((1, 4096), "bf16", 74)
    assert sl.gemm_any_workspace_bytes(L["fmt"], 1) == 0  # M = 1 runs the GEMV
    got = gpu_gemm_any(sl, L, xb)
    assert np.array_equal(got[0], gpu_gemv(sl, L, xb[0], "bf16"))
    # A full pass and a narrower last pass: the query covers the larger need.
    need = sl.gemm_any_workspace_bytes(L["fmt"], 300)
    assert need >= sl.gemm_any_workspace_bytes(L["fmt"], 256)
    assert need >= sl.gemm_any_workspace_bytes(L["fmt"], 44)
    assert sl.gemm_any_workspace_bytes(L["fmt"], 64) == sl.gemm_workspace_bytes(L["fmt"], 64)
    # Too small a workspace is refused before anything runs.
    rec, ep = planes(L)
    X = torch.zeros((300, 4096), dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros((300, 256), device="cuda")
    ws = torch.zeros(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(sl.SeedLMError) as exc:
        sl.gemm(L["fmt"], rec, ep, X, Y, workspace=ws)
    assert exc.value.code == -1


@pytest.mark.parametrize("cp,rows,cols,M", [(C8, 28672, 8192, 256), (C12, 8192, 28672, 300)])
def test_gemm_large_batches_full_size_sampled_rows(sl, oracle_mod, cp, rows, cols, M):
    L = inputs.make_layer(rows, cols, *cp, seed=rows + cols + M)
    Xb, Xv = inputs.make_activations((M, cols), "bf16", 92)
    got = gpu_gemm_any(sl, L, Xb)
    rng = np.random.default_rng(2)
    sample = np.unique(np.concatenate([np.arange(2), np.arange(rows - 2, rows),
                                       rng.integers(0, rows, 8)]))
    ref, refabs = oracle_mod.gemm_rows(L["fmt"], L["rec"], L["eplane"], Xv, sample)
    for m in range(M):
        assert_within(got[m, sample], ref[m], refabs[m])


def test_gemm_workspace_reuse_is_deterministic(sl):
    # The same workspace across calls (counters must be left at zero) and
    # bit-identical results (split-K partials are added in a fixed order).
    L = inputs.make_layer(1000, 8192, *C8, seed=81)
    Xb, _ = inputs.make_activations((64, 8192), "bf16", 82)
    ws = sl.gemm_workspace(L["fmt"], 64)
    a = gpu_gemm(sl, L, Xb, workspace=ws)
    b = gpu_gemm(sl, L, Xb, workspace=ws)
    assert np.array_equal(a.view(np.uint64), b.view(np.uint64))


@pytest.mark.parametrize("cp,rows,cols,M", [(C8, 8192, 28672, 64), (C8, 28672, 8192, 16),
                                            (C12, 8192, 28672, 16), (C12, 28672, 8192, 64)])
def test_gemm_full_size_sampled_rows(sl, oracle_mod, cp, rows, cols, M):
    L = inputs.make_layer(rows, cols, *cp, seed=rows + cols + M)
    Xb, Xv = inputs.make_activations((M, cols), "bf16", 91)
    got = gpu_gemm(sl, L, Xb)
    rng = np.random.default_rng(1)
    sample = np.unique(np.concatenate([np.arange(4), np.arange(rows - 4, rows),
                                       rng.integers(0, rows, 12)]))
    ref, refabs = oracle_mod.gemm_rows(L["fmt"], L["rec"], L["eplane"], Xv, sample)
    for m in range(M):
        assert_within(got[m, sample], ref[m], refabs[m])


def test_gemm_m1_equals_gemv_bitwise(sl):
    L = inputs.make_layer(256, 4096, *C8, seed=71)
    xb, _ = inputs.make_activations((1, 4096), "bf16", 72)
    got = gpu_gemm(sl, L, xb)
    y = gpu_gemv(sl, L, xb[0], "bf16")
    assert np.array_equal(got[0], y)


# --------------------------------------------------------- dense reference

def test_dense_f16_gemv(sl):
    rng = np.random.default_rng(5)
    rows, cols = 1001, 4104
    Wh = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float16)
    xh = rng.standard_normal(cols).astype(np.float16)
    y = torch.empty(rows, device="cuda")
    sl.dense_gemv_f16(dev(Wh.view(np.int16)), dev(xh.view(np.int16)), y)
    torch.cuda.synchronize()
    Wd, xd = Wh.astype(np.float64), xh.astype(np.float64)
    assert_within(y.cpu().numpy().astype(np.float64), Wd @ xd, np.abs(Wd) @ np.abs(xd))


def test_misaligned_record_pointer_is_rejected(sl):
    L = inputs.make_layer(8, 64, *C8, seed=1)
    rec, _ = planes(L)
    x = torch.zeros(64, dtype=torch.float16, device="cuda")
    y = torch.zeros(8, device="cuda")
    with pytest.raises(sl.SeedLMError):
        sl.gemv(L["fmt"], rec.data_ptr() + 4, None, x, y)


# ------------------------------------------------------------ CUDA graphs

def test_graph_replay_matches_eager_calls(sl):
    # GEMV and the two-launch GEMM (programmatic dependent launch between the
    # X staging and the GEMM) captured once and replayed: bit-identical to
    # eager calls, every replay.
    L = inputs.make_layer(512, 2048, *C8, seed=31)
    rec, _ = planes(L)
    xb, _ = inputs.make_activations((2048,), "f16", 32)
    Xb, _ = inputs.make_activations((16, 2048), "bf16", 33)
    x = act_tensor(xb, "f16")
    X = act_tensor(Xb, "bf16")
    ws = sl.gemm_workspace(L["fmt"], 16)
    y = torch.empty(512, device="cuda")
    Y = torch.empty((16, 512), device="cuda")
    sl.gemv(L["fmt"], rec, None, x, y)
    sl.gemm_smallM(L["fmt"], rec, None, X, Y, workspace=ws)
    torch.cuda.synchronize()
    y0, Y0 = y.clone(), Y.clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            sl.gemv(L["fmt"], rec, None, x, y, stream=s)
            sl.gemm_smallM(L["fmt"], rec, None, X, Y, workspace=ws, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        y.fill_(float("nan"))
        Y.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, y0) and torch.equal(Y, Y0)
    assert sl.device_error() == 0
    del g


# ------------------------------------------------------------ wide x

@pytest.mark.parametrize("cp,rows,cols", [
    # Large-product kernel (one CTA per SM, 16 warps, at least 64 items per
    # CTA): 15 spans of 1024 columns (4 bits, 4 blocks per lane) or 31 of
    # 768 (3 bits) per x segment.
    (C8, 2400, 70000), (C12, 2400, 50000), (C8, 2400, 15360), (C8, 2400, 15361),
    (C12, 2400, 23808), (C12, 2400, 23809),
    # 3 bits with half-warp spans (chosen where the busiest CTA has fewer
    # lane units: less span padding against 8-row items): 63 spans of 16
    # units of 24 columns per segment -- one segment exactly, two, and the
    # Llama-3-8B width; ragged row counts.
    (C12, 2365, 24192), (C12, 2365, 24720), (C12, 7101, 4096),
    # Small-product kernel (a few items per CTA): 32 KB of x slots, 16 spans
    # of 512 columns (4 bits, 2 blocks per lane) or 8 of 768 (3 bits).
    (C8, 40, 8192), (C8, 40, 8193), (C12, 40, 6144), (C12, 40, 6145),
])
def test_gemv_wide_x_in_column_segments(sl, oracle_mod, cp, rows, cols):
    # x is staged in shared memory in column segments, so any width works;
    # each kernel variant is checked exactly at, and one column past, its
    # one-segment width, and the large one at many segments.  gemm_smallM with M = 1 runs the same kernel, same
    # bits.
    L = inputs.make_layer(rows, cols, *cp, seed=cols + rows)
    xb, xv = inputs.make_activations((cols,), "f16", 3)
    y = gpu_gemv(sl, L, xb)
    ref, refabs = oracle_mod.gemv(L["fmt"], L["rec"], L["eplane"], xv,
                                  threads=os.cpu_count() or 1)
    assert_within(y, ref, refabs)
    assert sl.gemm_workspace_bytes(L["fmt"], 1) == 0
    got = gpu_gemm(sl, L, xb.reshape(1, cols), dtype="f16")
    assert np.array_equal(got[0].astype(np.float32).view(np.uint32),
                          y.astype(np.float32).view(np.uint32))


# ------------------------------------------------------------ batched GEMV

@pytest.mark.parametrize("cp,shapes,dtype,same_bits", [
    # Products large enough that each alone runs the batch's configuration
    # (the large-product kernel, 148 CTAs x 16 warps), as the projections of
    # a 70B decoder layer do: the bits must agree.
    (C8, [(8192, 8192), (10240, 8192), (8192, 28672), (16384, 8192)], "f16", True),
    # Mixed shapes: one and several x segments, fewer row groups than SMs,
    # an empty matrix; the batch's configuration may differ from an entry's
    # own (another summation order), so only the tolerance applies.
    (C8, [(1000, 8192), (40, 70000), (0, 512), (300, 999), (5000, 4096)], "f16", False),
    (C12, [(700, 4096), (33, 30000), (2000, 1000)], "bf16", False),
])
def test_gemv_batch_matches_separate_calls(sl, oracle_mod, cp, shapes, dtype, same_bits):
    # One launch for several GEMVs of one format.  Every output is within
    # tolerance of the oracle, repeated batches give the same bits, and when
    # the launch configuration is the one each entry would get alone, the
    # bits of the separate seedlm_gemv calls.
    items, refs = [], []
    for i, (rows, cols) in enumerate(shapes):
        L = inputs.make_layer(rows, cols, *cp, seed=500 + i)
        xb, xv = inputs.make_activations((cols,), dtype, 600 + i)
        rec, ep = planes(L)
        x = act_tensor(xb, dtype)
        y = torch.full((rows,), float("nan"), device="cuda")
        items.append((L["fmt"], rec, ep, x, y))
        refs.append((L, xv))
    sl.gemv_batch(items)
    torch.cuda.synchronize()
    first = [it[4].clone() for it in items]
    sl.gemv_batch(items)
    torch.cuda.synchronize()
    for (fmt, rec, ep, x, y), y0, (L, xv) in zip(items, first, refs):
        assert torch.equal(y.view(torch.int32), y0.view(torch.int32))
        if same_bits:
            ys = torch.full_like(y, float("nan"))
            sl.gemv(fmt, rec, ep, x, ys)
            torch.cuda.synchronize()
            assert torch.equal(y.view(torch.int32), ys.view(torch.int32))
        if fmt["rows"]:
            ref, refabs = oracle_mod.gemv(L["fmt"], L["rec"], L["eplane"], xv,
                                          threads=os.cpu_count() or 1)
            assert_within(y.cpu().numpy().astype(np.float64), ref, refabs)


def test_gemv_batch_rejects_mixed_formats_and_too_many(sl):
    L8 = inputs.make_layer(8, 64, *C8, seed=1)
    L12 = inputs.make_layer(8, 72, *C12, seed=2)
    x = torch.zeros(72, dtype=torch.float16, device="cuda")
    y = torch.zeros(8, device="cuda")
    r8, _ = planes(L8)
    r12, e12 = planes(L12)
    with pytest.raises(sl.SeedLMError) as exc:
        sl.gemv_batch([(L8["fmt"], r8, None, x, y), (L12["fmt"], r12, e12, x, y)])
    assert exc.value.code == -2
    with pytest.raises(sl.SeedLMError) as exc:
        sl.gemv_batch([(L8["fmt"], r8, None, x, y)] * 9)
    assert exc.value.code == -1
