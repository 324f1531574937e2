"""GPU parity of the dual-path product (osc_linear, osc_linear_fp8_fallback, osc_linear_grouped)
against the oracle's fp64 Y.

Tolerance: the fp32 accumulator (the Yf32 output of the same launch) must satisfy
max|dY| <= 1e-3 * max|Y_ref| over the compared rows. The bf16 output must equal the fp32
accumulator rounded to bf16, and lie within 1e-3 * max|Y_ref| + 1 bf16 ulp of Y_ref.

Every product is launched twice: once with the fp32 debug output (checked as above) and once
without it, which is the launch a caller (and the bench) makes; the two bf16 outputs must be
identical bit for bit. Full-size shapes are checked on every row (QKV at M = 2048) or on the
first, last and one seeded row of every 128-row block."""
import numpy as np
import pytest
import torch

from tests._layout import bf16_ulp
from tests.conftest import to_dev, to_np
from w4a4_outlier_separated_b200 import inputs as I

pytestmark = pytest.mark.gpu
REL = 1e-3


def _compare(Y_bf16, Y_f32, Yref):
    ymax = np.abs(Yref).max()
    d32 = np.abs(Y_f32.astype(np.float64) - Yref).max()
    assert d32 <= REL * ymax, (d32, ymax)
    yb = I.bf16_to_f32(Y_bf16).astype(np.float64)
    assert np.array_equal(Y_bf16, I.bf16_bits(Y_f32))            # bf16 = RNE(fp32 accumulator)
    assert np.all(np.abs(yb - Yref) <= REL * ymax + bf16_ulp(Yref))


def _run_osc(oracle, osc, X, W, G, L, rows=None, bn=0, pair=-1):
    M, K = X.shape
    N = W.shape[0]
    K_L = I.pad16(oracle.table_count(L)) if L is not None else 0
    Ld = to_dev(L) if L is not None else None
    prev, prev_pair = osc.osc_set_tile_n(bn), osc.osc_set_cta_pair(pair)
    try:
        QW, SW, WL = osc.prepare_weight(to_dev(W), G, Ld, K_L)
        QX, SX, B = osc.quantize(to_dev(X), G, Ld, K_L)
        Y, Yf = osc.linear(QX, SX, B, QW, SW, WL, M, N, K, G, K_L, want_f32=True)
        Y_plain, _ = osc.linear(QX, SX, B, QW, SW, WL, M, N, K, G, K_L)
        torch.cuda.synchronize()
    finally:
        osc.osc_set_tile_n(prev)
        osc.osc_set_cta_pair(prev_pair)
    assert osc.osc_status() == (0, 0)
    assert torch.equal(Y_plain.view(torch.int16), Y.view(torch.int16))   # launch without Yf32
    Lo = L if L is not None else np.full(K // G, -1, np.int8)
    cw, ew, WLr = oracle.osc_prepare_weight(W, G, Lo, K_L)
    sel = np.arange(M) if rows is None else np.asarray(rows)
    ref = oracle.osc_forward(X, G, Lo, K_L, cw, ew, WLr, rows=sel)["Y"]
    _compare(to_np(Y)[sel], to_np(Yf)[sel], ref)
    return ref


@pytest.mark.parametrize("bn", [128, 256])
def test_tiny(oracle, osc, bn):
    c = I.tiny_case()
    _run_osc(oracle, osc, c.X, c.W, 32, c.planted, bn=bn)


@pytest.mark.parametrize("M", [1, 16, 128, 2048])
def test_qkv(oracle, osc, M):
    """The headline shape (M = 2048) and the few-token shapes, every row and every column,
    in the automatic launch configuration (the CTA-pair tile at M = 2048)."""
    c = I.qkv_case(M)
    L = oracle.build_table(c.calib, 32)
    _run_osc(oracle, osc, c.X, c.W, 32, L)


@pytest.mark.parametrize("M, G, table, split", [(2048, 32, True, False), (2048, 16, True, False),
                                                 (130, 64, True, False), (16, 32, True, False),
                                                 (300, 32, False, False), (16, 32, True, True), (5, 16, True, True)])
def test_quantize_linear_matches_the_two_calls(oracle, osc, M, G, table, split):
    """osc_quantize_linear (one call; the product starts reading its weights before the quantize
    ends) against osc_quantize then osc_linear (or, with a workspace, osc_linear_splitk) on the
    same inputs: Q_X, S_X, B, Y and the fp32 accumulator bit for bit, in the CTA-pair (M = 2048),
    single-CTA, ragged and split (M <= 16) configurations, with and without a table; the
    two-call outputs are checked against the oracle elsewhere."""
    c = I.qkv_case(M)
    K, N = c.K, c.N
    L = oracle.build_table(c.calib, G) if table else None
    K_L = I.pad16(oracle.table_count(L)) if table else 0
    Ld = to_dev(L) if table else None
    QW, SW, WL = osc.prepare_weight(to_dev(c.W), G, Ld, K_L)
    Xd = to_dev(c.X)
    ws = None
    if split:
        nbytes = osc.osc_linear_workspace_bytes(M, N, K, K_L)
        assert nbytes > 0
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    QX, SX, B = osc.quantize(Xd, G, Ld, K_L)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    Yf = torch.empty((M, N), dtype=torch.float32, device="cuda")
    if split:
        osc.osc_linear_splitk(QX, SX, B, QW, SW, WL, M, N, K, G, K_L, Y, ws, Yf)
    else:
        osc.osc_linear(QX, SX, B, QW, SW, WL, M, N, K, G, K_L, Y, Yf)
    QX2, SX2, B2 = osc.alloc_quantize_outputs(M, K, G, K_L, "cuda")
    Y2 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    Yf2 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    Y3 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    osc.osc_quantize_linear(Xd, G, Ld, K_L, QX2, SX2, B2, QW, SW, WL, N, Y2, Yf2, workspace=ws)
    osc.osc_quantize_linear(Xd, G, Ld, K_L, QX2, SX2, B2, QW, SW, WL, N, Y3, workspace=ws)
    torch.cuda.synchronize()
    assert osc.osc_status() == (0, 0)
    assert torch.equal(QX2, QX) and torch.equal(SX2, SX)
    if K_L:
        assert torch.equal(B2, B)
    assert torch.equal(Y2.view(torch.int16), Y.view(torch.int16))
    assert torch.equal(Y3.view(torch.int16), Y.view(torch.int16))
    assert torch.equal(Yf2, Yf)


@pytest.mark.parametrize("G", [16, 64])
def test_qkv_group_sizes_full_size(oracle, osc, G):
    """The QKV shape at G = 16 and 64 in the launch configuration the bench times (automatic
    tile and CTA grouping), table by Algorithm 1 for that G."""
    c = I.qkv_case(2048)
    L = oracle.build_table(c.calib, G)
    _run_osc(oracle, osc, c.X, c.W, G, L, rows=I.block_rows(2048, seed=G + 1))


def test_qkv_tile_shapes(oracle, osc):
    """128- and 256-wide single-CTA tiles and the 2-CTA 256 x 256 pair tile."""
    c = I.qkv_case(2048)
    L = oracle.build_table(c.calib, 32)
    rows = I.block_rows(2048, seed=5)
    for bn, pair in ((128, 1), (256, 1), (256, 2)):
        _run_osc(oracle, osc, c.X, c.W, 32, L, rows=rows, bn=bn, pair=pair)


@pytest.mark.parametrize("G", [16, 64])
def test_cta_pair_group_sizes(oracle, osc, G):
    c = I.ffn_case(G, M=512, calib_tokens=512)
    L = oracle.build_table(c.calib, G)
    _run_osc(oracle, osc, c.X, c.W[:1024], G, L, rows=I.block_rows(512, seed=G), bn=256, pair=2)


@pytest.mark.parametrize("G", [16, 32, 64])
def test_ffn_full_size(oracle, osc, G):
    c = I.ffn_case(G, M=4096, calib_tokens=1536)
    L = oracle.build_table(c.calib, G)
    _run_osc(oracle, osc, c.X, c.W, G, L, rows=I.block_rows(4096, seed=G))


def test_w2_osc_full_size(oracle, osc):
    c = I.w2_case(M=4096)
    L = oracle.build_table(c.calib, 32)
    _run_osc(oracle, osc, c.X, c.W, 32, L, rows=I.block_rows(4096, seed=7))


@pytest.mark.parametrize("shape,pair", [((4096, 12288, 4096), -1), ((4096, 12288, 4096), 1), ((130, 512, 144), 1),
                                        ((130, 512, 256), 2), ((1, 256, 16), -1), ((2048, 4096, 6144), -1)])
def test_fp8_fallback(oracle, osc, shape, pair):
    """The MXFP8 path: the W2 fallback at full size, small ragged shapes, and the QKV shape
    (the W8A8 comparator of the OSC page's Table 2)."""
    M, K, N = shape
    if M == 4096:
        c = I.w2_case(M=4096)
        X, W = c.X, c.W
        rows = I.block_rows(M, seed=8)
    elif M == 2048:
        c = I.qkv_case(2048)
        X, W = c.X, c.W
        rows = I.block_rows(M, seed=9)
    else:
        rng = np.random.default_rng(M)
        X = I.bf16_bits(rng.standard_normal((M, K)) * np.exp2(rng.integers(-6, 6, (M, 1))))
        W = I.gen_weights(N, K, seed=N)
        rows = None
    Xd, Wd = to_dev(X), to_dev(W)
    QX, SX, _ = osc.alloc_quantize_outputs(M, K, 32, 0, fp8=True)
    QW, SW, _ = osc.alloc_quantize_outputs(N, K, 32, 0, fp8=True)
    osc.osc_quantize_fp8(Xd, QX, SX)
    osc.osc_quantize_fp8(Wd, QW, SW)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    Yf = torch.empty((M, N), dtype=torch.float32, device="cuda")
    Y_plain = torch.empty_like(Y)
    prev, prev_bn = osc.osc_set_cta_pair(pair), osc.osc_set_tile_n(256 if pair == 2 else 0)
    try:
        osc.osc_linear_fp8_fallback(QX, SX, QW, SW, M, N, K, Y, Yf)
        osc.osc_linear_fp8_fallback(QX, SX, QW, SW, M, N, K, Y_plain)
        torch.cuda.synchronize()
    finally:
        osc.osc_set_cta_pair(prev)
        osc.osc_set_tile_n(prev_bn)
    assert torch.equal(Y_plain.view(torch.int16), Y.view(torch.int16))   # launch without Yf32
    sel = np.arange(M) if rows is None else rows
    ref = oracle.fp8_forward(X[sel], W)["Y"]
    _compare(to_np(Y)[sel], to_np(Yf)[sel], ref)


@pytest.mark.parametrize("bn,pair", [(128, 1), (256, 1), (256, 2)])
def test_ragged_shapes_and_compensation_width(oracle, osc, bn, pair):
    """M not a multiple of 128, N not a multiple of the tile, two compensation stages with a
    partial second one (K_L = 80), entries at channel 0 and G-1."""
    rng = np.random.default_rng(21)
    M, K, N, G = 130, 2304, 400, 32
    x = rng.standard_normal((M, K))
    L = np.full(K // G, -1, np.int8)
    idx = rng.permutation(K // G)[:70]
    L[idx] = rng.integers(0, G, size=70)
    L[idx[0]], L[idx[1]] = 0, G - 1
    for k, j in enumerate(L):
        if j >= 0:
            x[:, k * G + int(j)] = rng.choice([-1, 1], M) * rng.uniform(20, 80, M)
    X = I.bf16_bits(x)
    W = I.gen_weights(N, K, seed=3)
    _run_osc(oracle, osc, X, W, G, L, bn=bn, pair=pair)


def test_all_minus_one_table_is_mxfp4_direct(oracle, osc):
    c = I.qkv_case(128)
    L = np.full(128, -1, np.int8)
    _run_osc(oracle, osc, c.X, c.W[:512], 32, L)
    _run_osc(oracle, osc, c.X, c.W[:512], 32, None)


def _moe(oracle, osc, counts, which="gateup", block_sample=False, R=1):
    case = I.moe_case(which, E=len(counts), counts_override=counts) if counts is not None else I.moe_case(which)
    K, N, G = case.K, case.N, 32
    counts, E = case.counts, case.E
    tables = np.stack([oracle.build_table(case.calib[e], G) if case.calib[e].shape[0] else
                       np.full(K // G, -1, np.int8) for e in range(E)])
    if R > 1:                                  # slot 1: a second channel in a third of the used groups
        rng = np.random.default_rng(77)
        second = np.full(tables.shape, -1, np.int8)
        for e in range(E):
            for k in np.nonzero(tables[e] >= 0)[0][::3]:
                second[e, k] = (int(tables[e, k]) + 1 + int(rng.integers(0, G - 1))) % G
        tables = np.stack([tables, second] + [np.full(tables.shape, -1, np.int8)] * (R - 2), axis=-1)
    kls = np.array([I.pad16(oracle.table_count(tables[e])) for e in range(E)], np.int32)
    K_L = max(16, int(kls.max()))
    off, poff, mbe = osc.osc_grouped_plan(counts)
    Mp = int(poff[-1])
    offd, poffd, mbed = off.cuda(), poff.cuda(), mbe.cuda()
    Ld = to_dev(tables)
    QX = torch.empty((Mp, K // 2), dtype=torch.uint8, device="cuda")
    SX = torch.empty(osc.osc_scale_bytes(Mp, K, G), dtype=torch.uint8, device="cuda")
    B = torch.empty((Mp, K_L), dtype=torch.int16, device="cuda")
    osc.osc_quantize_grouped(to_dev(case.X), E, offd, poffd, mbed, Mp, G, Ld, K_L, QX, SX, B)
    sw = osc.osc_scale_bytes(N, K, G)
    QW = torch.empty((E, N, K // 2), dtype=torch.uint8, device="cuda")
    SW = torch.empty((E, sw), dtype=torch.uint8, device="cuda")
    WL = torch.empty((E, N, K_L), dtype=torch.int16, device="cuda")
    Wd = to_dev(case.W)
    for e in range(E):
        osc.osc_prepare_weight(Wd[e], G, Ld[e], K_L, QW[e], SW[e], WL[e])
    Y = torch.empty((Mp, N), dtype=torch.bfloat16, device="cuda")
    Yf = torch.empty((Mp, N), dtype=torch.float32, device="cuda")
    kld = to_dev(kls)
    osc.osc_linear_grouped(QX, SX, B, QW, SW, WL, mbed, kld, E, Mp, N, K, G, K_L, Y, Yf)
    Y_plain = torch.empty_like(Y)
    osc.osc_linear_grouped(QX, SX, B, QW, SW, WL, mbed, kld, E, Mp, N, K, G, K_L, Y_plain)
    torch.cuda.synchronize()
    assert osc.osc_status() == (0, 0)
    assert torch.equal(Y_plain.view(torch.int16), Y.view(torch.int16))   # launch without Yf32
    Yn, Yfn = to_np(Y), to_np(Yf)
    off_n, poff_n = off.numpy(), poff.numpy()
    for e in range(E):
        cnt = int(counts[e])
        # padding rows of the expert's last block come out as zeros
        pad = slice(poff_n[e] + cnt, poff_n[e + 1])
        assert np.all(Yfn[pad] == 0)
        if cnt == 0:
            continue
        Xe = case.X[off_n[e]:off_n[e + 1]]
        # every 128-row block of every expert: its first, last and one seeded row
        sel = I.block_rows(cnt, seed=e) if block_sample else np.arange(cnt)
        cw, ew, WLr = oracle.osc_prepare_weight(case.W[e], G, tables[e], K_L)
        ref = oracle.osc_forward(Xe, G, tables[e], K_L, cw, ew, WLr, rows=sel)["Y"]
        _compare(Yn[poff_n[e] + sel], Yfn[poff_n[e] + sel], ref)


def test_moe_grouped_small(oracle, osc):
    _moe(oracle, osc, [130, 0, 1, 257, 64, 3, 128, 40])


def test_moe_grouped_small_down(oracle, osc):
    """The down projection of the expert layer (K = 768: three k-stages, 24 groups)."""
    _moe(oracle, osc, [130, 0, 1, 257, 64, 3, 128, 40], "down")


def test_moe_grouped_full_size_gateup(oracle, osc):
    _moe(oracle, osc, None, "gateup", block_sample=True)


def test_moe_grouped_full_size_down(oracle, osc):
    _moe(oracle, osc, None, "down", block_sample=True)


def _prep(osc, X, W, G, L, K_L):
    Ld = to_dev(L) if L is not None else None
    QW, SW, WL = osc.prepare_weight(to_dev(W), G, Ld, K_L)
    QX, SX, B = osc.quantize(to_dev(X), G, Ld, K_L)
    return QX, SX, B, QW, SW, WL


def _split_and_plain(oracle, osc, X, W, G, L, K_L):
    """osc_linear_splitk with its workspace (at M <= 16: K split over several SMs, partials added
    by the chained reduction; above that no split applies and it runs as osc_linear) and
    osc_linear (one part per weight tile), each launched with and without the fp32 output; both
    against the oracle on every row and column."""
    M, K = X.shape
    N = W.shape[0]
    QX, SX, B, QW, SW, WL = _prep(osc, X, W, G, L, K_L)
    nbytes = osc.osc_linear_workspace_bytes(M, N, K, K_L)
    if M <= 16:
        assert nbytes > 0 and nbytes % (4 * M * N) == 0            # S >= 2 parts of M x N fp32
    else:
        assert nbytes == 0                                         # no split above 16 rows
    ws = torch.empty(max(4, nbytes) // 4, dtype=torch.float32, device="cuda")
    Y = [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    Yf = [torch.empty((M, N), dtype=torch.float32, device="cuda") for _ in range(2)]
    osc.osc_linear_splitk(QX, SX, B, QW, SW, WL, M, N, K, G, K_L, Y[0], ws, Yf[0])
    osc.osc_linear_splitk(QX, SX, B, QW, SW, WL, M, N, K, G, K_L, Y[1], ws)
    osc.osc_linear(QX, SX, B, QW, SW, WL, M, N, K, G, K_L, Y[2], Yf[1])
    osc.osc_linear(QX, SX, B, QW, SW, WL, M, N, K, G, K_L, Y[3])
    torch.cuda.synchronize()
    assert osc.osc_status() == (0, 0)
    assert torch.equal(Y[1].view(torch.int16), Y[0].view(torch.int16))
    assert torch.equal(Y[3].view(torch.int16), Y[2].view(torch.int16))
    Lo = L if L is not None else np.full(K // G, -1, np.int8)
    cw, ew, WLr = oracle.osc_prepare_weight(W, G, Lo, K_L)
    ref = oracle.osc_forward(X, G, Lo, K_L, cw, ew, WLr)["Y"]
    _compare(to_np(Y[0]), to_np(Yf[0]), ref)
    _compare(to_np(Y[2]), to_np(Yf[1]), ref)
    return QX, SX, B, QW, SW, WL


@pytest.mark.parametrize("M", [1, 5, 16, 33, 64, 100, 128])
def test_few_rows_qkv(oracle, osc, M):
    """Few token rows at the QKV shape: the split product at M <= 16 (ragged M inside its 16-row
    token tile, the compensation stages dealt out with the FP4 ones), the general kernel's
    128-row tile at 33 .. 128 rows."""
    c = I.qkv_case(M)
    L = oracle.build_table(c.calib, 32)
    _split_and_plain(oracle, osc, c.X, c.W, 32, L, I.pad16(oracle.table_count(L)))


@pytest.mark.parametrize("G", [16, 64])
def test_few_rows_group_sizes(oracle, osc, G):
    c = I.qkv_case(16)
    L = oracle.build_table(c.calib, G)
    _split_and_plain(oracle, osc, c.X, c.W, G, L, I.pad16(oracle.table_count(L)))


def test_few_rows_ragged_and_small_workspace(oracle, osc):
    """A partial last weight tile (N = 400), two compensation stages with a partial one
    (K_L = 80), table channels 0 and G-1; then a workspace one byte too small, which must give
    the one-part result bit for bit."""
    rng = np.random.default_rng(31)
    M, K, N, G = 7, 2304, 400, 32
    x = rng.standard_normal((M, K))
    L = np.full(K // G, -1, np.int8)
    idx = rng.permutation(K // G)[:70]
    L[idx] = rng.integers(0, G, size=70)
    L[idx[0]], L[idx[1]] = 0, G - 1
    for k, j in enumerate(L):
        if j >= 0:
            x[:, k * G + int(j)] = rng.choice([-1, 1], M) * rng.uniform(20, 80, M)
    X = I.bf16_bits(x)
    W = I.gen_weights(N, K, seed=3)
    K_L = 80
    QX, SX, B, QW, SW, WL = _split_and_plain(oracle, osc, X, W, G, L, K_L)
    nbytes = osc.osc_linear_workspace_bytes(M, N, K, K_L)
    small = torch.empty(nbytes - 1, dtype=torch.uint8, device="cuda")
    Ya = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    Yb = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    osc.osc_linear_splitk(QX, SX, B, QW, SW, WL, M, N, K, G, K_L, Ya, small)
    osc.osc_linear(QX, SX, B, QW, SW, WL, M, N, K, G, K_L, Yb)
    torch.cuda.synchronize()
    assert torch.equal(Ya.view(torch.int16), Yb.view(torch.int16))


def test_few_rows_fp8_fallback(oracle, osc):
    """The MXFP8 product at few token rows (K = 12288, the W2 shape, 16 rows)."""
    c = I.w2_case(M=16)
    M, K, N = 16, 12288, 4096
    QX, SX, _ = osc.alloc_quantize_outputs(M, K, 32, 0, fp8=True)
    QW, SW, _ = osc.alloc_quantize_outputs(N, K, 32, 0, fp8=True)
    osc.osc_quantize_fp8(to_dev(c.X), QX, SX)
    osc.osc_quantize_fp8(to_dev(c.W), QW, SW)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    Yf = torch.empty((M, N), dtype=torch.float32, device="cuda")
    osc.osc_linear_fp8_fallback(QX, SX, QW, SW, M, N, K, Y, Yf)
    torch.cuda.synchronize()
    assert osc.osc_status() == (0, 0)
    _compare(to_np(Y), to_np(Yf), oracle.fp8_forward(c.X, c.W)["Y"])


# ---- several protected channels per group ---------------------------------------------------

@pytest.mark.parametrize("M", [256, 2048])
def test_multi_table_product(oracle, osc, M):
    """The dual-path product with a two-slot table (second outliers of the two-outlier
    workload on the 16-bit path): every row at M = 256, every 128-row block at M = 2048 in the
    CTA-pair configuration."""
    c = I.two_outlier_case(M)
    L = oracle.build_table_multi(c.calib, 32, 2)
    rows = None if M <= 256 else I.block_rows(M, seed=M)
    _run_osc(oracle, osc, c.X, c.W, 32, L, rows=rows)


def test_multi_table_few_rows(oracle, osc):
    c = I.two_outlier_case(16)
    L = oracle.build_table_multi(c.calib, 32, 2)
    _split_and_plain(oracle, osc, c.X, c.W, 32, L, I.pad16(oracle.table_count(L)))


def test_moe_grouped_multi_table(oracle, osc):
    """Grouped form with two-slot expert tables: the Algorithm 1 entry in slot 0 and, in a
    third of the groups that have one, a second channel in slot 1."""
    _moe(oracle, osc, [130, 0, 1, 257, 64, 3, 128, 40], R=2)
