"""GPU parity of the quantize side (osc_quantize, osc_quantize_fp8, osc_prepare_weight,
osc_build_table) against the oracle: codes, scales, B, W_L and table entries bit-exact, on
every row of every workload."""
import numpy as np
import pytest
import torch

from tests._layout import pad_rows_zero, unpack_e2m1, unswizzle_scales
from tests.conftest import to_dev, to_np
from w4a4_outlier_separated_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _gpu_quant(osc, X, G, L, K_L):
    M, K = X.shape
    Ld = to_dev(L) if L is not None else None
    QX, SX, B = osc.quantize(to_dev(X), G, Ld, K_L)
    torch.cuda.synchronize()
    assert osc.osc_status() == (0, 0)
    return to_np(QX), to_np(SX), (to_np(B) if B is not None else None)


def _check_quant(oracle, osc, X, G, L, K_L, rows=None):
    M, K = X.shape
    QX, SX, B = _gpu_quant(osc, X, G, L, K_L)
    V = 16 if G == 16 else 32
    codes = unpack_e2m1(QX, K)
    exps = unswizzle_scales(SX, M, K, V)
    assert pad_rows_zero(SX, M, K, V)
    sel = np.arange(M) if rows is None else np.asarray(rows)
    Xs = X[sel]
    if L is not None:
        Xz, Bref = oracle.extract(Xs, G, L, K_L)
        if K_L:
            assert np.array_equal(B[sel], Bref)
    else:
        Xz = Xs
    cref, eref = oracle.mx_quantize(Xz, G)
    bad = np.argwhere(codes[sel] != cref)
    assert bad.size == 0, f"{len(bad)} code mismatches, first {bad[:4]}"
    assert np.array_equal(exps[sel], eref)


def _anchor_rows(anchor, vals, K=256):
    per = 31
    n = len(vals)
    nb = (n + per - 1) // per
    nb = (nb + K // 32 - 1) // (K // 32) * (K // 32)
    pad = np.zeros(nb * per, dtype=np.uint16)
    pad[:n] = vals
    blocks = np.concatenate([np.full((nb, 1), anchor, np.uint16), pad.reshape(nb, per)], axis=1)
    return blocks.reshape(-1, K)


def _finite_bf16():
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    return b[(b & 0x7F80) != 0x7F80]


@pytest.mark.parametrize("shift", [0, 10, -60, -126, 100])
def test_every_bf16_value_e2m1(oracle, osc, shift):
    """All finite bf16 values under a block anchor: the hardware conversion, the exponent
    from the bf16 bits and the zero-sign rule agree with the oracle bit for bit."""
    anchor = I.bf16_bits(np.array([7.5 * 2.0 ** shift]))[0]
    b = _finite_bf16()
    f = I.bf16_to_f32(b).astype(np.float64)
    X = _anchor_rows(anchor, b[np.abs(f) <= 7.5 * 2.0 ** shift])
    _check_quant(oracle, osc, X, 32, None, 0)


@pytest.mark.parametrize("G", [16, 64])
def test_every_bf16_value_other_groups(oracle, osc, G):
    b = _finite_bf16()
    rng = np.random.default_rng(G)
    X = rng.permutation(b)[: (len(b) // 256) * 256].reshape(-1, 256)
    _check_quant(oracle, osc, X, G, None, 0)


@pytest.mark.parametrize("shift", [0, 7, -50, -120])
def test_every_bf16_value_e4m3(oracle, osc, shift):
    anchor = I.bf16_bits(np.array([480.0 * 2.0 ** shift]))[0]
    b = _finite_bf16()
    f = I.bf16_to_f32(b).astype(np.float64)
    X = _anchor_rows(anchor, b[np.abs(f) <= 480.0 * 2.0 ** shift])
    M, K = X.shape
    QX8, SX, _ = osc.alloc_quantize_outputs(M, K, 32, 0, fp8=True)
    osc.osc_quantize_fp8(to_dev(X), QX8, SX)
    torch.cuda.synchronize()
    cref, eref = oracle.mx_quantize(X, 32, oracle.FMT_E4M3)
    assert np.array_equal(to_np(QX8), cref)
    assert np.array_equal(unswizzle_scales(to_np(SX), M, K, 32), eref)


def test_tiny_planted(oracle, osc):
    c = I.tiny_case()
    _check_quant(oracle, osc, c.X, 32, c.planted, 16)


@pytest.mark.parametrize("M", [1, 16, 128, 2048])
def test_qkv_table_from_algorithm1(oracle, osc, M):
    c = I.qkv_case(M)
    L = oracle.build_table(c.calib, 32)
    K_L = I.pad16(oracle.table_count(L))
    assert K_L == 96
    _check_quant(oracle, osc, c.X, 32, L, K_L)


@pytest.mark.parametrize("G", [16, 32, 64])
def test_ffn_group_sizes_full_size(oracle, osc, G):
    c = I.ffn_case(G, M=4096, calib_tokens=1536)
    L = oracle.build_table(c.calib, G)
    K_L = I.pad16(oracle.table_count(L))
    _check_quant(oracle, osc, c.X, G, L, K_L)                # every row


def test_w2_osc_and_fp8_full_size(oracle, osc):
    c = I.w2_case(M=4096)
    L = oracle.build_table(c.calib, 32)
    K_L = I.pad16(oracle.table_count(L))
    _check_quant(oracle, osc, c.X, 32, L, K_L)               # every row
    QX8, SX, _ = osc.alloc_quantize_outputs(4096, 12288, 32, 0, fp8=True)
    osc.osc_quantize_fp8(to_dev(c.X), QX8, SX)
    torch.cuda.synchronize()
    cref, eref = oracle.mx_quantize(c.X, 32, oracle.FMT_E4M3)
    assert np.array_equal(to_np(QX8), cref)
    assert np.array_equal(unswizzle_scales(to_np(SX), 4096, 12288, 32), eref)


def test_edge_cases(oracle, osc):
    rng = np.random.default_rng(3)
    # ragged M, all-zero rows, negative zeros, K_L larger than the entry count, j* = 0 and G-1
    M, K, G = 130, 512, 32
    x = rng.standard_normal((M, K)) * 3
    x[5] = 0.0
    x[6] = -0.0
    X = I.bf16_bits(x)
    L = np.full(K // G, -1, np.int8)
    L[[0, 3, 15]] = [0, 31, 7]
    _check_quant(oracle, osc, X, G, L, 48)
    # all -1 table with K_L = 0, and no table at all
    _check_quant(oracle, osc, X, G, np.full(K // G, -1, np.int8), 0)
    _check_quant(oracle, osc, X, G, None, 0)
    # M = 0 is a no-op
    QX, SX, B = osc.alloc_quantize_outputs(0, K, G, 16)
    osc.osc_quantize(torch.zeros((0, K), dtype=torch.int16, device="cuda"), G, to_dev(L), 16, QX, SX, B)


def test_bad_table_is_reported_not_faulted(osc):
    X = to_dev(I.bf16_bits(np.ones((4, 256))))
    L = np.full(8, -1, np.int8)
    L[2] = 40                                   # >= G
    QX, SX, B = osc.quantize(X, 32, to_dev(L), 16)
    torch.cuda.synchronize()
    code, raw = osc.osc_status()
    assert code == -6 and raw == 2
    assert osc.osc_status() == (0, 0)           # cleared


def test_argument_errors(osc):
    X = torch.zeros((4, 256), dtype=torch.int16, device="cuda")
    QX, SX, B = osc.alloc_quantize_outputs(4, 256, 32, 16)
    with pytest.raises(osc.OSCError) as e:
        osc.osc_quantize(X, 24, None, 0, QX, SX, None)
    assert e.value.code == -3
    Xb = torch.zeros((4, 200), dtype=torch.int16, device="cuda")
    with pytest.raises(osc.OSCError) as e:
        osc.osc_quantize(Xb, 32, None, 0, QX, SX, None)
    assert e.value.code == -2


def test_prepare_weight(oracle, osc):
    c = I.qkv_case(1)
    L = c.planted
    K_L = I.pad16(oracle.table_count(L))
    QW, SW, WL = osc.prepare_weight(to_dev(c.W), 32, to_dev(L), K_L)
    torch.cuda.synchronize()
    cw, ew, WLr = oracle.osc_prepare_weight(c.W, 32, L, K_L)
    assert np.array_equal(unpack_e2m1(to_np(QW), 4096), cw)
    assert np.array_equal(unswizzle_scales(to_np(SW), 6144, 4096, 32), ew)
    assert np.array_equal(to_np(WL), WLr)


@pytest.mark.parametrize("case,G,alpha,min_hits", [
    ("qkv", 32, 5.0, 5), ("w2", 32, 5.0, 5), ("ffn", 16, 5.0, 5), ("ffn", 64, 5.0, 5),
    ("qkv", 32, 3.0, 2), ("random", 32, 2.5, 3)])
def test_build_table(oracle, osc, case, G, alpha, min_hits):
    if case == "qkv":
        X = I.qkv_case(1).calib
    elif case == "w2":
        X = I.w2_case(M=1).calib
    elif case == "ffn":
        X = I.ffn_case(G, M=1).calib
    else:
        X = I.bf16_bits(np.random.default_rng(9).standard_t(3, size=(700, 1024)))
    S, K = X.shape
    L = torch.empty(K // G, dtype=torch.int8, device="cuda")
    osc.osc_build_table(to_dev(X), G, alpha, min_hits, L)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(L), oracle.build_table(X, G, alpha, min_hits))


@pytest.mark.parametrize("case,G", [("qkv", 32), ("w2", 32), ("ffn", 16), ("ffn", 64), ("random", 32)])
def test_density_and_tier(oracle, osc, case, G):
    """§2.2 density on the GPU: per-group event and hit counts equal the oracle's, for a table
    built from calibration tokens and evaluated on other tokens; the tier chosen from the GPU
    counts is the one chosen from the oracle's."""
    if case == "qkv":
        c = I.qkv_case(512)
        X, L = c.X, oracle.build_table(c.calib, G)
    elif case == "w2":
        c = I.w2_case(M=512)
        X, L = c.X, oracle.build_table(c.calib, G)
    elif case == "ffn":
        c = I.ffn_case(G, M=512)
        X, L = c.X, oracle.build_table(c.calib, G)
    else:
        rng = np.random.default_rng(17)
        X = I.bf16_bits(rng.standard_t(3, size=(600, 1024)))
        L = rng.integers(-1, G, size=1024 // G).astype(np.int8)
        L[0], L[1], L[2] = 0, G - 1, -1
    S, K = X.shape
    nh = torch.empty(K // G, dtype=torch.int32, device="cuda")
    nt = torch.empty(K // G, dtype=torch.int32, device="cuda")
    osc.osc_density(to_dev(X), G, 5.0, to_dev(L), nh, nt)
    torch.cuda.synchronize()
    assert osc.osc_status() == (0, 0)
    rh, rt = oracle.density(X, G, L, 5.0)
    assert np.array_equal(to_np(nh), rh) and np.array_equal(to_np(nt), rt)
    (tg, cg), (tr, cr) = osc.osc_select_tier(to_np(nh), to_np(nt)), osc.osc_select_tier(rh, rt)
    assert tg == tr and (cg == cr or (np.isnan(cg) and np.isnan(cr)))


def test_density_bad_table_entry_is_reported(osc):
    X = to_dev(I.bf16_bits(np.random.default_rng(2).standard_normal((64, 256)) * 3))
    L = np.full(8, -1, np.int8)
    L[5] = 33                                   # >= G
    nh = torch.empty(8, dtype=torch.int32, device="cuda")
    nt = torch.empty(8, dtype=torch.int32, device="cuda")
    osc.osc_density(X, 32, 5.0, to_dev(L), nh, nt)
    torch.cuda.synchronize()
    assert osc.osc_status() == (-6, 2)
    assert to_np(nh)[5] == 0


def _gamma(K, seed):
    return I.bf16_bits(1.0 + 0.1 * np.random.default_rng(seed).standard_normal(K))


def _check_rmsnorm_quant(oracle, osc, X, gamma, eps, G, L, K_L):
    """osc_rmsnorm_quantize against the oracle's RMSNorm followed by extraction and
    microscaling: codes, scales (pad rows zero) and B bit for bit, every row."""
    M, K = X.shape
    Ld = to_dev(L) if L is not None else None
    QX, SX, B = osc.rmsnorm_quantize(to_dev(X), to_dev(gamma), eps, G, Ld, K_L)
    torch.cuda.synchronize()
    assert osc.osc_status() == (0, 0)
    Xn, _ = oracle.rmsnorm(X, gamma, eps)
    V = 16 if G == 16 else 32
    SXn = to_np(SX)
    assert pad_rows_zero(SXn, M, K, V)
    if L is not None:
        Xz, Bref = oracle.extract(Xn, G, L, K_L)
        if K_L:
            assert np.array_equal(to_np(B), Bref)
    else:
        Xz = Xn
    cref, eref = oracle.mx_quantize(Xz, G)
    codes = unpack_e2m1(to_np(QX), K)
    bad = np.argwhere(codes != cref)
    assert bad.size == 0, f"{len(bad)} code mismatches, first {bad[:4]}"
    assert np.array_equal(unswizzle_scales(SXn, M, K, V), eref)


@pytest.mark.parametrize("M", [1, 16, 130, 2048])
def test_rmsnorm_quantize_qkv(oracle, osc, M):
    """The fused input side at the QKV shape (K = 4096, G = 32), table by Algorithm 1 on
    calibration rows normalized the same way."""
    c = I.qkv_case(M)
    gamma = _gamma(4096, 1)
    L = oracle.build_table(oracle.rmsnorm(c.calib, gamma, 1e-6)[0], 32)
    K_L = I.pad16(oracle.table_count(L))
    _check_rmsnorm_quant(oracle, osc, c.X, gamma, 1e-6, 32, L, K_L)


@pytest.mark.parametrize("M, G", [(2048, 32), (130, 64)])
def test_rmsnorm_quantize_linear_matches_the_two_calls(oracle, osc, M, G):
    """osc_rmsnorm_quantize_linear (one call; the product may read its weights before the fused
    quantize ends) against osc_rmsnorm_quantize then osc_linear: Q_X, S_X, B, Y and the fp32
    accumulator bit for bit (the two-call outputs are checked against the oracle elsewhere)."""
    c = I.qkv_case(M)
    K, N = c.K, c.N
    gamma = _gamma(K, G)
    L = oracle.build_table(oracle.rmsnorm(c.calib[:512], gamma, 1e-6)[0], G)
    K_L = I.pad16(oracle.table_count(L))
    Ld, gd, Xd = to_dev(L), to_dev(gamma), to_dev(c.X)
    QW, SW, WL = osc.prepare_weight(to_dev(c.W), G, Ld, K_L)
    QX, SX, B = osc.rmsnorm_quantize(Xd, gd, 1e-6, G, Ld, K_L)
    Y, Yf = osc.linear(QX, SX, B, QW, SW, WL, M, N, K, G, K_L, want_f32=True)
    QX2, SX2, B2 = osc.alloc_quantize_outputs(M, K, G, K_L, "cuda")
    Y2 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    Yf2 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    osc.osc_rmsnorm_quantize_linear(Xd, gd, 1e-6, G, Ld, K_L, QX2, SX2, B2, QW, SW, WL, N, Y2, Yf2)
    torch.cuda.synchronize()
    assert osc.osc_status() == (0, 0)
    assert torch.equal(QX2, QX) and torch.equal(SX2, SX) and torch.equal(B2, B)
    assert torch.equal(Y2.view(torch.int16), Y.view(torch.int16))
    assert torch.equal(Yf2, Yf)


@pytest.mark.parametrize("G", [16, 64])
def test_rmsnorm_quantize_group_sizes(oracle, osc, G):
    c = I.qkv_case(256)
    gamma = _gamma(4096, G)
    L = oracle.build_table(oracle.rmsnorm(c.calib[:512], gamma, 1e-6)[0], G)
    _check_rmsnorm_quant(oracle, osc, c.X, gamma, 1e-6, G, L, I.pad16(oracle.table_count(L)))


@pytest.mark.parametrize("K", [256, 768, 1280, 2048, 6144])
def test_rmsnorm_quantize_row_lengths(oracle, osc, K):
    """Rows of 8 to 192 blocks: fewer blocks than lanes (K = 256, 768), a block count that is
    not a power of two (1280, 6144: partial last pass of the lanes), and the largest K."""
    rng = np.random.default_rng(K)
    M, G = 130, 32
    x = rng.standard_normal((M, K)) * np.exp2(rng.integers(-8, 8, (M, 1)))
    L = np.full(K // G, -1, np.int8)
    idx = rng.permutation(K // G)[: max(1, K // G // 2)]
    L[idx] = rng.integers(0, G, idx.size)
    for k, j in enumerate(L):
        if j >= 0:
            x[:, k * G + int(j)] *= 40.0
    X = I.bf16_bits(x)
    _check_rmsnorm_quant(oracle, osc, X, _gamma(K, K + 1), 1e-5, G, L, I.pad16(oracle.table_count(L)))


def test_rmsnorm_quantize_edge_rows(oracle, osc):
    """All-zero and negative-zero rows (eps > 0 keeps their scale finite), a constant row, rows
    whose squares overflow or underflow fp32 (both sides follow IEEE fp32: an infinite sum
    gives inv = 0), a negative and a zero gamma entry; with and without a table."""
    rng = np.random.default_rng(8)
    M, K = 9, 512
    x = rng.standard_normal((M, K))
    x[0] = 0.0
    x[1] = -0.0
    x[2] = 3.0
    x[3] *= 2.0 ** 100                                        # squares overflow fp32: inv = 0
    x[4] *= 2.0 ** -100                                       # squares underflow: eps decides
    x[5] *= 2.0 ** 50
    X = I.bf16_bits(x)
    gamma = _gamma(K, 3)
    gamma[7] = I.bf16_bits(np.array([-1.5]))[0]
    gamma[9] = 0
    _check_rmsnorm_quant(oracle, osc, X, gamma, 1e-6, 32, None, 0)
    L = np.full(K // 32, -1, np.int8)
    L[[0, 7, 15]] = [0, 31, 9]
    _check_rmsnorm_quant(oracle, osc, X, gamma, 1e-6, 32, L, 16)


# ---- several protected channels per group ---------------------------------------------------

@pytest.mark.parametrize("G,R", [(32, 2), (32, 3), (16, 2), (64, 3)])
def test_multi_table_build_and_quantize(oracle, osc, G, R):
    """Up to R channels per group: the GPU build (R rounds, earlier channels read as zero)
    equals the oracle's table, and the quantize moves every entry out in (group, slot) order:
    codes, scales and B bit for bit on every row."""
    c = I.two_outlier_case(512)
    Lref = oracle.build_table_multi(c.calib, G, R)
    Ld = torch.empty((4096 // G, R), dtype=torch.int8, device="cuda")
    osc.osc_build_table_multi(to_dev(c.calib), G, 5.0, 5, R, Ld)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(Ld), Lref)
    assert (Lref[:, 1] >= 0).sum() > 10                        # second slots are in use
    _check_quant(oracle, osc, c.X, G, Lref, I.pad16(oracle.table_count(Lref)))


def test_multi_table_hand_made_entries(oracle, osc):
    """A hand-made 3-slot table with a repeated channel, channels 0 and G-1 and a group whose
    later slot is set while an earlier one is not: the GPU follows the table order exactly
    (the repeated channel's second B column is 0). Also W_L of the same table."""
    rng = np.random.default_rng(41)
    M, K, G, R = 130, 512, 32, 3
    X = I.bf16_bits(rng.standard_normal((M, K)) * 4)
    L = np.full((K // G, R), -1, np.int8)
    L[0] = [4, 9, 4]
    L[3] = [0, 31, -1]
    L[7] = [-1, 12, -1]
    L[15] = [30, 2, 17]
    K_L = 16
    _check_quant(oracle, osc, X, G, L, K_L)
    W = I.gen_weights(96, K, seed=41)
    _, _, WL = osc.prepare_weight(to_dev(W), G, to_dev(L), K_L)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(WL), oracle.gather_wl(W, G, L, K_L))


@pytest.mark.parametrize("G", [32, 64])
def test_multi_table_rmsnorm_quantize(oracle, osc, G):
    c = I.two_outlier_case(256)
    gamma = _gamma(4096, 7)
    L = oracle.build_table_multi(oracle.rmsnorm(c.calib[:512], gamma, 1e-6)[0], G, 2)
    _check_rmsnorm_quant(oracle, osc, c.X, gamma, 1e-6, G, L, I.pad16(oracle.table_count(L)))
