"""Pins for the oracle: each check ties it to something other than itself.

Sources: the OSC page ("W4A4量化技术：OSC框架如何实现高效LLM部署", coreui.cn/article/2607942.html)
for the method (§2.2 density, §2.3 tiers, §3.1 Algorithm 1, §3.2 extraction, microscaling and the
dual-path equation), the OCP MX v1.0 element formats that the path names (E2M1, E4M3, E8M0), and
mathematics: brute-force nearest-value rounding, closed-form thresholds, library matmul on
dequantized values, exact-representability identities.
"""
import os

import numpy as np
import pytest

from w4a4_outlier_separated_b200 import inputs as I

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _read_table(name):
    rows = []
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append(line.split())
    return rows


def _all_finite_bf16():
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    return b[(b & 0x7F80) != 0x7F80]


# ---- element formats ------------------------------------------------------------------

def test_e2m1_code_table_and_counts(oracle):
    rows = _read_table("e2m1_code_table.txt")
    assert len(rows) == 16 == 2 ** 4                      # 4-bit code: 16 values
    for code_s, val_s in rows:
        v = oracle.decode_e2m1(int(code_s, 16))
        assert v == float(val_s) and np.signbit(v) == val_s.startswith("-")
    mags = sorted({abs(oracle.decode_e2m1(c)) for c in range(16)})
    assert len(mags) == 8 == 2 ** 3                       # 3 magnitude bits: 8 levels
    assert len({oracle.decode_e2m1(c) for c in range(16)}) == 15   # +0 == -0


def _nearest_even(a, table_vals, table_codes, mant_mask):
    """Brute force: the nearest representable magnitude; on a tie, the code with an even mantissa
    (adjacent codes always differ in their lowest mantissa bit)."""
    d = np.abs(a[:, None] - table_vals[None, :])
    cand = d == d.min(axis=1, keepdims=True)
    even = (table_codes & mant_mask) == 0
    score = cand.astype(np.int64) * 2 + (cand & even[None, :])
    return table_codes[np.argmax(score, axis=1)]


def _bruteforce_e2m1(v):
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    codes = np.arange(8)
    a = np.minimum(np.abs(v), 6.0)                # saturation beyond the largest element
    mag = _nearest_even(a, mags, codes, 1)
    return np.where(np.signbit(v), 8, 0) | mag


def _blocks_with_anchor(anchor_bits, vals_bits, per=31):
    n = len(vals_bits)
    nb = (n + per - 1) // per
    pad = np.zeros(nb * per, dtype=np.uint16)
    pad[:n] = vals_bits
    X = np.concatenate([np.full((nb, 1), anchor_bits, np.uint16), pad.reshape(nb, per)], axis=1)
    return X, n


@pytest.mark.parametrize("shift", [0, 10, -60, 100])
def test_e2m1_rounding_matches_bruteforce(oracle, shift):
    """Every finite bf16 value within the anchor's block range, at several scales: the oracle's
    binade-quantum rounding must equal a brute-force nearest search with ties to even."""
    anchor = I.bf16_bits(np.array([7.5 * 2.0 ** shift]))[0]       # floor(log2 7.5) - 2 = 0
    b = _all_finite_bf16()
    f = I.bf16_to_f32(b).astype(np.float64)
    keep = np.abs(f) <= 7.5 * 2.0 ** shift
    vals = b[keep]
    X, n = _blocks_with_anchor(anchor, vals)
    codes, exps = oracle.mx_quantize(X, 32)
    assert np.all(exps == shift)
    got = codes[:, 1:].reshape(-1)[:n]
    v = I.bf16_to_f32(vals).astype(np.float64) / 2.0 ** shift
    want = _bruteforce_e2m1(v)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (v[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_e2m1_known_ties(oracle):
    # ties: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4; saturation 7->6
    v = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, -0.1, -0.25])
    X = I.bf16_bits(np.concatenate([[7.5], v, np.zeros(32 - 1 - len(v))]))[None, :]
    codes, exps = oracle.mx_quantize(X, 32)
    assert exps[0, 0] == 0
    dec = [oracle.decode_e2m1(int(c)) for c in codes[0, 1:1 + len(v)]]
    assert dec[:8] == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0]
    assert codes[0, 9] == 0x8 and codes[0, 10] == 0x8     # negative values rounding to 0 keep the sign


def _e4m3_table():
    codes = np.arange(128)
    E, m = codes >> 3, codes & 7
    vals = np.where(E == 0, m * 2.0 ** -9, (1 + m / 8.0) * 2.0 ** (E - 7.0))
    ok = codes != 0x7F                                     # 0x7F is NaN
    return vals[ok], codes[ok]


def test_e4m3_decode_definition(oracle):
    vals, codes = _e4m3_table()
    for v, c in zip(vals, codes):
        assert oracle.decode_e4m3(int(c)) == v
        assert oracle.decode_e4m3(int(c) | 0x80) == -v
    assert vals.max() == 448.0 and np.isnan(oracle.decode_e4m3(0x7F))


def test_e4m3_spec_points(oracle):
    """The E4M3 decoder against the format's stated characteristic values (golden file), and
    the quantizer at the saturation and subnormal boundaries those values define."""
    rows = _read_table("e4m3_spec_points.txt")
    assert len(rows) == 10
    for r in rows:
        code, want = int(r[0], 16), float(r[1])
        got = oracle.decode_e4m3(code)
        if np.isnan(want):
            assert np.isnan(got)
        else:
            assert got == want and np.signbit(got) == np.signbit(want), (r, got)
    # with e = 0 (block max 480: floor(log2 480) - 8 = 0): 448 stays, 470 saturates to 448,
    # 2^-9 stays, 2^-10 is a tie with 0 (to the even code 0), 3 * 2^-11 rounds up to 2^-9
    v = np.array([480.0, 448.0, 470.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11, -(2.0 ** -10)])
    X = I.bf16_bits(np.concatenate([v, np.zeros(32 - len(v))]))[None, :]
    codes, exps = oracle.mx_quantize(X, 32, oracle.FMT_E4M3)
    assert exps[0, 0] == 0
    assert list(codes[0, :7]) == [0x7E, 0x7E, 0x7E, 0x01, 0x00, 0x01, 0x80]


@pytest.mark.parametrize("shift", [0, 7, -50])
def test_e4m3_rounding_matches_bruteforce(oracle, shift):
    anchor = I.bf16_bits(np.array([480.0 * 2.0 ** shift]))[0]      # floor(log2 480) - 8 = 0
    b = _all_finite_bf16()
    f = I.bf16_to_f32(b).astype(np.float64)
    vals = b[np.abs(f) <= 480.0 * 2.0 ** shift]
    X, n = _blocks_with_anchor(anchor, vals)
    codes, exps = oracle.mx_quantize(X, 32, oracle.FMT_E4M3)
    assert np.all(exps == shift)
    got = codes[:, 1:].reshape(-1)[:n]
    v = I.bf16_to_f32(vals).astype(np.float64) / 2.0 ** shift
    tv, tc = _e4m3_table()
    mag = _nearest_even(np.minimum(np.abs(v), 448.0), tv, tc, 1)
    want = np.where(np.signbit(v), 0x80, 0) | mag
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (v[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_shared_exponent_invariant(oracle):
    rng = np.random.default_rng(5)
    X = I.bf16_bits(rng.standard_normal((64, 256)) * np.exp2(rng.integers(-40, 40, (64, 1))))
    X[3, :32] = 0                                          # all-zero block
    codes, exps = oracle.mx_quantize(X, 32)
    f = I.bf16_to_f32(X).astype(np.float64).reshape(64, 8, 32)
    amax = np.abs(f).max(axis=2)
    e = exps.astype(np.float64)
    nz = amax > 0
    r = amax[nz] * 2.0 ** -e[nz]
    assert np.all((r >= 4) & (r < 8))                      # 4 <= amax * 2^-e < 8
    assert exps[3, 0] == -127
    # fp8: 256 <= amax * 2^-e < 512
    _, e8 = oracle.mx_quantize(X, 32, oracle.FMT_E4M3)
    r8 = amax[nz] * 2.0 ** -e8.astype(np.float64)[nz]
    assert np.all((r8 >= 256) & (r8 < 512))


def test_shared_exponent_clamps_low(oracle):
    tiny = np.array([2.0 ** -130, 2.0 ** -126, 2.0 ** -125], dtype=np.float64)
    X = I.bf16_bits(np.repeat(tiny, 32).reshape(3, 32))
    codes, exps = oracle.mx_quantize(X, 32)
    assert list(exps[:, 0]) == [-127, -127, -127]
    # 2^-125 * 2^127 = 4 -> code 6; 2^-126 -> 2 -> code 4; 2^-130 -> 0.125 -> 0
    assert list(codes[:, 0]) == [0, 4, 6]


def test_group_sizes_share_scales(oracle):
    rng = np.random.default_rng(6)
    X = I.bf16_bits(rng.standard_normal((4, 256)) * np.array([[1], [100], [0.01], [3]]))
    c64, e64 = oracle.mx_quantize(X, 64)
    assert e64.shape == (4, 8) and np.all(e64[:, 0::2] == e64[:, 1::2])
    c32, e32 = oracle.mx_quantize(X, 32)
    assert np.all(e64[:, 0::2] == np.maximum(e32[:, 0::2], e32[:, 1::2]))
    c16, e16 = oracle.mx_quantize(X, 16)
    assert e16.shape == (4, 16)
    assert np.all(e32 == np.maximum(e16[:, 0::2], e16[:, 1::2]))


def test_bf16_rounding_of_doubles(oracle):
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(2000) * np.exp2(rng.integers(-30, 30, 2000))).astype(np.float32)
    want = I.bf16_bits(x)                                   # fp32 -> bf16 by the bit trick
    got = np.array([oracle.double_to_bf16(float(v)) for v in x], dtype=np.uint16)
    assert np.array_equal(got, want)
    assert oracle.double_to_bf16(1.0 + 2.0 ** -8) == 0x3F80   # tie -> even
    assert oracle.double_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82


# ---- Algorithm 1 and the density --------------------------------------------------------

def _group_rows(vals_list, G=32):
    return I.bf16_bits(np.array(vals_list, dtype=np.float64))


def test_table_picks_consistent_channel(oracle):
    rng = np.random.default_rng(8)
    S, G = 40, 32
    X = rng.standard_normal((S, 3 * G)) * 0.5
    X[:, 0 * G + 3] = 100.0                  # group 0: channel 3 on every token
    X[:12, 1 * G + 0] = -90.0                # group 1: channel 0, 12 tokens (j* = 0 is valid)
    X[:3, 2 * G + 7] = 90.0                  # group 2: only 3 events < min_hits
    L = oracle.build_table(I.bf16_bits(X), G, alpha=5.0, min_hits=5)
    assert list(L) == [3, 0, -1]


def test_table_tie_goes_to_lowest_channel(oracle):
    S, G = 20, 32
    X = np.full((S, G), 0.25)
    X[:10, 9] = 50.0
    X[10:, 5] = 50.0
    L = oracle.build_table(I.bf16_bits(X), G, alpha=5.0, min_hits=5)
    assert list(L) == [5]
    X = np.zeros((S, G))                     # all-zero group: no events
    assert list(oracle.build_table(I.bf16_bits(X), G, 5.0, 1)) == [-1]
    X = np.full((S, G), 0.25)                # two channels share the token's maximum:
    X[:, 9] = X[:, 4] = 50.0                 # the event goes to the lower one on every token
    assert list(oracle.build_table(I.bf16_bits(X), G, 5.0, 5)) == [4]
    nh, nt = oracle.density(I.bf16_bits(X), G, np.array([9], np.int8), 5.0)
    assert nt[0] == S and nh[0] == 0


def test_table_min_hits_boundary(oracle):
    """A channel needs at least min_hits events: exactly min_hits qualifies, one fewer does not."""
    S, G = 30, 32
    X = np.full((S, 2 * G), 0.5)
    X[:5, 0 * G + 11] = 60.0                 # group 0: 5 events
    X[:4, 1 * G + 20] = 60.0                 # group 1: 4 events
    Xb = I.bf16_bits(X)
    assert list(oracle.build_table(Xb, G, alpha=5.0, min_hits=5)) == [11, -1]
    assert list(oracle.build_table(Xb, G, alpha=5.0, min_hits=4)) == [11, 20]
    assert list(oracle.build_table(Xb, G, alpha=5.0, min_hits=6)) == [-1, -1]


def test_event_threshold_closed_form(oracle):
    """Group [a, 1 x 31]: an event iff 32 a >= alpha (a + 31), i.e. a >= 31 alpha / (32 - alpha)."""
    alpha, G = 5.0, 32
    thr = 31 * alpha / (G - alpha)           # 5.7407...
    for a, expect in [(5.5, 0), (5.75, 1), (6.0, 1), (5.625, 0)]:
        X = np.ones((6, G))
        X[:, 4] = a
        nh, nt = oracle.density(I.bf16_bits(X), G, np.array([4], np.int8), alpha)
        assert nt[0] == 6 * expect and nh[0] == nt[0], (a, thr)
    # exact equality is an event ("at least alpha times the mean"): [155, 27 x 31] gives
    # 32 * 155 = 4960 = 5 * (155 + 31 * 27), every term exact in bf16 and in the fp32 sum
    for a, b, expect in [(155.0, 27.0, 1), (154.0, 27.0, 0)]:
        X = np.full((6, G), b)
        X[:, 4] = a
        nh, nt = oracle.density(I.bf16_bits(X), G, np.array([4], np.int8), alpha)
        assert nt[0] == 6 * expect, (a, b)
    # alpha + 1 raises the threshold: a = 6 stops being an event at alpha = 6 (thr = 7.15)
    X = np.ones((6, G)); X[:, 4] = 6.0
    assert oracle.density(I.bf16_bits(X), G, np.array([4], np.int8), 6.0)[1][0] == 0


def test_table_recovers_planted_qkv(oracle):
    c = I.qkv_case(1)
    L = oracle.build_table(c.calib, 32, alpha=5.0, min_hits=5)
    assert np.array_equal(L, c.planted)
    assert (L >= 0).sum() == round(0.7 * 128)


def test_density_on_planted_tiny(oracle):
    c = I.tiny_case()
    nh, nt = oracle.density(c.X, 32, c.planted, 5.0)
    planted = c.planted >= 0
    assert np.all(nh[planted] == nt[planted]) and np.all(nt[planted] > 0)   # C_k = 1
    assert nt[planted].sum() >= 0.8 * 16 * 6                                  # ~90% of tokens


def test_density_tiers_follow_table1(oracle):
    bands = {r[0]: tuple(map(float, r[1:])) for r in _read_table("table1_density_bands.txt")}
    q = I.qkv_case(1024)
    L = oracle.build_table(q.calib, 32)
    nh, nt = oracle.density(q.X, 32, L)
    cq = (nh[nt > 0] / nt[nt > 0]).mean()
    assert cq > bands["tier_high"][0]                       # attention input: static protection
    w = I.w2_case(M=512, calib_tokens=1536)
    Lw = oracle.build_table(w.calib, 32)
    nh, nt = oracle.density(w.X, 32, Lw)
    cw = (nh[nt > 0] / nt[nt > 0]).mean()
    lo, hi = bands["w2"]
    assert lo <= cw <= hi and cw < bands["tier_fp8"][0]     # W2: FP8 fallback tier


# ---- extraction, reconstruction and the dual-path product -----------------------------

def test_extract_moves_table_values(oracle):
    c = I.tiny_case()
    K_L = 16
    Xz, B = oracle.extract(c.X, 32, c.planted, K_L)
    cols = [k * 32 + int(j) for k, j in enumerate(c.planted) if j >= 0]
    assert np.array_equal(B[:, :len(cols)], c.X[:, cols])
    assert np.all(B[:, len(cols):] == 0)
    assert np.all(Xz[:, cols] == 0)
    mask = np.ones(256, bool); mask[cols] = False
    assert np.array_equal(Xz[:, mask], c.X[:, mask])
    with pytest.raises(ValueError):
        oracle.extract(c.X, 32, c.planted, len(cols) - 1)


def test_reconstruction_bound(oracle):
    c = I.qkv_case(64)
    L = c.planted
    K_L = I.pad16(oracle.table_count(L))
    Xz, B = oracle.extract(c.X, 32, L, K_L)
    codes, exps = oracle.mx_quantize(Xz, 32)
    deq = oracle.mx_dequantize(codes, exps)
    cols = [k * 32 + int(j) for k, j in enumerate(L) if j >= 0]
    rec = deq.copy()
    rec[:, cols] = I.bf16_to_f32(B[:, :len(cols)])
    x = I.bf16_to_f32(c.X).astype(np.float64)
    err = np.abs(rec - x)
    assert np.all(err[:, cols] == 0)                        # table slots are exact
    scale = np.repeat(2.0 ** exps.astype(np.float64), 32, axis=1)
    v = np.abs(I.bf16_to_f32(Xz).astype(np.float64)) / scale
    half = np.where(v <= 2, 0.25, np.where(v <= 4, 0.5, 1.0)) * scale
    inside = v <= 6
    assert np.all(err[inside] <= half[inside])
    sat = ~inside
    assert np.all(np.isclose(err[sat], (v[sat] - 6) * scale[sat], rtol=0, atol=0))
    assert np.all(err[sat] < 2 * scale[sat])


def test_linear_equals_matmul_of_dequantized(oracle):
    """The dual-path product is a matmul of dequantized operands plus B W_L^T (library matmul)."""
    c = I.tiny_case()
    L, K_L = c.planted, 16
    cw, ew, WL = oracle.osc_prepare_weight(c.W, 32, L, K_L)
    r = oracle.osc_forward(c.X, 32, L, K_L, cw, ew, WL)
    want = oracle.mx_dequantize(r["cx"], r["ex"]) @ oracle.mx_dequantize(cw, ew).T
    want += I.bf16_to_f32(r["B"]).astype(np.float64) @ I.bf16_to_f32(WL).astype(np.float64).T
    assert np.allclose(r["Y"], want, rtol=1e-12, atol=1e-12)
    rows = np.array([3, 0, 15], np.int32)
    r2 = oracle.osc_forward(c.X, 32, L, K_L, cw, ew, WL, rows=rows)
    assert np.array_equal(r2["Y"], r["Y"][rows])


@pytest.mark.parametrize("G", [16, 64])
def test_linear_equals_matmul_of_dequantized_group_sizes(oracle, G):
    """The same identity with 16-wide scale slots (G = 16) and 64-groups sharing one exponent
    over two 32-slots (G = 64), on activations with fixed outlier channels."""
    st = I.make_structure(1024, 0.7, seed=21)
    X = I.gen_tokens(st, 12, seed=22)
    W = I.bf16_bits(np.random.default_rng(23).standard_normal((24, 1024)) * 0.02)
    L = I.planted_table(st, G)
    K_L = I.pad16(oracle.table_count(L))
    cw, ew, WL = oracle.osc_prepare_weight(W, G, L, K_L)
    r = oracle.osc_forward(X, G, L, K_L, cw, ew, WL)
    assert r["ex"].shape == (12, 1024 // (16 if G == 16 else 32))
    want = oracle.mx_dequantize(r["cx"], r["ex"]) @ oracle.mx_dequantize(cw, ew).T
    want += I.bf16_to_f32(r["B"]).astype(np.float64) @ I.bf16_to_f32(WL).astype(np.float64).T
    assert np.allclose(r["Y"], want, rtol=1e-12, atol=1e-12)
    xf = I.bf16_to_f32(X).astype(np.float64)
    wf = I.bf16_to_f32(W).astype(np.float64)
    rel = np.abs(r["Y"] - xf @ wf.T).max() / np.abs(xf @ wf.T).max()
    assert rel < 0.25                                        # a 4-bit product, not a wrong one


def _representable(rng, rows, K, V=32, e_range=(-8, 3)):
    """Rows whose every V-block is exactly an E2M1 grid times 2^e, with the block max at 4 or 6."""
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    q = rng.choice(grid, size=(rows, K)) * rng.choice([-1, 1], size=(rows, K))
    q[:, ::V] = rng.choice([4.0, 6.0], size=(rows, K // V)) * rng.choice([-1, 1], size=(rows, K // V))
    e = rng.integers(e_range[0], e_range[1], size=(rows, K // V))
    return q * np.repeat(2.0 ** e, V, axis=1)


def test_osc_is_exact_on_representable_inputs(oracle):
    """If the non-table values of X and all of W are exactly MXFP4-representable, the dual-path
    output equals X W^T exactly: any dropped term, wrong column or transposed W_L breaks it."""
    rng = np.random.default_rng(11)
    M, K, N, G = 24, 256, 40, 32
    x = _representable(rng, M, K)
    w = _representable(rng, N, K)
    L = np.array([5, -1, 0, 31, -1, 12, 7, -1], np.int8)
    for k, j in enumerate(L):
        if j >= 0:
            x[:, k * G + int(j)] = rng.choice([-1, 1], size=M) * rng.uniform(200, 900, size=M)
    X, W = I.bf16_bits(x), I.bf16_bits(w)
    xf, wf = I.bf16_to_f32(X).astype(np.float64), I.bf16_to_f32(W).astype(np.float64)
    K_L = 16
    cw, ew, WL = oracle.osc_prepare_weight(W, G, L, K_L)
    r = oracle.osc_forward(X, G, L, K_L, cw, ew, WL)
    assert np.allclose(r["Y"], xf @ wf.T, rtol=1e-13, atol=1e-9)
    # and without the table the outliers wreck the same product (MXFP4 direct)
    L0 = np.full(8, -1, np.int8)
    cw0, ew0, _ = oracle.osc_prepare_weight(W, G, L0, 0)
    r0 = oracle.osc_forward(X, G, L0, 0, cw0, ew0, None)
    assert np.abs(r0["Y"] - xf @ wf.T).max() > 1.0


def test_all_minus_one_table_is_mxfp4_direct(oracle):
    c = I.tiny_case()
    L0 = np.full(8, -1, np.int8)
    assert oracle.table_count(L0) == 0
    cw, ew, WL = oracle.osc_prepare_weight(c.W, 32, L0, 0)
    r = oracle.osc_forward(c.X, 32, L0, 0, cw, ew, WL)
    assert r["B"].shape == (16, 0) and np.array_equal(r["Xz"], c.X)
    cx, ex = oracle.mx_quantize(c.X, 32)
    direct = oracle.mx_dequantize(cx, ex) @ oracle.mx_dequantize(cw, ew).T
    assert np.allclose(r["Y"], direct, rtol=1e-12, atol=1e-12)


def test_weight_codes_do_not_depend_on_table(oracle):
    """Weight side (§3.3): W is microscaled along K as it is; the table only selects the W_L
    columns. So Q_W and S_W are those of the empty table, and the table's weight columns keep
    their codes (they meet zeroed activation codes in the base product)."""
    rng = np.random.default_rng(13)
    W = I.bf16_bits(rng.standard_normal((20, 256)) * 0.02)
    W[:, 2 * 32 + 0] = I.bf16_bits(np.full(20, 0.5))           # a weight column that sets its
    L = np.array([-1, 3, 0, -1, 31, -1, -1, 9], np.int8)       # block's scale, in the table
    cw, ew, WL = oracle.osc_prepare_weight(W, 32, L, 16)
    cw0, ew0, _ = oracle.osc_prepare_weight(W, 32, np.full(8, -1, np.int8), 0)
    assert np.array_equal(cw, cw0) and np.array_equal(ew, ew0)
    assert np.all(cw[:, 64] == oracle.mx_quantize(W[:, 64:96], 32)[0][:, 0])
    assert np.array_equal(WL[:, :4], W[:, [1 * 32 + 3, 2 * 32 + 0, 4 * 32 + 31, 7 * 32 + 9]])
    assert np.all(WL[:, 4:] == 0)


def test_fp8_fallback_exact_on_representable(oracle):
    rng = np.random.default_rng(12)
    M, K, N = 8, 128, 16
    g = np.array([0, 2 ** -9, 0.5, 1.125, 3.5, 15, 104, 256, 448])
    def rep(rows):
        q = rng.choice(g, size=(rows, K)) * rng.choice([-1, 1], size=(rows, K))
        q[:, ::32] = 448.0
        return q * np.repeat(2.0 ** rng.integers(-12, -4, size=(rows, K // 32)), 32, axis=1)
    x, w = rep(M), rep(N)
    X, W = I.bf16_bits(x), I.bf16_bits(w)
    r = oracle.fp8_forward(X, W)
    xf, wf = I.bf16_to_f32(X).astype(np.float64), I.bf16_to_f32(W).astype(np.float64)
    assert np.allclose(r["Y"], xf @ wf.T, rtol=1e-13, atol=1e-12)


def test_group_size_sweep_roundtrip(oracle):
    """G = 16 / 32 / 64 all reduce the error of the same layer relative to MXFP4 direct."""
    c = I.ffn_case(32, M=32, calib_tokens=256)
    Wsmall = c.W[:64]
    xf = I.bf16_to_f32(c.X).astype(np.float64)
    ref = xf @ I.bf16_to_f32(Wsmall).astype(np.float64).T
    for G in (16, 32, 64):
        L = I.planted_table(I.make_structure(4096, 0.65, seed=1003), G)
        K_L = I.pad16(oracle.table_count(L))
        cw, ew, WL = oracle.osc_prepare_weight(Wsmall, G, L, K_L)
        r = oracle.osc_forward(c.X, G, L, K_L, cw, ew, WL)
        L0 = np.full(4096 // G, -1, np.int8)
        cw0, ew0, _ = oracle.osc_prepare_weight(Wsmall, G, L0, 0)
        r0 = oracle.osc_forward(c.X, G, L0, 0, cw0, ew0, None)
        assert np.abs(r["Y"] - ref).mean() < 0.8 * np.abs(r0["Y"] - ref).mean()


# ---- the producer step before the quantize (RMSNorm; the reading fixes its order) ----------

def _bf16_row(vals):
    return I.bf16_bits(np.asarray(vals, dtype=np.float64))


def test_rmsnorm_sum_order_closed_forms(oracle):
    """Totals worked out by hand in fp32 (ties to even; the spacing of fp32 at 2^24 is 2).
    Row A: 4096 then 31 ones in block 0, then seven blocks of 32 ones: in ascending order
    every 1 added to 2^24 is a tie that rounds back to 2^24, so block 0 sums to 2^24, the
    other blocks to 32 each, and the pairwise combination gives 2^24 + 224 exactly (a plain
    left-to-right sum over the row would lose every 1 and give 2^24; block 0 summed in
    descending order would give 2^24 + 32 for that block).
    Row B: 4096 alone in block 0, a single 1 in each of blocks 1..7: pairwise, 2^24 + 1 ties
    back to 2^24, then 2^24 + 2 and 2^24 + 6 are exact; left to right over the block sums
    every 1 ties back to 2^24."""
    a = np.ones(256)
    a[0] = 4096.0
    assert oracle.row_sumsq(_bf16_row(a)) == 16777216.0 + 224.0
    b = np.zeros(256)
    b[0] = 4096.0
    b[32::32] = 1.0
    assert oracle.row_sumsq(_bf16_row(b)) == 16777216.0 + 6.0


@pytest.mark.parametrize("K", [256, 768, 4096])
def test_rmsnorm_sum_within_fp32_bound(oracle, K):
    """On random rows (K/32 not always a power of two) the fp32 total stays within the error
    bound of its additions, (31 + log2 P) * 2^-24 relative, of the exact sum of squares."""
    import math
    rng = np.random.default_rng(K)
    for scale in (1.0, 1e-3, 300.0):
        x = I.bf16_bits(rng.standard_normal(K) * scale)
        v = I.bf16_to_f32(x).astype(np.float64)
        exact = math.fsum(float(t) * float(t) for t in v)      # each square is exact in fp64
        depth = 31 + math.ceil(math.log2(K // 32))
        assert abs(oracle.row_sumsq(x) - exact) <= depth * 2.0 ** -24 * exact


def test_rmsnorm_constant_rows_give_unit_output(oracle):
    """A row of one repeated value c (gamma = 1, eps = 0) normalizes to sign(c) * 1 exactly
    in bf16: its root mean square is |c|."""
    rng = np.random.default_rng(11)
    c = rng.choice([-1, 1], 40) * np.exp2(rng.uniform(-30, 30, 40))
    X = I.bf16_bits(np.repeat(c[:, None], 512, axis=1))
    Y, _ = oracle.rmsnorm(X, np.full(512, 0x3F80, np.uint16), 0.0)
    assert np.array_equal(Y, np.where(c[:, None] < 0, 0xBF80, 0x3F80).astype(np.uint16) * np.ones((1, 512), np.uint16))


def test_rmsnorm_scale_invariance(oracle):
    """Scaling a row by 2^k scales every square and sum exactly and the root by 2^k, so with
    eps = 0 the normalized row is bit-identical and the inverse root scales by 2^-k."""
    c = I.qkv_case(8)
    X = c.X[:, :1024]
    gamma = I.bf16_bits(1.0 + 0.1 * np.random.default_rng(2).standard_normal(1024))
    Y0, inv0 = oracle.rmsnorm(X, gamma, 0.0)
    for k in (-20, -3, 5, 17):
        Xk = I.bf16_bits(I.bf16_to_f32(X).astype(np.float64) * 2.0 ** k)
        Yk, invk = oracle.rmsnorm(Xk, gamma, 0.0)
        assert np.array_equal(Yk, Y0), k
        assert np.array_equal(invk.astype(np.float64), inv0.astype(np.float64) * 2.0 ** -k), k


def test_rmsnorm_matches_the_fp64_definition(oracle):
    """Against x / sqrt(mean(x^2) + eps) * gamma computed in fp64 from the same bf16 inputs:
    within one bf16 ulp (the fp32 steps add a few fp32 ulps before the final rounding). A row of
    tiny values, where eps dominates the mean, pins where eps enters."""
    from tests._layout import bf16_ulp
    rng = np.random.default_rng(5)
    c = I.qkv_case(16)
    X = np.concatenate([c.X, I.bf16_bits(rng.standard_normal((2, 4096)) * 1e-4)], axis=0)
    gamma = I.bf16_bits(1.0 + 0.2 * rng.standard_normal(4096))
    for eps in (1e-6, 1e-2):
        Y, _ = oracle.rmsnorm(X, gamma, eps)
        x = I.bf16_to_f32(X).astype(np.float64)
        g = I.bf16_to_f32(gamma).astype(np.float64)
        ref = x / np.sqrt((x * x).mean(axis=1, keepdims=True) + np.float64(np.float32(eps))) * g
        y = I.bf16_to_f32(Y).astype(np.float64)
        assert np.all(np.abs(y - ref) <= bf16_ulp(ref) + 1e-30), eps


def test_rmsnorm_then_osc_is_osc_of_the_normalized_rows(oracle):
    """The fused input side quantizes the normalized rows: rows that RMSNorm leaves unchanged
    (every value +-1, gamma = 1, eps = 0) give exactly the plain OSC outputs, and scaling them
    by 2^k changes nothing (the raw rows would get other scale exponents)."""
    rng = np.random.default_rng(9)
    K, G = 512, 32
    X = I.bf16_bits(rng.choice([-1.0, 1.0], (6, K)))
    W = I.gen_weights(64, K, seed=4)
    L = np.full(K // G, -1, np.int8)
    L[[1, 5, 9]] = [3, 0, 31]
    K_L = 16
    ones = np.full(K, 0x3F80, np.uint16)
    cw, ew, WL = oracle.osc_prepare_weight(W, G, L, K_L)
    plain = oracle.osc_forward(X, G, L, K_L, cw, ew, WL)
    Xk = I.bf16_bits(I.bf16_to_f32(X).astype(np.float64) * 2.0 ** 9)
    fused = oracle.rmsnorm_osc_forward(Xk, ones, 0.0, G, L, K_L, cw, ew, WL)
    for key in ("cx", "ex", "B"):
        assert np.array_equal(fused[key], plain[key]), key
    assert np.array_equal(fused["Y"], plain["Y"])


# ---- several protected channels per group (multi-outlier protection) ----------------------

def test_multi_table_finds_planted_second_channels(oracle):
    """Two persistent outliers in group 0 (channels 3 and 20), one in group 1 (channel 7), none
    in group 2, and in group 3 a second outlier on only 3 tokens (below min_hits): round 1
    finds the larger of each pair, round 2 the smaller one once the first is zeroed, and slots
    stay -1 once a round finds nothing. R = 1 is the single-entry table."""
    rng = np.random.default_rng(21)
    S, G = 60, 32
    X = rng.standard_normal((S, 4 * G)) * 0.5
    X[:, 0 * G + 3] = 100.0 * rng.choice([-1, 1], S)
    X[:, 0 * G + 20] = 60.0 * rng.choice([-1, 1], S)
    X[:, 1 * G + 7] = -90.0
    X[:, 3 * G + 11] = 80.0
    X[:3, 3 * G + 30] = 70.0
    Xb = I.bf16_bits(X)
    L3 = oracle.build_table_multi(Xb, G, 3)
    assert L3.tolist() == [[3, 20, -1], [7, -1, -1], [-1, -1, -1], [11, -1, -1]]
    assert np.array_equal(oracle.build_table_multi(Xb, G, 1)[:, 0], oracle.build_table(Xb, G))
    q = I.qkv_case(1)                                         # one planted channel per group
    L2 = oracle.build_table_multi(q.calib, 32, 2)
    assert np.array_equal(L2[:, 0], q.planted) and np.all(L2[:, 1] == -1)


def test_multi_extract_order_and_repeated_channel(oracle):
    """Entries are taken in (group, slot) order, each moved to its own B column and zeroed;
    a channel named twice in one group gives its value once and 0 the second time; W_L takes
    the same columns in the same order."""
    rng = np.random.default_rng(22)
    M, K, G = 5, 128, 32
    X = I.bf16_bits(rng.standard_normal((M, K)))
    L = np.array([[4, 9], [-1, -1], [30, 30], [0, -1]], np.int8)
    Xz, B = oracle.extract(X, G, L, 16)
    cols = [0 * G + 4, 0 * G + 9, 2 * G + 30, 3 * G + 0]
    assert np.array_equal(B[:, [0, 1, 2, 4]], X[:, cols])
    assert np.all(B[:, 3] == 0) and np.all(B[:, 5:] == 0)      # the repeated channel, the pad
    assert np.all(Xz[:, cols] == 0)
    keep = np.ones(K, bool); keep[cols] = False
    assert np.array_equal(Xz[:, keep], X[:, keep])
    W = I.bf16_bits(rng.standard_normal((7, K)))
    WL = oracle.gather_wl(W, G, L, 16)
    assert np.array_equal(WL[:, :5], W[:, [cols[0], cols[1], cols[2], cols[2], cols[3]]])
    assert oracle.table_count(L) == 5 and np.all(WL[:, 5:] == 0)


def test_multi_osc_is_exact_on_representable_inputs(oracle):
    """With two large outliers in some groups, a two-slot table makes the dual-path output
    equal X W^T exactly (both channels ride the 16-bit path); keeping only the first slot
    leaves the second outlier to set its block's scale and the product visibly off."""
    rng = np.random.default_rng(23)
    M, K, N, G = 16, 256, 24, 32
    x = _representable(rng, M, K)
    w = _representable(rng, N, K)
    L = np.array([[5, 17], [-1, -1], [0, 31], [12, -1], [-1, -1], [2, 3], [7, -1], [-1, -1]], np.int8)
    for k in range(8):
        for j in L[k]:
            if j >= 0:
                x[:, k * G + int(j)] = rng.choice([-1, 1], size=M) * rng.uniform(200, 900, size=M)
    X, W = I.bf16_bits(x), I.bf16_bits(w)
    xf, wf = I.bf16_to_f32(X).astype(np.float64), I.bf16_to_f32(W).astype(np.float64)
    cw, ew, WL = oracle.osc_prepare_weight(W, G, L, 16)
    r = oracle.osc_forward(X, G, L, 16, cw, ew, WL)
    assert np.allclose(r["Y"], xf @ wf.T, rtol=1e-13, atol=1e-9)
    L1 = L[:, 0].copy()
    cw1, ew1, WL1 = oracle.osc_prepare_weight(W, G, L1, 16)
    r1 = oracle.osc_forward(X, G, L1, 16, cw1, ew1, WL1)
    assert np.abs(r1["Y"] - xf @ wf.T).max() > 1.0
