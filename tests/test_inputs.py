"""The synthetic inputs have the structure the design notes state for each workload (the OSC
page's Qwen3 activations are not available, so these draws stand in for them): fixed outlier
channels in the stated fraction of 32-blocks with the stated magnitudes, random spikes on the
stated share of tokens, the diffuse W2 pattern, top-8 MoE routing with Zipf loads, and the same
arrays for the same seeds."""
import numpy as np

from w4a4_outlier_separated_b200 import inputs as I


def _f(bits):
    return I.bf16_to_f32(bits).astype(np.float64)


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 0.0, -0.0], np.float32)
    b = I.bf16_bits(x)
    # 1 + 2^-8 is the midpoint of 1 and 1 + 2^-7: ties go to the even mantissa (1.0);
    # 1 + 3 * 2^-8 is the midpoint of 1 + 2^-7 and 1 + 2^-6: even is 1 + 2^-6
    assert list(_f(b)) == [1.0, 1.0, 1.0 + 2.0 ** -6, -2.5, 0.0, 0.0]
    assert b[5] == 0x8000                                   # the sign of zero survives


def test_structure_fractions():
    for K, frac in ((4096, 0.70), (4096, 0.65), (12288, 0.25)):
        st = I.make_structure(K, frac, seed=7)
        nb = K // 32
        fixed = st.fixed_ch >= 0
        assert fixed.sum() == round(frac * nb)
        ch = st.fixed_ch[fixed]
        assert np.all(ch // 32 == np.nonzero(fixed)[0])     # each fixed channel lies in its own block


def test_qkv_tokens_carry_fixed_outliers_and_spikes():
    c = I.qkv_case(512)
    st = I.make_structure(4096, 0.70, seed=1002)
    x = _f(c.X)
    fixed = st.fixed_ch[st.fixed_ch >= 0]
    mag = np.abs(x[:, fixed])
    assert mag.min() >= 20.0 * 0.99 and mag.max() <= 80.0 * 1.01   # +-U(20, 80) on every token
    signs = np.sign(x[:, fixed])
    assert np.all(signs == st.sign[fixed // 32][None, :])          # one sign per channel
    rest = np.ones(4096, bool)
    rest[fixed] = False
    big = np.abs(x[:, rest]) >= 20.0
    spiked_tokens = np.count_nonzero(big.any(axis=1))
    assert abs(spiked_tokens - round(0.05 * 512)) <= 2             # one spike on ~5% of tokens
    assert np.abs(x[:, rest][~big]).max() < 8.0                    # the rest is N(0, 1)
    # the planted table names exactly the fixed channels
    L = c.planted
    assert np.array_equal(np.nonzero(L >= 0)[0], np.sort(fixed // 32))
    assert np.all(L[fixed // 32] == fixed % 32)


def test_tiny_case_shape_and_persistence():
    c = I.tiny_case()
    assert (c.M, c.K, c.N, c.G) == (16, 256, 128, 32)
    assert np.count_nonzero(c.planted >= 0) == 6
    x = _f(c.X)
    cols = [k * 32 + int(j) for k, j in enumerate(c.planted) if j >= 0]
    on = np.abs(x[:, cols]) >= 20.0
    assert 0.75 <= on.mean() <= 1.0                                 # present on ~90% of tokens
    assert np.abs(x[:, cols][on]).max() <= 60.0 * 1.01


def test_w2_diffuse_pattern():
    c = I.w2_case(M=256, calib_tokens=16)
    st = I.make_structure(12288, 0.25, seed=1004)
    x = _f(c.X)
    free = np.nonzero(st.fixed_ch < 0)[0]
    blk = np.abs(x[:, :].reshape(256, 384, 32))[:, free, :]
    hit = (blk >= 20.0).any(axis=2)
    assert 0.27 <= hit.mean() <= 0.33                               # a spike on 30% of tokens per block
    assert np.all((blk >= 20.0).sum(axis=2) <= 1)                   # at most one per block and token
    fixed = st.fixed_ch[st.fixed_ch >= 0]
    assert np.abs(x[:, fixed]).min() >= 20.0 * 0.99 and np.abs(x[:, fixed]).max() <= 60.0 * 1.01


def test_moe_routing_top8_zipf():
    ids, counts = I.moe_routing()
    assert ids.shape == (4096, 8)
    assert all(len(set(r)) == 8 for r in ids.tolist())             # 8 distinct experts per token
    assert counts.sum() == 4096 * 8 and counts.shape == (128,)
    assert np.array_equal(counts, np.bincount(ids.reshape(-1), minlength=128))
    s = np.sort(counts)[::-1]
    assert s[0] > 20 * np.median(counts)                            # heavy head, Zipf(1.1)
    assert s[-1] > 0


def test_same_seed_same_arrays():
    a, b = I.qkv_case(64), I.qkv_case(64)
    assert np.array_equal(a.X, b.X) and np.array_equal(a.W, b.W) and np.array_equal(a.calib, b.calib)
    assert not np.array_equal(I.gen_weights(8, 256, seed=1), I.gen_weights(8, 256, seed=2))


def test_block_rows_reach_every_block_edge():
    """The parity row sampler covers the first and last row of every 128-row block (ragged
    tail included), and nothing outside [0, M)."""
    for M in (1, 127, 128, 129, 300, 3712):
        r = I.block_rows(M, seed=M)
        assert r.min() >= 0 and r.max() < M and np.all(np.diff(r) > 0)
        for b0 in range(0, M, 128):
            assert b0 in r and min(M, b0 + 128) - 1 in r
