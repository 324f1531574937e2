"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This module holds none of the OSC arithmetic: it only draws activations,
weights, calibration sets and MoE routings with the shapes and outlier
structure that the OSC page ("W4A4量化技术：OSC框架如何实现高效LLM部署",
coreui.cn/article/2607942.html) describes for Qwen3-8B / Qwen3-30B-A3B
(§2.1 token-persistent outlier channels, §2.3 Table 1 per-module clustering
densities, §5.2 3x512 calibration tokens). Neither the model weights nor the
Pile are available, so these draws stand in for them.

Recipe (all draws from numpy's PCG64 with fixed seeds):
  * base activations N(0, 1); weights N(0, 0.02); rounded to bf16 (ties to even).
  * a *structure* fixes, per 32-channel block, whether it holds a fixed outlier
    channel (fraction ``frac_fixed`` of blocks), which channel, and its sign.
    The structure is a property of the activations, so the same structure serves
    every group size G (a 64-group can hold two fixed channels, a 16-group none).
  * per token, each fixed channel carries sign * U(lo, hi) with probability
    ``persist`` (1.0 = on every token).
  * ``spike_frac`` of tokens carry one extra spike, +-U(lo, hi), in a channel
    drawn uniformly over all K (random sign).
  * ``diffuse_frac``: in blocks without a fixed channel, each token carries a
    spike +-U(lo, hi) in a per-token random channel of the block with that
    probability (the diffuse W2 pattern).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

BLOCK = 32


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float array -> bf16 bit patterns (uint16), via fp32, round to nearest even."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32)
    r = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + r) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Structure:
    K: int
    fixed_ch: np.ndarray   # per 32-block: absolute channel index, or -1
    sign: np.ndarray       # per 32-block: +1 / -1


def make_structure(K: int, frac_fixed: float, seed: int, n_fixed: int | None = None) -> Structure:
    assert K % BLOCK == 0
    nb = K // BLOCK
    rng = np.random.default_rng(seed)
    cnt = int(round(frac_fixed * nb)) if n_fixed is None else n_fixed
    chosen = rng.permutation(nb)[:cnt]
    fixed = np.full(nb, -1, dtype=np.int64)
    fixed[chosen] = chosen * BLOCK + rng.integers(0, BLOCK, size=cnt)
    sign = np.where(rng.random(nb) < 0.5, -1.0, 1.0)
    return Structure(K=K, fixed_ch=fixed, sign=sign)


def gen_tokens(st: Structure, M: int, seed: int, mag=(20.0, 80.0), persist: float = 1.0,
               spike_frac: float = 0.0, spike_mag=(20.0, 80.0), diffuse_frac: float = 0.0,
               diffuse_mag=(20.0, 60.0)) -> np.ndarray:
    """M x K activations (bf16 bits) with the given outlier structure."""
    K = st.K
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K), dtype=np.float32)
    blocks = np.nonzero(st.fixed_ch >= 0)[0]
    if blocks.size and M:
        ch = st.fixed_ch[blocks]
        vals = rng.uniform(mag[0], mag[1], size=(M, blocks.size)).astype(np.float32)
        on = rng.random((M, blocks.size)) < persist
        cur = X[:, ch]
        X[:, ch] = np.where(on, vals * st.sign[blocks][None, :].astype(np.float32), cur)
    if diffuse_frac > 0 and M:
        free = np.nonzero(st.fixed_ch < 0)[0]
        if free.size:
            on = rng.random((M, free.size)) < diffuse_frac
            ch = free[None, :] * BLOCK + rng.integers(0, BLOCK, size=(M, free.size))
            vals = rng.uniform(diffuse_mag[0], diffuse_mag[1], size=(M, free.size))
            sg = np.where(rng.random((M, free.size)) < 0.5, -1.0, 1.0)
            t_idx, b_idx = np.nonzero(on)
            X[t_idx, ch[t_idx, b_idx]] = (vals * sg)[t_idx, b_idx]
    if spike_frac > 0 and M:
        nt = int(round(spike_frac * M))
        toks = rng.permutation(M)[:nt]
        ch = rng.integers(0, K, size=nt)
        sg = np.where(rng.random(nt) < 0.5, -1.0, 1.0)
        X[toks, ch] = (rng.uniform(spike_mag[0], spike_mag[1], size=nt) * sg).astype(np.float32)
    return bf16_bits(X)


def gen_weights(N: int, K: int, seed: int, std: float = 0.02) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return bf16_bits(rng.standard_normal((N, K), dtype=np.float32) * np.float32(std))


def planted_table(st: Structure, G: int) -> np.ndarray:
    """The fixed channels of a structure as a table (first fixed channel per G-group)."""
    Kg = st.K // G
    L = np.full(Kg, -1, dtype=np.int8)
    for c in st.fixed_ch[st.fixed_ch >= 0]:
        k = int(c) // G
        if L[k] < 0 or int(c) % G < L[k]:
            L[k] = int(c) % G
    return L


def pad16(n: int) -> int:
    return (n + 15) // 16 * 16


def block_rows(M: int, seed: int, block: int = 128) -> np.ndarray:
    """Sorted rows for parity checks that reach every `block`-row block of M rows: each
    block's first and last row and one seeded row inside it (so every output tile row block,
    and both CTAs of a 256-row CTA-pair tile, is checked at its edges)."""
    rng = np.random.default_rng(seed)
    pick = set()
    for b0 in range(0, M, block):
        b1 = min(M, b0 + block) - 1
        pick.update((b0, b1, int(rng.integers(b0, b1 + 1))))
    return np.array(sorted(pick), dtype=np.int32)


# ---- the named workloads ------------------------------------------------------

@dataclass
class LinearCase:
    name: str
    M: int
    K: int
    N: int
    G: int
    X: np.ndarray          # M x K bf16 bits
    W: np.ndarray          # N x K bf16 bits
    calib: np.ndarray      # S x K bf16 bits (calibration tokens), or None
    planted: np.ndarray    # planted table (int8, K/G)


def tiny_case() -> LinearCase:
    """M=16, K=256 (8 groups of 32), N=128: 6 of the 8 groups carry a fixed channel
    at +-U(20,60) on 90% of tokens; the table is those channels."""
    st = make_structure(256, 0.0, seed=1001, n_fixed=6)
    X = gen_tokens(st, 16, seed=1001, mag=(20.0, 60.0), persist=0.9)
    W = gen_weights(128, 256, seed=2001)
    return LinearCase("tiny", 16, 256, 128, 32, X, W, None, planted_table(st, 32))


def qkv_case(M: int, calib_tokens: int = 1536) -> LinearCase:
    """Qwen3-8B fused QKV: K=4096, N=6144, G=32; fixed channels in 70% of 32-blocks
    (+-U(20,80), every token) and a random-channel spike on 5% of tokens."""
    st = make_structure(4096, 0.70, seed=1002)
    X = gen_tokens(st, M, seed=1002 + M, spike_frac=0.05)
    calib = gen_tokens(st, calib_tokens, seed=1102, spike_frac=0.05)
    W = gen_weights(6144, 4096, seed=2002)
    return LinearCase(f"qkv_m{M}", M, 4096, 6144, 32, X, W, calib, planted_table(st, 32))


def second_channel(st: Structure, frac: float, seed: int) -> Structure:
    """A second fixed outlier channel in a fraction of the blocks that already hold one (the
    extreme case of the OSC page's §6 multi-outlier protection): a structure whose fixed
    channels are those second channels, drawn distinct from the first."""
    rng = np.random.default_rng(seed)
    fixed = np.full_like(st.fixed_ch, -1)
    blocks = np.nonzero(st.fixed_ch >= 0)[0]
    pick = rng.permutation(blocks)[: int(round(frac * blocks.size))]
    for b in pick:
        first = int(st.fixed_ch[b]) - b * BLOCK
        j = int(rng.integers(0, BLOCK - 1))
        fixed[b] = b * BLOCK + (j if j < first else j + 1)
    return Structure(K=st.K, fixed_ch=fixed, sign=np.where(rng.random(st.fixed_ch.size) < 0.5, -1.0, 1.0))


def two_outlier_case(M: int, calib_tokens: int = 1536) -> LinearCase:
    """The QKV shape (K=4096, N=6144, G=32) where 40% of the blocks with a fixed channel
    (+-U(20,80)) hold a second fixed channel at +-U(8,16) on every token: smaller than the
    first, yet still an outlier once the first is taken out."""
    st = make_structure(4096, 0.70, seed=1002)
    st2 = second_channel(st, 0.40, seed=1202)

    def draw(n, seed):
        X = bf16_to_f32(gen_tokens(st, n, seed=seed, spike_frac=0.05)).copy()
        rng = np.random.default_rng(seed + 1)
        b = np.nonzero(st2.fixed_ch >= 0)[0]
        vals = rng.uniform(8.0, 16.0, size=(n, b.size)) * st2.sign[b][None, :]
        X[:, st2.fixed_ch[b]] = vals
        return bf16_bits(X)

    X = draw(M, 1302 + M)
    calib = draw(calib_tokens, 1402)
    W = gen_weights(6144, 4096, seed=2002)
    return LinearCase(f"qkv2_m{M}", M, 4096, 6144, 32, X, W, calib, planted_table(st, 32))


def ffn_case(G: int, M: int = 4096, calib_tokens: int = 1536) -> LinearCase:
    """Qwen3-8B FFN up/gate: K=4096, N=24576, fixed channels in 65% of 32-blocks."""
    st = make_structure(4096, 0.65, seed=1003)
    X = gen_tokens(st, M, seed=1003, spike_frac=0.05)
    calib = gen_tokens(st, calib_tokens, seed=1103, spike_frac=0.05)
    W = gen_weights(24576, 4096, seed=2003)
    return LinearCase(f"ffn_g{G}", M, 4096, 24576, G, X, W, calib, planted_table(st, G))


def w2_case(M: int = 4096, calib_tokens: int = 1536) -> LinearCase:
    """Qwen3-8B down projection: K=12288, N=4096; fixed channels in 25% of blocks,
    the other blocks carry a +-U(20,60) spike in a per-token random channel on 30% of tokens."""
    st = make_structure(12288, 0.25, seed=1004)
    kw = dict(mag=(20.0, 60.0), diffuse_frac=0.30, diffuse_mag=(20.0, 60.0))
    X = gen_tokens(st, M, seed=1004, **kw)
    calib = gen_tokens(st, calib_tokens, seed=1104, **kw)
    W = gen_weights(4096, 12288, seed=2004)
    return LinearCase("w2", M, 12288, 4096, 32, X, W, calib, planted_table(st, 32))


@dataclass
class MoeCase:
    name: str
    E: int
    K: int
    N: int
    G: int
    counts: np.ndarray     # tokens per expert (E)
    X: np.ndarray          # sum(counts) x K, rows sorted by expert
    W: np.ndarray          # E x N x K
    calib: list            # per expert: S_e x K calibration rows


def moe_routing(T: int = 4096, E: int = 128, topk: int = 8, zipf: float = 1.1, seed: int = 1005):
    """Top-k routing with Zipf(zipf) expert popularity: each token picks topk distinct
    experts without replacement with probability proportional to rank^-zipf under a
    seeded rank permutation. Returns (token x topk expert ids, per-expert counts)."""
    rng = np.random.default_rng(seed)
    rank = rng.permutation(E) + 1
    p = rank.astype(np.float64) ** (-zipf)
    p /= p.sum()
    sel = np.empty((T, topk), dtype=np.int64)
    for t in range(T):
        sel[t] = rng.choice(E, size=topk, replace=False, p=p)
    counts = np.bincount(sel.reshape(-1), minlength=E)
    return sel, counts


def moe_case(which: str = "gateup", T: int = 4096, E: int = 128, calib_T: int = 1536,
             counts_override=None) -> MoeCase:
    """Qwen3-30B-A3B expert layer: hidden 2048, 128 experts, gate+up 2048 -> 1536
    (which='gateup') or down 768 -> 2048 (which='down'); top-8 routing of T tokens."""
    if which == "gateup":
        K, N, sseed = 2048, 1536, 1015
    else:
        K, N, sseed = 768, 2048, 1025
    _, counts = moe_routing(T, E)
    if counts_override is not None:
        counts = np.asarray(counts_override, dtype=np.int64)
    _, ccounts = moe_routing(calib_T, E, seed=1105)
    xs, calib = [], []
    for e in range(E):
        st = make_structure(K, 0.70, seed=sseed if which == "gateup" else sseed + 1000 + e)
        xs.append(gen_tokens(st, int(counts[e]), seed=sseed + 7 * e + 1, spike_frac=0.05))
        calib.append(gen_tokens(st, int(ccounts[e]), seed=sseed + 7 * e + 3, spike_frac=0.05))
    X = np.concatenate(xs, axis=0) if xs else np.zeros((0, K), np.uint16)
    rng = np.random.default_rng(sseed + 99)
    W = bf16_bits(rng.standard_normal((E, N, K), dtype=np.float32) * np.float32(0.02))
    return MoeCase(f"moe_{which}", E, K, N, 32, counts, X, W, calib)
