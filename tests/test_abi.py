"""The C ABI on the CPU: libosc.so loads, exports every function include/osc.h declares, and
its host-only logic (sizes, table width, grouped plan, argument checks) behaves as documented.
No compute call is made here."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from w4a4_outlier_separated_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def _declared():
    src = open(os.path.join(ROOT, "include", "osc.h")).read()
    return sorted(set(re.findall(r"OSC_API\s+[\w\s\*]+?\b(osc_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 16
    for n in names:
        assert hasattr(lib, n), n


def test_binding_names_match_header():
    from w4a4_outlier_separated_b200 import osc
    for n in _declared():
        if n in ("osc_version", "osc_error_string", "osc_last_cuda_error"):
            continue
        assert hasattr(osc, n), n


def test_scale_bytes(lib):
    f = lib.osc_scale_bytes
    f.restype = ctypes.c_size_t
    assert f(16, 256, 32) == 1 * 2 * 512
    assert f(2048, 4096, 32) == 16 * 32 * 512
    assert f(129, 4096, 16) == 2 * 64 * 512
    assert f(1, 4096, 64) == 1 * 32 * 512
    assert f(4096, 12288, 0) == 32 * 96 * 512
    assert f(16, 256, 24) == 0 and f(16, 100, 32) == 0


def test_table_kl(lib):
    L = np.array([-1, 5, 6, -1, 0, -1, 2, 15], np.int8)
    assert lib.osc_table_kl(L.ctypes.data_as(ctypes.c_void_p), 8) == 16
    L = np.full(128, 3, np.int8)
    assert lib.osc_table_kl(L.ctypes.data_as(ctypes.c_void_p), 128) == 128
    L[:39] = -1
    assert lib.osc_table_kl(L.ctypes.data_as(ctypes.c_void_p), 128) == 96


def test_grouped_plan(lib):
    counts = np.array([130, 0, 1, 257, 128], np.int32)
    off = np.zeros(6, np.int32)
    poff = np.zeros(6, np.int32)
    P = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    mp = lib.osc_grouped_plan(P(counts), 5, P(off), P(poff), None, 0)
    assert mp == 256 + 0 + 128 + 384 + 128
    mbe = np.full(mp // 128, -9, np.int32)
    assert lib.osc_grouped_plan(P(counts), 5, P(off), P(poff), P(mbe), mbe.size) == mp
    assert list(off) == [0, 130, 130, 131, 388, 516]
    assert list(poff) == [0, 256, 256, 384, 768, 896]
    assert list(mbe) == [0, 0, 2, 3, 3, 3, 4]
    assert lib.osc_grouped_plan(P(counts), 5, P(off), P(poff), P(mbe), 3) < 0


def test_argument_checks_return_before_any_cuda_call(lib):
    V = ctypes.c_void_p
    buf = (ctypes.c_uint8 * 4096)()
    p = ctypes.cast(buf, V)
    p16 = V((ctypes.addressof(buf) + 15) // 16 * 16)
    lib.osc_quantize.argtypes = [V, ctypes.c_int, ctypes.c_int, ctypes.c_int, V, ctypes.c_int, ctypes.c_int,
                                 V, V, V, V]
    assert lib.osc_quantize(p16, 4, 256, 24, None, 1, 0, p16, p16, None, None) == -3          # G
    assert lib.osc_quantize(None, 4, 256, 32, None, 1, 0, p16, p16, None, None) == -1         # null
    assert lib.osc_quantize(p16, 4, 200, 32, None, 1, 0, p16, p16, None, None) == -2          # K % 256
    assert lib.osc_quantize(V(p16.value + 2), 4, 256, 32, None, 1, 0, p16, p16, None, None) == -2  # alignment
    assert lib.osc_quantize(p16, 4, 256, 32, None, 1, 16, p16, p16, p16, None) == -1          # K_L without table
    assert lib.osc_quantize(p16, 4, 256, 32, p16, 0, 0, p16, p16, None, None) == -1           # R < 1
    assert lib.osc_quantize(p16, 4, 256, 32, p16, 4, 0, p16, p16, None, None) == -1           # R > 3
    lib.osc_linear.argtypes = [V] * 6 + [ctypes.c_int] * 5 + [V, V, V]
    assert lib.osc_linear(p16, p16, None, p16, p16, None, 4, 100, 256, 32, 0, p16, None, None) == -2  # N % 16
    assert lib.osc_linear(p16, p16, None, p16, p16, None, 4, 128, 256, 32, 8, p16, None, None) == -2  # K_L % 16
    assert lib.osc_linear(p16, p16, None, p16, p16, None, 4, 128, 256, 32, 16, p16, None, None) == -1  # B missing
    lib.osc_error_string.restype = ctypes.c_char_p
    assert b"group size" in lib.osc_error_string(-3)
    lib.osc_set_tile_n.argtypes = [ctypes.c_int]
    assert lib.osc_set_tile_n(96) == -1
    assert lib.osc_set_tile_n(128) == 0 and lib.osc_set_tile_n(0) == 128
    _ = p


def test_argument_limits_of_every_entry_point(lib):
    """Each entry point rejects out-of-range or misaligned arguments with the documented code
    before touching a device: table longer than 1024 groups, K_L above 32767, row counts whose
    scale indexing would overflow, bad group sizes, missing buffers, unaligned K or row padding."""
    V, I = ctypes.c_void_p, ctypes.c_int
    buf = (ctypes.c_uint8 * 4096)()
    p16 = V((ctypes.addressof(buf) + 15) // 16 * 16)
    q = lib.osc_quantize
    q.argtypes = [V, I, I, I, V, I, I, V, V, V, V]
    assert q(p16, 4, 131328, 32, p16, 1, 0, p16, p16, None, None) == -1    # K / G = 4104 > 4096 entries
    assert q(p16, 4, 45056, 32, p16, 3, 0, p16, p16, None, None) == -1     # 1408 groups x 3 slots > 4096
    assert q(p16, 4, 4096, 32, p16, 1, 32784, p16, p16, p16, None) == -1   # K_L > 32767
    assert q(p16, 1 << 30, 256, 32, None, 1, 0, p16, p16, None, None) == -1   # (M + 127) * K / 32 >= 2^31
    assert q(p16, 4, 256, 32, p16, 1, 16, p16, p16, None, None) == -1      # K_L > 0 needs B
    assert q(p16, 0, 256, 32, None, 1, 0, None, None, None, None) == 0     # M = 0: no-op, NULLs allowed
    li = lib.osc_linear
    li.argtypes = [V] * 6 + [I] * 5 + [V, V, V]
    assert li(None, None, None, None, None, None, 0, 128, 256, 32, 0, None, None, None) == 0   # M = 0: no-op
    assert li(None, None, None, None, None, None, 0, 128, 256, 24, 0, None, None, None) == -3  # G still checked
    q8 = lib.osc_quantize_fp8
    q8.argtypes = [V, I, I, V, V, V]
    assert q8(None, 0, 256, None, None, None) == 0                          # M = 0: no-op
    l8 = lib.osc_linear_fp8_fallback
    l8.argtypes = [V, V, V, V, I, I, I, V, V, V]
    assert l8(None, None, None, None, 0, 64, 256, None, None, None) == 0  # M = 0: no-op
    w = lib.osc_prepare_weight
    w.argtypes = [V, I, I, I, V, I, I, V, V, V, V]
    assert w(p16, 4, 256, 48, None, 1, 0, p16, p16, None, None) == -3      # G
    assert w(p16, 4, 256, 32, None, 1, 16, p16, p16, p16, None) == -1      # K_L > 0 needs L
    assert w(p16, 4, 512, 32, p16, 1, 8, p16, p16, p16, None) == -2        # K_L % 16
    assert w(p16, 4, 512, 32, p16, 5, 16, p16, p16, p16, None) == -1       # R > 3
    f8 = lib.osc_quantize_fp8
    f8.argtypes = [V, I, I, V, V, V]
    assert f8(p16, 4, 384, p16, p16, None) == -2                           # K % 256
    assert f8(None, 4, 256, p16, p16, None) == -1
    lf8 = lib.osc_linear_fp8_fallback
    lf8.argtypes = [V, V, V, V, I, I, I, V, V, V]
    assert lf8(p16, p16, p16, p16, 4, 40, 256, p16, None, None) == -2     # N % 16
    assert lf8(p16, p16, p16, p16, -1, 32, 256, p16, None, None) == -1    # M < 0
    bt = lib.osc_build_table
    bt.argtypes = [V, I, I, I, ctypes.c_float, I, V, V]
    assert bt(p16, 8, 250, 32, 5.0, 5, p16, None) == -1                    # K % G
    assert bt(p16, 8, 256, 8, 5.0, 5, p16, None) == -3                     # G
    qg = lib.osc_quantize_grouped
    qg.argtypes = [V, I, I, V, V, V, I, I, I, V, I, I, V, V, V, V]
    assert qg(p16, 100, 2, p16, p16, p16, 200, 256, 32, p16, 1, 0, p16, p16, None, None) == -2   # Mp % 128
    assert qg(p16, 100, 2, p16, p16, p16, 256, 256, 32, None, 1, 0, p16, p16, None, None) == -1  # tables required
    assert qg(p16, 100, 2, p16, p16, p16, 1 << 30, 256, 32, p16, 1, 0, p16, p16, None, None) == -1  # scale index
    assert qg(p16, 300, 2, p16, p16, p16, 256, 256, 32, p16, 1, 0, p16, p16, None, None) == -1   # T > Mp
    assert qg(p16, -1, 2, p16, p16, p16, 256, 256, 32, p16, 1, 0, p16, p16, None, None) == -1    # T < 0
    assert qg(p16, 100, 2, p16, p16, p16, 256, 256, 32, p16, 0, 0, p16, p16, None, None) == -1   # R < 1
    bm = lib.osc_build_table_multi
    bm.argtypes = [V, I, I, I, ctypes.c_float, I, I, V, V]
    assert bm(p16, 8, 256, 32, 5.0, 5, 4, p16, None) == -1                 # R > 3
    assert bm(p16, 8, 256, 32, 5.0, 5, 0, p16, None) == -1                 # R < 1
    assert bm(p16, 8, 256, 24, 5.0, 5, 2, p16, None) == -3                 # G
    lg = lib.osc_linear_grouped
    lg.argtypes = [V, V, V, V, V, V, V, V, I, I, I, I, I, I, V, V, V]
    assert lg(p16, p16, None, p16, p16, None, p16, None, 2, 200, 256, 256, 32, 0, p16, None, None) == -2  # Mp % 128
    assert lg(p16, p16, None, p16, p16, None, None, None, 2, 256, 256, 256, 32, 0, p16, None, None) == -1  # no map
    dn = lib.osc_density
    dn.argtypes = [V, I, I, I, ctypes.c_float, V, V, V, V]
    assert dn(p16, 8, 256, 24, 5.0, p16, p16, p16, None) == -3              # G
    assert dn(p16, 8, 250, 32, 5.0, p16, p16, p16, None) == -1              # K % G
    assert dn(p16, 8, 256, 32, 5.0, None, p16, p16, None) == -1             # table required
    assert dn(V(p16.value + 2), 8, 256, 32, 5.0, p16, p16, p16, None) == -2  # alignment
    st = lib.osc_select_tier
    st.argtypes = [V, V, I, V]
    assert st(None, None, 0, None) == 2 and st(None, None, 3, None) == -1
    stt = lib.osc_selftest_timeout
    stt.argtypes = [I, V]
    assert stt(0, None) == -1 and stt(2_000_000, None) == -1                # limit out of range
    rq = lib.osc_rmsnorm_quantize
    rq.argtypes = [V, V, ctypes.c_float, I, I, I, V, I, I, V, V, V, V]
    assert rq(p16, p16, -1.0, 4, 256, 32, None, 1, 0, p16, p16, None, None) == -1       # eps < 0
    assert rq(p16, p16, float("nan"), 4, 256, 32, None, 1, 0, p16, p16, None, None) == -1
    assert rq(p16, p16, 1e-6, 4, 8192, 32, None, 1, 0, p16, p16, None, None) == -1       # K above 6144
    assert rq(p16, None, 1e-6, 4, 256, 32, None, 1, 0, p16, p16, None, None) == -1       # gamma required
    assert rq(p16, V(p16.value + 2), 1e-6, 4, 256, 32, None, 1, 0, p16, p16, None, None) == -2  # gamma alignment
    assert rq(p16, p16, 1e-6, 4, 256, 24, None, 1, 0, p16, p16, None, None) == -3        # G
    assert rq(None, None, 1e-6, 0, 256, 32, None, 1, 0, None, None, None, None) == 0     # M = 0: no-op
    assert rq(p16, p16, 1e-6, 4, 256, 32, p16, 4, 0, p16, p16, None, None) == -1         # R > 3
    sk = lib.osc_linear_splitk
    sk.argtypes = [V] * 6 + [I] * 5 + [V, V, V, ctypes.c_size_t, V]
    assert sk(p16, p16, None, p16, p16, None, 4, 128, 256, 32, 0, p16, None, None, 64, None) == -1   # bytes, no buffer
    assert sk(p16, p16, None, p16, p16, None, 4, 128, 256, 32, 0, p16, None, V(p16.value + 4), 64, None) == -2
    assert sk(p16, p16, None, p16, p16, None, 4, 100, 256, 32, 0, p16, None, p16, 64, None) == -2    # N % 16
    assert sk(None, None, None, None, None, None, 0, 128, 256, 32, 0, None, None, None, 0, None) == 0  # M = 0
    ql = lib.osc_quantize_linear
    ql.argtypes = [V, I, I, I, V, I, I, V, V, V, V, V, V, I, V, V, V, ctypes.c_size_t, V]
    assert ql(None, 0, 256, 32, None, 1, 0, None, None, None, None, None, None, 128, None, None, None, 0, None) == 0  # M = 0
    assert ql(p16, 4, 256, 24, None, 1, 0, p16, p16, None, p16, p16, None, 128, p16, None, None, 0, None) == -3  # G
    assert ql(p16, 4, 256, 32, p16, 4, 0, p16, p16, None, p16, p16, None, 128, p16, None, None, 0, None) == -1   # R > 3
    assert ql(None, 4, 256, 32, None, 1, 0, p16, p16, None, p16, p16, None, 128, p16, None, None, 0, None) == -1  # X
    assert ql(p16, 4, 256, 32, None, 1, 0, p16, p16, None, p16, p16, None, 128, None, None, None, 0, None) == -1  # Y
    assert ql(p16, 4, 256, 32, None, 1, 16, p16, p16, p16, p16, p16, p16, 128, p16, None, None, 0, None) == -1   # K_L, no table
    assert ql(p16, 4, 256, 32, p16, 1, 16, p16, p16, p16, p16, p16, None, 128, p16, None, None, 0, None) == -1   # W_L missing
    assert ql(p16, 4, 256, 32, None, 1, 0, p16, p16, None, p16, p16, None, 100, p16, None, None, 0, None) == -2  # N % 16
    assert ql(V(p16.value + 2), 4, 256, 32, None, 1, 0, p16, p16, None, p16, p16, None, 128, p16, None, None, 0, None) == -2
    rl = lib.osc_rmsnorm_quantize_linear
    rl.argtypes = [V, V, ctypes.c_float, I, I, I, V, I, I, V, V, V, V, V, V, I, V, V, V]
    assert rl(None, None, 1e-6, 0, 256, 32, None, 1, 0, None, None, None, None, None, None, 128, None, None, None) == 0
    assert rl(p16, p16, -1.0, 4, 256, 32, None, 1, 0, p16, p16, None, p16, p16, None, 128, p16, None, None) == -1
    assert rl(p16, None, 1e-6, 4, 256, 32, None, 1, 0, p16, p16, None, p16, p16, None, 128, p16, None, None) == -1
    assert rl(p16, p16, 1e-6, 4, 8192, 32, None, 1, 0, p16, p16, None, p16, p16, None, 128, p16, None, None) == -1
    assert rl(p16, p16, 1e-6, 4, 256, 24, None, 1, 0, p16, p16, None, p16, p16, None, 128, p16, None, None) == -3
    assert rl(p16, p16, 1e-6, 4, 256, 32, None, 1, 0, p16, p16, None, p16, p16, None, 100, p16, None, None) == -2
    assert ql(p16, 4, 256, 32, None, 1, 0, p16, p16, None, p16, p16, None, 128, p16, None, None, 64, None) == -1  # bytes, no buffer
    assert ql(p16, 4, 256, 32, None, 1, 0, p16, p16, None, p16, p16, None, 128, p16, None, V(p16.value + 4), 64,
              None) == -2                                                                 # workspace alignment
    wb = lib.osc_linear_workspace_bytes
    wb.argtypes = [I, I, I, I]
    wb.restype = ctypes.c_size_t
    assert wb(17, 6144, 4096, 96) == 0 and wb(16, 6144, 4000, 96) == 0                 # M > 16, K % 256
    lib.osc_set_cta_pair.argtypes = [I]
    assert lib.osc_set_cta_pair(3) == -1
    prev = lib.osc_set_cta_pair(1)
    assert lib.osc_set_cta_pair(prev) == 1


def test_scale_layout_fills_the_buffer_exactly(lib):
    """The documented scale layout maps every (row, slot) of the padded rows to a distinct byte,
    and together they cover the buffer osc_scale_bytes sizes, with no gap or overlap."""
    from tests._layout import scale_offsets
    f = lib.osc_scale_bytes
    f.restype = ctypes.c_size_t
    for rows, K, G in ((128, 256, 32), (256, 4096, 32), (384, 512, 16), (128, 1024, 64), (130, 768, 32)):
        V = 16 if G == 16 else 32
        mpad = (rows + 127) // 128 * 128
        offs = scale_offsets(mpad, K, V).reshape(-1)
        size = f(rows, K, G)
        assert np.array_equal(np.sort(offs), np.arange(size)), (rows, K, G)
