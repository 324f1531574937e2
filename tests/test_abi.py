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
    lib.osc_quantize.argtypes = [V, ctypes.c_int, ctypes.c_int, ctypes.c_int, V, ctypes.c_int, V, V, V, V]
    assert lib.osc_quantize(p16, 4, 256, 24, None, 0, p16, p16, None, None) == -3          # G
    assert lib.osc_quantize(None, 4, 256, 32, None, 0, p16, p16, None, None) == -1         # null
    assert lib.osc_quantize(p16, 4, 200, 32, None, 0, p16, p16, None, None) == -2          # K % 256
    assert lib.osc_quantize(V(p16.value + 2), 4, 256, 32, None, 0, p16, p16, None, None) == -2  # alignment
    assert lib.osc_quantize(p16, 4, 256, 32, None, 16, p16, p16, p16, None) == -1          # K_L without table
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
