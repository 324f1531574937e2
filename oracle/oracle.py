"""Python face of the OSC oracle (oracle/osc_oracle.c): numpy in, numpy out.

TEST INFRASTRUCTURE ONLY. Only tests/, ``__graft_entry__.smoke()`` and the
cpu_baseline / reference leg of ``bench.py`` may import this module. The
product path never does, and shares no code with it.

Every function marshals arrays to the plain-C oracle and back; the arithmetic
lives in the C file, which cites the OSC page ("W4A4量化技术：OSC框架如何实现高效LLM部署",
coreui.cn/article/2607942.html) section by section.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "osc_oracle.c")
_LIB = os.path.join(_HERE, "liboscref.so")

FMT_E2M1 = 0
FMT_E4M3 = 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, f32 = ctypes.c_int, ctypes.c_int64, ctypes.c_float
        L.orc_build_table.argtypes = [P, i32, i32, i32, f32, i32, P]
        L.orc_density.argtypes = [P, i32, i32, i32, f32, P, P, P]
        L.orc_table_count.argtypes = [P, i32]
        L.orc_extract.argtypes = [P, i32, i32, i32, P, i32, i32, P, P]
        L.orc_gather_wl.argtypes = [P, i32, i32, i32, P, i32, i32, P]
        L.orc_build_table_multi.argtypes = [P, i32, i32, i32, f32, i32, i32, P]
        L.orc_mx_quantize.argtypes = [P, i32, i32, i32, i32, P, P]
        L.orc_mx_dequantize.argtypes = [P, P, i32, i32, i32, i32, P]
        L.orc_linear.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, P, i32, P]
        L.orc_decode_e2m1.argtypes = [ctypes.c_uint8]
        L.orc_decode_e2m1.restype = ctypes.c_double
        L.orc_decode_e4m3.argtypes = [ctypes.c_uint8]
        L.orc_decode_e4m3.restype = ctypes.c_double
        L.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_double.restype = ctypes.c_double
        L.orc_double_to_bf16.argtypes = [ctypes.c_double]
        L.orc_double_to_bf16.restype = ctypes.c_uint16
        L.orc_row_sumsq.argtypes = [P, i32]
        L.orc_row_sumsq.restype = ctypes.c_float
        L.orc_rmsnorm.argtypes = [P, i32, i32, P, f32, P, P]
        _ = (i64,)
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _chk(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


def slot_width(G: int, fmt: int = FMT_E2M1) -> int:
    """Elements per shared-exponent slot: 16 for G=16, else 32."""
    return 16 if (fmt == FMT_E2M1 and G == 16) else 32


def build_table(X: np.ndarray, G: int, alpha: float = 5.0, min_hits: int = 5) -> np.ndarray:
    """Algorithm 1 for one (position, layer): X is S x K bf16 bits -> L (int8, K/G)."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    S, K = X.shape
    L = np.empty(K // G, dtype=np.int8)
    _chk(lib().orc_build_table(_p(X), S, K, G, float(alpha), int(min_hits), _p(L)), "build_table")
    return L


def build_table_multi(X: np.ndarray, G: int, R: int, alpha: float = 5.0, min_hits: int = 5) -> np.ndarray:
    """Up to R protected channels per group: K/G x R int8 (slot r from round r of Algorithm 1
    on the calibration rows with the earlier rounds' channels zeroed)."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    S, K = X.shape
    L = np.empty((K // G, R), dtype=np.int8)
    _chk(lib().orc_build_table_multi(_p(X), S, K, G, float(alpha), int(min_hits), int(R), _p(L)),
         "build_table_multi")
    return L


def _table_shape(L: np.ndarray, K: int, G: int):
    """A table as K/G entries (one per group) or K/G x R entries: (flat int8 array, R)."""
    L = np.ascontiguousarray(L, dtype=np.int8)
    R = 1 if L.ndim == 1 else L.shape[1]
    if L.size != (K // G) * R:
        raise ValueError("table size does not match K / G")
    return L.reshape(-1), R


def density(X: np.ndarray, G: int, L: np.ndarray, alpha: float = 5.0):
    """Per-group (N_hit, N_total) of the clustering density C_k = N_hit / N_total."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    L = np.ascontiguousarray(L, dtype=np.int8)
    S, K = X.shape
    nh = np.zeros(K // G, dtype=np.int64)
    nt = np.zeros(K // G, dtype=np.int64)
    _chk(lib().orc_density(_p(X), S, K, G, float(alpha), _p(L), _p(nh), _p(nt)), "density")
    return nh, nt


def table_count(L: np.ndarray) -> int:
    """Number of table entries >= 0 (any table shape)."""
    L = np.ascontiguousarray(L, dtype=np.int8).reshape(-1)
    return int(lib().orc_table_count(_p(L), L.size))


def extract(X: np.ndarray, G: int, L: np.ndarray, K_L: int):
    """Outlier extraction: returns (X with table slots zeroed, B as M x K_L bf16 bits). L is
    one entry per group (K/G) or K/G x R entries (columns of B in group, slot order)."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    M, K = X.shape
    Lf, R = _table_shape(L, K, G)
    Xz = np.empty_like(X)
    B = np.empty((M, K_L), dtype=np.uint16)
    _chk(lib().orc_extract(_p(X), M, K, G, _p(Lf), R, K_L, _p(Xz), _p(B)), "extract")
    return Xz, B


def gather_wl(W: np.ndarray, G: int, L: np.ndarray, K_L: int) -> np.ndarray:
    """W_L: N x K_L bf16 bits, the weight columns of the table's channels."""
    W = np.ascontiguousarray(W, dtype=np.uint16)
    N, K = W.shape
    Lf, R = _table_shape(L, K, G)
    WL = np.empty((N, K_L), dtype=np.uint16)
    _chk(lib().orc_gather_wl(_p(W), N, K, G, _p(Lf), R, K_L, _p(WL)), "gather_wl")
    return WL


def mx_quantize(X: np.ndarray, G: int, fmt: int = FMT_E2M1):
    """MX quantization: returns (codes rows x K uint8, exps rows x K/V int16)."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    rows, K = X.shape
    V = slot_width(G, fmt)
    codes = np.empty((rows, K), dtype=np.uint8)
    exps = np.empty((rows, K // V), dtype=np.int16)
    _chk(lib().orc_mx_quantize(_p(X), rows, K, G, fmt, _p(codes), _p(exps)), "mx_quantize")
    return codes, exps


def mx_dequantize(codes: np.ndarray, exps: np.ndarray, fmt: int = FMT_E2M1) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    exps = np.ascontiguousarray(exps, dtype=np.int16)
    rows, K = codes.shape
    V = K // exps.shape[1]
    out = np.empty((rows, K), dtype=np.float64)
    _chk(lib().orc_mx_dequantize(_p(codes), _p(exps), rows, K, V, fmt, _p(out)), "mx_dequantize")
    return out


def linear(cx, ex, cw, ew, B, WL, fmt: int = FMT_E2M1, rows=None) -> np.ndarray:
    """Y = (Q_X (x) Q_W) * S + B * W_L in fp64 for the selected rows (all if None)."""
    cx = np.ascontiguousarray(cx, dtype=np.uint8)
    cw = np.ascontiguousarray(cw, dtype=np.uint8)
    ex = np.ascontiguousarray(ex, dtype=np.int16)
    ew = np.ascontiguousarray(ew, dtype=np.int16)
    M, K = cx.shape
    N = cw.shape[0]
    V = K // ex.shape[1]
    K_L = 0 if B is None else int(B.shape[1])
    if K_L:
        B = np.ascontiguousarray(B, dtype=np.uint16)
        WL = np.ascontiguousarray(WL, dtype=np.uint16)
        pB, pWL = _p(B), _p(WL)
    else:
        pB = pWL = None
    if rows is None:
        r_arr, nr, pr = None, M, None
    else:
        r_arr = np.ascontiguousarray(rows, dtype=np.int32)
        nr, pr = r_arr.size, _p(r_arr)
    Y = np.empty((nr, N), dtype=np.float64)
    _chk(lib().orc_linear(_p(cx), _p(ex), _p(cw), _p(ew), pB, pWL, M, N, K, V, fmt, K_L,
                          pr, nr, _p(Y)), "linear")
    return Y


def decode_e2m1(code: int) -> float:
    return float(lib().orc_decode_e2m1(code))


def decode_e4m3(code: int) -> float:
    return float(lib().orc_decode_e4m3(code))


def bf16_to_double(h: int) -> float:
    return float(lib().orc_bf16_to_double(h))


def double_to_bf16(x: float) -> int:
    return int(lib().orc_double_to_bf16(x))


def to_bf16_array(Y: np.ndarray) -> np.ndarray:
    """Round each fp64 value to bf16 (ties to even), element by element."""
    f = lib().orc_double_to_bf16
    out = np.empty(Y.shape, dtype=np.uint16)
    flat_in, flat_out = Y.reshape(-1), out.reshape(-1)
    for i in range(flat_in.size):
        flat_out[i] = f(float(flat_in[i]))
    return out


def row_sumsq(x: np.ndarray) -> float:
    """fp32 sum of squares of one bf16 row, in the order the RMSNorm reading fixes."""
    x = np.ascontiguousarray(x, dtype=np.uint16).reshape(-1)
    return float(lib().orc_row_sumsq(_p(x), x.size))


def rmsnorm(X: np.ndarray, gamma: np.ndarray, eps: float = 1e-6):
    """RMSNorm of each row (the producer step before the quantize): returns (Y bf16 bits,
    inv_rms fp32 per row)."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    gamma = np.ascontiguousarray(gamma, dtype=np.uint16).reshape(-1)
    M, K = X.shape
    Y = np.empty_like(X)
    inv = np.empty(M, dtype=np.float32)
    _chk(lib().orc_rmsnorm(_p(X), M, K, _p(gamma), float(eps), _p(Y), _p(inv)), "rmsnorm")
    return Y, inv


# ---- the whole OSC layer, step by step -----------------------------------------

def osc_prepare_weight(W: np.ndarray, G: int, L: np.ndarray, K_L: int):
    """Offline weight side (§3.3 'zero-overhead weight preprocessing'): W is quantized along K
    with no table (its outlier columns stay and meet zeroed activations), and W_L is gathered."""
    cw, ew = mx_quantize(W, G, FMT_E2M1)
    WL = gather_wl(W, G, L, K_L)
    return cw, ew, WL


def osc_forward(X: np.ndarray, G: int, L: np.ndarray, K_L: int, cw, ew, WL, rows=None):
    """Online path (§3.2): extract + zero, microscale the zeroed tensor, dual-path product."""
    Xz, B = extract(X, G, L, K_L)
    cx, ex = mx_quantize(Xz, G, FMT_E2M1)
    Y = linear(cx, ex, cw, ew, B if K_L else None, WL if K_L else None, FMT_E2M1, rows)
    return dict(Xz=Xz, B=B, cx=cx, ex=ex, Y=Y)


def rmsnorm_osc_forward(X: np.ndarray, gamma: np.ndarray, eps: float, G: int, L: np.ndarray, K_L: int,
                        cw, ew, WL, rows=None):
    """The producer-fused input side: RMSNorm, then the online OSC path on its output."""
    Yn, _ = rmsnorm(X, gamma, eps)
    out = osc_forward(Yn, G, L, K_L, cw, ew, WL, rows)
    out["Xn"] = Yn
    return out


def fp8_forward(X: np.ndarray, W: np.ndarray, rows=None):
    """Fallback (§4): no separation; X and W both MXFP8 (E4M3, 32-blocks)."""
    cx, ex = mx_quantize(X, 32, FMT_E4M3)
    cw, ew = mx_quantize(W, 32, FMT_E4M3)
    Y = linear(cx, ex, cw, ew, None, None, FMT_E4M3, rows)
    return dict(cx=cx, ex=ex, cw=cw, ew=ew, Y=Y)
