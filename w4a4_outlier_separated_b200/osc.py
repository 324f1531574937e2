"""Thin Python binding of libosc.so (the C ABI declared in include/osc.h).

Argument marshalling only: every step of the OSC path runs in the library's sm_100a kernels.
Tensors are PyTorch CUDA tensors; the current torch stream is used unless one is given.
The library must exist (``python -m w4a4_outlier_separated_b200.build``); there is no fallback.

Names follow the C ABI; ``alloc_*`` helpers allocate the output tensors of a call with torch.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libosc.so")

OSC_OK = 0
ERRORS = {-1: "OSC_ERR_ARG", -2: "OSC_ERR_ALIGN", -3: "OSC_ERR_G", -4: "OSC_ERR_CUDA",
          -5: "OSC_ERR_TIMEOUT", -6: "OSC_ERR_TABLE", -7: "OSC_ERR_DEVICE",
          -8: "OSC_ERR_SCRATCH"}


class OSCError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str, cuda_err: int = 0):
        super().__init__(f"{fn}: {ERRORS.get(code, code)} ({msg})" + (f", cudaError {cuda_err}" if cuda_err else ""))
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    """Load libosc.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"libosc.so not found at {_LIB_PATH}: build it with "
                              "`python -m w4a4_outlier_separated_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        P, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        sig = {
            "osc_version": ([], ctypes.c_char_p),
            "osc_error_string": ([i32], ctypes.c_char_p),
            "osc_last_cuda_error": ([], i32),
            "osc_scale_bytes": ([i32, i32, i32], ctypes.c_size_t),
            "osc_table_kl": ([P, i32], i32),
            "osc_build_table": ([P, i32, i32, i32, f32, i32, P, P], i32),
            "osc_build_table_multi": ([P, i32, i32, i32, f32, i32, i32, P, P], i32),
            "osc_density": ([P, i32, i32, i32, f32, P, P, P, P], i32),
            "osc_select_tier": ([P, P, i32, P], i32),
            "osc_select_group_size": ([P, P], i32),
            "osc_quantize": ([P, i32, i32, i32, P, i32, i32, P, P, P, P], i32),
            "osc_rmsnorm_quantize": ([P, P, f32, i32, i32, i32, P, i32, i32, P, P, P, P], i32),
            "osc_prepare_weight": ([P, i32, i32, i32, P, i32, i32, P, P, P, P], i32),
            "osc_linear": ([P, P, P, P, P, P, i32, i32, i32, i32, i32, P, P, P], i32),
            "osc_quantize_linear": ([P, i32, i32, i32, P, i32, i32, P, P, P, P, P, P, i32, P, P, P, ctypes.c_size_t, P],
                                    i32),
            "osc_rmsnorm_quantize_linear": ([P, P, f32, i32, i32, i32, P, i32, i32, P, P, P, P, P, P, i32, P, P, P],
                                            i32),
            "osc_linear_workspace_bytes": ([i32, i32, i32, i32], ctypes.c_size_t),
            "osc_linear_splitk": ([P, P, P, P, P, P, i32, i32, i32, i32, i32, P, P, P, ctypes.c_size_t, P], i32),
            "osc_linear_splitk_noalloc": ([P, P, P, P, P, P, i32, i32, i32, i32, i32, P, P, P], i32),
            "osc_quantize_fp8": ([P, i32, i32, P, P, P], i32),
            "osc_linear_fp8_fallback": ([P, P, P, P, i32, i32, i32, P, P, P], i32),
            "osc_grouped_plan": ([P, i32, P, P, P, i32], i32),
            "osc_quantize_grouped": ([P, i32, i32, P, P, P, i32, i32, i32, P, i32, i32, P, P, P, P], i32),
            "osc_linear_grouped": ([P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, P, P, P], i32),
            "osc_status": ([P, P], i32),
            "osc_selftest_timeout": ([i32, P], i32),
            "osc_set_tile_n": ([i32], i32),
            "osc_set_cta_pair": ([i32], i32),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(name: str, rc: int):
    if rc != OSC_OK:
        L = lib()
        raise OSCError(name, rc, L.osc_error_string(rc).decode(), L.osc_last_cuda_error())


# ---- sizes --------------------------------------------------------------------------------

def osc_scale_bytes(rows: int, K: int, G: int) -> int:
    return int(lib().osc_scale_bytes(rows, K, G))


def osc_table_kl(L) -> int:
    """K_L for a table (numpy int8 array or CPU tensor)."""
    t = torch.as_tensor(L, dtype=torch.int8).contiguous().cpu()
    rc = lib().osc_table_kl(ctypes.c_void_p(t.data_ptr()), t.numel())
    if rc < 0:
        _check("osc_table_kl", rc)
    return int(rc)


def osc_set_tile_n(bn: int) -> int:
    return int(lib().osc_set_tile_n(bn))


def osc_set_cta_pair(mode: int) -> int:
    return int(lib().osc_set_cta_pair(mode))


# ---- raw calls (outputs given) -----------------------------------------------------------------

def osc_build_table(Xcal, G: int, alpha: float, min_hits: int, L, stream=None):
    S, K = Xcal.shape
    _check("osc_build_table", lib().osc_build_table(_ptr(Xcal), S, K, G, alpha, min_hits, _ptr(L), _stream(stream)))


def osc_build_table_multi(Xcal, G: int, alpha: float, min_hits: int, R: int, L, stream=None):
    """Up to R protected channels per group into L (int8 CUDA tensor of K/G x R entries)."""
    S, K = Xcal.shape
    _check("osc_build_table_multi", lib().osc_build_table_multi(_ptr(Xcal), S, K, G, alpha, min_hits, R, _ptr(L),
                                                                _stream(stream)))


def _slots(L, groups: int) -> int:
    """Protected channels per group of a table tensor holding `groups` groups (1 without one)."""
    if L is None:
        return 1
    if L.numel() % groups:
        raise ValueError("table size is not a multiple of the group count")
    return L.numel() // groups


def osc_density(X, G: int, alpha: float, L, n_hit, n_total, stream=None):
    """Per-group outlier-event and table-hit counts (int32 CUDA tensors of K/G entries)."""
    S, K = X.shape
    _check("osc_density", lib().osc_density(_ptr(X), S, K, G, alpha, _ptr(L), _ptr(n_hit), _ptr(n_total),
                                            _stream(stream)))


TIERS = {0: "fp8_fallback", 1: "mid", 2: "high"}


def osc_select_tier(n_hit, n_total):
    """Host counts (numpy or CPU tensors) -> (tier code, C-bar). The tier codes are those of
    include/osc.h: 0 = MXFP8 fallback, 1 = mid, 2 = high clustering."""
    h = torch.as_tensor(n_hit, dtype=torch.int32).contiguous().cpu()
    t = torch.as_tensor(n_total, dtype=torch.int32).contiguous().cpu()
    if h.numel() != t.numel():
        raise ValueError("n_hit and n_total differ in length")
    c = ctypes.c_double(0.0)
    rc = lib().osc_select_tier(ctypes.c_void_p(h.data_ptr()), ctypes.c_void_p(t.data_ptr()), h.numel(),
                               ctypes.byref(c))
    if rc < 0:
        _check("osc_select_tier", rc)
    return int(rc), float(c.value)


def osc_select_group_size(c_bar16: float, c_bar32: float, c_bar64: float):
    """(G, tier) for one module from its C-bar at G = 16, 32, 64; G = 0 means the MXFP8
    fallback. Host logic of the library (include/osc.h)."""
    arr = (ctypes.c_double * 3)(c_bar16, c_bar32, c_bar64)
    tier = ctypes.c_int(0)
    g = lib().osc_select_group_size(arr, ctypes.byref(tier))
    if g < 0:
        _check("osc_select_group_size", g)
    return int(g), int(tier.value)


def osc_quantize(X, G: int, L, K_L: int, QX, SX, B, stream=None):
    M, K = X.shape
    _check("osc_quantize", lib().osc_quantize(_ptr(X), M, K, G, _ptr(L), _slots(L, K // G), K_L, _ptr(QX), _ptr(SX),
                                              _ptr(B) if K_L else None, _stream(stream)))


def osc_rmsnorm_quantize(X, gamma, eps: float, G: int, L, K_L: int, QX, SX, B, stream=None):
    M, K = X.shape
    _check("osc_rmsnorm_quantize", lib().osc_rmsnorm_quantize(_ptr(X), _ptr(gamma), eps, M, K, G, _ptr(L),
                                                              _slots(L, K // G), K_L,
                                                              _ptr(QX), _ptr(SX), _ptr(B) if K_L else None,
                                                              _stream(stream)))


def osc_prepare_weight(W, G: int, L, K_L: int, QW, SW, WL, stream=None):
    N, K = W.shape
    _check("osc_prepare_weight", lib().osc_prepare_weight(_ptr(W), N, K, G, _ptr(L), _slots(L, K // G), K_L,
                                                          _ptr(QW), _ptr(SW),
                                                          _ptr(WL) if K_L else None, _stream(stream)))


def osc_linear(QX, SX, B, QW, SW, WL, M: int, N: int, K: int, G: int, K_L: int, Y, Yf32=None, stream=None):
    _check("osc_linear", lib().osc_linear(_ptr(QX), _ptr(SX), _ptr(B) if K_L else None, _ptr(QW), _ptr(SW),
                                          _ptr(WL) if K_L else None, M, N, K, G, K_L, _ptr(Y), _ptr(Yf32),
                                          _stream(stream)))


def osc_quantize_linear(X, G: int, L, K_L: int, QX, SX, B, QW, SW, WL, N: int, Y, Yf32=None, workspace=None,
                        stream=None):
    """osc_quantize then osc_linear (or, with a workspace, osc_linear_splitk) in one call: the
    product may stream its weights while the quantize finishes; same outputs as the two calls.
    `workspace`: a CUDA tensor (any dtype) for the split's fp32 partials, or None."""
    M, K = X.shape
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("osc_quantize_linear", lib().osc_quantize_linear(
        _ptr(X), M, K, G, _ptr(L), _slots(L, K // G), K_L, _ptr(QX), _ptr(SX), _ptr(B) if K_L else None,
        _ptr(QW), _ptr(SW), _ptr(WL) if K_L else None, N, _ptr(Y), _ptr(Yf32), _ptr(workspace), nbytes,
        _stream(stream)))


def osc_rmsnorm_quantize_linear(X, gamma, eps: float, G: int, L, K_L: int, QX, SX, B, QW, SW, WL, N: int, Y,
                                Yf32=None, stream=None):
    """osc_rmsnorm_quantize then osc_linear in one call; same outputs as the two calls."""
    M, K = X.shape
    _check("osc_rmsnorm_quantize_linear", lib().osc_rmsnorm_quantize_linear(
        _ptr(X), _ptr(gamma), eps, M, K, G, _ptr(L), _slots(L, K // G), K_L, _ptr(QX), _ptr(SX),
        _ptr(B) if K_L else None, _ptr(QW), _ptr(SW), _ptr(WL) if K_L else None, N, _ptr(Y), _ptr(Yf32),
        _stream(stream)))


def osc_linear_workspace_bytes(M: int, N: int, K: int, K_L: int) -> int:
    """Bytes of fp32 partials osc_linear_splitk needs on the current device (0: no split)."""
    return int(lib().osc_linear_workspace_bytes(M, N, K, K_L))


def osc_linear_splitk(QX, SX, B, QW, SW, WL, M: int, N: int, K: int, G: int, K_L: int, Y, workspace, Yf32=None,
                      stream=None):
    """osc_linear for few token rows with the K range of each weight tile split over several SMs;
    `workspace` is a CUDA tensor (any dtype) whose bytes hold the fp32 partials."""
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("osc_linear_splitk", lib().osc_linear_splitk(_ptr(QX), _ptr(SX), _ptr(B) if K_L else None, _ptr(QW),
                                                        _ptr(SW), _ptr(WL) if K_L else None, M, N, K, G, K_L,
                                                        _ptr(Y), _ptr(Yf32), _ptr(workspace), nbytes,
                                                        _stream(stream)))


def osc_linear_splitk_noalloc(QX, SX, B, QW, SW, WL, M: int, N: int, K: int, G: int, K_L: int, Y, Yf32=None,
                              stream=None):
    """osc_linear_splitk with the partials in the library's fixed device buffer (no workspace):
    for callers that cannot allocate device memory."""
    _check("osc_linear_splitk_noalloc", lib().osc_linear_splitk_noalloc(
        _ptr(QX), _ptr(SX), _ptr(B) if K_L else None, _ptr(QW), _ptr(SW), _ptr(WL) if K_L else None,
        M, N, K, G, K_L, _ptr(Y), _ptr(Yf32), _stream(stream)))


def osc_quantize_fp8(X, QX8, SX, stream=None):
    M, K = X.shape
    _check("osc_quantize_fp8", lib().osc_quantize_fp8(_ptr(X), M, K, _ptr(QX8), _ptr(SX), _stream(stream)))


def osc_linear_fp8_fallback(QX8, SX, QW8, SW, M: int, N: int, K: int, Y, Yf32=None, stream=None):
    _check("osc_linear_fp8_fallback", lib().osc_linear_fp8_fallback(_ptr(QX8), _ptr(SX), _ptr(QW8), _ptr(SW), M, N, K,
                                                                    _ptr(Y), _ptr(Yf32), _stream(stream)))


def osc_grouped_plan(counts):
    """Per-expert token counts -> (off, poff, mblock_expert) as int32 CPU tensors."""
    c = torch.as_tensor(counts, dtype=torch.int32).contiguous().cpu()
    E = c.numel()
    off = torch.empty(E + 1, dtype=torch.int32)
    poff = torch.empty(E + 1, dtype=torch.int32)
    mp = lib().osc_grouped_plan(ctypes.c_void_p(c.data_ptr()), E, ctypes.c_void_p(off.data_ptr()),
                                ctypes.c_void_p(poff.data_ptr()), None, 0)
    if mp < 0:
        _check("osc_grouped_plan", mp)
    mbe = torch.empty(max(mp // 128, 1), dtype=torch.int32)
    rc = lib().osc_grouped_plan(ctypes.c_void_p(c.data_ptr()), E, ctypes.c_void_p(off.data_ptr()),
                                ctypes.c_void_p(poff.data_ptr()), ctypes.c_void_p(mbe.data_ptr()), mbe.numel())
    if rc < 0:
        _check("osc_grouped_plan", rc)
    return off, poff, mbe[: mp // 128]


def osc_quantize_grouped(X, E: int, off, poff, mblock_expert, Mp: int, G: int, L, K_L: int, QX, SX, B, stream=None):
    T, K = X.shape
    _check("osc_quantize_grouped", lib().osc_quantize_grouped(_ptr(X), T, E, _ptr(off), _ptr(poff), _ptr(mblock_expert),
                                                              Mp, K, G, _ptr(L), _slots(L, E * (K // G)), K_L,
                                                              _ptr(QX), _ptr(SX),
                                                              _ptr(B) if K_L else None, _stream(stream)))


def osc_linear_grouped(QX, SX, B, QW, SW, WL, mblock_expert, kl, E: int, Mp: int, N: int, K: int, G: int, K_L: int,
                       Y, Yf32=None, stream=None):
    _check("osc_linear_grouped", lib().osc_linear_grouped(_ptr(QX), _ptr(SX), _ptr(B) if K_L else None, _ptr(QW),
                                                          _ptr(SW), _ptr(WL) if K_L else None, _ptr(mblock_expert),
                                                          _ptr(kl), E, Mp, N, K, G, K_L, _ptr(Y), _ptr(Yf32),
                                                          _stream(stream)))


def osc_selftest_timeout(limit_us: int = 10000, stream=None):
    """Launch the failure-detection self-test: a bounded wait that runs out after limit_us."""
    _check("osc_selftest_timeout", lib().osc_selftest_timeout(limit_us, _stream(stream)))


def osc_status(stream=None):
    """(code, raw device word); reads and clears the device status word (synchronizes)."""
    raw = ctypes.c_int(0)
    rc = lib().osc_status(ctypes.byref(raw), _stream(stream))
    return int(rc), int(raw.value)


# ---- allocation helpers ------------------------------------------------------------------------

def alloc_quantize_outputs(M: int, K: int, G: int, K_L: int, device="cuda", fp8: bool = False):
    dev = torch.device(device)
    QX = torch.empty((M, K if fp8 else K // 2), dtype=torch.uint8, device=dev)
    SX = torch.empty(osc_scale_bytes(M, K, 0 if fp8 else G), dtype=torch.uint8, device=dev)
    B = torch.empty((M, K_L), dtype=torch.int16, device=dev) if K_L else None
    return QX, SX, B


def quantize(X, G: int, L=None, K_L: int = 0, stream=None):
    """X (bf16 or int16 bits, M x K) -> (QX, SX, B)."""
    M, K = X.shape
    QX, SX, B = alloc_quantize_outputs(M, K, G, K_L, X.device)
    osc_quantize(X, G, L, K_L, QX, SX, B, stream)
    return QX, SX, B


def rmsnorm_quantize(X, gamma, eps: float, G: int, L=None, K_L: int = 0, stream=None):
    """X (M x K) and gamma (K) -> (QX, SX, B) of the normalized rows."""
    M, K = X.shape
    QX, SX, B = alloc_quantize_outputs(M, K, G, K_L, X.device)
    osc_rmsnorm_quantize(X, gamma, eps, G, L, K_L, QX, SX, B, stream)
    return QX, SX, B


def prepare_weight(W, G: int, L=None, K_L: int = 0, stream=None):
    N, K = W.shape
    QW, SW, _ = alloc_quantize_outputs(N, K, G, 0, W.device)
    WL = torch.empty((N, K_L), dtype=torch.int16, device=W.device) if K_L else None
    osc_prepare_weight(W, G, L, K_L, QW, SW, WL, stream)
    return QW, SW, WL


def linear(QX, SX, B, QW, SW, WL, M: int, N: int, K: int, G: int, K_L: int, want_f32: bool = False, stream=None):
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=QX.device)
    Yf = torch.empty((M, N), dtype=torch.float32, device=QX.device) if want_f32 else None
    osc_linear(QX, SX, B, QW, SW, WL, M, N, K, G, K_L, Y, Yf, stream)
    return Y, Yf
