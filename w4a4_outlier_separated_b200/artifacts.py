"""Offline artifacts of one OSC layer, saved and loaded: the suppression table of Algorithm 1
(the OSC page, §3.1; the page sizes it at a few kilobytes) and the prepared weights of §3.3
(Q_W, S_W in the tensor-core scale layout, W_L).

File format, little-endian:
  header  8-byte magic b"OSCLAYR1", then uint32 version (1), G, K, N, K_L, float32 alpha,
          uint32 min_hits, uint32 kind (0 = MXFP4 with table), then uint64 byte sizes of
          L, QW, SW, WL
  body    the four arrays' raw bytes in that order (L int8, QW uint8, SW uint8, WL bf16 bits)
Loading checks the magic, the version and every size against the layer's shape (the scale
size comes from the library's osc_scale_bytes), so a file from another shape or a truncated
file is rejected instead of misread. Both directions also check the table against the layer:
entries in [-1, G) and no more entries than K_L columns hold. Host IO only: no computation
of the path happens here.
"""
from __future__ import annotations

import struct

import numpy as np
import torch

MAGIC = b"OSCLAYR1"
VERSION = 1
_HEAD = struct.Struct("<8sIIIIIfII4Q")


def _bytes_of(t: torch.Tensor) -> bytes:
    return t.detach().contiguous().cpu().view(torch.uint8).numpy().tobytes()


def expected_sizes(G: int, K: int, N: int, K_L: int) -> tuple[int, int, int, int]:
    """Byte sizes of L, QW, SW and WL for a layer of N outputs, K inputs, group size G."""
    from w4a4_outlier_separated_b200 import osc
    return K // G, N * K // 2, osc.osc_scale_bytes(N, K, G), N * K_L * 2


def check_table(L_bytes: bytes, G: int, K_L: int) -> None:
    """A table fits its layer when every entry is -1 or a channel 0..G-1 and its entries fit
    the compensation width: K_L a multiple of 16 and at least osc_table_kl(L) (the kernels
    would otherwise drop the extra entries and report OSC_ERR_TABLE at run time)."""
    from w4a4_outlier_separated_b200 import osc
    t = np.frombuffer(L_bytes, dtype=np.int8).copy()
    if t.size and (t.min() < -1 or t.max() >= G):
        raise ValueError(f"table entries must lie in [-1, {G})")
    if K_L < 0 or K_L % 16:
        raise ValueError(f"K_L = {K_L} is not a non-negative multiple of 16")
    need = osc.osc_table_kl(t)
    if need > K_L:
        raise ValueError(f"the table has entries for K_L = {need}, more than K_L = {K_L}")


def save_layer(path: str, L, QW, SW, WL, *, G: int, K: int, N: int, K_L: int,
               alpha: float = 5.0, min_hits: int = 5) -> None:
    """Write one layer's table and prepared weights (tensors on any device) to `path`."""
    parts = [_bytes_of(L), _bytes_of(QW), _bytes_of(SW), _bytes_of(WL) if K_L else b""]
    if G not in (16, 32, 64):
        raise ValueError(f"G = {G} is not 16, 32 or 64")
    want = expected_sizes(G, K, N, K_L)
    for name, got, w in zip(("L", "QW", "SW", "WL"), parts, want):
        if len(got) != w:
            raise ValueError(f"{name}: {len(got)} bytes, the layer shape needs {w}")
    check_table(parts[0], G, K_L)
    head = _HEAD.pack(MAGIC, VERSION, G, K, N, K_L, float(alpha), min_hits, 0, *[len(p) for p in parts])
    with open(path, "wb") as f:
        f.write(head)
        for p in parts:
            f.write(p)


def load_layer(path: str, device="cuda") -> dict:
    """Read a layer written by save_layer; tensors are placed on `device`."""
    with open(path, "rb") as f:
        raw = f.read()
    if len(raw) < _HEAD.size:
        raise ValueError("file too short for the header")
    magic, version, G, K, N, K_L, alpha, min_hits, kind, *sizes = _HEAD.unpack_from(raw, 0)
    if magic != MAGIC:
        raise ValueError("not an OSC layer file")
    if version != VERSION or kind != 0:
        raise ValueError(f"unsupported version {version} / kind {kind}")
    if G not in (16, 32, 64) or K <= 0 or K % G or N <= 0 or K_L < 0 or K_L % 16:
        raise ValueError("invalid layer shape in the header")
    if tuple(sizes) != expected_sizes(G, K, N, K_L):
        raise ValueError("array sizes do not match the layer shape")
    if len(raw) != _HEAD.size + sum(sizes):
        raise ValueError("file length does not match the header")
    off = _HEAD.size
    arrays = []
    for n in sizes:
        arrays.append(np.frombuffer(raw, dtype=np.uint8, count=n, offset=off).copy())
        off += n
    check_table(arrays[0].tobytes(), G, K_L)
    dev = torch.device(device)
    L = torch.from_numpy(arrays[0].view(np.int8)).to(dev)
    QW = torch.from_numpy(arrays[1]).reshape(N, K // 2).to(dev)
    SW = torch.from_numpy(arrays[2]).to(dev)
    WL = torch.from_numpy(arrays[3].view(np.int16)).reshape(N, K_L).to(dev) if K_L else None
    return dict(L=L, QW=QW, SW=SW, WL=WL, G=G, K=K, N=N, K_L=K_L, alpha=alpha, min_hits=min_hits)
