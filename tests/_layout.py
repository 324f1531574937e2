"""Test harness: turn the library's packed layouts back into logical arrays (numpy).

Not part of either implementation: it only reads bytes at the positions the C ABI documents
(include/osc.h) so that GPU outputs can be compared with the oracle's logical outputs.
"""
import numpy as np


def unpack_e2m1(q: np.ndarray, K: int) -> np.ndarray:
    """rows x K/2 bytes -> rows x K codes (even k in the low nibble)."""
    q = np.asarray(q, dtype=np.uint8).reshape(-1, K // 2)
    out = np.empty((q.shape[0], K), dtype=np.uint8)
    out[:, 0::2] = q & 0xF
    out[:, 1::2] = q >> 4
    return out


def scale_offsets(rows: int, K: int, V: int) -> np.ndarray:
    """Byte offset of (row r, slot s) in the tensor-core scale layout, rows x K/V."""
    nslot = K // V
    r = np.arange(rows)[:, None]
    s = np.arange(nslot)[None, :]
    return ((r // 128) * (nslot // 4) + s // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + s % 4


def unswizzle_scales(sbytes: np.ndarray, rows: int, K: int, V: int) -> np.ndarray:
    """Scale buffer -> rows x K/V shared exponents e (int16, byte - 127)."""
    b = np.asarray(sbytes, dtype=np.uint8).reshape(-1)
    return b[scale_offsets(rows, K, V)].astype(np.int16) - 127


def pad_rows_zero(sbytes: np.ndarray, rows: int, K: int, V: int) -> bool:
    """True if every scale byte of the rows between `rows` and the next multiple of 128 is 0."""
    mpad = (rows + 127) // 128 * 128
    if mpad == rows:
        return True
    b = np.asarray(sbytes, dtype=np.uint8).reshape(-1)
    offs = scale_offsets(mpad, K, V)[rows:]
    return bool(np.all(b[offs] == 0))


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (2^(floor(log2|x|) - 7)); subnormal floor 2^-133."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)
