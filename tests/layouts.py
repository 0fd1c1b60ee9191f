"""Test-side readers of the library's documented byte layouts (include/svdq.h).

Written from the header's layout description, independently of both the
CUDA code and the oracle; tests/test_abi.py checks it against the library's
own svdq_scale_offset.
"""
import numpy as np


def scale_offsets(rows: int, K: int) -> np.ndarray:
    """[rows, K/16] int64 byte offsets of each (row, kblock) scale in the tiled layout."""
    r = np.arange(rows, dtype=np.int64)[:, None]
    kb = np.arange(K // 16, dtype=np.int64)[None, :]
    atom = (r // 128) * (K // 64) + kb // 4
    rr = r % 128
    return atom * 512 + (rr % 32) * 16 + (rr // 32) * 4 + kb % 4


def untile_scales(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Tiled scale bytes -> [rows, K/16] uint8 in plain row-major order."""
    return np.asarray(buf, dtype=np.uint8)[scale_offsets(rows, K)]


def unpack_codes(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    """[rows][K/2] packed bytes -> [rows, K] 4-bit codes (element 2j = low nibble of byte j)."""
    b = np.asarray(buf, dtype=np.uint8).reshape(rows, K // 2)
    out = np.empty((rows, K), dtype=np.uint8)
    out[:, 0::2] = b & 0xF
    out[:, 1::2] = b >> 4
    return out


def bf16_ulp_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """|ordinal(a) - ordinal(b)| for float64 arrays holding bf16 values."""
    def ordinal(x):
        u = (np.asarray(x, dtype=np.float64).astype(np.float32).view(np.uint32) >> 16).astype(np.int64)
        return np.where(u & 0x8000, 0x8000 - u, u)
    return np.abs(ordinal(a) - ordinal(b))
