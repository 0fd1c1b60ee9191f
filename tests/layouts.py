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


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the bf16 spacing at |x| (8 significant bits): the largest error of
    rounding a real number to the nearest bf16 value x."""
    return np.ldexp(1.0, np.frexp(np.abs(np.asarray(x, dtype=np.float64)))[1] - 9)


def sum_error_bound(n_roundings: int, abs_sum, unit_roundoff: float) -> np.ndarray:
    """Higham's bound on the error of a sum evaluated with n_roundings rounded
    additions in any order (Accuracy and Stability of Numerical Algorithms,
    2nd ed., eq. 4.4): gamma_n * sum|terms| with gamma_n = n u / (1 - n u).
    Each term must be exact in the working precision (a product of two bf16
    values is exact in fp32). u = 2^-24 for round-to-nearest fp32; u = 2^-23
    covers any faithful rounding (round-toward-zero included), the guarantee
    used for the tensor cores' internal accumulation, whose rounding is not
    specified."""
    nu = n_roundings * unit_roundoff
    assert nu < 0.5
    return nu / (1.0 - nu) * np.asarray(abs_sum, dtype=np.float64)
