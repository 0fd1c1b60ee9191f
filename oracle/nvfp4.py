"""NVFP4 number formats and the NVFP4 block quantiser, written from their definitions.

TEST INFRASTRUCTURE ONLY. This is the slow CPU oracle that the CUDA path is
checked against. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import it; the library never does.

Source of the definitions
-------------------------
* The blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers",
  section "Native loading in Diffusers", fixes the scheme's parameters:
  precision "nvfp4", group size 16 (one scale per 16 contiguous K-elements),
  rank 32.
* The pages do not spell out NVFP4 itself. The reading used here: an element
  is an E2M1 code (1 sign, 2 exponent bits with bias 1, 1 mantissa bit, no
  Inf/NaN), each group of 16 contiguous K-elements carries one E4M3 scale
  (OCP FP8 E4M3: bias 7, no Inf, 0x7F/0xFF are NaN, max 448), and each tensor
  carries one FP32 global decode scale g. Decoded value = e2m1 * e4m3 * g.
* Rounding is round-to-nearest-even with saturation to the largest finite
  value (the ".rn.satfinite" conversions of the target ISA).

Readings where the pages are silent:
* g = fp32(amax / 2688), 2688 = 6 * 448, so the largest block of the tensor
  maps to the largest E2M1 magnitude times the largest E4M3 scale; g = 1 when
  the tensor is all zero.
* Per block: t = fp32(amax_block / fp32(6*g)); S = e4m3_rn_satfinite(t);
  sd = fp32(dec(S) * g); inv = fp32(1/sd) (0 when sd == 0);
  q = fp32(x * inv); code = e2m1_rn_satfinite(q). One reciprocal per block.
* A negative value that rounds to zero keeps its sign (code 0x8).
* Packing: byte j of a row holds element 2j in its low nibble and element
  2j+1 in its high nibble.
All float32 steps here are single IEEE-754 binary32 operations (numpy
float32 arithmetic), so each is correctly rounded.
"""
from __future__ import annotations

import numpy as np

GROUP = 16               # elements per block scale ("group_size": 16)
E2M1_MAX = 6.0
E4M3_MAX = 448.0
GLOBAL_DIVISOR = np.float32(E2M1_MAX * E4M3_MAX)   # 2688


# ---------------------------------------------------------------- E2M1 (FP4)
def e2m1_decode(code) -> np.ndarray:
    """Value of 4-bit E2M1 codes: s | e(2 bits, bias 1) | m(1 bit)."""
    c = np.asarray(code, dtype=np.int64) & 0xF
    s = (c >> 3) & 1
    e = (c >> 1) & 3
    m = c & 1
    mag = np.where(e == 0, m * 0.5, (1.0 + m * 0.5) * np.exp2(e - 1.0))
    return np.where(s == 1, -mag, mag)


_E2M1_POS = e2m1_decode(np.arange(8))            # ascending: 0 .5 1 1.5 2 3 4 6


def _nearest_even(a: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the nearest entry of an ascending table of non-negative values.

    Ties go to the even index (the code whose mantissa LSB is 0, since the
    codes here are consecutive integers starting at code 0). Values above the
    last entry saturate to it.
    """
    a = np.asarray(a, dtype=np.float64)
    hi = np.searchsorted(table, a, side="left")          # table[hi-1] < a <= table[hi]
    hi = np.clip(hi, 0, len(table) - 1)
    lo = np.clip(hi - 1, 0, len(table) - 1)
    d_lo = a - table[lo]
    d_hi = table[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(a >= table[-1], len(table) - 1, idx)
    return idx


def e2m1_encode(q) -> np.ndarray:
    """fp32 -> E2M1 code, round-to-nearest-even, saturate to +-6, sign kept."""
    q = np.asarray(q, dtype=np.float32)
    mag_code = _nearest_even(np.abs(q), _E2M1_POS)
    sign = np.signbit(q).astype(np.int64)
    return (mag_code | (sign << 3)).astype(np.uint8)


# ---------------------------------------------------------------- E4M3 (FP8)
def e4m3_decode(code) -> np.ndarray:
    """Value of OCP E4M3 codes (bias 7, subnormals, 0x7F/0xFF NaN, no Inf)."""
    c = np.asarray(code, dtype=np.int64) & 0xFF
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


_E4M3_POS = e4m3_decode(np.arange(0x7F))          # codes 0x00..0x7E, ascending


def e4m3_encode(t) -> np.ndarray:
    """fp32 -> E4M3 code, round-to-nearest-even, saturate to +-448, sign kept."""
    t = np.asarray(t, dtype=np.float32)
    mag_code = _nearest_even(np.abs(t), _E4M3_POS)
    sign = np.signbit(t).astype(np.int64)
    return (mag_code | (sign << 7)).astype(np.uint8)


# ---------------------------------------------------------------- bfloat16
def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), as float64.

    bfloat16 keeps 8 significant bits; the quantum of a value with
    frexp exponent e is 2^(e-8), never below the subnormal quantum 2^-133.
    Scaling by a power of two and np.rint (ties to even) are exact in float64.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    qe = np.maximum(e - 8, -133)
    y = np.ldexp(np.rint(np.ldexp(x, -qe)), qe)
    return np.where(np.abs(y) > 3.3895313892515355e38, np.copysign(np.inf, x), y)


def bf16_bits_to_f64(u16) -> np.ndarray:
    """uint16 bfloat16 bit patterns -> float64 (exact)."""
    u = np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- quantiser
def global_scale(a) -> np.float32:
    """Per-tensor decode scale g = fp32(amax|a| / 2688); 1 for an all-zero tensor."""
    amax = np.float32(np.max(np.abs(np.asarray(a, dtype=np.float32)))) if np.size(a) else np.float32(0)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(amax / GLOBAL_DIVISOR)


def quantize_rows(a, g) -> tuple[np.ndarray, np.ndarray]:
    """NVFP4-quantise the rows of ``a`` (float32, shape [rows, K], K % 16 == 0).

    Returns (codes uint8 [rows, K] one E2M1 code per element,
             scales uint8 [rows, K/16] one E4M3 code per block).
    """
    a = np.asarray(a, dtype=np.float32)
    rows, K = a.shape
    assert K % GROUP == 0
    g = np.float32(g)
    d = np.float32(np.float32(6.0) * g)
    blocks = a.reshape(rows, K // GROUP, GROUP)
    amax = np.max(np.abs(blocks), axis=-1)                     # exact
    t = (amax / d).astype(np.float32)                          # one fp32 divide
    S = e4m3_encode(t)
    sd = (e4m3_decode(S).astype(np.float32) * g).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(sd == 0, np.float32(0), np.float32(1.0) / sd).astype(np.float32)
    q = (blocks * inv[..., None]).astype(np.float32)
    codes = e2m1_encode(q).reshape(rows, K)
    return codes, S


def dequantize_rows(codes, scales) -> np.ndarray:
    """float64 values dec(code) * dec(S) for [rows, K] codes and [rows, K/16] scales
    (the global decode scale is not applied here)."""
    codes = np.asarray(codes)
    rows, K = codes.shape
    v = e2m1_decode(codes).reshape(rows, K // GROUP, GROUP)
    s = e4m3_decode(scales)[..., None]
    return (v * s).reshape(rows, K)


def pack_nibbles(codes) -> np.ndarray:
    """[rows, K] 4-bit codes -> [rows, K/2] bytes; element 2j in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out
