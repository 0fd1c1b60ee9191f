"""The AWQ W4A16 weight-only linear layer, step by step, on the CPU.

TEST INFRASTRUCTURE ONLY: see the package docstring.

Blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers", section
"Introducing Nunchaku Lite": the second kernel family, awq_w4a16, keeps
4-bit weights with 16-bit activations for the adaptive-normalisation and
modulation projections (memory-bound, precision-sensitive layers); section
"Native loading in Diffusers" fixes its parameters: precision "int4",
group_size 64, compute dtype bfloat16.

The pages give no formulas. Readings:
* Asymmetric INT4 per output row and group of 64 contiguous K-elements, with
  the rule of the AWQ reference implementation's pseudo-quantiser: over the
  group's values w (fp32), s = bf16(fp32(max(fp32(max w - min w), 1e-5) / 15))
  is the stored scale, z = clamp(rne(fp32(-min w / s)), 0, 15) the stored
  zero point, q = clamp(rne(fp32(w / s)) + z, 0, 15) the code; every step
  one correctly rounded fp32 operation, quantising with the stored bf16 scale
  so that storing and dequantising agree.
* Dequantised weight w' = (q - z) * s, exact in fp32 (a 5-bit integer times
  an 8-bit significand).
* The activation-aware part of AWQ is an optional per-input-channel factor
  a_k: the weight quantised is fp32(w * a_k) and the activation x * fp32(1/a_k)
  (the same form as SVDQuant's smoothing); how a_k is searched is calibration
  and not part of this layer.
* Y = bf16(sum_k x^_k w'[n,k] + b[n]) with float64 accumulation here.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import nvfp4

GROUP = 64
QMAX = 15


def _f32(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64).astype(np.float32)


@dataclass
class AwqWeight:
    codes: np.ndarray      # uint8 [N, K], one 4-bit code per element
    scales: np.ndarray     # float32 [N, K/64] (bf16 values)
    zeros: np.ndarray      # uint8 [N, K/64]
    inv_act: np.ndarray | None = None   # float32 [K] = fp32(1 / a_k), or None


def quantize(W, act_scale=None) -> AwqWeight:
    """INT4 group-64 asymmetric quantisation of W [N, K] (bf16 values)."""
    w = _f32(W)
    if act_scale is not None:
        w = (w * np.asarray(act_scale, dtype=np.float32)[None, :]).astype(np.float32)
    N, K = w.shape
    g = w.reshape(N, K // GROUP, GROUP)
    mx = g.max(axis=2)
    mn = g.min(axis=2)
    d = np.maximum((mx - mn).astype(np.float32), np.float32(1e-5))
    s = nvfp4.bf16_round((d / np.float32(QMAX)).astype(np.float32)).astype(np.float32)
    z = np.clip(np.rint((-mn / s).astype(np.float32)), 0, QMAX)
    q = np.clip(np.rint((g / s[:, :, None]).astype(np.float32)) + z[:, :, None], 0, QMAX)
    inv = None
    if act_scale is not None:
        inv = (np.float32(1.0) / np.asarray(act_scale, dtype=np.float32)).astype(np.float32)
    return AwqWeight(q.reshape(N, K).astype(np.uint8), s, z.astype(np.uint8), inv)


def dequantize(aw: AwqWeight) -> np.ndarray:
    """w'[n,k] = (q - z) * s, float64 (exact)."""
    N, K = aw.codes.shape
    q = aw.codes.reshape(N, K // GROUP, GROUP).astype(np.float64)
    w = (q - aw.zeros[:, :, None].astype(np.float64)) * aw.scales[:, :, None].astype(np.float64)
    return w.reshape(N, K)


@dataclass
class AwqForward:
    y64: np.ndarray    # float64 [M, N]
    y_ref: np.ndarray  # y64 rounded to bf16


def forward(X, aw: AwqWeight, bias=None) -> AwqForward:
    """Y = X^ . W'^T + b in float64, X^ = fp32(x * inv_act[k]) (or X)."""
    x = _f32(X)
    if aw.inv_act is not None:
        x = (x * aw.inv_act[None, :]).astype(np.float32)
    y = x.astype(np.float64) @ dequantize(aw).T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return AwqForward(y, nvfp4.bf16_round(y))
