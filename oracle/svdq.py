"""The SVDQuant W4A4 linear layer, step by step, on the CPU in float64.

TEST INFRASTRUCTURE ONLY: see the package docstring.

The layer (blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers",
section "Background: SVDQuant and Nunchaku"): outliers are first moved into
the weights, the hardest part of each weight matrix is kept in a small
16-bit low-rank branch, and the remaining residual is quantised to 4 bits;
activations are quantised to 4 bits on the fly (section "Introducing Nunchaku
Lite": 4-bit weights and activations). Written as one formula:

    Y = (X . L1) . L2  +  Q4(X) . Q4(R)^T  +  b,    R = W - (L1 . L2)^T

with L1: K x r and L2: r x N in bfloat16 (the figure caption in that section:
the down projection X.L1 is fused with the activation quantiser, the up
projection (X.L1).L2 with the 4-bit GEMM).

Smoothing ("moving activation outliers into the weights", same section) is a
per-input-channel factor lambda: the 4-bit branch sees X^ = X diag(1/lambda)
and W^ = W diag(lambda), so X^ W^T = X W^T. lambda = 1 (smooth=None) is
exactly the formula above. With smoothing the low-rank factors approximate
W^T scaled by lambda, and L1 is stored with 1/lambda folded in, so the
16-bit branch reads the raw X: X . L1 = X^ . (U_r S_r).

Functions, in the order the method applies them:
  smooth_factors    lambda from channel amaxima       (calibration)
  lowrank_factors   truncated SVD of W^T             (load time)
  residual          R = W - (L1 L2)^T                 (load time)
  pack_weight       NVFP4 of R, its global scale      (load time)
  quantize_act      NVFP4 of X                        (every call)
  down_proj         XL1 = bf16(X . L1)                (every call)
  forward           Y                                  (every call)
  qkv_norm_rope     per-head RMSNorm of Q and K and rotary embedding on a
                    fused QKV output (section "Quantizing models with
                    structural rewrites": the fused operator consumes the QKV
                    projection, the Q/K normalisation and the rotary embedding
                    together)
  mlp_pair          up projection, GELU, down projection (section
                    "Introducing Nunchaku Lite" names the full engine's fused
                    GELU / MLP kernels)
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import nvfp4


def to_f64(t) -> np.ndarray:
    """A CPU tensor (any float dtype, bf16 included) or array -> float64 array, exactly."""
    if isinstance(t, torch.Tensor):
        return t.detach().to(torch.float64).cpu().numpy()
    return np.asarray(t, dtype=np.float64)


# ------------------------------------------------------------------ load time
def smooth_factors(X, W, alpha: float = 0.5) -> np.ndarray:
    """Per-input-channel smoothing factors (calibration), float32 [K]:
    lambda_k = amax_m|X[m,k]|^alpha / amax_n|W[n,k]|^(1-alpha), in float64,
    clamped to [2^-32, 2^32] and rounded once to fp32 (alpha = 0.5:
    sqrt(ax) / sqrt(aw), each step correctly rounded); lambda_k = 1 where
    either amax is 0. alpha is taken as an fp32 value. The pages say only that
    outliers move into the weights; this is SmoothQuant's rule (Xiao et al.
    2023), which balances the two channel ranges."""
    alpha = float(np.float32(alpha))
    ax = np.max(np.abs(to_f64(X)), axis=0)
    aw = np.max(np.abs(to_f64(W)), axis=0)
    lam = np.ones(ax.shape, dtype=np.float64)
    ok = (ax > 0) & (aw > 0)
    if alpha == 0.5:
        lam[ok] = np.sqrt(ax[ok]) / np.sqrt(aw[ok])
    else:
        lam[ok] = ax[ok] ** alpha / aw[ok] ** (1.0 - alpha)
    lam[ok] = np.clip(lam[ok], 2.0 ** -32, 2.0 ** 32)
    return lam.astype(np.float32)


def inv_smooth(lam) -> np.ndarray:
    """fp32(1 / lambda), the factor the activation quantiser applies."""
    return (np.float32(1.0) / np.asarray(lam, dtype=np.float32)).astype(np.float32)


def lowrank_factors(W, r: int, smooth=None):
    """Rank-r factors of W^T (K x N) from a float64 SVD.

    W^T = U diag(s) V^T; L1 = bf16(U_r diag(s_r)) (K x r), L2 = bf16(V_r^T)
    (r x N). The pages do not say how the singular values are split between
    the factors; any split is valid because everything downstream uses these
    exact bf16 factors. With smoothing (lambda = smooth) the SVD is of
    diag(lambda) W^T and L1 = bf16(diag(1/lambda) U_r diag(s_r)), the
    division in float64. Returns (L1, L2, s) with s all singular values
    (float64) of the matrix decomposed.
    """
    Wt = to_f64(W).T
    if smooth is not None:
        Wt = Wt * to_f64(smooth)[:, None]
    U, s, Vt = np.linalg.svd(Wt, full_matrices=False)
    L1 = U[:, :r] * s[:r]
    if smooth is not None:
        L1 = L1 / to_f64(smooth)[:, None]
    return nvfp4.bf16_round(L1), nvfp4.bf16_round(Vt[:r, :]), s


def residual(W, L1, L2, smooth=None) -> np.ndarray:
    """R[n,k] = W[n,k] - sum_j L1[k,j] L2[j,n], float64, j ascending, then fp32 RN.

    Each product of two bf16 numbers is exact in float64; the running sum is
    rounded after each addition in the stated order, so the result is fully
    determined. With smoothing the float64 difference is multiplied by
    lambda_k (one more float64 rounding) before the fp32 rounding: the
    residual of W^ = W diag(lambda) against the folded factors.
    """
    W = to_f64(W)
    L1 = to_f64(L1)
    L2 = to_f64(L2)
    s = np.zeros_like(W)
    for j in range(L1.shape[1]):
        s += np.outer(L2[j, :], L1[:, j])
    d = W - s
    if smooth is not None:
        d = d * to_f64(smooth)[None, :]
    return d.astype(np.float32)


@dataclass
class PackedWeight:
    codes: np.ndarray    # uint8 [N, K] one E2M1 code per element
    scales: np.ndarray   # uint8 [N, K/16] E4M3 block scales
    g_w: np.float32      # global decode scale of R
    L1: np.ndarray       # float64 [K, r] (bf16 values)
    L2: np.ndarray       # float64 [r, N] (bf16 values)
    inv_smooth: np.ndarray | None = None   # float32 [K] = fp32(1/lambda), or None


def pack_weight(W, L1, L2, smooth=None) -> PackedWeight:
    R = residual(W, L1, L2, smooth)
    g_w = nvfp4.global_scale(R)
    codes, scales = nvfp4.quantize_rows(R, g_w)
    inv = inv_smooth(smooth) if smooth is not None else None
    return PackedWeight(codes, scales, g_w, to_f64(L1), to_f64(L2), inv)


# ------------------------------------------------------------------ per call
def smooth_act(X, inv=None) -> np.ndarray:
    """X^ = fp32(fp32(x) * inv[k]) (one fp32 rounding), or fp32(X) without smoothing."""
    x = to_f64(X).astype(np.float32)
    if inv is None:
        return x
    return (x * np.asarray(inv, dtype=np.float32)[None, :]).astype(np.float32)


def act_global_scale(X, inv=None) -> np.float32:
    """Activation decode scale, g_X = fp32(amax|X^| / 2688): static (calibrated
    once) or computed every call (dynamic), the same formula."""
    return nvfp4.global_scale(smooth_act(X, inv))


def quantize_act(X, g_x, inv=None):
    """NVFP4 of the (smoothed) activation rows: (codes [M, K], scales [M, K/16])."""
    return nvfp4.quantize_rows(smooth_act(X, inv), g_x)


def down_proj(X, L1) -> np.ndarray:
    """XL1 = bf16(X . L1), accumulated in float64 (the 16-bit branch's input)."""
    return nvfp4.bf16_round(to_f64(X) @ to_f64(L1))


@dataclass
class Forward:
    codes: np.ndarray    # activation codes [M, K]
    scales: np.ndarray   # activation scales [M, K/16]
    xl1: np.ndarray      # float64 [M, r] (bf16 values)
    y64: np.ndarray      # float64 [M, N] exact-precision output
    y_ref: np.ndarray    # float64 [M, N] y64 rounded to bf16


def gemm_4bit(codes_x, scales_x, codes_w, scales_w) -> np.ndarray:
    """acc[m,n] = sum_k dec(cX)dec(SX) * dec(cR)dec(SR), in float64 (no global scales)."""
    xq = nvfp4.dequantize_rows(codes_x, scales_x)
    wq = nvfp4.dequantize_rows(codes_w, scales_w)
    return xq @ wq.T


def forward(X, pw: PackedWeight, bias, g_x) -> Forward:
    """Y = acc * g_X * g_W + XL1 . L2 + b, float64; y_ref = bf16(Y). The 4-bit
    branch quantises the smoothed X^ (pw.inv_smooth), the 16-bit branch reads X."""
    codes, scales = quantize_act(X, g_x, pw.inv_smooth)
    xl1 = down_proj(X, pw.L1)
    acc = gemm_4bit(codes, scales, pw.codes, pw.scales)
    y = acc * float(g_x) * float(pw.g_w) + xl1 @ pw.L2
    if bias is not None:
        y = y + to_f64(bias)[None, :]
    return Forward(codes, scales, xl1, y, nvfp4.bf16_round(y))


# ------------------------------------------------------------------ fused QKV post-processing
def rms_norm_heads(y, heads: int, head_dim: int, weight, eps: float) -> np.ndarray:
    """Per-head RMSNorm of an [M, heads * head_dim] block, float64:
    x / sqrt(mean over the head of x^2 + eps) * weight (weight: head_dim)."""
    y = np.asarray(y, dtype=np.float64)
    M = y.shape[0]
    x = y.reshape(M, heads, head_dim)
    ms = np.mean(x * x, axis=2, keepdims=True)
    out = x / np.sqrt(ms + eps) * to_f64(weight)[None, None, :]
    return out.reshape(M, heads * head_dim)


def rotary_pairs(y, heads: int, head_dim: int, cos, sin) -> np.ndarray:
    """Rotary embedding of every head on adjacent pairs (2j, 2j+1), float64:
    each pair is rotated by the angle theta_j of its token position,
    (x0, x1) -> (x0 cos_j - x1 sin_j, x1 cos_j + x0 sin_j), with
    cos, sin: [M, head_dim // 2] (cos and sin of theta_j per token and pair)."""
    y = np.asarray(y, dtype=np.float64)
    M = y.shape[0]
    x = y.reshape(M, heads, head_dim)
    c = np.asarray(cos, dtype=np.float64)[:, None, :]
    s = np.asarray(sin, dtype=np.float64)[:, None, :]
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x1 * c + x0 * s
    return out.reshape(M, heads * head_dim)


def qkv_norm_rope(y_ref, heads: int, head_dim: int, w_q, w_k, eps: float, cos, sin):
    """The fused QKV post-processing of a [M, 3 * heads * head_dim] projection
    output laid out [Q | K | V]: Q and K get per-head RMSNorm (weights w_q, w_k)
    then the rotary embedding; V passes through. The input is the layer output
    rounded to bf16 (what the unfused sequence hands to the norm). Returns
    (float64 result, the result rounded to bf16)."""
    y = np.asarray(y_ref, dtype=np.float64)
    hd = heads * head_dim
    out = y.copy()
    for blk, w in ((0, w_q), (1, w_k)):
        part = y[:, blk * hd:(blk + 1) * hd]
        out[:, blk * hd:(blk + 1) * hd] = rotary_pairs(rms_norm_heads(part, heads, head_dim, w, eps),
                                                        heads, head_dim, cos, sin)
    return out, nvfp4.bf16_round(out)


# ------------------------------------------------------------------ MLP pair (GELU between two layers)
def gelu(x, approximate: bool = False) -> np.ndarray:
    """GELU in float64: x * Phi(x) = x (1 + erf(x / sqrt 2)) / 2, or with
    approximate=True the tanh form x (1 + tanh(u)) / 2, u = sqrt(2/pi) (x +
    0.044715 x^3) (the one FLUX's feed-forward blocks use). Evaluated as
    x erfc(-x / sqrt 2) / 2 and x / (1 + exp(-2u)), the same functions written
    without the cancellation of 1 + erf and 1 + tanh for negative x."""
    x = np.asarray(x, dtype=np.float64)
    if approximate:
        u = np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)
        with np.errstate(over="ignore"):
            return x / (1.0 + np.exp(-2.0 * u))
    from scipy.special import erfc
    return 0.5 * x * erfc(-x / np.sqrt(2.0))


@dataclass
class MlpPair:
    up: Forward          # the up projection (its y_ref is the bf16 layer output)
    h: np.ndarray        # float64 [M, K_down] (bf16 values): bf16(GELU(up.y_ref))
    down: Forward        # the down projection of h


def mlp_pair(X, pw_up: PackedWeight, b_up, g_up, pw_down: PackedWeight, b_down, g_h,
             approximate: bool = False) -> MlpPair:
    """The feed-forward pair of a transformer block as two W4A4 layers with GELU
    between them (blog section "Introducing Nunchaku Lite": part of the full
    engine's speed comes from fused GELU / MLP kernels): h = bf16(GELU(bf16(up(X)))), what the
    unfused sequence hands the down projection, which quantises h with its own
    activation scale g_h."""
    up = forward(X, pw_up, b_up, g_up)
    h = nvfp4.bf16_round(gelu(up.y_ref, approximate))
    down = forward(h, pw_down, b_down, g_h)
    return MlpPair(up, h, down)


# ------------------------------------------------------------------ metrics
def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def max_abs_over_row_rms(a, ref) -> float:
    """max_{m,n} |a - ref| / rms(ref[m, :])."""
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = np.sqrt(np.mean(ref * ref, axis=1, keepdims=True))
    return float(np.max(np.abs(a - ref) / rms))
