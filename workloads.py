"""Seeded synthetic workloads for the SVDQuant W4A4 linear layer.

This module only draws random tensors of the shapes and value distributions
that the workload definitions below describe. It holds none of the method's
arithmetic (no quantisation, no SVD of the weight, no layer product; the one
product here builds a planted low-rank weight part from random orthonormal
bases, part of the input recipe); both the CPU oracle and the CUDA path take
their inputs from here.

Shapes come from the benchmark set built for the layer described in the
Hugging Face blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers"
(sections "Native loading in Diffusers": rank 32, group size 16, NVFP4; and
"Structural adapters": Q, K, V fused along the output dimension). The pages
measure whole diffusion pipelines on real checkpoints and prompts; none of
those are available here, so these seeded tensors stand in for the
activations and weights of such a model.

Every tensor is drawn in float32 with numpy's ``default_rng`` and then
rounded once to bfloat16 (round-to-nearest-even, by torch's conversion).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class LayerSpec:
    """One linear layer of a workload: Y[M,N] = X[M,K] . W[N,K]^T + b."""

    name: str
    M: int
    K: int
    N: int
    r: int
    seed: tuple
    x_outlier_frac: float | None = None  # fraction of K channels made outliers
    x_outlier_count: int | None = None   # or an absolute count
    x_outlier_gain: float = 50.0
    w_std: float = 0.02
    planted_rank: int = 0                # rank of a planted low-rank weight part
    planted_norm_ratio: float = 0.0      # ||P||_F / ||W_gauss||_F
    bias_std: float = 0.0

    @property
    def n_outliers(self) -> int:
        if self.x_outlier_count is not None:
            return self.x_outlier_count
        return int(round(self.x_outlier_frac * self.K))


@dataclass(frozen=True)
class Workload:
    name: str
    description: str
    layers: tuple = field(default_factory=tuple)


def _cfg1() -> Workload:
    return Workload(
        "single_linear_256x1024x1024_r32",
        "Single SVDQ linear, M=256, K=N=1024, r=32; X ~ N(0,1) with 8 outlier "
        "channels x50; W ~ N(0, 0.02^2); zero bias; seed 0.",
        (LayerSpec("linear", 256, 1024, 1024, 32, (0,), x_outlier_count=8,
                   x_outlier_gain=50.0, w_std=0.02),),
    )


def _cfg2() -> Workload:
    return Workload(
        "dit_qkv_4608x3072x9216_r32",
        "FLUX-like DiT fused QKV projection: M=4608 tokens (4096 latent patches "
        "+ 512 text), K=3072, N=9216, r=32; X ~ N(0,1) with 1% outlier "
        "channels x30; W ~ N(0,0.02^2) plus a planted rank-8 part with 5x the "
        "Frobenius norm; bias ~ N(0, 0.01^2).",
        (LayerSpec("qkv", 4608, 3072, 9216, 32, (2, 0), x_outlier_frac=0.01,
                   x_outlier_gain=30.0, w_std=0.02, planted_rank=8,
                   planted_norm_ratio=5.0, bias_std=0.01),),
    )


def _cfg3() -> Workload:
    kw = dict(x_outlier_count=8, x_outlier_gain=50.0, w_std=0.02)
    return Workload(
        "dit_mlp_pair_4608_3072x12288_r32",
        "FLUX-like DiT MLP pair, M=4608, r=32: up 3072->12288 and down "
        "12288->3072, each with config-1 value distributions and its own seed.",
        (LayerSpec("mlp_up", 4608, 3072, 12288, 32, (3, 0), **kw),
         LayerSpec("mlp_down", 4608, 12288, 3072, 32, (3, 1), **kw)),
    )


def _cfg4() -> Workload:
    kw = dict(x_outlier_count=8, x_outlier_gain=50.0, w_std=0.02)
    M = 4 * 4608
    return Workload(
        "dit_block_4x4608_r32",
        "Batched DiT block linear set, M=4x4608=18432: QKV 3072->9216, attention "
        "out 3072->3072, MLP up 3072->12288, MLP down 12288->3072, r=32; config-1 "
        "value distributions.",
        (LayerSpec("qkv", M, 3072, 9216, 32, (4, 0), **kw),
         LayerSpec("attn_out", M, 3072, 3072, 32, (4, 1), **kw),
         LayerSpec("mlp_up", M, 3072, 12288, 32, (4, 2), **kw),
         LayerSpec("mlp_down", M, 12288, 3072, 32, (4, 3), **kw)),
    )


def _cfg5() -> Workload:
    layers = []
    for M in (128, 1024, 8192):
        for r in (16, 32, 64, 128):
            layers.append(LayerSpec(f"sweep_M{M}_r{r}", M, 4096, 4096, r, (5, M, r),
                                    x_outlier_frac=0.005, x_outlier_gain=100.0,
                                    w_std=0.015))
    return Workload(
        "sweep_4096x4096_M128-8192_r16-128",
        "Rank and shape sweep: K=N=4096, M in {128,1024,8192}, r in "
        "{16,32,64,128}; X ~ N(0,1) with 0.5% outlier channels x100; "
        "W ~ N(0, 0.015^2).",
        tuple(layers),
    )


WORKLOADS = {i + 1: f() for i, f in enumerate((_cfg1, _cfg2, _cfg3, _cfg4, _cfg5))}


def _to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def make_layer(spec: LayerSpec, rows: int | None = None):
    """Draw (X, W, bias) for one layer as CPU bfloat16 tensors.

    Draw order from one generator seeded with ``spec.seed``: outlier channel
    indices, X, W (Gaussian part), the planted factors, bias. ``rows`` limits
    the number of X rows returned (the first ``rows`` of the full draw), so a
    sample of a large workload has exactly the values of the full one.
    """
    rng = np.random.default_rng(list(spec.seed))
    idx = rng.choice(spec.K, size=spec.n_outliers, replace=False)
    x = rng.standard_normal((spec.M, spec.K), dtype=np.float32)
    x[:, idx] *= np.float32(spec.x_outlier_gain)
    if rows is not None:
        x = x[:rows]
    w = rng.normal(0.0, spec.w_std, size=(spec.N, spec.K)).astype(np.float32)
    if spec.planted_rank:
        k = spec.planted_rank
        u, _ = np.linalg.qr(rng.standard_normal((spec.N, k)))
        v, _ = np.linalg.qr(rng.standard_normal((spec.K, k)))
        sigma = spec.planted_norm_ratio * np.linalg.norm(w.astype(np.float64)) / np.sqrt(k)
        w = (w.astype(np.float64) + sigma * (u @ v.T)).astype(np.float32)
    if spec.bias_std > 0:
        b = rng.normal(0.0, spec.bias_std, size=spec.N).astype(np.float32)
    else:
        b = np.zeros(spec.N, dtype=np.float32)
    return _to_bf16(x), _to_bf16(w), _to_bf16(b)


def small_layer(M: int, K: int, N: int, r: int, seed: int = 1234, outliers: int = 4,
                gain: float = 40.0, w_std: float = 0.02, bias_std: float = 0.01):
    """A small ad-hoc layer (for parity tests at oracle-friendly sizes)."""
    spec = LayerSpec(f"small_{M}x{K}x{N}_r{r}", M, K, N, r, (seed, M, K, N, r),
                     x_outlier_count=min(outliers, K), x_outlier_gain=gain,
                     w_std=w_std, bias_std=bias_std)
    return spec, make_layer(spec)


def rope_tables(M: int, head_dim: int = 128, base: float = 10000.0, seed: int = 0):
    """Rotary tables for token positions: cos and sin of theta[m, j] = pos[m] *
    base^(-2j/head_dim), [M, head_dim // 2] float32, one angle per pair
    (2j, 2j+1); pos is a seeded permutation of 0..M-1, so the tables are not
    monotone in the row index."""
    rng = np.random.default_rng([seed, M, head_dim])
    pos = rng.permutation(M).astype(np.float64)
    freq = base ** (-np.arange(0, head_dim, 2, dtype=np.float64) / head_dim)
    ang = pos[:, None] * freq[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)

def modulation_layer(M: int = 1, K: int = 3072, N: int = 6 * 3072, seed: int = 0):
    """An adaptive-normalisation modulation projection (the AWQ W4A16 layers of
    the blog's section "Introducing Nunchaku Lite"): FLUX's adaLN modulation
    maps the conditioning vector (K = 3072) to six 3072-wide shift / scale /
    gate vectors (N = 18432), one row per sample (M = batch). Returns (X, W, b):
    X ~ N(0, 1), W ~ N(0, 0.02^2), b ~ N(0, 0.01^2), bf16, drawn in that order."""
    rng = np.random.default_rng([7, M, K, N, seed])
    X = rng.standard_normal((M, K), dtype=np.float32)
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    b = rng.standard_normal(N, dtype=np.float32) * np.float32(0.01)
    return _to_bf16(X), _to_bf16(W), _to_bf16(b)
