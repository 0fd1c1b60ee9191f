"""Pins of the oracle's smoothing (outliers moved from the activations into the
weights, blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers",
section "Background: SVDQuant and Nunchaku") against facts that do not depend
on the oracle's own code: exact power-of-two scalings, closed forms of the
calibration rule, the float64 identity X^ W^T = X W^T, Eckart-Young on the
smoothed weight, and the accuracy gain on outlier channels."""
import numpy as np
import pytest

from oracle import nvfp4, svdq

rng0 = np.random.default_rng


def _layer(M=24, K=96, N=80, seed=0, outliers=4, gain=40.0):
    rng = rng0(seed)
    X = rng.standard_normal((M, K))
    X[:, rng.choice(K, outliers, replace=False)] *= gain
    W = rng.standard_normal((N, K)) * 0.02
    return nvfp4.bf16_round(X), nvfp4.bf16_round(W)


def test_unit_smoothing_is_the_plain_method():
    X, W = _layer()
    lam = np.ones(W.shape[1], dtype=np.float32)
    r = 8
    L1, L2, s = svdq.lowrank_factors(W, r)
    L1s, L2s, ss = svdq.lowrank_factors(W, r, lam)
    assert np.array_equal(L1, L1s) and np.array_equal(L2, L2s) and np.array_equal(s, ss)
    assert np.array_equal(svdq.residual(W, L1, L2), svdq.residual(W, L1, L2, lam))
    g = svdq.act_global_scale(X)
    assert g == svdq.act_global_scale(X, svdq.inv_smooth(lam))
    a = svdq.forward(X, svdq.pack_weight(W, L1, L2), None, g)
    b = svdq.forward(X, svdq.pack_weight(W, L1, L2, lam), None, g)
    assert np.array_equal(a.codes, b.codes) and np.array_equal(a.y64, b.y64)


def test_power_of_two_smoothing_is_exact_per_input_channel():
    """lambda_k = 2^e_k (different per k, N != K): the smoothed residual is the
    plain one times lambda_k column by column, bit for bit, and X^ = X / lambda."""
    X, W = _layer(K=64, N=48)
    e = rng0(1).integers(-3, 4, W.shape[1])
    lam = np.ldexp(np.ones(W.shape[1]), e).astype(np.float32)
    L1, L2, _ = svdq.lowrank_factors(W, 4)
    R = svdq.residual(W, L1, L2)
    Rs = svdq.residual(W, L1, L2, lam)
    assert np.array_equal(Rs, (R * lam[None, :]).astype(np.float32))
    inv = svdq.inv_smooth(lam)
    assert np.array_equal(inv, np.ldexp(np.ones(W.shape[1]), -e).astype(np.float32))
    assert np.array_equal(svdq.smooth_act(X, inv), (X * np.ldexp(1.0, -e)[None, :]).astype(np.float32))


def test_uniform_power_of_two_smoothing_leaves_codes_unchanged():
    """NVFP4 is invariant under a power-of-two scaling of the tensor and its
    global scale: X^ = X / 4 with g / 4 gives the same codes and block scales."""
    X, _ = _layer(M=16, K=64)
    inv = np.full(X.shape[1], 0.25, dtype=np.float32)
    g = svdq.act_global_scale(X)
    gs = svdq.act_global_scale(X, inv)
    assert gs == np.float32(g * 0.25)
    c, s = svdq.quantize_act(X, g)
    cs, ss = svdq.quantize_act(X, gs, inv)
    assert np.array_equal(c, cs) and np.array_equal(s, ss)


def test_calibration_closed_forms():
    """alpha = 0.5 balances the channel ranges (amax|X^_k| = amax|W^_k| =
    sqrt(ax aw)); alpha = 1 makes every activation channel's amax 1, alpha = 0
    every weight channel's; an all-zero channel gets lambda = 1."""
    X, W = _layer(K=40, N=30)
    X[:, 3] = 0.0
    W[:, 7] = 0.0
    ax = np.max(np.abs(X), axis=0)
    aw = np.max(np.abs(W), axis=0)
    lam = svdq.smooth_factors(X, W, 0.5).astype(np.float64)
    ok = (ax > 0) & (aw > 0)
    assert lam[3] == 1.0 and lam[7] == 1.0
    assert np.allclose(ax[ok] / lam[ok], np.sqrt(ax[ok] * aw[ok]), rtol=1e-6, atol=0)
    assert np.allclose(aw[ok] * lam[ok], np.sqrt(ax[ok] * aw[ok]), rtol=1e-6, atol=0)
    assert np.allclose((ax / svdq.smooth_factors(X, W, 1.0))[ok], 1.0, rtol=1e-6, atol=0)
    assert np.allclose((aw * svdq.smooth_factors(X, W, 0.0))[ok], 1.0, rtol=1e-6, atol=0)
    assert svdq.smooth_factors(X, W).dtype == np.float32
    # the factors are clamped to [2^-32, 2^32]: an extreme channel ratio of 2^160 saturates
    Xe, We = X.copy(), W.copy()
    Xe[:, 0], We[:, 0] = 2.0 ** 80, 2.0 ** -80
    Xe[:, 1], We[:, 1] = 2.0 ** -80, 2.0 ** 80
    le = svdq.smooth_factors(Xe, We)
    assert le[0] == np.float32(2.0 ** 32) and le[1] == np.float32(2.0 ** -32)


def test_smoothed_factors_satisfy_eckart_young_on_the_smoothed_weight():
    """The factors approximate diag(lambda) W^T: the residual energy of
    diag(lambda) (W^T - L1 L2) is the tail of the smoothed spectrum (up to the
    bf16 rounding of the factors), and the returned singular values are those
    of the smoothed matrix (eigvalsh of its Gram matrix)."""
    X, W = _layer(K=64, N=48)
    lam = svdq.smooth_factors(X, W).astype(np.float64)
    r = 6
    L1, L2, s = svdq.lowrank_factors(W, r, lam)
    A = W.T * lam[:, None]
    ev = np.sort(np.linalg.eigvalsh(A @ A.T))[::-1][:len(s)]
    assert np.allclose(s ** 2, np.clip(ev, 0, None), rtol=1e-9, atol=1e-12 * ev[0])
    tail = float(np.sum(s[r:] ** 2))
    e = float(np.linalg.norm(A - lam[:, None] * (L1 @ L2)) ** 2)
    assert tail <= e <= tail * 1.01
    # L1 carries 1/lambda: without it the residual is far from the tail
    e_unfolded = float(np.linalg.norm(A - L1 @ L2) ** 2)
    assert e_unfolded > 2 * tail


def test_full_rank_smoothed_layer_reproduces_x_wt():
    """r = K: the low-rank branch holds the whole (smoothed) weight, the
    residual is bf16-rounding noise, and Y = X W^T to that precision: the
    float64 identity X^ W^^T = X W^T with everything else exact."""
    X, W = _layer(M=12, K=32, N=24)
    lam = svdq.smooth_factors(X, W)
    L1, L2, _ = svdq.lowrank_factors(W, 32, lam)
    pw = svdq.pack_weight(W, L1, L2, lam)
    g = svdq.act_global_scale(X, pw.inv_smooth)
    y = svdq.forward(X, pw, None, g).y64
    ref = X @ W.T
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 2e-2


def test_smoothing_improves_accuracy_on_outlier_channels():
    """The reason for smoothing: with outlier activation channels, the error of
    the W4A4 layer against X W^T drops when they move into the weights."""
    X, W = _layer(M=64, K=256, N=128, outliers=8, gain=50.0, seed=3)
    r = 16
    ref = X @ W.T

    def err(lam):
        L1, L2, _ = svdq.lowrank_factors(W, r, lam)
        pw = svdq.pack_weight(W, L1, L2, lam)
        y = svdq.forward(X, pw, None, svdq.act_global_scale(X, pw.inv_smooth)).y64
        return np.linalg.norm(y - ref) / np.linalg.norm(ref)

    e_plain = err(None)
    e_smooth = err(svdq.smooth_factors(X, W))
    assert e_smooth < 0.7 * e_plain, (e_smooth, e_plain)


@pytest.mark.parametrize("alpha", [0.5, 0.3])
def test_smoothed_forward_matches_elementwise_loops(alpha):
    """The 4-bit branch quantises x * inv[k] and the 16-bit branch reads the raw
    X, written out with per-element Python loops on a tiny case."""
    X, W = _layer(M=3, K=32, N=4, outliers=2)
    lam = svdq.smooth_factors(X, W, alpha)
    inv = svdq.inv_smooth(lam)
    L1, L2, _ = svdq.lowrank_factors(W, 2, lam)
    pw = svdq.pack_weight(W, L1, L2, lam)
    g = svdq.act_global_scale(X, inv)
    out = svdq.forward(X, pw, None, g)
    M, K = X.shape
    xs = np.empty((M, K), dtype=np.float32)
    for m in range(M):
        for k in range(K):
            xs[m, k] = np.float32(np.float32(X[m, k]) * inv[k])
    codes, scales = nvfp4.quantize_rows(xs, g)
    assert np.array_equal(codes, out.codes) and np.array_equal(scales, out.scales)
    for m in range(M):
        for j in range(2):
            assert out.xl1[m, j] == nvfp4.bf16_round(sum(X[m, k] * L1[k, j] for k in range(K)))
