"""Pins of the oracle's quantiser, decomposition and forward pass.

Each test ties an oracle function to an independent fact: a brute-force
search, a closed form, the Eckart-Young theorem, a special case that reduces
to plain NVFP4 W4A4 or to X.W^T, a pure-Python triple loop, or the accuracy
claim of the blog (low-rank correction beats plain 4-bit on outlier-heavy
inputs, section "Background: SVDQuant and Nunchaku")."""
import numpy as np
import pytest

from oracle import nvfp4, svdq
import workloads


def _rand(shape, seed=0, outl=3, gain=40.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape).astype(np.float32)
    x[:, rng.choice(shape[1], outl, replace=False)] *= gain
    return x


# ---------------------------------------------------------------- quantiser
def test_global_scale_maps_amax_to_6x448():
    a = _rand((8, 64))
    g = nvfp4.global_scale(a)
    assert np.isclose(float(g) * 2688.0, np.abs(a).max(), rtol=1e-7)
    assert nvfp4.global_scale(np.zeros((2, 16), np.float32)) == 1.0


def test_block_scale_is_nearest_e4m3_of_amax_over_6g():
    a = _rand((16, 256), seed=1)
    g = nvfp4.global_scale(a)
    _, S = nvfp4.quantize_rows(a, g)
    pos = nvfp4.e4m3_decode(np.arange(0x7F))
    amax = np.abs(a.reshape(16, 16, 16)).max(-1).astype(np.float64)
    target = amax / (6.0 * float(g))
    for t, s in zip(target.ravel(), S.ravel()):
        d = np.abs(pos - min(t, 448.0))
        assert abs(nvfp4.e4m3_decode(s) - pos[np.argmin(d)]) == 0 or np.isclose(d.min(), np.sort(d)[1])


def test_codes_are_nearest_grid_points_16x16_brute_force():
    """Every code of a 16x16 tile is the argmin over the 16 E2M1 values of
    |x / (dec(S) g) - v| (float64), except at exact ties."""
    a = _rand((16, 16), seed=2)
    g = nvfp4.global_scale(a)
    codes, S = nvfp4.quantize_rows(a, g)
    grid = nvfp4.e2m1_decode(np.arange(16))
    for i in range(16):
        sd = nvfp4.e4m3_decode(S[i, 0]) * float(g)
        for k in range(16):
            q = min(max(float(a[i, k]) / sd, -6.0), 6.0)
            d = np.abs(grid - q)
            order = np.argsort(d, kind="stable")
            if np.isclose(d[order[0]], d[order[1]], rtol=0, atol=1e-6) and grid[order[0]] != grid[order[1]]:
                continue                                      # a tie: both codes are valid
            assert grid[codes[i, k]] == grid[order[0]] or (grid[codes[i, k]] == 0 and grid[order[0]] == 0)


def test_zero_block_gives_zero_scale_and_codes():
    a = _rand((2, 64), seed=4)
    a[0, 16:32] = 0.0
    g = nvfp4.global_scale(a)
    codes, S = nvfp4.quantize_rows(a, g)
    assert S[0, 1] == 0 and np.all(codes[0, 16:32] == 0)


def test_quantisation_error_within_half_grid_step():
    """|x - dec(q)| <= half the local E2M1 spacing (<= 1) times the block's decode scale,
    plus the in-range rounding of the scale itself (no block saturates here)."""
    a = _rand((64, 512), seed=5)
    g = nvfp4.global_scale(a)
    codes, S = nvfp4.quantize_rows(a, g)
    deq = nvfp4.dequantize_rows(codes, S) * float(g)
    sd = (nvfp4.e4m3_decode(S) * float(g))[..., None]
    err = np.abs(deq.reshape(64, 32, 16) - a.reshape(64, 32, 16))
    assert np.all(err <= 1.0 * sd + 1e-12)


# ---------------------------------------------------------------- decomposition
def test_planted_low_rank_is_recovered():
    """W = U diag(s) V^T with orthonormal U, V: the SVD's singular values are s
    (closed form) and the bf16 factors reproduce W to bf16 precision."""
    rng = np.random.default_rng(9)
    N, K, k = 96, 64, 5
    U, _ = np.linalg.qr(rng.standard_normal((N, k)))
    V, _ = np.linalg.qr(rng.standard_normal((K, k)))
    s = np.array([9.0, 7.0, 5.0, 3.0, 1.0])
    W = (U * s) @ V.T
    L1, L2, sv = svdq.lowrank_factors(W, k)
    assert np.allclose(sv[:k], s, rtol=1e-12)
    assert np.all(sv[k:] < 1e-12)
    approx = (L1 @ L2).T
    assert np.linalg.norm(approx - W) / np.linalg.norm(W) < 2 ** -7


def test_eckart_young_and_singular_values_from_eigvalsh():
    rng = np.random.default_rng(10)
    W = rng.normal(0, 0.02, (80, 48))
    r = 8
    L1, L2, sv = svdq.lowrank_factors(W, r)
    ev = np.sort(np.linalg.eigvalsh(W.T @ W))[::-1]          # independent routine
    assert np.allclose(sv ** 2, ev, rtol=1e-9, atol=1e-15)
    tail = np.sum(ev[r:])
    R = svdq.residual(W, L1, L2).astype(np.float64)
    # best rank-r error (theorem) plus the bf16 rounding of the factors
    assert tail <= np.sum(R ** 2) <= tail * (1 + 2e-2)
    # dropping the top pair leaves sigma_1^2 more energy in the residual
    L1b, L2b = L1.copy(), L2.copy()
    L1b[:, 0] = 0
    assert np.sum(svdq.residual(W, L1b, L2b).astype(np.float64) ** 2) > tail + 0.95 * ev[0]


def test_residual_rank0_is_w_and_full_rank_is_small():
    rng = np.random.default_rng(12)
    W = nvfp4.bf16_round(rng.normal(0, 0.02, (32, 48)))
    L1, L2, _ = svdq.lowrank_factors(W, 0)
    assert np.array_equal(svdq.residual(W, L1, L2), W.astype(np.float32))
    L1, L2, _ = svdq.lowrank_factors(W, 32)
    R = svdq.residual(W, L1, L2)
    assert np.linalg.norm(R) / np.linalg.norm(W) < 2 ** -6


def test_residual_orientation():
    """R[n,k] = W[n,k] - sum_j L1[k,j] L2[j,n] element by element (tiny case)."""
    W = np.arange(6, dtype=np.float64).reshape(2, 3)          # N=2, K=3
    L1 = np.array([[1.0], [2.0], [3.0]])                      # K x r
    L2 = np.array([[0.5, -1.0]])                              # r x N
    R = svdq.residual(W, L1, L2)
    expect = [[W[n, k] - L1[k, 0] * L2[0, n] for k in range(3)] for n in range(2)]
    assert np.array_equal(R, np.float32(expect))


# ---------------------------------------------------------------- forward
def _tiny_layer(M=16, K=32, N=16, r=4, seed=3):
    rng = np.random.default_rng(seed)
    X = nvfp4.bf16_round(_rand((M, K), seed=seed))
    W = nvfp4.bf16_round(rng.normal(0, 0.05, (N, K)))
    b = nvfp4.bf16_round(rng.normal(0, 0.01, N))
    return X, W, b


def test_forward_matches_python_triple_loop():
    X, W, b = _tiny_layer()
    L1, L2, _ = svdq.lowrank_factors(W, 4)
    pw = svdq.pack_weight(W, L1, L2)
    g_x = svdq.act_global_scale(X)
    out = svdq.forward(X, pw, b, g_x)
    M, K = X.shape
    N = W.shape[0]
    cx, sx = out.codes, out.scales
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                xv = nvfp4.e2m1_decode(cx[m, k]) * nvfp4.e4m3_decode(sx[m, k // 16])
                wv = nvfp4.e2m1_decode(pw.codes[n, k]) * nvfp4.e4m3_decode(pw.scales[n, k // 16])
                acc += xv * wv
            lr = sum(out.xl1[m, j] * L2[j, n] for j in range(4))
            y = acc * float(g_x) * float(pw.g_w) + lr + b[n]
            assert np.isclose(out.y64[m, n], y, rtol=1e-12, atol=1e-15)
    # the down projection, by its definition
    for m in range(M):
        for j in range(4):
            assert out.xl1[m, j] == nvfp4.bf16_round(sum(X[m, k] * L1[k, j] for k in range(K)))


def test_rank0_reduces_to_plain_nvfp4_w4a4():
    X, W, b = _tiny_layer(M=8, K=64, N=32)
    L1, L2, _ = svdq.lowrank_factors(W, 0)
    pw = svdq.pack_weight(W, L1, L2)
    g_x = svdq.act_global_scale(X)
    out = svdq.forward(X, pw, b, g_x)
    cw, sw = nvfp4.quantize_rows(W.astype(np.float32), nvfp4.global_scale(W.astype(np.float32)))
    assert np.array_equal(pw.codes, cw) and np.array_equal(pw.scales, sw)
    plain = (nvfp4.dequantize_rows(out.codes, out.scales) * float(g_x)) @ \
            (nvfp4.dequantize_rows(cw, sw) * float(pw.g_w)).T + b
    assert np.allclose(out.y64, plain, rtol=1e-12, atol=1e-12)


def test_full_rank_reduces_to_x_wt():
    X, W, b = _tiny_layer(M=8, K=32, N=32)
    L1, L2, _ = svdq.lowrank_factors(W, 32)
    pw = svdq.pack_weight(W, L1, L2)
    out = svdq.forward(X, pw, b, svdq.act_global_scale(X))
    exact = X @ W.T + b
    assert svdq.rel_fro(out.y64, exact) < 1e-2


def test_rows_are_independent():
    X, W, b = _tiny_layer(M=32, K=64, N=16)
    L1, L2, _ = svdq.lowrank_factors(W, 4)
    pw = svdq.pack_weight(W, L1, L2)
    g_x = svdq.act_global_scale(X)
    full = svdq.forward(X, pw, b, g_x)
    part = svdq.forward(X[5:9], pw, b, g_x)
    assert np.array_equal(part.y64, full.y64[5:9])
    assert np.array_equal(part.codes, full.codes[5:9])


@pytest.mark.parametrize("outlier_gain", [50.0])
def test_low_rank_correction_beats_plain_w4a4_on_outliers(outlier_gain):
    """The blog's claim: the low-rank branch absorbs outliers, so the
    rank-corrected output is closer to X.W^T than plain NVFP4 W4A4."""
    spec = workloads.WORKLOADS[1].layers[0]
    X, W, b = workloads.make_layer(spec)
    X64, W64, b64 = svdq.to_f64(X), svdq.to_f64(W), svdq.to_f64(b)
    exact = X64 @ W64.T + b64
    g_x = svdq.act_global_scale(X64)
    L1, L2, _ = svdq.lowrank_factors(W64, 32)
    e_svdq = svdq.rel_fro(svdq.forward(X64, svdq.pack_weight(W64, L1, L2), b64, g_x).y64, exact)
    L10, L20, _ = svdq.lowrank_factors(W64, 0)
    e_naive = svdq.rel_fro(svdq.forward(X64, svdq.pack_weight(W64, L10, L20), b64, g_x).y64, exact)
    assert e_svdq < e_naive


# ------------------------------------------------------------------ fused QKV norm + rotary
def test_rms_norm_closed_forms():
    rng = np.random.default_rng(41)
    y = rng.standard_normal((5, 3 * 16)) * 7.0
    out = svdq.rms_norm_heads(y, 3, 16, np.ones(16), 0.0)
    ms = np.mean(out.reshape(5, 3, 16) ** 2, axis=2)
    assert np.allclose(ms, 1.0, rtol=0, atol=1e-12)           # unit RMS per head with eps = 0
    c = np.full((2, 16), -2.5)
    w = np.arange(1, 17, dtype=np.float64)
    assert np.allclose(svdq.rms_norm_heads(c, 1, 16, w, 0.0), -w[None, :], atol=1e-12)  # constant row -> sign * w
    # eps dominates a zero row: the result stays zero
    assert not svdq.rms_norm_heads(np.zeros((1, 16)), 1, 16, w, 1e-6).any()


def test_rotary_is_complex_multiplication():
    """Each pair is the complex product (x0 + i x1) e^(i theta_j): an independent
    formulation of the rotation by theta_j."""
    rng = np.random.default_rng(42)
    M, H, D = 4, 2, 8
    y = rng.standard_normal((M, H * D))
    theta = rng.uniform(-np.pi, np.pi, (M, D // 2))
    out = svdq.rotary_pairs(y, H, D, np.cos(theta), np.sin(theta)).reshape(M, H, D)
    z = y.reshape(M, H, D)[..., 0::2] + 1j * y.reshape(M, H, D)[..., 1::2]
    ref = z * np.exp(1j * theta)[:, None, :]
    assert np.allclose(out[..., 0::2], ref.real, atol=1e-13)
    assert np.allclose(out[..., 1::2], ref.imag, atol=1e-13)
    # pair norms are preserved, rotating back by -theta restores the input, cos = 1 / sin = 0 is the identity
    assert np.allclose(np.abs(ref), np.abs(z), atol=1e-13)
    back = svdq.rotary_pairs(out.reshape(M, H * D), H, D, np.cos(theta), -np.sin(theta))
    assert np.allclose(back, y, atol=1e-13)
    assert np.array_equal(svdq.rotary_pairs(y, H, D, np.ones((M, D // 2)), np.zeros((M, D // 2))), y)
    # a quarter turn maps (x0, x1) to (-x1, x0)
    q = svdq.rotary_pairs(y, H, D, np.zeros((M, D // 2)), np.ones((M, D // 2))).reshape(M, H, D)
    assert np.array_equal(q[..., 0::2], -y.reshape(M, H, D)[..., 1::2])
    assert np.array_equal(q[..., 1::2], y.reshape(M, H, D)[..., 0::2])


def test_qkv_norm_rope_against_loops():
    """The fused post-processing against per-element Python loops on a tiny case;
    V passes through unchanged; the bf16 output is the float64 result rounded."""
    rng = np.random.default_rng(43)
    M, H, D = 3, 2, 4
    y = nvfp4.bf16_round(rng.standard_normal((M, 3 * H * D)) * 3.0)
    wq, wk = rng.uniform(0.5, 1.5, D), rng.uniform(0.5, 1.5, D)
    cos, sin = rng.uniform(-1, 1, (M, D // 2)), rng.uniform(-1, 1, (M, D // 2))
    eps = 1e-6
    out, out_bf16 = svdq.qkv_norm_rope(y, H, D, wq, wk, eps, cos, sin)
    ref = y.copy()
    for blk, w in ((0, wq), (1, wk)):
        for m in range(M):
            for h in range(H):
                base = blk * H * D + h * D
                x = [y[m, base + i] for i in range(D)]
                rstd = 1.0 / np.sqrt(sum(v * v for v in x) / D + eps)
                n = [x[i] * rstd * w[i] for i in range(D)]
                for j in range(D // 2):
                    ref[m, base + 2 * j] = n[2 * j] * cos[m, j] - n[2 * j + 1] * sin[m, j]
                    ref[m, base + 2 * j + 1] = n[2 * j + 1] * cos[m, j] + n[2 * j] * sin[m, j]
    assert np.allclose(out, ref, rtol=0, atol=1e-12)
    assert np.array_equal(out[:, 2 * H * D:], y[:, 2 * H * D:])
    assert np.array_equal(out_bf16, nvfp4.bf16_round(out))
