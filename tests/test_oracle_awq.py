"""Pins of the AWQ W4A16 oracle (oracle/awq.py) against facts that do not
depend on its code: exact round trips of weights that lie on a 4-bit grid,
brute-force nearest grid points, the half-step error bound, the power-of-two
scaling of the activation-aware factor, and element loops for the layer."""
import numpy as np

from oracle import awq, nvfp4

rng0 = np.random.default_rng


def _grid_weight(N=6, K=256, seed=0):
    """W = (q - z) s with q, z, s drawn per group; every group uses codes 0 and 15."""
    rng = rng0(seed)
    G = K // awq.GROUP
    q = rng.integers(0, 16, (N, G, awq.GROUP))
    q[:, :, 0] = 0
    q[:, :, 1] = 15
    z = rng.integers(0, 16, (N, G))
    s = nvfp4.bf16_round(rng.uniform(0.001, 0.1, (N, G)))
    W = (q - z[:, :, None]) * s[:, :, None]
    return W.reshape(N, K), q.reshape(N, K), z, s


def test_weights_on_the_grid_round_trip_exactly():
    W, q, z, s = _grid_weight()
    aw = awq.quantize(W)
    assert np.array_equal(aw.codes, q)
    assert np.array_equal(aw.zeros, z)
    assert np.array_equal(aw.scales, s.astype(np.float32))
    assert np.array_equal(awq.dequantize(aw), W)


def test_codes_are_the_nearest_grid_points():
    """Given the stored (s, z), each code is the argmin over the 16 codes of
    |w - (q - z) s| (brute force; ties and clamped values excluded)."""
    rng = rng0(1)
    W = nvfp4.bf16_round(rng.standard_normal((8, 128)) * 0.05)
    aw = awq.quantize(W)
    N, K = W.shape
    s = np.repeat(aw.scales, awq.GROUP, axis=1).astype(np.float64)
    z = np.repeat(aw.zeros, awq.GROUP, axis=1).astype(np.float64)
    cand = (np.arange(16)[None, None, :] - z[:, :, None]) * s[:, :, None]
    err = np.abs(W[:, :, None] - cand)
    best = np.argmin(err, axis=2)
    srt = np.sort(err, axis=2)
    clear = (srt[:, :, 1] - srt[:, :, 0]) > 1e-6 * s
    assert clear.mean() > 0.99
    assert np.array_equal(aw.codes[clear], best[clear])


def test_error_within_half_a_step():
    rng = rng0(2)
    W = nvfp4.bf16_round(rng.standard_normal((16, 512)) * 0.02)
    aw = awq.quantize(W)
    s = np.repeat(aw.scales, awq.GROUP, axis=1).astype(np.float64)
    d = np.abs(awq.dequantize(aw) - W)
    # the grid spans [min, max] up to the rounding of s to bf16 and of z: half a step plus that slack
    assert np.all(d <= 0.5 * s * (1 + 2 ** -7) + 1e-12 + np.abs(W) * 2 ** -8)
    assert np.mean(d <= 0.5 * s + 1e-12) > 0.99


def test_zero_group_and_codes_in_range():
    W = np.zeros((2, 128))
    W[1, 64:] = nvfp4.bf16_round(rng0(3).standard_normal(64))
    aw = awq.quantize(W)
    assert not awq.dequantize(aw)[0].any()          # an all-zero group dequantises to zero
    assert aw.codes.max() <= 15 and aw.zeros.max() <= 15


def test_uniform_power_of_two_activation_factor_is_exact():
    """a = 4: the weight quantised is 4 W (scales 4x, same codes and zeros) and
    X is divided by 4, so the layer output is unchanged bit for bit."""
    rng = rng0(4)
    W = nvfp4.bf16_round(rng.standard_normal((12, 256)) * 0.03)
    X = nvfp4.bf16_round(rng.standard_normal((3, 256)))
    a = np.full(256, 4.0, dtype=np.float32)
    p, q = awq.quantize(W), awq.quantize(W, a)
    assert np.array_equal(p.codes, q.codes) and np.array_equal(p.zeros, q.zeros)
    assert np.array_equal(q.scales, (4 * p.scales).astype(np.float32))
    assert np.array_equal(q.inv_act, np.full(256, 0.25, dtype=np.float32))
    assert np.array_equal(awq.forward(X, p).y64, awq.forward(X, q).y64)


def test_activation_factor_scales_input_channels():
    """a_k varies per input channel (N != K): the weight quantised is W diag(a)."""
    rng = rng0(5)
    W = nvfp4.bf16_round(rng.standard_normal((8, 128)) * 0.03)
    a = rng.uniform(0.5, 2.0, 128).astype(np.float32)
    aw = awq.quantize(W, a)
    Wa = (W.astype(np.float32) * a[None, :]).astype(np.float32)
    assert np.array_equal(aw.codes, awq.quantize(Wa).codes)


def test_forward_matches_element_loops():
    rng = rng0(6)
    M, N, K = 2, 3, 128
    W = nvfp4.bf16_round(rng.standard_normal((N, K)) * 0.05)
    X = nvfp4.bf16_round(rng.standard_normal((M, K)))
    b = nvfp4.bf16_round(rng.standard_normal(N) * 0.01)
    a = rng.uniform(0.5, 2.0, K).astype(np.float32)
    aw = awq.quantize(W, a)
    out = awq.forward(X, aw, b)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                g = k // awq.GROUP
                w = (int(aw.codes[n, k]) - int(aw.zeros[n, g])) * float(aw.scales[n, g])
                x = float(np.float32(np.float32(X[m, k]) * aw.inv_act[k]))
                acc += x * w
            assert abs(out.y64[m, n] - (acc + b[n])) <= 1e-12 * (1 + abs(acc))


def test_w4a16_is_far_more_accurate_than_its_step():
    """Group-64 INT4 keeps the layer within a few percent of X W^T on Gaussian data."""
    rng = rng0(7)
    W = nvfp4.bf16_round(rng.standard_normal((64, 1024)) * 0.02)
    X = nvfp4.bf16_round(rng.standard_normal((4, 1024)))
    y = awq.forward(X, awq.quantize(W)).y64
    ref = X @ W.T
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 0.1
