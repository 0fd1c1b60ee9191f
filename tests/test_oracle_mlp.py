"""Pins of the oracle's MLP pair (up projection, GELU, down projection):
GELU against math.erf element loops, its closed forms (odd part, limits,
slope at zero), the tanh form's known distance from the exact one, and the
pair as the composition of two independently packed layers."""
import math

import numpy as np

import workloads
from oracle import nvfp4, svdq


def test_gelu_matches_math_erf_loops():
    x = np.linspace(-6, 6, 97)
    ref = np.array([0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0))) for v in x])
    assert np.allclose(svdq.gelu(x), ref, rtol=0, atol=1e-15)
    ref_t = np.array([0.5 * v * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (v + 0.044715 * v ** 3))) for v in x])
    assert np.allclose(svdq.gelu(x, approximate=True), ref_t, rtol=0, atol=1e-15)


def test_gelu_negative_tail_has_no_cancellation():
    """Far in the negative tail GELU is tiny but not zero: x Phi(x) with Phi(x)
    from the complementary error function (math.erfc) keeps full relative
    precision where 1 + erf(x / sqrt 2) would cancel to zero."""
    x = np.array([-6.0, -9.0, -12.0])
    ref = np.array([0.5 * v * math.erfc(-v / math.sqrt(2.0)) for v in x])
    g = svdq.gelu(x)
    assert np.all(g < 0) and np.allclose(g, ref, rtol=1e-14, atol=0)
    # the tanh form equals x sigma(2u): its tail follows exp(2u)
    u = math.sqrt(2.0 / math.pi) * (-9.0 + 0.044715 * (-9.0) ** 3)
    assert np.isclose(svdq.gelu(np.array([-9.0]), approximate=True)[0], -9.0 / (1.0 + math.exp(-2.0 * u)),
                      rtol=1e-14, atol=0)


def test_gelu_closed_forms():
    x = np.linspace(-8, 8, 161)
    g = svdq.gelu(x)
    assert np.allclose(g - svdq.gelu(-x), x, atol=1e-14)        # Phi(x) + Phi(-x) = 1
    assert svdq.gelu(np.array([0.0]))[0] == 0.0
    assert abs(svdq.gelu(np.array([10.0]))[0] - 10.0) < 1e-20 + 1e-15
    assert abs(svdq.gelu(np.array([-10.0]))[0]) < 1e-20
    eps = 1e-6
    slope = (svdq.gelu(np.array([eps]))[0] - svdq.gelu(np.array([-eps]))[0]) / (2 * eps)
    assert abs(slope - 0.5) < 1e-9                               # GELU'(0) = Phi(0) = 1/2
    # the tanh form stays within 5e-4 of the exact one (its maximal gap is about 4.7e-4)
    assert np.max(np.abs(svdq.gelu(x, approximate=True) - g)) < 5e-4


def test_mlp_pair_is_the_composition_of_two_layers():
    M, D, F, r = 16, 256, 512, 16
    _, (X, Wu, bu) = workloads.small_layer(M, D, F, r, seed=3)
    _, (_, Wd, bd) = workloads.small_layer(M, F, D, r, seed=4)
    Lu1, Lu2, _ = svdq.lowrank_factors(Wu, r)
    Ld1, Ld2, _ = svdq.lowrank_factors(Wd, r)
    pu, pd = svdq.pack_weight(Wu, Lu1, Lu2), svdq.pack_weight(Wd, Ld1, Ld2)
    gu = svdq.act_global_scale(X)
    up = svdq.forward(X, pu, bu, gu)
    h = nvfp4.bf16_round(svdq.gelu(up.y_ref))
    gh = svdq.act_global_scale(h)
    pair = svdq.mlp_pair(X, pu, bu, gu, pd, bd, gh)
    assert np.array_equal(pair.up.y_ref, up.y_ref)
    assert np.array_equal(pair.h, h)
    down = svdq.forward(h, pd, bd, gh)
    assert np.array_equal(pair.down.y64, down.y64) and np.array_equal(pair.down.codes, down.codes)
    # GELU output is bounded below by its minimum, about -0.17
    assert pair.h.min() >= -0.1701
