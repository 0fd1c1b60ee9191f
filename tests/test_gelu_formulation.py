"""CPU check of the GELU formulation the fused MLP epilogue evaluates
(blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers", section
"Introducing Nunchaku Lite": fused GELU / MLP kernels).

The kernel computes GELU in fp32 without a tail branch:
* the erf form x erfc(-x/sqrt 2)/2 takes erfc(a) = t exp(-a^2 + P(t)), t = 1/(1 + a/2),
  from the Chebyshev fit of Numerical Recipes in C (2nd ed., section 6.2, erfcc);
* the tanh form is x sigma(2u) with u = sqrt(2/pi)(x + 0.044715 x^3);
* both take the exponential as 2^(e + 64) and scale the product by 2^-64 last, so that
  a subnormal result is rounded once.

This test restates those steps in numpy float32, with an exact exp2 and
reciprocal in place of the hardware approximations, which flushes exp2 results
below the normal range to zero as the hardware does. It checks that the
formulation rounds to the correctly rounded bf16 GELU for every bf16 input in
[-40, 40], the far negative tail included. The kernel's own outputs are checked
against the oracle on the GPU, in tests/test_gpu_mlp.py.
"""
import numpy as np
import pytest
import torch
from scipy.special import erfc

F = np.float32
NR_ERFCC = [0.17087277, -0.82215223, 1.48851587, -1.13520398, 0.27886807, -0.18628806, 0.09678418, 0.37409196,
            1.00002368, -1.26551223]


def _ex2(v):
    r = np.exp2(v.astype(np.float64)).astype(F)
    r[np.abs(r) < F(2.0 ** -126)] = 0  # the flush of ex2.approx.ftz
    return r


def _rcp(v):
    return (1.0 / v.astype(np.float64)).astype(F)


def erf_form(x):
    z = (x * F(-0.7071067811865476)).astype(F)
    a = np.minimum(np.abs(z), F(16))
    t = _rcp((a * F(0.5) + F(1)).astype(F))
    p = np.full_like(t, F(NR_ERFCC[0]))
    for c in NR_ERFCC[1:]:
        p = (p * t + F(c)).astype(F)
    arg = ((-a * a + p).astype(F) * F(1.4426950408889634) + F(64)).astype(F)
    e = (t * _ex2(arg)).astype(F)                          # 2^64 erfc(a)
    c2 = (e * F(-2.0 ** -64) + F(2)).astype(F)             # 2 - erfc(a)
    phi = np.where(z >= 0, e, c2)
    sc = np.where(z >= 0, F(2.0 ** -65), F(0.5))
    return ((x * phi).astype(F) * sc).astype(F)


def tanh_form(x):
    u = (F(0.7978845608028654) * ((F(0.044715) * x).astype(F) * (x * x).astype(F) + x).astype(F)).astype(F)
    au = np.minimum(np.abs(u), F(128))
    e = _ex2((au * F(-2 * 1.4426950408889634) + F(64)).astype(F))  # 2^64 e^{-2|u|}
    den = (e * F(2.0 ** -64) + F(1)).astype(F)
    num = np.where(u >= 0, x, (x * e).astype(F))
    sc = np.where(u >= 0, F(1), F(2.0 ** -64))
    return ((num * _rcp(den)).astype(F) * sc).astype(F)


def _bf16_inputs(lo=-40.0, hi=40.0):
    bits = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    return bits[np.isfinite(bits) & (bits >= lo) & (bits <= hi)]


def _to_bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float64)).to(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("form", ["erf", "tanh"])
def test_formulation_rounds_like_the_exact_gelu(form):
    x = _bf16_inputs()
    xd = x.astype(np.float64)
    if form == "erf":
        got, ref = erf_form(x), 0.5 * xd * erfc(-xd / np.sqrt(2.0))
    else:
        u = np.sqrt(2.0 / np.pi) * (xd + 0.044715 * xd ** 3)
        with np.errstate(over="ignore", invalid="ignore"):
            ref = np.where(u >= 0, xd / (1.0 + np.exp(-2.0 * u)), xd * np.exp(2.0 * u) / (1.0 + np.exp(2.0 * u)))
        got = tanh_form(x)
    # the same bf16 value as the correctly rounded exact GELU, every input
    assert np.array_equal(_to_bf16(got), _to_bf16(ref))
    # and far inside the 2^-9 relative error that one bf16 step allows
    normal = np.abs(ref) > 2.0 ** -126
    rel = np.abs(got.astype(np.float64)[normal] - ref[normal]) / np.abs(ref[normal])
    assert rel.max() < 2.0 ** -14


def test_far_tail_keeps_tiny_values():
    # a result below the normal fp32 range is still produced, not flushed
    x = np.array([-12.0, -13.0, -13.5, -14.0], dtype=np.float32)
    got = erf_form(x)
    assert np.all(got < 0) and np.all(np.abs(got) < 2.0 ** -100)
    assert np.abs(got[-1]) < 2.0 ** -126  # subnormal, kept
    xd = x.astype(np.float64)
    ref = 0.5 * xd * erfc(-xd / np.sqrt(2.0))
    assert np.array_equal(_to_bf16(got), _to_bf16(ref))
