"""GPU parity of smoothing (outliers moved from the activations into the
weights, blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers",
section "Background: SVDQuant and Nunchaku") against the oracle
(oracle/svdq.py: smooth_factors, lowrank_factors, pack_weight, quantize_act,
forward with lambda).

Bars: calibration factors bit-exact for alpha = 0.5 (square roots and one
division, each correctly rounded) and within 1 fp32 ulp for other alpha (a
float64 power function on each side); inv_smooth, activation codes and
scales, packed residual codes / scales / g_w bit-exact; XL1 and Y as in
test_gpu_parity.py; the GPU truncated SVD of the smoothed weight by its
residual energy against the oracle's (Eckart-Young). The oracle computes
every expected value from the seeded inputs; nothing flows from the GPU into
the oracle.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import svdq as osv
from tests import layouts
from tests.test_gpu_parity import MAX_ROWRMS, REL_FRO, _bf16_np, _check_xl1, _to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from w4a4_rank_corrected_svdq_b200 import _lib, build
    build.build()
    return _lib


def _smoothed_layer(M, K, N, r, seed=11, alpha=0.5):
    _, (X, W, b) = workloads.small_layer(M, K, N, r, seed=seed, outliers=8, gain=50.0)
    lam = osv.smooth_factors(X, W, alpha)
    L1, L2, _ = osv.lowrank_factors(W, r, lam)
    return X, W, b, lam, L1, L2


def _f32_ulps(a, b):
    ia = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    ib = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(ia - ib)


@pytest.mark.parametrize("M,K,N", [(300, 1024, 256), (1, 256, 128), (4608, 3072, 1024)])
def test_smooth_factors_bitexact_at_half(lib, M, K, N):
    _, (X, W, b) = workloads.small_layer(M, K, N, 16, seed=5, outliers=8, gain=50.0)
    X = X.clone()
    W = W.clone()
    X[:, 5] = 0            # zero channels get lambda = 1
    W[:, 9] = 0
    lam = lib.svdq_smooth_factors(X.cuda(), W.cuda(), 0.5)
    torch.cuda.synchronize()
    ref = osv.smooth_factors(X, W, 0.5)
    got = lam.cpu().numpy()
    assert got[5] == 1.0 and got[9] == 1.0
    assert np.array_equal(got, ref), f"{np.sum(got != ref)} factors differ"


@pytest.mark.parametrize("alpha", [0.375, 0.8, 0.0, 1.0])
def test_smooth_factors_other_alpha(lib, alpha):
    _, (X, W, b) = workloads.small_layer(200, 512, 384, 16, seed=6, outliers=8, gain=50.0)
    lam = lib.svdq_smooth_factors(X.cuda(), W.cuda(), alpha)
    torch.cuda.synchronize()
    assert _f32_ulps(lam.cpu().numpy(), osv.smooth_factors(X, W, alpha)).max() <= 1


def test_strided_calibration_input(lib):
    _, (X, W, b) = workloads.small_layer(130, 512, 256, 16, seed=8)
    big = torch.zeros((130, 512 + 64), dtype=torch.bfloat16)
    big[:, :512] = X
    lam = lib.svdq_smooth_factors(big.cuda()[:, :512], W.cuda(), 0.5)
    torch.cuda.synchronize()
    assert np.array_equal(lam.cpu().numpy(), osv.smooth_factors(X, W, 0.5))


@pytest.mark.parametrize("N,K,r", [(256, 512, 32), (384, 1024, 64), (128, 256, 16)])
def test_pack_smoothed_bitexact(lib, N, K, r):
    X, W, b, lam, L1, L2 = _smoothed_layer(64, K, N, r)
    ref = osv.pack_weight(W, L1, L2, lam)
    g_x = osv.act_global_scale(X, ref.inv_smooth)
    pw = lib.svdq_pack_weight(W.cuda(), _to_dev(L1), _to_dev(L2), float(g_x),
                              smooth=torch.from_numpy(lam).cuda())
    torch.cuda.synchronize()
    assert lib.svdq_read_device_error() == 0
    assert np.array_equal(pw.inv_smooth.cpu().numpy(), ref.inv_smooth)
    assert np.array_equal(layouts.unpack_codes(pw.codes.cpu().numpy(), N, K), ref.codes)
    assert np.array_equal(layouts.untile_scales(pw.scales.cpu().numpy(), N, K), ref.scales)
    assert pw.gscale.cpu().numpy()[1] == ref.g_w


def test_pack_rejects_a_bad_factor_on_the_device(lib):
    """A lambda that is not positive and finite is reported in the device error word."""
    X, W, b, lam, L1, L2 = _smoothed_layer(8, 256, 128, 16)
    bad = lam.copy()
    bad[3] = 0.0
    lib.svdq_pack_weight(W.cuda(), _to_dev(L1), _to_dev(L2), 1.0, smooth=torch.from_numpy(bad).cuda())
    torch.cuda.synchronize()
    assert lib.svdq_read_device_error() == 1


def test_act_global_scale_smoothed_bitexact(lib):
    X, W, b, lam, L1, L2 = _smoothed_layer(300, 512, 128, 16)
    inv = osv.inv_smooth(lam)
    g = lib.svdq_act_global_scale(X.cuda(), inv_smooth=torch.from_numpy(inv).cuda()).item()
    assert np.float32(g) == osv.act_global_scale(X, inv)


def _act_weight(lib, K, r, L1, g_x, inv):
    pw = lib.PackedWeight(128, K, r, "cuda")
    pw.gscale.copy_(torch.tensor([float(g_x), 1.0, float(g_x), 0.0]))
    pw.l1t.copy_(_to_dev(L1.T))
    pw.inv_smooth = torch.from_numpy(inv).cuda()
    return pw


@pytest.mark.parametrize("rows,ks", [(128, 1), (128, 4), (64, 2), (64, 8)])
@pytest.mark.parametrize("r", [16, 128])
def test_quantize_act_smoothed_every_plan(lib, monkeypatch, rows, ks, r):
    """The smoothed activation kernel under several launch plans: codes and
    scales bit-exact against the oracle's NVFP4 of x * inv[k]; XL1 from the raw
    X with the folded L1. M = 200 leaves a ragged last tile."""
    M, K = 200, 1024
    monkeypatch.setenv("SVDQ_QUANT_PLAN", f"{rows},{ks}")
    X, W, b, lam, L1, L2 = _smoothed_layer(M, K, 128, r)
    inv = osv.inv_smooth(lam)
    g_x = osv.act_global_scale(X, inv)
    pw = _act_weight(lib, K, r, L1, g_x, inv)
    qa = lib.QuantAct(M, K, r, "cuda")
    for buf in (qa.codes, qa.scales, qa.xl1.view(torch.uint8)):
        buf.fill_(0xA5)
    lib.svdq_quantize_act(X.cuda(), pw, out=qa)
    torch.cuda.synchronize()
    codes, scales = osv.quantize_act(X, g_x, inv)
    assert np.array_equal(layouts.unpack_codes(qa.codes.cpu().numpy(), M, K), codes)
    assert np.array_equal(layouts.untile_scales(qa.scales.cpu().numpy(), M, K), scales)
    _check_xl1(_bf16_np(qa.xl1), X, L1)


def _forward_case(lib, X, W, b, lam, L1, L2, rows=None):
    ref_pw = osv.pack_weight(W, L1, L2, lam)
    g_x = osv.act_global_scale(X, ref_pw.inv_smooth)
    pw = lib.svdq_pack_weight(W.cuda(), _to_dev(L1), _to_dev(L2), float(g_x), smooth=torch.from_numpy(lam).cuda())
    Y = lib.svdq_linear_forward(X.cuda(), pw, b.cuda())
    torch.cuda.synchronize()
    assert lib.svdq_read_device_error() == 0
    y = _bf16_np(Y)
    Xr = X if rows is None else X[rows]
    fwd = osv.forward(Xr, ref_pw, b, g_x)
    if rows is not None:
        y = y[rows]
    assert osv.rel_fro(y, fwd.y_ref) <= REL_FRO
    assert osv.max_abs_over_row_rms(y, fwd.y64) <= MAX_ROWRMS
    return y


@pytest.mark.parametrize("M,K,N,r", [(256, 1024, 1024, 32), (129, 512, 384, 64), (517, 1280, 640, 16)])
def test_linear_forward_smoothed(lib, M, K, N, r):
    _forward_case(lib, *_smoothed_layer(M, K, N, r))


def test_smoothed_layer_is_more_accurate_config1(lib):
    """Config 1 end to end on the GPU: calibration, SVD of the smoothed weight,
    pack and forward; the result matches the oracle and is closer to X W^T than
    the unsmoothed layer (oracle: 0.030 against 0.108)."""
    spec = workloads.WORKLOADS[1].layers[0]
    X, W, b = workloads.make_layer(spec)
    Xd, Wd = X.cuda(), W.cuda()
    lam = lib.svdq_smooth_factors(Xd, Wd, 0.5)
    L1, L2, _ = lib.svdq_lowrank_init(Wd, spec.r, smooth=lam)
    pw0 = lib.svdq_pack_weight(Wd, L1, L2, 1.0, smooth=lam)
    g = lib.svdq_act_global_scale(Xd, inv_smooth=pw0.inv_smooth)
    pw = lib.svdq_pack_weight(Wd, L1, L2, g, smooth=lam)
    Y = lib.svdq_linear_forward(Xd, pw, b.cuda())
    torch.cuda.synchronize()
    assert lib.svdq_read_device_error() == 0
    lam_o = osv.smooth_factors(X, W, 0.5)
    assert np.array_equal(lam.cpu().numpy(), lam_o)
    L1h, L2h = _bf16_np(L1), _bf16_np(L2)
    ref_pw = osv.pack_weight(W, L1h, L2h, lam_o)
    g_o = osv.act_global_scale(X, ref_pw.inv_smooth)
    assert np.float32(g.item()) == g_o
    fwd = osv.forward(X, ref_pw, b, g_o)
    y = _bf16_np(Y)
    assert osv.rel_fro(y, fwd.y_ref) <= REL_FRO
    assert osv.max_abs_over_row_rms(y, fwd.y64) <= MAX_ROWRMS
    exact = osv.to_f64(X) @ osv.to_f64(W).T + osv.to_f64(b)[None, :]
    Lp1, Lp2, _ = lib.svdq_lowrank_init(Wd, spec.r)
    gp = lib.svdq_act_global_scale(Xd)
    Yp = lib.svdq_linear_forward(Xd, lib.svdq_pack_weight(Wd, Lp1, Lp2, gp), b.cuda())
    e_s = osv.rel_fro(y, exact)
    e_p = osv.rel_fro(_bf16_np(Yp), exact)
    assert e_s < 0.5 * e_p, (e_s, e_p)


def test_lowrank_smoothed_eckart_young(lib):
    """The GPU truncated SVD of diag(lambda) W^T: residual energy within 1e-4 of
    the oracle's (both bf16-rounded, L1 carrying 1/lambda)."""
    X, W, b, lam, L1o, L2o = _smoothed_layer(64, 1024, 768, 32)
    L1, L2, sig = lib.svdq_lowrank_init(W.cuda(), 32, smooth=torch.from_numpy(lam).cuda())
    torch.cuda.synchronize()
    A = osv.to_f64(W).T * lam.astype(np.float64)[:, None]
    lam64 = lam.astype(np.float64)[:, None]
    e_gpu = float(np.linalg.norm(A - lam64 * (_bf16_np(L1) @ _bf16_np(L2))) ** 2)
    e_ora = float(np.linalg.norm(A - lam64 * (osv.to_f64(L1o) @ osv.to_f64(L2o))) ** 2)
    assert e_gpu <= e_ora * (1 + 1e-4), (e_gpu / e_ora - 1)


def test_config2_smoothed_full_size_sampled(lib):
    """The DiT fused-QKV layer (M=4608, K=3072, N=9216) with smoothing, through
    the launch path the bench times; 96 sampled rows against the oracle."""
    spec = workloads.WORKLOADS[2].layers[0]
    X, W, b = workloads.make_layer(spec)
    lam = osv.smooth_factors(X, W, 0.5)
    L1, L2, _ = osv.lowrank_factors(W, spec.r, lam)
    rows = np.unique(np.concatenate([[0, 1, spec.M - 1], np.random.default_rng(4).choice(spec.M, 93, replace=False)]))
    _forward_case(lib, X, W, b, lam, L1, L2, rows=rows)
