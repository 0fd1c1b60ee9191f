"""GPU parity of the dynamic activation scale (svdq_linear_forward_dynamic):
g_x computed from each call's X instead of the calibrated value.

The oracle's forward with g = act_global_scale(X, inv_smooth) of the same X
is the expected result (the oracle formula is the same for a calibrated and a
per-call scale): activation codes and scales bit-exact (read back from the
workspace), the per-call scales bit-exact, Y within the layer's bars. With a
calibration on the same X the calibrated and the dynamic layer are the same
computation, so Y is bit-identical.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import svdq as osv
from tests import layouts
from tests.test_gpu_parity import MAX_ROWRMS, REL_FRO, _bf16_np, _to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from w4a4_rank_corrected_svdq_b200 import _lib, build
    build.build()
    return _lib


def _layer(M, K, N, r, seed=21, smooth=False):
    _, (X, W, b) = workloads.small_layer(M, K, N, r, seed=seed, outliers=8, gain=50.0)
    lam = osv.smooth_factors(X, W) if smooth else None
    L1, L2, _ = osv.lowrank_factors(W, r, lam)
    return X, W, b, lam, L1, L2


def _pack(lib, W, L1, L2, g, lam):
    return lib.svdq_pack_weight(W.cuda(), _to_dev(L1), _to_dev(L2), g,
                                smooth=None if lam is None else torch.from_numpy(lam).cuda())


@pytest.mark.parametrize("smooth", [False, True])
def test_dynamic_equals_calibration_on_the_same_input(lib, smooth):
    X, W, b, lam, L1, L2 = _layer(300, 1024, 512, 32, smooth=smooth)
    inv = None if lam is None else osv.inv_smooth(lam)
    g = osv.act_global_scale(X, inv)
    pw = _pack(lib, W, L1, L2, float(g), lam)
    Xd, bd = X.cuda(), b.cuda()
    Ys = lib.svdq_linear_forward(Xd, pw, bd)
    Yd = lib.svdq_linear_forward_dynamic(Xd, pw, bd)
    torch.cuda.synchronize()
    assert lib.svdq_read_device_error() == 0
    assert torch.equal(Ys, Yd)


@pytest.mark.parametrize("M,K,N,r,smooth", [(300, 1024, 512, 32, False), (129, 512, 384, 64, True),
                                            (1000, 768, 256, 16, True), (1, 256, 128, 128, False)])
def test_dynamic_scale_tracks_the_call(lib, M, K, N, r, smooth):
    """Packed with a scale calibrated on other data (X / 8): the dynamic layer
    uses this call's scale; codes, scales and the per-call scales bit-exact."""
    X, W, b, lam, L1, L2 = _layer(M, K, N, r, smooth=smooth)
    inv = None if lam is None else osv.inv_smooth(lam)
    g_cal = osv.act_global_scale(osv.to_f64(X) / 8.0, inv)
    pw = _pack(lib, W, L1, L2, float(g_cal), lam)
    ws = torch.empty(lib.svdq_dynamic_workspace_size(M, N, K, r), dtype=torch.uint8, device="cuda")
    Y = lib.svdq_linear_forward_dynamic(X.cuda(), pw, b.cuda(), workspace=ws)
    torch.cuda.synchronize()
    assert lib.svdq_read_device_error() == 0
    g = osv.act_global_scale(X, inv)
    ref_pw = osv.pack_weight(W, L1, L2, lam)
    base = lib.svdq_forward_workspace_size(M, K, r)
    gs = ws[base:base + 16].view(torch.float32).cpu().numpy()
    assert gs[0] == g and gs[1] == ref_pw.g_w and gs[2] == np.float32(g * ref_pw.g_w)
    cb, sb, _ = lib.svdq_act_sizes(M, K, r)
    codes, scales = osv.quantize_act(X, g, inv)
    wsn = ws.cpu().numpy()
    assert np.array_equal(layouts.unpack_codes(wsn[:cb], M, K), codes)
    s_off = (cb + 255) // 256 * 256
    assert np.array_equal(layouts.untile_scales(wsn[s_off:s_off + sb], M, K), scales)
    fwd = osv.forward(X, ref_pw, b, g)
    y = _bf16_np(Y)
    assert osv.rel_fro(y, fwd.y_ref) <= REL_FRO
    assert osv.max_abs_over_row_rms(y, fwd.y64) <= MAX_ROWRMS


def test_dynamic_zero_input(lib):
    """An all-zero X: g = 1, Y = bias."""
    X, W, b, lam, L1, L2 = _layer(64, 512, 256, 16)
    pw = _pack(lib, W, L1, L2, 0.5, None)
    Y = lib.svdq_linear_forward_dynamic(torch.zeros_like(X).cuda(), pw, b.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(_bf16_np(Y), np.broadcast_to(osv.to_f64(b), (64, 256)))


def test_dynamic_config2_full_size_sampled(lib):
    """The DiT fused-QKV layer at full size, calibrated on other data, 96 sampled rows."""
    spec = workloads.WORKLOADS[2].layers[0]
    X, W, b = workloads.make_layer(spec)
    L1, L2, _ = osv.lowrank_factors(W, spec.r)
    pw = _pack(lib, W, L1, L2, float(osv.act_global_scale(osv.to_f64(X) * 3.0)), None)
    Y = lib.svdq_linear_forward_dynamic(X.cuda(), pw, b.cuda())
    torch.cuda.synchronize()
    assert lib.svdq_read_device_error() == 0
    rows = np.unique(np.concatenate([[0, 1, spec.M - 1], np.random.default_rng(5).choice(spec.M, 93, replace=False)]))
    g = osv.act_global_scale(X)
    fwd = osv.forward(X[rows], osv.pack_weight(W, L1, L2), b, g)
    y = _bf16_np(Y)[rows]
    assert osv.rel_fro(y, fwd.y_ref) <= REL_FRO
    assert osv.max_abs_over_row_rms(y, fwd.y64) <= MAX_ROWRMS
