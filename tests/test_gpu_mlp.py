"""GPU parity of the MLP pair's fused up projection (svdq_mlp_up_forward):
GELU and the down projection's activation quantisation in the up
projection's GEMM epilogue, against oracle/svdq.py (gelu, quantize_act,
down_proj, forward).

Staged, so that each step is checked on the GPU's own input to it:
  * h against bf16(GELU(y)) of the GPU's plain up-projection output y (the
    same epilogue arithmetic): within 1 bf16 ulp (fp32 GELU against float64);
  * codes and block scales bit-exact against the oracle's NVFP4 of the
    kernel's own h, padding rows' scales zero;
  * XL1 within half a bf16 ulp plus the fp32 summation bound of bf16(h . L1);
  * the down projection, run on these buffers, within the layer bars against
    the oracle's forward of h.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import nvfp4, svdq as osv
from tests import layouts

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from w4a4_rank_corrected_svdq_b200 import _lib, build
    build.build()
    return _lib


def _f64(t):
    return t.detach().to(torch.float64).cpu().numpy()


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()


def _case(lib, M, D, F, r, approximate, seed=1):
    _, (X, Wu, bu) = workloads.small_layer(M, D, F, r, seed=seed)
    _, (_, Wd, bd) = workloads.small_layer(M, F, D, r, seed=seed + 1)
    Lu1, Lu2, _ = osv.lowrank_factors(Wu, r)
    Ld1, Ld2, _ = osv.lowrank_factors(Wd, 32)
    pu = lib.svdq_pack_weight(Wu.cuda(), _dev(Lu1), _dev(Lu2), float(osv.act_global_scale(X)))
    Yup = lib.svdq_linear_forward(X.cuda(), pu, bu.cuda())
    torch.cuda.synchronize()
    h_st = nvfp4.bf16_round(osv.gelu(_f64(Yup), approximate))
    gh = osv.act_global_scale(h_st)
    return X, Wd, bu, bd, Ld1, Ld2, pu, h_st, gh


@pytest.mark.parametrize("M,D,F,r,approximate", [(300, 512, 1024, 32, False), (600, 256, 512, 16, True),
                                                 (129, 512, 768, 64, False)])
def test_mlp_up_staged(lib, monkeypatch, M, D, F, r, approximate):
    # the plain reference run takes the CTA-pair kernel the fused path uses (same epilogue arithmetic for y)
    monkeypatch.setenv("SVDQ_GEMM_KERNEL", "2sm")
    X, Wd, bu, bd, Ld1, Ld2, pu, h_st, gh = _case(lib, M, D, F, r, approximate)
    qa = lib.QuantAct(M, F, 32, "cuda")
    for b in (qa.codes, qa.scales, qa.xl1.view(torch.uint8)):
        b.fill_(0xA5)
    H = torch.empty((M, F), dtype=torch.bfloat16, device="cuda")
    ghd = torch.tensor([float(gh)], dtype=torch.float32, device="cuda")
    lib.svdq_mlp_up_forward(X.cuda(), pu, bu.cuda(), ghd, _dev(Ld1), approximate, out=qa, h_out=H)
    pd = lib.svdq_pack_weight(Wd.cuda(), _dev(Ld1), _dev(Ld2), float(gh))
    Yd = lib.svdq_w4a4_gemm(qa, pd, bd.cuda())
    torch.cuda.synchronize()
    assert lib.svdq_read_device_error() == 0
    h = _f64(H)
    assert layouts.bf16_ulp_distance(h, h_st).max() <= 1
    codes, scales = osv.quantize_act(h, gh)
    assert np.array_equal(layouts.unpack_codes(qa.codes.cpu().numpy(), M, F), codes)
    sbuf = qa.scales.cpu().numpy()
    assert np.array_equal(layouts.untile_scales(sbuf, M, F), scales)
    mpad = (M + 127) // 128 * 128
    if mpad > M:
        assert not layouts.untile_scales(sbuf, mpad, F)[M:].any()
    exact = h @ osv.to_f64(Ld1)
    absum = np.abs(h) @ np.abs(osv.to_f64(Ld1))
    xg = _f64(qa.xl1)
    bound = np.ldexp(1.0, np.frexp(np.abs(xg))[1] - 9) + 2.0 * (F + 96) * 2.0 ** -24 * absum
    assert np.all(np.abs(xg - exact) <= bound)
    fwd = osv.forward(h, osv.pack_weight(Wd, Ld1, Ld2), bd, gh)
    y = _f64(Yd)
    assert osv.rel_fro(y, fwd.y_ref) <= 1e-3
    assert osv.max_abs_over_row_rms(y, fwd.y64) <= 2e-2


def test_mlp_up_without_storing_h(lib):
    """Without h_out the kernel writes the same codes, scales and XL1."""
    M, D, F, r = 300, 512, 1024, 32
    X, Wd, bu, bd, Ld1, Ld2, pu, h_st, gh = _case(lib, M, D, F, r, False, seed=5)
    ghd = torch.tensor([float(gh)], dtype=torch.float32, device="cuda")
    H = torch.empty((M, F), dtype=torch.bfloat16, device="cuda")
    a = lib.svdq_mlp_up_forward(X.cuda(), pu, bu.cuda(), ghd, _dev(Ld1), out=None, h_out=H)
    b = lib.svdq_mlp_up_forward(X.cuda(), pu, bu.cuda(), ghd, _dev(Ld1))
    torch.cuda.synchronize()
    assert lib.svdq_read_device_error() == 0
    assert torch.equal(a.codes[: M * F // 2], b.codes[: M * F // 2])
    assert torch.equal(a.scales, b.scales) and torch.equal(a.xl1, b.xl1)
