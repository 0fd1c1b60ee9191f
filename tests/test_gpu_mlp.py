"""GPU parity of the MLP pair's fused up projection (svdq_mlp_up_forward):
GELU and the down projection's activation quantisation in the up
projection's GEMM epilogue, against oracle/svdq.py (gelu, quantize_act,
down_proj, forward).

Staged, so that each step is checked on the GPU's own input to it:
  * h against bf16(GELU(y)) of the GPU's plain up-projection output y (the
    same epilogue arithmetic): within 1 bf16 ulp (fp32 GELU against float64);
  * codes and block scales bit-exact against the oracle's NVFP4 of the
    kernel's own h, padding rows' scales zero;
  * XL1 within half a bf16 ulp plus the fp32 summation bound of bf16(h . L1)
    (_check_xl1_of_h);
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


def _check_xl1_of_h(xg, h, Ld1):
    """XL1 = bf16(h . L1_down), F exact products (bf16 x bf16) summed in fp32:
    at most one rounding per product plus one per partial sum (at most one
    partial per 128 columns of h), in any order; u = 2^-23 covers any faithful
    rounding (tensor-core accumulation included). Then one rounding to bf16."""
    F = h.shape[1]
    L = osv.to_f64(Ld1)
    exact = h @ L
    absum = np.abs(h) @ np.abs(L)
    bound = layouts.bf16_half_ulp(xg) + layouts.sum_error_bound(F + F // 128, absum, 2.0 ** -23) + \
        layouts.sum_error_bound(F, absum, 2.0 ** -53)
    err = np.abs(xg - exact)
    assert np.all(err <= bound), f"XL1 error {np.max(err / bound):.2f} x bound"


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
    lib.svdq_mlp_up_forward(X.cuda(), pu, bu.cuda(), ghd, _dev(Ld1.T), approximate, out=qa, h_out=H)
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
    _check_xl1_of_h(_f64(qa.xl1), h, Ld1)
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
    a = lib.svdq_mlp_up_forward(X.cuda(), pu, bu.cuda(), ghd, _dev(Ld1.T), out=None, h_out=H)
    b = lib.svdq_mlp_up_forward(X.cuda(), pu, bu.cuda(), ghd, _dev(Ld1.T))
    torch.cuda.synchronize()
    assert lib.svdq_read_device_error() == 0
    assert torch.equal(a.codes[: M * F // 2], b.codes[: M * F // 2])
    assert torch.equal(a.scales, b.scales) and torch.equal(a.xl1, b.xl1)


# ------------------------------------------------------------------ the DiT feed-forward at full size
@pytest.fixture(scope="module")
def config3(lib):
    """The DiT MLP pair of the benchmark set at full size: M = 4608 tokens,
    3072 -> 12288 -> 3072, rank 32 both ways, seeded inputs of workloads.py.
    The down projection's activation scale g_h is calibrated by the oracle on
    its own h of every row (bf16(GELU(bf16(up(X)))), erf form), computed in row
    chunks; the same g_h serves both GELU forms."""
    up_s, dn_s = workloads.WORKLOADS[3].layers
    X, Wu, bu = workloads.make_layer(up_s)
    Wd, bd = workloads.make_layer(dn_s, rows=1)[1:]
    Lu1, Lu2, _ = osv.lowrank_factors(Wu, up_s.r)
    Ld1, Ld2, _ = osv.lowrank_factors(Wd, dn_s.r)
    g_up = osv.act_global_scale(X)
    ref_pu = osv.pack_weight(Wu, Lu1, Lu2)
    ref_pd = osv.pack_weight(Wd, Ld1, Ld2)
    amax = 0.0
    for m0 in range(0, up_s.M, 1152):
        y = osv.forward(X[m0:m0 + 1152], ref_pu, bu, g_up).y_ref
        amax = max(amax, float(np.max(np.abs(nvfp4.bf16_round(osv.gelu(y))))))
    g_h = nvfp4.global_scale(np.array([amax]))
    pu = lib.svdq_pack_weight(Wu.cuda(), _dev(Lu1), _dev(Lu2), float(g_up))
    pd = lib.svdq_pack_weight(Wd.cuda(), _dev(Ld1), _dev(Ld2), float(g_h))
    rng = np.random.default_rng(31)
    rows = np.unique(np.concatenate([[0, 1, up_s.M - 1], rng.choice(up_s.M, 93, replace=False)]))
    return dict(X=X, bu=bu, bd=bd, Ld1=Ld1, g_up=g_up, g_h=g_h, ref_pu=ref_pu, ref_pd=ref_pd, pu=pu, pd=pd,
                rows=rows, M=up_s.M, F=up_s.N, D=dn_s.N)


@pytest.mark.parametrize("approximate", [False, True])
def test_mlp_pair_config3_full_size(lib, monkeypatch, config3, approximate):
    """The fused up projection plus the down GEMM on the full DiT feed-forward
    (48 N tiles of the up projection, F = 12288 columns of h per row), through
    the launch path the bench times, on 96 sampled rows (first, second, last
    and random ones):
      * staged, each step against the oracle on the GPU's own input to it: h
        within 1 bf16 ulp of bf16(GELU(y)) of the GPU's plain up-projection
        output y; codes and block scales bit-exact; XL1 within its summation
        bound; the down projection within the layer bars;
      * end to end against oracle.mlp_pair on X alone: the up projection's y
        and the pair's output within the layer bars (relative Frobenius <= 1e-3
        against the bf16 reference, max |err| <= 2e-2 x row RMS against
        float64); h within GELU's slope times y's own difference plus the
        roundings, elementwise (h inherits the up projection's last-bit
        differences, which the layer bars allow, so it is not held to 1 ulp)."""
    c = config3
    monkeypatch.setenv("SVDQ_GEMM_KERNEL", "2sm")
    M, F, rows = c["M"], c["F"], c["rows"]
    Xd = c["X"].cuda()
    qa = lib.QuantAct(M, F, 32, "cuda")
    for b in (qa.codes, qa.scales, qa.xl1.view(torch.uint8)):
        b.fill_(0xA5)
    H = torch.empty((M, F), dtype=torch.bfloat16, device="cuda")
    ghd = torch.tensor([float(c["g_h"])], dtype=torch.float32, device="cuda")
    lib.svdq_mlp_up_forward(Xd, c["pu"], c["bu"].cuda(), ghd, _dev(c["Ld1"].T), approximate, out=qa, h_out=H)
    Yd = lib.svdq_w4a4_gemm(qa, c["pd"], c["bd"].cuda())
    Yup = lib.svdq_linear_forward(Xd, c["pu"], c["bu"].cuda())
    torch.cuda.synchronize()
    assert lib.svdq_read_device_error() == 0
    h = _f64(H)[rows]
    codes = layouts.unpack_codes(qa.codes.cpu().numpy(), M, F)[rows]
    scales = layouts.untile_scales(qa.scales.cpu().numpy(), M, F)[rows]
    xl1 = _f64(qa.xl1)[rows]
    y_dn = _f64(Yd)[rows]
    # staged
    h_st = nvfp4.bf16_round(osv.gelu(_f64(Yup)[rows], approximate))
    assert layouts.bf16_ulp_distance(h, h_st).max() <= 1
    ref_codes, ref_scales = osv.quantize_act(h, c["g_h"])
    assert np.array_equal(codes, ref_codes) and np.array_equal(scales, ref_scales)
    _check_xl1_of_h(xl1, h, c["Ld1"])
    st = osv.forward(h, c["ref_pd"], c["bd"], c["g_h"])
    assert osv.rel_fro(y_dn, st.y_ref) <= 1e-3
    assert osv.max_abs_over_row_rms(y_dn, st.y64) <= 2e-2
    # end to end
    pair = osv.mlp_pair(c["X"][rows], c["ref_pu"], c["bu"], c["g_up"], c["ref_pd"], c["bd"], c["g_h"], approximate)
    y_up = _f64(Yup)[rows]
    assert osv.rel_fro(y_up, pair.up.y_ref) <= 1e-3
    assert osv.max_abs_over_row_rms(y_up, pair.up.y64) <= 2e-2
    # h = bf16(GELU(y)) inherits y's differences through GELU's slope: within
    # L |y - y_ref| plus the roundings (1 ulp staged, 1/2 ulp of each bf16 GELU)
    lip = _gelu_lipschitz(approximate)
    bound = lip * np.abs(y_up - pair.up.y_ref) + 3.0 * layouts.bf16_half_ulp(h) + layouts.bf16_half_ulp(pair.h)
    assert np.all(np.abs(h - pair.h) <= bound)
    assert osv.rel_fro(h, pair.h) <= 1e-3
    assert osv.rel_fro(y_dn, pair.down.y_ref) <= 1e-3
    assert osv.max_abs_over_row_rms(y_dn, pair.down.y64) <= 2e-2


def _gelu_lipschitz(approximate):
    """sup |GELU'| (1.129 at x = sqrt 2 for x Phi(x)), from the oracle's GELU on a
    fine grid (difference quotients over the whole real line's relevant range),
    with 1 % margin for the grid."""
    x = np.linspace(-12.0, 12.0, 480001)
    g = osv.gelu(x, approximate)
    return 1.01 * float(np.max(np.abs(np.diff(g) / np.diff(x))))
