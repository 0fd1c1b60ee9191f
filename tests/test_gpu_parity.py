"""GPU parity: the CUDA path through the C ABI against the float64 CPU oracle.

Bars (from the layer's acceptance criteria):
  * activation codes and scales, packed weight codes / scales / g_w: bit-exact;
  * XL1: within half a bf16 ulp of its own value plus the fp32 summation error
    bound of the exact float64 product (the blog's fused down projection
    accumulates in fp32 in an order it does not fix; see _check_xl1), and within
    1 bf16 ulp of the oracle wherever that bound is below a quarter ulp;
  * Y: relative Frobenius error <= 1e-3 against the oracle output rounded to
    bf16, and max |Y - y64| <= 2e-2 * RMS of the y64 row.
Inputs come from the seeded generators in workloads.py; the oracle computes
the expected values; nothing flows from the GPU into the oracle.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import nvfp4, svdq as osv
from tests import layouts

pytestmark = pytest.mark.gpu

REL_FRO = 1e-3
MAX_ROWRMS = 2e-2


@pytest.fixture(scope="module")
def lib():
    from w4a4_rank_corrected_svdq_b200 import _lib, build
    build.build()
    return _lib


def _bf16_np(t):
    return t.detach().to(torch.float64).cpu().numpy()


def _to_dev(a64):
    return torch.from_numpy(np.ascontiguousarray(a64)).to(torch.bfloat16).cuda()


def _layer(M, K, N, r, seed=7, bias=True):
    spec, (X, W, b) = workloads.small_layer(M, K, N, r, seed=seed, bias_std=0.01 if bias else 0.0)
    L1, L2, _ = osv.lowrank_factors(W, r)
    return X, W, b, L1, L2


def _act_only_weight(lib, K, r, L1, g_x):
    """A packed-weight holder carrying only what svdq_quantize_act reads (g_x, l1t)."""
    pw = lib.PackedWeight(128, K, r, "cuda")
    pw.gscale.copy_(torch.tensor([float(g_x), 1.0, float(g_x), 0.0]))
    pw.l1t.copy_(_to_dev(L1.T))
    return pw


def _check_act(lib, X, L1, r, g_x, qa, M, K):
    ref = osv.quantize_act(X, g_x)
    codes = layouts.unpack_codes(qa.codes.cpu().numpy(), M, K)
    scales_buf = qa.scales.cpu().numpy()
    scales = layouts.untile_scales(scales_buf, M, K)
    assert np.array_equal(codes, ref[0]), f"codes differ at {np.argwhere(codes != ref[0])[:5]}"
    assert np.array_equal(scales, ref[1]), f"scales differ at {np.argwhere(scales != ref[1])[:5]}"
    mpad = (M + 127) // 128 * 128
    if mpad > M:   # padding rows must hold zero scales
        pad = layouts.untile_scales(scales_buf, mpad, K)[M:]
        assert not pad.any()
    _check_xl1(_bf16_np(qa.xl1), X, L1)


def _check_xl1(xl1_gpu, X, L1):
    """XL1 = bf16(X . L1): K exact products (bf16 x bf16 fits fp32) summed in
    fp32 by the tensor cores and the K-split's partial additions, K - 1
    roundings in an order the pages leave open, then one rounding to bf16.
      * bound: |gpu - exact| <= 1/2 ulp_bf16(gpu) + gamma_{K-1} sum_k |x_k L1_kj|
        with u = 2^-23 (any faithful rounding; the tensor cores' internal
        rounding is not specified), plus the oracle's own float64 error;
      * where that summation bound is below a quarter of a bf16 ulp of the
        oracle's value, the fp32 sum and the exact sum round to bf16 values at
        most one step apart, so those elements must be within 1 ulp."""
    X64, L164 = osv.to_f64(X), osv.to_f64(L1)
    exact = X64 @ L164
    absum = np.abs(X64) @ np.abs(L164)
    K = X64.shape[1]
    summ = layouts.sum_error_bound(K - 1, absum, 2.0 ** -23) + layouts.sum_error_bound(K, absum, 2.0 ** -53)
    bound = layouts.bf16_half_ulp(xl1_gpu) + summ
    err = np.abs(xl1_gpu - exact)
    assert np.all(err <= bound), f"XL1 error {np.max(err / bound):.2f} x bound"
    oracle = osv.down_proj(X, L1)
    tight = summ < 0.5 * layouts.bf16_half_ulp(oracle)
    ulps = layouts.bf16_ulp_distance(xl1_gpu, oracle)
    assert np.all(ulps[tight] <= 1), f"XL1: {np.sum(ulps[tight] > 1)} elements beyond 1 ulp where the bound allows 1"


def _check_y(Y, fwd, rows=None):
    y = _bf16_np(Y)
    if rows is not None:
        y = y[rows]
    rel = osv.rel_fro(y, fwd.y_ref)
    mx = osv.max_abs_over_row_rms(y, fwd.y64)
    assert rel <= REL_FRO, f"rel Frobenius {rel:.3e}"
    assert mx <= MAX_ROWRMS, f"max |err| / row-RMS {mx:.3e}"
    return rel, mx


# ------------------------------------------------------------------ calibration
def test_act_global_scale_bitexact(lib):
    X, *_ = _layer(300, 512, 128, 16)
    g = lib.svdq_act_global_scale(X.cuda()).item()
    assert np.float32(g) == osv.act_global_scale(X)
    z = lib.svdq_act_global_scale(torch.zeros((5, 256), dtype=torch.bfloat16, device="cuda")).item()
    assert z == 1.0


# ------------------------------------------------------------------ activation kernel
@pytest.mark.parametrize("M,K,r", [(256, 1024, 32), (1, 256, 16), (127, 512, 32), (129, 512, 64),
                                   (300, 768, 128), (64, 4096, 32), (1000, 256, 16)])
def test_quantize_act_bitexact(lib, M, K, r):
    X, W, b, L1, L2 = _layer(M, K, 128, r)
    g_x = osv.act_global_scale(X)
    pw = _act_only_weight(lib, K, r, L1, g_x)
    qa = lib.svdq_quantize_act(X.cuda(), pw)
    torch.cuda.synchronize()
    _check_act(lib, X, L1, r, g_x, qa, M, K)


@pytest.mark.parametrize("rows", [64, 128])
@pytest.mark.parametrize("ks", [1, 2, 4, 8])
@pytest.mark.parametrize("r", [16, 32, 64, 128])
def test_quantize_act_every_launch_plan(lib, monkeypatch, rows, ks, r):
    """Every launch plan of the activation kernel: 64- or 128-row tiles, K split
    over a cluster of 1, 2, 4 or 8 CTAs, every rank; M = 200 leaves a ragged
    last tile for both heights and an odd count of 64-row tiles."""
    M, K = 200, 1024
    monkeypatch.setenv("SVDQ_QUANT_PLAN", f"{rows},{ks}")
    X, W, b, L1, L2 = _layer(M, K, 128, r)
    g_x = osv.act_global_scale(X)
    pw = _act_only_weight(lib, K, r, L1, g_x)
    qa = lib.QuantAct(M, K, r, "cuda")
    for buf in (qa.codes, qa.scales, qa.xl1.view(torch.uint8)):
        buf.fill_(0xA5)   # every output byte, padding included, must be written
    lib.svdq_quantize_act(X.cuda(), pw, out=qa)
    torch.cuda.synchronize()
    _check_act(lib, X, L1, r, g_x, qa, M, K)


def test_quantize_act_zero_rows_and_strided_input(lib):
    M, K, r = 130, 512, 32
    X, W, b, L1, L2 = _layer(M, K, 128, r)
    X = X.clone()
    X[3] = 0
    X[7, 16:48] = 0
    big = torch.zeros((M, K + 64), dtype=torch.bfloat16)
    big[:, :K] = X
    g_x = osv.act_global_scale(X)
    pw = _act_only_weight(lib, K, r, L1, g_x)
    qa = lib.svdq_quantize_act(big.cuda()[:, :K], pw)
    torch.cuda.synchronize()
    _check_act(lib, X, L1, r, g_x, qa, M, K)


# ------------------------------------------------------------------ weight packing
@pytest.mark.parametrize("N,K,r", [(128, 256, 16), (256, 512, 32), (384, 1024, 64), (256, 512, 128)])
def test_pack_weight_bitexact(lib, N, K, r):
    X, W, b, L1, L2 = _layer(8, K, N, r)
    g_x = osv.act_global_scale(X)
    pw = lib.svdq_pack_weight(W.cuda(), _to_dev(L1), _to_dev(L2), float(g_x))
    torch.cuda.synchronize()
    ref = osv.pack_weight(W, L1, L2)
    codes = layouts.unpack_codes(pw.codes.cpu().numpy(), N, K)
    scales = layouts.untile_scales(pw.scales.cpu().numpy(), N, K)
    gs = pw.gscale.cpu().numpy()
    assert gs[0] == g_x and gs[1] == ref.g_w and gs[2] == np.float32(g_x * ref.g_w) and gs[3] == 0
    assert np.array_equal(scales, ref.scales)
    assert np.array_equal(codes, ref.codes)
    assert np.array_equal(_bf16_np(pw.l1t), L1.T)
    # l2s: documented encoding of L2^T / alpha as bf16 hi + lo (include/svdq.h)
    v = (L2.T.astype(np.float32) / np.float32(gs[2])).astype(np.float32)
    hi = nvfp4.bf16_round(v)
    lo = nvfp4.bf16_round((v - hi.astype(np.float32)).astype(np.float32))
    l2s = _bf16_np(pw.l2s)
    assert np.array_equal(l2s[0], hi) and np.array_equal(l2s[1], lo)
    assert np.max(np.abs((l2s[0] + l2s[1]) * float(gs[2]) - L2.T)) <= 2 ** -15 * np.max(np.abs(L2))


# ------------------------------------------------------------------ full layer
@pytest.mark.parametrize("splitk", ["0", "1"])
@pytest.mark.parametrize("M,K,N,r,bias", [(256, 1024, 1024, 32, True), (1, 256, 128, 16, True),
                                          (129, 512, 384, 64, False), (300, 768, 256, 128, True),
                                          (517, 1280, 640, 32, True), (128, 4096, 1024, 16, True),
                                          (200, 2048, 768, 128, True), (64, 512, 2048, 32, False)])
def test_linear_forward_parity(lib, monkeypatch, splitk, M, K, N, r, bias):
    """The layer through the library's own kernel choice, and with few rows also
    with K split across a thread-block cluster (SVDQ_GEMM_SPLITK=1)."""
    monkeypatch.setenv("SVDQ_GEMM_SPLITK", splitk)
    X, W, b, L1, L2 = _layer(M, K, N, r, bias=bias)
    g_x = osv.act_global_scale(X)
    pw = lib.svdq_pack_weight(W.cuda(), _to_dev(L1), _to_dev(L2), float(g_x))
    Y = lib.svdq_linear_forward(X.cuda(), pw, b.cuda() if bias else None)
    torch.cuda.synchronize()
    assert lib.svdq_read_device_error() == 0
    fwd = osv.forward(X, osv.pack_weight(W, L1, L2), b if bias else None, g_x)
    _check_y(Y, fwd)


def test_linear_forward_config1(lib):
    spec = workloads.WORKLOADS[1].layers[0]
    X, W, b = workloads.make_layer(spec)
    L1, L2, _ = osv.lowrank_factors(W, spec.r)
    g_x = lib.svdq_act_global_scale(X.cuda())      # calibration on the GPU, then pack
    assert np.float32(g_x.item()) == osv.act_global_scale(X)
    pw = lib.svdq_pack_weight(W.cuda(), _to_dev(L1), _to_dev(L2), g_x)
    g_x = osv.act_global_scale(X)
    qa = lib.svdq_quantize_act(X.cuda(), pw)
    Y = lib.svdq_w4a4_gemm(qa, pw, b.cuda())
    torch.cuda.synchronize()
    _check_act(lib, X, L1, spec.r, g_x, qa, spec.M, spec.K)
    fwd = osv.forward(X, osv.pack_weight(W, L1, L2), b, g_x)
    _check_y(Y, fwd)
    # deterministic: a second call gives identical bits
    Y2 = lib.svdq_linear_forward(X.cuda(), pw, b.cuda())
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)


def test_m_zero_is_noop(lib):
    pw = lib.PackedWeight(128, 256, 16, "cuda")
    X = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    Y = lib.svdq_linear_forward(X, pw)
    assert Y.shape == (0, 128)


# ------------------------------------------------------------------ CTA-pair (2-SM) GEMM
@pytest.mark.parametrize("M,K,N,r", [(1, 256, 256, 16), (129, 512, 512, 64), (300, 768, 256, 128),
                                     (600, 1280, 768, 32), (4096, 512, 4096, 32), (2304, 256, 2560, 128)])
def test_linear_forward_parity_pair_kernel(lib, monkeypatch, M, K, N, r):
    """The 256x256-tile CTA-pair kernel (forced), including persistent loops over
    several tiles per pair, partial row tiles and every rank."""
    monkeypatch.setenv("SVDQ_GEMM_KERNEL", "2sm")
    X, W, b, L1, L2 = _layer(M, K, N, r)
    g_x = osv.act_global_scale(X)
    pw = lib.svdq_pack_weight(W.cuda(), _to_dev(L1), _to_dev(L2), float(g_x))
    Y = lib.svdq_linear_forward(X.cuda(), pw, b.cuda())
    torch.cuda.synchronize()
    assert lib.svdq_read_device_error() == 0
    fwd = osv.forward(X, osv.pack_weight(W, L1, L2), b, g_x)
    _check_y(Y, fwd)
    # the single-CTA kernel computes the same layer
    monkeypatch.setenv("SVDQ_GEMM_KERNEL", "1sm")
    Y1 = lib.svdq_linear_forward(X.cuda(), pw, b.cuda())
    torch.cuda.synchronize()
    assert osv.rel_fro(_bf16_np(Y1), _bf16_np(Y)) <= REL_FRO


def _full_size_sampled(lib, spec, n_sample=96, seed=17):
    """One workload layer at full size through the launch path bench.py times
    (svdq_quantize_act + svdq_w4a4_gemm, kernel plans chosen by the library);
    the oracle checks the packed weight in full and `n_sample` rows (the first,
    second and last plus random ones) of the activation codes, scales and Y."""
    X, W, b = workloads.make_layer(spec)
    L1, L2, _ = osv.lowrank_factors(W, spec.r)
    g_x = osv.act_global_scale(X)
    pw = lib.svdq_pack_weight(W.cuda(), _to_dev(L1), _to_dev(L2), float(g_x))
    qa = lib.svdq_quantize_act(X.cuda(), pw)
    Y = lib.svdq_w4a4_gemm(qa, pw, b.cuda())
    torch.cuda.synchronize()
    assert lib.svdq_read_device_error() == 0
    rng = np.random.default_rng(seed)
    extra = min(spec.M, n_sample) - 3
    rows = np.unique(np.concatenate([[0, 1, spec.M - 1], rng.choice(spec.M, max(extra, 0), replace=False)]))
    ref_pw = osv.pack_weight(W, L1, L2)
    codes = layouts.unpack_codes(pw.codes.cpu().numpy(), spec.N, spec.K)
    assert np.array_equal(codes, ref_pw.codes)
    fwd = osv.forward(X[rows], ref_pw, b, g_x)
    act_codes = layouts.unpack_codes(qa.codes.cpu().numpy(), spec.M, spec.K)[rows]
    act_scales = layouts.untile_scales(qa.scales.cpu().numpy(), spec.M, spec.K)[rows]
    assert np.array_equal(act_codes, fwd.codes) and np.array_equal(act_scales, fwd.scales)
    _check_xl1(_bf16_np(qa.xl1)[rows], X[rows], L1)
    return _check_y(Y, fwd, rows=rows)


def test_config2_full_size_sampled_rows(lib):
    """The DiT fused-QKV workload at full size (M=4608, K=3072, N=9216, r=32),
    the configuration bench.py times."""
    _full_size_sampled(lib, workloads.WORKLOADS[2].layers[0])


@pytest.mark.parametrize("layer", range(len(workloads.WORKLOADS[3].layers)),
                         ids=[l.name for l in workloads.WORKLOADS[3].layers])
def test_config3_full_size_sampled_rows(lib, layer):
    """DiT MLP pair at full size: up 3072->12288 and down 12288->3072, M=4608."""
    _full_size_sampled(lib, workloads.WORKLOADS[3].layers[layer])


@pytest.mark.parametrize("layer", range(len(workloads.WORKLOADS[4].layers)),
                         ids=[l.name for l in workloads.WORKLOADS[4].layers])
def test_config4_full_size_sampled_rows(lib, layer):
    """Batched DiT block at M=18432: QKV, attention out, MLP up and MLP down."""
    _full_size_sampled(lib, workloads.WORKLOADS[4].layers[layer])


@pytest.mark.parametrize("layer", range(len(workloads.WORKLOADS[5].layers)),
                         ids=[l.name for l in workloads.WORKLOADS[5].layers])
def test_config5_full_size_sampled_rows(lib, layer):
    """Rank and shape sweep K=N=4096, M in {128, 1024, 8192}, r in {16..128}
    (M=128 runs the single-CTA GEMM, the others the CTA-pair GEMM)."""
    _full_size_sampled(lib, workloads.WORKLOADS[5].layers[layer])
