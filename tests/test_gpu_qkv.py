"""GPU parity of the fused QKV post-processing (svdq_linear_forward_qkv):
per-head RMSNorm of Q and K and the rotary embedding applied in the GEMM
epilogue, against oracle/svdq.py::qkv_norm_rope.

Two checks per case:
  * staged: the oracle transform applied to the GPU's own plain layer output
    (same bf16 q values) isolates the epilogue arithmetic: every element
    within 1 bf16 ulp of the float64 result (fp32 vs float64, one rounding),
    V columns bit-identical to the plain layer;
  * end to end: against the oracle's whole chain (its y_ref): relative
    Frobenius error <= 1e-3 on each block; max |err| <= 2e-2 x row RMS on V
    (the plain layer's bar) and 4e-2 on Q and K. The normalised blocks pass
    through two bf16 roundings in series (the layer output the norm reads and
    the final output): a last-bit flip of q on an element of up to ~5x the
    head RMS moves the normalised value by 2^-8 x 5 = 0.02 of the RMS, and the
    final rounding adds up to 2^-9 x 5 = 0.01.
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


def _bf16_cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()


def _run(lib, X, W, b, r, heads, seed, rows=None):
    L1, L2, _ = osv.lowrank_factors(W, r)
    g_x = osv.act_global_scale(X)
    pw = lib.svdq_pack_weight(W.cuda(), _bf16_cuda(L1), _bf16_cuda(L2), float(g_x))
    M = X.shape[0]
    rng = np.random.default_rng(seed)
    wq = nvfp4.bf16_round(rng.uniform(0.5, 1.5, 128))
    wk = nvfp4.bf16_round(rng.uniform(0.5, 1.5, 128))
    cos, sin = workloads.rope_tables(M, 128, seed=seed)
    Xd, bd = X.cuda(), b.cuda()
    Yq = lib.svdq_linear_forward_qkv(Xd, pw, bd, heads, _bf16_cuda(wq), _bf16_cuda(wk), 1e-6,
                                     torch.from_numpy(cos).cuda(), torch.from_numpy(sin).cuda())
    Yp = lib.svdq_linear_forward(Xd, pw, bd)
    torch.cuda.synchronize()
    assert lib.svdq_read_device_error() == 0
    yq, yp = _f64(Yq), _f64(Yp)
    if rows is not None:
        yq, yp, cos, sin = yq[rows], yp[rows], cos[rows], sin[rows]
    hd = heads * 128
    # staged: the same q values through the oracle transform
    st64, _ = osv.qkv_norm_rope(yp, heads, 128, wq, wk, 1e-6, cos, sin)
    ulp = layouts.bf16_ulp_distance(yq[:, :2 * hd], nvfp4.bf16_round(st64[:, :2 * hd]))
    assert ulp.max() <= 1, f"fused epilogue off by {ulp.max()} bf16 ulps"
    assert np.array_equal(yq[:, 2 * hd:], yp[:, 2 * hd:]), "V must be the plain layer output"
    # end to end against the oracle's chain
    ref_pw = osv.pack_weight(W, L1, L2)
    fwd = osv.forward(X if rows is None else X[rows], ref_pw, b, g_x)
    e64, eref = osv.qkv_norm_rope(fwd.y_ref, heads, 128, wq, wk, 1e-6, cos, sin)
    for blk in range(3):
        cols = slice(blk * hd, (blk + 1) * hd)
        assert osv.rel_fro(yq[:, cols], eref[:, cols]) <= 1e-3, f"block {blk}"
        bar = 2e-2 if blk == 2 else 4e-2
        assert osv.max_abs_over_row_rms(yq[:, cols], e64[:, cols]) <= bar, f"block {blk}"


@pytest.mark.parametrize("kernel", ["1sm", "2sm"])
@pytest.mark.parametrize("M,heads,r", [(300, 2, 32), (129, 1, 16), (520, 2, 64)])
def test_qkv_norm_rope_small(lib, monkeypatch, kernel, M, heads, r):
    """Both GEMM kernels (forced), ragged M, several ranks; N = 3 * heads * 128."""
    N = 3 * heads * 128
    if kernel == "2sm" and N % 256 != 0:
        pytest.skip("the CTA-pair GEMM needs N % 256 == 0")
    monkeypatch.setenv("SVDQ_GEMM_KERNEL", kernel)
    _, (X, W, b) = workloads.small_layer(M, 512, N, r, seed=19)
    _run(lib, X, W, b, r, heads, seed=5)


def test_qkv_norm_rope_config2_full_size(lib):
    """The DiT fused-QKV layer at full size (M=4608, 24 heads of 128), 96 sampled rows."""
    spec = workloads.WORKLOADS[2].layers[0]
    X, W, b = workloads.make_layer(spec)
    rows = np.unique(np.concatenate([[0, 1, spec.M - 1], np.random.default_rng(3).choice(spec.M, 93, replace=False)]))
    _run(lib, X, W, b, spec.r, spec.N // 384, seed=7, rows=rows)
