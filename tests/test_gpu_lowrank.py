"""GPU truncated SVD (svdq_lowrank_init, the load-time step S0) against the
oracle's float64 LAPACK SVD (oracle/svdq.py::lowrank_factors).

The GPU method (randomized subspace iteration in float64) approximates the
truncated SVD, so it is compared by what the mathematics fixes rather than
element by element (singular vectors of a flat spectrum are not unique):
  * Eckart-Young: the residual energy ||W^T - L1 L2||_F^2 of the GPU factors
    is at most (1 + tol) times that of the oracle's factors (both rounded to
    bf16). tol follows the method's convergence with 32 power iterations and
    32 oversampling columns, measured on these spectra by a float64 restatement
    of the iteration: about 1e-6 at rank 32 and 2e-4 at rank 128 on flat
    Gaussian spectra;
  * singular values separated by a planted low-rank part agree to 1e-9;
  * the rows of L2 are orthonormal to bf16 precision;
  * an exactly rank-5 weight leaves a residual at the bf16 rounding level;
  * W = 0 gives zero factors; a seed gives identical bytes;
  * the GPU factors, packed and run through the forward pass, match the
    oracle given the same factors.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import svdq as osv
from tests import layouts

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from w4a4_rank_corrected_svdq_b200 import _lib, build
    build.build()
    return _lib


def _f64(t):
    return t.detach().to(torch.float64).cpu().numpy()


def _residual_energy(W, L1, L2):
    A = osv.to_f64(W).T
    return float(np.linalg.norm(A - np.asarray(L1, np.float64) @ np.asarray(L2, np.float64)) ** 2)


def _compare(lib, W, r, tol, seed=3):
    L1, L2, sig = lib.svdq_lowrank_init(W.cuda(), r, seed=seed)
    torch.cuda.synchronize()
    assert lib.svdq_read_device_error() == 0
    L1o, L2o, so = osv.lowrank_factors(W, r)
    e_gpu = _residual_energy(W, _f64(L1), _f64(L2))
    e_ora = _residual_energy(W, osv.to_f64(L1o), osv.to_f64(L2o))
    assert e_gpu <= e_ora * (1.0 + tol), f"residual energy {e_gpu / e_ora - 1:.3e} above the oracle's"
    s = sig.cpu().numpy()
    assert np.all(np.diff(s) <= 0), "sigma must be non-increasing"
    return L1, L2, s, so, e_gpu, e_ora


def test_lowrank_planted_qkv_full_size(lib):
    """Config 2's weight (9216 x 3072, planted rank 8 with 5x the Gaussian part's
    norm): the planted singular values to 1e-9, the residual within 1e-4."""
    spec = workloads.WORKLOADS[2].layers[0]
    _, W, _ = workloads.make_layer(spec)
    L1, L2, s, so, e_gpu, e_ora = _compare(lib, W, spec.r, tol=1e-4)
    assert np.max(np.abs(s[:8] - so[:8]) / so[:8]) < 1e-9
    assert np.max(np.abs(s - so[:spec.r]) / so[:spec.r]) < 1e-2


def test_lowrank_flat_spectrum(lib):
    """Config 1's Gaussian weight (1024 x 1024, r = 32): no gap in the spectrum."""
    spec = workloads.WORKLOADS[1].layers[0]
    _, W, _ = workloads.make_layer(spec)
    _compare(lib, W, spec.r, tol=1e-4)


def test_lowrank_rank128_sweep_weight(lib):
    """A K = N = 4096 sweep weight at the largest rank (160-column sketch)."""
    spec = workloads.WORKLOADS[5].layers[3]
    assert spec.r == 128
    _, W, _ = workloads.make_layer(spec)
    _compare(lib, W, spec.r, tol=5e-4)


@pytest.mark.parametrize("N,K,r", [(768, 1280, 16), (1280, 768, 64), (200, 1000, 16)])
def test_lowrank_rectangular_shapes(lib, N, K, r):
    """N != K either way, and N not a multiple of 128 (the SVD has no GEMM shape rules)."""
    _, (X, W, b) = workloads.small_layer(8, K, N, r, seed=11)
    L1, L2, *_ = _compare(lib, W, r, tol=1e-3)
    assert L1.shape == (K, r) and L2.shape == (r, N)


def test_lowrank_rows_of_l2_orthonormal(lib):
    spec = workloads.WORKLOADS[1].layers[0]
    _, W, _ = workloads.make_layer(spec)
    _, L2, _ = lib.svdq_lowrank_init(W.cuda(), spec.r)
    V = _f64(L2)
    gram = V @ V.T
    # bf16 rounding of unit vectors moves each inner product by at most about 2 * 2^-9
    assert np.max(np.abs(gram - np.eye(spec.r))) < 1e-2


def test_lowrank_exact_rank_weight(lib):
    """W = bf16(U diag(s) V^T) of rank 5 < r: everything beyond bf16 rounding is captured."""
    rng = np.random.default_rng(5)
    N, K, r = 512, 1024, 16
    U, _ = np.linalg.qr(rng.standard_normal((N, 5)))
    V, _ = np.linalg.qr(rng.standard_normal((K, 5)))
    W = torch.from_numpy(((U * np.array([9.0, 7.0, 5.0, 3.0, 1.0])) @ V.T).astype(np.float32)).to(torch.bfloat16)
    L1, L2, s, so, e_gpu, e_ora = _compare(lib, W, r, tol=1e-2)
    assert e_gpu <= 1e-4 * float(np.linalg.norm(osv.to_f64(W)) ** 2)
    assert np.max(np.abs(s[:5] - so[:5]) / so[:5]) < 1e-9


def test_lowrank_zero_weight(lib):
    W = torch.zeros((256, 512), dtype=torch.bfloat16)
    L1, L2, s = lib.svdq_lowrank_init(W.cuda(), 16)
    torch.cuda.synchronize()
    assert not _f64(L1).any() and not _f64(L2).any() and not s.cpu().numpy().any()


def test_lowrank_deterministic_for_a_seed(lib):
    spec = workloads.WORKLOADS[1].layers[0]
    _, W, _ = workloads.make_layer(spec)
    a = lib.svdq_lowrank_init(W.cuda(), 32, seed=9)
    b = lib.svdq_lowrank_init(W.cuda(), 32, seed=9)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_lowrank_factors_feed_pack_and_forward(lib):
    """Config 1 end to end with GPU-made factors: the packed weight is bit-exact
    and the forward output within the layer's bars of the oracle given the same
    factors."""
    spec = workloads.WORKLOADS[1].layers[0]
    X, W, b = workloads.make_layer(spec)
    L1, L2, _ = lib.svdq_lowrank_init(W.cuda(), spec.r)
    g_x = osv.act_global_scale(X)
    pw = lib.svdq_pack_weight(W.cuda(), L1, L2, float(g_x))
    Y = lib.svdq_linear_forward(X.cuda(), pw, b.cuda())
    torch.cuda.synchronize()
    L1h, L2h = _f64(L1), _f64(L2)
    ref_pw = osv.pack_weight(W, L1h, L2h)
    codes = layouts.unpack_codes(pw.codes.cpu().numpy(), spec.N, spec.K)
    assert np.array_equal(codes, ref_pw.codes)
    fwd = osv.forward(X, ref_pw, b, g_x)
    y = _f64(Y)
    assert osv.rel_fro(y, fwd.y_ref) <= 1e-3
    assert osv.max_abs_over_row_rms(y, fwd.y64) <= 2e-2
