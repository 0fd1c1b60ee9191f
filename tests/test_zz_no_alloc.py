"""GPU test of svdq_linear_forward_noalloc, the forward for callers that cannot
provide a workspace (runtime plugin interfaces that pass only a layer's inputs
and outputs; code that must not call an allocator once its memory budget is
fixed). It is called through the C ABI and compared with svdq_linear_forward,
which takes a caller-provided workspace, on two calls in a row after a larger
call has dirtied the shared scratch; the outputs must be bit-identical. This
file is collected last so that a run stopping at its first failure has already run
every other test."""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from oracle import svdq as osv

pytestmark = pytest.mark.gpu

REL_FRO = 1e-3
MAX_ROWRMS = 2e-2


@pytest.fixture(scope="module")
def lib():
    from w4a4_rank_corrected_svdq_b200 import _lib, build
    build.build()
    return _lib


def _p(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _noalloc(L, X, pw, bias, Y):
    M, K = X.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.svdq_linear_forward_noalloc(M, pw.N, K, pw.r, _p(X), X.stride(0), _p(pw.codes), _p(pw.scales),
                                         _p(pw.gscale), _p(pw.l1t), _p(pw.l2s), _p(pw.inv_smooth), _p(bias), _p(Y),
                                         Y.stride(0), stream)


def _layer(lib, M, K, N, r, seed):
    _, (X, W, b) = workloads.small_layer(M, K, N, r, seed=seed)
    L1, L2, _ = osv.lowrank_factors(W, r)
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).cuda()  # noqa: E731
    g_x = osv.act_global_scale(X)
    pw = lib.svdq_pack_weight(W.cuda(), to_dev(L1), to_dev(L2), float(g_x))
    return X, W, b, L1, L2, g_x, pw


@pytest.mark.parametrize("M,K,N,r", [(256, 1024, 1024, 32), (333, 768, 384, 64)])
def test_noalloc_forward_matches_workspace_forward(lib, M, K, N, r):
    L = lib.lib()
    # Leave non-zero bytes in the shared scratch first (a larger call with
    # another K and rank), so nothing below can rely on it starting at zero.
    Xp, _, bp, _, _, _, pwp = _layer(lib, 640, 2048, 256, 128, seed=5)
    Yp = torch.empty((640, 256), dtype=torch.bfloat16, device="cuda")
    assert _noalloc(L, Xp.cuda(), pwp, bp.cuda(), Yp) == 0
    torch.cuda.synchronize()

    X, W, b, L1, L2, g_x, pw = _layer(lib, M, K, N, r, seed=21)
    Xd, bd = X.cuda(), b.cuda()
    # the workspace forward, its workspace filled with 0xFF bytes (NaN patterns)
    ws = torch.full((lib.svdq_forward_workspace_size(M, K, r),), 0xFF, dtype=torch.uint8, device="cuda")
    ref = lib.svdq_linear_forward(Xd, pw, bd, workspace=ws)
    outs = []
    for _ in range(2):                       # two calls in a row share the scratch
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(L, Xd, pw, bd, Y) == 0
        torch.cuda.synchronize()
        outs.append(Y)
    assert lib.svdq_read_device_error() == 0
    # the same kernels on the same inputs: bit-identical to the workspace forward
    for y in outs:
        assert torch.equal(y, ref)
    # and within the layer's bars of the CPU oracle
    o = osv.forward(X, osv.pack_weight(W, L1, L2), b, g_x)
    y = outs[-1].double().cpu().numpy()
    assert osv.rel_fro(y, o.y_ref) <= REL_FRO
    assert osv.max_abs_over_row_rms(y, o.y64) <= MAX_ROWRMS


def test_noalloc_rejects_shapes_beyond_the_scratch_limit(lib):
    L = lib.lib()
    p = ctypes.c_void_p(0x10000)             # never dereferenced: the size check fails first
    M, K, N, r = 18432, 3072, 128, 32        # workspace about 33 MB > 16 MiB
    assert lib.svdq_forward_workspace_size(M, K, r) > (16 << 20)
    assert L.svdq_linear_forward_noalloc(M, N, K, r, p, K, p, p, p, p, p, None, None, p, N, None) == 7
