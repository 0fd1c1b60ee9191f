"""GPU test of the bounded waits every kernel relies on (blog "Bringing
Nunchaku 4-bit Diffusion Inference to Diffusers", section "Hardware support":
a failure must surface as a clear error, not as wrong outputs or a hang).

svdq_selftest_bounded_wait launches one kernel whose only wait is on an
mbarrier that nothing arrives on, with a short limit. The wait must give up,
record SVDQ_ERR_TIMEOUT in the device error word and return normally; the
CUDA context must stay usable, so a forward of the layer right after it
still matches the oracle and leaves no error behind. No kernel here traps,
faults or spins without bound."""
import numpy as np
import pytest
import torch

import workloads
from oracle import svdq as osv
from tests import layouts

pytestmark = pytest.mark.gpu

SVDQ_ERR_TIMEOUT = 6


@pytest.fixture(scope="module")
def svdq():
    from w4a4_rank_corrected_svdq_b200 import build
    build.build()
    import w4a4_rank_corrected_svdq_b200 as m
    return m


def _small_forward_matches_oracle(svdq):
    M, K, N, r = 200, 512, 256, 32
    _, (X, W, b) = workloads.small_layer(M, K, N, r, seed=17)
    L1, L2, _ = osv.lowrank_factors(W, r)
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).cuda()  # noqa: E731
    g_x = osv.act_global_scale(X)
    pw = svdq.svdq_pack_weight(W.cuda(), to_dev(L1), to_dev(L2), float(g_x))
    qa = svdq.svdq_quantize_act(X.cuda(), pw)
    Y = svdq.svdq_w4a4_gemm(qa, pw, b.cuda())
    torch.cuda.synchronize()
    ref = osv.forward(X, osv.pack_weight(W, L1, L2), b, g_x)
    assert np.array_equal(layouts.unpack_codes(qa.codes.cpu().numpy(), M, K), ref.codes)
    assert np.array_equal(layouts.untile_scales(qa.scales.cpu().numpy(), M, K), ref.scales)
    y = Y.double().cpu().numpy()
    assert osv.rel_fro(y, ref.y_ref) <= 1e-3
    assert osv.max_abs_over_row_rms(y, ref.y64) <= 2e-2


@pytest.mark.parametrize("limit_us", [1000, 20000])
def test_wait_that_runs_out_reports_timeout_and_context_survives(svdq, limit_us):
    assert svdq.svdq_read_device_error(clear=True) in (0, SVDQ_ERR_TIMEOUT)
    assert svdq.svdq_read_device_error(clear=True) == 0
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    svdq.svdq_selftest_bounded_wait(limit_us)
    t1.record()
    torch.cuda.synchronize()
    # the kernel waited at least its limit, then gave up well before the
    # library-wide 2 s bound
    ms = t0.elapsed_time(t1)
    assert limit_us / 1e3 <= ms < limit_us / 1e3 + 500.0, ms
    assert svdq.svdq_read_device_error(clear=True) == SVDQ_ERR_TIMEOUT
    assert svdq.svdq_read_device_error(clear=True) == 0
    _small_forward_matches_oracle(svdq)
    assert svdq.svdq_read_device_error(clear=True) == 0


def test_selftest_rejects_bad_limits(svdq):
    L = svdq.lib()
    for bad in (0, -5, 1000001):
        assert L.svdq_selftest_bounded_wait(bad, None) == 1   # SVDQ_ERR_INVALID_ARG, nothing launched
    torch.cuda.synchronize()
    assert svdq.svdq_read_device_error(clear=True) == 0
