"""Host-side checks of the C ABI: the library loads without a GPU, exports every
symbol include/svdq.h declares, validates arguments before touching a device,
and reports a missing/unsupported device as SVDQ_ERR_UNSUPPORTED_DEVICE."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from tests import layouts
from w4a4_rank_corrected_svdq_b200 import _lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "svdq.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from w4a4_rank_corrected_svdq_b200 import build
    build.build()
    return _lib.lib()


def test_every_declared_symbol_is_exported_and_bound(L):
    names = _declared_functions()
    assert "svdq_linear_forward" in names and "svdq_pack_weight" in names and "svdq_quantize_act" in names
    for n in names:
        assert hasattr(L, n), n
        assert n in _lib.SIGNATURES, n


def test_status_strings_and_version(L):
    assert L.svdq_status_string(0) == b"SVDQ_OK"
    assert L.svdq_status_string(6) == b"SVDQ_ERR_TIMEOUT"
    assert L.svdq_status_string(99) == b"SVDQ_ERR_UNKNOWN"
    assert L.svdq_version() >= 100


def test_scale_offset_matches_documented_layout(L):
    K = 512
    offs = layouts.scale_offsets(300, K)
    for row in (0, 1, 31, 32, 100, 127, 128, 255, 299):
        for kb in (0, 1, 3, 4, 17, K // 16 - 1):
            assert _lib.svdq_scale_offset(K, row, kb) == offs[row, kb]
    # a 128-row block of a K-column tensor is a permutation of its K/16*128 bytes
    blk = layouts.scale_offsets(128, K).ravel()
    assert np.array_equal(np.sort(blk), np.arange(128 * K // 16))


def test_scale_offset_errors(L):
    out = ctypes.c_size_t()
    assert L.svdq_scale_offset(100, 0, 0, ctypes.byref(out)) == 2
    assert L.svdq_scale_offset(256, -1, 0, ctypes.byref(out)) == 1
    assert L.svdq_scale_offset(256, 0, 16, ctypes.byref(out)) == 1
    assert L.svdq_scale_offset(256, 0, 0, None) == 1


def test_sizes(L):
    assert _lib.svdq_weight_sizes(256, 512, 32) == (256 * 256, 256 * 32, 32 * 512 * 2, 2 * 256 * 32 * 2)
    assert _lib.svdq_act_sizes(129, 512, 16) == (129 * 256, 256 * 32, 129 * 16 * 2)
    ws = _lib.svdq_forward_workspace_size(129, 512, 16)
    assert ws >= sum(_lib.svdq_act_sizes(129, 512, 16))
    with pytest.raises(_lib.SvdqError):
        _lib.svdq_weight_sizes(100, 512, 32)      # N % 128
    with pytest.raises(_lib.SvdqError):
        _lib.svdq_weight_sizes(128, 500, 32)      # K % 256
    with pytest.raises(_lib.SvdqError):
        _lib.svdq_weight_sizes(128, 512, 24)      # rank


def test_validation_happens_before_device_checks(L):
    p = ctypes.c_void_p(0x10000)          # never dereferenced: validation fails first
    odd = ctypes.c_void_p(0x10008)
    # bad K
    assert L.svdq_quantize_act(4, 100, 32, p, 100, p, p, None, p, p, p, None) == 2
    # null pointer
    assert L.svdq_quantize_act(4, 256, 32, None, 256, p, p, None, p, p, p, None) == 1
    # misaligned pointer
    assert L.svdq_quantize_act(4, 256, 32, odd, 256, p, p, None, p, p, p, None) == 3
    assert L.svdq_quantize_act(4, 256, 32, p, 256, p, p, ctypes.c_void_p(0x10004), p, p, p, None) == 3  # inv_smooth
    # bad leading dimension
    assert L.svdq_w4a4_gemm(4, 128, 256, 32, p, p, p, p, p, p, p, None, p, 100, None) == 2
    # workspace too small
    assert L.svdq_linear_forward(4, 128, 256, 32, p, 256, p, p, p, p, p, None, None, p, 128, p, 16, None) == 7
    # M == 0 is a valid no-op
    assert L.svdq_w4a4_gemm(0, 128, 256, 32, None, None, None, None, None, None, None, None, None, 128,
                            None) == 0


def test_lowrank_sizes_and_validation(L):
    p = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    ws = _lib.svdq_lowrank_workspace_size(9216, 3072, 32)
    assert ws >= 8 * (2 * 9216 + 2 * 3072) * 64        # two N x p and two K x p float64 buffers, p = r + 32
    assert _lib.svdq_lowrank_workspace_size(200, 1000, 16) > 0   # no GEMM shape rules
    out = ctypes.c_size_t()
    assert L.svdq_lowrank_workspace_size(128, 256, 24, ctypes.byref(out)) == 1    # rank
    assert L.svdq_lowrank_workspace_size(16, 256, 32, ctypes.byref(out)) == 2     # r > min(N, K)
    big = ctypes.c_size_t(1 << 40)
    # rank, then shape, then alignment, then workspace size, all before any device check
    assert L.svdq_lowrank_init(128, 256, 24, p, None, p, p, None, 0, 4, p, big, None) == 1
    assert L.svdq_lowrank_init(128, 256, 32, p, None, p, p, None, 0, 65, p, big, None) == 1   # power_iters
    assert L.svdq_lowrank_init(128, 252, 32, p, None, p, p, None, 0, 4, p, big, None) == 2    # K % 8
    assert L.svdq_lowrank_init(128, 256, 32, odd, None, p, p, None, 0, 4, p, big, None) == 3
    assert L.svdq_lowrank_init(128, 256, 32, p, None, p, p, ctypes.c_void_p(0x10004), 0, 4, p, big, None) == 3
    assert L.svdq_lowrank_init(128, 256, 32, p, odd, p, p, None, 0, 4, p, big, None) == 3     # smooth
    assert L.svdq_lowrank_init(128, 256, 32, p, None, p, p, None, 0, 4, p, ctypes.c_size_t(16), None) == 7


def test_smoothing_validation(L):
    p = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    f = ctypes.c_float
    # smooth and inv_smooth come together
    assert L.svdq_pack_weight(128, 256, 32, p, p, p, p, p, p, p, p, p, p, None, None) == 1
    assert L.svdq_pack_weight(128, 256, 32, p, p, p, None, p, p, p, p, p, p, p, None) == 1
    assert L.svdq_pack_weight(128, 256, 32, p, p, p, odd, p, p, p, p, p, p, p, None) == 3
    # calibration: alpha in [0, 1], K % 8, alignment
    assert L.svdq_smooth_factors(4, 128, 256, p, 256, p, f(1.5), p, None) == 1
    assert L.svdq_smooth_factors(4, 128, 256, p, 256, p, f(-0.1), p, None) == 1
    assert L.svdq_smooth_factors(4, 128, 252, p, 256, p, f(0.5), p, None) == 2
    assert L.svdq_smooth_factors(4, 128, 256, odd, 256, p, f(0.5), p, None) == 3
    assert L.svdq_act_global_scale(4, 256, p, 256, odd, p, None) == 3


def test_dynamic_forward_sizes_and_validation(L):
    p = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    base = _lib.svdq_forward_workspace_size(300, 512, 32)
    assert _lib.svdq_dynamic_workspace_size(300, 384, 512, 32) == base + 8192 + 384 * 32 * 4
    with pytest.raises(_lib.SvdqError):
        _lib.svdq_dynamic_workspace_size(300, 100, 512, 32)     # N % 128
    need = _lib.svdq_dynamic_workspace_size(4, 128, 256, 32)
    args = lambda ws, wsb, x: (4, 128, 256, 32, x, 256, p, p, p, p, p, None, None, p, 128, ws, ctypes.c_size_t(wsb),
                               None)
    assert L.svdq_linear_forward_dynamic(*args(p, need - 1, p)) == 7     # workspace too small
    assert L.svdq_linear_forward_dynamic(*args(odd, need, p)) == 3       # misaligned workspace
    assert L.svdq_linear_forward_dynamic(*args(p, need, None)) == 1      # no X
    assert L.svdq_linear_forward_dynamic(0, 128, 256, 32, None, 256, None, None, None, None, None, None, None, None,
                                         128, None, 0, None) == 0          # M == 0: no-op


def test_awq_sizes_and_validation(L):
    p = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    assert _lib.svdq_awq_sizes(100, 576) == (100 * 288, 100 * 9 * 2, 100 * 9)
    with pytest.raises(_lib.SvdqError):
        _lib.svdq_awq_sizes(100, 500)                                  # K % 64
    assert L.svdq_awq_pack(100, 576, p, p, p, p, p, None, None) == 1    # act_scale without inv_act
    assert L.svdq_awq_pack(100, 576, odd, None, p, p, p, None, None) == 3
    assert L.svdq_awq_gemv(2, 100, 576, p, 500, p, p, p, None, None, p, 100, None) == 2    # ldx < K
    assert L.svdq_awq_gemv(2, 100, 576, odd, 576, p, p, p, None, None, p, 100, None) == 3
    assert L.svdq_awq_gemv(2, 100, 32768, p, 32768, p, p, p, None, None, p, 100, None) == 2  # K * 4 > 96 KB
    assert L.svdq_awq_gemv(0, 100, 576, None, 576, None, None, None, None, None, None, 100, None) == 0


def test_mlp_up_sizes_and_validation(L):
    p = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    base = _lib.svdq_forward_workspace_size(300, 512, 32)
    # one 256-row fp32 partial slot of r_down = 32 per 256 x 256 tile: 2 x 4 tiles
    assert _lib.svdq_mlp_workspace_size(300, 1024, 512, 32, 32) == base + 2 * 4 * 256 * 32 * 4
    with pytest.raises(_lib.SvdqError):
        _lib.svdq_mlp_workspace_size(300, 1024, 512, 32, 16)          # r_down must be 32
    with pytest.raises(_lib.SvdqError):
        _lib.svdq_mlp_workspace_size(300, 896, 512, 32, 32)           # N % 256
    need = _lib.svdq_mlp_workspace_size(4, 256, 256, 32, 32)
    args = lambda ws, wsb, l1d: (4, 256, 256, 32, p, 256, p, p, p, p, p, None, None, 32, p, l1d, 0, p, p, p, None,
                                 0, ws, ctypes.c_size_t(wsb), None)
    assert L.svdq_mlp_up_forward(*args(p, need - 1, p)) == 7          # workspace too small
    assert L.svdq_mlp_up_forward(*args(p, need, None)) == 1           # no L1 of the down projection
    assert L.svdq_mlp_up_forward(*args(p, need, odd)) == 3            # misaligned L1
    bad_bias = (4, 256, 256, 32, p, 256, p, p, p, p, p, None, odd, 32, p, p, 0, p, p, p, None, 0, p,
                ctypes.c_size_t(need), None)
    assert L.svdq_mlp_up_forward(*bad_bias) == 3                       # misaligned bias


def test_qkv_forward_validation(L):
    p = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    f = ctypes.c_float
    ws = ctypes.c_size_t(1 << 40)
    args = lambda N, heads, eps, cs, ld: (4, N, 256, 32, p, 256, p, p, p, p, p, None, None, heads, p, p, f(eps), cs,
                                          p, ld, p, N, p, ws, None)
    assert L.svdq_linear_forward_qkv(*args(768, 2, 1e-6, p, 128)) in (0, 4)     # valid (no GPU here: 4)
    assert L.svdq_linear_forward_qkv(*args(768, 1, 1e-6, p, 128)) == 2          # N != 3 * heads * 128
    assert L.svdq_linear_forward_qkv(*args(768, 2, -1.0, p, 128)) == 1          # eps < 0
    assert L.svdq_linear_forward_qkv(*args(768, 2, 1e-6, p, 64)) in (0, 4)      # 64 angles per token suffice
    assert L.svdq_linear_forward_qkv(*args(768, 2, 1e-6, p, 60)) == 2           # ld_rope < 64
    assert L.svdq_linear_forward_qkv(*args(768, 2, 1e-6, p, 66)) == 2           # ld_rope % 4 != 0
    assert L.svdq_linear_forward_qkv(*args(768, 2, 1e-6, odd, 128)) == 3        # misaligned rope table
    assert L.svdq_linear_forward_qkv(*args(768, 0, 1e-6, p, 128)) == 1          # heads


def test_device_rule_on_simulated_capabilities(L):
    """The capability rule the entry points apply, fed simulated devices: only
    compute capability 10.0 (B200) is supported; Hopper, Ada, Ampere, other
    Blackwell parts and later families get SVDQ_ERR_UNSUPPORTED_DEVICE."""
    assert L.svdq_device_supported(10, 0) == 0
    for major, minor in ((9, 0), (8, 9), (8, 0), (7, 5), (10, 3), (12, 0), (11, 0), (0, 0)):
        assert L.svdq_device_supported(major, minor) == 4, (major, minor)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_no_gpu_is_unsupported_device(L):
    p = ctypes.c_void_p(0x10000)
    assert L.svdq_quantize_act(4, 256, 32, p, 256, p, p, None, p, p, p, None) == 4
    assert L.svdq_pack_weight(128, 256, 32, p, p, p, None, p, p, p, p, p, p, None, None) == 4
    assert L.svdq_lowrank_init(128, 256, 32, p, None, p, p, None, 0, 4, p, ctypes.c_size_t(1 << 40), None) == 4
    assert L.svdq_smooth_factors(4, 128, 256, p, 256, p, ctypes.c_float(0.5), p, None) == 4
    code = ctypes.c_int()
    assert L.svdq_read_device_error(ctypes.byref(code), 0) == 4


def test_ulp_helper():
    a = np.array([1.0, 1.0, -1.0, 0.0])
    b = np.array([1.0 + 2 ** -7, 1.0, -1.0 - 2 ** -7, -0.0])
    assert layouts.bf16_ulp_distance(a, b).tolist() == [1, 0, 1, 0]
