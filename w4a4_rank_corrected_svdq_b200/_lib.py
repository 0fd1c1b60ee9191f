"""ctypes binding of libsvdq.so (the C ABI in include/svdq.h).

Argument marshalling only: every function here checks tensor dtypes, shapes,
devices and contiguity, passes raw device pointers and the current CUDA
stream to the C function of the same name, and raises SvdqError on a non-OK
status. No arithmetic of the layer happens in Python, and there is no
fallback: if the library cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsvdq.so")

STATUS = {
    0: "SVDQ_OK", 1: "SVDQ_ERR_INVALID_ARG", 2: "SVDQ_ERR_UNSUPPORTED_SHAPE", 3: "SVDQ_ERR_MISALIGNED",
    4: "SVDQ_ERR_UNSUPPORTED_DEVICE", 5: "SVDQ_ERR_CUDA", 6: "SVDQ_ERR_TIMEOUT", 7: "SVDQ_ERR_WORKSPACE",
}

# (name, restype, argtypes) for every symbol declared in include/svdq.h
_i, _i64, _f, _p, _sz = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
_psz, _pi = ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_int)
SIGNATURES = {
    "svdq_status_string": (ctypes.c_char_p, [_i]),
    "svdq_version": (_i, []),
    "svdq_scale_offset": (_i, [_i, _i, _i, _psz]),
    "svdq_device_supported": (_i, [_i, _i]),
    "svdq_weight_sizes": (_i, [_i, _i, _i, _psz, _psz, _psz, _psz]),
    "svdq_act_sizes": (_i, [_i, _i, _i, _psz, _psz, _psz]),
    "svdq_forward_workspace_size": (_i, [_i, _i, _i, _psz]),
    "svdq_pack_weight": (_i, [_i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p]),
    "svdq_smooth_factors": (_i, [_i, _i, _i, _p, _i64, _p, _f, _p, _p]),
    "svdq_act_global_scale": (_i, [_i, _i, _p, _i64, _p, _p, _p]),
    "svdq_quantize_act": (_i, [_i, _i, _i, _p, _i64, _p, _p, _p, _p, _p, _p, _p]),
    "svdq_w4a4_gemm": (_i, [_i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p, _i64, _p]),
    "svdq_linear_forward": (_i, [_i, _i, _i, _i, _p, _i64, _p, _p, _p, _p, _p, _p, _p, _p, _i64, _p, _sz, _p]),
    "svdq_read_device_error": (_i, [_pi, _i]),
    "svdq_selftest_bounded_wait": (_i, [_i, _p]),
    "svdq_linear_forward_noalloc": (_i, [_i, _i, _i, _i, _p, _i64, _p, _p, _p, _p, _p, _p, _p, _p, _i64, _p]),
    "svdq_linear_forward_qkv": (_i, [_i, _i, _i, _i, _p, _i64, _p, _p, _p, _p, _p, _p, _p, _i, _p, _p, _f, _p,
                                     _p, _i64, _p, _i64, _p, _sz, _p]),
    "svdq_dynamic_workspace_size": (_i, [_i, _i, _i, _i, _psz]),
    "svdq_linear_forward_dynamic": (_i, [_i, _i, _i, _i, _p, _i64, _p, _p, _p, _p, _p, _p, _p, _p, _i64, _p, _sz,
                                         _p]),
    "svdq_mlp_workspace_size": (_i, [_i, _i, _i, _i, _i, _psz]),
    "svdq_mlp_up_forward": (_i, [_i, _i, _i, _i, _p, _i64, _p, _p, _p, _p, _p, _p, _p, _i, _p, _p, _i, _p, _p, _p,
                                 _p, _i64, _p, _sz, _p]),
    "svdq_awq_sizes": (_i, [_i, _i, _psz, _psz, _psz]),
    "svdq_awq_pack": (_i, [_i, _i, _p, _p, _p, _p, _p, _p, _p]),
    "svdq_awq_gemv": (_i, [_i, _i, _i, _p, _i64, _p, _p, _p, _p, _p, _p, _i64, _p]),
    "svdq_lowrank_workspace_size": (_i, [_i, _i, _i, _psz]),
    "svdq_lowrank_init": (_i, [_i, _i, _i, _p, _p, _p, _p, _p, ctypes.c_ulonglong, _i, _p, _sz, _p]),
}


class SvdqError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsvdq.so (built in-tree by build.py); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libsvdq.so not built ({LIB_PATH}); run python -m w4a4_rank_corrected_svdq_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(name: str, status: int) -> None:
    if status != 0:
        raise SvdqError(name, status)


def _stream(t: torch.Tensor | None = None):
    dev = t.device if t is not None else torch.device("cuda")
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _ptr(t: torch.Tensor | None):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _dev(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _rows(t: torch.Tensor, name: str, cols: int) -> int:
    """Leading dimension (elements) of a 2-D tensor with unit column stride."""
    if t.dim() != 2 or t.shape[1] != cols or t.stride(1) != 1:
        raise ValueError(f"{name} must be 2-D [rows, {cols}] with unit column stride")
    return t.stride(0)


# ------------------------------------------------------------------ sizes
def svdq_scale_offset(K: int, row: int, kblock: int) -> int:
    out = ctypes.c_size_t()
    _check("svdq_scale_offset", lib().svdq_scale_offset(K, row, kblock, ctypes.byref(out)))
    return out.value


def svdq_weight_sizes(N: int, K: int, r: int):
    a, b, c, d = (ctypes.c_size_t() for _ in range(4))
    _check("svdq_weight_sizes", lib().svdq_weight_sizes(N, K, r, *(ctypes.byref(x) for x in (a, b, c, d))))
    return a.value, b.value, c.value, d.value


def svdq_act_sizes(M: int, K: int, r: int):
    a, b, c = (ctypes.c_size_t() for _ in range(3))
    _check("svdq_act_sizes", lib().svdq_act_sizes(M, K, r, *(ctypes.byref(x) for x in (a, b, c))))
    return a.value, b.value, c.value


def svdq_forward_workspace_size(M: int, K: int, r: int) -> int:
    out = ctypes.c_size_t()
    _check("svdq_forward_workspace_size", lib().svdq_forward_workspace_size(M, K, r, ctypes.byref(out)))
    return out.value


def svdq_lowrank_workspace_size(N: int, K: int, r: int) -> int:
    out = ctypes.c_size_t()
    _check("svdq_lowrank_workspace_size", lib().svdq_lowrank_workspace_size(N, K, r, ctypes.byref(out)))
    return out.value


def _smooth_vec(t: torch.Tensor | None, K: int, name: str):
    if t is not None:
        _dev(t, name, torch.float32, (K,))
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    return t


def svdq_lowrank_init(W: torch.Tensor, r: int, seed: int = 0, power_iters: int = 32,
                      workspace: torch.Tensor | None = None, smooth: torch.Tensor | None = None):
    """Rank-r factors of the 16-bit branch from a truncated SVD of W^T on the GPU
    (of diag(smooth) W^T with L1 carrying 1/smooth when smoothing):
    returns (L1 [K, r] bf16, L2 [r, N] bf16, sigma [r] float64)."""
    _dev(W, "W", torch.bfloat16)
    if not W.is_contiguous():
        raise ValueError("W must be contiguous")
    N, K = W.shape
    _smooth_vec(smooth, K, "smooth")
    need = svdq_lowrank_workspace_size(N, K, r)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    L1 = torch.empty((K, r), dtype=torch.bfloat16, device=W.device)
    L2 = torch.empty((r, N), dtype=torch.bfloat16, device=W.device)
    sigma = torch.empty(r, dtype=torch.float64, device=W.device)
    _check("svdq_lowrank_init", lib().svdq_lowrank_init(
        N, K, r, _ptr(W), _ptr(smooth), _ptr(L1), _ptr(L2), _ptr(sigma), seed, power_iters, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(W)))
    return L1, L2, sigma


# ------------------------------------------------------------------ packed weight
class PackedWeight:
    """Device buffers of one packed layer (allocated by torch, filled by svdq_pack_weight).

    gscale = [g_x, g_w, g_x*g_w, 0]; l2s = [2, N, r] bf16 hi / lo parts of L2^T / (g_x g_w);
    inv_smooth = fp32(1 / lambda) [K] of a smoothed layer, else None."""

    def __init__(self, N: int, K: int, r: int, device):
        cb, sb, lb1, lb2 = svdq_weight_sizes(N, K, r)
        self.N, self.K, self.r = N, K, r
        self.codes = torch.empty(cb, dtype=torch.uint8, device=device)
        self.scales = torch.empty(sb, dtype=torch.uint8, device=device)
        self.gscale = torch.empty(4, dtype=torch.float32, device=device)
        self.l1t = torch.empty((r, K), dtype=torch.bfloat16, device=device)
        self.l2s = torch.empty((2, N, r), dtype=torch.bfloat16, device=device)
        self.inv_smooth = None

    @property
    def g_x(self) -> torch.Tensor:
        return self.gscale[0:1]

    @property
    def g_w(self) -> torch.Tensor:
        return self.gscale[1:2]


def svdq_pack_weight(W: torch.Tensor, L1: torch.Tensor, L2: torch.Tensor, g_x, out: PackedWeight | None = None,
                     smooth: torch.Tensor | None = None):
    """Pack one layer. g_x: the calibrated activation scale, a CUDA float32 tensor of
    one element (e.g. from svdq_act_global_scale) or a Python float. smooth: the
    smoothing factors lambda [K] float32 (L1 then from svdq_lowrank_init with the
    same smooth), or None."""
    N, K = W.shape
    r = L1.shape[1]
    _dev(W, "W", torch.bfloat16)
    _dev(L1, "L1", torch.bfloat16, (K, r))
    _dev(L2, "L2", torch.bfloat16, (r, N))
    for t, n in ((W, "W"), (L1, "L1"), (L2, "L2")):
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    if not isinstance(g_x, torch.Tensor):
        g_x = torch.tensor([float(g_x)], dtype=torch.float32, device=W.device)
    _dev(g_x, "g_x", torch.float32)
    _smooth_vec(smooth, K, "smooth")
    pw = out if out is not None else PackedWeight(N, K, r, W.device)
    pw.inv_smooth = None if smooth is None else torch.empty(K, dtype=torch.float32, device=W.device)
    _check("svdq_pack_weight", lib().svdq_pack_weight(
        N, K, r, _ptr(W), _ptr(L1), _ptr(L2), _ptr(smooth), _ptr(g_x), _ptr(pw.codes), _ptr(pw.scales),
        _ptr(pw.gscale), _ptr(pw.l1t), _ptr(pw.l2s), _ptr(pw.inv_smooth), _stream(W)))
    return pw


def svdq_smooth_factors(X: torch.Tensor, W: torch.Tensor, alpha: float = 0.5,
                        out: torch.Tensor | None = None) -> torch.Tensor:
    """Smoothing factors lambda [K] (float32) from calibration activations X [M, K]
    and the weight W [N, K]."""
    _dev(X, "X", torch.bfloat16)
    _dev(W, "W", torch.bfloat16)
    M, K = X.shape
    ldx = _rows(X, "X", K)
    if W.dim() != 2 or W.shape[1] != K or not W.is_contiguous():
        raise ValueError("W must be contiguous [N, K]")
    lam = out if out is not None else torch.empty(K, dtype=torch.float32, device=X.device)
    _check("svdq_smooth_factors", lib().svdq_smooth_factors(M, W.shape[0], K, _ptr(X), ldx, _ptr(W), float(alpha),
                                                            _ptr(lam), _stream(X)))
    return lam


def svdq_act_global_scale(X: torch.Tensor, out: torch.Tensor | None = None,
                          inv_smooth: torch.Tensor | None = None) -> torch.Tensor:
    """fp32(amax|X^| / 2688) with X^ = X * inv_smooth (or X), on the device."""
    _dev(X, "X", torch.bfloat16)
    M, K = X.shape
    ldx = _rows(X, "X", K)
    _smooth_vec(inv_smooth, K, "inv_smooth")
    g = out if out is not None else torch.empty(1, dtype=torch.float32, device=X.device)
    _check("svdq_act_global_scale", lib().svdq_act_global_scale(M, K, _ptr(X), ldx, _ptr(inv_smooth), _ptr(g),
                                                                _stream(X)))
    return g


# ------------------------------------------------------------------ per call
class QuantAct:
    def __init__(self, M: int, K: int, r: int, device):
        cb, sb, xb = svdq_act_sizes(M, K, r)
        self.M, self.K, self.r = M, K, r
        self.codes = torch.empty(cb, dtype=torch.uint8, device=device)
        self.scales = torch.empty(sb, dtype=torch.uint8, device=device)
        self.xl1 = torch.empty((M, r), dtype=torch.bfloat16, device=device)


def svdq_quantize_act(X: torch.Tensor, pw: PackedWeight, out: QuantAct | None = None) -> QuantAct:
    """Quantise X with the layer's calibrated g_x (pw.gscale[0]) and project it onto L1."""
    _dev(X, "X", torch.bfloat16)
    M, K = X.shape
    ldx = _rows(X, "X", K)
    qa = out if out is not None else QuantAct(M, K, pw.r, X.device)
    _check("svdq_quantize_act", lib().svdq_quantize_act(
        M, K, pw.r, _ptr(X), ldx, _ptr(pw.gscale), _ptr(pw.l1t), _ptr(pw.inv_smooth), _ptr(qa.codes),
        _ptr(qa.scales), _ptr(qa.xl1), _stream(X)))
    return qa


def svdq_w4a4_gemm(qa: QuantAct, pw: PackedWeight, bias: torch.Tensor | None = None,
                   out: torch.Tensor | None = None) -> torch.Tensor:
    M, N, K, r = qa.M, pw.N, pw.K, pw.r
    if bias is not None:
        _dev(bias, "bias", torch.bfloat16, (N,))
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=qa.codes.device)
    _dev(Y, "Y", torch.bfloat16)
    ldy = _rows(Y, "Y", N)
    _check("svdq_w4a4_gemm", lib().svdq_w4a4_gemm(
        M, N, K, r, _ptr(qa.codes), _ptr(qa.scales), _ptr(qa.xl1), _ptr(pw.codes), _ptr(pw.scales),
        _ptr(pw.gscale), _ptr(pw.l2s), _ptr(bias), _ptr(Y), ldy, _stream(Y)))
    return Y


def svdq_linear_forward(X: torch.Tensor, pw: PackedWeight, bias: torch.Tensor | None = None,
                        out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    _dev(X, "X", torch.bfloat16)
    M, K = X.shape
    N, r = pw.N, pw.r
    ldx = _rows(X, "X", K)
    if bias is not None:
        _dev(bias, "bias", torch.bfloat16, (N,))
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _dev(Y, "Y", torch.bfloat16)
    ldy = _rows(Y, "Y", N)
    need = svdq_forward_workspace_size(M, K, r)
    ws = workspace if workspace is not None else torch.empty(max(need, 16), dtype=torch.uint8, device=X.device)
    _check("svdq_linear_forward", lib().svdq_linear_forward(
        M, N, K, r, _ptr(X), ldx, _ptr(pw.codes), _ptr(pw.scales), _ptr(pw.gscale), _ptr(pw.l1t),
        _ptr(pw.l2s), _ptr(pw.inv_smooth), _ptr(bias), _ptr(Y), ldy, _ptr(ws), ws.numel(), _stream(X)))
    return Y


def svdq_linear_forward_qkv(X: torch.Tensor, pw: PackedWeight, bias: torch.Tensor | None, heads: int,
                            norm_q_weight: torch.Tensor, norm_k_weight: torch.Tensor, eps: float,
                            rope_cos: torch.Tensor, rope_sin: torch.Tensor, out: torch.Tensor | None = None,
                            workspace: torch.Tensor | None = None) -> torch.Tensor:
    """The layer with the fused QKV post-processing (per-head RMSNorm of Q and K,
    rotary embedding; head_dim 128). rope_cos / rope_sin: float32 [M, >=64],
    cos / sin of each token's angle per pair (2j, 2j+1)."""
    _dev(X, "X", torch.bfloat16)
    M, K = X.shape
    ldx = _rows(X, "X", K)
    N = pw.N
    for t, n in ((norm_q_weight, "norm_q_weight"), (norm_k_weight, "norm_k_weight")):
        _dev(t, n, torch.bfloat16, (128,))
    for t, n in ((rope_cos, "rope_cos"), (rope_sin, "rope_sin")):
        _dev(t, n, torch.float32)
        if t.dim() != 2 or t.shape[0] != M or t.stride(1) != 1:
            raise ValueError(f"{n} must be [M, >=64] with unit column stride")
    if rope_cos.stride(0) != rope_sin.stride(0):
        raise ValueError("rope_cos and rope_sin must share a row stride")
    if bias is not None:
        _dev(bias, "bias", torch.bfloat16, (N,))
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    ldy = _rows(Y, "Y", N)
    if workspace is None:
        workspace = torch.empty(max(1, svdq_forward_workspace_size(M, K, pw.r)), dtype=torch.uint8, device=X.device)
    _check("svdq_linear_forward_qkv", lib().svdq_linear_forward_qkv(
        M, N, K, pw.r, _ptr(X), ldx, _ptr(pw.codes), _ptr(pw.scales), _ptr(pw.gscale), _ptr(pw.l1t), _ptr(pw.l2s),
        _ptr(pw.inv_smooth), _ptr(bias), heads, _ptr(norm_q_weight), _ptr(norm_k_weight), float(eps), _ptr(rope_cos), _ptr(rope_sin),
        rope_cos.stride(0), _ptr(Y), ldy, _ptr(workspace), workspace.numel(), _stream(X)))
    return Y


def svdq_dynamic_workspace_size(M: int, N: int, K: int, r: int) -> int:
    out = ctypes.c_size_t()
    _check("svdq_dynamic_workspace_size", lib().svdq_dynamic_workspace_size(M, N, K, r, ctypes.byref(out)))
    return out.value


def svdq_linear_forward_dynamic(X: torch.Tensor, pw: PackedWeight, bias: torch.Tensor | None = None,
                                out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """The layer with the activation scale computed from this call's X."""
    _dev(X, "X", torch.bfloat16)
    M, K = X.shape
    N, r = pw.N, pw.r
    ldx = _rows(X, "X", K)
    if bias is not None:
        _dev(bias, "bias", torch.bfloat16, (N,))
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _dev(Y, "Y", torch.bfloat16)
    ldy = _rows(Y, "Y", N)
    need = svdq_dynamic_workspace_size(M, N, K, r)
    ws = workspace if workspace is not None else torch.empty(need, dtype=torch.uint8, device=X.device)
    _check("svdq_linear_forward_dynamic", lib().svdq_linear_forward_dynamic(
        M, N, K, r, _ptr(X), ldx, _ptr(pw.codes), _ptr(pw.scales), _ptr(pw.gscale), _ptr(pw.l1t),
        _ptr(pw.l2s), _ptr(pw.inv_smooth), _ptr(bias), _ptr(Y), ldy, _ptr(ws), ws.numel(), _stream(X)))
    return Y


# ------------------------------------------------------------------ MLP pair
def svdq_mlp_workspace_size(M: int, N: int, K: int, r: int, r_down: int = 32) -> int:
    out = ctypes.c_size_t()
    _check("svdq_mlp_workspace_size", lib().svdq_mlp_workspace_size(M, N, K, r, r_down, ctypes.byref(out)))
    return out.value


def svdq_mlp_up_forward(X: torch.Tensor, pw: PackedWeight, bias: torch.Tensor | None, g_h: torch.Tensor,
                        l1t_down: torch.Tensor, approximate: bool = False, out: QuantAct | None = None,
                        h_out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> QuantAct:
    """The up projection with GELU, writing h quantised for the down projection:
    returns the down projection's QuantAct (codes, scales, xl1 of h). g_h: the
    down projection's activation scale (CUDA float32, one element); l1t_down:
    its L1 transposed, bf16 [r_down, N] (the down projection's packed
    PackedWeight.l1t); h_out: optional bf16 [M, N] copy of h."""
    _dev(X, "X", torch.bfloat16)
    M, K = X.shape
    N, r = pw.N, pw.r
    ldx = _rows(X, "X", K)
    _dev(g_h, "g_h", torch.float32)
    _dev(l1t_down, "l1t_down", torch.bfloat16)
    if l1t_down.dim() != 2 or l1t_down.shape[1] != N or not l1t_down.is_contiguous():
        raise ValueError("l1t_down must be a contiguous [r_down, N] tensor")
    rd = l1t_down.shape[0]
    if bias is not None:
        _dev(bias, "bias", torch.bfloat16, (N,))
    ldh = 0
    if h_out is not None:
        _dev(h_out, "h_out", torch.bfloat16)
        ldh = _rows(h_out, "h_out", N)
    qa = out if out is not None else QuantAct(M, N, rd, X.device)
    need = svdq_mlp_workspace_size(M, N, K, r, rd)
    ws = workspace if workspace is not None else torch.empty(need, dtype=torch.uint8, device=X.device)
    _check("svdq_mlp_up_forward", lib().svdq_mlp_up_forward(
        M, N, K, r, _ptr(X), ldx, _ptr(pw.codes), _ptr(pw.scales), _ptr(pw.gscale), _ptr(pw.l1t), _ptr(pw.l2s),
        _ptr(pw.inv_smooth), _ptr(bias), rd, _ptr(g_h), _ptr(l1t_down), int(approximate), _ptr(qa.codes),
        _ptr(qa.scales), _ptr(qa.xl1), _ptr(h_out), ldh, _ptr(ws), ws.numel(), _stream(X)))
    return qa


# ------------------------------------------------------------------ AWQ W4A16
def svdq_awq_sizes(N: int, K: int):
    a, b, c = (ctypes.c_size_t() for _ in range(3))
    _check("svdq_awq_sizes", lib().svdq_awq_sizes(N, K, *(ctypes.byref(x) for x in (a, b, c))))
    return a.value, b.value, c.value


class AwqWeight:
    """Device buffers of one INT4 group-64 weight (filled by svdq_awq_pack):
    codes u8 [N, K/2], scales bf16 [N, K/64], zeros u8 [N, K/64], inv_act [K] or None."""

    def __init__(self, N: int, K: int, device):
        cb, sb, zb = svdq_awq_sizes(N, K)
        self.N, self.K = N, K
        self.codes = torch.empty(cb, dtype=torch.uint8, device=device)
        self.scales = torch.empty((N, K // 64), dtype=torch.bfloat16, device=device)
        self.zeros = torch.empty((N, K // 64), dtype=torch.uint8, device=device)
        self.inv_act = None


def svdq_awq_pack(W: torch.Tensor, act_scale: torch.Tensor | None = None, out: AwqWeight | None = None) -> AwqWeight:
    """INT4 group-64 quantisation of W [N, K] bf16 (act_scale: activation-aware factors [K] or None)."""
    _dev(W, "W", torch.bfloat16)
    if W.dim() != 2 or not W.is_contiguous():
        raise ValueError("W must be a contiguous [N, K] tensor")
    N, K = W.shape
    _smooth_vec(act_scale, K, "act_scale")
    aw = out if out is not None else AwqWeight(N, K, W.device)
    aw.inv_act = None if act_scale is None else torch.empty(K, dtype=torch.float32, device=W.device)
    _check("svdq_awq_pack", lib().svdq_awq_pack(N, K, _ptr(W), _ptr(act_scale), _ptr(aw.codes), _ptr(aw.scales),
                                                _ptr(aw.zeros), _ptr(aw.inv_act), _stream(W)))
    return aw


def svdq_awq_gemv(X: torch.Tensor, aw: AwqWeight, bias: torch.Tensor | None = None,
                  out: torch.Tensor | None = None) -> torch.Tensor:
    """Y = X^ . W'^T + b for an AWQ W4A16 weight (X bf16 [M, K])."""
    _dev(X, "X", torch.bfloat16)
    M, K = X.shape
    N = aw.N
    ldx = _rows(X, "X", K)
    if bias is not None:
        _dev(bias, "bias", torch.bfloat16, (N,))
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _dev(Y, "Y", torch.bfloat16)
    ldy = _rows(Y, "Y", N)
    _check("svdq_awq_gemv", lib().svdq_awq_gemv(M, N, K, _ptr(X), ldx, _ptr(aw.codes), _ptr(aw.scales),
                                                _ptr(aw.zeros), _ptr(aw.inv_act), _ptr(bias), _ptr(Y), ldy,
                                                _stream(X)))
    return Y


def svdq_selftest_bounded_wait(limit_us: int = 1000) -> None:
    """Launch the bounded-wait self-test on the current stream (its wait gives up
    after limit_us and records SVDQ_ERR_TIMEOUT in the device error word)."""
    _check("svdq_selftest_bounded_wait", lib().svdq_selftest_bounded_wait(int(limit_us), _stream()))


def svdq_read_device_error(clear: bool = True) -> int:
    code = ctypes.c_int()
    _check("svdq_read_device_error", lib().svdq_read_device_error(ctypes.byref(code), int(clear)))
    return code.value
