"""B200 (sm_100a) SVDQuant W4A4 NVFP4 linear layer.

Y = (X . L1) . L2 + Q4(X) . Q4(R)^T + b with a rank-r bf16 low-rank branch and
an NVFP4 residual R = W - (L1 . L2)^T (blog "Bringing Nunchaku 4-bit Diffusion
Inference to Diffusers"). The work runs in hand-written CUDA kernels behind
the C ABI of include/svdq.h; this package is its ctypes binding.

Typical use (device tensors):
    lam = svdq_smooth_factors(X_cal, W)                  # optional smoothing
    L1, L2, _ = svdq_lowrank_init(W, 32, smooth=lam)     # truncated SVD
    pw = svdq_pack_weight(W, L1, L2, 1.0, smooth=lam)    # (for inv_smooth)
    g_x = svdq_act_global_scale(X_cal, inv_smooth=pw.inv_smooth)
    pw = svdq_pack_weight(W, L1, L2, g_x, smooth=lam)
    Y = svdq_linear_forward(X, pw, bias)                 # or _dynamic, _qkv
The AWQ W4A16 family: svdq_awq_pack, svdq_awq_gemv.
"""
from ._lib import (  # noqa: F401
    AwqWeight,
    PackedWeight,
    QuantAct,
    SvdqError,
    lib,
    svdq_act_global_scale,
    svdq_act_sizes,
    svdq_awq_gemv,
    svdq_awq_pack,
    svdq_awq_sizes,
    svdq_dynamic_workspace_size,
    svdq_forward_workspace_size,
    svdq_linear_forward,
    svdq_linear_forward_dynamic,
    svdq_linear_forward_qkv,
    svdq_lowrank_init,
    svdq_mlp_up_forward,
    svdq_mlp_workspace_size,
    svdq_lowrank_workspace_size,
    svdq_pack_weight,
    svdq_quantize_act,
    svdq_read_device_error,
    svdq_scale_offset,
    svdq_selftest_bounded_wait,
    svdq_smooth_factors,
    svdq_w4a4_gemm,
    svdq_weight_sizes,
)
