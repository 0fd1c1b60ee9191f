// smooth.cuh — smoothing: activation outliers moved into the weights.
//
// Blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers", section
// "Background: SVDQuant and Nunchaku": outliers are first moved from the
// activations into the weights. A per-input-channel factor lambda_k does it:
// the 4-bit branch quantises x^ = x * fp32(1 / lambda_k) and a weight whose
// residual carries lambda_k (pack_weight.cuh), so x^ . W^T is unchanged.
//
// Calibration (this file) takes SmoothQuant's rule (Xiao et al. 2023), the
// one the blog's method builds on but does not spell out:
//   lambda_k = amax_m|X[m,k]|^alpha / amax_n|W[n,k]|^(1 - alpha)
// in float64, clamped to [2^-32, 2^32], rounded once to fp32; lambda_k = 1
// where either amax is 0. alpha = 0.5 uses correctly rounded square roots and
// one correctly rounded division, so it is exactly reproducible.
#pragma once

#include "nvfp4.cuh"

namespace svdq {

constexpr int kSmoothCols = 64;      // columns per block (8 lanes x 8 bf16)
constexpr int kSmoothThreads = 256;  // 8 column lanes x 32 row lanes

// Column amaxima of the bf16 matrices X (M x K, pitch ldx) and W (N x K,
// pitch K) for the block's 64 columns, then lambda for each of them.
__global__ void __launch_bounds__(kSmoothThreads) smooth_factors_kernel(const __nv_bfloat16* __restrict__ X,
                                                                        int64_t ldx, int M,
                                                                        const __nv_bfloat16* __restrict__ W, int N,
                                                                        int K, float alpha, float* __restrict__ lam) {
  __shared__ float sx[32][kSmoothCols + 1], sw[32][kSmoothCols + 1];
  const int cl = threadIdx.x & 7;   // 8-column chunk
  const int rl = threadIdx.x >> 3;  // row lane
  const int col = blockIdx.x * kSmoothCols + 8 * cl;
  float ax[8], aw[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) ax[i] = aw[i] = 0.0f;
  if (col < K) {
#pragma unroll 4
    for (int m = rl; m < M; m += 32) {
      float f[8];
      bf16x8_to_f32(ldg_nc_v4(X + static_cast<int64_t>(m) * ldx + col), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) ax[i] = fmaxf(ax[i], fabsf(f[i]));
    }
#pragma unroll 4
    for (int n = rl; n < N; n += 32) {
      float f[8];
      bf16x8_to_f32(ldg_nc_v4(W + static_cast<int64_t>(n) * K + col), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) aw[i] = fmaxf(aw[i], fabsf(f[i]));
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    sx[rl][8 * cl + i] = ax[i];
    sw[rl][8 * cl + i] = aw[i];
  }
  __syncthreads();
  const int c = threadIdx.x;
  const int k = blockIdx.x * kSmoothCols + c;
  if (c < kSmoothCols && k < K) {
    float mx = 0.0f, mw = 0.0f;
    for (int j = 0; j < 32; ++j) {
      mx = fmaxf(mx, sx[j][c]);
      mw = fmaxf(mw, sw[j][c]);
    }
    double l = 1.0;
    if (mx > 0.0f && mw > 0.0f) {
      const double dx = mx, dw = mw;
      if (alpha == 0.5f)
        l = __ddiv_rn(__dsqrt_rn(dx), __dsqrt_rn(dw));
      else
        l = pow(dx, static_cast<double>(alpha)) / pow(dw, 1.0 - static_cast<double>(alpha));
      l = fmin(fmax(l, 0x1.0p-32), 0x1.0p32);
    }
    lam[k] = __double2float_rn(l);
  }
}

// inv[k] = fp32(1 / lambda_k) (correctly rounded). A lambda that is not a
// positive finite number records SVDQ_ERR_INVALID_ARG and gives inv = 0.
__global__ void inv_smooth_kernel(const float* __restrict__ lam, float* __restrict__ inv, int K) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const float l = lam[k];
  if (!(l > 0.0f && l < INFINITY)) {
    record_error(1);
    inv[k] = 0.0f;
    return;
  }
  inv[k] = __frcp_rn(l);
}

}  // namespace svdq
