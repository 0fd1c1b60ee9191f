// pack_weight.cuh — load-time packing of one layer: residual, its NVFP4 codes
// and scales, and the transposed low-rank factors the per-call kernels read.
//
// Blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers", section
// "Background: SVDQuant and Nunchaku": the hardest part of each weight matrix
// is kept in a small 16-bit low-rank branch and the remaining residual is
// quantised to 4 bits. Here
//   R[n,k] = W[n,k] - sum_j L1[k,j] L2[j,n]
// is formed in float64 with j ascending (each bf16 x bf16 product is exact in
// float64, so a fused multiply-add gives the same value) and rounded once to
// float32; g_w = fp32(amax|R| / 2688) (1 if R == 0); R is then quantised with
// the same NVFP4 rule as the activations, blocks of 16 along K. With smoothing
// (outliers moved into the weights, same section) the float64 difference is
// multiplied by lambda_k before the fp32 rounding: the residual of
// W diag(lambda) against factors whose L1 carries 1/lambda.
//
// Work split: a warp owns 32 consecutive K-columns (two 16-element blocks) and
// walks `rows_per_warp` rows n; each lane keeps its column's L1 row in
// registers and reads the row of L2^T (r contiguous bf16) as broadcast loads.
#pragma once

#include "nvfp4.cuh"

namespace svdq {

constexpr int kPackThreads = 256;
constexpr int kPackRowsPerWarp = 32;

// l1t[j][k] = L1[k][j]   (L1: K x r  ->  r x K)
__global__ void transpose_bf16_kernel(const __nv_bfloat16* __restrict__ in, __nv_bfloat16* __restrict__ out,
                                      int rows, int cols) {
  __shared__ __nv_bfloat16 tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8 threads
  for (int i = ty; i < 32; i += 8) {
    const int r = r0 + i, c = c0 + tx;
    if (r < rows && c < cols) tile[i][tx] = in[static_cast<int64_t>(r) * cols + c];
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int c = c0 + i, r = r0 + tx;
    if (c < cols && r < rows) out[static_cast<int64_t>(c) * rows + r] = tile[tx][i];
  }
}

template <int R>
__device__ __forceinline__ float residual_at(const __nv_bfloat16* __restrict__ W, const float (&l1row)[R],
                                             const __nv_bfloat16* __restrict__ l2t, int N, int K, int n, int k,
                                             double lam) {
  double s = 0.0;
  const __nv_bfloat16* l2 = l2t + static_cast<int64_t>(n) * R;
#pragma unroll
  for (int j8 = 0; j8 < R; j8 += 8) {
    const uint4 v = ldg_v4(l2 + j8);
    float f[8];
    bf16x8_to_f32(v, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) s = __dadd_rn(s, __dmul_rn(static_cast<double>(l1row[j8 + i]), static_cast<double>(f[i])));
  }
  const double w = static_cast<double>(__bfloat162float(W[static_cast<int64_t>(n) * K + k]));
  return __double2float_rn(__dmul_rn(__dsub_rn(w, s), lam));
}

template <int R>
__device__ __forceinline__ void load_l1_row(const __nv_bfloat16* __restrict__ L1, int k, float (&l1row)[R]) {
  const __nv_bfloat16* p = L1 + static_cast<int64_t>(k) * R;
#pragma unroll
  for (int j8 = 0; j8 < R; j8 += 8) {
    float f[8];
    bf16x8_to_f32(ldg_v4(p + j8), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) l1row[j8 + i] = f[i];
  }
}

// Pass 1: amax |R| over the whole matrix -> *amax_bits (as fp32 bits; |R| >= 0
// so unsigned comparison of the bit patterns orders the values).
template <int R>
__global__ void __launch_bounds__(kPackThreads) residual_amax_kernel(const __nv_bfloat16* __restrict__ W,
                                                                      const __nv_bfloat16* __restrict__ L1,
                                                                      const __nv_bfloat16* __restrict__ l2t,
                                                                      const float* __restrict__ smooth, int N,
                                                                      int K, unsigned* amax_bits) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (kPackThreads / 32) + (threadIdx.x >> 5);
  const int slabs = K / 32;
  const int slab = gw % slabs;
  const int n_begin = (gw / slabs) * kPackRowsPerWarp;
  if (n_begin >= N) return;
  const int k = slab * 32 + lane;
  float l1row[R];
  load_l1_row<R>(L1, k, l1row);
  const double lam = smooth != nullptr ? static_cast<double>(smooth[k]) : 1.0;
  float am = 0.0f;
  const int n_end = min(N, n_begin + kPackRowsPerWarp);
  for (int n = n_begin; n < n_end; ++n) am = fmaxf(am, fabsf(residual_at<R>(W, l1row, l2t, N, K, n, k, lam)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  if (lane == 0) atomicMax(amax_bits, __float_as_uint(am));
}

// amax bits -> g = fp32(amax / 2688), or 1 for an all-zero tensor (in place).
__global__ void finalize_global_scale_kernel(float* g) {
  const float am = __uint_as_float(*reinterpret_cast<unsigned*>(g));
  *g = (am == 0.0f) ? 1.0f : __fdiv_rn(am, kGlobalDivisor);
}

// gscale = {g_x, g_w, alpha = fp32(g_x g_w), 0}; gscale[1] holds the amax bits of R on entry.
__global__ void finalize_gscale_kernel(float* gscale, const float* g_x) {
  const float am = __uint_as_float(*reinterpret_cast<unsigned*>(gscale + 1));
  const float gw = (am == 0.0f) ? 1.0f : __fdiv_rn(am, kGlobalDivisor);
  const float gx = *g_x;
  gscale[0] = gx;
  gscale[1] = gw;
  gscale[2] = __fmul_rn(gx, gw);
  gscale[3] = 0.0f;
}

// l2s[0][n][j] = hi, l2s[1][n][j] = lo with v = fp32(L2[j][n] / alpha), hi = bf16(v), lo = bf16(v - hi).
__global__ void make_l2s_kernel(const __nv_bfloat16* __restrict__ L2, const float* __restrict__ gscale,
                                __nv_bfloat16* __restrict__ l2s, int N, int r) {
  const float alpha = gscale[2];
  const int64_t total = static_cast<int64_t>(N) * r;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = i / r;
    const int j = static_cast<int>(i % r);
    const float v = __fdiv_rn(__bfloat162float(L2[static_cast<int64_t>(j) * N + n]), alpha);
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(v, __bfloat162float(hi)));
    l2s[i] = hi;
    l2s[total + i] = lo;
  }
}

// Pass 2: quantise R with g_w. Lanes 0-15 hold one 16-element block, 16-31 the next.
template <int R>
__global__ void __launch_bounds__(kPackThreads) residual_quant_kernel(
    const __nv_bfloat16* __restrict__ W, const __nv_bfloat16* __restrict__ L1,
    const __nv_bfloat16* __restrict__ l2t, const float* __restrict__ smooth, int N, int K,
    const float* __restrict__ gscale, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (kPackThreads / 32) + (threadIdx.x >> 5);
  const int slabs = K / 32;
  const int slab = gw % slabs;
  const int n_begin = (gw / slabs) * kPackRowsPerWarp;
  if (n_begin >= N) return;
  const int k = slab * 32 + lane;
  float l1row[R];
  load_l1_row<R>(L1, k, l1row);
  const double lam = smooth != nullptr ? static_cast<double>(smooth[k]) : 1.0;
  const float g = gscale[1];
  const float d = __fmul_rn(6.0f, g);
  const int n_end = min(N, n_begin + kPackRowsPerWarp);
  for (int n = n_begin; n < n_end; ++n) {
    const float x = residual_at<R>(W, l1row, l2t, N, K, n, k, lam);
    float am = fabsf(x);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    const float t = __fdiv_rn(am, d);
    const uint32_t S = f32_to_e4m3(t);
    const float sd = __fmul_rn(e4m3_to_f32(S), g);
    const float inv = (sd == 0.0f) ? 0.0f : __frcp_rn(sd);
    const float q = __fmul_rn(x, inv);
    // one code per lane; even lanes pair their code with the odd neighbour's
    const float qv[8] = {q, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
    const uint32_t mine = f32x8_to_e2m1(qv) & 0xFu;
    const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
    uint32_t byte = (mine | (other << 4)) & 0xFFu;  // valid on even lanes
    // gather 4 bytes (lanes 8i, 8i+2, 8i+4, 8i+6) into lane 8i
    const uint32_t b1 = __shfl_down_sync(0xffffffffu, byte, 2);
    const uint32_t b2 = __shfl_down_sync(0xffffffffu, byte, 4);
    const uint32_t b3 = __shfl_down_sync(0xffffffffu, byte, 6);
    if ((lane & 7) == 0) {
      const uint32_t word = byte | (b1 << 8) | (b2 << 16) | (b3 << 24);
      *reinterpret_cast<uint32_t*>(codes + static_cast<int64_t>(n) * (K / 2) + (slab * 32 + lane) / 2) = word;
    }
    if ((lane & 15) == 0) scales[scale_offset(K, n, (slab * 32 + lane) / 16)] = static_cast<uint8_t>(S);
  }
}

}  // namespace svdq
