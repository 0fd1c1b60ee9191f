// quantize_act.cuh — activation NVFP4 quantisation fused with the low-rank
// down projection XL1 = X . L1 (one read of X).
//
// Blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers", figure
// caption in "Background: SVDQuant and Nunchaku": the low-rank down
// projection is fused with the quantisation kernel, so the 16-bit branch adds
// no extra pass over the activations.
//
// Work split: a CTA owns 128 rows (8 warps x 16 rows) and a K-range; the
// K-ranges of one row block form a thread-block cluster (KS CTAs, KS | 8). Each
// thread loads 16 contiguous bytes (8 bf16) of two rows per 32-column step:
//  * quantisation: a 16-element block spans two neighbouring lanes, whose
//    amax is exchanged with one shuffle;
//  * down projection: the same registers are the A fragments of two
//    m16n8k16 bf16 MMAs under a fixed permutation of K (the dot product does
//    not depend on the order of K), and 16 bytes of l1t = L1^T give the
//    matching B fragments.
// Partial XL1 sums of the KS CTAs are added in a fixed order through
// distributed shared memory, so the result is deterministic.
#pragma once

#include <cooperative_groups.h>

#include "nvfp4.cuh"

namespace svdq {

constexpr int kQuantThreads = 256;
constexpr int kQuantRows = 128;

template <int R>
__global__ void __launch_bounds__(kQuantThreads) quantize_act_kernel(
    const __nv_bfloat16* __restrict__ X, int64_t ldx, int M, int K, const float* __restrict__ g_x,
    const __nv_bfloat16* __restrict__ l1t, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
    __nv_bfloat16* __restrict__ xl1, int kchunk) {
  namespace cg = cooperative_groups;
  constexpr int NT = R / 8;  // n-tiles of 8 columns of XL1
  extern __shared__ float part[];  // [128][R] partial XL1 of this CTA

  cg::cluster_group cluster = cg::this_cluster();
  const int KS = static_cast<int>(cluster.num_blocks());
  const int ks = static_cast<int>(cluster.block_rank());

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int gq = lane >> 2;  // group id (row within the 8-row half)
  const int c = lane & 3;    // thread in group
  const int m0 = blockIdx.y * kQuantRows;
  const int row0 = m0 + warp * 16 + gq;
  const int row1 = row0 + 8;
  const bool v0 = row0 < M;
  const bool v1 = row1 < M;
  const int k_begin = ks * kchunk;
  const int k_end = min(K, k_begin + kchunk);
  const float g = *g_x;
  const float d = __fmul_rn(6.0f, g);

  const __nv_bfloat16* x0 = X + static_cast<int64_t>(v0 ? row0 : 0) * ldx;
  const __nv_bfloat16* x1 = X + static_cast<int64_t>(v1 ? row1 : 0) * ldx;
  const int64_t code_ld = K / 2;

  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[t][i] = 0.0f;

  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  uint4 a0 = zero, a1 = zero;
  if (k_begin < k_end) {
    a0 = v0 ? ldg_nc_v4(x0 + k_begin + 8 * c) : zero;
    a1 = v1 ? ldg_nc_v4(x1 + k_begin + 8 * c) : zero;
  }
#pragma unroll 1
  for (int k = k_begin; k < k_end; k += 32) {
    const int col = k + 8 * c;
    // prefetch the next step's activations
    uint4 n0 = zero, n1 = zero;
    if (k + 32 < k_end) {
      n0 = v0 ? ldg_nc_v4(x0 + col + 32) : zero;
      n1 = v1 ? ldg_nc_v4(x1 + col + 32) : zero;
    }
    // ---- NVFP4 quantisation of the two rows' 8-element slices
    {
      float f[8];
      bf16x8_to_f32(a0, f);
      const QuantOut q0 = quantize8(f, g, d, 1);
      bf16x8_to_f32(a1, f);
      const QuantOut q1 = quantize8(f, g, d, 1);
      if (v0) *reinterpret_cast<uint32_t*>(codes + row0 * code_ld + col / 2) = q0.codes;
      if (v1) *reinterpret_cast<uint32_t*>(codes + row1 * code_ld + col / 2) = q1.codes;
      if ((c & 1) == 0) {  // rows in [M, 128*ceil(M/128)) get a zero scale
        scales[scale_offset(K, row0, col / 16)] = static_cast<uint8_t>(q0.scale);
        scales[scale_offset(K, row1, col / 16)] = static_cast<uint8_t>(q1.scale);
      }
    }
    // ---- down projection on the tensor cores
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const uint4 b = ldg_v4(l1t + static_cast<int64_t>(8 * t + gq) * K + col);
      mma_m16n8k16_bf16(acc[t], a0.x, a1.x, a0.y, a1.y, b.x, b.y);
      mma_m16n8k16_bf16(acc[t], a0.z, a1.z, a0.w, a1.w, b.z, b.w);
    }
    a0 = n0;
    a1 = n1;
  }

  // ---- partial XL1 of this CTA to shared memory
  {
    const int r0 = warp * 16 + gq;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int j = 8 * t + 2 * c;
      part[r0 * R + j] = acc[t][0];
      part[r0 * R + j + 1] = acc[t][1];
      part[(r0 + 8) * R + j] = acc[t][2];
      part[(r0 + 8) * R + j + 1] = acc[t][3];
    }
  }
  cluster.sync();
  // ---- fixed-order reduction over the cluster; CTA ks finishes rows [ks*rpc, (ks+1)*rpc)
  const int rpc = kQuantRows / KS;
  for (int i = threadIdx.x; i < rpc * R; i += kQuantThreads) {
    const int rr = ks * rpc + i / R;
    const int j = i % R;
    float s = 0.0f;
    for (int p = 0; p < KS; ++p) {
      const float* peer = cluster.map_shared_rank(part, p);
      s += peer[rr * R + j];
    }
    if (m0 + rr < M) xl1[static_cast<int64_t>(m0 + rr) * R + j] = __float2bfloat16_rn(s);
  }
  cluster.sync();
}

}  // namespace svdq
