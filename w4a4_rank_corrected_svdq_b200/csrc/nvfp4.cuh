// nvfp4.cuh — the NVFP4 block quantiser and the tiled scale layout, device side.
//
// NVFP4 as used by the SVDQuant W4A4 layer (blog "Bringing Nunchaku 4-bit
// Diffusion Inference to Diffusers", section "Native loading in Diffusers":
// precision nvfp4, group size 16): E2M1 codes, one E4M3 scale per 16
// contiguous K-elements, one fp32 decode scale g per tensor. Per block:
//   t  = fp32(amax / fp32(6 g))           S  = e4m3_rn_satfinite(t)
//   sd = fp32(dec(S) * g)                 inv = fp32(1 / sd)   (0 if sd == 0)
//   q  = fp32(x * inv)                    code = e2m1_rn_satfinite(q)
// Every step is one correctly rounded fp32 operation, so the result is
// bit-reproducible by any IEEE implementation of the same steps.
#pragma once

#include "ptx.cuh"

namespace svdq {

// Decode-scale divisor: 6 (largest E2M1 magnitude) * 448 (largest E4M3 value).
constexpr float kGlobalDivisor = 2688.0f;

// Byte offset of the scale of (row, kb) in the tiled layout: 128-row x 64-K
// atoms of 512 bytes, K-atoms contiguous inside a 128-row block; inside an atom
// row r sits at (r%32)*16 + (r/32)*4 and the 4 K-blocks are consecutive bytes.
// This is the order tcgen05.cp (32x128b, warpx4) moves into TMEM for the
// block-scaled MMA.
__host__ __device__ __forceinline__ size_t scale_offset(int K, int row, int kb) {
  const size_t atom = static_cast<size_t>(row / 128) * static_cast<size_t>(K / 64) + static_cast<size_t>(kb / 4);
  const int r = row % 128;
  return atom * 512 + static_cast<size_t>((r % 32) * 16 + (r / 32) * 4 + (kb % 4));
}

struct QuantOut {
  uint32_t codes;  // 8 E2M1 codes, element i in bits 4i..4i+3
  uint32_t scale;  // E4M3 code of the block
};

// Block amax -> scale -> codes for the 8 values this thread holds; the other
// half of the 16-element block is held by the lane whose id differs in bit
// `pair_mask` (the amax is exchanged with one shuffle). All 32 lanes must call.
__device__ __forceinline__ QuantOut quantize8(const float (&f)[8], float g, float d, int pair_mask) {
  float am = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(f[i]));
  am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, pair_mask));
  const float t = __fdiv_rn(am, d);
  const uint32_t S = f32_to_e4m3(t);
  const float sd = __fmul_rn(e4m3_to_f32(S), g);
  const float inv = (sd == 0.0f) ? 0.0f : __frcp_rn(sd);
  float q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(f[i], inv);
  return {f32x8_to_e2m1(q), S};
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

}  // namespace svdq
