// qkv_post.cuh — fused QKV post-processing in the GEMM epilogue: per-head
// RMSNorm of the Q and K heads and the rotary embedding, applied to the
// layer's bf16 output before it is stored.
//
// Blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers", section
// "Quantizing models with structural rewrites": the Q, K and V projections
// are fused into one to_qkv layer, and the fused operator consumes that
// projection, the Q/K normalisation and the rotary embedding together.
// For a [M, 3 * H * 128] output laid out [Q | K | V] (head_dim 128):
//   q = bf16(alpha * acc + b)                       (the layer output)
//   n_i = q_i / sqrt(mean_i(q_i^2) + eps) * w_i     (RMSNorm per head, fp32)
//   (n0, n1) -> (n0 c_j - n1 s_j, n1 c_j + n0 s_j)  (pair 2j, 2j+1 rotated by theta_j)
// rounded to bf16 once; V is stored unchanged. An epilogue warp holds 32 rows
// of one 128-column head, so each thread owns a whole head row: the norm is
// thread-local and each rotation pair lies in one 32-column chunk.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace svdq {

constexpr int kHeadDim = 128;

struct QkvPost {
  const __nv_bfloat16* w_q;  // [128] RMSNorm weight of the Q heads
  const __nv_bfloat16* w_k;  // [128] RMSNorm weight of the K heads
  const float* cos;          // [M][ld_rope] cos(theta_j) per token and pair (64 used)
  const float* sin;          // [M][ld_rope] sin(theta_j)
  int64_t ld_rope;
  int hd;                    // columns of each of Q, K and V (heads * 128)
  float eps;
};

// Epilogue of an MLP pair's up projection (blog "Bringing Nunchaku 4-bit
// Diffusion Inference to Diffusers", section "Introducing Nunchaku Lite":
// the full engine's speed comes partly from fused GELU / MLP kernels):
// h = bf16(GELU(bf16(alpha acc + b))) quantised in place for the down
// projection (NVFP4 codes and tiled block scales with the down projection's
// activation scale g_h), and h . L1_down accumulated on the tensor cores over
// each CTA pair's run of tiles that share their rows (one fp32 XL1 partial per
// run, summed afterwards in tile order).
struct MlpPost {
  const float* g_h;           // device float: the down projection's activation decode scale
  uint8_t* codes;             // [M][N/2]
  uint8_t* scales;            // tiled, rows padded to 128 (padding rows get zero scales)
  float* partial;             // [tiles][256][r_down] fp32: XL1 partial of each run of tiles (slot = first tile)
  int m_pad;                  // M rounded up to 128
  int store_h;                // also store h (bf16) through the output map
  int approximate;            // tanh form of GELU
};

// GELU in fp32: x Phi(x) = x erfc(-x / sqrt 2) / 2, or the tanh form
// x (1 + tanh u) / 2 = x / (1 + exp(-2u)), u = sqrt(2/pi) (x + 0.044715 x^3);
// both written without the cancellation of 1 + erf / 1 + tanh for negative x.
//
// h is rounded to bf16 (8 significant bits), so a relative error far below
// 2^-10 is enough for the result to lie within one bf16 step of the correctly
// rounded value. The fast paths below stay far inside that:
//  * erfc(z), z >= 0, by the Chebyshev fit of Press, Teukolsky, Vetterling and
//    Flannery (Numerical Recipes in C, 2nd ed., section 6.2, erfcc): with
//    t = 1 / (1 + z/2), erfc(z) = t exp(-z^2 + P(t)), P of degree 9, fractional
//    error below 1.2e-7 for every z >= 0; erfc(-z) = 2 - erfc(z);
//  * exponentials by the hardware exp2 (__expf, relative error ~2^-21),
//    reciprocals by __fdividef.
// Where a result would fall below the normal fp32 range (|z| > 9 for erfc,
// 2u < -80 in the tanh form) the accurate library functions take over, so the
// far negative tail keeps its tiny values (subnormals included) instead of
// flushing them to zero.
__device__ __forceinline__ float erfc_fast_nonneg(float z) {
  const float t = __fdividef(1.0f, __fmaf_rn(0.5f, z, 1.0f));
  float p = 0.17087277f;
  p = __fmaf_rn(p, t, -0.82215223f);
  p = __fmaf_rn(p, t, 1.48851587f);
  p = __fmaf_rn(p, t, -1.13520398f);
  p = __fmaf_rn(p, t, 0.27886807f);
  p = __fmaf_rn(p, t, -0.18628806f);
  p = __fmaf_rn(p, t, 0.09678418f);
  p = __fmaf_rn(p, t, 0.37409196f);
  p = __fmaf_rn(p, t, 1.00002368f);
  p = __fmaf_rn(p, t, -1.26551223f);
  return t * __expf(__fmaf_rn(-z, z, p));
}

// The far negative tail with the accurate library functions (rarely reached,
// kept out of line so the fast paths stay compact).
__device__ __noinline__ float gelu_tail(float x, bool approximate) {
  if (approximate) {
    const float u = __fmul_rn(0.7978845608028654f, __fmaf_rn(__fmul_rn(0.044715f, x), __fmul_rn(x, x), x));
    const float e = expf(__fmul_rn(2.0f, u));
    return __fdiv_rn(__fmul_rn(x, e), __fadd_rn(1.0f, e));
  }
  return __fmul_rn(__fmul_rn(0.5f, x), erfcf(__fmul_rn(x, -0.7071067811865476f)));
}

// tanh form, x sigma(2u) with the logistic sigma evaluated as 1 / (1 + e^{-t})
// for t >= 0 and e^{t} / (1 + e^{t}) for t < 0 (e^{-|t|} <= 1 never
// overflows), branch-free; *tail is set where the result may fall below the
// normal fp32 range (u <= -40), for which gelu_tail recomputes it.
__device__ __forceinline__ float gelu_tanh_fast(float x, bool& tail) {
  const float u = __fmul_rn(0.7978845608028654f, __fmaf_rn(__fmul_rn(0.044715f, x), __fmul_rn(x, x), x));
  const float e = __expf(-2.0f * fabsf(u));
  tail = u <= -40.0f;
  return __fdividef(u >= 0.0f ? x : x * e, 1.0f + e);
}

// erf form, x erfc(-x / sqrt 2) / 2, branch-free; *tail where |z| > 9.
__device__ __forceinline__ float gelu_erf_fast(float x, bool& tail) {
  const float z = x * -0.7071067811865476f;
  const float az = fabsf(z);
  const float e = erfc_fast_nonneg(fminf(az, 9.0f));
  tail = az > 9.0f;
  return 0.5f * x * (z >= 0.0f ? e : 2.0f - e);
}

__device__ __forceinline__ float gelu_tanh_f32(float x) {
  bool tail;
  const float h = gelu_tanh_fast(x, tail);
  return tail ? gelu_tail(x, true) : h;
}
__device__ __forceinline__ float gelu_erf_f32(float x) {
  bool tail;
  const float h = gelu_erf_fast(x, tail);
  return tail ? gelu_tail(x, false) : h;
}

__device__ __forceinline__ float gelu_f32(float x, bool approximate) {
  return approximate ? gelu_tanh_f32(x) : gelu_erf_f32(x);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// One head row held as 64 packed bf16 pairs (element 2j in the low half of
// p[j]): RMSNorm with weight w, then the rotation of each pair j by this
// row's angle (cs[j], sn[j]: 64 floats each, 16-byte aligned), in place.
__device__ __forceinline__ void qk_norm_rope_row(uint32_t (&p)[64], const __nv_bfloat16* __restrict__ w,
                                                 const float* __restrict__ cs, const float* __restrict__ sn,
                                                 float eps) {
  float ss = 0.0f;
#pragma unroll
  for (int j = 0; j < 64; ++j) {
    const float x0 = bf16_lo(p[j]), x1 = bf16_hi(p[j]);
    ss = __fmaf_rn(x0, x0, ss);
    ss = __fmaf_rn(x1, x1, ss);
  }
  const float rstd = 1.0f / sqrtf(__fmaf_rn(ss, 1.0f / kHeadDim, eps));
#pragma unroll
  for (int g = 0; g < 16; ++g) {  // 8 columns = 4 pairs per group
    const uint4 wv = *reinterpret_cast<const uint4*>(w + 8 * g);
    const float4 c4 = *reinterpret_cast<const float4*>(cs + 4 * g);
    const float4 s4 = *reinterpret_cast<const float4*>(sn + 4 * g);
    const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
    const float cc[4] = {c4.x, c4.y, c4.z, c4.w};
    const float ssn[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int j = 4 * g + t;
      const float n0 = bf16_lo(p[j]) * rstd * bf16_lo(ww[t]);
      const float n1 = bf16_hi(p[j]) * rstd * bf16_hi(ww[t]);
      p[j] = pack_bf16(__fmaf_rn(n0, cc[t], -n1 * ssn[t]), __fmaf_rn(n1, cc[t], n0 * ssn[t]));
    }
  }
}

// bf16 pairs of y = alpha * acc + b for one 32-column chunk (bias: 32 bf16 at
// bcol, or none).
__device__ __forceinline__ void pack_chunk(const uint32_t (&v)[32], const __nv_bfloat16* __restrict__ bcol,
                                           float alpha, uint32_t* out) {
  uint32_t bw[16];
  if (bcol != nullptr) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 u = *reinterpret_cast<const uint4*>(bcol + 8 * q);
      bw[4 * q] = u.x;
      bw[4 * q + 1] = u.y;
      bw[4 * q + 2] = u.z;
      bw[4 * q + 3] = u.w;
    }
  } else {
#pragma unroll
    for (int q = 0; q < 16; ++q) bw[q] = 0u;
  }
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    const float y0 = __fmaf_rn(__uint_as_float(v[2 * p]), alpha, bf16_lo(bw[p]));
    const float y1 = __fmaf_rn(__uint_as_float(v[2 * p + 1]), alpha, bf16_hi(bw[p]));
    out[p] = pack_bf16(y0, y1);
  }
}

}  // namespace svdq
