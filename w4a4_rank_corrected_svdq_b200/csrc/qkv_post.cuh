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
// rounded value. The paths below stay far inside that:
//  * erfc(z), z >= 0, by the Chebyshev fit of Press, Teukolsky, Vetterling and
//    Flannery (Numerical Recipes in C, 2nd ed., section 6.2, erfcc): with
//    t = 1 / (1 + z/2), erfc(z) = t exp(-z^2 + P(t)), P of degree 9, fractional
//    error below 1.2e-7 for every z >= 0; erfc(-z) = 2 - erfc(z);
//  * exponentials by the hardware exp2 (ex2.approx, relative error ~2^-22),
//    reciprocals by rcp.approx.
// The far negative tail keeps its tiny values (subnormals included): the
// exponential is taken as 2^(e + 64), which stays a normal number for every
// exponent e >= -190, and the product is scaled by 2^-64 (and 1/2) last, so
// a result below the normal range is rounded once, by that multiplication.
// Where e < -190 the true result is below 2^-180 in magnitude, rounds to zero
// in fp32, and the flushed exponential gives that zero. Both forms are
// branch-free and work on a pair of values (packed f32x2 arithmetic for the
// polynomial and products; the hardware exp2 and reciprocal per lane).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kTwoPowM64 = 0x1p-64f;
constexpr float kTwoPowM65 = 0x1p-65f;

// erf form: z = -x / sqrt 2, a = |z|, E = 2^64 erfc(a); x <= 0 (z >= 0):
// (x E) 2^-65; x > 0: (x/2) (2 - E 2^-64). a is capped at 16, where erfc is
// below 2^-370 (the product rounds to zero either way); the cap keeps a huge
// |x| from turning a^2 into inf.
__device__ __forceinline__ float2 gelu_erf_pair(float2 x) {
  const float2 z = __fmul2_rn(x, f2(-0.7071067811865476f));
  const float2 a = make_float2(fminf(fabsf(z.x), 16.0f), fminf(fabsf(z.y), 16.0f));
  const float2 d = __ffma2_rn(a, f2(0.5f), f2(1.0f));
  const float2 t = make_float2(rcp_approx(d.x), rcp_approx(d.y));
  float2 p = f2(0.17087277f);
  p = __ffma2_rn(p, t, f2(-0.82215223f));
  p = __ffma2_rn(p, t, f2(1.48851587f));
  p = __ffma2_rn(p, t, f2(-1.13520398f));
  p = __ffma2_rn(p, t, f2(0.27886807f));
  p = __ffma2_rn(p, t, f2(-0.18628806f));
  p = __ffma2_rn(p, t, f2(0.09678418f));
  p = __ffma2_rn(p, t, f2(0.37409196f));
  p = __ffma2_rn(p, t, f2(1.00002368f));
  p = __ffma2_rn(p, t, f2(-1.26551223f));
  // log2 of erfc(a) 2^64
  const float2 arg = __ffma2_rn(__ffma2_rn(make_float2(-a.x, -a.y), a, p), f2(kLog2e), f2(64.0f));
  const float2 E = __fmul2_rn(t, make_float2(ex2_approx(arg.x), ex2_approx(arg.y)));
  const float2 c = __ffma2_rn(E, f2(-kTwoPowM64), f2(2.0f));
  const float2 phi = make_float2(z.x >= 0.0f ? E.x : c.x, z.y >= 0.0f ? E.y : c.y);
  const float2 sc = make_float2(z.x >= 0.0f ? kTwoPowM65 : 0.5f, z.y >= 0.0f ? kTwoPowM65 : 0.5f);
  return __fmul2_rn(__fmul2_rn(x, phi), sc);
}

// tanh form: x sigma(2u) with sigma(s) = 1 / (1 + e^{-s}) for s >= 0 and
// e^{s} / (1 + e^{s}) for s < 0 (e^{-|s|} <= 1 never overflows). With
// E = 2^64 e^{-2|u|}: u >= 0: x / (1 + E 2^-64); u < 0: (x E / (1 + E 2^-64)) 2^-64.
// |u| is capped at 128, beyond which e^{-2|u|} < 2^-369.
__device__ __forceinline__ float2 gelu_tanh_pair(float2 x) {
  const float2 x2 = __fmul2_rn(x, x);
  const float2 u = __fmul2_rn(f2(0.7978845608028654f), __ffma2_rn(__fmul2_rn(f2(0.044715f), x), x2, x));
  const float2 au = make_float2(fminf(fabsf(u.x), 128.0f), fminf(fabsf(u.y), 128.0f));
  const float2 arg = __ffma2_rn(au, f2(-2.0f * kLog2e), f2(64.0f));
  const float2 E = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
  const float2 den = __ffma2_rn(E, f2(kTwoPowM64), f2(1.0f));
  const float2 num = make_float2(u.x >= 0.0f ? x.x : x.x * E.x, u.y >= 0.0f ? x.y : x.y * E.y);
  const float2 sc = make_float2(u.x >= 0.0f ? 1.0f : kTwoPowM64, u.y >= 0.0f ? 1.0f : kTwoPowM64);
  return __fmul2_rn(__fmul2_rn(num, make_float2(rcp_approx(den.x), rcp_approx(den.y))), sc);
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
