// awq_w4a16.cuh — the weight-only AWQ W4A16 layer (INT4 weights, group 64,
// bf16 activations) for memory-bound modulation projections.
//
// Blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers", section
// "Introducing Nunchaku Lite": the awq_w4a16 kernel family keeps 4-bit weights
// with 16-bit activations for adaptive-normalisation and modulation layers,
// which are memory-bound and precision-sensitive; section "Native loading in
// Diffusers" fixes precision int4 and group size 64.
//
// Quantisation (load time), per output row n and group of 64 K-elements, with
// the AWQ reference pseudo-quantiser's rule, each step one correctly rounded
// fp32 operation:
//   w = fp32(W[n,k] * a_k)   (a = the activation-aware factor, or w = W)
//   s = bf16(fp32(max(fp32(max w - min w), 1e-5) / 15))     stored scale
//   z = clamp(rne(fp32(-min w / s)), 0, 15)                  stored zero point
//   q = clamp(rne(fp32(w / s)) + z, 0, 15)                   code
// Layer (every call): Y[m,n] = bf16(sum_k x^_k w'[n,k] + b[n]) with
// w' = (q - z) s (exact in fp32), x^ = fp32(x * fp32(1/a_k)) (or x), fp32
// accumulation.
//
// The layer reads N K / 2 bytes of codes for M K multiply-adds per row block:
// for the few activation rows of a modulation projection it is bound by HBM,
// not by the tensor cores, so it runs on the CUDA cores: each warp streams one
// weight row as coalesced 4-byte code words while the activations sit in
// shared memory.
#pragma once

#include "nvfp4.cuh"

namespace svdq {

constexpr int kAwqGroup = 64;
constexpr int kAwqThreads = 256;

// One thread per (row, group): codes (element 2j in the low nibble of byte j),
// bf16 scale, u8 zero point.
__global__ void __launch_bounds__(kAwqThreads) awq_pack_kernel(const __nv_bfloat16* __restrict__ W, int N, int K,
                                                               const float* __restrict__ act,
                                                               uint8_t* __restrict__ codes,
                                                               __nv_bfloat16* __restrict__ scales,
                                                               uint8_t* __restrict__ zeros) {
  const int G = K / kAwqGroup;
  const int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (t >= static_cast<int64_t>(N) * G) return;
  const int64_t n = t / G;
  const int g = static_cast<int>(t % G);
  const __nv_bfloat16* src = W + n * K + g * kAwqGroup;
  float w[kAwqGroup];
#pragma unroll
  for (int v = 0; v < kAwqGroup / 8; ++v) bf16x8_to_f32(ldg_v4(src + 8 * v), *reinterpret_cast<float(*)[8]>(w + 8 * v));
  if (act != nullptr) {
#pragma unroll
    for (int i = 0; i < kAwqGroup; ++i) w[i] = __fmul_rn(w[i], act[g * kAwqGroup + i]);
  }
  float mx = w[0], mn = w[0];
#pragma unroll
  for (int i = 1; i < kAwqGroup; ++i) {
    mx = fmaxf(mx, w[i]);
    mn = fminf(mn, w[i]);
  }
  const float d = fmaxf(__fsub_rn(mx, mn), 1e-5f);
  const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(d, 15.0f));
  const float s = __bfloat162float(sb);
  const float z = fminf(fmaxf(rintf(__fdiv_rn(-mn, s)), 0.0f), 15.0f);
  uint32_t packed[kAwqGroup / 8];
#pragma unroll
  for (int j = 0; j < kAwqGroup / 8; ++j) {
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float q = fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(w[8 * j + e], s)), z), 0.0f), 15.0f);
      word |= static_cast<uint32_t>(q) << (4 * e);
    }
    packed[j] = word;
  }
  uint4* dst = reinterpret_cast<uint4*>(codes + n * (K / 2) + g * (kAwqGroup / 2));
  dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  scales[t] = sb;
  zeros[t] = static_cast<uint8_t>(z);
}

// Y (the first min(M, MT) rows of X) = X^ . W'^T + b. Shared memory holds X^
// as fp32 in two planes of float4 per 8-element group (elements 0-3 and 4-7),
// so that lanes reading consecutive groups touch consecutive 16-byte words.
// Each warp takes output rows n = warp_id, warp_id + total_warps, ...; lane l
// takes the row's code words (8 codes, all of one 64-group) l, l + 32, ...:
// coalesced 128-byte loads per warp. Per word the integers q - z are formed
// exactly (2^23 + q from one byte permute, minus the exact 2^23 + z), the
// eight products x (q - z) are summed as two fp32 pair partials and scaled by
// s once; the row keeps two fp32 partial sums (even and odd elements), added
// at the end. Packed f32x2 arithmetic throughout.
template <int MT>
__global__ void __launch_bounds__(kAwqThreads) awq_gemv_kernel(int M, int N, int K,
                                                               const __nv_bfloat16* __restrict__ X, int64_t ldx,
                                                               const uint8_t* __restrict__ codes,
                                                               const __nv_bfloat16* __restrict__ scales,
                                                               const uint8_t* __restrict__ zeros,
                                                               const float* __restrict__ inv_act,
                                                               const __nv_bfloat16* __restrict__ bias,
                                                               __nv_bfloat16* __restrict__ Y, int64_t ldy) {
  extern __shared__ float4 xs4[];  // [MT][2][K/8]
  const int rows = M < MT ? M : MT;
  const int K8 = K / 8;
  for (int i = threadIdx.x; i < MT * K8; i += blockDim.x) {
    const int m = i / K8, j = i % K8;
    float f[8];
    if (m < rows) {
      bf16x8_to_f32(ldg_nc_v4(X + static_cast<int64_t>(m) * ldx + 8 * j), f);
      if (inv_act != nullptr) {
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __fmul_rn(f[e], inv_act[8 * j + e]);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = 0.0f;
    }
    xs4[(2 * m) * K8 + j] = make_float4(f[0], f[1], f[2], f[3]);
    xs4[(2 * m + 1) * K8 + j] = make_float4(f[4], f[5], f[6], f[7]);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int warps = static_cast<int>(gridDim.x) * (kAwqThreads / 32);
  const int G = K / kAwqGroup;
  for (int n = blockIdx.x * (kAwqThreads / 32) + (threadIdx.x >> 5); n < N; n += warps) {
    const uint32_t* crow = reinterpret_cast<const uint32_t*>(codes + static_cast<int64_t>(n) * (K / 2));
    const __nv_bfloat16* srow = scales + static_cast<int64_t>(n) * G;
    const uint8_t* zrow = zeros + static_cast<int64_t>(n) * G;
    float2 acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = make_float2(0.0f, 0.0f);
#pragma unroll 4
    for (int j = lane; j < K8; j += 32) {
      const uint32_t v = __ldg(crow + j);
      const int g = j >> 3;
      const float s = __bfloat162float(srow[g]);
      const float zf = __fadd_rn(8388608.0f, static_cast<float>(zrow[g]));  // 2^23 + z, exact
      const float2 s2 = make_float2(s, s), nz2 = make_float2(-zf, -zf);
      const uint32_t lo = v & 0x0F0F0F0Fu, hi = (v >> 4) & 0x0F0F0F0Fu;
      float2 d[4];  // (q - z) of elements (2b, 2b + 1): the low and high nibble of byte b
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const float2 q = make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7650u + b)),
                                     __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7650u + b)));
        d[b] = __fadd2_rn(q, nz2);
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const float4 a = xs4[(2 * m) * K8 + j];
        const float4 c = xs4[(2 * m + 1) * K8 + j];
        float2 t = __fmul2_rn(make_float2(a.x, a.y), d[0]);
        t = __ffma2_rn(make_float2(a.z, a.w), d[1], t);
        t = __ffma2_rn(make_float2(c.x, c.y), d[2], t);
        t = __ffma2_rn(make_float2(c.z, c.w), d[3], t);
        acc[m] = __ffma2_rn(t, s2, acc[m]);
      }
    }
    float r[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      r[m] = __fadd_rn(acc[m].x, acc[m].y);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) r[m] += __shfl_xor_sync(0xffffffffu, r[m], o);
    }
    if (lane == 0) {
      const float bn = bias != nullptr ? __bfloat162float(bias[n]) : 0.0f;
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (m < rows) Y[static_cast<int64_t>(m) * ldy + n] = __float2bfloat16_rn(__fadd_rn(r[m], bn));
    }
  }
}

}  // namespace svdq
