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
// weight row with coalesced 16-byte loads while the activations sit in shared
// memory.
#pragma once

#include "nvfp4.cuh"

namespace svdq {

constexpr int kAwqGroup = 64;
constexpr int kAwqThreads = 256;
constexpr int kAwqRows = 4;  // weight rows per warp pass of the GEMV
static_assert(kAwqGroup / 2 == 32, "a row's code bytes are 32 per group (the GEMV's scale offset is n K/2 >> 5)");

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

// Y (the first min(M, MT) rows of X) = X^ . W'^T + b.
// Shared memory holds X^ as fp32, per row m and 32-element chunk c as eight
// float4 (elements 4f..4f+3), float4 f stored at slot f ^ (c & 7): lanes
// reading consecutive chunks then touch eight different 16-byte bank groups.
// Each warp takes kAwqRows output rows per pass (passes strided by the number
// of warps); lane l takes the rows' chunks l, l + 32, ... (32 codes = 16 bytes,
// half a 64-group, so one scale and zero point each). Per
// 8-code word the integers q - z are formed exactly (2^23 + q from one byte
// permute, plus -(2^23 + z) built from its bit pattern), the products
// x (q - z) are summed as fp32 pairs over the chunk and scaled by s once.
// Packed f32x2 arithmetic.
template <int MT>
__global__ void __launch_bounds__(kAwqThreads) awq_gemv_kernel(int M, int N, int K,
                                                               const __nv_bfloat16* __restrict__ X, int64_t ldx,
                                                               const uint8_t* __restrict__ codes,
                                                               const __nv_bfloat16* __restrict__ scales,
                                                               const uint8_t* __restrict__ zeros,
                                                               const float* __restrict__ inv_act,
                                                               const __nv_bfloat16* __restrict__ bias,
                                                               __nv_bfloat16* __restrict__ Y, int64_t ldy) {
  extern __shared__ float4 xs4[];  // [MT][K/32][8], swizzled
  const int rows = M < MT ? M : MT;
  const int C = K / 32;
  const int lane = threadIdx.x & 31;
  const int warps = static_cast<int>(gridDim.x) * (kAwqThreads / 32);
  const int nstep = warps * kAwqRows;
  int n0 = (blockIdx.x * (kAwqThreads / 32) + (threadIdx.x >> 5)) * kAwqRows;
  // chunk loads are software-pipelined: the next chunk's codes, scales and zero
  // points (after a pass's last chunk: the next pass's first) are requested
  // before the current chunk's arithmetic, and the first pass's first chunk
  // before the activations are staged
  uint4 vn[kAwqRows];
  __nv_bfloat16 sn[kAwqRows];
  uint8_t zn[kAwqRows];
  // the code-row offsets n K/2 of the pass being fetched (rows past N repeat
  // the last one and are not stored); a row's scales and zero points start at
  // n G = n K/2 / 32
  int64_t ro[kAwqRows];
  auto bases = [&](int nb) {
#pragma unroll
    for (int r = 0; r < kAwqRows; ++r) ro[r] = static_cast<int64_t>(nb + r < N ? nb + r : N - 1) * (K / 2);
  };
  auto fetch = [&](int c) {
#pragma unroll
    for (int r = 0; r < kAwqRows; ++r) {
      vn[r] = ldg_nc_v4(codes + ro[r] + 16 * c);
      sn[r] = scales[(ro[r] >> 5) + (c >> 1)];
      zn[r] = zeros[(ro[r] >> 5) + (c >> 1)];
    }
  };
  if (n0 < N) {
    bases(n0);
    if (lane < C) fetch(lane);
  }
  for (int i = threadIdx.x; i < MT * (K / 4); i += blockDim.x) {
    const int m = i / (K / 4), q4 = i % (K / 4);  // float4 q4 of row m: elements 4 q4 .. 4 q4 + 3
    float4 f = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (m < rows) {
      const __nv_bfloat16* src = X + static_cast<int64_t>(m) * ldx + 4 * q4;
      const uint2 raw = *reinterpret_cast<const uint2*>(src);
      f = make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                      __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u));
      if (inv_act != nullptr) {
        const float4 iv = *reinterpret_cast<const float4*>(inv_act + 4 * q4);
        f = make_float4(__fmul_rn(f.x, iv.x), __fmul_rn(f.y, iv.y), __fmul_rn(f.z, iv.z), __fmul_rn(f.w, iv.w));
      }
    }
    const int c = q4 >> 3, fi = q4 & 7;
    xs4[(m * C + c) * 8 + (fi ^ (c & 7))] = f;
  }
  __syncthreads();
  // kAwqRows weight rows per warp pass: each X^ value read from shared memory
  // serves all of them (shared-memory bandwidth, not HBM, bounds a pass over
  // one row at a time).
  for (; n0 < N; n0 += nstep) {
    float2 acc[kAwqRows][MT];
#pragma unroll
    for (int r = 0; r < kAwqRows; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m] = make_float2(0.0f, 0.0f);
    for (int c = lane; c < C; c += 32) {
      uint4 v[kAwqRows];
      float sv[kAwqRows], nz[kAwqRows];
#pragma unroll
      for (int r = 0; r < kAwqRows; ++r) {
        v[r] = vn[r];
        sv[r] = __bfloat162float(sn[r]);
        nz[r] = __uint_as_float(0xCB000000u | zn[r]);  // -(2^23 + z), exact
      }
      if (c + 32 < C) {
        fetch(c + 32);
      } else if (n0 + nstep < N) {
        bases(n0 + nstep);
        fetch(lane);
      }
      const int sw = c & 7;
      float2 t[kAwqRows][MT];
#pragma unroll
      for (int r = 0; r < kAwqRows; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) t[r][m] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) {
        float2 d[kAwqRows][4];  // (q - z) of elements (2b, 2b + 1): low and high nibble of byte b of the word
#pragma unroll
        for (int r = 0; r < kAwqRows; ++r) {
          const uint32_t word = wd == 0 ? v[r].x : (wd == 1 ? v[r].y : (wd == 2 ? v[r].z : v[r].w));
          const uint32_t lo = word & 0x0F0F0F0Fu, hi = (word >> 4) & 0x0F0F0F0Fu;
          const float2 nz2 = make_float2(nz[r], nz[r]);
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const float2 q = make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7650u + b)),
                                         __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7650u + b)));
            d[r][b] = __fadd2_rn(q, nz2);
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const float4* xc = xs4 + (m * C + c) * 8;
          const float4 a = xc[(2 * wd) ^ sw];
          const float4 e = xc[(2 * wd + 1) ^ sw];
          const float2 x01 = make_float2(a.x, a.y), x23 = make_float2(a.z, a.w);
          const float2 x45 = make_float2(e.x, e.y), x67 = make_float2(e.z, e.w);
#pragma unroll
          for (int r = 0; r < kAwqRows; ++r) {
            t[r][m] = __ffma2_rn(x01, d[r][0], t[r][m]);
            t[r][m] = __ffma2_rn(x23, d[r][1], t[r][m]);
            t[r][m] = __ffma2_rn(x45, d[r][2], t[r][m]);
            t[r][m] = __ffma2_rn(x67, d[r][3], t[r][m]);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < kAwqRows; ++r) {
        const float2 s2 = make_float2(sv[r], sv[r]);
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = __ffma2_rn(t[r][m], s2, acc[r][m]);
      }
    }
#pragma unroll
    for (int r = 0; r < kAwqRows; ++r) {
      const int n = n0 + r;
      float res[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        res[m] = __fadd_rn(acc[r][m].x, acc[r][m].y);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) res[m] += __shfl_xor_sync(0xffffffffu, res[m], o);
      }
      if (lane == 0 && n < N) {
        const float bn = bias != nullptr ? __bfloat162float(bias[n]) : 0.0f;
#pragma unroll
        for (int m = 0; m < MT; ++m)
          if (m < rows) Y[static_cast<int64_t>(m) * ldy + n] = __float2bfloat16_rn(__fadd_rn(res[m], bn));
      }
    }
  }
}

// ------------------------------------------------------------------ bulk-copy ring variant
// The same layer with the weight rows streamed by one producer thread through a
// ring of shared-memory stages (cp.async.bulk, completion counted on an
// mbarrier), so each SM keeps a whole stage ring of weight bytes in flight
// instead of the 16 bytes per lane and row of direct loads. A stage holds
// kAwqRingRows consecutive weight rows: their codes (rows x K/2 bytes), bf16
// scales and zero points (rows x K/64 each) as three contiguous bulk copies,
// which needs K % 1024 == 0 (16-byte multiples for every row count). Each CTA
// owns one contiguous run of rows; its 8 consumer warps take kAwqRows rows of
// every stage each, with the activations staged as in awq_gemv_kernel. Every
// wait is bounded (mbar_wait).
constexpr int kAwqRingRows = 8 * kAwqRows;  // rows per stage (8 consumer warps)
constexpr int kAwqRingThreads = 288;        // 8 consumer warps + 1 producer warp
constexpr int kAwqRingMaxStages = 8;

__host__ __device__ constexpr int awq_ring_stage_bytes(int K) {
  return kAwqRingRows * (K / 2 + (K / kAwqGroup) * 3);
}

template <int MT>
__global__ void __launch_bounds__(kAwqRingThreads, 1) awq_gemv_ring_kernel(
    int M, int N, int K, const __nv_bfloat16* __restrict__ X, int64_t ldx, const uint8_t* __restrict__ codes,
    const __nv_bfloat16* __restrict__ scales, const uint8_t* __restrict__ zeros, const float* __restrict__ inv_act,
    const __nv_bfloat16* __restrict__ bias, __nv_bfloat16* __restrict__ Y, int64_t ldy, int stages) {
  extern __shared__ __align__(16) uint8_t ring_smem[];
  const int rows = M < MT ? M : MT;
  const int C = K / 32;
  const int G = K / kAwqGroup;
  float4* xs4 = reinterpret_cast<float4*>(ring_smem);  // [MT][K/32][8], swizzled
  uint8_t* ring = ring_smem + MT * K * 4;
  const int stage_bytes = awq_ring_stage_bytes(K);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + stages * stage_bytes);
  uint64_t* empty = full + kAwqRingMaxStages;
  int* abort_flag = reinterpret_cast<int*>(empty + kAwqRingMaxStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's rows [r0, r1) (balanced split) and their stages
  const int base = N / static_cast<int>(gridDim.x), rem = N % static_cast<int>(gridDim.x);
  const int r0 = static_cast<int>(blockIdx.x) * base + (static_cast<int>(blockIdx.x) < rem ? blockIdx.x : rem);
  const int r1 = r0 + base + (static_cast<int>(blockIdx.x) < rem ? 1 : 0);
  const int nst = (r1 - r0 + kAwqRingRows - 1) / kAwqRingRows;
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 8);  // the 8 consumer warps
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort = abort_flag;
  if (warp == 8) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      for (int i = 0; i < nst; ++i) {
        const int s = i % stages;
        if (!mbar_wait(&empty[s], ((i / stages) & 1) ^ 1, abort)) break;
        const int n0 = r0 + i * kAwqRingRows;
        const int nr = r1 - n0 < kAwqRingRows ? r1 - n0 : kAwqRingRows;
        uint8_t* st = ring + s * stage_bytes;
        const uint32_t cb = static_cast<uint32_t>(nr) * (K / 2), sb = static_cast<uint32_t>(nr) * G * 2,
                       zb = static_cast<uint32_t>(nr) * G;
        mbar_arrive_expect_tx(&full[s], cb + sb + zb);
        bulk_load(st, codes + static_cast<int64_t>(n0) * (K / 2), cb, &full[s]);
        bulk_load(st + kAwqRingRows * (K / 2), scales + static_cast<int64_t>(n0) * G, sb, &full[s]);
        bulk_load(st + kAwqRingRows * (K / 2 + 2 * G), zeros + static_cast<int64_t>(n0) * G, zb, &full[s]);
      }
      if (*abort) {  // error path: give copies that may still be in flight time to land
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 2000000ull) {
        }
      }
    }
    return;
  }
  // ------------------------------------------------------------------ consumers: stage the activations
  for (int i = threadIdx.x; i < MT * (K / 4); i += 256) {
    const int m = i / (K / 4), q4 = i % (K / 4);
    float4 f = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (m < rows) {
      const __nv_bfloat16* src = X + static_cast<int64_t>(m) * ldx + 4 * q4;
      const uint2 raw = *reinterpret_cast<const uint2*>(src);
      f = make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                      __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u));
      if (inv_act != nullptr) {
        const float4 iv = *reinterpret_cast<const float4*>(inv_act + 4 * q4);
        f = make_float4(__fmul_rn(f.x, iv.x), __fmul_rn(f.y, iv.y), __fmul_rn(f.z, iv.z), __fmul_rn(f.w, iv.w));
      }
    }
    const int c = q4 >> 3, fi = q4 & 7;
    xs4[(m * C + c) * 8 + (fi ^ (c & 7))] = f;
  }
  asm volatile("bar.sync 1, 256;" ::: "memory");  // the 8 consumer warps only
  for (int i = 0; i < nst; ++i) {
    const int s = i % stages;
    if (!mbar_wait(&full[s], (i / stages) & 1, abort)) break;
    const uint8_t* st = ring + s * stage_bytes;
    const __nv_bfloat16* st_sc = reinterpret_cast<const __nv_bfloat16*>(st + kAwqRingRows * (K / 2));
    const uint8_t* st_z = st + kAwqRingRows * (K / 2 + 2 * G);
    const int lr0 = warp * kAwqRows;                 // this warp's first row of the stage
    const int n0 = r0 + i * kAwqRingRows + lr0;
    float2 acc[kAwqRows][MT];
#pragma unroll
    for (int r = 0; r < kAwqRows; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m] = make_float2(0.0f, 0.0f);
    for (int c = lane; c < C; c += 32) {
      uint4 v[kAwqRows];
      float sv[kAwqRows], nz[kAwqRows];
#pragma unroll
      for (int r = 0; r < kAwqRows; ++r) {
        // rows past the CTA's run read the stage's stale bytes and are not stored
        v[r] = *reinterpret_cast<const uint4*>(st + (lr0 + r) * (K / 2) + 16 * c);
        sv[r] = __bfloat162float(st_sc[(lr0 + r) * G + (c >> 1)]);
        nz[r] = __uint_as_float(0xCB000000u | st_z[(lr0 + r) * G + (c >> 1)]);  // -(2^23 + z), exact
      }
      const int sw = c & 7;
      float2 t[kAwqRows][MT];
#pragma unroll
      for (int r = 0; r < kAwqRows; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) t[r][m] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) {
        float2 d[kAwqRows][4];
#pragma unroll
        for (int r = 0; r < kAwqRows; ++r) {
          const uint32_t word = wd == 0 ? v[r].x : (wd == 1 ? v[r].y : (wd == 2 ? v[r].z : v[r].w));
          const uint32_t lo = word & 0x0F0F0F0Fu, hi = (word >> 4) & 0x0F0F0F0Fu;
          const float2 nz2 = make_float2(nz[r], nz[r]);
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const float2 q = make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7650u + b)),
                                         __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7650u + b)));
            d[r][b] = __fadd2_rn(q, nz2);
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const float4* xc = xs4 + (m * C + c) * 8;
          const float4 a = xc[(2 * wd) ^ sw];
          const float4 e = xc[(2 * wd + 1) ^ sw];
          const float2 x01 = make_float2(a.x, a.y), x23 = make_float2(a.z, a.w);
          const float2 x45 = make_float2(e.x, e.y), x67 = make_float2(e.z, e.w);
#pragma unroll
          for (int r = 0; r < kAwqRows; ++r) {
            t[r][m] = __ffma2_rn(x01, d[r][0], t[r][m]);
            t[r][m] = __ffma2_rn(x23, d[r][1], t[r][m]);
            t[r][m] = __ffma2_rn(x45, d[r][2], t[r][m]);
            t[r][m] = __ffma2_rn(x67, d[r][3], t[r][m]);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < kAwqRows; ++r) {
        const float2 s2 = make_float2(sv[r], sv[r]);
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = __ffma2_rn(t[r][m], s2, acc[r][m]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);  // this warp is done with the stage
#pragma unroll
    for (int r = 0; r < kAwqRows; ++r) {
      const int n = n0 + r;
      float res[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        res[m] = __fadd_rn(acc[r][m].x, acc[r][m].y);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) res[m] += __shfl_xor_sync(0xffffffffu, res[m], o);
      }
      if (lane == 0 && n < r1) {
        const float bn = bias != nullptr ? __bfloat162float(bias[n]) : 0.0f;
#pragma unroll
        for (int m = 0; m < MT; ++m)
          if (m < rows) Y[static_cast<int64_t>(m) * ldy + n] = __float2bfloat16_rn(__fadd_rn(res[m], bn));
      }
    }
  }
}

}  // namespace svdq
