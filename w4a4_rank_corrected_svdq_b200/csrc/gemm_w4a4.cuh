// gemm_w4a4.cuh — NVFP4 x NVFP4 block-scaled GEMM on the 5th-generation tensor
// cores (tcgen05, kind::mxf4nvf4, UE4M3 scales per 16 K-elements) with the
// low-rank up projection, the global scales and the bias fused in the epilogue:
//
//   Y[m,n] = bf16( alpha * ( sum_k (cX SX)(cR SR) + sum_j XL1[m,j] (hi + lo)[n,j] ) + b[n] )
//
// where alpha = g_x g_w and hi + lo = L2^T / alpha (two bf16 parts, packed at
// load time), so the low-rank term carries the up projection to ~2^-17.
//
// Blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers", figure
// caption in "Background: SVDQuant and Nunchaku": the low-rank up projection
// is fused with the 4-bit compute kernel, so the 16-bit branch costs no extra
// memory pass.
//
// Design (one CTA per SM, persistent over 128 x 128 output tiles):
//  * warp 0     TMA producer: E2M1 code tiles (128 rows x 128 bytes, 128-byte
//               swizzle) for A and B, their scale atoms (2 KB each, one bulk
//               copy: the tiled scale layout is exactly what the MMA wants), and
//               per tile the XL1, hi and lo tiles for the low-rank MMA.
//  * warp 1     TMEM owner and MMA issuer (one thread): per 256-wide K block it
//               moves the scales smem -> TMEM (tcgen05.cp) and issues four
//               128x128x64 block-scaled MMAs; per tile it then issues 2r/16
//               128x128x16 bf16 MMAs for XL1 . (hi + lo) into a separate
//               accumulator.
//  * warps 2-5  epilogue: TMEM -> registers, y = alpha * (acc + lr) + b,
//               bf16, global stores.
// TMEM (512 columns): two 4-bit accumulators [0,128) and [128,256) so the
// epilogue of one tile overlaps the main loop of the next, the low-rank
// accumulator [256,384) and the scale factors [384,416).
// Every wait is bounded (see mbar_wait); on a timeout the CTA records the
// error, stops issuing work, waits for its in-flight copies and MMAs, frees
// TMEM and returns.
#pragma once

#include "ptx.cuh"
#include "qkv_post.cuh"

namespace svdq {

constexpr int kGemmThreads = 192;
constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kBKBytes = 128;  // 256 E2M1 elements per K block

template <int R>
struct GemmCfg {
  static constexpr int kABytes = kBM * kBKBytes;
  static constexpr int kBBytes = kBN * kBKBytes;
  static constexpr int kSFBytes = 2048;  // 4 scale atoms of 512 bytes
  static constexpr int kStageBytes = kABytes + kBBytes + 2 * kSFBytes;
  static constexpr int kStages = (R == 128) ? 3 : (R == 64 ? 4 : 5);
  static constexpr int kLrAtomCols = R < 64 ? R : 64;  // bf16 columns per swizzle atom row
  static constexpr int kLrAtoms = R / kLrAtomCols;
  static constexpr int kLrRowBytes = kLrAtomCols * 2;
  static constexpr int kLrAtomBytes = 128 * kLrRowBytes;
  static constexpr int kLrTileBytes = kLrAtoms * kLrAtomBytes;  // 128 x R bf16
  static constexpr int kLrOff = kStages * kStageBytes;
  static constexpr int kBarOff = kLrOff + 3 * kLrTileBytes;  // XL1, hi, lo tiles
  static constexpr int kBarBytes = 256;
  static constexpr int kSmemBytes = kBarOff + kBarBytes + 1024;  // + alignment slack
  static constexpr SwizzleMode kLrSwizzle =
      kLrRowBytes == 128 ? kSwizzle128B : (kLrRowBytes == 64 ? kSwizzle64B : kSwizzle32B);
};

struct GemmBarriers {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t lr_full;
  uint64_t lr_empty;
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t teardown;
  uint32_t tmem_base;
  int abort;
};

template <int R, bool QKV>
__global__ void __launch_bounds__(kGemmThreads, 1) w4a4_gemm_kernel(
    const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
    const __grid_constant__ CUtensorMap tm_xl1, const __grid_constant__ CUtensorMap tm_l2s,
    const uint8_t* __restrict__ a_scales, const uint8_t* __restrict__ w_scales,
    const float* __restrict__ gscale, const __nv_bfloat16* __restrict__ bias, __nv_bfloat16* __restrict__ Y,
    int64_t ldy, int M, int N, int K, const QkvPost post) {
  using C = GemmCfg<R>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  GemmBarriers* bars = reinterpret_cast<GemmBarriers*>(smem + C::kBarOff);
  uint8_t* lr_x = smem + C::kLrOff;
  uint8_t* lr_hi = lr_x + C::kLrTileBytes;
  uint8_t* lr_lo = lr_hi + C::kLrTileBytes;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_mb = (M + kBM - 1) / kBM;
  const int num_nb = N / kBN;
  const int num_tiles = num_mb * num_nb;
  const int nk = K / 256;
  const int sf_atoms_per_row = K / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->lr_full, 1);
    mbar_init(&bars->lr_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->acc_full[b], 1);
      mbar_init(&bars->acc_empty[b], 128);
    }
    mbar_init(&bars->teardown, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_xl1);
    prefetch_tmap(&tm_l2s);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();  // the prologue above overlaps the previous kernel (programmatic dependent launch)
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      bool ok = true;
      uint32_t filled[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // loads issued per stage
      uint32_t lr_filled = 0;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        const int mb = tile % num_mb, nb = tile / num_mb;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&bars->empty[s], ph ^ 1, abort)) { ok = false; break; }
          uint8_t* st = smem + s * C::kStageBytes;
          mbar_arrive_expect_tx(&bars->full[s], C::kStageBytes);
          tma_load_2d(st, &tm_a, kb * kBKBytes, mb * kBM, &bars->full[s]);
          tma_load_2d(st + C::kABytes, &tm_b, kb * kBKBytes, nb * kBN, &bars->full[s]);
          bulk_load(st + C::kABytes + C::kBBytes,
                    a_scales + (static_cast<size_t>(mb) * sf_atoms_per_row + kb * 4) * 512, C::kSFBytes,
                    &bars->full[s]);
          bulk_load(st + C::kABytes + C::kBBytes + C::kSFBytes,
                    w_scales + (static_cast<size_t>(nb) * sf_atoms_per_row + kb * 4) * 512, C::kSFBytes,
                    &bars->full[s]);
          ++filled[s];
          if (++s == S) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        if (!mbar_wait(&bars->lr_empty, (it & 1) ^ 1, abort)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars->lr_full, 3 * C::kLrTileBytes);
        for (int a = 0; a < C::kLrAtoms; ++a) {
          tma_load_2d(lr_x + a * C::kLrAtomBytes, &tm_xl1, a * 64, mb * kBM, &bars->lr_full);
          tma_load_2d(lr_hi + a * C::kLrAtomBytes, &tm_l2s, a * 64, nb * kBN, &bars->lr_full);
          tma_load_2d(lr_lo + a * C::kLrAtomBytes, &tm_l2s, a * 64, N + nb * kBN, &bars->lr_full);
        }
        ++lr_filled;
      }
      if (!ok) {
        // give the copies still in flight time to land before the CTA exits
        volatile int never = 0;
        for (int i = 0; i < S; ++i)
          if (filled[i] > 0) mbar_wait(&bars->full[i], (filled[i] - 1) & 1, &never);
        if (lr_filled > 0) mbar_wait(&bars->lr_full, (lr_filled - 1) & 1, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_fp4 = (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
      const uint32_t idesc_bf16 =
          (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
      const uint32_t t_lr = tmem + 256;
      const uint32_t t_sfa = tmem + 384;
      const uint32_t t_sfb = tmem + 400;
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        const int b = it & 1;
        const uint32_t t_acc = tmem + b * kBN;
        if (!mbar_wait(&bars->acc_empty[b], ((it >> 1) & 1) ^ 1, abort)) { ok = false; break; }
        tc_fence_after();
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&bars->full[s], ph, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * C::kStageBytes);
          const uint32_t sfa = st + C::kABytes + C::kBBytes;
          const uint32_t sfb = sfa + C::kSFBytes;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tmem_cp_32x128b_x4(t_sfa + 4 * j, smem_desc(sfa + 512 * j, 0, 128, kSwizzleNone));
            tmem_cp_32x128b_x4(t_sfb + 4 * j, smem_desc(sfb + 512 * j, 0, 128, kSwizzleNone));
          }
          const uint64_t adesc = smem_desc(st, 16, 1024, kSwizzle128B);
          const uint64_t bdesc = smem_desc(st + C::kABytes, 16, 1024, kSwizzle128B);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_nvf4(t_acc, adesc + 2 * j, bdesc + 2 * j, idesc_fp4, t_sfa + 4 * j, t_sfb + 4 * j,
                     (kb | j) != 0 ? 1u : 0u);
          tc_commit(&bars->empty[s]);
          if (++s == S) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        // low-rank up projection into its own accumulator
        if (!mbar_wait(&bars->lr_full, it & 1, abort)) { ok = false; break; }
        if (it > 0 && !mbar_wait(&bars->acc_empty[b ^ 1], ((it - 1) >> 1) & 1, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sx = smem_u32(lr_x), shi = smem_u32(lr_hi), slo = smem_u32(lr_lo);
        constexpr int kStepsPerAtom = C::kLrAtomCols / 16;
#pragma unroll
        for (int j = 0; j < R / 16; ++j) {
          const uint32_t off = (j / kStepsPerAtom) * C::kLrAtomBytes + (j % kStepsPerAtom) * 32;
          const uint64_t xdesc = smem_desc(sx + off, 16, 8 * C::kLrRowBytes, C::kLrSwizzle);
          mma_bf16(t_lr, xdesc, smem_desc(shi + off, 16, 8 * C::kLrRowBytes, C::kLrSwizzle), idesc_bf16,
                   j != 0 ? 1u : 0u);
          mma_bf16(t_lr, xdesc, smem_desc(slo + off, 16, 8 * C::kLrRowBytes, C::kLrSwizzle), idesc_bf16, 1u);
        }
        tc_commit(&bars->lr_empty);
        tc_commit(&bars->acc_full[b]);
      }
      // all MMAs issued by this thread complete before TMEM is released
      tc_commit(&bars->teardown);
      volatile int never = 0;
      mbar_wait(&bars->teardown, 0, &never);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const float alpha = gscale[2];
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int mb = tile % num_mb, nb = tile / num_mb;
      const int b = it & 1;
      if (!mbar_wait(&bars->acc_full[b], (it >> 1) & 1, abort)) break;
      tc_fence_after();
      const int row = mb * kBM + 32 * q + lane;
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
      if constexpr (QKV) {
        // The tile is one 128-column head of Q, K or V: gather the row, then
        // normalise and rotate Q / K rows before storing.
        const int n_tile = nb * kBN;
        const int seg = n_tile / post.hd;
        const __nv_bfloat16* w = seg == 0 ? post.w_q : (seg == 1 ? post.w_k : nullptr);
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t va[32], vl[32];
          tmem_ld_32x32b_x32(lane_base + b * kBN + 32 * c, va);
          tmem_ld_32x32b_x32(lane_base + 256 + 32 * c, vl);
          tmem_ld_wait();
          uint32_t bw[16];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 u = bias != nullptr ? ldg_v4(bias + n_tile + 32 * c + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
            bw[4 * v] = u.x;
            bw[4 * v + 1] = u.y;
            bw[4 * v + 2] = u.z;
            bw[4 * v + 3] = u.w;
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float s0 = __fadd_rn(__uint_as_float(va[2 * i]), __uint_as_float(vl[2 * i]));
            const float s1 = __fadd_rn(__uint_as_float(va[2 * i + 1]), __uint_as_float(vl[2 * i + 1]));
            pk[16 * c + i] = pack_bf16(__fmaf_rn(s0, alpha, bf16_lo(bw[i])), __fmaf_rn(s1, alpha, bf16_hi(bw[i])));
          }
        }
        if (w != nullptr) {
          const int64_t rr = row < M ? row : M - 1;
          qk_norm_rope_row(pk, w, post.cos + rr * post.ld_rope, post.sin + rr * post.ld_rope, post.eps);
        }
        if (row < M) {
          uint4* dst = reinterpret_cast<uint4*>(Y + static_cast<int64_t>(row) * ldy + n_tile);
#pragma unroll
          for (int v = 0; v < 16; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t va[32], vl[32];
          tmem_ld_32x32b_x32(lane_base + b * kBN + 32 * c, va);
          tmem_ld_32x32b_x32(lane_base + 256 + 32 * c, vl);
          tmem_ld_wait();
          const int n0 = nb * kBN + 32 * c;
          float bf[32];
          if (bias != nullptr) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint4 u = ldg_v4(bias + n0 + 8 * v);
              const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                bf[8 * v + 2 * i] = __uint_as_float(w4[i] << 16);
                bf[8 * v + 2 * i + 1] = __uint_as_float(w4[i] & 0xFFFF0000u);
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) bf[i] = 0.0f;
          }
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float s0 = __fadd_rn(__uint_as_float(va[2 * i]), __uint_as_float(vl[2 * i]));
            const float s1 = __fadd_rn(__uint_as_float(va[2 * i + 1]), __uint_as_float(vl[2 * i + 1]));
            const float y0 = __fmaf_rn(s0, alpha, bf[2 * i]);
            const float y1 = __fmaf_rn(s1, alpha, bf[2 * i + 1]);
            const __nv_bfloat162 h = __floats2bfloat162_rn(y0, y1);
            packed[i] = *reinterpret_cast<const uint32_t*>(&h);
          }
          if (row < M) {
            uint4* dst = reinterpret_cast<uint4*>(Y + static_cast<int64_t>(row) * ldy + n0);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace svdq
