// gemm_w4a4_splitk.cuh — the NVFP4 block-scaled GEMM of the SVDQuant W4A4 layer
// for few rows (small M), with K split across a thread-block cluster:
//
//   Y[m,n] = bf16( alpha * ( sum_k (cX SX)(cR SR) + sum_j XL1[m,j] (hi + lo)[n,j] ) + b[n] )
//
// (alpha = g_x g_w, hi + lo = L2^T / alpha; blog "Bringing Nunchaku 4-bit
// Diffusion Inference to Diffusers", figure caption in "Background: SVDQuant
// and Nunchaku": the up projection is fused with the 4-bit compute kernel).
//
// With few rows there are few 128 x 128 output tiles (a 128-token layer with
// N = 4096 has 32), so one CTA per tile would leave most SMs idle and each
// would stream the whole of K alone. Here a cluster of KS CTAs owns a tile and
// CTA ks takes K blocks [ks nk / KS, (ks + 1) nk / KS):
//  * warp 0     TMA producer: A and B code tiles (128 rows x 128 bytes,
//               128-byte swizzle) and the two 2 KB scale blocks per 256-deep K
//               block; CTA 0 also loads the low-rank tiles (XL1, hi, lo).
//  * warp 1     TMEM owner and MMA issuer: tcgen05.cp of the scale atoms, four
//               128x128x64 block-scaled MMAs per K block into one fp32
//               accumulator; CTA 0 adds XL1 . (hi + lo) into the same
//               accumulator with bf16 MMAs.
//  * warps 2-5  epilogue: after a cluster barrier (every CTA's ring is drained),
//               each thread reads its row of the partial accumulator from TMEM
//               and sends column slab o (128 / KS columns) to CTA o with
//               asynchronous 16-byte stores into CTA o's shared memory (slot =
//               source rank), counted on CTA o's mbarrier. CTA o then adds the
//               KS partials of its slab in rank order (deterministic), applies
//               alpha and the bias and stores bf16.
// TMEM: accumulator [0, 128), scale factors [128, 160) (256 columns).
// Every mbarrier wait is bounded (see mbar_wait).
#pragma once

#include "gemm_w4a4.cuh"

namespace svdq {

constexpr int kSplitThreads = 192;
constexpr int kSplitMaxKS = 8;

template <int R>
struct SplitCfg {
  static constexpr int kABytes = kBM * kBKBytes;
  static constexpr int kBBytes = kBN * kBKBytes;
  static constexpr int kSFBytes = 2048;
  static constexpr int kStageBytes = kABytes + kBBytes + 2 * kSFBytes;  // 36 KB
  static constexpr int kStages = R == 128 ? 3 : 4;  // the rank-128 low-rank tiles take 96 KB
  static constexpr int kLrAtomCols = R < 64 ? R : 64;
  static constexpr int kLrAtoms = R / kLrAtomCols;
  static constexpr int kLrRowBytes = kLrAtomCols * 2;
  static constexpr int kLrAtomBytes = 128 * kLrRowBytes;
  static constexpr int kLrTileBytes = kLrAtoms * kLrAtomBytes;  // 128 x R bf16
  static constexpr int kLrOff = kStages * kStageBytes;
  // partial slots [KS][128 rows][128 / KS fp32] = 64 KB for any KS; they alias
  // the stage ring once every CTA of the cluster has drained it
  static constexpr int kRecvBytes = 128 * 128 * 4;
  static_assert(kRecvBytes <= kLrOff, "partials alias the ring");
  static constexpr int kBarOff = kLrOff + 3 * kLrTileBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;
  static constexpr SwizzleMode kLrSwizzle =
      kLrRowBytes == 128 ? kSwizzle128B : (kLrRowBytes == 64 ? kSwizzle64B : kSwizzle32B);
};

struct SplitBarriers {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t lr_full;
  uint64_t acc_full;
  uint64_t recv;      // every partial of this CTA's column slab has arrived
  uint64_t teardown;
  uint32_t tmem_base;
  int abort;
};

template <int R>
__global__ void __launch_bounds__(kSplitThreads, 1) w4a4_gemm_splitk_kernel(
    const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
    const __grid_constant__ CUtensorMap tm_xl1, const __grid_constant__ CUtensorMap tm_l2s,
    const uint8_t* __restrict__ a_scales, const uint8_t* __restrict__ w_scales, const float* __restrict__ gscale,
    const __nv_bfloat16* __restrict__ bias, __nv_bfloat16* __restrict__ Y, int64_t ldy, int M, int N, int K) {
  using C = SplitCfg<R>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SplitBarriers* bars = reinterpret_cast<SplitBarriers*>(smem + C::kBarOff);
  uint8_t* lr_x = smem + C::kLrOff;
  uint8_t* lr_hi = lr_x + C::kLrTileBytes;
  uint8_t* lr_lo = lr_hi + C::kLrTileBytes;
  float* recv = reinterpret_cast<float*>(smem);  // valid after the cluster barrier

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int KS = static_cast<int>(gridDim.x);   // one cluster per tile
  const int ks = static_cast<int>(cluster_rank());
  const int num_mb = (M + kBM - 1) / kBM;
  const int tile = static_cast<int>(blockIdx.y);
  const int mb = tile % num_mb, nb = tile / num_mb;
  const int nk = K / 256;
  const int kb0 = ks * (nk / KS), kb1 = kb0 + nk / KS;
  const int sf_atoms_per_row = K / 64;
  const int W = kBN / KS;  // columns of each CTA's output slab
  const bool lr = ks == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->lr_full, 1);
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->recv, 1);
    mbar_init(&bars->teardown, 1);
    bars->abort = 0;
    fence_barrier_init();
    // KS partials of 128 rows x W fp32 = 64 KB arrive as st.async bytes
    mbar_arrive_expect_tx(&bars->recv, C::kRecvBytes);
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    if (lr) {
      prefetch_tmap(&tm_xl1);
      prefetch_tmap(&tm_l2s);
    }
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  // every CTA's barriers are initialised before any peer sends to them
  cluster_sync_all();
  tc_fence_after();
  pdl_wait();  // the prologue above overlaps the previous kernel (programmatic dependent launch)
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      if (lr) {  // the low-rank tiles have their own buffers: requested first
        mbar_arrive_expect_tx(&bars->lr_full, 3 * C::kLrTileBytes);
        for (int a = 0; a < C::kLrAtoms; ++a) {
          tma_load_2d(lr_x + a * C::kLrAtomBytes, &tm_xl1, a * 64, mb * kBM, &bars->lr_full);
          tma_load_2d(lr_hi + a * C::kLrAtomBytes, &tm_l2s, a * 64, nb * kBN, &bars->lr_full);
          tma_load_2d(lr_lo + a * C::kLrAtomBytes, &tm_l2s, a * 64, N + nb * kBN, &bars->lr_full);
        }
      }
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&bars->empty[s], ph ^ 1, abort)) { ok = false; break; }
        uint8_t* st = smem + s * C::kStageBytes;
        mbar_arrive_expect_tx(&bars->full[s], C::kStageBytes);
        tma_load_2d(st, &tm_a, kb * kBKBytes, mb * kBM, &bars->full[s]);
        tma_load_2d(st + C::kABytes, &tm_b, kb * kBKBytes, nb * kBN, &bars->full[s]);
        bulk_load(st + C::kABytes + C::kBBytes, a_scales + (static_cast<size_t>(mb) * sf_atoms_per_row + kb * 4) * 512,
                  C::kSFBytes, &bars->full[s]);
        bulk_load(st + C::kABytes + C::kBBytes + C::kSFBytes,
                  w_scales + (static_cast<size_t>(nb) * sf_atoms_per_row + kb * 4) * 512, C::kSFBytes,
                  &bars->full[s]);
        if (++s == S) { s = 0; ph ^= 1; }
      }
      if (!ok) {  // error path: give copies that may still be in flight time to land
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 2000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_fp4 = (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
      const uint32_t idesc_bf16 =
          (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
      const uint32_t t_sfa = tmem + 128;
      const uint32_t t_sfb = tmem + 144;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
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
          mma_nvf4(tmem, adesc + 2 * j, bdesc + 2 * j, idesc_fp4, t_sfa + 4 * j, t_sfb + 4 * j,
                   (kb != kb0 || j != 0) ? 1u : 0u);
        tc_commit(&bars->empty[s]);
        if (++s == S) { s = 0; ph ^= 1; }
      }
      if (ok && lr) {  // the low-rank up projection into the same accumulator
        if (mbar_wait(&bars->lr_full, 0, abort)) {
          tc_fence_after();
          const uint32_t sx = smem_u32(lr_x), shi = smem_u32(lr_hi), slo = smem_u32(lr_lo);
          constexpr int kStepsPerAtom = C::kLrAtomCols / 16;
#pragma unroll
          for (int j = 0; j < R / 16; ++j) {
            const uint32_t off = (j / kStepsPerAtom) * C::kLrAtomBytes + (j % kStepsPerAtom) * 32;
            const uint64_t xdesc = smem_desc(sx + off, 16, 8 * C::kLrRowBytes, C::kLrSwizzle);
            mma_bf16(tmem, xdesc, smem_desc(shi + off, 16, 8 * C::kLrRowBytes, C::kLrSwizzle), idesc_bf16, 1u);
            mma_bf16(tmem, xdesc, smem_desc(slo + off, 16, 8 * C::kLrRowBytes, C::kLrSwizzle), idesc_bf16, 1u);
          }
        }
      }
      tc_commit(&bars->acc_full);
      // all MMAs issued by this thread complete before TMEM is released
      tc_commit(&bars->teardown);
      volatile int never = 0;
      mbar_wait(&bars->teardown, 0, &never);
    }
  } else {
    // ------------------------------------------------------------ epilogue part 1: wait for the partial
    mbar_wait(&bars->acc_full, 0, abort);
    tc_fence_after();
  }

  // ---- every CTA of the cluster has drained its ring and finished its MMAs:
  // partial slots may now be written into any CTA's ring. (The arrive is
  // relaxed: nothing written before the barrier is read through it.)
  __syncwarp();
  tc_fence_before();
  cluster_arrive_relaxed();
  cluster_wait();
  tc_fence_after();

  if (warp >= 2) {
    const int q = warp & 3;      // TMEM lane quadrant
    const int rloc = 32 * q + lane;  // this thread's row of the tile
    const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * q) << 16);
    const int chunks = W / 4;    // 16-byte chunks of a slab row
    const int swz = chunks < 8 ? chunks - 1 : 7;
    // send column slab o of this row to CTA o (slot ks), 16 bytes at a time
#pragma unroll 1
    for (int c0 = 0; c0 < kBN; c0 += 32) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(taddr + c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int col = c0 + 4 * j;
        const int o = col / W, ch = (col % W) / 4;
        const uint32_t slot = smem_u32(recv) + static_cast<uint32_t>(((ks * 128 + rloc) * W + 4 * (ch ^ (rloc & swz))) * 4);
        st_async_v4(mapa_shared(slot, static_cast<uint32_t>(o)), v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3],
                    mapa_shared(smem_u32(&bars->recv), static_cast<uint32_t>(o)));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  if (warp >= 2) {
    // ------------------------------------------------------------ epilogue part 2: this CTA's slab
    const int q = warp & 3;
    const int rloc = 32 * q + lane;
    const int row = mb * kBM + rloc;
    const int chunks = W / 4;
    const int swz = chunks < 8 ? chunks - 1 : 7;
    if (!mbar_wait_cluster(&bars->recv, 0, abort)) {
      // error path: partials already sent may still be landing here
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait_cluster(smem_u32(&bars->recv), 0) && globaltimer() - t0 < 1000000ull) {
      }
      return;
    }
    const float alpha = gscale[2];
    const int n0 = nb * kBN + ks * W;
#pragma unroll 1
    for (int ch = 0; ch < chunks; ch += 2) {  // 8 columns per step: one 16-byte bf16 store
      float a[8];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int pc = (ch + u) ^ (rloc & swz);
        float4 acc = *reinterpret_cast<const float4*>(recv + (static_cast<size_t>(rloc)) * W + 4 * pc);
        for (int p = 1; p < KS; ++p) {
          const float4 o = *reinterpret_cast<const float4*>(recv + static_cast<size_t>(p * 128 + rloc) * W + 4 * pc);
          acc.x = __fadd_rn(acc.x, o.x);
          acc.y = __fadd_rn(acc.y, o.y);
          acc.z = __fadd_rn(acc.z, o.z);
          acc.w = __fadd_rn(acc.w, o.w);
        }
        a[4 * u] = acc.x;
        a[4 * u + 1] = acc.y;
        a[4 * u + 2] = acc.z;
        a[4 * u + 3] = acc.w;
      }
      const int n = n0 + 4 * ch;
      uint4 bv = make_uint4(0u, 0u, 0u, 0u);
      if (bias != nullptr) bv = ldg_v4(bias + n);
      const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
      uint32_t pk[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float y0 = __fmaf_rn(a[2 * i], alpha, __uint_as_float(bw[i] << 16));
        const float y1 = __fmaf_rn(a[2 * i + 1], alpha, __uint_as_float(bw[i] & 0xFFFF0000u));
        const __nv_bfloat162 h = __floats2bfloat162_rn(y0, y1);
        pk[i] = *reinterpret_cast<const uint32_t*>(&h);
      }
      if (row < M)
        *reinterpret_cast<uint4*>(Y + static_cast<int64_t>(row) * ldy + n) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
}

}  // namespace svdq
