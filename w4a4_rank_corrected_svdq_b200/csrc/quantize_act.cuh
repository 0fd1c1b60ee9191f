// quantize_act.cuh — activation NVFP4 quantisation fused with the low-rank
// down projection XL1 = X . L1 (one read of X from HBM).
//
// Blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers", figure
// caption in "Background: SVDQuant and Nunchaku": the low-rank down
// projection is fused with the quantisation kernel, so the 16-bit branch adds
// no extra pass over the activations.
//
// A CTA owns 128 rows and a K-range; the K-ranges of one 128-row block form a
// thread-block cluster of KS CTAs whose partial XL1 sums are added in a fixed
// order through distributed shared memory (deterministic).
// Roles (320 threads):
//  * warp 0     TMA producer: per 64-column step one X tile (128 rows x 128 B,
//               128-byte swizzle) and one L1^T tile (r rows x 128 B) into a
//               ring of shared-memory stages;
//  * warp 1     TMEM owner; lane 0 issues four 128 x r x 16 bf16 tcgen05 MMAs
//               per step (XL1 accumulates in TMEM) and releases the stage;
//  * warps 2-9  quantisers: thread t takes row t/2, 32 columns (two NVFP4
//               blocks) of the step, read from the swizzled tile with
//               conflict-free 16-byte loads; per block one divide gives the
//               scale and a 127-entry table of correctly rounded reciprocals
//               (dec(S) g takes at most 127 values) gives 1/sd; 16 code bytes
//               per thread go out in one store, the scales are staged as whole
//               512-byte atoms and written once.
// After the K-range the quantisers move XL1 from TMEM to shared memory for the
// cluster reduction. Every wait is bounded (see mbar_wait).
#pragma once

#include <cooperative_groups.h>

#include "nvfp4.cuh"

namespace svdq {

constexpr int kQuantThreads = 320;
constexpr int kQuantRows = 128;
constexpr int kQuantStep = 64;  // columns per step (128 bytes of bf16)

template <int R>
struct QuantCfg {
  static constexpr int kXBytes = kQuantRows * 128;        // 16 KB
  static constexpr int kLBytes = R * 128;                  // L1^T tile
  static constexpr int kStageBytes = kXBytes + kLBytes;
  static constexpr int kStages = (R >= 128) ? 3 : 4;
  static constexpr int kTmemCols = R < 32 ? 32 : R;
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kPartBytes = kQuantRows * R * 4;   // aliases the ring after the loop
  static constexpr int kBody = kRingBytes > kPartBytes ? kRingBytes : kPartBytes;
};

struct QuantBarriers {
  uint64_t full[4];
  uint64_t empty[4];
  uint64_t acc_done;
  uint32_t tmem_base;
  int abort;
};

// Dynamic shared memory: stage ring (later XL1 partials), scale staging for
// the CTA's K-range, reciprocal table, barriers, alignment slack.
template <int R>
__host__ __device__ constexpr size_t quantize_smem_bytes(int kchunk) {
  return static_cast<size_t>(QuantCfg<R>::kBody) + static_cast<size_t>(kchunk / 64) * 512 + 512 + 128 + 1024;
}

template <int R>
__global__ void __launch_bounds__(kQuantThreads) quantize_act_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l1t, int M, int K,
    const float* __restrict__ g_x, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
    __nv_bfloat16* __restrict__ xl1, int kchunk) {
  namespace cg = cooperative_groups;
  using C = QuantCfg<R>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t qsmem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qsmem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sc_stage = smem + C::kBody;
  float* inv_tab = reinterpret_cast<float*>(sc_stage + (kchunk / 64) * 512);
  QuantBarriers* bars = reinterpret_cast<QuantBarriers*>(inv_tab + 128);
  float* part = reinterpret_cast<float*>(smem);  // [128][R], valid after the main loop

  cg::cluster_group cluster = cg::this_cluster();
  const int KS = static_cast<int>(cluster.num_blocks());
  const int ks = static_cast<int>(cluster.block_rank());
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * kQuantRows;
  const int k_begin = ks * kchunk;
  const int nsteps = kchunk / kQuantStep;
  const float g = *g_x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1 + 8);  // MMA commit + 8 quantiser warps
    }
    mbar_init(&bars->acc_done, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (threadIdx.x >= 64 && threadIdx.x < 64 + 128) {  // reciprocal of every possible block decode scale
    const int code = threadIdx.x - 64;
    const float sd = __fmul_rn(e4m3_to_f32(code), g);
    inv_tab[code] = (sd == 0.0f || code >= 0x7F) ? 0.0f : __frcp_rn(sd);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_l1t);
      uint32_t ph = 0;
      int s = 0;
      for (int st = 0; st < nsteps; ++st) {
        if (!mbar_wait(&bars->empty[s], ph ^ 1, abort)) break;
        uint8_t* dst = smem + s * C::kStageBytes;
        mbar_arrive_expect_tx(&bars->full[s], C::kStageBytes);
        tma_load_2d(dst, &tm_x, k_begin + st * kQuantStep, m0, &bars->full[s]);
        tma_load_2d(dst + C::kXBytes, &tm_l1t, k_begin + st * kQuantStep, 0, &bars->full[s]);
        if (++s == S) { s = 0; ph ^= 1; }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ XL1 MMAs
    if (lane == 0) {
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(R >> 3) << 17) | (uint32_t(128 >> 4) << 24);
      uint32_t ph = 0;
      int s = 0;
      for (int st = 0; st < nsteps; ++st) {
        if (!mbar_wait(&bars->full[s], ph, abort)) break;
        tc_fence_after();
        const uint32_t a = smem_u32(smem + s * C::kStageBytes);
        const uint64_t adesc = smem_desc(a, 16, 1024, kSwizzle128B);
        const uint64_t bdesc = smem_desc(a + C::kXBytes, 16, 1024, kSwizzle128B);
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16)
          mma_bf16(tmem, adesc + 2 * k16, bdesc + 2 * k16, idesc, (st | k16) != 0 ? 1u : 0u);
        tc_commit(&bars->empty[s]);
        if (++s == S) { s = 0; ph ^= 1; }
      }
      tc_commit(&bars->acc_done);
    }
  } else {
    // ------------------------------------------------------------ quantisers
    const int t = threadIdx.x - 64;
    const int rl = t >> 1;     // local row
    const int h = t & 1;       // which 32 columns of the step
    const int row = m0 + rl;
    const bool valid = row < M;
    const float d = __fmul_rn(6.0f, g);
    uint8_t* cp = codes + static_cast<int64_t>(valid ? row : 0) * (K / 2) + k_begin / 2 + 16 * h;
    uint32_t ph = 0;
    int s = 0;
    for (int st = 0; st < nsteps; ++st) {
      if (!mbar_wait(&bars->full[s], ph, abort)) break;
      const uint8_t* tile = smem + s * C::kStageBytes + rl * 128;
      uint4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = *reinterpret_cast<const uint4*>(tile + (((4 * h + j) ^ (rl & 7)) << 4));
      uint32_t word = 0;
      uint4 outc;
#pragma unroll
      for (int blk = 0; blk < 2; ++blk) {
        float f[8], e[8];
        bf16x8_to_f32(v[2 * blk], f);
        bf16x8_to_f32(v[2 * blk + 1], e);
        float am = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) am = fmaxf(am, fmaxf(fabsf(f[i]), fabsf(e[i])));
        const uint32_t sc = f32_to_e4m3(__fdiv_rn(am, d));
        const float inv = inv_tab[sc];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          f[i] = __fmul_rn(f[i], inv);
          e[i] = __fmul_rn(e[i], inv);
        }
        const uint32_t lo = f32x8_to_e2m1(f), hi = f32x8_to_e2m1(e);
        if (blk == 0) { outc.x = lo; outc.y = hi; } else { outc.z = lo; outc.w = hi; }
        word |= sc << (8 * (2 * h + blk));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->empty[s]);  // this warp is done reading the stage
      if (valid) *reinterpret_cast<uint4*>(cp + st * (kQuantStep / 2)) = outc;
      word |= __shfl_xor_sync(0xffffffffu, word, 1);
      if (h == 0) *reinterpret_cast<uint32_t*>(sc_stage + st * 512 + (rl & 31) * 16 + (rl >> 5) * 4) = word;
      if (++s == S) { s = 0; ph ^= 1; }
    }
  }

  // ---- all stages consumed: scale atoms out (coalesced), XL1 partial TMEM -> smem
  __syncthreads();
  {
    uint8_t* dst = scales + (static_cast<size_t>(m0 / 128) * (K / 64) + k_begin / 64) * 512;
    for (int i = threadIdx.x; i < nsteps * 32; i += kQuantThreads)
      reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(sc_stage)[i];
  }
  if (warp >= 2 && warp < 6) {
    volatile int never = 0;
    mbar_wait(&bars->acc_done, 0, &never);
    tc_fence_after();
    const int q = warp & 3;
    const int rloc = 32 * q + lane;
#pragma unroll
    for (int c0 = 0; c0 < R; c0 += 16) {
      uint32_t v[16];
      tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(32 * q) << 16) + c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) part[rloc * R + c0 + i] = __uint_as_float(v[i]);
    }
  }
  tc_fence_before();
  cluster.sync();
  // ---- fixed-order reduction over the cluster; CTA ks finishes rows [ks*rpc, (ks+1)*rpc)
  const int rpc = kQuantRows / KS;
  for (int i = threadIdx.x; i < rpc * R; i += kQuantThreads) {
    const int rr = ks * rpc + i / R;
    const int j = i % R;
    float sum = 0.0f;
    for (int p = 0; p < KS; ++p) {
      const float* peer = cluster.map_shared_rank(part, p);
      sum += peer[rr * R + j];
    }
    if (m0 + rr < M) xl1[static_cast<int64_t>(m0 + rr) * R + j] = __float2bfloat16_rn(sum);
  }
  cluster.sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace svdq
