// quantize_act.cuh — activation NVFP4 quantisation fused with the low-rank
// down projection XL1 = X . L1 (one read of X from HBM).
//
// Blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers", figure
// caption in "Background: SVDQuant and Nunchaku": the low-rank down
// projection is fused with the quantisation kernel, so the 16-bit branch adds
// no extra pass over the activations.
//
// A CTA owns 128 rows and a K-range; the KS K-ranges of one 128-row block form
// a thread-block cluster. Roles (288 threads; two CTAs fit an SM, so clusters
// of four still fill the GPU in one wave):
//  * warp 0      barrier setup and TMEM allocation; then lane 0 is both the
//                TMA producer (per 64-column step one X tile, 128 rows x 128 B
//                with 128-byte swizzle, and one L1^T tile, r rows x 128 B, into
//                a ring of shared-memory stages) and the MMA issuer (four
//                128 x r x 16 bf16 tcgen05 MMAs per step, XL1 accumulating in
//                TMEM). The first stages are requested before the CTA-wide
//                sync so the setup hides under their latency;
//  * warps 1-8   quantisers, two steps per iteration for independent work in
//                flight: thread t takes row t/2 and 32 columns (two NVFP4
//                blocks) of each step, read from the swizzled tile with
//                conflict-free 16-byte loads; per block one divide gives the
//                scale and a 127-entry table of correctly rounded reciprocals
//                (dec(S) g takes at most 127 values) gives 1/sd; products are
//                formed two at a time (packed fp32); 16 code bytes per thread
//                go out in one store and the scale bytes into staged 512-byte
//                atoms that are written once.
// XL1 reduction over the cluster (deterministic): CTA q finishes rows
// [q*128/KS, (q+1)*128/KS). After one cluster barrier (every ring is drained),
// each CTA reads its TMEM partial row by row and sends it with asynchronous
// 16-byte stores into the owning CTA's shared memory (slot = source rank);
// the stores count their bytes on the owner's mbarrier, which was armed with
// the total at setup, so no thread waits for its own stores to land. The owner
// adds the KS slots in rank order. Every mbarrier wait is bounded (see
// mbar_wait).
#pragma once

#include "nvfp4.cuh"

namespace svdq {

constexpr int kQuantThreads = 288;
constexpr int kQuantWarps = 8;     // quantiser warps (1..8)
constexpr int kQuantRows = 128;
constexpr int kQuantStep = 64;     // columns per step (128 bytes of bf16)

template <int R>
struct QuantCfg {
  static constexpr int kXBytes = kQuantRows * 128;        // 16 KB
  static constexpr int kLBytes = R * 128;                  // L1^T tile
  static constexpr int kStageBytes = kXBytes + kLBytes;
  static constexpr int kStages = (R >= 128) ? 3 : (R >= 64 ? 4 : 5);
  static constexpr int kTmemCols = R < 32 ? 32 : R;
  static constexpr int kRingBytes = kStages * kStageBytes;
  // Partial-sum slots [KS][128/KS rows][R] fp32 = 128 x R x 4 bytes whatever
  // KS is; they alias the ring once every CTA of the cluster has drained it.
  static constexpr int kPartBytes = kQuantRows * R * 4;
  static constexpr int kBody = kRingBytes > kPartBytes ? kRingBytes : kPartBytes;
  static constexpr int kSwzMask = (R / 4 < 8 ? R / 4 : 8) - 1;  // 16-byte chunk swizzle of a partial row
};

struct QuantBarriers {
  uint64_t full[5];
  uint64_t empty[5];
  uint64_t acc_done;
  uint64_t xl1_in;   // every partial row for this CTA's output rows has arrived
  uint32_t tmem_base;
  int abort;
};

// Dynamic shared memory: stage ring (later XL1 partial slots), scale staging
// for the CTA's K-range, reciprocal table, barriers, alignment slack.
template <int R>
__host__ __device__ constexpr size_t quantize_smem_bytes(int kchunk) {
  return static_cast<size_t>(QuantCfg<R>::kBody) + static_cast<size_t>(kchunk / 64) * 512 + 512 + 128 + 1024;
}

// Two NVFP4 blocks (32 bf16 values, four 16-byte words) -> 16 code bytes and
// the two scale bytes (low byte = first block). Every step is one correctly
// rounded fp32 operation: S = e4m3(amax / (6 g)), q = x * (1 / fp32(dec(S) g)).
__device__ __forceinline__ void quantize_32(const uint4 (&v)[4], float d, const float* inv_tab, uint4& codes,
                                            uint32_t& sc2) {
  uint32_t c[4];
  sc2 = 0;
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
    for (int i = 0; i < 8; i += 2) {
      mul2_rn(f[i], f[i + 1], inv);
      mul2_rn(e[i], e[i + 1], inv);
    }
    c[2 * blk] = f32x8_to_e2m1(f);
    c[2 * blk + 1] = f32x8_to_e2m1(e);
    sc2 |= sc << (8 * blk);
  }
  codes = make_uint4(c[0], c[1], c[2], c[3]);
}

template <int R>
__global__ void __launch_bounds__(kQuantThreads, 2) quantize_act_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l1t, int M, int K,
    const float* __restrict__ g_x, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
    __nv_bfloat16* __restrict__ xl1, int kchunk) {
  using C = QuantCfg<R>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t qsmem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qsmem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sc_stage = smem + C::kBody;
  float* inv_tab = reinterpret_cast<float*>(sc_stage + (kchunk / 64) * 512);
  QuantBarriers* bars = reinterpret_cast<QuantBarriers*>(inv_tab + 128);
  float* part = reinterpret_cast<float*>(smem);  // slots, valid after the cluster barrier

  const int KS = static_cast<int>(gridDim.x);  // the launch makes one cluster per row block
  const int ks = static_cast<int>(cluster_rank());
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * kQuantRows;
  const int k_begin = ks * kchunk;
  const int nsteps = kchunk / kQuantStep;
  const int rpc = kQuantRows / KS;  // output rows finished by each CTA of the cluster
  const float g = *g_x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1 + kQuantWarps);  // MMA commit + quantiser warps
    }
    mbar_init(&bars->acc_done, 1);
    mbar_init(&bars->xl1_in, 1);
    bars->abort = 0;
    fence_barrier_init();
    // rpc rows of R fp32 from each of the KS CTAs = 128 x R x 4 bytes
    mbar_arrive_expect_tx(&bars->xl1_in, C::kPartBytes);
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_l1t);
    for (int st = 0; st < S && st < nsteps; ++st) {
      uint8_t* dst = smem + st * C::kStageBytes;
      mbar_arrive_expect_tx(&bars->full[st], C::kStageBytes);
      tma_load_2d(dst, &tm_x, k_begin + st * kQuantStep, m0, &bars->full[st]);
      tma_load_2d(dst + C::kXBytes, &tm_l1t, k_begin + st * kQuantStep, 0, &bars->full[st]);
    }
  }
  if (warp == 0) {
    __syncwarp();
    tmem_alloc(&bars->tmem_base, C::kTmemCols);
    tmem_relinquish();
  } else if (threadIdx.x < 32 + 128) {  // reciprocal of every possible block decode scale
    const int code = threadIdx.x - 32;
    const float sd = __fmul_rn(e4m3_to_f32(code), g);
    inv_tab[code] = (sd == 0.0f || code >= 0x7F) ? 0.0f : __frcp_rn(sd);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  if (warp == 0) {
    // ------------------------------------------------- producer + XL1 MMA issuer
    if (lane == 0) {
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(R >> 3) << 17) | (uint32_t(128 >> 4) << 24);
      for (int st = 0; st < nsteps; ++st) {
        const int s = st % S;
        const uint32_t ph = (st / S) & 1;
        if (!mbar_wait(&bars->full[s], ph, abort)) break;
        tc_fence_after();
        const uint32_t a = smem_u32(smem + s * C::kStageBytes);
        const uint64_t adesc = smem_desc(a, 16, 1024, kSwizzle128B);
        const uint64_t bdesc = smem_desc(a + C::kXBytes, 16, 1024, kSwizzle128B);
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16)
          mma_bf16(tmem, adesc + 2 * k16, bdesc + 2 * k16, idesc, (st | k16) != 0 ? 1u : 0u);
        tc_commit(&bars->empty[s]);
        // Refill this stage with step st + S once the quantisers and the MMAs are done with it.
        const int nx = st + S;
        if (nx < nsteps) {
          if (!mbar_wait(&bars->empty[s], ph, abort)) break;
          uint8_t* dst = smem + s * C::kStageBytes;
          mbar_arrive_expect_tx(&bars->full[s], C::kStageBytes);
          tma_load_2d(dst, &tm_x, k_begin + nx * kQuantStep, m0, &bars->full[s]);
          tma_load_2d(dst + C::kXBytes, &tm_l1t, k_begin + nx * kQuantStep, 0, &bars->full[s]);
        }
      }
      tc_commit(&bars->acc_done);
    }
  } else {
    // ------------------------------------------------------------ quantisers
    const int t = threadIdx.x - 32;
    const int rl = t >> 1;     // local row
    const int h = t & 1;       // which 32 columns of the step
    const int row = m0 + rl;
    const bool valid = row < M;
    const float d = __fmul_rn(6.0f, g);
    uint8_t* cp = codes + static_cast<int64_t>(valid ? row : 0) * (K / 2) + k_begin / 2 + 16 * h;
    uint8_t* sp = sc_stage + (rl & 31) * 16 + (rl >> 5) * 4 + 2 * h;
    const int swz = rl & 7;
    auto load_stage = [&](int st, uint4 (&v)[4]) -> bool {
      const int s = st % S;
      if (!mbar_wait(&bars->full[s], (st / S) & 1, abort)) return false;
      const uint8_t* tile = smem + s * C::kStageBytes + rl * 128;
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = *reinterpret_cast<const uint4*>(tile + (((4 * h + j) ^ swz) << 4));
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->empty[s]);  // this warp is done reading the stage
      return true;
    };
    auto emit = [&](int st, const uint4 (&v)[4]) {
      uint4 c;
      uint32_t sc2;
      quantize_32(v, d, inv_tab, c, sc2);
      if (valid) *reinterpret_cast<uint4*>(cp + st * (kQuantStep / 2)) = c;
      *reinterpret_cast<uint16_t*>(sp + st * 512) = static_cast<uint16_t>(sc2);
    };
    int st = 0;
    for (; st + 1 < nsteps; st += 2) {
      uint4 v0[4], v1[4];
      if (!load_stage(st, v0) || !load_stage(st + 1, v1)) break;
      emit(st, v0);
      emit(st + 1, v1);
    }
    if (st + 1 == nsteps) {
      uint4 v0[4];
      if (load_stage(st, v0)) emit(st, v0);
    }
    if (warp <= 4) {  // warps 1-4 read XL1 from TMEM below: every MMA must have completed
      volatile int never = 0;
      mbar_wait(&bars->acc_done, 0, &never);
    }
  }

  // ---- every CTA of the cluster has drained its ring: partial slots may now be
  // written. Nothing written before this barrier is read through it (the ring's
  // reads and TMA writes have completed and the MMAs have committed), so the
  // arrive is relaxed; the barrier-init fence above publishes the mbarriers.
  __syncwarp();
  tc_fence_before();
  cluster_arrive_relaxed();
  cluster_wait();
  tc_fence_after();
  if (warp >= 1 && warp <= 4) {
    const int q = warp & 3;          // TMEM lane quarter this warp may read
    const int rloc = 32 * q + lane;  // local row held by this thread
    const int owner = rloc / rpc;
    const int orow = rloc - owner * rpc;
    const uint32_t slot = smem_u32(part) + static_cast<uint32_t>((ks * rpc + orow) * R * 4);
    const uint32_t remote = mapa_shared(slot, static_cast<uint32_t>(owner));
    const uint32_t remote_bar = mapa_shared(smem_u32(&bars->xl1_in), static_cast<uint32_t>(owner));
#pragma unroll
    for (int c0 = 0; c0 < R; c0 += 16) {
      uint32_t vv[16];
      tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(32 * q) << 16) + c0, vv);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int chunk = (c0 / 4 + j) ^ (orow & C::kSwzMask);
        st_async_v4(remote + chunk * 16, vv[4 * j], vv[4 * j + 1], vv[4 * j + 2], vv[4 * j + 3], remote_bar);
      }
    }
  }
  {
    uint8_t* dst = scales + (static_cast<size_t>(m0 / 128) * (K / 64) + k_begin / 64) * 512;
    for (int i = threadIdx.x; i < nsteps * 32; i += kQuantThreads)
      reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(sc_stage)[i];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
  // ---- this CTA's output rows: add the KS slots in rank order
  if (!mbar_wait_cluster(&bars->xl1_in, 0, abort)) return;
  constexpr int kChunks = R / 4;
  for (int i = threadIdx.x; i < rpc * kChunks; i += kQuantThreads) {
    const int orow = i / kChunks;
    const int ch = i % kChunks;
    const int pch = ch ^ (orow & C::kSwzMask);
    float4 acc = *reinterpret_cast<const float4*>(part + static_cast<size_t>(orow) * R + pch * 4);
    for (int p = 1; p < KS; ++p) {
      const float4 o = *reinterpret_cast<const float4*>(part + static_cast<size_t>(p * rpc + orow) * R + pch * 4);
      acc.x += o.x;
      acc.y += o.y;
      acc.z += o.z;
      acc.w += o.w;
    }
    const int grow = m0 + ks * rpc + orow;
    if (grow < M) {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t*>(&lo);
      pk.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(xl1 + static_cast<int64_t>(grow) * R + ch * 4) = pk;
    }
  }
}

}  // namespace svdq
