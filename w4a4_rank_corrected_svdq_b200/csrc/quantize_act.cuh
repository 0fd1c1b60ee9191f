// quantize_act.cuh — activation NVFP4 quantisation fused with the low-rank
// down projection XL1 = X . L1 (one read of X from HBM).
//
// Blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers", figure
// caption in "Background: SVDQuant and Nunchaku": the low-rank down
// projection is fused with the quantisation kernel, so the 16-bit branch adds
// no extra pass over the activations.
//
// A CTA owns ROWS (64 or 128) rows and a K-range; the KS K-ranges of one row
// block form a thread-block cluster. Roles (288 threads):
//  * warp 0      barrier setup and TMEM allocation; then lane 0 is both the
//                TMA producer (per 64-column step one X tile, ROWS rows x
//                128 B with 128-byte swizzle, and one L1^T tile, r rows x
//                128 B, into a ring of shared-memory stages) and the MMA issuer
//                (four 128 x r x 16 bf16 tcgen05 MMAs per step, XL1
//                accumulating in TMEM). With 64-row tiles the MMA still has
//                M = 128: its rows 64-127 read the bytes after the tile (the
//                ring is padded so they stay inside the allocation) and land in
//                TMEM lanes that are never read. The first stages are requested
//                before the CTA-wide sync so the setup hides under their
//                latency;
//  * warps 1-8   quantisers, several steps per iteration for independent work
//                in flight: each thread takes one row and ROWS/64 NVFP4 blocks
//                (16 columns each) of every step, read from the swizzled tile
//                with conflict-free 16-byte loads; per block one divide gives
//                the scale and a 127-entry table of correctly rounded
//                reciprocals (dec(S) g takes at most 127 values) gives 1/sd;
//                products are formed two at a time (packed fp32); code bytes go
//                out in one store per step and the scale bytes into staged
//                512-byte atoms written out after the K-range (a 64-row tile
//                owns half of every atom).
// XL1 reduction over the cluster (deterministic): CTA q finishes rows
// [q*ROWS/KS, (q+1)*ROWS/KS) of the tile. After one cluster barrier (every
// ring is drained), each CTA reads its TMEM partial row by row and sends it
// with asynchronous 16-byte stores into the owning CTA's shared memory
// (slot = source rank); the stores count their bytes on the owner's mbarrier,
// which was armed with the total at setup, so no thread waits for its own
// stores to land. The owner adds the KS slots in rank order. Every mbarrier
// wait is bounded (see mbar_wait).
#pragma once

#include "nvfp4.cuh"

namespace svdq {

constexpr int kQuantThreads = 288;
constexpr int kQuantWarps = 8;     // quantiser warps (1..8)
constexpr int kQuantStep = 64;     // columns per step (128 bytes of bf16)
constexpr int kQuantMaxStages = 8;

template <int R, int ROWS>
struct QuantCfg {
  static_assert(ROWS == 64 || ROWS == 128, "row tile");
  static constexpr int kXBytes = ROWS * 128;
  static constexpr int kLBytes = R * 128;                  // L1^T tile
  static constexpr int kStageBytes = kXBytes + kLBytes;
  static constexpr int kStages = ROWS == 128 ? ((R >= 128) ? 3 : (R >= 64 ? 4 : 5))
                                             : ((R >= 128) ? 4 : (R >= 64 ? 6 : 8));
  static constexpr int kTmemCols = R < 32 ? 32 : R;
  // MMA rows past a 64-row tile read up to 8 KB beyond the last stage.
  static constexpr int kRingBytes = kStages * kStageBytes + (ROWS == 64 ? 8192 : 0);
  // Partial-sum slots [KS][ROWS/KS rows][R] fp32 = ROWS x R x 4 bytes whatever
  // KS is; they alias the ring once every CTA of the cluster has drained it.
  static constexpr int kPartBytes = ROWS * R * 4;
  static constexpr int kBody = kRingBytes > kPartBytes ? kRingBytes : kPartBytes;
  // Smoothing factors of each step (64 floats), loaded with the step's tiles
  // into a ring of 2 x kStages slots: the slot of step st is rewritten only
  // with step st + 2 kStages, whose load waits for every quantiser warp to
  // release step st + kStages, which each does after quantising step st.
  static constexpr int kSmoothSlots = 2 * kStages;
  static constexpr int kSmoothBytes = kSmoothSlots * kQuantStep * 4;
  static constexpr int kSwzMask = (R / 4 < 8 ? R / 4 : 8) - 1;  // 16-byte chunk swizzle of a partial row
  static constexpr int kBpt = ROWS / 64;   // NVFP4 blocks per quantiser thread per step
  static constexpr int kTpr = 4 / kBpt;    // quantiser threads per row
  static constexpr int kBatch = 4 / kBpt;  // steps per quantiser iteration
  static_assert(kStages <= kQuantMaxStages, "barrier arrays");
  static_assert(kStages >= kBatch, "the smoothing ring needs a step's release to follow its quantisation");
};

struct QuantBarriers {
  uint64_t full[kQuantMaxStages];
  uint64_t empty[kQuantMaxStages];
  uint64_t acc_done;
  uint64_t xl1_in;   // every partial row for this CTA's output rows has arrived
  uint32_t tmem_base;
  int abort;
  float red[kQuantThreads / 32];  // per-warp maxima of the per-call activation scale
};
static_assert(sizeof(QuantBarriers) <= 256, "the barrier block of quantize_smem_bytes");

// Per-call (dynamic) activation scale, computed by every CTA of the quantiser
// from the amax pass's per-block maxima instead of read from g_x:
// g = fp32(amax / 2688) (1 for amax = 0), alpha' = fp32(g g_w). CTA 0 writes
// {g, g_w, alpha', amax} to gs_out, and the CTAs together re-express the
// packed hi/lo planes of L2^T / alpha for alpha' (reexpress_planes) while their
// first stages are in flight. partial == nullptr: the calibrated scale *g_x.
struct DynScale {
  const float* partial;         // [nparts] block maxima of |X^|
  int nparts;
  const float* gscale;          // the layer's {g_x, g_w, alpha, 0}
  float* gs_out;                // this call's {g, g_w, alpha', amax}
  const __nv_bfloat16* l2s;     // [2][total]: hi, lo planes for alpha
  __nv_bfloat16* l2s_out;       // [2][total]: for alpha'
  int64_t total;                // N r (a multiple of 16)
};

// Elements [8 i0, 8 i1) of the planes: v = hi + lo (exact in fp32),
// v' = fp32(v * ratio), hi' = bf16(v'), lo' = bf16(v' - hi'); copied
// unchanged when alpha' == alpha (same).
__device__ __forceinline__ void reexpress_planes(const DynScale& dyn, int64_t i0, int64_t i1, int64_t stride,
                                                 bool same, float ratio) {
  const uint4* hi8 = reinterpret_cast<const uint4*>(dyn.l2s);
  const uint4* lo8 = reinterpret_cast<const uint4*>(dyn.l2s + dyn.total);
  uint4* ohi8 = reinterpret_cast<uint4*>(dyn.l2s_out);
  uint4* olo8 = reinterpret_cast<uint4*>(dyn.l2s_out + dyn.total);
  for (int64_t i = i0; i < i1; i += stride) {
    const uint4 h = ldg_v4(hi8 + i), l = ldg_v4(lo8 + i);
    if (same) {
      ohi8[i] = h;
      olo8[i] = l;
      continue;
    }
    const uint32_t hw[4] = {h.x, h.y, h.z, h.w}, lw[4] = {l.x, l.y, l.z, l.w};
    uint32_t oh[4], ol[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float v0 = __fmul_rn(__fadd_rn(__uint_as_float(hw[j] << 16), __uint_as_float(lw[j] << 16)), ratio);
      const float v1 =
          __fmul_rn(__fadd_rn(__uint_as_float(hw[j] & 0xFFFF0000u), __uint_as_float(lw[j] & 0xFFFF0000u)), ratio);
      const __nv_bfloat162 hh = __floats2bfloat162_rn(v0, v1);
      const float h0 = __low2float(hh), h1 = __high2float(hh);
      const __nv_bfloat162 ll = __floats2bfloat162_rn(__fsub_rn(v0, h0), __fsub_rn(v1, h1));
      oh[j] = *reinterpret_cast<const uint32_t*>(&hh);
      ol[j] = *reinterpret_cast<const uint32_t*>(&ll);
    }
    ohi8[i] = make_uint4(oh[0], oh[1], oh[2], oh[3]);
    olo8[i] = make_uint4(ol[0], ol[1], ol[2], ol[3]);
  }
}

// Dynamic shared memory: stage ring (later XL1 partial slots), smoothing-factor
// ring, scale staging for the CTA's K-range, reciprocal table, barriers,
// alignment slack. (Both instantiations reserve the smoothing ring, so the
// launch plan does not depend on smoothing.)
template <int R, int ROWS>
__host__ __device__ constexpr size_t quantize_smem_bytes(int kchunk) {
  return static_cast<size_t>(QuantCfg<R, ROWS>::kBody) + QuantCfg<R, ROWS>::kSmoothBytes +
         static_cast<size_t>(kchunk / 64) * 512 + 512 + 256 + 1024;
}

// NB NVFP4 blocks (16 bf16 values = two 16-byte words each) -> 8 code bytes
// per block in c[2b], c[2b+1] and the scale bytes in sc (block b in byte b).
// Every step is one correctly rounded fp32 operation:
// x^ = x * inv_smooth[k] (when smoothing), S = e4m3(amax / (6 g)),
// q = x^ * (1 / fp32(dec(S) g)). sm: the blocks' 16 * NB smoothing factors
// (16-byte aligned, in shared memory), or nullptr.
template <int NB>
__device__ __forceinline__ void quantize_blocks(const uint4 (&v)[2 * NB], float d, const float* inv_tab,
                                                const float* __restrict__ sm, uint32_t (&c)[2 * NB], uint32_t& sc) {
  sc = 0;
#pragma unroll
  for (int blk = 0; blk < NB; ++blk) {
    float f[8], e[8];
    bf16x8_to_f32(v[2 * blk], f);
    bf16x8_to_f32(v[2 * blk + 1], e);
    if (sm != nullptr) {
      const float4* s4 = reinterpret_cast<const float4*>(sm + 16 * blk);
      const float4 a = s4[0], b = s4[1], cc = s4[2], dd = s4[3];
      const float fa[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      const float fe[8] = {cc.x, cc.y, cc.z, cc.w, dd.x, dd.y, dd.z, dd.w};
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        mul2x2_rn(f[i], f[i + 1], fa[i], fa[i + 1]);
        mul2x2_rn(e[i], e[i + 1], fe[i], fe[i + 1]);
      }
    }
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) am = fmaxf(am, fmaxf(fabsf(f[i]), fabsf(e[i])));
    const uint32_t s = f32_to_e4m3(__fdiv_rn(am, d));
    const float inv = inv_tab[s];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      mul2_rn(f[i], f[i + 1], inv);
      mul2_rn(e[i], e[i + 1], inv);
    }
    c[2 * blk] = f32x8_to_e2m1(f);
    c[2 * blk + 1] = f32x8_to_e2m1(e);
    sc |= s << (8 * blk);
  }
}

// SMOOTH: the 4-bit branch quantises x * inv_smooth[k] (smoothing); the plain
// instantiation ignores inv_smooth.
template <int R, int ROWS, bool SMOOTH>
__global__ void __launch_bounds__(kQuantThreads, 2) quantize_act_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l1t, int M, int K,
    const float* __restrict__ g_x, const float* __restrict__ inv_smooth, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales, __nv_bfloat16* __restrict__ xl1, int kchunk, const DynScale dyn) {
  using C = QuantCfg<R, ROWS>;
  constexpr int S = C::kStages;
  constexpr int BPT = C::kBpt;
  extern __shared__ uint8_t qsmem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qsmem_raw) + 1023) & ~uintptr_t(1023));
  float* sm_ring = reinterpret_cast<float*>(smem + C::kBody);
  uint8_t* sc_stage = smem + C::kBody + C::kSmoothBytes;
  float* inv_tab = reinterpret_cast<float*>(sc_stage + (kchunk / 64) * 512);
  QuantBarriers* bars = reinterpret_cast<QuantBarriers*>(inv_tab + 128);
  float* part = reinterpret_cast<float*>(smem);  // slots, valid after the cluster barrier

  const int KS = static_cast<int>(gridDim.x);  // the launch makes one cluster per row block
  const int ks = static_cast<int>(cluster_rank());
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * ROWS;
  const int k_begin = ks * kchunk;
  const int nsteps = kchunk / kQuantStep;
  const int rpc = ROWS / KS;  // output rows finished by each CTA of the cluster

  // The prologue reads only X, L1^T and the smoothing factors, which no kernel
  // of the layer writes; g_x may come from the kernel before this one (the
  // dynamic scale), so it is read after griddepcontrol.wait (a no-op unless
  // this grid was launched as a programmatic dependent).
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1 + kQuantWarps);  // MMA commit + quantiser warps
    }
    mbar_init(&bars->acc_done, 1);
    mbar_init(&bars->xl1_in, 1);
    bars->abort = 0;
    fence_barrier_init();
    // rpc rows of R fp32 from each of the KS CTAs = ROWS x R x 4 bytes
    mbar_arrive_expect_tx(&bars->xl1_in, C::kPartBytes);
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_l1t);
    for (int st = 0; st < S && st < nsteps; ++st) {
      uint8_t* dst = smem + st * C::kStageBytes;
      mbar_arrive_expect_tx(&bars->full[st], C::kStageBytes + (SMOOTH ? kQuantStep * 4 : 0));
      tma_load_2d(dst, &tm_x, k_begin + st * kQuantStep, m0, &bars->full[st]);
      tma_load_2d(dst + C::kXBytes, &tm_l1t, k_begin + st * kQuantStep, 0, &bars->full[st]);
      if (SMOOTH)
        bulk_load(sm_ring + (st % C::kSmoothSlots) * kQuantStep, inv_smooth + k_begin + st * kQuantStep,
                  kQuantStep * 4, &bars->full[st]);
    }
  }
  pdl_wait();
  float g;
  if (dyn.partial != nullptr) {
    // this call's scale from the amax pass's block maxima (the same maximum,
    // hence the same g, in every CTA)
    float am = 0.0f;
    for (int i = threadIdx.x; i < dyn.nparts; i += kQuantThreads) am = fmaxf(am, dyn.partial[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    if (lane == 0) bars->red[warp] = am;
    __syncthreads();
    am = bars->red[0];
#pragma unroll
    for (int w = 1; w < kQuantThreads / 32; ++w) am = fmaxf(am, bars->red[w]);
    g = (am == 0.0f) ? 1.0f : __fdiv_rn(am, kGlobalDivisor);
    const float gw = dyn.gscale[1], alpha = dyn.gscale[2];
    const float alpha_d = __fmul_rn(g, gw);
    const int cta = blockIdx.y * gridDim.x + blockIdx.x;
    if (cta == 0 && threadIdx.x == 0) {
      dyn.gs_out[0] = g;
      dyn.gs_out[1] = gw;
      dyn.gs_out[2] = alpha_d;
      dyn.gs_out[3] = am;
    }
    if (warp > 0) {  // the quantiser warps, while the first stages are in flight
      const int64_t vecs = dyn.total / 8, ncta = static_cast<int64_t>(gridDim.x) * gridDim.y;
      const int64_t per = (vecs + ncta - 1) / ncta;
      const int64_t i0 = cta * per, i1 = i0 + per < vecs ? i0 + per : vecs;
      reexpress_planes(dyn, i0 + threadIdx.x - 32, i1, kQuantThreads - 32, alpha_d == alpha,
                       __fdiv_rn(alpha, alpha_d));
    }
  } else {
    g = *g_x;
  }
  // The GEMM that consumes this kernel's output may be scheduled now: it
  // prepares its shared memory and TMEM, then waits for this grid to finish.
  pdl_launch_dependents();
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
  // Warps whose TMEM lane quarter (warp % 4) holds the tile's rows read XL1.
  const bool xl1_reader = warp >= 4 && warp < 4 + ROWS / 32;

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
          mbar_arrive_expect_tx(&bars->full[s], C::kStageBytes + (SMOOTH ? kQuantStep * 4 : 0));
          tma_load_2d(dst, &tm_x, k_begin + nx * kQuantStep, m0, &bars->full[s]);
          tma_load_2d(dst + C::kXBytes, &tm_l1t, k_begin + nx * kQuantStep, 0, &bars->full[s]);
          if (SMOOTH)
            bulk_load(sm_ring + (nx % C::kSmoothSlots) * kQuantStep, inv_smooth + k_begin + nx * kQuantStep,
                      kQuantStep * 4, &bars->full[s]);
        }
      }
      tc_commit(&bars->acc_done);
    }
  } else {
    // ------------------------------------------------------------ quantisers
    const int t = threadIdx.x - 32;
    const int rl = t / C::kTpr;            // local row
    const int b0 = (t % C::kTpr) * BPT;    // first NVFP4 block of the step
    const int r128 = (m0 & 127) + rl;      // row inside its 128-row scale atom
    const int row = m0 + rl;
    const bool valid = row < M;
    const float d = __fmul_rn(6.0f, g);
    uint8_t* cp = codes + static_cast<int64_t>(valid ? row : 0) * (K / 2) + k_begin / 2 + 8 * b0;
    uint8_t* sp = sc_stage + (r128 & 31) * 16 + (r128 >> 5) * 4 + b0;
    const int swz = rl & 7;
    auto load_stage = [&](int st, uint4 (&v)[2 * BPT]) -> bool {
      const int s = st % S;
      if (!mbar_wait(&bars->full[s], (st / S) & 1, abort)) return false;
      const uint8_t* tile = smem + s * C::kStageBytes + rl * 128;
#pragma unroll
      for (int j = 0; j < 2 * BPT; ++j) v[j] = *reinterpret_cast<const uint4*>(tile + (((2 * b0 + j) ^ swz) << 4));
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->empty[s]);  // this warp is done reading the stage
      return true;
    };
    auto emit = [&](int st, const uint4 (&v)[2 * BPT]) {
      uint32_t c[2 * BPT];
      uint32_t sc;
      quantize_blocks<BPT>(v, d, inv_tab, SMOOTH ? sm_ring + (st % C::kSmoothSlots) * kQuantStep + 16 * b0 : nullptr,
                           c, sc);
      if constexpr (BPT == 2) {
        if (valid) *reinterpret_cast<uint4*>(cp + st * (kQuantStep / 2)) = make_uint4(c[0], c[1], c[2], c[3]);
        *reinterpret_cast<uint16_t*>(sp + st * 512) = static_cast<uint16_t>(sc);
      } else {
        if (valid) *reinterpret_cast<uint2*>(cp + st * (kQuantStep / 2)) = make_uint2(c[0], c[1]);
        sp[st * 512] = static_cast<uint8_t>(sc);
      }
    };
    int st = 0;
    for (; st + C::kBatch <= nsteps; st += C::kBatch) {
      uint4 v[C::kBatch][2 * BPT];
      bool ok = true;
#pragma unroll
      for (int i = 0; i < C::kBatch; ++i) ok = ok && load_stage(st + i, v[i]);
      if (!ok) break;
#pragma unroll
      for (int i = 0; i < C::kBatch; ++i) emit(st + i, v[i]);
    }
    for (; st < nsteps; ++st) {
      uint4 v[2 * BPT];
      if (!load_stage(st, v)) break;
      emit(st, v);
    }
    if (xl1_reader) {  // XL1 is read from TMEM below: every MMA must have completed
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
  if (xl1_reader) {
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
    // Scale atoms of this K-range: whole 512-byte atoms, or this tile's half
    // (8 bytes of every 16-byte line) for a 64-row tile.
    uint8_t* dst = scales + (static_cast<size_t>(m0 / 128) * (K / 64) + k_begin / 64) * 512;
    if (ROWS == 128) {
      for (int i = threadIdx.x; i < nsteps * 32; i += kQuantThreads)
        reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(sc_stage)[i];
    } else {
      const int half = (m0 & 127) >> 6;
      // The last tile of an odd count also zeroes the padding half of its atoms.
      const bool pad_other = half == 0 && m0 + 64 >= M;
      for (int i = threadIdx.x; i < nsteps * 32; i += kQuantThreads) {
        const int off = (i >> 5) * 512 + (i & 31) * 16 + 8 * half;
        *reinterpret_cast<uint2*>(dst + off) = *reinterpret_cast<const uint2*>(sc_stage + off);
        if (pad_other) *reinterpret_cast<uint2*>(dst + off + 8) = make_uint2(0u, 0u);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
  // ---- this CTA's output rows: add the KS slots in rank order
  if (!mbar_wait_cluster(&bars->xl1_in, 0, abort)) {
    // Error path: the reduction is skipped, but partial rows that cluster peers
    // have already sent may still be landing in this CTA's shared memory; give
    // them a bounded time to arrive before the CTA exits.
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait_cluster(smem_u32(&bars->xl1_in), 0) && globaltimer() - t0 < 1000000ull) {
    }
    return;
  }
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
