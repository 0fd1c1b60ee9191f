// gemm_w4a4_2sm.cuh — the block-scaled NVFP4 GEMM of the SVDQuant W4A4 layer on
// CTA pairs (tcgen05 cta_group::2), 256 x 256 output tiles:
//
//   Y[m,n] = bf16( alpha * ( sum_k (cX SX)(cR SR) + sum_j XL1[m,j] (hi + lo)[n,j] ) + b[n] )
//
// with alpha = g_x g_w and hi + lo = L2^T / alpha (packed at load time), so the
// 4-bit product and the low-rank up projection share one fp32 accumulator
// (blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers", figure
// caption in "Background: SVDQuant and Nunchaku": the up projection is fused
// with the 4-bit compute kernel).
//
// A cluster of two CTAs on two SMs owns a 256 x 256 tile. Each CTA loads its
// own 128 rows of A and its own 128 rows of B; one thread of the even CTA issues
// 256x256xK MMAs that read both CTAs' shared memory and write each CTA's
// 128 x 256 half of the accumulator into that CTA's TMEM. No load uses cluster
// multicast: each CTA fetches every byte it stores.
//
// Tile order: the tiles are numbered M-block-major (N fastest) and each CTA
// pair takes one contiguous run of them, so consecutive tiles of a pair mostly
// share their 128-row A block. The A block's scale factors are then copied
// into TMEM once per run of tiles with the same A block (when all of K fits:
// K <= 14 x 256) and stay there: per 256-deep K block only the weight scales
// (SFB) are copied, four tcgen05.cp of 128x256b instead of six.
//
// Stages (one 256-deep K block each): the plain layer with resident A scales
// runs four 48 KB stages (A, B, SFB), its A scales loaded through a two-slot
// ring of their own and its epilogue staged 32 x 32 per warp (2 KB). The
// fused epilogues, and K too long for resident A scales, run three 56 KB
// stages that carry the A scales too. The fourth stage covers the load delay
// the epilogue's burst of Y stores causes at every tile start.
//
// Roles (320 threads per CTA):
//  * warp 0     TMA producer (both CTAs): per tile K/256 stages of E2M1
//               codes (128-byte swizzle) and UE4M3 scale atoms (SFA only when
//               the tile starts a new A block), then r/c low-rank stages (XL1
//               columns, hi and lo columns of l2s; c = min(r, 32)). The small
//               low-rank stages come last: when the ring refills at a tile
//               boundary its first stages are then full K blocks, whose MMAs
//               cover the load latency of the next ones.
//               Completion bytes of both CTAs land on the even CTA's barrier
//               (cp.async.bulk.tensor .cta_group::2).
//  * warp 1     TMEM owner (both CTAs, 512 columns); in the even CTA lane 0
//               issues the MMAs and the scale copies smem -> TMEM.
//  * warps 2-9  epilogue (both CTAs): two warps per 32-lane TMEM quadrant, one
//               per 128-column half. Each warp first drains its whole
//               32 x 128 share of the accumulator into registers and releases
//               it, so the next tile's MMAs start at once; then y = alpha acc + b
//               (bias staged in shared memory per tile), bf16, TMA stores. The
//               epilogue mode EPI selects the plain layer (0), the fused QKV
//               post-processing (1: per-head RMSNorm of Q/K and the rotary
//               embedding; the two warps of a quadrant then split a tile by
//               chunks) or the MLP up projection (2: GELU and the down
//               projection's NVFP4 codes, scales and XL1 partials instead of y).
// TMEM (512 columns): accumulator [0, 256), weight scales of the current K
// block [256, 288), A scales [288, 512) in 14 slots of 16 columns, one per K
// block. Every wait is bounded; see mbar_wait.
#pragma once

#include "ptx.cuh"
#include "nvfp4.cuh"
#include "qkv_post.cuh"

namespace svdq {

// ------------------------------------------------------------------ cluster / 2-SM PTX
// 2-D tiled load into this CTA's shared memory; the completion bytes are counted
// on the barrier at `bar_cluster` (the even CTA's barrier).
__device__ __forceinline__ void tma_load_2d_cg2(void* dst, const CUtensorMap* m, int x, int y, uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}
// 4-D / 5-D tiled loads with .cta_group::2 completion (used for the scale
// factors, whose tensor maps repeat each 512-byte atom four times through a
// zero-stride dimension, producing the replicated layout TMEM needs).
__device__ __forceinline__ void tma_load_4d_cg2(void* dst, const CUtensorMap* m, int c0, int c1, int c2, int c3,
                                                uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
      "%4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void tma_load_5d_cg2(void* dst, const CUtensorMap* m, int c0, int c1, int c2, int c3, int c4,
                                                uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.5d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
      "%4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void tmem_cp_128x256b_cg2(uint32_t taddr, uint64_t s_desc) {
  asm volatile("tcgen05.cp.cta_group::2.128x256b [%0], %1;" ::"r"(taddr), "l"(s_desc) : "memory");
}
__device__ __forceinline__ void tmem_alloc_cg2(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_cg2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_cg2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma_nvf4_cg2(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
__device__ __forceinline__ void mma_bf16_cg2(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives on the barrier at this shared-memory offset in every CTA of `mask`
// once all prior tcgen05 operations of this thread have completed.
__device__ __forceinline__ void tc_commit_cg2_mc(uint64_t* bar, uint16_t mask) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "h"(mask)
               : "memory");
}

// ------------------------------------------------------------------ configuration
constexpr int k2Threads = 320;
constexpr int k2TileM = 256;   // per CTA pair; 128 rows per CTA
constexpr int k2TileN = 256;   // per CTA pair; each CTA loads 128 rows of B
constexpr int k2SfbCol = 256;  // weight scales of one K block: 4 K-steps x 8 columns
constexpr int k2SfaCol = 288;  // A scales: kSfaSlots slots of 16 columns (4 K-steps x 4)

constexpr int k2Xl1Col = 480;  // MLP up projection: h . L1_down accumulator (32 columns)

template <int R, int EPI = 0, bool LEAN = (EPI == 0)>
struct Gemm2Cfg {
  static constexpr bool QKV = EPI == 1;
  static constexpr bool MLP = EPI == 2;
  // the MLP up projection adds one warp that loads L1_down and issues h . L1_down
  static constexpr int kThreads = MLP ? 352 : 320;
  static constexpr int kABytes = 128 * 128;     // 128 rows x 256 E2M1
  static constexpr int kBBytes = 128 * 128;
  // Scale factors are staged in smem already replicated four times (the
  // layout TMEM needs), so that each tcgen05.cp 128x256b moves 32 bytes per
  // lane: two K-steps of A scales, or one K-step of both 128-row halves of B.
  static constexpr int kSfaBytes = 4 * 2048;    // 4 K-steps x 4 replicas x 512 B (128 rows)
  static constexpr int kSfbBytes = 2 * 4 * 2048;  // 2 row blocks x 4 K-steps x 4 replicas x 512 B
  // LEAN (plain layer, EPI 0, when its A scales stay resident in TMEM): four
  // stages; the A scales, needed only when a tile starts a new A block, move to
  // a two-slot ring of their own, and the epilogue stages 32 x 32 (2 KB) per
  // warp. Otherwise three stages with the A scales in every stage (the fused
  // modes need the room; a K too long for resident A scales needs them with
  // every K block, which a two-slot ring would hold back).
  static_assert(!LEAN || EPI == 0, "the lean layout is for the plain epilogue");
  static constexpr bool kLean = LEAN;
  static constexpr int kSfbOff = kABytes + kBBytes + (kLean ? 0 : kSfaBytes);  // within a stage
  static constexpr int kStageBytes = kSfbOff + kSfbBytes;  // 48 or 56 KB
  static constexpr int kStages = kLean ? 4 : 3;
  // K blocks of A scales held in TMEM (MLP: the last 32 columns hold h . L1_down)
  static constexpr int kSfaSlots = ((MLP ? k2Xl1Col : 512) - k2SfaCol) / 16;
  static constexpr int kLrCols = R < 32 ? R : 32;           // low-rank columns per stage
  static constexpr int kLrSteps = R / kLrCols;              // low-rank stages per tile
  static constexpr int kLrRowBytes = kLrCols * 2;
  static constexpr int kLrTileBytes = 128 * kLrRowBytes;    // per operand per CTA
  static constexpr SwizzleMode kLrSwizzle = kLrRowBytes == 64 ? kSwizzle64B : kSwizzle32B;
  static constexpr uint32_t kMainTx = 2u * kStageBytes;     // both CTAs
  static constexpr uint32_t kSfaTx = 2u * kSfaBytes;
  static constexpr uint32_t kLrTx = 2u * 3u * kLrTileBytes;
  // Epilogue staging per warp: the plain layer one 32 x 32 buffer (2 KB,
  // 64-byte swizzle, four TMA stores per tile); the fused QKV mode two such
  // buffers; the MLP mode one 32-row x 64-column chunk (4 KB, 128-byte swizzle).
  static constexpr int kOutPerWarp = kLean ? 2048 : 4096;  // (the plain layer uses 2 KB either way)
  static constexpr int kOutOff = kStages * kStageBytes;
  static constexpr int kOutBytes = 8 * kOutPerWarp;
  // Plain layer: the A-scale ring (two slots of one K block's A scales).
  static constexpr int kSfaRingOff = kOutOff + kOutBytes;
  static constexpr int kSfaRingBytes = kLean ? 2 * kSfaBytes : 0;
  // The tile's 256 bias values, double-buffered by tile parity.
  static constexpr int kBiasOff = kSfaRingOff + kSfaRingBytes;
  static constexpr int kBiasBytes = 2 * k2TileN * 2;
  // Fused QKV: per warp, partial sums of squares of its rows for the two heads
  // of a tile, double-buffered (2 x 2 x 32 floats).
  static constexpr int kXchgOff = kBiasOff + kBiasBytes;
  static constexpr int kXchgBytes = QKV ? 8 * 512 : 0;
  // MLP: L1_down^T for a tile's 256 columns, each CTA its 16 of the 32 rows
  // (4 chunks of 16 rows x 64 columns, 128-byte swizzle), double-buffered.
  static constexpr int kL1dOff = kXchgOff + kXchgBytes;
  static constexpr int kL1dChunk = 16 * 128;
  static constexpr int kL1dBytes = MLP ? 2 * 4 * kL1dChunk : 0;
  // MLP: the 128 reciprocals 1 / fp32(dec(S) g_h) of every E4M3 scale code
  static constexpr int kInvOff = kL1dOff + kL1dBytes;
  static constexpr int kInvBytes = MLP ? 512 : 0;
  static constexpr int kBarOff = kInvOff + kInvBytes;
  static constexpr int kSmemBytes = kBarOff + 512 + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "dynamic shared memory per CTA");
};

struct Gemm2Barriers {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full;       // the tile's MMAs have completed (one commit, both CTAs)
  uint64_t acc_empty;      // the accumulator has been drained (8 epilogue warps x 2 CTAs)
  uint64_t bias_ready[2];  // the tile's bias is in shared memory (256 epilogue threads)
  uint64_t teardown;
  uint64_t xchg[4];        // fused QKV: the two epilogue warps of a TMEM lane quadrant (64 arrivals)
  // MLP up projection
  uint64_t chunk_ready[2];  // per column half: a 64-column chunk of h is staged (4 warps x 2 CTAs)
  uint64_t chunk_free[2];   // per column half: the h . L1_down MMAs of the staged chunk completed
  uint64_t l1d_full[2];     // L1_down^T of a tile is in shared memory (both CTAs' halves)
  uint64_t l1d_free[2];     // its MMAs completed
  uint64_t xl1_done;        // the run's h . L1_down accumulator is complete
  uint64_t xl1_free;        // and has been read out (4 warps x 2 CTAs)
  uint64_t xl1_teardown;    // every h . L1_down MMA has completed
  // plain layer: the A-scale ring
  uint64_t sfa_full[2];     // a K block's A scales are in the slot (both CTAs' halves)
  uint64_t sfa_empty[2];    // and have been copied into TMEM
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Gemm2Barriers) <= 512, "the barrier block of Gemm2Cfg::kSmemBytes");

// The contiguous run of tiles [t0, t1) of CTA pair `pair` (balanced: runs
// differ by at most one tile).
__device__ __forceinline__ void pair_tile_range(int pair, int num_pairs, int num_tiles, int& t0, int& t1) {
  const int base = num_tiles / num_pairs, rem = num_tiles % num_pairs;
  t0 = pair * base + (pair < rem ? pair : rem);
  t1 = t0 + base + (pair < rem ? 1 : 0);
}

// bf16 tile store from shared memory (TMA, async bulk group).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(x), "r"(y), "r"(smem_u32(src))
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Drains this warp's four 32-column chunks of the accumulator (TMEM columns
// c0, c1, c2, c3 of its lane quadrant at tq) into registers and releases the
// accumulator to the MMA issuer (a relaxed arrive: the loads have completed,
// nothing is published).
__device__ __forceinline__ void drain4(uint32_t tq, int c0, int c1, int c2, int c3, uint32_t (&v0)[32],
                                       uint32_t (&v1)[32], uint32_t (&v2)[32], uint32_t (&v3)[32],
                                       uint32_t acc_empty_remote, int lane) {
  tmem_ld_32x32b_x32(tq + c0, v0);
  tmem_ld_32x32b_x32(tq + c1, v1);
  tmem_ld_32x32b_x32(tq + c2, v2);
  tmem_ld_32x32b_x32(tq + c3, v3);
  tmem_ld_wait();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive_cluster_relaxed(acc_empty_remote);
}

// ------------------------------------------------------------------ fused QKV epilogue
// The two epilogue warps of a TMEM lane quadrant split a 256-column tile (two
// 128-column heads) by chunks rather than by heads: warp h takes chunks 2h,
// 2h+1 of both heads, so the rotary angles it needs (pairs 32h..32h+31 of its
// rows) are the same for both heads; those of its first chunk are fetched
// before the accumulator is ready. The per-row sums of squares of the two
// warps are combined through shared memory.

// Writes / reads this lane's row of 16 packed bf16 pairs in a 2 KB staging
// buffer (32 rows x 64 bytes, the 64-byte swizzle of the store map).
__device__ __forceinline__ void stage_row16(uint8_t* buf, const uint32_t (&pk)[16], int lane) {
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ sw) << 4)) =
        make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
}
// This lane's row of 16 rotary angles (cos at cr, sin at sr; 16-byte aligned).
__device__ __forceinline__ void load_angles16(const float* cr, const float* sr, float (&tc)[16], float (&ts)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 c = reinterpret_cast<const float4*>(cr)[i];
    const float4 sv = reinterpret_cast<const float4*>(sr)[i];
    tc[4 * i] = c.x;
    tc[4 * i + 1] = c.y;
    tc[4 * i + 2] = c.z;
    tc[4 * i + 3] = c.w;
    ts[4 * i] = sv.x;
    ts[4 * i + 1] = sv.y;
    ts[4 * i + 2] = sv.z;
    ts[4 * i + 3] = sv.w;
  }
}

// Publishes a staged buffer to the async proxy and stores it with TMA.
__device__ __forceinline__ void store_staged(const uint8_t* buf, const CUtensorMap* tm_y, int x, int y, int lane) {
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tm_y, buf, x, y);
    bulk_commit();
  }
}

// 32 columns of this lane's row (16 packed bf16 pairs) into the warp's
// 32 x 64-byte staging buffer (64-byte swizzle) and one TMA store, once the
// previous store from the buffer has read it.
__device__ __forceinline__ void store_row32(uint8_t* buf, const uint32_t (&pk)[16], const CUtensorMap* tm_y, int x,
                                            int y, int lane) {
  if (lane == 0) bulk_wait_read0();
  __syncwarp();
  stage_row16(buf, pk, lane);
  store_staged(buf, tm_y, x, y, lane);
}

// Sum of squares of 16 packed bf16 pairs, added to ss in element order.
__device__ __forceinline__ float sumsq16(const uint32_t (&pk)[16], float ss) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float a = bf16_lo(pk[i]), b = bf16_hi(pk[i]);
    ss = __fmaf_rn(a, a, ss);
    ss = __fmaf_rn(b, b, ss);
  }
  return ss;
}

// RMSNorm (rstd, weights wcol: the chunk's 32 bf16) and rotation of the 16
// pairs of a chunk of this lane's row by their angles (tc, ts: cos, sin), in
// fp32, one rounding to bf16.
__device__ __forceinline__ void qk_rot16(uint32_t (&pk)[16], float rstd, const __nv_bfloat16* __restrict__ wcol,
                                         const float (&tc)[16], const float (&ts)[16]) {
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    const uint4 wv = *reinterpret_cast<const uint4*>(wcol + 8 * q4);
    const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int j = 4 * q4 + t;
      const float c = tc[j], sn = ts[j];
      const float n0 = bf16_lo(pk[j]) * rstd * bf16_lo(ww[t]);
      const float n1 = bf16_hi(pk[j]) * rstd * bf16_hi(ww[t]);
      pk[j] = pack_bf16(__fmaf_rn(n0, c, -n1 * sn), __fmaf_rn(n1, c, n0 * sn));
    }
  }
}


// One fused-QKV tile for one epilogue warp, y already packed (bf16 pairs):
// y0c, y0d = head 0's chunks c0 = 2h, c0 + 1; y1c, y1d = head 1's. For a Q/K
// tile (w0, w1: the norm weights of heads 0 and 1; cr/sr: this lane's row of
// rotary angles from chunk c0's first pair on; xs_*: the exchange slots) the
// rows are normalised and rotated, chunk c0 of both heads first so that only
// one chunk's angles are held at a time; a V tile (w0 == nullptr) is stored as
// computed. Returns false on abort.
__device__ __forceinline__ bool epilogue_qkv_tile(uint32_t (&y0c)[16], uint32_t (&y0d)[16], uint32_t (&y1c)[16],
                                                  uint32_t (&y1d)[16], int h, uint8_t* stage,
                                                  const CUtensorMap* tm_y, int xt, int y0, int lane,
                                                  const __nv_bfloat16* w0, const __nv_bfloat16* w1, const float* cr,
                                                  const float* sr, float* xs_mine, const float* xs_peer,
                                                  uint64_t* xbar, uint32_t xpar, float eps, volatile int* abort) {
  const int c0 = 2 * h;
  if (lane == 0) bulk_wait_read0();  // both staging buffers are free
  __syncwarp();
  if (w0 == nullptr) {
    stage_row16(stage, y0c, lane);
    store_staged(stage, tm_y, xt + 32 * c0, y0, lane);
    stage_row16(stage + 2048, y0d, lane);
    store_staged(stage + 2048, tm_y, xt + 32 * (c0 + 1), y0, lane);
    if (lane == 0) bulk_wait_read1();  // the store from buffer 0 has read it
    __syncwarp();
    stage_row16(stage, y1c, lane);
    store_staged(stage, tm_y, xt + 128 + 32 * c0, y0, lane);
    if (lane == 0) bulk_wait_read1();
    __syncwarp();
    stage_row16(stage + 2048, y1d, lane);
    store_staged(stage + 2048, tm_y, xt + 128 + 32 * (c0 + 1), y0, lane);
    return true;
  }
  // this warp's part of each row's sum of squares, chunk c0 then c0 + 1
  const float s0 = sumsq16(y0d, sumsq16(y0c, 0.0f));
  const float s1 = sumsq16(y1d, sumsq16(y1c, 0.0f));
  xs_mine[lane] = s0;
  xs_mine[32 + lane] = s1;
  mbar_arrive(xbar);
  float tc[16], ts[16];
  load_angles16(cr, sr, tc, ts);  // chunk c0's pairs
  if (!mbar_wait(xbar, xpar, abort)) return false;
  const float p0 = xs_peer[lane], p1 = xs_peer[32 + lane];
  // rows' sums in chunk order: warp 0's chunks 0, 1 then warp 1's chunks 2, 3
  const float t0 = h == 0 ? s0 + p0 : p0 + s0;
  const float t1 = h == 0 ? s1 + p1 : p1 + s1;
  const float r0 = 1.0f / sqrtf(__fmaf_rn(t0, 1.0f / kHeadDim, eps));
  const float r1 = 1.0f / sqrtf(__fmaf_rn(t1, 1.0f / kHeadDim, eps));
  qk_rot16(y0c, r0, w0 + 32 * c0, tc, ts);
  stage_row16(stage, y0c, lane);
  store_staged(stage, tm_y, xt + 32 * c0, y0, lane);
  qk_rot16(y1c, r1, w1 + 32 * c0, tc, ts);
  stage_row16(stage + 2048, y1c, lane);
  store_staged(stage + 2048, tm_y, xt + 128 + 32 * c0, y0, lane);
  load_angles16(cr + 16, sr + 16, tc, ts);  // chunk c0 + 1's pairs
  qk_rot16(y0d, r0, w0 + 32 * (c0 + 1), tc, ts);
  if (lane == 0) bulk_wait_read1();  // the store from buffer 0 has read it
  __syncwarp();
  stage_row16(stage, y0d, lane);
  store_staged(stage, tm_y, xt + 32 * (c0 + 1), y0, lane);
  qk_rot16(y1d, r1, w1 + 32 * (c0 + 1), tc, ts);
  if (lane == 0) bulk_wait_read1();
  __syncwarp();
  stage_row16(stage + 2048, y1d, lane);
  store_staged(stage + 2048, tm_y, xt + 128 + 32 * (c0 + 1), y0, lane);
  return true;
}

// ------------------------------------------------------------------ MLP up-projection epilogue
constexpr int kMlpRank = 32;  // the down projection's rank the fused epilogue supports

// In place on this lane's staged row of 64 columns (rowp: its 128 bytes in the
// 128-byte swizzle, sw = row % 8), holding y as bf16: h = bf16(GELU(y)),
// written back, and its four NVFP4 blocks by the activation quantiser's rule
// (S = e4m3(amax / fp32(6 g)), q = h * fp32(1 / fp32(dec(S) g)), with the
// reciprocal from inv_tab, zero for a zero or saturated scale): the 32 code
// bytes into cw (block b in bytes 8b .. 8b + 7) and the four scale bytes into
// sc (block b in byte b), for mlp_store_row64 to write once the staged chunk
// has been handed to the MMA (a release arrive waits for this thread's earlier
// global stores). One block per iteration keeps the code compact (the codes
// shift through cw so it stays in registers); within a block the values are
// processed as pairs.
__device__ __forceinline__ void mlp_gelu_quant_row64(uint8_t* rowp, int sw, bool approximate, float d,
                                                     const float* inv_tab, uint4 (&cw)[2], uint32_t& sc) {
  uint2 c0 = make_uint2(0u, 0u), c1 = c0, c2 = c0, c3 = c0;
  sc = 0;
#pragma unroll 1
  for (int blk = 0; blk < 4; ++blk) {
    uint4* p0 = reinterpret_cast<uint4*>(rowp + (((2 * blk) ^ sw) << 4));
    uint4* p1 = reinterpret_cast<uint4*>(rowp + (((2 * blk + 1) ^ sw) << 4));
    const uint4 v0 = *p0, v1 = *p1;
    uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    // branch-free GELU of all 16 values (8 independent pairs)
    float2 hv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 y = make_float2(bf16_lo(w[i]), bf16_hi(w[i]));
      hv[i] = approximate ? gelu_tanh_pair(y) : gelu_erf_pair(y);
    }
    __nv_bfloat162 am2 = __float2bfloat162_rn(0.0f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w[i] = pack_bf16(hv[i].x, hv[i].y);
      const uint32_t ab = w[i] & 0x7FFF7FFFu;  // |h| of both halves, exact
      am2 = __hmax2(am2, *reinterpret_cast<const __nv_bfloat162*>(&ab));
    }
    *p0 = make_uint4(w[0], w[1], w[2], w[3]);
    *p1 = make_uint4(w[4], w[5], w[6], w[7]);
    const float am = fmaxf(__low2float(am2), __high2float(am2));
    const uint32_t S = f32_to_e4m3(__fdiv_rn(am, d));
    const float2 inv = f2(inv_tab[S]);
    float q0[8], q1[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 a = __fmul2_rn(make_float2(bf16_lo(w[i]), bf16_hi(w[i])), inv);
      const float2 c = __fmul2_rn(make_float2(bf16_lo(w[4 + i]), bf16_hi(w[4 + i])), inv);
      q0[2 * i] = a.x;
      q0[2 * i + 1] = a.y;
      q1[2 * i] = c.x;
      q1[2 * i + 1] = c.y;
    }
    c0 = c1;
    c1 = c2;
    c2 = c3;
    c3 = make_uint2(f32x8_to_e2m1(q0), f32x8_to_e2m1(q1));
    sc |= S << (8 * blk);
  }
  cw[0] = make_uint4(c0.x, c0.y, c1.x, c1.y);
  cw[1] = make_uint4(c2.x, c2.y, c3.x, c3.y);
}

// The codes and scale word of mlp_gelu_quant_row64 for this lane's row of
// columns x0 .. x0 + 63: 32 code bytes for the down projection and the row's
// scale word of the tiled layout (zero for padding rows M <= row < m_pad).
__device__ __forceinline__ void mlp_store_row64(const uint4 (&cw)[2], uint32_t sc, int x0, int row, int M, int N,
                                                const MlpPost& mp) {
  if (row < M) {
    uint4* dst = reinterpret_cast<uint4*>(mp.codes + static_cast<int64_t>(row) * (N / 2) + x0 / 2);
    dst[0] = cw[0];
    dst[1] = cw[1];
  }
  if (row < mp.m_pad)  // the four scale bytes of a row's 64 columns are one aligned word of the tiled layout
    *reinterpret_cast<uint32_t*>(mp.scales + scale_offset(N, row, x0 / 16)) = row < M ? sc : 0u;
}

// 64 columns of packed bf16 pairs (pa, pb) of this lane's row into a 32-row x
// 128-byte buffer in the 128-byte swizzle (the K-major layout the MMA reads,
// and the box layout of the 64-column store map).
__device__ __forceinline__ void stage_row64(uint8_t* buf, const uint32_t (&pa)[16], const uint32_t (&pb)[16],
                                            int lane) {
  uint8_t* row = buf + lane * 128;
  const int sw = lane & 7;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    *reinterpret_cast<uint4*>(row + ((j ^ sw) << 4)) = make_uint4(pa[4 * j], pa[4 * j + 1], pa[4 * j + 2], pa[4 * j + 3]);
    *reinterpret_cast<uint4*>(row + (((j + 4) ^ sw) << 4)) =
        make_uint4(pb[4 * j], pb[4 * j + 1], pb[4 * j + 2], pb[4 * j + 3]);
  }
}

// Arrival that publishes this thread's earlier writes to a cluster CTA's observer.
__device__ __forceinline__ void mbar_arrive_cluster_release(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// The first tile of CTA pair p's run (the pair_tile_range split) and the pair
// that owns tile t.
__host__ __device__ __forceinline__ int pair_first_tile(int p, int num_pairs, int num_tiles) {
  const int base = num_tiles / num_pairs, rem = num_tiles % num_pairs;
  return p * base + (p < rem ? p : rem);
}
__host__ __device__ __forceinline__ int pair_of_tile(int t, int num_pairs, int num_tiles) {
  const int base = num_tiles / num_pairs, rem = num_tiles % num_pairs;
  const int big = rem * (base + 1);
  return t < big ? t / (base + 1) : rem + (t - big) / base;
}

// Sums the XL1 partials of an MLP up projection: the partial of a run of tiles
// sits in the slot of the run's first tile; the runs covering row block
// m / 256 start at that block's first tile and at every CTA pair's first tile
// inside it. xl1[m][j] = bf16(sum over those runs in tile order) (fp32,
// deterministic).
__global__ void mlp_xl1_reduce_kernel(const float* __restrict__ partial, int num_tiles, int num_pairs, int num_nt,
                                      int M, __nv_bfloat16* __restrict__ xl1) {
  const int64_t total = static_cast<int64_t>(M) * kMlpRank;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int m = static_cast<int>(i / kMlpRank), j = static_cast<int>(i % kMlpRank);
    const int mt = m / k2TileM, lr = m % k2TileM;
    const int t_lo = mt * num_nt, t_hi = t_lo + num_nt;
    float s = 0.0f;
    for (int p = pair_of_tile(t_lo, num_pairs, num_tiles); p < num_pairs; ++p) {
      const int f = pair_first_tile(p, num_pairs, num_tiles);
      if (f >= t_hi) break;
      const int t = f > t_lo ? f : t_lo;
      s = __fadd_rn(s, partial[(static_cast<int64_t>(t) * k2TileM + lr) * kMlpRank + j]);
    }
    xl1[i] = __float2bfloat16_rn(s);
  }
}

template <int R, int EPI, bool LEAN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Gemm2Cfg<R, EPI, LEAN>::kThreads, 1) w4a4_gemm_2sm_kernel(
    const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
    const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
    const __grid_constant__ CUtensorMap tm_xl1, const __grid_constant__ CUtensorMap tm_l2s,
    const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_l1d, const float* __restrict__ gscale,
    const __nv_bfloat16* __restrict__ bias, int M, int N, int K, const QkvPost post, const MlpPost mlp) {
  using C = Gemm2Cfg<R, EPI, LEAN>;
  constexpr bool QKV = EPI == 1;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Gemm2Barriers* bars = reinterpret_cast<Gemm2Barriers*>(smem + C::kBarOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int num_mt = (M + k2TileM - 1) / k2TileM;
  const int num_nt = N / k2TileN;
  const int num_tiles = num_mt * num_nt;
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;
  const int nk = K / 256;
  const int steps = C::kLrSteps + nk;
  const int sf_row_stride = K / 64;  // scale atoms per 128-row block
  // A scales stay in TMEM across the tiles of one A block when every K block has a slot
  const bool sfa_resident = nk <= C::kSfaSlots;
  int t_begin, t_end;
  pair_tile_range(pair, num_pairs, num_tiles, t_begin, t_end);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, 16);  // 8 epilogue warps x 2 CTAs
    mbar_init(&bars->bias_ready[0], 256);
    mbar_init(&bars->bias_ready[1], 256);
    mbar_init(&bars->teardown, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&bars->xchg[i], 64);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->chunk_ready[i], 8);  // 4 warps x 2 CTAs
      mbar_init(&bars->chunk_free[i], 1);
      mbar_init(&bars->l1d_full[i], 1);
      mbar_init(&bars->l1d_free[i], 1);
    }
    mbar_init(&bars->xl1_done, 1);
    mbar_init(&bars->xl1_free, 8);
    mbar_init(&bars->xl1_teardown, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->sfa_full[i], 1);
      mbar_init(&bars->sfa_empty[i], 1);
    }
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_sfa);
    prefetch_tmap(&tm_sfb);
    prefetch_tmap(&tm_xl1);
    prefetch_tmap(&tm_l2s);
    prefetch_tmap(&tm_y);
    if (C::MLP) prefetch_tmap(&tm_l1d);
  }
  if (warp == 1) {
    tmem_alloc_cg2(&bars->tmem_base, 512);
    tmem_relinquish_cg2();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;
  // Everything above overlaps the previous kernel of the stream (programmatic
  // dependent launch); nothing global is read or written before this wait.
  pdl_wait();
  if constexpr (C::MLP) {
    // reciprocal of every possible block decode scale of h (dec(S) g_h takes at
    // most 127 finite values); the epilogue warps read it after their first
    // acc_full wait, which follows this CTA-wide barrier
    float* inv_tab = reinterpret_cast<float*>(smem + C::kInvOff);
    if (threadIdx.x < 128) {
      const float sd = __fmul_rn(e4m3_to_f32(threadIdx.x), *mlp.g_h);
      inv_tab[threadIdx.x] = (sd == 0.0f || threadIdx.x >= 0x7Fu) ? 0.0f : __frcp_rn(sd);
    }
    __syncthreads();
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int prev_mt = -1;
      int nsfa = 0;  // plain layer: A-scale loads so far (ring slot nsfa & 1)
      for (int tile = t_begin; tile < t_end && ok; ++tile) {
        const int mt = tile / num_nt, nt = tile % num_nt;
        const bool sfa_load = !sfa_resident || mt != prev_mt;
        prev_mt = mt;
        const int m_own = mt * k2TileM + static_cast<int>(rank) * 128;
        const int n_own = nt * k2TileN + static_cast<int>(rank) * 128;
        const int nblk = nt * 2;  // first 128-row block of B in this tile
        for (int step = 0; step < steps; ++step) {
          if (!mbar_wait(&bars->empty[s], ph ^ 1, abort)) { ok = false; break; }
          uint8_t* st = smem + s * C::kStageBytes;
          const uint32_t bar = mapa_shared(smem_u32(&bars->full[s]), 0);
          if (step >= nk) {  // the low-rank stages come last, after the K blocks
            if (rank == 0) mbar_arrive_expect_tx(&bars->full[s], C::kLrTx);
            const int x = (step - nk) * C::kLrCols;
            tma_load_2d_cg2(st, &tm_xl1, x, m_own, bar);
            tma_load_2d_cg2(st + C::kABytes, &tm_l2s, x, n_own, bar);
            tma_load_2d_cg2(st + C::kABytes + C::kLrTileBytes, &tm_l2s, x, N + n_own, bar);
          } else {
            const int kb = step;
            if (rank == 0)
              mbar_arrive_expect_tx(&bars->full[s], (C::kLean || sfa_load) ? C::kMainTx : C::kMainTx - C::kSfaTx);
            tma_load_2d_cg2(st, &tm_a, kb * 128, m_own, bar);
            tma_load_2d_cg2(st + C::kABytes, &tm_b, kb * 128, n_own, bar);
            if (sfa_load) {
              const int sfa_c = (m_own / 128) * sf_row_stride + 4 * kb;
              if constexpr (C::kLean) {
                const int slot = nsfa & 1;
                if (!mbar_wait(&bars->sfa_empty[slot], ((nsfa >> 1) & 1) ^ 1, abort)) { ok = false; break; }
                if (rank == 0) mbar_arrive_expect_tx(&bars->sfa_full[slot], C::kSfaTx);
                tma_load_4d_cg2(smem + C::kSfaRingOff + slot * C::kSfaBytes, &tm_sfa, 0, 0, 0, sfa_c,
                                mapa_shared(smem_u32(&bars->sfa_full[slot]), 0));
                ++nsfa;
              } else {
                tma_load_4d_cg2(st + C::kABytes + C::kBBytes, &tm_sfa, 0, 0, 0, sfa_c, bar);
              }
            }
            tma_load_5d_cg2(st + C::kSfbOff, &tm_sfb, 0, 0, 0, 4 * kb, nblk, bar);
          }
          if (++s == S) { s = 0; ph ^= 1; }
        }
      }
      if (!ok) {
        // error path: give copies that may still be in flight time to land
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 2000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (rank == 0 && lane == 0) {
      const uint32_t idesc_fp4 = (1u << 7) | (1u << 10) | (uint32_t(k2TileN >> 3) << 17) | (uint32_t(k2TileM >> 4) << 24);
      const uint32_t idesc_bf16 =
          (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(k2TileN >> 3) << 17) | (uint32_t(k2TileM >> 4) << 24);
      const uint32_t t_sfb = tmem + k2SfbCol;
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      bool ok = true;
      int prev_mt = -1;
      int nsfa = 0;  // plain layer: A-scale slots consumed so far
      for (int tile = t_begin; tile < t_end && ok; ++tile, ++it) {
        const int mt = tile / num_nt;
        const bool sfa_load = !sfa_resident || mt != prev_mt;
        prev_mt = mt;
        // the epilogue has drained the previous tile's accumulator
        if (!mbar_wait_cluster(&bars->acc_empty, (it & 1) ^ 1, abort)) { ok = false; break; }
        tc_fence_after();
        for (int step = 0; step < steps; ++step) {
          if (!mbar_wait(&bars->full[s], ph, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * C::kStageBytes);
          if (step >= nk) {  // low-rank stages, after the K blocks: XL1 . (hi, lo) into the same accumulator
#pragma unroll
            for (int k16 = 0; k16 < C::kLrCols / 16; ++k16) {
              const uint64_t a = smem_desc(st + 32 * k16, 16, 8 * C::kLrRowBytes, C::kLrSwizzle);
              const uint64_t bh = smem_desc(st + C::kABytes + 32 * k16, 16, 8 * C::kLrRowBytes, C::kLrSwizzle);
              const uint64_t bl =
                  smem_desc(st + C::kABytes + C::kLrTileBytes + 32 * k16, 16, 8 * C::kLrRowBytes, C::kLrSwizzle);
              mma_bf16_cg2(tmem, a, bh, idesc_bf16, 1u);
              mma_bf16_cg2(tmem, a, bl, idesc_bf16, 1u);
            }
          } else {
            const int kb = step;
            const uint32_t t_sfa = tmem + k2SfaCol + 16 * (kb % C::kSfaSlots);
            const uint32_t sfb = st + C::kSfbOff;
            // A: K-steps (0,1) and (2,3), 2 KB apart (only when the tile starts a new A block);
            // B: K-step j, row blocks 8 KB apart
            if (sfa_load) {
              uint32_t sfa = st + C::kABytes + C::kBBytes;
              if constexpr (C::kLean) {
                const int slot = nsfa & 1;
                if (!mbar_wait(&bars->sfa_full[slot], (nsfa >> 1) & 1, abort)) { ok = false; break; }
                tc_fence_after();
                sfa = smem_u32(smem + C::kSfaRingOff + slot * C::kSfaBytes);
              }
              tmem_cp_128x256b_cg2(t_sfa, smem_desc(sfa, 2048, 128, kSwizzleNone));
              tmem_cp_128x256b_cg2(t_sfa + 8, smem_desc(sfa + 4096, 2048, 128, kSwizzleNone));
              if constexpr (C::kLean) tc_commit_cg2_mc(&bars->sfa_empty[nsfa++ & 1], 0x3);  // the slot may be refilled
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tmem_cp_128x256b_cg2(t_sfb + 8 * j, smem_desc(sfb + 2048 * j, 8192, 128, kSwizzleNone));
            const uint64_t adesc = smem_desc(st, 16, 1024, kSwizzle128B);
            const uint64_t bdesc = smem_desc(st + C::kABytes, 16, 1024, kSwizzle128B);
#pragma unroll
            for (int j = 0; j < 4; ++j)  // the tile's first MMA overwrites the accumulator
              mma_nvf4_cg2(tmem, adesc + 2 * j, bdesc + 2 * j, idesc_fp4, t_sfa + 4 * j, t_sfb + 8 * j,
                           (kb | j) != 0 ? 1u : 0u);
          }
          tc_commit_cg2_mc(&bars->empty[s], 0x3);
          if (++s == S) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        tc_commit_cg2_mc(&bars->acc_full, 0x3);
      }
      // every MMA this thread issued completes before TMEM is released
      tc_commit(&bars->teardown);
      volatile int never = 0;
      mbar_wait(&bars->teardown, 0, &never);
    }
  } else if (C::MLP && warp == 10) {
    // ------------------------------------------------------------ MLP: h . L1_down (both CTAs load, even CTA issues)
    // Per tile: L1_down^T for the tile's 256 columns (each CTA its 16 of the 32
    // rows; completion bytes on the even CTA's barrier), then for each staged
    // 64-column chunk of h four bf16 MMAs (M = 256, N = 32, K = 16) into the
    // h . L1_down accumulator, which runs over the pair's tiles that share
    // their rows and is read out at the end of each such run.
    if (lane == 0) {
      const uint32_t idesc =
          (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kMlpRank >> 3) << 17) | (uint32_t(k2TileM >> 4) << 24);
      uint8_t* l1d = smem + C::kL1dOff;
      const uint32_t t_xl1 = tmem + k2Xl1Col;
      // L1_down^T of the pair's it-th tile into buffer it & 1 (once the MMAs of
      // tile it - 2 have read that buffer)
      auto load_l1d = [&](int it, int tile) -> bool {
        const int b = it & 1;
        if (!mbar_wait(&bars->l1d_free[b], ((it >> 1) & 1) ^ 1, abort)) return false;
        if (rank == 0) mbar_arrive_expect_tx(&bars->l1d_full[b], 2u * 4u * C::kL1dChunk);
        const uint32_t lbar = mapa_shared(smem_u32(&bars->l1d_full[b]), 0);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tma_load_2d_cg2(l1d + (4 * b + k) * C::kL1dChunk, &tm_l1d, (tile % num_nt) * k2TileN + 64 * k,
                          16 * static_cast<int>(rank), lbar);
        return true;
      };
      int it = 0, run = 0, prev_mt = -1;
      bool ok = t_begin >= t_end || load_l1d(0, t_begin);
      for (int tile = t_begin; tile < t_end && ok; ++tile, ++it) {
        const int mt = tile / num_nt;
        const bool first = mt != prev_mt;
        prev_mt = mt;
        const bool last = tile + 1 == t_end || (tile + 1) / num_nt != mt;
        const int b = it & 1;
        if (tile + 1 < t_end && !load_l1d(it + 1, tile + 1)) { ok = false; break; }  // the next tile's, early
        if (rank != 0) continue;
        // a new run starts once the previous run's accumulator has been read out
        if (first && it > 0 && !mbar_wait_cluster(&bars->xl1_free, (run - 1) & 1, abort)) { ok = false; break; }
        if (!mbar_wait(&bars->l1d_full[b], (it >> 1) & 1, abort)) { ok = false; break; }
        // chunks alternate between the column halves' warps: (half 0, chunk 0),
        // (half 1, chunk 0), (half 0, chunk 1), (half 1, chunk 1), so each half
        // stages its next chunk while the other half's is multiplied
        for (int k = 0; k < 4; ++k) {
          const int hh = k & 1, cc = k >> 1;
          if (!mbar_wait_cluster(&bars->chunk_ready[hh], cc, abort)) { ok = false; break; }
          tc_fence_after();
          const uint64_t a = smem_desc(smem_u32(smem + C::kOutOff + hh * 16384), 16, 1024, kSwizzle128B);
          const uint64_t bd =
              smem_desc(smem_u32(l1d + (4 * b + 2 * hh + cc) * C::kL1dChunk), 16, 1024, kSwizzle128B);
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16)
            mma_bf16_cg2(t_xl1, a + 2 * k16, bd + 2 * k16, idesc, (first && k == 0 && k16 == 0) ? 0u : 1u);
          tc_commit_cg2_mc(&bars->chunk_free[hh], 0x3);
        }
        if (!ok) break;
        tc_commit_cg2_mc(&bars->l1d_free[b], 0x3);
        if (last) {
          tc_commit_cg2_mc(&bars->xl1_done, 0x3);
          ++run;
        }
      }
      if (rank == 0) {  // every MMA this thread issued completes before TMEM is released
        tc_commit(&bars->xl1_teardown);
        volatile int never = 0;
        mbar_wait(&bars->xl1_teardown, 0, &never);
      }
      if (!ok) {
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 2000000ull) {
        }
      }
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int e = warp - 2;
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int h = e >> 2;    // 128-column half of the tile (fused QKV: chunk pair)
    const float alpha = gscale[2];
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    const uint32_t acc_empty_remote = mapa_shared(smem_u32(&bars->acc_empty), 0);
    // staging buffer of warp (h, q): the MLP epilogue's chunk buffer of half h
    // holds the four quadrants' rows in order (rows 32 q .. 32 q + 31 at q x 4 KB)
    uint8_t* stage = smem + C::kOutOff + (4 * h + q) * C::kOutPerWarp;
    __nv_bfloat16* bias_s = reinterpret_cast<__nv_bfloat16*>(smem + C::kBiasOff);
    uint32_t nx = 0;  // fused QKV: exchanges of row sums done by this warp
    int mlp_prev_mt = -1, run_first = 0, nrun = 0;  // MLP: runs of tiles sharing their rows
    int it = 0;
    for (int tile = t_begin; tile < t_end; ++tile, ++it) {
      const int mt = tile / num_nt, nt = tile % num_nt;
      const int y0 = mt * k2TileM + static_cast<int>(rank) * 128 + 32 * q;
      const int col0 = nt * k2TileN + 128 * h;
      // the tile's bias into shared memory (thread 32 e + lane loads one value)
      __nv_bfloat16* bb = bias_s + (it & 1) * k2TileN;
      if (bias != nullptr) bb[32 * e + lane] = bias[nt * k2TileN + 32 * e + lane];
      mbar_arrive(&bars->bias_ready[it & 1]);
      if constexpr (QKV) {
        // A tile is all Q/K or all V (the V block starts at 2 * hd, a multiple of 256).
        if (!mbar_wait(&bars->acc_full, it & 1, abort)) break;
        tc_fence_after();
        uint32_t y0c[16], y0d[16], y1c[16], y1d[16];
        {
          uint32_t va[32], vb[32], vc[32], vd[32];
          const int c0 = 2 * h;
          drain4(lane_base, 32 * c0, 32 * (c0 + 1), 128 + 32 * c0, 128 + 32 * (c0 + 1), va, vb, vc, vd,
                 acc_empty_remote, lane);
          if (!mbar_wait(&bars->bias_ready[it & 1], (it >> 1) & 1, abort)) break;
          const __nv_bfloat16* bt = bias != nullptr ? bb : nullptr;
          pack_chunk(va, bt ? bt + 32 * c0 : nullptr, alpha, y0c);
          pack_chunk(vb, bt ? bt + 32 * (c0 + 1) : nullptr, alpha, y0d);
          pack_chunk(vc, bt ? bt + 128 + 32 * c0 : nullptr, alpha, y1c);
          pack_chunk(vd, bt ? bt + 128 + 32 * (c0 + 1) : nullptr, alpha, y1d);
        }

        const int xt = nt * k2TileN;
        const bool qk = xt < 2 * post.hd;
        const int64_t row = (y0 + lane < M) ? y0 + lane : M - 1;
        const float* cr = post.cos + row * post.ld_rope + 32 * h;
        const float* sr = post.sin + row * post.ld_rope + 32 * h;
        const __nv_bfloat16* w0 = qk ? (xt < post.hd ? post.w_q : post.w_k) : nullptr;
        const __nv_bfloat16* w1 = qk ? (xt + 128 < post.hd ? post.w_q : post.w_k) : nullptr;
        float* xs = reinterpret_cast<float*>(smem + C::kXchgOff) + 128 * (2 * q + h) + 64 * (nx & 1);
        const float* xp = reinterpret_cast<const float*>(smem + C::kXchgOff) + 128 * (2 * q + (h ^ 1)) + 64 * (nx & 1);
        // (the accumulator is already released: the angles' latency no longer holds the MMAs up)
        const bool ok = epilogue_qkv_tile(y0c, y0d, y1c, y1d, h, stage, &tm_y, xt, y0, lane, w0, w1, cr, sr, xs,
                                          xp, &bars->xchg[q], nx & 1, post.eps, abort);
        if (!ok) break;
        if (qk) ++nx;
        continue;
      }
      if (!mbar_wait(&bars->acc_full, it & 1, abort)) break;
      tc_fence_after();
      uint32_t va[32], vb[32], vc[32], vd[32];
      drain4(lane_base + 128 * h, 0, 32, 64, 96, va, vb, vc, vd, acc_empty_remote, lane);
      if (!mbar_wait(&bars->bias_ready[it & 1], (it >> 1) & 1, abort)) break;
      const __nv_bfloat16* bcol = bias != nullptr ? bb + 128 * h : nullptr;
      if constexpr (EPI == 2) {
        const int row = y0 + lane;
        const float g = *mlp.g_h;
        const float d = __fmul_rn(6.0f, g);
        uint32_t pk0[16], pk1[16], pk2[16], pk3[16];
        pack_chunk(va, bcol, alpha, pk0);
        pack_chunk(vb, bcol ? bcol + 32 : nullptr, alpha, pk1);
        pack_chunk(vc, bcol ? bcol + 64 : nullptr, alpha, pk2);
        pack_chunk(vd, bcol ? bcol + 96 : nullptr, alpha, pk3);
        const bool first = mt != mlp_prev_mt;
        mlp_prev_mt = mt;
        if (first) run_first = tile;
        const bool last = tile + 1 == t_end || (tile + 1) / num_nt != mt;
        const uint32_t ready = mapa_shared(smem_u32(&bars->chunk_ready[h]), 0);
        bool ok = true;
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          // this half's chunk buffer: its previous chunk's MMAs have read it
          if (!mbar_wait(&bars->chunk_free[h], cc ^ 1, abort)) { ok = false; break; }
          if (mlp.store_h && lane == 0) bulk_wait_read0();  // and so has the previous store of h
          __syncwarp();
          uint32_t ta[16], tb[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            ta[i] = cc == 0 ? pk0[i] : pk2[i];
            tb[i] = cc == 0 ? pk1[i] : pk3[i];
          }
          stage_row64(stage, ta, tb, lane);  // y, then GELU and the quantisation in place
          uint4 cw[2];
          uint32_t scw;
          mlp_gelu_quant_row64(stage + lane * 128, lane & 7, mlp.approximate != 0, d,
                               reinterpret_cast<const float*>(smem + C::kInvOff), cw, scw);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive_cluster_release(ready);
            if (mlp.store_h) {
              tma_store_2d(&tm_y, stage, col0 + 64 * cc, y0);
              bulk_commit();
            }
          }
          mlp_store_row64(cw, scw, col0 + 64 * cc, row, M, N, mlp);
        }
        if (!ok) break;
        if (last) {
          if (h == 0) {  // the first half's warps read the run's accumulator out (their lane quadrant)
            if (!mbar_wait(&bars->xl1_done, nrun & 1, abort)) break;
            tc_fence_after();
            uint32_t xv[32];
            tmem_ld_32x32b_x32(lane_base + k2Xl1Col, xv);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&bars->xl1_free), 0));
            float4* dst = reinterpret_cast<float4*>(
                mlp.partial + (static_cast<int64_t>(run_first) * k2TileM + static_cast<int>(rank) * 128 + 32 * q + lane) *
                                  kMlpRank);
#pragma unroll
            for (int j = 0; j < kMlpRank / 4; ++j)
              dst[j] = make_float4(__uint_as_float(xv[4 * j]), __uint_as_float(xv[4 * j + 1]),
                                   __uint_as_float(xv[4 * j + 2]), __uint_as_float(xv[4 * j + 3]));
          }
          ++nrun;
        }
        continue;
      }
      uint32_t pk[16];
      pack_chunk(va, bcol, alpha, pk);
      store_row32(stage, pk, &tm_y, col0, y0, lane);
      pack_chunk(vb, bcol ? bcol + 32 : nullptr, alpha, pk);
      store_row32(stage, pk, &tm_y, col0 + 32, y0, lane);
      pack_chunk(vc, bcol ? bcol + 64 : nullptr, alpha, pk);
      store_row32(stage, pk, &tm_y, col0 + 64, y0, lane);
      pack_chunk(vd, bcol ? bcol + 96 : nullptr, alpha, pk);
      store_row32(stage, pk, &tm_y, col0 + 96, y0, lane);
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_cg2(tmem, 512);
  }
}

}  // namespace svdq
