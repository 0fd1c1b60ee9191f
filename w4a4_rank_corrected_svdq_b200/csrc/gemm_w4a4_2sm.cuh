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
// 128 x 256 half of the accumulator into that CTA's TMEM. Per 256-wide K block
// and SM this moves 38 KB for 8.4 MFLOP (half the bytes per FLOP of a 128 x 128
// single-CTA tile), which keeps the L2 -> SM traffic within what L2 delivers.
// No load uses cluster multicast: each CTA fetches every byte it stores.
//
// Roles (320 threads per CTA):
//  * warp 0     TMA producer (both CTAs): per tile first r/c low-rank stages
//               (XL1 columns, hi and lo columns of l2s; c = min(r, 32)), then
//               K/256 stages of E2M1 codes (128-byte swizzle) and UE4M3 scale
//               atoms. Completion bytes of both CTAs land on the even CTA's
//               barrier (cp.async.bulk.tensor .cta_group::2).
//  * warp 1     TMEM owner (both CTAs, 512 columns); in the even CTA lane 0
//               issues the MMAs and the scale copies smem -> TMEM.
//  * warps 2-9  epilogue (both CTAs): TMEM -> registers, y = alpha acc + b,
//               bf16 stores; two warps per 32-lane TMEM quadrant, one per
//               128-column half. The epilogue mode EPI selects the plain
//               layer (0), the fused QKV post-processing (1: per-head RMSNorm
//               of Q/K and the rotary embedding; the two warps of a quadrant
//               then split a tile by chunks) or the MLP up projection (2:
//               GELU and the down projection's NVFP4 codes, scales and XL1
//               partials instead of y).
// TMEM: accumulator 0 = columns [0,256), accumulator 1 = [208,464): the two
// share [208,256), which the epilogue reads first and releases early, so the
// next tile's MMAs start long before the previous tile is fully stored; scale
// factors at [464,480) (A) and [480,512) (B, 256 rows).
// Every wait is bounded; see mbar_wait.
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
__device__ __forceinline__ void tmem_cp_cg2(uint32_t taddr, uint64_t s_desc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(s_desc) : "memory");
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
constexpr int k2TileM = 256;  // per CTA pair; 128 rows per CTA
constexpr int k2TileN = 256;  // per CTA pair; each CTA loads 128 rows of B
constexpr int k2Acc1Col = 208;
constexpr int k2SfaCol = 464;
constexpr int k2SfbCol = 480;

template <int R, int EPI = 0>
struct Gemm2Cfg {
  static constexpr bool QKV = EPI == 1;
  static constexpr int kABytes = 128 * 128;     // 128 rows x 256 E2M1
  static constexpr int kBBytes = 128 * 128;
  // Scale factors are staged in smem already replicated four times (the
  // layout TMEM needs), so that each tcgen05.cp 128x256b moves 32 bytes per
  // lane: two K-steps of A scales, or one K-step of both 128-row halves of B.
  static constexpr int kSfaBytes = 4 * 2048;    // 4 K-steps x 4 replicas x 512 B (128 rows)
  static constexpr int kSfbBytes = 2 * 4 * 2048;  // 2 row blocks x 4 K-steps x 4 replicas x 512 B
  static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;  // 56 KB
  static constexpr int kStages = 3;
  static constexpr int kLrCols = R < 32 ? R : 32;           // low-rank columns per stage
  static constexpr int kLrSteps = R / kLrCols;              // low-rank stages per tile
  static constexpr int kLrRowBytes = kLrCols * 2;
  static constexpr int kLrTileBytes = 128 * kLrRowBytes;    // per operand per CTA
  static constexpr SwizzleMode kLrSwizzle = kLrRowBytes == 64 ? kSwizzle64B : kSwizzle32B;
  static constexpr uint32_t kMainTx = 2u * kStageBytes;     // both CTAs
  static constexpr uint32_t kLrTx = 2u * 3u * kLrTileBytes;
  // Epilogue staging per warp: two 2 KB bf16 TMA-store buffers.
  static constexpr int kOutPerWarp = 4096;
  static constexpr int kOutOff = kStages * kStageBytes;
  static constexpr int kOutBytes = 8 * kOutPerWarp;
  // Fused QKV: per warp, partial sums of squares of its rows for the two heads
  // of a tile, double-buffered (2 x 2 x 32 floats).
  static constexpr int kXchgOff = kOutOff + kOutBytes;
  static constexpr int kXchgBytes = QKV ? 8 * 512 : 0;
  static constexpr int kBarOff = kXchgOff + kXchgBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;
};

struct Gemm2Barriers {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t ovl_free;
  uint64_t teardown;
  uint64_t xchg[4];  // fused QKV: the two epilogue warps of a TMEM lane quadrant (64 arrivals)
  uint32_t tmem_base;
  int abort;
};

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

// y = alpha * acc + b for one 32-column chunk of this lane's row, packed to
// bf16 and written into a 32-row x 64-byte staging buffer in the 64-byte
// swizzled order the Y tensor map expects; then lane 0 issues the TMA store.
__device__ __forceinline__ void store_chunk(const uint32_t (&v)[32], const uint4 (&bv)[16], int c, float alpha,
                                            uint8_t* stage, const CUtensorMap* tm_y, int x, int y, int lane) {
  uint32_t packed[16];
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    const uint4 bq = bv[4 * c + p / 4];
    const uint32_t bw = (p % 4 == 0) ? bq.x : (p % 4 == 1) ? bq.y : (p % 4 == 2) ? bq.z : bq.w;
    const float y0 = __fmaf_rn(__uint_as_float(v[2 * p]), alpha, __uint_as_float(bw << 16));
    const float y1 = __fmaf_rn(__uint_as_float(v[2 * p + 1]), alpha, __uint_as_float(bw & 0xFFFF0000u));
    const __nv_bfloat162 hv = __floats2bfloat162_rn(y0, y1);
    packed[p] = *reinterpret_cast<const uint32_t*>(&hv);
  }
  if (lane == 0) bulk_wait_read1();  // the previous store from this buffer has read it
  __syncwarp();
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    *reinterpret_cast<uint4*>(stage + lane * 64 + ((j ^ sw) << 4)) =
        make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tm_y, stage, x, y);
    bulk_commit();
  }
}

// One epilogue warp's 128-column half of a tile, in four 32-column chunks.
// If the warp holds the columns shared by the two accumulators (chunks 2,3 of
// accumulator 0's upper half; chunks 0,1 of accumulator 1's lower half), it
// reads those first and releases them before doing any other work.
template <int FIRST>
__device__ __forceinline__ void epilogue_half(uint32_t taddr, const uint4 (&bv)[16], float alpha, uint8_t* stage,
                                              int& nbuf, const CUtensorMap* tm_y, int x0, int y0, bool holds_overlap,
                                              uint32_t ovl_bar, int lane) {
  uint32_t va[32], vb[32];
  tmem_ld_32x32b_x32(taddr + 32 * ((FIRST + 0) & 3), va);
  tmem_ld_32x32b_x32(taddr + 32 * ((FIRST + 1) & 3), vb);
  tmem_ld_wait();
  if (holds_overlap) {  // the loads above have completed (tcgen05.wait::ld): nothing else to publish
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster_relaxed(ovl_bar);
  }
  store_chunk(va, bv, (FIRST + 0) & 3, alpha, stage + 2048 * (nbuf & 1), tm_y, x0 + 32 * ((FIRST + 0) & 3), y0, lane);
  ++nbuf;
  store_chunk(vb, bv, (FIRST + 1) & 3, alpha, stage + 2048 * (nbuf & 1), tm_y, x0 + 32 * ((FIRST + 1) & 3), y0, lane);
  ++nbuf;
  tmem_ld_32x32b_x32(taddr + 32 * ((FIRST + 2) & 3), va);
  tmem_ld_32x32b_x32(taddr + 32 * ((FIRST + 3) & 3), vb);
  tmem_ld_wait();
  store_chunk(va, bv, (FIRST + 2) & 3, alpha, stage + 2048 * (nbuf & 1), tm_y, x0 + 32 * ((FIRST + 2) & 3), y0, lane);
  ++nbuf;
  store_chunk(vb, bv, (FIRST + 3) & 3, alpha, stage + 2048 * (nbuf & 1), tm_y, x0 + 32 * ((FIRST + 3) & 3), y0, lane);
  ++nbuf;
}

// ------------------------------------------------------------------ fused QKV epilogue
// For the fused QKV variant the two epilogue warps of a TMEM lane quadrant
// split a 256-column tile (two 128-column heads) by chunks rather than by
// heads: warp h takes chunks 2h, 2h+1 of both heads, so the rotary angles it
// needs (pairs 32h..32h+31 of its rows) are the same for both heads and are
// fetched once, before the accumulator is ready. The per-row sums of squares
// of the two warps are combined through shared memory.

// Writes / reads this lane's row of 16 packed bf16 pairs in a 2 KB staging
// buffer (32 rows x 64 bytes, the 64-byte swizzle of the store map).
__device__ __forceinline__ void stage_row16(uint8_t* buf, const uint32_t (&pk)[16], int lane) {
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ sw) << 4)) =
        make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
}
__device__ __forceinline__ void load_row16(const uint8_t* buf, uint32_t (&pk)[16], int lane) {
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 v = *reinterpret_cast<const uint4*>(buf + lane * 64 + ((j ^ sw) << 4));
    pk[4 * j] = v.x;
    pk[4 * j + 1] = v.y;
    pk[4 * j + 2] = v.z;
    pk[4 * j + 3] = v.w;
  }
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

// bf16 pairs of alpha * acc + b for one 32-column chunk (bias at bcol, or none).
__device__ __forceinline__ void pack32(const uint32_t (&v)[32], const __nv_bfloat16* bcol, float alpha,
                                       uint32_t (&pk)[16]) {
  pack_chunk(v, bcol, alpha, pk);
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

// One fused-QKV tile for one epilogue warp: chunks c0 = 2h, c0 + 1 of head F
// (read first: it holds the columns shared by the two accumulators when
// holds_overlap) and of head 1 - F. tacc: the accumulator's TMEM address for
// this lane quadrant. For a Q/K tile (w_f, w_s the norm weights of heads F
// and 1 - F)
// tc0/ts0 hold the angles of chunk c0's pairs (fetched before the
// accumulator was ready), cr/sr point at those of chunk c0 + 1 (fetched once
// the first head is read) and xs_* are the exchange slots; a V tile
// (w_f == nullptr) is stored as computed. Returns false on abort.
__device__ __forceinline__ bool epilogue_qkv_tile(uint32_t tacc, int F, int h, const __nv_bfloat16* btile, float alpha,
                                                  uint8_t* stage, const CUtensorMap* tm_y, int xt, int y0,
                                                  bool holds_overlap, uint32_t ovl_bar, int lane,
                                                  const __nv_bfloat16* w_f, const __nv_bfloat16* w_s,
                                                  const float (&tc0)[16],
                                                  const float (&ts0)[16], const float* cr, const float* sr,
                                                  float* xs_mine, const float* xs_peer,
                                                  uint64_t* xbar, uint32_t xpar, float eps, volatile int* abort) {
  const int S = 1 - F;
  const bool qk = w_f != nullptr;
  const int c0 = 2 * h;
  const auto bcol = [&](int head, int c) { return btile != nullptr ? btile + 128 * head + 32 * c : nullptr; };
  float ssf = 0.0f, sss = 0.0f;  // this warp's part of the rows' sums of squares
  if (lane == 0) bulk_wait_read0();  // both staging buffers are free
  __syncwarp();
  {
    uint32_t va[32], vb[32];
    tmem_ld_32x32b_x32(tacc + 128 * F + 32 * c0, va);
    tmem_ld_32x32b_x32(tacc + 128 * F + 32 * (c0 + 1), vb);
    tmem_ld_wait();
    if (holds_overlap) {  // the loads above have completed (tcgen05.wait::ld): nothing else to publish
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(ovl_bar);
    }
    uint32_t pk[16];
    pack32(va, bcol(F, c0), alpha, pk);
    ssf = sumsq16(pk, ssf);
    stage_row16(stage, pk, lane);
    if (!qk) store_staged(stage, tm_y, xt + 128 * F + 32 * c0, y0, lane);
    pack32(vb, bcol(F, c0 + 1), alpha, pk);
    ssf = sumsq16(pk, ssf);
    stage_row16(stage + 2048, pk, lane);
    if (!qk) store_staged(stage + 2048, tm_y, xt + 128 * F + 32 * (c0 + 1), y0, lane);
  }
  float tc1[16], ts1[16];
  if (qk) {
    load_angles16(cr, sr, tc1, ts1);
    // head 1 - F never holds shared columns: read it for its sums now and
    // again, to store it, after the exchange
#pragma unroll 1
    for (int k = 0; k < 2; ++k) {
      uint32_t va[32], pk[16];
      tmem_ld_32x32b_x32(tacc + 128 * S + 32 * (c0 + k), va);
      tmem_ld_wait();
      pack32(va, bcol(S, c0 + k), alpha, pk);
      sss = sumsq16(pk, sss);
    }
    // this warp's partial sums for heads 0 / 1, then the partner's
    xs_mine[32 * F + lane] = ssf;
    xs_mine[32 * S + lane] = sss;
    mbar_arrive(xbar);
    if (!mbar_wait(xbar, xpar, abort)) return false;
    const float pf = xs_peer[32 * F + lane], pss = xs_peer[32 * S + lane];
    // rows' sums in chunk order: warp 0's chunks 0, 1 then warp 1's chunks 2, 3
    const float tf = h == 0 ? ssf + pf : pf + ssf;
    const float tsum = h == 0 ? sss + pss : pss + sss;
    const float rs_f = 1.0f / sqrtf(__fmaf_rn(tf, 1.0f / kHeadDim, eps));
    const float rs_s = 1.0f / sqrtf(__fmaf_rn(tsum, 1.0f / kHeadDim, eps));
    uint32_t pk[16];
    load_row16(stage, pk, lane);
    qk_rot16(pk, rs_f, w_f + 32 * c0, tc0, ts0);
    stage_row16(stage, pk, lane);
    store_staged(stage, tm_y, xt + 128 * F + 32 * c0, y0, lane);
    load_row16(stage + 2048, pk, lane);
    qk_rot16(pk, rs_f, w_f + 32 * (c0 + 1), tc1, ts1);
    stage_row16(stage + 2048, pk, lane);
    store_staged(stage + 2048, tm_y, xt + 128 * F + 32 * (c0 + 1), y0, lane);
    {
      uint32_t va[32];
      tmem_ld_32x32b_x32(tacc + 128 * S + 32 * c0, va);
      tmem_ld_wait();
      pack32(va, bcol(S, c0), alpha, pk);
    }
    qk_rot16(pk, rs_s, w_s + 32 * c0, tc0, ts0);
    if (lane == 0) bulk_wait_read1();  // the store from buffer 0 has read it
    __syncwarp();
    stage_row16(stage, pk, lane);
    store_staged(stage, tm_y, xt + 128 * S + 32 * c0, y0, lane);
    {
      uint32_t va[32];
      tmem_ld_32x32b_x32(tacc + 128 * S + 32 * (c0 + 1), va);
      tmem_ld_wait();
      pack32(va, bcol(S, c0 + 1), alpha, pk);
    }
    qk_rot16(pk, rs_s, w_s + 32 * (c0 + 1), tc1, ts1);
    if (lane == 0) bulk_wait_read1();
    __syncwarp();
    stage_row16(stage + 2048, pk, lane);
    store_staged(stage + 2048, tm_y, xt + 128 * S + 32 * (c0 + 1), y0, lane);
    return true;
  }
#pragma unroll 1
  for (int k = 0; k < 2; ++k) {  // V: head 1 - F as computed
    uint32_t va[32], pk[16];
    tmem_ld_32x32b_x32(tacc + 128 * S + 32 * (c0 + k), va);
    tmem_ld_wait();
    pack32(va, bcol(S, c0 + k), alpha, pk);
    if (lane == 0) bulk_wait_read1();
    __syncwarp();
    stage_row16(stage + 2048 * k, pk, lane);
    store_staged(stage + 2048 * k, tm_y, xt + 128 * S + 32 * (c0 + k), y0, lane);
  }
  return true;
}

// ------------------------------------------------------------------ MLP up-projection epilogue
constexpr int kMlpRank = 32;  // the down projection's rank the fused epilogue supports
// One 32-column chunk c (columns x0 + 32 c ..) of this lane's row: y, h =
// bf16(GELU(y)), the two NVFP4 blocks of h (the activation quantiser's rule:
// S = e4m3(amax / fp32(6 g)), q = h * fp32(1 / fp32(dec(S) g))), their codes
// and scales stored for the down projection, h added into the XL1 partial
// (part[j] += h_i L1d[x0 + 32 c + i][j]), and h optionally staged for a TMA
// store.
template <int RD>
__device__ __forceinline__ void mlp_chunk(const uint32_t (&v)[32], const __nv_bfloat16* bcol, float alpha, int c,
                                          int x0, int row, int M, int N, const MlpPost& mp, float g, float d,
                                          float (&part)[RD], uint8_t* stage, int& nbuf, const CUtensorMap* tm_y,
                                          int y0, int lane) {
  uint32_t pk[16];
  pack_chunk(v, bcol != nullptr ? bcol + 32 * c : nullptr, alpha, pk);  // y, exactly as the plain epilogue
  float hf[32];
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    const uint32_t hp = pack_bf16(gelu_f32(bf16_lo(pk[p]), mp.approximate != 0),
                                  gelu_f32(bf16_hi(pk[p]), mp.approximate != 0));
    pk[p] = hp;
    hf[2 * p] = bf16_lo(hp);
    hf[2 * p + 1] = bf16_hi(hp);
  }
  const int col = x0 + 32 * c;
  uint32_t words[4];
  uint32_t sc = 0;
#pragma unroll
  for (int blk = 0; blk < 2; ++blk) {
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) am = fmaxf(am, fabsf(hf[16 * blk + i]));
    const uint32_t S = f32_to_e4m3(__fdiv_rn(am, d));
    const float sd = __fmul_rn(e4m3_to_f32(S), g);
    const float inv = (sd == 0.0f || S >= 0x7Fu) ? 0.0f : __frcp_rn(sd);
    float q0[8], q1[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      q0[i] = __fmul_rn(hf[16 * blk + i], inv);
      q1[i] = __fmul_rn(hf[16 * blk + 8 + i], inv);
    }
    words[2 * blk] = f32x8_to_e2m1(q0);
    words[2 * blk + 1] = f32x8_to_e2m1(q1);
    sc |= S << (8 * blk);
  }
  if (row < M) {
    *reinterpret_cast<uint4*>(mp.codes + static_cast<int64_t>(row) * (N / 2) + col / 2) =
        make_uint4(words[0], words[1], words[2], words[3]);
  }
  if (row < mp.m_pad)
    *reinterpret_cast<uint16_t*>(mp.scales + scale_offset(N, row, col / 16)) =
        static_cast<uint16_t>(row < M ? sc : 0u);
  // XL1 partial: the L1 rows of these 32 columns are the same for every lane (broadcast loads);
  // fully unrolled so that hf stays in registers
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint4* lrow = reinterpret_cast<const uint4*>(mp.l1d + static_cast<int64_t>(col + i) * RD);
#pragma unroll
    for (int j8 = 0; j8 < RD / 8; ++j8) {
      float l[8];
      bf16x8_to_f32(__ldg(lrow + j8), l);
#pragma unroll
      for (int e = 0; e < 8; ++e) part[8 * j8 + e] = __fmaf_rn(hf[i], l[e], part[8 * j8 + e]);
    }
  }
  if (mp.store_h) {
    uint8_t* out = stage + 2048 * (nbuf & 1);
    ++nbuf;
    if (lane == 0) bulk_wait_read1();
    __syncwarp();
    stage_row16(out, pk, lane);
    store_staged(out, tm_y, col, y0, lane);
  }
}

// The MLP variant of epilogue_half: the warp's 128-column half in four chunks
// (the shared accumulator columns first, released at once), then its XL1
// partial for rows y0 .. y0 + 31 written to partial slot 2 nt + h.
template <int RD, int FIRST>
__device__ __forceinline__ void epilogue_half_mlp(uint32_t taddr, const __nv_bfloat16* bcol, float alpha,
                                                  uint8_t* stage, int& nbuf, const CUtensorMap* tm_y, int x0, int y0,
                                                  bool holds_overlap, uint32_t ovl_bar, int lane, const MlpPost& mp,
                                                  int M, int N, int slot) {
  const int row = y0 + lane;
  const float g = *mp.g_h;
  const float d = __fmul_rn(6.0f, g);
  float part[RD];
#pragma unroll
  for (int j = 0; j < RD; ++j) part[j] = 0.0f;
  {
    uint32_t va[32], vb[32];
    tmem_ld_32x32b_x32(taddr + 32 * ((FIRST + 0) & 3), va);
    tmem_ld_32x32b_x32(taddr + 32 * ((FIRST + 1) & 3), vb);
    tmem_ld_wait();
    if (holds_overlap) {  // the loads above have completed (tcgen05.wait::ld): nothing else to publish
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(ovl_bar);
    }
    mlp_chunk<RD>(va, bcol, alpha, (FIRST + 0) & 3, x0, row, M, N, mp, g, d, part, stage, nbuf, tm_y, y0, lane);
    mlp_chunk<RD>(vb, bcol, alpha, (FIRST + 1) & 3, x0, row, M, N, mp, g, d, part, stage, nbuf, tm_y, y0, lane);
  }
#pragma unroll 1
  for (int k = 2; k < 4; ++k) {
    uint32_t va[32];
    tmem_ld_32x32b_x32(taddr + 32 * ((FIRST + k) & 3), va);
    tmem_ld_wait();
    mlp_chunk<RD>(va, bcol, alpha, (FIRST + k) & 3, x0, row, M, N, mp, g, d, part, stage, nbuf, tm_y, y0, lane);
  }
  if (row < M) {
    float4* dst = reinterpret_cast<float4*>(mp.partial + (static_cast<int64_t>(slot) * M + row) * RD);
#pragma unroll
    for (int j = 0; j < RD / 4; ++j) dst[j] = make_float4(part[4 * j], part[4 * j + 1], part[4 * j + 2], part[4 * j + 3]);
  }
}

// Sums the XL1 partials of an MLP up projection in slot order:
// xl1[m][j] = bf16(sum_p partial[p][m][j]) (fp32, p ascending: deterministic).
__global__ void mlp_xl1_reduce_kernel(const float* __restrict__ partial, int slots, int M, int rd,
                                      __nv_bfloat16* __restrict__ xl1) {
  const int64_t total = static_cast<int64_t>(M) * rd;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = 0.0f;
    for (int p = 0; p < slots; ++p) s = __fadd_rn(s, partial[p * total + i]);
    xl1[i] = __float2bfloat16_rn(s);
  }
}

template <int R, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(k2Threads, 1) w4a4_gemm_2sm_kernel(
    const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
    const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
    const __grid_constant__ CUtensorMap tm_xl1, const __grid_constant__ CUtensorMap tm_l2s,
    const __grid_constant__ CUtensorMap tm_y, const float* __restrict__ gscale,
    const __nv_bfloat16* __restrict__ bias, int M, int N, int K, const QkvPost post, const MlpPost mlp) {
  using C = Gemm2Cfg<R, EPI>;
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

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->acc_full[b], 1);
      mbar_init(&bars->acc_empty[b], 16);  // 8 epilogue warps x 2 CTAs
    }
    mbar_init(&bars->ovl_free, 8);         // 4 warps (the half holding the shared columns) x 2 CTAs
    mbar_init(&bars->teardown, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&bars->xchg[i], 64);
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        const int mt = tile % num_mt, nt = tile / num_mt;
        const int m_own = mt * k2TileM + static_cast<int>(rank) * 128;
        const int n_own = nt * k2TileN + static_cast<int>(rank) * 128;
        const int nblk = nt * 2;  // first 128-row block of B in this tile
        for (int step = 0; step < steps; ++step) {
          if (!mbar_wait(&bars->empty[s], ph ^ 1, abort)) { ok = false; break; }
          uint8_t* st = smem + s * C::kStageBytes;
          const uint32_t bar = mapa_shared(smem_u32(&bars->full[s]), 0);
          if (step < C::kLrSteps) {
            if (rank == 0) mbar_arrive_expect_tx(&bars->full[s], C::kLrTx);
            const int x = step * C::kLrCols;
            tma_load_2d_cg2(st, &tm_xl1, x, m_own, bar);
            tma_load_2d_cg2(st + C::kABytes, &tm_l2s, x, n_own, bar);
            tma_load_2d_cg2(st + C::kABytes + C::kLrTileBytes, &tm_l2s, x, N + n_own, bar);
          } else {
            const int kb = step - C::kLrSteps;
            if (rank == 0) mbar_arrive_expect_tx(&bars->full[s], C::kMainTx);
            tma_load_2d_cg2(st, &tm_a, kb * 128, m_own, bar);
            tma_load_2d_cg2(st + C::kABytes, &tm_b, kb * 128, n_own, bar);
            uint8_t* sf = st + C::kABytes + C::kBBytes;
            tma_load_4d_cg2(sf, &tm_sfa, 0, 0, 0, (m_own / 128) * sf_row_stride + 4 * kb, bar);
            tma_load_5d_cg2(sf + C::kSfaBytes, &tm_sfb, 0, 0, 0, 4 * kb, nblk, bar);
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
      const uint32_t t_sfa = tmem + k2SfaCol;
      const uint32_t t_sfb = tmem + k2SfbCol;
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs, ++it) {
        const int b = it & 1;
        const uint32_t t_acc = tmem + (b ? k2Acc1Col : 0);
        if (!mbar_wait_cluster(&bars->acc_empty[b], ((it >> 1) & 1) ^ 1, abort)) { ok = false; break; }
        if (it > 0 && !mbar_wait_cluster(&bars->ovl_free, (it - 1) & 1, abort)) { ok = false; break; }
        tc_fence_after();
        for (int step = 0; step < steps; ++step) {
          if (!mbar_wait(&bars->full[s], ph, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * C::kStageBytes);
          if (step < C::kLrSteps) {
#pragma unroll
            for (int k16 = 0; k16 < C::kLrCols / 16; ++k16) {
              const uint64_t a = smem_desc(st + 32 * k16, 16, 8 * C::kLrRowBytes, C::kLrSwizzle);
              const uint64_t bh = smem_desc(st + C::kABytes + 32 * k16, 16, 8 * C::kLrRowBytes, C::kLrSwizzle);
              const uint64_t bl =
                  smem_desc(st + C::kABytes + C::kLrTileBytes + 32 * k16, 16, 8 * C::kLrRowBytes, C::kLrSwizzle);
              mma_bf16_cg2(t_acc, a, bh, idesc_bf16, (step | k16) != 0 ? 1u : 0u);
              mma_bf16_cg2(t_acc, a, bl, idesc_bf16, 1u);
            }
          } else {
            const uint32_t sfa = st + C::kABytes + C::kBBytes;
            const uint32_t sfb = sfa + C::kSfaBytes;
            // A: K-steps (0,1) and (2,3), 2 KB apart; B: K-step j, row blocks 8 KB apart
            tmem_cp_128x256b_cg2(t_sfa, smem_desc(sfa, 2048, 128, kSwizzleNone));
            tmem_cp_128x256b_cg2(t_sfa + 8, smem_desc(sfa + 4096, 2048, 128, kSwizzleNone));
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tmem_cp_128x256b_cg2(t_sfb + 8 * j, smem_desc(sfb + 2048 * j, 8192, 128, kSwizzleNone));
            const uint64_t adesc = smem_desc(st, 16, 1024, kSwizzle128B);
            const uint64_t bdesc = smem_desc(st + C::kABytes, 16, 1024, kSwizzle128B);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              mma_nvf4_cg2(t_acc, adesc + 2 * j, bdesc + 2 * j, idesc_fp4, t_sfa + 4 * j, t_sfb + 8 * j, 1u);
          }
          tc_commit_cg2_mc(&bars->empty[s], 0x3);
          if (++s == S) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        tc_commit_cg2_mc(&bars->acc_full[b], 0x3);
      }
      // every MMA this thread issued completes before TMEM is released
      tc_commit(&bars->teardown);
      volatile int never = 0;
      mbar_wait(&bars->teardown, 0, &never);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int e = warp - 2;
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int h = e >> 2;    // 128-column half of the tile
    const float alpha = gscale[2];
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    const uint32_t ovl_bar = mapa_shared(smem_u32(&bars->ovl_free), 0);
    uint8_t* stage = smem + C::kOutOff + e * C::kOutPerWarp;
    int nbuf = 0;
    uint32_t nx = 0;  // fused QKV: exchanges of row sums done by this warp
    int it = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs, ++it) {
      const int mt = tile % num_mt, nt = tile / num_mt;
      const int b = it & 1;
      const int y0 = mt * k2TileM + static_cast<int>(rank) * 128 + 32 * q;
      const int col0 = nt * k2TileN + 128 * h;
      if constexpr (QKV) {
        // Q / K tiles: this lane's rotary angles for the warp's first chunk,
        // fetched before the accumulator is ready. A tile is all Q/K or all V (the
        // V block starts at 2 * hd, a multiple of 256).
        const int xt = nt * k2TileN;
        const bool qk = xt < 2 * post.hd;
        float tc0[16], ts0[16];
        const int64_t row = (y0 + lane < M) ? y0 + lane : M - 1;
        const float* cr = post.cos + row * post.ld_rope + 32 * h;
        const float* sr = post.sin + row * post.ld_rope + 32 * h;
        if (qk) {
          load_angles16(cr, sr, tc0, ts0);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) tc0[i] = ts0[i] = 0.0f;
        }
        const __nv_bfloat16* w0 = qk ? (xt < post.hd ? post.w_q : post.w_k) : nullptr;
        const __nv_bfloat16* w1 = qk ? (xt + 128 < post.hd ? post.w_q : post.w_k) : nullptr;
        if (!mbar_wait(&bars->acc_full[b], (it >> 1) & 1, abort)) break;
        tc_fence_after();
        const uint32_t tacc = lane_base + (b ? k2Acc1Col : 0);
        const __nv_bfloat16* btile = bias != nullptr ? bias + xt : nullptr;
        float* xs = reinterpret_cast<float*>(smem + C::kXchgOff) + 128 * (2 * q + h) + 64 * (nx & 1);
        const float* xp = reinterpret_cast<const float*>(smem + C::kXchgOff) + 128 * (2 * q + (h ^ 1)) + 64 * (nx & 1);
        // accumulator 0's shared columns lie in head 1 (warp 1's chunks),
        // accumulator 1's in head 0 (warp 0's chunks)
        const bool ok = epilogue_qkv_tile(tacc, b == 0 ? 1 : 0, h, btile, alpha, stage, &tm_y, xt, y0, h == (b == 0),
                                          ovl_bar, lane, b == 0 ? w1 : w0, b == 0 ? w0 : w1, tc0, ts0, cr + 16, sr + 16, xs, xp, &bars->xchg[q], nx & 1,
                                          post.eps, abort);
        if (!ok) break;
        if (qk) ++nx;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&bars->acc_empty[b]), 0));
        continue;
      }
      if constexpr (EPI == 2) {
        if (!mbar_wait(&bars->acc_full[b], (it >> 1) & 1, abort)) break;
        tc_fence_after();
        const uint32_t acc = lane_base + (b ? k2Acc1Col : 0) + 128 * h;
        const __nv_bfloat16* bcol = bias != nullptr ? bias + col0 : nullptr;
        const int slot = 2 * nt + h;
        if (b == 0 && h == 1)
          epilogue_half_mlp<kMlpRank, 2>(acc, bcol, alpha, stage, nbuf, &tm_y, col0, y0, true, ovl_bar, lane, mlp, M,
                                         N, slot);
        else
          epilogue_half_mlp<kMlpRank, 0>(acc, bcol, alpha, stage, nbuf, &tm_y, col0, y0, b == 1 && h == 0, ovl_bar,
                                         lane, mlp, M, N, slot);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&bars->acc_empty[b]), 0));
        continue;
      }
      // bias of this warp's 128 columns, fetched before the accumulator is ready
      uint4 bv[16];
      if (bias != nullptr) {
#pragma unroll
        for (int i = 0; i < 16; ++i) bv[i] = ldg_v4(bias + col0 + 8 * i);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) bv[i] = make_uint4(0u, 0u, 0u, 0u);
      }
      if (!mbar_wait(&bars->acc_full[b], (it >> 1) & 1, abort)) break;
      tc_fence_after();
      const uint32_t acc = lane_base + (b ? k2Acc1Col : 0) + 128 * h;
      if (b == 0 && h == 1)
        epilogue_half<2>(acc, bv, alpha, stage, nbuf, &tm_y, col0, y0, true, ovl_bar, lane);
      else
        epilogue_half<0>(acc, bv, alpha, stage, nbuf, &tm_y, col0, y0, b == 1 && h == 0, ovl_bar, lane);
      tc_fence_before();
      __syncwarp();
      // every TMEM load of this accumulator has completed; the MMAs read nothing this warp wrote
      if (lane == 0) mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&bars->acc_empty[b]), 0));
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
