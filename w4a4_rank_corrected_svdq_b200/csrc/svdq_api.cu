// svdq_api.cu — the C ABI (include/svdq.h): argument validation, device
// checks, tensor-map encoding and kernel launches. One translation unit holds
// every kernel so the per-device error word is a single symbol.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/svdq.h"
#include "gemm_w4a4.cuh"
#include "gemm_w4a4_2sm.cuh"
#include "gemm_w4a4_splitk.cuh"
#include "lowrank_svd.cuh"
#include "pack_weight.cuh"
#include "smooth.cuh"
#include "awq_w4a16.cuh"
#include "quantize_act.cuh"

#include <nvtx3/nvToolsExt.h>

namespace svdq {
namespace {

constexpr int kVersion = 100;  // 0.1.0

// NVTX range around one entry point (for timeline profilers; a no-op when no
// tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool valid_rank(int r) { return r == 16 || r == 32 || r == 64 || r == 128; }
size_t round_up(size_t x, size_t m) { return (x + m - 1) / m * m; }

// ------------------------------------------------------------------ device checks
}  // namespace
}  // namespace svdq

// The kernels are built for sm_100a (tcgen05, TMEM, mxf4nvf4 block-scaled MMA):
// compute capability 10.0 exactly.
extern "C" svdq_status svdq_device_supported(int major, int minor) {
  return (major == 10 && minor == 0) ? SVDQ_OK : SVDQ_ERR_UNSUPPORTED_DEVICE;
}

namespace svdq {
namespace {
struct DeviceInfo {
  int sm_count = 0;
  int ok = -1;  // -1 unknown, 0 unsupported, 1 supported
};
constexpr int kMaxDevices = 64;
DeviceInfo g_devices[kMaxDevices];
std::mutex g_dev_mutex;

svdq_status current_device(int* dev_out, DeviceInfo* info_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_UNSUPPORTED_DEVICE;
  }
  if (dev < 0 || dev >= kMaxDevices) return SVDQ_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceInfo& di = g_devices[dev];
  if (di.ok < 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return SVDQ_ERR_UNSUPPORTED_DEVICE;
    }
    di.sm_count = sms;
    di.ok = svdq_device_supported(major, minor) == SVDQ_OK ? 1 : 0;
  }
  if (di.ok != 1) return SVDQ_ERR_UNSUPPORTED_DEVICE;
  if (dev_out) *dev_out = dev;
  if (info_out) *info_out = di;
  return SVDQ_OK;
}

// cudaFuncSetAttribute for the dynamic shared memory size, once per (kernel, device).
template <typename Kernel>
void ensure_smem_attr(Kernel kern, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  // Every kernel here stages through shared memory and barely uses L1: ask for
  // the largest shared-memory carveout so that the occupancy queries (and the
  // launches) count every CTA that fits.
  cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  done.fetch_or(bit, std::memory_order_acq_rel);
}

// cudaOccupancyMaxActiveClusters costs far more host time than a launch; its
// answer depends only on (kernel, device, cluster size, dynamic shared memory),
// so each answer is kept. A full table simply stops caching.
class ClusterOccupancyCache {
 public:
  template <typename Kernel>
  int get(Kernel kern, cudaLaunchConfig_t* cfg, int dev) {
    const uint64_t key = (static_cast<uint64_t>(dev & 0xFF) << 56) |
                         (static_cast<uint64_t>(cfg->attrs[0].val.clusterDim.x & 0xFF) << 48) |
                         (static_cast<uint64_t>(cfg->dynamicSmemBytes) & 0xFFFFFFFFull);
    {
      std::lock_guard<std::mutex> lock(mu_);
      for (int i = 0; i < n_; ++i)
        if (keys_[i] == key) return vals_[i];
    }
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, cfg) != cudaSuccess) {
      cudaGetLastError();
      clusters = 0;
    }
    std::lock_guard<std::mutex> lock(mu_);
    if (n_ < kSlots) {
      keys_[n_] = key;
      vals_[n_] = clusters;
      ++n_;
    }
    return clusters;
  }

 private:
  static constexpr int kSlots = 64;
  uint64_t keys_[kSlots] = {};
  int vals_[kSlots] = {};
  int n_ = 0;
  std::mutex mu_;
};

// Launch attributes for a kernel that may start while the previous kernel of
// the stream is finishing (programmatic dependent launch); the kernel itself
// waits (griddepcontrol.wait) before touching global memory.
struct PdlLaunch {
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = {};
  PdlLaunch(dim3 grid, dim3 block, size_t smem, cudaStream_t st) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
};

svdq_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    std::fprintf(stderr, "svdq: CUDA error: %s\n", cudaGetErrorString(e));
    return SVDQ_ERR_CUDA;
  }
  return SVDQ_OK;
}

// ------------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// 2-D row-major tensor [rows][cols] of `elem_bytes` elements, row pitch `pitch_bytes`.
bool make_tmap_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t cols,
                  uint64_t rows, uint64_t pitch_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  (void)elem_bytes;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map of rank 2..5 over bytes or bf16 (dims / strides in elements / bytes).
bool make_tmap(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int rank, const uint64_t* dims,
               const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[5];
  cuuint64_t st[4];
  cuuint32_t b[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides_bytes[i];
  }
  return fn(m, dt, rank, const_cast<void*>(base), d, st, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Scale atoms (512 B) read four times each through a zero-stride dimension:
// SFA: {256 B, 2 halves, 4 replicas, atoms}; box = 4 consecutive atoms (one
// 256-wide K block of one 128-row block). SFB adds the row-block dimension;
// box = 4 atoms of two consecutive 128-row blocks.
bool make_sf_tmaps(CUtensorMap* sfa, const void* a_scales, uint64_t a_rows_pad, CUtensorMap* sfb,
                   const void* w_scales, uint64_t n_rows, int K) {
  const uint64_t atoms_per_rb = static_cast<uint64_t>(K / 64);
  const uint64_t da[4] = {256, 2, 4, (a_rows_pad / 128) * atoms_per_rb};
  const uint64_t sa[3] = {256, 0, 512};
  const uint32_t ba[4] = {256, 2, 4, 4};
  const uint64_t db[5] = {256, 2, 4, atoms_per_rb, n_rows / 128};
  const uint64_t sb[4] = {256, 0, 512, atoms_per_rb * 512};
  const uint32_t bb[5] = {256, 2, 4, 4, 2};
  return make_tmap(sfa, a_scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, da, sa, ba, CU_TENSOR_MAP_SWIZZLE_NONE) &&
         make_tmap(sfb, w_scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, db, sb, bb, CU_TENSOR_MAP_SWIZZLE_NONE);
}

CUtensorMapSwizzle lr_swizzle(int r) {
  const int row_bytes = (r < 64 ? r : 64) * 2;
  return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : (row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

// ------------------------------------------------------------------ launches
// Launch plan of the quantiser: row-tile height (64 or 128) and K-split ks
// (CTAs per cluster).
struct QuantPlan {
  int rows = 128;
  int ks = 1;
};

// Is (ROWS, ks) a one-wave grid of at most one CTA per SM whose clusters are
// all resident at once? Clusters are placed within a GPC, so at about one CTA
// per SM a few clusters may find no whole free group of SMs and then share SMs
// with running CTAs (*shares = true), which needs two CTAs' shared memory to
// fit an SM (registers are bounded for two CTAs by __launch_bounds__).
// cudaOccupancyMaxActiveClusters counts one CTA per SM for any kernel that
// allocates tensor memory: on B200 it reports 33 clusters of four, yet 36
// start together when two CTAs' shared memory fits an SM.
template <int R, int ROWS>
bool quant_candidate(int M, int K, int ks, int sm_count, int dev, bool* shares) {
  static ClusterOccupancyCache occupancy;
  const int tiles = (M + ROWS - 1) / ROWS;
  if (K % (kQuantStep * ks) != 0 || tiles * ks > sm_count) return false;
  const size_t smem = quantize_smem_bytes<R, ROWS>(K / ks);
  if (smem > 227 * 1024) return false;
  *shares = false;
  if (ks == 1) return true;
  auto kern = quantize_act_kernel<R, ROWS, false>;
  static std::atomic<uint64_t> attr_done{0};
  ensure_smem_attr(kern, 227 * 1024, attr_done);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = ks;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.blockDim = dim3(kQuantThreads, 1, 1);
  cfg.gridDim = dim3(ks, tiles, 1);
  cfg.dynamicSmemBytes = smem;
  if (occupancy.get(kern, &cfg, dev) >= tiles) return true;
  *shares = true;
  return 2 * (smem + 1024) <= 228 * 1024;
}

// Most CTAs (up to one per SM) wins; ties go to the taller tile (fewer L1^T
// tile reloads and half the steps: on B200, 36 x 128-row tiles split four ways
// run 10 % faster than 72 x 64-row tiles split two ways although three of
// their clusters share SMs). With
// no one-wave plan (very large M, or K too long for the shared-memory
// staging) the smallest K-split whose shared memory fits, 128-row tiles.
// SVDQ_QUANT_PLAN="rows,ks" (tests, benchmarks) forces a plan when K splits
// into whole 64-column steps and its shared memory fits; otherwise it is
// ignored.
template <int R>
QuantPlan plan_quantize(int M, int K, int sm_count) {
  int dev = 0;
  cudaGetDevice(&dev);
  QuantPlan best;
  if (const char* env = std::getenv("SVDQ_QUANT_PLAN")) {
    int rows = 0, ks = 0;
    if (std::sscanf(env, "%d,%d", &rows, &ks) == 2 && (rows == 64 || rows == 128) &&
        (ks == 1 || ks == 2 || ks == 4 || ks == 8) && K % (kQuantStep * ks) == 0) {
      const size_t smem =
          rows == 64 ? quantize_smem_bytes<R, 64>(K / ks) : quantize_smem_bytes<R, 128>(K / ks);
      if (smem <= 227 * 1024) {
        best.rows = rows;
        best.ks = ks;
        return best;
      }
    }
  }
  long best_score = -1;
  for (int rows : {128, 64})
    for (int ks : {1, 2, 4, 8}) {
      bool shares = false;  // clusters may share SMs; measured not to cost more than the extra steps
      const bool ok = rows == 128 ? quant_candidate<R, 128>(M, K, ks, sm_count, dev, &shares)
                                  : quant_candidate<R, 64>(M, K, ks, sm_count, dev, &shares);
      if (!ok) continue;
      const long ctas = static_cast<long>((M + rows - 1) / rows) * ks;
      const long score = ctas;
      if (score > best_score) {
        best_score = score;
        best.rows = rows;
        best.ks = ks;
      }
    }
  if (best_score < 0) {
    best.rows = 128;
    best.ks = 1;
    while (best.ks < 8 && K % (kQuantStep * best.ks * 2) == 0 &&
           quantize_smem_bytes<R, 128>(K / best.ks) > 227 * 1024)
      best.ks *= 2;
  }
  return best;
}

template <int R, int ROWS>
svdq_status launch_quantize(int M, int K, int ks, const void* X, int64_t ldx, const float* g_x, const void* l1t,
                            const float* inv_smooth, void* codes, void* scales, void* xl1, cudaStream_t stream,
                            bool pdl, const DynScale& dyn) {
  const int row_tiles = (M + ROWS - 1) / ROWS;
  const int kchunk = K / ks;
  const size_t smem = quantize_smem_bytes<R, ROWS>(kchunk);
  if (smem > 227 * 1024) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  auto kern = inv_smooth != nullptr ? quantize_act_kernel<R, ROWS, true> : quantize_act_kernel<R, ROWS, false>;
  static std::atomic<uint64_t> attr_done[2] = {};
  ensure_smem_attr(kern, 227 * 1024, attr_done[inv_smooth != nullptr]);
  CUtensorMap tm_x, tm_l;
  if (!make_tmap_2d(&tm_x, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, M, static_cast<uint64_t>(ldx) * 2, 64, ROWS,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tm_l, l1t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, R, static_cast<uint64_t>(K) * 2, 64, R,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return SVDQ_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kQuantThreads, 1, 1);
  cfg.gridDim = dim3(ks, row_tiles, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = ks;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // pdl: a programmatic dependent of the previous kernel on the stream (the
  // kernel reads g_x only after griddepcontrol.wait).
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  cudaLaunchKernelEx(&cfg, kern, tm_x, tm_l, M, K, g_x, inv_smooth, static_cast<uint8_t*>(codes),
                     static_cast<uint8_t*>(scales), static_cast<__nv_bfloat16*>(xl1), kchunk, dyn);
  return launch_status();
}

template <int R>
svdq_status launch_quantize_planned(int M, int K, const void* X, int64_t ldx, const float* g_x, const void* l1t,
                                    const float* inv_smooth, void* codes, void* scales, void* xl1, cudaStream_t st,
                                    int sms, bool pdl, const DynScale& dyn) {
  const QuantPlan plan = plan_quantize<R>(M, K, sms);
  if (plan.rows == 64)
    return launch_quantize<R, 64>(M, K, plan.ks, X, ldx, g_x, l1t, inv_smooth, codes, scales, xl1, st, pdl, dyn);
  return launch_quantize<R, 128>(M, K, plan.ks, X, ldx, g_x, l1t, inv_smooth, codes, scales, xl1, st, pdl, dyn);
}

// dyn: the per-call scale (svdq_linear_forward_dynamic), or none (g from g_x).
svdq_status quantize_dispatch(int M, int K, int r, const void* X, int64_t ldx, const float* g_x, const void* l1t,
                              const float* inv_smooth, void* codes, void* scales, void* xl1, cudaStream_t st,
                              int sms, bool pdl = false, const DynScale& dyn = DynScale{}) {
#define SVDQ_Q_ARGS M, K, X, ldx, g_x, l1t, inv_smooth, codes, scales, xl1, st, sms, pdl, dyn
  switch (r) {
    case 16: return launch_quantize_planned<16>(SVDQ_Q_ARGS);
    case 32: return launch_quantize_planned<32>(SVDQ_Q_ARGS);
    case 64: return launch_quantize_planned<64>(SVDQ_Q_ARGS);
    default: return launch_quantize_planned<128>(SVDQ_Q_ARGS);
  }
#undef SVDQ_Q_ARGS
}

template <int R, bool QKV>
svdq_status launch_gemm(int M, int N, int K, const void* a_codes, const void* a_scales, const void* xl1,
                        const void* w_codes, const void* w_scales, const float* gscale, const void* l2s,
                        const void* bias, void* Y, int64_t ldy, cudaStream_t stream, int sm_count,
                        const QkvPost& post) {
  using C = GemmCfg<R>;
  CUtensorMap tm_a, tm_b, tm_x, tm_l;
  const uint64_t kb = static_cast<uint64_t>(K / 2);
  if (!make_tmap_2d(&tm_a, a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kb, M, kb, kBKBytes, kBM,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tm_b, w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kb, N, kb, kBKBytes, kBN,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tm_x, xl1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, R, M, R * 2, C::kLrAtomCols, kBM,
                    lr_swizzle(R)) ||
      !make_tmap_2d(&tm_l, l2s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, R, 2 * static_cast<uint64_t>(N), R * 2,
                    C::kLrAtomCols, kBN, lr_swizzle(R)))
    return SVDQ_ERR_CUDA;
  auto kern = w4a4_gemm_kernel<R, QKV>;
  static std::atomic<uint64_t> attr_done{0};
  ensure_smem_attr(kern, C::kSmemBytes, attr_done);
  const int tiles = ((M + kBM - 1) / kBM) * (N / kBN);
  const int grid = tiles < sm_count ? tiles : sm_count;
  PdlLaunch pl(dim3(grid), dim3(kGemmThreads), C::kSmemBytes, stream);
  cudaLaunchKernelEx(&pl.cfg, kern, tm_a, tm_b, tm_x, tm_l, static_cast<const uint8_t*>(a_scales),
                     static_cast<const uint8_t*>(w_scales), gscale, static_cast<const __nv_bfloat16*>(bias),
                     static_cast<__nv_bfloat16*>(Y), ldy, M, N, K, post);
  return launch_status();
}

// K split of the few-row GEMM: the largest KS in {8, 4, 2} that divides the
// K blocks and keeps one CTA per SM for every tile's cluster; 1 = no split.
// Opt-in (SVDQ_GEMM_SPLITK=1): on B200 it measured slower than one CTA per
// tile for the few-row layers (the cluster exchange costs more than the split
// saves at these sizes).
int gemm_split(int M, int N, int K, int sm_count) {
  const char* env = std::getenv("SVDQ_GEMM_SPLITK");
  if (env == nullptr || std::strcmp(env, "1") != 0) return 1;
  const int tiles = ((M + kBM - 1) / kBM) * (N / kBN);
  const int nk = K / 256;
  for (int ks = kSplitMaxKS; ks >= 2; ks /= 2)
    if (nk % ks == 0 && tiles * ks <= sm_count) return ks;
  return 1;
}

template <int R>
svdq_status launch_gemm_splitk(int M, int N, int K, int ks, const void* a_codes, const void* a_scales,
                               const void* xl1, const void* w_codes, const void* w_scales, const float* gscale,
                               const void* l2s, const void* bias, void* Y, int64_t ldy, cudaStream_t stream) {
  using C = SplitCfg<R>;
  CUtensorMap tm_a, tm_b, tm_x, tm_l;
  const uint64_t kb = static_cast<uint64_t>(K / 2);
  if (!make_tmap_2d(&tm_a, a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kb, M, kb, kBKBytes, kBM,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tm_b, w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kb, N, kb, kBKBytes, kBN,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tm_x, xl1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, R, M, R * 2, C::kLrAtomCols, kBM,
                    lr_swizzle(R)) ||
      !make_tmap_2d(&tm_l, l2s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, R, 2 * static_cast<uint64_t>(N), R * 2,
                    C::kLrAtomCols, kBN, lr_swizzle(R)))
    return SVDQ_ERR_CUDA;
  auto kern = w4a4_gemm_splitk_kernel<R>;
  static std::atomic<uint64_t> attr_done{0};
  ensure_smem_attr(kern, C::kSmemBytes, attr_done);
  const int tiles = ((M + kBM - 1) / kBM) * (N / kBN);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = ks;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cfg.blockDim = dim3(kSplitThreads, 1, 1);
  cfg.gridDim = dim3(ks, tiles, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchKernelEx(&cfg, kern, tm_a, tm_b, tm_x, tm_l, static_cast<const uint8_t*>(a_scales),
                     static_cast<const uint8_t*>(w_scales), gscale, static_cast<const __nv_bfloat16*>(bias),
                     static_cast<__nv_bfloat16*>(Y), ldy, M, N, K);
  return launch_status();
}

// CTA pairs the 2-SM GEMM launches: one per tile, at most one per two SMs.
int gemm2_pairs(int M, int N, int sm_count) {
  const int tiles = ((M + k2TileM - 1) / k2TileM) * (N / k2TileN);
  const int max_pairs = sm_count / 2;
  return tiles < max_pairs ? tiles : max_pairs;
}

template <int R, int EPI>
svdq_status launch_gemm_2sm(int M, int N, int K, const void* a_codes, const void* a_scales, const void* xl1,
                            const void* w_codes, const void* w_scales, const float* gscale, const void* l2s,
                            const void* bias, void* Y, int64_t ldy, cudaStream_t stream, int sm_count,
                            const QkvPost& post, const MlpPost& mlp, const void* l1t_down) {
  using C = Gemm2Cfg<R, EPI, false>;
  CUtensorMap tm_a, tm_b, tm_sfa, tm_sfb, tm_x, tm_l, tm_y, tm_l1d;
  const uint64_t kb = static_cast<uint64_t>(K / 2);
  const uint64_t mpad = round_up(static_cast<size_t>(M), 128);
  const CUtensorMapSwizzle lr_sw = C::kLrRowBytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  if (!make_tmap_2d(&tm_a, a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kb, M, kb, 128, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tm_b, w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kb, N, kb, 128, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_sf_tmaps(&tm_sfa, a_scales, mpad, &tm_sfb, w_scales, static_cast<uint64_t>(N), K) ||
      !make_tmap_2d(&tm_x, xl1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, R, M, R * 2, C::kLrCols, 128, lr_sw) ||
      !make_tmap_2d(&tm_l, l2s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, R, 2 * static_cast<uint64_t>(N), R * 2,
                    C::kLrCols, 128, lr_sw) ||
      // the plain and fused QKV epilogues store 32 rows x 32 columns (64-byte swizzle), the MLP one 32 x 64 (128-byte)
      !make_tmap_2d(&tm_y, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, M, static_cast<uint64_t>(ldy) * 2,
                    EPI == 2 ? 64 : 32, 32, EPI == 2 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
    return SVDQ_ERR_CUDA;
  // MLP: L1_down^T [32][N] (bf16, row pitch 2N), boxes of 16 rows x 64 columns; otherwise unused
  if (EPI == 2) {
    if (!make_tmap_2d(&tm_l1d, l1t_down, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, kMlpRank,
                      static_cast<uint64_t>(N) * 2, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B))
      return SVDQ_ERR_CUDA;
  } else {
    tm_l1d = tm_y;
  }
  // the plain layer takes the four-stage layout when its A scales stay in TMEM
  using CL = Gemm2Cfg<R, 0, true>;
  const bool lean = EPI == 0 && K / 256 <= CL::kSfaSlots;
  auto kern = lean ? w4a4_gemm_2sm_kernel<R, EPI, EPI == 0> : w4a4_gemm_2sm_kernel<R, EPI, false>;
  const int smem = lean ? CL::kSmemBytes : C::kSmemBytes;
  static std::atomic<uint64_t> attr_done[2] = {};
  ensure_smem_attr(kern, smem, attr_done[lean ? 1 : 0]);
  const int pairs = gemm2_pairs(M, N, sm_count);
  PdlLaunch pl(dim3(2 * pairs), dim3(C::kThreads), smem, stream);
  cudaLaunchKernelEx(&pl.cfg, kern, tm_a, tm_b, tm_sfa, tm_sfb, tm_x, tm_l, tm_y, tm_l1d, gscale,
                     static_cast<const __nv_bfloat16*>(bias), M, N, K, post, mlp);
  return launch_status();
}

// Kernel choice: CTA-pair 256x256 tiles when N is a multiple of 256 and there
// are enough rows to keep most SM pairs busy; otherwise single-CTA 128x128
// tiles. SVDQ_GEMM_KERNEL=1sm|2sm overrides the choice (tests, benchmarks).
bool use_2sm(int M, int N) {
  if (N % 256 != 0) return false;
  const char* env = std::getenv("SVDQ_GEMM_KERNEL");
  if (env != nullptr) {
    if (std::strcmp(env, "2sm") == 0) return true;
    if (std::strcmp(env, "1sm") == 0) return false;
  }
  return M >= 512;
}

// The plain layer, or with post the fused QKV post-processing, or with mlp the
// MLP up projection (CTA-pair GEMM only).
svdq_status gemm_dispatch(int M, int N, int K, int r, const void* a_codes, const void* a_scales, const void* xl1,
                          const void* w_codes, const void* w_scales, const float* gscale, const void* l2s,
                          const void* bias, void* Y, int64_t ldy, cudaStream_t st, int sms,
                          const QkvPost* post = nullptr, const MlpPost* mlp = nullptr,
                          const void* l1t_down = nullptr) {
  const QkvPost none{};
  const QkvPost& pp = post != nullptr ? *post : none;
  const MlpPost mnone{};
  const MlpPost& mp = mlp != nullptr ? *mlp : mnone;
  if (mlp != nullptr) {  // the MLP up-projection epilogue exists for the CTA-pair GEMM only
    if (N % 256 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
#define SVDQ_GEMM2_ARGS M, N, K, a_codes, a_scales, xl1, w_codes, w_scales, gscale, l2s, bias, Y, ldy, st, sms, pp, mp, \
                        l1t_down
    switch (r) {
      case 16: return launch_gemm_2sm<16, 2>(SVDQ_GEMM2_ARGS);
      case 32: return launch_gemm_2sm<32, 2>(SVDQ_GEMM2_ARGS);
      case 64: return launch_gemm_2sm<64, 2>(SVDQ_GEMM2_ARGS);
      default: return launch_gemm_2sm<128, 2>(SVDQ_GEMM2_ARGS);
    }
  }
#define SVDQ_GEMM_ARGS M, N, K, a_codes, a_scales, xl1, w_codes, w_scales, gscale, l2s, bias, Y, ldy, st, sms, pp
#define SVDQ_GEMM_CASES(F, Q)                 \
  switch (r) {                                \
    case 16: return F<16, Q>(SVDQ_GEMM_ARGS); \
    case 32: return F<32, Q>(SVDQ_GEMM_ARGS); \
    case 64: return F<64, Q>(SVDQ_GEMM_ARGS); \
    default: return F<128, Q>(SVDQ_GEMM_ARGS); \
  }
  if (use_2sm(M, N)) {
    if (post != nullptr) {
      switch (r) {
        case 16: return launch_gemm_2sm<16, 1>(SVDQ_GEMM2_ARGS);
        case 32: return launch_gemm_2sm<32, 1>(SVDQ_GEMM2_ARGS);
        case 64: return launch_gemm_2sm<64, 1>(SVDQ_GEMM2_ARGS);
        default: return launch_gemm_2sm<128, 1>(SVDQ_GEMM2_ARGS);
      }
    }
    switch (r) {
      case 16: return launch_gemm_2sm<16, 0>(SVDQ_GEMM2_ARGS);
      case 32: return launch_gemm_2sm<32, 0>(SVDQ_GEMM2_ARGS);
      case 64: return launch_gemm_2sm<64, 0>(SVDQ_GEMM2_ARGS);
      default: return launch_gemm_2sm<128, 0>(SVDQ_GEMM2_ARGS);
    }
  }
  if (post != nullptr) SVDQ_GEMM_CASES(launch_gemm, true)
  // few rows: K split across a cluster when that fills more SMs (16-byte aligned bias)
  const int ks = gemm_split(M, N, K, sms);
  if (ks > 1 && (bias == nullptr || (reinterpret_cast<uintptr_t>(bias) & 15u) == 0)) {
#define SVDQ_SPLIT_ARGS M, N, K, ks, a_codes, a_scales, xl1, w_codes, w_scales, gscale, l2s, bias, Y, ldy, st
    switch (r) {
      case 16: return launch_gemm_splitk<16>(SVDQ_SPLIT_ARGS);
      case 32: return launch_gemm_splitk<32>(SVDQ_SPLIT_ARGS);
      case 64: return launch_gemm_splitk<64>(SVDQ_SPLIT_ARGS);
      default: return launch_gemm_splitk<128>(SVDQ_SPLIT_ARGS);
    }
#undef SVDQ_SPLIT_ARGS
  }
  SVDQ_GEMM_CASES(launch_gemm, false)
#undef SVDQ_GEMM_CASES
#undef SVDQ_GEMM_ARGS
#undef SVDQ_GEMM2_ARGS
}

// max |fp32(x * inv[col + j])| (or |x|) over one 16-byte vector of 8 bf16.
__device__ __forceinline__ float vec_amax(const __nv_bfloat16* p, const float* __restrict__ inv, int col, float am) {
  float f[8];
  bf16x8_to_f32(ldg_nc_v4(p), f);
  if (inv != nullptr) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(inv + col));
    const float4 b = __ldg(reinterpret_cast<const float4*>(inv + col) + 1);
    const float s8[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = __fmul_rn(f[j], s8[j]);
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) am = fmaxf(am, fabsf(f[j]));
  return am;
}

// amax|X^| over an M x K bf16 matrix with row pitch ldx, X^ = fp32(x * inv[k])
// with smoothing (inv != nullptr), else X. A grid-stride walk over the 16-byte
// vectors, four loads in flight per thread, then per block either one
// atomicMax into *bits (fp32 bits: |x| >= 0, so the unsigned order of the bits
// is the order of the values) or, with partial != nullptr, the block's
// maximum in partial[blockIdx.x]. Idx: 32-bit indexing when the vector count
// fits.
template <typename Idx>
__global__ void __launch_bounds__(256) act_amax_kernel(const __nv_bfloat16* __restrict__ X, int64_t ldx, int M,
                                                       int K, const float* __restrict__ inv, unsigned* bits,
                                                       float* __restrict__ partial) {
  pdl_launch_dependents();  // a programmatic dependent waits for this grid's completion anyway
  const Idx vpr = static_cast<Idx>(K / 8);
  const Idx total = static_cast<Idx>(M) * vpr;
  const Idx stride = static_cast<Idx>(gridDim.x) * blockDim.x;
  float am = 0.0f;
  Idx i = static_cast<Idx>(blockIdx.x) * blockDim.x + threadIdx.x;
  auto at = [&](Idx v) { return X + static_cast<int64_t>(v / vpr) * ldx + static_cast<int64_t>(v % vpr) * 8; };
  for (; i + 3 * stride < total; i += 4 * stride) {
    const Idx i1 = i + stride, i2 = i + 2 * stride, i3 = i + 3 * stride;
    const uint4 v0 = ldg_nc_v4(at(i)), v1 = ldg_nc_v4(at(i1)), v2 = ldg_nc_v4(at(i2)), v3 = ldg_nc_v4(at(i3));
    const uint4 vv[4] = {v0, v1, v2, v3};
    const Idx ii[4] = {i, i1, i2, i3};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float f[8];
      bf16x8_to_f32(vv[u], f);
      if (inv != nullptr) {
        const int col = static_cast<int>(ii[u] % vpr) * 8;
        const float4 a = __ldg(reinterpret_cast<const float4*>(inv + col));
        const float4 b = __ldg(reinterpret_cast<const float4*>(inv + col) + 1);
        const float s8[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = __fmul_rn(f[j], s8[j]);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) am = fmaxf(am, fabsf(f[j]));
    }
  }
  for (; i < total; i += stride) am = vec_amax(at(i), inv, static_cast<int>(i % vpr) * 8, am);
  __shared__ float warp_max[8];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = am;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) am = fmaxf(am, warp_max[w]);
    if (partial != nullptr)
      partial[blockIdx.x] = am;
    else
      atomicMax(bits, __float_as_uint(am));
  }
}

constexpr int kAmaxMaxBlocks = 1984;  // partial maxima of the dynamic scale: 8 KB block minus 256 bytes

// Launches act_amax_kernel over M x K: into *bits (atomicMax; the caller
// zeroes it) or, with partial, one maximum per block. Returns the block count.
int launch_act_amax(const __nv_bfloat16* X, int64_t ldx, int M, int K, const float* inv, unsigned* bits,
                    float* partial, int sm_count, cudaStream_t st) {
  const uint64_t vecs = static_cast<uint64_t>(M) * static_cast<uint64_t>(K / 8);
  uint64_t blocks = (vecs + 1023) / 1024;
  if (blocks > static_cast<uint64_t>(4 * sm_count)) blocks = 4 * sm_count;
  if (blocks > static_cast<uint64_t>(kAmaxMaxBlocks)) blocks = kAmaxMaxBlocks;
  if (blocks == 0) blocks = 1;  // an empty X still writes its (zero) partial
  if (vecs + 4ull * blocks * 256 < (1ull << 32))
    act_amax_kernel<uint32_t><<<static_cast<int>(blocks), 256, 0, st>>>(X, ldx, M, K, inv, bits, partial);
  else
    act_amax_kernel<uint64_t><<<static_cast<int>(blocks), 256, 0, st>>>(X, ldx, M, K, inv, bits, partial);
  return static_cast<int>(blocks);
}

template <int R>
svdq_status launch_pack(int N, int K, const void* W, const void* L1, const void* L2, const float* smooth,
                        const float* g_x, void* codes, void* scales, float* gscale, void* l2s, cudaStream_t st) {
  // The residual kernels read L2 transposed (N x r); plane 1 of l2s serves as
  // that scratch until make_l2s_kernel overwrites both planes at the end.
  __nv_bfloat16* l2t_scratch = static_cast<__nv_bfloat16*>(l2s) + static_cast<size_t>(N) * R;
  transpose_bf16_kernel<<<dim3((N + 31) / 32, (R + 31) / 32), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(L2), l2t_scratch, R, N);
  const int warps = (K / 32) * ((N + kPackRowsPerWarp - 1) / kPackRowsPerWarp);
  const int blocks = (warps + kPackThreads / 32 - 1) / (kPackThreads / 32);
  if (cudaMemsetAsync(gscale, 0, 4 * sizeof(float), st) != cudaSuccess) return launch_status();
  residual_amax_kernel<R><<<blocks, kPackThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(W),
                                                           static_cast<const __nv_bfloat16*>(L1), l2t_scratch, smooth,
                                                           N, K, reinterpret_cast<unsigned*>(gscale + 1));
  finalize_gscale_kernel<<<1, 1, 0, st>>>(gscale, g_x);
  residual_quant_kernel<R><<<blocks, kPackThreads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(W), static_cast<const __nv_bfloat16*>(L1), l2t_scratch, smooth, N, K, gscale,
      static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales));
  const int64_t total = static_cast<int64_t>(N) * R;
  make_l2s_kernel<<<static_cast<int>((total + 255) / 256), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(L2), gscale, static_cast<__nv_bfloat16*>(l2s), N, R);
  return launch_status();
}

svdq_status check_layer_shape(int N, int K, int r) {
  if (N <= 0 || K <= 0 || !valid_rank(r)) return SVDQ_ERR_INVALID_ARG;
  if (K % 256 != 0 || N % 128 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  return SVDQ_OK;
}

// ------------------------------------------------------------------ truncated SVD (load time)
// Sketch width p = r + 32 oversampling columns (a multiple of 16, at most 160).
int svd_width(int r) { return r + 32; }

// Split of the long dimension for the tall-skinny GEMM: enough CTAs for about
// two per SM of a 148-SM B200 (fixed, so that workspace sizes do not depend
// on the device), slices of at least 64.
int ts_splits(int M, int L) {
  const int mtiles = (M + kTsRows - 1) / kTsRows;
  int splits = (296 + mtiles - 1) / mtiles;
  const int max_splits = L / 64 > 0 ? L / 64 : 1;
  if (splits > max_splits) splits = max_splits;
  return splits < 1 ? 1 : splits;
}

size_t ts_part_elems(int M, int L, int P) {
  const int sp = ts_splits(M, L);
  return sp > 1 ? static_cast<size_t>(sp) * M * P : 0;
}

// Workspace layout (float64 buffers, each 256-byte aligned).
struct SvdLayout {
  size_t om, zt, y, yt, part, g, rr, rinv, c, v, lam, m1, m2, u1, v2, total;
};

SvdLayout svd_layout(int N, int K, int r) {
  const int p = svd_width(r);
  SvdLayout l{};
  size_t off = 0;
  auto take = [&](size_t elems) {
    const size_t at = off;
    off = round_up(off + elems * sizeof(double), 256);
    return at;
  };
  size_t part = 0;
  const int shapes[][3] = {{K, N, p}, {N, K, p}, {p, K, p}, {p, N, p}, {K, p, p}, {N, p, p}, {K, p, r}, {N, p, r}};
  for (const auto& sh : shapes) {
    const size_t e = ts_part_elems(sh[0], sh[1], sh[2]);
    if (e > part) part = e;
  }
  l.om = take(static_cast<size_t>(N) * p);
  l.zt = take(static_cast<size_t>(N) * p);
  l.y = take(static_cast<size_t>(K) * p);
  l.yt = take(static_cast<size_t>(K) * p);
  l.part = take(part > 0 ? part : 1);
  l.g = take(static_cast<size_t>(p) * p);
  l.rr = take(static_cast<size_t>(p) * p);
  l.rinv = take(static_cast<size_t>(p) * p);
  l.c = take(static_cast<size_t>(p) * p);
  l.v = take(static_cast<size_t>(p) * p);
  l.lam = take(p);
  l.m1 = take(static_cast<size_t>(p) * r);
  l.m2 = take(static_cast<size_t>(p) * r);
  l.u1 = take(static_cast<size_t>(K) * r);
  l.v2 = take(static_cast<size_t>(N) * r);
  l.total = off;
  return l;
}

// C (M x P) = op(A) B with op(A) = A (M x L) or A^T (A: L x M); B: L x P.
template <bool TRANS_A, typename TA>
svdq_status ts_gemm(int M, int L, int P, const TA* A, int64_t lda, const double* B, double* C, double* part,
                    cudaStream_t st, const float* colscale = nullptr) {
  const int splits = ts_splits(M, L);
  const int lchunk = (L + splits - 1) / splits;
  const dim3 grid((M + kTsRows - 1) / kTsRows, splits);
  static std::atomic<uint64_t> attr_done{0};  // static tile + up to 40 KB of B slice exceed the 48 KB default
  ensure_smem_attr(ts_gemm_kernel<TRANS_A, TA>, kTsL * kSvdMaxP * static_cast<int>(sizeof(double)), attr_done);
  ts_gemm_kernel<TRANS_A, TA><<<grid, kTsThreads, kTsL * P * sizeof(double), st>>>(
      M, L, P, A, lda, colscale, B, splits > 1 ? part : C, lchunk);
  if (splits > 1) {
    const int64_t n = static_cast<int64_t>(M) * P;
    split_sum_kernel<<<static_cast<int>((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184), 256, 0, st>>>(
        part, splits, n, C);
  }
  return launch_status();
}

// T (L x p, float64) <- an orthonormal basis of its column space: Cholesky QR
// three times, the first with the diagonal shift 11 (L p + p (p + 1)) u ||T||^2
// of Fukaya et al. (||T||_2^2 estimated by the largest squared column norm),
// the others with only a floor against breakdown. `tmp` is L x p.
svdq_status orth(double* T, double* tmp, int L, int p, const SvdLayout& lay, uint8_t* ws, cudaStream_t st) {
  double* G = reinterpret_cast<double*>(ws + lay.g);
  double* R = reinterpret_cast<double*>(ws + lay.rr);
  double* Rinv = reinterpret_cast<double*>(ws + lay.rinv);
  double* part = reinterpret_cast<double*>(ws + lay.part);
  const double shift_rel = 11.0 * (static_cast<double>(L) * p + static_cast<double>(p) * (p + 1)) * 0x1.0p-53;
  double* src = T;
  double* dst = tmp;
  svdq_status s;
  for (int pass = 0; pass < 3; ++pass) {
    if ((s = ts_gemm<true, double>(p, L, p, src, p, src, G, part, st)) != SVDQ_OK) return s;
    chol_inv_kernel<<<1, 1024, 0, st>>>(G, p, pass == 0 ? shift_rel : 0.0, R, Rinv);
    if ((s = launch_status()) != SVDQ_OK) return s;
    if ((s = ts_gemm<false, double>(L, p, p, src, p, Rinv, dst, part, st)) != SVDQ_OK) return s;
    double* t = src;
    src = dst;
    dst = t;
  }
  // three passes: the result is in tmp; copy it back
  if (cudaMemcpyAsync(T, src, static_cast<size_t>(L) * p * sizeof(double), cudaMemcpyDeviceToDevice, st) !=
      cudaSuccess)
    return launch_status();
  return SVDQ_OK;
}

svdq_status run_lowrank(int N, int K, int r, const __nv_bfloat16* W, const float* smooth, __nv_bfloat16* L1,
                        __nv_bfloat16* L2, double* sigma, uint64_t seed, int power_iters, uint8_t* ws,
                        cudaStream_t st) {
  const int p = svd_width(r);
  const SvdLayout lay = svd_layout(N, K, r);
  double* Om = reinterpret_cast<double*>(ws + lay.om);   // N x p: Omega, later Z
  double* Zt = reinterpret_cast<double*>(ws + lay.zt);   // N x p scratch
  double* Y = reinterpret_cast<double*>(ws + lay.y);     // K x p
  double* Yt = reinterpret_cast<double*>(ws + lay.yt);   // K x p scratch
  double* part = reinterpret_cast<double*>(ws + lay.part);
  double* C = reinterpret_cast<double*>(ws + lay.c);
  double* V = reinterpret_cast<double*>(ws + lay.v);
  double* lam = reinterpret_cast<double*>(ws + lay.lam);
  double* M1 = reinterpret_cast<double*>(ws + lay.m1);
  double* M2 = reinterpret_cast<double*>(ws + lay.m2);
  double* U1 = reinterpret_cast<double*>(ws + lay.u1);
  double* V2 = reinterpret_cast<double*>(ws + lay.v2);
  svdq_status s;
  const int64_t n_om = static_cast<int64_t>(N) * p;
  gauss_fill_kernel<<<static_cast<int>(((n_om + 1) / 2 + 255) / 256 < 1184 ? ((n_om + 1) / 2 + 255) / 256 : 1184),
                      256, 0, st>>>(Om, n_om, seed);
  if ((s = launch_status()) != SVDQ_OK) return s;
  // A = diag(lambda) W^T (lambda = 1 without smoothing): every read of W scales its column k by lambda_k.
  // Y = A Omega
  if ((s = ts_gemm<true, __nv_bfloat16>(K, N, p, W, K, Om, Y, part, st, smooth)) != SVDQ_OK) return s;
  for (int it = 0; it < power_iters; ++it) {
    if ((s = orth(Y, Yt, K, p, lay, ws, st)) != SVDQ_OK) return s;
    if ((s = ts_gemm<false, __nv_bfloat16>(N, K, p, W, K, Y, Om, part, st, smooth)) != SVDQ_OK) return s;  // Z = A^T Y
    if ((s = orth(Om, Zt, N, p, lay, ws, st)) != SVDQ_OK) return s;
    if ((s = ts_gemm<true, __nv_bfloat16>(K, N, p, W, K, Om, Y, part, st, smooth)) != SVDQ_OK) return s;  // Y = A Z
  }
  if ((s = orth(Y, Yt, K, p, lay, ws, st)) != SVDQ_OK) return s;                                            // Q
  if ((s = ts_gemm<false, __nv_bfloat16>(N, K, p, W, K, Y, Om, part, st, smooth)) != SVDQ_OK) return s;  // B^T = A^T Q
  if ((s = ts_gemm<true, double>(p, N, p, Om, p, Om, C, part, st)) != SVDQ_OK) return s;          // B B^T = Z^T Z
  jacobi_eig_kernel<<<1, 1024, 0, st>>>(C, p, V, lam, 60);
  svd_coeff_kernel<<<1, 256, 0, st>>>(lam, V, p, r, M1, M2, sigma);
  if ((s = launch_status()) != SVDQ_OK) return s;
  if ((s = ts_gemm<false, double>(K, p, r, Y, p, M1, U1, part, st)) != SVDQ_OK) return s;   // U_r S_r = Q U_B,r S_r
  if ((s = ts_gemm<false, double>(N, p, r, Om, p, M2, V2, part, st)) != SVDQ_OK) return s;  // V_r = B^T U_B,r / S_r
  const int64_t tot = static_cast<int64_t>(K + N) * r;
  svd_store_kernel<<<static_cast<int>((tot + 255) / 256 < 1184 ? (tot + 255) / 256 : 1184), 256, 0, st>>>(
      U1, K, V2, N, r, smooth, L1, L2);
  return launch_status();
}

svdq_status gemm_checked(int M, int N, int K, int r, const void* a_codes, const void* a_scales, const void* xl1,
                         const void* w_codes, const void* w_scales, const float* gscale, const void* l2s,
                         const void* bias, void* Y, int64_t ldy, void* stream, const QkvPost* post);

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" {

const char* svdq_status_string(int status) {
  switch (status) {
    case SVDQ_OK: return "SVDQ_OK";
    case SVDQ_ERR_INVALID_ARG: return "SVDQ_ERR_INVALID_ARG";
    case SVDQ_ERR_UNSUPPORTED_SHAPE: return "SVDQ_ERR_UNSUPPORTED_SHAPE";
    case SVDQ_ERR_MISALIGNED: return "SVDQ_ERR_MISALIGNED";
    case SVDQ_ERR_UNSUPPORTED_DEVICE: return "SVDQ_ERR_UNSUPPORTED_DEVICE";
    case SVDQ_ERR_CUDA: return "SVDQ_ERR_CUDA";
    case SVDQ_ERR_TIMEOUT: return "SVDQ_ERR_TIMEOUT";
    case SVDQ_ERR_WORKSPACE: return "SVDQ_ERR_WORKSPACE";
    default: return "SVDQ_ERR_UNKNOWN";
  }
}

int svdq_version(void) { return kVersion; }

svdq_status svdq_scale_offset(int K, int row, int kblock, size_t* out) {
  if (out == nullptr || row < 0 || K <= 0 || kblock < 0) return SVDQ_ERR_INVALID_ARG;
  if (K % 64 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (kblock >= K / 16) return SVDQ_ERR_INVALID_ARG;
  *out = scale_offset(K, row, kblock);
  return SVDQ_OK;
}

svdq_status svdq_weight_sizes(int N, int K, int r, size_t* codes_bytes, size_t* scales_bytes, size_t* l1t_bytes,
                              size_t* l2s_bytes) {
  const svdq_status s = check_layer_shape(N, K, r);
  if (s != SVDQ_OK) return s;
  if (!codes_bytes || !scales_bytes || !l1t_bytes || !l2s_bytes) return SVDQ_ERR_INVALID_ARG;
  *codes_bytes = static_cast<size_t>(N) * (K / 2);
  *scales_bytes = static_cast<size_t>(N) * (K / 16);
  *l1t_bytes = static_cast<size_t>(r) * K * 2;
  *l2s_bytes = static_cast<size_t>(N) * r * 2 * 2;
  return SVDQ_OK;
}

svdq_status svdq_act_sizes(int M, int K, int r, size_t* codes_bytes, size_t* scales_bytes, size_t* xl1_bytes) {
  if (M < 0 || K <= 0 || !valid_rank(r) || !codes_bytes || !scales_bytes || !xl1_bytes) return SVDQ_ERR_INVALID_ARG;
  if (K % 256 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  *codes_bytes = static_cast<size_t>(M) * (K / 2);
  *scales_bytes = round_up(static_cast<size_t>(M), 128) * (K / 16);
  *xl1_bytes = static_cast<size_t>(M) * r * 2;
  return SVDQ_OK;
}

svdq_status svdq_forward_workspace_size(int M, int K, int r, size_t* bytes) {
  size_t c, s, x;
  const svdq_status st = svdq_act_sizes(M, K, r, &c, &s, &x);
  if (st != SVDQ_OK) return st;
  if (!bytes) return SVDQ_ERR_INVALID_ARG;
  *bytes = round_up(c, 256) + round_up(s, 256) + round_up(x, 256);
  return SVDQ_OK;
}

svdq_status svdq_pack_weight(int N, int K, int r, const void* W, const void* L1, const void* L2, const float* smooth,
                             const float* g_x, void* w_codes, void* w_scales, float* gscale, void* l1t, void* l2s,
                             float* inv_smooth, void* stream) {
  NvtxRange nvtx_range("svdq_pack_weight");
  svdq_status s = check_layer_shape(N, K, r);
  if (s != SVDQ_OK) return s;
  if (!W || !L1 || !L2 || !g_x || !w_codes || !w_scales || !gscale || !l1t || !l2s) return SVDQ_ERR_INVALID_ARG;
  if ((smooth == nullptr) != (inv_smooth == nullptr)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(L1) || !aligned16(L2) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(l1t) || !aligned16(l2s) || !aligned16(gscale) || (reinterpret_cast<uintptr_t>(g_x) & 3u) ||
      (smooth && (!aligned16(smooth) || !aligned16(inv_smooth))))
    return SVDQ_ERR_MISALIGNED;
  DeviceInfo di;
  if ((s = current_device(nullptr, &di)) != SVDQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (smooth != nullptr) {
    inv_smooth_kernel<<<(K + 255) / 256, 256, 0, st>>>(smooth, inv_smooth, K);
    if ((s = launch_status()) != SVDQ_OK) return s;
  }
  // l1t = L1^T (r x K)
  transpose_bf16_kernel<<<dim3((r + 31) / 32, (K + 31) / 32), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(L1), static_cast<__nv_bfloat16*>(l1t), K, r);
  if ((s = launch_status()) != SVDQ_OK) return s;
  switch (r) {
    case 16: return launch_pack<16>(N, K, W, L1, L2, smooth, g_x, w_codes, w_scales, gscale, l2s, st);
    case 32: return launch_pack<32>(N, K, W, L1, L2, smooth, g_x, w_codes, w_scales, gscale, l2s, st);
    case 64: return launch_pack<64>(N, K, W, L1, L2, smooth, g_x, w_codes, w_scales, gscale, l2s, st);
    default: return launch_pack<128>(N, K, W, L1, L2, smooth, g_x, w_codes, w_scales, gscale, l2s, st);
  }
}

svdq_status svdq_lowrank_workspace_size(int N, int K, int r, size_t* bytes) {
  if (N <= 0 || K <= 0 || !valid_rank(r) || !bytes) return SVDQ_ERR_INVALID_ARG;
  if (r > N || r > K) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  *bytes = svd_layout(N, K, r).total;
  return SVDQ_OK;
}

svdq_status svdq_lowrank_init(int N, int K, int r, const void* W, const float* smooth, void* L1, void* L2,
                              double* sigma, unsigned long long seed, int power_iters, void* workspace,
                              size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("svdq_lowrank_init");
  if (N <= 0 || K <= 0 || !valid_rank(r) || !W || !L1 || !L2 || !workspace || power_iters < 0 || power_iters > 64)
    return SVDQ_ERR_INVALID_ARG;
  if (r > N || r > K || K % 8 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(W) || !aligned16(L1) || !aligned16(L2) || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      (reinterpret_cast<uintptr_t>(sigma) & 7u) || (smooth && !aligned16(smooth)))
    return SVDQ_ERR_MISALIGNED;
  if (ws_bytes < svd_layout(N, K, r).total) return SVDQ_ERR_WORKSPACE;
  svdq_status s;
  DeviceInfo di;
  if ((s = current_device(nullptr, &di)) != SVDQ_OK) return s;
  return run_lowrank(N, K, r, static_cast<const __nv_bfloat16*>(W), smooth, static_cast<__nv_bfloat16*>(L1),
                     static_cast<__nv_bfloat16*>(L2), sigma, seed, power_iters, static_cast<uint8_t*>(workspace),
                     static_cast<cudaStream_t>(stream));
}

svdq_status svdq_act_global_scale(int M, int K, const void* X, int64_t ldx, const float* inv_smooth, float* g_out,
                                  void* stream) {
  NvtxRange nvtx_range("svdq_act_global_scale");
  if (M < 0 || K <= 0 || !X || !g_out) return SVDQ_ERR_INVALID_ARG;
  if (K % 8 != 0 || ldx < K || ldx % 8 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(X) || (reinterpret_cast<uintptr_t>(g_out) & 3u) || (inv_smooth && !aligned16(inv_smooth)))
    return SVDQ_ERR_MISALIGNED;
  svdq_status s;
  DeviceInfo di;
  if ((s = current_device(nullptr, &di)) != SVDQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(g_out, 0, sizeof(float), st) != cudaSuccess) return launch_status();
  if (M > 0) {
    launch_act_amax(static_cast<const __nv_bfloat16*>(X), ldx, M, K, inv_smooth, reinterpret_cast<unsigned*>(g_out),
                    nullptr, di.sm_count, st);
  }
  finalize_global_scale_kernel<<<1, 1, 0, st>>>(g_out);
  return launch_status();
}

svdq_status svdq_smooth_factors(int M, int N, int K, const void* X, int64_t ldx, const void* W, float alpha,
                                float* lambda, void* stream) {
  NvtxRange nvtx_range("svdq_smooth_factors");
  if (M < 0 || N <= 0 || K <= 0 || !X || !W || !lambda || !(alpha >= 0.0f && alpha <= 1.0f))
    return SVDQ_ERR_INVALID_ARG;
  if (K % 8 != 0 || ldx < K || ldx % 8 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(X) || !aligned16(W) || (reinterpret_cast<uintptr_t>(lambda) & 3u)) return SVDQ_ERR_MISALIGNED;
  svdq_status s;
  DeviceInfo di;
  if ((s = current_device(nullptr, &di)) != SVDQ_OK) return s;
  smooth_factors_kernel<<<(K + kSmoothCols - 1) / kSmoothCols, kSmoothThreads, 0,
                          static_cast<cudaStream_t>(stream)>>>(static_cast<const __nv_bfloat16*>(X), ldx, M,
                                                               static_cast<const __nv_bfloat16*>(W), N, K, alpha,
                                                               lambda);
  return launch_status();
}

svdq_status svdq_quantize_act(int M, int K, int r, const void* X, int64_t ldx, const float* g_x, const void* l1t,
                              const float* inv_smooth, void* codes, void* scales, void* xl1, void* stream) {
  NvtxRange nvtx_range("svdq_quantize_act");
  if (M < 0 || K <= 0 || !valid_rank(r)) return SVDQ_ERR_INVALID_ARG;
  if (K % 256 != 0 || ldx < K || ldx % 8 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!X || !g_x || !l1t || !codes || !scales || !xl1) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(l1t) || !aligned16(codes) || !aligned16(scales) || !aligned16(xl1) ||
      (reinterpret_cast<uintptr_t>(g_x) & 3u) || (inv_smooth && !aligned16(inv_smooth)))
    return SVDQ_ERR_MISALIGNED;
  svdq_status s;
  DeviceInfo di;
  if ((s = current_device(nullptr, &di)) != SVDQ_OK) return s;
  return quantize_dispatch(M, K, r, X, ldx, g_x, l1t, inv_smooth, codes, scales, xl1,
                           static_cast<cudaStream_t>(stream), di.sm_count);
}

svdq_status svdq_w4a4_gemm(int M, int N, int K, int r, const void* a_codes, const void* a_scales, const void* xl1,
                           const void* w_codes, const void* w_scales, const float* gscale, const void* l2s,
                           const void* bias, void* Y, int64_t ldy, void* stream) {
  NvtxRange nvtx_range("svdq_w4a4_gemm");
  return gemm_checked(M, N, K, r, a_codes, a_scales, xl1, w_codes, w_scales, gscale, l2s, bias, Y, ldy, stream,
                      nullptr);
}

svdq_status svdq_linear_forward_qkv(int M, int N, int K, int r, const void* X, int64_t ldx, const void* w_codes,
                                    const void* w_scales, const float* gscale, const void* l1t, const void* l2s,
                                    const float* inv_smooth, const void* bias, int heads, const void* norm_q_weight,
                                    const void* norm_k_weight, float eps, const float* rope_cos,
                                    const float* rope_sin, int64_t ld_rope, void* Y, int64_t ldy, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("svdq_linear_forward_qkv");
  if (M < 0 || heads <= 0 || !(eps >= 0.0f && eps < 1e30f)) return SVDQ_ERR_INVALID_ARG;
  svdq_status s = check_layer_shape(N, K, r);
  if (s != SVDQ_OK) return s;
  if (static_cast<int64_t>(N) != 3ll * heads * kHeadDim) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (ldx < K || ldx % 8 != 0 || ldy < N || ldy % 8 != 0 || ld_rope < kHeadDim / 2 || ld_rope % 4 != 0)
    return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!norm_q_weight || !norm_k_weight || !rope_cos || !rope_sin || !workspace || !gscale)
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(norm_q_weight) || !aligned16(norm_k_weight) || !aligned16(rope_cos) || !aligned16(rope_sin) ||
      !aligned16(workspace))
    return SVDQ_ERR_MISALIGNED;
  size_t need = 0, c = 0, sc = 0, x = 0;
  svdq_forward_workspace_size(M, K, r, &need);
  svdq_act_sizes(M, K, r, &c, &sc, &x);
  if (workspace_bytes < need) return SVDQ_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* a_codes = ws;
  uint8_t* a_scales = ws + round_up(c, 256);
  uint8_t* xl1 = a_scales + round_up(sc, 256);
  s = svdq_quantize_act(M, K, r, X, ldx, gscale, l1t, inv_smooth, a_codes, a_scales, xl1, stream);
  if (s != SVDQ_OK) return s;
  QkvPost post{};
  post.w_q = static_cast<const __nv_bfloat16*>(norm_q_weight);
  post.w_k = static_cast<const __nv_bfloat16*>(norm_k_weight);
  post.cos = rope_cos;
  post.sin = rope_sin;
  post.ld_rope = ld_rope;
  post.hd = heads * kHeadDim;
  post.eps = eps;
  return gemm_checked(M, N, K, r, a_codes, a_scales, xl1, w_codes, w_scales, gscale, l2s, bias, Y, ldy, stream,
                      &post);
}

svdq_status svdq_mlp_workspace_size(int M, int N, int K, int r, int r_down, size_t* bytes) {
  size_t base = 0;
  svdq_status s = check_layer_shape(N, K, r);
  if (s != SVDQ_OK) return s;
  if (r_down != kMlpRank || N % 256 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if ((s = svdq_forward_workspace_size(M, K, r, &base)) != SVDQ_OK) return s;
  if (!bytes) return SVDQ_ERR_INVALID_ARG;
  // one fp32 XL1 partial slot of 256 rows per 256 x 256 tile (used by the tiles that start a run)
  const size_t tiles = static_cast<size_t>((M + 255) / 256) * (N / 256);
  *bytes = base + round_up(tiles * 256 * r_down * 4, 256);
  return SVDQ_OK;
}

svdq_status svdq_mlp_up_forward(int M, int N, int K, int r, const void* X, int64_t ldx, const void* w_codes,
                                const void* w_scales, const float* gscale, const void* l1t, const void* l2s,
                                const float* inv_smooth, const void* bias, int r_down, const float* g_h,
                                const void* l1t_down, int approximate, void* h_codes, void* h_scales, void* h_xl1,
                                void* h_out, int64_t ldh, void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("svdq_mlp_up_forward");
  if (M < 0) return SVDQ_ERR_INVALID_ARG;
  svdq_status s = check_layer_shape(N, K, r);
  if (s != SVDQ_OK) return s;
  if (r_down != kMlpRank || N % 256 != 0 || ldx < K || ldx % 8 != 0 || (h_out && (ldh < N || ldh % 8 != 0)))
    return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!X || !gscale || !l1t || !g_h || !l1t_down || !h_codes || !h_scales || !h_xl1 || !workspace || !w_codes ||
      !w_scales || !l2s)
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(l1t_down) || !aligned16(h_codes) || !aligned16(h_scales) || !aligned16(h_xl1) ||
      !aligned16(workspace) || (h_out && !aligned16(h_out)) || (reinterpret_cast<uintptr_t>(g_h) & 3u) ||
      !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(l2s) || !aligned16(gscale) ||
      (bias && !aligned16(bias)))
    return SVDQ_ERR_MISALIGNED;
  size_t need = 0, base = 0, c = 0, sc = 0, x = 0;
  svdq_mlp_workspace_size(M, N, K, r, r_down, &need);
  svdq_forward_workspace_size(M, K, r, &base);
  svdq_act_sizes(M, K, r, &c, &sc, &x);
  if (workspace_bytes < need) return SVDQ_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* a_codes = ws;
  uint8_t* a_scales = ws + round_up(c, 256);
  uint8_t* xl1 = a_scales + round_up(sc, 256);
  float* partial = reinterpret_cast<float*>(ws + base);
  s = svdq_quantize_act(M, K, r, X, ldx, gscale, l1t, inv_smooth, a_codes, a_scales, xl1, stream);
  if (s != SVDQ_OK) return s;
  DeviceInfo di;
  if ((s = current_device(nullptr, &di)) != SVDQ_OK) return s;
  MlpPost mp{};
  mp.g_h = g_h;
  mp.codes = static_cast<uint8_t*>(h_codes);
  mp.scales = static_cast<uint8_t*>(h_scales);
  mp.partial = partial;
  mp.m_pad = static_cast<int>(round_up(static_cast<size_t>(M), 128));
  mp.store_h = h_out != nullptr;
  mp.approximate = approximate != 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // without h_out nothing is stored through the output map; it is built on h_codes only to be valid
  s = gemm_dispatch(M, N, K, r, a_codes, a_scales, xl1, w_codes, w_scales, gscale, l2s, bias,
                    h_out ? h_out : h_codes, h_out ? ldh : N, st, di.sm_count, nullptr, &mp, l1t_down);
  if (s != SVDQ_OK) return s;
  const int64_t tot = static_cast<int64_t>(M) * r_down;
  int64_t blocks = (tot + 255) / 256;
  if (blocks > 4 * di.sm_count) blocks = 4 * di.sm_count;
  const int num_nt = N / k2TileN;
  const int num_tiles = ((M + k2TileM - 1) / k2TileM) * num_nt;
  mlp_xl1_reduce_kernel<<<static_cast<int>(blocks), 256, 0, st>>>(partial, num_tiles, gemm2_pairs(M, N, di.sm_count),
                                                                    num_nt, M, static_cast<__nv_bfloat16*>(h_xl1));
  return launch_status();
}

}  // extern "C"

namespace svdq {
namespace {
svdq_status gemm_checked(int M, int N, int K, int r, const void* a_codes, const void* a_scales, const void* xl1,
                         const void* w_codes, const void* w_scales, const float* gscale, const void* l2s,
                         const void* bias, void* Y, int64_t ldy, void* stream, const QkvPost* post) {
  if (M < 0) return SVDQ_ERR_INVALID_ARG;
  svdq_status s = check_layer_shape(N, K, r);
  if (s != SVDQ_OK) return s;
  if (ldy < N || ldy % 8 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!a_codes || !a_scales || !xl1 || !w_codes || !w_scales || !gscale || !l2s || !Y) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(xl1) || !aligned16(w_codes) ||
      !aligned16(w_scales) || !aligned16(l2s) || !aligned16(Y) || (bias && !aligned16(bias)) || !aligned16(gscale))
    return SVDQ_ERR_MISALIGNED;
  DeviceInfo di;
  if ((s = current_device(nullptr, &di)) != SVDQ_OK) return s;
  return gemm_dispatch(M, N, K, r, a_codes, a_scales, xl1, w_codes, w_scales, gscale, l2s, bias, Y, ldy,
                       static_cast<cudaStream_t>(stream), di.sm_count, post);
}
}  // namespace
}  // namespace svdq

extern "C" {

svdq_status svdq_linear_forward(int M, int N, int K, int r, const void* X, int64_t ldx, const void* w_codes,
                                const void* w_scales, const float* gscale, const void* l1t, const void* l2s,
                                const float* inv_smooth, const void* bias, void* Y, int64_t ldy, void* workspace,
                                size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("svdq_linear_forward");
  if (M < 0) return SVDQ_ERR_INVALID_ARG;
  svdq_status s = check_layer_shape(N, K, r);
  if (s != SVDQ_OK) return s;
  if (ldx < K || ldx % 8 != 0 || ldy < N || ldy % 8 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SVDQ_OK;
  size_t need = 0, c = 0, sc = 0, x = 0;
  svdq_forward_workspace_size(M, K, r, &need);
  svdq_act_sizes(M, K, r, &c, &sc, &x);
  if (!workspace) return SVDQ_ERR_INVALID_ARG;
  if (workspace_bytes < need) return SVDQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SVDQ_ERR_MISALIGNED;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* a_codes = ws;
  uint8_t* a_scales = ws + round_up(c, 256);
  uint8_t* xl1 = a_scales + round_up(sc, 256);
  if (!gscale) return SVDQ_ERR_INVALID_ARG;
  s = svdq_quantize_act(M, K, r, X, ldx, gscale, l1t, inv_smooth, a_codes, a_scales, xl1, stream);
  if (s != SVDQ_OK) return s;
  return svdq_w4a4_gemm(M, N, K, r, a_codes, a_scales, xl1, w_codes, w_scales, gscale, l2s, bias, Y, ldy, stream);
}

}  // extern "C"
namespace svdq {
namespace {
// Per-call scale block of the dynamic forward: {g, g_w, alpha', amax} at 0,
// the amax pass's per-block maxima from byte 256.
constexpr size_t kDynScaleBytes = 8192;
}  // namespace
}  // namespace svdq
extern "C" {

svdq_status svdq_dynamic_workspace_size(int M, int N, int K, int r, size_t* bytes) {
  size_t base = 0;
  svdq_status s = check_layer_shape(N, K, r);
  if (s != SVDQ_OK) return s;
  if ((s = svdq_forward_workspace_size(M, K, r, &base)) != SVDQ_OK) return s;
  if (!bytes) return SVDQ_ERR_INVALID_ARG;
  *bytes = base + kDynScaleBytes + round_up(static_cast<size_t>(N) * r * 2 * 2, 256);
  return SVDQ_OK;
}

svdq_status svdq_linear_forward_dynamic(int M, int N, int K, int r, const void* X, int64_t ldx, const void* w_codes,
                                        const void* w_scales, const float* gscale, const void* l1t, const void* l2s,
                                        const float* inv_smooth, const void* bias, void* Y, int64_t ldy,
                                        void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("svdq_linear_forward_dynamic");
  if (M < 0) return SVDQ_ERR_INVALID_ARG;
  svdq_status s = check_layer_shape(N, K, r);
  if (s != SVDQ_OK) return s;
  if (ldx < K || ldx % 8 != 0 || ldy < N || ldy % 8 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!workspace || !gscale || !l2s || !X || !l1t) return SVDQ_ERR_INVALID_ARG;
  size_t need = 0, base = 0;
  svdq_dynamic_workspace_size(M, N, K, r, &need);
  svdq_forward_workspace_size(M, K, r, &base);
  if (workspace_bytes < need) return SVDQ_ERR_WORKSPACE;
  if (!aligned16(workspace) || !aligned16(gscale) || !aligned16(l2s) || !aligned16(X) || !aligned16(l1t) ||
      (inv_smooth && !aligned16(inv_smooth)))
    return SVDQ_ERR_MISALIGNED;
  DeviceInfo di;
  if ((s = current_device(nullptr, &di)) != SVDQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* gs = reinterpret_cast<float*>(ws + base);
  float* partial = reinterpret_cast<float*>(ws + base + 256);
  __nv_bfloat16* l2s_d = reinterpret_cast<__nv_bfloat16*>(ws + base + kDynScaleBytes);
  // amax|X^| of this call as per-block maxima; the quantiser (a programmatic
  // dependent of the amax pass) reduces them to this call's scale, writes
  // {g, g_w, alpha', amax} and re-expresses the l2 planes; then the GEMM.
  const int nparts = launch_act_amax(static_cast<const __nv_bfloat16*>(X), ldx, M, K, inv_smooth, nullptr, partial,
                                     di.sm_count, st);
  if ((s = launch_status()) != SVDQ_OK) return s;
  size_t c = 0, sc = 0, x = 0;
  svdq_act_sizes(M, K, r, &c, &sc, &x);
  uint8_t* a_codes = ws;
  uint8_t* a_scales = ws + round_up(c, 256);
  uint8_t* xl1 = a_scales + round_up(sc, 256);
  DynScale dyn{};
  dyn.partial = partial;
  dyn.nparts = nparts;
  dyn.gscale = gscale;
  dyn.gs_out = gs;
  dyn.l2s = static_cast<const __nv_bfloat16*>(l2s);
  dyn.l2s_out = l2s_d;
  dyn.total = static_cast<int64_t>(N) * r;
  s = quantize_dispatch(M, K, r, X, ldx, gs, l1t, inv_smooth, a_codes, a_scales, xl1, st, di.sm_count, true, dyn);
  if (s != SVDQ_OK) return s;
  return svdq_w4a4_gemm(M, N, K, r, a_codes, a_scales, xl1, w_codes, w_scales, gs, l2s_d, bias, Y, ldy, stream);
}

svdq_status svdq_awq_sizes(int N, int K, size_t* codes_bytes, size_t* scales_bytes, size_t* zeros_bytes) {
  if (N <= 0 || K <= 0 || !codes_bytes || !scales_bytes || !zeros_bytes) return SVDQ_ERR_INVALID_ARG;
  if (K % kAwqGroup != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  *codes_bytes = static_cast<size_t>(N) * (K / 2);
  *scales_bytes = static_cast<size_t>(N) * (K / kAwqGroup) * 2;
  *zeros_bytes = static_cast<size_t>(N) * (K / kAwqGroup);
  return SVDQ_OK;
}

svdq_status svdq_awq_pack(int N, int K, const void* W, const float* act_scale, void* codes, void* scales,
                          void* zeros, float* inv_act, void* stream) {
  NvtxRange nvtx_range("svdq_awq_pack");
  if (N <= 0 || K <= 0 || !W || !codes || !scales || !zeros) return SVDQ_ERR_INVALID_ARG;
  if ((act_scale == nullptr) != (inv_act == nullptr)) return SVDQ_ERR_INVALID_ARG;
  if (K % kAwqGroup != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(W) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 1u) ||
      (act_scale && (!aligned16(act_scale) || !aligned16(inv_act))))
    return SVDQ_ERR_MISALIGNED;
  svdq_status s;
  DeviceInfo di;
  if ((s = current_device(nullptr, &di)) != SVDQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (act_scale != nullptr) inv_smooth_kernel<<<(K + 255) / 256, 256, 0, st>>>(act_scale, inv_act, K);
  const int64_t groups = static_cast<int64_t>(N) * (K / kAwqGroup);
  awq_pack_kernel<<<static_cast<int>((groups + kAwqThreads - 1) / kAwqThreads), kAwqThreads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(W), N, K, act_scale, static_cast<uint8_t*>(codes),
      static_cast<__nv_bfloat16*>(scales), static_cast<uint8_t*>(zeros));
  return launch_status();
}

}  // extern "C"
namespace svdq {
namespace {
constexpr int kAwqSmemCap = 96 * 1024;  // activation rows staged per CTA: at most 96 KB
constexpr int kAwqRingSmemCap = 226 * 1024;  // the ring variant: staged activations + stage ring

template <int MT>
svdq_status launch_awq_gemv(int M, int N, int K, const __nv_bfloat16* X, int64_t ldx, const uint8_t* codes,
                            const __nv_bfloat16* scales, const uint8_t* zeros, const float* inv_act,
                            const __nv_bfloat16* bias, __nv_bfloat16* Y, int64_t ldy, int sm_count,
                            cudaStream_t st) {
  // The bulk-copy ring variant: K % 1024 == 0 (every row count's codes, scales
  // and zero points are 16-byte multiples), 16-byte aligned scales and zero
  // points, and room for at least two stages next to the staged activations.
  // SVDQ_AWQ_KERNEL=direct|ring overrides the choice where both apply (tests).
  {
    const char* env = std::getenv("SVDQ_AWQ_KERNEL");
    const int stage = awq_ring_stage_bytes(K);
    const int room = kAwqRingSmemCap - MT * K * 4 - 2 * kAwqRingMaxStages * 8 - 16;
    int stages = room > 0 ? room / stage : 0;
    if (stages > kAwqRingMaxStages) stages = kAwqRingMaxStages;
    // by default from four activation rows on: with one or two rows the direct
    // kernel (two CTAs per SM) measured faster on B200
    const bool ring_default = MT >= 4;
    const bool use_ring = env == nullptr ? ring_default : std::strcmp(env, "ring") == 0;
    if (use_ring && K % 1024 == 0 && aligned16(scales) && aligned16(zeros) && stages >= 2) {
      const int smem_r = MT * K * 4 + stages * stage + 2 * kAwqRingMaxStages * 8 + 16;
      static std::atomic<uint64_t> attr_r{0};
      ensure_smem_attr(awq_gemv_ring_kernel<MT>, kAwqRingSmemCap, attr_r);
      int blocks = (N + kAwqRingRows - 1) / kAwqRingRows;
      if (blocks > sm_count) blocks = sm_count;  // one CTA per SM, each a contiguous run of rows
      for (int m0 = 0; m0 < M; m0 += MT) {
        awq_gemv_ring_kernel<MT><<<blocks, kAwqRingThreads, smem_r, st>>>(
            M - m0, N, K, X + static_cast<int64_t>(m0) * ldx, ldx, codes, scales, zeros, inv_act, bias,
            Y + static_cast<int64_t>(m0) * ldy, ldy, stages);
        const svdq_status s = launch_status();
        if (s != SVDQ_OK) return s;
      }
      return SVDQ_OK;
    }
  }
  const int smem = MT * K * 4;
  static std::atomic<uint64_t> attr_done{0};  // set once to the cap, which covers every K accepted
  ensure_smem_attr(awq_gemv_kernel<MT>, kAwqSmemCap, attr_done);
  int per_sm = 0;  // resident blocks per SM (registers and shared memory): one wave
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, awq_gemv_kernel<MT>, kAwqThreads, smem) != cudaSuccess)
    return launch_status();
  if (per_sm < 1) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  int blocks = (N + kAwqThreads / 32 - 1) / (kAwqThreads / 32);
  if (blocks > per_sm * sm_count) blocks = per_sm * sm_count;
  for (int m0 = 0; m0 < M; m0 += MT) {
    awq_gemv_kernel<MT><<<blocks, kAwqThreads, smem, st>>>(M - m0, N, K, X + static_cast<int64_t>(m0) * ldx, ldx,
                                                            codes, scales, zeros, inv_act, bias,
                                                            Y + static_cast<int64_t>(m0) * ldy, ldy);
    const svdq_status s = launch_status();
    if (s != SVDQ_OK) return s;
  }
  return SVDQ_OK;
}
}  // namespace
}  // namespace svdq
extern "C" {

svdq_status svdq_awq_gemv(int M, int N, int K, const void* X, int64_t ldx, const void* codes, const void* scales,
                          const void* zeros, const float* inv_act, const void* bias, void* Y, int64_t ldy,
                          void* stream) {
  NvtxRange nvtx_range("svdq_awq_gemv");
  if (M < 0 || N <= 0 || K <= 0) return SVDQ_ERR_INVALID_ARG;
  if (K % kAwqGroup != 0 || ldx < K || ldx % 8 != 0 || ldy < N) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!X || !codes || !scales || !zeros || !Y) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 1u) ||
      (reinterpret_cast<uintptr_t>(Y) & 1u) || (bias && (reinterpret_cast<uintptr_t>(bias) & 1u)) ||
      (inv_act && !aligned16(inv_act)))
    return SVDQ_ERR_MISALIGNED;
  if (K * 4 > kAwqSmemCap) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  svdq_status s;
  DeviceInfo di;
  if ((s = current_device(nullptr, &di)) != SVDQ_OK) return s;
  const auto* x = static_cast<const __nv_bfloat16*>(X);
  const auto* c = static_cast<const uint8_t*>(codes);
  const auto* sc = static_cast<const __nv_bfloat16*>(scales);
  const auto* z = static_cast<const uint8_t*>(zeros);
  const auto* b = static_cast<const __nv_bfloat16*>(bias);
  auto* y = static_cast<__nv_bfloat16*>(Y);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // rows per launch: the smallest power of two covering M (at most 8) whose
  // staged activations fit the cap
  int mt = 1;
  while (mt < 8 && mt < M && 2 * mt * K * 4 <= kAwqSmemCap) mt *= 2;
  switch (mt) {
    case 1: return launch_awq_gemv<1>(M, N, K, x, ldx, c, sc, z, inv_act, b, y, ldy, di.sm_count, st);
    case 2: return launch_awq_gemv<2>(M, N, K, x, ldx, c, sc, z, inv_act, b, y, ldy, di.sm_count, st);
    case 4: return launch_awq_gemv<4>(M, N, K, x, ldx, c, sc, z, inv_act, b, y, ldy, di.sm_count, st);
    default: return launch_awq_gemv<8>(M, N, K, x, ldx, c, sc, z, inv_act, b, y, ldy, di.sm_count, st);
  }
}

}  // extern "C"

namespace svdq {
namespace {
// The bounded wait of every kernel, exercised on purpose: one thread waits on
// an mbarrier that nothing arrives on, with a short limit, so the wait gives
// up, records SVDQ_ERR_TIMEOUT and the kernel returns normally.
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_for(&bar, 0, &abort_flag, limit_ns);
  __syncthreads();
}
}  // namespace
}  // namespace svdq

extern "C" {

svdq_status svdq_selftest_bounded_wait(int limit_us, void* stream) {
  NvtxRange nvtx_range("svdq_selftest_bounded_wait");
  if (limit_us < 1 || limit_us > 1000000) return SVDQ_ERR_INVALID_ARG;
  svdq_status s;
  if ((s = current_device(nullptr, nullptr)) != SVDQ_OK) return s;
  bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_us) * 1000ull);
  return launch_status();
}

svdq_status svdq_read_device_error(int* code, int clear) {
  if (!code) return SVDQ_ERR_INVALID_ARG;
  svdq_status s;
  if ((s = current_device(nullptr, nullptr)) != SVDQ_OK) return s;
  if (cudaDeviceSynchronize() != cudaSuccess) return launch_status();
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return launch_status();
  *code = v;
  if (clear) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return launch_status();
  }
  return SVDQ_OK;
}

}  // extern "C"

// ----------------------------------------------------------------------------
// Forward without caller-provided workspace.
//
// Some callers cannot hand the library a workspace buffer: plugin interfaces
// of inference runtimes that pass only the layer's inputs and outputs, and
// code that runs after the process has fixed its device-memory budget, where
// calling the allocator (and its implicit synchronisation) is not allowed.
// For them the intermediates of svdq_linear_forward (activation codes, block
// scales, XL1) live in one fixed scratch array inside the library.
//
// The array is a file-scope __device__ object of kNoAllocScratchBytes bytes;
// every GPU that loads the library holds it until the process exits. Host code
// must not pass the array's name to a kernel (on the host it names a shadow
// variable, not device memory): the device address is fetched with
// cudaGetSymbolAddress once per device, with that device current, on the
// first call made on that device.
// ----------------------------------------------------------------------------
namespace svdq {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mutex;

// Device address of the scratch array on the current device (set up once per device).
svdq_status noalloc_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      std::fprintf(stderr, "svdq: cudaGetSymbolAddress(scratch) failed: %s\n", cudaGetErrorString(e));
      cudaGetLastError();
      return SVDQ_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return SVDQ_OK;
}

}  // namespace
}  // namespace svdq

extern "C" svdq_status svdq_linear_forward_noalloc(int M, int N, int K, int r, const void* X, int64_t ldx,
                                                   const void* w_codes, const void* w_scales, const float* gscale,
                                                   const void* l1t, const void* l2s, const float* inv_smooth,
                                                   const void* bias, void* Y, int64_t ldy, void* stream) {
  if (M < 0) return SVDQ_ERR_INVALID_ARG;
  svdq_status s = check_layer_shape(N, K, r);
  if (s != SVDQ_OK) return s;
  if (ldx < K || ldx % 8 != 0 || ldy < N || ldy % 8 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SVDQ_OK;
  size_t need = 0;
  if ((s = svdq_forward_workspace_size(M, K, r, &need)) != SVDQ_OK) return s;
  if (need > kNoAllocScratchBytes) {
    std::fprintf(stderr,
                 "svdq_linear_forward_noalloc: M=%d K=%d r=%d needs %zu bytes of scratch, the built-in limit is "
                 "%zu bytes; use svdq_linear_forward with a workspace\n",
                 M, K, r, need, kNoAllocScratchBytes);
    return SVDQ_ERR_WORKSPACE;
  }
  int dev = 0;
  if ((s = current_device(&dev, nullptr)) != SVDQ_OK) return s;
  void* scratch = nullptr;
  if ((s = noalloc_scratch(dev, &scratch)) != SVDQ_OK) return s;
  // Nothing in the scratch has to start at zero: the quantize kernel of this
  // call writes every byte the GEMM of this call reads.
  return svdq_linear_forward(M, N, K, r, X, ldx, w_codes, w_scales, gscale, l1t, l2s, inv_smooth, bias, Y, ldy,
                             scratch, kNoAllocScratchBytes, stream);
}
