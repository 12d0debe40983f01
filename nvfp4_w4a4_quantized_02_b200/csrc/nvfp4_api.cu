// C ABI of the NVFP4 W4A4 linear library (declared in include/nvfp4.h):
// argument validation, TMA descriptor creation and kernel launches.
// Everything runs asynchronously on the caller's stream; nothing is allocated.
#include <cuda.h>
#include <cuda_runtime.h>

#include <nvtx3/nvToolsExt.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "nvfp4.h"
#include "quantize.cuh"
#include "gemm.cuh"
#include "fold.cuh"
#include "kvcache.cuh"
#include "gdn.cuh"
#include "gdn_chunk.cuh"
#include "layout.cuh"

using namespace nvfp4;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool init = false;
  bool ok = false;
  int sms = 0;
  bool attrs = false;
  int quant_ctas_per_sm = 1;
  int gemm2_clusters = 1;  // co-resident 2-CTA clusters of gemm2_kernel
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Current device, checked to be an sm_100 part; fills `info`.
nvfp4_status_t current_device(DeviceInfo **info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo &d = g_dev[dev];
  if (!d.init) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return NVFP4_ERR_CUDA;
    d.ok = (major == 10 && minor == 0);
    d.sms = sms;
    d.init = true;
  }
  if (!d.ok) return NVFP4_ERR_UNSUPPORTED_DEVICE;
  if (!d.attrs) {
    if (cudaFuncSetAttribute(gemm::gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             gemm::Plan1::BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(gemm::gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             gemm::Plan1::BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(gemm::gemm_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             gemm::Plan1::BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(gemm::gemm2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             gemm::Plan2::BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(gemm::decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             gemm::PlanD::BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(gemm::gemm2_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 0) !=
            cudaSuccess ||
        cudaFuncSetAttribute(quantize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmemBytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(gdn::recurrence_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(sizeof(gdn::Smem<32>))) != cudaSuccess ||
        cudaFuncSetAttribute(gdn::recurrence_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(sizeof(gdn::Smem<16>))) != cudaSuccess ||
        cudaFuncSetAttribute(gdn::chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(sizeof(gdn::ChunkSmem))) != cudaSuccess)
      return NVFP4_ERR_CUDA;
    {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * d.sms, 1, 1);
      cfg.blockDim = dim3(gemm::NUM_THREADS, 1, 1);
      cfg.dynamicSmemBytes = gemm::Plan2::BYTES;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, gemm::gemm2_kernel, &cfg) != cudaSuccess) return NVFP4_ERR_CUDA;
      d.gemm2_clusters = clusters < 1 ? 1 : clusters;
    }
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, quantize_kernel, kQThreads, kQSmemBytes) != cudaSuccess)
      return NVFP4_ERR_CUDA;
    d.quant_ctas_per_sm = occ < 1 ? 1 : occ;
    d.attrs = true;
  }
  *info = &d;
  return NVFP4_OK;
}

// NVTX range around one C-ABI call, named after the entry point, so that profilers
// (Nsight Systems / Compute) show which call launched which kernels.  Without a tool
// attached each push / pop is a call through a no-op pointer.
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Cache of encoded tensor maps.  A map is a pure function of (kind, base address,
// sizes, box), so an entry can never go stale: a buffer freed and reallocated at the
// same address with the same sizes gets the same map.  Keyed also by device.  The
// cache is bounded: when full it is cleared and refilled.
struct MapKey {
  int dev, kind;
  const void *ptr;
  int64_t a, b, c;
  bool operator==(const MapKey &o) const {
    return dev == o.dev && kind == o.kind && ptr == o.ptr && a == o.a && b == o.b && c == o.c;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey &k) const {
    uint64_t h = reinterpret_cast<uintptr_t>(k.ptr) * 0x9E3779B97F4A7C15ull;
    for (uint64_t v : {uint64_t(k.dev), uint64_t(k.kind), uint64_t(k.a), uint64_t(k.b), uint64_t(k.c)})
      h = (h ^ v) * 0x100000001B3ull + (h >> 29);
    return static_cast<size_t>(h);
  }
};
constexpr size_t kMapCacheMax = 4096;
std::unordered_map<MapKey, CUtensorMap, MapKeyHash> g_maps;
std::mutex g_maps_mu;

enum MapKind : int { MAP_CODES = 0, MAP_BF16 = 1, MAP_SCALES = 2 };

// Looks `key` up; on a miss runs `encode(m)` and keeps its result.
template <typename F>
bool cached_map(CUtensorMap *m, MapKey key, F &&encode) {
  if (cudaGetDevice(&key.dev) != cudaSuccess) return false;
  {
    std::lock_guard<std::mutex> lk(g_maps_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
      std::memcpy(m, &it->second, sizeof(CUtensorMap));
      return true;
    }
  }
  if (!encode(m)) return false;
  std::lock_guard<std::mutex> lk(g_maps_mu);
  if (g_maps.size() >= kMapCacheMax) g_maps.clear();
  g_maps.emplace(key, *m);
  return true;
}

// Tensor map of packed codes [rows x K/2] bytes: 128-byte x box_rows boxes with the
// 128-byte swizzle (the smem layout the MMA descriptors describe); rows beyond
// `rows` read as zero.
bool encode_codes_map(CUtensorMap *m, const uint8_t *codes, int64_t rows, int64_t K, unsigned box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(codes), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_codes_map(CUtensorMap *m, const uint8_t *codes, int64_t rows, int64_t K, unsigned box_rows = 128) {
  return cached_map(m, MapKey{0, MAP_CODES, codes, rows, K, box_rows},
                    [&](CUtensorMap *mm) { return encode_codes_map(mm, codes, rows, K, box_rows); });
}

// Tensor map of a BF16 matrix [rows x cols] with row stride ld elements: 64-column x
// 128-row boxes (128 bytes per box row) with the 128-byte swizzle; coordinates
// outside the matrix read as zero.
bool encode_bf16_map(CUtensorMap *m, const void *x, int64_t rows, int64_t cols, int64_t ld) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kQTileCols), static_cast<cuuint32_t>(kQTileRows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_bf16_map(CUtensorMap *m, const void *x, int64_t rows, int64_t cols, int64_t ld) {
  return cached_map(m, MapKey{0, MAP_BF16, x, rows, cols, ld},
                    [&](CUtensorMap *mm) { return encode_bf16_map(mm, x, rows, cols, ld); });
}

// Tensor map of a swizzled scale buffer of a [rows x K] operand, viewed as 8-byte
// elements: one row per 128-row group (K/64 atoms of 512 bytes), boxes of 256
// elements = the 4 atoms (2 KB) of one 256-wide K tile of one group.
bool encode_scales_map(CUtensorMap *m, const uint8_t *scales, int64_t rows, int64_t K) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const int64_t groups = (rows + 127) / 128;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 64 * 64), static_cast<cuuint64_t>(groups)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 64 * 512)};
  cuuint32_t box[2] = {256, 1};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<uint8_t *>(scales), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_scales_map(CUtensorMap *m, const uint8_t *scales, int64_t rows, int64_t K) {
  return cached_map(m, MapKey{0, MAP_SCALES, scales, rows, K, 0},
                    [&](CUtensorMap *mm) { return encode_scales_map(mm, scales, rows, K); });
}

// Launches `kernel` with programmatic stream serialization: it may begin (shared
// memory, barriers, TMEM) while the previous kernel on the stream finishes, and waits
// for it in griddepcontrol.wait before touching global memory (every kernel of the
// library does).  In a CUDA graph of many small launches (a decode step) this hides
// most of each launch's latency and prologue.  cluster_x > 1 adds a cluster shape.
template <typename... KArgs, typename... Args>
nvfp4_status_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                          unsigned cluster_x, Args &&...args) {
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...) == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

// Validates the arguments of a linear and fills everything of Params but the tiling.
nvfp4_status_t prepare_linear(const nvfp4_operand_t *A, const float *gs_a, const nvfp4_operand_t *W,
                              const nvfp4_segment_t *segs, int nseg, int epilogue,
                              const nvfp4_epilogue_params_t *ep, void *out, int out_kind, int64_t ldo,
                              gemm::Params &p) {
  using namespace gemm;
  if (!A || !W || !gs_a || !segs || !out) return NVFP4_ERR_INVALID_ARG;
  if (!A->codes || !A->scales || !W->codes || !W->scales) return NVFP4_ERR_INVALID_ARG;
  if (A->rows < 1 || W->rows < 1 || A->K < 1 || A->K != W->K) return NVFP4_ERR_INVALID_ARG;
  if (epilogue < NVFP4_EPI_NONE || epilogue > NVFP4_EPI_GDN_GATES) return NVFP4_ERR_INVALID_ARG;
  if (out_kind < NVFP4_OUT_BF16 || out_kind > NVFP4_OUT_NVFP4) return NVFP4_ERR_INVALID_ARG;
  if (nseg < 1 || nseg > NVFP4_MAX_SEGMENTS) return NVFP4_ERR_INVALID_ARG;
  const int64_t M = A->rows, N = W->rows, K = A->K;
  if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (K % BK != 0 || N % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  // segments: sorted, disjoint, 16-aligned, covering [0, N)
  int64_t expect = 0;
  for (int i = 0; i < nseg; ++i) {
    if (!segs[i].gs_w || !aligned(segs[i].gs_w, 4)) return NVFP4_ERR_INVALID_ARG;
    if (segs[i].n_begin != expect || segs[i].n_end <= segs[i].n_begin) return NVFP4_ERR_INVALID_ARG;
    if (segs[i].n_begin % 16 != 0 || segs[i].n_end % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    expect = segs[i].n_end;
  }
  if (expect != N) return NVFP4_ERR_INVALID_ARG;
  int64_t Nout = N;
  if (epilogue == NVFP4_EPI_SILU_MUL) {
    if (N % (2 * 128) != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    Nout = N / 2;
  }
  if (epilogue == NVFP4_EPI_GDN_GATES) {
    if (!ep || !ep->A_log || !ep->dt_bias || ep->n_heads < 1) return NVFP4_ERR_INVALID_ARG;
    const int64_t h = ep->n_heads;
    if (ep->beta_begin < 0 || ep->beta_begin + h > N || ep->alpha_begin < 0 || ep->alpha_begin + h > N)
      return NVFP4_ERR_INVALID_ARG;
    if (ep->beta_begin < ep->alpha_begin + h && ep->alpha_begin < ep->beta_begin + h) return NVFP4_ERR_INVALID_ARG;
    if (!aligned(ep->A_log, 4) || !aligned(ep->dt_bias, 4) || (ep->beta_out && !aligned(ep->beta_out, 4)) ||
        (ep->g_out && !aligned(ep->g_out, 4)))
      return NVFP4_ERR_MISALIGNED;
  }
  if (out_kind == NVFP4_OUT_NVFP4) {
    if (!ep || !ep->gs_out || !ep->out_scales) return NVFP4_ERR_INVALID_ARG;
    if (Nout % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(out, 16) || !aligned(ep->out_scales, 16) || !aligned(ep->gs_out, 4)) return NVFP4_ERR_MISALIGNED;
  } else {
    const int64_t elem = out_kind == NVFP4_OUT_BF16 ? 2 : 4;
    if (ldo < Nout) return NVFP4_ERR_INVALID_ARG;
    if (!aligned(out, 16) || (ldo * elem) % 16 != 0) return NVFP4_ERR_MISALIGNED;
  }
  if (!aligned(A->codes, 16) || !aligned(W->codes, 16) || !aligned(A->scales, 16) || !aligned(W->scales, 16) ||
      !aligned(gs_a, 4))
    return NVFP4_ERR_MISALIGNED;

  p = Params{};
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.Nout = static_cast<int>(Nout);
  p.mode = epilogue;
  p.tile_mode = epilogue;
  p.out_kind = out_kind;
  p.k_tiles = static_cast<int>(K / BK);
  p.splits = 1;
  p.kt_per_split = p.k_tiles;
  p.partial = nullptr;
  p.up_row0 = static_cast<int>(Nout);
  p.kb_atoms = K / 64;
  p.sfa = A->scales;
  p.sfb = W->scales;
  p.gs_a = gs_a;
  p.nseg = nseg;
  for (int i = 0; i < nseg; ++i) {
    p.seg[i].n_begin = static_cast<int>(segs[i].n_begin);
    p.seg[i].n_end = static_cast<int>(segs[i].n_end);
    p.seg[i].gs_w = segs[i].gs_w;
  }
  p.out = out;
  p.ldo = ldo;
  p.beta_begin = p.alpha_begin = -1;
  p.n_heads = 0;
  if (epilogue == NVFP4_EPI_GDN_GATES) {
    p.beta_begin = static_cast<int>(ep->beta_begin);
    p.alpha_begin = static_cast<int>(ep->alpha_begin);
    p.n_heads = static_cast<int>(ep->n_heads);
    p.A_log = ep->A_log;
    p.dt_bias = ep->dt_bias;
    p.beta_out = ep->beta_out;
    p.g_out = ep->g_out;
  }
  if (out_kind == NVFP4_OUT_NVFP4) {
    p.gs_out = ep->gs_out;
    p.out_scales = ep->out_scales;
    p.out_kb_atoms = Nout / 64;
  }
  // 32-byte epilogue stores when every row of the output starts 32-byte aligned (an
  // NVFP4 row is Nout / 2 bytes, a multiple of 32)
  const int64_t row_bytes = out_kind == NVFP4_OUT_NVFP4 ? Nout / 2 : ldo * (out_kind == NVFP4_OUT_BF16 ? 2 : 4);
  p.st32 = aligned(out, 32) && row_bytes % 32 == 0;
  p.group_m = GROUP_M;
  return NVFP4_OK;
}

// Split count of the split-K linear: as many splits as keep all work units in one
// wave on the SMs (SMs / tiles, rounded down), with at least 4 K tiles (1024 K) per
// split.  Tiles are 128 weight rows for the decode kernel (M <= 64), else 128 x 256.
// On the decode kernel at 32 rows the rule picks the fastest of splits 1, 2, 3, 4, 6
// for five of the six shapes of the 496-linear decode step; for the 12352-row GDN
// in-projection it picks 1 (13.2 us), where 3 measured 12.8 us.
int default_splits(int64_t M, int64_t N, int64_t K, int sms) {
  const int64_t tiles = M <= gemm::DEC_DN_MAX ? (N + gemm::DEC_BM - 1) / gemm::DEC_BM
                                               : (M + gemm::BM - 1) / gemm::BM * ((N + gemm::BN - 1) / gemm::BN);
  const int64_t k_tiles = K / gemm::BK;
  int64_t s = sms / tiles;
  if (s > k_tiles / 4) s = k_tiles / 4;
  return static_cast<int>(s < 1 ? 1 : s);
}

// Launches the 1-CTA GEMM in split-K mode and the epilogue kernel on `p` (prepared
// by prepare_linear); `splits` >= 1 and the workspace were checked by the caller.
nvfp4_status_t launch_splitk(gemm::Params p, const nvfp4_operand_t *A, const nvfp4_operand_t *W, int splits,
                             float *workspace, const DeviceInfo *dev, cudaStream_t st) {
  using namespace gemm;
  p.kt_per_split = (p.k_tiles + splits - 1) / splits;
  p.splits = (p.k_tiles + p.kt_per_split - 1) / p.kt_per_split;  // no empty split
  p.partial = workspace;
  p.tile_mode = MODE_NONE;
  CUtensorMap tmA, tmB;
  if (p.M <= DEC_DN_MAX) {  // decode size: weight rows are the MMA's M, tokens its N
    p.dn = p.M <= 32 ? 32 : DEC_DN_MAX;
    p.m_tiles = 1;
    p.n_tiles = (p.N + DEC_BM - 1) / DEC_BM;
    if (!make_codes_map(&tmB, W->codes, p.N, p.K) || !make_codes_map(&tmA, A->codes, p.M, p.K, p.dn))
      return NVFP4_ERR_CUDA;
    const int64_t units = int64_t(p.n_tiles) * p.splits;
    if (units > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const int grid = static_cast<int>(units < dev->sms ? units : dev->sms);
    // One split, an element-wise epilogue and a BF16 / FP32 output: the kernel applies
    // the epilogue itself (no partials, no reduction kernel).  SiLU*mul pairs columns of
    // two tiles and an NVFP4 output needs 16 columns of a row; both keep the reduction.
    const bool direct = p.splits == 1 && p.mode != MODE_SILU_MUL && p.out_kind != OUT_NVFP4;
    if (direct) p.partial = nullptr;
    if (nvfp4_status_t e = launch_pdl(decode_kernel, dim3(grid), dim3(DEC_THREADS), PlanD::BYTES, st, 1, tmB, tmA, p))
      return e;
    if (direct) return NVFP4_OK;
  } else {
    if (!make_codes_map(&tmA, A->codes, p.M, p.K) || !make_codes_map(&tmB, W->codes, p.N, p.K)) return NVFP4_ERR_CUDA;
    p.m_tiles = (p.M + BM - 1) / BM;
    p.n_tiles = (p.N + BN - 1) / BN;
    const int64_t units = int64_t(p.m_tiles) * p.n_tiles * p.splits;
    if (units > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const int grid = static_cast<int>(units < dev->sms ? units : dev->sms);
    if (nvfp4_status_t e =
            launch_pdl(gemm_kernel<true>, dim3(grid), dim3(NUM_THREADS), Plan1::BYTES, st, 1, tmA, tmB, p))
      return e;
  }
  // one thread per 16 columns (an E4M3 block) for an NVFP4 output, else per 4 columns
  const bool nvfp4_out = p.out_kind == OUT_NVFP4;
  const int64_t rows_cover = nvfp4_out ? (p.M + 127) / 128 * 128 : p.M;
  const int64_t threads = rows_cover * (p.Nout / (nvfp4_out ? 16 : 4));
  const int64_t blocks = (threads + REDUCE_THREADS - 1) / REDUCE_THREADS;
  if (blocks > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  return launch_pdl(nvfp4_out ? splitk_epilogue_kernel<16> : splitk_epilogue_kernel<4>,
                    dim3(static_cast<unsigned>(blocks)), dim3(REDUCE_THREADS), 0, st, 1, p);
}

// ------------------------------------------------- scratch for callers that cannot allocate
// nvfp4_linear_splitk_noalloc keeps its split-K partial sums in this fixed array, so
// that callers which cannot allocate device memory (no workspace to hand in) can
// still run the decode-regime linear.  Every GPU that loads the library holds these
// NVFP4_NOALLOC_SCRATCH_BYTES until the process exits.
static __device__ __align__(256) float g_noalloc_scratch[NVFP4_NOALLOC_SCRATCH_BYTES / sizeof(float)];

// Device address of g_noalloc_scratch on each device, looked up once per device (the
// host-side name of the array is not a device address).
float *g_noalloc_ptr[kMaxDevices] = {};

nvfp4_status_t noalloc_scratch(float **ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return NVFP4_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<float *>(p);
  }
  *ptr = g_noalloc_ptr[dev];
  return NVFP4_OK;
}

// max|x| of a BF16 matrix into *out (device FP32): zero it, then the amax kernel's
// atomicMax over the bit patterns (non-negative floats order as unsigned integers).
nvfp4_status_t launch_amax(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, float *out,
                           const DeviceInfo *dev, cudaStream_t s) {
  if (cudaMemsetAsync(out, 0, sizeof(float), s) != cudaSuccess) return NVFP4_ERR_CUDA;
  AmaxArgs a;
  a.x = static_cast<const uint16_t *>(x_bf16);
  a.rows = rows;
  a.cols = cols;
  a.ld = ld;
  a.amax_bits = reinterpret_cast<unsigned int *>(out);
  const int64_t vecs = rows * (cols / 8);
  const int64_t want = (vecs / 4 + kAmaxThreads - 1) / kAmaxThreads;
  const int64_t cap = int64_t(dev->sms) * 4;
  const int grid = static_cast<int>(want < 1 ? 1 : (want < cap ? want : cap));
  return launch_pdl(amax_kernel, dim3(grid), dim3(kAmaxThreads), 0, s, 1, a);
}

}  // namespace

extern "C" {

const char *nvfp4_status_string(int s) {
  switch (s) {
    case NVFP4_OK: return "NVFP4_OK";
    case NVFP4_ERR_INVALID_ARG: return "NVFP4_ERR_INVALID_ARG";
    case NVFP4_ERR_UNSUPPORTED_SHAPE: return "NVFP4_ERR_UNSUPPORTED_SHAPE";
    case NVFP4_ERR_MISALIGNED: return "NVFP4_ERR_MISALIGNED";
    case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA";
    case NVFP4_ERR_DEVICE_TIMEOUT: return "NVFP4_ERR_DEVICE_TIMEOUT";
    case NVFP4_ERR_UNSUPPORTED_DEVICE: return "NVFP4_ERR_UNSUPPORTED_DEVICE";
    case NVFP4_ERR_DEVICE_INDEX: return "NVFP4_ERR_DEVICE_INDEX";
    default: return "NVFP4_ERR_UNKNOWN";
  }
}

size_t nvfp4_scale_bytes(int64_t rows, int64_t cols) {
  if (rows < 1 || cols < 16 || cols % 16 != 0 || rows > kMaxDim || cols > kMaxDim) return 0;
  const int64_t rows_pad = (rows + 127) / 128 * 128;
  const int64_t kb_pad = (cols / 16 + 3) / 4 * 4;
  return static_cast<size_t>(rows_pad * kb_pad);
}

nvfp4_status_t nvfp4_amax(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, float *amax_out,
                          nvfp4_stream_t stream) {
  NvtxRange nvtx("nvfp4_amax");
  if (!x_bf16 || !amax_out || rows < 1 || cols < 1 || ld < cols) return NVFP4_ERR_INVALID_ARG;
  if (cols % 16 != 0 || rows > kMaxDim || cols > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(x_bf16, 16) || ld % 8 != 0 || !aligned(amax_out, 4)) return NVFP4_ERR_MISALIGNED;
  DeviceInfo *dev = nullptr;
  if (nvfp4_status_t st = current_device(&dev)) return st;
  return launch_amax(x_bf16, rows, cols, ld, amax_out, dev, reinterpret_cast<cudaStream_t>(stream));
}

nvfp4_status_t nvfp4_global_scale(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, float *gs_out,
                                  nvfp4_stream_t stream) {
  NvtxRange nvtx("nvfp4_global_scale");
  if (!x_bf16 || !gs_out || rows < 1 || cols < 1 || ld < cols) return NVFP4_ERR_INVALID_ARG;
  if (cols % 16 != 0 || rows > kMaxDim || cols > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(x_bf16, 16) || ld % 8 != 0 || !aligned(gs_out, 4)) return NVFP4_ERR_MISALIGNED;
  DeviceInfo *dev = nullptr;
  if (nvfp4_status_t st = current_device(&dev)) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (nvfp4_status_t e = launch_amax(x_bf16, rows, cols, ld, gs_out, dev, s)) return e;
  return launch_pdl(global_scale_finalize_kernel, dim3(1), dim3(1), 0, s, 1, gs_out);
}

nvfp4_status_t nvfp4_quantize_rows(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, const float *gs,
                                   uint8_t *codes, uint8_t *scales, int64_t row_offset, int64_t total_rows,
                                   nvfp4_stream_t stream) {
  NvtxRange nvtx("nvfp4_quantize_rows");
  if (!x_bf16 || !gs || !codes || !scales || rows < 1 || cols < 1 || ld < cols) return NVFP4_ERR_INVALID_ARG;
  if (row_offset < 0 || total_rows < row_offset + rows) return NVFP4_ERR_INVALID_ARG;
  if (cols < 16 || cols % 16 != 0 || total_rows > kMaxDim || cols > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(x_bf16, 16) || ld % 8 != 0 || !aligned(codes, 16) || !aligned(scales, 16) || !aligned(gs, 4))
    return NVFP4_ERR_MISALIGNED;
  DeviceInfo *dev = nullptr;
  if (nvfp4_status_t st = current_device(&dev)) return st;
  QuantArgs a;
  a.gs = gs;
  a.codes = codes;
  a.scales = scales;
  a.rows = rows;
  a.cols = cols;
  a.row_offset = row_offset;
  const bool last = row_offset + rows == total_rows;
  a.own_end = last ? (total_rows + 127) / 128 * 128 : row_offset + rows;
  a.code_ld = cols / 2;
  a.kb_atoms = (cols + 63) / 64;
  a.tile_r0 = row_offset / 128;
  a.n_tiles = ((a.own_end + 127) / 128 - a.tile_r0) * a.kb_atoms;
  if (rows <= 64) {  // decode sizes: one thread per 16-element block, no TMA staging
    const int64_t threads = (a.own_end - row_offset) * 4 * a.kb_atoms;
    const int64_t blocks = (threads + kQSmallThreads - 1) / kQSmallThreads;
    if (blocks > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    return launch_pdl(quantize_small_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kQSmallThreads), 0,
                      reinterpret_cast<cudaStream_t>(stream), 1, static_cast<const uint16_t *>(x_bf16), ld, a);
  }
  CUtensorMap tmX;
  if (!make_bf16_map(&tmX, x_bf16, rows, cols, ld)) return NVFP4_ERR_CUDA;
  const int64_t cap = int64_t(dev->sms) * dev->quant_ctas_per_sm;
  const int grid = static_cast<int>(a.n_tiles < cap ? a.n_tiles : cap);
  return launch_pdl(quantize_kernel, dim3(grid), dim3(kQThreads), kQSmemBytes, reinterpret_cast<cudaStream_t>(stream), 1,
                    tmX, a);
}

nvfp4_status_t nvfp4_quantize(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, const float *gs,
                              uint8_t *codes, uint8_t *scales, nvfp4_stream_t stream) {
  NvtxRange nvtx("nvfp4_quantize");
  return nvfp4_quantize_rows(x_bf16, rows, cols, ld, gs, codes, scales, 0, rows, stream);
}

nvfp4_status_t nvfp4_linear(const nvfp4_operand_t *A, const float *gs_a, const nvfp4_operand_t *W,
                            const nvfp4_segment_t *segs, int nseg, int epilogue, const nvfp4_epilogue_params_t *ep,
                            void *out, int out_kind, int64_t ldo, nvfp4_stream_t stream) {
  NvtxRange nvtx("nvfp4_linear");
  using namespace gemm;
  Params p;
  if (nvfp4_status_t st = prepare_linear(A, gs_a, W, segs, nseg, epilogue, ep, out, out_kind, ldo, p)) return st;
  DeviceInfo *dev = nullptr;
  if (nvfp4_status_t st = current_device(&dev)) return st;
  const int64_t M = p.M, N = p.N, K = p.K;

  const bool pair = M > BM;  // 2-CTA tiles of 256 rows; one CTA per tile for M <= 128
  CUtensorMap tmA, tmB, tmSFA, tmSFB;
  if (!make_codes_map(&tmA, A->codes, M, K) || !make_codes_map(&tmB, W->codes, N, K)) return NVFP4_ERR_CUDA;
  if (pair && (!make_scales_map(&tmSFA, A->scales, M, K) || !make_scales_map(&tmSFB, W->scales, N, K)))
    return NVFP4_ERR_CUDA;
  const int64_t tile_m = pair ? 2 * BM : BM;
  p.m_tiles = static_cast<int>((M + tile_m - 1) / tile_m);
  p.n_tiles = epilogue == NVFP4_EPI_SILU_MUL ? p.Nout / 128 : static_cast<int>((N + BN - 1) / BN);
  const int64_t tiles = int64_t(p.m_tiles) * p.n_tiles;
  if (tiles > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!pair) {
    const int grid = static_cast<int>(tiles < dev->sms ? tiles : dev->sms);
    return launch_pdl(gemm_kernel<false>, dim3(grid), dim3(NUM_THREADS), Plan1::BYTES, st, 1, tmA, tmB, p);
  }
  // A wide weight (64 N-tiles or more) is streamed from DRAM once per raster group:
  // groups of 32 M-tiles halve those re-reads while the group's A rows (codes and
  // scales) stay within 32 MB, a quarter of the B200's L2.  MLP gate|up at 32768
  // tokens: DRAM reads 895 -> 496 MB per launch, 1.6 % faster; a longer K (the down
  // projection) keeps 16.
  if (p.n_tiles >= 64 && int64_t(2 * GROUP_M) * (2 * BM) * (K / 2) * 9 / 8 <= (int64_t(32) << 20))
    p.group_m = 2 * GROUP_M;
  const int64_t clusters = tiles < dev->gemm2_clusters ? tiles : dev->gemm2_clusters;
  return launch_pdl(gemm2_kernel, dim3(static_cast<unsigned>(2 * clusters)), dim3(NUM_THREADS), Plan2::BYTES, st, 2, tmA,
                    tmB, tmSFA, tmSFB, p);
}

int nvfp4_splitk_default(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 16 || K < gemm::BK || K % gemm::BK != 0) return 0;
  DeviceInfo *dev = nullptr;
  if (current_device(&dev) != NVFP4_OK) return 0;
  return default_splits(M, N, K, dev->sms);
}

size_t nvfp4_splitk_workspace_bytes(int64_t M, int64_t N, int split_k) {
  if (M < 1 || N < 1 || split_k < 1 || M > kMaxDim || N > kMaxDim) return 0;
  return static_cast<size_t>(M) * static_cast<size_t>(N) * static_cast<size_t>(split_k) * sizeof(float);
}

nvfp4_status_t nvfp4_linear_splitk(const nvfp4_operand_t *A, const float *gs_a, const nvfp4_operand_t *W,
                                   const nvfp4_segment_t *segs, int nseg, int epilogue,
                                   const nvfp4_epilogue_params_t *ep, void *out, int out_kind, int64_t ldo,
                                   int split_k, void *workspace, size_t workspace_bytes, nvfp4_stream_t stream) {
  NvtxRange nvtx("nvfp4_linear_splitk");
  using namespace gemm;
  Params p;
  if (nvfp4_status_t st = prepare_linear(A, gs_a, W, segs, nseg, epilogue, ep, out, out_kind, ldo, p)) return st;
  if (split_k < 1 || split_k > p.k_tiles) return NVFP4_ERR_INVALID_ARG;
  if (!workspace) return NVFP4_ERR_INVALID_ARG;
  if (workspace_bytes < nvfp4_splitk_workspace_bytes(p.M, p.N, split_k)) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(workspace, 16)) return NVFP4_ERR_MISALIGNED;
  // One split above decode size: the ordinary kernel, without partials or the second
  // kernel.  Up to 64 rows the decode kernel and the reduction beat it even unsplit
  // (a 496-linear decode step at 32 rows: 4.74 ms against 6.86 ms).
  if (split_k == 1 && p.M > DEC_DN_MAX)
    return nvfp4_linear(A, gs_a, W, segs, nseg, epilogue, ep, out, out_kind, ldo, stream);
  DeviceInfo *dev = nullptr;
  if (nvfp4_status_t st = current_device(&dev)) return st;
  return launch_splitk(p, A, W, split_k, static_cast<float *>(workspace), dev,
                       reinterpret_cast<cudaStream_t>(stream));
}

nvfp4_status_t nvfp4_linear_splitk_noalloc(const nvfp4_operand_t *A, const float *gs_a, const nvfp4_operand_t *W,
                                           const nvfp4_segment_t *segs, int nseg, int epilogue,
                                           const nvfp4_epilogue_params_t *ep, void *out, int out_kind, int64_t ldo,
                                           int split_k, nvfp4_stream_t stream) {
  NvtxRange nvtx("nvfp4_linear_splitk_noalloc");
  using namespace gemm;
  Params p;
  if (nvfp4_status_t st = prepare_linear(A, gs_a, W, segs, nseg, epilogue, ep, out, out_kind, ldo, p)) return st;
  if (split_k < 1 || split_k > p.k_tiles) return NVFP4_ERR_INVALID_ARG;
  // One split above decode size needs no partials: the ordinary kernel, which allocates
  // nothing either (as in nvfp4_linear_splitk).
  if (split_k == 1 && p.M > DEC_DN_MAX)
    return nvfp4_linear(A, gs_a, W, segs, nseg, epilogue, ep, out, out_kind, ldo, stream);
  if (nvfp4_splitk_workspace_bytes(p.M, p.N, split_k) > NVFP4_NOALLOC_SCRATCH_BYTES)
    return NVFP4_ERR_UNSUPPORTED_SHAPE;  // the partials do not fit the fixed scratch array
  DeviceInfo *dev = nullptr;
  if (nvfp4_status_t st = current_device(&dev)) return st;
  float *scratch = nullptr;
  if (nvfp4_status_t st = noalloc_scratch(&scratch)) return st;
  return launch_splitk(p, A, W, split_k, scratch, dev, reinterpret_cast<cudaStream_t>(stream));
}

nvfp4_status_t nvfp4_unswizzle_scales(const uint8_t *scales, int64_t rows, int64_t cols, uint8_t *out, int64_t ld,
                                      nvfp4_stream_t stream) {
  NvtxRange nvtx("nvfp4_unswizzle_scales");
  if (!scales || !out || rows < 1 || cols < 16 || ld < cols / 16) return NVFP4_ERR_INVALID_ARG;
  if (cols % 16 != 0 || rows > kMaxDim || cols > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(scales, 16)) return NVFP4_ERR_MISALIGNED;
  DeviceInfo *dev = nullptr;
  if (nvfp4_status_t st = current_device(&dev)) return st;
  UnswizzleArgs a;
  a.scales = scales;
  a.out = out;
  a.rows = rows;
  a.kb = cols / 16;
  a.kb_atoms = (a.kb + 3) / 4;
  a.ld = ld;
  const int64_t want = (rows * a.kb_atoms + kLayoutThreads - 1) / kLayoutThreads;
  const int64_t cap = int64_t(dev->sms) * 8;
  const int grid = static_cast<int>(want < cap ? want : cap);
  return launch_pdl(unswizzle_scales_kernel, dim3(grid), dim3(kLayoutThreads), 0,
                    reinterpret_cast<cudaStream_t>(stream), 1, a);
}

nvfp4_status_t nvfp4_pack_weight(const nvfp4_operand_t *parts, int nparts, uint8_t *codes, uint8_t *scales,
                                 int64_t rows_out, nvfp4_stream_t stream) {
  NvtxRange nvtx("nvfp4_pack_weight");
  if (!parts || !codes || !scales || nparts < 1 || nparts > NVFP4_MAX_SEGMENTS) return NVFP4_ERR_INVALID_ARG;
  PackArgs a{};
  const int64_t K = parts[0].K;
  int64_t row = 0;
  for (int i = 0; i < nparts; ++i) {
    const nvfp4_operand_t &q = parts[i];
    if (!q.codes || !q.scales || q.rows < 1 || q.K != K) return NVFP4_ERR_INVALID_ARG;
    if (!aligned(q.codes, 16) || !aligned(q.scales, 16)) return NVFP4_ERR_MISALIGNED;
    a.codes[i] = q.codes;
    a.scales[i] = q.scales;
    a.row0[i] = row;
    row += q.rows;
  }
  a.row0[nparts] = row;
  if (K < 64 || rows_out < row) return NVFP4_ERR_INVALID_ARG;
  if (K % 64 != 0 || rows_out > kMaxDim || K > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(codes, 16) || !aligned(scales, 16)) return NVFP4_ERR_MISALIGNED;
  DeviceInfo *dev = nullptr;
  if (nvfp4_status_t st = current_device(&dev)) return st;
  a.nparts = nparts;
  a.out_codes = codes;
  a.out_scales = scales;
  a.rows_out = rows_out;
  a.code_vecs = K / 32;
  a.kb_atoms = K / 64;
  const int64_t tasks = rows_out * a.code_vecs + (rows_out + 127) / 128 * 128 * a.kb_atoms;
  const int64_t want = (tasks + kLayoutThreads - 1) / kLayoutThreads;
  const int64_t cap = int64_t(dev->sms) * 8;
  const int grid = static_cast<int>(want < cap ? want : cap);
  return launch_pdl(pack_weight_kernel, dim3(grid), dim3(kLayoutThreads), 0, reinterpret_cast<cudaStream_t>(stream), 1,
                    a);
}

nvfp4_status_t nvfp4_fold_segments(uint8_t *scales, int64_t rows, int64_t cols, const nvfp4_segment_t *segs,
                                   int nseg, float *gs_common_out, nvfp4_stream_t stream) {
  NvtxRange nvtx("nvfp4_fold_segments");
  if (!scales || !segs || !gs_common_out || rows < 1 || cols < 1) return NVFP4_ERR_INVALID_ARG;
  if (nseg < 1 || nseg > NVFP4_MAX_SEGMENTS) return NVFP4_ERR_INVALID_ARG;
  if (cols % 16 != 0 || rows > kMaxDim || cols > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(scales, 16) || !aligned(gs_common_out, 4)) return NVFP4_ERR_MISALIGNED;
  FoldArgs a{};
  int64_t expect = 0;
  for (int i = 0; i < nseg; ++i) {
    if (!segs[i].gs_w || !aligned(segs[i].gs_w, 4)) return NVFP4_ERR_INVALID_ARG;
    if (segs[i].gs_w == gs_common_out) return NVFP4_ERR_INVALID_ARG;  // read while written
    if (segs[i].n_begin != expect || segs[i].n_end <= segs[i].n_begin) return NVFP4_ERR_INVALID_ARG;
    a.seg_begin[i] = static_cast<int>(segs[i].n_begin);
    a.seg_end[i] = static_cast<int>(segs[i].n_end);
    a.gs[i] = segs[i].gs_w;
    expect = segs[i].n_end;
  }
  if (expect != rows) return NVFP4_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  if (nvfp4_status_t st = current_device(&dev)) return st;
  a.scales = scales;
  a.rows = rows;
  a.kb = cols / 16;
  a.kb_atoms = (a.kb + 3) / 4;
  a.bytes = static_cast<int64_t>(nvfp4_scale_bytes(rows, cols));
  a.nseg = nseg;
  a.gs_common = gs_common_out;
  const int64_t want = (a.bytes / 16 + kFoldThreads - 1) / kFoldThreads;
  const int64_t cap = int64_t(dev->sms) * 8;
  const int grid = static_cast<int>(want < cap ? want : cap);
  return launch_pdl(fold_scales_kernel, dim3(grid), dim3(kFoldThreads), 0, reinterpret_cast<cudaStream_t>(stream), 1,
                    a);
}

nvfp4_status_t nvfp4_fp8_scale(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, float *scale_out,
                               nvfp4_stream_t stream) {
  NvtxRange nvtx("nvfp4_fp8_scale");
  if (!x_bf16 || !scale_out || rows < 1 || cols < 1 || ld < cols) return NVFP4_ERR_INVALID_ARG;
  if (cols % 16 != 0 || rows > kMaxDim || cols > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(x_bf16, 16) || ld % 8 != 0 || !aligned(scale_out, 4)) return NVFP4_ERR_MISALIGNED;
  DeviceInfo *dev = nullptr;
  if (nvfp4_status_t st = current_device(&dev)) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scale_out, 0, sizeof(float), s) != cudaSuccess) return NVFP4_ERR_CUDA;
  AmaxArgs a;
  a.x = static_cast<const uint16_t *>(x_bf16);
  a.rows = rows;
  a.cols = cols;
  a.ld = ld;
  a.amax_bits = reinterpret_cast<unsigned int *>(scale_out);
  const int64_t vecs = rows * (cols / 8);
  const int64_t want = (vecs / 4 + kAmaxThreads - 1) / kAmaxThreads;
  const int64_t cap = int64_t(dev->sms) * 4;
  const int grid = static_cast<int>(want < 1 ? 1 : (want < cap ? want : cap));
  if (nvfp4_status_t e = launch_pdl(amax_kernel, dim3(grid), dim3(kAmaxThreads), 0, s, 1, a)) return e;
  return launch_pdl(fp8_scale_finalize_kernel, dim3(1), dim3(1), 0, s, 1, scale_out);
}

nvfp4_status_t nvfp4_kv_cache_fp8(const void *k_bf16, const void *v_bf16, int64_t tokens, int64_t width,
                                  int64_t ld, const float *k_scale, const float *v_scale, const int64_t *slots,
                                  uint8_t *k_cache, uint8_t *v_cache, int64_t num_slots, nvfp4_stream_t stream) {
  NvtxRange nvtx("nvfp4_kv_cache_fp8");
  if (!k_bf16 || !v_bf16 || !k_scale || !v_scale || !slots || !k_cache || !v_cache) return NVFP4_ERR_INVALID_ARG;
  if (tokens < 1 || width < 1 || ld < width || num_slots < 1) return NVFP4_ERR_INVALID_ARG;
  if (width % 16 != 0 || tokens > kMaxDim || width > kMaxDim) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(k_bf16, 16) || !aligned(v_bf16, 16) || ld % 8 != 0 || !aligned(k_scale, 4) ||
      !aligned(v_scale, 4) || !aligned(slots, 8) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
    return NVFP4_ERR_MISALIGNED;
  DeviceInfo *dev = nullptr;
  if (nvfp4_status_t st = current_device(&dev)) return st;
  KvArgs a;
  a.k = static_cast<const uint16_t *>(k_bf16);
  a.v = static_cast<const uint16_t *>(v_bf16);
  a.tokens = tokens;
  a.width = width;
  a.ld = ld;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.slots = slots;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.num_slots = num_slots;
  const int64_t chunks = tokens * (width / 16);
  const int64_t want = (chunks + kKvThreads - 1) / kKvThreads;
  const int64_t cap = int64_t(dev->sms) * 8;
  const int grid = static_cast<int>(want < cap ? want : cap);
  return launch_pdl(kv_cache_fp8_kernel, dim3(grid), dim3(kKvThreads), 0, reinterpret_cast<cudaStream_t>(stream), 1,
                    a);
}

nvfp4_status_t nvfp4_gdn_recurrence(const void *q_bf16, const void *k_bf16, int64_t ld_qk, const void *v_bf16,
                                    int64_t ld_v, const float *g, const float *beta, int64_t ld_gate,
                                    const int32_t *cu_seqlens, int64_t n_seqs, int64_t tokens, int n_key_heads,
                                    int n_value_heads, int head_dim, float *state, int initial_state, void *out,
                                    int64_t ld_out, int out_kind, nvfp4_stream_t stream) {
  NvtxRange nvtx("nvfp4_gdn_recurrence");
  if (!q_bf16 || !k_bf16 || !v_bf16 || !g || !beta || !cu_seqlens || !state || !out) return NVFP4_ERR_INVALID_ARG;
  if (n_seqs < 1 || tokens < 0 || n_key_heads < 1 || n_value_heads < 1 || n_value_heads % n_key_heads != 0)
    return NVFP4_ERR_INVALID_ARG;
  if (out_kind != NVFP4_OUT_BF16 && out_kind != NVFP4_OUT_F32) return NVFP4_ERR_INVALID_ARG;
  if (head_dim != gdn::kDim || n_seqs > 65535 || n_value_heads > 65535 || tokens > kMaxDim)
    return NVFP4_ERR_UNSUPPORTED_SHAPE;
  const int64_t wk = int64_t(n_key_heads) * gdn::kDim, wv = int64_t(n_value_heads) * gdn::kDim;
  if (ld_qk < wk || ld_v < wv || ld_gate < n_value_heads || ld_out < wv) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(q_bf16, 16) || !aligned(k_bf16, 16) || !aligned(v_bf16, 16) || ld_qk % 8 != 0 || ld_v % 8 != 0 ||
      !aligned(g, 4) || !aligned(beta, 4) || !aligned(cu_seqlens, 4) || !aligned(state, 16) || !aligned(out, 16) ||
      ld_out % (out_kind == NVFP4_OUT_BF16 ? 8 : 4) != 0)
    return NVFP4_ERR_MISALIGNED;
  DeviceInfo *dev = nullptr;
  if (nvfp4_status_t st = current_device(&dev)) return st;
  gdn::Args a;
  a.q = static_cast<const uint16_t *>(q_bf16);
  a.k = static_cast<const uint16_t *>(k_bf16);
  a.v = static_cast<const uint16_t *>(v_bf16);
  a.ld_qk = ld_qk;
  a.ld_v = ld_v;
  a.g = g;
  a.beta = beta;
  a.ld_gate = ld_gate;
  a.cu_seqlens = cu_seqlens;
  a.tokens = tokens;
  a.heads_per_key = n_value_heads / n_key_heads;
  a.state = state;
  a.initial = initial_state != 0;
  a.out = out;
  a.ld_out = ld_out;
  a.out_fp32 = out_kind == NVFP4_OUT_F32;
  const dim3 grid(gdn::kColBlocks, n_value_heads, static_cast<unsigned>(n_seqs));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // Long sequences (prefill): the chunked form on the tensor cores.
  if (tokens >= 64 * n_seqs)
    return launch_pdl(gdn::chunk_kernel, dim3(gdn::kChunkColBlocks, n_value_heads, static_cast<unsigned>(n_seqs)),
                      dim3(gdn::kChunkThreads), sizeof(gdn::ChunkSmem), s, 1, a);
  // Shorter sequences stage fewer tokens at a time: a smaller shared-memory footprint,
  // so more CTAs per SM in the state-bound case, and less staging work spent on the
  // empty slots of a chunk.
  if (tokens >= 16 * n_seqs)
    return launch_pdl(gdn::recurrence_kernel<32>, grid, dim3(gdn::kThreads), sizeof(gdn::Smem<32>), s, 1, a);
  if (tokens >= 4 * n_seqs)
    return launch_pdl(gdn::recurrence_kernel<16>, grid, dim3(gdn::kThreads), sizeof(gdn::Smem<16>), s, 1, a);
  // About one token per sequence (decode): one warp per four state columns.
  return launch_pdl(gdn::column_kernel, dim3(gdn::kColBlocksPerHead, n_value_heads, static_cast<unsigned>(n_seqs)),
                    dim3(gdn::kColThreads), 0, s, 1, a);
}

nvfp4_status_t nvfp4_selftest_stalled_linear(const nvfp4_operand_t *A, const float *gs_a, const nvfp4_operand_t *W,
                                             const nvfp4_segment_t *segs, int nseg, float *out, int64_t ldo,
                                             int stall_stage, nvfp4_stream_t stream) {
  NvtxRange nvtx("nvfp4_selftest_stalled_linear");
  using namespace gemm;
  Params p;
  if (nvfp4_status_t st = prepare_linear(A, gs_a, W, segs, nseg, NVFP4_EPI_NONE, nullptr, out, NVFP4_OUT_F32, ldo, p))
    return st;
  if (p.M > BM || p.N > BN) return NVFP4_ERR_UNSUPPORTED_SHAPE;  // one tile, one CTA
  if (stall_stage < 0 || stall_stage >= p.k_tiles) return NVFP4_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  if (nvfp4_status_t st = current_device(&dev)) return st;
  CUtensorMap tmA, tmB;
  if (!make_codes_map(&tmA, A->codes, p.M, p.K) || !make_codes_map(&tmB, W->codes, p.N, p.K)) return NVFP4_ERR_CUDA;
  p.m_tiles = 1;
  p.n_tiles = 1;
  p.stall_stage = stall_stage;
  return launch_pdl(gemm_kernel<false, true>, dim3(1), dim3(NUM_THREADS), Plan1::BYTES,
                    reinterpret_cast<cudaStream_t>(stream), 1, tmA, tmB, p);
}

nvfp4_status_t nvfp4_get_device_status(int *code) {
  NvtxRange nvtx("nvfp4_get_device_status");
  if (!code) return NVFP4_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return NVFP4_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return NVFP4_ERR_CUDA;
  *code = v;
  return NVFP4_OK;
}

}  // extern "C"
