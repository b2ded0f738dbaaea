// fp4_api.cu -- the C ABI of libfp4 (declared in include/fp4.h): host-side argument
// validation, TMA descriptor construction and kernel launches on the caller's stream.
// The library allocates no device memory; all buffers belong to the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/fp4.h"
#include "common.cuh"
#include "gemm.cuh"
#include "quantize.cuh"

using namespace fp4k;

namespace {

// NVTX range around each compute entry point (named after it), so that a profiler's
// timeline shows which ABI call launched which kernels. Header-only NVTX: without a
// profiler attached a push/pop is a check of one pointer.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultWaitLimitNs = 1000000000ull;  // 1 s per pipeline wait

// ---------------------------------------------------------------- device facts (cached)
struct DeviceInfo {
  int sm_count = 0;
  int cc_major = 0;
  bool ok = false;
};
DeviceInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];

fp4_status current_device(int* dev_out, const DeviceInfo** info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP4_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FP4_ERR_UNSUPPORTED_DEVICE;
  std::call_once(g_dev_once[dev], [dev] {
    DeviceInfo d;
    if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) ==
            cudaSuccess)
      d.ok = true;
    g_dev[dev] = d;
  });
  const DeviceInfo& d = g_dev[dev];
  if (!d.ok) return FP4_ERR_CUDA;
  if (d.cc_major != 10) return FP4_ERR_UNSUPPORTED_DEVICE;
  *dev_out = dev;
  *info = &d;
  return FP4_OK;
}

// ---------------------------------------------------------------- TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

EncodeTiledFn encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode;
}

// 2-D row-major tensor [outer][inner] of `elem_bytes` elements.
bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, int elem_bytes, const void* base,
                 uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * static_cast<uint64_t>(elem_bytes)};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Raise a kernel's dynamic shared-memory limit once per device.
template <typename K>
cudaError_t ensure_smem(K kernel, int bytes, int dev, std::atomic<uint64_t>& done) {
  const uint64_t bit = 1ull << dev;
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int block_of(fp4_format f) { return f == FP4_NVFP4 ? 16 : 32; }
inline bool valid_format(fp4_format f) {
  return f == FP4_MXFP4 || f == FP4_NVFP4 || f == FP4_MXFP8;
}
// code bytes per element: 1/2 (FP4) or 1 (MXFP8)
inline int64_t code_bytes(int64_t elems, fp4_format f) { return f == FP4_MXFP8 ? elems : elems / 2; }

// ---------------------------------------------------------------- quantise launch
// The plain NVFP4 instances run the 512-thread quantize_wide_kernel (measured 2027 ->
// 2384 GB/s over the Llama layer's dual quantisations); MXFP4 (where the 256-thread
// kernel measured 4% faster), the variants (EXT) and MXFP8 run quantize_kernel. Both
// take two CTAs per SM.
template <int FMT, int HN, int MODE, bool AMAX, bool EXT, bool BANDED, int NITEMS = 1>
cudaError_t launch_q_kernel(const QuantBatch& qb, int grid, int dev, cudaStream_t s) {
  static std::atomic<uint64_t> done{0};
  if constexpr (!EXT && FMT == kFmtNV) {
    auto k = quantize_wide_kernel<FMT, HN, MODE, AMAX, BANDED, NITEMS>;
    cudaError_t e = ensure_smem(k, kQWSmemBytes, dev, done);
    if (e != cudaSuccess) return e;
    k<<<grid, kQWThreads, kQWSmemBytes, s>>>(qb);
  } else {
    auto k = quantize_kernel<FMT, HN, MODE, AMAX, EXT, BANDED, NITEMS>;
    constexpr int smem = kQSmemBytesOf(FMT, EXT);
    cudaError_t e = ensure_smem(k, smem, dev, done);
    if (e != cudaSuccess) return e;
    k<<<grid, kQThreads, smem, s>>>(qb);
  }
  return cudaGetLastError();
}

// Banded tile order (band_c < tiles_c) only for single-tensor launches of the
// column-layout modes of the plain kernels; everything else walks tiles row-major.
// Batches of several tensors (dual layout, plain quantiser only) take the instances
// compiled for kQMaxItems tensors.
template <int FMT, int HN, int MODE, bool AMAX, bool EXT>
cudaError_t launch_q(const QuantBatch& qb, int grid, int dev, cudaStream_t s) {
  if (qb.n > 1) {
    if constexpr (MODE == kModeDual && !EXT)
      return launch_q_kernel<FMT, HN, MODE, AMAX, EXT, false, kQMaxItems>(qb, grid, dev, s);
    else
      return cudaErrorInvalidValue;  // not reached: batches are dual and plain
  }
  if constexpr (MODE != kModeRow && !EXT) {
    if (qb.item[0].a.band_c < qb.item[0].a.tiles_c)
      return launch_q_kernel<FMT, HN, MODE, AMAX, EXT, true>(qb, grid, dev, s);
  }
  return launch_q_kernel<FMT, HN, MODE, AMAX, EXT, false>(qb, grid, dev, s);
}

template <int FMT, int HN, bool AMAX, bool EXT>
cudaError_t dispatch_mode(int mode, const QuantBatch& qb, int grid, int dev, cudaStream_t s) {
  switch (mode) {
    case kModeRow: return launch_q<FMT, HN, kModeRow, AMAX, EXT>(qb, grid, dev, s);
    case kModeCol: return launch_q<FMT, HN, kModeCol, AMAX, EXT>(qb, grid, dev, s);
    default: return launch_q<FMT, HN, kModeDual, AMAX, EXT>(qb, grid, dev, s);
  }
}

// ext: the variant kernels (random signs and/or stochastic rounding requested)
template <int FMT, bool AMAX>
cudaError_t dispatch_hn(int hn, int mode, const QuantBatch& qb, int grid, int dev,
                        cudaStream_t s) {
  const bool ext = qb.item[0].a.sr != 0 || qb.item[0].a.rht != 0;
  if (ext) {
    switch (hn) {
      case 0: return dispatch_mode<FMT, 0, AMAX, true>(mode, qb, grid, dev, s);
      case 16: return dispatch_mode<FMT, 16, AMAX, true>(mode, qb, grid, dev, s);
      default: return dispatch_mode<FMT, 32, AMAX, true>(mode, qb, grid, dev, s);
    }
  }
  switch (hn) {
    case 0: return dispatch_mode<FMT, 0, AMAX, false>(mode, qb, grid, dev, s);
    case 16: return dispatch_mode<FMT, 16, AMAX, false>(mode, qb, grid, dev, s);
    default: return dispatch_mode<FMT, 32, AMAX, false>(mode, qb, grid, dev, s);
  }
}

fp4_status validate_quant_common(const void* x, int64_t rows, int64_t cols, fp4_format fmt,
                                 int hn) {
  if (!valid_format(fmt)) return FP4_ERR_INVALID_ARG;
  if (hn != 0 && hn != 16 && hn != 32) return FP4_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0) return FP4_ERR_SHAPE;
  if (rows % 32 != 0 || cols % 32 != 0) return FP4_ERR_SHAPE;
  if (rows > (int64_t(1) << 31) - 128 || cols > (int64_t(1) << 31) - 128) return FP4_ERR_SHAPE;
  if (rows == 0 || cols == 0) return FP4_OK;
  if (!x) return FP4_ERR_INVALID_ARG;
  if (!aligned16(x)) return FP4_ERR_ALIGN;
  return FP4_OK;
}

// Host-side checks of one tensor of a quantise call (no device access). *skip is set
// for an empty tensor (nothing to do).
fp4_status check_item(bool* skip, const void* x, void* rcodes, void* rscales, void* ccodes,
                      void* cscales, float* ts, int64_t rows, int64_t cols, fp4_format fmt,
                      int hn, int mode, const fp4_quant_opts* opts) {
  *skip = false;
  fp4_status st = validate_quant_common(x, rows, cols, fmt, hn);
  if (st != FP4_OK) return st;
  const bool do_row = mode & kModeRow, do_col = mode & kModeCol;
  if (fmt != FP4_NVFP4 && ts) return FP4_ERR_INVALID_ARG;
  if (fmt == FP4_NVFP4 && !ts) return FP4_ERR_INVALID_ARG;
  if (fmt == FP4_MXFP8 && opts && (opts->amax || opts->stochastic || opts->random_signs))
    return FP4_ERR_INVALID_ARG;
  const float* amax_in = opts ? opts->amax : nullptr;
  if (amax_in && fmt != FP4_NVFP4) return FP4_ERR_INVALID_ARG;
  if (amax_in && (reinterpret_cast<uintptr_t>(amax_in) & 3u)) return FP4_ERR_ALIGN;
  if (rows == 0 || cols == 0) {
    *skip = true;
    return FP4_OK;
  }
  if ((do_row && (!rcodes || !rscales)) || (do_col && (!ccodes || !cscales)))
    return FP4_ERR_INVALID_ARG;
  if ((do_row && (!aligned16(rcodes) || !aligned16(rscales))) ||
      (do_col && (!aligned16(ccodes) || !aligned16(cscales))) ||
      (ts && (reinterpret_cast<uintptr_t>(ts) & 3u)))
    return FP4_ERR_ALIGN;
  return FP4_OK;
}

// One tensor of a quantise launch: validated arguments, TMA maps and kernel arguments.
// *skip is set for an empty tensor (nothing to do). For NVFP4 without a supplied amax,
// *amax_cells / *amax_bytes name the reduction cells the amax pass needs zeroed first.
fp4_status prepare_item(QuantItem* item, bool* skip, float** amax_cells, size_t* amax_bytes,
                        const void* x, void* rcodes, void* rscales, void* ccodes, void* cscales,
                        float* ts, int64_t rows, int64_t cols, fp4_format fmt, int hn, int mode,
                        const fp4_quant_opts* opts) {
  *amax_cells = nullptr;
  *amax_bytes = 0;
  fp4_status st = check_item(skip, x, rcodes, rscales, ccodes, cscales, ts, rows, cols, fmt, hn,
                             mode, opts);
  if (st != FP4_OK || *skip) return st;
  const bool do_row = mode & kModeRow, do_col = mode & kModeCol;
  const float* amax_in = opts ? opts->amax : nullptr;

  std::memset(item, 0, sizeof(*item));
  if (!make_map_2d(&item->in, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, cols, rows, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return FP4_ERR_CUDA;
  // code tiles: 128 rows x 64 bytes (FP4, 64B swizzle) or x 128 bytes (MXFP8, 128B swizzle)
  const uint32_t cbox = fmt == FP4_MXFP8 ? 128 : 64;
  const CUtensorMapSwizzle csw = fmt == FP4_MXFP8 ? CU_TENSOR_MAP_SWIZZLE_128B
                                                  : CU_TENSOR_MAP_SWIZZLE_64B;
  if (do_row && !make_map_2d(&item->rcodes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rcodes,
                             code_bytes(cols, fmt), rows, cbox, 128, csw))
    return FP4_ERR_CUDA;
  if (do_col && !make_map_2d(&item->ccodes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ccodes,
                             code_bytes(rows, fmt), cols, cbox, 128, csw))
    return FP4_ERR_CUDA;

  const int bs = block_of(fmt);
  QuantArgs& a = item->a;
  a.rows = rows;
  a.cols = cols;
  a.tiles_c = static_cast<int>(ceil_div(cols, 128));
  a.tiles_r = static_cast<int>(ceil_div(rows, 128));
  const int64_t tiles = int64_t(a.tiles_r) * a.tiles_c;
  // Bands of 32 tile columns once the column-layout codes are far larger than L2
  // (measured: a 2^30-element dual pass 0.57 -> 0.70 of HBM; at 2^27 and below plain
  // row-major order was 4% faster).
  // Bands of 16 tile columns for the MXFP4 column layout alone, else 32 (measured on
  // 2^30-element tensors: the MXFP4 column layout 0.76 -> 0.84 of HBM with 16; the dual
  // pass and NVFP4 no better, and worse on 4096-column tensors, which 32 leaves
  // unbanded).
  const int band = (!do_row && fmt == FP4_MXFP4) ? 16 : 32;
  a.band_c = (do_col && !(opts && (opts->stochastic || opts->random_signs)) && a.tiles_c > band &&
              code_bytes(rows * cols, fmt) > (int64_t(256) << 20))
                 ? band : a.tiles_c;
  if (tiles > INT32_MAX) return FP4_ERR_SHAPE;
  a.num_tiles = static_cast<int>(tiles);
  a.row_scales = static_cast<uint8_t*>(rscales);
  a.col_scales = static_cast<uint8_t*>(cscales);
  a.row_kb4 = static_cast<int>(ceil_div(cols / bs, 4));
  a.col_kb4 = static_cast<int>(ceil_div(rows / bs, 4));
  a.wait_limit_ns = kDefaultWaitLimitNs;
  if (opts) {
    a.sr = opts->stochastic != 0;
    a.rht = opts->random_signs != 0;
    a.sr_key[0] = static_cast<uint32_t>(opts->sr_seed);
    a.sr_key[1] = static_cast<uint32_t>(opts->sr_seed >> 32);
    a.sign_key[0] = static_cast<uint32_t>(opts->sign_seed);
    a.sign_key[1] = static_cast<uint32_t>(opts->sign_seed >> 32);
  }
  if (fmt == FP4_NVFP4) {
    // ts layout: single -> {S, amax}; dual -> {S_row, S_col, amax_row, amax_col}
    float* amax_r = nullptr;
    float* amax_c = nullptr;
    if (mode == kModeDual) {
      a.s_row_out = ts;
      a.s_col_out = ts + 1;
      amax_r = ts + 2;
      amax_c = ts + 3;
    } else if (mode == kModeRow) {
      a.s_row_out = ts;
      amax_r = ts + 1;
    } else {
      a.s_col_out = ts;
      amax_c = ts + 1;
    }
    if (amax_in) {
      // caller-supplied tensor amax: no amax pass; CTA 0 copies T into the amax slots
      a.amax_row = amax_r ? amax_in : nullptr;
      a.amax_col = amax_c ? (amax_r ? amax_in + 1 : amax_in) : nullptr;
      a.amax_row_copy = amax_r;
      a.amax_col_copy = amax_c;
    } else {
      a.amax_row = amax_r;
      a.amax_col = amax_c;
      a.amax_row_acc = reinterpret_cast<unsigned*>(amax_r);
      a.amax_col_acc = reinterpret_cast<unsigned*>(amax_c);
      *amax_cells = amax_r ? amax_r : amax_c;
      *amax_bytes = (amax_r && amax_c) ? 2 * sizeof(float) : sizeof(float);
    }
  }
  return FP4_OK;
}

// Launch the kernels of up to kQMaxItems prepared tensors of one format, rotation and
// mode: NVFP4 without supplied amaxes zeroes the amax cells, runs the amax pass and then
// the quantise pass; the other formats one quantise pass. `need_amax_pass` is whether
// the (all-alike) tensors take the amax pass.
fp4_status launch_batch(QuantBatch& qb, const float* const* amax_cells, const size_t* amax_bytes,
                        fp4_format fmt, int hn, int mode, bool need_amax_pass,
                        const DeviceInfo* info, int dev, cudaStream_t stream) {
  int tiles = 0;
  for (int k = 0; k < qb.n; ++k) {
    qb.item[k].tile0 = tiles;
    if (int64_t(tiles) + qb.item[k].a.num_tiles > INT32_MAX) return FP4_ERR_SHAPE;
    tiles += qb.item[k].a.num_tiles;
  }
  qb.num_tiles = tiles;
  if (qb.n == 0 || tiles == 0) return FP4_OK;
  const bool ext = qb.item[0].a.sr != 0 || qb.item[0].a.rht != 0;
  const int per_sm = fmt == FP4_MXFP8 ? kQCtasPerSMOf(kFmtMX8, false)
                     : fmt == FP4_MXFP4 ? kQCtasPerSMOf(kFmtMX, ext)
                                        : kQCtasPerSMOf(kFmtNV, ext);
  const int resident = per_sm * info->sm_count;
  const int grid = tiles < resident ? tiles : resident;
  cudaError_t e = cudaSuccess;
  if (fmt == FP4_MXFP4) {
    e = dispatch_hn<kFmtMX, false>(hn, mode, qb, grid, dev, stream);
  } else if (fmt == FP4_MXFP8) {
    switch (hn) {
      case 0: e = dispatch_mode<kFmtMX8, 0, false, false>(mode, qb, grid, dev, stream); break;
      case 16: e = dispatch_mode<kFmtMX8, 16, false, false>(mode, qb, grid, dev, stream); break;
      default: e = dispatch_mode<kFmtMX8, 32, false, false>(mode, qb, grid, dev, stream);
    }
  } else {
    if (need_amax_pass) {
      for (int k = 0; k < qb.n && e == cudaSuccess; ++k)
        e = cudaMemsetAsync(const_cast<float*>(amax_cells[k]), 0, amax_bytes[k], stream);
      if (e == cudaSuccess) e = dispatch_hn<kFmtNV, true>(hn, mode, qb, grid, dev, stream);
    }
    if (e == cudaSuccess) e = dispatch_hn<kFmtNV, false>(hn, mode, qb, grid, dev, stream);
  }
  return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

fp4_status quantize_impl(const void* x, void* rcodes, void* rscales, void* ccodes, void* cscales,
                         float* ts, int64_t rows, int64_t cols, fp4_format fmt, int hn, int mode,
                         cudaStream_t stream, const fp4_quant_opts* opts = nullptr) {
  // thread-local storage keeps the batch (2.3 KB of tensor maps and arguments) off
  // small host stacks
  static thread_local QuantBatch qb;
  bool skip;
  float* cells;
  size_t cell_bytes;
  fp4_status st = prepare_item(&qb.item[0], &skip, &cells, &cell_bytes, x, rcodes, rscales,
                               ccodes, cscales, ts, rows, cols, fmt, hn, mode, opts);
  if (st != FP4_OK || skip) return st;
  int dev;
  const DeviceInfo* info;
  st = current_device(&dev, &info);
  if (st != FP4_OK) return st;
  qb.n = 1;
  const float* cell_list[1] = {cells};
  return launch_batch(qb, cell_list, &cell_bytes, fmt, hn, mode, cells != nullptr, info, dev,
                      stream);
}

// ---------------------------------------------------------------- GEMM launch
template <int FMT, int OUT>
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& sa,
                        const CUtensorMap& sb, const GemmArgs& g, int grid, int dev,
                        cudaStream_t s) {
  static std::atomic<uint64_t> done{0};
  auto k = gemm_fp4_kernel<FMT, OUT>;
  cudaError_t e = ensure_smem(k, GemmCfg<FMT>::kSmemBytes, dev, done);
  if (e != cudaSuccess) return e;
  k<<<grid, kGSingleThreads, GemmCfg<FMT>::kSmemBytes, s>>>(a, b, sa, sb, g);
  return cudaGetLastError();
}

// CTA-pair kernel: the grid is two CTAs per pair tile, capped at the number of CTA pairs
// the device can hold at once (queried once per device), so the persistent loop never
// waits for a pair that is not resident.
template <int FMT, int QHN = -1>
cudaError_t launch_gemm_pair(const GemmGroup& grp, int dev, cudaStream_t s) {
  static std::atomic<uint64_t> done{0};
  static int max_pairs[kMaxDevices];
  static std::once_flag once[kMaxDevices];
  auto k = gemm_fp4_pair_kernel<FMT, QHN>;
  cudaError_t e = ensure_smem(k, PairCfg<FMT>::kSmemBytes, dev, done);
  if (e != cudaSuccess) return e;
  std::call_once(once[dev], [&] {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * g_dev[dev].sm_count / 2, 1, 1);
    cfg.blockDim = dim3(PairCfg<FMT>::kThreads, 1, 1);
    cfg.dynamicSmemBytes = PairCfg<FMT>::kSmemBytes;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k, &cfg) != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = g_dev[dev].sm_count / 2;
    }
    max_pairs[dev] = n;
  });
  const int pairs = grp.num_tiles < max_pairs[dev] ? grp.num_tiles : max_pairs[dev];
  k<<<2 * pairs, PairCfg<FMT>::kThreads, PairCfg<FMT>::kSmemBytes, s>>>(grp);
  return cudaGetLastError();
}

// Tile order for L2 reuse (see tile_coords). A band of tile rows keeps its A panels in
// L2 while B is streamed once per band, and the reverse for a band of tile columns. The
// band is as wide as a panel budget allows (a third of B200's 126 MB L2, which also
// carries the output stream), and the orientation with fewer estimated HBM operand bytes
// is taken.
constexpr double kL2PanelBudget = 40.0 * (1 << 20);

void choose_tile_order(GemmArgs& g, int64_t tile_rows, int64_t row_bytes_i) {
  const double row_bytes = double(row_bytes_i);  // code + scale bytes of one operand row
  const double panel_a = double(tile_rows) * row_bytes, panel_b = double(kGBN) * row_bytes;
  auto fit = [](double panel, int tiles) {
    const double n = kL2PanelBudget / panel;
    return n < 1.0 ? 1 : (n >= tiles ? tiles : static_cast<int>(n));
  };
  const int ga = fit(panel_a, g.tiles_m), gb = fit(panel_b, g.tiles_n);
  const double a_all = panel_a * g.tiles_m, b_all = panel_b * g.tiles_n;
  const double by_rows = a_all + b_all * double(ceil_div(g.tiles_m, ga));
  const double by_cols = b_all + a_all * double(ceil_div(g.tiles_n, gb));
  g.band_n = by_cols < by_rows ? 1 : 0;
  g.band = g.band_n ? gb : ga;
}

// Host checks of one GEMM (fp4_gemm, fp4_gemm_quant, a member of fp4_gemm_group); a
// problem with M or N zero passes them and is then skipped (*empty).
fp4_status check_gemm(const void* A, const void* As, const float* Ats, const void* B,
                      const void* Bs, const float* Bts, const void* C, int64_t M, int64_t N,
                      int64_t K, fp4_format fmt, fp4_out_dtype od, const void* q_codes,
                      const void* q_scales, int q_hn, bool* empty) {
  *empty = false;
  if (!valid_format(fmt)) return FP4_ERR_INVALID_ARG;
  if (od != FP4_OUT_F32 && od != FP4_OUT_BF16) return FP4_ERR_INVALID_ARG;
  const bool quant = q_hn >= 0;
  if (quant && (fmt == FP4_MXFP8 || od != FP4_OUT_BF16 || (q_hn != 0 && q_hn != 16 && q_hn != 32)))
    return FP4_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0 || M % 32 || N % 32 || K % 32) return FP4_ERR_SHAPE;
  if (M > (int64_t(1) << 31) - 256 || N > (int64_t(1) << 31) - 256 ||
      K > (int64_t(1) << 31) - 256)
    return FP4_ERR_SHAPE;
  if (fmt != FP4_NVFP4 && (Ats || Bts)) return FP4_ERR_INVALID_ARG;
  if (fmt == FP4_NVFP4 && (!Ats || !Bts)) return FP4_ERR_INVALID_ARG;
  if (M == 0 || N == 0) {
    *empty = true;
    return FP4_OK;
  }
  if (!C && !quant) return FP4_ERR_INVALID_ARG;
  if (quant && (!q_codes || !q_scales)) return FP4_ERR_INVALID_ARG;
  if (K == 0) return FP4_ERR_SHAPE;  // an empty contraction is not a launch the tiles express
  if (!A || !As || !B || !Bs) return FP4_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(As) || !aligned16(B) || !aligned16(Bs) || (C && !aligned16(C)))
    return FP4_ERR_ALIGN;
  if (quant && (!aligned16(q_codes) || !aligned16(q_scales))) return FP4_ERR_ALIGN;
  return FP4_OK;
}

// Operand maps and arguments of one GEMM for either kernel: the pair kernel (256-row
// tiles) or the one-CTA kernel (M <= 128, 128-row tiles). The output map (fp32 TMA-store
// epilogue of the pair kernel) is made by the caller.
fp4_status build_gemm(GemmProblem* P, bool pair, const void* A, const void* As,
                      const float* Ats, const void* B, const void* Bs, const float* Bts,
                      void* C, int64_t M, int64_t N, int64_t K, fp4_format fmt,
                      fp4_out_dtype od, void* q_codes, void* q_scales) {
  const int bs = block_of(fmt);
  const int64_t kb4 = ceil_div(K / bs, 4);
  const int slab_k = !pair ? kGBK
                     : fmt == FP4_MXFP4 ? PairCfg<kFmtMX>::kSlabK
                     : fmt == FP4_NVFP4 ? PairCfg<kFmtNV>::kSlabK
                                        : PairCfg<kFmtMX8>::kSlabK;
  const int atoms = slab_k / (4 * bs);
  const uint32_t b_box_rows = pair ? 128 : kGBN;
  const int64_t kbytes = code_bytes(K, fmt);
  if (!make_map_2d(&P->a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, A, kbytes, M, 128, kGBM,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&P->b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, kbytes, N, 128, b_box_rows,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&P->sa, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, As, kb4 * 64, ceil_div(M, 128),
                   atoms * 64, 1, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map_2d(&P->sb, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, Bs, kb4 * 64, ceil_div(N, 128),
                   atoms * 64, 2, CU_TENSOR_MAP_SWIZZLE_NONE))
    return FP4_ERR_CUDA;
  std::memset(&P->c, 0, sizeof(P->c));
  GemmArgs& g = P->g;
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.K = static_cast<int>(K);
  g.tiles_m = static_cast<int>(ceil_div(M, pair ? 256 : kGBM));
  g.tiles_n = static_cast<int>(ceil_div(N, kGBN));
  const int64_t tiles = int64_t(g.tiles_m) * g.tiles_n;
  if (tiles > INT32_MAX) return FP4_ERR_SHAPE;
  g.num_tiles = static_cast<int>(tiles);
  g.k_tiles = static_cast<int>(ceil_div(K, slab_k));
  choose_tile_order(g, pair ? 256 : kGBM, kbytes + K / bs);
  g.C = C;
  g.c_v8 = (reinterpret_cast<uintptr_t>(C) & 31) == 0 ? 1 : 0;
  g.sa = Ats;
  g.sb = Bts;
  g.wait_limit_ns = kDefaultWaitLimitNs;
  g.q_codes = static_cast<uint8_t*>(q_codes);
  g.q_scales = static_cast<uint8_t*>(q_scales);
  g.q_kb4 = static_cast<int>(ceil_div(N / 32, 4));
  g.m_pad = static_cast<int>(ceil_div(M, 128) * 128);
  P->tile0 = 0;
  P->out_bf16 = od == FP4_OUT_BF16 ? 1 : 0;
  if (pair && !P->out_bf16 &&
      !make_map_2d(&P->c, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, C, N, M, 8, 32,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return FP4_ERR_CUDA;
  return FP4_OK;
}

cudaError_t launch_group(const GemmGroup& grp, fp4_format fmt, int q_hn, int dev,
                         cudaStream_t stream) {
  if (q_hn >= 0) {
    switch (q_hn) {
      case 0:
        return fmt == FP4_MXFP4 ? launch_gemm_pair<kFmtMX, 0>(grp, dev, stream)
                                : launch_gemm_pair<kFmtNV, 0>(grp, dev, stream);
      case 16:
        return fmt == FP4_MXFP4 ? launch_gemm_pair<kFmtMX, 16>(grp, dev, stream)
                                : launch_gemm_pair<kFmtNV, 16>(grp, dev, stream);
      default:
        return fmt == FP4_MXFP4 ? launch_gemm_pair<kFmtMX, 32>(grp, dev, stream)
                                : launch_gemm_pair<kFmtNV, 32>(grp, dev, stream);
    }
  }
  if (fmt == FP4_MXFP4) return launch_gemm_pair<kFmtMX>(grp, dev, stream);
  if (fmt == FP4_MXFP8) return launch_gemm_pair<kFmtMX8>(grp, dev, stream);
  return launch_gemm_pair<kFmtNV>(grp, dev, stream);
}

// thread_local: the group is ~2.4 KB and copied into the launch's parameters.
thread_local GemmGroup t_group;

fp4_status gemm_impl(const void* A, const void* As, const float* Ats, const void* B,
                     const void* Bs, const float* Bts, void* C, int64_t M, int64_t N, int64_t K,
                     fp4_format fmt, fp4_out_dtype od, cudaStream_t stream,
                     void* q_codes = nullptr, void* q_scales = nullptr, int q_hn = -1) {
  bool empty;
  fp4_status st = check_gemm(A, As, Ats, B, Bs, Bts, C, M, N, K, fmt, od, q_codes, q_scales,
                             q_hn, &empty);
  if (st != FP4_OK || empty) return st;
  int dev;
  const DeviceInfo* info;
  st = current_device(&dev, &info);
  if (st != FP4_OK) return st;
  // Rows of 256 (M > 128) go to the CTA-pair kernel; a single 128-row band of M to the
  // one-CTA kernel. Each kernel has its own K per pipeline stage.
  // (The MXFP8 comparator always takes the pair kernel; M <= 128 is then one zero-filled
  // 256-row band.)
  const bool quant = q_hn >= 0;
  const bool pair = M > 128 || fmt == FP4_MXFP8 || quant;
  GemmGroup& grp = t_group;
  st = build_gemm(&grp.p[0], pair, A, As, Ats, B, Bs, Bts, C, M, N, K, fmt, od, q_codes,
                  q_scales);
  if (st != FP4_OK) return st;
  cudaError_t e;
  if (pair) {
    grp.n = 1;
    grp.num_tiles = grp.p[0].g.num_tiles;
    e = launch_group(grp, fmt, q_hn, dev, stream);
  } else {
    const GemmProblem& P = grp.p[0];
    const int grid = P.g.num_tiles < info->sm_count ? P.g.num_tiles : info->sm_count;
    if (fmt == FP4_MXFP4)
      e = od == FP4_OUT_F32 ? launch_gemm<kFmtMX, 0>(P.a, P.b, P.sa, P.sb, P.g, grid, dev, stream)
                            : launch_gemm<kFmtMX, 1>(P.a, P.b, P.sa, P.sb, P.g, grid, dev, stream);
    else
      e = od == FP4_OUT_F32 ? launch_gemm<kFmtNV, 0>(P.a, P.b, P.sa, P.sb, P.g, grid, dev, stream)
                            : launch_gemm<kFmtNV, 1>(P.a, P.b, P.sa, P.sb, P.g, grid, dev, stream);
  }
  return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

// Up to kGMaxProblems GEMMs of one format in one launch of the pair kernel. Problems
// with M or N zero are skipped; the rest run in order of decreasing K, so that the tiles
// left for the last wave are the cheapest ones.
// q_index >= 0: that member's epilogue also quantises its bf16 output (as fp4_gemm_quant,
// rotation q_hn) into q_codes / q_scales.
fp4_status gemm_group_impl(const fp4_gemm_desc* d, int n, fp4_format fmt, cudaStream_t stream,
                           int q_index = -1, void* q_codes = nullptr, void* q_scales = nullptr,
                           int q_hn = -1) {
  if (n < 1 || n > FP4_GEMM_GROUP_MAX || !d) return FP4_ERR_INVALID_ARG;
  if (q_index >= n || (q_index >= 0) != (q_hn >= 0)) return FP4_ERR_INVALID_ARG;
  int order[kGMaxProblems], used = 0;
  bool q_used = false;
  for (int i = 0; i < n; ++i) {
    bool empty;
    const bool qi = i == q_index;
    const fp4_status st = check_gemm(d[i].A_codes, d[i].A_scales, d[i].A_tensor_scale,
                                     d[i].B_codes, d[i].B_scales, d[i].B_tensor_scale, d[i].C,
                                     d[i].M, d[i].N, d[i].K, fmt, d[i].out_dtype,
                                     qi ? q_codes : nullptr, qi ? q_scales : nullptr,
                                     qi ? q_hn : -1, &empty);
    if (st != FP4_OK) return st;
    if (!empty) {
      order[used++] = i;
      q_used = q_used || qi;
    }
  }
  if (used == 0) return FP4_OK;
  for (int i = 1; i < used; ++i)  // stable insertion sort by decreasing K
    for (int j = i; j > 0 && d[order[j]].K > d[order[j - 1]].K; --j) {
      const int t = order[j];
      order[j] = order[j - 1];
      order[j - 1] = t;
    }
  int dev;
  const DeviceInfo* info;
  fp4_status st = current_device(&dev, &info);
  if (st != FP4_OK) return st;
  GemmGroup& grp = t_group;
  int64_t tiles = 0;
  for (int q = 0; q < used; ++q) {
    const fp4_gemm_desc& x = d[order[q]];
    const bool qi = order[q] == q_index;
    st = build_gemm(&grp.p[q], true, x.A_codes, x.A_scales, x.A_tensor_scale, x.B_codes,
                    x.B_scales, x.B_tensor_scale, x.C, x.M, x.N, x.K, fmt, x.out_dtype,
                    qi ? q_codes : nullptr, qi ? q_scales : nullptr);
    if (st != FP4_OK) return st;
    grp.p[q].tile0 = static_cast<int>(tiles);
    tiles += grp.p[q].g.num_tiles;
    if (tiles > INT32_MAX) return FP4_ERR_SHAPE;
  }
  grp.n = used;
  grp.num_tiles = static_cast<int>(tiles);
  return launch_group(grp, fmt, q_used ? q_hn : -1, dev, stream) == cudaSuccess ? FP4_OK
                                                                                 : FP4_ERR_CUDA;
}

// ---------------------------------------------------------------- linear-layer passes
inline size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

// Workspace of one pass: operand A (R_a x K') and operand B (R_b x K') quantised
// along the contraction K', plus 16 floats of NVFP4 tensor-scale cells.
struct WsPlan {
  size_t a_codes, a_scales, b_codes, b_scales, ts, total;
};

WsPlan plan_ws(int64_t ra, int64_t rb, int64_t kc, fp4_format fmt) {
  WsPlan p;
  size_t off = 0;
  p.a_codes = off;  off += align256(fp4_codes_bytes_fmt(ra, kc, fmt));
  p.a_scales = off; off += align256(fp4_scales_bytes(ra, kc, fmt));
  p.b_codes = off;  off += align256(fp4_codes_bytes_fmt(rb, kc, fmt));
  p.b_scales = off; off += align256(fp4_scales_bytes(rb, kc, fmt));
  p.ts = off;       off += 256;
  p.total = off;
  return p;
}

void pass_dims(fp4_pass pass, int64_t M, int64_t N, int64_t K, int64_t* ra, int64_t* rb,
               int64_t* kc) {
  switch (pass) {
    case FP4_PASS_FPROP: *ra = M; *rb = N; *kc = K; break;  // Y = X W^T
    case FP4_PASS_DGRAD: *ra = M; *rb = K; *kc = N; break;  // dX = dY W
    default: *ra = N; *rb = K; *kc = M; break;              // dW = dY^T X
  }
}

fp4_status linear_impl(fp4_pass pass, const void* P, const void* Q, void* out, int64_t M,
                       int64_t N, int64_t K, fp4_format fmt, int hn, fp4_out_dtype od, void* ws,
                       size_t ws_bytes, cudaStream_t stream) {
  if (!valid_format(fmt)) return FP4_ERR_INVALID_ARG;
  if (hn != 0 && hn != 16 && hn != 32) return FP4_ERR_INVALID_ARG;
  if (od != FP4_OUT_F32 && od != FP4_OUT_BF16) return FP4_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0 || M % 32 || N % 32 || K % 32) return FP4_ERR_SHAPE;
  int64_t ra, rb, kc;
  pass_dims(pass, M, N, K, &ra, &rb, &kc);
  if (ra == 0 || rb == 0) return FP4_OK;
  if (kc == 0) return FP4_ERR_SHAPE;
  if (!P || !Q || !out) return FP4_ERR_INVALID_ARG;
  const WsPlan p = plan_ws(ra, rb, kc, fmt);
  if (!ws || ws_bytes < p.total) return FP4_ERR_WORKSPACE;
  if (!aligned16(ws)) return FP4_ERR_ALIGN;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* ts = fmt == FP4_NVFP4 ? reinterpret_cast<float*>(w + p.ts) : nullptr;
  float* tsa = ts;
  float* tsb = ts ? ts + 4 : nullptr;
  fp4_status st;
  switch (pass) {
    case FP4_PASS_FPROP:  // A = X [M][K] rows, B = W [N][K] rows
      st = quantize_impl(P, w + p.a_codes, w + p.a_scales, nullptr, nullptr, tsa, M, K, fmt, hn,
                         kModeRow, stream);
      if (st == FP4_OK)
        st = quantize_impl(Q, w + p.b_codes, w + p.b_scales, nullptr, nullptr, tsb, N, K, fmt, hn,
                           kModeRow, stream);
      break;
    case FP4_PASS_DGRAD:  // A = dY [M][N] rows, B = W [N][K] along N -> [K][N]
      st = quantize_impl(P, w + p.a_codes, w + p.a_scales, nullptr, nullptr, tsa, M, N, fmt, hn,
                         kModeRow, stream);
      if (st == FP4_OK)
        st = quantize_impl(Q, nullptr, nullptr, w + p.b_codes, w + p.b_scales, tsb, N, K, fmt, hn,
                           kModeCol, stream);
      break;
    default:  // A = dY [M][N] along M -> [N][M], B = X [M][K] along M -> [K][M]
      st = quantize_impl(P, nullptr, nullptr, w + p.a_codes, w + p.a_scales, tsa, M, N, fmt, hn,
                         kModeCol, stream);
      if (st == FP4_OK)
        st = quantize_impl(Q, nullptr, nullptr, w + p.b_codes, w + p.b_scales, tsb, M, K, fmt, hn,
                           kModeCol, stream);
      break;
  }
  if (st != FP4_OK) return st;
  return gemm_impl(w + p.a_codes, w + p.a_scales, tsa, w + p.b_codes, w + p.b_scales, tsb, out, ra,
                   rb, kc, fmt, od, stream);
}

// ---------------------------------------------------------------- failure-path self test
__global__ void wait_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  // Nobody arrives: the bounded wait must give up and record the timeout.
  (void)mbar_wait(&bar, 0u, limit_ns);
}

}  // namespace

// ---------------------------------------------------------------- no-allocation scratch
// Scratch of fp4_linear_fprop_noalloc: a file-scope device array, so callers that
// cannot allocate still get the workspace the fprop pass needs. Host code must not
// pass g_noalloc_scratch itself to a kernel (on the host that name is only a
// stand-in); it passes the device address looked up once per device below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[FP4_NOALLOC_SCRATCH_BYTES];

std::atomic<void*> g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mutex;

// Device address of the scratch array on the current device, looked up with that
// device current. Only a successful lookup is cached: a failed one (for example a
// module load refused during a stream capture) clears the CUDA error it raised, so
// later calls and status checks do not see it, and is retried on the next call.
fp4_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP4_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FP4_ERR_UNSUPPORTED_DEVICE;
  void* p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    p = g_noalloc_ptr[dev].load(std::memory_order_relaxed);
    if (!p) {
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
        (void)cudaGetLastError();
        return FP4_ERR_CUDA;
      }
      g_noalloc_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return FP4_OK;
}

// ==================================================================== C ABI
extern "C" {

int fp4_abi_version(void) { return 2; }

size_t fp4_codes_bytes(int64_t rows, int64_t cols) {
  if (rows <= 0 || cols <= 0) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(cols) / 2;
}

size_t fp4_codes_bytes_fmt(int64_t rows, int64_t cols, fp4_format fmt) {
  if (rows <= 0 || cols <= 0 || !valid_format(fmt)) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(code_bytes(cols, fmt));
}

size_t fp4_scales_bytes(int64_t rows, int64_t cols, fp4_format fmt) {
  if (rows <= 0 || cols <= 0) return 0;
  const int64_t kb = cols / block_of(fmt);
  return static_cast<size_t>(ceil_div(rows, 128) * 128) * static_cast<size_t>(ceil_div(kb, 4) * 4);
}

fp4_status fp4_quantize(const void* x, void* codes, void* scales, float* ts, int64_t rows,
                        int64_t cols, fp4_format fmt, int hn, fp4_axis axis, fp4_stream_t stream) {
  NvtxRange nvtx_range("fp4_quantize");
  if (axis != FP4_AXIS_ROW && axis != FP4_AXIS_COL) return FP4_ERR_INVALID_ARG;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (axis == FP4_AXIS_ROW)
    return quantize_impl(x, codes, scales, nullptr, nullptr, ts, rows, cols, fmt, hn, kModeRow, s);
  return quantize_impl(x, nullptr, nullptr, codes, scales, ts, rows, cols, fmt, hn, kModeCol, s);
}

fp4_status fp4_quantize_dual(const void* x, void* row_codes, void* row_scales, void* col_codes,
                             void* col_scales, float* ts, int64_t rows, int64_t cols,
                             fp4_format fmt, int hn, fp4_stream_t stream) {
  NvtxRange nvtx_range("fp4_quantize_dual");
  return quantize_impl(x, row_codes, row_scales, col_codes, col_scales, ts, rows, cols, fmt, hn,
                       kModeDual, reinterpret_cast<cudaStream_t>(stream));
}
fp4_status fp4_quantize_opts(const void* x, void* codes, void* scales, float* ts, int64_t rows,
                             int64_t cols, fp4_format fmt, int hn, fp4_axis axis,
                             const fp4_quant_opts* opts, fp4_stream_t stream) {
  NvtxRange nvtx_range("fp4_quantize_opts");
  if (axis != FP4_AXIS_ROW && axis != FP4_AXIS_COL) return FP4_ERR_INVALID_ARG;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (axis == FP4_AXIS_ROW)
    return quantize_impl(x, codes, scales, nullptr, nullptr, ts, rows, cols, fmt, hn, kModeRow, s,
                         opts);
  return quantize_impl(x, nullptr, nullptr, codes, scales, ts, rows, cols, fmt, hn, kModeCol, s,
                       opts);
}
fp4_status fp4_quantize_dual_opts(const void* x, void* row_codes, void* row_scales,
                                  void* col_codes, void* col_scales, float* ts, int64_t rows,
                                  int64_t cols, fp4_format fmt, int hn,
                                  const fp4_quant_opts* opts, fp4_stream_t stream) {
  NvtxRange nvtx_range("fp4_quantize_dual_opts");
  return quantize_impl(x, row_codes, row_scales, col_codes, col_scales, ts, rows, cols, fmt, hn,
                       kModeDual, reinterpret_cast<cudaStream_t>(stream), opts);
}

fp4_status fp4_quantize_dual_batch(const fp4_quant_item* items, int n, fp4_format fmt, int hn,
                                   fp4_stream_t stream) {
  NvtxRange nvtx_range("fp4_quantize_dual_batch");
  if (n < 0 || (n > 0 && !items)) return FP4_ERR_INVALID_ARG;
  // every tensor is checked, then every map built, before anything is launched
  for (int i = 0; i < n; ++i) {
    const fp4_quant_item& t = items[i];
    bool skip;
    const fp4_status st = check_item(&skip, t.x_bf16, t.row_codes, t.row_scales, t.col_codes,
                                     t.col_scales, t.tensor_scale, t.rows, t.cols, fmt, hn,
                                     kModeDual, nullptr);
    if (st != FP4_OK) return st;
  }
  std::vector<QuantItem> prepared;
  std::vector<float*> cells;
  std::vector<size_t> cell_bytes;
  prepared.reserve(n);
  for (int i = 0; i < n; ++i) {
    const fp4_quant_item& t = items[i];
    QuantItem q;
    bool skip;
    float* c;
    size_t cb;
    const fp4_status st =
        prepare_item(&q, &skip, &c, &cb, t.x_bf16, t.row_codes, t.row_scales, t.col_codes,
                     t.col_scales, t.tensor_scale, t.rows, t.cols, fmt, hn, kModeDual, nullptr);
    if (st != FP4_OK) return st;
    if (skip) continue;
    prepared.push_back(q);
    cells.push_back(c);
    cell_bytes.push_back(cb);
  }
  if (prepared.empty()) return FP4_OK;
  int dev;
  const DeviceInfo* info;
  fp4_status st = current_device(&dev, &info);
  if (st != FP4_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  static thread_local QuantBatch qb;
  // tensors whose transposed codes want the banded tile order go alone; the rest in
  // groups of up to kQMaxItems, in the order given
  size_t i = 0;
  while (i < prepared.size() && st == FP4_OK) {
    qb.n = 0;
    const float* group_cells[kQMaxItems];
    size_t group_bytes[kQMaxItems];
    while (i < prepared.size() && qb.n < kQMaxItems) {
      const bool banded = prepared[i].a.band_c < prepared[i].a.tiles_c;
      if (banded && qb.n > 0) break;
      group_cells[qb.n] = cells[i];
      group_bytes[qb.n] = cell_bytes[i];
      qb.item[qb.n++] = prepared[i++];
      if (banded) break;
    }
    st = launch_batch(qb, group_cells, group_bytes, fmt, hn, kModeDual, fmt == FP4_NVFP4, info,
                      dev, s);
  }
  return st;
}

fp4_status fp4_gemm(const void* A, const void* As, const float* Ats, const void* B, const void* Bs,
                    const float* Bts, void* C, int64_t M, int64_t N, int64_t K, fp4_format fmt,
                    fp4_out_dtype od, fp4_stream_t stream) {
  NvtxRange nvtx_range("fp4_gemm");
  return gemm_impl(A, As, Ats, B, Bs, Bts, C, M, N, K, fmt, od,
                   reinterpret_cast<cudaStream_t>(stream));
}

fp4_status fp4_gemm_group(const fp4_gemm_desc* descs, int n, fp4_format fmt,
                          fp4_stream_t stream) {
  NvtxRange nvtx_range("fp4_gemm_group");
  return gemm_group_impl(descs, n, fmt, reinterpret_cast<cudaStream_t>(stream));
}

fp4_status fp4_gemm_group_quant(const fp4_gemm_desc* descs, int n, fp4_format fmt, int q_index,
                                void* Q_codes, void* Q_scales, int q_hadamard_n,
                                fp4_stream_t stream) {
  NvtxRange nvtx_range("fp4_gemm_group_quant");
  if (q_hadamard_n != 0 && q_hadamard_n != 16 && q_hadamard_n != 32) return FP4_ERR_INVALID_ARG;
  if (q_index < 0 || q_index >= n) return FP4_ERR_INVALID_ARG;
  return gemm_group_impl(descs, n, fmt, reinterpret_cast<cudaStream_t>(stream), q_index, Q_codes,
                         Q_scales, q_hadamard_n);
}

fp4_status fp4_gemm_quant(const void* A, const void* As, const float* Ats, const void* B,
                          const void* Bs, const float* Bts, void* C, void* Q_codes,
                          void* Q_scales, int64_t M, int64_t N, int64_t K, fp4_format fmt,
                          int q_hadamard_n, fp4_stream_t stream) {
  NvtxRange nvtx_range("fp4_gemm_quant");
  if (q_hadamard_n != 0 && q_hadamard_n != 16 && q_hadamard_n != 32) return FP4_ERR_INVALID_ARG;
  return gemm_impl(A, As, Ats, B, Bs, Bts, C, M, N, K, fmt, FP4_OUT_BF16,
                   reinterpret_cast<cudaStream_t>(stream), Q_codes, Q_scales, q_hadamard_n);
}

size_t fp4_linear_workspace_size(fp4_pass pass, int64_t M, int64_t N, int64_t K, fp4_format fmt) {
  if (pass != FP4_PASS_FPROP && pass != FP4_PASS_DGRAD && pass != FP4_PASS_WGRAD) return 0;
  if (!valid_format(fmt)) return 0;
  if (M < 0 || N < 0 || K < 0) return 0;
  int64_t ra, rb, kc;
  pass_dims(pass, M, N, K, &ra, &rb, &kc);
  return plan_ws(ra, rb, kc, fmt).total;
}

fp4_status fp4_linear_fprop(const void* X, const void* W, void* Y, int64_t M, int64_t N, int64_t K,
                            fp4_format fmt, int hn, fp4_out_dtype od, void* ws, size_t ws_bytes,
                            fp4_stream_t stream) {
  NvtxRange nvtx_range("fp4_linear_fprop");
  return linear_impl(FP4_PASS_FPROP, X, W, Y, M, N, K, fmt, hn, od, ws, ws_bytes,
                     reinterpret_cast<cudaStream_t>(stream));
}

fp4_status fp4_linear_dgrad(const void* dY, const void* W, void* dX, int64_t M, int64_t N,
                            int64_t K, fp4_format fmt, int hn, fp4_out_dtype od, void* ws,
                            size_t ws_bytes, fp4_stream_t stream) {
  NvtxRange nvtx_range("fp4_linear_dgrad");
  return linear_impl(FP4_PASS_DGRAD, dY, W, dX, M, N, K, fmt, hn, od, ws, ws_bytes,
                     reinterpret_cast<cudaStream_t>(stream));
}

fp4_status fp4_linear_wgrad(const void* dY, const void* X, void* dW, int64_t M, int64_t N,
                            int64_t K, fp4_format fmt, int hn, fp4_out_dtype od, void* ws,
                            size_t ws_bytes, fp4_stream_t stream) {
  NvtxRange nvtx_range("fp4_linear_wgrad");
  return linear_impl(FP4_PASS_WGRAD, dY, X, dW, M, N, K, fmt, hn, od, ws, ws_bytes,
                     reinterpret_cast<cudaStream_t>(stream));
}

// Workspace of fp4_linear_step: for X [M][K], W [N][K] and dY [M][N] in turn, the row
// codes and scales, the column codes and scales and 16 floats of NVFP4 tensor-scale
// cells ({row S, column S, ...} as fp4_quantize_dual writes them), each 256-byte aligned.
struct StepPlan {
  size_t rc[3], rs[3], cc[3], cs[3], ts[3], total;
};
StepPlan plan_step(int64_t M, int64_t N, int64_t K, fp4_format fmt) {
  const int64_t rows[3] = {M, N, M}, cols[3] = {K, K, N};
  StepPlan p;
  size_t off = 0;
  for (int t = 0; t < 3; ++t) {
    p.rc[t] = off; off += align256(fp4_codes_bytes_fmt(rows[t], cols[t], fmt));
    p.rs[t] = off; off += align256(fp4_scales_bytes(rows[t], cols[t], fmt));
    p.cc[t] = off; off += align256(fp4_codes_bytes_fmt(cols[t], rows[t], fmt));
    p.cs[t] = off; off += align256(fp4_scales_bytes(cols[t], rows[t], fmt));
    p.ts[t] = off; off += 256;
  }
  p.total = off;
  return p;
}

size_t fp4_linear_step_workspace_size(int64_t M, int64_t N, int64_t K, fp4_format fmt) {
  if (!valid_format(fmt) || M < 0 || N < 0 || K < 0) return 0;
  return plan_step(M, N, K, fmt).total;
}

fp4_status fp4_linear_step(const void* X, const void* W, const void* dY, void* Y, void* dX,
                           void* dW, int64_t M, int64_t N, int64_t K, fp4_format fmt, int hn,
                           void* ws, size_t ws_bytes, fp4_stream_t stream) {
  NvtxRange nvtx_range("fp4_linear_step");
  if (!valid_format(fmt)) return FP4_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0 || M % 32 || N % 32 || K % 32) return FP4_ERR_SHAPE;
  if (M == 0 || N == 0 || K == 0) return FP4_OK;
  const StepPlan p = plan_step(M, N, K, fmt);
  if (!ws || ws_bytes < p.total) return FP4_ERR_WORKSPACE;
  if (!aligned16(ws)) return FP4_ERR_ALIGN;
  uint8_t* w = static_cast<uint8_t*>(ws);
  const bool nv = fmt == FP4_NVFP4;
  const void* src[3] = {X, W, dY};
  const int64_t rows[3] = {M, N, M}, cols[3] = {K, K, N};
  fp4_quant_item items[3];
  float* ts[3];
  for (int t = 0; t < 3; ++t) {
    ts[t] = reinterpret_cast<float*>(w + p.ts[t]);
    items[t] = fp4_quant_item{src[t], w + p.rc[t], w + p.rs[t], w + p.cc[t], w + p.cs[t],
                              nv ? ts[t] : nullptr, rows[t], cols[t]};
  }
  enum { kX = 0, kW = 1, kDY = 2 };
  auto S = [&](int t, int layout) -> const float* { return nv ? ts[t] + layout : nullptr; };
  // Fprop: Q_row(X) . Q_row(W)^T; Dgrad: Q_row(dY) . Q_col(W)^T; Wgrad: Q_col(dY) . Q_col(X)^T
  const fp4_gemm_desc descs[3] = {
      {w + p.rc[kX], w + p.rs[kX], S(kX, 0), w + p.rc[kW], w + p.rs[kW], S(kW, 0), Y, M, N, K,
       FP4_OUT_BF16},
      {w + p.rc[kDY], w + p.rs[kDY], S(kDY, 0), w + p.cc[kW], w + p.cs[kW], S(kW, 1), dX, M, K, N,
       FP4_OUT_BF16},
      {w + p.cc[kDY], w + p.cs[kDY], S(kDY, 1), w + p.cc[kX], w + p.cs[kX], S(kX, 1), dW, N, K, M,
       FP4_OUT_F32}};
  // both calls' host checks before either launches
  for (int i = 0; i < 3; ++i) {
    bool empty;
    const fp4_gemm_desc& d = descs[i];
    const fp4_status st = check_gemm(d.A_codes, d.A_scales, d.A_tensor_scale, d.B_codes,
                                     d.B_scales, d.B_tensor_scale, d.C, d.M, d.N, d.K, fmt,
                                     d.out_dtype, nullptr, nullptr, -1, &empty);
    if (st != FP4_OK) return st;
  }
  for (int t = 0; t < 3; ++t) {
    bool skip;
    const fp4_quant_item& q = items[t];
    const fp4_status st = check_item(&skip, q.x_bf16, q.row_codes, q.row_scales, q.col_codes,
                                     q.col_scales, q.tensor_scale, q.rows, q.cols, fmt, hn,
                                     kModeDual, nullptr);
    if (st != FP4_OK) return st;
  }
  fp4_status st = fp4_quantize_dual_batch(items, 3, fmt, hn, stream);
  if (st != FP4_OK) return st;
  return gemm_group_impl(descs, 3, fmt, reinterpret_cast<cudaStream_t>(stream));
}

fp4_status fp4_linear_fprop_noalloc(const void* X, const void* W, void* Y, int64_t M, int64_t N,
                                    int64_t K, fp4_format fmt, int hn, fp4_out_dtype od,
                                    fp4_stream_t stream) {
  NvtxRange nvtx_range("fp4_linear_fprop_noalloc");
  if (fp4_linear_workspace_size(FP4_PASS_FPROP, M, N, K, fmt) > FP4_NOALLOC_SCRATCH_BYTES)
    return FP4_ERR_WORKSPACE;
  int dev;
  const DeviceInfo* info;
  fp4_status st = current_device(&dev, &info);
  if (st != FP4_OK) return st;
  void* ws = nullptr;
  st = noalloc_scratch(&ws);
  if (st != FP4_OK) return st;
  return linear_impl(FP4_PASS_FPROP, X, W, Y, M, N, K, fmt, hn, od, ws, FP4_NOALLOC_SCRATCH_BYTES,
                     reinterpret_cast<cudaStream_t>(stream));
}

fp4_status fp4_check_status(fp4_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FP4_ERR_CUDA;
  unsigned word = 0;
  const unsigned zero = 0;
  if (cudaMemcpyFromSymbol(&word, g_status_word, sizeof(word)) != cudaSuccess) return FP4_ERR_CUDA;
  if (word != 0 && cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero)) != cudaSuccess)
    return FP4_ERR_CUDA;
  if (word & kDevErrBounds) return FP4_ERR_BOUNDS;
  return (word & kDevErrTimeout) ? FP4_ERR_TIMEOUT : FP4_OK;
}

fp4_status fp4_selftest_timeout(uint64_t timeout_ns, fp4_stream_t stream) {
  NvtxRange nvtx_range("fp4_selftest_timeout");
  int dev;
  const DeviceInfo* info;
  fp4_status st = current_device(&dev, &info);
  if (st != FP4_OK) return st;
  wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(timeout_ns);
  return cudaGetLastError() == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

const char* fp4_status_string(fp4_status s) {
  switch (s) {
    case FP4_OK: return "ok";
    case FP4_ERR_INVALID_ARG: return "invalid argument";
    case FP4_ERR_SHAPE: return "unsupported shape";
    case FP4_ERR_ALIGN: return "pointer not 16-byte aligned";
    case FP4_ERR_UNSUPPORTED_DEVICE: return "device is not sm_100 (B200)";
    case FP4_ERR_CUDA: return "CUDA error";
    case FP4_ERR_TIMEOUT: return "device pipeline wait timed out";
    case FP4_ERR_WORKSPACE: return "workspace missing or too small";
    case FP4_ERR_BOUNDS: return "device-side bounds check failed (debug build)";
  }
  return "unknown status";
}

}  // extern "C"
