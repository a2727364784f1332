// C ABI of the FP8 block-scaled GEMM library (see include/fp8gemm.h):
// argument validation, TMA descriptor encoding, tile-shape and split-K
// selection, and kernel launches. One translation unit holds every kernel.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "fp8gemm.h"
#include "gemm.cuh"
#include "ep.cuh"
#include "peak.cuh"
#include "gemm_mx.cuh"
#include "quant.cuh"

namespace fg {
namespace {

__device__ int g_status_word;  // device status (FG_DEVICE_*), read by fg_get_device_status

thread_local std::string g_last_error;

fg_status fail(fg_status code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

fg_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FG_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sm_count = 0;
  int* status = nullptr;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

fg_status device_info(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FG_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
      return fail(FG_ERR_UNSUPPORTED, "built for sm_100a, device %d is sm_%d%d", dev, major,
                  minor);
    e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_status_word);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
    d.status = static_cast<int*>(p);
    d.ready = true;
  }
  *out = &d;
  return FG_OK;
}

uint64_t wait_limit_ns() {
  static uint64_t v = [] {
    const char* s = std::getenv("FG_WAIT_TIMEOUT_MS");
    const long ms = s ? std::atol(s) : 2000;
    return static_cast<uint64_t>(ms > 0 ? ms : 2000) * 1000000ull;
  }();
  return v;
}

// ---------------------------------------------------------------- TMA maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

fg_status encode_fn(EncodeTiledFn* out) {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (!fn) return fail(FG_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(err));
  *out = fn;
  return FG_OK;
}

// Encoded tensor maps, reused across calls: a map is a pure function of its
// encoding parameters, so a hit is always exact. Direct-mapped by a hash of
// the parameters; a miss re-encodes and replaces the slot.
struct MapKey {
  const void* base;
  uint64_t inner, outer, row_bytes;
  uint32_t box_inner, box_outer;
  int dt, swz;
  bool operator==(const MapKey& o) const {
    return base == o.base && inner == o.inner && outer == o.outer && row_bytes == o.row_bytes &&
           box_inner == o.box_inner && box_outer == o.box_outer && dt == o.dt && swz == o.swz;
  }
};
struct MapSlot {
  bool used = false;
  MapKey key{};
  CUtensorMap map;
};
constexpr int kMapSlots = 256;
std::mutex g_map_mu;
MapSlot g_map_slots[kMapSlots];

size_t map_slot(const MapKey& k) {
  uint64_t h = reinterpret_cast<uintptr_t>(k.base) * 0x9E3779B97F4A7C15ull;
  h ^= (k.inner * 31 + k.outer) * 0xC2B2AE3D27D4EB4Full;
  h ^= (static_cast<uint64_t>(k.box_inner) << 32 | k.box_outer) + static_cast<uint64_t>(k.dt * 7 + k.swz);
  return static_cast<size_t>((h ^ (h >> 29)) % kMapSlots);
}

// 2-D row-major tensor: `inner` elements per row (contiguous), `outer` rows,
// `row_bytes` between rows; box of box_inner x box_outer elements.
fg_status make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint64_t inner,
                   uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                   CUtensorMapSwizzle swz, const char* what) {
  const MapKey key{base, inner, outer, row_bytes, box_inner, box_outer, static_cast<int>(dt),
                   static_cast<int>(swz)};
  const size_t slot = map_slot(key);
  {
    std::lock_guard<std::mutex> lock(g_map_mu);
    if (g_map_slots[slot].used && g_map_slots[slot].key == key) {
      *map = g_map_slots[slot].map;
      return FG_OK;
    }
  }
  EncodeTiledFn fn;
  fg_status st = encode_fn(&fn);
  if (st != FG_OK) return st;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(FG_ERR_UNSUPPORTED, "cuTensorMapEncodeTiled(%s) failed with %d", what,
                static_cast<int>(r));
  std::lock_guard<std::mutex> lock(g_map_mu);
  g_map_slots[slot].used = true;
  g_map_slots[slot].key = key;
  g_map_slots[slot].map = *map;
  return FG_OK;
}

// ---------------------------------------------------------------- validation

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fg_status check_ptr(const void* p, const char* name) {
  if (!p) return fail(FG_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(FG_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return FG_OK;
}

#define FG_TRY(expr)                 \
  do {                               \
    const fg_status _s = (expr);     \
    if (_s != FG_OK) return _s;      \
  } while (0)

int sfa_stride(int M) { return (M + 3) / 4 * 4; }

// ---------------------------------------------------------------- GEMM configs

//                        BT   BW   swap  stages PW split K blocks/stage
using CfgNormal = GemmCfg<128, 256, false, 3, 8, 1, 1>;
using CfgPair = GemmCfg<128, 256, false, 4, 8, 1, 1, true>;  // dense: CTA pairs, 256 x 256 tiles
using CfgSwap16 = GemmCfg<16, 128, true, 5, 4, 1, 2>;
using CfgSwap32 = GemmCfg<32, 128, true, 5, 4, 1, 2>;
using CfgSwap64 = GemmCfg<64, 128, true, 4, 4, 1, 2>;
using CfgSwap16S2 = GemmCfg<16, 128, true, 5, 4, 2, 2>;
using CfgSwap32S2 = GemmCfg<32, 128, true, 4, 4, 2, 2>;
using CfgSwap64S2 = GemmCfg<64, 128, true, 3, 4, 2, 2>;
using CfgSwap16S4 = GemmCfg<16, 128, true, 5, 4, 4, 2>;
using CfgSwap32S4 = GemmCfg<32, 128, true, 4, 4, 4, 2>;
using CfgSwap64S4 = GemmCfg<64, 128, true, 3, 4, 4, 2>;

struct KernelInfo {
  std::atomic<bool> attr_set{false};  // published after max_clusters (release)
  int max_clusters = 0;  // max co-resident clusters (split-K and pair configs)
};

// One-time set-up of a kernel on a device, safe when several host threads
// make their first call at once: double-checked under g_mu, and the flag is
// published only after every field it guards has been written.
template <class C, int FORM>
fg_status kernel_info(int dev, KernelInfo** out) {
  static KernelInfo info[kMaxDevices];
  KernelInfo& k = info[dev];
  if (k.attr_set.load(std::memory_order_acquire)) {
    *out = &k;
    return FG_OK;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!k.attr_set.load(std::memory_order_relaxed)) {
    cudaError_t e = cudaFuncSetAttribute(fp8_gemm_kernel<C, FORM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::smem_bytes(FORM));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    if (C::REG_SPLIT) {
      // the warpgroup register split draws on the launch allocation: it must
      // be exactly what the split was sized for, or the increase would wait
      cudaFuncAttributes fa;
      e = cudaFuncGetAttributes(&fa, fp8_gemm_kernel<C, FORM>);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
      if (fa.numRegs != C::MAX_REGS)
        return fail(FG_ERR_UNSUPPORTED, "kernel built with %d registers per thread, register split needs %d",
                    fa.numRegs, C::MAX_REGS);
    }
    if (C::CLUSTER > 1) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = C::CLUSTER;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(C::CLUSTER * 64);
      cfg.blockDim = dim3(C::NUM_THREADS);
      cfg.dynamicSmemBytes = C::smem_bytes(FORM);
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      e = cudaOccupancyMaxActiveClusters(&n, fp8_gemm_kernel<C, FORM>, &cfg);
      if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveClusters");
      if (n < 1) return fail(FG_ERR_UNSUPPORTED, "no cluster of %d CTAs fits", C::CLUSTER);
      k.max_clusters = n;
    }
    k.attr_set.store(true, std::memory_order_release);
  }
  *out = &k;
  return FG_OK;
}

struct Problem {
  int form;
  const uint8_t* A;
  const float* sfa;
  const uint8_t* B;
  const float* sfb;
  uint16_t* D;
  const int32_t* m_indices;
  const int32_t* masked_m;
  int M;  // rows of one token slab
  int N, K, G;
  int slabs;  // token slabs in A (G for masked, else 1)
};

struct Plan {
  int bt;      // token rows per tile (128 = normal form, else swapped)
  int splits;  // CTAs per cluster sharing one tile's K blocks
  int num_mt, num_nt;
};

// Tile shape and split-K factor. The swapped product (tokens on the MMA's N
// side) is used for dense M <= 64 and for masked layouts whose expected rows
// per expert are <= 64; when it leaves most SMs idle, K is split across a
// cluster of 2 or 4 CTAs.
Plan plan_for(const Problem& pr, int sm_count, int expected_m) {
  Plan pl{};
  const int KB = pr.K / 128;
  int small_m = 1 << 30;
  if (pr.form == kFormDense) small_m = pr.M;
  if (pr.form == kFormMasked) small_m = expected_m;
  if (small_m <= 16) pl.bt = 16;
  else if (small_m <= 32) pl.bt = 32;
  else if (small_m <= 64) pl.bt = 64;
  else pl.bt = 128;
  if (pr.form == kFormMasked && pl.bt < 64) pl.bt = 64;  // one swapped shape for masked
  pl.num_mt = (pr.M + pl.bt - 1) / pl.bt;
  const int tile_w = pl.bt == 128 ? CfgNormal::BW : 128;  // weight rows per tile
  pl.num_nt = (pr.N + tile_w - 1) / tile_w;
  pl.splits = 1;
  if (pr.form == kFormDense && pl.bt < 128) {
    const int tiles = pl.num_mt * pl.num_nt;
    for (int s : {4, 2}) {
      if (tiles * s <= sm_count && KB >= 2 * s) {
        pl.splits = s;
        break;
      }
    }
  }
  return pl;
}

template <class C, int FORM>
fg_status launch_gemm(const Problem& pr, const Plan& pl, const DeviceInfo& dev, int dev_id,
                      cudaStream_t stream) {
  static_assert(C::smem_bytes(FORM) <= 232448, "shared memory per CTA");
  KernelInfo* ki = nullptr;
  FG_TRY((kernel_info<C, FORM>(dev_id, &ki)));
  const int KB = pr.K / 128;
  CUtensorMap tmA, tmB, tmSA, tmD;
  FG_TRY(make_map(&tmA, pr.A, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.K,
                  static_cast<uint64_t>(pr.slabs) * pr.M, pr.K, 128, C::BT,
                  CU_TENSOR_MAP_SWIZZLE_128B, "A"));
  FG_TRY(make_map(&tmB, pr.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.K,
                  static_cast<uint64_t>(pr.G) * pr.N, pr.K, 128, C::B_ROWS,
                  CU_TENSOR_MAP_SWIZZLE_128B, "B"));
  FG_TRY(make_map(&tmSA, pr.sfa, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, pr.M,
                  static_cast<uint64_t>(pr.slabs) * KB,
                  static_cast<uint64_t>(sfa_stride(pr.M)) * 4, C::BT, 1,
                  CU_TENSOR_MAP_SWIZZLE_NONE, "SFA"));
  // D as rows x N bf16: boxes of 32 rows x 64 columns with 128-byte
  // swizzling (normal-form epilogue) or SLICE_M rows x 128 columns (split-K
  // slices of the swapped form); unused, and left zero, otherwise
  std::memset(&tmD, 0, sizeof(tmD));
  if (C::EPI_TMA)
    FG_TRY(make_map(&tmD, pr.D, CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.N,
                    static_cast<uint64_t>(pr.slabs) * pr.M, static_cast<uint64_t>(pr.N) * 2,
                    64, 32, CU_TENSOR_MAP_SWIZZLE_128B, "D"));
  else if (C::RED_TMA && FORM == kFormDense)
    FG_TRY(make_map(&tmD, pr.D, CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.N,
                    static_cast<uint64_t>(pr.slabs) * pr.M, static_cast<uint64_t>(pr.N) * 2,
                    128, C::SLICE_M, CU_TENSOR_MAP_SWIZZLE_NONE, "D"));
  GemmParams p{};
  p.M = pr.M;
  p.N = pr.N;
  p.K = pr.K;
  p.G = pr.G;
  p.KB = KB;
  p.NB = (pr.N + 127) / 128;
  p.num_mt = pl.num_mt;
  p.num_nt = pl.num_nt;
  p.sfb = pr.sfb;
  p.D = pr.D;
  p.m_indices = pr.m_indices;
  p.masked_m = pr.masked_m;
  p.status = dev.status;
  p.timeout_ns = wait_limit_ns();
  int64_t tiles = static_cast<int64_t>(C::PAIR ? (pl.num_mt + 1) / 2 : pl.num_mt) * pl.num_nt;
  if (FORM == kFormMasked) tiles *= pr.G;  // upper bound: masked_m lives on the device
  int64_t grid;
  if (C::CLUSTER > 1) {
    grid = C::CLUSTER * std::max<int64_t>(1, std::min<int64_t>(tiles, ki->max_clusters));
  } else {
    grid = std::max<int64_t>(1, std::min<int64_t>(tiles, dev.sm_count));
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(C::NUM_THREADS);
  cfg.dynamicSmemBytes = C::smem_bytes(FORM);
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // prologue overlaps the
  attr[0].val.programmaticStreamSerializationAllowed = 1;           // previous kernel
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (C::CLUSTER > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = C::CLUSTER;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  const cudaError_t e = cudaLaunchKernelEx(&cfg, fp8_gemm_kernel<C, FORM>, tmA, tmB, tmSA, tmD, p);
  if (e != cudaSuccess) return cuda_fail(e, "fp8_gemm_kernel launch");
  return FG_OK;
}

template <int FORM>
fg_status dispatch(const Problem& pr, const Plan& pl, const DeviceInfo& dev, int dev_id,
                   cudaStream_t stream) {
  if (pl.bt == 128) {
    // dense: CTA pairs; grouped forms: single-CTA tiles, which are as fast
    // once promotion is the limit and keep groups 128-row aligned
    if constexpr (FORM == kFormDense) return launch_gemm<CfgPair, FORM>(pr, pl, dev, dev_id, stream);
    return launch_gemm<CfgNormal, FORM>(pr, pl, dev, dev_id, stream);
  }
  if constexpr (FORM == kFormMasked) {
    if (pl.bt == 64) return launch_gemm<CfgSwap64, FORM>(pr, pl, dev, dev_id, stream);
  }
  if constexpr (FORM == kFormDense) {
    switch (pl.bt * 10 + pl.splits) {
      case 161: return launch_gemm<CfgSwap16, FORM>(pr, pl, dev, dev_id, stream);
      case 162: return launch_gemm<CfgSwap16S2, FORM>(pr, pl, dev, dev_id, stream);
      case 164: return launch_gemm<CfgSwap16S4, FORM>(pr, pl, dev, dev_id, stream);
      case 321: return launch_gemm<CfgSwap32, FORM>(pr, pl, dev, dev_id, stream);
      case 322: return launch_gemm<CfgSwap32S2, FORM>(pr, pl, dev, dev_id, stream);
      case 324: return launch_gemm<CfgSwap32S4, FORM>(pr, pl, dev, dev_id, stream);
      case 641: return launch_gemm<CfgSwap64, FORM>(pr, pl, dev, dev_id, stream);
      case 642: return launch_gemm<CfgSwap64S2, FORM>(pr, pl, dev, dev_id, stream);
      case 644: return launch_gemm<CfgSwap64S4, FORM>(pr, pl, dev, dev_id, stream);
      default: break;
    }
  }
  return fail(FG_ERR_UNSUPPORTED, "no kernel for token tile %d, split %d", pl.bt, pl.splits);
}

fg_status run_gemm(const Problem& pr, int expected_m, cudaStream_t stream) {
  DeviceInfo* dev = nullptr;
  FG_TRY(device_info(&dev));
  int dev_id = 0;
  cudaGetDevice(&dev_id);
  const Plan pl = plan_for(pr, dev->sm_count, expected_m);
  if (pr.form == kFormContig && pl.num_mt > kTableMax)
    return fail(FG_ERR_UNSUPPORTED, "M_total %d exceeds %d rows", pr.M, kTableMax * pl.bt);
  if (pr.form == kFormMasked && pr.G + 1 > kTableMax)
    return fail(FG_ERR_UNSUPPORTED, "G %d exceeds %d experts", pr.G, kTableMax - 1);
  switch (pr.form) {
    case kFormDense: return dispatch<kFormDense>(pr, pl, *dev, dev_id, stream);
    case kFormContig: return dispatch<kFormContig>(pr, pl, *dev, dev_id, stream);
    default: return dispatch<kFormMasked>(pr, pl, *dev, dev_id, stream);
  }
}

// ---------------------------------------------------------------- UE8M0 GEMM

//                  BW  stages accumulators epilogue-warps/quadrant pair K-blocks/stage
using MxN128 = MxCfg<128, 5, 2, 1, false, 1>;
using MxN224 = MxCfg<224, 4, 2, 1, false, 1>;
using MxN256 = MxCfg<256, 3, 1, 2, false, 1>;
using MxP224 = MxCfg<224, 3, 2, 1, true, 2>;  // CTA pairs, 256 x 224 tiles
using MxP192 = MxCfg<192, 3, 2, 1, true, 2>;  // CTA pairs, 256 x 192 tiles (N = 11 x 192 = 2112 ...)
// first GEMM of the expert FFN with the fused SwiGLU + requantization epilogue
using MxFfnP = MxCfg<256, 3, 1, 1, true, 2, 1>;
using MxFfnS = MxCfg<256, 4, 1, 1, false, 1, 1>;
// the expert FFN in one launch: first-GEMM tiles with that epilogue, then
// second-GEMM tiles (224 wide, bf16 output)
using MxFfn1P = MxCfg<256, 3, 1, 1, true, 2, 3>;
using MxFfn1S = MxCfg<256, 4, 1, 1, false, 1, 3>;
// K-grouped GEMM (expert weight gradients): fp32 output, per-row B scales
using MxKgP = MxCfg<224, 3, 2, 1, true, 2, 2>;
using MxKgS = MxCfg<224, 4, 2, 1, false, 1, 2>;

// Outputs of the fused expert-FFN epilogue; for the one-kernel FFN also the
// second GEMM's operands, its output and the ready counters.
struct FfnOut {
  uint8_t* hq;
  float* sfh;
  uint16_t* gu;
  int I;
  const uint8_t* W2 = nullptr;
  const float* sfw2 = nullptr;
  uint16_t* Y = nullptr;
  int H = 0;
  int* ready = nullptr;
};

// Shared-memory attribute and, for pair configs, the number of co-resident
// clusters (the persistent grid's size).
template <class C, int FORM>
fg_status mx_kernel_attr(int dev, int* max_clusters) {
  static std::atomic<bool> done[kMaxDevices];  // (zero-initialised: false)
  static int clusters[kMaxDevices] = {};
  if (done[dev].load(std::memory_order_acquire)) {
    *max_clusters = clusters[dev];
    return FG_OK;
  }
  std::lock_guard<std::mutex> lock(g_mu);  // (see kernel_info)
  if (!done[dev].load(std::memory_order_relaxed)) {
    cudaError_t e = cudaFuncSetAttribute(fp8_gemm_mx_kernel<C, FORM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::smem_bytes(FORM));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    if (C::CLUSTER > 1) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = C::CLUSTER;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(C::CLUSTER * 64);
      cfg.blockDim = dim3(C::NUM_THREADS);
      cfg.dynamicSmemBytes = C::smem_bytes(FORM);
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      e = cudaOccupancyMaxActiveClusters(&n, fp8_gemm_mx_kernel<C, FORM>, &cfg);
      if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveClusters");
      if (n < 1) return fail(FG_ERR_UNSUPPORTED, "no cluster of %d CTAs fits", C::CLUSTER);
      clusters[dev] = n;
    }
    done[dev].store(true, std::memory_order_release);
  }
  *max_clusters = clusters[dev];
  return FG_OK;
}

// The K-grouped problem's fp32 output travels in the Problem's D slot.
float* ffn_d32(const Problem& pr) { return reinterpret_cast<float*>(pr.D); }

template <class C, int FORM>
fg_status launch_mx(const Problem& pr, const DeviceInfo& dev, int dev_id, cudaStream_t stream,
                    const FfnOut* ffn = nullptr, int kb_override = -1) {
  static_assert(C::smem_bytes(FORM) <= 232448, "shared memory per CTA");
  int max_clusters = 0;
  FG_TRY((mx_kernel_attr<C, FORM>(dev_id, &max_clusters)));
  const int KB = pr.K / 128;
  CUtensorMap tmA, tmB, tmSA, tmSB, tmD, tmA2, tmB2, tmSA2;
  FG_TRY(make_map(&tmA, pr.A, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.K,
                  static_cast<uint64_t>(pr.slabs) * pr.M, pr.K, 128, C::BT,
                  CU_TENSOR_MAP_SWIZZLE_128B, "A"));
  // one-kernel FFN: the second GEMM reads Hq [slabs * M][I], W2 [G * H][I]
  // and sfh (MN-major [slabs * I/128][stride(M)]); unused, and zero, otherwise
  std::memset(&tmA2, 0, sizeof(tmA2));
  std::memset(&tmB2, 0, sizeof(tmB2));
  std::memset(&tmSA2, 0, sizeof(tmSA2));
  if (C::FUSED) {
    FG_TRY(make_map(&tmA2, ffn->hq, CU_TENSOR_MAP_DATA_TYPE_UINT8, ffn->I,
                    static_cast<uint64_t>(pr.slabs) * pr.M, ffn->I, 128, C::BT,
                    CU_TENSOR_MAP_SWIZZLE_128B, "Hq"));
    FG_TRY(make_map(&tmB2, ffn->W2, CU_TENSOR_MAP_DATA_TYPE_UINT8, ffn->I,
                    static_cast<uint64_t>(pr.G) * ffn->H, ffn->I, 128, C::B_ROWS2,
                    CU_TENSOR_MAP_SWIZZLE_128B, "W2"));
    FG_TRY(make_map(&tmSA2, ffn->sfh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, pr.M,
                    static_cast<uint64_t>(pr.slabs) * (ffn->I / 128),
                    static_cast<uint64_t>(sfa_stride(pr.M)) * 4, C::BT, 4,
                    CU_TENSOR_MAP_SWIZZLE_NONE, "sfh"));
  }
  // (K-grouped: one B of N rows whose K range the experts share)
  FG_TRY(make_map(&tmB, pr.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.K,
                  static_cast<uint64_t>(FORM == kFormKGrouped ? 1 : pr.G) * pr.N, pr.K, 128, C::B_BOX,
                  CU_TENSOR_MAP_SWIZZLE_128B, "B"));
  // token scales: boxes of 128 tokens x 4 K blocks (one quad)
  FG_TRY(make_map(&tmSA, pr.sfa, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, pr.M,
                  static_cast<uint64_t>(pr.slabs) * KB,
                  static_cast<uint64_t>(sfa_stride(pr.M)) * 4, C::BT, 4,
                  CU_TENSOR_MAP_SWIZZLE_NONE, "SFA"));
  // K-grouped: per-row weight scales, MN-major [K/128][stride(N)], boxes of
  // BW rows x 4 K blocks
  std::memset(&tmSB, 0, sizeof(tmSB));
  if (C::EPI == 2)
    FG_TRY(make_map(&tmSB, pr.sfb, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, pr.N, KB,
                    static_cast<uint64_t>(sfa_stride(pr.N)) * 4, C::BW, 4,
                    CU_TENSOR_MAP_SWIZZLE_NONE, "SFB"));
  // D as rows x N bf16 in boxes of 32 rows x 32 columns, 64-byte swizzled
  // (K-grouped: fp32 in 32 x 32 boxes, 128-byte swizzled; the fused FFN
  // epilogue writes no D)
  std::memset(&tmD, 0, sizeof(tmD));
  if (C::EPI == 2)
    FG_TRY(make_map(&tmD, ffn_d32(pr), CU_TENSOR_MAP_DATA_TYPE_FLOAT32, pr.N,
                    static_cast<uint64_t>(pr.G) * pr.M, static_cast<uint64_t>(pr.N) * 4, 32, 32,
                    CU_TENSOR_MAP_SWIZZLE_128B, "D"));
  if (C::EPI == 0)
    FG_TRY(make_map(&tmD, pr.D, CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.N,
                    static_cast<uint64_t>(pr.slabs) * pr.M, static_cast<uint64_t>(pr.N) * 2, 32, 32,
                    CU_TENSOR_MAP_SWIZZLE_64B, "D"));
  GemmParams p{};
  p.M = pr.M;
  p.N = pr.N;
  p.K = pr.K;
  p.G = pr.G;
  p.KB = kb_override >= 0 ? kb_override : KB;  // (K-grouped with T = 0: no K blocks)
  p.NB = (pr.N + 127) / 128;
  p.num_mt = (pr.M + C::BT - 1) / C::BT;
  p.num_nt = (pr.N + C::BW - 1) / C::BW;
  p.sfb = pr.sfb;
  p.D = pr.D;
  p.m_indices = pr.m_indices;
  p.masked_m = pr.masked_m;
  p.status = dev.status;
  p.timeout_ns = wait_limit_ns();
  if (C::FFN) {
    p.hq = ffn->hq;
    p.sfh = ffn->sfh;
    p.gu = ffn->gu;
    p.I = ffn->I;
    p.sfh_stride = sfa_stride(pr.M);
    p.num_nt = ffn->I / 128;  // one tile = 128 gate + 128 up rows
  }
  if (C::FUSED) {
    p.D = ffn->Y;
    p.N2 = ffn->H;
    p.KB2 = ffn->I / 128;
    p.NB2 = ffn->H / 128;
    p.num_nt2 = (ffn->H + C::BW2 - 1) / C::BW2;
    p.sfb2 = ffn->sfw2;
    p.ready = ffn->ready;
    p.ready_target = C::EW * p.num_nt;  // every epilogue warp of every first-GEMM tile
  }
  if (C::EPI == 2) {
    p.ks = pr.m_indices;  // token counts per expert (device)
    p.d32 = ffn_d32(pr);
  }
  int64_t tiles = static_cast<int64_t>(C::PAIR ? (p.num_mt + 1) / 2 : p.num_mt) * p.num_nt;
  if (C::FUSED)  // both GEMMs' tiles (contiguous pairs: at most a unit per token tile)
    tiles = static_cast<int64_t>(FORM == kFormContig ? p.num_mt : (C::PAIR ? (p.num_mt + 1) / 2 : p.num_mt)) *
            (p.num_nt + p.num_nt2);
  if (FORM == kFormMasked || FORM == kFormKGrouped) tiles *= pr.G;  // (masked: an upper bound)
  // (one-kernel FFN: second-GEMM tiles wait for first-GEMM tiles of other
  // CTAs, so every CTA of the grid must be resident at once: at most one
  // CTA per SM, or the co-resident clusters)
  const int64_t grid = C::PAIR ? C::CLUSTER * std::max<int64_t>(1, std::min<int64_t>(tiles, max_clusters))
                               : std::max<int64_t>(1, std::min<int64_t>(tiles, dev.sm_count));
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(C::NUM_THREADS);
  cfg.dynamicSmemBytes = C::smem_bytes(FORM);
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (C::CLUSTER > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = C::CLUSTER;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  const cudaError_t e = cudaLaunchKernelEx(&cfg, fp8_gemm_mx_kernel<C, FORM>, tmA, tmB, tmSA,
                                           tmSB, tmD, tmA2, tmB2, tmSA2, p);
  if (e != cudaSuccess) return cuda_fail(e, "fp8_gemm_mx_kernel launch");
  return FG_OK;
}

// Tile of the block-scaled kernel: the candidate whose tiles fill the SMs in
// the fewest rounds, a round costed by its MMA work (the tile width) times a
// per-candidate factor for how close the candidate's MMAs run to the tensor
// peak (the single-CTA tiles stream more operand bytes per MMA than the stage
// ring keeps in flight; the narrow tile also reads more shared memory per
// flop; the single-accumulator tile waits for each accumulator to be read).
struct MxPlan {
  int bw;
  bool pair;
};

MxPlan mx_plan(const Problem& pr, int sm_count, int expected_m) {
  // token tiles, and token-tile pairs (pairs never span experts: masked
  // slabs pair within an expert; contiguous runs likewise, counted here as
  // if the groups' tiles paired perfectly)
  int64_t token_tiles = (pr.M + 127) / 128;
  int64_t pairs = (token_tiles + 1) / 2;
  if (pr.form == kFormMasked) {
    const int64_t per_expert = (expected_m + 127) / 128;
    token_tiles = per_expert * pr.G;
    pairs = (per_expert + 1) / 2 * pr.G;
  }
  // relative cost of one tile's MMA work per SM, measured on B200 (pair 192 vs 224: 1.04-1.11
  // on dense shapes of equal work per round)
  const struct { int bw; bool pair; double weight; } cand[] = {
      {224, true, 1.0}, {192, true, 1.07}, {224, false, 1.15}, {256, false, 1.4}, {128, false, 1.5}};
  MxPlan best{224, false};
  double best_cost = 1e300;
  for (const auto& c : cand) {
    const int64_t nt = (pr.N + c.bw - 1) / c.bw;
    const int64_t tiles = (c.pair ? pairs : token_tiles) * nt;
    const int64_t units = c.pair ? sm_count / 2 : sm_count;
    const int64_t rounds = (tiles + units - 1) / units;
    const double cost = static_cast<double>(rounds) * c.bw * c.weight;
    if (cost < best_cost) {
      best_cost = cost;
      best = MxPlan{c.bw, c.pair};
    }
  }
  return best;
}

template <int FORM>
fg_status dispatch_mx(const Problem& pr, MxPlan pl, const DeviceInfo& dev, int dev_id, cudaStream_t stream) {
  if (pl.pair) {
    if (pl.bw == 192) return launch_mx<MxP192, FORM>(pr, dev, dev_id, stream);
    return launch_mx<MxP224, FORM>(pr, dev, dev_id, stream);
  }
  switch (pl.bw) {
    case 128: return launch_mx<MxN128, FORM>(pr, dev, dev_id, stream);
    case 256: return launch_mx<MxN256, FORM>(pr, dev, dev_id, stream);
    default: return launch_mx<MxN224, FORM>(pr, dev, dev_id, stream);
  }
}

// fg_set_ue8m0_tile: 0 = automatic, else the forced width (+ pair flag)
std::atomic<int> g_mx_tile{0};

// Power-of-two scales: the block-scaled kernel for token tiles of 128 rows;
// thin shapes (dense M <= 64, masked with expected_m <= 64) take the swapped
// promotion kernel, whose per-block scaling is exact for such scales too.
fg_status run_gemm_mx(const Problem& pr, int expected_m, cudaStream_t stream) {
  const int forced = g_mx_tile.load(std::memory_order_relaxed);
  DeviceInfo* dev = nullptr;
  FG_TRY(device_info(&dev));
  int dev_id = 0;
  cudaGetDevice(&dev_id);
  const int small_m = pr.form == kFormDense ? pr.M : pr.form == kFormMasked ? expected_m : 1 << 30;
  if (small_m <= 64 && forced == 0) return run_gemm(pr, expected_m, stream);
  if (pr.form == kFormContig && (pr.M + 127) / 128 > kTableMax)
    return fail(FG_ERR_UNSUPPORTED, "M_total %d exceeds %d rows", pr.M, kTableMax * 128);
  if (pr.form == kFormMasked && pr.G + 1 > kTableMax)
    return fail(FG_ERR_UNSUPPORTED, "G %d exceeds %d experts", pr.G, kTableMax - 1);
  MxPlan pl = forced ? MxPlan{forced & 0xFFFF, (forced >> 16) != 0} : mx_plan(pr, dev->sm_count, expected_m);
  switch (pr.form) {
    case kFormDense: return dispatch_mx<kFormDense>(pr, pl, *dev, dev_id, stream);
    case kFormContig: return dispatch_mx<kFormContig>(pr, pl, *dev, dev_id, stream);
    default: return dispatch_mx<kFormMasked>(pr, pl, *dev, dev_id, stream);
  }
}

// The expert FFN. Two forms, chosen by the expected rows per expert:
//  - one persistent launch (rows per expert <= 128, decode-sized batches,
//    where the weights dominate): the first grouped GEMM's tiles with the
//    fused SwiGLU + requant epilogue, then the second grouped GEMM's tiles,
//    each waiting for its token tile's quantized activations through a ready
//    counter in the workspace; no second launch and no tail between the two
//    GEMMs (measured on B200, H = 7168, I = 2048: 256 vs 296 us for 32
//    experts x 8 rows, 104 vs 110 us for 8 x 128);
//  - two launches (larger batches): the first GEMM with the fused epilogue,
//    then the plain grouped GEMM, whose 224-wide tiles stream their output
//    through shared memory with tensor stores (8% faster than one launch on
//    the 8-expert contiguous workload, 519 vs 559 us).
// Pairs unless the masked layout's experts hold about one token tile.
std::atomic<int> g_ffn_mode{0};  // fg_set_ffn_mode: 0 automatic, 1 one launch, 2 two launches

// Ready counters of the one-kernel FFN: one int per token tile (masked: per
// expert and token tile of its slab).
size_t ffn_ready_count(int form, int M, int G) {
  const size_t tiles = static_cast<size_t>((M + 127) / 128);
  return form == kFormMasked ? tiles * static_cast<size_t>(G) : tiles;
}

size_t ffn_workspace_bytes(int form, int M, int G) {
  return (ffn_ready_count(form, M, G) * sizeof(int) + 255) / 256 * 256;
}

fg_status run_ffn(int form, const uint8_t* X, const float* sfx, const uint8_t* W1, const float* sfw1,
                  const uint8_t* W2, const float* sfw2, uint8_t* Hq, float* sfh, uint16_t* GU,
                  uint16_t* Y, const int32_t* m_indices, const int32_t* masked_m, int M, int H,
                  int I, int G, int expected_m, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (G < 1) return fail(FG_ERR_INVALID_ARG, "G=%d must be >= 1", G);
  if (H <= 0 || H % 128 != 0) return fail(FG_ERR_INVALID_ARG, "H=%d must be a positive multiple of 128", H);
  if (I <= 0 || I % 128 != 0) return fail(FG_ERR_INVALID_ARG, "I=%d must be a positive multiple of 128", I);
  if (form == kFormContig) {
    if (M < 0 || M % 128 != 0)
      return fail(FG_ERR_INVALID_ARG, "M_total=%d must be a non-negative multiple of 128", M);
    if (M == 0) return FG_OK;
    FG_TRY(check_ptr(m_indices, "m_indices"));
    if ((M + 127) / 128 > kTableMax)
      return fail(FG_ERR_UNSUPPORTED, "M_total %d exceeds %d rows", M, kTableMax * 128);
  } else {
    if (M < 1) return fail(FG_ERR_INVALID_ARG, "M_max=%d must be >= 1", M);
    FG_TRY(check_ptr(masked_m, "masked_m"));
    if (G + 1 > kTableMax) return fail(FG_ERR_UNSUPPORTED, "G %d exceeds %d experts", G, kTableMax - 1);
    if (expected_m <= 0) expected_m = M;
  }
  FG_TRY(check_ptr(X, "X"));
  FG_TRY(check_ptr(sfx, "sfx"));
  FG_TRY(check_ptr(W1, "W1"));
  FG_TRY(check_ptr(sfw1, "sfw1"));
  FG_TRY(check_ptr(W2, "W2"));
  FG_TRY(check_ptr(sfw2, "sfw2"));
  FG_TRY(check_ptr(Hq, "Hq"));
  FG_TRY(check_ptr(sfh, "sfh"));
  FG_TRY(check_ptr(Y, "Y"));
  if (GU) FG_TRY(check_ptr(GU, "GU"));
  FG_TRY(check_ptr(ws, "ws"));
  const size_t need = ffn_workspace_bytes(form, M, G);
  if (ws_bytes < need)
    return fail(FG_ERR_INVALID_ARG, "ws_bytes=%zu, the expert FFN needs %zu (fg_moe_ffn_workspace_bytes)",
                ws_bytes, need);
  DeviceInfo* dev = nullptr;
  FG_TRY(device_info(&dev));
  int dev_id = 0;
  cudaGetDevice(&dev_id);
  const int slabs = form == kFormMasked ? G : 1;
  FfnOut out{Hq, sfh, GU, I};
  Problem p1{form, X, sfx, W1, sfw1, nullptr, m_indices, masked_m, M, 2 * I, H, G, slabs};
  const bool pair = form == kFormContig || expected_m > 128;
  const int rows_per_expert = form == kFormMasked ? expected_m : M / G;
  const int mode = g_ffn_mode.load(std::memory_order_relaxed);
  if (mode == 2 || (mode == 0 && rows_per_expert > 128)) {
    fg_status st;
    if (form == kFormContig)
      st = pair ? launch_mx<MxFfnP, kFormContig>(p1, *dev, dev_id, stream, &out)
                : launch_mx<MxFfnS, kFormContig>(p1, *dev, dev_id, stream, &out);
    else
      st = pair ? launch_mx<MxFfnP, kFormMasked>(p1, *dev, dev_id, stream, &out)
                : launch_mx<MxFfnS, kFormMasked>(p1, *dev, dev_id, stream, &out);
    if (st != FG_OK) return st;
    Problem p2{form, Hq, sfh, W2, sfw2, Y, m_indices, masked_m, M, H, I, G, slabs};
    return run_gemm_mx(p2, expected_m, stream);
  }
  out.W2 = W2;
  out.sfw2 = sfw2;
  out.Y = Y;
  out.H = H;
  out.ready = static_cast<int*>(ws);
  // the counters start at zero (the memset precedes the kernel on the stream)
  const cudaError_t e = cudaMemsetAsync(ws, 0, ffn_ready_count(form, M, G) * sizeof(int), stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(ready counters)");
  if (form == kFormContig)
    return pair ? launch_mx<MxFfn1P, kFormContig>(p1, *dev, dev_id, stream, &out)
                : launch_mx<MxFfn1S, kFormContig>(p1, *dev, dev_id, stream, &out);
  return pair ? launch_mx<MxFfn1P, kFormMasked>(p1, *dev, dev_id, stream, &out)
              : launch_mx<MxFfn1S, kFormMasked>(p1, *dev, dev_id, stream, &out);
}

fg_status check_gemm_common(const uint8_t* A, const float* sfa, const uint8_t* B,
                            const float* sfb, uint16_t* D, int N, int K) {
  if (K <= 0 || K % 128 != 0) return fail(FG_ERR_INVALID_ARG, "K=%d must be a positive multiple of 128", K);
  if (N <= 0 || N % 16 != 0) return fail(FG_ERR_INVALID_ARG, "N=%d must be a positive multiple of 16", N);
  FG_TRY(check_ptr(A, "A"));
  FG_TRY(check_ptr(sfa, "sfa"));
  FG_TRY(check_ptr(B, "B"));
  FG_TRY(check_ptr(sfb, "sfb"));
  FG_TRY(check_ptr(D, "D"));
  return FG_OK;
}

// Launch with programmatic stream serialization (the kernel waits on the
// previous grid with griddepcontrol.wait before touching memory).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, cudaStream_t stream,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

__global__ void selftest_wait_kernel(int* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl ctl{&abort_flag, status, limit_ns};
    // Nobody arrives on `bar`: the wait must give up after limit_ns.
    (void)mbar_wait(&bar, 0, ctl);
  }
  __syncthreads();
}

fg_status run_per_token(const uint16_t* x, uint8_t* q, float* sfa, int num_groups, int M, int K,
                        bool ue8m0, cudaStream_t stream) {
  if (num_groups < 1) return fail(FG_ERR_INVALID_ARG, "num_groups=%d must be >= 1", num_groups);
  if (M < 0) return fail(FG_ERR_INVALID_ARG, "M=%d must be >= 0", M);
  if (K <= 0 || K % 128 != 0) return fail(FG_ERR_INVALID_ARG, "K=%d must be a positive multiple of 128", K);
  if (M == 0) return FG_OK;
  FG_TRY(check_ptr(x, "x"));
  FG_TRY(check_ptr(q, "q"));
  FG_TRY(check_ptr(sfa, "sfa"));
  DeviceInfo* dev = nullptr;
  FG_TRY(device_info(&dev));
  const int64_t slices = static_cast<int64_t>(num_groups) * M * (K / 128);
  if (slices >= (int64_t(1) << 31)) return fail(FG_ERR_UNSUPPORTED, "too many 128-element slices");
  // one warp per work item of QROW_ITEM slices of a row, up to 8 blocks of
  // 256 threads per SM (grid-stride beyond that)
  const int64_t items = static_cast<int64_t>(num_groups) * M * ((K / 128 + QROW_ITEM - 1) / QROW_ITEM);
  const int64_t blocks_needed = (items * 32 + 255) / 256;
  const int grid = static_cast<int>(std::min<int64_t>(blocks_needed, int64_t(dev->sm_count) * 8));
  const cudaError_t e = launch_pdl(ue8m0 ? per_token_cast_kernel<true> : per_token_cast_kernel<false>, dim3(grid), dim3(256), stream, x, q, sfa,
                                   num_groups, M, K, sfa_stride(M));
  if (e != cudaSuccess) return cuda_fail(e, "per_token_cast_kernel launch");
  return FG_OK;
}

fg_status run_per_block(const uint16_t* x, uint8_t* q, float* sfb, int num_groups, int N, int K,
                        bool ue8m0, cudaStream_t stream) {
  if (num_groups < 1) return fail(FG_ERR_INVALID_ARG, "num_groups=%d must be >= 1", num_groups);
  if (N <= 0) return fail(FG_ERR_INVALID_ARG, "N=%d must be >= 1", N);
  if (K <= 0 || K % 128 != 0) return fail(FG_ERR_INVALID_ARG, "K=%d must be a positive multiple of 128", K);
  FG_TRY(check_ptr(x, "x"));
  FG_TRY(check_ptr(q, "q"));
  FG_TRY(check_ptr(sfb, "sfb"));
  DeviceInfo* dev = nullptr;
  FG_TRY(device_info(&dev));
  const int64_t blocks = static_cast<int64_t>(num_groups) * ((N + 127) / 128) * (K / 128);
  if (blocks > 0x7FFFFFFF) return fail(FG_ERR_UNSUPPORTED, "too many blocks");
  const cudaError_t e = launch_pdl(ue8m0 ? per_block_cast_kernel<true> : per_block_cast_kernel<false>,
                                   dim3(static_cast<unsigned>(blocks)),
                                   dim3(256), stream, x, q, sfb, num_groups, N, K);
  if (e != cudaSuccess) return cuda_fail(e, "per_block_cast_kernel launch");
  return FG_OK;
}

// ---------------------------------------------------------------- FFN without allocation

// Ready counters of fp8_moe_ffn_masked_ue8m0_noalloc, for callers that are
// given device buffers for their inputs and outputs but may not allocate any
// further device memory. The array is this library's own: every GPU that
// loads the library holds it (16 KB) until the process exits. In host code
// `g_ffn_scratch` names a host-side stand-in, not device memory: kernels are
// given the device address looked up below.
constexpr size_t kFfnScratchCounters = 4096;
static __device__ __align__(256) int g_ffn_scratch[kFfnScratchCounters];

std::mutex g_scratch_mu;
int* g_scratch_dev[kMaxDevices] = {};

// Device address of g_ffn_scratch on the current device `dev`, looked up on
// the first call for that device (cudaGetSymbolAddress, with `dev` current)
// and cached.
fg_status ffn_scratch(int dev, int** out) {
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_dev[dev] == nullptr) {
    int* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress((void**)&ptr, g_ffn_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(FFN scratch)");
    g_scratch_dev[dev] = ptr;
  }
  *out = g_scratch_dev[dev];
  return FG_OK;
}

fg_status run_ffn_masked_noalloc(const uint8_t* X, const float* sfx, const uint8_t* W1,
                                 const float* sfw1, const uint8_t* W2, const float* sfw2,
                                 uint8_t* Hq, float* sfh, uint16_t* GU, uint16_t* Y,
                                 const int32_t* masked_m, int G, int M_max, int H, int I,
                                 int expected_m, cudaStream_t stream) {
  if (G < 1) return fail(FG_ERR_INVALID_ARG, "G=%d must be >= 1", G);
  if (H <= 0 || H % 128 != 0) return fail(FG_ERR_INVALID_ARG, "H=%d must be a positive multiple of 128", H);
  if (I <= 0 || I % 128 != 0) return fail(FG_ERR_INVALID_ARG, "I=%d must be a positive multiple of 128", I);
  if (M_max < 1) return fail(FG_ERR_INVALID_ARG, "M_max=%d must be >= 1", M_max);
  FG_TRY(check_ptr(masked_m, "masked_m"));
  if (G + 1 > kTableMax) return fail(FG_ERR_UNSUPPORTED, "G %d exceeds %d experts", G, kTableMax - 1);
  const size_t need = ffn_ready_count(kFormMasked, M_max, G);
  if (need > kFfnScratchCounters)
    return fail(FG_ERR_UNSUPPORTED,
                "fp8_moe_ffn_masked_ue8m0_noalloc: G * ceil(M_max / 128) = %zu token tiles exceed the "
                "%zu of its fixed scratch (use fp8_moe_ffn_masked_ue8m0 with a workspace)",
                need, kFfnScratchCounters);
  if (expected_m <= 0) expected_m = M_max;
  FG_TRY(check_ptr(X, "X"));
  FG_TRY(check_ptr(sfx, "sfx"));
  FG_TRY(check_ptr(W1, "W1"));
  FG_TRY(check_ptr(sfw1, "sfw1"));
  FG_TRY(check_ptr(W2, "W2"));
  FG_TRY(check_ptr(sfw2, "sfw2"));
  FG_TRY(check_ptr(Hq, "Hq"));
  FG_TRY(check_ptr(sfh, "sfh"));
  FG_TRY(check_ptr(Y, "Y"));
  if (GU) FG_TRY(check_ptr(GU, "GU"));
  DeviceInfo* dev = nullptr;
  FG_TRY(device_info(&dev));
  int dev_id = 0;
  cudaGetDevice(&dev_id);
  int* ready = nullptr;
  FG_TRY(ffn_scratch(dev_id, &ready));
  // the array keeps the previous call's counts: clear the ones this call uses
  const cudaError_t e = cudaMemsetAsync(ready, 0, need * sizeof(int), stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(FFN scratch)");
  FfnOut out{Hq, sfh, GU, I};
  out.W2 = W2;
  out.sfw2 = sfw2;
  out.Y = Y;
  out.H = H;
  out.ready = ready;
  Problem p1{kFormMasked, X, sfx, W1, sfw1, nullptr, nullptr, masked_m, M_max, 2 * I, H, G, G};
  return expected_m > 128 ? launch_mx<MxFfn1P, kFormMasked>(p1, *dev, dev_id, stream, &out)
                          : launch_mx<MxFfn1S, kFormMasked>(p1, *dev, dev_id, stream, &out);
}

}  // namespace
}  // namespace fg

using namespace fg;

extern "C" {

int fg_sfa_stride(int M) { return sfa_stride(M); }

fg_status per_token_cast_to_fp8(const uint16_t* x, uint8_t* q, float* sfa, int num_groups, int M,
                                int K, cudaStream_t stream) {
  return run_per_token(x, q, sfa, num_groups, M, K, false, stream);
}

fg_status per_token_cast_to_fp8_ue8m0(const uint16_t* x, uint8_t* q, float* sfa, int num_groups,
                                      int M, int K, cudaStream_t stream) {
  return run_per_token(x, q, sfa, num_groups, M, K, true, stream);
}

fg_status per_block_cast_to_fp8(const uint16_t* x, uint8_t* q, float* sfb, int num_groups, int N,
                                int K, cudaStream_t stream) {
  return run_per_block(x, q, sfb, num_groups, N, K, false, stream);
}

fg_status per_block_cast_to_fp8_ue8m0(const uint16_t* x, uint8_t* q, float* sfb, int num_groups,
                                      int N, int K, cudaStream_t stream) {
  return run_per_block(x, q, sfb, num_groups, N, K, true, stream);
}

fg_status per_block_dequant_to_bf16(const uint8_t* q, const float* sfb, uint16_t* x,
                                    int num_groups, int N, int K, cudaStream_t stream) {
  if (num_groups < 1) return fail(FG_ERR_INVALID_ARG, "num_groups=%d must be >= 1", num_groups);
  if (N <= 0) return fail(FG_ERR_INVALID_ARG, "N=%d must be >= 1", N);
  if (K <= 0 || K % 128 != 0) return fail(FG_ERR_INVALID_ARG, "K=%d must be a positive multiple of 128", K);
  FG_TRY(check_ptr(q, "q"));
  FG_TRY(check_ptr(sfb, "sfb"));
  FG_TRY(check_ptr(x, "x"));
  DeviceInfo* dev = nullptr;
  FG_TRY(device_info(&dev));
  const int64_t chunks = static_cast<int64_t>(num_groups) * N * (K / 16);
  const int grid = static_cast<int>(std::min<int64_t>((chunks + 255) / 256, int64_t(dev->sm_count) * 8));
  const cudaError_t e = launch_pdl(per_block_dequant_kernel, dim3(grid), dim3(256), stream, q, sfb, x,
                                   num_groups, N, K);
  if (e != cudaSuccess) return cuda_fail(e, "per_block_dequant_kernel launch");
  return FG_OK;
}

fg_status fp8_gemm_nt(const uint8_t* A, const float* sfa, const uint8_t* B, const float* sfb,
                      uint16_t* D, int M, int N, int K, cudaStream_t stream) {
  if (M < 0) return fail(FG_ERR_INVALID_ARG, "M=%d must be >= 0", M);
  if (M == 0) return FG_OK;
  FG_TRY(check_gemm_common(A, sfa, B, sfb, D, N, K));
  Problem pr{kFormDense, A, sfa, B, sfb, D, nullptr, nullptr, M, N, K, 1, 1};
  return run_gemm(pr, M, stream);
}

fg_status fp8_grouped_gemm_contiguous(const uint8_t* A, const float* sfa, const uint8_t* B,
                                      const float* sfb, uint16_t* D, const int32_t* m_indices,
                                      int M_total, int N, int K, int G, cudaStream_t stream) {
  if (M_total < 0 || M_total % 128 != 0)
    return fail(FG_ERR_INVALID_ARG, "M_total=%d must be a non-negative multiple of 128", M_total);
  if (G < 1) return fail(FG_ERR_INVALID_ARG, "G=%d must be >= 1", G);
  if (M_total == 0) return FG_OK;
  FG_TRY(check_gemm_common(A, sfa, B, sfb, D, N, K));
  FG_TRY(check_ptr(m_indices, "m_indices"));
  Problem pr{kFormContig, A, sfa, B, sfb, D, m_indices, nullptr, M_total, N, K, G, 1};
  return run_gemm(pr, M_total, stream);
}

fg_status fp8_grouped_gemm_masked(const uint8_t* A, const float* sfa, const uint8_t* B,
                                  const float* sfb, uint16_t* D, const int32_t* masked_m, int G,
                                  int M_max, int N, int K, int expected_m, cudaStream_t stream) {
  if (G < 1) return fail(FG_ERR_INVALID_ARG, "G=%d must be >= 1", G);
  if (M_max < 1) return fail(FG_ERR_INVALID_ARG, "M_max=%d must be >= 1", M_max);
  FG_TRY(check_gemm_common(A, sfa, B, sfb, D, N, K));
  FG_TRY(check_ptr(masked_m, "masked_m"));
  if (expected_m <= 0) expected_m = M_max;
  Problem pr{kFormMasked, A, sfa, B, sfb, D, nullptr, masked_m, M_max, N, K, G, G};
  return run_gemm(pr, expected_m, stream);
}

fg_status fp8_gemm_nt_ue8m0(const uint8_t* A, const float* sfa, const uint8_t* B, const float* sfb,
                            uint16_t* D, int M, int N, int K, cudaStream_t stream) {
  if (M < 0) return fail(FG_ERR_INVALID_ARG, "M=%d must be >= 0", M);
  if (M == 0) return FG_OK;
  FG_TRY(check_gemm_common(A, sfa, B, sfb, D, N, K));
  Problem pr{kFormDense, A, sfa, B, sfb, D, nullptr, nullptr, M, N, K, 1, 1};
  return run_gemm_mx(pr, M, stream);
}

fg_status fp8_grouped_gemm_contiguous_ue8m0(const uint8_t* A, const float* sfa, const uint8_t* B,
                                            const float* sfb, uint16_t* D,
                                            const int32_t* m_indices, int M_total, int N, int K,
                                            int G, cudaStream_t stream) {
  if (M_total < 0 || M_total % 128 != 0)
    return fail(FG_ERR_INVALID_ARG, "M_total=%d must be a non-negative multiple of 128", M_total);
  if (G < 1) return fail(FG_ERR_INVALID_ARG, "G=%d must be >= 1", G);
  if (M_total == 0) return FG_OK;
  FG_TRY(check_gemm_common(A, sfa, B, sfb, D, N, K));
  FG_TRY(check_ptr(m_indices, "m_indices"));
  Problem pr{kFormContig, A, sfa, B, sfb, D, m_indices, nullptr, M_total, N, K, G, 1};
  return run_gemm_mx(pr, M_total, stream);
}

fg_status fp8_grouped_gemm_masked_ue8m0(const uint8_t* A, const float* sfa, const uint8_t* B,
                                        const float* sfb, uint16_t* D, const int32_t* masked_m,
                                        int G, int M_max, int N, int K, int expected_m,
                                        cudaStream_t stream) {
  if (G < 1) return fail(FG_ERR_INVALID_ARG, "G=%d must be >= 1", G);
  if (M_max < 1) return fail(FG_ERR_INVALID_ARG, "M_max=%d must be >= 1", M_max);
  FG_TRY(check_gemm_common(A, sfa, B, sfb, D, N, K));
  FG_TRY(check_ptr(masked_m, "masked_m"));
  if (expected_m <= 0) expected_m = M_max;
  Problem pr{kFormMasked, A, sfa, B, sfb, D, nullptr, masked_m, M_max, N, K, G, G};
  return run_gemm_mx(pr, expected_m, stream);
}

fg_status fg_set_ffn_mode(int mode) {
  if (mode < 0 || mode > 2) return fail(FG_ERR_INVALID_ARG, "ffn mode %d (0, 1 or 2)", mode);
  g_ffn_mode.store(mode, std::memory_order_relaxed);
  return FG_OK;
}

size_t fg_moe_ffn_workspace_bytes(int layout, int M, int G) {
  if (M < 0 || G < 1 || (layout != FG_LAYOUT_CONTIGUOUS && layout != FG_LAYOUT_MASKED)) return 0;
  return ffn_workspace_bytes(layout == FG_LAYOUT_MASKED ? kFormMasked : kFormContig, M, G);
}

fg_status fp8_moe_ffn_contiguous_ue8m0(const uint8_t* X, const float* sfx, const uint8_t* W1,
                                      const float* sfw1, const uint8_t* W2, const float* sfw2,
                                      uint8_t* Hq, float* sfh, uint16_t* GU, uint16_t* Y,
                                      const int32_t* m_indices, int M_total, int H, int I, int G,
                                      void* ws, size_t ws_bytes, cudaStream_t stream) {
  return run_ffn(kFormContig, X, sfx, W1, sfw1, W2, sfw2, Hq, sfh, GU, Y, m_indices, nullptr,
                 M_total, H, I, G, M_total, ws, ws_bytes, stream);
}

fg_status fp8_moe_ffn_masked_ue8m0(const uint8_t* X, const float* sfx, const uint8_t* W1,
                                  const float* sfw1, const uint8_t* W2, const float* sfw2,
                                  uint8_t* Hq, float* sfh, uint16_t* GU, uint16_t* Y,
                                  const int32_t* masked_m, int G, int M_max, int H, int I,
                                  int expected_m, void* ws, size_t ws_bytes, cudaStream_t stream) {
  return run_ffn(kFormMasked, X, sfx, W1, sfw1, W2, sfw2, Hq, sfh, GU, Y, nullptr, masked_m, M_max,
                 H, I, G, expected_m, ws, ws_bytes, stream);
}

fg_status fp8_moe_ffn_masked_ue8m0_noalloc(const uint8_t* X, const float* sfx, const uint8_t* W1,
                                          const float* sfw1, const uint8_t* W2, const float* sfw2,
                                          uint8_t* Hq, float* sfh, uint16_t* GU, uint16_t* Y,
                                          const int32_t* masked_m, int G, int M_max, int H, int I,
                                          int expected_m, cudaStream_t stream) {
  return run_ffn_masked_noalloc(X, sfx, W1, sfw1, W2, sfw2, Hq, sfh, GU, Y, masked_m, G, M_max, H, I,
                                expected_m, stream);
}

// ---------------------------------------------------------------- expert-parallel dispatch / combine

fg_status ep_dispatch_layout(const int32_t* topk_idx, int T, int k, int E, int32_t* counts,
                             int32_t* send_pos, cudaStream_t stream) {
  if (T < 0 || k < 1 || E < 1) return fail(FG_ERR_INVALID_ARG, "T=%d k=%d E=%d", T, k, E);
  FG_TRY(check_ptr(counts, "counts"));
  if (T == 0) {
    const cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, stream);
    return e == cudaSuccess ? FG_OK : cuda_fail(e, "cudaMemsetAsync(counts)");
  }
  FG_TRY(check_ptr(topk_idx, "topk_idx"));
  FG_TRY(check_ptr(send_pos, "send_pos"));
  DeviceInfo* dev = nullptr;
  FG_TRY(device_info(&dev));
  const int P = T * k;
  cudaError_t e = launch_pdl(ep_count_kernel, dim3(E), dim3(kEpBlock), stream, topk_idx, P, E, counts,
                             send_pos, dev->status);
  if (e != cudaSuccess) return cuda_fail(e, "ep_count_kernel launch");
  e = launch_pdl(ep_position_kernel, dim3(E), dim3(kEpBlock), stream, topk_idx, P,
                 static_cast<const int32_t*>(counts), 1, 0, send_pos, dev->status);
  return e == cudaSuccess ? FG_OK : cuda_fail(e, "ep_position_kernel launch");
}

fg_status ep_dispatch_layout_capacity(const int32_t* topk_idx, int T, int k, int E, int W, int C,
                                      int32_t* counts, int32_t* send_pos, cudaStream_t stream) {
  if (T < 0 || k < 1 || E < 1 || W < 1 || C < 1)
    return fail(FG_ERR_INVALID_ARG, "T=%d k=%d E=%d W=%d C=%d", T, k, E, W, C);
  if (E % W != 0) return fail(FG_ERR_INVALID_ARG, "E=%d is not a multiple of W=%d", E, W);
  if (static_cast<int64_t>(W) * C > INT32_MAX)
    return fail(FG_ERR_UNSUPPORTED, "W * C = %lld rows", static_cast<long long>(W) * C);
  FG_TRY(check_ptr(counts, "counts"));
  if (T == 0) {
    const cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, stream);
    return e == cudaSuccess ? FG_OK : cuda_fail(e, "cudaMemsetAsync(counts)");
  }
  FG_TRY(check_ptr(topk_idx, "topk_idx"));
  FG_TRY(check_ptr(send_pos, "send_pos"));
  DeviceInfo* dev = nullptr;
  FG_TRY(device_info(&dev));
  const int P = T * k;
  cudaError_t e = launch_pdl(ep_count_kernel, dim3(E), dim3(kEpBlock), stream, topk_idx, P, E, counts,
                             send_pos, dev->status);
  if (e != cudaSuccess) return cuda_fail(e, "ep_count_kernel launch");
  e = launch_pdl(ep_position_kernel, dim3(E), dim3(kEpBlock), stream, topk_idx, P,
                 static_cast<const int32_t*>(counts), E / W, C, send_pos, dev->status);
  if (e != cudaSuccess) return cuda_fail(e, "ep_position_kernel launch");
  e = launch_pdl(ep_cap_counts_kernel, dim3(1), dim3(kEpBlock), stream, counts, E, E / W, C);
  return e == cudaSuccess ? FG_OK : cuda_fail(e, "ep_cap_counts_kernel launch");
}

fg_status ep_dispatch_pack(const uint8_t* q, const float* sfa, const int32_t* send_pos, int T, int k,
                           int K, uint8_t* send_q, float* send_s, cudaStream_t stream) {
  if (T < 0 || k < 1) return fail(FG_ERR_INVALID_ARG, "T=%d k=%d", T, k);
  if (K <= 0 || K % 128 != 0) return fail(FG_ERR_INVALID_ARG, "K=%d must be a positive multiple of 128", K);
  if (T == 0) return FG_OK;
  FG_TRY(check_ptr(q, "q"));
  FG_TRY(check_ptr(sfa, "sfa"));
  FG_TRY(check_ptr(send_pos, "send_pos"));
  FG_TRY(check_ptr(send_q, "send_q"));
  FG_TRY(check_ptr(send_s, "send_s"));
  const int P = T * k;
  const int per = kEpBlock / 32;
  const cudaError_t e = launch_pdl(ep_pack_kernel, dim3((P + per - 1) / per), dim3(kEpBlock), stream, q,
                                   sfa, sfa_stride(T), send_pos, P, k, K, send_q, send_s);
  return e == cudaSuccess ? FG_OK : cuda_fail(e, "ep_pack_kernel launch");
}

static fg_status run_unpack(const uint8_t* recv_q, const float* recv_s, const int32_t* recv_counts, int W, int G,
                     int C, int R, int M_max, int K, uint8_t* A, float* sfa, int32_t* masked_m,
                     int32_t* recv_slot, cudaStream_t stream) {
  if (W < 1 || G < 1 || R < 0 || M_max < 1)
    return fail(FG_ERR_INVALID_ARG, "W=%d G=%d R=%d M_max=%d", W, G, R, M_max);
  if (static_cast<int64_t>(W) * G > kEpMaxTable)
    return fail(FG_ERR_UNSUPPORTED, "W * G = %lld exceeds %d", static_cast<long long>(W) * G, kEpMaxTable);
  if (K <= 0 || K % 128 != 0) return fail(FG_ERR_INVALID_ARG, "K=%d must be a positive multiple of 128", K);
  FG_TRY(check_ptr(recv_counts, "recv_counts"));
  FG_TRY(check_ptr(A, "A"));
  FG_TRY(check_ptr(sfa, "sfa"));
  FG_TRY(check_ptr(masked_m, "masked_m"));
  if (R > 0) {
    FG_TRY(check_ptr(recv_q, "recv_q"));
    FG_TRY(check_ptr(recv_s, "recv_s"));
    FG_TRY(check_ptr(recv_slot, "recv_slot"));
  }
  DeviceInfo* dev = nullptr;
  FG_TRY(device_info(&dev));
  const int per = kEpBlock / 32;
  const int blocks = R > 0 ? (R + per - 1) / per : 1;  // (block 0 writes masked_m)
  const cudaError_t e = launch_pdl(ep_unpack_kernel, dim3(blocks), dim3(kEpBlock), stream, recv_q, recv_s,
                                   recv_counts, W, G, C, R, M_max, K, A, sfa, masked_m, recv_slot,
                                   dev->status);
  return e == cudaSuccess ? FG_OK : cuda_fail(e, "ep_unpack_kernel launch");
}

fg_status ep_dispatch_unpack_masked(const uint8_t* recv_q, const float* recv_s,
                                    const int32_t* recv_counts, int W, int G, int R, int M_max,
                                    int K, uint8_t* A, float* sfa, int32_t* masked_m,
                                    int32_t* recv_slot, cudaStream_t stream) {
  return run_unpack(recv_q, recv_s, recv_counts, W, G, 0, R, M_max, K, A, sfa, masked_m, recv_slot, stream);
}

fg_status ep_dispatch_unpack_masked_capacity(const uint8_t* recv_q, const float* recv_s,
                                             const int32_t* recv_counts, int W, int G, int C, int M_max,
                                             int K, uint8_t* A, float* sfa, int32_t* masked_m,
                                             int32_t* recv_slot, cudaStream_t stream) {
  if (C < 1) return fail(FG_ERR_INVALID_ARG, "C=%d must be >= 1", C);
  if (static_cast<int64_t>(W) * C > INT32_MAX)
    return fail(FG_ERR_UNSUPPORTED, "W * C = %lld rows", static_cast<long long>(W) * C);
  return run_unpack(recv_q, recv_s, recv_counts, W, G, C, W * C, M_max, K, A, sfa, masked_m, recv_slot,
                    stream);
}

fg_status ep_combine_gather(const uint16_t* D, const int32_t* recv_slot, int R, int N, uint16_t* out,
                            cudaStream_t stream) {
  if (R < 0 || N <= 0 || N % 8 != 0) return fail(FG_ERR_INVALID_ARG, "R=%d N=%d (N %% 8 == 0)", R, N);
  if (R == 0) return FG_OK;
  FG_TRY(check_ptr(D, "D"));
  FG_TRY(check_ptr(recv_slot, "recv_slot"));
  FG_TRY(check_ptr(out, "out"));
  const int per = kEpBlock / 32;
  const cudaError_t e = launch_pdl(ep_gather_kernel, dim3((R + per - 1) / per), dim3(kEpBlock), stream, D,
                                   recv_slot, R, N, out);
  return e == cudaSuccess ? FG_OK : cuda_fail(e, "ep_gather_kernel launch");
}

fg_status ep_combine_reduce(const uint16_t* y, const int32_t* send_pos, const float* topk_w, int T, int k,
                            int N, uint16_t* out, cudaStream_t stream) {
  if (T < 0 || k < 1 || N <= 0 || N % 8 != 0) return fail(FG_ERR_INVALID_ARG, "T=%d k=%d N=%d", T, k, N);
  if (T == 0) return FG_OK;
  FG_TRY(check_ptr(y, "y"));
  FG_TRY(check_ptr(send_pos, "send_pos"));
  FG_TRY(check_ptr(topk_w, "topk_w"));
  FG_TRY(check_ptr(out, "out"));
  const cudaError_t e = launch_pdl(ep_combine_kernel, dim3(T), dim3(kEpBlock), stream, y, send_pos, topk_w,
                                   k, N, out);
  return e == cudaSuccess ? FG_OK : cuda_fail(e, "ep_combine_kernel launch");
}

fg_status fp8_k_grouped_gemm_nt_ue8m0(const uint8_t* A, const float* sfa, const uint8_t* B,
                                     const float* sfb, float* D, const int32_t* ks, int G, int M,
                                     int N, int T, cudaStream_t stream) {
  if (G < 1) return fail(FG_ERR_INVALID_ARG, "G=%d must be >= 1", G);
  if (G + 1 > kTableMax) return fail(FG_ERR_UNSUPPORTED, "G %d exceeds %d groups", G, kTableMax - 1);
  if (M < 1) return fail(FG_ERR_INVALID_ARG, "M=%d must be >= 1", M);
  if (N <= 0 || N % 16 != 0) return fail(FG_ERR_INVALID_ARG, "N=%d must be a positive multiple of 16", N);
  if (T < 0 || T % 128 != 0) return fail(FG_ERR_INVALID_ARG, "T=%d must be a non-negative multiple of 128", T);
  FG_TRY(check_ptr(A, "A"));
  FG_TRY(check_ptr(sfa, "sfa"));
  FG_TRY(check_ptr(B, "B"));
  FG_TRY(check_ptr(sfb, "sfb"));
  FG_TRY(check_ptr(D, "D"));
  FG_TRY(check_ptr(ks, "ks"));
  DeviceInfo* dev = nullptr;
  FG_TRY(device_info(&dev));
  int dev_id = 0;
  cudaGetDevice(&dev_id);
  // (T = 0: every group is empty; the kernel writes zeros. The tensor maps
  // need a nonzero extent, so the K extent is at least one block.)
  Problem pr{kFormKGrouped, A, sfa, B, sfb, reinterpret_cast<uint16_t*>(D), ks, nullptr, M, N,
             std::max(T, 128), G, 1};
  if (T == 0) pr.K = 128;
  // pairs unless there is a single token tile
  if (M > 128) return launch_mx<MxKgP, kFormKGrouped>(pr, *dev, dev_id, stream, nullptr, T / 128);
  return launch_mx<MxKgS, kFormKGrouped>(pr, *dev, dev_id, stream, nullptr, T / 128);
}

fg_status fg_set_ue8m0_tile(int width, int pair) {
  const bool ok = width == 0 || (pair ? (width == 224 || width == 192)
                                      : (width == 128 || width == 224 || width == 256));
  if (!ok)
    return fail(FG_ERR_INVALID_ARG, "tile %d%s: 0 (automatic), 128, 224, 256, or 224 as a pair",
                width, pair ? " (pair)" : "");
  g_mx_tile.store(width == 0 ? 0 : (width | (pair ? 1 << 16 : 0)), std::memory_order_relaxed);
  return FG_OK;
}

fg_status fg_get_device_status(cudaStream_t stream, int* code) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_status_word, sizeof v);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol(status)");
  if (code) *code = v;
  if (v == 0) return FG_OK;
  const int zero = 0;
  e = cudaMemcpyToSymbol(g_status_word, &zero, sizeof zero);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyToSymbol(status)");
  const char* what = v == FG_DEVICE_WAIT_TIMEOUT   ? "a pipeline wait timed out"
                     : v == FG_DEVICE_BAD_MASKED_M ? "masked_m outside [0, M_max]"
                     : v == FG_DEVICE_BAD_M_INDEX  ? "m_indices entry >= G"
                     : v == FG_DEVICE_BAD_K_GROUP  ? "ks entry negative, not a multiple of 128, or past T"
                     : v == FG_DEVICE_BAD_SCALE    ? "a scale of a block-scaled (_ue8m0) GEMM is not a power of two"
                     : v == FG_DEVICE_EP_OVERFLOW  ? "a local expert received more than M_max rows"
                                                   : "unknown device status";
  return fail(FG_ERR_DEVICE, "device status %d: %s", v, what);
}

fg_status fg_selftest_wait_timeout(int timeout_us, cudaStream_t stream) {
  if (timeout_us <= 0 || timeout_us > 10000000)
    return fail(FG_ERR_INVALID_ARG, "timeout_us=%d must be in (0, 1e7]", timeout_us);
  DeviceInfo* dev = nullptr;
  FG_TRY(device_info(&dev));
  selftest_wait_kernel<<<1, 32, 0, stream>>>(dev->status, static_cast<uint64_t>(timeout_us) * 1000ull);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "selftest_wait_kernel launch");
  return FG_OK;
}

const char* fg_status_string(fg_status s) {
  switch (s) {
    case FG_OK: return "FG_OK";
    case FG_ERR_INVALID_ARG: return "FG_ERR_INVALID_ARG";
    case FG_ERR_UNSUPPORTED: return "FG_ERR_UNSUPPORTED";
    case FG_ERR_CUDA: return "FG_ERR_CUDA";
    case FG_ERR_DEVICE: return "FG_ERR_DEVICE";
  }
  return "FG_ERR_UNKNOWN";
}

const char* fg_last_error(void) { return g_last_error.c_str(); }

// ---------------------------------------------------------------- tensor-core rate

int fg_fp8_mma_peak_ctas(void) {
  DeviceInfo* dev = nullptr;
  if (device_info(&dev) != FG_OK) return 0;
  return dev->sm_count;
}

fg_status fg_fp8_mma_peak(int iters, float* out, cudaStream_t stream) {
  if (iters < 1 || iters > kPeakMaxIters)
    return fail(FG_ERR_INVALID_ARG, "iters=%d must be in [1, %d]", iters, kPeakMaxIters);
  FG_TRY(check_ptr(out, "out"));
  DeviceInfo* dev = nullptr;
  FG_TRY(device_info(&dev));
  int d = 0;
  cudaError_t e = cudaGetDevice(&d);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  static std::atomic<bool> attr_set[kMaxDevices];
  if (!attr_set[d].load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!attr_set[d].load(std::memory_order_relaxed)) {
      e = cudaFuncSetAttribute(fp8_mma_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kPeakSmem + 1024);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
      attr_set[d].store(true, std::memory_order_release);
    }
  }
  fp8_mma_peak_kernel<<<dev->sm_count, 128, kPeakSmem + 1024, stream>>>(iters, out, dev->status,
                                                                      wait_limit_ns());
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fp8_mma_peak_kernel launch");
  return FG_OK;
}

}  // extern "C"
