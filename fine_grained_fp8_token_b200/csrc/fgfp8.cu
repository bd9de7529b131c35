// C ABI of the fine-grained FP8 W8A8 library (declared in include/fgfp8.h):
// host-side validation, TMA descriptor encoding and kernel launches.  All
// kernels live in this translation unit so that they share the device status
// word without relocatable device code.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstdio>
#include <map>
#include <mutex>
#include <set>
#include <unordered_map>
#include <utility>
#include <string>

#include "fgfp8.h"
#include "gemm.cuh"
#include "layout.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace {

thread_local std::string t_last_error;

fgfp8_status fail(fgfp8_status code, const std::string& msg) {
  t_last_error = msg;
  return code;
}

fgfp8_status ok() {
  t_last_error.clear();
  return FGFP8_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

fgfp8_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FGFP8_ERR_CUDA, std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")");
}

struct DeviceInfo {
  int sm_count = 0;
  int cc_major = 0, cc_minor = 0;
};

constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];

fgfp8_status current_device(int* dev_out, DeviceInfo* info) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FGFP8_ERR_CUDA, "device index out of range");
  std::call_once(g_dev_once[dev], [dev] {
    cudaDeviceGetAttribute(&g_dev[dev].sm_count, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&g_dev[dev].cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&g_dev[dev].cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
  });
  *info = g_dev[dev];
  *dev_out = dev;
  if (info->cc_major != 10 || info->cc_minor != 0)
    return fail(FGFP8_ERR_CUDA, "this library is built for sm_100a (B200); device " + std::to_string(dev) +
                                    " has compute capability " + std::to_string(info->cc_major) + "." +
                                    std::to_string(info->cc_minor));
  return FGFP8_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// Encoded tensor maps, keyed by everything the encoding depends on (device,
// base address, shape, row stride, box height).  A map holds no reference to
// the memory: a later buffer at the same address with the same shape gets
// the same, still valid, map.  The cache is cleared when it reaches
// kMapCacheMax entries, so a caller cycling through many buffers never makes
// it grow without bound.
struct MapKey {
  int dev;
  const void* base;
  uint64_t rows, cols, ld;
  uint32_t box_rows;
  bool operator==(const MapKey& o) const {
    return dev == o.dev && base == o.base && rows == o.rows && cols == o.cols && ld == o.ld && box_rows == o.box_rows;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    uint64_t h = reinterpret_cast<uintptr_t>(k.base) * 0x9E3779B97F4A7C15ull;
    for (uint64_t v : {static_cast<uint64_t>(k.dev), k.rows, k.cols, k.ld, static_cast<uint64_t>(k.box_rows)})
      h = (h ^ v) * 0x100000001B3ull;
    return static_cast<size_t>(h ^ (h >> 29));
  }
};
constexpr size_t kMapCacheMax = 4096;

// 2-D map over a row-major u8 matrix [rows, cols] (row stride ld bytes) with a
// box of 128 columns (one 128-byte swizzle row) by box_rows rows, on device
// dev; encoded once per distinct key and then served from the cache.
fgfp8_status make_map_u8_sw128(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                               uint32_t box_rows, int dev) {
  static std::mutex mu;
  static std::unordered_map<MapKey, CUtensorMap, MapKeyHash> cache;
  const MapKey key{dev, base, rows, cols, ld, box_rows};
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *map = it->second;
      return FGFP8_OK;
    }
  }
  auto fn = encode_fn();
  if (!fn) return fail(FGFP8_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FGFP8_ERR_CUDA, "cuTensorMapEncodeTiled failed with code " + std::to_string(r));
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() >= kMapCacheMax) cache.clear();
  cache.emplace(key, *map);
  return FGFP8_OK;
}

// Raise the dynamic shared-memory limit of a kernel, once per (kernel, device).
fgfp8_status set_smem(const void* kernel, size_t bytes, int dev) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({kernel, dev})) return FGFP8_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  done.insert({kernel, dev});
  return FGFP8_OK;
}

// Launch with programmatic stream serialization: the grid may be scheduled
// while the preceding kernel in the stream is finishing; the kernels wait
// (griddepcontrol.wait) before touching memory that kernel may write.
template <typename... KArgs, typename... Args>
fgfp8_status launch_dependent(void (*kernel)(KArgs...), unsigned grid, unsigned threads, size_t smem,
                              cudaStream_t stream, const char* what, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) return cuda_fail(e, what);
  return ok();
}

fgfp8_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return ok();
}

fgfp8_status check_fmt(int fmt) {
  if (fmt != FGFP8_SCALE_F32 && fmt != FGFP8_SCALE_UE8M0)
    return fail(FGFP8_ERR_INVALID_ARG, "fmt must be FGFP8_SCALE_F32 (0) or FGFP8_SCALE_UE8M0 (1)");
  return FGFP8_OK;
}

fgfp8_status check_act_scales(const void* Xs, int64_t ld_s, int64_t M, int fmt) {
  if (!Xs) return fail(FGFP8_ERR_INVALID_ARG, "Xs is NULL");
  if (ld_s < M) return fail(FGFP8_ERR_SHAPE, "ld_s must be >= M");
  if (ld_s >= (int64_t(1) << 31)) return fail(FGFP8_ERR_SHAPE, "ld_s must be < 2^31");
  const int64_t unit = (fmt == FGFP8_SCALE_F32) ? 4 : 16;
  if (ld_s % unit != 0)
    return fail(FGFP8_ERR_ALIGN, fmt == FGFP8_SCALE_F32 ? "ld_s must be a multiple of 4 for fp32 scales"
                                                        : "ld_s must be a multiple of 16 for UE8M0 scales");
  if (!aligned(Xs, 16)) return fail(FGFP8_ERR_ALIGN, "Xs must be 16-byte aligned");
  return FGFP8_OK;
}

// M tiles per band of the dense tile order (see grouped_tile): the plain
// M-fastest order while the activation codes fit comfortably in L2 (every
// weight tile is then read once), else bands of 16 M tiles, whose activation
// rows and the weight tiles a wave touches fit in L2 together.
int dense_group_m(int64_t M, int64_t K, int bm) {
  const int64_t num_m = (M + bm - 1) / bm;
  if (M * K <= (int64_t(48) << 20)) return static_cast<int>(num_m);
  return static_cast<int>(num_m < 16 ? num_m : 16);
}

// Launch one GEMM instantiation as a persistent grid (one CTA per SM at most).
// kFuse: the SwiGLU gate/up projection writing the down projection's
// quantized input (Hq, Hs, ld_h) instead of Y.
template <int BN, int CW, int FMT, bool kGrouped, bool kFuse = false>
fgfp8_status launch_gemm(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq, const void* Ws,
                         void* Y, int64_t M, int64_t N, int64_t K, const int32_t* offs, int E, int64_t b_rows,
                         cudaStream_t stream, int dev, int sm_count, int early, int cap = 0, uint8_t* Hq = nullptr,
                         float* Hs = nullptr, int64_t ld_h = 0, int withhold_kb = -1) {
  using C = fgfp8::GemmCfg<BN, CW>;
  CUtensorMap mA, mB, mBh;
  fgfp8_status st = make_map_u8_sw128(&mA, Xq, static_cast<uint64_t>(M), static_cast<uint64_t>(K),
                                      static_cast<uint64_t>(K), 128, dev);
  if (st != FGFP8_OK) return st;
  st = make_map_u8_sw128(&mB, Wq, static_cast<uint64_t>(b_rows), static_cast<uint64_t>(K), static_cast<uint64_t>(K),
                         BN, dev);
  if (st != FGFP8_OK) return st;
  // the same weights with a 128-row box, for half tiles
  st = make_map_u8_sw128(&mBh, Wq, static_cast<uint64_t>(b_rows), static_cast<uint64_t>(K), static_cast<uint64_t>(K),
                         BN / 2, dev);
  if (st != FGFP8_OK) return st;
  auto kernel = fgfp8::gemm_blockscaled_kernel<BN, CW, FMT, kGrouped, kFuse>;
  st = set_smem(reinterpret_cast<const void*>(kernel), C::kSmemBytes, dev);
  if (st != FGFP8_OK) return st;
  if (C::kRegSplit) {
    // setmaxnreg.inc waits until registers are free: the warpgroups' shares
    // must fit in what the block is launched with, or it would wait forever.
    cudaFuncAttributes fa{};
    cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
    const long launch = static_cast<long>(fa.numRegs) * C::kThreads;
    const long after = 128L * C::kRegsLow + static_cast<long>(C::kThreads - 128) * C::kRegsHigh;
    if (after > launch)
      return fail(FGFP8_ERR_UNSUPPORTED, "register split exceeds the launch allocation (" + std::to_string(fa.numRegs) +
                                            " registers x " + std::to_string(C::kThreads) + " threads)");
  }
  const int64_t tiles = ((M + C::kBM - 1) / C::kBM) * (N / BN);
  if (tiles == 0) return ok();
  const int64_t grid = tiles < sm_count ? tiles : sm_count;
  // Dense 256-wide tiles: when the last partial wave of R full tiles fits
  // twice into one wave (2R <= grid), those R tiles run as 2R half tiles,
  // so that wave takes about half a tile's time instead of a whole one.
  int64_t num_full = tiles, items = tiles;
  if (!kGrouped && !kFuse && BN == 256) {
    const int64_t waves = tiles / grid, rest = tiles - waves * grid;
    if (waves >= 1 && rest > 0 && 2 * rest <= grid) {
      num_full = waves * grid;
      items = num_full + 2 * rest;
    }
  }
  return launch_dependent(kernel, static_cast<unsigned>(grid), C::kThreads, C::kSmemBytes, stream, "gemm launch", mA,
                          mB, mBh, Xs, static_cast<uint32_t>(ld_s), Ws, reinterpret_cast<__nv_bfloat16*>(Y),
                          static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), offs, E, cap,
                          static_cast<int>(items), static_cast<int>(num_full), early, Hq, Hs,
                          static_cast<uint32_t>(ld_h), withhold_kb, dense_group_m(M, K, C::kBM));
}

// UE8M0 launch with hardware block scaling (persistent, 128 x BN tiles).
template <int BN, bool kGrouped>
fgfp8_status launch_gemm_mx(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq, const void* Ws,
                            void* Y, int64_t M, int64_t N, int64_t K, const int32_t* offs, int E, int64_t b_rows,
                            cudaStream_t stream, int dev, int sm_count, int early, int cap, int withhold_kb = -1) {
  using C = fgfp8::MxCfg<BN>;
  CUtensorMap mA, mB, mBh;
  fgfp8_status st = make_map_u8_sw128(&mA, Xq, static_cast<uint64_t>(M), static_cast<uint64_t>(K),
                                      static_cast<uint64_t>(K), 128, dev);
  if (st != FGFP8_OK) return st;
  st = make_map_u8_sw128(&mB, Wq, static_cast<uint64_t>(b_rows), static_cast<uint64_t>(K), static_cast<uint64_t>(K),
                         C::kBN, dev);
  if (st != FGFP8_OK) return st;
  st = make_map_u8_sw128(&mBh, Wq, static_cast<uint64_t>(b_rows), static_cast<uint64_t>(K), static_cast<uint64_t>(K),
                         C::kBN / 2, dev);
  if (st != FGFP8_OK) return st;
  auto kernel = fgfp8::gemm_mx_kernel<BN, kGrouped>;
  st = set_smem(reinterpret_cast<const void*>(kernel), C::kSmemBytes, dev);
  if (st != FGFP8_OK) return st;
  const int64_t tiles = ((M + C::kBM - 1) / C::kBM) * (N / C::kBN);
  if (tiles == 0) return ok();
  const int64_t grid = tiles < sm_count ? tiles : sm_count;
  // dense 128 x 256 tiles: the last partial wave as half tiles when it fits
  // twice into one wave
  int64_t num_full = tiles, items = tiles;
  if (!kGrouped && BN == 256) {
    const int64_t waves = tiles / grid, rest = tiles - waves * grid;
    if (waves >= 1 && rest > 0 && 2 * rest <= grid) {
      num_full = waves * grid;
      items = num_full + 2 * rest;
    }
  }
  return launch_dependent(kernel, static_cast<unsigned>(grid), C::kThreads, C::kSmemBytes, stream,
                          "block-scaled gemm launch", mA, mB, mBh, reinterpret_cast<const uint8_t*>(Xs),
                          static_cast<uint32_t>(ld_s), reinterpret_cast<const uint8_t*>(Ws),
                          reinterpret_cast<__nv_bfloat16*>(Y), static_cast<int>(M), static_cast<int>(N),
                          static_cast<int>(K), offs, E, cap, static_cast<int>(items), static_cast<int>(num_full),
                          early, withhold_kb, dense_group_m(M, K, C::kBM));
}

template <bool kGrouped>
fgfp8_status dispatch_gemm(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq, const void* Ws, void* Y,
                           int64_t M, int64_t N, int64_t K, int fmt, const int32_t* offs, int E, int64_t b_rows,
                           cudaStream_t s, int dev, int sms, int early, int cap = 0) {
  // 128x256 tiles: measured faster per FLOP than 128x128 on B200 even where
  // 128x128 tiles would fill the last wave better (4096^3: 95 us vs 119 us);
  // 128x128 only when N is not a multiple of 256.
  const bool wide = (N % 256 == 0);
  constexpr int kWideCW = 128;
  // UE8M0 scales: the tensor core applies them (block-scaled MMA), no promotion.
  if (fmt == FGFP8_SCALE_UE8M0)
    return wide ? launch_gemm_mx<256, kGrouped>(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, offs, E, b_rows, s, dev, sms, early,
                                                cap)
                : launch_gemm_mx<128, kGrouped>(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, offs, E, b_rows, s, dev, sms, early,
                                                cap);
  return wide ? launch_gemm<256, kWideCW, 0, kGrouped>(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, offs, E, b_rows, s, dev, sms,
                                                       early, cap)
              : launch_gemm<128, 64, 0, kGrouped>(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, offs, E, b_rows, s, dev, sms,
                                                  early, cap);
}

// Few-token (M <= 64) launch: one CTA per 128 output columns, operands swapped.
template <int BNT, int FMT>
fgfp8_status launch_decode(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq, const void* Ws,
                           void* Y, int64_t M, int64_t N, int64_t K, cudaStream_t stream, int dev, int early) {
  using C = fgfp8::DecodeCfg<BNT>;
  CUtensorMap mX, mW;
  fgfp8_status st = make_map_u8_sw128(&mX, Xq, static_cast<uint64_t>(M), static_cast<uint64_t>(K),
                                      static_cast<uint64_t>(K), BNT, dev);
  if (st != FGFP8_OK) return st;
  st = make_map_u8_sw128(&mW, Wq, static_cast<uint64_t>(N), static_cast<uint64_t>(K), static_cast<uint64_t>(K), 128, dev);
  if (st != FGFP8_OK) return st;
  auto kernel = fgfp8::gemm_decode_kernel<BNT, FMT>;
  st = set_smem(reinterpret_cast<const void*>(kernel), C::kSmemBytes, dev);
  if (st != FGFP8_OK) return st;
  return launch_dependent(kernel, static_cast<unsigned>(N / 128), C::kThreads, C::kSmemBytes, stream,
                          "decode gemm launch", mX, mW, Xs, static_cast<uint32_t>(ld_s), Ws,
                          reinterpret_cast<__nv_bfloat16*>(Y), static_cast<int>(M), static_cast<int>(N),
                          static_cast<int>(K), early);
}

// UE8M0 few-token launch: the block-scaled MMA applies the scales.
template <int BNT>
fgfp8_status launch_decode_mx(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq, const void* Ws,
                              void* Y, int64_t M, int64_t N, int64_t K, cudaStream_t stream, int dev, int early) {
  using C = fgfp8::DecodeMxCfg<BNT>;
  CUtensorMap mX, mW;
  fgfp8_status st = make_map_u8_sw128(&mX, Xq, static_cast<uint64_t>(M), static_cast<uint64_t>(K),
                                      static_cast<uint64_t>(K), BNT, dev);
  if (st != FGFP8_OK) return st;
  st = make_map_u8_sw128(&mW, Wq, static_cast<uint64_t>(N), static_cast<uint64_t>(K), static_cast<uint64_t>(K), 128, dev);
  if (st != FGFP8_OK) return st;
  auto kernel = fgfp8::gemm_decode_mx_kernel<BNT>;
  st = set_smem(reinterpret_cast<const void*>(kernel), C::kSmemBytes, dev);
  if (st != FGFP8_OK) return st;
  return launch_dependent(kernel, static_cast<unsigned>(N / 128), C::kThreads, C::kSmemBytes, stream,
                          "decode gemm launch", mX, mW, reinterpret_cast<const uint8_t*>(Xs),
                          static_cast<uint32_t>(ld_s), reinterpret_cast<const uint8_t*>(Ws),
                          reinterpret_cast<__nv_bfloat16*>(Y), static_cast<int>(M), static_cast<int>(N),
                          static_cast<int>(K), early);
}

template <int FMT>
fgfp8_status dispatch_decode(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq, const void* Ws,
                             void* Y, int64_t M, int64_t N, int64_t K, cudaStream_t s, int dev, int early) {
  if constexpr (FMT == FGFP8_SCALE_UE8M0) {
    if (M <= 16) return launch_decode_mx<16>(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, s, dev, early);
    if (M <= 32) return launch_decode_mx<32>(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, s, dev, early);
    return launch_decode_mx<64>(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, s, dev, early);
  } else {
    if (M <= 16) return launch_decode<16, FMT>(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, s, dev, early);
    if (M <= 32) return launch_decode<32, FMT>(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, s, dev, early);
    return launch_decode<64, FMT>(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, s, dev, early);
  }
}

// Row/column-scaled GEMM: persistent grid of 128 x BN tiles.
template <int BN>
fgfp8_status launch_gemm_rowcol(const uint8_t* Xq, const float* sx, int x_per_tensor, const uint8_t* Wq,
                                const float* sw, int w_per_tensor, void* Y, int64_t M, int64_t N, int64_t K,
                                cudaStream_t stream, int dev, int sm_count) {
  using C = fgfp8::RowColCfg<BN>;
  CUtensorMap mA, mB, mBh;
  fgfp8_status st = make_map_u8_sw128(&mA, Xq, static_cast<uint64_t>(M), static_cast<uint64_t>(K),
                                      static_cast<uint64_t>(K), 128, dev);
  if (st != FGFP8_OK) return st;
  st = make_map_u8_sw128(&mB, Wq, static_cast<uint64_t>(N), static_cast<uint64_t>(K), static_cast<uint64_t>(K), BN, dev);
  if (st != FGFP8_OK) return st;
  st = make_map_u8_sw128(&mBh, Wq, static_cast<uint64_t>(N), static_cast<uint64_t>(K), static_cast<uint64_t>(K),
                         BN / 2, dev);
  if (st != FGFP8_OK) return st;
  auto kernel = fgfp8::gemm_rowcol_kernel<BN>;
  st = set_smem(reinterpret_cast<const void*>(kernel), C::kSmemBytes, dev);
  if (st != FGFP8_OK) return st;
  const int64_t tiles = ((M + C::kBM - 1) / C::kBM) * (N / BN);
  if (tiles == 0) return ok();
  const int64_t grid = tiles < sm_count ? tiles : sm_count;
  // the last partial wave as half tiles when it fits twice into one wave
  int64_t num_full = tiles, items = tiles;
  if (BN == 256) {
    const int64_t waves = tiles / grid, rest = tiles - waves * grid;
    if (waves >= 1 && rest > 0 && 2 * rest <= grid) {
      num_full = waves * grid;
      items = num_full + 2 * rest;
    }
  }
  return launch_dependent(kernel, static_cast<unsigned>(grid), C::kThreads, C::kSmemBytes, stream,
                          "row/column-scaled gemm launch", mA, mB, mBh, sx, x_per_tensor, sw, w_per_tensor,
                          reinterpret_cast<__nv_bfloat16*>(Y), static_cast<int>(M), static_cast<int>(N),
                          static_cast<int>(K), static_cast<int>(items), static_cast<int>(num_full),
                          dense_group_m(M, K, C::kBM));
}

// Shared checks of the row / tensor quantizers' input X bf16 [R, K] (row
// stride ldx) and, when given, their codes Xq u8 [R, K].
fgfp8_status check_rows_common(const void* X, int64_t R, int64_t K, int64_t ldx, bool has_codes,
                               const uint8_t* Xq) {
  if (R < 0 || K < 0 || ldx < 0) return fail(FGFP8_ERR_INVALID_ARG, "negative size");
  if (K == 0 || K % 128 != 0) return fail(FGFP8_ERR_SHAPE, "K must be a positive multiple of 128");
  if (ldx < K) return fail(FGFP8_ERR_SHAPE, "ldx must be >= K");
  if (R >= (int64_t(1) << 31) || R * (K / 8) >= (int64_t(1) << 32))
    return fail(FGFP8_ERR_SHAPE, "R must be < 2^31 and R*K/8 < 2^32");
  if (R > 0 && !X) return fail(FGFP8_ERR_INVALID_ARG, "X is NULL");
  if (!aligned(X, 16) || ldx % 8 != 0) return fail(FGFP8_ERR_ALIGN, "X must be 16-byte aligned with ldx % 8 == 0");
  if (has_codes) {
    if (R > 0 && !Xq) return fail(FGFP8_ERR_INVALID_ARG, "Xq is NULL");
    if (!aligned(Xq, 16)) return fail(FGFP8_ERR_ALIGN, "Xq must be 16-byte aligned");
  }
  return FGFP8_OK;
}

// CTAs of `kernel` (with `threads` threads, no dynamic shared memory) that
// are resident on the device at once, from the occupancy calculator, cached
// per (kernel, device).  A grid-stride kernel launched with more CTAs than
// this runs the excess as a partial second wave that finishes last.
int64_t resident_blocks(const void* kernel, int threads, int dev, int sm_count) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int64_t> cache;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find({kernel, dev});
  if (it != cache.end()) return it->second;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int64_t n = static_cast<int64_t>(sm_count) * per_sm;
  cache[{kernel, dev}] = n;
  return n;
}

// Grid of a grid-stride kernel over work_items items of one thread each:
// enough 256-thread CTAs for the work, at most one resident wave.  (For the
// static quantizer, 16 bytes per item, this measured faster than a grid
// covering every item in one pass: 16.0 against 19.0 us on 4096 x 4096.)
unsigned grid_stride_blocks(const void* kernel, int64_t work_items, int dev, int sm_count) {
  const int64_t want = (work_items + 255) / 256;
  const int64_t cap = resident_blocks(kernel, 256, dev, sm_count);
  return static_cast<unsigned>(want < 1 ? 1 : (want < cap ? want : cap));
}

fgfp8_status check_gemm_common(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq, const void* Ws,
                               void* Y, int64_t M, int64_t N, int64_t K, int fmt) {
  fgfp8_status st = check_fmt(fmt);
  if (st != FGFP8_OK) return st;
  if (M < 0 || N < 0 || K < 0) return fail(FGFP8_ERR_INVALID_ARG, "negative size");
  if (K == 0 || K % 128 != 0) return fail(FGFP8_ERR_SHAPE, "K must be a positive multiple of 128");
  if (N == 0 || N % 128 != 0) return fail(FGFP8_ERR_SHAPE, "N must be a positive multiple of 128");
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
    return fail(FGFP8_ERR_SHAPE, "M, N and K must be < 2^31");
  if (!Xq || !Wq || !Ws || !Y) return fail(FGFP8_ERR_INVALID_ARG, "a required pointer is NULL");
  st = check_act_scales(Xs, ld_s, M, fmt);
  if (st != FGFP8_OK) return st;
  if (!aligned(Xq, 16) || !aligned(Wq, 16) || !aligned(Y, 16))
    return fail(FGFP8_ERR_ALIGN, "Xq, Wq and Y must be 16-byte aligned");
  if (fmt == FGFP8_SCALE_F32 && !aligned(Ws, 4)) return fail(FGFP8_ERR_ALIGN, "fp32 Ws must be 4-byte aligned");
  return FGFP8_OK;
}

}  // namespace

namespace {

// Dynamic 1x128 activation quantization; with dry set, only validates.
fgfp8_status quant_act_impl(const void* X, int64_t M, int64_t K, int64_t ldx, uint8_t* Xq, void* Xs, int64_t ld_s,
                            int fmt, void* stream, bool dry) {
  fgfp8_status st = check_fmt(fmt);
  if (st != FGFP8_OK) return st;
  if (M < 0 || K < 0 || ldx < 0) return fail(FGFP8_ERR_INVALID_ARG, "negative size");
  if (K == 0 || K % 128 != 0) return fail(FGFP8_ERR_SHAPE, "K must be a positive multiple of 128");
  if (ldx < K) return fail(FGFP8_ERR_SHAPE, "ldx must be >= K");
  if (M == 0) return ok();
  if (M * (K / 128) >= (int64_t(1) << 32) || K >= (int64_t(1) << 31))
    return fail(FGFP8_ERR_SHAPE, "M*K/128 must be < 2^32 and K < 2^31");
  if (!X || !Xq) return fail(FGFP8_ERR_INVALID_ARG, "X or Xq is NULL");
  st = check_act_scales(Xs, ld_s, M, fmt);
  if (st != FGFP8_OK) return st;
  if (!aligned(X, 16) || ldx % 8 != 0) return fail(FGFP8_ERR_ALIGN, "X must be 16-byte aligned with ldx % 8 == 0");
  if (!aligned(Xq, 16)) return fail(FGFP8_ERR_ALIGN, "Xq must be 16-byte aligned");
  if (dry) return FGFP8_OK;
  int dev;
  DeviceInfo info;
  st = current_device(&dev, &info);
  if (st != FGFP8_OK) return st;

  // One 8-lane team per 1x128 group and one or two groups per team.  The
  // grid covers every group in one pass (up to 2^23 blocks; the kernel
  // strides over the rest): the block scheduler hands out blocks as others
  // finish, which measured faster than one resident wave striding over the
  // groups (ncu, 8192x14336: 62.2 -> 58.4 us; 4096x4096: 11.4 -> 11.0 us).
  // Inputs of up to 2^26 elements take one group per team (more blocks),
  // larger ones two (more bytes in flight per lane).
  const uint64_t groups = static_cast<uint64_t>(M) * (K / 128);
  const bool one = static_cast<uint64_t>(M) * static_cast<uint64_t>(K) <= (uint64_t(1) << 26);
  const uint64_t per_block = 32u * (one ? 1u : 2u);
  const uint64_t want = (groups + per_block - 1) / per_block;
  const unsigned blocks = static_cast<unsigned>(want == 0 ? 1 : (want < (uint64_t(1) << 23) ? want : (uint64_t(1) << 23)));
  fgfp8::FastDiv kbd(static_cast<uint32_t>(K / 128));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  auto go = [&](auto kernel) {
    kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const uint16_t*>(X), static_cast<uint32_t>(M),
                                  static_cast<uint32_t>(K), static_cast<uint64_t>(ldx), Xq, Xs,
                                  static_cast<uint64_t>(ld_s), kbd);
  };
  if (fmt == FGFP8_SCALE_F32) {
    if (one) go(fgfp8::quant_act_kernel<0, 1>);
    else go(fgfp8::quant_act_kernel<0, 2>);
  } else {
    if (one) go(fgfp8::quant_act_kernel<1, 1>);
    else go(fgfp8::quant_act_kernel<1, 2>);
  }
  return check_launch("quant_act launch");
}

// Dense block-scaled GEMM; early lets the weight loads start before the wait
// for the preceding grid; with dry set, only validates.
fgfp8_status gemm_impl(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq, const void* Ws, void* Y,
                       int64_t M, int64_t N, int64_t K, int fmt, void* stream, int early, bool dry) {
  if (M == 0 && fmt >= 0 && fmt <= 1 && N >= 0 && K >= 0) return ok();
  fgfp8_status st = check_gemm_common(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, fmt);
  if (st != FGFP8_OK) return st;
  if (dry) return FGFP8_OK;
  int dev;
  DeviceInfo info;
  st = current_device(&dev, &info);
  if (st != FGFP8_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (M <= 64) {
    return fmt == FGFP8_SCALE_F32 ? dispatch_decode<0>(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, s, dev, early)
                                  : dispatch_decode<1>(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, s, dev, early);
  }
  return dispatch_gemm<false>(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, fmt, nullptr, 1, N, s, dev, info.sm_count, early);
}

// M-grouped expert GEMM; with dry set, only validates.
fgfp8_status grouped_impl(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq, const void* Ws, void* Y,
                          const int32_t* group_offs, int32_t E, int64_t M_total, int64_t N, int64_t K, int fmt,
                          void* stream, bool dry) {
  if (E <= 0) return fail(FGFP8_ERR_INVALID_ARG, "E must be >= 1");
  if (M_total % 128 != 0) return fail(FGFP8_ERR_SHAPE, "M_total must be a multiple of 128");
  if (M_total == 0 && fmt >= 0 && fmt <= 1 && N >= 0 && K >= 0) return ok();
  fgfp8_status st = check_gemm_common(Xq, Xs, ld_s, Wq, Ws, Y, M_total, N, K, fmt);
  if (st != FGFP8_OK) return st;
  if (!group_offs) return fail(FGFP8_ERR_INVALID_ARG, "group_offs is NULL");
  if (!aligned(group_offs, 4)) return fail(FGFP8_ERR_ALIGN, "group_offs must be 4-byte aligned");
  if (static_cast<int64_t>(E) * N >= (int64_t(1) << 31))
    return fail(FGFP8_ERR_SHAPE, "E*N must be < 2^31");
  if (dry) return FGFP8_OK;
  int dev;
  DeviceInfo info;
  st = current_device(&dev, &info);
  if (st != FGFP8_OK) return st;
  return dispatch_gemm<true>(Xq, Xs, ld_s, Wq, Ws, Y, M_total, N, K, fmt, group_offs, E,
                             static_cast<int64_t>(E) * N, reinterpret_cast<cudaStream_t>(stream), dev, info.sm_count, 0);
}

}  // namespace

// ---------------------------------------------------------------------------
// Static scratch of fgfp8_linear_noalloc: the quantized activations (codes,
// then scales) of one call live here instead of in caller-allocated buffers.
// Every device that loads this library holds FGFP8_NOALLOC_SCRATCH_BYTES of
// it until the process exits.  Host code must not pass the symbol itself to
// a kernel (on the host it names a stand-in object, not device memory): the
// device address comes from cudaGetSymbolAddress, once per device.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_noalloc_scratch[FGFP8_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of g_noalloc_scratch on the current device `dev`, looked up
// on the first call for that device and cached.  A failed lookup is reported
// and retried on the next call.
fgfp8_status noalloc_scratch(int dev, uint8_t** out) {
  static std::mutex mu;
  static uint8_t* addr[kMaxDevices] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the static scratch");
    if (!p || !aligned(p, 256)) return fail(FGFP8_ERR_CUDA, "the static scratch has no 256-byte aligned address");
    addr[dev] = static_cast<uint8_t*>(p);
  }
  *out = addr[dev];
  return FGFP8_OK;
}

// Masked expert GEMM; with dry set, only validates.
fgfp8_status masked_impl(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq, const void* Ws, void* Y,
                         const int32_t* counts, int32_t E, int64_t cap, int64_t N, int64_t K, int fmt, void* stream,
                         bool dry) {
  if (E <= 0) return fail(FGFP8_ERR_INVALID_ARG, "E must be >= 1");
  if (cap <= 0 || cap % 128 != 0) return fail(FGFP8_ERR_SHAPE, "cap must be a positive multiple of 128");
  if (static_cast<int64_t>(E) * cap >= (int64_t(1) << 31)) return fail(FGFP8_ERR_SHAPE, "E*cap must be < 2^31");
  const int64_t M_total = static_cast<int64_t>(E) * cap;
  fgfp8_status st = check_gemm_common(Xq, Xs, ld_s, Wq, Ws, Y, M_total, N, K, fmt);
  if (st != FGFP8_OK) return st;
  if (!counts) return fail(FGFP8_ERR_INVALID_ARG, "counts is NULL");
  if (!aligned(counts, 4)) return fail(FGFP8_ERR_ALIGN, "counts must be 4-byte aligned");
  if (static_cast<int64_t>(E) * N >= (int64_t(1) << 31)) return fail(FGFP8_ERR_SHAPE, "E*N must be < 2^31");
  if (dry) return FGFP8_OK;
  int dev;
  DeviceInfo info;
  st = current_device(&dev, &info);
  if (st != FGFP8_OK) return st;
  return dispatch_gemm<true>(Xq, Xs, ld_s, Wq, Ws, Y, M_total, N, K, fmt, counts, E, static_cast<int64_t>(E) * N,
                             reinterpret_cast<cudaStream_t>(stream), dev, info.sm_count, 0, static_cast<int>(cap));
}

// Activation quantizer over the token rows of the masked layout; with dry
// set, only validates.
fgfp8_status quant_act_masked_impl(const void* X, int64_t ldx, const int32_t* counts, int32_t E, int64_t cap,
                                   int64_t K, uint8_t* Xq, void* Xs, int64_t ld_s, int fmt, void* stream, bool dry) {
  if (E <= 0) return fail(FGFP8_ERR_INVALID_ARG, "E must be >= 1");
  if (cap <= 0 || cap % 128 != 0) return fail(FGFP8_ERR_SHAPE, "cap must be a positive multiple of 128");
  if (static_cast<int64_t>(E) * cap >= (int64_t(1) << 31)) return fail(FGFP8_ERR_SHAPE, "E*cap must be < 2^31");
  if (E > 65535) return fail(FGFP8_ERR_SHAPE, "E must be <= 65535");
  if (!counts) return fail(FGFP8_ERR_INVALID_ARG, "counts is NULL");
  if (!aligned(counts, 4)) return fail(FGFP8_ERR_ALIGN, "counts must be 4-byte aligned");
  const int64_t M = static_cast<int64_t>(E) * cap;
  // the same checks as the quantizer over all E * cap rows
  fgfp8_status st = quant_act_impl(X, M, K, ldx, Xq, Xs, ld_s, fmt, stream, true);
  if (st != FGFP8_OK) return st;
  if (dry) return FGFP8_OK;
  int dev;
  DeviceInfo info;
  st = current_device(&dev, &info);
  if (st != FGFP8_OK) return st;
  // blocks per expert: a full expert block in about seven passes of 32
  // groups each; blocks beyond an expert's count exit at once
  const int64_t most = cap * (K / 128);                       // groups of a full expert block
  int64_t bx = (most + 255) / 256;
  bx = bx < 1 ? 1 : (bx > 32 ? 32 : bx);
  const dim3 grid(static_cast<unsigned>(bx), static_cast<unsigned>(E));
  fgfp8::FastDiv kbd(static_cast<uint32_t>(K / 128));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (fmt == FGFP8_SCALE_F32)
    fgfp8::quant_act_masked_kernel<0><<<grid, 256, 0, s>>>(reinterpret_cast<const uint16_t*>(X), counts,
                                                           static_cast<uint32_t>(cap), static_cast<uint32_t>(K),
                                                           static_cast<uint64_t>(ldx), Xq, Xs,
                                                           static_cast<uint64_t>(ld_s), kbd);
  else
    fgfp8::quant_act_masked_kernel<1><<<grid, 256, 0, s>>>(reinterpret_cast<const uint16_t*>(X), counts,
                                                           static_cast<uint32_t>(cap), static_cast<uint32_t>(K),
                                                           static_cast<uint64_t>(ldx), Xq, Xs,
                                                           static_cast<uint64_t>(ld_s), kbd);
  return check_launch("masked quant_act launch");
}

}  // namespace

extern "C" {

int fgfp8_version(void) { return FGFP8_VERSION; }

const char* fgfp8_last_error_string(void) { return t_last_error.c_str(); }


fgfp8_status fgfp8_quant_weight(const void* W, int64_t N, int64_t K, int64_t ldw, uint8_t* Wq, void* Ws, int fmt,
                                void* stream) {
  fgfp8_status st = check_fmt(fmt);
  if (st != FGFP8_OK) return st;
  if (N < 0 || K < 0 || ldw < 0) return fail(FGFP8_ERR_INVALID_ARG, "negative size");
  if (K == 0 || K % 128 != 0) return fail(FGFP8_ERR_SHAPE, "K must be a positive multiple of 128");
  if (N % 128 != 0) return fail(FGFP8_ERR_SHAPE, "N must be a multiple of 128");
  if (ldw < K) return fail(FGFP8_ERR_SHAPE, "ldw must be >= K");
  if (N == 0) return ok();
  if ((N / 128) * (K / 128) >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
    return fail(FGFP8_ERR_SHAPE, "(N/128)*(K/128) must be < 2^31");
  if (!W || !Wq || !Ws) return fail(FGFP8_ERR_INVALID_ARG, "W, Wq or Ws is NULL");
  if (!aligned(W, 16) || ldw % 8 != 0) return fail(FGFP8_ERR_ALIGN, "W must be 16-byte aligned with ldw % 8 == 0");
  if (!aligned(Wq, 16)) return fail(FGFP8_ERR_ALIGN, "Wq must be 16-byte aligned");
  if (fmt == FGFP8_SCALE_F32 && !aligned(Ws, 4)) return fail(FGFP8_ERR_ALIGN, "fp32 Ws must be 4-byte aligned");
  int dev;
  DeviceInfo info;
  st = current_device(&dev, &info);
  if (st != FGFP8_OK) return st;
  const unsigned blocks = static_cast<unsigned>((N / 128) * (K / 128));
  fgfp8::FastDiv kbd(static_cast<uint32_t>(K / 128));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (fmt == FGFP8_SCALE_F32)
    fgfp8::quant_weight_kernel<0><<<blocks, 256, 0, s>>>(reinterpret_cast<const uint16_t*>(W),
                                                         static_cast<uint32_t>(K), static_cast<uint64_t>(ldw), Wq, Ws,
                                                         kbd);
  else
    fgfp8::quant_weight_kernel<1><<<blocks, 256, 0, s>>>(reinterpret_cast<const uint16_t*>(W),
                                                         static_cast<uint32_t>(K), static_cast<uint64_t>(ldw), Wq, Ws,
                                                         kbd);
  return check_launch("quant_weight launch");
}



fgfp8_status fgfp8_quant_act(const void* X, int64_t M, int64_t K, int64_t ldx, uint8_t* Xq, void* Xs, int64_t ld_s,
                             int fmt, void* stream) {
  return quant_act_impl(X, M, K, ldx, Xq, Xs, ld_s, fmt, stream, false);
}

fgfp8_status fgfp8_gemm(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq, const void* Ws, void* Y,
                        int64_t M, int64_t N, int64_t K, int fmt, void* stream) {
  return gemm_impl(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, fmt, stream, 0, false);
}

fgfp8_status fgfp8_grouped_gemm(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq, const void* Ws,
                                void* Y, const int32_t* group_offs, int32_t E, int64_t M_total, int64_t N, int64_t K,
                                int fmt, void* stream) {
  return grouped_impl(Xq, Xs, ld_s, Wq, Ws, Y, group_offs, E, M_total, N, K, fmt, stream, false);
}

fgfp8_status fgfp8_linear(const void* X, int64_t ldx, uint8_t* Xq, void* Xs, int64_t ld_s, const uint8_t* Wq,
                          const void* Ws, void* Y, int64_t M, int64_t N, int64_t K, int fmt, void* stream) {
  fgfp8_status st = quant_act_impl(X, M, K, ldx, Xq, Xs, ld_s, fmt, stream, true);
  if (st != FGFP8_OK) return st;
  st = gemm_impl(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, fmt, stream, 1, true);
  if (st != FGFP8_OK) return st;
  st = quant_act_impl(X, M, K, ldx, Xq, Xs, ld_s, fmt, stream, false);
  if (st != FGFP8_OK) return st;
  // the quantizer writes only Xq and Xs: the GEMM may request weight tiles early
  return gemm_impl(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, fmt, stream, 1, false);
}

fgfp8_status fgfp8_grouped_linear(const void* X, int64_t ldx, uint8_t* Xq, void* Xs, int64_t ld_s, const uint8_t* Wq,
                                  const void* Ws, void* Y, const int32_t* group_offs, int32_t E, int64_t M_total,
                                  int64_t N, int64_t K, int fmt, void* stream) {
  fgfp8_status st = quant_act_impl(X, M_total, K, ldx, Xq, Xs, ld_s, fmt, stream, true);
  if (st != FGFP8_OK) return st;
  st = grouped_impl(Xq, Xs, ld_s, Wq, Ws, Y, group_offs, E, M_total, N, K, fmt, stream, true);
  if (st != FGFP8_OK) return st;
  st = quant_act_impl(X, M_total, K, ldx, Xq, Xs, ld_s, fmt, stream, false);
  if (st != FGFP8_OK) return st;
  return grouped_impl(Xq, Xs, ld_s, Wq, Ws, Y, group_offs, E, M_total, N, K, fmt, stream, false);
}

fgfp8_status fgfp8_linear_noalloc(const void* X, int64_t ldx, const uint8_t* Wq, const void* Ws, void* Y,
                                  int64_t M, int64_t N, int64_t K, int fmt, void* stream) {
  // Everything that can be checked without a device comes first, so an
  // oversized request is rejected before any CUDA call.
  fgfp8_status st = check_fmt(fmt);
  if (st != FGFP8_OK) return st;
  if (M < 0 || N < 0 || K < 0 || ldx < 0) return fail(FGFP8_ERR_INVALID_ARG, "negative size");
  if (K == 0 || K % 128 != 0) return fail(FGFP8_ERR_SHAPE, "K must be a positive multiple of 128");
  if (N == 0 || N % 128 != 0) return fail(FGFP8_ERR_SHAPE, "N must be a positive multiple of 128");
  if (M == 0) return ok();
  const int64_t ld_s = (M + 15) / 16 * 16;              // valid for both scale formats
  const int64_t scale_bytes = (fmt == FGFP8_SCALE_F32) ? 4 : 1;
  const int64_t limit = static_cast<int64_t>(FGFP8_NOALLOC_SCRATCH_BYTES);
  if (M > limit || K > limit) return fail(FGFP8_ERR_SHAPE, "M or K exceeds the static scratch");
  const int64_t codes = (M * K + 255) / 256 * 256;      // Xq, then Xs at a 256-byte boundary
  const int64_t need = codes + (K / 128) * ld_s * scale_bytes;
  if (need > limit)
    return fail(FGFP8_ERR_SHAPE, "M x K too large for the static scratch: the quantized activations need " +
                                     std::to_string(need) + " bytes, the limit is " + std::to_string(limit) +
                                     " (FGFP8_NOALLOC_SCRATCH_BYTES); use fgfp8_linear with caller buffers");
  if (!X || !Wq || !Ws || !Y) return fail(FGFP8_ERR_INVALID_ARG, "X, Wq, Ws or Y is NULL");
  int dev;
  DeviceInfo info;
  st = current_device(&dev, &info);
  if (st != FGFP8_OK) return st;
  uint8_t* scratch = nullptr;
  st = noalloc_scratch(dev, &scratch);
  if (st != FGFP8_OK) return st;
  uint8_t* Xq = scratch;
  void* Xs = scratch + codes;
  // the same validation-first sequence as fgfp8_linear, on the scratch buffers
  st = quant_act_impl(X, M, K, ldx, Xq, Xs, ld_s, fmt, stream, true);
  if (st != FGFP8_OK) return st;
  st = gemm_impl(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, fmt, stream, 1, true);
  if (st != FGFP8_OK) return st;
  st = quant_act_impl(X, M, K, ldx, Xq, Xs, ld_s, fmt, stream, false);
  if (st != FGFP8_OK) return st;
  return gemm_impl(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, fmt, stream, 1, false);
}

fgfp8_status fgfp8_quant_rows(const void* X, int64_t R, int64_t K, int64_t ldx, uint8_t* Xq, float* scales,
                              void* stream) {
  fgfp8_status st = check_rows_common(X, R, K, ldx, true, Xq);
  if (st != FGFP8_OK) return st;
  if (R == 0) return ok();
  if (!scales) return fail(FGFP8_ERR_INVALID_ARG, "scales is NULL");
  if (!aligned(scales, 4)) return fail(FGFP8_ERR_ALIGN, "scales must be 4-byte aligned");
  int dev;
  DeviceInfo info;
  st = current_device(&dev, &info);
  if (st != FGFP8_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K <= fgfp8::kWarpRowChunks * 32 * 8)
    fgfp8::quant_rows_warp_kernel<<<static_cast<unsigned>((R + 7) / 8), 256, 0, s>>>(
        reinterpret_cast<const uint16_t*>(X), static_cast<uint32_t>(R), static_cast<uint32_t>(K),
        static_cast<uint64_t>(ldx), Xq, scales);
  else
    fgfp8::quant_rows_kernel<<<static_cast<unsigned>(R), fgfp8::kRowThreads, 0, s>>>(
        reinterpret_cast<const uint16_t*>(X), static_cast<uint32_t>(K), static_cast<uint64_t>(ldx), Xq, scales);
  return check_launch("quant_rows launch");
}

fgfp8_status fgfp8_tensor_scale(const void* X, int64_t R, int64_t K, int64_t ldx, float* scale, void* stream) {
  fgfp8_status st = check_rows_common(X, R, K, ldx, false, nullptr);
  if (st != FGFP8_OK) return st;
  if (!scale) return fail(FGFP8_ERR_INVALID_ARG, "scale is NULL");
  if (!aligned(scale, 4)) return fail(FGFP8_ERR_ALIGN, "scale must be 4-byte aligned");
  int dev;
  DeviceInfo info;
  st = current_device(&dev, &info);
  if (st != FGFP8_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* word = reinterpret_cast<uint32_t*>(scale);
  cudaError_t e = cudaMemsetAsync(word, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the amax word");
  if (R > 0) {
    fgfp8::FastDiv chunks(static_cast<uint32_t>(K / 8));
    fgfp8::tensor_amax_kernel<<<grid_stride_blocks(reinterpret_cast<const void*>(fgfp8::tensor_amax_kernel),
                                                   R * (K / 8), dev, info.sm_count),
                                256, 0, s>>>(
        reinterpret_cast<const uint16_t*>(X), static_cast<uint32_t>(R), static_cast<uint32_t>(K),
        static_cast<uint64_t>(ldx), chunks, word);
    st = check_launch("tensor amax launch");
    if (st != FGFP8_OK) return st;
  }
  fgfp8::tensor_scale_finish_kernel<<<1, 32, 0, s>>>(word);
  return check_launch("tensor scale launch");
}

fgfp8_status fgfp8_quant_static(const void* X, int64_t R, int64_t K, int64_t ldx, const float* scale, uint8_t* Xq,
                                void* stream) {
  fgfp8_status st = check_rows_common(X, R, K, ldx, true, Xq);
  if (st != FGFP8_OK) return st;
  if (R == 0) return ok();
  if (!scale) return fail(FGFP8_ERR_INVALID_ARG, "scale is NULL");
  if (!aligned(scale, 4)) return fail(FGFP8_ERR_ALIGN, "scale must be 4-byte aligned");
  int dev;
  DeviceInfo info;
  st = current_device(&dev, &info);
  if (st != FGFP8_OK) return st;
  fgfp8::FastDiv chunks(static_cast<uint32_t>(K / 8));
  fgfp8::quant_static_kernel<<<grid_stride_blocks(reinterpret_cast<const void*>(fgfp8::quant_static_kernel),
                                                  R * (K / 8), dev, info.sm_count),
                               256, 0,
                               reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint16_t*>(X), static_cast<uint32_t>(R), static_cast<uint32_t>(K),
      static_cast<uint64_t>(ldx), chunks, scale, Xq);
  return check_launch("quant_static launch");
}

fgfp8_status fgfp8_gemm_rowcol(const uint8_t* Xq, const float* sx, int x_per_tensor, const uint8_t* Wq,
                               const float* sw, int w_per_tensor, void* Y, int64_t M, int64_t N, int64_t K,
                               void* stream) {
  if (x_per_tensor != 0 && x_per_tensor != 1) return fail(FGFP8_ERR_INVALID_ARG, "x_per_tensor must be 0 or 1");
  if (w_per_tensor != 0 && w_per_tensor != 1) return fail(FGFP8_ERR_INVALID_ARG, "w_per_tensor must be 0 or 1");
  if (M < 0 || N < 0 || K < 0) return fail(FGFP8_ERR_INVALID_ARG, "negative size");
  if (K == 0 || K % 128 != 0) return fail(FGFP8_ERR_SHAPE, "K must be a positive multiple of 128");
  if (N == 0 || N % 128 != 0) return fail(FGFP8_ERR_SHAPE, "N must be a positive multiple of 128");
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
    return fail(FGFP8_ERR_SHAPE, "M, N and K must be < 2^31");
  if (M == 0) return ok();
  if (!Xq || !Wq || !sx || !sw || !Y) return fail(FGFP8_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(Xq, 16) || !aligned(Wq, 16) || !aligned(Y, 16))
    return fail(FGFP8_ERR_ALIGN, "Xq, Wq and Y must be 16-byte aligned");
  if (!aligned(sx, 4)) return fail(FGFP8_ERR_ALIGN, "sx must be 4-byte aligned");
  if (!aligned(sw, w_per_tensor ? 4 : 16))
    return fail(FGFP8_ERR_ALIGN, "per-channel sw must be 16-byte aligned (4 bytes for one per-tensor scale)");
  int dev;
  DeviceInfo info;
  fgfp8_status st = current_device(&dev, &info);
  if (st != FGFP8_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (N % 256 == 0)
    return launch_gemm_rowcol<256>(Xq, sx, x_per_tensor, Wq, sw, w_per_tensor, Y, M, N, K, s, dev, info.sm_count);
  return launch_gemm_rowcol<128>(Xq, sx, x_per_tensor, Wq, sw, w_per_tensor, Y, M, N, K, s, dev, info.sm_count);
}

fgfp8_status fgfp8_masked_gemm(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq, const void* Ws,
                               void* Y, const int32_t* counts, int32_t E, int64_t cap, int64_t N, int64_t K, int fmt,
                               void* stream) {
  return masked_impl(Xq, Xs, ld_s, Wq, Ws, Y, counts, E, cap, N, K, fmt, stream, false);
}

fgfp8_status fgfp8_quant_act_masked(const void* X, int64_t ldx, const int32_t* counts, int32_t E, int64_t cap,
                                    int64_t K, uint8_t* Xq, void* Xs, int64_t ld_s, int fmt, void* stream) {
  return quant_act_masked_impl(X, ldx, counts, E, cap, K, Xq, Xs, ld_s, fmt, stream, false);
}

fgfp8_status fgfp8_masked_linear(const void* X, int64_t ldx, uint8_t* Xq, void* Xs, int64_t ld_s, const uint8_t* Wq,
                                 const void* Ws, void* Y, const int32_t* counts, int32_t E, int64_t cap, int64_t N,
                                 int64_t K, int fmt, void* stream) {
  fgfp8_status st = quant_act_masked_impl(X, ldx, counts, E, cap, K, Xq, Xs, ld_s, fmt, stream, true);
  if (st != FGFP8_OK) return st;
  st = masked_impl(Xq, Xs, ld_s, Wq, Ws, Y, counts, E, cap, N, K, fmt, stream, true);
  if (st != FGFP8_OK) return st;
  st = quant_act_masked_impl(X, ldx, counts, E, cap, K, Xq, Xs, ld_s, fmt, stream, false);
  if (st != FGFP8_OK) return st;
  return masked_impl(Xq, Xs, ld_s, Wq, Ws, Y, counts, E, cap, N, K, fmt, stream, false);
}

fgfp8_status fgfp8_gemm_swiglu_quant(const uint8_t* Xq, const float* Xs, int64_t ld_s, const uint8_t* Wq_gu,
                                     const float* Ws_gu, uint8_t* Hq, float* Hs, int64_t ld_h, int64_t M, int64_t I,
                                     int64_t K, void* stream) {
  if (M < 0 || I < 0) return fail(FGFP8_ERR_INVALID_ARG, "negative size");
  if (I == 0 || I % 128 != 0) return fail(FGFP8_ERR_SHAPE, "I must be a positive multiple of 128");
  if (M == 0) return ok();
  fgfp8_status st = check_gemm_common(Xq, Xs, ld_s, Wq_gu, Ws_gu, Hq, M, 2 * I, K, FGFP8_SCALE_F32);
  if (st != FGFP8_OK) return st;
  st = check_act_scales(Hs, ld_h, M, FGFP8_SCALE_F32);
  if (st != FGFP8_OK) return st;
  int dev;
  DeviceInfo info;
  st = current_device(&dev, &info);
  if (st != FGFP8_OK) return st;
  return launch_gemm<256, 128, 0, false, true>(Xq, Xs, ld_s, Wq_gu, Ws_gu, nullptr, M, 2 * I, K, nullptr, 1, 2 * I,
                                               reinterpret_cast<cudaStream_t>(stream), dev, info.sm_count, 0, 0, Hq,
                                               Hs, ld_h);
}

fgfp8_status fgfp8_gather_cols(const void* parts, int64_t P, int64_t M, int64_t n, void* Y, void* stream) {
  if (P < 0 || M < 0 || n < 0) return fail(FGFP8_ERR_INVALID_ARG, "negative size");
  if (P == 0 || M == 0 || n == 0) return ok();
  if (n % 8 != 0) return fail(FGFP8_ERR_SHAPE, "n must be a multiple of 8 (16-byte rows)");
  if (P * M * (n / 8) >= (int64_t(1) << 32) || M >= (int64_t(1) << 31))
    return fail(FGFP8_ERR_SHAPE, "P * M * n / 8 must be < 2^32");
  if (!parts || !Y) return fail(FGFP8_ERR_INVALID_ARG, "parts or Y is NULL");
  if (!aligned(parts, 16) || !aligned(Y, 16)) return fail(FGFP8_ERR_ALIGN, "parts and Y must be 16-byte aligned");
  int dev;
  DeviceInfo info;
  fgfp8_status st = current_device(&dev, &info);
  if (st != FGFP8_OK) return st;
  const uint32_t total = static_cast<uint32_t>(P * M * (n / 8));
  fgfp8::gather_cols_kernel<<<grid_stride_blocks(reinterpret_cast<const void*>(fgfp8::gather_cols_kernel), total,
                                                 dev, info.sm_count),
                              256, 0,
                              reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint4*>(parts), total, fgfp8::FastDiv(static_cast<uint32_t>(n / 8)),
      fgfp8::FastDiv(static_cast<uint32_t>(M)), reinterpret_cast<uint4*>(Y));
  return check_launch("gather_cols launch");
}

fgfp8_status fgfp8_selftest_expired_wait(void* stream) {
  int dev;
  DeviceInfo info;
  fgfp8_status st = current_device(&dev, &info);
  if (st != FGFP8_OK) return st;
  fgfp8::selftest_expired_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
  return check_launch("self-test launch");
}

fgfp8_status fgfp8_selftest_gemm_timeout(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq,
                                         const void* Ws, void* Y, int64_t M, int64_t N, int64_t K, int fmt,
                                         int64_t withhold_kb, void* stream) {
  fgfp8_status st = check_gemm_common(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, fmt);
  if (st != FGFP8_OK) return st;
  if (M <= 64 || N % 256 != 0)
    return fail(FGFP8_ERR_SHAPE, "the self-test runs the persistent 128x256-tile GEMM: M > 64 and N % 256 == 0");
  if (withhold_kb < 0 || withhold_kb >= K / 128) return fail(FGFP8_ERR_INVALID_ARG, "withhold_kb must be in [0, K/128)");
  int dev;
  DeviceInfo info;
  st = current_device(&dev, &info);
  if (st != FGFP8_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int kb = static_cast<int>(withhold_kb);
  if (fmt == FGFP8_SCALE_UE8M0)
    return launch_gemm_mx<256, false>(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, nullptr, 1, N, s, dev, info.sm_count, 0, 0, kb);
  return launch_gemm<256, 128, 0, false>(Xq, Xs, ld_s, Wq, Ws, Y, M, N, K, nullptr, 1, N, s, dev, info.sm_count, 0, 0,
                                         nullptr, nullptr, 0, kb);
}

fgfp8_status fgfp8_check_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, fgfp8::g_device_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  if (v == fgfp8::kDevOk) return ok();
  const int zero = 0;
  e = cudaMemcpyToSymbol(fgfp8::g_device_status, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "clearing the device status word");
  switch (v) {
    case fgfp8::kDevTimeoutProducer:
      return fail(FGFP8_ERR_TIMEOUT, "a GEMM producer wait exceeded its limit");
    case fgfp8::kDevTimeoutMma:
      return fail(FGFP8_ERR_TIMEOUT, "a GEMM MMA wait exceeded its limit");
    case fgfp8::kDevTimeoutEpilogue:
      return fail(FGFP8_ERR_TIMEOUT, "a GEMM epilogue wait exceeded its limit");
    case fgfp8::kDevTimeoutSelftest:
      return fail(FGFP8_ERR_TIMEOUT, "the bounded-wait self-test's wait expired");
    case fgfp8::kDevBadGroupOffsets:
      return fail(FGFP8_ERR_DEVICE,
                  "group_offs is inconsistent (not a non-decreasing 0..M_total cover) or a masked count is outside "
                  "[0, cap]");
    case fgfp8::kDevBadIndex:
      return fail(FGFP8_ERR_DEVICE, "a debug-build index check failed (a tile, row, column or expert out of bounds)");
    case fgfp8::kDevBadScale:
      return fail(FGFP8_ERR_DEVICE, "the static quantizer's scale is not positive (<= 0 or NaN)");
    default:
      return fail(FGFP8_ERR_DEVICE, "unknown device status " + std::to_string(v));
  }
}

}  // extern "C"
