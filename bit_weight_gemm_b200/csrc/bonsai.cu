// bonsai.cu - the C ABI declared in include/bonsai.h: argument checks, tensor
// maps, kernel selection (the planner) and launches, the batched small-M
// launches, and the host-buffer pipeline.  All arithmetic runs in the kernels
// of pack_dequant.cuh, gemm_tc.cuh, gemm_persistent.cuh, gemm_small.cuh and
// gemm_batch.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "bonsai.h"
#include "gemm_batch.cuh"
#include "gemm_persistent.cuh"
#include "gemm_small.cuh"
#include "gemm_tc.cuh"
#include "pack_dequant.cuh"

namespace bonsai {
namespace {

constexpr uint64_t kDefaultWaitLimitNs = 4000000000ull;  // 4 s: far above any launch's run time

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_mode(int mode) {
  return mode == BONSAI_BINARY || mode == BONSAI_TERNARY_INT2 || mode == BONSAI_TERNARY_B3;
}

// Packed words of one row: K/32 (binary), K/16 (INT2), 28 per 4 groups (base-3).
int64_t row_words(int64_t K, int mode) {
  if (mode == BONSAI_TERNARY_B3) return (K / kGroup + kB3BlockGroups - 1) / kB3BlockGroups * (kB3BlockBytes / 4);
  if (mode == kModeHqq4) return K / 8;
  return K / (mode == BONSAI_BINARY ? 32 : 16);
}

// Tensor map of the packed weights: [N rows][row_words] uint32, copied in
// boxes of one word stage (128 bytes of a row with 128-byte swizzling, or one
// 112-byte base-3 block unswizzled) x 128 rows.
bool make_weight_map(CUtensorMap* map, const void* packed, int N, int K, int mode);

// K multiple of 128, sizes non-negative and small enough for 32-bit tile
// coordinates and 64-bit byte counts.
int check_shape(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K < 0) return BONSAI_ERR_SHAPE;
  if (K % kGroup != 0) return BONSAI_ERR_SHAPE;
  const int64_t lim = int64_t(1) << 31;
  if (M >= lim || N >= lim || K >= lim) return BONSAI_ERR_SHAPE;
  if (N > 0 && K > (int64_t(1) << 62) / N) return BONSAI_ERR_SHAPE;
  if (M > 0 && K > (int64_t(1) << 62) / M) return BONSAI_ERR_SHAPE;
  if (M > 0 && N > (int64_t(1) << 62) / M) return BONSAI_ERR_SHAPE;
  return BONSAI_OK;
}

// The kernels use tcgen05 and TMA: the device must be sm_100.
int check_device() {
  static std::mutex mu;
  static int cached[64];  // 0 unknown, 1 ok, 2 wrong arch
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BONSAI_ERR_CUDA;
  if (dev < 0 || dev >= 64) return BONSAI_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return BONSAI_ERR_CUDA;
    cached[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return cached[dev] == 1 ? BONSAI_OK : BONSAI_ERR_ARCH;
}

int launch_status() {
  return cudaGetLastError() == cudaSuccess ? BONSAI_OK : BONSAI_ERR_CUDA;
}

int grid_for(int64_t work_items, int threads) {
  int64_t blocks = (work_items + threads - 1) / threads;
  const int64_t cap = 148 * 16;
  if (blocks > cap) blocks = cap;
  return blocks < 1 ? 1 : static_cast<int>(blocks);
}

// ----------------------------------------------------------- tensor maps --
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
  });
  return fn;
}

// Encoded tensor maps are kept in a small cache: encoding costs
// microseconds of host time per call, comparable to a small-M launch.  A map
// holds only an address, sizes and a box shape, so a hit is always valid.
struct MapKey {
  const void* base;
  uint64_t inner, rows;
  uint32_t box_inner, box_rows;
  int dtype, swizzle, device;
  bool operator==(const MapKey& o) const {
    return base == o.base && inner == o.inner && rows == o.rows && box_inner == o.box_inner &&
           box_rows == o.box_rows && dtype == o.dtype && swizzle == o.swizzle && device == o.device;
  }
};

constexpr int kMapCacheSize = 256;
struct MapCache {
  std::mutex mu;
  MapKey keys[kMapCacheSize];
  CUtensorMap maps[kMapCacheSize];
  bool used[kMapCacheSize] = {};
  int next = 0;
};

MapCache& map_cache() {
  static MapCache cache;
  return cache;
}

// Row-major 2-D tensor [rows, inner] of `elem` bytes per element, copied in
// boxes of box_rows x box_inner.
bool make_map(CUtensorMap* map, CUtensorMapDataType dtype, int elem, const void* base, uint64_t inner,
              uint64_t rows, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  int device = 0;
  cudaGetDevice(&device);
  const MapKey key{base, inner, rows, box_inner, box_rows, static_cast<int>(dtype), static_cast<int>(swizzle), device};
  MapCache& cache = map_cache();
  uint64_t h = reinterpret_cast<uintptr_t>(base) * 0x9E3779B97F4A7C15ull;
  h ^= (inner * 0xC2B2AE3D27D4EB4Full) ^ (rows * 0x165667B19E3779F9ull) ^
       (static_cast<uint64_t>(box_inner) << 40) ^ (static_cast<uint64_t>(box_rows) << 20) ^
       (static_cast<uint64_t>(dtype) << 8) ^ static_cast<uint64_t>(swizzle) ^ (static_cast<uint64_t>(device) << 56);
  const int home = static_cast<int>((h >> 32) % kMapCacheSize);
  constexpr int kProbe = 8;
  {
    std::lock_guard<std::mutex> lock(cache.mu);
    for (int i = 0; i < kProbe; ++i) {
      const int slot = (home + i) % kMapCacheSize;
      if (cache.used[slot] && cache.keys[slot] == key) {
        *map = cache.maps[slot];
        return true;
      }
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * static_cast<uint64_t>(elem)};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  if (fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  std::lock_guard<std::mutex> lock(cache.mu);
  int slot = -1;
  for (int i = 0; i < kProbe && slot < 0; ++i)
    if (!cache.used[(home + i) % kMapCacheSize]) slot = (home + i) % kMapCacheSize;
  if (slot < 0) {  // all probe slots taken: replace them in turn
    slot = (home + cache.next) % kMapCacheSize;
    cache.next = (cache.next + 1) % kProbe;
  }
  cache.keys[slot] = key;
  cache.maps[slot] = *map;
  cache.used[slot] = true;
  return true;
}

bool make_weight_map(CUtensorMap* map, const void* packed, int N, int K, int mode) {
  const bool b3 = mode == BONSAI_TERNARY_B3;
  return make_map(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, packed, static_cast<uint64_t>(row_words(K, mode)), N,
                  b3 ? kB3BlockBytes / 4 : 32, 128, b3 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B);
}

// ------------------------------------------------------------------ GEMM --
int sm_count() {
  static int count[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (count[dev] == 0) {
    int c = 0;
    cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev);
    count[dev] = c > 0 ? c : 148;
  }
  return count[dev];
}

// Raises a kernel's dynamic shared-memory limit to what it uses, once per
// device (the attribute is per device, and the occupancy queries below
// depend on it).
template <auto KERNEL>
int smem_opt_in(int bytes) {
  static std::mutex mu;
  static bool done[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BONSAI_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev]) {
    if (cudaFuncSetAttribute(KERNEL, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) {
      cudaGetLastError();
      return BONSAI_ERR_CUDA;
    }
    done[dev] = true;
  }
  return BONSAI_OK;
}

// Clusters of `ksplit` CTAs that can be resident at once on the current
// device (0 if unknown).
template <int MODE, int BLOCK_T>
int resident_clusters(int ksplit) {
  using T = GemmTile<MODE, BLOCK_T>;
  static std::mutex mu;
  static int cache[64][9] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (ksplit < 1 || ksplit > 8) return 0;
  if (smem_opt_in<lowbit_gemm_kernel<MODE, BLOCK_T>>(T::kSmemBytes) != BONSAI_OK) return 0;
  if (cache[dev][ksplit] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, ksplit);
    cfg.blockDim = dim3(T::kThreads);
    cfg.dynamicSmemBytes = T::kSmemBytes;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 1;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = ksplit;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, lowbit_gemm_kernel<MODE, BLOCK_T>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = -1;
    }
    cache[dev][ksplit] = n;
  }
  return cache[dev][ksplit] > 0 ? cache[dev][ksplit] : 0;
}

template <int MODE, int BLOCK_T>
int launch_gemm(const uint16_t* A, const void* packed, const uint16_t* scales, const uint16_t* zeros, int M, int N,
                int K, int ksplit,
                uint16_t* out, cudaStream_t stream) {
  using T = GemmTile<MODE, BLOCK_T>;
  auto kernel = lowbit_gemm_kernel<MODE, BLOCK_T>;
  if (smem_opt_in<lowbit_gemm_kernel<MODE, BLOCK_T>>(T::kSmemBytes) != BONSAI_OK) return BONSAI_ERR_CUDA;

  CUtensorMap map_act, map_w, map_out;
  // Boxes of one MMA's tokens (half of a two-half tile).
  if (!make_map(&map_act, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, A, K, M, 64, T::kMmaN, CU_TENSOR_MAP_SWIZZLE_128B))
    return BONSAI_ERR_CUDA;
  if (!make_weight_map(&map_w, packed, N, K, MODE)) return BONSAI_ERR_CUDA;
  const bool tma_store = (N % 8) == 0;
  if (tma_store) {
    if (!make_map(&map_out, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, out, N, M, T::kRows, T::kMmaN,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
      return BONSAI_ERR_CUDA;
  } else {
    map_out = map_act;  // unused: rows of N halves are not 16-byte multiples, the kernel stores directly
  }
  const int groups = K / kGroup;
  const int tiles_n = (N + T::kRows - 1) / T::kRows, tiles_m = (M + BLOCK_T - 1) / BLOCK_T;
  if (ksplit < 1 || ksplit > 8 || ksplit > groups || (T::kHalves > 1 && ksplit > 1)) return BONSAI_ERR_SHAPE;
  // Scale tile by TMA: rows of the scale matrix must be 16-byte multiples
  // (groups % 8 == 0); the box covers a CTA's groups from an 8-aligned start.
  CUtensorMap map_s = map_act;  // placeholder when unused
  int scale_box = 0;
  if (T::kScaleBytes > 0 && groups % 8 == 0) {
    const int per_cta = (groups + ksplit - 1) / ksplit;
    int box = ((per_cta + 7 + 7) / 8) * 8;
    if (box > groups) box = groups;
    if (box <= 256 && box * T::kRows * 2 <= T::kScaleBytes) {
      if (!make_map(&map_s, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, scales, groups, N, box, T::kRows,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
        return BONSAI_ERR_CUDA;
      scale_box = box;
    }
  }

  GemmArgs args;
  args.scales = scales;
  args.zeros = zeros;
  args.out = out;
  args.M = M;
  args.N = N;
  args.K = K;
  args.ksplit = ksplit;
  args.tma_store = tma_store ? 1 : 0;
  args.scale_box = scale_box;
  args.wait_limit_ns = kDefaultWaitLimitNs;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles_n, tiles_m, ksplit);
  cfg.blockDim = dim3(T::kThreads);
  cfg.dynamicSmemBytes = T::kSmemBytes;
  cfg.stream = stream;
  // Programmatic dependent launch: the kernel's prologue may overlap the
  // previous kernel in the stream; it waits for that kernel before touching
  // global memory (griddepcontrol.wait), so stream order is preserved.
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  if (ksplit > 1) {
    attrs[1].id = cudaLaunchAttributeClusterDimension;
    attrs[1].val.clusterDim.x = 1;
    attrs[1].val.clusterDim.y = 1;
    attrs[1].val.clusterDim.z = ksplit;
    cfg.numAttrs = 2;
  }
  if (cudaLaunchKernelEx(&cfg, kernel, map_act, map_w, map_out, map_s, args) != cudaSuccess) return BONSAI_ERR_CUDA;
  return launch_status();
}

// Persistent form (gemm_persistent.cuh): more BLOCK_T-token tiles than SMs
// and whole word stages per tile.
template <int MODE, int BLOCK_T>
bool use_persistent(int M, int N, int K) {
  using T = PersistTile<MODE, BLOCK_T>;
  // Whole word stages per tile, and a group count per tile that is a
  // multiple of 4 (each converter warp keeps its TMEM stage across tiles).
  const int per_stage = T::kWGroups > 4 ? T::kWGroups : 4;
  if (M <= 128 || K % (kGroup * per_stage) != 0) return false;
  const int64_t tiles = static_cast<int64_t>((N + T::kRows - 1) / T::kRows) * ((M + T::kBlockT - 1) / T::kBlockT);
  return tiles > sm_count();
}

template <int MODE, int BLOCK_T>
int launch_gemm_persistent(const uint16_t* A, const void* packed, const uint16_t* scales, const uint16_t* zeros, int M,
                           int N, int K,
                           uint16_t* out, cudaStream_t stream) {
  using T = PersistTile<MODE, BLOCK_T>;
  auto kernel = lowbit_gemm_persistent_kernel<MODE, BLOCK_T>;
  if (smem_opt_in<lowbit_gemm_persistent_kernel<MODE, BLOCK_T>>(T::kSmemBytes) != BONSAI_OK) return BONSAI_ERR_CUDA;
  CUtensorMap map_act, map_w;
  if (!make_map(&map_act, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, A, K, M, 64, T::kBlockT, CU_TENSOR_MAP_SWIZZLE_128B))
    return BONSAI_ERR_CUDA;
  if (!make_weight_map(&map_w, packed, N, K, MODE)) return BONSAI_ERR_CUDA;
  PersistArgs args;
  args.scales = scales;
  args.zeros = zeros;
  args.out = out;
  args.M = M;
  args.N = N;
  args.K = K;
  args.tiles_n = (N + T::kRows - 1) / T::kRows;
  args.tiles = args.tiles_n * ((M + T::kBlockT - 1) / T::kBlockT);
  args.wait_limit_ns = kDefaultWaitLimitNs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(args.tiles < sm_count() ? args.tiles : sm_count());
  cfg.blockDim = dim3(T::kThreads);
  cfg.dynamicSmemBytes = T::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, map_act, map_w, args) != cudaSuccess) return BONSAI_ERR_CUDA;
  return launch_status();
}

// Clusters of `ksplit` small-M CTAs that can be resident at once on the
// current device (the kernel takes one SM per CTA; clusters must fit within
// a GPC, so fewer than SMs / ksplit may fit).  0 if unknown.
template <int MODE>
int small_resident_clusters(int ksplit) {
  using T = SmallTile<MODE>;
  static std::mutex mu;
  static int cache[64][9] = {};
  int dev = 0;
  if (ksplit < 1 || ksplit > T::kMaxSplit) return 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (smem_opt_in<lowbit_gemm_small_kernel<MODE>>(T::kSmemBytes) != BONSAI_OK) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev][ksplit] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, ksplit);
    cfg.blockDim = dim3(T::kThreads);
    cfg.dynamicSmemBytes = T::kSmemBytes;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 1;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = ksplit;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, lowbit_gemm_small_kernel<MODE>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = -1;
    }
    cache[dev][ksplit] = n;
  }
  return cache[dev][ksplit] > 0 ? cache[dev][ksplit] : 0;
}

// Small-M form (gemm_small.cuh): the K split for up to 16 tokens, 0 when the
// form does not apply.  Every CTA's range must fit its shared memory
// (kMaxGroups groups).  A kernel with tensor memory takes a whole SM, so a
// launch's CTAs start as the previous launch's leave; a launch on at most
// half the SMs lets the next one start on the other half.  So: no split when
// the tiles fit half the SMs and a tile's groups fit one CTA (measured on the
// fused QKV layer, 9216x3072: 7.2 us per launch on 72 SMs against 8.2 split
// two ways on 144); else the largest split whose tiles x ksplit CTAs are all
// resident at once (one wave), else the smallest feasible one.
template <int MODE>
int small_ksplit(int M, int N, int K) {
  using T = SmallTile<MODE>;
  if constexpr (MODE == kModeHqq4) return 0;  // (its weights are formed with the scale, in the other kernels)
  if (M > T::kBlockT) return 0;
  const int groups = K / kGroup;
  const int tiles = (N + T::kRows - 1) / T::kRows;
  if (2 * tiles <= sm_count() && groups <= T::kMaxGroups) return 1;
  int best = 0;
  bool best_fits = false;
  for (int ks = 1; ks <= T::kMaxSplit && ks * T::kGroupAlign <= (groups > T::kGroupAlign ? groups : T::kGroupAlign);
       ++ks) {
    int widest = 0;
    for (int z = 0; z < ks; ++z) {
      const int w = split_bound<T::kGroupAlign>(z + 1, groups, ks) - split_bound<T::kGroupAlign>(z, groups, ks);
      if (w < 1) widest = 1 << 30;  // an empty range
      widest = w > widest ? w : widest;
    }
    if (widest > T::kMaxGroups) continue;
    const int resident = ks == 1 ? sm_count() : small_resident_clusters<MODE>(ks);
    if (tiles <= resident) {  // one wave: the largest such split wins
      best = ks;
      best_fits = true;
    } else if (!best_fits && best == 0) {  // none in one wave (yet): the smallest feasible split
      best = ks;
    }
  }
  return best;
}

template <int MODE>
int launch_gemm_small(const uint16_t* A, const void* packed, const uint16_t* scales, int M, int N, int K, int ksplit,
                      uint16_t* out, cudaStream_t stream) {
  using T = SmallTile<MODE>;
  auto kernel = lowbit_gemm_small_kernel<MODE>;
  if (smem_opt_in<lowbit_gemm_small_kernel<MODE>>(T::kSmemBytes) != BONSAI_OK) return BONSAI_ERR_CUDA;
  CUtensorMap map_act, map_w;
  if (!make_map(&map_act, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, A, K, M, 64, T::kBlockT, CU_TENSOR_MAP_SWIZZLE_128B))
    return BONSAI_ERR_CUDA;
  if (!make_weight_map(&map_w, packed, N, K, MODE)) return BONSAI_ERR_CUDA;
  SmallArgs args;
  args.scales = scales;
  args.out = out;
  args.M = M;
  args.N = N;
  args.K = K;
  args.ksplit = ksplit;
  args.wait_limit_ns = kDefaultWaitLimitNs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((N + T::kRows - 1) / T::kRows, 1, ksplit);
  cfg.blockDim = dim3(T::kThreads);
  cfg.dynamicSmemBytes = T::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  attrs[1].id = cudaLaunchAttributeClusterDimension;
  attrs[1].val.clusterDim.x = 1;
  attrs[1].val.clusterDim.y = 1;
  attrs[1].val.clusterDim.z = ksplit;
  cfg.attrs = attrs;
  cfg.numAttrs = ksplit > 1 ? 2 : 1;
  if (cudaLaunchKernelEx(&cfg, kernel, map_act, map_w, args) != cudaSuccess) return BONSAI_ERR_CUDA;
  return launch_status();
}

// ------------------------------------------------- batched small M --
// One persistent launch over `count` problems of up to 16 tokens
// (gemm_batch.cuh): their 128-row tiles form one unit list, cut into one
// contiguous range per CTA with nearly equal numbers of K groups.
template <int MODE>
int launch_gemm_batch(const bonsai_gemm_problem* const* probs, int count, cudaStream_t stream) {
  using T = BatchTile<MODE>;
  if (count < 1 || count > kBatchMaxLayers) return BONSAI_ERR_INVALID_ARG;
  if (smem_opt_in<lowbit_gemm_batch_kernel<MODE>>(T::kSmemBytes) != BONSAI_OK) return BONSAI_ERR_CUDA;
  static thread_local BatchParams params;  // 28 KB: kept off the stack
  int units = 0;
  int64_t total = 0;  // K groups of all units
  for (int i = 0; i < count; ++i) {
    const bonsai_gemm_problem& q = *probs[i];
    const int M = static_cast<int>(q.M), N = static_cast<int>(q.N), K = static_cast<int>(q.K);
    if (!make_map(&params.act[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, q.A, K, M, 64, T::kBlockT,
                  CU_TENSOR_MAP_SWIZZLE_128B))
      return BONSAI_ERR_CUDA;
    // Binary word stages are 64-byte rows (four groups), the others as in the other kernels.
    if (MODE == BONSAI_BINARY ? !make_map(&params.w[i], CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, q.packed,
                                          static_cast<uint64_t>(row_words(K, MODE)), N, T::kWRowBytes / 4, 128,
                                          CU_TENSOR_MAP_SWIZZLE_64B)
                              : !make_weight_map(&params.w[i], q.packed, N, K, MODE))
      return BONSAI_ERR_CUDA;
    params.layer[i] = BatchLayer{q.scales, q.out, M, N, K, units};
    const int tiles = (N + T::kRows - 1) / T::kRows;
    units += tiles;
    total += static_cast<int64_t>(tiles) * (K / kGroup);
  }
  params.count = count;
  params.units = units;
  params.wait_limit_ns = kDefaultWaitLimitNs;
  int ctas = sm_count();
  if (ctas > kBatchMaxCtas) ctas = kBatchMaxCtas;
  if (ctas > units) ctas = units;
  // Boundary c: units go to the earlier CTA while at least half of a unit's
  // groups lie before c * total / ctas.
  params.cta_unit0[0] = 0;
  int u = 0, li = 0;
  int64_t before = 0;  // groups of units 0 .. u-1
  for (int c = 1; c < ctas; ++c) {
    const int64_t target = total * c / ctas;
    while (u < units) {
      while (li + 1 < count && params.layer[li + 1].unit0 <= u) ++li;
      const int g = params.layer[li].K / kGroup;
      if (2 * (before + g) > 2 * target + g) break;
      before += g;
      ++u;
    }
    params.cta_unit0[c] = u;
  }
  params.cta_unit0[ctas] = units;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(T::kThreads);
  cfg.dynamicSmemBytes = T::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, lowbit_gemm_batch_kernel<MODE>, params) != cudaSuccess) return BONSAI_ERR_CUDA;
  return launch_status();
}

// ------------------------------------------------------------- planning --
// Launch costs in microseconds, measured on a B200 with an M sweep of single
// launches (16..4608 tokens on the MMDiT layer shapes, clocks under the power
// cap of a long run): per 128-wide K group of one CTA, per wave of one-tile
// CTAs (start, accumulator read-out, store, exit), and per split-K cluster
// reduction.  The persistent kernel pays about 1 us per tile boundary
// instead of a wave's start and end.
struct TileCost {
  double group, wave, reduce;
};

constexpr TileCost tile_cost(int block_t) {
  return block_t <= 32    ? TileCost{0.31, 1.5, 1.0}
         : block_t == 64  ? TileCost{0.31, 2.0, 1.5}
         : block_t == 128 ? TileCost{0.50, 2.5, 2.0}
         : block_t == 176 ? TileCost{0.59, 2.7, 2.75}  // interpolated between 128 and 192
         : block_t == 192 ? TileCost{0.62, 2.75, 3.0}
         : block_t == 256 ? TileCost{0.75, 3.0, 4.0}
                          : TileCost{1.12, 3.5, 0.0};  // 352 (two halves; not split), measured at 2048 tokens
}
constexpr double kLaunchCost = 2.5;
constexpr double kPersistentBoundary = 1.0;

struct Plan {
  int block_t = 0, ksplit = 0, ctas = 0, tiles = 0;
  bool persistent = false;
  bool small = false;  // the bandwidth-bound form of gemm_small.cuh
  double cost = 1e30;
};

// Every split of K (1..8, a cluster of that many CTAs per tile) for
// BLOCK_T-token tiles: waves x (groups per CTA + per-wave costs).
template <int MODE, int BLOCK_T>
void consider(int M, int N, int K, Plan* best) {
  const int groups = K / kGroup;
  const int tiles = ((N + 127) / 128) * ((M + BLOCK_T - 1) / BLOCK_T);
  const TileCost c = tile_cost(BLOCK_T);
  const int sms = sm_count();
  // Base-3 ranges start on 4-group blocks: at most groups / 4 of them.
  const int max_ks = MODE == BONSAI_TERNARY_B3 ? (groups / kB3BlockGroups > 1 ? groups / kB3BlockGroups : 1) : groups;
  for (int ks = 1; ks <= 8 && ks <= max_ks; ++ks) {
    if constexpr (BLOCK_T > 256) {
      if (ks > 1) break;  // two-half tiles are not split
    }
    const int per_wave = ks == 1 ? sms : resident_clusters<MODE, BLOCK_T>(ks);
    if (per_wave <= 0) continue;
    const int waves = (tiles + per_wave - 1) / per_wave;
    // 176-token tiles only where they fit one wave (1024 tokens on the N=3072
    // layers); with more tiles the persistent 192- or 256-token forms win
    // (measured at 2048 tokens, N=3072, K=9216: 1068 TFLOP/s against ~1300).
    if (BLOCK_T == 176 && waves > 1) continue;
    // 352-token tiles (two 176-token halves) likewise, and unsplit: at 2048
    // tokens the N=3072 layers make 144 of them, one wave, where 192-token
    // tiles need 1.8 waves of the persistent kernel; on ragged mid-M shapes
    // just past one wave of 256-token tiles they save a second wave.
    if (BLOCK_T == 352 && waves > 1) continue;
    bool persistent = false;
    if constexpr (BLOCK_T >= 192 && BLOCK_T <= 256) persistent = ks == 1 && use_persistent<MODE, BLOCK_T>(M, N, K);
    const double per_wave_cost = ((groups + ks - 1) / ks) * c.group + (persistent ? kPersistentBoundary : c.wave) +
                                 (ks > 1 ? c.reduce : 0.0);
    const double cost = kLaunchCost + waves * per_wave_cost;
    if (cost < best->cost) {
      best->block_t = BLOCK_T;
      best->ksplit = ks;
      best->tiles = tiles;
      best->persistent = persistent;
      best->ctas = persistent ? (tiles < sms ? tiles : sms) : tiles * ks;
      best->cost = cost;
    }
  }
}

// Tokens per tile: the smallest MMA N that covers M up to 128; above that
// 128-, 176-, 192- or 256-token tiles, whichever the cost model prefers (256
// amortises each converted weight over the most tokens; the narrower ones
// waste fewer rows and fill more SMs at mid M: M=1024 with N=3072 makes 96
// 256-token tiles for 148 SMs but 144 of 192 or 176 tokens, and 176-token
// tiles leave 32 empty token rows where 192-token ones leave 128).
template <int MODE>
Plan plan_gemm(int M, int N, int K) {
  Plan best;
  if (const int ks = small_ksplit<MODE>(M, N, K)) {
    best.block_t = SmallTile<MODE>::kBlockT;
    best.ksplit = ks;
    best.tiles = (N + 127) / 128;
    best.ctas = best.tiles * ks;
    best.small = true;
    return best;
  }
  if (M <= 16) {
    consider<MODE, 16>(M, N, K, &best);
  } else if (M <= 32) {
    consider<MODE, 32>(M, N, K, &best);
  } else if (M <= 64) {
    consider<MODE, 64>(M, N, K, &best);
  } else if (M <= 128) {
    consider<MODE, 128>(M, N, K, &best);
  } else {
    consider<MODE, 128>(M, N, K, &best);
    consider<MODE, 176>(M, N, K, &best);
    consider<MODE, 192>(M, N, K, &best);
    consider<MODE, 256>(M, N, K, &best);
    // Ternary weights only: binary ones measured 6% slower in 352-token tiles
    // than in the persistent kernel's 192-token tiles at 2048 tokens.
    if constexpr (MODE == BONSAI_TERNARY_INT2 || MODE == BONSAI_TERNARY_B3) consider<MODE, 352>(M, N, K, &best);
  }
  return best;
}

template <int MODE>
int dispatch_gemm(const uint16_t* A, const void* packed, const uint16_t* scales, const uint16_t* zeros, int M, int N,
                  int K,
                  uint16_t* out, cudaStream_t stream) {
  const Plan p = plan_gemm<MODE>(M, N, K);
  if constexpr (MODE != kModeHqq4)
    if (p.small) return launch_gemm_small<MODE>(A, packed, scales, M, N, K, p.ksplit, out, stream);
  if (p.persistent)
    return p.block_t == 192 ? launch_gemm_persistent<MODE, 192>(A, packed, scales, zeros, M, N, K, out, stream)
                            : launch_gemm_persistent<MODE, 256>(A, packed, scales, zeros, M, N, K, out, stream);
  switch (p.block_t) {
    case 16: return launch_gemm<MODE, 16>(A, packed, scales, zeros, M, N, K, p.ksplit, out, stream);
    case 32: return launch_gemm<MODE, 32>(A, packed, scales, zeros, M, N, K, p.ksplit, out, stream);
    case 64: return launch_gemm<MODE, 64>(A, packed, scales, zeros, M, N, K, p.ksplit, out, stream);
    case 128: return launch_gemm<MODE, 128>(A, packed, scales, zeros, M, N, K, p.ksplit, out, stream);
    case 176: return launch_gemm<MODE, 176>(A, packed, scales, zeros, M, N, K, p.ksplit, out, stream);
    case 192: return launch_gemm<MODE, 192>(A, packed, scales, zeros, M, N, K, p.ksplit, out, stream);
    case 256: return launch_gemm<MODE, 256>(A, packed, scales, zeros, M, N, K, p.ksplit, out, stream);
    case 352:
      if constexpr (MODE == BONSAI_TERNARY_INT2 || MODE == BONSAI_TERNARY_B3)
        return launch_gemm<MODE, 352>(A, packed, scales, zeros, M, N, K, p.ksplit, out, stream);
      return BONSAI_ERR_CUDA;
    default: return BONSAI_ERR_CUDA;  // no plan: the occupancy queries failed
  }
}

// ------------------------------------------------ host-buffer pipeline --
// Three streams per device (copies in, GEMMs, copies out) and the events that
// chain a call's chunks, created on first use and kept for the process.
constexpr int kMaxChunks = 16;

struct HostPipeline {
  bool ready = false;
  cudaStream_t in = nullptr, comp = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t copied[kMaxChunks] = {}, computed[kMaxChunks] = {};
};

std::mutex g_pipe_mu;
HostPipeline g_pipes[64];

int pipeline_for_device(HostPipeline** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BONSAI_ERR_CUDA;
  HostPipeline& p = g_pipes[dev];
  if (!p.ready) {
    const unsigned ev = cudaEventDisableTiming;
    bool ok = cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p.comp, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&p.start, ev) == cudaSuccess &&
              cudaEventCreateWithFlags(&p.done, ev) == cudaSuccess;
    for (int c = 0; ok && c < kMaxChunks; ++c)
      ok = cudaEventCreateWithFlags(&p.copied[c], ev) == cudaSuccess &&
           cudaEventCreateWithFlags(&p.computed[c], ev) == cudaSuccess;
    if (!ok) {  // release what was created; the next call starts over
      cudaGetLastError();
      for (cudaStream_t* st : {&p.in, &p.comp, &p.out})
        if (*st) cudaStreamDestroy(*st), *st = nullptr;
      for (cudaEvent_t* ev : {&p.start, &p.done})
        if (*ev) cudaEventDestroy(*ev), *ev = nullptr;
      for (int c = 0; c < kMaxChunks; ++c) {
        if (p.copied[c]) cudaEventDestroy(p.copied[c]), p.copied[c] = nullptr;
        if (p.computed[c]) cudaEventDestroy(p.computed[c]), p.computed[c] = nullptr;
      }
      return BONSAI_ERR_CUDA;
    }
    p.ready = true;
  }
  *out = &p;
  return BONSAI_OK;
}

// Rows per chunk: a multiple of 256 (whole 256-token tiles), about a quarter
// of M so that copies in, GEMMs and copies out of neighbouring chunks overlap,
// and at most kMaxChunks chunks.
int64_t chunk_rows(int64_t M) {
  const int64_t quarter = (M + 3) / 4;
  const int64_t cap = (M + kMaxChunks - 1) / kMaxChunks;
  int64_t rows = quarter > cap ? quarter : cap;
  rows = (rows + 255) / 256 * 256;
  return rows < 256 ? 256 : rows;
}

template <int MODE>
int gemm_host_pipelined(const uint16_t* A_host, const void* packed, const uint16_t* scales, int64_t M, int64_t N,
                        int64_t K, uint16_t* out_host, uint16_t* A_dev, uint16_t* out_dev, cudaStream_t user) {
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipeline* p = nullptr;
  int rc = pipeline_for_device(&p);
  if (rc != BONSAI_OK) return rc;
  const int64_t rows = chunk_rows(M);
  const int chunks = static_cast<int>((M + rows - 1) / rows);
  // Fork: all three streams start after the work already on the caller's stream.
  if (cudaEventRecord(p->start, user) != cudaSuccess || cudaStreamWaitEvent(p->in, p->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(p->comp, p->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(p->out, p->start, 0) != cudaSuccess)
    return BONSAI_ERR_CUDA;
  for (int c = 0; c < chunks; ++c) {
    const int64_t r0 = c * rows, m = (M - r0) < rows ? (M - r0) : rows;
    const size_t a_off = static_cast<size_t>(r0) * K, o_off = static_cast<size_t>(r0) * N;
    if (cudaMemcpyAsync(A_dev + a_off, A_host + a_off, static_cast<size_t>(m) * K * 2, cudaMemcpyHostToDevice,
                        p->in) != cudaSuccess ||
        cudaEventRecord(p->copied[c], p->in) != cudaSuccess || cudaStreamWaitEvent(p->comp, p->copied[c], 0) != cudaSuccess)
      return BONSAI_ERR_CUDA;
    rc = dispatch_gemm<MODE>(A_dev + a_off, packed, scales, nullptr, static_cast<int>(m), static_cast<int>(N),
                             static_cast<int>(K), out_dev + o_off, p->comp);
    if (rc != BONSAI_OK) return rc;
    if (cudaEventRecord(p->computed[c], p->comp) != cudaSuccess ||
        cudaStreamWaitEvent(p->out, p->computed[c], 0) != cudaSuccess ||
        cudaMemcpyAsync(out_host + o_off, out_dev + o_off, static_cast<size_t>(m) * N * 2, cudaMemcpyDeviceToHost,
                        p->out) != cudaSuccess)
      return BONSAI_ERR_CUDA;
  }
  // Join: the caller's stream continues after the last copy out (which
  // follows every chunk's GEMM and copy in).
  if (cudaEventRecord(p->done, p->out) != cudaSuccess || cudaStreamWaitEvent(user, p->done, 0) != cudaSuccess)
    return BONSAI_ERR_CUDA;
  return BONSAI_OK;
}

}  // namespace
}  // namespace bonsai

using namespace bonsai;

extern "C" {

size_t bonsai_packed_bytes(int64_t N, int64_t K, int mode) {
  if (!valid_mode(mode) || check_shape(0, N, K) != BONSAI_OK) return 0;
  return static_cast<size_t>(N) * static_cast<size_t>(row_words(K, mode)) * 4;
}

size_t bonsai_scale_bytes(int64_t N, int64_t K) {
  if (check_shape(0, N, K) != BONSAI_OK) return 0;
  return static_cast<size_t>(N) * static_cast<size_t>(K / kGroup) * 2;
}

int bonsai_pack(const int8_t* codes, int64_t N, int64_t K, int mode, void* packed, void* stream) {
  if (!valid_mode(mode)) return BONSAI_ERR_INVALID_ARG;
  int rc = check_shape(0, N, K);
  if (rc != BONSAI_OK) return rc;
  if (N == 0 || K == 0) return BONSAI_OK;
  if (!codes || !packed) return BONSAI_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(packed)) return BONSAI_ERR_ALIGN;
  if ((rc = check_device()) != BONSAI_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned zero = 0;
  if (cudaMemcpyToSymbolAsync(g_pack_bad_code, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return BONSAI_ERR_CUDA;
  if (mode == BONSAI_TERNARY_B3) {
    const int64_t slots = N * (row_words(K, mode) / (kB3BlockBytes / 4)) * kB3BlockGroups;
    if ((reinterpret_cast<uintptr_t>(codes) & 31u) == 0)
      pack_b3_kernel<true><<<grid_for(slots, 256), 256, 0, st>>>(codes, static_cast<uint32_t*>(packed), N, K);
    else
      pack_b3_kernel<false><<<grid_for(slots, 256), 256, 0, st>>>(codes, static_cast<uint32_t*>(packed), N, K);
  } else {
    const int64_t words = N * K / (mode == BONSAI_BINARY ? 32 : 16);
    const int grid = grid_for(words / (mode == BONSAI_BINARY ? 4 : 8), 256);  // 4-word steps: one binary, two ternary
    if (mode == BONSAI_BINARY && (reinterpret_cast<uintptr_t>(codes) & 31u) == 0)
      pack_kernel<BONSAI_BINARY, true><<<grid, 256, 0, st>>>(codes, static_cast<uint32_t*>(packed), words);
    else if (mode == BONSAI_BINARY)
      pack_kernel<BONSAI_BINARY><<<grid, 256, 0, st>>>(codes, static_cast<uint32_t*>(packed), words);
    else
      pack_kernel<BONSAI_TERNARY_INT2><<<grid, 256, 0, st>>>(codes, static_cast<uint32_t*>(packed), words);
  }
  if ((rc = launch_status()) != BONSAI_OK) return rc;
  unsigned bad = 0;
  if (cudaMemcpyFromSymbolAsync(&bad, g_pack_bad_code, sizeof(bad), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return BONSAI_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return BONSAI_ERR_CUDA;
  return bad ? BONSAI_ERR_BAD_CODE : BONSAI_OK;
}

int bonsai_dequant(const void* packed, const uint16_t* scales, int64_t N, int64_t K, int mode, uint16_t* w,
                   void* stream) {
  if (!valid_mode(mode)) return BONSAI_ERR_INVALID_ARG;
  int rc = check_shape(0, N, K);
  if (rc != BONSAI_OK) return rc;
  if (N == 0 || K == 0) return BONSAI_OK;
  if (!packed || !scales || !w) return BONSAI_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(scales) || !aligned16(w)) return BONSAI_ERR_ALIGN;
  if ((rc = check_device()) != BONSAI_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (mode == BONSAI_TERNARY_B3) {
    dequant_b3_kernel<<<grid_for(N * (K / kGroup), 256), 256, 0, st>>>(static_cast<const uint32_t*>(packed), scales, w,
                                                                          N, K);
    return launch_status();
  }
  const int64_t words = N * K / (mode == BONSAI_BINARY ? 32 : 16);
  const int grid = grid_for(words, 256);
  const auto* pk = static_cast<const uint32_t*>(packed);
  const bool wide = (reinterpret_cast<uintptr_t>(w) & 31u) == 0;  // 32-byte stores
  if (mode == BONSAI_BINARY && wide)
    dequant_kernel<BONSAI_BINARY, true><<<grid, 256, 0, st>>>(pk, scales, w, N, K);
  else if (mode == BONSAI_BINARY)
    dequant_kernel<BONSAI_BINARY, false><<<grid, 256, 0, st>>>(pk, scales, w, N, K);
  else if (wide)
    dequant_kernel<BONSAI_TERNARY_INT2, true><<<grid, 256, 0, st>>>(pk, scales, w, N, K);
  else
    dequant_kernel<BONSAI_TERNARY_INT2, false><<<grid, 256, 0, st>>>(pk, scales, w, N, K);
  return launch_status();
}

int bonsai_lowbit_gemm(const uint16_t* A, const void* packed, const uint16_t* scales, int64_t M, int64_t N, int64_t K,
                       int mode, uint16_t* out, void* stream) {
  if (!valid_mode(mode)) return BONSAI_ERR_INVALID_ARG;
  int rc = check_shape(M, N, K);
  if (rc != BONSAI_OK) return rc;
  if (M == 0 || N == 0) return BONSAI_OK;
  if (!out) return BONSAI_ERR_INVALID_ARG;
  if (!aligned16(out)) return BONSAI_ERR_ALIGN;
  if ((rc = check_device()) != BONSAI_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (K == 0) {  // empty sum
    return cudaMemsetAsync(out, 0, static_cast<size_t>(M) * N * 2, st) == cudaSuccess ? BONSAI_OK : BONSAI_ERR_CUDA;
  }
  if (!A || !packed || !scales) return BONSAI_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(packed) || !aligned16(scales)) return BONSAI_ERR_ALIGN;
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  if (mode == BONSAI_BINARY) return dispatch_gemm<BONSAI_BINARY>(A, packed, scales, nullptr, m, n, k, out, st);
  if (mode == BONSAI_TERNARY_B3)
    return dispatch_gemm<BONSAI_TERNARY_B3>(A, packed, scales, nullptr, m, n, k, out, st);
  return dispatch_gemm<BONSAI_TERNARY_INT2>(A, packed, scales, nullptr, m, n, k, out, st);
}

int bonsai_lowbit_gemm_host(const uint16_t* A_host, const void* packed, const uint16_t* scales, int64_t M, int64_t N,
                            int64_t K, int mode, uint16_t* out_host, uint16_t* A_dev, uint16_t* out_dev, void* stream) {
  if (!valid_mode(mode)) return BONSAI_ERR_INVALID_ARG;
  int rc = check_shape(M, N, K);
  if (rc != BONSAI_OK) return rc;
  if (M == 0 || N == 0) return BONSAI_OK;
  if (!A_host || !out_host || !A_dev || !out_dev || (K > 0 && (!packed || !scales))) return BONSAI_ERR_INVALID_ARG;
  if (!aligned16(A_dev) || !aligned16(out_dev) || (K > 0 && (!aligned16(packed) || !aligned16(scales))))
    return BONSAI_ERR_ALIGN;
  if ((rc = check_device()) != BONSAI_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (K == 0) {  // empty sum: zeros, written through the device buffer
    if (cudaMemsetAsync(out_dev, 0, static_cast<size_t>(M) * N * 2, st) != cudaSuccess ||
        cudaMemcpyAsync(out_host, out_dev, static_cast<size_t>(M) * N * 2, cudaMemcpyDeviceToHost, st) != cudaSuccess)
      return BONSAI_ERR_CUDA;
    return BONSAI_OK;
  }
  if (mode == BONSAI_BINARY)
    return gemm_host_pipelined<BONSAI_BINARY>(A_host, packed, scales, M, N, K, out_host, A_dev, out_dev, st);
  if (mode == BONSAI_TERNARY_B3)
    return gemm_host_pipelined<BONSAI_TERNARY_B3>(A_host, packed, scales, M, N, K, out_host, A_dev, out_dev, st);
  return gemm_host_pipelined<BONSAI_TERNARY_INT2>(A_host, packed, scales, M, N, K, out_host, A_dev, out_dev, st);
}

int bonsai_lowbit_gemm_batch(const bonsai_gemm_problem* problems, int count, int mode, void* stream) {
  if (!valid_mode(mode)) return BONSAI_ERR_INVALID_ARG;
  if (count < 0 || (count > 0 && !problems)) return BONSAI_ERR_INVALID_ARG;
  bool any = false;
  for (int i = 0; i < count; ++i) {
    const bonsai_gemm_problem& q = problems[i];
    int rc = check_shape(q.M, q.N, q.K);
    if (rc != BONSAI_OK) return rc;
    if (q.M == 0 || q.N == 0) continue;
    if (!q.out) return BONSAI_ERR_INVALID_ARG;
    if (!aligned16(q.out)) return BONSAI_ERR_ALIGN;
    if (q.K > 0) {
      if (!q.A || !q.packed || !q.scales) return BONSAI_ERR_INVALID_ARG;
      if (!aligned16(q.A) || !aligned16(q.packed) || !aligned16(q.scales)) return BONSAI_ERR_ALIGN;
    }
    any = true;
  }
  if (!any) return BONSAI_OK;
  int rc = check_device();
  if (rc != BONSAI_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::vector<const bonsai_gemm_problem*> small;
  for (int i = 0; i < count; ++i) {
    const bonsai_gemm_problem& q = problems[i];
    if (q.M == 0 || q.N == 0) continue;
    if (q.K == 0) {  // empty sums
      if (cudaMemsetAsync(q.out, 0, static_cast<size_t>(q.M) * q.N * 2, st) != cudaSuccess) return BONSAI_ERR_CUDA;
    } else if (q.M <= 16) {
      small.push_back(&q);
    }
  }
  // Launches of nearly equal numbers of problems, at most kBatchMaxLayers each.
  const int n_small = static_cast<int>(small.size());
  const int launches = (n_small + kBatchMaxLayers - 1) / kBatchMaxLayers;
  for (int l = 0; l < launches; ++l) {
    const int b = static_cast<int>(static_cast<int64_t>(n_small) * l / launches);
    const int e = static_cast<int>(static_cast<int64_t>(n_small) * (l + 1) / launches);
    rc = mode == BONSAI_BINARY      ? launch_gemm_batch<BONSAI_BINARY>(small.data() + b, e - b, st)
         : mode == BONSAI_TERNARY_B3 ? launch_gemm_batch<BONSAI_TERNARY_B3>(small.data() + b, e - b, st)
                                     : launch_gemm_batch<BONSAI_TERNARY_INT2>(small.data() + b, e - b, st);
    if (rc != BONSAI_OK) return rc;
  }
  for (int i = 0; i < count; ++i) {
    const bonsai_gemm_problem& q = problems[i];
    if (q.M <= 16 || q.N == 0 || q.K == 0) continue;
    const int m = static_cast<int>(q.M), n = static_cast<int>(q.N), k = static_cast<int>(q.K);
    rc = mode == BONSAI_BINARY ? dispatch_gemm<BONSAI_BINARY>(q.A, q.packed, q.scales, nullptr, m, n, k, q.out, st)
         : mode == BONSAI_TERNARY_B3
             ? dispatch_gemm<BONSAI_TERNARY_B3>(q.A, q.packed, q.scales, nullptr, m, n, k, q.out, st)
             : dispatch_gemm<BONSAI_TERNARY_INT2>(q.A, q.packed, q.scales, nullptr, m, n, k, q.out, st);
    if (rc != BONSAI_OK) return rc;
  }
  return BONSAI_OK;
}

// ------------------------------------------ 4-bit group-affine weights --
size_t bonsai_hqq4_packed_bytes(int64_t N, int64_t K) {
  if (check_shape(0, N, K) != BONSAI_OK) return 0;
  return static_cast<size_t>(N) * static_cast<size_t>(K) / 2;
}

int bonsai_hqq4_pack(const uint8_t* q, int64_t N, int64_t K, void* packed, void* stream) {
  int rc = check_shape(0, N, K);
  if (rc != BONSAI_OK) return rc;
  if (N == 0 || K == 0) return BONSAI_OK;
  if (!q || !packed) return BONSAI_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(packed)) return BONSAI_ERR_ALIGN;
  if ((rc = check_device()) != BONSAI_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned zero = 0;
  if (cudaMemcpyToSymbolAsync(g_pack_bad_code, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return BONSAI_ERR_CUDA;
  const int64_t words = N * K / 8;
  pack_hqq4_kernel<<<grid_for(words / 4, 256), 256, 0, st>>>(q, static_cast<uint32_t*>(packed), words);
  if ((rc = launch_status()) != BONSAI_OK) return rc;
  unsigned bad = 0;
  if (cudaMemcpyFromSymbolAsync(&bad, g_pack_bad_code, sizeof(bad), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return BONSAI_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return BONSAI_ERR_CUDA;
  return bad ? BONSAI_ERR_BAD_CODE : BONSAI_OK;
}

int bonsai_hqq4_dequant(const void* packed, const uint16_t* scales, const uint16_t* zeros, int64_t N, int64_t K,
                        uint16_t* w, void* stream) {
  int rc = check_shape(0, N, K);
  if (rc != BONSAI_OK) return rc;
  if (N == 0 || K == 0) return BONSAI_OK;
  if (!packed || !scales || !zeros || !w) return BONSAI_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(scales) || !aligned16(zeros) || !aligned16(w)) return BONSAI_ERR_ALIGN;
  if ((rc = check_device()) != BONSAI_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dequant_hqq4_kernel<<<grid_for(N * K / 8, 256), 256, 0, st>>>(static_cast<const uint32_t*>(packed), scales, zeros,
                                                                  w, N, K);
  return launch_status();
}

int bonsai_hqq4_gemm(const uint16_t* A, const void* packed, const uint16_t* scales, const uint16_t* zeros, int64_t M,
                     int64_t N, int64_t K, uint16_t* out, void* stream) {
  int rc = check_shape(M, N, K);
  if (rc != BONSAI_OK) return rc;
  if (M == 0 || N == 0) return BONSAI_OK;
  if (!out || (K > 0 && (!A || !packed || !scales || !zeros))) return BONSAI_ERR_INVALID_ARG;
  if (!aligned16(out) || (K > 0 && (!aligned16(A) || !aligned16(packed) || !aligned16(scales) || !aligned16(zeros))))
    return BONSAI_ERR_ALIGN;
  if ((rc = check_device()) != BONSAI_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (K == 0)
    return cudaMemsetAsync(out, 0, static_cast<size_t>(M) * N * 2, st) == cudaSuccess ? BONSAI_OK : BONSAI_ERR_CUDA;
  return dispatch_gemm<kModeHqq4>(A, packed, scales, zeros, static_cast<int>(M), static_cast<int>(N),
                                  static_cast<int>(K), out, st);
}

int bonsai_gemm_plan(int64_t M, int64_t N, int64_t K, int mode, int* block_t, int* ksplit, int* ctas, int* tiles) {
  if (!valid_mode(mode) && mode != kModeHqq4) return BONSAI_ERR_INVALID_ARG;
  int rc = check_shape(M, N, K);
  if (rc != BONSAI_OK) return rc;
  if (!block_t || !ksplit || !ctas || !tiles) return BONSAI_ERR_INVALID_ARG;
  if (M == 0 || N == 0 || K == 0) {
    *block_t = 0;
    *ksplit = 0;
    *ctas = 0;
    *tiles = 0;
    return BONSAI_OK;
  }
  if ((rc = check_device()) != BONSAI_OK) return rc;
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  const Plan p = mode == BONSAI_BINARY      ? plan_gemm<BONSAI_BINARY>(m, n, k)
                 : mode == BONSAI_TERNARY_B3 ? plan_gemm<BONSAI_TERNARY_B3>(m, n, k)
                 : mode == kModeHqq4         ? plan_gemm<kModeHqq4>(m, n, k)
                                             : plan_gemm<BONSAI_TERNARY_INT2>(m, n, k);
  if (p.block_t == 0) return BONSAI_ERR_CUDA;
  *block_t = p.block_t;
  *ksplit = p.ksplit;
  *ctas = p.ctas;
  *tiles = p.tiles;
  return BONSAI_OK;
}

int bonsai_get_device_error(void) {
  int rc = check_device();
  if (rc == BONSAI_ERR_CUDA) return rc;
  if (cudaDeviceSynchronize() != cudaSuccess) return BONSAI_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpyFromSymbol(&word, g_device_error, sizeof(word)) != cudaSuccess) return BONSAI_ERR_CUDA;
  const unsigned zero = 0;
  if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return BONSAI_ERR_CUDA;
  if (word & kErrBitTimeout) return BONSAI_ERR_TIMEOUT;
  return word ? BONSAI_ERR_CUDA : BONSAI_OK;
}

const char* bonsai_status_string(int status) {
  switch (status) {
    case BONSAI_OK: return "ok";
    case BONSAI_ERR_INVALID_ARG: return "invalid argument";
    case BONSAI_ERR_SHAPE: return "invalid shape";
    case BONSAI_ERR_ALIGN: return "pointer not 16-byte aligned";
    case BONSAI_ERR_BAD_CODE: return "code outside the alphabet";
    case BONSAI_ERR_CUDA: return "CUDA error";
    case BONSAI_ERR_ARCH: return "device is not sm_100";
    case BONSAI_ERR_TIMEOUT: return "a bounded wait in a kernel ran out";
    default: return "unknown status";
  }
}

int bonsai_selftest_wait_timeout(uint64_t limit_ns) {
  int rc = check_device();
  if (rc != BONSAI_OK) return rc;
  if ((rc = bonsai_get_device_error()) == BONSAI_ERR_CUDA) return rc;
  wait_timeout_selftest_kernel<<<1, 32>>>(limit_ns);
  if (launch_status() != BONSAI_OK) return BONSAI_ERR_CUDA;
  return bonsai_get_device_error();
}

}  // extern "C"
