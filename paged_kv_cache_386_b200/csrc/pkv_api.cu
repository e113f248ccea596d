// pkv_api.cu -- C ABI of libpagedkv.so (declared in include/pagedkv.h):
// argument checks, per-device set-up, tensor-map encoding and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "pagedkv.h"
#include "pkv_kernels.cuh"
#include "pkv_prefix.cuh"
#include "pkv_prefix_tc.cuh"

namespace pkv {
namespace {

constexpr int kMaxDevices = 64;
constexpr int32_t kVersion = 10000;  // 1.0.0

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceInfo {
  bool ready = false;
  int sm_count = 0;
  int smem_optin = 0;
};

std::mutex g_mutex;
DeviceInfo g_devices[kMaxDevices];
EncodeTiledFn g_encode = nullptr;

pkv_status device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_devices[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      return PKV_ERR_CUDA;
    d.ready = true;
  }
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qres) != cudaSuccess ||
        qres != cudaDriverEntryPointSuccess || fn == nullptr)
      return PKV_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  *out = d;
  return PKV_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_bytes(pkv_dtype dt) {
  switch (dt) {
    case PKV_F32: return 4;
    case PKV_F16: return 2;
    case PKV_BF16: return 2;
    default: return 0;
  }
}

// Query heads handled together on one kv head by the tensor-core path: the
// largest divisor of the group size that is at most 16; 1 selects the
// CUDA-core path.
int heads_per_segment(int group, pkv_dtype dt, bool force_simt) {
  if (dt == PKV_F32 || force_simt || group < 2) return 1;
  for (int gp = 16; gp >= 2; --gp)
    if (group % gp == 0) return gp;
  return 1;
}

int record_floats(int gp, int head_dim) { return (gp * (head_dim + 2) + 3) & ~3; }

size_t meta_bytes(int chunks) { return (static_cast<size_t>(chunks) * sizeof(int4) + 255) & ~static_cast<size_t>(255); }

constexpr int kDefaultSubChunks = 0;  // balancing chunks cost more than they recover on B200
constexpr int kDefaultStaticPermille = 800;
constexpr size_t kSchedBytes = 256;  // claim counter of the balancing chunks

// Workspace: the claim counter, then per chunk (units x (1 + sub_chunks)) one
// metadata entry and two partial-softmax records (its first and last
// segment).
size_t workspace_for(int units, int sub_chunks, int gp, int head_dim) {
  const size_t chunks = static_cast<size_t>(units) * (1 + sub_chunks);
  return kSchedBytes + meta_bytes(static_cast<int>(chunks)) + chunks * 2 * record_floats(gp, head_dim) * sizeof(float);
}

struct DecodeShape {
  int batch, n_q, n_kv, head_dim, group, gp, ng, units;
  pkv_dtype dtype;
};

pkv_status check_decode_args(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                             int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t batch,
                             int32_t num_blocks, float scale, int32_t n_q_heads, int32_t n_kv_heads,
                             int32_t head_dim, int32_t block_size, void* out, pkv_dtype dtype) {
  if (batch < 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 ||
      head_dim <= 0 || block_size <= 0)
    return PKV_ERR_INVALID_ARG;
  if (n_q_heads % n_kv_heads != 0) return PKV_ERR_INVALID_ARG;
  if (!(scale == scale)) return PKV_ERR_INVALID_ARG;  // NaN scale
  if (elem_bytes(dtype) == 0) return PKV_ERR_UNSUPPORTED;
  if (block_size != kBlockTokens) return PKV_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
  if (batch > PKV_MAX_BATCH) return PKV_ERR_UNSUPPORTED;
  if (max_blocks_per_seq > (1 << 26)) return PKV_ERR_UNSUPPORTED;  // context lengths stay below 2^30
  if (batch == 0) return PKV_OK;
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PKV_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3u) || (reinterpret_cast<uintptr_t>(context_lens) & 3u))
    return PKV_ERR_INVALID_ARG;
  // Tile counts are 32-bit on the device: bound the worst case.
  const int64_t worst = static_cast<int64_t>(batch) * max_blocks_per_seq * n_q_heads;
  if (worst >= (int64_t(1) << 31)) return PKV_ERR_UNSUPPORTED;
  return PKV_OK;
}

pkv_status encode_cache_map(CUtensorMap* map, const void* cache, pkv_dtype dt, int num_blocks, int n_kv,
                            int head_dim) {
  const int es = elem_bytes(dt);
  const CUtensorMapDataType ty = dt == PKV_F32   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : dt == PKV_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  // [block][kv head][token][dim], innermost first.
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(kBlockTokens),
                              static_cast<cuuint64_t>(n_kv), static_cast<cuuint64_t>(num_blocks)};
  const cuuint64_t row = static_cast<cuuint64_t>(head_dim) * es;
  const cuuint64_t strides[3] = {row, row * kBlockTokens, row * kBlockTokens * n_kv};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / es), static_cast<cuuint32_t>(kBlockTokens), 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = g_encode(map, ty, 4, const_cast<void*>(cache), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : PKV_ERR_CUDA;
}

// A block's whole K or V tile of one kv head as one TMA box: dims {128
// bytes of dims, 16 tokens, head_dim * es / 128 chunks, kv head, block}, box
// {128 bytes, 16, chunks, 1, 1}, landing as [chunk][token][128 B] with the
// 128-byte swizzle -- the layout of `chunks` separate 16-row boxes, in one
// request.
pkv_status encode_cache_map_tile(CUtensorMap* map, const void* cache, pkv_dtype dt, int num_blocks, int n_kv,
                                 int head_dim) {
  const int es = elem_bytes(dt);
  const CUtensorMapDataType ty = dt == PKV_F32   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : dt == PKV_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const cuuint64_t row = static_cast<cuuint64_t>(head_dim) * es;
  const cuuint32_t x = static_cast<cuuint32_t>(128 / es), chunks = static_cast<cuuint32_t>(row / 128);
  const cuuint64_t dims[5] = {x, static_cast<cuuint64_t>(kBlockTokens), chunks, static_cast<cuuint64_t>(n_kv),
                              static_cast<cuuint64_t>(num_blocks)};
  const cuuint64_t strides[4] = {row, 128, row * kBlockTokens, row * kBlockTokens * n_kv};
  const cuuint32_t box[5] = {x, static_cast<cuuint32_t>(kBlockTokens), chunks, 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = g_encode(map, ty, 5, const_cast<void*>(cache), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : PKV_ERR_CUDA;
}

// K of a block for the tensor-memory prefix kernel (16-bit, head dim 128) as
// one TMA box: dims {64 dims, 8 tokens, dim half, 8-token group, block x kv
// head} (the cache's [block][kv head] pairs are 4 KiB apart), landing as
// [token group][dim half][8 tokens][128 B] with the 128-byte swizzle, so that
// the 8-token atoms of one dim half lie 2 KiB apart in shared memory.
pkv_status encode_cache_map_kgroups(CUtensorMap* map, const void* cache, pkv_dtype dt, int num_blocks, int n_kv,
                                    int head_dim) {
  if (elem_bytes(dt) != 2 || head_dim != 128) return PKV_ERR_UNSUPPORTED;
  const CUtensorMapDataType ty = dt == PKV_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const cuuint64_t row = 256;
  const cuuint64_t dims[5] = {64, 8, 2, 2, static_cast<cuuint64_t>(num_blocks) * static_cast<cuuint64_t>(n_kv)};
  const cuuint64_t strides[4] = {row, 128, 8 * row, kBlockTokens * row};
  const cuuint32_t box[5] = {64, 8, 2, 2, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = g_encode(map, ty, 5, const_cast<void*>(cache), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : PKV_ERR_CUDA;
}

// Encoded tensor maps, cached per (kind, base address, dtype, shape): a map
// depends only on those, so a serving loop that calls with the same caches
// every step pays the encode once.  A small table with least-recently-used
// replacement, shared by every device and host thread.
enum MapKind { kMapBox = 0, kMapTile = 1, kMapKGroups = 2 };
struct MapKey {
  const void* base;
  int kind, dtype, num_blocks, n_kv, head_dim;
  bool operator==(const MapKey& o) const {
    return base == o.base && kind == o.kind && dtype == o.dtype && num_blocks == o.num_blocks && n_kv == o.n_kv &&
           head_dim == o.head_dim;
  }
};
struct MapEntry {
  MapKey key;
  CUtensorMap map;
  uint64_t last_use;  // 0: empty
};
constexpr int kMapCacheSize = 32;
std::mutex g_map_mutex;
MapEntry g_map_cache[kMapCacheSize];
uint64_t g_map_clock = 0;

pkv_status cached_map(MapKind kind, CUtensorMap* map, const void* cache, pkv_dtype dt, int num_blocks, int n_kv,
                      int head_dim) {
  const MapKey key = {cache, static_cast<int>(kind), static_cast<int>(dt), num_blocks, n_kv, head_dim};
  {
    std::lock_guard<std::mutex> lock(g_map_mutex);
    for (MapEntry& e : g_map_cache) {
      if (e.last_use != 0 && e.key == key) {
        e.last_use = ++g_map_clock;
        *map = e.map;
        return PKV_OK;
      }
    }
  }
  const pkv_status st = kind == kMapTile      ? encode_cache_map_tile(map, cache, dt, num_blocks, n_kv, head_dim)
                        : kind == kMapKGroups ? encode_cache_map_kgroups(map, cache, dt, num_blocks, n_kv, head_dim)
                                              : encode_cache_map(map, cache, dt, num_blocks, n_kv, head_dim);
  if (st != PKV_OK) return st;
  std::lock_guard<std::mutex> lock(g_map_mutex);
  MapEntry* victim = &g_map_cache[0];
  for (MapEntry& e : g_map_cache)
    if (e.last_use < victim->last_use) victim = &e;
  victim->key = key;
  victim->map = *map;
  victim->last_use = ++g_map_clock;
  return PKV_OK;
}

// The decode kernel is launched cooperatively: its CTAs (at most one per SM)
// are guaranteed to be co-resident, which its grid-wide barrier needs.
template <int DT, int D, int GPAD, bool kI8 = false, bool kMQ = false, bool kFused = false>
pkv_status launch_decode(const CUtensorMap& mk, const CUtensorMap& mv, const DecodeParams& p, int grid, size_t smem,
                         cudaStream_t stream) {
  auto kern = pkv_decode_kernel<DT, D, GPAD, kI8, kMQ, kFused>;
  // Opt in to the largest dynamic shared memory once per device (the launch
  // itself passes the size it needs).
  static bool opted_in[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
  if (!opted_in[dev]) {
    int optin = 0;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - 256) != cudaSuccess)
      return PKV_ERR_CUDA;
    opted_in[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kDecodeThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, mk, mv, p) != cudaSuccess) return PKV_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

template <int DT, int D, bool kFused>
pkv_status dispatch_gpad_f(int gpad, const CUtensorMap& mk, const CUtensorMap& mv, const DecodeParams& p, int grid,
                           size_t smem, cudaStream_t stream) {
  if constexpr (DT == kF32) {
    return launch_decode<DT, D, 0, false, false, kFused>(mk, mv, p, grid, smem, stream);
  } else {
    switch (gpad) {
      case 0: return launch_decode<DT, D, 0, false, false, kFused>(mk, mv, p, grid, smem, stream);
      case 8: return launch_decode<DT, D, 8, false, false, kFused>(mk, mv, p, grid, smem, stream);
      default: return launch_decode<DT, D, 16, false, false, kFused>(mk, mv, p, grid, smem, stream);
    }
  }
}

// The plain decode, or with the new tokens' append fused in front of it.
template <int DT, int D>
pkv_status dispatch_gpad(int gpad, const CUtensorMap& mk, const CUtensorMap& mv, const DecodeParams& p, int grid,
                         size_t smem, cudaStream_t stream) {
  return p.app.total > 0 ? dispatch_gpad_f<DT, D, true>(gpad, mk, mv, p, grid, smem, stream)
                         : dispatch_gpad_f<DT, D, false>(gpad, mk, mv, p, grid, smem, stream);
}

template <int DT>
pkv_status dispatch_dim(int head_dim, int gpad, const CUtensorMap& mk, const CUtensorMap& mv, const DecodeParams& p,
                        int grid, size_t smem, cudaStream_t stream) {
  return head_dim == 64 ? dispatch_gpad<DT, 64>(gpad, mk, mv, p, grid, smem, stream)
                        : dispatch_gpad<DT, 128>(gpad, mk, mv, p, grid, smem, stream);
}

// INT8 cache (head_dim 128, tensor-core consumer for every head group).
template <int DT>
pkv_status dispatch_i8(int gpad, const CUtensorMap& mk, const DecodeParams& p, int grid, size_t smem,
                       cudaStream_t stream) {
  return gpad == 8 ? launch_decode<DT, 128, 8, true>(mk, mk, p, grid, smem, stream)
                   : launch_decode<DT, 128, 16, true>(mk, mk, p, grid, smem, stream);
}

// Several queries per sequence (16-bit data, tensor-core consumer).
template <int DT>
pkv_status dispatch_mq(int head_dim, int gpad, const CUtensorMap& mk, const CUtensorMap& mv, const DecodeParams& p,
                       int grid, size_t smem, cudaStream_t stream) {
  if (head_dim == 64)
    return gpad == 8 ? launch_decode<DT, 64, 8, false, true>(mk, mv, p, grid, smem, stream)
                     : launch_decode<DT, 64, 16, false, true>(mk, mv, p, grid, smem, stream);
  return gpad == 8 ? launch_decode<DT, 128, 8, false, true>(mk, mv, p, grid, smem, stream)
                   : launch_decode<DT, 128, 16, false, true>(mk, mv, p, grid, smem, stream);
}

// Heads per segment with q_len queries: the largest divisor of the head group
// whose rows (heads x queries) fit the 16 rows of a tensor-core tile.
int heads_per_segment_mq(int group, int q_len) {
  for (int gp = 16 / q_len; gp >= 1; --gp)
    if (group % gp == 0) return gp;
  return 1;
}

// The INT8 cache (one record per (block, kv head); null for 16-bit caches).
struct KvI8 {
  const uint8_t* records;
};

// Shared-memory ring of the prefix kernel: three stages of 64 tokens of K and V.
constexpr int kPrefixStages = 3;

size_t prefix_init_bytes(int batch, int n_q_heads, int head_dim) {
  return (static_cast<size_t>(batch) * n_q_heads * (head_dim + 2) * sizeof(float) + 255) & ~static_cast<size_t>(255);
}

template <int DT, int D>
pkv_status launch_prefix(const CUtensorMap& mk, const CUtensorMap& mv, const PrefixParams& pp, int n_kv, size_t smem,
                         cudaStream_t stream) {
  auto kern = pkv_prefix_kernel<DT, D>;
  static bool opted_in[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
  if (!opted_in[dev]) {
    int optin = 0;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - 256) != cudaSuccess)
      return PKV_ERR_CUDA;
    opted_in[dev] = true;
  }
  const int rows = pp.batch * pp.group;
  const dim3 grid((rows + kPrefixRows - 1) / kPrefixRows, n_kv, pp.n_groups);
  kern<<<grid, kPrefixThreads, smem, stream>>>(mk, mv, pp);
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

// The tensor-memory prefix kernel (head dim 128): 128-row tiles, 192 KiB of
// operands plus barriers and the member list.
size_t prefix_tc_smem(int batch) {
  return 1024 + kTcSmemBytes + kTcBarBytes + kTcExchBytes + static_cast<size_t>(batch) * 4;
}

// Launch configuration of the tensor-memory prefix kernel: one cluster of
// `splits` CTAs per 128-row tile of every (group, kv head).
cudaLaunchConfig_t prefix_tc_config(const PrefixParams& pp, int n_kv, int splits, cudaStream_t stream,
                                    cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  const int rows = pp.batch * pp.group;
  cfg.gridDim = dim3(static_cast<unsigned>((rows + kTcRows - 1) / kTcRows * splits), n_kv, pp.n_groups);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = prefix_tc_smem(pp.batch);
  cfg.stream = stream;
  attr->id = cudaLaunchAttributeClusterDimension;
  attr->val.clusterDim.x = static_cast<unsigned>(splits);
  attr->val.clusterDim.y = 1;
  attr->val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

// Prefix shares per tile: enough clusters to cover the SMs once, at most
// kTcMaxSplit, and only sizes the device can co-schedule.  Rows per group are
// not known on the host; the estimate takes every group's tiles as full but
// the total as at most the tiles of the batch plus one ragged tile per group.
template <int DT>
int prefix_tc_splits(const PrefixParams& pp, int n_kv, int sm_count, cudaStream_t stream) {
  const long tiles_batch = (static_cast<long>(pp.batch) * pp.group + kTcRows - 1) / kTcRows;
  const long ctas = static_cast<long>(n_kv) * std::min(tiles_batch * pp.n_groups, tiles_batch + pp.n_groups - 1);
  int splits = static_cast<int>(std::max(1L, std::min<long>(kTcMaxSplit, sm_count / std::max(1L, ctas))));
  // Whether clusters of each size can be co-scheduled, per device (0 unknown, 1 yes, -1 no).
  static int feasible[kMaxDevices][kTcMaxSplit + 1] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 1;
  for (; splits > 1; --splits) {
    if (feasible[dev][splits] == 0) {
      cudaLaunchAttribute attr;
      cudaLaunchConfig_t cfg = prefix_tc_config(pp, n_kv, splits, stream, &attr);
      int clusters = 0;
      const bool yes =
          cudaOccupancyMaxActiveClusters(&clusters, pkv_prefix_tc_kernel<DT>, &cfg) == cudaSuccess && clusters > 0;
      (void)cudaGetLastError();
      feasible[dev][splits] = yes ? 1 : -1;
    }
    if (feasible[dev][splits] > 0) break;
  }
  return splits;
}

template <int DT>
pkv_status launch_prefix_tc(const CUtensorMap& mk, const CUtensorMap& mv, const PrefixParams& pp, int n_kv,
                            int splits, int sm_count, cudaStream_t stream) {
  auto kern = pkv_prefix_tc_kernel<DT>;
  static bool opted_in[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
  if (!opted_in[dev]) {
    int optin = 0;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - 256) != cudaSuccess)
      return PKV_ERR_CUDA;
    opted_in[dev] = true;
  }
  if (splits <= 0) splits = prefix_tc_splits<DT>(pp, n_kv, sm_count, stream);
  if (splits > kTcMaxSplit) return PKV_ERR_INVALID_ARG;
  cudaLaunchAttribute attr;
  cudaLaunchConfig_t cfg = prefix_tc_config(pp, n_kv, splits, stream, &attr);
  if (cfg.gridDim.x > 0x7fffffffu / 2) return PKV_ERR_INVALID_ARG;
  return cudaLaunchKernelEx(&cfg, kern, mk, mv, pp) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

}  // namespace
}  // namespace pkv

namespace pkv {
namespace {
// Checks of paged_kv_append's arguments and its kernel parameters.
pkv_status append_params(const void* k, const void* v, const int64_t* slot_mapping, int32_t num_tokens,
                         void* k_cache, void* v_cache, int32_t num_blocks, int32_t block_size, int32_t n_kv_heads,
                         int32_t head_dim, pkv_dtype dtype, AppendParams* p) {
  if (num_tokens < 0 || num_blocks <= 0 || block_size <= 0 || n_kv_heads <= 0 || head_dim <= 0)
    return PKV_ERR_INVALID_ARG;
  const int es = elem_bytes(dtype);
  if (es == 0 || block_size != kBlockTokens || (head_dim * es) % 16 != 0) return PKV_ERR_UNSUPPORTED;
  *p = {};
  if (num_tokens == 0) return PKV_OK;
  if (!k || !v || !slot_mapping || !k_cache || !v_cache) return PKV_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return PKV_ERR_INVALID_ARG;
  p->k = static_cast<const uint8_t*>(k);
  p->v = static_cast<const uint8_t*>(v);
  p->slot_mapping = slot_mapping;
  p->k_cache = static_cast<uint8_t*>(k_cache);
  p->v_cache = static_cast<uint8_t*>(v_cache);
  p->num_slots = static_cast<int64_t>(num_blocks) * block_size;
  p->n_kv_heads = n_kv_heads;
  p->row_chunks = head_dim * es / 16;
  p->total = static_cast<int64_t>(num_tokens) * n_kv_heads * p->row_chunks;
  return PKV_OK;
}
}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" {

int32_t pkv_version(void) { return kVersion; }

const char* pkv_status_string(pkv_status s) {
  switch (s) {
    case PKV_OK: return "ok";
    case PKV_ERR_INVALID_ARG: return "invalid argument";
    case PKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case PKV_ERR_OUT_OF_RANGE: return "a kernel saw an out-of-range block id, context length or slot";
    case PKV_ERR_CUDA: return "CUDA runtime error";
    case PKV_ERR_WORKSPACE: return "workspace too small";
    case PKV_ERR_NO_BLOCKS: return "not enough free or evictable blocks";
    case PKV_ERR_HOST_MEMORY: return "host allocation failed";
    default: return "unknown status";
  }
}

pkv_status paged_kv_append(const void* k, const void* v, const int64_t* slot_mapping, int32_t num_tokens,
                           void* k_cache, void* v_cache, int32_t num_blocks, int32_t block_size,
                           int32_t n_kv_heads, int32_t head_dim, pkv_dtype dtype, void* stream) {
  AppendParams p;
  const pkv_status st = append_params(k, v, slot_mapping, num_tokens, k_cache, v_cache, num_blocks, block_size,
                                      n_kv_heads, head_dim, dtype, &p);
  if (st != PKV_OK || num_tokens == 0) return st;
  DeviceInfo di;
  if (device_info(&di) != PKV_OK) return PKV_ERR_CUDA;
  const int64_t want = (p.total + 255) / 256;
  const int grid = static_cast<int>(want < int64_t(di.sm_count) * 8 ? want : int64_t(di.sm_count) * 8);
  pkv_append_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status paged_kv_copy_blocks(void* k_cache, void* v_cache, const int32_t* src_blocks, const int32_t* dst_blocks,
                                int32_t n_pairs, int32_t num_blocks, int32_t block_size, int32_t n_kv_heads,
                                int32_t head_dim, pkv_dtype dtype, void* stream) {
  if (n_pairs < 0 || num_blocks <= 0 || block_size <= 0 || n_kv_heads <= 0 || head_dim <= 0)
    return PKV_ERR_INVALID_ARG;
  const int es = elem_bytes(dtype);
  if (es == 0 || block_size != kBlockTokens || (head_dim * es) % 16 != 0) return PKV_ERR_UNSUPPORTED;
  if (n_pairs == 0) return PKV_OK;
  if (!k_cache || !v_cache || !src_blocks || !dst_blocks || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(src_blocks) & 3u) || (reinterpret_cast<uintptr_t>(dst_blocks) & 3u))
    return PKV_ERR_INVALID_ARG;
  const int64_t chunks = static_cast<int64_t>(n_kv_heads) * block_size * head_dim * es / 16;
  if (chunks > INT32_MAX) return PKV_ERR_UNSUPPORTED;
  DeviceInfo di;
  if (device_info(&di) != PKV_OK) return PKV_ERR_CUDA;
  CopyParams p;
  p.k_cache = static_cast<uint8_t*>(k_cache);
  p.v_cache = static_cast<uint8_t*>(v_cache);
  p.src = src_blocks;
  p.dst = dst_blocks;
  p.n_pairs = n_pairs;
  p.num_blocks = num_blocks;
  p.chunks = static_cast<int32_t>(chunks);
  const int grid = n_pairs < di.sm_count * 8 ? n_pairs : di.sm_count * 8;
  pkv_copy_blocks_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status paged_kv_append_int8(const void* k, const void* v, pkv_dtype dtype, const int64_t* slot_mapping,
                                int32_t num_tokens, uint8_t* kv_cache, int32_t num_blocks, int32_t block_size,
                                int32_t n_kv_heads, int32_t head_dim, void* stream) {
  if (num_tokens < 0 || num_blocks <= 0 || block_size <= 0 || n_kv_heads <= 0 || head_dim <= 0)
    return PKV_ERR_INVALID_ARG;
  if (elem_bytes(dtype) == 0 || block_size != kBlockTokens || (head_dim != 64 && head_dim != 128))
    return PKV_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PKV_OK;
  if (!k || !v || !slot_mapping || !kv_cache || !aligned16(kv_cache) || (reinterpret_cast<uintptr_t>(slot_mapping) & 7u) ||
      (reinterpret_cast<uintptr_t>(k) & 3u) || (reinterpret_cast<uintptr_t>(v) & 3u))
    return PKV_ERR_INVALID_ARG;
  DeviceInfo di;
  if (device_info(&di) != PKV_OK) return PKV_ERR_CUDA;
  AppendI8Params p;
  p.k = k;
  p.v = v;
  p.slot_mapping = slot_mapping;
  p.cache = kv_cache;
  p.num_slots = static_cast<int64_t>(num_blocks) * block_size;
  p.num_tokens = num_tokens;
  p.n_kv_heads = n_kv_heads;
  const int64_t warps = static_cast<int64_t>(num_tokens) * n_kv_heads;
  const int64_t want = (warps + 7) / 8;  // 8 warps per 256-thread CTA
  const int grid = static_cast<int>(want < int64_t(di.sm_count) * 8 ? want : int64_t(di.sm_count) * 8);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool d128 = head_dim == 128;
  switch (dtype) {
    case PKV_F32:
      d128 ? pkv_append_i8_kernel<kF32, 128><<<grid, 256, 0, s>>>(p) : pkv_append_i8_kernel<kF32, 64><<<grid, 256, 0, s>>>(p);
      break;
    case PKV_F16:
      d128 ? pkv_append_i8_kernel<kF16, 128><<<grid, 256, 0, s>>>(p) : pkv_append_i8_kernel<kF16, 64><<<grid, 256, 0, s>>>(p);
      break;
    default:
      d128 ? pkv_append_i8_kernel<kBF16, 128><<<grid, 256, 0, s>>>(p)
           : pkv_append_i8_kernel<kBF16, 64><<<grid, 256, 0, s>>>(p);
      break;
  }
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status paged_attention_workspace_size(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                          pkv_dtype dtype, size_t* bytes) {
  return paged_attention_workspace_size_ex(batch, n_q_heads, n_kv_heads, head_dim, dtype, nullptr, bytes);
}

pkv_status paged_attention_workspace_size_ex(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                             pkv_dtype dtype, const pkv_decode_options* options, size_t* bytes) {
  if (!bytes || batch < 0 || n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads % n_kv_heads != 0 || head_dim <= 0)
    return PKV_ERR_INVALID_ARG;
  if (elem_bytes(dtype) == 0 || (head_dim != 64 && head_dim != 128)) return PKV_ERR_UNSUPPORTED;
  DeviceInfo di;
  if (device_info(&di) != PKV_OK) return PKV_ERR_CUDA;
  // Sized for the widest head group so that force_simt never needs more.
  const int gp = heads_per_segment(n_q_heads / n_kv_heads, dtype, false);
  const int sub = (options && options->balance_chunks > 0) ? options->balance_chunks : kDefaultSubChunks;
  if (sub > 4) return PKV_ERR_INVALID_ARG;
  *bytes = workspace_for(di.sm_count * kConsumerWarps, sub, gp, head_dim);
  return PKV_OK;
}

}  // extern "C"

namespace pkv {
namespace {
// The decode launch behind paged_attention_decode_ex and the cascade: `init`
// and `seq_group` (both null for a plain decode) give an initial softmax state
// per (sequence, query head).
pkv_status decode_impl(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                       int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t batch, int32_t num_blocks,
                       float scale, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int32_t block_size,
                       void* out, pkv_dtype dtype, void* workspace, size_t workspace_bytes, void* stream,
                       const pkv_decode_options* options, const float* init, const int32_t* seq_group,
                       int32_t n_groups, const KvI8* i8 = nullptr, int32_t q_len = 1,
                       const AppendParams* app = nullptr) {
  pkv_status st = check_decode_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, batch,
                                    num_blocks, scale, n_q_heads, n_kv_heads, head_dim, block_size, out, dtype);
  if (st != PKV_OK) return st;
  if (i8 && (dtype == PKV_F32 || head_dim != 128)) return PKV_ERR_UNSUPPORTED;
  if (q_len < 1) return PKV_ERR_INVALID_ARG;
  if (q_len > 1 && (q_len > 16 || dtype == PKV_F32 || i8 || init)) return PKV_ERR_UNSUPPORTED;
  if (batch == 0) return st;
  pkv_decode_options opt = {};
  if (options) {
    opt = *options;
    for (int i = 0; i < 2; ++i)
      if (opt.reserved[i] != 0) return PKV_ERR_INVALID_ARG;
    if (opt.wait_limit_us < 0 || opt.test_withhold_unit < 0) return PKV_ERR_INVALID_ARG;
    if (opt.num_units < 0 || (opt.force_simt != 0 && opt.force_simt != 1)) return PKV_ERR_INVALID_ARG;
    if (opt.balance_chunks < 0 || opt.balance_chunks > 4) return PKV_ERR_INVALID_ARG;
    if (opt.static_permille != 0 && (opt.static_permille < 500 || opt.static_permille > 999))
      return PKV_ERR_INVALID_ARG;
  }
  const int sub_chunks = opt.balance_chunks == 0 ? kDefaultSubChunks : opt.balance_chunks;
  const int static_permille = opt.static_permille == 0 ? kDefaultStaticPermille : opt.static_permille;
  DeviceInfo di;
  if (device_info(&di) != PKV_OK) return PKV_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  const int group = n_q_heads / n_kv_heads;
  const bool mq = q_len > 1;
  const int gp = mq ? heads_per_segment_mq(group, q_len) : heads_per_segment(group, dtype, opt.force_simt == 1 && !i8);
  const int rows = gp * q_len;
  // The INT8 cache and several queries always take the tensor-core consumer.
  const int gpad = (rows == 1 && !i8 && !mq) ? 0 : (rows <= 8 ? 8 : 16);
  // One CTA per SM at most (the kernel's grid barrier needs every CTA
  // resident), so the unit count is capped at one per consumer warp of
  // every SM.
  const int default_units = di.sm_count * kConsumerWarps;
  const int units = (opt.num_units > 0 && opt.num_units < default_units) ? opt.num_units : default_units;
  const int grid = (units + kConsumerWarps - 1) / kConsumerWarps;

  // Ring depth: as many slots per consumer warp as shared memory allows
  // (at most 4; 2 with ten consumer warps and 8 KiB tiles).
  const int es = elem_bytes(dtype);
  // INT8: one record (K and transposed V codes, 2 x 16 scales).
  const size_t stage_bytes = i8 ? static_cast<size_t>(i8_record_bytes(head_dim))
                                : static_cast<size_t>(2) * (head_dim * es / 128) * kBoxBytes;
  // 1 KiB alignment slack, abort word, prefix sums and clamped lengths, and
  // 256 bytes for the kernel's static shared memory.
  const size_t qbuf_bytes = static_cast<size_t>(gpad == 0 ? 1 : gpad) * head_dim * es;
  const size_t fixed =
      1024 + kConsumerWarps * qbuf_bytes + 16 + static_cast<size_t>(2 * batch + 1) * sizeof(int) + 256;
  const size_t per_round = kConsumerWarps * (stage_bytes + 2 * sizeof(uint64_t) + 4 * sizeof(int));
  if (fixed + per_round > static_cast<size_t>(di.smem_optin)) return PKV_ERR_UNSUPPORTED;
  int stages = static_cast<int>((di.smem_optin - fixed) / per_round);
  if (stages > 4) stages = 4;
  const size_t smem = fixed - 256 + stages * per_round;

  const size_t need = workspace_for(units, sub_chunks, rows, head_dim);
  void* ws = workspace;
  bool own = false;
  if (ws == nullptr) {
    if (cudaMallocAsync(&ws, need, s) != cudaSuccess) return PKV_ERR_CUDA;
    own = true;
    if (cudaMemsetAsync(ws, 0, kSchedBytes, s) != cudaSuccess) {
      cudaFreeAsync(ws, s);
      return PKV_ERR_CUDA;
    }
  } else if (workspace_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) {
    return PKV_ERR_WORKSPACE;
  }

  CUtensorMap mk = {}, mv = {};
  if (!i8) {
    st = cached_map(kMapTile, &mk, k_cache, dtype, num_blocks, n_kv_heads, head_dim);
    if (st == PKV_OK) st = cached_map(kMapTile, &mv, v_cache, dtype, num_blocks, n_kv_heads, head_dim);
  }

  DecodeParams p;
  p.kv_i8 = i8 ? i8->records : nullptr;
  p.n_kv_heads = n_kv_heads;
  p.q = q;
  p.out = out;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  const int chunks = units * (1 + sub_chunks);
  p.sched = static_cast<int*>(ws);
  p.meta = reinterpret_cast<int4*>(static_cast<uint8_t*>(ws) + kSchedBytes);
  p.records = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kSchedBytes + meta_bytes(chunks));
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.batch = batch;
  p.num_blocks = num_blocks;
  p.n_q_heads = n_q_heads;
  p.group = group;
  p.gp = gp;
  p.ng = n_q_heads / gp;
  p.num_units = units;
  p.sub_chunks = sub_chunks;
  p.static_permille = static_permille;
  p.stages = stages;
  p.rec_floats = record_floats(rows, head_dim);
  p.q_len = q_len;
  p.rows = rows;
  p.head_dim = head_dim;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.init = init;
  p.seq_group = seq_group;
  p.n_groups = n_groups;
  p.wait_limit_ns = opt.wait_limit_us > 0 ? static_cast<uint64_t>(opt.wait_limit_us) * 1000u : kWaitLimitNs;
  p.withhold_unit = opt.test_withhold_unit - 1;
  p.app = {};
  if (app) p.app = *app;

  if (st == PKV_OK && mq) {
    st = dtype == PKV_F16 ? dispatch_mq<kF16>(head_dim, gpad, mk, mv, p, grid, smem, s)
                          : dispatch_mq<kBF16>(head_dim, gpad, mk, mv, p, grid, smem, s);
  } else if (st == PKV_OK && i8) {
    st = dtype == PKV_F16 ? dispatch_i8<kF16>(gpad, mk, p, grid, smem, s) : dispatch_i8<kBF16>(gpad, mk, p, grid, smem, s);
  } else if (st == PKV_OK) {
    switch (dtype) {
      case PKV_F32: st = dispatch_dim<kF32>(head_dim, gpad, mk, mv, p, grid, smem, s); break;
      case PKV_F16: st = dispatch_dim<kF16>(head_dim, gpad, mk, mv, p, grid, smem, s); break;
      default: st = dispatch_dim<kBF16>(head_dim, gpad, mk, mv, p, grid, smem, s); break;
    }
  }
  if (own && cudaFreeAsync(ws, s) != cudaSuccess && st == PKV_OK) st = PKV_ERR_CUDA;
  return st;
}
}  // namespace
}  // namespace pkv

extern "C" {

pkv_status paged_attention_decode_ex(const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                                     const int32_t* context_lens, int32_t batch, int32_t num_blocks, float scale,
                                     int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int32_t block_size,
                                     void* out, pkv_dtype dtype, void* workspace, size_t workspace_bytes,
                                     void* stream, const pkv_decode_options* options) {
  return decode_impl(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, batch, num_blocks, scale,
                     n_q_heads, n_kv_heads, head_dim, block_size, out, dtype, workspace, workspace_bytes, stream,
                     options, nullptr, nullptr, 0);
}

pkv_status paged_attention_decode(const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* block_tables, int32_t max_blocks_per_seq,
                                  const int32_t* context_lens, int32_t batch, int32_t num_blocks, float scale,
                                  int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int32_t block_size,
                                  void* out, pkv_dtype dtype, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  return paged_attention_decode_ex(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, batch,
                                   num_blocks, scale, n_q_heads, n_kv_heads, head_dim, block_size, out, dtype,
                                   workspace, workspace_bytes, stream, nullptr);
}

pkv_status paged_kv_append_and_decode(const void* q, const void* k, const void* v, const int64_t* slot_mapping,
                                      int32_t num_tokens, void* k_cache, void* v_cache,
                                      const int32_t* block_tables, int32_t max_blocks_per_seq,
                                      const int32_t* context_lens, int32_t batch, int32_t num_blocks, float scale,
                                      int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int32_t block_size,
                                      void* out, pkv_dtype dtype, void* workspace, size_t workspace_bytes,
                                      void* stream) {
  AppendParams app;
  pkv_status st = append_params(k, v, slot_mapping, num_tokens, k_cache, v_cache, num_blocks, block_size,
                                n_kv_heads, head_dim, dtype, &app);
  if (st != PKV_OK) return st;
  st = check_decode_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, batch, num_blocks,
                         scale, n_q_heads, n_kv_heads, head_dim, block_size, out, dtype);
  if (st != PKV_OK) return st;
  if (batch == 0)  // no decode: the append alone
    return paged_kv_append(k, v, slot_mapping, num_tokens, k_cache, v_cache, num_blocks, block_size, n_kv_heads,
                           head_dim, dtype, stream);
  return decode_impl(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, batch, num_blocks, scale,
                     n_q_heads, n_kv_heads, head_dim, block_size, out, dtype, workspace, workspace_bytes, stream,
                     nullptr, nullptr, nullptr, 0, nullptr, 1, &app);
}

pkv_status paged_attention_decode_int8(const void* q, const uint8_t* kv_cache, const int32_t* block_tables,
                                       int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t batch,
                                       int32_t num_blocks, float scale, int32_t n_q_heads, int32_t n_kv_heads,
                                       int32_t head_dim, int32_t block_size, void* out, pkv_dtype dtype,
                                       void* workspace, size_t workspace_bytes, void* stream) {
  const KvI8 i8 = {kv_cache};
  return decode_impl(q, kv_cache, kv_cache, block_tables, max_blocks_per_seq, context_lens, batch, num_blocks, scale,
                     n_q_heads, n_kv_heads, head_dim, block_size, out, dtype, workspace, workspace_bytes, stream,
                     nullptr, nullptr, nullptr, 0, &i8);
}

pkv_status paged_attention_mq_workspace_size(int32_t batch, int32_t q_len, int32_t n_q_heads, int32_t n_kv_heads,
                                             int32_t head_dim, pkv_dtype dtype, size_t* bytes) {
  if (!bytes || batch < 0 || q_len < 1 || n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads % n_kv_heads != 0)
    return PKV_ERR_INVALID_ARG;
  if (q_len > 16 || dtype == PKV_F32 || elem_bytes(dtype) == 0 || (head_dim != 64 && head_dim != 128))
    return PKV_ERR_UNSUPPORTED;
  DeviceInfo di;
  if (device_info(&di) != PKV_OK) return PKV_ERR_CUDA;
  const int rows = heads_per_segment_mq(n_q_heads / n_kv_heads, q_len) * q_len;
  *bytes = workspace_for(di.sm_count * kConsumerWarps, kDefaultSubChunks, rows, head_dim);
  return PKV_OK;
}

pkv_status paged_attention_decode_mq(const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                                     const int32_t* context_lens, int32_t batch, int32_t q_len, int32_t num_blocks,
                                     float scale, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                     int32_t block_size, void* out, pkv_dtype dtype, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  return decode_impl(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, batch, num_blocks, scale,
                     n_q_heads, n_kv_heads, head_dim, block_size, out, dtype, workspace, workspace_bytes, stream,
                     nullptr, nullptr, nullptr, 0, nullptr, q_len);
}

// ---------------------------------------------------------------------------
// Decode without any allocation: the split-context scratch lives in a
// file-scope device array instead of caller or library allocations.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_pkv_static_workspace[PKV_STATIC_WORKSPACE_BYTES];

namespace {
std::mutex g_static_mutex;
void* g_static_workspace_ptr[kMaxDevices] = {};

// Device address of the static array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
pkv_status static_workspace(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (g_static_workspace_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_pkv_static_workspace) != cudaSuccess || ptr == nullptr) return PKV_ERR_CUDA;
    g_static_workspace_ptr[dev] = ptr;
  }
  *out = g_static_workspace_ptr[dev];
  return PKV_OK;
}
}  // namespace

pkv_status paged_attention_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                          const int32_t* block_tables, int32_t max_blocks_per_seq,
                                          const int32_t* context_lens, int32_t batch, int32_t num_blocks,
                                          float scale, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                          int32_t block_size, void* out, pkv_dtype dtype, void* stream) {
  pkv_status st = check_decode_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, batch,
                                    num_blocks, scale, n_q_heads, n_kv_heads, head_dim, block_size, out, dtype);
  if (st != PKV_OK || batch == 0) return st;
  if (n_q_heads % n_kv_heads != 0) return PKV_ERR_INVALID_ARG;
  DeviceInfo di;
  if (device_info(&di) != PKV_OK) return PKV_ERR_CUDA;
  const int gp = heads_per_segment(n_q_heads / n_kv_heads, dtype, false);
  if (workspace_for(di.sm_count * kConsumerWarps, kDefaultSubChunks, gp, head_dim) > PKV_STATIC_WORKSPACE_BYTES)
    return PKV_ERR_WORKSPACE;
  void* ws = nullptr;
  st = static_workspace(&ws);
  if (st != PKV_OK) return st;
  return paged_attention_decode_ex(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, batch,
                                   num_blocks, scale, n_q_heads, n_kv_heads, head_dim, block_size, out, dtype, ws,
                                   PKV_STATIC_WORKSPACE_BYTES, stream, nullptr);
}

pkv_status paged_attention_cascade_workspace_size(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                                  int32_t head_dim, pkv_dtype dtype, size_t* bytes) {
  size_t dec = 0;
  const pkv_status st = paged_attention_workspace_size(batch, n_q_heads, n_kv_heads, head_dim, dtype, &dec);
  if (st != PKV_OK) return st;
  *bytes = prefix_init_bytes(batch, n_q_heads, head_dim) + dec;
  return PKV_OK;
}

pkv_status paged_attention_decode_cascade(const void* q, const void* k_cache, const void* v_cache, int32_t n_groups,
                                          const int32_t* prefix_block_tables, int32_t max_prefix_blocks,
                                          const int32_t* prefix_lens, const int32_t* seq_group,
                                          const int32_t* block_tables, int32_t max_blocks_per_seq,
                                          const int32_t* context_lens, int32_t batch, int32_t num_blocks,
                                          float scale, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                          int32_t block_size, void* out, pkv_dtype dtype, void* workspace,
                                          size_t workspace_bytes, void* stream) {
  return paged_attention_decode_cascade_ex(q, k_cache, v_cache, n_groups, prefix_block_tables, max_prefix_blocks,
                                           prefix_lens, seq_group, block_tables, max_blocks_per_seq, context_lens,
                                           batch, num_blocks, scale, n_q_heads, n_kv_heads, head_dim, block_size, out,
                                           dtype, workspace, workspace_bytes, stream, nullptr);
}

pkv_status paged_attention_decode_cascade_ex(const void* q, const void* k_cache, const void* v_cache,
                                             int32_t n_groups, const int32_t* prefix_block_tables,
                                             int32_t max_prefix_blocks, const int32_t* prefix_lens,
                                             const int32_t* seq_group, const int32_t* block_tables,
                                             int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t batch,
                                             int32_t num_blocks, float scale, int32_t n_q_heads, int32_t n_kv_heads,
                                             int32_t head_dim, int32_t block_size, void* out, pkv_dtype dtype,
                                             void* workspace, size_t workspace_bytes, void* stream,
                                             const pkv_cascade_options* options) {
  pkv_cascade_options opt = {};
  if (options) opt = *options;
  if (opt.prefix_splits < 0 || opt.prefix_splits > kTcMaxSplit || opt.prefix_kernel < 0 || opt.prefix_kernel > 2)
    return PKV_ERR_INVALID_ARG;
  for (int i = 0; i < 6; ++i)
    if (opt.reserved[i] != 0) return PKV_ERR_INVALID_ARG;
  pkv_status st = check_decode_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, batch,
                                    num_blocks, scale, n_q_heads, n_kv_heads, head_dim, block_size, out, dtype);
  if (st != PKV_OK || batch == 0) return st;
  if (n_groups < 0 || n_groups > 65535) return PKV_ERR_INVALID_ARG;
  if (dtype == PKV_F32) return PKV_ERR_UNSUPPORTED;  // the prefix GEMM runs on 16-bit tensor-core operands
  if (n_groups > 0 && (!prefix_block_tables || !prefix_lens || !seq_group || max_prefix_blocks <= 0 ||
                       max_prefix_blocks > (1 << 26)))
    return PKV_ERR_INVALID_ARG;
  if (n_groups == 0)
    return decode_impl(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, batch, num_blocks,
                       scale, n_q_heads, n_kv_heads, head_dim, block_size, out, dtype, workspace, workspace_bytes,
                       stream, nullptr, nullptr, nullptr, 0);
  DeviceInfo di;
  if (device_info(&di) != PKV_OK) return PKV_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  size_t need = 0;
  st = paged_attention_cascade_workspace_size(batch, n_q_heads, n_kv_heads, head_dim, dtype, &need);
  if (st != PKV_OK) return st;
  void* ws = workspace;
  bool own = false;
  const size_t init_bytes = prefix_init_bytes(batch, n_q_heads, head_dim);
  if (ws == nullptr) {
    if (cudaMallocAsync(&ws, need, s) != cudaSuccess) return PKV_ERR_CUDA;
    own = true;
    // The decode part's scheduling counter starts at zero.
    if (cudaMemsetAsync(static_cast<uint8_t*>(ws) + init_bytes, 0, kSchedBytes, s) != cudaSuccess) {
      cudaFreeAsync(ws, s);
      return PKV_ERR_CUDA;
    }
  } else if (workspace_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) {
    return PKV_ERR_WORKSPACE;
  }
  float* init = static_cast<float*>(ws);

  CUtensorMap mk, mv;
  st = cached_map(kMapBox, &mk, k_cache, dtype, num_blocks, n_kv_heads, head_dim);
  if (st == PKV_OK) st = cached_map(kMapBox, &mv, v_cache, dtype, num_blocks, n_kv_heads, head_dim);
  PrefixParams pp;
  pp.q = q;
  pp.prefix_tables = prefix_block_tables;
  pp.prefix_lens = prefix_lens;
  pp.seq_group = seq_group;
  pp.init = init;
  pp.batch = batch;
  pp.n_groups = n_groups;
  pp.max_prefix_blocks = max_prefix_blocks;
  pp.num_blocks = num_blocks;
  pp.n_q_heads = n_q_heads;
  pp.group = n_q_heads / n_kv_heads;
  pp.stages = kPrefixStages;
  pp.scale_log2 = scale * 1.4426950408889634f;
  const size_t stage_bytes = static_cast<size_t>(2) * kPrefixBlocks * (head_dim * 2 / 128) * kBoxBytes;
  const size_t smem = 1024 + kPrefixStages * (stage_bytes + 2 * sizeof(uint64_t)) + 16 + static_cast<size_t>(batch) * 4;
  // Head dim 128 runs on the tensor-memory kernel when its operands fit (and
  // its K map's block x kv-head coordinate fits 32 bits).
  const bool tc_fits = head_dim == 128 && prefix_tc_smem(batch) + 256 <= static_cast<size_t>(di.smem_optin) &&
                       static_cast<int64_t>(num_blocks) * n_kv_heads < (int64_t(1) << 31);
  if (opt.prefix_kernel == 1 && !tc_fits && st == PKV_OK) st = PKV_ERR_UNSUPPORTED;  // the owned workspace is freed below
  const bool tc = tc_fits && opt.prefix_kernel != 2;
  if (!tc && smem + 256 > static_cast<size_t>(di.smem_optin)) st = st == PKV_OK ? PKV_ERR_UNSUPPORTED : st;
  if (st == PKV_OK && tc) {
    CUtensorMap mk_groups, mv_tile;
    st = cached_map(kMapKGroups, &mk_groups, k_cache, dtype, num_blocks, n_kv_heads, head_dim);
    if (st == PKV_OK) st = cached_map(kMapTile, &mv_tile, v_cache, dtype, num_blocks, n_kv_heads, head_dim);
    if (st == PKV_OK)
      st = dtype == PKV_F16
               ? launch_prefix_tc<kF16>(mk_groups, mv_tile, pp, n_kv_heads, opt.prefix_splits, di.sm_count, s)
               : launch_prefix_tc<kBF16>(mk_groups, mv_tile, pp, n_kv_heads, opt.prefix_splits, di.sm_count, s);
  } else if (st == PKV_OK) {
    if (dtype == PKV_F16)
      st = head_dim == 64 ? launch_prefix<kF16, 64>(mk, mv, pp, n_kv_heads, smem, s)
                          : launch_prefix<kF16, 128>(mk, mv, pp, n_kv_heads, smem, s);
    else
      st = head_dim == 64 ? launch_prefix<kBF16, 64>(mk, mv, pp, n_kv_heads, smem, s)
                          : launch_prefix<kBF16, 128>(mk, mv, pp, n_kv_heads, smem, s);
  }
  if (st == PKV_OK)
    st = decode_impl(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, batch, num_blocks, scale,
                     n_q_heads, n_kv_heads, head_dim, block_size, out, dtype, static_cast<uint8_t*>(ws) + init_bytes,
                     need - init_bytes, stream, nullptr, init, seq_group, n_groups);
  if (own && cudaFreeAsync(ws, s) != cudaSuccess && st == PKV_OK) st = PKV_ERR_CUDA;
  return st;
}

pkv_status pkv_get_device_error(void* stream, uint32_t* flags) {
  if (!flags) return PKV_ERR_INVALID_ARG;
  *flags = 0;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PKV_ERR_CUDA;
  uint32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof v) != cudaSuccess) return PKV_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero) != cudaSuccess) return PKV_ERR_CUDA;
  *flags = v;
  return v ? PKV_ERR_OUT_OF_RANGE : PKV_OK;
}

}  // extern "C"
