// C ABI of libparallax.so (declared in include/parallax.h): argument checks,
// the split-count heuristic, TMA descriptor encoding and kernel launches.
// The host never synchronises and never allocates; every launch goes to the
// caller's stream.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <map>
#include <mutex>
#include <tuple>

#include "parallax.h"
#include "parallax_testing.h"

#include "common.cuh"
#include "kernel_cluster.cuh"
#include "kernel_copy.cuh"
#include "kernel_generic.cuh"
#include "kernel_merge.cuh"
#include "kernel_prefill.cuh"
#include "kernel_tc.cuh"

using namespace plx;

namespace {

constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait
constexpr long long kMinKeysPerSplit = 128;  // smallest key range worth a TMA-kernel CTA (two tiles)
// The generic kernel walks a CTA's keys in serial chunks of 32, so it takes
// ranges half as long (the fp32 tiny decode: 17.8 us per step at 128 keys
// per split, 11.5 us at 64; the TMA kernel is faster at 128: 6.6 vs 6.9 us
// for 8192 keys).
constexpr long long kMinKeysPerSplitGeneric = 64;
constexpr int kCtasPerSm = 1;                // split-KV CTAs per SM (a 96-128 KB ring each)

struct Call {
  int phases;  // bit 0: split-KV kernel, bit 1: merge kernel
  bool probe;
  const void *q, *r, *k, *v;
  const int32_t* seqlens;
  void* out;
  int B, Hq, Hkv, D;
  float scale;
  cudaStream_t stream;
  int Lmax, in_dtype, out_dtype, num_splits;
  void* ws;
  size_t ws_bytes;
  int kv_layout, window;
  unsigned long long timeout_ns;
  int debug_skip_first_tile;
  // paged / block-sparse rows (partition.cuh, KvMode)
  int kv_mode;
  const int32_t* table;  // page ids or block ids, [B][table_stride]
  int table_stride;
  const int32_t* num_blocks;
  int page_size, num_pages;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// SM count of the current device, cached per device (host threads may call
// concurrently: the cache entries are atomics).
int current_sm_count(int* out) {
  static std::atomic<int> cache[256];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PARALLAX_ERR_CUDA;
  if (dev >= 0 && dev < 256) {
    const int n = cache[dev].load(std::memory_order_relaxed);
    if (n > 0) {
      *out = n;
      return PARALLAX_OK;
    }
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
    return PARALLAX_ERR_CUDA;
  if (dev >= 0 && dev < 256) cache[dev].store(n, std::memory_order_relaxed);
  *out = n;
  return PARALLAX_OK;
}

// PARALLAX_SPLITS (a positive integer, read once per process) overrides the
// split heuristic, for experiments; 0 when unset or invalid.
int env_splits() {
  static const int value = [] {
    const char* e = std::getenv("PARALLAX_SPLITS");
    const long v = e ? std::strtol(e, nullptr, 10) : 0;
    return (v > 0 && v <= PARALLAX_MAX_SPLITS) ? (int)v : 0;
  }();
  return value;
}

// PARALLAX_CLUSTER (read once per process), for experiments: a value in
// 2..16 forces that cluster size on the cluster path, -1 turns the cluster
// path off; 0 when unset or invalid (the occupancy-based choice).
int env_cluster() {
  static const int value = [] {
    const char* e = std::getenv("PARALLAX_CLUSTER");
    const long v = e ? std::strtol(e, nullptr, 10) : 0;
    return (v == -1 || (v >= 2 && v <= 16)) ? (int)v : 0;
  }();
  return value;
}

int choose_splits_impl(int B, int Hkv, int Lmax, int sm_count,
                       long long keys_per_split = kMinKeysPerSplit) {
  if (env_splits() > 0) return env_splits();
  const long long max_keys = (long long)B * Hkv * Lmax;
  const long long slots = (long long)kCtasPerSm * sm_count;
  const long long by_work = std::max(1LL, (max_keys + keys_per_split - 1) / keys_per_split);
  return (int)std::min(slots, by_work);
}

bool shape_ok(int B, int Hq, int Hkv, int D, int Lmax) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Lmax < 1 || D < 1) return false;
  if (Hq % Hkv != 0) return false;
  if (Hq / Hkv > kMergeMaxG) return false;  // query heads per kv head
  if ((long long)B * Hkv > 0x7fffffffLL) return false;     // TMA item coordinate is int32
  if ((long long)Hkv * Lmax > 0x7fffffffLL) return false;  // key offsets inside a batch row
  return true;
}

size_t workspace_bytes_for(int G, int D, int P) {
  return kWorkspaceHeaderBytes + (size_t)2 * P * G * rec_floats(D) * sizeof(float);
}

int effective_len(int Lmax, int window) { return window > 0 && window < Lmax ? window : Lmax; }

// num_splits, or for 0 the default of the kernel the call runs on (generic:
// the generic kernel's finer split, which is also what the workspace size
// function plans for, so that one workspace fits either kernel).
int resolve_splits(int num_splits, int B, int Hkv, int Lmax, bool generic, int* P) {
  if (num_splits < 0 || num_splits > PARALLAX_MAX_SPLITS) return PARALLAX_ERR_BAD_SPLITS;
  if (num_splits > 0) {
    *P = num_splits;
    return PARALLAX_OK;
  }
  int sm = 0;
  const int st = current_sm_count(&sm);
  if (st != PARALLAX_OK) return st;
  *P = choose_splits_impl(B, Hkv, Lmax, sm, generic ? kMinKeysPerSplitGeneric : kMinKeysPerSplit);
  return PARALLAX_OK;
}

// Keys per row the partition heuristic plans for.
int planned_len(const Call& c) {
  if (c.kv_mode == kKvPaged) return c.table_stride * c.page_size;
  if (c.kv_mode == kKvBlockSparse) return c.table_stride * kTileKeys;
  return effective_len(c.Lmax, c.window);
}

int validate(const Call& c) {
  if (!c.q || !c.k || !c.v || !c.out || !c.ws) return PARALLAX_ERR_NULL_POINTER;
  if (c.kv_mode != kKvContiguous) {
    if (!c.table || (c.kv_mode == kKvBlockSparse && !c.num_blocks)) return PARALLAX_ERR_NULL_POINTER;
    if ((reinterpret_cast<uintptr_t>(c.table) & 3u) ||
        (reinterpret_cast<uintptr_t>(c.num_blocks) & 3u))
      return PARALLAX_ERR_MISALIGNED;
    if (c.table_stride < 1 || c.window != 0) return PARALLAX_ERR_BAD_SHAPE;
    if (c.kv_mode == kKvPaged &&
        (c.page_size < kTileKeys || c.page_size % kTileKeys != 0 || c.num_pages < 1 ||
         (long long)c.table_stride * c.page_size > 0x7fffffffLL))
      return PARALLAX_ERR_BAD_SHAPE;
    if (c.kv_mode == kKvBlockSparse && (long long)c.table_stride * kTileKeys > 0x7fffffffLL)
      return PARALLAX_ERR_BAD_SHAPE;
  }
  if (c.probe && !c.r) return PARALLAX_ERR_NULL_POINTER;
  if (!shape_ok(c.B, c.Hq, c.Hkv, c.D, c.Lmax)) return PARALLAX_ERR_BAD_SHAPE;
  if ((c.kv_layout != PARALLAX_KV_BHSD && c.kv_layout != PARALLAX_KV_BSHD) || c.window < 0)
    return PARALLAX_ERR_BAD_SHAPE;
  if (c.D != 64 && c.D != 128) return PARALLAX_ERR_UNSUPPORTED_HEAD_DIM;
  if ((c.in_dtype != PARALLAX_DTYPE_BF16 && c.in_dtype != PARALLAX_DTYPE_F32) ||
      (c.out_dtype != PARALLAX_DTYPE_BF16 && c.out_dtype != PARALLAX_DTYPE_F32))
    return PARALLAX_ERR_UNSUPPORTED_DTYPE;
  if (!aligned16(c.q) || (c.probe && !aligned16(c.r)) || !aligned16(c.k) || !aligned16(c.v) ||
      !aligned16(c.out) || !aligned16(c.ws) || (reinterpret_cast<uintptr_t>(c.seqlens) & 3u))
    return PARALLAX_ERR_MISALIGNED;
  if (c.num_splits < 0 || c.num_splits > PARALLAX_MAX_SPLITS) return PARALLAX_ERR_BAD_SPLITS;
  return PARALLAX_OK;
}

// --------------------------------------------------------- TMA descriptors --

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// Element strides of (batch row, kv head, key) in a cache of either layout.
struct KvStrides {
  long long b, h, k;
};
KvStrides kv_strides(int layout, int Hkv, int Lmax, int D) {
  if (layout == PARALLAX_KV_BSHD)
    return {(long long)Lmax * Hkv * D, (long long)D, (long long)Hkv * D};
  return {(long long)Hkv * Lmax * D, (long long)Lmax * D, (long long)D};
}

// A bf16 cache of either layout viewed as {64 dims, Lmax keys, D/64 halves,
// Hkv heads, B rows}: one box of 64 keys x D dims lands as D/64 swizzled
// [64 keys][128 bytes] blocks, one per 64-dim half.
int encode_cache_map(CUtensorMap* map, const void* cache, int D, int Lmax, int Hkv, int B,
                     int layout) {
  auto enc = tensor_map_encoder();
  if (!enc) return PARALLAX_ERR_CUDA;
  const KvStrides st = kv_strides(layout, Hkv, Lmax, D);
  cuuint64_t dims[5] = {64, (cuuint64_t)Lmax, (cuuint64_t)(D / 64), (cuuint64_t)Hkv,
                        (cuuint64_t)B};
  cuuint64_t strides[4] = {(cuuint64_t)st.k * 2, 128, (cuuint64_t)st.h * 2, (cuuint64_t)st.b * 2};
  cuuint32_t box[5] = {64, (cuuint32_t)kTileKeys, (cuuint32_t)(D / 64), 1, 1};
  cuuint32_t elem[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(cache), dims,
                   strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PARALLAX_OK : PARALLAX_ERR_CUDA;
}

// ----------------------------------------------------------------- launch --

// Raises the kernel's dynamic shared-memory limit once per device (the
// attribute call is idempotent, so two threads racing here both succeed).
template <typename Kernel>
int set_smem_once(Kernel kernel, int bytes, std::atomic<int>* done_dev) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PARALLAX_ERR_CUDA;
  if (dev >= 0 && dev < 256 && done_dev[dev].load(std::memory_order_acquire) >= bytes)
    return PARALLAX_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return PARALLAX_ERR_CUDA;
  if (dev >= 0 && dev < 256) done_dev[dev].store(bytes, std::memory_order_release);
  return PARALLAX_OK;
}

template <int D, bool PROBE, bool OUT_F32>
int launch_tc(const Call& c, const DecodeParams& prm, int P) {
  // probabilities as bf16 hi + lo: always with the probe, else for fp32 output
  constexpr bool kPsplit = PROBE || OUT_F32;
  auto kernel = parallax_tc_kernel<D, PROBE, OUT_F32, kPsplit>;
  static std::atomic<int> done[256];
  const TcSmemLayout L =
      tc_smem_layout(D, TcGeom<D>::kStageBytes, TcGeom<D>::kStages, prm.G, PROBE);
  int st = set_smem_once(kernel, L.total, done);
  if (st != PARALLAX_OK) return st;
  CUtensorMap tmK, tmV;
  // paged: the page pool [num_pages][page_size][Hkv][D] is a cache of num_pages
  // rows of page_size keys in the (B, L, H, D) layout
  const bool paged = c.kv_mode == kKvPaged;
  const int rows = paged ? c.num_pages : c.B, len = paged ? c.page_size : c.Lmax;
  const int layout = paged ? PARALLAX_KV_BSHD : c.kv_layout;
  if ((st = encode_cache_map(&tmK, c.k, D, len, c.Hkv, rows, layout)) != PARALLAX_OK) return st;
  if ((st = encode_cache_map(&tmV, c.v, D, len, c.Hkv, rows, layout)) != PARALLAX_OK) return st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)P);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = (size_t)L.total;
  cfg.stream = c.stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, tmK, tmV, prm) == cudaSuccess ? PARALLAX_OK
                                                                        : PARALLAX_ERR_CUDA;
}

template <typename T, int D, bool PROBE, bool OUT_F32>
int launch_generic(const Call& c, const DecodeParams& prm, int P) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)P);
  cfg.blockDim = dim3(kGenericThreads);
  cfg.stream = c.stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, parallax_generic_kernel<T, D, PROBE, OUT_F32>, prm) == cudaSuccess
             ? PARALLAX_OK
             : PARALLAX_ERR_CUDA;
}

template <bool PROBE, bool OUT_F32>
int launch_merge(const Call& c, const DecodeParams& prm, int P) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)P, (unsigned)merge_slices(prm.G, prm.D, PROBE));
  cfg.blockDim = dim3(kMergeThreads);
  cfg.stream = c.stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, parallax_merge_kernel<PROBE, OUT_F32>, prm) == cudaSuccess
             ? PARALLAX_OK
             : PARALLAX_ERR_CUDA;
}

// ------------------------------------------------------- cluster path --

bool tma_path(const Call& c);

// Dynamic shared memory of the cluster kernel for a group of G query heads
// and clusters of S CTAs.
template <int D>
int cluster_smem_bytes(int G, int S) {
  return cluster_layout(TcGeom<D>::kStageBytes, ClusterGeom<D>::kStages, G, D, S).total;
}

// Raises the kernel's shared-memory limit and allows clusters above the
// portable size of 8, once per device.
template <typename Kernel>
int prepare_cluster_kernel(Kernel kernel, int smem, std::atomic<int>* done_dev) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PARALLAX_ERR_CUDA;
  if (dev >= 0 && dev < 256 && done_dev[dev].load(std::memory_order_acquire) >= smem)
    return PARALLAX_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
          cudaSuccess)
    return PARALLAX_ERR_CUDA;
  if (dev >= 0 && dev < 256) done_dev[dev].store(smem, std::memory_order_release);
  return PARALLAX_OK;
}

template <int D, bool PROBE, bool OUT_F32>
auto cluster_kernel() {
  return parallax_cluster_kernel<D, PROBE, OUT_F32, PROBE || OUT_F32>;
}

template <int D, bool PROBE, bool OUT_F32>
std::atomic<int>* cluster_prepared() {
  static std::atomic<int> done[256];
  return done;
}

// How many clusters of S CTAs of this kernel the current device holds at once
// (cudaOccupancyMaxActiveClusters), cached per device, kernel, G and S.
template <int D, bool PROBE, bool OUT_F32>
int max_active_clusters(int G, int S, int* out) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PARALLAX_ERR_CUDA;
  const auto key = std::make_tuple(dev, G, S);
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *out = it->second;
      return PARALLAX_OK;
    }
  }
  auto kernel = cluster_kernel<D, PROBE, OUT_F32>();
  const int smem = cluster_smem_bytes<D>(G, S);
  int st = prepare_cluster_kernel(kernel, smem, cluster_prepared<D, PROBE, OUT_F32>());
  if (st != PARALLAX_OK) return st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)S);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;  // a size the device can not run: never chosen
  }
  std::lock_guard<std::mutex> lock(mu);
  cache[key] = n;
  *out = n;
  return PARALLAX_OK;
}

template <int D, bool PROBE, bool OUT_F32>
int choose_cluster_impl(int items, int G, int sm, int* S_out) {
  *S_out = 0;
  if (items < 1 || items > sm / 2) return PARALLAX_OK;
  for (int S = std::min(kClusterAuto, sm / items); S >= 2; --S) {
    int n = 0;
    const int st = max_active_clusters<D, PROBE, OUT_F32>(G, S, &n);
    if (st != PARALLAX_OK) return st;
    if (n >= items) {
      *S_out = S;
      return PARALLAX_OK;
    }
  }
  return PARALLAX_OK;
}

// The cluster size a call runs with (0: the split-KV + merge path). The
// cluster path takes the TMA kernel's inputs (bf16 caches of any key space:
// contiguous rows with or without a window, paged, block-sparse) with the
// default split (num_splits = 0), when every (batch row, kv head) item can
// have a cluster of at least two CTAs resident at once.
int cluster_plan(const Call& c, int* S) {
  *S = 0;
  if (c.phases != 3 || c.num_splits != 0 || env_splits() > 0 || env_cluster() < 0 ||
      !tma_path(c))
    return PARALLAX_OK;
  int sm = 0;
  int st = current_sm_count(&sm);
  if (st != PARALLAX_OK) return st;
  const long long items = (long long)c.B * c.Hkv;
  if (items > sm / 2) return PARALLAX_OK;
  if (env_cluster() > 0) {
    *S = env_cluster();
    return PARALLAX_OK;
  }
  const int G = c.Hq / c.Hkv, it = (int)items;
  const bool f32 = c.out_dtype == PARALLAX_DTYPE_F32;
  if (c.D == 128) {
    if (c.probe) return f32 ? choose_cluster_impl<128, true, true>(it, G, sm, S)
                            : choose_cluster_impl<128, true, false>(it, G, sm, S);
    return f32 ? choose_cluster_impl<128, false, true>(it, G, sm, S)
               : choose_cluster_impl<128, false, false>(it, G, sm, S);
  }
  if (c.probe) return f32 ? choose_cluster_impl<64, true, true>(it, G, sm, S)
                          : choose_cluster_impl<64, true, false>(it, G, sm, S);
  return f32 ? choose_cluster_impl<64, false, true>(it, G, sm, S)
             : choose_cluster_impl<64, false, false>(it, G, sm, S);
}

template <int D, bool PROBE, bool OUT_F32>
int launch_cluster(const Call& c, const DecodeParams& prm, int S) {
  auto kernel = cluster_kernel<D, PROBE, OUT_F32>();
  const int smem = cluster_smem_bytes<D>(prm.G, S);
  int st = prepare_cluster_kernel(kernel, smem, cluster_prepared<D, PROBE, OUT_F32>());
  if (st != PARALLAX_OK) return st;
  CUtensorMap tmK, tmV;
  // a paged pool is viewed as a (kv_len, H, D) cache of page_size keys per page
  const bool paged = c.kv_mode == kKvPaged;
  const int rows = paged ? c.num_pages : c.B, len = paged ? c.page_size : c.Lmax;
  const int layout = paged ? PARALLAX_KV_BSHD : c.kv_layout;
  if ((st = encode_cache_map(&tmK, c.k, D, len, c.Hkv, rows, layout)) != PARALLAX_OK) return st;
  if ((st = encode_cache_map(&tmV, c.v, D, len, c.Hkv, rows, layout)) != PARALLAX_OK) return st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(c.B * c.Hkv * S));
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = c.stream;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, tmK, tmV, prm) == cudaSuccess ? PARALLAX_OK
                                                                        : PARALLAX_ERR_CUDA;
}

template <bool PROBE, bool OUT_F32>
int run_cluster(const Call& c, const DecodeParams& prm, int S) {
  return c.D == 128 ? launch_cluster<128, PROBE, OUT_F32>(c, prm, S)
                    : launch_cluster<64, PROBE, OUT_F32>(c, prm, S);
}

// The TMA kernel takes bf16 caches whose GQA group (q and r rows with the
// probe) fits its 8 mma columns; everything else runs on the generic kernel.
bool tma_path(const Call& c) {
  const int G = c.Hkv > 0 ? c.Hq / c.Hkv : 0;
  return c.in_dtype == PARALLAX_DTYPE_BF16 && (c.probe ? 2 * G <= 8 : G <= 8);
}

template <bool PROBE, bool OUT_F32>
int launch_split_kv(const Call& c, const DecodeParams& prm, int P) {
  if (tma_path(c)) {
    if (c.D == 128) return launch_tc<128, PROBE, OUT_F32>(c, prm, P);
    return launch_tc<64, PROBE, OUT_F32>(c, prm, P);
  }
  if (c.in_dtype == PARALLAX_DTYPE_BF16)
    return c.D == 128 ? launch_generic<__nv_bfloat16, 128, PROBE, OUT_F32>(c, prm, P)
                      : launch_generic<__nv_bfloat16, 64, PROBE, OUT_F32>(c, prm, P);
  return c.D == 128 ? launch_generic<float, 128, PROBE, OUT_F32>(c, prm, P)
                    : launch_generic<float, 64, PROBE, OUT_F32>(c, prm, P);
}

template <bool PROBE, bool OUT_F32>
int run_phases(const Call& c, const DecodeParams& prm, int P) {
  if (c.phases & 1) {
    const int st = launch_split_kv<PROBE, OUT_F32>(c, prm, P);
    if (st != PARALLAX_OK) return st;
  }
  if (c.phases & 2) return launch_merge<PROBE, OUT_F32>(c, prm, P);
  return PARALLAX_OK;
}

int run(const Call& c) {
  int st = validate(c);
  if (st != PARALLAX_OK) return st;
  int S = 0;
  if ((st = cluster_plan(c, &S)) != PARALLAX_OK) return st;
  int P = 0;
  if (S == 0 &&
      (st = resolve_splits(c.num_splits, c.B, c.Hkv, planned_len(c), !tma_path(c), &P)) !=
          PARALLAX_OK)
    return st;
  const int G = c.Hq / c.Hkv;
  if (c.ws_bytes < (S > 0 ? kWorkspaceHeaderBytes : workspace_bytes_for(G, c.D, P)))
    return PARALLAX_ERR_WORKSPACE_TOO_SMALL;

  DecodeParams prm{};
  prm.q = c.q;
  prm.r = c.probe ? c.r : nullptr;
  prm.k = c.k;
  prm.v = c.v;
  // a paged pool [pages][page_size][Hkv][D] is a (kv_len, H, D) cache of
  // page_size keys per page (the TMA kernel's tensor map views it the same way)
  const KvStrides kst = c.kv_mode == kKvPaged
                            ? kv_strides(PARALLAX_KV_BSHD, c.Hkv, c.page_size, c.D)
                            : kv_strides(c.kv_layout, c.Hkv, c.Lmax, c.D);
  prm.kv_sb = kst.b;
  prm.kv_sh = kst.h;
  prm.kv_sk = kst.k;
  prm.seqlens = c.seqlens;
  prm.window = c.window;
  prm.out = c.out;
  prm.status = static_cast<unsigned int*>(c.ws);
  prm.partials = reinterpret_cast<float*>(static_cast<char*>(c.ws) + kWorkspaceHeaderBytes);
  prm.B = c.B;
  prm.Hq = c.Hq;
  prm.Hkv = c.Hkv;
  prm.G = G;
  prm.D = c.D;
  prm.Lmax = c.kv_mode == kKvPaged ? c.table_stride * c.page_size : c.Lmax;
  prm.kv_mode = c.kv_mode;
  prm.table = c.table;
  prm.table_stride = c.table_stride;
  prm.num_blocks = c.num_blocks;
  prm.page_size = c.page_size;
  prm.num_pages = c.num_pages;
  prm.scale_log2 = (float)((double)c.scale * 1.4426950408889634);  // log2(e)
  prm.timeout_ns = c.timeout_ns;
  prm.debug_skip_first_tile = c.debug_skip_first_tile;

  const bool f32 = c.out_dtype == PARALLAX_DTYPE_F32;
  if (S > 0) {
    if (c.probe) return f32 ? run_cluster<true, true>(c, prm, S) : run_cluster<true, false>(c, prm, S);
    return f32 ? run_cluster<false, true>(c, prm, S) : run_cluster<false, false>(c, prm, S);
  }
  if (c.probe) return f32 ? run_phases<true, true>(c, prm, P) : run_phases<true, false>(c, prm, P);
  return f32 ? run_phases<false, true>(c, prm, P) : run_phases<false, false>(c, prm, P);
}

Call make_call(int phases, bool probe, const void* q, const void* r, const void* k, const void* v,
               const int32_t* seqlens, void* out, int B, int Hq, int Hkv, int D, float scale,
               void* stream, int Lmax, int in_dtype, int out_dtype, int num_splits, void* ws,
               size_t ws_bytes) {
  Call c;
  c.phases = phases;
  c.probe = probe;
  c.q = q;
  c.r = r;
  c.k = k;
  c.v = v;
  c.seqlens = seqlens;
  c.out = out;
  c.B = B;
  c.Hq = Hq;
  c.Hkv = Hkv;
  c.D = D;
  c.scale = scale;
  c.stream = static_cast<cudaStream_t>(stream);
  c.Lmax = Lmax;
  c.in_dtype = in_dtype;
  c.out_dtype = out_dtype;
  c.num_splits = num_splits;
  c.ws = ws;
  c.ws_bytes = ws_bytes;
  c.kv_layout = PARALLAX_KV_BHSD;
  c.window = 0;
  c.timeout_ns = kDefaultTimeoutNs;
  c.debug_skip_first_tile = 0;
  c.kv_mode = kKvContiguous;
  c.table = nullptr;
  c.table_stride = 0;
  c.num_blocks = nullptr;
  c.page_size = 0;
  c.num_pages = 0;
  return c;
}

}  // namespace

extern "C" {

int parallax_choose_splits(int B, int Hkv, int Lmax, int sm_count) {
  if (B < 1 || Hkv < 1 || Lmax < 1) return PARALLAX_ERR_BAD_SHAPE;
  if (sm_count <= 0) {
    const int st = current_sm_count(&sm_count);
    if (st != PARALLAX_OK) return st;
  }
  return choose_splits_impl(B, Hkv, Lmax, sm_count);
}

int parallax_default_splits(int B, int Hq, int Hkv, int Lmax, int in_dtype, int probe,
                            int sm_count) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Lmax < 1 || Hq % Hkv != 0) return PARALLAX_ERR_BAD_SHAPE;
  if (in_dtype != PARALLAX_DTYPE_BF16 && in_dtype != PARALLAX_DTYPE_F32)
    return PARALLAX_ERR_UNSUPPORTED_DTYPE;
  if (sm_count <= 0) {
    const int st = current_sm_count(&sm_count);
    if (st != PARALLAX_OK) return st;
  }
  Call c{};
  c.Hq = Hq;
  c.Hkv = Hkv;
  c.in_dtype = in_dtype;
  c.probe = probe != 0;
  return choose_splits_impl(B, Hkv, Lmax, sm_count,
                            tma_path(c) ? kMinKeysPerSplit : kMinKeysPerSplitGeneric);
}

int parallax_decode_plan(int B, int Hq, int Hkv, int D, int Lmax, int in_dtype, int out_dtype,
                         int probe, int* grid_ctas, int* cluster_ctas) {
  if (!grid_ctas || !cluster_ctas) return PARALLAX_ERR_NULL_POINTER;
  if (!shape_ok(B, Hq, Hkv, D, Lmax)) return PARALLAX_ERR_BAD_SHAPE;
  if (D != 64 && D != 128) return PARALLAX_ERR_UNSUPPORTED_HEAD_DIM;
  if ((in_dtype != PARALLAX_DTYPE_BF16 && in_dtype != PARALLAX_DTYPE_F32) ||
      (out_dtype != PARALLAX_DTYPE_BF16 && out_dtype != PARALLAX_DTYPE_F32))
    return PARALLAX_ERR_UNSUPPORTED_DTYPE;
  Call c = make_call(3, probe != 0, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, B, Hq,
                     Hkv, D, 1.f, nullptr, Lmax, in_dtype, out_dtype, 0, nullptr, 0);
  int S = 0;
  int st = cluster_plan(c, &S);
  if (st != PARALLAX_OK) return st;
  if (S > 0) {
    *grid_ctas = B * Hkv * S;
    *cluster_ctas = S;
    return PARALLAX_OK;
  }
  int P = 0;
  if ((st = resolve_splits(0, B, Hkv, Lmax, !tma_path(c), &P)) != PARALLAX_OK) return st;
  *grid_ctas = P;
  *cluster_ctas = 0;
  return PARALLAX_OK;
}

size_t parallax_decode_workspace_bytes(int B, int Hq, int Hkv, int D, int Lmax, int num_splits) {
  if (!shape_ok(B, Hq, Hkv, D, Lmax) || (D != 64 && D != 128)) return 0;
  int P = 0;
  if (resolve_splits(num_splits, B, Hkv, Lmax, true, &P) != PARALLAX_OK) return 0;
  return workspace_bytes_for(Hq / Hkv, D, P);
}

int parallax_decode(const void* q, const void* r, const void* k_cache, const void* v_cache,
                    const int32_t* cache_seqlens, void* out, int B, int Hq, int Hkv, int D,
                    float scale, void* stream, int Lmax, int in_dtype, int out_dtype,
                    int num_splits, void* workspace, size_t workspace_bytes) {
  return run(make_call(3, true, q, r, k_cache, v_cache, cache_seqlens, out, B, Hq, Hkv, D, scale,
                       stream, Lmax, in_dtype, out_dtype, num_splits, workspace, workspace_bytes));
}

int parallax_softmax_decode(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* cache_seqlens, void* out, int B, int Hq, int Hkv, int D,
                            float scale, void* stream, int Lmax, int in_dtype, int out_dtype,
                            int num_splits, void* workspace, size_t workspace_bytes) {
  return run(make_call(3, false, q, nullptr, k_cache, v_cache, cache_seqlens, out, B, Hq, Hkv, D,
                       scale, stream, Lmax, in_dtype, out_dtype, num_splits, workspace,
                       workspace_bytes));
}

int parallax_decode_ex(const void* q, const void* r, const void* k_cache, const void* v_cache,
                       const int32_t* cache_seqlens, void* out, int B, int Hq, int Hkv, int D,
                       float scale, void* stream, int Lmax, int in_dtype, int out_dtype,
                       int num_splits, void* workspace, size_t workspace_bytes, int probe,
                       int kv_layout, int window, int phases) {
  if (phases < 1 || phases > 3) return PARALLAX_ERR_BAD_PHASE;
  Call c = make_call(phases, probe != 0, q, r, k_cache, v_cache, cache_seqlens, out, B, Hq, Hkv,
                     D, scale, stream, Lmax, in_dtype, out_dtype, num_splits, workspace,
                     workspace_bytes);
  c.kv_layout = kv_layout;
  c.window = window;
  return run(c);
}

int parallax_decode_paged(const void* q, const void* r, const void* k_pages, const void* v_pages,
                          const int32_t* block_table, const int32_t* cache_seqlens, void* out,
                          int B, int Hq, int Hkv, int D, float scale, void* stream, int num_pages,
                          int page_size, int max_pages_per_seq, int probe, int in_dtype,
                          int out_dtype, int num_splits, void* workspace, size_t workspace_bytes) {
  if (page_size < 1 || max_pages_per_seq < 1) return PARALLAX_ERR_BAD_SHAPE;
  const long long lmax = (long long)page_size * max_pages_per_seq;
  if (lmax > 0x7fffffffLL) return PARALLAX_ERR_BAD_SHAPE;
  Call c = make_call(3, probe != 0, q, r, k_pages, v_pages, cache_seqlens, out, B, Hq, Hkv, D,
                     scale, stream, (int)lmax, in_dtype, out_dtype, num_splits, workspace,
                     workspace_bytes);
  c.kv_mode = kKvPaged;
  c.table = block_table;
  c.table_stride = max_pages_per_seq;
  c.page_size = page_size;
  c.num_pages = num_pages;
  return run(c);
}

int parallax_decode_block_sparse(const void* q, const void* r, const void* k_cache,
                                 const void* v_cache, const int32_t* cache_seqlens,
                                 const int32_t* block_ids, const int32_t* num_blocks, void* out,
                                 int B, int Hq, int Hkv, int D, float scale, void* stream, int Lmax,
                                 int kv_layout, int max_blocks, int probe, int in_dtype,
                                 int out_dtype, int num_splits, void* workspace,
                                 size_t workspace_bytes) {
  Call c = make_call(3, probe != 0, q, r, k_cache, v_cache, cache_seqlens, out, B, Hq, Hkv, D,
                     scale, stream, Lmax, in_dtype, out_dtype, num_splits, workspace,
                     workspace_bytes);
  c.kv_layout = kv_layout;
  c.kv_mode = kKvBlockSparse;
  c.table = block_ids;
  c.table_stride = max_blocks;
  c.num_blocks = num_blocks;
  return run(c);
}

int parallax_decode_phase(int phase, int probe, const void* q, const void* r, const void* k_cache,
                          const void* v_cache, const int32_t* cache_seqlens, void* out, int B,
                          int Hq, int Hkv, int D, float scale, void* stream, int Lmax, int in_dtype,
                          int out_dtype, int num_splits, void* workspace, size_t workspace_bytes) {
  if (phase != 1 && phase != 2) return PARALLAX_ERR_BAD_PHASE;
  return run(make_call(phase, probe != 0, q, r, k_cache, v_cache, cache_seqlens, out, B, Hq, Hkv,
                       D, scale, stream, Lmax, in_dtype, out_dtype, num_splits, workspace,
                       workspace_bytes));
}

}  // extern "C"

namespace {

// The address a kernel on the current device uses for p (for page-locked host
// memory, its mapping into the device's address space), and whether p is host
// memory; false for pageable or unmapped host memory.
bool device_address(const void* p, void** dev, bool* is_host) {
  cudaPointerAttributes attr{};
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  *is_host = attr.type == cudaMemoryTypeHost;
  if (attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged) {
    *dev = const_cast<void*>(p);
    return true;
  }
  if (attr.type != cudaMemoryTypeHost) return false;  // pageable host memory
  if (attr.devicePointer == nullptr) return false;    // not mapped for this device
  *dev = attr.devicePointer;
  return true;
}

}  // namespace

extern "C" {

int parallax_copy(void* dst, const void* src, size_t bytes, void* stream) {
  if (!dst || !src) return PARALLAX_ERR_NULL_POINTER;
  if (!aligned16(dst) || !aligned16(src) || bytes % 16 != 0) return PARALLAX_ERR_MISALIGNED;
  if (bytes == 0) return PARALLAX_OK;
  void *d_dst = nullptr, *d_src = nullptr;
  bool dst_host = false, src_host = false;
  if (!device_address(dst, &d_dst, &dst_host) || !device_address(src, &d_src, &src_host))
    return PARALLAX_ERR_BAD_SHAPE;
  const long long n16 = (long long)(bytes / 16);
  int sm = 0;
  int st = current_sm_count(&sm);
  if (st != PARALLAX_OK) return st;
  const long long want = (n16 + kCopyThreads - 1) / kCopyThreads;
  const unsigned blocks = (unsigned)std::max(1LL, std::min<long long>(want, 4LL * sm));
  parallax_copy_kernel<<<blocks, kCopyThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(d_dst), static_cast<const uint4*>(d_src), n16, dst_host ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? PARALLAX_OK : PARALLAX_ERR_CUDA;
}

int parallax_workspace_status(void* workspace, int clear, uint32_t* device_status) {
  if (!workspace || !device_status) return PARALLAX_ERR_NULL_POINTER;
  uint32_t word = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return PARALLAX_ERR_CUDA;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return PARALLAX_ERR_CUDA;
  if (clear && cudaMemset(workspace, 0, sizeof(word)) != cudaSuccess) return PARALLAX_ERR_CUDA;
  *device_status = word;
  if (word & PARALLAX_DEVICE_STATUS_TIMEOUT) return PARALLAX_ERR_DEVICE_TIMEOUT;
  if (word & PARALLAX_DEVICE_STATUS_SEQLEN_CLAMPED) return PARALLAX_ERR_SEQLEN_CLAMPED;
  return PARALLAX_OK;
}

const char* parallax_status_string(int status) {
  switch (status) {
    case PARALLAX_OK: return "ok";
    case PARALLAX_ERR_NULL_POINTER: return "a required pointer is NULL";
    case PARALLAX_ERR_BAD_SHAPE: return "bad shape (B, Hq, Hkv, Lmax >= 1 and Hq % Hkv == 0 required)";
    case PARALLAX_ERR_UNSUPPORTED_HEAD_DIM: return "unsupported head dimension (64 or 128)";
    case PARALLAX_ERR_UNSUPPORTED_DTYPE: return "unsupported dtype selector";
    case PARALLAX_ERR_MISALIGNED: return "a pointer is not 16-byte aligned";
    case PARALLAX_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case PARALLAX_ERR_BAD_SPLITS: return "num_splits out of range";
    case PARALLAX_ERR_CUDA: return "CUDA runtime error (launch or descriptor encoding)";
    case PARALLAX_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel timed out";
    case PARALLAX_ERR_BAD_PHASE: return "phase must be 1 or 2";
    case PARALLAX_ERR_SEQLEN_CLAMPED: return "a cache_seqlens value was outside [0, Lmax] and was clamped";
    case PARALLAX_ERR_SCRATCH_LIMIT:
      return "the workspace this call needs exceeds PARALLAX_NOALLOC_SCRATCH_BYTES (lower num_splits)";
    default: return "unknown status";
  }
}

}  // extern "C"

// ------------------------------------------------------------- prefill ----
namespace {

// [rows_per_item * items][D] bf16 viewed as {64 dims, L rows, D/64 halves,
// items}: one box of `box_rows` rows x D dims lands as D/64 swizzled
// [box_rows][128 bytes] blocks (the UMMA operand layout).
int encode_rows_map(CUtensorMap* map, const void* base, int D, int L, long long items,
                    int box_rows, CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto enc = tensor_map_encoder();
  if (!enc) return PARALLAX_ERR_CUDA;
  cuuint64_t dims[4] = {64, (cuuint64_t)L, (cuuint64_t)(D / 64), (cuuint64_t)items};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, 128, (cuuint64_t)L * D * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)box_rows, (cuuint32_t)(D / 64), 1};
  cuuint32_t elem[4] = {1, 1, 1, 1};
  CUresult r = enc(map, dtype, 4, const_cast<void*>(base), dims,
                   strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PARALLAX_OK : PARALLAX_ERR_CUDA;
}

// Packed [total][H][D] bf16 viewed as {64 dims, total rows, D/64 halves, H
// heads}: a box of `box_rows` consecutive rows of one head lands in the same
// swizzled layout as encode_rows_map's.
int encode_packed_map(CUtensorMap* map, const void* base, int D, int total, int H,
                      int box_rows, CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto enc = tensor_map_encoder();
  if (!enc) return PARALLAX_ERR_CUDA;
  cuuint64_t dims[4] = {64, (cuuint64_t)total, (cuuint64_t)(D / 64), (cuuint64_t)H};
  cuuint64_t strides[3] = {(cuuint64_t)H * D * 2, 128, (cuuint64_t)D * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)box_rows, (cuuint32_t)(D / 64), 1};
  cuuint32_t elem[4] = {1, 1, 1, 1};
  CUresult r = enc(map, dtype, 4, const_cast<void*>(base), dims,
                   strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PARALLAX_OK : PARALLAX_ERR_CUDA;
}

// Workspace of the bf16-output prefill: the 256-byte header, then (from byte
// 1024) the fp16 copy of V, then one record per (kv item, 64-row block).
// Dense: B batch rows of L keys, items = B * Hkv; packed: B = 1, L = total.
struct PrefillWorkspace {
  size_t v16_off, info_off, total;
  int nblk;
  long long items;
};

PrefillWorkspace prefill_workspace(int B, int L, int Hkv, int D) {
  PrefillWorkspace w{};
  w.nblk = (L + 63) / 64;
  w.items = (long long)B * Hkv;
  w.v16_off = 1024;
  const size_t v16 = (size_t)B * (size_t)L * (size_t)Hkv * (size_t)D * 2;
  w.info_off = w.v16_off + (v16 + 255) / 256 * 256;
  w.total = w.info_off + (size_t)w.items * (size_t)w.nblk * 4;
  return w;
}

// The fp16 copy of V and the per-block records, when the workspace holds
// them (bf16 output only); then the prefill, chained with programmatic
// dependent launch so that its set-up overlaps the end of the copy.
template <int D, bool OUT_F32, bool VARLEN>
int launch_prefill(const void* q, const void* r, const void* k, const void* v,
                   PrefillParams prm, int grid_x, void* workspace, size_t workspace_bytes,
                   cudaStream_t stream) {
  auto kernel = parallax_prefill_kernel<D, OUT_F32, VARLEN>;
  static std::atomic<int> done[256];
  int st = set_smem_once(kernel, PfGeom<D, OUT_F32>::kSmem, done);
  if (st != PARALLAX_OK) return st;
  const int rows = VARLEN ? prm.total : prm.L;
  const PrefillWorkspace w = prefill_workspace(VARLEN ? 1 : prm.B, rows, prm.Hkv, D);
  const long long nprep = w.items * w.nblk;
  const bool use16 = !OUT_F32 && workspace_bytes >= w.total && nprep <= 0x7fffffffLL;
  char* const ws = static_cast<char*>(workspace);
  CUtensorMap tq, tr, tk, tv, tv16;
  const void* src[4] = {q, r, k, v};
  CUtensorMap* maps[4] = {&tq, &tr, &tk, &tv};
  for (int i = 0; i < 4; ++i) {
    const int H = i < 2 ? prm.Hq : prm.Hkv, box = i < 2 ? kPfRows : kPfKeys;
    st = VARLEN ? encode_packed_map(maps[i], src[i], D, prm.total, H, box)
                : encode_rows_map(maps[i], src[i], D, prm.L, (long long)prm.B * H, box);
    if (st != PARALLAX_OK) return st;
  }
  tv16 = tv;
  if (use16) {
    st = VARLEN ? encode_packed_map(&tv16, ws + w.v16_off, D, prm.total, prm.Hkv, kPfKeys,
                                    CU_TENSOR_MAP_DATA_TYPE_FLOAT16)
                : encode_rows_map(&tv16, ws + w.v16_off, D, prm.L, (long long)prm.B * prm.Hkv,
                                  kPfKeys, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    if (st != PARALLAX_OK) return st;
    prm.vinfo = reinterpret_cast<const uint32_t*>(ws + w.info_off);
    prm.nblk = w.nblk;
    dim3 grid((unsigned)w.nblk, 1, 1);
    // one linear index would overflow gridDim.y's 65535 items: blocks in x, items in y and z
    const long long items = w.items;
    grid.y = (unsigned)std::min<long long>(items, 65535);
    grid.z = (unsigned)((items + grid.y - 1) / grid.y);
    if (grid.z > 65535) return PARALLAX_ERR_BAD_SHAPE;
    parallax_prefill_prep_kernel<D, VARLEN><<<grid, 256, 0, stream>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v),
        reinterpret_cast<uint4*>(ws + w.v16_off), reinterpret_cast<uint32_t*>(ws + w.info_off),
        rows, prm.Hkv, w.nblk, (int)grid.y, items);
    if (cudaGetLastError() != cudaSuccess) return PARALLAX_ERR_CUDA;
  } else {
    prm.vinfo = nullptr;
    prm.nblk = 0;
  }
  cudaLaunchConfig_t cfg = {};
  // one linear index over tile slots x Hq x B (slot slowest)
  const long long lin = (long long)grid_x * prm.Hq * prm.B;
  if (lin > 0x7fffffffLL) return PARALLAX_ERR_BAD_SHAPE;
  cfg.gridDim = dim3((unsigned)lin);
  cfg.blockDim = dim3(kPfThreads);
  cfg.dynamicSmemBytes = PfGeom<D, OUT_F32>::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (use16) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kernel, tq, tr, tk, tv, tv16, prm) == cudaSuccess
             ? PARALLAX_OK
             : PARALLAX_ERR_CUDA;
}

template <bool VARLEN>
int dispatch_prefill(const void* q, const void* r, const void* k, const void* v,
                     const PrefillParams& prm, int D, bool f32, int grid_x, void* ws,
                     size_t ws_bytes, cudaStream_t s) {
  if (D == 128)
    return f32 ? launch_prefill<128, true, VARLEN>(q, r, k, v, prm, grid_x, ws, ws_bytes, s)
               : launch_prefill<128, false, VARLEN>(q, r, k, v, prm, grid_x, ws, ws_bytes, s);
  return f32 ? launch_prefill<64, true, VARLEN>(q, r, k, v, prm, grid_x, ws, ws_bytes, s)
             : launch_prefill<64, false, VARLEN>(q, r, k, v, prm, grid_x, ws, ws_bytes, s);
}

// The checks both prefill layouts share.
int check_prefill_args(const void* q, const void* r, const void* k, const void* v, void* out,
                       int Hq, int Hkv, int D, float scale, int out_dtype, void* workspace,
                       size_t workspace_bytes) {
  if (!q || !r || !k || !v || !out || !workspace) return PARALLAX_ERR_NULL_POINTER;
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Hq > 65535) return PARALLAX_ERR_BAD_SHAPE;
  if (!(scale > 0.f) || !(scale < 3.0e38f)) return PARALLAX_ERR_BAD_SHAPE;  // positive, finite
  if (D != 64 && D != 128) return PARALLAX_ERR_UNSUPPORTED_HEAD_DIM;
  if (out_dtype != PARALLAX_DTYPE_BF16 && out_dtype != PARALLAX_DTYPE_F32)
    return PARALLAX_ERR_UNSUPPORTED_DTYPE;
  if (!aligned16(q) || !aligned16(r) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      !aligned16(workspace))
    return PARALLAX_ERR_MISALIGNED;
  if (workspace_bytes < kWorkspaceHeaderBytes) return PARALLAX_ERR_WORKSPACE_TOO_SMALL;
  return PARALLAX_OK;
}

}  // namespace

namespace {

int run_prefill(const void* q, const void* r, const void* k, const void* v, void* out, int B,
                int Hq, int Hkv, int L, int D, float scale, int causal, void* stream,
                int out_dtype, void* workspace, size_t workspace_bytes,
                unsigned long long timeout_ns, int debug_skip_first_k) {
  int st = check_prefill_args(q, r, k, v, out, Hq, Hkv, D, scale, out_dtype, workspace,
                              workspace_bytes);
  if (st != PARALLAX_OK) return st;
  if (B < 1 || L < 1 || B > 65535) return PARALLAX_ERR_BAD_SHAPE;
  PrefillParams prm{};
  prm.out = out;
  prm.status = static_cast<unsigned int*>(workspace);
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = Hq / Hkv;
  prm.L = L;
  prm.num_qt = (L + kPfRows - 1) / kPfRows;
  prm.causal = causal != 0;
  prm.scale_log2 = (float)((double)scale * 1.4426950408889634);
  prm.timeout_ns = timeout_ns;
  prm.debug_skip_first_k = debug_skip_first_k;
  return dispatch_prefill<false>(q, r, k, v, prm, D, out_dtype == PARALLAX_DTYPE_F32,
                                 prm.num_qt, workspace, workspace_bytes,
                                 static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" int parallax_prefill(const void* q, const void* r, const void* k, const void* v,
                                void* out, int B, int Hq, int Hkv, int L, int D, float scale,
                                int causal, void* stream, int out_dtype, void* workspace,
                                size_t workspace_bytes) {
  return run_prefill(q, r, k, v, out, B, Hq, Hkv, L, D, scale, causal, stream, out_dtype,
                     workspace, workspace_bytes, kDefaultTimeoutNs, 0);
}

extern "C" size_t parallax_prefill_workspace_bytes(int B, int L, int Hkv, int D) {
  if (B < 1 || L < 1 || Hkv < 1 || (D != 64 && D != 128)) return 0;
  return prefill_workspace(B, L, Hkv, D).total;
}

extern "C" int parallax_testing_prefill_stalled(const void* q, const void* r, const void* k,
                                                const void* v, void* out, int B, int Hq,
                                                int Hkv, int L, int D, float scale, int causal,
                                                void* stream, int out_dtype, void* workspace,
                                                size_t workspace_bytes, int timeout_ms) {
  if (timeout_ms < 1 || timeout_ms > 10000) return PARALLAX_ERR_BAD_SHAPE;
  return run_prefill(q, r, k, v, out, B, Hq, Hkv, L, D, scale, causal, stream, out_dtype,
                     workspace, workspace_bytes, (unsigned long long)timeout_ms * 1000000ull, 1);
}

extern "C" int parallax_varlen_prefill(const void* q, const void* r, const void* k,
                                       const void* v, const int32_t* cu_seqlens, void* out,
                                       int B, int total_tokens, int max_seqlen, int Hq, int Hkv,
                                       int D, float scale, int causal, void* stream,
                                       int out_dtype, void* workspace, size_t workspace_bytes) {
  int st = check_prefill_args(q, r, k, v, out, Hq, Hkv, D, scale, out_dtype, workspace,
                              workspace_bytes);
  if (st != PARALLAX_OK) return st;
  if (!cu_seqlens) return PARALLAX_ERR_NULL_POINTER;
  if (B < 1 || B > 65535 || total_tokens < 1 || max_seqlen < 1 || max_seqlen > total_tokens)
    return PARALLAX_ERR_BAD_SHAPE;
  PrefillParams prm{};
  prm.out = out;
  prm.status = static_cast<unsigned int*>(workspace);
  prm.cu_seqlens = cu_seqlens;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = Hq / Hkv;
  prm.L = 0;
  prm.num_qt = (max_seqlen + kPfRows - 1) / kPfRows;  // tile slots: the longest sequence's
  prm.total = total_tokens;
  prm.causal = causal != 0;
  prm.scale_log2 = (float)((double)scale * 1.4426950408889634);
  prm.timeout_ns = kDefaultTimeoutNs;
  return dispatch_prefill<true>(q, r, k, v, prm, D, out_dtype == PARALLAX_DTYPE_F32, prm.num_qt,
                                workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

extern "C" int parallax_testing_decode_stalled(const void* q, const void* r, const void* k_cache,
                                               const void* v_cache, const int32_t* cache_seqlens,
                                               void* out, int B, int Hq, int Hkv, int D,
                                               float scale, void* stream, int Lmax,
                                               int num_splits, void* workspace,
                                               size_t workspace_bytes, int timeout_ms) {
  if (timeout_ms < 1 || timeout_ms > 10000) return PARALLAX_ERR_BAD_SHAPE;
  Call c = make_call(3, true, q, r, k_cache, v_cache, cache_seqlens, out, B, Hq, Hkv, D, scale,
                     stream, Lmax, PARALLAX_DTYPE_BF16, PARALLAX_DTYPE_BF16, num_splits, workspace,
                     workspace_bytes);
  c.timeout_ns = (unsigned long long)timeout_ms * 1000000ull;
  c.debug_skip_first_tile = 1;
  return run(c);
}

// --------------------------------------------------------------------------
// parallax_decode_noalloc: the same decode for callers that cannot allocate
// device memory (see include/parallax.h). Its workspace is this file-scope
// array in the library's device memory. In host code the array's name is
// only a host-side stand-in, so the device address is looked up once per
// device with cudaGetSymbolAddress and passed to the kernels like any
// caller-provided workspace.
namespace {

constexpr size_t kNoallocScratchBytes = PARALLAX_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_addr[256] = {};

// Device address of g_noalloc_scratch on the current device (first call per
// device does the lookup, with that device current).
int noalloc_scratch_address(void** addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return PARALLAX_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return PARALLAX_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *addr = g_noalloc_addr[dev];
  return PARALLAX_OK;
}

}  // namespace

extern "C" int parallax_decode_noalloc(const void* q, const void* r, const void* k_cache,
                                       const void* v_cache, const int32_t* cache_seqlens,
                                       void* out, int B, int Hq, int Hkv, int D, float scale,
                                       void* stream, int Lmax, int in_dtype, int out_dtype,
                                       int num_splits) {
  void* scratch = nullptr;
  int st = noalloc_scratch_address(&scratch);
  if (st != PARALLAX_OK) return st;
  Call c = make_call(3, true, q, r, k_cache, v_cache, cache_seqlens, out, B, Hq, Hkv, D, scale,
                     stream, Lmax, in_dtype, out_dtype, num_splits, scratch, kNoallocScratchBytes);
  if ((st = validate(c)) != PARALLAX_OK) return st;
  int P = 0;
  if ((st = resolve_splits(num_splits, B, Hkv, Lmax, !tma_path(c), &P)) != PARALLAX_OK) return st;
  // The default count is capped at what the array holds for this group and
  // head size; an explicit count beyond it is an error.
  const size_t per_split = workspace_bytes_for(Hq / Hkv, D, 1) - kWorkspaceHeaderBytes;
  const int capacity = (int)std::min<size_t>(
      PARALLAX_MAX_SPLITS, (kNoallocScratchBytes - kWorkspaceHeaderBytes) / per_split);
  if (num_splits == 0) P = std::min(P, capacity);
  if (P < 1 || workspace_bytes_for(Hq / Hkv, D, P) > kNoallocScratchBytes)
    return PARALLAX_ERR_SCRATCH_LIMIT;
  c.num_splits = P;
  // The array keeps the previous call's contents: the status word must start
  // at zero; the partial records are always written before they are read.
  if (cudaMemsetAsync(scratch, 0, kWorkspaceHeaderBytes, c.stream) != cudaSuccess)
    return PARALLAX_ERR_CUDA;
  return run(c);
}
