// Definitions shared by the host launcher and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>

namespace plx {

// Workspace: a 256-byte header whose first word is the device status word,
// then 2 * P * G partial records of kRecHead + 2*D floats each:
//   [0] m (running max, log2 domain) [1] l [2] b [3] unused [4..4+D) A [4+D..4+2D) C
constexpr size_t kWorkspaceHeaderBytes = 256;
constexpr int kRecHead = 4;

__host__ __device__ constexpr int rec_floats(int D) { return kRecHead + 2 * D; }

struct DecodeParams {
  const void* q;          // [B][Hq][D]
  const void* r;          // [B][Hq][D] (unused by the softmax kernels)
  const void* k;          // K cache (generic kernel only; the TMA kernel uses tensor maps)
  const void* v;
  long long kv_sb, kv_sh, kv_sk;  // element strides of batch row, kv head and key in K and V
  const int32_t* seqlens; // [B], or NULL: every row holds Lmax keys
  int window;             // > 0: attend only the last `window` keys of each row
  void* out;              // [B][Hq][D]
  float* partials;        // 2 * P * G records
  unsigned int* status;   // device status word (workspace header)
  int B, Hq, Hkv, G, D, Lmax;
  float scale_log2;       // qk_scale * log2(e): logits are kept in the log2 domain
  unsigned long long timeout_ns;  // bound of every wait inside the kernels
  int debug_skip_first_tile;      // testing hook: the producer never fills stage 0
  // where the keys of a row come from (partition.cuh, KvMode)
  int kv_mode;
  const int32_t* table;   // paged: [B][table_stride] page ids; block-sparse: block ids
  int table_stride;
  const int32_t* num_blocks;  // block-sparse: [B] listed blocks
  int page_size, num_pages;   // paged
};

// ------------------------------------------------ TMA kernel geometry ------
constexpr int kTileKeys = 64;        // keys per pipeline stage
constexpr int kConsumerWarps = 4;    // warps per stage: each owns 16 of its keys
constexpr int kConsumerGroups = 2;   // groups of kConsumerWarps that take alternate stages
constexpr int kTcConsumers = kConsumerWarps * kConsumerGroups;
constexpr int kTcThreads = (kTcConsumers + 1) * 32;  // + one producer warp
constexpr int kBoxBytes = kTileKeys * 128;             // one 64-key x 128-byte swizzled box

// A 96-128 KB ring of K+V per CTA: measured on B200, one CTA per SM with
// ~100 KB in flight streams faster than 192 KB per SM (one CTA with a 6-stage
// ring, or two CTAs), and it leaves shared memory for the merge kernel's blocks
// to become resident early. The stage count is a multiple of the consumer
// groups, so every stage is always consumed by the same group: a group then
// waits on each of its stages' fills in order, never two phases ahead of an
// mbarrier (where a parity wait can not tell the fills apart).
template <int D>
struct TcGeom {
  static constexpr int kHalves = D / 64;                 // 128-byte boxes per key row
  static constexpr int kKBytes = kHalves * kBoxBytes;    // K tile of one stage
  static constexpr int kStageBytes = 2 * kKBytes;        // K + V
  static constexpr int kStages = D == 128 ? 4 : 6;
  static_assert(kStages % kConsumerGroups == 0, "a stage must always belong to one group");
};

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

// Byte offsets inside the (1024-aligned) dynamic shared memory of the TMA kernel.
struct TcSmemLayout {
  int off_p, off_merge, off_bar, off_misc, total;
};

__host__ __device__ inline TcSmemLayout tc_smem_layout(int D, int stage_bytes, int stages, int G,
                                                       bool probe) {
  (void)probe;
  TcSmemLayout L{};
  L.off_p = stages * stage_bytes;
  L.off_merge = L.off_p + kTcConsumers * 512;
  L.off_bar = align_up(L.off_merge + kTcConsumers * G * rec_floats(D) * 4, 16);
  // full[stages], empty[stages], fin[2]
  L.off_misc = L.off_bar + 8 * (2 * stages + 2);
  L.total = L.off_misc + 48 + 1024;  // abort flag, per-stage valid keys, alignment slack
  return L;
}

constexpr int kGenericThreads = 128;
constexpr int kMergeThreads = 128;  // one warp per SM sub-partition: fits beside a split-KV CTA
constexpr int kMergeMaxG = 128;  // query heads per kv head handled by the merge kernel
constexpr int kMergeChunk = 16;  // partial records one merge thread holds in registers

// Merge blocks per partition: one float4 column of A (and C) per thread.
__host__ __device__ inline int merge_slices(int G, int D, bool probe) {
  const int cols = G * (D / 4) * (probe ? 2 : 1);
  return (cols + kMergeThreads - 1) / kMergeThreads;
}

}  // namespace plx
