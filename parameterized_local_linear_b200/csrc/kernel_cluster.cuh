// Parallax decode for few (batch row, kv head) items: one thread-block cluster
// per item, the split pieces combined in distributed shared memory (sm_100a).
//
// When B * Hkv is small (one sequence: the latency-bound single-user decode
// step), the split-KV kernel's fixed costs dominate: locating a partition
// from the lengths, writing partial records to global memory and a second
// kernel that merges them. Here the S CTAs that share item (b, g) form one
// cluster. CTA `rank` takes the item's 64-key tiles rank, rank + S,
// rank + 2S, ... of the row's key space (partition.cuh: the cache row, its
// last W keys with a sliding window, a paged row, or a block-sparse list;
// paged and block-sparse tiles are resolved by tile_source and publish their
// attended prefix per stage). On a contiguous row without a window the
// first tiles are known before the length is read: one producer lane per
// stage issues the tiles that fit in the ring (and lie inside the cache)
// right after the dependency wait, and the length is read while they fly.
// The consumer warps are those of the split-KV kernel
// (TcConsumer: GQA-packed mma.sync scores and value products, online
// (m, l, b, A, C)).
//
// The end, with no partial records in global memory and no merge kernel:
//  1. the eight consumer warps write their records into the drained ring and
//     combine them into this CTA's (M, L, B, A_d, C_d) per query head;
//  2. the G*D output values of the item are dealt to the S CTAs in slices;
//     each CTA pushes its combined values of slice o into CTA o's shared
//     memory with st.async, whose bytes count off CTA o's "slots" mbarrier as
//     they land (the cluster barrier, arrived at the start and waited for
//     here, guarantees every CTA is running with its barriers initialised);
//  3. CTA o waits on its own mbarrier for the bytes of all S sources (armed
//     with their total at the start; every source pushes on every path, also
//     after a timed-out wait, so the count always completes), then finishes
//     its slice from the S records in its own shared memory:
//       M = max m_s, w_s = 2^(m_s - M), l = sum w_s l_s (likewise b, A, C),
//       o = A/l + C/l - (b/l)(A/l)   (A/l without the probe; 0 when l = 0).
//     A release barrier after the pushes is not needed: a sender only leaves
//     once its own incoming bytes have landed, and nothing reads a sender's
//     shared memory.
//
// Tiles past the item's length that were issued before the length was known
// are consumed with zero attended keys. Every mbarrier wait is bounded; every
// thread reaches both cluster barrier phases on every path (the bounded waits
// end), so they always complete.
#pragma once

#include "common.cuh"
#include "kernel_tc.cuh"
#include "ptx.cuh"

namespace plx {

constexpr int kClusterMax = 16;  // CTAs per cluster the kernel takes (above 8: non-portable)
// The largest size the host chooses by itself. Measured on a B200 at the
// Qwen-3 B = 1 step (8 items, 64 tiles each): 8 CTAs per item (8 tiles each)
// 6.62 us, 9 -> 6.87, 10 -> 6.75; 11 and more fit only 7 clusters at a time.
constexpr int kClusterAuto = 8;

template <int D>
struct ClusterGeom {
  // a deeper ring than the split-KV kernel's: one CTA's few tiles all in flight
  static constexpr int kStages = D == 128 ? 6 : 8;
  static_assert(kStages % kConsumerGroups == 0, "a stage must always belong to one group");
};

// Byte offsets inside the (1024-aligned) dynamic shared memory of the cluster
// kernel: the K/V ring (the consumer warps' records reuse it once drained),
// the P tiles, the barriers, the abort flag, then the S incoming records of
// this CTA's output slice: per source rank, G headers (m, l, b, -) and the
// (A, C) pairs of the slice's `per` values.
struct ClusterLayout {
  int off_p, off_bar, off_misc, off_slots, per, slot_stride, total;
};

__host__ __device__ inline ClusterLayout cluster_layout(int stage_bytes, int stages, int G, int D,
                                                        int S) {
  ClusterLayout L{};
  L.off_p = stages * stage_bytes;
  L.off_bar = L.off_p + kTcConsumers * 512;
  L.off_misc = align_up(L.off_bar + 8 * (2 * stages + 2), 16);  // full, empty, fin, slots
  L.off_slots = L.off_misc + 16 + 4 * stages;  // abort flag, then each stage's attended keys
  L.per = (G * D + S - 1) / S;
  L.off_slots = align_up(L.off_slots, 16);
  L.slot_stride = align_up(4 * G + 2 * L.per, 4);  // floats; rows stay 16-byte aligned
  L.total = L.off_slots + S * L.slot_stride * 4 + 1024;  // + alignment slack
  return L;
}

template <int D, bool PROBE, bool OUT_F32, bool PSPLIT>
__global__ void __launch_bounds__(kTcThreads, 1)
    parallax_cluster_kernel(const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  static_assert(!PROBE || PSPLIT, "the probe kernel needs the hi + lo split of P");
  constexpr int kStages = ClusterGeom<D>::kStages;
  constexpr int kStageBytes = TcGeom<D>::kStageBytes;
  constexpr int kKBytes = TcGeom<D>::kKBytes;
  constexpr int REC = rec_floats(D);
  const float kNegInf = __int_as_float(0xff800000u);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = (int)cluster_nctarank(), rank = (int)cluster_ctarank();
  const int item = (int)blockIdx.x / S;  // a cluster is S consecutive CTAs along x
  const int b = item / p.Hkv, g = item - b * p.Hkv;
  const int G = p.G;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - raw);
  const ClusterLayout L = cluster_layout(kStageBytes, kStages, G, D, S);
  const uint32_t bar_full = base + L.off_bar;
  const uint32_t bar_empty = bar_full + 8 * kStages;
  const uint32_t bar_fin = bar_empty + 8 * kStages;
  const uint32_t bar_slots = bar_fin + 8;  // the pushes into this CTA's slots
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L.off_misc);
  // paged / block-sparse rows: attended keys (a prefix) of the tile in each stage
  volatile int* stage_valid = reinterpret_cast<volatile int*>(gbase + L.off_misc + 16);
  float* const merge_scr = reinterpret_cast<float*>(gbase);  // the drained ring
  const uint32_t slots = base + L.off_slots;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, kConsumerWarps);
    }
    mbar_init(bar_fin, kTcConsumers);
    mbar_init(bar_slots, 1);
    *abort_flag = 0;
    mbar_fence_init();
    // the bytes S sources push into this CTA's slice: G headers of 16 bytes
    // and an (A, C) pair of 8 bytes per value of the slice
    const int nvals = min(L.per, G * D - rank * L.per);
    mbar_arrive_expect_tx(bar_slots, (uint32_t)(S * (16 * G + 8 * max(nvals, 0))));
  }
  uint64_t policy = 0;
  if (warp == kTcConsumers) {
    if (lane == 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
    }
    policy = l2_policy_evict_first();
  }
  __syncthreads();
  cluster_arrive_release();  // phase 0: this CTA runs, its barriers initialised
  // Launched with programmatic stream serialisation: nothing below may read
  // what the previous kernel in the stream writes before this wait.
  pdl_wait_primary();

  // tile j of this CTA is the item's tile rank + S j; on a contiguous row
  // without a window, and on a paged row, the first ones that fit in the ring
  // and lie inside the row's capacity are issued before the length is known
  // (a paged tile's page id and attended prefix come with it from tile_source;
  // one past the length attends nothing)
  const KeySpace ks = key_space(p);
  const bool contiguous = p.kv_mode == kKvContiguous;
  const int cache_tiles = (p.Lmax + kTileKeys - 1) / kTileKeys;
  const bool speculate = (contiguous && p.window == 0) || p.kv_mode == kKvPaged;
  const int nspec = (speculate && rank < cache_tiles)
                        ? min(kStages, (cache_tiles - rank + S - 1) / S)
                        : 0;
  const bool skip0 = p.debug_skip_first_tile != 0;  // testing hook: stage 0 never filled
  bool ok = true;

  if (warp == kTcConsumers) {
    // ---------------------------------------------------------- producer --
    // tile j's first key and row on the K/V view: kbase + its position on a
    // contiguous row, else where tile_source finds it (and its attended keys,
    // published in the stage's word before the arrive below)
    auto issue = [&](int j, int kbase) {
      const int stage = j % kStages;
      const uint32_t full = bar_full + 8 * stage;
      const uint32_t sK = base + stage * kStageBytes;
      int key = kbase + (rank + S * j) * kTileKeys, row = b;
      if (!contiguous) {
        int nv;
        tile_source(p, b, (rank + S * j) * kTileKeys, &key, &row, &nv);
        stage_valid[stage] = nv;
      }
      mbar_arrive_expect_tx(full, kStageBytes);
      tma_load_5d(sK, &tmK, 0, key, 0, g, row, full, policy);
      tma_load_5d(sK + kKBytes, &tmV, 0, key, 0, g, row, full, policy);
    };
    if (lane < nspec && !(lane == 0 && skip0)) issue(lane, 0);  // fresh stages, one lane each
    pdl_launch_dependents();
    __syncwarp();
    if (lane == 0) {
      uint32_t issued_mask = ((1u << nspec) - 1u) & (skip0 ? ~1u : ~0u), issued_par = 0;
      int kbase;
      const int nkeys = item_keys(ks, b, &kbase);  // positions of the row's key space
      const int ntiles = (nkeys + kTileKeys - 1) / kTileKeys;
      const int nreal = rank < ntiles ? (ntiles - rank + S - 1) / S : 0;
      bool skip = skip0 && nspec == 0;
      for (int j = nspec; j < nreal; ++j) {
        const int stage = j % kStages;
        const uint32_t par = (uint32_t)(j / kStages) & 1u;
        if (!mbar_wait_bounded(bar_empty + 8 * stage, par ^ 1u, p.timeout_ns, abort_flag)) {
          ok = false;
          break;
        }
        if (skip) {  // testing hook: the first stage is never filled
          skip = false;
          continue;
        }
        issue(j, kbase);
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (par << stage);
      }
      if (!ok) {
        // Give up: tell the consumers, record the timeout, and wait (bounded)
        // for this CTA's copies still in flight.
        *abort_flag = 1;
        atomicOr(p.status, 1u /* PARALLAX_DEVICE_STATUS_TIMEOUT */);
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s))
            mbar_wait_bounded(bar_full + 8 * s, (issued_par >> s) & 1u, p.timeout_ns, nullptr);
      }
    }
    __syncwarp();
    cluster_wait();  // phase 0
  } else {
    // --------------------------------------------------------- consumers --
    pdl_launch_dependents();
    if (rank == 0 && tid == 0 && g == 0 && item_clamped(ks, b))
      atomicOr(p.status, 2u /* PARALLAX_DEVICE_STATUS_SEQLEN_CLAMPED */);
    int kbase;
    const int nkeys = item_keys(ks, b, &kbase);
    const int ntiles = (nkeys + kTileKeys - 1) / kTileKeys;
    const int nreal = rank < ntiles ? (ntiles - rank + S - 1) / S : 0;
    const int J = max(nspec, nreal);
    const int group = warp / kConsumerWarps;
    TcConsumer<D, PROBE, PSPLIT> cs;
    cs.init(warp, lane, base + L.off_p + warp * 512);
    cs.load_rows(p, b, g);
    cs.reset();
    for (int j = group; j < J; j += kConsumerGroups) {
      const int stage = j % kStages;
      const uint32_t par = (uint32_t)(j / kStages) & 1u;
      if (!mbar_wait_bounded(bar_full + 8 * stage, par, p.timeout_ns, abort_flag)) {
        ok = false;
        break;
      }
      const int k0 = (rank + S * j) * kTileKeys;  // position in the row's key space
      const uint32_t sK = base + stage * kStageBytes;
      const int nvalid = contiguous ? max(0, min(kTileKeys, nkeys - k0)) : stage_valid[stage];
      cs.tile(sK, sK + kKBytes, nvalid, p.scale_log2);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty + 8 * stage);
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) atomicOr(p.status, 1u /* PARALLAX_DEVICE_STATUS_TIMEOUT */);
    }
    // 1. every consumer warp is done with the ring: the warps' records go there
    asm volatile("bar.sync 1, %0;" ::"n"(kTcConsumers * 32) : "memory");
    cs.write_record(merge_scr + warp * G * REC, G);
    asm volatile("bar.sync 1, %0;" ::"n"(kTcConsumers * 32) : "memory");
    cluster_wait();  // phase 0: every CTA of the cluster is running
    // 2. this CTA's combined values, each pushed to the CTA that owns its slice
    const uint32_t row = (uint32_t)(rank * L.slot_stride);  // this CTA's row in every slot area
    for (int idx = tid; idx < G * D; idx += kTcConsumers * 32) {
      const int h = idx / D, d = idx - h * D;
      float M, Lw, Bw, Aw, Cw;
      tc_combine_warps<D, PROBE>(merge_scr, G, h, d, M, Lw, Bw, Aw, Cw);
      const int o = idx / L.per, j = idx - o * L.per;
      st_async_f32x2(cluster_map(slots + (row + 4 * G + 2 * j) * 4u, (uint32_t)o), Aw, Cw,
                     cluster_map(bar_slots, (uint32_t)o));
      if (d == 0) {
        for (int t = 0; t < S; ++t)
          st_async_f32x4(cluster_map(slots + (row + 4 * h) * 4u, (uint32_t)t), M, Lw, Bw, 0.f,
                         cluster_map(bar_slots, (uint32_t)t));
      }
    }
  }

  // 3. this CTA's slice has landed (bounded wait, no abort shortcut: every
  // source pushes, and this CTA must not leave before its bytes arrive)
  if (!mbar_wait_bounded(bar_slots, 0, p.timeout_ns, nullptr)) {
    if (tid == 0) atomicOr(p.status, 1u /* PARALLAX_DEVICE_STATUS_TIMEOUT */);
    return;
  }
  // W lanes per output value (W >= S, a power of two dividing 32), one
  // source record each, reduced with shuffles; whole warps iterate together
  const float* const slot = reinterpret_cast<const float*>(gbase + L.off_slots);
  const int W = S <= 2 ? 2 : (S <= 4 ? 4 : (S <= 8 ? 8 : 16));
  const int total = L.per * W;
  for (int base0 = warp * 32; base0 < total; base0 += kTcThreads) {
    const int idx = base0 + lane, j = idx / W, src = idx - j * W;
    const int gi = rank * L.per + j;
    const bool value = idx < total && gi < G * D;
    const int h = value ? gi / D : 0, d = value ? gi - h * D : 0;
    float m = kNegInf, l = 0.f, bb = 0.f, a = 0.f, c = 0.f;
    if (value && src < S) {
      const float4 hd = *reinterpret_cast<const float4*>(slot + src * L.slot_stride + 4 * h);
      const float2 ac =
          *reinterpret_cast<const float2*>(slot + src * L.slot_stride + 4 * G + 2 * j);
      m = hd.x;
      l = hd.y;
      bb = hd.z;
      a = ac.x;
      c = ac.y;
    }
    float M = m;
    for (int o = 1; o < W; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float w = m == kNegInf ? 0.f : ex2_approx(m - M);
    l *= w;
    a *= w;
    bb *= w;
    c *= w;
    for (int o = 1; o < W; o <<= 1) {
      l += __shfl_xor_sync(0xffffffffu, l, o);
      a += __shfl_xor_sync(0xffffffffu, a, o);
      if (PROBE) {
        bb += __shfl_xor_sync(0xffffffffu, bb, o);
        c += __shfl_xor_sync(0xffffffffu, c, o);
      }
    }
    if (value && src == 0) {
      const float inv = l > 0.f ? 1.f / l : 0.f;  // no attended key: o = 0
      const float vbar = a * inv;
      const float o = PROBE ? vbar + c * inv - (bb * inv) * vbar : vbar;
      const size_t oi = ((size_t)b * p.Hq + (size_t)g * G + h) * D + d;
      if (OUT_F32)
        static_cast<float*>(p.out)[oi] = o;
      else
        static_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(o);
    }
  }
}

}  // namespace plx
