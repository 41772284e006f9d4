// Parallax decode for few (batch row, kv head) items: one thread-block cluster
// per item, the split pieces combined in distributed shared memory (sm_100a).
//
// When B * Hkv is small (one sequence: the latency-bound single-user decode
// step), the split-KV kernel's fixed costs dominate: locating a partition
// from the lengths, writing partial records to global memory and a second
// kernel that merges them. Here the S CTAs that share item (b, g) form one
// cluster. CTA `rank` takes the item's 64-key tiles rank, rank + S,
// rank + 2S, ... so the first tiles are known before the length is read: the
// producer issues the tiles that fit in its ring (and lie inside the cache)
// right after the dependency wait, and reads the length while they fly. The
// consumer warps are those of the split-KV kernel (TcConsumer: GQA-packed
// mma.sync scores and value products, online (m, l, b, A, C)). At the end the
// eight warps combine in shared memory into one record per query head, the
// cluster synchronises, and CTA `rank` finishes its slice of the item's
// outputs from the S records of the cluster (the same rescaled sums as the
// merge kernel, read with ld.shared::cluster):
//   M = max m_s, w_s = 2^(m_s - M), l = sum w_s l_s (likewise b, A, C),
//   o = A/l + C/l - (b/l)(A/l)   (A/l without the probe; 0 when l = 0).
// A second cluster barrier keeps every CTA alive until the others have read
// its record. No workspace beyond the status word, no merge kernel.
//
// Tiles past the item's length that were issued before the length was known
// are consumed with zero attended keys. Every mbarrier wait is bounded; the
// cluster barriers are reached by every thread on every path (the bounded
// waits end), so they always complete.
#pragma once

#include "common.cuh"
#include "kernel_tc.cuh"
#include "ptx.cuh"

namespace plx {

constexpr int kClusterMax = 16;  // CTAs per cluster (above 8 needs the non-portable size)

// Shared memory of the cluster kernel: the split-KV kernel's layout, then one
// combined record per query head of the group (read by the whole cluster).
__host__ __device__ inline int cluster_off_crec(const TcSmemLayout& L) {
  return align_up(L.off_misc + 48, 16);
}
__host__ __device__ inline int cluster_smem_total(const TcSmemLayout& L, int G, int D) {
  return cluster_off_crec(L) + G * rec_floats(D) * 4 + 1024;
}

template <int D, bool PROBE, bool OUT_F32, bool PSPLIT>
__global__ void __launch_bounds__(kTcThreads, 1)
    parallax_cluster_kernel(const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  static_assert(!PROBE || PSPLIT, "the probe kernel needs the hi + lo split of P");
  using Geom = TcGeom<D>;
  constexpr int kStages = Geom::kStages;
  constexpr int kStageBytes = Geom::kStageBytes;
  constexpr int kKBytes = Geom::kKBytes;
  constexpr int REC = rec_floats(D);
  const float kNegInf = __int_as_float(0xff800000u);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - raw);
  const TcSmemLayout L = tc_smem_layout(D, kStageBytes, kStages, p.G, PROBE);
  const uint32_t bar_full = base + L.off_bar;
  const uint32_t bar_empty = bar_full + 8 * kStages;
  const uint32_t bar_fin = bar_empty + 8 * kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L.off_misc);
  float* const merge_scr = reinterpret_cast<float*>(gbase + L.off_merge);
  float* const crec = reinterpret_cast<float*>(gbase + cluster_off_crec(L));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = (int)cluster_nctarank(), rank = (int)cluster_ctarank();
  const int item = (int)blockIdx.x / S;  // a cluster is S consecutive CTAs along x
  const int b = item / p.Hkv, g = item - b * p.Hkv;
  const int G = p.G;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, kConsumerWarps);
    }
    mbar_init(bar_fin, kTcConsumers);
    *abort_flag = 0;
    mbar_fence_init();
  }
  uint64_t policy = 0;
  if (tid == kTcConsumers * 32) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    policy = l2_policy_evict_first();
  }
  __syncthreads();
  // Launched with programmatic stream serialisation: nothing below may read
  // what the previous kernel in the stream writes before this wait.
  pdl_wait_primary();

  // tile j of this CTA is the item's tile rank + S j; the first ones that fit
  // in the ring and lie inside the cache are issued before the length is known
  const int cache_tiles = (p.Lmax + kTileKeys - 1) / kTileKeys;
  const int nspec = rank < cache_tiles ? min(kStages, (cache_tiles - rank + S - 1) / S) : 0;
  bool ok = true;

  if (warp == kTcConsumers) {
    // ---------------------------------------------------------- producer --
    if (lane == 0) {
      bool skip = p.debug_skip_first_tile != 0;
      uint32_t issued_mask = 0, issued_par = 0;
      auto issue = [&](int j) {
        const int stage = j % kStages;
        const uint32_t par = (uint32_t)(j / kStages) & 1u;
        if (skip) {
          skip = false;  // testing hook: leave this stage empty forever
          return;
        }
        const uint32_t full = bar_full + 8 * stage;
        const uint32_t sK = base + stage * kStageBytes;
        const int key = (rank + S * j) * kTileKeys;
        mbar_arrive_expect_tx(full, kStageBytes);
        tma_load_5d(sK, &tmK, 0, key, 0, g, b, full, policy);
        tma_load_5d(sK + kKBytes, &tmV, 0, key, 0, g, b, full, policy);
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (par << stage);
      };
      for (int j = 0; j < nspec; ++j) issue(j);  // fresh stages: no wait for room
      pdl_launch_dependents();
      const int n = p.seqlens ? clamp_len(__ldg(p.seqlens + b), p.Lmax) : p.Lmax;
      const int ntiles = (n + kTileKeys - 1) / kTileKeys;
      const int nreal = rank < ntiles ? (ntiles - rank + S - 1) / S : 0;
      for (int j = nspec; j < nreal; ++j) {
        const int stage = j % kStages;
        const uint32_t par = (uint32_t)(j / kStages) & 1u;
        if (!mbar_wait_bounded(bar_empty + 8 * stage, par ^ 1u, p.timeout_ns, abort_flag)) {
          ok = false;
          break;
        }
        issue(j);
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(p.status, 1u /* PARALLAX_DEVICE_STATUS_TIMEOUT */);
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s))
            mbar_wait_bounded(bar_full + 8 * s, (issued_par >> s) & 1u, p.timeout_ns, nullptr);
      }
    } else {
      pdl_launch_dependents();
    }
    __syncwarp();
  } else {
    // --------------------------------------------------------- consumers --
    pdl_launch_dependents();
    const int nraw = p.seqlens ? __ldg(p.seqlens + b) : p.Lmax;
    const int n = clamp_len(nraw, p.Lmax);
    if (rank == 0 && tid == 0 && g == 0 && nraw != n)
      atomicOr(p.status, 2u /* PARALLAX_DEVICE_STATUS_SEQLEN_CLAMPED */);
    const int ntiles = (n + kTileKeys - 1) / kTileKeys;
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
      const int k0 = (rank + S * j) * kTileKeys;
      const uint32_t sK = base + stage * kStageBytes;
      cs.tile(sK, sK + kKBytes, max(0, min(kTileKeys, n - k0)), p.scale_log2);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty + 8 * stage);
    }
    // the eight warps' records, combined into this CTA's record per head
    if (ok) {
      cs.write_record(merge_scr + warp * G * REC, G);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_fin);
      ok = mbar_wait_bounded(bar_fin, 0, p.timeout_ns, abort_flag);
    }
    if (ok) {
      for (int idx = tid; idx < G * D; idx += kTcConsumers * 32) {
        const int h = idx / D, d = idx - h * D;
        float M, Lw, Bw, Aw, Cw;
        tc_combine_warps<D, PROBE>(merge_scr, G, h, d, M, Lw, Bw, Aw, Cw);
        float* rec = crec + h * REC;
        if (d == 0) {
          rec[0] = M;
          rec[1] = Lw;
          rec[2] = Bw;
        }
        rec[kRecHead + d] = Aw;
        if (PROBE) rec[kRecHead + D + d] = Cw;
      }
    } else {
      *abort_flag = 1;
      if (lane == 0) atomicOr(p.status, 1u /* PARALLAX_DEVICE_STATUS_TIMEOUT */);
    }
  }

  // ---- the cluster's records, this CTA's slice of the item's outputs ----
  __syncwarp();
  cluster_sync_all();
  const int per = (G * D + S - 1) / S;
  const uint32_t crec_addr = smem_u32(crec);
  for (int v = tid; v < per; v += kTcThreads) {
    const int gi = rank * per + v;
    if (gi >= G * D) break;
    const int h = gi / D, d = gi - h * D;
    const uint32_t off = (uint32_t)(h * REC) * 4u;
    float ms[kClusterMax], ls[kClusterMax], bs[kClusterMax], as[kClusterMax], cs_[kClusterMax];
#pragma unroll
    for (int s = 0; s < kClusterMax; ++s) {
      if (s < S) {
        const uint32_t r = cluster_map(crec_addr + off, (uint32_t)s);
        const float4 hd = ld_cluster_f32x4(r);
        ms[s] = hd.x;
        ls[s] = hd.y;
        bs[s] = hd.z;
        as[s] = ld_cluster_f32(r + (uint32_t)(kRecHead + d) * 4u);
        cs_[s] = PROBE ? ld_cluster_f32(r + (uint32_t)(kRecHead + D + d) * 4u) : 0.f;
      }
    }
    float M = kNegInf;
#pragma unroll
    for (int s = 0; s < kClusterMax; ++s)
      if (s < S) M = fmaxf(M, ms[s]);
    float Lw = 0.f, Bw = 0.f, Aw = 0.f, Cw = 0.f;
#pragma unroll
    for (int s = 0; s < kClusterMax; ++s) {
      if (s < S) {
        const float w = ms[s] == kNegInf ? 0.f : ex2_approx(ms[s] - M);
        Lw += w * ls[s];
        Aw += w * as[s];
        if (PROBE) {
          Bw += w * bs[s];
          Cw += w * cs_[s];
        }
      }
    }
    const float inv = Lw > 0.f ? 1.f / Lw : 0.f;  // no attended key: o = 0
    const float vbar = Aw * inv;
    const float o = PROBE ? vbar + Cw * inv - (Bw * inv) * vbar : vbar;
    const size_t oi = ((size_t)b * p.Hq + (size_t)g * G + h) * D + d;
    if (OUT_F32)
      static_cast<float*>(p.out)[oi] = o;
    else
      static_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(o);
  }
  __syncwarp();
  cluster_sync_all();  // no CTA leaves while another may still read its record
}

}  // namespace plx
