// Split-KV Parallax decode kernel for bf16 caches (sm_100a).
//
// One CTA per partition of the flattened key range (see partition.cuh),
// persistent over the pieces of that range. Warp 8 is the producer: one lane
// streams 64-key K and V tiles of the current item with one TMA each (5-D
// tensor maps {64 dims, keys, D/64 halves, kv heads, batch rows} over either
// cache layout, 128-byte swizzle, no multicast) into a ring of shared-memory
// stages guarded by full/empty mbarriers. Warps 0..7 consume in two groups of
// four that take alternate stages (two tiles in flight through the math at
// once): warp w owns keys 16 (w % 4) .. +15 of its group's stages and keeps its
// own online accumulators, so the consumer warps never synchronise inside the
// key loop. They read the q (and r) rows of the item's GQA group straight into
// mma fragments from global memory, overlapped with the first K/V tile's
// flight.
//
// The method streams the same K/V tiles as FlashAttention and does twice its
// work per byte ("Parallax: Parameterized Local Linear Attention for Language
// Modeling", neuraltrendhub summary, "What the paper found"; bayesiansapien
// blog, "What changes vs prior work"). Per 16-key block a consumer warp runs:
//   scores  S[16 keys x 8] = K[16 x D] * [q_0 r_0 q_1 r_1 ...]^T   (mma.sync)
//           (the GQA group's q and r rows are the 8 columns, so every K tile
//            read from HBM serves 2*G query-side rows)
//   online  m' = max(m, t), alpha = 2^(m-m'), e = 2^(t-m'),
//           l = alpha l + sum e, b = alpha b + sum e s     (per query head)
//   values  O^T[D x 8] = V^T[D x 16] * P[16 x 8],  P = [e_0, e_0 s_0, e_1, ...]
//           accumulating A (column e_h) and C (column e_h s_h) in fp32.
// t = qk_scale * log2(e) * q.k is kept in the log2 domain. With PSPLIT the
// probabilities go through the tensor cores as a bf16 hi + lo pair (~16
// significant bits). The probe kernel always splits: the correction
// C/l - (b/l)(A/l) subtracts two terms of size |s||v|, so a single bf16
// rounding of e and e*s (2^-9) would leave an error of ~2^-9 |s||v| where the
// result itself can be ~0 (one dominant key); l and b are summed from the same
// hi + lo values the tensor cores apply. The softmax kernel splits only for
// the fp32-output mode.
// At the end of a piece the eight warps combine their (m, l, b, A, C) in shared
// memory; a whole item is finished (o = A/l + C/l - (b/l)(A/l), or A/l without
// the probe) and stored, a partial item writes a partial record for the merge
// kernel.
#pragma once

#include "common.cuh"
#include "partition.cuh"
#include "ptx.cuh"

namespace plx {

static_assert(kTileKeys == kRangeAlign, "partition ranges are whole tiles of this kernel");

// One consumer warp of the TMA kernels: its lane constants, the mma fragments
// of the item's q (and r) rows, and its online accumulators over the keys it
// owns (16 per stage of its group). With the probe each thread carries one
// query head h = lane % 4 (column pair = its logit and probe score); the
// softmax kernel carries two heads 2 (lane % 4), +1 (two logit columns).
template <int D, bool PROBE, bool PSPLIT>
struct TcConsumer {
  static constexpr int kJ = D / 16;  // 16-wide slices of the head dimension
  using Geom = TcGeom<D>;
  int lane, g8, c4, my0;
  int k_row, k_cadd, v_row, v_cadd, sw;
  uint32_t p_tile;
  uint32_t bq[kJ][2];
  float acc[kJ][4];
  float m0, m1, l0, l1, bsum;  // (m1, l1) softmax only; bsum probe only

  __device__ __forceinline__ void init(int warp, int lane_, uint32_t p_tile_) {
    lane = lane_;
    g8 = lane >> 2;
    c4 = lane & 3;
    my0 = 16 * (warp % kConsumerWarps);  // this warp's first key row inside a stage
    p_tile = p_tile_;
    // ldmatrix row addresses (before the stage base and the D-slice offset).
    // K (scores, A operand, row-major): matrices {rows 0-7, rows 8-15} x {k 0-7, k 8-15}.
    k_row = my0 + (lane & 7) + ((lane >> 3) & 1) * 8;
    k_cadd = lane >> 4;  // +1 chunk for matrices 2, 3
    // V (values, A operand = V^T via .trans): matrices {dims 0-7, 8-15} x {keys 0-7, keys 8-15}.
    v_row = my0 + (lane & 7) + (lane >> 4) * 8;
    v_cadd = (lane >> 3) & 1;
    sw = lane & 7;  // row index mod 8 = the 128-byte swizzle phase of both rows
  }

  // B fragments of the group's q (and r) rows of item (b, g); column n = lane / 4.
  __device__ __forceinline__ void load_rows(const DecodeParams& p, int b, int g) {
    const int G = p.G;
    int h, is_r;
    if (PROBE) {
      h = g8 >> 1;
      is_r = g8 & 1;  // odd columns hold the probe rows
    } else {
      h = g8;
      is_r = 0;
    }
    const bool valid = h < G;  // columns past the group stay zero
    const size_t row = ((size_t)b * p.Hq + (size_t)g * G + (valid ? h : 0)) * D;
    const uint32_t* src = reinterpret_cast<const uint32_t*>(
        static_cast<const __nv_bfloat16*>(is_r ? p.r : p.q) + row);
#pragma unroll
    for (int j = 0; j < kJ; ++j) {
      bq[j][0] = valid ? __ldg(src + 8 * j + c4) : 0u;      // dims 16j + 2c4, +1
      bq[j][1] = valid ? __ldg(src + 8 * j + c4 + 4) : 0u;  // dims 16j + 2c4 + 8, +9
    }
  }

  __device__ __forceinline__ void reset() {
    const float kNegInf = __int_as_float(0xff800000u);
#pragma unroll
    for (int i = 0; i < kJ; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    m0 = m1 = kNegInf;
    l0 = l1 = bsum = 0.f;
  }

  // This warp's 16 keys of the stage at sK (K) / sV (V), of which the first
  // `nvalid` keys of the stage are attended (rows past them are masked).
  __device__ __forceinline__ void tile(uint32_t sK, uint32_t sV, int nvalid, float scale_log2) {
    const float kNegInf = __int_as_float(0xff800000u);
    if (my0 >= nvalid) return;
    if (my0 + 16 > nvalid) {
      // Rows past the piece's end hold other keys, padding (maybe NaN)
      // or TMA zero fill: zero this warp's such V rows so that 0 * NaN
      // can not reach the accumulators (their probabilities are 0).
      const int first_bad = nvalid - my0;  // 1..15
      for (int idx = lane; idx < (16 - first_bad) * 8 * Geom::kHalves; idx += 32) {
        const int row = my0 + first_bad + idx / (8 * Geom::kHalves);
        const int rem = idx % (8 * Geom::kHalves);
        const uint32_t a = sV + (rem >> 3) * kBoxBytes + row * 128 + (rem & 7) * 16;
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0) : "memory");
      }
      fence_proxy_async_smem();
      __syncwarp();
    }
    // --- scores: two accumulation chains over the D slices ---
    float sc[4] = {0.f, 0.f, 0.f, 0.f}, sc2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < kJ; ++j) {
      const int chunk = 2 * (j & 3) + k_cadd;
      const uint32_t a = sK + (j >> 2) * kBoxBytes + k_row * 128 + ((chunk ^ sw) << 4);
      uint32_t fr[4];
      ldmatrix_x4(fr, a);
      if (j & 1)
        mma_bf16_16816(sc2, fr, bq[j][0], bq[j][1]);
      else
        mma_bf16_16816(sc, fr, bq[j][0], bq[j][1]);
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) sc[x] += sc2[x];
    // sc[0], sc[1]: key my0+g8, columns 2*c4, 2*c4+1; sc[2], sc[3]: key my0+g8+8
    const bool va = my0 + g8 < nvalid, vb = my0 + g8 + 8 < nvalid;
    float pa0, pa1, pb0, pb1;  // P entries: key a cols (2c4, 2c4+1), key b likewise
    float alpha0 = 1.f;        // PROBE: rescale of this thread's head
    if (PROBE) {
      const float ta = va ? sc[0] * scale_log2 : kNegInf;
      const float sa = va ? sc[1] : 0.f;
      const float tb = vb ? sc[2] * scale_log2 : kNegInf;
      const float sb = vb ? sc[3] : 0.f;
      float mx = fmaxf(ta, tb);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float mn = fmaxf(m0, mx);
      const float mu = mn == kNegInf ? 0.f : mn;
      alpha0 = ex2_approx(m0 - mu);
      const float ea = ex2_approx(ta - mu), eb = ex2_approx(tb - mu);
      m0 = mn;
      pa0 = ea;
      pa1 = ea * sa;
      pb0 = eb;
      pb1 = eb * sb;
#pragma unroll
      for (int i = 0; i < kJ; ++i) {
        acc[i][0] *= alpha0;
        acc[i][1] *= alpha0;
        acc[i][2] *= alpha0;
        acc[i][3] *= alpha0;
      }
    } else {
      const float ta0 = va ? sc[0] * scale_log2 : kNegInf;
      const float ta1 = va ? sc[1] * scale_log2 : kNegInf;
      const float tb0 = vb ? sc[2] * scale_log2 : kNegInf;
      const float tb1 = vb ? sc[3] * scale_log2 : kNegInf;
      float mx0 = fmaxf(ta0, tb0), mx1 = fmaxf(ta1, tb1);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float mu0 = mn0 == kNegInf ? 0.f : mn0, mu1 = mn1 == kNegInf ? 0.f : mn1;
      const float al0 = ex2_approx(m0 - mu0), al1 = ex2_approx(m1 - mu1);
      pa0 = ex2_approx(ta0 - mu0);
      pa1 = ex2_approx(ta1 - mu1);
      pb0 = ex2_approx(tb0 - mu0);
      pb1 = ex2_approx(tb1 - mu1);
      l0 = l0 * al0 + (pa0 + pb0);
      l1 = l1 * al1 + (pa1 + pb1);
      m0 = mn0;
      m1 = mn1;
#pragma unroll
      for (int i = 0; i < kJ; ++i) {
        acc[i][0] *= al0;
        acc[i][1] *= al1;
        acc[i][2] *= al0;
        acc[i][3] *= al1;
      }
    }
    // --- P to shared memory ([16 keys][8 columns] bf16), then B fragments ---
    const uint32_t hia = pack_bf16x2(pa0, pa1), hib = pack_bf16x2(pb0, pb1);
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(p_tile + g8 * 16 + c4 * 4), "r"(hia) : "memory");
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(p_tile + (g8 + 8) * 16 + c4 * 4), "r"(hib)
                 : "memory");
    if (PSPLIT) {
      const uint32_t loa = pack_bf16x2(pa0 - bf16_lo_to_float(hia), pa1 - bf16_hi_to_float(hia));
      const uint32_t lob = pack_bf16x2(pb0 - bf16_lo_to_float(hib), pb1 - bf16_hi_to_float(hib));
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(p_tile + 256 + g8 * 16 + c4 * 4), "r"(loa)
                   : "memory");
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(p_tile + 256 + (g8 + 8) * 16 + c4 * 4),
                   "r"(lob)
                   : "memory");
      if (PROBE) {
        // l and b from exactly the weights the tensor cores apply to A and
        // C (hi + lo), so that C/l - (b/l)(A/l) cancels consistently.
        const float ea = bf16_lo_to_float(hia) + bf16_lo_to_float(loa);
        const float esa = bf16_hi_to_float(hia) + bf16_hi_to_float(loa);
        const float eb = bf16_lo_to_float(hib) + bf16_lo_to_float(lob);
        const float esb = bf16_hi_to_float(hib) + bf16_hi_to_float(lob);
        l0 = l0 * alpha0 + (ea + eb);
        bsum = bsum * alpha0 + (esa + esb);
      }
    }
    __syncwarp();
    uint32_t bp[4];
    if (PSPLIT) {
      uint32_t t4[4];
      ldmatrix_x4_trans(t4, p_tile + (lane >> 4) * 256 + (lane & 15) * 16);
      bp[0] = t4[0];
      bp[1] = t4[1];
      bp[2] = t4[2];
      bp[3] = t4[3];
    } else {
      uint32_t t2[2];
      ldmatrix_x2_trans(t2, p_tile + (lane & 15) * 16);
      bp[0] = t2[0];
      bp[1] = t2[1];
      bp[2] = bp[3] = 0u;
    }
    // --- values: O^T[16 dims x 8] += V^T[16 dims x 16 keys] * P ---
#pragma unroll
    for (int i = 0; i < kJ; ++i) {
      const int chunk = 2 * (i & 3) + v_cadd;
      const uint32_t a = sV + (i >> 2) * kBoxBytes + v_row * 128 + ((chunk ^ sw) << 4);
      uint32_t fr[4];
      ldmatrix_x4_trans(fr, a);
      mma_bf16_16816(acc[i], fr, bp[0], bp[1]);
      if (PSPLIT) mma_bf16_16816(acc[i], fr, bp[2], bp[3]);
    }
    __syncwarp();
  }

  // The warp's (m, l, b, A, C) of each head of the group as records
  // [m, l, b, -, A[D], C[D]] at scr + h * rec_floats(D) (the warp's l and b
  // are first summed over its lanes).
  __device__ __forceinline__ void write_record(float* scr, int G) {
    constexpr int REC = rec_floats(D);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
      bsum += __shfl_xor_sync(0xffffffffu, bsum, o);
    }
    if (PROBE) {
      if (c4 < G) {
        float* rec = scr + c4 * REC;
        if (g8 == 0) {
          rec[0] = m0;
          rec[1] = l0;
          rec[2] = bsum;
        }
#pragma unroll
        for (int i = 0; i < kJ; ++i) {
          rec[kRecHead + 16 * i + g8] = acc[i][0];
          rec[kRecHead + D + 16 * i + g8] = acc[i][1];
          rec[kRecHead + 16 * i + g8 + 8] = acc[i][2];
          rec[kRecHead + D + 16 * i + g8 + 8] = acc[i][3];
        }
      }
    } else {
      const int ha = 2 * c4, hb = 2 * c4 + 1;
      if (ha < G) {
        float* rec = scr + ha * REC;
        if (g8 == 0) {
          rec[0] = m0;
          rec[1] = l0;
        }
#pragma unroll
        for (int i = 0; i < kJ; ++i) {
          rec[kRecHead + 16 * i + g8] = acc[i][0];
          rec[kRecHead + 16 * i + g8 + 8] = acc[i][2];
        }
      }
      if (hb < G) {
        float* rec = scr + hb * REC;
        if (g8 == 0) {
          rec[0] = m1;
          rec[1] = l1;
        }
#pragma unroll
        for (int i = 0; i < kJ; ++i) {
          rec[kRecHead + 16 * i + g8] = acc[i][1];
          rec[kRecHead + 16 * i + g8 + 8] = acc[i][3];
        }
      }
    }
  }
};

// The eight consumer warps' records of head h (written by write_record at
// merge_scr + (w * G + h) * rec_floats(D)) combined at dimension d: the
// common max M and the rescaled sums of l, b, A_d, C_d.
template <int D, bool PROBE>
__device__ __forceinline__ void tc_combine_warps(const float* merge_scr, int G, int h, int d,
                                                 float& M, float& Lw, float& Bw, float& Aw,
                                                 float& Cw) {
  constexpr int REC = rec_floats(D);
  const float kNegInf = __int_as_float(0xff800000u);
  M = kNegInf;
#pragma unroll
  for (int w = 0; w < kTcConsumers; ++w) M = fmaxf(M, merge_scr[(w * G + h) * REC]);
  Lw = Bw = Aw = Cw = 0.f;
#pragma unroll
  for (int w = 0; w < kTcConsumers; ++w) {
    const float* rec = merge_scr + (w * G + h) * REC;
    const float mw = rec[0];
    const float a = mw == kNegInf ? 0.f : ex2_approx(mw - M);
    Lw += a * rec[1];
    Aw += a * rec[kRecHead + d];
    if (PROBE) {
      Bw += a * rec[2];
      Cw += a * rec[kRecHead + D + d];
    }
  }
}

template <int D, bool PROBE, bool OUT_F32, bool PSPLIT>
__global__ void __launch_bounds__(kTcThreads, 1)
    parallax_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  static_assert(!PROBE || PSPLIT, "the probe kernel needs the hi + lo split of P");
  using Geom = TcGeom<D>;
  constexpr int kStages = Geom::kStages;
  constexpr int kStageBytes = Geom::kStageBytes;
  constexpr int kKBytes = Geom::kKBytes;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - raw);
  const TcSmemLayout L = tc_smem_layout(D, kStageBytes, kStages, p.G, PROBE);

  const uint32_t bar_full = base + L.off_bar;
  const uint32_t bar_empty = bar_full + 8 * kStages;
  const uint32_t bar_fin = bar_empty + 8 * kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L.off_misc);
  // paged / block-sparse rows: valid keys (a prefix) of the tile in each stage
  volatile int* stage_valid = reinterpret_cast<volatile int*>(gbase + L.off_misc + 16);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, kConsumerWarps);
    }
    for (int s = 0; s < 2; ++s) mbar_init(bar_fin + 8 * s, kTcConsumers);
    *abort_flag = 0;
    mbar_fence_init();
  }
  uint64_t policy = 0;
  if (tid == kTcConsumers * 32) {  // the producer lane: descriptors are kernel parameters
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    policy = l2_policy_evict_first();
  }
  __syncthreads();  // barriers initialised before anyone uses them
  // Launched with programmatic stream serialisation: everything above overlaps
  // the previous kernel in the stream; nothing below may run before it ends.
  pdl_wait_primary();
  const PartitionInfo part =
      locate_partition(key_space(p), p.B, p.Hkv, blockIdx.x, gridDim.x);
  if (blockIdx.x == 0 && tid == 0 && part.clamped)
    atomicOr(p.status, 2u /* PARALLAX_DEVICE_STATUS_SEQLEN_CLAMPED */);
  // The merge grid may be scheduled once every CTA has its first stage in
  // flight (threads that return early count as triggered): early enough to
  // hide its prologue, late enough not to slow this kernel's start.
  if (part.lo >= part.hi) return;

  const int G = p.G;

  // ------------------------------------------------------------ producer --
  if (warp == kTcConsumers) {
    if (lane != 0) return;
    PieceCursor cur;
    cur.init(part, key_space(p), p.B, p.Hkv);
    Piece pc;
    int stage = 0;
    uint32_t ph = 0, issued_mask = 0, issued_par = 0;
    bool ok = true, skip = p.debug_skip_first_tile != 0;
    while (ok && cur.next(pc)) {
      for (int k0 = pc.i; k0 < pc.i + pc.len; k0 += kTileKeys) {
        if (!mbar_wait_bounded(bar_empty + 8 * stage, ph ^ 1, p.timeout_ns, abort_flag)) {
          ok = false;
          break;
        }
        if (skip) {
          skip = false;  // testing hook: leave this stage empty forever
        } else {
          const uint32_t full = bar_full + 8 * stage;
          const uint32_t sK = base + stage * kStageBytes;
          // source of the tile: (key or page slot, batch row or page) on the maps
          int key = pc.kbase + k0, item = pc.b;
          if (p.kv_mode != kKvContiguous) {
            int nv;
            tile_source(p, pc.b, k0, &key, &item, &nv);
            stage_valid[stage] = nv;  // published by the arrive below
          }
          mbar_arrive_expect_tx(full, kStageBytes);
          tma_load_5d(sK, &tmK, 0, key, 0, pc.g, item, full, policy);
          tma_load_5d(sK + kKBytes, &tmV, 0, key, 0, pc.g, item, full, policy);
          if (issued_mask == 0) pdl_launch_dependents();
          issued_mask |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (ph << stage);
        }
        if (++stage == kStages) {
          stage = 0;
          ph ^= 1;
        }
      }
    }
    if (issued_mask == 0) pdl_launch_dependents();
    if (!ok) {
      // Give up: tell the consumers, record the timeout, and wait (bounded)
      // for this CTA's copies still in flight before leaving.
      *abort_flag = 1;
      atomicOr(p.status, 1u /* PARALLAX_DEVICE_STATUS_TIMEOUT */);
      for (int s = 0; s < kStages; ++s)
        if (issued_mask & (1u << s))
          mbar_wait_bounded(bar_full + 8 * s, (issued_par >> s) & 1u, p.timeout_ns, nullptr);
    }
    return;
  }

  // ----------------------------------------------------------- consumers --
  const int group = warp / kConsumerWarps;  // takes the stages of tiles group, group + 2, ...
  float* const merge_scr = reinterpret_cast<float*>(gbase + L.off_merge);
  const int REC = rec_floats(D);
  TcConsumer<D, PROBE, PSPLIT> cs;
  cs.init(warp, lane, base + L.off_p + warp * 512);

  PieceCursor cur;
  cur.init(part, key_space(p), p.B, p.Hkv);
  Piece pc;
  int stage = 0;
  uint32_t ph = 0, fph = 0, tseq = 0;  // tseq: the CTA's tile count, all pieces
  bool ok = true, triggered = false;

  while (ok && cur.next(pc)) {
    cs.load_rows(p, pc.b, pc.g);
    cs.reset();
    for (int k0 = pc.i; k0 < pc.i + pc.len; k0 += kTileKeys, ++tseq) {
      if ((int)(tseq % kConsumerGroups) != group) {  // the other group's tile
        if (++stage == kStages) {
          stage = 0;
          ph ^= 1;
        }
        continue;
      }
      if (!mbar_wait_bounded(bar_full + 8 * stage, ph, p.timeout_ns, abort_flag)) {
        ok = false;
        break;
      }
      if (!triggered) {
        pdl_launch_dependents();
        triggered = true;
      }
      const int nvalid = p.kv_mode == kKvContiguous ? min(kTileKeys, pc.i + pc.len - k0)
                                                    : stage_valid[stage];
      const uint32_t sK = base + stage * kStageBytes;
      cs.tile(sK, sK + kKBytes, nvalid, p.scale_log2);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty + 8 * stage);
      if (++stage == kStages) {
        stage = 0;
        ph ^= 1;
      }
    }
    if (!ok) break;

    // --- end of piece: combine the eight warps, finish or write a partial ---
    cs.write_record(merge_scr + warp * G * REC, G);
    __syncwarp();  // orders the warp's scratch writes before lane 0's release
    if (lane == 0) mbar_arrive(bar_fin);
    if (!mbar_wait_bounded(bar_fin, fph, p.timeout_ns, abort_flag)) {
      ok = false;
      break;
    }
    for (int idx = tid; idx < G * D; idx += kTcConsumers * 32) {
      const int h = idx / D, d = idx - h * D;
      float M, Lw, Bw, Aw, Cw;
      tc_combine_warps<D, PROBE>(merge_scr, G, h, d, M, Lw, Bw, Aw, Cw);
      if (pc.complete) {
        const float inv = Lw > 0.f ? 1.f / Lw : 0.f;  // no attended key: o = 0
        const float vbar = Aw * inv;
        const float o = PROBE ? vbar + Cw * inv - (Bw * inv) * vbar : vbar;
        const size_t oi = ((size_t)pc.b * p.Hq + (size_t)pc.g * G + h) * D + d;
        if (OUT_F32)
          static_cast<float*>(p.out)[oi] = o;
        else
          static_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(o);
      } else {
        float* rec = p.partials + ((size_t)piece_slot(blockIdx.x, pc.first) * G + h) * REC;
        if (d == 0) {
          rec[0] = M;
          rec[1] = Lw;
          rec[2] = Bw;
        }
        rec[kRecHead + d] = Aw;
        if (PROBE) rec[kRecHead + D + d] = Cw;
      }
    }
    if (cur.pos >= cur.hi) break;  // the CTA's last piece: no one overwrites the scratch
    __syncwarp();  // scratch may be overwritten by the next piece
    if (lane == 0) mbar_arrive(bar_fin + 8);
    if (!mbar_wait_bounded(bar_fin + 8, fph, p.timeout_ns, abort_flag)) {
      ok = false;
      break;
    }
    fph ^= 1;
  }
  if (!triggered) pdl_launch_dependents();
  if (!ok) {
    *abort_flag = 1;
    if (lane == 0) atomicOr(p.status, 1u /* PARALLAX_DEVICE_STATUS_TIMEOUT */);
  }
}

}  // namespace plx
