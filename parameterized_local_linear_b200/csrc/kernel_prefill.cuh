// Parallax prefill forward (training shape) on the 5th-generation tensor
// cores: tcgen05.mma with accumulators in TMEM.
//
// parallax-kernel 0.1.0 README, "Training (Triton)": parallax_func(q, r, k, v)
// maps (B, H, L, D) tensors to (B, H, L, D), causal. Row i of query head h
// is the decode output over keys 0..i of kv head h / G:
//   t_ij = scale q_i.k_j, s_ij = r_i.k_j, e_ij = 2^(t_ij log2e - m_i),
//   l = sum e, b = sum e s, A = sum e v, C = sum e s v,
//   o_i = A/l + C/l - (b/l)(A/l).
// Both products are dense contractions here: S = Q K^T and T = R K^T
// (128 query rows x 64 keys x D, operands in shared memory) and O_A = P V,
// O_C = (P o T) V (128 rows x D x 64 keys, P read from TMEM), so they go
// through UMMA.
//
// One CTA per (128-row query tile, query head, batch row); late (heavier,
// causal) tiles first across the whole grid, so that the last wave holds the
// lightest tiles. 320 threads:
//   warp 8  TMA producer: the Q and R tiles once, then 64-key K and V tiles
//           into two rings (128-byte swizzle, the UMMA operand layout)
//   warp 9  owns the 512 TMEM columns and issues every UMMA (one lane), in
//           the order S_j, T_j, then O += P_{j-1} V_{j-1}: the score products
//           of a tile run while the softmax of the tile before finishes
//   warps 0-7  softmax, two threads per query row (TMEM lane): warp w reads
//           lanes 32 (w % 4).. and keys 32 (w / 4).. of each tile. Each takes
//           the row max over all 64 keys (no exchange needed) and writes its
//           32 keys of e and e*s into the P operand in TMEM. O is rescaled in
//           TMEM only when the max grows by more than 2^8 (otherwise the stale
//           max keeps every e <= 2^8); each thread of a row rescales one of
//           O_A, O_C.
// The weights. The value of key i is weighted by e_i (1 + s_i - b/l), so a
// weight's rounding error is multiplied by |s|, which for these probes reaches
// tens: one bf16 per weight is not enough. l and b are always summed from the
// exact values the products apply, so the weights stay consistent.
//   - bf16 output, tile in fp16 range: e 2^-8 (<= 1) and e*s 2^-sigma as one
//     fp16 each (11 significant bits), against an fp16 copy of V that
//     parallax_prefill_prep_kernel wrote beforehand (exact for every bf16
//     below 2^16; it also records, per 64 keys, whether V is in that range
//     and the largest |k|). sigma, a power of two per row fixed at the start
//     from |r_i|_1 max|k| >= |s|, keeps e*s far from fp16's largest value;
//     it is 0 unless r and k are huge.
//   - bf16 output, any other tile (V at or above 2^16, or no workspace for
//     the copy): e and e*s (with the same factors) rounded to 17 significant
//     bits and split exactly into bf16 hi + lo pairs, against bf16 V.
//   - fp32 output: e and e*s (fp32) split into three bf16 terms hi + mid + lo,
//     which sum to them exactly; hi and mid sit where P_hi and P_lo do, and
//     the two lo tiles are A operands in shared memory (TMEM has no room left
//     at D = 128).
// TMEM columns: S [0,64) T [64,128) P [128,256) (per key half, 64 columns:
// P_hi, P_lo, PT_hi, PT_lo, 16 each; an fp16 tile uses the P_hi and PT_hi
// columns), O_A [256, 256+D), O_C [256+D, 256+2D).
// Every wait is bounded; on a timeout the kernel records it, waits (bounded)
// for its own TMA copies and UMMAs in flight, frees TMEM and returns.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace plx {

constexpr int kPfRows = 128;     // query rows per CTA (UMMA M)
constexpr int kPfKeys = 64;      // keys per tile (UMMA N of S, T; K of the PV products)
constexpr int kPfSoftmaxWarps = 8;
constexpr int kPfThreads = 320;  // warps 0-7 softmax, 8 producer, 9 UMMA issuer
constexpr int kPfTmemCols = 512;
constexpr uint32_t kPfColS = 0, kPfColT = 64, kPfColP = 128;

struct PrefillParams {
  void* out;                // dense [B][Hq][L][D]; packed [total][Hq][D]
  unsigned int* status;     // device status word
  const int* cu_seqlens;    // packed layout: [B + 1] sequence starts (nullptr when dense)
  int B, Hq, Hkv, G, L, num_qt, causal;
  int total;                // packed layout: rows of q, k (cu_seqlens is clamped to it)
  float scale_log2;         // > 0
  unsigned long long timeout_ns;
  int debug_skip_first_k;   // testing hook: the producer never loads the first K tile
  // bf16 output with the fp16 copy of V (written by parallax_prefill_prep_kernel):
  // per kv item (dense b * Hkv + g, packed g) and 64-row block of its key rows,
  // bit 16 = V in fp16 range, bits 0-15 = the largest |k| (bf16 bits)
  const uint32_t* vinfo;    // nullptr: every tile takes the bf16 hi + lo weights
  int nblk;                 // blocks per kv item
};

// Before the bf16-output prefill: one CTA per (kv item, 64-row block) reads
// the block's K and V rows once, writes V as fp16 into the workspace copy
// (same layout as V), and records whether every value is below 2^16 in
// magnitude (fp16 then holds each one exactly, down to 2^-17 and within
// 2^-25 below) and the largest |k| of the block. Rows past the item's last
// are skipped. Dense: item = b * Hkv + g, row t at ((item * rows) + t) * D;
// packed: item = g, row t at (t * Hkv + g) * D.
template <int D, bool VARLEN>
__global__ void __launch_bounds__(256)
    parallax_prefill_prep_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                 uint4* __restrict__ v16, uint32_t* __restrict__ vinfo, int rows,
                                 int Hkv, int nblk, int items_per_y, long long items) {
  pdl_launch_dependents();  // the prefill may set up meanwhile; it waits before reading these
  constexpr int kVecPerRow = D / 8;  // 16-byte words of one row
  // grid: blocks in x, items in y (then z past 65535 items)
  const int blk = (int)blockIdx.x;
  const long long item_ll = (long long)blockIdx.z * items_per_y + blockIdx.y;
  if (item_ll >= items) return;
  const int item = (int)item_ll;
  uint32_t km = 0, bad = 0;
#pragma unroll
  for (int it = 0; it < 64 * kVecPerRow / 256; ++it) {
    const int idx = it * 256 + (int)threadIdx.x;
    const int t = blk * 64 + idx / kVecPerRow, c = idx % kVecPerRow;
    if (t >= rows) continue;
    const size_t off =
        (VARLEN ? (size_t)t * Hkv + item : (size_t)item * rows + t) * kVecPerRow + c;
    const uint4 kw = __ldg(k + off), vw = __ldg(v + off);
    const uint32_t kk[4] = {kw.x, kw.y, kw.z, kw.w}, vv[4] = {vw.x, vw.y, vw.z, vw.w};
    uint32_t h[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      km = __vmaxu2(km, kk[x] & 0x7fff7fffu);
      // a half at or above 0x4780 (2^16, inf, NaN) carries into its top bit
      bad |= ((vv[x] & 0x7fff7fffu) + 0x38803880u) & 0x80008000u;
      h[x] = pack_f16x2(bf16_lo_to_float(vv[x]), bf16_hi_to_float(vv[x]));
    }
    v16[off] = make_uint4(h[0], h[1], h[2], h[3]);
  }
  km = max(km & 0xffffu, km >> 16);
  __shared__ uint32_t s_km, s_bad;
  if (threadIdx.x == 0) {
    s_km = 0;
    s_bad = 0;
  }
  __syncthreads();
  km = __reduce_max_sync(0xffffffffu, km);
  bad = __reduce_or_sync(0xffffffffu, bad);
  if ((threadIdx.x & 31) == 0) {
    atomicMax(&s_km, km);
    atomicOr(&s_bad, bad);
  }
  __syncthreads();
  if (threadIdx.x == 0) vinfo[(size_t)item * nblk + blk] = (s_bad ? 0u : 0x10000u) | s_km;
}

template <int D, bool F32 = false>
struct PfGeom {
  static constexpr int kStages = F32 ? 3 : 4;  // depth of the K ring and of the V ring
  static constexpr int kH = D / 64;
  static constexpr int kQBytes = kH * kPfRows * 128;   // Q (or R) tile
  static constexpr int kKVBytes = kH * kPfKeys * 128;  // K (or V) tile
  static constexpr int kOffQ = 0, kOffR = kQBytes, kOffK = 2 * kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKVBytes;
  // fp32 output: the lo terms of e and of e*s, one [128 rows][64 keys] bf16
  // tile each, K-major with the 128-byte swizzle (the UMMA A-operand layout)
  static constexpr int kP3Bytes = kPfRows * kPfKeys * 2;
  static constexpr int kOffP3 = kOffV + kStages * kKVBytes;  // 1024-byte aligned
  static constexpr int kOffRed = kOffP3 + (F32 ? 2 * kP3Bytes : 0);  // l, b of both key halves
  static constexpr int kOffBar = kOffRed + 4 * kPfRows * 4;
  static constexpr int kSmem = kOffBar + 512 + 1024;            // barriers, slots, alignment
  static constexpr uint32_t kColOA = 256, kColOC = 256 + D;
};

// x rounded (half away from zero) to 17 significant bits.
__device__ __forceinline__ float round17(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x40u) & 0xFFFFFF80u);
}

// x0, x1 rounded to 17 significant bits (y), split exactly into bf16 hi + lo:
// hi = y rounded to nearest bf16, lo = y - hi (at most 8 significant bits, so
// exact in bf16). Packed as bf16x2 words (x0 in the low half). Returns y0 + y1.
__device__ __forceinline__ float split_hi_lo(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const float y0 = round17(x0), y1 = round17(x1);
  hi = pack_bf16x2(y0, y1);
  const float l0 = y0 - bf16_lo_to_float(hi), l1 = y1 - bf16_hi_to_float(hi);
  lo = __byte_perm(__float_as_uint(l0), __float_as_uint(l1), 0x7632);
  return y0 + y1;
}

// x0, x1 split into three bf16 terms hi + mid + lo that sum to them exactly
// (each term rounds the remainder of the ones before to nearest; an fp32
// value has 24 significant bits and each term takes 8). Packed as bf16x2
// words (x0 in the low half). Returns x0 + x1.
__device__ __forceinline__ float split3(float x0, float x1, uint32_t& hi, uint32_t& mid,
                                        uint32_t& lo) {
  hi = pack_bf16x2(x0, x1);
  const float r0 = x0 - bf16_lo_to_float(hi), r1 = x1 - bf16_hi_to_float(hi);
  mid = pack_bf16x2(r0, r1);
  lo = pack_bf16x2(r0 - bf16_lo_to_float(mid), r1 - bf16_hi_to_float(mid));
  return x0 + x1;
}

// VARLEN: the packed layout of parallax_varlen_func (q, r, out [total][Hq][D],
// k, v [total][Hkv][D], sequence b in rows cu_seqlens[b] .. cu_seqlens[b+1]);
// otherwise the dense [B][H][L][D] layout.
template <int D, bool OUT_F32, bool VARLEN>
__global__ void __launch_bounds__(kPfThreads, 1)
    parallax_prefill_kernel(const __grid_constant__ CUtensorMap tmQ,
                            const __grid_constant__ CUtensorMap tmR,
                            const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV,
                            const __grid_constant__ CUtensorMap tmV16, const PrefillParams p) {
  using Geo = PfGeom<D, OUT_F32>;
  constexpr int kSt = Geo::kStages;
  constexpr uint32_t kIdescS = umma_idesc_bf16(kPfRows, kPfKeys, false);
  constexpr uint32_t kIdescPV = umma_idesc_bf16(kPfRows, D, true);
  constexpr uint32_t kIdescPV16 = umma_idesc_f16(kPfRows, D, true);
  const float kNegInf = __int_as_float(0xff800000u);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + Geo::kOffQ, sR = base + Geo::kOffR;
  const uint32_t sK = base + Geo::kOffK, sV = base + Geo::kOffV;
  const uint32_t sP3 = base + Geo::kOffP3;  // fp32 output: lo of e, then lo of e*s
  const uint32_t bar = base + Geo::kOffBar;
  // one barrier per ring stage: K full / empty, V full / empty
  const uint32_t bar_q = bar, k_full = bar + 8, k_empty = k_full + 8 * kSt,
                 v_full = k_empty + 8 * kSt, v_empty = v_full + 8 * kSt;
  const uint32_t s_full = v_empty + 8 * kSt, s_free = s_full + 8, p_full = s_full + 16,
                 o_done = s_full + 24, bar_drain = s_full + 32;
  constexpr int kOffMisc = Geo::kOffBar + 8 + 4 * 8 * kSt + 40;
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gbase + kOffMisc);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(gbase + kOffMisc + 4);
  float* const red = reinterpret_cast<float*>(gbase + Geo::kOffRed);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // CTA -> (query tile slot, head h, batch row b): one linear index with the
  // slot slowest (slot 0 is every sequence's last, heaviest causal tile), then
  // h, then b. Slots run to the longest sequence's tile count.
  const int hb = p.Hq * p.B, slot = (int)blockIdx.x / hb;
  const int h = ((int)blockIdx.x - slot * hb) % p.Hq, b = ((int)blockIdx.x - slot * hb) / p.Hq;
  const int g = h / p.G;
  // this sequence: its length L and, packed, its first row s0
  int L = p.L, s0 = 0;
  if (VARLEN) {
    const int a = __ldg(p.cu_seqlens + b), e = __ldg(p.cu_seqlens + b + 1);
    s0 = min(max(a, 0), p.total);
    L = min(max(e, s0), p.total) - s0;
    const bool bad = s0 != a || s0 + L != e;  // outside [0, total] or decreasing
    if (tid == 0 && slot == 0 && h == 0 && (bad || (L + kPfRows - 1) / kPfRows > p.num_qt))
      atomicOr(p.status, 2u /* PARALLAX_DEVICE_STATUS_SEQLEN_CLAMPED */);
  }
  const int num_qt = VARLEN ? (L + kPfRows - 1) / kPfRows : p.num_qt;
  if (slot >= num_qt) return;  // shorter sequence: nothing for this CTA
  const int qt = num_qt - 1 - slot;  // heavy causal tiles first
  const int q0 = qt * kPfRows;
  const int kend = p.causal ? min(L, q0 + kPfRows) : L;  // keys this tile can see
  const int nkt = (kend + kPfKeys - 1) / kPfKeys;
  // TMA coordinates: (row, item) of the Q, R box and of the K, V boxes
  const int qrow = VARLEN ? s0 + q0 : q0, qitem = VARLEN ? h : b * p.Hq + h;
  const int krow = VARLEN ? s0 : 0, kitem = VARLEN ? g : b * p.Hkv + g;
  // fp16 value products for tile j: the 64-row blocks its K/V box covers
  // (rows krow + 64 j .. +63, the tail past the sequence included: masked
  // keys still meet V in the products) all hold V in fp16 range. Every role
  // reads this after the prep kernel has finished (griddepcontrol.wait).
  // Each role loads the two records of tile j + 1 while it works on tile j,
  // so that their latency stays off its critical path.
  const uint32_t* const vinfo_item =
      OUT_F32 || p.vinfo == nullptr ? nullptr : p.vinfo + (size_t)kitem * p.nblk;
  struct TileRecords {
    uint32_t w0 = 0, w1 = 0;
    __device__ bool f16() const { return (w0 & w1 & 0x10000u) != 0u; }
  };
  const auto load_records = [&](int j) {
    TileRecords t;
    if (vinfo_item != nullptr && j < nkt) {
      const int a = krow + j * kPfKeys;
      t.w0 = __ldg(vinfo_item + (a >> 6));
      t.w1 = __ldg(vinfo_item + min((a + kPfKeys - 1) >> 6, p.nblk - 1));
    }
    return t;
  };

  if (tid == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < kSt; ++s) {
      mbar_init(k_full + 8 * s, 1);
      mbar_init(k_empty + 8 * s, 1);
      mbar_init(v_full + 8 * s, 1);
      mbar_init(v_empty + 8 * s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, kPfSoftmaxWarps);
    mbar_init(p_full, kPfSoftmaxWarps);
    mbar_init(o_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 9) tmem_alloc(smem_u32(tmem_slot), kPfTmemCols);
  uint64_t policy = 0;
  if (tid == 8 * 32) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmR);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    if (vinfo_item != nullptr) prefetch_tensormap(&tmV16);
    policy = l2_policy_evict_first();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      bool ok = true;
      bool skipped_k0 = false;  // testing hook
      int last = -1;  // the last tile whose K and V loads were both started
      mbar_arrive_expect_tx(bar_q, 2 * Geo::kQBytes);
      tma_load_4d(sQ, &tmQ, 0, qrow, 0, qitem, bar_q, policy);
      tma_load_4d(sR, &tmR, 0, qrow, 0, qitem, bar_q, policy);
      if (vinfo_item != nullptr) pdl_wait_primary();  // the fp16 copy of V is complete
      TileRecords rec = load_records(0);
      int st = 0;
      uint32_t ph = 0;
      for (int j = 0; j < nkt; ++j) {
        if (!mbar_wait_bounded(k_empty + 8 * st, ph ^ 1, p.timeout_ns, abort_flag)) {
          ok = false;
          break;
        }
        if (j == 0 && p.debug_skip_first_k) {
          skipped_k0 = true;  // the UMMA issuer's wait on this tile must run out
        } else {
          mbar_arrive_expect_tx(k_full + 8 * st, Geo::kKVBytes);
          tma_load_4d(sK + st * Geo::kKVBytes, &tmK, 0, krow + j * kPfKeys, 0, kitem,
                      k_full + 8 * st, policy);
        }
        if (!mbar_wait_bounded(v_empty + 8 * st, ph ^ 1, p.timeout_ns, abort_flag)) {
          if (!skipped_k0 || j > 0)
            mbar_wait_bounded(k_full + 8 * st, ph, p.timeout_ns, nullptr);  // K_j in flight
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(v_full + 8 * st, Geo::kKVBytes);
        const bool f16 = rec.f16();
        rec = load_records(j + 1);
        tma_load_4d(sV + st * Geo::kKVBytes, f16 ? &tmV16 : &tmV, 0, krow + j * kPfKeys, 0,
                    kitem, v_full + 8 * st, policy);
        last = j;
        if (++st == kSt) {
          st = 0;
          ph ^= 1;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(p.status, 1u /* PARALLAX_DEVICE_STATUS_TIMEOUT */);
      }
      // Wait (bounded) until every copy this CTA started has landed: the
      // latest load into each stage is the last one started there.
      mbar_wait_bounded(bar_q, 0, p.timeout_ns, nullptr);
      for (int j = max(0, last - kSt + 1); j <= last; ++j) {
        const int s = j % kSt;
        const uint32_t par = (uint32_t)(j / kSt) & 1u;
        if (!(j == 0 && skipped_k0)) mbar_wait_bounded(k_full + 8 * s, par, p.timeout_ns, nullptr);
        mbar_wait_bounded(v_full + 8 * s, par, p.timeout_ns, nullptr);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------- UMMA issuer --
    if (lane == 0) {
      if (vinfo_item != nullptr) pdl_wait_primary();
      TileRecords rec = load_records(0);
      bool ok = mbar_wait_bounded(bar_q, 0, p.timeout_ns, abort_flag);
      tc_fence_after_sync();
      for (int jj = 0; jj <= nkt && ok; ++jj) {
        if (jj < nkt) {  // S_jj = Q K^T, T_jj = R K^T once the softmax has read S_jj-1
          const int st = jj % kSt;
          const uint32_t par = (uint32_t)(jj / kSt) & 1u;
          if ((jj > 0 && !mbar_wait_bounded(s_free, (jj - 1) & 1, p.timeout_ns, abort_flag)) ||
              !mbar_wait_bounded(k_full + 8 * st, par, p.timeout_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sKs = sK + st * Geo::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t ko = (kk >> 2) * (kPfKeys * 128) + (kk & 3) * 32;
            const uint32_t qo = (kk >> 2) * (kPfRows * 128) + (kk & 3) * 32;
            umma_bf16(tmem + kPfColS, umma_smem_desc(sQ + qo, 16, 1024),
                      umma_smem_desc(sKs + ko, 16, 1024), kIdescS, kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t ko = (kk >> 2) * (kPfKeys * 128) + (kk & 3) * 32;
            const uint32_t qo = (kk >> 2) * (kPfRows * 128) + (kk & 3) * 32;
            umma_bf16(tmem + kPfColT, umma_smem_desc(sR + qo, 16, 1024),
                      umma_smem_desc(sKs + ko, 16, 1024), kIdescS, kk > 0);
          }
          umma_commit(s_full);  // also frees K_jj's stage: softmax warp 0 passes it on
        }
        if (jj >= 1) {  // O_A += P V, O_C += (P o T) V for tile j = jj - 1
          const int j = jj - 1, st = j % kSt;
          const uint32_t par = (uint32_t)(j / kSt) & 1u;
          if (!mbar_wait_bounded(p_full, j & 1, p.timeout_ns, abort_flag) ||
              !mbar_wait_bounded(v_full + 8 * st, par, p.timeout_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sVs = sV + st * Geo::kKVBytes;
          const bool f16 = rec.f16();
          rec = load_records(j + 1);
          if (f16) {
            // fp16 tile: P -> O_A, PT -> O_C, one term each
#pragma unroll
            for (int pm = 0; pm < 4; pm += 2) {
              const uint32_t dO = tmem + (pm == 0 ? Geo::kColOA : Geo::kColOC);
#pragma unroll
              for (int kk = 0; kk < kPfKeys / 16; ++kk)
                umma_ts(dO, tmem + kPfColP + 64 * (kk >> 1) + 16 * pm + 8 * (kk & 1),
                        umma_smem_desc(sVs + kk * 16 * 128, kPfKeys * 128, 1024), kIdescPV16,
                        !(j == 0 && kk == 0));
            }
          } else {
#pragma unroll
            for (int pm = 0; pm < 4; ++pm) {  // P_hi, P_lo -> O_A; PT_hi, PT_lo -> O_C
              const uint32_t dO = tmem + (pm < 2 ? Geo::kColOA : Geo::kColOC);
#pragma unroll
              for (int kk = 0; kk < kPfKeys / 16; ++kk) {
                const bool acc = !(j == 0 && (pm & 1) == 0 && kk == 0);
                // keys 16 kk .. +15 sit in half kk / 2's 64 columns: 16 per operand
                umma_ts(dO, tmem + kPfColP + 64 * (kk >> 1) + 16 * pm + 8 * (kk & 1),
                        umma_smem_desc(sVs + kk * 16 * 128, kPfKeys * 128, 1024), kIdescPV, acc);
              }
            }
          }
          if constexpr (OUT_F32) {  // the lo terms, A from shared memory: e -> O_A, e*s -> O_C
#pragma unroll
            for (int pm = 0; pm < 2; ++pm) {
              const uint32_t dO = tmem + (pm == 0 ? Geo::kColOA : Geo::kColOC);
              const uint32_t sA = sP3 + pm * Geo::kP3Bytes;
#pragma unroll
              for (int kk = 0; kk < kPfKeys / 16; ++kk)
                umma_bf16(dO, umma_smem_desc(sA + 32 * kk, 16, 1024),
                          umma_smem_desc(sVs + kk * 16 * 128, kPfKeys * 128, 1024), kIdescPV,
                          true);
            }
          }
          umma_commit(o_done);  // also frees V_j's stage: softmax warp 0 passes it on
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(p.status, 1u);
      }
      umma_commit(bar_drain);  // every UMMA issued above is done once this arrives
      mbar_wait_bounded(bar_drain, 0, p.timeout_ns, nullptr);
    }
  } else {
    // ------------------------------------- softmax: two threads per row --
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane, qi = q0 + r;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + kPfColS, tT = tmem + lane_base + kPfColT;
    const uint32_t tP = tmem + lane_base + kPfColP + 64 * half;  // this half's 64 columns
    const float c = p.scale_log2;
    float m_used = kNegInf, l = 0.f, bsum = 0.f;
    bool ok = true;
    // e*s enters the products (and b) as e*s 2^-sigma: sigma is the smallest
    // power keeping |r_i|_1 max|k| 2^-sigma, a bound on |s|, below 2^14 for
    // every key this CTA reads, so that fp16 holds e*s. Both threads of a row
    // compute the same sigma.
    float pt_scale = 1.f, pt_unscale = 1.f;
    if constexpr (!OUT_F32) {
      if (vinfo_item != nullptr) {
        pdl_wait_primary();  // the prep kernel's records are complete
        const int b_lo = krow >> 6, b_hi = min((krow + nkt * kPfKeys - 1) >> 6, p.nblk - 1);
        uint32_t km = 0;
        for (int bb = b_lo + lane; bb <= b_hi; bb += 32) km = max(km, __ldg(vinfo_item + bb) & 0xffffu);
        km = __reduce_max_sync(0xffffffffu, km);
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar_q, 0, p.timeout_ns, abort_flag));
        float rl1 = 0.f;
        if (ok) {
          const uint4* const rrow = reinterpret_cast<const uint4*>(gbase + Geo::kOffR) + r * 8;
#pragma unroll
          for (int hh = 0; hh < Geo::kH; ++hh) {
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {  // staggered 16-byte chunks of the row
              const uint4 w = rrow[hh * (kPfRows * 8) + ((cc + lane) & 7)];
              const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int x = 0; x < 4; ++x)
                rl1 += bf16_lo_to_float(u[x] & 0x7fffu) + bf16_hi_to_float(u[x] & 0x7fff0000u);
            }
          }
        }
        const float bound = rl1 * __uint_as_float(km << 16);
        // 2^-sigma and 2^sigma stay normal floats for sigma <= 126, which covers
        // every finite bound (below 2^128); an infinite bound (its product
        // overflowed) takes 126, which brings any finite |s| below 4
        int sigma = 0;
        if (!(bound < 16384.f))  // also inf and NaN
          sigma = bound < 3.0e38f ? (int)((__float_as_uint(bound) >> 23) & 0xffu) - 127 - 13 : 126;
        sigma = min(max(sigma, 0), 126);
        pt_scale = __int_as_float((127 - sigma) << 23);
        pt_unscale = __int_as_float((127 + sigma) << 23);
      }
    }
    TileRecords rec = load_records(0);
    for (int j = 0; j < nkt && ok; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(s_full, j & 1, p.timeout_ns, abort_flag))) {
        ok = false;
        *abort_flag = 1;
        break;
      }
      tc_fence_after_sync();
      float sv[32], so[32], tv[32];
      tmem_ld32(tS + 32 * half, sv);
      tmem_ld32(tS + 32 * (half ^ 1), so);
      tmem_ld32(tT + 32 * half, tv);
      tmem_wait_ld();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      // S_j, T_j complete: the score UMMAs have read K_j, so its stage can be
      // refilled (an arrive here instead of a second commit by the issuer,
      // each of which costs the tensor pipe ~50 ns)
      if (warp == 0 && lane == 0) mbar_arrive(k_empty + 8 * (j % kSt));
      // causal mask (only tiles that reach past this tile's first row or the
      // end of the sequence need one) and the row max over all 64 keys
      const int k0 = j * kPfKeys, kown = k0 + 32 * half, kother = k0 + 32 * (half ^ 1);
      float mx = kNegInf;
      if (k0 + kPfKeys <= (p.causal ? min(kend, q0 + 1) : kend)) {
#pragma unroll
        for (int x = 0; x < 32; ++x) mx = fmaxf(mx, fmaxf(sv[x], so[x]));
      } else {
        const int klim = p.causal ? min(kend, qi + 1) : kend;  // keys below klim are seen
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const bool own = kown + x < klim;
          sv[x] = own ? sv[x] : kNegInf;
          tv[x] = own ? tv[x] : 0.f;
          mx = fmaxf(mx, fmaxf(sv[x], kother + x < klim ? so[x] : kNegInf));
        }
      }
      mx *= c;  // the scale is positive: this is the max of the scaled scores
      // lazy rescale: keep the stale max unless this tile exceeds it by 2^8
      float alpha = 1.f;
      const bool grow = mx > m_used + 8.f;
      if (grow) {
        alpha = m_used == kNegInf ? 0.f : ex2_approx(m_used - mx);
        m_used = mx;
      }
      // bf16 output: the weights are e 2^-8 (<= 1 under the lazy max), in
      // every tile, so that fp16 holds them; l, b, A, C share the factor
      const float neg_m = OUT_F32 ? -m_used : -m_used - 8.f;
      bool f16 = false;  // this tile's value products take fp16 operands
      if constexpr (!OUT_F32) {
        f16 = rec.f16();
        rec = load_records(j + 1);
      }
      // The previous PV products must be done before P is overwritten (it is
      // single-buffered) and before O is rescaled. Each weight format below
      // computes its weights first, so that they overlap those products.
      auto prev_done_and_rescale = [&]() -> bool {
        if (j == 0) return true;
        if (!__all_sync(0xffffffffu,
                        mbar_wait_bounded(o_done, (j - 1) & 1, p.timeout_ns, abort_flag)))
          return false;
        tc_fence_after_sync();
        // the value UMMAs of tile j - 1 have read V_{j-1}: its stage can be refilled
        if (warp == 0 && lane == 0) mbar_arrive(v_empty + 8 * ((j - 1) % kSt));
        if (__any_sync(0xffffffffu, grow)) {  // warp-uniform: alpha is 1 on the other rows
          const uint32_t tO = tmem + lane_base + (half ? Geo::kColOC : Geo::kColOA);
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            float o[32];
            tmem_ld32(tO + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] *= alpha;
            tmem_st32(tO + c0, o);
          }
        }
        return true;
      };
      float lt = 0.f, bt = 0.f;
      if (f16) {
        // one fp16 term each, at the P_hi and PT_hi columns; l and b add the
        // rounded values the products apply
        uint32_t ph[16], th[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const uint32_t pe = pack_f16x2(ex2_approx(fmaf(sv[2 * u], c, neg_m)),
                                         ex2_approx(fmaf(sv[2 * u + 1], c, neg_m)));
          const float a0 = f16_lo_to_float(pe), a1 = f16_hi_to_float(pe);
          const uint32_t pes =
              pack_f16x2(a0 * pt_scale * tv[2 * u], a1 * pt_scale * tv[2 * u + 1]);
          lt += a0 + a1;
          bt += f16_lo_to_float(pes) + f16_hi_to_float(pes);
          ph[u] = pe;
          th[u] = pes;
        }
        if (!prev_done_and_rescale()) {
          ok = false;
          *abort_flag = 1;
          break;
        }
        tmem_st16u(tP, ph);
        tmem_st16u(tP + 32, th);
      } else {
        // e and e*s of this thread's 32 keys as exact bf16 hi + lo pairs, in
        // the order of this half's P columns: P_hi | P_lo then PT_hi | PT_lo.
        // With fp32 output: hi | mid in those columns and the lo terms in p3, pt3.
        uint32_t pp[32], pt[32];
        uint32_t p3[OUT_F32 ? 16 : 1], pt3[OUT_F32 ? 16 : 1];
        uint32_t* const ph = pp;
        uint32_t* const pl = pp + 16;
        uint32_t* const th = pt;
        uint32_t* const tl = pt + 16;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float e0 = ex2_approx(fmaf(sv[2 * u], c, neg_m));
          const float e1 = ex2_approx(fmaf(sv[2 * u + 1], c, neg_m));
          if constexpr (OUT_F32) {
            lt += split3(e0, e1, ph[u], pl[u], p3[u]);
            bt += split3(e0 * tv[2 * u], e1 * tv[2 * u + 1], th[u], tl[u], pt3[u]);
          } else {
            lt += split_hi_lo(e0, e1, ph[u], pl[u]);
            // e*s from the rounded e: the weights P applies
            const float es0 = round17(e0) * pt_scale * tv[2 * u];
            const float es1 = round17(e1) * pt_scale * tv[2 * u + 1];
            bt += split_hi_lo(es0, es1, th[u], tl[u]);
          }
        }
        if (!prev_done_and_rescale()) {
          ok = false;
          *abort_flag = 1;
          break;
        }
        if constexpr (OUT_F32) {
          // row r of the lo tiles: keys 32 half .. +31 are 16-byte chunks
          // 4 half .. +3, each at chunk position (chunk ^ (r mod 8)) of the row
          const uint32_t row = sP3 + (uint32_t)r * 128u, sw = (uint32_t)r & 7u;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const uint32_t off = (((uint32_t)(4 * half + c4)) ^ sw) << 4;
            st_shared_v4(row + off, p3[4 * c4], p3[4 * c4 + 1], p3[4 * c4 + 2], p3[4 * c4 + 3]);
            st_shared_v4(row + Geo::kP3Bytes + off, pt3[4 * c4], pt3[4 * c4 + 1], pt3[4 * c4 + 2],
                         pt3[4 * c4 + 3]);
          }
          fence_proxy_async_smem();  // the UMMAs read these tiles through the async proxy
        }
        tmem_st32u(tP, pp);
        tmem_st32u(tP + 32, pt);
      }
      l = l * alpha + lt;
      bsum = bsum * alpha + bt;
      tmem_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // epilogue: l and b of the two key halves, then o = A/l + C/l - (b/l)(A/l)
    red[half * kPfRows + r] = l;
    red[(2 + half) * kPfRows + r] = bsum;
    asm volatile("bar.sync 1, %0;" ::"n"(kPfSoftmaxWarps * 32) : "memory");
    const float lsum = red[r] + red[kPfRows + r];
    const float bfull = red[2 * kPfRows + r] + red[3 * kPfRows + r];
    if (ok && __all_sync(0xffffffffu,
                         mbar_wait_bounded(o_done, (nkt - 1) & 1, p.timeout_ns, abort_flag))) {
      tc_fence_after_sync();
      const float inv = 1.f / lsum, bl = bfull * inv;
#pragma unroll 1
      for (int c0 = half * (D / 2); c0 < (half + 1) * (D / 2); c0 += 32) {
        float a[32], cc[32];
        tmem_ld32(tmem + lane_base + Geo::kColOA + c0, a);
        tmem_ld32(tmem + lane_base + Geo::kColOC + c0, cc);
        tmem_wait_ld();
        if (qi < L) {
          const size_t oi = (VARLEN ? ((size_t)(s0 + qi) * p.Hq + h)
                                    : (((size_t)b * p.Hq + h) * L + qi)) * D + c0;
#pragma unroll
          for (int x = 0; x < 32; x += 4) {
            float o4[4];
#pragma unroll
            for (int y = 0; y < 4; ++y) {  // C and b carry the factor 2^-sigma
              const float vbar = a[x + y] * inv;
              o4[y] = vbar + pt_unscale * (cc[x + y] * inv - bl * vbar);
            }
            if (OUT_F32) {
              *reinterpret_cast<float4*>(static_cast<float*>(p.out) + oi + x) =
                  make_float4(o4[0], o4[1], o4[2], o4[3]);
            } else {
              uint2 pk;
              pk.x = pack_bf16x2(o4[0], o4[1]);
              pk.y = pack_bf16x2(o4[2], o4[3]);
              *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.out) + oi + x) = pk;
            }
          }
        }
      }
    } else {
      ok = false;
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) atomicOr(p.status, 1u);
    }
  }
  // teardown: every role is done with TMEM (UMMAs drained, loads waited)
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 9) tmem_dealloc(tmem, kPfTmemCols);
}

}  // namespace plx
