// Parallax prefill forward (training shape) on the 5th-generation tensor
// cores: tcgen05.mma with operands in shared memory and accumulators in TMEM.
//
// parallax-kernel 0.1.0 README, "Training (Triton)": parallax_func(q, r, k, v)
// maps (B, H, L, D) tensors to (B, H, L, D), causal. Row i of query head h
// is the decode output over keys 0..i of kv head h / G:
//   t_ij = scale q_i.k_j, s_ij = r_i.k_j, e_ij = 2^(t_ij log2e - m_i),
//   l = sum e, b = sum e s, A = sum e v, C = sum e s v,
//   o_i = A/l + C/l - (b/l)(A/l).
// Both products are dense contractions here: S = Q K^T and T = R K^T
// (128 query rows x 64 keys x D) and O_A = P V, O_C = (P o T) V
// (128 rows x D x 64 keys), so they go through UMMA.
//
// One CTA per (128-row query tile, query head, batch row); late (heavier,
// causal) tiles first. 192 threads:
//   warp 4  TMA producer: the Q and R tiles once, then 64-key K and V tiles
//           into a 2-stage ring (128-byte swizzle, the UMMA operand layout)
//   warp 5  owns the 512 TMEM columns and issues every UMMA (one lane):
//           S_j, T_j into double-buffered TMEM, then O += P_j V_j
//   warps 0-3  one query row per thread (= its TMEM lane): causal mask,
//           online max, e and e*s as bf16 hi + lo pairs written as swizzled
//           A operands for the PV products, l and b from the same hi + lo
//           values; O is rescaled in TMEM only when the max grows by more
//           than 2^8 (otherwise the stale max keeps every e <= 2^8).
// TMEM columns: S_0 [0,64) T_0 [64,128) S_1 [128,192) T_1 [192,256),
// O_A [256, 256+D), O_C [256+D, 256+2D).
// Every wait is bounded; on a timeout the kernel records it, waits (bounded)
// for its own TMA copies and UMMAs in flight, frees TMEM and returns.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace plx {

constexpr int kPfRows = 128;     // query rows per CTA (UMMA M)
constexpr int kPfKeys = 64;      // keys per tile (UMMA N of S, T; K of the PV products)
constexpr int kPfThreads = 192;  // warps 0-3 softmax, 4 producer, 5 UMMA issuer
constexpr int kPfTmemCols = 512;

struct PrefillParams {
  void* out;             // [B][Hq][L][D]
  unsigned int* status;  // device status word
  int B, Hq, Hkv, G, L, num_qt, causal;
  float scale_log2;
  unsigned long long timeout_ns;
};

template <int D>
struct PfGeom {
  static constexpr int kH = D / 64;
  static constexpr int kQBytes = kH * kPfRows * 128;   // Q (or R) tile
  static constexpr int kKVBytes = kH * kPfKeys * 128;  // K (or V) tile
  static constexpr int kPBytes = kPfRows * 128;        // one [128 rows][64 keys] bf16 tile
  static constexpr int kOffQ = 0, kOffR = kQBytes, kOffKV = 2 * kQBytes;
  static constexpr int kOffP = kOffKV + 2 * 2 * kKVBytes;  // 2 stages of K + V
  static constexpr int kOffBar = kOffP + 4 * kPBytes;     // P_hi, P_lo, PT_hi, PT_lo
  static constexpr int kSmem = kOffBar + 128 + 1024;      // barriers, slots, alignment
  static constexpr int kColOA = 256, kColOC = 256 + D;
};

template <int D, bool OUT_F32>
__global__ void __launch_bounds__(kPfThreads, 1)
    parallax_prefill_kernel(const __grid_constant__ CUtensorMap tmQ,
                            const __grid_constant__ CUtensorMap tmR,
                            const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using Geo = PfGeom<D>;
  constexpr int kH = Geo::kH;
  constexpr uint32_t kIdescS = umma_idesc_bf16(kPfRows, kPfKeys, false);
  constexpr uint32_t kIdescPV = umma_idesc_bf16(kPfRows, D, true);
  const float kNegInf = __int_as_float(0xff800000u);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + Geo::kOffQ, sR = base + Geo::kOffR, sKV = base + Geo::kOffKV;
  const uint32_t sP = base + Geo::kOffP;
  const uint32_t bar = base + Geo::kOffBar;
  const uint32_t bar_q = bar, bar_kv_full = bar + 8, bar_kv_empty = bar + 24;
  const uint32_t bar_s = bar + 40, bar_p = bar + 56, bar_o = bar + 64, bar_drain = bar + 72;
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gbase + Geo::kOffBar + 96);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(gbase + Geo::kOffBar + 100);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = p.num_qt - 1 - (int)blockIdx.x;  // heavy causal tiles first
  const int h = blockIdx.y, b = blockIdx.z, g = h / p.G;
  const int q0 = qt * kPfRows;
  const int kend = p.causal ? min(p.L, q0 + kPfRows) : p.L;  // keys this tile can see
  const int nkt = (kend + kPfKeys - 1) / kPfKeys;

  if (tid == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_kv_full + 8 * s, 1);
      mbar_init(bar_kv_empty + 8 * s, 1);
      mbar_init(bar_s + 8 * s, 1);
    }
    mbar_init(bar_p, kPfRows);
    mbar_init(bar_o, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 5) tmem_alloc(smem_u32(tmem_slot), kPfTmemCols);
  uint64_t policy = 0;
  if (tid == 4 * 32) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmR);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    policy = l2_policy_evict_first();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      bool ok = true;
      uint32_t issued = 0;  // bit s: stage s has a load in flight of tile `last[s]`
      int last[2] = {0, 0};
      mbar_arrive_expect_tx(bar_q, 2 * Geo::kQBytes);
      tma_load_4d(sQ, &tmQ, 0, q0, 0, b * p.Hq + h, bar_q, policy);
      tma_load_4d(sR, &tmR, 0, q0, 0, b * p.Hq + h, bar_q, policy);
      for (int j = 0; j < nkt && ok; ++j) {
        const int st = j & 1;
        if (!mbar_wait_bounded(bar_kv_empty + 8 * st, ((j >> 1) & 1) ^ 1, p.timeout_ns,
                               abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t full = bar_kv_full + 8 * st;
        const uint32_t sK = sKV + st * 2 * Geo::kKVBytes;
        mbar_arrive_expect_tx(full, 2 * Geo::kKVBytes);
        tma_load_4d(sK, &tmK, 0, j * kPfKeys, 0, b * p.Hkv + g, full, policy);
        tma_load_4d(sK + Geo::kKVBytes, &tmV, 0, j * kPfKeys, 0, b * p.Hkv + g, full, policy);
        issued |= 1u << st;
        last[st] = j;
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(p.status, 1u /* PARALLAX_DEVICE_STATUS_TIMEOUT */);
      }
      // Wait (bounded) until every copy this CTA started has landed.
      mbar_wait_bounded(bar_q, 0, p.timeout_ns, nullptr);
      for (int s = 0; s < 2; ++s)
        if (issued & (1u << s))
          mbar_wait_bounded(bar_kv_full + 8 * s, (last[s] >> 1) & 1, p.timeout_ns, nullptr);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------- UMMA issuer --
    if (lane == 0) {
      bool ok = mbar_wait_bounded(bar_q, 0, p.timeout_ns, abort_flag);
      tc_fence_after_sync();
      for (int jj = 0; jj <= nkt && ok; ++jj) {
        if (jj < nkt) {  // S_jj = Q K^T, T_jj = R K^T
          const int st = jj & 1;
          if (!mbar_wait_bounded(bar_kv_full + 8 * st, (jj >> 1) & 1, p.timeout_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sK = sKV + st * 2 * Geo::kKVBytes;
          const uint32_t dS = tmem + 128 * st, dT = dS + 64;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t ko = (kk >> 2) * (kPfKeys * 128) + (kk & 3) * 32;
            const uint32_t qo = (kk >> 2) * (kPfRows * 128) + (kk & 3) * 32;
            umma_bf16(dS, umma_smem_desc(sQ + qo, 16, 1024), umma_smem_desc(sK + ko, 16, 1024),
                      kIdescS, kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t ko = (kk >> 2) * (kPfKeys * 128) + (kk & 3) * 32;
            const uint32_t qo = (kk >> 2) * (kPfRows * 128) + (kk & 3) * 32;
            umma_bf16(dT, umma_smem_desc(sR + qo, 16, 1024), umma_smem_desc(sK + ko, 16, 1024),
                      kIdescS, kk > 0);
          }
          umma_commit(bar_s + 8 * st);
        }
        if (jj >= 1) {  // O_A += P V, O_C += (P o T) V for tile j = jj - 1
          const int j = jj - 1, st = j & 1;
          if (!mbar_wait_bounded(bar_p, j & 1, p.timeout_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sV = sKV + st * 2 * Geo::kKVBytes + Geo::kKVBytes;
#pragma unroll
          for (int pm = 0; pm < 4; ++pm) {  // P_hi, P_lo -> O_A; PT_hi, PT_lo -> O_C
            const uint32_t dO = tmem + (pm < 2 ? Geo::kColOA : Geo::kColOC);
#pragma unroll
            for (int kk = 0; kk < kPfKeys / 16; ++kk) {
              const bool acc = !(j == 0 && (pm & 1) == 0 && kk == 0);
              umma_bf16(dO, umma_smem_desc(sP + pm * Geo::kPBytes + kk * 32, 16, 1024),
                        umma_smem_desc(sV + kk * 16 * 128, kPfKeys * 128, 1024), kIdescPV, acc);
            }
          }
          umma_commit(bar_o);
          umma_commit(bar_kv_empty + 8 * st);
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
    // ------------------------------------------- softmax: one row / thread --
    const int r = tid, qi = q0 + r;
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    float m_used = kNegInf, l = 0.f, bsum = 0.f;
    bool ok = true;
    for (int j = 0; j < nkt && ok; ++j) {
      const int sb = j & 1;
      if (!mbar_wait_bounded(bar_s + 8 * sb, (j >> 1) & 1, p.timeout_ns, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      float sv[64], tv[64];
      {
        float a[32], c[32];
        tmem_ld32(tmem + lane_base + 128 * sb, a);
        tmem_ld32(tmem + lane_base + 128 * sb + 32, c);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          sv[x] = a[x];
          sv[32 + x] = c[x];
        }
        tmem_ld32(tmem + lane_base + 128 * sb + 64, a);
        tmem_ld32(tmem + lane_base + 128 * sb + 96, c);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          tv[x] = a[x];
          tv[32 + x] = c[x];
        }
      }
      // causal mask and the row max of this tile (log2 domain)
      const int k0 = j * kPfKeys;
      const int klim = p.causal ? min(kend, qi + 1) : kend;  // keys k0 + x < klim are seen
      float mx = kNegInf;
#pragma unroll
      for (int x = 0; x < 64; ++x) {
        const bool valid = k0 + x < klim;
        sv[x] = valid ? sv[x] * p.scale_log2 : kNegInf;
        tv[x] = valid ? tv[x] : 0.f;
        mx = fmaxf(mx, sv[x]);
      }
      // lazy rescale: keep the stale max unless this tile exceeds it by 2^8
      float alpha = 1.f;
      const bool grow = mx > m_used + 8.f;
      if (grow) {
        alpha = m_used == kNegInf ? 0.f : ex2_approx(m_used - mx);
        m_used = mx;
      }
      // the previous PV product must be done: P is single-buffered and O may be rescaled
      if (j > 0) {
        if (!mbar_wait_bounded(bar_o, (j - 1) & 1, p.timeout_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        if (grow) {
#pragma unroll 1
          for (int c0 = 0; c0 < 2 * D; c0 += 32) {
            float o[32];
            tmem_ld32(tmem + lane_base + Geo::kColOA + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] *= alpha;
            tmem_st32(tmem + lane_base + Geo::kColOA + c0, o);
          }
          tmem_wait_st();
        }
      }
      l *= alpha;
      bsum *= alpha;
      // e and e*s as bf16 hi + lo, written row r of the four swizzled P tiles
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        uint32_t ph[4], pl[4], th[4], tl[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int x = 8 * c8 + 2 * u;
          const float e0 = ex2_approx(sv[x] - m_used), e1 = ex2_approx(sv[x + 1] - m_used);
          const float es0 = e0 * tv[x], es1 = e1 * tv[x + 1];
          ph[u] = pack_bf16x2(e0, e1);
          pl[u] = pack_bf16x2(e0 - bf16_lo_to_float(ph[u]), e1 - bf16_hi_to_float(ph[u]));
          th[u] = pack_bf16x2(es0, es1);
          tl[u] = pack_bf16x2(es0 - bf16_lo_to_float(th[u]), es1 - bf16_hi_to_float(th[u]));
          l += (bf16_lo_to_float(ph[u]) + bf16_lo_to_float(pl[u])) +
               (bf16_hi_to_float(ph[u]) + bf16_hi_to_float(pl[u]));
          bsum += (bf16_lo_to_float(th[u]) + bf16_lo_to_float(tl[u])) +
                  (bf16_hi_to_float(th[u]) + bf16_hi_to_float(tl[u]));
        }
        const uint32_t off = r * 128 + ((c8 ^ (r & 7)) << 4);
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sP + off), "r"(ph[0]),
                     "r"(ph[1]), "r"(ph[2]), "r"(ph[3])
                     : "memory");
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sP + Geo::kPBytes + off),
                     "r"(pl[0]), "r"(pl[1]), "r"(pl[2]), "r"(pl[3])
                     : "memory");
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sP + 2 * Geo::kPBytes + off),
                     "r"(th[0]), "r"(th[1]), "r"(th[2]), "r"(th[3])
                     : "memory");
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sP + 3 * Geo::kPBytes + off),
                     "r"(tl[0]), "r"(tl[1]), "r"(tl[2]), "r"(tl[3])
                     : "memory");
      }
      fence_proxy_async_smem();  // the tensor cores read P through the async proxy
      tc_fence_before_sync();
      mbar_arrive(bar_p);
    }
    // epilogue: o = A/l + C/l - (b/l)(A/l)
    if (ok && mbar_wait_bounded(bar_o, (nkt - 1) & 1, p.timeout_ns, abort_flag)) {
      tc_fence_after_sync();
      const float inv = 1.f / l, bl = bsum * inv;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        float a[32], c[32];
        tmem_ld32(tmem + lane_base + Geo::kColOA + c0, a);
        tmem_ld32(tmem + lane_base + Geo::kColOC + c0, c);
        tmem_wait_ld();
        if (qi < p.L) {
          const size_t oi = (((size_t)b * p.Hq + h) * p.L + qi) * D + c0;
#pragma unroll
          for (int x = 0; x < 32; x += 4) {
            float o4[4];
#pragma unroll
            for (int y = 0; y < 4; ++y) {
              const float vbar = a[x + y] * inv;
              o4[y] = vbar + c[x + y] * inv - bl * vbar;
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
    } else if (ok) {
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
  if (warp == 5) tmem_dealloc(tmem, kPfTmemCols);
}

}  // namespace plx
