// Generic split-KV Parallax decode kernel: fp32 (or bf16) inputs, plain FMA
// arithmetic, any GQA group size. It serves the fp32 input mode and shapes
// the tensor-core kernel does not cover; it shares the partitioning, the
// partial-record format and the merge kernel with that kernel.
//
// A piece's keys go through shared memory in chunks of 32, the loads of chunk
// c + 1 in flight (in registers) while chunk c is processed, for up to four
// query heads of the group per pass. Paged and block-sparse rows resolve each
// chunk through tile_source (a chunk never straddles a 64-key tile, since
// pieces start on whole tiles), and only the attended prefix of a tile is
// loaded. Warp w scores head w, one key per lane
// (t = scale*log2(e) q.k, s = r.k; K padded by one float per row so the lanes
// hit distinct banks), takes the chunk max with shuffles and writes the
// weights e = 2^(t-m') and e*s; then thread d (< D) updates the accumulators
// of dimension d of each head:
//   m' = max(m, max t), alpha = 2^(m-m'),
//   l = alpha l + sum e, b = alpha b + sum e s,
//   A_d = alpha A_d + sum e v_d, C_d = alpha C_d + sum e s v_d.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"
#include "partition.cuh"
#include "ptx.cuh"

namespace plx {

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

constexpr int kGenericChunk = 32;                        // keys per chunk: one per lane
constexpr int kGenericHeads = kGenericThreads / 32;      // query heads per pass: one per warp

template <typename T, int D, bool PROBE, bool OUT_F32>
__global__ void __launch_bounds__(kGenericThreads)
    parallax_generic_kernel(const DecodeParams p) {
  static_assert(D % 4 == 0 && D <= kGenericThreads, "one thread per output dimension");
  constexpr int HP = kGenericHeads;
  constexpr int kPer = kGenericChunk * D / kGenericThreads;  // staged values per thread
  __shared__ float s_k[kGenericChunk][D + 1];
  __shared__ float s_v[kGenericChunk][D];
  __shared__ float s_q[HP][D], s_r[HP][D];
  __shared__ float s_e[HP][kGenericChunk], s_es[HP][kGenericChunk];
  __shared__ float s_m[HP], s_alpha[HP];
  const float kNegInf = __int_as_float(0xff800000u);

  pdl_wait_primary();  // launched with programmatic stream serialisation
  const PartitionInfo part =
      locate_partition(key_space(p), p.B, p.Hkv, blockIdx.x, gridDim.x);
  if (blockIdx.x == 0 && threadIdx.x == 0 && part.clamped) atomicOr(p.status, 2u);
  pdl_launch_dependents();
  if (part.lo >= part.hi) return;

  const T* q = static_cast<const T*>(p.q);
  const T* r = static_cast<const T*>(p.r);
  const T* k = static_cast<const T*>(p.k);
  const T* v = static_cast<const T*>(p.v);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, G = p.G;
  constexpr int REC = rec_floats(D);

  PieceCursor cur;
  cur.init(part, key_space(p), p.B, p.Hkv);
  Piece pc;
  while (cur.next(pc)) {
    const int nchunks = (pc.len + kGenericChunk - 1) / kGenericChunk;
    for (int h0 = 0; h0 < G; h0 += HP) {
      const int nh = min(HP, G - h0);
      const size_t row0 = ((size_t)pc.b * p.Hq + (size_t)pc.g * G + h0) * D;
      __syncthreads();  // the previous pass is done with the shared arrays
      for (int idx = tid; idx < nh * D; idx += kGenericThreads) {
        s_q[idx / D][idx % D] = to_f32(q[row0 + idx]);
        s_r[idx / D][idx % D] = PROBE ? to_f32(r[row0 + idx]) : 0.f;
      }
      if (tid < HP) s_m[tid] = kNegInf;
      float l[HP], bs[HP], A[HP], C[HP];
#pragma unroll
      for (int hh = 0; hh < HP; ++hh) l[hh] = bs[hh] = A[hh] = C[hh] = 0.f;

      float kr[kPer], vr[kPer];
      int nv_next = 0;
      // chunk c's K and V values of this thread (coalesced), and its count of
      // attended keys (a prefix of the chunk)
      auto load_chunk = [&](int c) {
        const int k0 = pc.i + c * kGenericChunk;  // position in the item's key space
        int nv = min(kGenericChunk, pc.i + pc.len - k0);
        long long first;  // element offset of the chunk's first key in K and V
        if (p.kv_mode == kKvContiguous) {
          first = pc.b * p.kv_sb + pc.g * p.kv_sh + (long long)(pc.kbase + k0) * p.kv_sk;
        } else {
          const int o = k0 & (kRangeAlign - 1);
          int key, item, nvt;
          tile_source(p, pc.b, k0 - o, &key, &item, &nvt);
          nv = max(0, min(nv, nvt - o));
          first = item * p.kv_sb + pc.g * p.kv_sh + (long long)(key + o) * p.kv_sk;
        }
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
          const int idx = tid + u * kGenericThreads, j = idx / D, d = idx % D;
          const long long off = first + (long long)(j < nv ? j : 0) * p.kv_sk + d;
          kr[u] = j < nv ? to_f32(k[off]) : 0.f;
          vr[u] = j < nv ? to_f32(v[off]) : 0.f;
        }
        nv_next = nv;
      };
      load_chunk(0);
      for (int c = 0; c < nchunks; ++c) {
        const int nk = nv_next;  // attended keys of this chunk
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
          const int idx = tid + u * kGenericThreads;
          s_k[idx / D][idx % D] = kr[u];
          s_v[idx / D][idx % D] = vr[u];
        }
        __syncthreads();
        if (c + 1 < nchunks) load_chunk(c + 1);  // in flight while this chunk is used
        if (warp < nh) {  // warp = head, lane = key
          float t0 = 0.f, t1 = 0.f, s0 = 0.f, s1 = 0.f;
#pragma unroll 8
          for (int d = 0; d < D; d += 2) {
            const float k0d = s_k[lane][d], k1d = s_k[lane][d + 1];
            t0 = fmaf(s_q[warp][d], k0d, t0);
            t1 = fmaf(s_q[warp][d + 1], k1d, t1);
            if (PROBE) {
              s0 = fmaf(s_r[warp][d], k0d, s0);
              s1 = fmaf(s_r[warp][d + 1], k1d, s1);
            }
          }
          const float t = lane < nk ? (t0 + t1) * p.scale_log2 : kNegInf;
          float mc = t;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
          const float mo = s_m[warp], mn = fmaxf(mo, mc);
          const float e = lane < nk ? exp2f(t - mn) : 0.f;
          s_e[warp][lane] = e;
          s_es[warp][lane] = e * (s0 + s1);
          __syncwarp();
          if (lane == 0) {
            // no key attended yet (mo = -inf): the sums are 0, whatever mn is
            s_alpha[warp] = mo == kNegInf ? 0.f : exp2f(mo - mn);
            s_m[warp] = mn;
          }
        }
        __syncthreads();
#pragma unroll
        for (int hh = 0; hh < HP; ++hh) {
          if (hh < nh) {
            const float alpha = s_alpha[hh];
            float lh = 0.f, bh = 0.f, ah = 0.f, ch = 0.f;
#pragma unroll 8
            for (int j = 0; j < nk; ++j) {
              const float e = s_e[hh][j], es = s_es[hh][j];
              lh += e;
              if (PROBE) bh += es;
              if (tid < D) {
                const float vd = s_v[j][tid];
                ah = fmaf(e, vd, ah);
                if (PROBE) ch = fmaf(es, vd, ch);
              }
            }
            l[hh] = fmaf(l[hh], alpha, lh);
            bs[hh] = fmaf(bs[hh], alpha, bh);
            A[hh] = fmaf(A[hh], alpha, ah);
            C[hh] = fmaf(C[hh], alpha, ch);
          }
        }
        __syncthreads();  // the chunk's readers are done before the next one is staged
      }
#pragma unroll
      for (int hh = 0; hh < HP; ++hh) {
        if (hh < nh && tid < D) {
          const size_t row = row0 + (size_t)hh * D;
          if (pc.complete) {
            const float inv = l[hh] > 0.f ? 1.f / l[hh] : 0.f;  // no attended key: o = 0
            const float vbar = A[hh] * inv;
            const float o = PROBE ? vbar + C[hh] * inv - (bs[hh] * inv) * vbar : vbar;
            if (OUT_F32)
              static_cast<float*>(p.out)[row + tid] = o;
            else
              static_cast<__nv_bfloat16*>(p.out)[row + tid] = __float2bfloat16_rn(o);
          } else {
            float* rec =
                p.partials + ((size_t)piece_slot(blockIdx.x, pc.first) * G + h0 + hh) * REC;
            if (tid == 0) {
              rec[0] = s_m[hh];
              rec[1] = l[hh];
              rec[2] = bs[hh];
            }
            rec[kRecHead + tid] = A[hh];
            if (PROBE) rec[kRecHead + D + tid] = C[hh];
          }
        }
      }
    }
  }
}

}  // namespace plx
