// Generic split-KV Parallax decode kernel: fp32 (or bf16) inputs, plain FMA
// arithmetic, any GQA group size. It serves the fp32 input mode and shapes
// the tensor-core kernel does not cover; it shares the partitioning, the
// partial-record format and the merge kernel with that kernel.
//
// Per piece and per query head of the group, chunks of 128 keys are scored
// one key per thread (t = scale*log2(e) q.k, s = r.k into shared memory),
// then thread d (< D) updates the online accumulators of dimension d:
//   m' = max(m, max t), alpha = 2^(m-m'), e = 2^(t-m'),
//   l = alpha l + sum e, b = alpha b + sum e s,
//   A_d = alpha A_d + sum e v_d, C_d = alpha C_d + sum e s v_d.
// (m, l, b) are the same in every thread: each reads the whole chunk.
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

template <typename T, bool PROBE, bool OUT_F32>
__global__ void __launch_bounds__(kGenericThreads)
    parallax_generic_kernel(const DecodeParams p) {
  __shared__ float s_t[kGenericThreads];
  __shared__ float s_s[kGenericThreads];
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
  const int tid = threadIdx.x, D = p.D, G = p.G, REC = rec_floats(D);

  PieceCursor cur;
  cur.init(part, key_space(p), p.B, p.Hkv);
  Piece pc;
  while (cur.next(pc)) {
    const long long kv0 = pc.b * p.kv_sb + pc.g * p.kv_sh + pc.kbase * p.kv_sk;
    const T* kb = k + kv0;  // key j of the piece's item: kb + j * kv_sk
    const T* vb = v + kv0;
    for (int h = 0; h < G; ++h) {
      const size_t row = ((size_t)pc.b * p.Hq + (size_t)pc.g * G + h) * D;
      float m = kNegInf, l = 0.f, bs = 0.f, A = 0.f, C = 0.f;
      for (int k0 = pc.i; k0 < pc.i + pc.len; k0 += kGenericThreads) {
        const int nk = min(kGenericThreads, pc.i + pc.len - k0);
        if (tid < nk) {
          const T* kr = kb + (long long)(k0 + tid) * p.kv_sk;
          float t = 0.f, s = 0.f;
          for (int d = 0; d < D; ++d) {
            const float kd = to_f32(kr[d]);
            t = fmaf(to_f32(q[row + d]), kd, t);
            if (PROBE) s = fmaf(to_f32(r[row + d]), kd, s);
          }
          s_t[tid] = t * p.scale_log2;
          s_s[tid] = s;
        }
        __syncthreads();
        float mc = kNegInf;
        for (int j = 0; j < nk; ++j) mc = fmaxf(mc, s_t[j]);
        const float mn = fmaxf(m, mc);
        const float alpha = exp2f(m - mn);  // m = -inf on the first chunk: 0
        l *= alpha;
        bs *= alpha;
        A *= alpha;
        C *= alpha;
        for (int j = 0; j < nk; ++j) {
          const float e = exp2f(s_t[j] - mn);
          l += e;
          if (PROBE) bs = fmaf(e, s_s[j], bs);
          if (tid < D) {
            const float vd = to_f32(vb[(long long)(k0 + j) * p.kv_sk + tid]);
            A = fmaf(e, vd, A);
            if (PROBE) C = fmaf(e * s_s[j], vd, C);
          }
        }
        m = mn;
        __syncthreads();
      }
      if (tid < D) {
        if (pc.complete) {
          const float inv = 1.f / l;
          const float vbar = A * inv;
          const float o = PROBE ? vbar + C * inv - (bs * inv) * vbar : vbar;
          if (OUT_F32)
            static_cast<float*>(p.out)[row + tid] = o;
          else
            static_cast<__nv_bfloat16*>(p.out)[row + tid] = __float2bfloat16_rn(o);
        } else {
          float* rec = p.partials + ((size_t)piece_slot(blockIdx.x, pc.first) * G + h) * REC;
          if (tid == 0) {
            rec[0] = m;
            rec[1] = l;
            rec[2] = bs;
          }
          rec[kRecHead + tid] = A;
          if (PROBE) rec[kRecHead + D + tid] = C;
        }
      }
    }
  }
}

}  // namespace plx
