// Split-merge kernel: combines the partial records of every item that the
// split-KV kernel cut across partitions, and writes the zero output of
// sequences with no keys.
//
// Block c owns the item whose range ENDS in partition c but began in an
// earlier one (at most one such item per partition). Its pieces are partition
// c_lo's last piece (or first, if the item starts exactly at c_lo's range),
// then the first piece of every partition up to c. They are combined in that
// fixed order with the max-rescaling merge of the online softmax:
//   M = max_j m_j, w_j = 2^(m_j - M),
//   l = sum w_j l_j, b = sum w_j b_j, A = sum w_j A_j, C = sum w_j C_j,
// and the output is o = A/l + C/l - (b/l)(A/l) (or A/l without the probe).
//
// Per query head, records are taken in chunks of kMergeThreads: their
// (m, l, b) go to shared memory, warp 0 forms the weights w_j once (and
// rescales the running sums when the chunk raises the max), then thread d
// accumulates A_d and C_d with independent loads across the chunk.
//
// Launched with programmatic stream serialisation: the prologue overlaps the
// tail of the split-KV kernel and griddepcontrol.wait guards every read of
// the partial records.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"
#include "partition.cuh"
#include "ptx.cuh"

namespace plx {

template <bool PROBE, bool OUT_F32>
__global__ void __launch_bounds__(kMergeThreads) parallax_merge_kernel(const DecodeParams p) {
  __shared__ PrologueScratch scratch;
  __shared__ float s_m[kMergeThreads], s_l[kMergeThreads], s_b[kMergeThreads], s_w[kMergeThreads];
  __shared__ float s_run[4];  // running M, L, B and the rescale of the previous chunks
  const float kNegInf = __int_as_float(0xff800000u);
  const int tid = threadIdx.x, lane = tid & 31, c = blockIdx.x, P = gridDim.x;
  const PartitionInfo part =
      locate_partition<kMergeThreads>(p.seqlens, p.B, p.Hkv, p.Lmax, c, P, &scratch);

  // Sequences without keys: zero output (nothing else writes these rows).
  for (int b = c; b < p.B; b += P) {
    if (clamp_len(p.seqlens[b], p.Lmax) != 0) continue;
    for (int idx = tid; idx < p.Hq * p.D; idx += kMergeThreads) {
      const size_t oi = (size_t)b * p.Hq * p.D + idx;
      if (OUT_F32)
        static_cast<float*>(p.out)[oi] = 0.f;
      else
        static_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(0.f);
    }
  }
  // Every block waits for the split-KV grid (so this grid's completion implies
  // that one's), then only owners read partial records.
  pdl_wait_primary();
  if (part.lo >= part.hi || part.i == 0) return;  // no item started before this range
  const int n = clamp_len(p.seqlens[part.b], p.Lmax);
  if ((long long)(n - part.i) > part.hi - part.lo) return;  // the item ends in a later partition

  const long long s0 = part.lo - part.i;  // item start
  const int c_lo = (int)(s0 / part.per);
  const int S = c - c_lo + 1;  // pieces of the item, in partition order
  const int D = p.D, G = p.G, REC = rec_floats(D);
  const bool lo_is_first = s0 == (long long)c_lo * part.per;
  auto record = [&](int j, int h) -> const float* {
    const int cc = c_lo + j;
    const bool first = !(j == 0 && !lo_is_first);
    return p.partials + ((size_t)piece_slot(cc, first) * G + h) * REC;
  };

  for (int h = 0; h < G; ++h) {
    float A = 0.f, C = 0.f;
    if (tid == 0) {
      s_run[0] = kNegInf;
      s_run[1] = 0.f;
      s_run[2] = 0.f;
    }
    for (int j0 = 0; j0 < S; j0 += kMergeThreads) {
      const int nch = min(kMergeThreads, S - j0);
      if (tid < nch) {
        const float* rec = record(j0 + tid, h);
        s_m[tid] = rec[0];
        s_l[tid] = rec[1];
        s_b[tid] = PROBE ? rec[2] : 0.f;
      }
      __syncthreads();
      if (tid < 32) {
        float mx = kNegInf;
        for (int t = lane; t < nch; t += 32) mx = fmaxf(mx, s_m[t]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float M_old = s_run[0];
        const float M = fmaxf(M_old, mx);
        float lsum = 0.f, bsum = 0.f;
        for (int t = lane; t < nch; t += 32) {
          const float w = ex2_approx(s_m[t] - M);
          s_w[t] = w;
          lsum += w * s_l[t];
          bsum += w * s_b[t];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
          bsum += __shfl_xor_sync(0xffffffffu, bsum, o);
        }
        __syncwarp();
        if (lane == 0) {
          const float so = M_old == kNegInf ? 0.f : ex2_approx(M_old - M);
          s_run[0] = M;
          s_run[1] = s_run[1] * so + lsum;
          s_run[2] = s_run[2] * so + bsum;
          s_run[3] = so;
        }
      }
      __syncthreads();
      if (tid < D) {
        const float so = s_run[3];
        float a0 = 0.f, a1 = 0.f, c0 = 0.f, c1 = 0.f;
        int t = 0;
#pragma unroll 4
        for (; t + 1 < nch; t += 2) {
          const float* r0 = record(j0 + t, h);
          const float* r1 = record(j0 + t + 1, h);
          a0 += s_w[t] * r0[kRecHead + tid];
          a1 += s_w[t + 1] * r1[kRecHead + tid];
          if (PROBE) {
            c0 += s_w[t] * r0[kRecHead + D + tid];
            c1 += s_w[t + 1] * r1[kRecHead + D + tid];
          }
        }
        if (t < nch) {
          const float* r0 = record(j0 + t, h);
          a0 += s_w[t] * r0[kRecHead + tid];
          if (PROBE) c0 += s_w[t] * r0[kRecHead + D + tid];
        }
        A = A * so + (a0 + a1);
        C = C * so + (c0 + c1);
      }
      __syncthreads();  // s_m/s_w/s_run are rewritten by the next chunk or head
    }
    if (tid < D) {
      const float inv = 1.f / s_run[1];
      const float vbar = A * inv;
      const float o = PROBE ? vbar + C * inv - (s_run[2] * inv) * vbar : vbar;
      const size_t oi = ((size_t)part.b * p.Hq + (size_t)part.g * G + h) * D + tid;
      if (OUT_F32)
        static_cast<float*>(p.out)[oi] = o;
      else
        static_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(o);
    }
    __syncthreads();  // s_run is reset for the next head
  }
}

}  // namespace plx
