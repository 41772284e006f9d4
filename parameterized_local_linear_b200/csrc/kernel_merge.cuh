// Split-merge kernel: combines the partial records of every item that the
// split-KV kernel cut across partitions, and writes the zero output of
// sequences with no keys.
//
// Blocks (c, y): partition c owns the item whose range ENDS in partition c
// but began in an earlier one (at most one such item per partition); slice y
// of the owner's output columns is merged by block (c, y). The item's pieces
// are partition c_lo's last piece (or first, if the item starts exactly at
// c_lo's range), then the first piece of every partition up to c. They are
// combined in that fixed order with the max-rescaling merge of the online
// softmax:
//   M = max_j m_j, w_j = 2^(m_j - M),
//   l = sum w_j l_j, b = sum w_j b_j, A = sum w_j A_j, C = sum w_j C_j,
// and the output is o = A/l + C/l - (b/l)(A/l) (or A/l without the probe).
//
// The slice's A and C float4 columns are summed by groups of threads that
// each take every jg-th record; the groups are added in a fixed order, so the
// result is deterministic. Records come in chunks whose (m, l, b) go to
// shared memory; every thread derives the chunk max of its head and its own
// weights from there, rescaling its running sums when a chunk raises the max
// (thread h < G also keeps head h's running l and b). When all records fit
// (the common case) each thread's A/C loads are issued right after the
// (m, l, b) loads, before the chunk's only barrier, so the merge costs about
// one memory round trip.
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
__global__ void __launch_bounds__(kMergeThreads, 3) parallax_merge_kernel(const DecodeParams p) {
  constexpr int kAC = PROBE ? 2 : 1;  // A (and C) per output group
  __shared__ float s_m[kMergeThreads], s_l[kMergeThreads], s_b[kMergeThreads];
  __shared__ float s_L[kMergeMaxG], s_B[kMergeMaxG];
  __shared__ float4 s_red[kMergeThreads];
  const float kNegInf = __int_as_float(0xff800000u);
  const int tid = threadIdx.x;
  const int c = blockIdx.x, P = gridDim.x;
  const PartitionInfo part = locate_partition(p.seqlens, p.B, p.Hkv, p.Lmax, c, P);

  // Sequences without keys: zero output (nothing else writes these rows).
  if (blockIdx.y == 0) {
    for (int b = c; b < p.B; b += P) {
      if (clamp_len(__ldg(p.seqlens + b), p.Lmax) != 0) continue;
      for (int idx = tid; idx < p.Hq * p.D; idx += kMergeThreads) {
        const size_t oi = (size_t)b * p.Hq * p.D + idx;
        if (OUT_F32)
          static_cast<float*>(p.out)[oi] = 0.f;
        else
          static_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(0.f);
      }
    }
  }
  // Every block waits for the split-KV grid (so this grid's completion implies
  // that one's), then only owners read partial records. The next call's
  // split-KV kernel may be scheduled from here on; it waits for this grid
  // before it touches global memory.
  pdl_wait_primary();
  pdl_launch_dependents();
  if (part.lo >= part.hi || part.i == 0) return;  // no item started before this range
  if ((long long)(part.n - part.i) > part.hi - part.lo) return;  // it ends in a later partition

  const long long s0 = part.lo - part.i;  // item start
  const int c_lo = (int)(s0 / part.per);
  const int S = c - c_lo + 1;  // pieces of the item, in partition order
  const int D = p.D, G = p.G, REC = rec_floats(D), D4 = D / 4;
  const bool lo_is_first = s0 == (long long)c_lo * part.per;
  auto record = [&](int j, int h) -> const float* {
    const bool first = !(j == 0 && !lo_is_first);
    return p.partials + ((size_t)piece_slot(c_lo + j, first) * G + h) * REC;
  };

  // This block's output groups: (head, 4 dims) pairs [og0, og1).
  const int n_og = G * D4;
  const int og_per = (n_og + gridDim.y - 1) / gridDim.y;
  const int og0 = min(n_og, (int)blockIdx.y * og_per), og1 = min(n_og, og0 + og_per);
  if (og0 >= og1) return;
  const int cols = (og1 - og0) * kAC;               // float4 columns summed here
  const int groups = max(1, kMergeThreads / cols);  // record groups per column
  const int col = tid % cols, jg = tid / cols;
  const bool active = tid < cols * groups;
  const int og = og0 + col / kAC, ac = col % kAC;
  const int h_col = og / D4, d4 = og % D4;
  const int chunk = max(1, kMergeThreads / G);  // records per chunk: chunk * G <= threads
  const bool one_pass = S <= chunk && S <= groups * kMergeMaxPerThread;

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float M_run = kNegInf;                            // running max of head h_col
  float Mh_run = kNegInf, Lh_run = 0.f, Bh_run = 0.f;  // head tid (threads tid < G)
  for (int j0 = 0; j0 < S; j0 += chunk) {
    const int nch = min(chunk, S - j0);
    float m = kNegInf, l = 0.f, bb = 0.f;
    if (tid < nch * G) {
      const float* rec = record(j0 + tid / G, tid % G);
      m = rec[0];
      l = rec[1];
      bb = PROBE ? rec[2] : 0.f;
    }
    float4 v[kMergeMaxPerThread];
    if (one_pass && active) {
#pragma unroll
      for (int k = 0; k < kMergeMaxPerThread; ++k) {
        const int t = jg + k * groups;
        v[k] = t < S ? *reinterpret_cast<const float4*>(record(t, h_col) + kRecHead + ac * D + 4 * d4)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    if (tid < nch * G) {
      s_m[tid] = m;
      s_l[tid] = l;
      s_b[tid] = bb;
    }
    __syncthreads();
    if (active) {
      float mc = kNegInf;  // chunk max of head h_col: the same value in every thread
      for (int t = 0; t < nch; ++t) mc = fmaxf(mc, s_m[t * G + h_col]);
      const float M_new = fmaxf(M_run, mc);
      const float so = M_run == kNegInf ? 0.f : ex2_approx(M_run - M_new);
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
      if (one_pass) {
#pragma unroll
        for (int k = 0; k < kMergeMaxPerThread; ++k) {
          const int t = jg + k * groups;
          const float w = t < S ? ex2_approx(s_m[t * G + h_col] - M_new) : 0.f;
          sum.x += w * v[k].x;
          sum.y += w * v[k].y;
          sum.z += w * v[k].z;
          sum.w += w * v[k].w;
        }
      } else {
#pragma unroll 4
        for (int t = jg; t < nch; t += groups) {
          const float w = ex2_approx(s_m[t * G + h_col] - M_new);
          const float4 x = *reinterpret_cast<const float4*>(record(j0 + t, h_col) + kRecHead +
                                                            ac * D + 4 * d4);
          sum.x += w * x.x;
          sum.y += w * x.y;
          sum.z += w * x.z;
          sum.w += w * x.w;
        }
      }
      acc.x = acc.x * so + sum.x;
      acc.y = acc.y * so + sum.y;
      acc.z = acc.z * so + sum.z;
      acc.w = acc.w * so + sum.w;
      M_run = M_new;
    }
    if (tid < G) {  // head tid's running l and b, with the same max as above
      float mh = kNegInf;
      for (int t = 0; t < nch; ++t) mh = fmaxf(mh, s_m[t * G + tid]);
      const float Mn = fmaxf(Mh_run, mh);
      const float soh = Mh_run == kNegInf ? 0.f : ex2_approx(Mh_run - Mn);
      float lc = 0.f, bc = 0.f;
      for (int t = 0; t < nch; ++t) {
        const float w = ex2_approx(s_m[t * G + tid] - Mn);
        lc += w * s_l[t * G + tid];
        bc += w * s_b[t * G + tid];
      }
      Lh_run = Lh_run * soh + lc;
      Bh_run = Bh_run * soh + bc;
      Mh_run = Mn;
    }
    __syncthreads();  // s_m, s_l, s_b are rewritten by the next chunk
  }
  if (tid < G) {
    s_L[tid] = Lh_run;
    s_B[tid] = Bh_run;
  }
  // add the record groups of every column in a fixed order
  s_red[tid] = acc;
  __syncthreads();
  if (tid < cols) {
    float4 t = s_red[tid];
    for (int g2 = 1; g2 < groups; ++g2) {
      const float4 u = s_red[g2 * cols + tid];
      t.x += u.x;
      t.y += u.y;
      t.z += u.z;
      t.w += u.w;
    }
    s_red[tid] = t;  // column tid's total (groups >= 1 reads only other slots)
  }
  __syncthreads();
  const int n_out = (og1 - og0) * 4;
  for (int e = tid; e < n_out; e += kMergeThreads) {
    const int ogl = e >> 2, k = e & 3;
    const int og_e = og0 + ogl, h = og_e / D4, d = 4 * (og_e % D4) + k;
    const float* a4 = reinterpret_cast<const float*>(&s_red[ogl * kAC]);
    const float inv = 1.f / s_L[h];
    const float vbar = a4[k] * inv;
    float o = vbar;
    if (PROBE) {
      const float* c4v = reinterpret_cast<const float*>(&s_red[ogl * kAC + 1]);
      o = vbar + c4v[k] * inv - (s_B[h] * inv) * vbar;
    }
    const size_t oi = ((size_t)part.b * p.Hq + (size_t)part.g * G + h) * D + d;
    if (OUT_F32)
      static_cast<float*>(p.out)[oi] = o;
    else
      static_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(o);
  }
}

}  // namespace plx
