// Split-merge kernel: combines the partial records of every item that the
// split-KV kernel cut across partitions, and writes the zero output of
// sequences with no keys.
//
// Blocks (c, y): partition c owns the item whose range ENDS in partition c
// but began in an earlier one (at most one such item per partition); block
// (c, y) merges slice y of the owner's float4 columns (one column per
// thread; a single slice unless G * D/4 * 2 > kMergeThreads). The item's
// pieces are partition c_lo's last piece (or first, if the item starts
// exactly at c_lo's range), then the first piece of every partition up to c.
// They are combined with the max-rescaling merge of the online softmax:
//   M = max_j m_j, w_j = 2^(m_j - M),
//   l = sum w_j l_j, b = sum w_j b_j, A = sum w_j A_j, C = sum w_j C_j,
// and the output is o = A/l + C/l - (b/l)(A/l) (or A/l without the probe).
//
// A column is one float4 of A or C of one (head, 4 dims) output group; the A
// and C columns of a group are neighbouring threads. Records come in chunks of
// up to kMergeChunk: each thread loads its column of every record of the chunk
// into registers right after the chunk's (m, l, b) loads, all before the
// chunk's only block barrier, then takes the chunk max, the weights and the
// l and b sums of its head from shared memory in record order. One memory
// round trip per chunk (one chunk in the common case), deterministic order.
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
__global__ void __launch_bounds__(kMergeThreads, 4) parallax_merge_kernel(const DecodeParams p) {
  constexpr int kAC = PROBE ? 2 : 1;  // A (and C) columns per output group
  __shared__ float s_m[kMergeThreads], s_l[kMergeThreads], s_b[kMergeThreads];
  const float kNegInf = __int_as_float(0xff800000u);
  const int tid = threadIdx.x;
  const int c = blockIdx.x, P = gridDim.x;
  const PartitionInfo part = locate_partition(key_space(p), p.B, p.Hkv, c, P);

  // Sequences without keys: zero output (nothing else writes these rows).
  if (blockIdx.y == 0) {
    for (int b = c; b < p.B; b += P) {
      int kb;
      if (item_keys(key_space(p), b, &kb) != 0) continue;
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
  const int c_lo = (int)div_pos(s0, part.per);
  const int S = c - c_lo + 1;  // pieces of the item, in partition order
  const int D = p.D, G = p.G, REC = rec_floats(D), D4 = D / 4;
  const bool lo_is_first = s0 == (long long)c_lo * part.per;
  auto record = [&](int j, int h) -> const float* {
    const bool first = !(j == 0 && !lo_is_first);
    return p.partials + ((size_t)piece_slot(c_lo + j, first) * G + h) * REC;
  };

  // This thread's column: slice y holds columns [y * threads, ...).
  const int n_cols = G * D4 * kAC;
  const int col = blockIdx.y * kMergeThreads + tid;
  const bool active = col < n_cols;
  const int cc = active ? col : n_cols - 1;
  const int og = cc / kAC, ac = cc % kAC;
  const int h_col = og / D4, d4 = og % D4;
  const int chunk = min(kMergeChunk, kMergeThreads / G);  // chunk * G <= threads

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float M_run = kNegInf, L_run = 0.f, B_run = 0.f;  // of head h_col
  for (int j0 = 0; j0 < S; j0 += chunk) {
    const int nch = min(chunk, S - j0);
    float m = kNegInf, l = 0.f, bb = 0.f;
    if (tid < nch * G) {  // the record header (m, l, b, -) in one load
      const float4 hd = ld_cg_f4(record(j0 + tid / G, tid % G));
      m = hd.x;
      l = hd.y;
      bb = PROBE ? hd.z : 0.f;
    }
    // every thread loads kMergeChunk records unconditionally (past the chunk it
    // re-reads the chunk's last record, weighted 0 below), so the loads issue
    // back to back with no branch between them
    float4 v[kMergeChunk];
#pragma unroll
    for (int k = 0; k < kMergeChunk; ++k)
      v[k] = ld_cg_f4(record(j0 + min(k, nch - 1), h_col) + kRecHead + ac * D + 4 * d4);
    if (tid < nch * G) {
      s_m[tid] = m;
      s_l[tid] = l;
      s_b[tid] = bb;
    }
    __syncthreads();
    float mc = kNegInf;
    for (int t = 0; t < nch; ++t) mc = fmaxf(mc, s_m[t * G + h_col]);
    const float M_new = fmaxf(M_run, mc);
    const float so = M_run == kNegInf ? 0.f : ex2_approx(M_run - M_new);
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
    float lsum = 0.f, bsum = 0.f;
#pragma unroll
    for (int k = 0; k < kMergeChunk; ++k) {
      if (k < nch) {
        const float mk = s_m[k * G + h_col];
        const float w = mk == kNegInf ? 0.f : ex2_approx(mk - M_new);  // a piece with no key
        sum.x += w * v[k].x;
        sum.y += w * v[k].y;
        sum.z += w * v[k].z;
        sum.w += w * v[k].w;
        lsum += w * s_l[k * G + h_col];
        bsum += w * s_b[k * G + h_col];
      }
    }
    acc.x = acc.x * so + sum.x;
    acc.y = acc.y * so + sum.y;
    acc.z = acc.z * so + sum.z;
    acc.w = acc.w * so + sum.w;
    L_run = L_run * so + lsum;
    B_run = B_run * so + bsum;
    M_run = M_new;
    if (j0 + chunk < S) __syncthreads();  // s_m, s_l, s_b are rewritten by the next chunk
  }
  // Output: the A-column thread writes its 4 dimensions; with the probe the C
  // column is the next thread.
  const float inv = L_run > 0.f ? 1.f / L_run : 0.f;  // no attended key: o = 0
  float4 o = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (PROBE) {
    const float cx = __shfl_down_sync(0xffffffffu, acc.x, 1);
    const float cy = __shfl_down_sync(0xffffffffu, acc.y, 1);
    const float cz = __shfl_down_sync(0xffffffffu, acc.z, 1);
    const float cw = __shfl_down_sync(0xffffffffu, acc.w, 1);
    const float bl = B_run * inv;
    o.x = o.x + cx * inv - bl * o.x;
    o.y = o.y + cy * inv - bl * o.y;
    o.z = o.z + cz * inv - bl * o.z;
    o.w = o.w + cw * inv - bl * o.w;
  }
  if (active && ac == 0) {
    const size_t oi = ((size_t)part.b * p.Hq + (size_t)part.g * G + h_col) * D + 4 * d4;
    if (OUT_F32) {
      *reinterpret_cast<float4*>(static_cast<float*>(p.out) + oi) = o;
    } else {
      __nv_bfloat162 lo2 = __floats2bfloat162_rn(o.x, o.y), hi2 = __floats2bfloat162_rn(o.z, o.w);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo2);
      pk.y = *reinterpret_cast<uint32_t*>(&hi2);
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.out) + oi) = pk;
    }
  }
}

}  // namespace plx
