// Work partitioning shared by the split-KV kernels and the merge kernel.
//
// The keys of all (batch b, kv head g) items are laid end to end: item
// (b, g) holds n_b = clamp(cache_seqlens[b], 0, Lmax) keys and starts at
// position Hkv * (n_0 + ... + n_{b-1}) + g * n_b. The P partitions (one CTA
// each) cut this sequence of total = Hkv * sum_b n_b keys into equal ranges
// [c*per, min((c+1)*per, total)), per = ceil(total / P), so every CTA streams
// the same number of K/V bytes whatever the lengths (flash-decoding split-KV
// with a balanced, length-aware cut). A range is processed as a series of
// "pieces", the parts of the items it overlaps. A piece that is a whole item
// is finished in place; any other piece writes a partial record to slot 2c
// (the first piece of partition c) or 2c+1 (its last piece), and the
// partition in which the item ends merges them.
#pragma once

#include <cstdint>

namespace plx {

__device__ __forceinline__ int clamp_len(int n, int Lmax) {
  return n < 0 ? 0 : (n > Lmax ? Lmax : n);
}

struct PartitionInfo {
  long long total;  // keys over all items
  long long per;    // keys per partition
  long long lo, hi; // this partition's range
  int b, g, i;      // item and key offset at position lo (valid if lo < hi)
  int clamped;      // some cache_seqlens value was outside [0, Lmax]
};

struct PrologueScratch {
  long long warp_sum[32];
  long long total;
  long long within;
  int b;
  int clamped;
};

// Block-cooperative (every thread of the block must call it, NT threads).
// Reads cache_seqlens once, computes the partition of this block (index c of
// P) and locates its first key.
template <int NT>
__device__ PartitionInfo locate_partition(const int32_t* __restrict__ seqlens, int B, int Hkv,
                                          int Lmax, int c, int P, PrologueScratch* s) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = NT / 32;
  const int chunk = (B + NT - 1) / NT;
  const int b0 = min(B, tid * chunk), b1 = min(B, b0 + chunk);
  long long local = 0;
  int clamped = 0;
  for (int b = b0; b < b1; ++b) {
    int n = seqlens[b];
    clamped |= (n < 0 || n > Lmax);
    local += clamp_len(n, Lmax);
  }
  // inclusive warp scan of `local`
  long long incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    long long x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  clamped = __any_sync(0xffffffffu, clamped);
  if (tid == 0) {
    s->b = -1;
    s->clamped = 0;
  }
  if (lane == 31) s->warp_sum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    long long w = lane < kWarps ? s->warp_sum[lane] : 0;
    long long wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      long long x = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += x;
    }
    if (lane < kWarps) s->warp_sum[lane] = wi - w;  // exclusive warp offsets
    if (lane == kWarps - 1) s->total = wi;
  }
  if (clamped && lane == 0) atomicOr(&s->clamped, 1);
  __syncthreads();
  const long long excl = s->warp_sum[warp] + incl - local;  // lengths before b0
  PartitionInfo p;
  p.total = (long long)Hkv * s->total;
  p.per = (p.total + P - 1) / P;
  p.lo = min(p.total, (long long)c * p.per);
  p.hi = min(p.total, p.lo + p.per);
  // the thread whose batches contain position lo records the item there
  if (p.lo < p.hi && local > 0) {
    long long pos = (long long)Hkv * excl;
    if (p.lo >= pos && p.lo < pos + (long long)Hkv * local) {
      for (int b = b0; b < b1; ++b) {
        const long long blk = (long long)Hkv * clamp_len(seqlens[b], Lmax);
        if (p.lo < pos + blk) {
          s->b = b;
          s->within = p.lo - pos;
          break;
        }
        pos += blk;
      }
    }
  }
  __syncthreads();
  p.clamped = s->clamped;
  p.b = s->b;
  p.g = 0;
  p.i = 0;
  if (p.b >= 0) {
    const int n = clamp_len(seqlens[p.b], Lmax);
    p.g = (int)(s->within / n);
    p.i = (int)(s->within % n);
  }
  return p;
}

struct Piece {
  int b, g;      // item
  int i, len;    // keys [i, i+len) of the item
  int n;         // item length
  bool complete; // the piece is the whole item
  bool first;    // the first piece of this partition
};

// Walks the pieces of one partition; every role of a CTA walks the same list.
struct PieceCursor {
  int b, g, i;
  long long pos, lo, hi;
  const int32_t* seqlens;
  int B, Hkv, Lmax;

  __device__ void init(const PartitionInfo& p, const int32_t* sl, int B_, int Hkv_, int Lmax_) {
    b = p.b;
    g = p.g;
    i = p.i;
    pos = p.lo;
    lo = p.lo;
    hi = p.hi;
    seqlens = sl;
    B = B_;
    Hkv = Hkv_;
    Lmax = Lmax_;
  }

  __device__ bool next(Piece& pc) {
    if (pos >= hi) return false;
    const int n = clamp_len(seqlens[b], Lmax);
    const long long room = hi - pos;
    const int len = (long long)(n - i) < room ? n - i : (int)room;
    pc.b = b;
    pc.g = g;
    pc.i = i;
    pc.len = len;
    pc.n = n;
    pc.complete = (i == 0) && (len == n);
    pc.first = (pos == lo);
    pos += len;
    i += len;
    if (i == n) {
      i = 0;
      if (++g == Hkv) {
        g = 0;
        ++b;
        while (pos < hi && b < B && clamp_len(seqlens[b], Lmax) == 0) ++b;
      }
    }
    return true;
  }
};

// Slot of the partial record of a piece of partition c.
__device__ __forceinline__ int piece_slot(int c, bool first) { return 2 * c + (first ? 0 : 1); }

}  // namespace plx
