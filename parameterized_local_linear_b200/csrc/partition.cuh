// Work partitioning shared by the split-KV kernels and the merge kernel.
//
// The keys of all (batch b, kv head g) items are laid end to end: item
// (b, g) holds n_b = clamp(cache_seqlens[b], 0, Lmax) keys and starts at
// position Hkv * (n_0 + ... + n_{b-1}) + g * n_b. The P partitions (one CTA
// each) cut this sequence of total = Hkv * sum_b n_b keys into equal ranges
// [c*per, min((c+1)*per, total)), per = ceil(total / P) rounded up to whole
// 64-key tiles, so every CTA streams the same number of K/V bytes whatever the
// lengths (flash-decoding split-KV with a balanced, length-aware cut). A range is processed as a series of
// "pieces", the parts of the items it overlaps. A piece that is a whole item
// is finished in place; any other piece writes a partial record to slot 2c
// (the first piece of partition c) or 2c+1 (its last piece), and the
// partition in which the item ends merges them.
#pragma once

#include <cstdint>

namespace plx {

constexpr int kRangeAlign = 64;  // partition ranges are multiples of one K/V tile

// x / d for x >= 0, d > 0: one 32-bit division when x fits (the usual case;
// a 64-bit division is a long software sequence on the critical path).
__device__ __forceinline__ long long div_pos(long long x, long long d) {
  if (x <= 0x7fffffffLL && d <= 0x7fffffffLL) return (long long)((unsigned)x / (unsigned)d);
  return x / d;
}

__device__ __forceinline__ int clamp_len(int n, int Lmax) {
  return n < 0 ? 0 : (n > Lmax ? Lmax : n);
}

// Where the keys of each batch row come from.
//   kKvContiguous  the cache row itself: keys 0..n-1 (with a sliding window
//                  W > 0 only the last min(n, W)).
//   kKvPaged       fixed-size pages listed per row in a block table: key i is
//                  slot i % page_size of page table[b][i / page_size].
//   kKvBlockSparse a per-row list of 64-key blocks of the cache row: logical
//                  tile t is cache keys 64 table[b][t] .. +63 (keys >= n masked).
// The paged and block-sparse rows are walked in whole 64-key tiles, so every
// tile a CTA loads sits inside one page or block.
enum KvMode { kKvContiguous = 0, kKvPaged = 1, kKvBlockSparse = 2 };

struct KeySpace {
  const int32_t* seqlens;     // [B], or NULL: every row holds Lmax keys
  const int32_t* num_blocks;  // block-sparse: [B] listed blocks per row
  int Lmax, window, mode, max_blocks;
};

// The keys batch row b contributes to the end-to-end key sequence the
// partitions cut, and (contiguous rows) *kbase = the cache position of the
// first one. Paged rows count their n keys rounded up to whole tiles and
// block-sparse rows 64 per listed block; the kernels mask the keys past n.
__device__ __forceinline__ int item_keys(const KeySpace& ks, int b, int* kbase) {
  const int n = ks.seqlens ? clamp_len(__ldg(ks.seqlens + b), ks.Lmax) : ks.Lmax;
  *kbase = 0;
  if (ks.mode == kKvPaged) return (n + kRangeAlign - 1) / kRangeAlign * kRangeAlign;
  if (ks.mode == kKvBlockSparse) {
    const int nb = __ldg(ks.num_blocks + b);
    return kRangeAlign * (nb < 0 ? 0 : (nb > ks.max_blocks ? ks.max_blocks : nb));
  }
  const int ne = (ks.window > 0 && n > ks.window) ? ks.window : n;
  *kbase = n - ne;
  return ne;
}

template <typename Params>
__device__ __forceinline__ KeySpace key_space(const Params& p) {
  return KeySpace{p.seqlens, p.num_blocks, p.Lmax, p.window, p.kv_mode, p.table_stride};
}

// A length or block count outside its range (clamped by item_keys).
__device__ __forceinline__ bool item_clamped(const KeySpace& ks, int b) {
  bool bad = false;
  if (ks.seqlens) {
    const int n = __ldg(ks.seqlens + b);
    bad = n < 0 || n > ks.Lmax;
  }
  if (ks.mode == kKvBlockSparse) {
    const int nb = __ldg(ks.num_blocks + b);
    bad = bad || nb < 0 || nb > ks.max_blocks;
  }
  return bad;
}

struct PartitionInfo {
  long long total;  // keys over all items
  long long per;    // keys per partition
  long long lo, hi; // this partition's range
  int b, g, i;      // item and key offset at position lo (valid if lo < hi)
  int n;            // keys of batch b (item_keys)
  int kbase;        // first attended key of batch b
  int clamped;      // some cache_seqlens value was outside [0, Lmax]
};

// Warp-cooperative: every warp of a block calls it and gets the same result,
// with no block barrier and no shared memory. Each lane sums a contiguous
// chunk of cache_seqlens (read-only path, so the re-reads hit L1), a warp scan
// gives the prefix sums, and the lane whose chunk holds position lo walks it
// to find the item there. c is this block's index among P partitions.
__device__ inline PartitionInfo locate_partition(const KeySpace& ks, int B, int Hkv, int c,
                                                 int P) {
  const int lane = threadIdx.x & 31;
  const int chunk = (B + 31) / 32;
  const int b0 = min(B, lane * chunk), b1 = min(B, b0 + chunk);
  long long local = 0;
  int clamped = 0, kb;
  for (int b = b0; b < b1; ++b) {
    clamped |= item_clamped(ks, b);
    local += item_keys(ks, b, &kb);
  }
  long long incl = local;  // inclusive scan over lanes
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  PartitionInfo p;
  p.clamped = __any_sync(0xffffffffu, clamped);
  p.total = (long long)Hkv * __shfl_sync(0xffffffffu, incl, 31);
  // ranges are whole 64-key tiles, so a range starts on a tile of its item
  // whenever the items are tile multiples (trailing partitions may be empty)
  p.per = (div_pos(p.total + P - 1, P) + kRangeAlign - 1) / kRangeAlign * kRangeAlign;
  p.lo = min(p.total, (long long)c * p.per);
  p.hi = min(p.total, p.lo + p.per);
  p.b = -1;
  p.g = p.i = p.n = p.kbase = 0;
  // the lane whose batches contain position lo finds the item there
  long long pos = (long long)Hkv * (incl - local);
  int fb = -1, fn = 0, fk = 0;
  long long within = 0;
  if (p.lo < p.hi && p.lo >= pos && p.lo < pos + (long long)Hkv * local) {
    for (int b = b0; b < b1; ++b) {
      const int n = item_keys(ks, b, &kb);
      const long long blk = (long long)Hkv * n;
      if (p.lo < pos + blk) {
        fb = b;
        fn = n;
        fk = kb;
        within = p.lo - pos;
        break;
      }
      pos += blk;
    }
  }
  const unsigned owner = __ballot_sync(0xffffffffu, fb >= 0);
  if (owner) {
    const int src = __ffs(owner) - 1;
    p.b = __shfl_sync(0xffffffffu, fb, src);
    p.n = __shfl_sync(0xffffffffu, fn, src);
    p.kbase = __shfl_sync(0xffffffffu, fk, src);
    const int w = (int)__shfl_sync(0xffffffffu, within, src);  // < Hkv * n <= Hkv * Lmax
    p.g = w / p.n;
    p.i = w - p.g * p.n;
  }
  return p;
}

struct Piece {
  int b, g;      // item
  int i, len;    // keys [i, i+len) of the item's attended range
  int n;         // attended keys of the item
  int kbase;     // cache position of the item's first attended key
  bool complete; // the piece is the whole item
  bool first;    // the first piece of this partition
};

// Walks the pieces of one partition; every role of a CTA walks the same list.
struct PieceCursor {
  int b, g, i, n, kbase;  // n, kbase: keys of batch b (item_keys) and the first one
  long long pos, lo, hi;
  KeySpace ks;
  int B, Hkv;

  __device__ void init(const PartitionInfo& p, const KeySpace& ks_, int B_, int Hkv_) {
    b = p.b;
    g = p.g;
    i = p.i;
    n = p.n;
    kbase = p.kbase;
    pos = p.lo;
    lo = p.lo;
    hi = p.hi;
    ks = ks_;
    B = B_;
    Hkv = Hkv_;
  }

  __device__ bool next(Piece& pc) {
    if (pos >= hi) return false;
    const long long room = hi - pos;
    const int len = (long long)(n - i) < room ? n - i : (int)room;
    pc.b = b;
    pc.g = g;
    pc.i = i;
    pc.len = len;
    pc.n = n;
    pc.kbase = kbase;
    pc.complete = (i == 0) && (len == n);
    pc.first = (pos == lo);
    pos += len;
    i += len;
    if (i == n) {
      i = 0;
      if (++g == Hkv) {
        g = 0;
        ++b;
        n = 0;
        while (pos < hi && b < B && (n = item_keys(ks, b, &kbase)) == 0) ++b;
      }
    }
    return true;
  }
};

// Paged and block-sparse rows: where logical 64-key tile k0 (a multiple of 64)
// of batch row b lives, as (*key, *item): the first key and the batch row (or
// page) of the tile in the K/V view the split-KV kernels read (the paged pool
// is viewed as a cache of page_size keys per "row" in the (kv_len, H, D)
// layout), and how many of its keys are attended (*nv, a prefix of the tile).
// An id outside the pool or the cache gives an empty tile and sets the
// clamped status bit.
template <typename Params>
__device__ __forceinline__ void tile_source(const Params& p, int b, int k0, int* key, int* item,
                                            int* nv) {
  const int n = p.seqlens ? clamp_len(__ldg(p.seqlens + b), p.Lmax) : p.Lmax;
  if (p.kv_mode == kKvPaged) {
    const int page = __ldg(p.table + (size_t)b * p.table_stride + k0 / p.page_size);
    const bool ok = page >= 0 && page < p.num_pages;
    *key = ok ? k0 % p.page_size : 0;
    *item = ok ? page : 0;
    *nv = ok ? max(0, min(kRangeAlign, n - k0)) : 0;
    // an entry past the length (read when the cluster kernel fetches a row's
    // first tiles before its length) attends nothing and is not an error
    if (!ok && k0 < n) atomicOr(p.status, 2u /* PARALLAX_DEVICE_STATUS_SEQLEN_CLAMPED */);
  } else {  // block-sparse: the listed block of the cache row
    const int blk = __ldg(p.table + (size_t)b * p.table_stride + k0 / kRangeAlign);
    const bool ok = blk >= 0 && (long long)blk * kRangeAlign < p.Lmax;
    *key = ok ? blk * kRangeAlign : 0;
    *item = b;
    *nv = ok ? max(0, min(kRangeAlign, n - blk * kRangeAlign)) : 0;
    if (!ok) atomicOr(p.status, 2u);
  }
}

// Slot of the partial record of a piece of partition c.
__device__ __forceinline__ int piece_slot(int c, bool first) { return 2 * c + (first ? 0 : 1); }

}  // namespace plx
