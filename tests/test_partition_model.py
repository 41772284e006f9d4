"""A host model of the work partition the split-KV kernels and the merge kernel
share (csrc/partition.cuh, the merge ownership in csrc/kernel_merge.cuh), run
over many random shapes: the invariants the design relies on.

The keys of all (batch row, kv head) items are laid end to end (row b holds
Hkv * n_b positions: n_b keys per kv head, or whole 64-key tiles for paged and
block-sparse rows); P partitions take equal ranges, rounded up to whole tiles.
Checked here:
- every position is covered by exactly one piece of one partition;
- a piece that is not a whole item writes its record to a slot no other
  piece writes (2c for the first piece of partition c, 2c+1 for its last);
- exactly one partition owns each split item (the one where it ends), and
  the slots it merges are exactly the slots that item's pieces wrote, in
  partition order;
- pieces of tile-multiple items start on whole tiles, so the generic kernel's
  32-key chunks and the TMA kernel's 64-key tiles never straddle a page or a
  listed block.
"""
import random

import pytest

TILE = 64


def item_keys(mode, n, Lmax, window, nblocks):
    """Positions batch row b contributes per kv head (partition.cuh item_keys)."""
    n = max(0, min(n, Lmax))
    if mode == "paged":
        return (n + TILE - 1) // TILE * TILE
    if mode == "block_sparse":
        return TILE * nblocks
    return min(n, window) if window > 0 else n


def partition_model(keys, Hkv, P):
    pref = [0]
    for k in keys:
        pref.append(pref[-1] + k)
    total = Hkv * pref[-1]
    per = ((total + P - 1) // P + TILE - 1) // TILE * TILE if total else 0

    def locate(lo):
        b = next(b for b in range(len(keys)) if Hkv * pref[b] <= lo < Hkv * pref[b + 1])
        within = lo - Hkv * pref[b]
        return b, within // keys[b], within % keys[b]

    cover, slots, pieces_by_item, starts = {}, {}, {}, []
    for c in range(P):
        lo, hi = min(total, c * per), min(total, c * per + per)
        if lo >= hi:
            continue
        b, g, i = locate(lo)
        pos = lo
        while pos < hi:
            nb = keys[b]
            ln = min(nb - i, hi - pos)
            complete, first = i == 0 and ln == nb, pos == lo
            starts.append((b, i))
            for kk in range(i, i + ln):
                assert (b, g, kk) not in cover, "a position covered twice"
                cover[(b, g, kk)] = c
            if not complete:
                s = 2 * c + (0 if first else 1)
                assert s not in slots, "two pieces write one record slot"
                slots[s] = (b, g)
                pieces_by_item.setdefault((b, g), []).append(s)
            pos += ln
            i += ln
            if i == nb:
                i, g = 0, g + 1
                if g == Hkv:
                    g, b = 0, b + 1
                    while pos < hi and b < len(keys) and keys[b] == 0:
                        b += 1
    assert len(cover) == total, "a position left uncovered"
    # merge ownership: partition c owns the item whose range ends in c but began earlier
    merged = {}
    for c in range(P):
        lo, hi = min(total, c * per), min(total, c * per + per)
        if lo >= hi:
            continue
        b, g, i = locate(lo)
        if i == 0 or keys[b] - i > hi - lo:
            continue
        s0 = lo - i
        c_lo = s0 // per
        used = [2 * cc + (0 if not (cc == c_lo and s0 != c_lo * per) else 1)
                for cc in range(c_lo, c + 1)]
        assert (b, g) not in merged, "an item merged twice"
        merged[(b, g)] = used
    assert set(merged) == set(pieces_by_item), "a split item without exactly one owner"
    for item, sl in pieces_by_item.items():
        assert merged[item] == sl, (item, sl, merged[item])
    return per, starts


@pytest.mark.parametrize("mode", ["contiguous", "window", "paged", "block_sparse"])
def test_partition_invariants(mode):
    rng = random.Random(["contiguous", "window", "paged", "block_sparse"].index(mode) + 11)
    for _ in range(600):
        B = rng.randint(1, 7)
        Hkv = rng.choice([1, 2, 3, 8])
        Lmax = rng.randint(1, 400)
        window = rng.randint(1, Lmax) if mode == "window" else 0
        lens = [rng.choice([0, 1, Lmax, rng.randint(0, Lmax), Lmax + 5, -3]) for _ in range(B)]
        nblocks = [rng.randint(0, 6) for _ in range(B)]
        keys = [item_keys(mode, n, Lmax, window, nb) for n, nb in zip(lens, nblocks)]
        P = rng.choice([1, 2, 3, 7, 64, 296, rng.randint(1, 500)])
        per, starts = partition_model(keys, Hkv, P)
        assert per % TILE == 0
        if mode in ("paged", "block_sparse"):
            # every item is whole tiles: every piece starts on a tile
            assert all(i % TILE == 0 for _, i in starts)
