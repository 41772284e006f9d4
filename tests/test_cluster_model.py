"""A host model of the cluster schedule's index arithmetic
(csrc/kernel_cluster.cuh), run over many shapes: the invariants the kernel
relies on, checked without a GPU.

Per (batch row, kv head) item, a cluster of S CTAs; CTA `rank` takes tiles
rank, rank + S, ... of the row's key space. Checked here:
- every tile of the row is taken by exactly one CTA, and the count each CTA
  waits for (max of its speculative and real tiles) covers what its producer
  issues, so no stage is left in flight;
- speculative tiles (issued before the length is known) fit in the ring and
  start inside the cache;
- a stage is always consumed by the same consumer group (the ring depth is a
  multiple of the groups), and a stage's fill j waits for the release of
  fill j - stages;
- the output values of the item (G heads x D dims) are dealt to the S CTAs in
  slices that cover each value exactly once; every push lands inside the
  owner's slot area, header and value rows do not overlap, the bytes an
  owner's barrier expects equal the bytes its sources push, and the area
  fits in the kernel's shared memory;
- the reduction lanes (W >= S per value) stay inside whole warps.
"""
import itertools

import pytest

TILE = 64
GROUPS = 2
CONSUMER_WARPS = 8
THREADS = 288
STAGE_BYTES = {64: 2 * 64 * 128, 128: 2 * 2 * 64 * 128}  # K + V of one 64-key tile
STAGES = {64: 8, 128: 6}
SMEM_LIMIT = 227 * 1024


def align_up(x, a):
    return (x + a - 1) // a * a


def layout(D, G, S):
    """The cluster kernel's shared-memory layout (cluster_layout)."""
    stages = STAGES[D]
    off_p = stages * STAGE_BYTES[D]
    off_bar = off_p + CONSUMER_WARPS * 512
    off_misc = align_up(off_bar + 8 * (2 * stages + 2), 16)
    off_slots = align_up(off_misc + 16 + 4 * stages, 16)
    per = (G * D + S - 1) // S
    stride = align_up(4 * G + 2 * per, 4)
    total = off_slots + S * stride * 4 + 1024
    return dict(stages=stages, off_slots=off_slots, per=per, stride=stride, total=total,
                rec_area=CONSUMER_WARPS * G * (4 + 2 * D) * 4, ring=stages * STAGE_BYTES[D])


def tiles_of(rank, S, ntiles):
    return list(range(rank, ntiles, S))


@pytest.mark.parametrize("D", [64, 128])
def test_tile_deal_and_ring(D):
    stages = STAGES[D]
    assert stages % GROUPS == 0
    for S, Lmax, n in itertools.product(range(2, 17), (1, 63, 64, 100, 700, 4096, 4097),
                                        (0, 1, 64, 65, 699, 4096)):
        n = min(n, Lmax)
        cache_tiles = (Lmax + TILE - 1) // TILE
        ntiles = (n + TILE - 1) // TILE
        seen = []
        for rank in range(S):
            nspec = min(stages, (cache_tiles - rank + S - 1) // S) if rank < cache_tiles else 0
            nreal = (ntiles - rank + S - 1) // S if rank < ntiles else 0
            J = max(nspec, nreal)
            # the producer issues 0..nspec-1, then nspec..nreal-1: exactly 0..J-1
            issued = list(range(nspec)) + list(range(nspec, nreal))
            assert issued == list(range(J))
            for j in range(nspec):  # speculative tiles start inside the cache
                assert (rank + S * j) * TILE < Lmax
            assert nspec <= stages
            real = [rank + S * j for j in range(nreal)]
            assert real == tiles_of(rank, S, ntiles)
            seen += real
            # each stage belongs to one group; fill j of a stage follows fill j - stages
            for j in range(J):
                assert (j % stages) % GROUPS == j % GROUPS
                if j >= stages:
                    assert (j - stages) % stages == j % stages
        assert sorted(seen) == list(range(ntiles))


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 3, 4, 8])
def test_slices_slots_and_shared_memory(D, G):
    for S in range(2, 17):
        L = layout(D, G, S)
        assert L["total"] <= SMEM_LIMIT, (D, G, S, L["total"])
        assert L["rec_area"] <= L["ring"]  # the warps' records reuse the drained ring
        assert L["off_slots"] % 16 == 0 and L["stride"] % 4 == 0
        owners = {}
        for idx in range(G * D):
            o, j = divmod(idx, L["per"])
            assert o < S and j < L["per"]
            owners.setdefault(o, set()).add(j)
            for rank in range(S):
                row = rank * L["stride"]
                val = row + 4 * G + 2 * j  # (A, C) pair
                assert val % 2 == 0 and val + 2 <= S * L["stride"]
                assert val >= row + 4 * G and val + 2 <= row + L["stride"]
                hdr = row + 4 * (idx // D)  # (m, l, b, -) of the head
                assert hdr % 4 == 0 and hdr + 4 <= row + 4 * G
        # every value owned exactly once: owner o holds its consecutive slice
        covered = sorted(o * L["per"] + j for o, js in owners.items() for j in js)
        assert covered == list(range(G * D))
        # the bytes each owner arms its barrier with = the bytes its sources push
        for o in range(S):
            nvals = max(0, min(L["per"], G * D - o * L["per"]))
            pushed = S * (16 * G + 8 * len(owners.get(o, ())))
            assert pushed == S * (16 * G + 8 * nvals)


def test_reduction_lanes_stay_in_whole_warps():
    for S in range(2, 17):
        W = 2 if S <= 2 else 4 if S <= 4 else 8 if S <= 8 else 16
        assert W >= S and 32 % W == 0 and THREADS % W == 0
        for per in (1, 7, 16, 26, 32, 64, 128, 256):
            total = per * W
            for base in range(0, total, THREADS):  # warp w starts at w * 32
                for lane in range(32):
                    idx = base + lane
                    j, src = divmod(idx, W)
                    # the W lanes of one value share a warp and an iteration
                    first = base + (lane // W) * W
                    assert divmod(first, W)[0] == j and first // 32 == idx // 32
                    assert src < W


@pytest.mark.parametrize("page_size", [64, 128, 256, 1024])
def test_paged_speculative_tiles_stay_in_the_table_row(page_size):
    """Paged rows fetch their first tiles before the length is known: tile j of
    CTA `rank` is row position (rank + S j) * 64, and its page id is entry
    position / page_size of the row's table. With Lmax = max_pages *
    page_size, every speculative tile reads an entry inside the row (never
    the next row's), and a tile at or past the length attends nothing."""
    for D in (64, 128):
        stages = STAGES[D]
        for S, max_pages, n in itertools.product(range(2, 17), (1, 2, 3, 16, 64),
                                                 (0, 1, 64, 200, 4096)):
            Lmax = max_pages * page_size
            n = min(n, Lmax)
            cache_tiles = (Lmax + TILE - 1) // TILE
            for rank in range(S):
                nspec = min(stages, (cache_tiles - rank + S - 1) // S) if rank < cache_tiles else 0
                for j in range(nspec):
                    k0 = (rank + S * j) * TILE
                    assert 0 <= k0 // page_size < max_pages
                    attended = max(0, min(TILE, n - k0))
                    assert (attended == 0) == (k0 >= n)
