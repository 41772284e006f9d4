"""CPU model of the split-KV kernel's shared-memory ring (kernel_tc.cuh):
one producer fills stages in tile order after an empty-barrier wait; the
consumer warps, in groups that take alternate tiles, wait on the stage's full
barrier by phase parity and release it with one arrival per warp; every piece
ends with two all-consumer barriers. Random interleavings check that each tile
is consumed exactly once by all warps of its group, from the stage it was
loaded into, and that no stage is refilled while in use, for the stage and
group counts the kernel is built with (read from common.cuh). The model also
has to catch the broken case: an odd stage count with two groups lets a group
wait two phases ahead of a barrier, where a parity wait passes too early."""
import os
import random
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
COMMON = os.path.join(ROOT, "parameterized_local_linear_b200", "csrc", "common.cuh")


class Barrier:
    """An mbarrier: arrival count, transaction bytes, phase; try_wait.parity(P)
    succeeds once the phase with parity P has completed (a fresh barrier counts
    the phase before it, parity 1, as completed)."""

    def __init__(self, count):
        self.count, self.pending, self.phase, self.tx = count, count, 0, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than the barrier expects"
        self._advance()

    def expect_tx(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._advance()

    def _advance(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):
        return (self.phase & 1) != parity


def simulate(seed, pieces, stages, groups, warps_per_group=4):
    rnd = random.Random(seed)
    nwarps = groups * warps_per_group
    full = [Barrier(1) for _ in range(stages)]
    empty = [Barrier(warps_per_group) for _ in range(stages)]
    fin = [Barrier(nwarps), Barrier(nwarps)]
    tiles = [(pi, t) for pi, n in enumerate(pieces) for t in range(n)]
    in_stage = [None] * stages
    landing = []
    prod = {"i": 0, "stage": 0, "ph": 0}
    warps = [{"pi": 0, "t": 0, "tseq": 0, "stage": 0, "ph": 0, "fph": 0, "mode": "tile"}
             for _ in range(nwarps)]
    seen = {}
    for _ in range(10 ** 6):
        actors = (["producer"] if prod["i"] < len(tiles) else []) + (["tma"] if landing else [])
        actors += [w for w in range(nwarps) if warps[w]["pi"] < len(pieces)]
        if not actors:
            break
        a = rnd.choice(actors)
        if a == "producer":
            st = prod["stage"]
            if empty[st].done(prod["ph"] ^ 1):
                assert in_stage[st] is None, f"stage {st} refilled while in use"
                full[st].expect_tx(1)
                in_stage[st] = tiles[prod["i"]]
                landing.append(st)
                prod["i"] += 1
                prod["stage"] = (st + 1) % stages
                prod["ph"] ^= int(prod["stage"] == 0)
        elif a == "tma":
            full[landing.pop(rnd.randrange(len(landing)))].complete_tx(1)
        else:
            w, c = a, warps[a]
            if c["mode"] == "tile":
                if c["t"] == pieces[c["pi"]]:
                    c["mode"] = "fin0"
                    continue
                tile = (c["pi"], c["t"])
                if c["tseq"] % groups == w // warps_per_group:  # this group's tile
                    st = c["stage"]
                    if not full[st].done(c["ph"]):
                        continue
                    assert in_stage[st] == tile, f"warp {w} read stage {st} too early"
                    seen.setdefault(tile, set()).add(w)
                    empty[st].arrive()
                    if len(seen[tile]) == warps_per_group:
                        in_stage[st] = None
                c["stage"] = (c["stage"] + 1) % stages
                c["ph"] ^= int(c["stage"] == 0)
                c["t"] += 1
                c["tseq"] += 1
            elif c["mode"] in ("fin0", "fin1"):
                fin[c["mode"] == "fin1"].arrive()
                c["mode"] = "wait0" if c["mode"] == "fin0" else "wait1"
            elif fin[c["mode"] == "wait1"].done(c["fph"]):
                if c["mode"] == "wait0":
                    c["mode"] = "fin1"
                else:
                    c["fph"] ^= 1
                    c["pi"] += 1
                    c["t"] = 0
                    c["mode"] = "tile"
    else:
        raise AssertionError("deadlock")
    for tile in tiles:
        assert len(seen.get(tile, ())) == warps_per_group, f"tile {tile} not consumed once"


def kernel_config():
    text = open(COMMON).read()
    groups = int(re.search(r"kConsumerGroups\s*=\s*(\d+)", text).group(1))
    warps = int(re.search(r"kConsumerWarps\s*=\s*(\d+)", text).group(1))
    m = re.search(r"kStages\s*=\s*D\s*==\s*128\s*\?\s*(\d+)\s*:\s*(\d+)", text)
    return groups, warps, {128: int(m.group(1)), 64: int(m.group(2))}


def run_many(stages, groups, warps, n=200):
    rnd = random.Random(stages * 31 + groups)
    for seed in range(n):
        pieces = [rnd.randint(1, 12) for _ in range(rnd.randint(1, 8))]
        simulate(seed, pieces, stages, groups, warps)


@pytest.mark.parametrize("D", [64, 128])
def test_kernel_ring_is_consistent(D):
    groups, warps, stages = kernel_config()
    run_many(stages[D], groups, warps)


def test_model_catches_an_odd_ring_with_two_groups():
    with pytest.raises(AssertionError):
        run_many(3, 2, 4)
