"""A host model of the prefill's fp16-path arithmetic (csrc/kernel_prefill.cuh,
parallax_prefill_workspace_bytes), checked over many shapes without a GPU:

- the workspace layout: the header, the fp16 copy of V from byte 1024, and
  the per-block records 256-byte aligned after it, without overlap, and the
  size parallax_prefill_workspace_bytes returns;
- the two records a tile checks: tile j of a sequence starting at packed row
  s0 has the K/V box rows s0 + 64 j .. +63. The records of blocks
  (s0 + 64 j) / 64 and min((s0 + 64 j + 63) / 64, nblk - 1) must cover every
  row of the box that lies inside the tensor, the neighbour's masked rows
  included, and no block past the last;
- the blocks a CTA scans for its bound on |k| cover every row of every box it
  loads;
- sigma: the smallest power of two with |r|_1 max|k| 2^-sigma below 2^14
  (126 for inf and NaN; 2^-126 is still a normal float), so that e*s 2^-sigma, with e <= 1, stays
  far below fp16's largest value 65504.
"""
import math
import random

import numpy as np
import pytest

from parameterized_local_linear_b200 import binding, build

ROWS, KEYS = 128, 64


def layout(B, L, Hkv, D):
    nblk = (L + 63) // 64
    v16 = B * L * Hkv * D * 2
    info_off = 1024 + (v16 + 255) // 256 * 256
    return nblk, info_off, info_off + B * Hkv * nblk * 4


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def test_workspace_layout_matches_the_library(lib):
    rnd = random.Random(5)
    for _ in range(200):
        B, L, Hkv, D = rnd.randint(1, 9), rnd.randint(1, 9000), rnd.randint(1, 16), rnd.choice((64, 128))
        nblk, info_off, total = layout(B, L, Hkv, D)
        assert binding.parallax_prefill_workspace_bytes(B, L, Hkv, D) == total
        assert info_off >= 1024 + B * L * Hkv * D * 2 and info_off % 256 == 0
        assert total - info_off == B * Hkv * nblk * 4


def tile_blocks(s0, j, nblk):
    a = s0 + j * KEYS
    return a >> 6, min((a + KEYS - 1) >> 6, nblk - 1)


@pytest.mark.parametrize("seed", range(20))
def test_tile_records_cover_every_box_row(seed):
    rnd = random.Random(seed)
    lens = [rnd.choice((0, 1, 63, 64, 65, rnd.randint(1, 700))) for _ in range(rnd.randint(1, 6))]
    total = sum(lens)
    if total == 0:
        return
    nblk = (total + 63) // 64
    s0 = 0
    for n in lens:
        nq = (n + ROWS - 1) // ROWS
        for qt in range(nq):  # causal: a query tile sees keys below its end
            kend = min(n, (qt + 1) * ROWS)
            nkt = (kend + KEYS - 1) // KEYS
            scanned = set()
            b_lo, b_hi = s0 >> 6, min((s0 + nkt * KEYS - 1) >> 6, nblk - 1)
            for j in range(nkt):
                b0, b1 = tile_blocks(s0, j, nblk)
                assert 0 <= b0 <= b1 < nblk and b1 - b0 <= 1
                box = range(s0 + j * KEYS, min(s0 + j * KEYS + KEYS, total))  # rows inside the tensor
                for row in box:
                    assert row // 64 in (b0, b1)
                    scanned.add(row // 64)
            # the CTA's bound on |k| scans blocks b_lo..b_hi: every box row is in one
            assert scanned <= set(range(b_lo, b_hi + 1))
        s0 += n


def sigma_of(bound):
    """The kernel's choice of sigma from the bound (fp32 arithmetic)."""
    b = np.float32(bound)
    if not (b < np.float32(16384.0)):
        if b < np.float32(3.0e38):
            e = int((b.view(np.uint32) >> 23) & 0xFF) - 127
            sigma = e - 13
        else:
            sigma = 126
    else:
        sigma = 0
    return min(max(sigma, 0), 126)


def test_sigma_keeps_the_scaled_bound_below_2_14():
    rnd = random.Random(9)
    values = [0.0, 1.0, 16383.0, 16384.0, 16385.0, 32767.0, 32768.0, 1e6, 2.15e35, 2.9e38, 3.3e38,
              float("inf"), float("nan")] + [10 ** rnd.uniform(-3, 38.4) for _ in range(4000)]
    for bound in values:
        sigma = sigma_of(bound)
        assert 0 <= sigma <= 126
        if math.isnan(bound) or math.isinf(bound) or bound >= 3.0e38:
            assert sigma == 126
            assert 3.4028235e38 * 2.0 ** -sigma < 4  # any finite |s|
            continue
        scaled = bound * 2.0 ** -sigma
        assert scaled < 16384.0, (bound, sigma)
        if sigma > 0:  # and sigma is the smallest that does it
            assert bound * 2.0 ** -(sigma - 1) >= 16384.0 * (1 - 1e-7), (bound, sigma)
        # e <= 1, so |e s 2^-sigma| <= |s| 2^-sigma <= bound 2^-sigma: far below 65504
        assert scaled * 3.99 < 65504.0


def test_l1_bound_dominates_the_probe_score():
    """|r . k| <= |r|_1 max|k| for bf16-like vectors (the bound sigma is set from)."""
    rng = np.random.default_rng(3)
    for _ in range(200):
        D = int(rng.choice((64, 128)))
        r = rng.standard_normal(D) * float(10 ** rng.uniform(-2, 3))
        k = rng.standard_normal((64, D)) * float(10 ** rng.uniform(-2, 3))
        s = k @ r
        assert np.max(np.abs(s)) <= np.sum(np.abs(r)) * np.max(np.abs(k)) * (1 + 1e-12)
