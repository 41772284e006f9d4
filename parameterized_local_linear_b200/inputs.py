"""Seeded synthetic decode workloads.

This module only draws random inputs; it holds none of the method's
arithmetic. It is the one module that both the CUDA path (tests, bench,
smoke) and the oracle's tests use.

The workloads are Qwen-3-shaped decode steps (head_dim 128, 16 query heads
over 8 kv heads), the backbone the Parallax pretraining runs use ("Come
Parallax cambia ..." / "I guadagni di pretraining ..." on the encorp.ai page;
"What the paper found" on the neuraltrendhub summary), plus a tiny fp32 case.
The pages train and evaluate on datasets that are not available here; these
seeded inputs stand in for them.

Layouts (contiguous, row-major):
    q, r     [B, Hq, D]
    k, v     [B, Hkv, Lmax, D]   (a max-length-padded cache)
    seqlens  [B] int32           (keys 0 .. seqlens[b]-1 are valid)

Draw order for one workload: q, r, K, V, then the per-(batch, kv head) key
offset mu (long-context workload only), then seqlens (ragged workload only),
all from one torch.Generator seeded with the workload's seed, on the device
the tensors are made on.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    Lmax: int
    dtype: torch.dtype
    seed: int
    # "full": every sequence is Lmax long; "uniform": U{1..Lmax} per sequence;
    # otherwise an explicit tuple of lengths.
    lengths: object = "full"
    r_scale: float = 1.0
    k_offset_std: float = 0.0
    scale: Optional[float] = None  # default 1/sqrt(D)

    @property
    def qk_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.D)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def kv_bytes_full(self) -> int:
        """Bytes of the allocated (padded) K and V caches."""
        return 2 * self.B * self.Hkv * self.Lmax * self.D * _itemsize(self.dtype)


def _itemsize(dtype: torch.dtype) -> int:
    return torch.tensor([], dtype=dtype).element_size()


WORKLOADS = {
    # fp32 debug case; also run with r = 0
    "tiny": Workload("tiny", B=2, Hq=4, Hkv=2, D=64, Lmax=128, dtype=torch.float32,
                     seed=0, lengths=(37, 128), scale=1.0 / 8.0),
    # one Qwen-3-0.6B-shaped layer at context 4096
    "qwen": Workload("qwen", B=1, Hq=16, Hkv=8, D=128, Lmax=4096, dtype=torch.bfloat16,
                     seed=1, r_scale=0.5),
    # large batch, ~34 GB of KV
    "large": Workload("large", B=2048, Hq=16, Hkv=8, D=128, Lmax=4096,
                      dtype=torch.bfloat16, seed=2),
    # long context, keys with per-(batch, kv head) mean offsets of variance 0.5
    "long": Workload("long", B=256, Hq=16, Hkv=8, D=128, Lmax=32768,
                     dtype=torch.bfloat16, seed=3, k_offset_std=math.sqrt(0.5)),
    # ragged lengths U{1..32768}, r = 0.3 N(0,1), padded to 32768
    "ragged": Workload("ragged", B=512, Hq=16, Hkv=8, D=128, Lmax=32768,
                       dtype=torch.bfloat16, seed=4, lengths="uniform", r_scale=0.3),
}


def draw_lengths(w: Workload, gen: torch.Generator, device) -> torch.Tensor:
    if w.lengths == "full":
        return torch.full((w.B,), w.Lmax, dtype=torch.int32, device=device)
    if w.lengths == "uniform":
        return torch.randint(1, w.Lmax + 1, (w.B,), generator=gen, device=device,
                             dtype=torch.int64).to(torch.int32)
    lens = torch.tensor(list(w.lengths), dtype=torch.int32, device=device)
    assert lens.numel() == w.B
    return lens


def make_inputs(w: Workload, device="cpu", pad_value: Optional[float] = float("nan"),
                zero_r: bool = False) -> dict:
    """Draw one decode step of workload `w` on `device`.

    pad_value fills cache positions >= seqlens[b] (NaN in correctness runs, so
    that a kernel reading padding shows it); None leaves the random values.
    zero_r replaces the probe by zeros (the R = 0 case).
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    dt = w.dtype
    q = torch.randn((w.B, w.Hq, w.D), generator=gen, device=device, dtype=dt)
    r = torch.randn((w.B, w.Hq, w.D), generator=gen, device=device, dtype=dt)
    if w.r_scale != 1.0:
        r = (r * w.r_scale).to(dt)
    if zero_r:
        r = torch.zeros_like(r)
    kv_shape = (w.B, w.Hkv, w.Lmax, w.D)
    k = torch.randn(kv_shape, generator=gen, device=device, dtype=dt)
    v = torch.randn(kv_shape, generator=gen, device=device, dtype=dt)
    if w.k_offset_std > 0.0:
        mu = torch.randn((w.B, w.Hkv, 1, w.D), generator=gen, device=device,
                         dtype=torch.float32) * w.k_offset_std
        for b in range(w.B):  # in place, one batch row at a time, to bound memory
            k[b] = (k[b].float() + mu[b]).to(dt)
    seqlens = draw_lengths(w, gen, device)
    if pad_value is not None:
        fill_padding(k, v, seqlens, pad_value)
    return {"q": q, "r": r, "k": k, "v": v, "seqlens": seqlens, "scale": w.qk_scale}


def fill_padding(k: torch.Tensor, v: torch.Tensor, seqlens: torch.Tensor,
                 value: float) -> None:
    """Write `value` into every cache position at or beyond seqlens[b]."""
    Lmax = k.shape[2]
    lens = seqlens.to(torch.int64).tolist()
    for b, n in enumerate(lens):
        n = max(0, min(int(n), Lmax))
        if n < Lmax:
            k[b, :, n:, :] = value
            v[b, :, n:, :] = value


def custom_workload(name: str, B: int, Hq: int, Hkv: int, D: int, Lmax: int,
                    lengths: Sequence[int] | str = "full", dtype=torch.bfloat16,
                    seed: int = 0, r_scale: float = 1.0, k_offset_std: float = 0.0,
                    scale: Optional[float] = None) -> Workload:
    if not isinstance(lengths, str):
        lengths = tuple(int(x) for x in lengths)
    return Workload(name, B, Hq, Hkv, D, Lmax, dtype, seed, lengths, r_scale,
                    k_offset_std, scale)


def make_paged(w: Workload, page_size: int, device="cpu") -> dict:
    """Workload `w` with its cache in pages: a pool [B * ceil(Lmax / page_size),
    page_size, Hkv, D] of N(0,1) keys and values (the workload's key offsets
    are not applied) and a block table that scatters each sequence's pages
    through the pool in a seeded random order."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    dt = w.dtype
    q = torch.randn((w.B, w.Hq, w.D), generator=gen, device=device, dtype=dt)
    r = torch.randn((w.B, w.Hq, w.D), generator=gen, device=device, dtype=dt)
    if w.r_scale != 1.0:
        r = (r * w.r_scale).to(dt)
    per = (w.Lmax + page_size - 1) // page_size
    pool = (w.B * per, page_size, w.Hkv, w.D)
    k = torch.randn(pool, generator=gen, device=device, dtype=dt)
    v = torch.randn(pool, generator=gen, device=device, dtype=dt)
    seqlens = draw_lengths(w, gen, device)
    perm = torch.randperm(w.B * per, generator=gen, device=device)
    table = perm.reshape(w.B, per).to(torch.int32)
    return {"q": q, "r": r, "k": k, "v": v, "seqlens": seqlens, "table": table,
            "page_size": page_size, "scale": w.qk_scale}


def make_block_sparse(w: Workload, density: float, device="cpu") -> dict:
    """Workload `w` (dense cache, padding left as drawn) plus, per sequence, a
    seeded random subset of about `density` of the 64-key blocks below its
    length (at least one), sorted, padded to the longest list."""
    x = make_inputs(w, device=device, pad_value=None)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed + 1000)
    lens = x["seqlens"].cpu().tolist()
    lists = []
    for n in lens:
        nb = max(1, (int(n) + 63) // 64)
        take = max(1, int(round(density * nb)))
        lists.append(torch.sort(torch.randperm(nb, generator=gen)[:take]).values)
    width = max(len(a) for a in lists)
    ids = torch.zeros((w.B, width), dtype=torch.int32)
    for b, a in enumerate(lists):
        ids[b, :len(a)] = a.to(torch.int32)
    x["block_ids"] = ids.to(device)
    x["num_blocks"] = torch.tensor([len(a) for a in lists], dtype=torch.int32, device=device)
    return x
