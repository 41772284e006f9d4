"""GPU parity of the paged-KV and block-sparse decode (the split-KV kernel
reading 64-key tiles through a page table or a per-sequence block list)
against the fp64 oracle, which gathers the same keys into a dense cache:
ragged lengths that end inside a page or block, a shuffled page pool, unsorted
and repeated block lists, empty selections, both cache layouts, GQA groups,
Parallax and R = 0, bf16 and fp32 inputs and outputs, several split counts,
and the device-side handling of ids outside the pool or the cache."""
import numpy as np
import pytest
import torch

import oracle
from parameterized_local_linear_b200 import binding

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}


def scaled_error(got, ref):
    g = got.float().cpu().double().numpy()
    assert np.all(np.isfinite(g)), "non-finite output"
    return float(np.max(np.abs(g - ref) / np.maximum(1.0, np.abs(ref))))


def status_bits(ws):
    rc, bits = ws.status(clear=True)
    return bits


def paged_case(seed, B, Hq, Hkv, D, page_size, max_pages, lens, spare=5, dtype=torch.bfloat16):
    g = torch.Generator(device="cuda").manual_seed(seed)
    num_pages = B * max_pages + spare
    q = torch.randn(B, Hq, D, device="cuda", generator=g).to(dtype)
    r = (torch.randn(B, Hq, D, device="cuda", generator=g) * 0.5).to(dtype)
    kp = torch.randn(num_pages, page_size, Hkv, D, device="cuda", generator=g).to(dtype)
    vp = torch.randn(num_pages, page_size, Hkv, D, device="cuda", generator=g).to(dtype)
    perm = torch.randperm(num_pages, generator=torch.Generator().manual_seed(seed))
    table = perm[:B * max_pages].reshape(B, max_pages).to(torch.int32).cuda()
    n = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return q, r, kp, vp, table, n


@pytest.mark.parametrize("D,Hq,Hkv", [(128, 16, 8), (64, 8, 8), (128, 8, 2), (128, 16, 2),
                                      (64, 32, 4)])
@pytest.mark.parametrize("page_size", [64, 256])
def test_paged_matches_oracle(D, Hq, Hkv, page_size):
    """G = Hq / Hkv up to 8: groups of more than 4 query heads with the probe
    (or 8 without) go through the generic kernel, the rest the TMA kernel."""
    max_pages = 4096 // page_size
    lens = [1, 700, 4096]
    q, r, kp, vp, table, n = paged_case(500 + D + page_size, 3, Hq, Hkv, D, page_size,
                                        max_pages, lens)
    for probe in (True, False):
        want = oracle.parallax_decode_paged(q, r, kp, vp, table, n, D ** -0.5, probe=probe)
        for out_dtype in (torch.bfloat16, torch.float32):
            for splits in (0, 1, 7):
                ws = binding.Workspace(3, Hq, Hkv, D, max_pages * page_size, splits)
                got = binding.parallax_decode_paged(q, r, kp, vp, table, n, out_dtype=out_dtype,
                                                    workspace=ws, num_splits=splits, probe=probe)
                err = scaled_error(got, want)
                assert err <= TOL[out_dtype], (probe, out_dtype, splits, err)
                assert status_bits(ws) == 0


@pytest.mark.parametrize("D,Hq,Hkv", [(128, 16, 8), (64, 8, 8), (128, 16, 2)])
@pytest.mark.parametrize("page_size", [64, 192])
def test_paged_f32_pool_matches_oracle(D, Hq, Hkv, page_size):
    """fp32 pools (q, r, pages all fp32) on the generic kernel, lengths that
    end inside a page, both output dtypes, Parallax and R = 0."""
    max_pages = (2048 + page_size - 1) // page_size
    lens = [1, 333, 2048]
    q, r, kp, vp, table, n = paged_case(530 + D + page_size, 3, Hq, Hkv, D, page_size,
                                        max_pages, lens, dtype=torch.float32)
    for probe in (True, False):
        want = oracle.parallax_decode_paged(q, r, kp, vp, table, n, D ** -0.5, probe=probe)
        for out_dtype in (torch.bfloat16, torch.float32):
            for splits in (0, 3):
                ws = binding.Workspace(3, Hq, Hkv, D, max_pages * page_size, splits)
                got = binding.parallax_decode_paged(q, r, kp, vp, table, n, out_dtype=out_dtype,
                                                    workspace=ws, num_splits=splits, probe=probe)
                err = scaled_error(got, want)
                assert err <= TOL[out_dtype], (probe, out_dtype, splits, err)
                assert status_bits(ws) == 0


def test_paged_without_lengths_and_bad_page():
    q, r, kp, vp, table, n = paged_case(520, 2, 16, 8, 128, 64, 10, [640, 640])
    want = oracle.parallax_decode_paged(q, r, kp, vp, table, None, 128 ** -0.5)
    ws = binding.Workspace(2, 16, 8, 128, 640)
    got = binding.parallax_decode_paged(q, r, kp, vp, table, None, out_dtype=torch.float32,
                                        workspace=ws)
    assert scaled_error(got, want) <= 1e-4
    assert status_bits(ws) == 0
    bad = table.clone()
    bad[1, 3] = kp.shape[0] + 7  # outside the pool: its keys are left out
    got = binding.parallax_decode_paged(q, r, kp, vp, bad, n, out_dtype=torch.float32,
                                        workspace=ws)
    assert status_bits(ws) & 2
    assert torch.isfinite(got).all()
    assert scaled_error(got[0], want[0]) <= 1e-4  # the other sequence is untouched


@pytest.mark.parametrize("page_size", [64, 256])
def test_paged_entries_past_the_length_are_ignored(page_size):
    """The cluster schedule (few items, num_splits = 0) fetches a row's first
    tiles before its length is known, so it reads table entries past the
    length. Whatever they hold (ids outside the pool here, or -1), those keys
    attend nothing and no status bit is set; an out-of-range id the length
    reaches still sets it."""
    max_pages = 2048 // page_size
    lens = [1, 300, 2048]
    q, r, kp, vp, table, n = paged_case(540 + page_size, 3, 16, 8, 128, page_size, max_pages,
                                        lens)
    for b, nb in enumerate(lens):
        used = (nb + page_size - 1) // page_size
        table[b, used:] = -1 if b % 2 else kp.shape[0] + 1000
    want = oracle.parallax_decode_paged(q, r, kp, vp, table, n, 128 ** -0.5)
    assert binding.parallax_decode_plan(3, 16, 8, 128, max_pages * page_size)["cluster_ctas"] > 0
    ws = binding.Workspace(3, 16, 8, 128, max_pages * page_size)
    for out_dtype in (torch.bfloat16, torch.float32):
        got = binding.parallax_decode_paged(q, r, kp, vp, table, n, out_dtype=out_dtype,
                                            workspace=ws)
        assert scaled_error(got, want) <= TOL[out_dtype], out_dtype
        assert status_bits(ws) == 0
    bad = table.clone()
    bad[1, 0] = kp.shape[0] + 3  # the length reaches this one
    binding.parallax_decode_paged(q, r, kp, vp, bad, n, workspace=ws)
    assert status_bits(ws) & 2


def sparse_case(seed, B, Hq, Hkv, D, Lmax, lens, layout, dtype=torch.bfloat16):
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn(B, Hq, D, device="cuda", generator=g).to(dtype)
    r = (torch.randn(B, Hq, D, device="cuda", generator=g) * 0.5).to(dtype)
    shape = (B, Hkv, Lmax, D) if layout == "bhsd" else (B, Lmax, Hkv, D)
    k = torch.randn(*shape, device="cuda", generator=g).to(dtype)
    v = torch.randn(*shape, device="cuda", generator=g).to(dtype)
    n = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return q, r, k, v, n


@pytest.mark.parametrize("layout", ["bhsd", "bshd"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(16, 8), (16, 2)])
def test_block_sparse_matches_oracle(layout, D, Hq, Hkv):
    B, Lmax, nblk = 4, 4096, 64
    lens = [4096, 1000, 37, 4096]
    q, r, k, v, n = sparse_case(600 + D, B, Hq, Hkv, D, Lmax, lens, layout)
    rng = np.random.default_rng(601)
    ids = np.zeros((B, 24), dtype=np.int32)
    cnt = np.array([24, 10, 3, 0], dtype=np.int32)
    ids[0] = rng.choice(nblk, 24, replace=False)        # unsorted
    ids[1, :10] = np.sort(rng.choice(nblk, 10, replace=False))  # some past the length
    ids[2, :3] = [0, 0, 5]                              # a repeat and a block past the end
    bid = torch.from_numpy(ids).cuda()
    bcnt = torch.from_numpy(cnt).cuda()
    k_o = k if layout == "bhsd" else k.transpose(1, 2)
    v_o = v if layout == "bhsd" else v.transpose(1, 2)
    for probe in (True, False):
        want = oracle.parallax_decode_block_sparse(q, r, k_o, v_o, ids, cnt, n, D ** -0.5,
                                                   probe=probe)
        for out_dtype in (torch.bfloat16, torch.float32):
            for splits in (0, 5):
                ws = binding.Workspace(B, Hq, Hkv, D, 64 * 24, splits)
                got = binding.parallax_decode_block_sparse(
                    q, r, k, v, bid, bcnt, n, out_dtype=out_dtype, workspace=ws,
                    num_splits=splits, probe=probe, kv_layout=layout)
                err = scaled_error(got, want)
                assert err <= TOL[out_dtype], (probe, out_dtype, splits, err)
                assert torch.all(got[3] == 0)  # no block listed: zero output
                assert status_bits(ws) == 0


@pytest.mark.parametrize("layout", ["bhsd", "bshd"])
@pytest.mark.parametrize("D,Hq,Hkv", [(64, 8, 4), (128, 16, 8)])
def test_block_sparse_f32_matches_oracle(layout, D, Hq, Hkv):
    """fp32 caches on the generic kernel: unsorted, repeated and
    past-the-length blocks, an empty list, both layouts and output dtypes."""
    B, Lmax, nblk = 4, 2048, 32
    lens = [2048, 700, 37, 2048]
    q, r, k, v, n = sparse_case(620 + D, B, Hq, Hkv, D, Lmax, lens, layout, dtype=torch.float32)
    rng = np.random.default_rng(621)
    ids = np.zeros((B, 12), dtype=np.int32)
    cnt = np.array([12, 8, 3, 0], dtype=np.int32)
    ids[0] = rng.choice(nblk, 12, replace=False)
    ids[1, :8] = np.sort(rng.choice(nblk, 8, replace=False))
    ids[2, :3] = [0, 0, 5]
    bid, bcnt = torch.from_numpy(ids).cuda(), torch.from_numpy(cnt).cuda()
    k_o = k if layout == "bhsd" else k.transpose(1, 2)
    v_o = v if layout == "bhsd" else v.transpose(1, 2)
    for probe in (True, False):
        want = oracle.parallax_decode_block_sparse(q, r, k_o, v_o, ids, cnt, n, D ** -0.5,
                                                   probe=probe)
        for out_dtype in (torch.bfloat16, torch.float32):
            for splits in (0, 4):
                ws = binding.Workspace(B, Hq, Hkv, D, 64 * 12, splits)
                got = binding.parallax_decode_block_sparse(
                    q, r, k, v, bid, bcnt, n, out_dtype=out_dtype, workspace=ws,
                    num_splits=splits, probe=probe, kv_layout=layout)
                err = scaled_error(got, want)
                assert err <= TOL[out_dtype], (probe, out_dtype, splits, err)
                assert torch.all(got[3] == 0)
                assert status_bits(ws) == 0


@pytest.mark.parametrize("Hq,Hkv", [(16, 8), (16, 2)])
def test_block_sparse_bad_ids_are_flagged(Hq, Hkv):
    B, D, Lmax = 2, 128, 1024
    q, r, k, v, n = sparse_case(610, B, Hq, Hkv, D, Lmax, [1024, 1024], "bhsd")
    ids = torch.tensor([[0, 99, 2], [1, 2, 3]], dtype=torch.int32, device="cuda")
    cnt = torch.tensor([3, 5], dtype=torch.int32, device="cuda")  # 5 > max_blocks: clamped
    ws = binding.Workspace(B, Hq, Hkv, D, 64 * 3)
    got = binding.parallax_decode_block_sparse(q, r, k, v, ids, cnt, n, out_dtype=torch.float32,
                                               workspace=ws)
    assert status_bits(ws) & 2
    assert torch.isfinite(got).all()
    want = oracle.parallax_decode_block_sparse(q, r, k, v, np.array([[0, 2, 0], [1, 2, 3]]),
                                               np.array([2, 3]), n, D ** -0.5)
    assert scaled_error(got, want) <= 1e-4


@pytest.mark.parametrize("mode", ["paged", "block_sparse"])
def test_full_size_sampled(mode):
    """The bench's paged (large workload, page 256) and block-sparse (long
    workload, half the blocks) steps at full size, in the bench's launch
    configuration: two batch rows against the oracle (gathering only their
    keys), every output finite."""
    from parameterized_local_linear_b200 import inputs
    if mode == "paged":
        w = inputs.WORKLOADS["large"]
        x = inputs.make_paged(w, 256, "cuda")
        plan = x["table"].shape[1] * 256
    else:
        w = inputs.WORKLOADS["long"]
        x = inputs.make_block_sparse(w, 0.5, "cuda")
        plan = 64 * x["block_ids"].shape[1]
    try:
        ws = binding.Workspace(w.B, w.Hq, w.Hkv, w.D, plan)
        if mode == "paged":
            got = binding.parallax_decode_paged(x["q"], x["r"], x["k"], x["v"], x["table"],
                                                x["seqlens"], scale=x["scale"],
                                                out_dtype=torch.float32, workspace=ws)
        else:
            got = binding.parallax_decode_block_sparse(x["q"], x["r"], x["k"], x["v"],
                                                       x["block_ids"], x["num_blocks"],
                                                       x["seqlens"], scale=x["scale"],
                                                       out_dtype=torch.float32, workspace=ws)
        assert bool(torch.isfinite(got).all())
        assert status_bits(ws) == 0
        for b in (0, w.B - 1):
            sl = slice(b, b + 1)
            if mode == "paged":
                table = x["table"][sl].cpu()
                used = torch.unique(table)
                remap = torch.full((int(used.max()) + 1,), -1, dtype=torch.int64)
                remap[used] = torch.arange(used.numel())
                dev_used = used.cuda()
                want = oracle.parallax_decode_paged(x["q"][sl], x["r"][sl], x["k"][dev_used],
                                                    x["v"][dev_used], remap[table.long()].numpy(),
                                                    x["seqlens"][sl], x["scale"])
            else:
                want = oracle.parallax_decode_block_sparse(
                    x["q"][sl], x["r"][sl], x["k"][sl], x["v"][sl], x["block_ids"][sl],
                    x["num_blocks"][sl], x["seqlens"][sl], x["scale"])
            assert scaled_error(got[sl], want) <= TOL[torch.float32], (mode, b)
    finally:
        del x
        torch.cuda.empty_cache()
