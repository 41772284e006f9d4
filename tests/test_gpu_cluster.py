"""GPU parity of the cluster schedule: for few (batch row, kv head) items a
num_splits = 0 decode runs one thread-block cluster per item, the CTAs taking
the item's 64-key tiles round-robin and combining their (m, l, b, A, C) in
distributed shared memory, with no merge kernel. Checked against the fp64
oracle (bf16 and fp32 outputs, Parallax and R = 0, GQA groups, both head
sizes, lengths that end inside a tile, lengths shorter than one tile per CTA,
empty and clamped lengths, NaN padding, and the other key spaces: a sliding
window, a shuffled page pool, block-sparse lists with repeats and ids
outside the cache), against the split-KV + merge schedule, for determinism,
and for its bounded waits."""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle
from parameterized_local_linear_b200 import binding, inputs

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}


def scaled_error(got, ref):
    g = got.detach().float().cpu().double().numpy()
    assert np.all(np.isfinite(g)), "non-finite output"
    return float(np.max(np.abs(g - ref) / np.maximum(1.0, np.abs(ref))))


def plan(w, out_dtype=torch.bfloat16, probe=True):
    return binding.parallax_decode_plan(w.B, w.Hq, w.Hkv, w.D, w.Lmax, w.dtype, out_dtype, probe)


def test_plan_takes_clusters_for_one_sequence_and_partitions_for_a_large_batch():
    q = plan(inputs.WORKLOADS["qwen"])
    assert 2 <= q["cluster_ctas"] <= 16 and q["grid_ctas"] == 8 * q["cluster_ctas"]
    big = plan(inputs.WORKLOADS["large"])
    assert big["cluster_ctas"] == 0 and big["grid_ctas"] >= 1
    fp32 = plan(inputs.WORKLOADS["tiny"])  # fp32 caches: the generic kernel's partitions
    assert fp32["cluster_ctas"] == 0


CASES = [
    # B, Hq, Hkv, D, Lmax, lengths
    (1, 16, 8, 128, 4096, (4096,)),        # the Qwen-3 decode step
    (1, 16, 8, 128, 4000, (3999,)),        # ends inside a tile, Lmax not a tile multiple
    (2, 32, 8, 128, 3000, (0, 2999)),      # an empty sequence, G = 4
    (3, 8, 8, 64, 2048, (1, 65, 2048)),    # MHA, D = 64
    (1, 4, 1, 128, 700, (700,)),           # G = 4, one item, fewer tiles than CTAs
    (2, 16, 8, 64, 100, (37, 100)),        # a cache shorter than two tiles
]


@pytest.mark.parametrize("B,Hq,Hkv,D,Lmax,lengths", CASES)
def test_cluster_matches_oracle(B, Hq, Hkv, D, Lmax, lengths):
    w = inputs.custom_workload("cluster", B=B, Hq=Hq, Hkv=Hkv, D=D, Lmax=Lmax, lengths=lengths,
                               seed=700 + B + Hq + D + Lmax, r_scale=1.0)
    assert plan(w)["cluster_ctas"] >= 2, plan(w)
    x = inputs.make_inputs(w, device="cuda")  # NaN padding past each length
    ref = oracle.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"], x["scale"])
    soft = oracle.softmax_decode(x["q"], x["k"], x["v"], x["seqlens"], x["scale"])
    for out_dtype in (torch.bfloat16, torch.float32):
        ws = binding.Workspace(B, Hq, Hkv, D, Lmax)
        got = binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"],
                                      scale=x["scale"], out_dtype=out_dtype, workspace=ws)
        err = scaled_error(got, ref)
        assert err <= TOL[out_dtype], (out_dtype, err)
        for b, n in enumerate(lengths):
            if n == 0:
                assert torch.all(got[b] == 0)
        got = binding.parallax_softmax_decode(x["q"], x["k"], x["v"], x["seqlens"],
                                              scale=x["scale"], out_dtype=out_dtype, workspace=ws)
        assert scaled_error(got, soft) <= TOL[out_dtype], out_dtype
        assert ws.status() == (0, 0)


def test_cluster_agrees_with_split_merge_and_is_deterministic():
    w = inputs.WORKLOADS["qwen"]
    x = inputs.make_inputs(w, device="cuda")
    a = binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"], scale=x["scale"],
                                out_dtype=torch.float32)
    b = binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"], scale=x["scale"],
                                out_dtype=torch.float32)
    assert torch.equal(a, b)
    P = binding.parallax_default_splits(w.B, w.Hq, w.Hkv, w.Lmax, w.dtype)
    c = binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"], scale=x["scale"],
                                out_dtype=torch.float32, num_splits=P)
    d = (a.double() - c.double()).abs() / c.double().abs().clamp(min=1.0)
    assert float(d.max()) <= 1e-4


def test_cluster_clamps_and_reports_lengths():
    w = inputs.custom_workload("cluster_clamp", B=2, Hq=16, Hkv=8, D=128, Lmax=300,
                               lengths=(300, 120), seed=711)
    x = inputs.make_inputs(w, device="cuda", pad_value=None)
    assert plan(w)["cluster_ctas"] >= 2
    ws = binding.Workspace(2, 16, 8, 128, 300)
    bad = torch.tensor([10_000, -3], dtype=torch.int32, device="cuda")
    got = binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], bad, scale=x["scale"],
                                  out_dtype=torch.float32, workspace=ws)
    rc, bits = ws.status(clear=True)
    assert bits & 2
    clamped = torch.tensor([300, 0], dtype=torch.int32)
    ref = oracle.parallax_decode(x["q"], x["r"], x["k"], x["v"], clamped, x["scale"])
    assert scaled_error(got, ref) <= 1e-4
    assert torch.all(got[1] == 0)


def test_cluster_bounded_wait_gives_up_and_context_survives():
    """The testing hook leaves the first stage of every CTA unfilled; the
    consumers' wait runs out (50 ms), the timeout is recorded, both cluster
    barriers are still reached, and a normal decode afterwards is correct."""
    lib = binding.load_library()
    fn = lib.parallax_testing_decode_stalled
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp] * 6 + [i] * 4 + [ctypes.c_float, vp, i, i, vp, ctypes.c_size_t, i]
    fn.restype = i
    w = inputs.custom_workload("cluster_stall", B=2, Hq=16, Hkv=8, D=128, Lmax=512, seed=712)
    assert plan(w)["cluster_ctas"] >= 2
    x = inputs.make_inputs(w, device="cuda")
    ws = binding.Workspace(2, 16, 8, 128, 512)
    out = torch.empty((2, 16, 128), device="cuda", dtype=torch.bfloat16)
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.perf_counter()
    rc = fn(x["q"].data_ptr(), x["r"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(),
            x["seqlens"].data_ptr(), out.data_ptr(), 2, 16, 8, 128, x["scale"], stream, 512, 0,
            ws.ptr(), ws.nbytes, 50)
    assert rc == 0
    status, bits = ws.status(clear=True)
    assert bits & 1 and status == -9
    assert time.perf_counter() - t0 < 5.0
    got = binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"], scale=x["scale"],
                                  out_dtype=torch.float32, workspace=ws)
    ref = oracle.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"], x["scale"])
    assert scaled_error(got, ref) <= 1e-4
    assert ws.status() == (0, 0)


# --------------------------------------- other key spaces on the cluster path --

def _windowed(x, W):
    """The cache holding only each row's last min(n, W) keys, for the oracle."""
    n = x["seqlens"].cpu().to(torch.int64)
    k, v = torch.zeros_like(x["k"]), torch.zeros_like(x["v"])
    for b in range(k.shape[0]):
        e = int(n[b]); s = max(0, e - W)
        k[b, :, :e - s] = x["k"][b, :, s:e]
        v[b, :, :e - s] = x["v"][b, :, s:e]
    return dict(x, k=k, v=v, seqlens=(n - (n - W).clamp(min=0)).to(torch.int32))


@pytest.mark.parametrize("W", [1, 200, 5000])
def test_cluster_sliding_window(W):
    w = inputs.custom_workload("cluster_win", B=2, Hq=16, Hkv=8, D=128, Lmax=3000,
                               lengths=(3000, 777), seed=720 + W, r_scale=1.0)
    x = inputs.make_inputs(w, device="cuda")
    assert plan(w)["cluster_ctas"] >= 2
    y = _windowed(x, W)
    want = oracle.parallax_decode(y["q"], y["r"], y["k"], y["v"], y["seqlens"], y["scale"])
    for out_dtype in (torch.bfloat16, torch.float32):
        got = binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"],
                                      scale=x["scale"], out_dtype=out_dtype, window=W)
        assert scaled_error(got, want) <= TOL[out_dtype], (W, out_dtype)


@pytest.mark.parametrize("page_size", [64, 256])
def test_cluster_paged(page_size):
    """One sequence's pages scattered through a pool (the Qwen-3 shape), and
    three sequences of ragged lengths: the cluster path against the oracle,
    and against the split-KV + merge path."""
    for w in (inputs.custom_workload("cluster_paged1", B=1, Hq=16, Hkv=8, D=128, Lmax=4096,
                                     seed=730, r_scale=1.0),
              inputs.custom_workload("cluster_paged3", B=3, Hq=16, Hkv=8, D=128, Lmax=2048,
                                     lengths=(1, 1000, 2048), seed=731, r_scale=1.0)):
        assert plan(w)["cluster_ctas"] >= 2
        x = inputs.make_paged(w, page_size, "cuda")
        want = oracle.parallax_decode_paged(x["q"], x["r"], x["k"], x["v"], x["table"],
                                            x["seqlens"], x["scale"])
        for out_dtype in (torch.bfloat16, torch.float32):
            ws = binding.Workspace(w.B, w.Hq, w.Hkv, w.D, x["table"].shape[1] * page_size)
            got = binding.parallax_decode_paged(x["q"], x["r"], x["k"], x["v"], x["table"],
                                                x["seqlens"], scale=x["scale"],
                                                out_dtype=out_dtype, workspace=ws)
            assert scaled_error(got, want) <= TOL[out_dtype], (w.name, page_size, out_dtype)
            assert ws.status() == (0, 0)
        split = binding.parallax_decode_paged(x["q"], x["r"], x["k"], x["v"], x["table"],
                                              x["seqlens"], scale=x["scale"],
                                              out_dtype=torch.float32, num_splits=23)
        assert scaled_error(got, split.double().cpu().numpy()) <= 1e-4


def test_cluster_block_sparse_and_bad_ids():
    w = inputs.custom_workload("cluster_bs", B=2, Hq=16, Hkv=8, D=128, Lmax=4096,
                               lengths=(4096, 1500), seed=740, r_scale=1.0)
    assert plan(w)["cluster_ctas"] >= 2
    x = inputs.make_inputs(w, device="cuda")
    ids = torch.tensor([[5, 0, 63, 17, 17, 40], [1, 22, 30, 0, 0, 0]], dtype=torch.int32)
    cnt = torch.tensor([6, 3], dtype=torch.int32)
    want = oracle.parallax_decode_block_sparse(x["q"], x["r"], x["k"], x["v"], ids.numpy(),
                                               cnt.numpy(), x["seqlens"], x["scale"])
    ws = binding.Workspace(2, 16, 8, 128, 64 * 6)
    for out_dtype in (torch.bfloat16, torch.float32):
        got = binding.parallax_decode_block_sparse(x["q"], x["r"], x["k"], x["v"], ids.cuda(),
                                                   cnt.cuda(), x["seqlens"], scale=x["scale"],
                                                   out_dtype=out_dtype, workspace=ws)
        assert scaled_error(got, want) <= TOL[out_dtype], out_dtype
        assert ws.status() == (0, 0)
    bad = ids.clone()
    bad[1, 1] = 1000  # outside the cache: left out and reported
    got = binding.parallax_decode_block_sparse(x["q"], x["r"], x["k"], x["v"], bad.cuda(),
                                               cnt.cuda(), x["seqlens"], scale=x["scale"],
                                               out_dtype=torch.float32, workspace=ws)
    rc, bits = ws.status(clear=True)
    assert bits & 2
    want_bad = oracle.parallax_decode_block_sparse(
        x["q"], x["r"], x["k"], x["v"], torch.tensor([[5, 0, 63, 17, 17, 40], [1, 30, 0, 0, 0, 0]],
                                                     dtype=torch.int32).numpy(),
        torch.tensor([6, 2], dtype=torch.int32).numpy(), x["seqlens"], x["scale"])
    assert scaled_error(got, want_bad) <= 1e-4
