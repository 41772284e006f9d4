"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances (element-wise, e = |o - o_ref| / max(1, |o_ref|)):
  bf16 output  e <= 2e-2
  fp32 output  e <= 1e-4   (the fp32 debug mode)
Cache lengths are checked exactly: padding is NaN, so any padding key that
reached an accumulator would make the output non-finite.
"""
import numpy as np
import pytest
import torch

import oracle
from parameterized_local_linear_b200 import binding, inputs

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    binding.load_library()
    yield
    torch.cuda.synchronize()


def scaled_error(got, ref):
    g = got.detach().float().cpu().double().numpy()
    assert np.all(np.isfinite(g)), "non-finite output"
    return float(np.max(np.abs(g - ref) / np.maximum(1.0, np.abs(ref)))) if g.size else 0.0


def assert_close(got, ref, tol, what=""):
    err = scaled_error(got, ref)
    assert err <= tol, f"{what}: max scaled error {err:.3e} > {tol:.1e}"


def run(x, out_dtype, num_splits=0, zero_r=False, ws=None):
    r = torch.zeros_like(x["r"]) if zero_r else x["r"]
    return binding.parallax_decode(x["q"], r, x["k"], x["v"], x["seqlens"], scale=x["scale"],
                                   out_dtype=out_dtype, num_splits=num_splits, workspace=ws)


def run_softmax(x, out_dtype, num_splits=0):
    return binding.parallax_softmax_decode(x["q"], x["k"], x["v"], x["seqlens"],
                                           scale=x["scale"], out_dtype=out_dtype,
                                           num_splits=num_splits)


def ref_parallax(x, rows=None, zero_r=False):
    sl = slice(None) if rows is None else rows
    r = torch.zeros_like(x["r"][sl]) if zero_r else x["r"][sl]
    return oracle.parallax_decode(x["q"][sl], r, x["k"][sl], x["v"][sl], x["seqlens"][sl],
                                  x["scale"])


def ref_softmax(x, rows=None):
    sl = slice(None) if rows is None else rows
    return oracle.softmax_decode(x["q"][sl], x["k"][sl], x["v"][sl], x["seqlens"][sl], x["scale"])


# ------------------------------------------------------------- the configs --

def test_tiny_fp32():
    """fp32 q/r/K/V, lengths [37, 128], fp32 output; also with r = 0."""
    x = inputs.make_inputs(inputs.WORKLOADS["tiny"], device="cuda")
    assert_close(run(x, torch.float32), ref_parallax(x), 1e-4, "tiny")
    soft = ref_softmax(x)
    assert_close(run(x, torch.float32, zero_r=True), soft, 1e-4, "tiny r=0")
    assert_close(run_softmax(x, torch.float32), soft, 1e-4, "tiny softmax kernel")
    assert_close(run(x, torch.bfloat16), ref_parallax(x), 2e-2, "tiny bf16 out")


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_qwen(out_dtype):
    x = inputs.make_inputs(inputs.WORKLOADS["qwen"], device="cuda")
    ref = ref_parallax(x)
    assert_close(run(x, out_dtype), ref, TOL[out_dtype], "qwen")
    assert_close(run_softmax(x, out_dtype), ref_softmax(x), TOL[out_dtype], "qwen softmax")


# ------------------------------------------------- shapes, splits, lengths --

LENGTHS = (1, 63, 64, 65, 0, 300, 1000, 17)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(16, 8), (8, 8), (16, 4), (32, 4)])
def test_shapes_and_splits(D, Hq, Hkv):
    w = inputs.custom_workload("shape", B=len(LENGTHS), Hq=Hq, Hkv=Hkv, D=D, Lmax=1000,
                               lengths=LENGTHS, seed=100 + D + Hq + Hkv, r_scale=0.5)
    x = inputs.make_inputs(w, device="cuda")
    ref = ref_parallax(x)
    soft = ref_softmax(x)
    for out_dtype in (torch.bfloat16, torch.float32):
        for splits in (0, 1, 2, 3, 7, 64, 1000):
            tag = f"D={D} G={Hq // Hkv} splits={splits} out={out_dtype}"
            got = run(x, out_dtype, splits)
            assert_close(got, ref, TOL[out_dtype], tag)
            assert torch.all(got[4] == 0), f"{tag}: empty sequence not zero"
            assert_close(run_softmax(x, out_dtype, splits), soft, TOL[out_dtype],
                         tag + " softmax")


def test_all_sequences_empty():
    w = inputs.custom_workload("empty", B=3, Hq=16, Hkv=8, D=128, Lmax=64, lengths=(0, 0, 0))
    x = inputs.make_inputs(w, device="cuda")
    out = torch.full((3, 16, 128), 7.0, device="cuda", dtype=torch.bfloat16)
    binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"], scale=x["scale"],
                            out=out)
    assert torch.all(out == 0)


def test_lengths_are_clamped_and_reported():
    w = inputs.custom_workload("clamp", B=3, Hq=16, Hkv=8, D=128, Lmax=200, lengths=(5, 150, 200))
    x = inputs.make_inputs(w, device="cuda", pad_value=None)
    ws = binding.Workspace(3, 16, 8, 128, 200)
    bad = torch.tensor([-4, 150, 10_000], dtype=torch.int32, device="cuda")
    y = dict(x, seqlens=bad)
    got = run(y, torch.float32, ws=ws)
    rc, bits = ws.status(clear=True)
    assert rc == -11 and bits == 2
    clamped = dict(x, seqlens=torch.tensor([0, 150, 200], dtype=torch.int32))
    assert_close(got, ref_parallax(clamped), 1e-4, "clamped lengths")
    run(x, torch.float32, ws=ws)
    assert ws.status() == (0, 0)


# ------------------------------------------------------- execution checks --

def test_deterministic_and_phases():
    x = inputs.make_inputs(inputs.custom_workload("det", B=5, Hq=16, Hkv=8, D=128, Lmax=3000,
                                                  lengths="uniform", seed=7), device="cuda")
    ws = binding.Workspace(5, 16, 8, 128, 3000)
    # the default schedule (40 items: one cluster each) and the split-KV +
    # merge schedule at the default partition count are each deterministic
    P = binding.parallax_default_splits(5, 16, 8, 3000)
    for splits in (0, P):
        a = run(x, torch.bfloat16, num_splits=splits, ws=ws)
        b = run(x, torch.bfloat16, num_splits=splits, ws=ws)
        assert torch.equal(a, b), f"two identical calls differ (num_splits={splits})"
    c = torch.empty_like(a)
    binding.parallax_decode_phase(1, True, x["q"], x["r"], x["k"], x["v"], x["seqlens"], c, ws,
                                  scale=x["scale"], num_splits=P)
    binding.parallax_decode_phase(2, True, x["q"], x["r"], x["k"], x["v"], x["seqlens"], c, ws,
                                  scale=x["scale"], num_splits=P)
    assert torch.equal(a, c), "phase 1 + phase 2 differs from one call"
    assert ws.status() == (0, 0)


def test_r_zero_equals_softmax_kernel():
    x = inputs.make_inputs(inputs.custom_workload("r0", B=4, Hq=16, Hkv=8, D=128, Lmax=2048,
                                                  lengths="uniform", seed=8), device="cuda")
    soft = ref_softmax(x)
    a = run(x, torch.float32, zero_r=True)
    b = run_softmax(x, torch.float32)
    assert_close(a, soft, 1e-4, "parallax r=0")
    assert_close(b, soft, 1e-4, "softmax kernel")
    assert_close(a, b.double().cpu().numpy(), 1e-5, "parallax r=0 vs softmax kernel")


def test_streams_and_graph_capture():
    x = inputs.make_inputs(inputs.WORKLOADS["qwen"], device="cuda", pad_value=None)
    ws = binding.Workspace(1, 16, 8, 128, 4096)
    out = torch.empty((1, 16, 128), device="cuda", dtype=torch.bfloat16)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"], scale=x["scale"],
                                out=out, workspace=ws)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"],
                                    scale=x["scale"], out=out, workspace=ws)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert_close(out, ref_parallax(x), 2e-2, "graph replay")


# ------------------------------------------- full-size configs (sampled) ----

def _sample_rows(x, n_random=2, seed=0):
    n = x["seqlens"].cpu()
    B = n.numel()
    rows = {0, B - 1, int(torch.argmin(n)), int(torch.argmax(n))}
    g = torch.Generator().manual_seed(seed)
    rows |= set(torch.randint(0, B, (n_random,), generator=g).tolist())
    return sorted(rows)


@pytest.mark.parametrize("name", ["large", "long", "ragged"])
def test_full_size_sampled(name):
    """The bench's workload and launch configuration (auto split count); the
    oracle checks sampled batch rows, every output must be finite, and r = 0
    must agree with the softmax kernel everywhere."""
    w = inputs.WORKLOADS[name]
    x = inputs.make_inputs(w, device="cuda", pad_value=float("nan"))
    try:
        rows = _sample_rows(x, seed=w.seed)
        idx = torch.tensor(rows, device="cuda")
        sub = {k: (v[idx] if torch.is_tensor(v) else v) for k, v in x.items()}
        ref = ref_parallax(sub)
        for out_dtype in (torch.bfloat16, torch.float32):
            out = run(x, out_dtype)
            assert bool(torch.isfinite(out.float()).all()), f"{name}: non-finite output"
            assert_close(out[idx], ref, TOL[out_dtype], f"{name} {out_dtype}")
        a = run(x, torch.float32, zero_r=True)
        b = run_softmax(x, torch.float32)
        err = float(((a - b).abs() / b.abs().clamp_min(1.0)).max())
        assert err <= 1e-5, f"{name}: r=0 vs softmax kernel {err:.3e}"
        assert_close(b[idx], ref_softmax(sub), 1e-4, f"{name} softmax")
    finally:
        del x
        torch.cuda.empty_cache()


def test_merge_many_pieces_and_workspace_reuse():
    """Sequences cut into 2 to ~250 pieces (more than one register chunk of
    partial records in the merge), a keyless sequence among them, the probe
    and the softmax kernel, and one workspace reused across calls and split
    counts: every call writes the records it reads."""
    w = inputs.custom_workload("merge", B=4, Hq=8, Hkv=2, D=128, Lmax=3000, lengths="uniform",
                               seed=41)
    x = inputs.make_inputs(w, device="cuda")
    x["seqlens"][2] = 0  # no keys: o = 0, written by the partition that covers row 2
    ref = ref_parallax(x)
    soft = ref_softmax(x)
    ws = binding.Workspace(4, 8, 2, 128, 3000, num_splits=1000)
    for splits in (3, 17, 160, 1000):
        outs = [run(x, torch.float32, num_splits=splits, ws=ws) for _ in range(3)]
        for o in outs[1:]:
            assert torch.equal(o, outs[0]), f"{splits} splits: calls differ"
        assert_close(outs[0], ref, 1e-4, f"{splits} splits")
        assert float(outs[0][2].abs().max()) == 0.0
        b = binding.parallax_softmax_decode(x["q"], x["k"], x["v"], x["seqlens"],
                                            scale=x["scale"], out_dtype=torch.float32,
                                            num_splits=splits, workspace=ws)
        assert_close(b, soft, 1e-4, f"softmax, {splits} splits")
    assert ws.status() == (0, 0)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(16, 8), (16, 4)])
def test_fp32_output_large_probe_few_keys(D, Hq, Hkv):
    """The fp32-output bound where the weights' rounding weighs most: r at
    twice the large configs' scale (|s| ~ 2 sqrt(D)) and rows of 1 to 300
    keys, on the cluster schedule (num_splits = 0) and the split-KV + merge
    schedule."""
    w = inputs.custom_workload("few", B=6, Hq=Hq, Hkv=Hkv, D=D, Lmax=300,
                               lengths=(1, 2, 5, 17, 64, 300), seed=900 + D + Hkv, r_scale=2.0)
    x = inputs.make_inputs(w, device="cuda")
    ref = ref_parallax(x)
    for splits in (0, 7):
        assert_close(run(x, torch.float32, splits), ref, 1e-4, f"D={D} G={Hq // Hkv} {splits}")
