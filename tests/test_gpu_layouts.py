"""GPU parity for the cache layouts, absent lengths and sliding windows.

- The pages' cache layout (B, kv_len, H, D) ("parallax-kernel 0.1.0" README,
  "Quickstart / Decoding (CuTeDSL)") gives exactly the result of the
  [B, Hkv, Lmax, D] layout on the same values, and matches the oracle.
- The pages' call form: q, r of shape (B, 1, H, D), no lengths.
- A sliding window W attends the last min(n, W) keys of each sequence (the
  README's introduction: sliding windows are structurally compatible). The
  reference is the oracle on a cache that holds only those keys.
"""
import numpy as np
import pytest
import torch

import oracle
from parameterized_local_linear_b200 import binding, inputs

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}
LENGTHS = (1, 63, 64, 65, 0, 300, 1000, 17)


def scaled_error(got, ref):
    g = got.detach().float().cpu().double().numpy()
    assert np.all(np.isfinite(g)), "non-finite output"
    return float(np.max(np.abs(g - ref) / np.maximum(1.0, np.abs(ref))))


def bshd(t):
    return t.permute(0, 2, 1, 3).contiguous()


def windowed(x, W):
    """The cache and lengths the oracle sees for window W: each row's last
    min(n, W) keys, moved to the front."""
    k = torch.full_like(x["k"], float("nan"))
    v = torch.full_like(x["v"], float("nan"))
    lens = x["seqlens"].cpu().tolist()
    new = []
    for b, n in enumerate(lens):
        m = min(n, W)
        k[b, :, :m] = x["k"][b, :, n - m:n]
        v[b, :, :m] = x["v"][b, :, n - m:n]
        new.append(m)
    return dict(x, k=k, v=v, seqlens=torch.tensor(new, dtype=torch.int32, device=x["k"].device))


def ref(x):
    return oracle.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"], x["scale"])


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(16, 8), (8, 8), (16, 4)])
def test_bshd_layout(D, Hq, Hkv):
    w = inputs.custom_workload("bshd", B=len(LENGTHS), Hq=Hq, Hkv=Hkv, D=D, Lmax=1000,
                               lengths=LENGTHS, seed=200 + D + Hq + Hkv, r_scale=0.5)
    x = inputs.make_inputs(w, device="cuda")
    kb, vb = bshd(x["k"]), bshd(x["v"])
    want = ref(x)
    want_soft = oracle.softmax_decode(x["q"], x["k"], x["v"], x["seqlens"], x["scale"])
    for out_dtype in (torch.bfloat16, torch.float32):
        for splits in (0, 3, 7):
            a = binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"],
                                        scale=x["scale"], out_dtype=out_dtype,
                                        num_splits=splits)
            b = binding.parallax_decode(x["q"], x["r"], kb, vb, x["seqlens"], scale=x["scale"],
                                        out_dtype=out_dtype, num_splits=splits,
                                        kv_layout="bshd")
            assert torch.equal(a, b), "layouts differ on the same values"
            assert scaled_error(b, want) <= TOL[out_dtype]
            s = binding.parallax_softmax_decode(x["q"], kb, vb, x["seqlens"], scale=x["scale"],
                                                out_dtype=out_dtype, num_splits=splits,
                                                kv_layout="bshd")
            assert scaled_error(s, want_soft) <= TOL[out_dtype]


def test_bshd_fp32_inputs():
    w = inputs.custom_workload("bshd32", B=3, Hq=4, Hkv=2, D=64, Lmax=130, lengths=(130, 5, 77),
                               dtype=torch.float32, seed=210)
    x = inputs.make_inputs(w, device="cuda")
    got = binding.parallax_decode(x["q"], x["r"], bshd(x["k"]), bshd(x["v"]), x["seqlens"],
                                  scale=x["scale"], out_dtype=torch.float32, kv_layout="bshd")
    assert scaled_error(got, ref(x)) <= 1e-4


def test_pages_call_form():
    """q, r (B, 1, H, D); k, v (B, kv_len, H, D); no lengths; MHA."""
    B, H, D, L = 4, 8, 128, 4096
    g = torch.Generator(device="cuda").manual_seed(220)
    q = torch.randn(B, 1, H, D, device="cuda", dtype=torch.bfloat16, generator=g)
    r = torch.randn(B, 1, H, D, device="cuda", dtype=torch.bfloat16, generator=g)
    k = torch.randn(B, L, H, D, device="cuda", dtype=torch.bfloat16, generator=g)
    v = torch.randn(B, L, H, D, device="cuda", dtype=torch.bfloat16, generator=g)
    o = binding.parallax_decode(q, r, k, v, scale=D ** -0.5)
    assert o.shape == (B, 1, H, D)
    want = oracle.parallax_decode(q[:, 0], r[:, 0], k.permute(0, 2, 1, 3), v.permute(0, 2, 1, 3),
                                  [L] * B, D ** -0.5)
    assert scaled_error(o[:, 0], want) <= 2e-2


def test_absent_lengths_mean_full():
    w = inputs.custom_workload("full", B=3, Hq=16, Hkv=8, D=128, Lmax=777, seed=230)
    x = inputs.make_inputs(w, device="cuda", pad_value=None)
    a = binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], None, scale=x["scale"])
    b = binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"], scale=x["scale"])
    assert torch.equal(a, b)


@pytest.mark.parametrize("W", [1, 50, 64, 100, 5000])
@pytest.mark.parametrize("layout", ["bhsd", "bshd"])
def test_sliding_window(W, layout):
    w = inputs.custom_workload("win", B=len(LENGTHS), Hq=16, Hkv=8, D=128, Lmax=1000,
                               lengths=LENGTHS, seed=240 + W, r_scale=0.5)
    x = inputs.make_inputs(w, device="cuda")
    want = ref(windowed(x, W))
    kc, vc = (bshd(x["k"]), bshd(x["v"])) if layout == "bshd" else (x["k"], x["v"])
    for out_dtype in (torch.bfloat16, torch.float32):
        for splits in (0, 5):
            got = binding.parallax_decode(x["q"], x["r"], kc, vc, x["seqlens"], scale=x["scale"],
                                          out_dtype=out_dtype, num_splits=splits,
                                          kv_layout=layout, window=W)
            assert scaled_error(got, want) <= TOL[out_dtype], (W, layout, out_dtype, splits)
            assert torch.all(got[4] == 0)  # empty sequence


def test_window_without_lengths():
    w = inputs.custom_workload("winfull", B=2, Hq=16, Hkv=8, D=128, Lmax=700, seed=250)
    x = inputs.make_inputs(w, device="cuda", pad_value=None)
    got = binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], None, scale=x["scale"],
                                  out_dtype=torch.float32, window=129)
    assert scaled_error(got, ref(windowed(x, 129))) <= 1e-4
