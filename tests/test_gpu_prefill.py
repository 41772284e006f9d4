"""GPU parity of the tcgen05 prefill forward (the README's parallax_func,
"Training (Triton)": (B, H, L, D) -> (B, H, L, D), causal) against the fp64
oracle's prefill. Partial 128-row query tiles and 64-key tiles, GQA, both
head dimensions, causal and not, bf16 and fp32 outputs, and probes at the
README's recipe (r drawn like q, N(0,1)) as well as half and twice that
scale: the probe score's size multiplies every weight's rounding error."""
import numpy as np
import pytest
import torch

import oracle
from parameterized_local_linear_b200 import binding

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}


def make(B, Hq, Hkv, L, D, seed, r_scale=1.0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn(B, Hq, L, D, device="cuda", dtype=torch.bfloat16, generator=g)
    r = (torch.randn(B, Hq, L, D, device="cuda", dtype=torch.bfloat16, generator=g) * r_scale).to(
        torch.bfloat16)
    k = torch.randn(B, Hkv, L, D, device="cuda", dtype=torch.bfloat16, generator=g)
    v = torch.randn(B, Hkv, L, D, device="cuda", dtype=torch.bfloat16, generator=g)
    return q, r, k, v


def scaled_error(got, ref):
    g = got.float().cpu().double().numpy()
    assert np.all(np.isfinite(g)), "non-finite output"
    return float(np.max(np.abs(g - ref) / np.maximum(1.0, np.abs(ref))))


@pytest.mark.parametrize("r_scale", [0.5, 1.0, 2.0])
@pytest.mark.parametrize("L", [1, 64, 200, 384])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2)])
def test_prefill_matches_oracle(L, D, Hq, Hkv, r_scale):
    q, r, k, v = make(2, Hq, Hkv, L, D, seed=300 + L + D + Hq, r_scale=r_scale)
    scale = D ** -0.5
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    for causal in (True, False):
        want = oracle.parallax_prefill(q, r, k, v, scale, causal)
        for out_dtype in (torch.bfloat16, torch.float32):
            got = binding.parallax_prefill(q, r, k, v, scale=scale, causal=causal,
                                           out_dtype=out_dtype, workspace=ws)
            err = scaled_error(got, want)
            assert err <= TOL[out_dtype], (L, D, Hq, Hkv, r_scale, causal, out_dtype, err)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0  # no device timeout


def test_prefill_r_zero_and_deterministic():
    q, r, k, v = make(1, 4, 4, 300, 128, seed=320)
    z = torch.zeros_like(r)
    want = oracle.parallax_prefill(q, z, k, v, 128 ** -0.5, True)
    a = binding.parallax_prefill(q, z, k, v, out_dtype=torch.float32)
    b = binding.parallax_prefill(q, z, k, v, out_dtype=torch.float32)
    assert torch.equal(a, b)
    assert scaled_error(a, want) <= 1e-4


@pytest.mark.parametrize("r_scale", [0.5, 1.0])
def test_prefill_full_size_sampled(r_scale):
    """The bench's prefill workload (Qwen-3 attention heads at the training
    length: B=4, Hq=16, Hkv=8, L=4096, D=128, the README's N(0,1) recipe, and
    r at half scale): two (batch, head) slices against the oracle, every
    output finite."""
    B, Hq, Hkv, L, D = 4, 16, 8, 4096, 128
    q, r, k, v = make(B, Hq, Hkv, L, D, seed=7, r_scale=r_scale)
    outs = {dt: binding.parallax_prefill(q, r, k, v, out_dtype=dt)
            for dt in (torch.bfloat16, torch.float32)}  # bf16: the bench's configuration
    for dt, got in outs.items():
        assert bool(torch.isfinite(got).all()), dt
    for b, h in ((0, 0), (3, 15)):
        g = h // (Hq // Hkv)
        sl = lambda t, i: t[b:b + 1, i:i + 1]
        want = oracle.parallax_prefill(sl(q, h), sl(r, h), sl(k, g), sl(v, g), D ** -0.5, True)
        for dt, got in outs.items():
            err = scaled_error(got[b:b + 1, h:h + 1], want)
            assert err <= TOL[dt], (b, h, dt, r_scale, err)
