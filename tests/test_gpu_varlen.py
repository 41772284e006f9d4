"""GPU parity of the packed variable-length forward (the README's
parallax_varlen_func, "Training (dense + varlen)") against the fp64 oracle:
ragged sequences that span several 128-row query tiles and partial 64-key
tiles, an empty sequence, GQA, both head dimensions, causal and not, bf16 and
fp32 outputs, plus the device-side clamping of malformed cu_seqlens."""
import numpy as np
import pytest
import torch

import oracle
from parameterized_local_linear_b200 import binding

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}


def make(lens, Hq, Hkv, D, seed, r_scale=1.0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    total = int(sum(lens))
    rnd = lambda H, s=1.0: (torch.randn(total, H, D, device="cuda", generator=g) * s).to(torch.bfloat16)
    q, r, k, v = rnd(Hq), rnd(Hq, r_scale), rnd(Hkv), rnd(Hkv)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    return q, r, k, v, cu


def status_bits(ws):
    """The device status word (first 4 bytes of the workspace), then cleared."""
    torch.cuda.synchronize()
    bits = int(ws[:4].view(torch.int32).item())
    ws.zero_()
    return bits


def scaled_error(got, ref):
    g = got.float().cpu().double().numpy()
    assert np.all(np.isfinite(g)), "non-finite output"
    return float(np.max(np.abs(g - ref) / np.maximum(1.0, np.abs(ref))))


@pytest.mark.parametrize("ws_kind", ["full", "header"])
@pytest.mark.parametrize("r_scale", [0.5, 1.0, 2.0])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2)])
def test_varlen_matches_oracle(D, Hq, Hkv, r_scale, ws_kind):
    """'full': a workspace with room for the fp16 copy of V (fp16 value
    products on in-range tiles, bf16 output); 'header': the status header only."""
    lens = [1, 130, 64, 0, 257, 5, 128]
    q, r, k, v, cu = make(lens, Hq, Hkv, D, seed=400 + D + Hq, r_scale=r_scale)
    scale = D ** -0.5
    ws = (binding.prefill_workspace(1, sum(lens), Hkv, D, "cuda") if ws_kind == "full"
          else torch.zeros(256, dtype=torch.uint8, device="cuda"))
    for causal in (True, False):
        want = oracle.parallax_varlen_prefill(q, r, k, v, cu, scale, causal)
        for out_dtype in (torch.bfloat16, torch.float32):
            got = binding.parallax_varlen_prefill(q, r, k, v, cu, max(lens), scale=scale,
                                                  causal=causal, out_dtype=out_dtype, workspace=ws)
            err = scaled_error(got, want)
            assert err <= TOL[out_dtype], (D, Hq, Hkv, r_scale, ws_kind, causal, out_dtype, err)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0


def test_varlen_equal_lengths_match_dense_kernel():
    B, Hq, Hkv, L, D = 3, 4, 2, 200, 128
    g = torch.Generator(device="cuda").manual_seed(410)
    mk = lambda H: torch.randn(B, H, L, D, device="cuda", generator=g).to(torch.bfloat16)
    q, r, k, v = mk(Hq), mk(Hq), mk(Hkv), mk(Hkv)
    dense = binding.parallax_prefill(q, r, k, v, out_dtype=torch.float32)
    pack = lambda x: x.transpose(1, 2).reshape(B * L, x.shape[1], D).contiguous()
    cu = torch.arange(0, B * L + 1, L, dtype=torch.int32, device="cuda")
    got = binding.parallax_varlen_prefill(pack(q), pack(r), pack(k), pack(v), cu,
                                          out_dtype=torch.float32)
    # same tiles, same arithmetic: identical bits
    assert torch.equal(got, pack(dense))


def test_varlen_malformed_lengths_are_clamped():
    lens = [50, 70]
    q, r, k, v, cu = make(lens, 2, 2, 64, seed=420)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    out = torch.full_like(q, 7.0)
    bad = torch.tensor([0, 90, 60], dtype=torch.int32, device="cuda")  # decreasing pair
    binding.parallax_varlen_prefill(q, r, k, v, bad, 90, out=out, workspace=ws)
    assert status_bits(ws) & 2
    # the first sequence (rows 0..89) is computed; the clamped-empty second
    # sequence writes nothing
    want = oracle.parallax_varlen_prefill(q[:90], r[:90], k[:90], v[:90],
                                          np.array([0, 90]), 64 ** -0.5)
    assert scaled_error(out[:90], want) <= 2e-2
    assert torch.all(out[90:] == 7.0)
    # a max_seqlen that leaves a sequence's query tiles out is flagged too
    q, r, k, v, cu = make([50, 200], 2, 2, 64, seed=421)
    binding.parallax_varlen_prefill(q, r, k, v, cu, 100, workspace=ws)
    assert status_bits(ws) & 2
    binding.parallax_varlen_prefill(q, r, k, v, cu, 200, workspace=ws)
    assert status_bits(ws) == 0


def test_varlen_full_size_sampled():
    """The bench's varlen workload (16 sequences of lengths U{1..4096}, Hq=16,
    Hkv=8, D=128): the shortest and the longest sequence, one head each,
    against the oracle."""
    lens = torch.randint(1, 4097, (16,), generator=torch.Generator().manual_seed(11)).tolist()
    q, r, k, v, cu = make(lens, 16, 8, 128, seed=430)
    got = binding.parallax_varlen_prefill(q, r, k, v, cu, max(lens), out_dtype=torch.float32)
    assert bool(torch.isfinite(got).all())
    cuh = cu.cpu().tolist()
    for s in (int(np.argmin(lens)), int(np.argmax(lens))):
        a, e = cuh[s], cuh[s + 1]
        for h in (0, 13):
            g = h // 2
            want = oracle.parallax_varlen_prefill(q[a:e, h:h + 1], r[a:e, h:h + 1],
                                                  k[a:e, g:g + 1], v[a:e, g:g + 1],
                                                  np.array([0, e - a]), 128 ** -0.5)
            err = scaled_error(got[a:e, h:h + 1], want)
            assert err <= TOL[torch.float32], (s, h, err)


def row_scaled_error(got, ref):
    """Error over the largest |ref| of the row (at least 1): with values of V
    in the hundreds of thousands, any fp32 evaluation of o is off by units on
    outputs that happen to be near zero."""
    g = got.float().cpu().double().numpy()
    assert np.all(np.isfinite(g)), "non-finite output"
    return float(np.max(np.abs(g - ref) / np.maximum(1.0, np.max(np.abs(ref), -1, keepdims=True))))


@pytest.mark.parametrize("D", [64, 128])
def test_varlen_neighbour_rows_outside_fp16_range(D):
    """A tile's K/V box can reach into the next sequence's rows, which are
    masked (weight 0) but still multiplied. Here the second sequence's first
    rows hold V above fp16's range: the first sequence's last tile, whose box
    covers them, must not take the fp16 copy (inf times 0 would be NaN), and
    the second sequence itself runs its first tile on the bf16 weights."""
    lens = [100, 90, 200]
    q, r, k, v, cu = make(lens, 4, 2, D, seed=460)
    v[100:110] = (v[100:110].float() * 3e5).to(torch.bfloat16)  # rows 0..9 of sequence 1
    want = oracle.parallax_varlen_prefill(q, r, k, v, cu, D ** -0.5, True)
    ws = binding.prefill_workspace(1, sum(lens), 2, D, "cuda")
    got = binding.parallax_varlen_prefill(q, r, k, v, cu, max(lens), workspace=ws)
    assert row_scaled_error(got, want) <= TOL[torch.bfloat16]
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
