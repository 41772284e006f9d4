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


def workspace(kind, B, L, Hkv, D):
    """'full': room for the fp16 copy of V (the fp16 value products with bf16
    output); 'header': the 256-byte status header only (every tile takes the
    bf16 hi + lo weights)."""
    if kind == "full":
        return binding.prefill_workspace(B, L, Hkv, D, "cuda")
    return torch.zeros(256, dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("ws_kind", ["full", "header"])
@pytest.mark.parametrize("r_scale", [0.5, 1.0, 2.0])
@pytest.mark.parametrize("L", [1, 64, 200, 384])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2)])
def test_prefill_matches_oracle(L, D, Hq, Hkv, r_scale, ws_kind):
    q, r, k, v = make(2, Hq, Hkv, L, D, seed=300 + L + D + Hq, r_scale=r_scale)
    scale = D ** -0.5
    ws = workspace(ws_kind, 2, L, Hkv, D)
    for causal in (True, False):
        want = oracle.parallax_prefill(q, r, k, v, scale, causal)
        for out_dtype in (torch.bfloat16, torch.float32):
            got = binding.parallax_prefill(q, r, k, v, scale=scale, causal=causal,
                                           out_dtype=out_dtype, workspace=ws)
            err = scaled_error(got, want)
            assert err <= TOL[out_dtype], (L, D, Hq, Hkv, r_scale, ws_kind, causal, out_dtype,
                                           err)
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


def row_scaled_error(got, ref):
    """Error of each output over the largest |ref| of its row (at least 1).
    With values of V in the hundreds of thousands the terms of
    o = A/l + C/l - (b/l)(A/l) are ~1e6 and cancel: any fp32 evaluation is
    off by units on the outputs of such a row that happen to be near zero,
    so their error is measured against the row's magnitude."""
    g = got.float().cpu().double().numpy()
    assert np.all(np.isfinite(g)), "non-finite output"
    scale = np.maximum(1.0, np.max(np.abs(ref), axis=-1, keepdims=True))
    return float(np.max(np.abs(g - ref) / scale))


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("case", ["v_over_2e16", "v_near_f16_max", "probe_bound", "probe_huge",
                                  "v_one_huge"])
def test_prefill_tiles_outside_fp16_range(case, D):
    """With bf16 output the value products take fp16 operands on tiles whose
    V and probe-score bounds fit fp16, and the exact bf16 hi + lo weights on
    the others; one sequence can mix both. Each case puts some tiles outside
    the fp16 bounds (or right at their edge) and checks the result against
    the oracle. A tile that took fp16 by mistake would turn V above 2^16
    into inf; a row whose e*s were not scaled down would overflow fp16."""
    B, Hq, Hkv, L = 1, 4, 2, 320
    q, r, k, v = make(B, Hq, Hkv, L, D, seed=340 + D)
    if case == "v_over_2e16":  # keys 64..127 of kv head 0 above fp16's range
        v[:, 0, 64:128] = (v[:, 0, 64:128].float() * 3e5).to(torch.bfloat16)
    elif case == "v_near_f16_max":  # in range, up to 65280 (exact in fp16)
        v[:, 1, 128:192] = (v[:, 1, 128:192].float().clamp(-1, 1) * 65280).to(torch.bfloat16)
    elif case == "probe_bound":  # |r|_1 max|k| above 2^14 for query heads 0 and 3: sigma > 0
        r[:, 0] = (r[:, 0].float() * 400).to(torch.bfloat16)
        r[:, 3] = (r[:, 3].float() * 400).to(torch.bfloat16)
    elif case == "probe_huge":  # |s| itself beyond fp16's range, on some rows of head 1
        r[:, 1, 100:140] = (r[:, 1, 100:140].float() * 2e4).to(torch.bfloat16)
    else:  # one value just above fp16's range (inf in fp16) in the middle of a tile
        # (not far above it: on the bf16 hi + lo path a weight's rounding error times
        # that value is the error, which a row whose weight nearly cancels does not
        # dwarf; the check here is on the tile's decision)
        v[:, 1, 200, 5] = 8e4
    want = oracle.parallax_prefill(q, r, k, v, D ** -0.5, True)
    got = binding.parallax_prefill(q, r, k, v, out_dtype=torch.bfloat16)
    assert row_scaled_error(got, want) <= TOL[torch.bfloat16], (case, D)


def test_prefill_workspace_one_byte_short_takes_the_exact_weights():
    """A workspace one byte smaller than parallax_prefill_workspace_bytes holds
    no fp16 copy of V: every tile takes the bf16 hi + lo weights, and the call
    matches the oracle within the fp32-accurate weights' error (well inside the
    bf16 output's bound), as does the full workspace."""
    B, Hq, Hkv, L, D = 1, 4, 2, 200, 128
    q, r, k, v = make(B, Hq, Hkv, L, D, seed=350)
    want = oracle.parallax_prefill(q, r, k, v, D ** -0.5, True)
    n = binding.parallax_prefill_workspace_bytes(B, L, Hkv, D)
    for size in (n - 1, n):
        ws = torch.zeros(size, dtype=torch.uint8, device="cuda")
        got = binding.parallax_prefill(q, r, k, v, out_dtype=torch.bfloat16, workspace=ws)
        assert scaled_error(got, want) <= TOL[torch.bfloat16], size
        torch.cuda.synchronize()
        assert int(ws[:4].view(torch.int32).item()) == 0


def _expected_records(k, v, items_rows):
    """Per (kv item, 64-row block): bits 0-15 the largest |k| as bf16 bits,
    bit 16 set when every |v| is below 2^16 (a bf16 magnitude below 0x4780).
    `items_rows` gives each item's rows as [rows, D] views."""
    out = []
    for kk, vv in items_rows(k, v):
        kb = kk.contiguous().view(torch.int16).to(torch.int32) & 0x7FFF
        vb = vv.contiguous().view(torch.int16).to(torch.int32) & 0x7FFF
        rows = kb.shape[0]
        for b0 in range(0, rows, 64):
            km = int(kb[b0:b0 + 64].max())
            ok = int(vb[b0:b0 + 64].max()) < 0x4780
            out.append(km | (0x10000 if ok else 0))
    return out


@pytest.mark.parametrize("layout", ["dense", "packed"])
@pytest.mark.parametrize("D", [64, 128])
def test_prefill_prep_copy_and_records_are_exact(layout, D):
    """The kernel launched before a bf16-output prefill writes, from byte 1024
    of the workspace, V converted to fp16 (round to nearest even, inf at and
    above 65520: the conversion torch performs) and, 256-byte aligned after
    it, one 32-bit record per (kv item, 64-row block). Both are checked bit
    for bit, on a V with one block out of fp16's range."""
    Hq, Hkv = 4, 2
    if layout == "dense":
        B, L = 2, 200
        q, r, k, v = make(B, Hq, Hkv, L, D, seed=360 + D)
        v[1, 0, 70, 3] = 7e4  # item 2 (b = 1, g = 0), block 1
        rows, items = L, B * Hkv
        binding.parallax_prefill(q, r, k, v, out_dtype=torch.bfloat16,
                                 workspace=(ws := binding.prefill_workspace(B, L, Hkv, D, "cuda")))
        per_item = lambda kk, vv: [(kk[b, g], vv[b, g]) for b in range(B) for g in range(Hkv)]
        v_elems = v.numel()
    else:
        lens = [130, 7, 200]
        q, r, k, v, cu = _packed(lens, Hq, Hkv, D, seed=370 + D)
        v[135, 1, 2] = -7e4  # head 1, packed row 135: block 2
        rows, items = sum(lens), Hkv
        ws = binding.prefill_workspace(1, rows, Hkv, D, "cuda")
        binding.parallax_varlen_prefill(q, r, k, v, cu, max(lens), out_dtype=torch.bfloat16,
                                        workspace=ws)
        per_item = lambda kk, vv: [(kk[:, g], vv[:, g]) for g in range(Hkv)]
        v_elems = v.numel()
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    copy = ws[1024:1024 + 2 * v_elems].view(torch.float16).view(v.shape)
    want = v.float().to(torch.float16)
    assert torch.equal(copy.view(torch.int16), want.view(torch.int16))
    info_off = 1024 + (2 * v_elems + 255) // 256 * 256
    nblk = (rows + 63) // 64
    rec = ws[info_off:info_off + 4 * items * nblk].view(torch.int32).cpu().tolist()
    assert rec == _expected_records(k.cpu(), v.cpu(), per_item)
    assert sum(1 for x in rec if not x & 0x10000) == 1  # the one out-of-range block


def _packed(lens, Hq, Hkv, D, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    total = int(sum(lens))
    rnd = lambda H: torch.randn(total, H, D, device="cuda", generator=g).to(torch.bfloat16)
    q, r, k, v = rnd(Hq), rnd(Hq), rnd(Hkv), rnd(Hkv)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    return q, r, k, v, cu
