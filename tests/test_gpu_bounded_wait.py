"""Failure detection without a GPU fault: the split-KV kernel's waits are
bounded. A testing hook tells the producer never to fill a CTA's first
pipeline stage, so the consumers' wait on it runs out (50 ms here); the kernel
must record PARALLAX_DEVICE_STATUS_TIMEOUT and return, and the same CUDA
context must then run a normal decode correctly."""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle
from parameterized_local_linear_b200 import binding, inputs

pytestmark = pytest.mark.gpu

TIMEOUT_BIT, ERR_DEVICE_TIMEOUT = 1, -9


def test_bounded_wait_gives_up_and_context_survives():
    assert torch.cuda.is_available()
    lib = binding.load_library()
    fn = lib.parallax_testing_decode_stalled
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp] * 6 + [i] * 4 + [ctypes.c_float, vp, i, i, vp, ctypes.c_size_t, i]
    fn.restype = i
    w = inputs.custom_workload("stall", B=2, Hq=16, Hkv=8, D=128, Lmax=512, seed=31)
    x = inputs.make_inputs(w, device="cuda")
    ws = binding.Workspace(2, 16, 8, 128, 512, num_splits=4)
    out = torch.empty((2, 16, 128), device="cuda", dtype=torch.bfloat16)
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.perf_counter()
    rc = fn(x["q"].data_ptr(), x["r"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(),
            x["seqlens"].data_ptr(), out.data_ptr(), 2, 16, 8, 128, x["scale"], stream, 512, 4,
            ws.ptr(), ws.nbytes, 50)
    assert rc == 0
    status, bits = ws.status(clear=True)  # synchronises
    elapsed = time.perf_counter() - t0
    assert bits & TIMEOUT_BIT and status == ERR_DEVICE_TIMEOUT
    assert elapsed < 5.0, f"the stalled call took {elapsed:.2f} s"
    assert ws.status() == (0, 0)

    # the context is intact: a normal decode afterwards matches the oracle
    got = binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"], scale=x["scale"],
                                  out_dtype=torch.float32, num_splits=4, workspace=ws)
    ref = oracle.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"], x["scale"])
    g = got.double().cpu().numpy()
    assert np.all(np.isfinite(g))
    assert np.max(np.abs(g - ref) / np.maximum(1.0, np.abs(ref))) <= 1e-4
    assert ws.status() == (0, 0)


@pytest.mark.parametrize("ws_kind", ["header", "full"])
def test_prefill_bounded_wait_gives_up_and_context_survives(ws_kind):
    """The tcgen05 prefill: the producer never loads a CTA's first K tile, so
    the UMMA issuer's wait runs out (50 ms); every CTA must record the timeout,
    drain its own copies, free its tensor memory and return, and a normal
    prefill on the same context (which allocates tensor memory again on every
    SM) must then match the oracle. 'full': with the workspace for the fp16
    copy of V, so the stalled launch follows the copy kernel."""
    lib = binding.load_library()
    fn = lib.parallax_testing_prefill_stalled
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp] * 5 + [i] * 5 + [ctypes.c_float, i, vp, i, vp, ctypes.c_size_t, i]
    fn.restype = i
    B, Hq, Hkv, L, D = 2, 4, 2, 300, 128
    g = torch.Generator(device="cuda").manual_seed(33)
    mk = lambda H, sc=1.0: (torch.randn(B, H, L, D, device="cuda", generator=g) * sc).to(
        torch.bfloat16)
    q, r, k, v = mk(Hq), mk(Hq, 0.5), mk(Hkv), mk(Hkv)
    out = torch.empty_like(q)
    ws = (binding.prefill_workspace(B, L, Hkv, D, "cuda") if ws_kind == "full"
          else torch.zeros(256, dtype=torch.uint8, device="cuda"))
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.perf_counter()
    rc = fn(q.data_ptr(), r.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hq, Hkv, L,
            D, D ** -0.5, 1, stream, 0, ws.data_ptr(), ws.numel(), 50)
    assert rc == 0
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    bits = int(ws[:4].view(torch.int32).item())
    assert bits & TIMEOUT_BIT, bits
    assert elapsed < 5.0, f"the stalled call took {elapsed:.2f} s"
    ws[:256].zero_()
    got = binding.parallax_prefill(q, r, k, v, out_dtype=torch.float32, workspace=ws)
    want = oracle.parallax_prefill(q, r, k, v, D ** -0.5, True)
    gg = got.double().cpu().numpy()
    assert np.all(np.isfinite(gg))
    assert np.max(np.abs(gg - want) / np.maximum(1.0, np.abs(want))) <= 1e-4
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
