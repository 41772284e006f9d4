"""parallax_decode_noalloc: the decode entry point for callers that cannot
allocate device memory (a plugin or host program next to a framework whose
pool already holds the GPU's memory, or a decode loop that must not call
cudaMalloc). It uses a fixed array inside the library instead of a caller
workspace. Checked through the C ABI against parallax_decode, two calls in a
row (the array keeps the previous call's contents), plus its size limit.

Kept in its own file, named to be collected last."""
import ctypes

import numpy as np
import pytest
import torch

from parameterized_local_linear_b200 import binding, inputs

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = -12


def _lib():
    lib = binding.load_library()
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.parallax_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, f, vp, i, i, i, i]
    lib.parallax_decode_noalloc.restype = i
    return lib


def _call(lib, x, out, num_splits=0, stream=None):
    B, Hq, D = x["q"].shape
    _, Hkv, Lmax, _ = x["k"].shape
    s = torch.cuda.current_stream().cuda_stream if stream is None else stream
    return lib.parallax_decode_noalloc(
        x["q"].data_ptr(), x["r"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(),
        x["seqlens"].data_ptr(), out.data_ptr(), B, Hq, Hkv, D, float(x["scale"]), s, Lmax,
        0, 1 if out.dtype == torch.float32 else 0, num_splits)


def _scaled_err(got, ref):
    g = got.float().cpu().double().numpy()
    r = ref.float().cpu().double().numpy()
    assert np.all(np.isfinite(g))
    return float(np.max(np.abs(g - r) / np.maximum(1.0, np.abs(r))))


@pytest.mark.parametrize("out_dtype,tol", [(torch.bfloat16, 2e-2), (torch.float32, 1e-4)])
def test_noalloc_matches_decode_twice(out_dtype, tol):
    assert torch.cuda.is_available()
    lib = _lib()
    w = inputs.custom_workload("noalloc", B=4, Hq=16, Hkv=8, D=128, Lmax=3000,
                               lengths=(3000, 1, 777, 2048), seed=21, r_scale=0.5)
    x = inputs.make_inputs(w, device="cuda")
    ref = binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"],
                                  scale=x["scale"], out_dtype=out_dtype)
    for _ in range(2):  # the second call starts from the first call's leftovers
        out = torch.full_like(ref, float("nan"))
        assert _call(lib, x, out) == 0
        torch.cuda.synchronize()
        assert _scaled_err(out, ref) <= tol


def test_noalloc_rejects_oversized_split_counts():
    lib = _lib()
    w = inputs.custom_workload("noalloc_big", B=2, Hq=16, Hkv=8, D=128, Lmax=256, seed=22)
    x = inputs.make_inputs(w, device="cuda")
    out = torch.empty((2, 16, 128), device="cuda", dtype=torch.bfloat16)
    assert _call(lib, x, out, num_splits=5000) == SCRATCH_LIMIT
    assert "NOALLOC" in binding.parallax_status_string(SCRATCH_LIMIT)
    assert _call(lib, x, out, num_splits=1008) == 0  # the largest that fits at G = 2
    torch.cuda.synchronize()
