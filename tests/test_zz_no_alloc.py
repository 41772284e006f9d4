"""parallax_decode_noalloc: the decode entry point for callers that cannot
allocate device memory (a plugin or host program next to a framework whose
pool already holds the GPU's memory, or a decode loop that must not call
cudaMalloc). It uses a fixed array inside the library instead of a caller
workspace.

Checked through the C ABI:
- against parallax_decode at the same split count, two calls in a row (the
  array keeps the previous call's contents). The two run the same kernels on
  the same partition, so the outputs must be bit-identical;
- one call against the fp64 oracle, within the decode tolerances;
- default calls (num_splits = 0) with 8 and 16 query heads per kv head,
  whose default count the array can only hold once it is capped;
- its size limit for explicit split counts.

Kept in its own file, named to be collected last."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
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
    r = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(g))
    return float(np.max(np.abs(g - r) / np.maximum(1.0, np.abs(r))))


@pytest.mark.parametrize("out_dtype,tol", [(torch.bfloat16, 2e-2), (torch.float32, 1e-4)])
def test_noalloc_equals_decode_twice_and_matches_oracle(out_dtype, tol):
    assert torch.cuda.is_available()
    lib = _lib()
    w = inputs.custom_workload("noalloc", B=4, Hq=16, Hkv=8, D=128, Lmax=3000,
                               lengths=(3000, 1, 777, 2048), seed=21, r_scale=0.5)
    x = inputs.make_inputs(w, device="cuda")
    P = binding.parallax_default_splits(w.B, w.Hq, w.Hkv, w.Lmax, w.dtype)
    ref = binding.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"],
                                  scale=x["scale"], out_dtype=out_dtype, num_splits=P)
    for _ in range(2):  # the second call starts from the first call's leftovers
        out = torch.full_like(ref, float("nan"))
        assert _call(lib, x, out, num_splits=P) == 0
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    want = oracle.parallax_decode(x["q"].cpu(), x["r"].cpu(), x["k"].cpu(), x["v"].cpu(),
                                  x["seqlens"].cpu(), x["scale"])
    assert _scaled_err(out, want) <= tol


@pytest.mark.parametrize("Hq,Hkv", [(16, 2), (32, 2)])
def test_noalloc_default_count_fits_large_groups(Hq, Hkv):
    """8 and 16 query heads per kv head at D = 128: the array holds 252 and
    126 partitions, and a default call must fit without an explicit count."""
    lib = _lib()
    w = inputs.custom_workload("noalloc_group", B=3, Hq=Hq, Hkv=Hkv, D=128, Lmax=2500,
                               lengths=(2500, 64, 1300), seed=23, r_scale=0.5)
    x = inputs.make_inputs(w, device="cuda")
    out = torch.full((w.B, w.Hq, w.D), float("nan"), device="cuda", dtype=torch.float32)
    assert _call(lib, x, out) == 0
    torch.cuda.synchronize()
    want = oracle.parallax_decode(x["q"].cpu(), x["r"].cpu(), x["k"].cpu(), x["v"].cpu(),
                                  x["seqlens"].cpu(), x["scale"])
    assert _scaled_err(out, want) <= 1e-4


def test_noalloc_rejects_oversized_split_counts():
    lib = _lib()
    w = inputs.custom_workload("noalloc_big", B=2, Hq=16, Hkv=8, D=128, Lmax=256, seed=22)
    x = inputs.make_inputs(w, device="cuda")
    out = torch.empty((2, 16, 128), device="cuda", dtype=torch.bfloat16)
    assert _call(lib, x, out, num_splits=5000) == SCRATCH_LIMIT
    assert "NOALLOC" in binding.parallax_status_string(SCRATCH_LIMIT)
    assert _call(lib, x, out, num_splits=1008) == 0  # the largest that fits at G = 2
    torch.cuda.synchronize()
