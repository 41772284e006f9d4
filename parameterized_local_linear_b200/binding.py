"""ctypes binding of libparallax.so (include/parallax.h), same entry-point names.

Argument marshalling only: shapes are read off the torch tensors, pointers
and the current CUDA stream are passed through, and a non-zero status raises.
Every step of the decode runs in the library's CUDA kernels; there is no
other implementation behind these functions. If the library is not built or
no CUDA device is present, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import build as _build

BF16, F32 = 0, 1
_DTYPE_CODE = {torch.bfloat16: BF16, torch.float32: F32}
_CODE_DTYPE = {BF16: torch.bfloat16, F32: torch.float32}

_lib = None


def library_path() -> str:
    return _build.LIB


def load_library():
    """Load libparallax.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m parameterized_local_linear_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    decode_tail = [i, i, i, i, f, vp, i, i, i, i, vp, sz]
    lib.parallax_decode.argtypes = [vp, vp, vp, vp, vp, vp] + decode_tail
    lib.parallax_softmax_decode.argtypes = [vp, vp, vp, vp, vp] + decode_tail
    lib.parallax_decode_phase.argtypes = [i, i, vp, vp, vp, vp, vp, vp] + decode_tail
    lib.parallax_decode_workspace_bytes.argtypes = [i, i, i, i, i, i]
    lib.parallax_decode_workspace_bytes.restype = sz
    lib.parallax_choose_splits.argtypes = [i, i, i, i]
    lib.parallax_workspace_status.argtypes = [vp, i, ctypes.POINTER(ctypes.c_uint32)]
    lib.parallax_status_string.argtypes = [i]
    lib.parallax_status_string.restype = ctypes.c_char_p
    for fn in (lib.parallax_decode, lib.parallax_softmax_decode, lib.parallax_decode_phase,
               lib.parallax_choose_splits, lib.parallax_workspace_status):
        fn.restype = i
    _lib = lib
    return lib


def parallax_status_string(status: int) -> str:
    return load_library().parallax_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != 0:
        raise RuntimeError(f"{what} failed: {parallax_status_string(status)} (status {status})")


def parallax_choose_splits(B: int, Hkv: int, Lmax: int, sm_count: int = 0) -> int:
    n = load_library().parallax_choose_splits(B, Hkv, Lmax, sm_count)
    if n < 0:
        _check(n, "parallax_choose_splits")
    return n


def parallax_decode_workspace_bytes(B: int, Hq: int, Hkv: int, D: int, Lmax: int,
                                    num_splits: int = 0) -> int:
    n = load_library().parallax_decode_workspace_bytes(B, Hq, Hkv, D, Lmax, num_splits)
    if n == 0:
        raise RuntimeError("parallax_decode_workspace_bytes: invalid arguments")
    return int(n)


class Workspace:
    """Caller-owned scratch for the decode calls (zero-filled once, as the
    status word at its start requires)."""

    def __init__(self, B, Hq, Hkv, D, Lmax, num_splits=0, device=None):
        self.nbytes = parallax_decode_workspace_bytes(B, Hq, Hkv, D, Lmax, num_splits)
        self.buffer = torch.zeros(self.nbytes, dtype=torch.uint8,
                                  device=device if device is not None else "cuda")

    def ptr(self) -> int:
        return self.buffer.data_ptr()

    def status(self, clear: bool = False):
        """(status code, device status bits); synchronises the device."""
        torch.cuda.synchronize(self.buffer.device)
        word = ctypes.c_uint32(0)
        rc = load_library().parallax_workspace_status(ctypes.c_void_p(self.ptr()), int(clear),
                                                      ctypes.byref(word))
        return rc, word.value


def parallax_workspace_status(workspace: Workspace, clear: bool = False):
    return workspace.status(clear)


def _shapes(q, k_cache, v_cache, cache_seqlens):
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                    ("cache_seqlens", cache_seqlens)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if q.dim() != 3 or k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("expected q [B,Hq,D] and k_cache, v_cache [B,Hkv,Lmax,D]")
    if cache_seqlens.dtype != torch.int32 or cache_seqlens.shape != (q.shape[0],):
        raise ValueError("cache_seqlens must be int32 [B]")
    if k_cache.dtype != q.dtype or v_cache.dtype != q.dtype or q.dtype not in _DTYPE_CODE:
        raise ValueError("q, r, k_cache, v_cache must share one dtype (bf16 or fp32)")
    B, Hq, D = q.shape
    Bk, Hkv, Lmax, Dk = k_cache.shape
    if Bk != B or Dk != D:
        raise ValueError("k_cache shape does not match q")
    return B, Hq, Hkv, D, Lmax


def _prepare(q, k_cache, v_cache, cache_seqlens, out, out_dtype, workspace, num_splits):
    B, Hq, Hkv, D, Lmax = _shapes(q, k_cache, v_cache, cache_seqlens)
    if out is None:
        out = torch.empty((B, Hq, D), device=q.device,
                          dtype=out_dtype if out_dtype is not None else q.dtype)
    if out.shape != (B, Hq, D) or not out.is_contiguous() or out.dtype not in _DTYPE_CODE:
        raise ValueError("out must be a contiguous [B,Hq,D] bf16 or fp32 tensor")
    if workspace is None:
        workspace = Workspace(B, Hq, Hkv, D, Lmax, num_splits, device=q.device)
    return B, Hq, Hkv, D, Lmax, out, workspace


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def parallax_decode(q, r, k_cache, v_cache, cache_seqlens, scale: Optional[float] = None,
                    out=None, out_dtype=None, num_splits: int = 0,
                    workspace: Optional[Workspace] = None, stream=None):
    """Parallax decode: out[b,h] = vbar + C/l - (b/l) vbar over the cached keys."""
    B, Hq, Hkv, D, Lmax, out, workspace = _prepare(q, k_cache, v_cache, cache_seqlens, out,
                                                   out_dtype, workspace, num_splits)
    if r.shape != q.shape or r.dtype != q.dtype or not r.is_cuda or not r.is_contiguous():
        raise ValueError("r must be a contiguous CUDA tensor shaped like q")
    scale = D ** -0.5 if scale is None else scale
    rc = load_library().parallax_decode(
        q.data_ptr(), r.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
        cache_seqlens.data_ptr(), out.data_ptr(), B, Hq, Hkv, D, float(scale),
        _stream(stream), Lmax, _DTYPE_CODE[q.dtype], _DTYPE_CODE[out.dtype], int(num_splits),
        workspace.ptr(), workspace.nbytes)
    _check(rc, "parallax_decode")
    return out


def parallax_softmax_decode(q, k_cache, v_cache, cache_seqlens, scale: Optional[float] = None,
                            out=None, out_dtype=None, num_splits: int = 0,
                            workspace: Optional[Workspace] = None, stream=None):
    """The R = 0 comparator: softmax attention decode on the same pipeline."""
    B, Hq, Hkv, D, Lmax, out, workspace = _prepare(q, k_cache, v_cache, cache_seqlens, out,
                                                   out_dtype, workspace, num_splits)
    scale = D ** -0.5 if scale is None else scale
    rc = load_library().parallax_softmax_decode(
        q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), cache_seqlens.data_ptr(),
        out.data_ptr(), B, Hq, Hkv, D, float(scale), _stream(stream), Lmax,
        _DTYPE_CODE[q.dtype], _DTYPE_CODE[out.dtype], int(num_splits), workspace.ptr(),
        workspace.nbytes)
    _check(rc, "parallax_softmax_decode")
    return out


def parallax_decode_phase(phase: int, probe: bool, q, r, k_cache, v_cache, cache_seqlens,
                          out, workspace: Workspace, scale: Optional[float] = None,
                          num_splits: int = 0, stream=None):
    """Run only the split-KV kernel (phase 1) or only the merge kernel (phase 2)."""
    B, Hq, Hkv, D, Lmax, out, workspace = _prepare(q, k_cache, v_cache, cache_seqlens, out,
                                                   None, workspace, num_splits)
    scale = D ** -0.5 if scale is None else scale
    rc = load_library().parallax_decode_phase(
        int(phase), int(bool(probe)), q.data_ptr(), r.data_ptr() if r is not None else None,
        k_cache.data_ptr(), v_cache.data_ptr(), cache_seqlens.data_ptr(), out.data_ptr(),
        B, Hq, Hkv, D, float(scale), _stream(stream), Lmax, _DTYPE_CODE[q.dtype],
        _DTYPE_CODE[out.dtype], int(num_splits), workspace.ptr(), workspace.nbytes)
    _check(rc, "parallax_decode_phase")
    return out


def parallax_decode_noalloc(q, r, k_cache, v_cache, cache_seqlens, scale: Optional[float] = None,
                            out=None, out_dtype=None, num_splits: int = 0, stream=None):
    """parallax_decode without a caller workspace, for callers that cannot
    allocate device memory: the library uses its own fixed device array (see
    include/parallax.h). Calls that can overlap on the GPU race on it."""
    lib = load_library()
    fn = lib.parallax_decode_noalloc
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fn.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, f, vp, i, i, i, i]
    fn.restype = i
    B, Hq, Hkv, D, Lmax = _shapes(q, k_cache, v_cache, cache_seqlens)
    if out is None:
        out = torch.empty((B, Hq, D), device=q.device,
                          dtype=out_dtype if out_dtype is not None else q.dtype)
    if r.shape != q.shape or r.dtype != q.dtype or not r.is_cuda or not r.is_contiguous():
        raise ValueError("r must be a contiguous CUDA tensor shaped like q")
    scale = D ** -0.5 if scale is None else scale
    rc = fn(q.data_ptr(), r.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
            cache_seqlens.data_ptr(), out.data_ptr(), B, Hq, Hkv, D, float(scale),
            _stream(stream), Lmax, _DTYPE_CODE[q.dtype], _DTYPE_CODE[out.dtype], int(num_splits))
    _check(rc, "parallax_decode_noalloc")
    return out
