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
    lib.parallax_decode_ex.argtypes = [vp, vp, vp, vp, vp, vp] + decode_tail + [i, i, i, i]
    lib.parallax_decode_paged.argtypes = [vp] * 7 + [i, i, i, i, f, vp, i, i, i, i, i, i, i, vp,
                                                     sz]
    lib.parallax_decode_block_sparse.argtypes = ([vp] * 8 + [i, i, i, i, f, vp, i, i, i, i, i, i,
                                                             i, vp, sz])
    lib.parallax_decode_workspace_bytes.argtypes = [i, i, i, i, i, i]
    lib.parallax_decode_workspace_bytes.restype = sz
    lib.parallax_choose_splits.argtypes = [i, i, i, i]
    lib.parallax_workspace_status.argtypes = [vp, i, ctypes.POINTER(ctypes.c_uint32)]
    lib.parallax_status_string.argtypes = [i]
    lib.parallax_status_string.restype = ctypes.c_char_p
    for fn in (lib.parallax_decode, lib.parallax_softmax_decode, lib.parallax_decode_phase,
               lib.parallax_decode_ex, lib.parallax_choose_splits, lib.parallax_decode_paged,
               lib.parallax_decode_block_sparse,
               lib.parallax_workspace_status):
        fn.restype = i
    _lib = lib
    return lib


def parallax_status_string(status: int) -> str:
    return load_library().parallax_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != 0:
        raise RuntimeError(f"{what} failed: {parallax_status_string(status)} (status {status})")


def parallax_varlen_prefill(q, r, k, v, cu_seqlens, max_seqlen: Optional[int] = None,
                            scale: Optional[float] = None, causal: bool = True, out=None,
                            out_dtype=None, workspace=None, stream=None):
    """Packed variable-length forward (the README's parallax_varlen_func):
    q, r [total, Hq, D], k, v [total, Hkv, D] bf16, cu_seqlens int32 [B + 1] on
    the device; sequence b is rows cu_seqlens[b]:cu_seqlens[b+1]."""
    lib = load_library()
    fn = lib.parallax_varlen_prefill
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fn.argtypes = [vp] * 6 + [i] * 6 + [f, i, vp, i, vp, ctypes.c_size_t]
    fn.restype = i
    for name, t in (("q", q), ("r", r), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != torch.bfloat16 or t.dim() != 3:
            raise ValueError(f"{name} must be a contiguous 3-D bf16 CUDA tensor")
    total, Hq, D = q.shape
    if r.shape != q.shape or k.shape != v.shape or k.shape[0] != total or k.shape[2] != D:
        raise ValueError("expected q, r [total, Hq, D] and k, v [total, Hkv, D]")
    if (not cu_seqlens.is_cuda or cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1
            or not cu_seqlens.is_contiguous()):
        raise ValueError("cu_seqlens must be a contiguous 1-D int32 CUDA tensor")
    B = cu_seqlens.numel() - 1
    if max_seqlen is None:  # one device read; pass it to stay asynchronous
        max_seqlen = int((cu_seqlens[1:] - cu_seqlens[:-1]).max().item()) if B > 0 else 0
    if out is None:
        out = torch.empty_like(q, dtype=out_dtype if out_dtype is not None else q.dtype)
    if workspace is None:
        workspace = prefill_workspace(1, total, k.shape[1], D, q.device)
    buf = workspace.buffer if isinstance(workspace, Workspace) else workspace
    scale = D ** -0.5 if scale is None else scale
    rc = fn(q.data_ptr(), r.data_ptr(), k.data_ptr(), v.data_ptr(), cu_seqlens.data_ptr(),
            out.data_ptr(), B, total, int(max_seqlen), Hq, k.shape[1], D, float(scale),
            int(bool(causal)), _stream(stream), _DTYPE_CODE[out.dtype], buf.data_ptr(),
            buf.numel())
    _check(rc, "parallax_varlen_prefill")
    return out


def parallax_choose_splits(B: int, Hkv: int, Lmax: int, sm_count: int = 0) -> int:
    n = load_library().parallax_choose_splits(B, Hkv, Lmax, sm_count)
    if n < 0:
        _check(n, "parallax_choose_splits")
    return n


def parallax_default_splits(B: int, Hq: int, Hkv: int, Lmax: int, dtype=torch.bfloat16,
                            probe: bool = True, sm_count: int = 0) -> int:
    """The partition count a decode call with num_splits=0 uses for these
    shapes, input dtype and probe setting."""
    fn = load_library().parallax_default_splits
    fn.argtypes = [ctypes.c_int] * 7
    fn.restype = ctypes.c_int
    n = fn(B, Hq, Hkv, Lmax, _DTYPE_CODE[dtype], int(bool(probe)), sm_count)
    if n < 1:
        raise RuntimeError(f"parallax_default_splits failed: {parallax_status_string(n)}")
    return n


def parallax_decode_plan(B: int, Hq: int, Hkv: int, D: int, Lmax: int, dtype=torch.bfloat16,
                         out_dtype=torch.bfloat16, probe: bool = True) -> dict:
    """How a decode call with num_splits=0 runs these shapes: the grid size and
    the CTAs per cluster (0: split-KV partitions + merge kernel)."""
    fn = load_library().parallax_decode_plan
    fn.argtypes = [ctypes.c_int] * 8 + [ctypes.POINTER(ctypes.c_int)] * 2
    fn.restype = ctypes.c_int
    grid, cl = ctypes.c_int(0), ctypes.c_int(0)
    _check(fn(B, Hq, Hkv, D, Lmax, _DTYPE_CODE[dtype], _DTYPE_CODE[out_dtype], int(bool(probe)),
              ctypes.byref(grid), ctypes.byref(cl)), "parallax_decode_plan")
    return {"grid_ctas": grid.value, "cluster_ctas": cl.value}


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


KV_LAYOUTS = {"bhsd": 0, "bshd": 1}


def _shapes(q, k_cache, v_cache, cache_seqlens, kv_layout="bhsd"):
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                    ("cache_seqlens", cache_seqlens)):
        if t is None and name == "cache_seqlens":
            continue
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if q.dim() != 3 or k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("expected q [B,Hq,D] and a 4-D k_cache, v_cache")
    if cache_seqlens is not None and (cache_seqlens.dtype != torch.int32
                                      or cache_seqlens.shape != (q.shape[0],)):
        raise ValueError("cache_seqlens must be int32 [B]")
    if k_cache.dtype != q.dtype or v_cache.dtype != q.dtype or q.dtype not in _DTYPE_CODE:
        raise ValueError("q, r, k_cache, v_cache must share one dtype (bf16 or fp32)")
    B, Hq, D = q.shape
    if kv_layout == "bshd":
        Bk, Lmax, Hkv, Dk = k_cache.shape
    elif kv_layout == "bhsd":
        Bk, Hkv, Lmax, Dk = k_cache.shape
    else:
        raise ValueError("kv_layout must be 'bhsd' or 'bshd'")
    if Bk != B or Dk != D:
        raise ValueError("k_cache shape does not match q")
    return B, Hq, Hkv, D, Lmax


def _prepare(q, k_cache, v_cache, cache_seqlens, out, out_dtype, workspace, num_splits,
             kv_layout="bhsd", window=0):
    B, Hq, Hkv, D, Lmax = _shapes(q, k_cache, v_cache, cache_seqlens, kv_layout)
    if out is None:
        out = torch.empty((B, Hq, D), device=q.device,
                          dtype=out_dtype if out_dtype is not None else q.dtype)
    if out.shape != (B, Hq, D) or not out.is_contiguous() or out.dtype not in _DTYPE_CODE:
        raise ValueError("out must be a contiguous [B,Hq,D] bf16 or fp32 tensor")
    if workspace is None:
        eff = min(Lmax, window) if window > 0 else Lmax
        workspace = Workspace(B, Hq, Hkv, D, eff, num_splits, device=q.device)
    return B, Hq, Hkv, D, Lmax, out, workspace


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def parallax_copy(dst, src, stream=None):
    """Stream-ordered copy of src into dst by a kernel (parallax_copy): for
    small per-step transfers between device tensors and page-locked host
    tensors (pin_memory()), where a DMA copy's fixed latency dominates. Both
    contiguous, the same number of bytes (a multiple of 16)."""
    if not (dst.is_contiguous() and src.is_contiguous()):
        raise ValueError("parallax_copy: tensors must be contiguous")
    nbytes = dst.numel() * dst.element_size()
    if src.numel() * src.element_size() != nbytes:
        raise ValueError("parallax_copy: dst and src differ in size")
    fn = load_library().parallax_copy
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    _check(fn(dst.data_ptr(), src.data_ptr(), nbytes, _stream(stream)), "parallax_copy")
    return dst


def parallax_decode(q, r, k_cache, v_cache, cache_seqlens=None, scale: Optional[float] = None,
                    out=None, out_dtype=None, num_splits: int = 0,
                    workspace: Optional[Workspace] = None, stream=None,
                    kv_layout: Optional[str] = None, window: int = 0):
    """Parallax decode: out[b,h] = vbar + C/l - (b/l) vbar over the cached keys.

    q, r: [B, Hq, D], or the pages' (B, 1, Hq, D) (the cache layout then
    defaults to (B, kv_len, Hkv, D) and the result has q's shape).
    cache_seqlens: int32 [B], or None for full-length sequences.
    kv_layout: 'bhsd' ([B, Hkv, Lmax, D], the default) or 'bshd'.
    window: 0, or attend only the last `window` keys of each sequence."""
    four_d = q.dim() == 4
    if four_d:
        if q.shape[1] != 1 or r.shape != q.shape:
            raise ValueError("4-D q and r must be (B, 1, H, D)")
        q, r = q.reshape(q.shape[0], q.shape[2], q.shape[3]), r.reshape(r.shape[0], r.shape[2], r.shape[3])
    layout = kv_layout or ("bshd" if four_d else "bhsd")
    B, Hq, Hkv, D, Lmax, out, workspace = _prepare(q, k_cache, v_cache, cache_seqlens, out,
                                                   out_dtype, workspace, num_splits, layout,
                                                   window)
    if r.shape != q.shape or r.dtype != q.dtype or not r.is_cuda or not r.is_contiguous():
        raise ValueError("r must be a contiguous CUDA tensor shaped like q")
    scale = D ** -0.5 if scale is None else scale
    lib = load_library()
    args = (q.data_ptr(), r.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
            _ptr(cache_seqlens), out.data_ptr(), B, Hq, Hkv, D, float(scale), _stream(stream),
            Lmax, _DTYPE_CODE[q.dtype], _DTYPE_CODE[out.dtype], int(num_splits),
            workspace.ptr(), workspace.nbytes)
    if layout == "bhsd" and window == 0:
        rc = lib.parallax_decode(*args)
    else:
        rc = lib.parallax_decode_ex(*args, 1, KV_LAYOUTS[layout], int(window), 3)
    _check(rc, "parallax_decode")
    return out.reshape(B, 1, Hq, D) if four_d else out


def parallax_softmax_decode(q, k_cache, v_cache, cache_seqlens=None,
                            scale: Optional[float] = None, out=None, out_dtype=None,
                            num_splits: int = 0, workspace: Optional[Workspace] = None,
                            stream=None, kv_layout: str = "bhsd", window: int = 0):
    """The R = 0 comparator: softmax attention decode on the same pipeline."""
    B, Hq, Hkv, D, Lmax, out, workspace = _prepare(q, k_cache, v_cache, cache_seqlens, out,
                                                   out_dtype, workspace, num_splits, kv_layout,
                                                   window)
    scale = D ** -0.5 if scale is None else scale
    lib = load_library()
    args = (q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), _ptr(cache_seqlens),
            out.data_ptr(), B, Hq, Hkv, D, float(scale), _stream(stream), Lmax,
            _DTYPE_CODE[q.dtype], _DTYPE_CODE[out.dtype], int(num_splits), workspace.ptr(),
            workspace.nbytes)
    if kv_layout == "bhsd" and window == 0:
        rc = lib.parallax_softmax_decode(*args)
    else:
        rc = lib.parallax_decode_ex(args[0], None, *args[1:], 0, KV_LAYOUTS[kv_layout],
                                    int(window), 3)
    _check(rc, "parallax_softmax_decode")
    return out


def parallax_decode_ex(q, r, k_cache, v_cache, cache_seqlens, out, workspace: Workspace,
                       scale: Optional[float] = None, num_splits: int = 0, probe: bool = True,
                       kv_layout: str = "bhsd", window: int = 0, phases: int = 3, stream=None):
    """The general entry point: probe (Parallax) or not (R = 0), either cache
    layout, an optional sliding window, and the phases to run."""
    B, Hq, Hkv, D, Lmax, out, workspace = _prepare(q, k_cache, v_cache, cache_seqlens, out,
                                                   None, workspace, num_splits, kv_layout,
                                                   window)
    scale = D ** -0.5 if scale is None else scale
    rc = load_library().parallax_decode_ex(
        q.data_ptr(), _ptr(r) if probe else None, k_cache.data_ptr(), v_cache.data_ptr(),
        _ptr(cache_seqlens), out.data_ptr(), B, Hq, Hkv, D, float(scale), _stream(stream), Lmax,
        _DTYPE_CODE[q.dtype], _DTYPE_CODE[out.dtype], int(num_splits), workspace.ptr(),
        workspace.nbytes, int(bool(probe)), KV_LAYOUTS[kv_layout], int(window), int(phases))
    _check(rc, "parallax_decode_ex")
    return out


def _check_int32(name, t, dim):
    if (t is None or not t.is_cuda or t.dtype != torch.int32 or t.dim() != dim
            or not t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous {dim}-D int32 CUDA tensor")


def parallax_decode_paged(q, r, k_pages, v_pages, block_table, cache_seqlens=None,
                          scale: Optional[float] = None, out=None, out_dtype=None,
                          workspace: Optional[Workspace] = None, num_splits: int = 0,
                          probe: bool = True, stream=None):
    """Decode over a paged cache: k_pages, v_pages [num_pages, page_size, Hkv, D]
    bf16 or fp32 (q's dtype), block_table int32 [B, max_pages_per_seq] (page
    ids per sequence), cache_seqlens int32 [B] or None (every sequence fills
    its table)."""
    for name, t in (("q", q), ("k_pages", k_pages), ("v_pages", v_pages)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype not in _DTYPE_CODE:
            raise ValueError(f"{name} must be a contiguous bf16 or fp32 CUDA tensor")
        if t.dtype != q.dtype:
            raise ValueError("q, r, k_pages, v_pages must share one dtype")
    if probe and (r is None or r.shape != q.shape or r.dtype != q.dtype or not r.is_cuda
                  or not r.is_contiguous()):
        raise ValueError("r must be a contiguous CUDA tensor shaped like q")
    if q.dim() != 3 or k_pages.dim() != 4 or v_pages.shape != k_pages.shape:
        raise ValueError("expected q [B,Hq,D] and k_pages, v_pages [num_pages,page_size,Hkv,D]")
    B, Hq, D = q.shape
    num_pages, page_size, Hkv, Dk = k_pages.shape
    if Dk != D:
        raise ValueError("head dimension of the pages does not match q")
    _check_int32("block_table", block_table, 2)
    if block_table.shape[0] != B:
        raise ValueError("block_table must be [B, max_pages_per_seq]")
    if cache_seqlens is not None:
        _check_int32("cache_seqlens", cache_seqlens, 1)
    max_pages = block_table.shape[1]
    if out is None:
        out = torch.empty((B, Hq, D), device=q.device,
                          dtype=out_dtype if out_dtype is not None else q.dtype)
    if workspace is None:
        workspace = Workspace(B, Hq, Hkv, D, max_pages * page_size, num_splits, device=q.device)
    scale = D ** -0.5 if scale is None else scale
    rc = load_library().parallax_decode_paged(
        q.data_ptr(), _ptr(r) if probe else None, k_pages.data_ptr(), v_pages.data_ptr(),
        block_table.data_ptr(), _ptr(cache_seqlens), out.data_ptr(), B, Hq, Hkv, D, float(scale),
        _stream(stream), num_pages, page_size, max_pages, int(bool(probe)), _DTYPE_CODE[q.dtype],
        _DTYPE_CODE[out.dtype], int(num_splits), workspace.ptr(), workspace.nbytes)
    _check(rc, "parallax_decode_paged")
    return out


def parallax_decode_block_sparse(q, r, k_cache, v_cache, block_ids, num_blocks,
                                 cache_seqlens=None, scale: Optional[float] = None, out=None,
                                 out_dtype=None, workspace: Optional[Workspace] = None,
                                 num_splits: int = 0, probe: bool = True, kv_layout: str = "bhsd",
                                 stream=None):
    """Decode over the listed 64-key blocks of each sequence: block_ids int32
    [B, max_blocks] (first num_blocks[b] used), num_blocks int32 [B]; bf16 or
    fp32 inputs."""
    B, Hq, Hkv, D, Lmax = _shapes(q, k_cache, v_cache, cache_seqlens, kv_layout)
    if probe and (r is None or r.shape != q.shape or r.dtype != q.dtype or not r.is_cuda
                  or not r.is_contiguous()):
        raise ValueError("r must be a contiguous CUDA tensor shaped like q")
    _check_int32("block_ids", block_ids, 2)
    _check_int32("num_blocks", num_blocks, 1)
    if block_ids.shape[0] != B or num_blocks.shape != (B,):
        raise ValueError("block_ids must be [B, max_blocks] and num_blocks [B]")
    max_blocks = block_ids.shape[1]
    if out is None:
        out = torch.empty((B, Hq, D), device=q.device,
                          dtype=out_dtype if out_dtype is not None else q.dtype)
    if workspace is None:
        workspace = Workspace(B, Hq, Hkv, D, 64 * max_blocks, num_splits, device=q.device)
    scale = D ** -0.5 if scale is None else scale
    rc = load_library().parallax_decode_block_sparse(
        q.data_ptr(), _ptr(r) if probe else None, k_cache.data_ptr(), v_cache.data_ptr(),
        _ptr(cache_seqlens), block_ids.data_ptr(), num_blocks.data_ptr(), out.data_ptr(), B, Hq,
        Hkv, D, float(scale), _stream(stream), Lmax, KV_LAYOUTS[kv_layout], max_blocks,
        int(bool(probe)), _DTYPE_CODE[q.dtype], _DTYPE_CODE[out.dtype], int(num_splits),
        workspace.ptr(), workspace.nbytes)
    _check(rc, "parallax_decode_block_sparse")
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
        k_cache.data_ptr(), v_cache.data_ptr(), _ptr(cache_seqlens), out.data_ptr(),
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
            _ptr(cache_seqlens), out.data_ptr(), B, Hq, Hkv, D, float(scale),
            _stream(stream), Lmax, _DTYPE_CODE[q.dtype], _DTYPE_CODE[out.dtype], int(num_splits))
    _check(rc, "parallax_decode_noalloc")
    return out


def parallax_prefill_workspace_bytes(B: int, L: int, Hkv: int, D: int) -> int:
    """Workspace bytes for the fp16 value products of a bf16-output prefill
    (dense: B rows of L keys; packed: B = 1, L = total tokens)."""
    lib = load_library()
    fn = lib.parallax_prefill_workspace_bytes
    fn.argtypes = [ctypes.c_int] * 4
    fn.restype = ctypes.c_size_t
    return int(fn(B, L, Hkv, D))


def prefill_workspace(B: int, L: int, Hkv: int, D: int, device):
    """A prefill workspace of parallax_prefill_workspace_bytes bytes with its
    256-byte header (the status word) zeroed."""
    ws = torch.empty(max(256, parallax_prefill_workspace_bytes(B, L, Hkv, D)), dtype=torch.uint8,
                     device=device)
    ws[:256].zero_()
    return ws


def parallax_prefill(q, r, k, v, scale: Optional[float] = None, causal: bool = True, out=None,
                     out_dtype=None, workspace=None, stream=None):
    """Training-shape forward (the README's parallax_func): q, r [B, Hq, L, D],
    k, v [B, Hkv, L, D] bf16 -> [B, Hq, L, D]; row i attends keys 0..i."""
    lib = load_library()
    fn = lib.parallax_prefill
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fn.argtypes = [vp] * 5 + [i] * 5 + [f, i, vp, i, vp, ctypes.c_size_t]
    fn.restype = i
    for name, t in (("q", q), ("r", r), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != torch.bfloat16 or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous 4-D bf16 CUDA tensor")
    B, Hq, L, D = q.shape
    if r.shape != q.shape or k.shape != v.shape or k.shape[0] != B or k.shape[2:] != (L, D):
        raise ValueError("expected q, r [B, Hq, L, D] and k, v [B, Hkv, L, D]")
    Hkv = k.shape[1]
    if out is None:
        out = torch.empty_like(q, dtype=out_dtype if out_dtype is not None else q.dtype)
    if workspace is None:
        workspace = prefill_workspace(B, L, Hkv, D, q.device)
    buf = workspace.buffer if isinstance(workspace, Workspace) else workspace
    scale = D ** -0.5 if scale is None else scale
    rc = fn(q.data_ptr(), r.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hq, Hkv,
            L, D, float(scale), int(bool(causal)), _stream(stream), _DTYPE_CODE[out.dtype],
            buf.data_ptr(), buf.numel())
    _check(rc, "parallax_prefill")
    return out
