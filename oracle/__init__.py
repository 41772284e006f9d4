"""fp64 CPU oracle for the Parallax decode forward.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
bench's CPU-baseline leg. The product path (the CUDA library and its binding)
never imports it and shares no code with it.

Every function takes arrays in the product layout and widens them to float64
(exact for bf16 and fp32 inputs):
    q, r, out : [B, Hq, D]
    k, v      : [B, Hkv, Lmax, D]
    seqlens   : [B] int32, each in [0, Lmax]

The arithmetic lives in parallax_oracle.c; its header gives the equations and
the passages of the pages they follow.
"""
import ctypes

import numpy as np

from . import build as _build


def _f64(x):
    if hasattr(x, "detach"):  # torch tensor: widen on the host, exactly
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a, ctype=ctypes.c_double):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


class Oracle:
    """The oracle functions of one compiled copy of parallax_oracle.c."""

    def __init__(self, path):
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        i = ctypes.c_int
        d = ctypes.c_double
        lib.oracle_parallax_covariance.argtypes = [dp, dp, dp, dp, ip, i, i, i, i, i, d, dp]
        lib.oracle_parallax_expanded.argtypes = [dp, dp, dp, dp, ip, i, i, i, i, i, d, dp]
        lib.oracle_parallax_streaming.argtypes = [dp, dp, dp, dp, ip, i, i, i, i, i, d, i, dp]
        lib.oracle_softmax_decode.argtypes = [dp, dp, dp, ip, i, i, i, i, i, d, dp]
        lib.oracle_parallax_prefill.argtypes = [dp, dp, dp, dp, i, i, i, i, i, d, i, dp]
        lib.oracle_parallax_prefill.restype = ctypes.c_int
        for f in (lib.oracle_parallax_covariance, lib.oracle_parallax_expanded,
                  lib.oracle_parallax_streaming, lib.oracle_softmax_decode,
                  lib.oracle_num_threads):
            f.restype = ctypes.c_int
        self._lib = lib
        self.path = path

    @staticmethod
    def _prep(q, k, v, seqlens):
        q, k, v = _f64(q), _f64(k), _f64(v)
        if hasattr(seqlens, "detach"):
            seqlens = seqlens.detach().cpu().numpy()
        seqlens = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
        if q.ndim != 3 or k.ndim != 4 or v.shape != k.shape:
            raise ValueError("expected q [B,Hq,D] and k, v [B,Hkv,Lmax,D]")
        B, Hq, D = q.shape
        _, Hkv, Lmax, Dk = k.shape
        if k.shape[0] != B or Dk != D or seqlens.shape != (B,):
            raise ValueError("shape mismatch between q, k, v and seqlens")
        return q, k, v, seqlens, B, Hq, Hkv, Lmax, D

    @staticmethod
    def _check(rc, name):
        if rc != 0:
            raise ValueError(f"{name} rejected its arguments (rc={rc})")

    def _parallax(self, fn, name, q, r, k, v, seqlens, scale, *extra):
        q, k, v, seqlens, B, Hq, Hkv, Lmax, D = self._prep(q, k, v, seqlens)
        r = _f64(r)
        if r.shape != q.shape:
            raise ValueError("r must have the shape of q")
        out = np.zeros((B, Hq, D))
        rc = fn(_ptr(q), _ptr(r), _ptr(k), _ptr(v), _ptr(seqlens, ctypes.c_int32),
                B, Hq, Hkv, Lmax, D, float(scale), *extra, _ptr(out))
        self._check(rc, name)
        return out

    def parallax_covariance(self, q, r, k, v, seqlens, scale):
        """o = vbar + sum_i w_i (s_i - sbar)(v_i - vbar): the definition form."""
        return self._parallax(self._lib.oracle_parallax_covariance,
                              "oracle_parallax_covariance", q, r, k, v, seqlens, scale)

    def parallax_expanded(self, q, r, k, v, seqlens, scale):
        """o = A/l + C/l - (b/l)(A/l) with l, A, b, C summed over all keys."""
        return self._parallax(self._lib.oracle_parallax_expanded,
                              "oracle_parallax_expanded", q, r, k, v, seqlens, scale)

    def parallax_streaming(self, q, r, k, v, seqlens, scale, chunk):
        """Online accumulators over chunks of `chunk` keys, merged by max-rescaling."""
        return self._parallax(self._lib.oracle_parallax_streaming,
                              "oracle_parallax_streaming", q, r, k, v, seqlens, scale,
                              int(chunk))

    def softmax_decode(self, q, k, v, seqlens, scale):
        """Plain softmax attention, the R = 0 special case."""
        q, k, v, seqlens, B, Hq, Hkv, Lmax, D = self._prep(q, k, v, seqlens)
        out = np.zeros((B, Hq, D))
        rc = self._lib.oracle_softmax_decode(_ptr(q), _ptr(k), _ptr(v),
                                             _ptr(seqlens, ctypes.c_int32), B, Hq, Hkv,
                                             Lmax, D, float(scale), _ptr(out))
        self._check(rc, "oracle_softmax_decode")
        return out

    def parallax_prefill(self, q, r, k, v, scale, causal=True):
        """Training-shape forward: q, r [B, Hq, L, D], k, v [B, Hkv, L, D];
        row i attends keys 0..i (all keys when causal is False)."""
        q, r, k, v = _f64(q), _f64(r), _f64(k), _f64(v)
        if q.ndim != 4 or r.shape != q.shape or k.ndim != 4 or v.shape != k.shape:
            raise ValueError("expected q, r [B,Hq,L,D] and k, v [B,Hkv,L,D]")
        B, Hq, L, D = q.shape
        if k.shape[0] != B or k.shape[2] != L or k.shape[3] != D:
            raise ValueError("shape mismatch between q and k")
        out = np.zeros_like(q)
        rc = self._lib.oracle_parallax_prefill(_ptr(q), _ptr(r), _ptr(k), _ptr(v), B, Hq,
                                               k.shape[1], L, D, float(scale), int(bool(causal)),
                                               _ptr(out))
        self._check(rc, "oracle_parallax_prefill")
        return out

    def parallax_varlen_prefill(self, q, r, k, v, cu_seqlens, scale, causal=True):
        """Packed variable-length forward: q, r [total, Hq, D], k, v [total,
        Hkv, D]; sequence b is rows cu_seqlens[b]:cu_seqlens[b+1] and attends to
        its own keys only. Each sequence goes through parallax_prefill on its
        own, moved to the [1, H, len, D] layout and back."""
        q, r, k, v = _f64(q), _f64(r), _f64(k), _f64(v)
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        if q.ndim != 3 or r.shape != q.shape or k.ndim != 3 or v.shape != k.shape:
            raise ValueError("expected q, r [total,Hq,D] and k, v [total,Hkv,D]")
        if cu.ndim != 1 or cu[0] != 0 or cu[-1] != q.shape[0] or np.any(np.diff(cu) < 0):
            raise ValueError("cu_seqlens must rise from 0 to total")
        out = np.zeros_like(q)
        for b in range(len(cu) - 1):
            a, e = int(cu[b]), int(cu[b + 1])
            if e == a:
                continue
            seq = [np.ascontiguousarray(x[a:e].transpose(1, 0, 2))[None] for x in (q, r, k, v)]
            o = self.parallax_prefill(*seq, scale, causal)
            out[a:e] = o[0].transpose(1, 0, 2)
        return out

    def _decode(self, q, r, k, v, n, scale, probe):
        if probe:
            return self.parallax_covariance(q, r, k, v, n, scale)
        return self.softmax_decode(q, k, v, n, scale)

    def parallax_decode_paged(self, q, r, k_pages, v_pages, block_table, seqlens, scale,
                              probe=True):
        """Decode over a paged cache: k_pages, v_pages [num_pages, page_size,
        Hkv, D]; key i of sequence b is slot i % page_size of page
        block_table[b][i // page_size]. The pages are gathered into a
        [B, Hkv, Lmax, D] cache and the decode above runs on it."""
        q, kp, vp = _f64(q), _f64(k_pages), _f64(v_pages)
        r = _f64(r) if probe else np.zeros_like(q)
        table = np.asarray(block_table.cpu() if hasattr(block_table, "cpu") else block_table)
        B, Hq, D = q.shape
        _, ps, Hkv, _ = kp.shape
        Lmax = table.shape[1] * ps
        n = (np.full(B, Lmax) if seqlens is None else
             np.asarray(seqlens.cpu() if hasattr(seqlens, "cpu") else seqlens)).astype(np.int32)
        k = np.zeros((B, Hkv, Lmax, D))
        v = np.zeros((B, Hkv, Lmax, D))
        for b in range(B):
            for i in range(int(n[b])):
                page, slot = table[b, i // ps], i % ps
                k[b, :, i] = kp[page, slot]
                v[b, :, i] = vp[page, slot]
        return self._decode(q, r, k, v, n, scale, probe)

    def parallax_decode_block_sparse(self, q, r, k, v, block_ids, num_blocks, seqlens, scale,
                                     probe=True):
        """Decode over the listed 64-key blocks of each cache row: the keys of
        blocks block_ids[b][:num_blocks[b]] below seqlens[b], in list order,
        gathered into a dense cache with per-row lengths (k, v [B, Hkv, Lmax, D])."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        r = _f64(r) if probe else np.zeros_like(q)
        ids = np.asarray(block_ids.cpu() if hasattr(block_ids, "cpu") else block_ids)
        cnt = np.asarray(num_blocks.cpu() if hasattr(num_blocks, "cpu") else num_blocks)
        B, Hkv, Lmax, D = k.shape
        n = (np.full(B, Lmax) if seqlens is None else
             np.asarray(seqlens.cpu() if hasattr(seqlens, "cpu") else seqlens)).astype(np.int64)
        rows = []
        for b in range(B):
            keys = [key for blk in ids[b, :int(cnt[b])]
                    for key in range(64 * int(blk), 64 * int(blk) + 64) if key < n[b]]
            rows.append(keys)
        width = max(1, max(len(x) for x in rows))
        kg = np.zeros((B, Hkv, width, D))
        vg = np.zeros((B, Hkv, width, D))
        for b, keys in enumerate(rows):
            kg[b, :, :len(keys)] = k[b][:, keys]
            vg[b, :, :len(keys)] = v[b][:, keys]
        lens = np.array([len(x) for x in rows], dtype=np.int32)
        return self._decode(q, r, kg, vg, lens, scale, probe)

    # The default used by parity checks: the definition (covariance) form.
    def parallax_decode(self, q, r, k, v, seqlens, scale):
        return self.parallax_covariance(q, r, k, v, seqlens, scale)

    def num_threads(self) -> int:
        return int(self._lib.oracle_num_threads())


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def parallax_covariance(*a, **kw):
    return default().parallax_covariance(*a, **kw)


def parallax_expanded(*a, **kw):
    return default().parallax_expanded(*a, **kw)


def parallax_streaming(*a, **kw):
    return default().parallax_streaming(*a, **kw)


def softmax_decode(*a, **kw):
    return default().softmax_decode(*a, **kw)


def parallax_decode(*a, **kw):
    return default().parallax_decode(*a, **kw)


def parallax_prefill(*a, **kw):
    return default().parallax_prefill(*a, **kw)


def parallax_varlen_prefill(*a, **kw):
    return default().parallax_varlen_prefill(*a, **kw)


def parallax_decode_paged(*a, **kw):
    return default().parallax_decode_paged(*a, **kw)


def parallax_decode_block_sparse(*a, **kw):
    return default().parallax_decode_block_sparse(*a, **kw)


def num_threads() -> int:
    return default().num_threads()
