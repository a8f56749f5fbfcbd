"""fp64 CPU oracle for exact attention (prefill and paged decode).

TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the benchmark's
CPU-baseline leg may import this package; the product path never does, and
this package imports nothing from the product package.

The arithmetic lives in ``oracle.c`` (plain definition, fp64, two-pass
softmax over a materialised score row).  This module only marshals arrays
into it: inputs may be torch CPU tensors or numpy arrays of bf16 (torch
``bfloat16``), float32 or float64, and are passed to C in that element type
so that the C code upcasts them exactly.

Module-level functions use the library built from ``oracle.c``;
``Oracle(path)`` binds any other build of the same source (the mutation
tests use this to load copies with a planted mistake).
"""
from __future__ import annotations

import ctypes
from typing import Sequence

import numpy as np

from . import build as _build

_BF16, _F32, _F64 = 0, 1, 2


def _as_np(x):
    """Return (numpy array, dtype code).  bf16 tensors become uint16 bit patterns."""
    try:
        import torch
    except ImportError:  # pragma: no cover
        torch = None
    if torch is not None and isinstance(x, torch.Tensor):
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy().view(np.uint16), _BF16
        if x.dtype == torch.float32:
            return x.numpy(), _F32
        if x.dtype == torch.float64:
            return x.numpy(), _F64
        raise TypeError(f"unsupported dtype {x.dtype}")
    a = np.ascontiguousarray(x)
    if a.dtype == np.float32:
        return a, _F32
    if a.dtype == np.float64:
        return a, _F64
    raise TypeError(f"unsupported dtype {a.dtype} (pass bf16 as a torch tensor)")


def _int_np(x, dtype):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x), dtype=dtype)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _ptr_or_null(a):
    return None if a is None else _ptr(a)


def _variant(window, softcap, alibi_slopes, B: int, Hq: int):
    """Marshals the mask-variant arguments: (left, right, softcap, slopes
    as contiguous float32 or None, slope stride per sequence)."""
    left, right = (int(window[0]), int(window[1]))
    if softcap < 0:
        raise ValueError("softcap must be >= 0")
    if alibi_slopes is None:
        return left, right, float(softcap), None, 0
    a = np.ascontiguousarray(_as_np(alibi_slopes)[0], dtype=np.float32)
    if a.shape == (Hq,):
        return left, right, float(softcap), a, 0
    if a.shape == (B, Hq):
        return left, right, float(softcap), a, Hq
    raise ValueError(f"alibi_slopes must be [Hq] or [B, Hq], got {a.shape}")


def _same_dtype(*arrs):
    codes = {c for _, c in arrs}
    if len(codes) != 1:
        raise TypeError("q, k and v must share one element type")
    return codes.pop()


class Oracle:
    """ctypes binding of one build of ``oracle.c``."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        vp = ctypes.c_void_p
        ci, cd, c64 = ctypes.c_int, ctypes.c_double, ctypes.c_int64
        lib.oracle_prefill_rows_ex.argtypes = [vp, vp, vp, ci, vp, ci, ci, ci, ci, ci, cd,
                                               ci, ci, cd, vp, ci, vp, vp, c64, vp, vp]
        lib.oracle_prefill_ex.argtypes = [vp, vp, vp, ci, vp, ci, ci, ci, ci, ci, cd,
                                          ci, ci, cd, vp, ci, vp, vp]
        lib.oracle_prefill_probs.argtypes = [vp, vp, ci, vp, ci, ci, ci, ci, ci, cd,
                                             ci, ci, cd, vp, ci, ci, ci, vp]
        lib.oracle_decode_paged.argtypes = [vp, vp, vp, ci, vp, vp, ci, ci, ci, ci, ci, ci,
                                            c64, cd, vp, vp]
        lib.oracle_rope.argtypes = [vp, ci, c64, ci, vp, vp, vp, c64, ci, ci, vp]
        lib.oracle_decode_paged_append.argtypes = [vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci,
                                                   ci, c64, cd, vp, vp, c64, ci, ci, vp, vp, vp]
        lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_prefill_fp8.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, cd, cd, cd, cd, vp, vp]
        lib.oracle_prefill_fp8.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        lib.oracle_set_num_threads.argtypes = [ci]
        for f in (lib.oracle_prefill_rows_ex, lib.oracle_prefill_ex, lib.oracle_prefill_probs,
                  lib.oracle_decode_paged, lib.oracle_num_threads, lib.oracle_rope,
                  lib.oracle_decode_paged_append):
            f.restype = ctypes.c_int
        lib.oracle_set_num_threads.restype = None
        self._lib = lib
        self.path = path

    def set_num_threads(self, n: int) -> None:
        self._lib.oracle_set_num_threads(int(n))

    def num_threads(self) -> int:
        return int(self._lib.oracle_num_threads())

    def prefill(self, q, k, v, cu_seqlens, causal: bool, scale: float, window=(-1, -1),
                softcap: float = 0.0, alibi_slopes=None):
        """Exact attention over packed sequences.

        q: [T, Hq, d]; k, v: [T, Hkv, d]; cu_seqlens: [B+1].
        window = (left, right): key j visible to query i when
        i - left <= j <= i + right (a negative bound: unlimited).
        softcap > 0: logits x become softcap * tanh(x / softcap).
        alibi_slopes: fp32 [Hq] or [B, Hq], adds -slope * |i - j|.
        Returns (o [T, Hq, d] float64, lse [Hq, T] float64).
        """
        (qa, c1), (ka, c2), (va, c3) = _as_np(q), _as_np(k), _as_np(v)
        dt = _same_dtype((qa, c1), (ka, c2), (va, c3))
        cu = _int_np(cu_seqlens, np.int32)
        T, Hq, d = qa.shape
        Hkv = ka.shape[1]
        B = cu.shape[0] - 1
        o = np.zeros((T, Hq, d), np.float64)
        lse = np.zeros((Hq, T), np.float64)
        wl, wr, sc, al, ast = _variant(window, softcap, alibi_slopes, B, Hq)
        rc = self._lib.oracle_prefill_ex(_ptr(qa), _ptr(ka), _ptr(va), dt, _ptr(cu), B, Hq, Hkv,
                                         d, int(bool(causal)), float(scale), wl, wr, sc,
                                         _ptr_or_null(al), ast, _ptr(o), _ptr(lse))
        if rc != 0:
            raise ValueError(f"oracle_prefill rejected its arguments (rc={rc})")
        return o, lse

    def prefill_rows(self, q, k, v, cu_seqlens, causal: bool, scale: float,
                     rows_t: Sequence[int], rows_h: Sequence[int], window=(-1, -1),
                     softcap: float = 0.0, alibi_slopes=None):
        """Exact attention for selected (token, head) rows only (variant
        arguments as in ``prefill``).

        Returns (o [n, d] float64, lse [n] float64).  Rows are independent,
        so a sample of rows is exact for those rows.
        """
        (qa, c1), (ka, c2), (va, c3) = _as_np(q), _as_np(k), _as_np(v)
        dt = _same_dtype((qa, c1), (ka, c2), (va, c3))
        cu = _int_np(cu_seqlens, np.int32)
        rt = _int_np(rows_t, np.int64)
        rh = _int_np(rows_h, np.int32)
        T, Hq, d = qa.shape
        Hkv = ka.shape[1]
        B = cu.shape[0] - 1
        n = rt.shape[0]
        o = np.zeros((n, d), np.float64)
        lse = np.zeros((n,), np.float64)
        wl, wr, sc, al, ast = _variant(window, softcap, alibi_slopes, B, Hq)
        rc = self._lib.oracle_prefill_rows_ex(_ptr(qa), _ptr(ka), _ptr(va), dt, _ptr(cu), B, Hq,
                                              Hkv, d, int(bool(causal)), float(scale), wl, wr,
                                              sc, _ptr_or_null(al), ast, _ptr(rt), _ptr(rh), n,
                                              _ptr(o), _ptr(lse))
        if rc != 0:
            raise ValueError(f"oracle_prefill_rows rejected its arguments (rc={rc})")
        return o, lse

    def prefill_probs(self, q, k, cu_seqlens, causal: bool, scale: float, b: int, h: int,
                      Hkv: int, window=(-1, -1), softcap: float = 0.0, alibi_slopes=None):
        """The [L, L] probability matrix P of one (sequence, head); zeros where
        masked (variant arguments as in ``prefill``)."""
        (qa, c1), (ka, c2) = _as_np(q), _as_np(k)
        dt = _same_dtype((qa, c1), (ka, c2))
        cu = _int_np(cu_seqlens, np.int32)
        T, Hq, d = qa.shape
        B = cu.shape[0] - 1
        L = int(cu[b + 1] - cu[b])
        P = np.zeros((L, L), np.float64)
        wl, wr, sc, al, ast = _variant(window, softcap, alibi_slopes, B, Hq)
        rc = self._lib.oracle_prefill_probs(_ptr(qa), _ptr(ka), dt, _ptr(cu), B, Hq, Hkv, d,
                                            int(bool(causal)), float(scale), wl, wr, sc,
                                            _ptr_or_null(al), ast, int(b), int(h), _ptr(P))
        if rc != 0:
            raise ValueError(f"oracle_prefill_probs rejected its arguments (rc={rc})")
        return P

    def decode_paged(self, q, k_pages, v_pages, block_table, seq_lens, scale: float):
        """Single-token attention of each request over its paged K/V cache.

        q: [B, Hq, d]; k_pages, v_pages: [num_pages, page_size, Hkv, d];
        block_table: [B, max_blocks] int32; seq_lens: [B] int32.
        Returns (o [B, Hq, d] float64, lse [B, Hq] float64).
        """
        (qa, c1), (ka, c2), (va, c3) = _as_np(q), _as_np(k_pages), _as_np(v_pages)
        dt = _same_dtype((qa, c1), (ka, c2), (va, c3))
        bt = _int_np(block_table, np.int32)
        sl = _int_np(seq_lens, np.int32)
        B, Hq, d = qa.shape
        num_pages, page_size, Hkv, _ = ka.shape
        max_blocks = bt.shape[1]
        o = np.zeros((B, Hq, d), np.float64)
        lse = np.zeros((B, Hq), np.float64)
        rc = self._lib.oracle_decode_paged(_ptr(qa), _ptr(ka), _ptr(va), dt, _ptr(bt),
                                           _ptr(sl), B, Hq, Hkv, d, page_size, max_blocks,
                                           num_pages, float(scale), _ptr(o), _ptr(lse))
        if rc == -2:
            raise IndexError("a used block_table entry is outside [0, num_pages)")
        if rc != 0:
            raise ValueError(f"oracle_decode_paged rejected its arguments (rc={rc})")
        return o, lse


    def rope(self, x, pos, cos, sin, rotary_dim: int, interleaved: bool = False):
        """Exact RoPE of rows x [n, d] at positions pos [n] with fp32 tables
        cos/sin [max_pos, rotary_dim/2].  Returns float64 [n, d] (unrounded)."""
        xa, dt = _as_np(x)
        n, d = xa.shape
        ps = _int_np(pos, np.int32)
        ca = np.ascontiguousarray(_as_np(cos)[0], dtype=np.float32)
        sa = np.ascontiguousarray(_as_np(sin)[0], dtype=np.float32)
        out = np.zeros((n, d), np.float64)
        rc = self._lib.oracle_rope(_ptr(xa), dt, n, d, _ptr(ps), _ptr(ca), _ptr(sa), ca.shape[0],
                                   int(rotary_dim), int(bool(interleaved)), _ptr(out))
        if rc != 0:
            raise ValueError(f"oracle_rope rejected its arguments (rc={rc})")
        return out

    def decode_paged_append(self, q, k_new, v_new, k_pages, v_pages, block_table, cache_seqlens,
                            scale: float, cos=None, sin=None, rotary_dim: int | None = None,
                            interleaved: bool = False):
        """Append one token per request to a copy of the paged cache (with
        RoPE when cos/sin are given) and attend.  bf16 tensors.

        Returns (o [B, Hq, d] float64, lse [B, Hq] float64, k_pages, v_pages
        (updated copies, bf16 bit patterns as uint16 arrays), q_rot [B, Hq, d]
        float64 (the bf16-rounded rotated queries)).
        """
        (qa, c1), (kn, c2), (vn, c3) = _as_np(q), _as_np(k_new), _as_np(v_new)
        (kp, c4), (vpg, c5) = _as_np(k_pages), _as_np(v_pages)
        if {c1, c2, c3, c4, c5} != {_BF16}:
            raise TypeError("decode_paged_append takes bf16 tensors")
        kp, vpg = kp.copy(), vpg.copy()
        bt = _int_np(block_table, np.int32)
        cs = _int_np(cache_seqlens, np.int32)
        B, Hq, d = qa.shape
        num_pages, page_size, Hkv, _ = kp.shape
        if cos is not None:
            ca = np.ascontiguousarray(_as_np(cos)[0], dtype=np.float32)
            sa = np.ascontiguousarray(_as_np(sin)[0], dtype=np.float32)
            rd = int(rotary_dim if rotary_dim is not None else 2 * ca.shape[1])
            mp = ca.shape[0]
        else:
            ca = sa = None
            rd, mp = 0, 0
        o = np.zeros((B, Hq, d), np.float64)
        lse = np.zeros((B, Hq), np.float64)
        qr = np.zeros((B, Hq, d), np.float64)
        rc = self._lib.oracle_decode_paged_append(
            _ptr(qa), _ptr(kn), _ptr(vn), _ptr(kp), _ptr(vpg), _ptr(bt), _ptr(cs), B, Hq, Hkv, d,
            page_size, bt.shape[1], num_pages, float(scale), _ptr_or_null(ca), _ptr_or_null(sa),
            mp, rd, int(bool(interleaved)), _ptr(qr), _ptr(o), _ptr(lse))
        if rc == -2:
            raise IndexError("a block_table entry the append or attention needs is out of the pool")
        if rc != 0:
            raise ValueError(f"oracle_decode_paged_append rejected its arguments (rc={rc})")
        return o, lse, kp, vpg, qr


    def e4m3_value(self, byte: int) -> float:
        """Exact value of one e4m3 byte."""
        return float(self._lib.oracle_e4m3_value(int(byte) & 0xFF))

    def prefill_fp8(self, q, k, v, cu_seqlens, causal: bool, scale: float, q_descale: float = 1.0,
                    k_descale: float = 1.0, v_descale: float = 1.0):
        """Exact attention of e4m3 inputs (torch float8_e4m3fn tensors, or uint8
        bytes) times their per-tensor descale factors.  Returns (o, lse) as
        in ``prefill``."""
        def raw(x):
            import torch
            if isinstance(x, torch.Tensor):
                x = x.detach().cpu().contiguous()
                if x.dtype != torch.uint8:
                    x = x.view(torch.uint8)
                return x.numpy()
            return np.ascontiguousarray(x, dtype=np.uint8)
        qa, ka, va = raw(q), raw(k), raw(v)
        cu = _int_np(cu_seqlens, np.int32)
        T, Hq, d = qa.shape
        Hkv = ka.shape[1]
        B = cu.shape[0] - 1
        o = np.zeros((T, Hq, d), np.float64)
        lse = np.zeros((Hq, T), np.float64)
        rc = self._lib.oracle_prefill_fp8(_ptr(qa), _ptr(ka), _ptr(va), _ptr(cu), B, Hq, Hkv, d,
                                          int(bool(causal)), float(scale), float(q_descale),
                                          float(k_descale), float(v_descale), _ptr(o), _ptr(lse))
        if rc != 0:
            raise ValueError(f"oracle_prefill_fp8 rejected its arguments (rc={rc})")
        return o, lse


_default: Oracle | None = None


def default() -> Oracle:
    """The oracle built from ``oracle.c`` (built on first use).

    ``ORACLE_LIB`` names another build of the same source instead; the
    mutation tests point it at copies with a planted mistake.
    """
    global _default
    if _default is None:
        import os
        _default = Oracle(os.environ.get("ORACLE_LIB") or _build.ensure_built())
    return _default


def prefill(*args, **kw):
    return default().prefill(*args, **kw)


def prefill_rows(*args, **kw):
    return default().prefill_rows(*args, **kw)


def prefill_probs(*args, **kw):
    return default().prefill_probs(*args, **kw)


def decode_paged(*args, **kw):
    return default().decode_paged(*args, **kw)


def rope(*args, **kw):
    return default().rope(*args, **kw)


def decode_paged_append(*args, **kw):
    return default().decode_paged_append(*args, **kw)


def e4m3_value(*args, **kw):
    return default().e4m3_value(*args, **kw)


def prefill_fp8(*args, **kw):
    return default().prefill_fp8(*args, **kw)


def set_num_threads(n: int) -> None:
    default().set_num_threads(n)


def num_threads() -> int:
    return default().num_threads()
