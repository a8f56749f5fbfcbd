"""Python binding of ``libfa.so`` (C ABI in ``include/fa.h``).

Argument marshalling only: shapes, dtypes and device pointers of torch
tensors are passed to the C entry points, which run every step of the
computation in this package's CUDA kernels.  There is no fallback: if the
library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

# Largest batch whose decode plan (the prefix of per-request range counts)
# each CTA of the split kernel builds itself; larger batches get it from a
# separate one-CTA plan kernel (FA_DECODE_PLAN_MAX_B in include/fa.h).
DECODE_PLAN_MAX_B = 2048

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_CUDA = 3
FA_ERR_DEVICE_BOUNDS = 4
FA_ERR_DEVICE_TIMEOUT = 5

_lib = None


class FAError(RuntimeError):
    """A non-OK status from the C ABI."""

    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {error_string(code)} (status {code})")


def load_library(path: str = LIB_PATH):
    """Load ``libfa.so`` and declare its signatures (idempotent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing; build it with `python -m exact_io_aware_86_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_prefill.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, i32, i32]
    lib.fa_prefill_ex.argtypes = lib.fa_prefill.argtypes + [i32, i32, f32, vp, i32]
    lib.fa_prefill_fp8.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, f32, f32,
                                   f32, vp, i32, i32]
    lib.fa_prefill_fp8.restype = ctypes.c_int
    lib.fa_decode_paged.argtypes = [vp, vp, vp, vp, vp, i32, i32, vp, vp, i32, i32, i32, i32, i32,
                                    i32, f32, vp, vp, sz]
    lib.fa_decode_paged_noalloc.argtypes = [vp, vp, vp, vp, vp, i32, i32, vp, vp, i32, i32, i32,
                                            i32, i32, i32, f32, vp]
    lib.fa_decode_paged_noalloc.restype = ctypes.c_int
    lib.fa_decode_paged_append.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, vp, vp, i32, i32,
                                           i32, i32, i32, i32, f32, vp, vp, vp, i32, i32, i32, vp,
                                           sz]
    lib.fa_decode_paged_append.restype = ctypes.c_int
    lib.fa_decode_append_workspace_size.argtypes = [i32, i32, i32, i32]
    lib.fa_decode_append_workspace_size.restype = sz
    lib.fa_decode_workspace_size.argtypes = [i32, i32, i32, i32]
    lib.fa_decode_workspace_size.restype = sz
    lib.fa_decode_auto_splits.argtypes = [i32, i32, i32, i32, i32, i32]
    lib.fa_prefill_f32.argtypes = lib.fa_prefill.argtypes
    lib.fa_decode_paged_f32.argtypes = [vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32,
                                        i32, f32, vp]
    lib.fa_get_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
    lib.fa_get_error_string.argtypes = [i32]
    lib.fa_get_error_string.restype = ctypes.c_char_p
    lib.fa_version.argtypes = []
    lib.fa_selftest_math.argtypes = [i32, vp, vp, i32, f32, f32, vp]
    lib.fa_selftest_math.restype = ctypes.c_int
    lib.fa_selftest_inject_stall.argtypes = [i32, ctypes.c_ulonglong]
    lib.fa_selftest_inject_stall.restype = ctypes.c_int
    for f in (lib.fa_prefill, lib.fa_prefill_ex, lib.fa_decode_paged, lib.fa_decode_auto_splits, lib.fa_prefill_f32,
              lib.fa_decode_paged_f32, lib.fa_get_device_error, lib.fa_version):
        f.restype = ctypes.c_int
    _lib = lib
    return lib


def error_string(code: int) -> str:
    return load_library().fa_get_error_string(int(code)).decode()


def _check(code: int, where: str) -> None:
    if code != FA_OK:
        raise FAError(code, where)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    return ctypes.c_void_p(int(stream))


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int, shape=None) -> None:
    """Type, dtype, rank, optional exact shape and contiguity of an argument.
    The device is checked separately (``_on_cuda``), after every shape, so a
    wrong shape is reported the same way on any device."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _on_cuda(**tensors) -> None:
    for name, t in tensors.items():
        if t is not None and not t.is_cuda:
            raise ValueError(f"{name} must be on a CUDA device")


# --------------------------------------------------------------------------
# prefill
# --------------------------------------------------------------------------
def fa_prefill(q, k, v, o, lse, cu_seqlens, causal: bool, scale: float = 0.0,
               max_seqlen: int | None = None, stream=None, *, window=(-1, -1),
               softcap: float = 0.0, alibi_slopes: torch.Tensor | None = None,
               _f32: bool = False) -> None:
    """Calls ``fa_prefill`` / ``fa_prefill_ex`` (bf16) or ``fa_prefill_f32``
    on torch CUDA tensors.

    q [T, Hq, d], k/v [T, Hkv, d], o [T, Hq, d], lse [Hq, T] fp32 or None,
    cu_seqlens int32 [B+1].  ``max_seqlen`` bounds every sequence length
    (defaults to T, which needs no device read).  ``window`` = (left, right)
    (negative = unlimited), ``softcap`` (0 = off) and ``alibi_slopes``
    (fp32 CUDA [Hq] or [B, Hq]) select the mask variants of ``fa_prefill_ex``.
    """
    dt = torch.float32 if _f32 else torch.bfloat16
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, n, dt, 3)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    if lse is not None:
        _need(lse, "lse", torch.float32, 2)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (T, Hkv, d) or v.shape != k.shape or o.shape != q.shape:
        raise ValueError("q/k/v/o shapes disagree")
    if lse is not None and lse.shape != (Hq, T):
        raise ValueError("lse must be [Hq, T]")
    _on_cuda(q=q, k=k, v=v, o=o, lse=lse, cu_seqlens=cu_seqlens, alibi_slopes=alibi_slopes)
    B = cu_seqlens.numel() - 1
    ms = T if max_seqlen is None else int(max_seqlen)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens), B, Hq, Hkv, d,
            int(bool(causal)), float(scale), _stream(stream), T, ms)
    left, right = int(window[0]), int(window[1])
    plain = left < 0 and right < 0 and softcap == 0 and alibi_slopes is None
    if _f32:
        if not plain:
            raise ValueError("the fp32 debug path has no mask variants")
        _check(load_library().fa_prefill_f32(*args), "fa_prefill_f32")
        return
    if plain:
        _check(load_library().fa_prefill(*args), "fa_prefill")
        return
    stride = 0
    if alibi_slopes is not None:
        if alibi_slopes.dim() == 1:
            _need(alibi_slopes, "alibi_slopes", torch.float32, 1)
            if alibi_slopes.shape[0] != Hq:
                raise ValueError("alibi_slopes must be [Hq] or [B, Hq]")
        else:
            _need(alibi_slopes, "alibi_slopes", torch.float32, 2)
            if tuple(alibi_slopes.shape) != (B, Hq):
                raise ValueError("alibi_slopes must be [Hq] or [B, Hq]")
            stride = Hq
    _check(load_library().fa_prefill_ex(*args, left, right, float(softcap), _ptr(alibi_slopes),
                                        stride), "fa_prefill_ex")


def prefill(q, k, v, cu_seqlens, causal: bool = True, scale: float = 0.0,
            max_seqlen: int | None = None, return_lse: bool = True, stream=None, *,
            window=(-1, -1), softcap: float = 0.0, alibi_slopes: torch.Tensor | None = None):
    """Allocates O (and LSE) and runs ``fa_prefill`` (``fa_prefill_ex`` when a
    mask variant is given).  Returns (o, lse or None)."""
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[1], q.shape[0], dtype=torch.float32, device=q.device) if return_lse else None
    fa_prefill(q, k, v, o, lse, cu_seqlens, causal, scale, max_seqlen, stream, window=window,
               softcap=softcap, alibi_slopes=alibi_slopes)
    return o, lse


def fa_prefill_fp8(q, k, v, o, lse, cu_seqlens, causal: bool, scale: float = 0.0,
                   q_descale: float = 1.0, k_descale: float = 1.0, v_descale: float = 1.0,
                   max_seqlen: int | None = None, stream=None) -> None:
    """Calls ``fa_prefill_fp8``: q [T, Hq, 128], k/v [T, Hkv, 128] as
    torch.float8_e4m3fn, o bf16 [T, Hq, 128], lse fp32 [Hq, T] or None."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.float8_e4m3fn, 3)
    _need(o, "o", torch.bfloat16, 3)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    if lse is not None:
        _need(lse, "lse", torch.float32, 2)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (T, Hkv, d) or v.shape != k.shape or o.shape != q.shape:
        raise ValueError("q/k/v/o shapes disagree")
    if lse is not None and lse.shape != (Hq, T):
        raise ValueError("lse must be [Hq, T]")
    _on_cuda(q=q, k=k, v=v, o=o, lse=lse, cu_seqlens=cu_seqlens)
    B = cu_seqlens.numel() - 1
    ms = T if max_seqlen is None else int(max_seqlen)
    _check(load_library().fa_prefill_fp8(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens), B, Hq, Hkv, d,
        int(bool(causal)), float(scale), float(q_descale), float(k_descale), float(v_descale),
        _stream(stream), T, ms), "fa_prefill_fp8")


def prefill_fp8(q, k, v, cu_seqlens, causal: bool = True, scale: float = 0.0,
                q_descale: float = 1.0, k_descale: float = 1.0, v_descale: float = 1.0,
                max_seqlen: int | None = None, return_lse: bool = True, stream=None):
    """Allocates O (bf16) and LSE and runs ``fa_prefill_fp8``.  Returns (o, lse or None)."""
    o = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    lse = torch.empty(q.shape[1], q.shape[0], dtype=torch.float32, device=q.device) if return_lse else None
    fa_prefill_fp8(q, k, v, o, lse, cu_seqlens, causal, scale, q_descale, k_descale, v_descale,
                   max_seqlen, stream)
    return o, lse


def prefill_f32(q, k, v, cu_seqlens, causal: bool = True, scale: float = 0.0, stream=None):
    """fp32 debug path: returns (o fp32, lse fp32)."""
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[1], q.shape[0], dtype=torch.float32, device=q.device)
    fa_prefill(q, k, v, o, lse, cu_seqlens, causal, scale, None, stream, _f32=True)
    return o, lse


# --------------------------------------------------------------------------
# paged decode
# --------------------------------------------------------------------------
def decode_workspace_size(B: int, Hq: int, d: int, num_splits: int) -> int:
    return int(load_library().fa_decode_workspace_size(B, Hq, d, num_splits))


def decode_auto_splits(B: int, Hq: int, Hkv: int, max_blocks_per_seq: int, page_size: int,
                       num_sms: int = 0) -> int:
    """The split count ``num_splits = 0`` resolves to (sizes the workspace)."""
    return int(load_library().fa_decode_auto_splits(B, Hq, Hkv, max_blocks_per_seq, page_size,
                                                    num_sms))


def _decode_shapes(q, k_pages, v_pages, block_table, seq_lens, dt, o=None, lse=None,
                   o_dtype=None):
    """Checks the decode arguments (o [B, Hq, d] and lse [B, Hq] when given:
    the kernels write exactly that many elements) and returns the shape
    scalars (B, Hq, Hkv, d, num_pages, page_size, max_blocks)."""
    _need(q, "q", dt, 3)
    _need(k_pages, "k_pages", dt, 4)
    _need(v_pages, "v_pages", dt, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    B, Hq, d = q.shape
    num_pages, page_size, Hkv, d2 = k_pages.shape
    if d2 != d or v_pages.shape != k_pages.shape:
        raise ValueError("q/k_pages/v_pages shapes disagree")
    if block_table.shape[0] != B or seq_lens.shape[0] != B:
        raise ValueError("block_table and seq_lens need one row per request")
    if o is not None:
        _need(o, "o", o_dtype or dt, 3, (B, Hq, d))
    if lse is not None:
        _need(lse, "lse", torch.float32, 2, (B, Hq))
    _on_cuda(q=q, k_pages=k_pages, v_pages=v_pages, block_table=block_table, seq_lens=seq_lens,
             o=o, lse=lse)
    return B, Hq, Hkv, d, num_pages, page_size, block_table.shape[1]


def fa_decode_paged(q, k_pages, v_pages, block_table, seq_lens, num_splits: int, o, lse=None,
                    scale: float = 0.0, workspace: torch.Tensor | None = None, stream=None) -> None:
    """Calls ``fa_decode_paged`` on torch CUDA tensors.

    q [B, Hq, d] bf16; k_pages/v_pages [num_pages, page_size, Hkv, d] bf16;
    block_table [B, max_blocks] int32; seq_lens [B] int32; o [B, Hq, d] bf16;
    lse [B, Hq] fp32 or None; workspace: a uint8 CUDA tensor of at least
    ``decode_workspace_size`` bytes, or None (the library then allocates
    stream-ordered scratch).
    """
    B, Hq, Hkv, d, num_pages, page_size, max_blocks = _decode_shapes(
        q, k_pages, v_pages, block_table, seq_lens, torch.bfloat16, o, lse)
    ws_bytes = 0
    if workspace is not None:
        if not workspace.is_cuda or not workspace.is_contiguous():
            raise ValueError("workspace must be a contiguous CUDA tensor")
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(load_library().fa_decode_paged(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens), page_size,
        int(num_splits), _ptr(o), _stream(stream), B, Hq, Hkv, d, max_blocks, num_pages,
        float(scale), _ptr(lse), _ptr(workspace), ws_bytes), "fa_decode_paged")


def fa_decode_paged_noalloc(q, k_pages, v_pages, block_table, seq_lens, num_splits: int, o,
                            lse=None, scale: float = 0.0, stream=None) -> None:
    """Calls ``fa_decode_paged_noalloc``: the same decode as
    ``fa_decode_paged``, with the split scratch taken from a fixed 64 MiB
    array inside the library, for callers that cannot allocate device memory
    at decode time.  Raises FAError(FA_ERR_UNSUPPORTED) when the split scratch
    this shape needs is larger than that array.  Concurrent calls on
    different streams share the array and must not overlap.
    """
    B, Hq, Hkv, d, num_pages, page_size, max_blocks = _decode_shapes(
        q, k_pages, v_pages, block_table, seq_lens, torch.bfloat16, o, lse)
    _check(load_library().fa_decode_paged_noalloc(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens), page_size,
        int(num_splits), _ptr(o), _stream(stream), B, Hq, Hkv, d, max_blocks, num_pages,
        float(scale), _ptr(lse)), "fa_decode_paged_noalloc")


def decode_paged(q, k_pages, v_pages, block_table, seq_lens, num_splits: int = 0,
                 scale: float = 0.0, return_lse: bool = True, stream=None):
    """Allocates O, LSE and the split workspace with torch and runs
    ``fa_decode_paged``.  Returns (o, lse or None)."""
    B, Hq, Hkv, d, num_pages, page_size, max_blocks = _decode_shapes(
        q, k_pages, v_pages, block_table, seq_lens, torch.bfloat16)
    S = num_splits if num_splits > 0 else decode_auto_splits(B, Hq, Hkv, max_blocks, page_size)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device) if return_lse else None
    nbytes = decode_workspace_size(B, Hq, d, S)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device) if nbytes else None
    fa_decode_paged(q, k_pages, v_pages, block_table, seq_lens, num_splits, o, lse, scale, ws,
                    stream)
    return o, lse


def decode_paged_f32(q, k_pages, v_pages, block_table, seq_lens, scale: float = 0.0, stream=None):
    """fp32 debug path: returns (o fp32, lse fp32)."""
    B, Hq, Hkv, d, num_pages, page_size, max_blocks = _decode_shapes(
        q, k_pages, v_pages, block_table, seq_lens, torch.float32)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    _check(load_library().fa_decode_paged_f32(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens), page_size,
        _ptr(o), _stream(stream), B, Hq, Hkv, d, max_blocks, num_pages, float(scale), _ptr(lse)),
        "fa_decode_paged_f32")
    return o, lse


MATH_EXP2_FMA, MATH_EXP2_MUFU, MATH_SOFTCAP_LOG2 = 0, 1, 2


def selftest_math(op: int, x: torch.Tensor, a: float = 0.0, b: float = 0.0, stream=None):
    """Calls ``fa_selftest_math``: y = f(x) elementwise on the GPU for one of
    the scalar functions of the prefill softmax (x: fp32 CUDA tensor)."""
    _need(x, "x", torch.float32, x.dim())
    _on_cuda(x=x)
    y = torch.empty_like(x)
    _check(load_library().fa_selftest_math(int(op), _ptr(x), _ptr(y), x.numel(), float(a),
                                           float(b), _stream(stream)), "fa_selftest_math")
    return y


STALL_NONE, STALL_PREFILL, STALL_DECODE = 0, 1, 2


def selftest_inject_stall(which: int, wait_limit_ns: int = 0) -> None:
    """Calls ``fa_selftest_inject_stall`` (timeout-path tests only): makes one
    warp of CTA 0 of the prefill (STALL_PREFILL) or decode (STALL_DECODE)
    kernels wait on a barrier nothing arrives at, with the abortable-wait
    limit set to wait_limit_ns (0 = the default 2 s).  (STALL_NONE, 0)
    restores normal operation."""
    _check(load_library().fa_selftest_inject_stall(int(which), int(wait_limit_ns)),
           "fa_selftest_inject_stall")


def device_error(stream=None) -> int:
    """Reads and clears the device error word (synchronises the stream)."""
    code = ctypes.c_int(0)
    _check(load_library().fa_get_device_error(_stream(stream), ctypes.byref(code)),
           "fa_get_device_error")
    return code.value


# --------------------------------------------------------------------------
# decode with cache append (+ RoPE)
# --------------------------------------------------------------------------
def decode_append_workspace_size(B: int, Hq: int, d: int, num_splits: int) -> int:
    return int(load_library().fa_decode_append_workspace_size(B, Hq, d, num_splits))


def fa_decode_paged_append(q, k_new, v_new, k_pages, v_pages, block_table, cache_seqlens,
                           num_splits: int, o, lse=None, scale: float = 0.0, rotary_cos=None,
                           rotary_sin=None, rotary_dim: int | None = None,
                           rotary_interleaved: bool = False,
                           workspace: torch.Tensor | None = None, stream=None) -> None:
    """Calls ``fa_decode_paged_append``: writes k_new/v_new (k rotated when
    tables are given) into the page pool at cache_seqlens, then attends.
    k_pages / v_pages are modified in place; cache_seqlens is not."""
    B, Hq, Hkv, d, num_pages, page_size, max_blocks = _decode_shapes(
        q, k_pages, v_pages, block_table, cache_seqlens, torch.bfloat16, o, lse)
    for t, n in ((k_new, "k_new"), (v_new, "v_new")):
        _need(t, n, torch.bfloat16, 3, (B, Hkv, d))
    _on_cuda(k_new=k_new, v_new=v_new)
    max_pos, rd = 0, 0
    if (rotary_cos is None) != (rotary_sin is None):
        raise ValueError("give both rotary_cos and rotary_sin, or neither")
    if rotary_cos is not None:
        _need(rotary_cos, "rotary_cos", torch.float32, 2)
        _need(rotary_sin, "rotary_sin", torch.float32, 2)
        _on_cuda(rotary_cos=rotary_cos, rotary_sin=rotary_sin)
        if rotary_sin.shape != rotary_cos.shape:
            raise ValueError("rotary_cos and rotary_sin shapes differ")
        max_pos = rotary_cos.shape[0]
        rd = int(rotary_dim) if rotary_dim is not None else 2 * rotary_cos.shape[1]
        if rotary_cos.shape[1] != rd // 2:
            raise ValueError("rotary tables need rotary_dim / 2 columns")
    ws_bytes = 0
    if workspace is not None:
        if not workspace.is_cuda or not workspace.is_contiguous():
            raise ValueError("workspace must be a contiguous CUDA tensor")
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(load_library().fa_decode_paged_append(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pages), _ptr(v_pages), _ptr(block_table),
        _ptr(cache_seqlens), page_size, int(num_splits), _ptr(o), _stream(stream), B, Hq, Hkv, d,
        max_blocks, num_pages, float(scale), _ptr(lse), _ptr(rotary_cos), _ptr(rotary_sin),
        max_pos, rd, int(bool(rotary_interleaved)), _ptr(workspace), ws_bytes),
        "fa_decode_paged_append")


def decode_paged_append(q, k_new, v_new, k_pages, v_pages, block_table, cache_seqlens,
                        num_splits: int = 0, scale: float = 0.0, rotary_cos=None, rotary_sin=None,
                        rotary_dim: int | None = None, rotary_interleaved: bool = False,
                        return_lse: bool = True, stream=None):
    """Allocates O (and LSE) and runs ``fa_decode_paged_append``.  Returns (o, lse or None)."""
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=q.device) if return_lse else None
    fa_decode_paged_append(q, k_new, v_new, k_pages, v_pages, block_table, cache_seqlens,
                           num_splits, o, lse, scale, rotary_cos, rotary_sin, rotary_dim,
                           rotary_interleaved, None, stream)
    return o, lse
