"""Python binding for the exact tiled attention library (``include/attn.h``).

Argument marshalling only: every function checks shapes and dtypes of torch
tensors, then calls the C entry point of the same name with raw device
pointers and the current CUDA stream. All arithmetic runs in the CUDA kernels
of ``libattn.so``; there is no fallback path. If the library is missing or
cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn.so")

ATTN_OK = 0
ATTN_ERR_INVALID = -1
ATTN_ERR_UNSUPPORTED = -2
ATTN_ERR_CUDA = -3
ATTN_ERR_TIMEOUT = -4
ATTN_ERR_SCRATCH = -5

# name -> (restype, argtypes); mirrors include/attn.h
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
SIGNATURES = {
    "attn_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "attn_fwd_f16": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "attn_decode": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _P]),
    "attn_decode_f16": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _P]),
    "attn_decode_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _P]),
    "attn_decode_num_splits": (_I, [_I, _I, _I, _I]),
    "attn_strerror": (ctypes.c_char_p, [_I]),
    "attn_get_device_status": (_I, [_P, ctypes.POINTER(ctypes.c_uint)]),
    "attn_fwd_stall_test": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I,
                                 ctypes.c_uint, _P]),
    "attn_fwd_window": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "attn_fwd_window_f16": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "attn_decode_window": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "attn_decode_window_f16": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "attn_last_cuda_error": (_I, []),
    "attn_merge": (_I, [_P, _P, _P, _P, _P, ctypes.c_longlong, _I, _P]),
    "attn_merge_f16": (_I, [_P, _P, _P, _P, _P, ctypes.c_longlong, _I, _P]),
    "attn_fwd_partial": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "attn_fwd_partial_f16": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "attn_merge_partial": (_I, [_P, _P, _P, _P, _P, ctypes.c_longlong, _I, _P]),
    "attn_merge_partial_f16": (_I, [_P, _P, _P, _P, _P, ctypes.c_longlong, _I, _P]),
}

_lib = None


class AttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        self.cuda_error = load_library().attn_last_cuda_error() if code == ATTN_ERR_CUDA else 0
        extra = f", cudaError {self.cuda_error}" if self.cuda_error else ""
        super().__init__(f"{where}: {strerror(code)} (code {code}{extra})")


def load_library(path: str = LIB_PATH):
    """Load ``libattn.so`` (once). Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is not built; run `python -m exact_tiled_attention_38_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def strerror(code: int) -> str:
    return load_library().attn_strerror(int(code)).decode()


def _stream_handle(stream) -> Optional[int]:
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return stream or None
    return stream.cuda_stream or None


def _check(code: int, where: str):
    if code != ATTN_OK:
        raise AttnError(code, where)


def _dev(t, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _on_device(*tensors):
    """The library works on the current CUDA device: every tensor of a call must
    live on one device, which is made current for the call (and whose current
    stream is used when none is given)."""
    import torch

    devs = {t.device for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError(f"all tensors of a call must be on one CUDA device, got {sorted(map(str, devs))}")
    return torch.cuda.device(next(iter(devs)))


def _fwd(fname, dtype, q, k, v, o, lse, scale, causal, stream, want_lse, window=None,
         out_dtype=None):
    import torch

    out_dtype = out_dtype or dtype
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
        if t.dtype != dtype or t.dim() != 4:
            raise ValueError(f"{n} must be a 4-D {dtype} tensor [B, H, N, d]")
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if Bk != B or dk != d or tuple(v.shape) != tuple(k.shape):
        raise ValueError("q/k/v shapes disagree")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty(q.shape, device=q.device, dtype=out_dtype)
    _dev(o, "o")
    if o.dtype != out_dtype or tuple(o.shape) != tuple(q.shape):
        raise ValueError(f"o must be a {out_dtype} tensor of q's shape")
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Nq), device=q.device, dtype=torch.float32)
    if lse is not None:
        _dev(lse, "lse")
        if lse.dtype != torch.float32 or tuple(lse.shape) != (B, Hq, Nq):
            raise ValueError("lse must be float32 [B, Hq, Nq]")
    fn = getattr(load_library(), fname)
    with _on_device(q, k, v, o, lse):
        code = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                  lse.data_ptr() if lse is not None else None, B, Hq, Hkv, Nq, Nk, d,
                  float(scale), *((int(window),) if window is not None else (1 if causal else 0,)),
                  _stream_handle(stream))
    _check(code, fname)
    return o, lse


def attn_fwd(q, k, v, o=None, lse=None, scale: Optional[float] = None, causal: bool = False,
             stream=None, want_lse: bool = True) -> Tuple:
    """Prefill attention, bf16. q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d] -> (o, lse)."""
    import torch

    return _fwd("attn_fwd", torch.bfloat16, q, k, v, o, lse, scale, causal, stream, want_lse)


def attn_fwd_f16(q, k, v, o=None, lse=None, scale: Optional[float] = None,
                 causal: bool = False, stream=None, want_lse: bool = True) -> Tuple:
    """Prefill attention, fp16."""
    import torch

    return _fwd("attn_fwd_f16", torch.float16, q, k, v, o, lse, scale, causal, stream,
                want_lse)


def attn_fwd_partial(q, k, v, o=None, lse=None, scale: Optional[float] = None,
                     causal: bool = False, stream=None, want_lse: bool = True) -> Tuple:
    """Prefill attention with O kept in float32 (unrounded), for results that
    are merged further (``attn_merge`` with a float32 ``o_part``). q, k, v bf16
    or fp16; returns (o float32 [B,Hq,Nq,d], lse)."""
    import torch

    if q.dtype == torch.float16:
        name, dt = "attn_fwd_partial_f16", torch.float16
    else:
        name, dt = "attn_fwd_partial", torch.bfloat16
    return _fwd(name, dt, q, k, v, o, lse, scale, causal, stream, want_lse,
                out_dtype=torch.float32)


def _decode(fname, dtype, q, kcache, vcache, seqlens, Hkv, o, lse, scale, stream, want_lse,
            window=None):
    import torch

    for t, n in ((q, "q"), (kcache, "kcache"), (vcache, "vcache"), (seqlens, "seqlens")):
        _dev(t, n)
    if q.dtype != dtype or q.dim() != 3:
        raise ValueError(f"q must be a 3-D {dtype} tensor [B, Hq, d]")
    if kcache.dtype != dtype or vcache.dtype != dtype:
        raise ValueError(f"caches must be {dtype}")
    if seqlens.dtype != torch.int32:
        raise ValueError("seqlens must be int32")
    B, Hq, d = q.shape
    if seqlens.numel() != B:
        raise ValueError("seqlens must have B entries")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty_like(q)
    _dev(o, "o")
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), device=q.device, dtype=torch.float32)
    fn = getattr(load_library(), fname)
    with _on_device(q, kcache, vcache, seqlens, o, lse):
        code = fn(q.data_ptr(), kcache.data_ptr(), vcache.data_ptr(), seqlens.data_ptr(),
                  o.data_ptr(), lse.data_ptr() if lse is not None else None, B, Hq, Hkv, d,
                  float(scale), *((int(window),) if window is not None else ()),
                  _stream_handle(stream))
    _check(code, fname)
    return o, lse


def attn_fwd_window(q, k, v, window: int, o=None, lse=None, scale: Optional[float] = None,
                    stream=None, want_lse: bool = True) -> Tuple:
    """Causal prefill with a sliding window of `window` keys, bf16 (fp16 if q is fp16)."""
    import torch

    name, dt = (("attn_fwd_window_f16", torch.float16) if q.dtype == torch.float16
                else ("attn_fwd_window", torch.bfloat16))
    return _fwd(name, dt, q, k, v, o, lse, scale, True, stream, want_lse, window=window)


def attn_decode_window(q, kcache, vcache, seqlens, Hkv: int, window: int, o=None, lse=None,
                       scale: Optional[float] = None, stream=None, want_lse: bool = True):
    """Decode reading the last `window` cached tokens, bf16 (fp16 if q is fp16)."""
    import torch

    name, dt = (("attn_decode_window_f16", torch.float16) if q.dtype == torch.float16
                else ("attn_decode_window", torch.bfloat16))
    return _decode(name, dt, q, kcache, vcache, seqlens, Hkv, o, lse, scale, stream, want_lse,
                   window=window)


def attn_decode(q, kcache, vcache, seqlens, Hkv: int, o=None, lse=None,
                scale: Optional[float] = None, stream=None, want_lse: bool = True):
    """One-token decode over a packed ragged cache, bf16. Returns (o [B,Hq,d], lse [B,Hq])."""
    import torch

    return _decode("attn_decode", torch.bfloat16, q, kcache, vcache, seqlens, Hkv, o, lse,
                   scale, stream, want_lse)


def attn_decode_f16(q, kcache, vcache, seqlens, Hkv: int, o=None, lse=None,
                    scale: Optional[float] = None, stream=None, want_lse: bool = True):
    """One-token decode, fp16."""
    import torch

    return _decode("attn_decode_f16", torch.float16, q, kcache, vcache, seqlens, Hkv, o, lse,
                   scale, stream, want_lse)


def attn_decode_noalloc(q, kcache, vcache, seqlens, Hkv: int, o=None, lse=None,
                        scale: Optional[float] = None, stream=None, want_lse: bool = True):
    """bf16 decode whose scratch is the library's fixed device array.

    For callers that cannot allocate device memory where decode runs. The
    library allocates nothing here; pass preallocated ``o`` / ``lse`` to keep
    this wrapper from allocating them either. Calls that may overlap on the GPU
    share the scratch and must be ordered (one stream, or events).
    """
    import torch

    return _decode("attn_decode_noalloc", torch.bfloat16, q, kcache, vcache, seqlens, Hkv, o,
                   lse, scale, stream, want_lse)


def attn_merge(o_acc, lse_acc, o_part, lse_part, o_out=None, stream=None) -> None:
    """Fold a partial result (o_part, lse_part) into the fp32 accumulator in place.

    o_acc float32 [..., d] and lse_acc float32 [...] (same leading shape as
    o_part / lse_part); o_part bf16, fp16 or float32 (an unrounded partial from
    ``attn_fwd_partial``); o_out (optional, o_part's shape; bf16 or fp16, o_part's
    dtype unless o_part is float32) also receives the merged O rounded. A row
    with lse_acc = -inf is empty (o_acc not read). Runs ``attn_merge`` /
    ``attn_merge_f16``, or ``attn_merge_partial`` / ``attn_merge_partial_f16``.
    """
    import torch

    for t, n in ((o_acc, "o_acc"), (lse_acc, "lse_acc"), (o_part, "o_part"),
                 (lse_part, "lse_part")):
        _dev(t, n)
    if o_part.dtype not in (torch.bfloat16, torch.float16, torch.float32):
        raise ValueError("o_part must be bf16, fp16 or float32")
    if o_acc.dtype != torch.float32 or lse_acc.dtype != torch.float32 or \
            lse_part.dtype != torch.float32:
        raise ValueError("o_acc, lse_acc and lse_part must be float32")
    d = o_part.shape[-1]
    if tuple(o_acc.shape) != tuple(o_part.shape) or \
            tuple(lse_acc.shape) != tuple(o_part.shape[:-1]) or \
            tuple(lse_part.shape) != tuple(o_part.shape[:-1]):
        raise ValueError("o_acc, lse_acc, o_part and lse_part shapes disagree")
    if o_out is not None:
        _dev(o_out, "o_out")
        if tuple(o_out.shape) != tuple(o_part.shape) or (
                o_out.dtype != o_part.dtype if o_part.dtype != torch.float32
                else o_out.dtype not in (torch.bfloat16, torch.float16)):
            raise ValueError("o_out must match o_part's shape (and dtype, or bf16 / fp16 "
                             "for a float32 o_part)")
    if o_part.dtype == torch.float32:
        f16 = o_out is not None and o_out.dtype == torch.float16
        name = "attn_merge_partial_f16" if f16 else "attn_merge_partial"
    else:
        name = "attn_merge_f16" if o_part.dtype == torch.float16 else "attn_merge"
    rows = o_part.numel() // d if d else 0
    with _on_device(o_acc, lse_acc, o_part, lse_part, o_out):
        code = getattr(load_library(), name)(
            o_acc.data_ptr(), lse_acc.data_ptr(), o_part.data_ptr(), lse_part.data_ptr(),
            o_out.data_ptr() if o_out is not None else None, rows, d, _stream_handle(stream))
    _check(code, name)


def attn_decode_num_splits(B: int, Hq: int, Hkv: int, d: int) -> int:
    r = load_library().attn_decode_num_splits(B, Hq, Hkv, d)
    if r < 0:
        raise AttnError(r, "attn_decode_num_splits")
    return r


def attn_get_device_status(stream=None) -> Tuple[int, int]:
    """(status code, raw site code) after synchronising the stream; clears the word."""
    raw = ctypes.c_uint(0)
    code = load_library().attn_get_device_status(_stream_handle(stream), ctypes.byref(raw))
    return code, raw.value
