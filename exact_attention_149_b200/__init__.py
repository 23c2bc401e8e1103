"""Python binding of the exact-attention C ABI (include/fa.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libfa.so``. PyTorch provides device memory and the current
stream; nothing here computes attention, and there is no fallback: if the
library is missing, importing this package raises.

Low-level names mirror the C ABI (``fa_fwd``, ``fa_bwd``, ``fa_fwd_kvcache``,
``fa_bwd_workspace_size``, ``fa_kvcache_workspace_size``,
``fa_get_device_status``, ``fa_last_error``, ``fa_version``) and take torch
tensors where the C call takes pointers. ``fwd``, ``bwd`` and
``fwd_kvcache`` additionally allocate outputs and workspaces with torch.
"""

from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "LIB_PATH", "FaError", "lib",
    "fa_fwd", "fa_bwd", "fa_fwd_kvcache", "fa_fwd_kvcache_noalloc", "fa_bwd_workspace_size",
    "fa_kvcache_workspace_size", "FA_NOALLOC_SCRATCH_BYTES",
    "fa_get_device_status", "fa_last_error", "fa_version",
    "fa_kernel_timing_enable", "fa_kernel_timing_read", "fa_kernel_timing_reset",
    "fwd", "bwd", "fwd_kvcache", "fwd_qkvpacked", "bwd_qkvpacked", "fa_fwd_qkvpacked",
    "fa_bwd_qkvpacked", "fa_fwd_kvcache_int8", "fa_kv_quantize_int8", "kv_quantize_int8",
    "fa_fwd_kvcache_int4", "fa_kv_quantize_int4", "kv_quantize_int4",
    "fa_fwd_fp8", "fwd_fp8", "fa_selftest_poly", "fa_selftest_fwd_timeout",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa.so")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(5)
_STATUS = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_CUDA",
           4: "FA_ERR_TIMEOUT"}
_DTYPE = {torch.bfloat16: 0, torch.float16: 1}


class FaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python exact_attention_149_b200/build.py` "
        "(nvcc, sm_100a). There is no CPU or library fallback.")

lib = ctypes.CDLL(LIB_PATH)

_p = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_z = ctypes.c_size_t

lib.fa_fwd.restype = _i
lib.fa_fwd.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _i, _i, _i, _f, _p, _i, _p, _i,
                       _i, _p]
lib.fa_fwd_fp8.restype = _i
lib.fa_fwd_fp8.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _f, _f, _f, _i, _i, _i, _f,
                           _p, _i, _p, _i, _i, _p]
lib.fa_selftest_fwd_timeout.restype = _i
lib.fa_selftest_fwd_timeout.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _f, ctypes.c_ulonglong, _i, _p]
lib.fa_selftest_poly.restype = _i
lib.fa_selftest_poly.argtypes = [_i, _p, _p, _p, _i, _p]
lib.fa_bwd.restype = _i
lib.fa_bwd.argtypes = [_p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _i, _i, _i, _f,
                       _p, _i, _p, _i, _i, _p, _z, _p]
lib.fa_fwd_qkvpacked.restype = _i
lib.fa_fwd_qkvpacked.argtypes = [_p, _p, _p, _i, _i, _i, _i, _f, _i, _i, _i, _f, _p, _i, _p, _i, _i,
                                 _p]
lib.fa_bwd_qkvpacked.restype = _i
lib.fa_bwd_qkvpacked.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _f, _i, _i, _i, _f, _p, _i, _p,
                                 _i, _i, _p, _z, _p]
lib.fa_fwd_kvcache.restype = _i
# q, k_new, v_new, k_cache, v_cache, block_table, cache_seqlens, rotary_cos, rotary_sin, out, lse;
# B, Sq, Hq, Hkv, D, page_size, max_pages_per_seq, num_pages, rotary_rows, rotary_dim,
# rotary_interleaved; scale, causal, window_left, window_right, softcap, alibi_slopes,
# alibi_batch_stride, num_splits, dtype
_KV_ARGS = [_p] * 11 + [_i] * 11 + [_f, _i, _i, _i, _f, _p, _i, _i, _i]
lib.fa_fwd_kvcache.restype = _i
lib.fa_fwd_kvcache.argtypes = _KV_ARGS + [_p, _z, _p]
lib.fa_fwd_kvcache_noalloc.restype = _i
lib.fa_fwd_kvcache_noalloc.argtypes = _KV_ARGS + [_p]
# as _KV_ARGS with k_scale, v_scale after v_cache
lib.fa_fwd_kvcache_int8.restype = _i
lib.fa_fwd_kvcache_int8.argtypes = [_p] * 13 + _KV_ARGS[11:] + [_p, _z, _p]
lib.fa_kv_quantize_int8.restype = _i
lib.fa_kv_quantize_int8.argtypes = [_p, _p, _p, _i, _i, _i, _i, _i, _p]
lib.fa_fwd_kvcache_int4.restype = _i
lib.fa_fwd_kvcache_int4.argtypes = [_p] * 13 + _KV_ARGS[11:] + [_p, _z, _p]
lib.fa_kv_quantize_int4.restype = _i
lib.fa_kv_quantize_int4.argtypes = [_p, _p, _p, _i, _i, _i, _i, _i, _p]
lib.fa_bwd_workspace_size.restype = _z
lib.fa_bwd_workspace_size.argtypes = [_i, _i, _i, _i, _i]
lib.fa_kvcache_workspace_size.restype = _z
lib.fa_kvcache_workspace_size.argtypes = [_i, _i, _i, _i, _i, _i]
lib.fa_get_device_status.restype = _i
lib.fa_get_device_status.argtypes = [ctypes.POINTER(_i)]
lib.fa_kernel_timing_enable.restype = _i
lib.fa_kernel_timing_enable.argtypes = [_i]
lib.fa_kernel_timing_read.restype = _i
lib.fa_kernel_timing_read.argtypes = [ctypes.c_char_p, ctypes.POINTER(_f), ctypes.POINTER(_i)]
lib.fa_kernel_timing_reset.restype = _i
lib.fa_kernel_timing_reset.argtypes = []
lib.fa_last_error.restype = ctypes.c_char_p
lib.fa_last_error.argtypes = []
lib.fa_version.restype = ctypes.c_char_p
lib.fa_version.argtypes = []


def fa_last_error() -> str:
    return lib.fa_last_error().decode()


def fa_version() -> str:
    return lib.fa_version().decode()


def _check(status: int):
    if status != FA_OK:
        raise FaError(status, fa_last_error())


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dt(t) -> int:
    if t.dtype not in _DTYPE:
        raise FaError(FA_ERR_INVALID_ARG, f"dtype {t.dtype} not supported (bf16/fp16)")
    return _DTYPE[t.dtype]


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not isinstance(t, int):
            if not t.is_cuda:
                raise FaError(FA_ERR_INVALID_ARG, "tensors must live on a CUDA device")
            if not t.is_contiguous():
                raise FaError(FA_ERR_INVALID_ARG, "tensors must be contiguous")


# ---------------------------------------------------------------------------
# C-ABI mirrors
# ---------------------------------------------------------------------------
def fa_fwd(q, k, v, out, lse, B, Hq, Hkv, S, D, scale, causal, window_left, window_right,
           softcap, alibi_slopes, alibi_batch_stride, cu_seqlens, total_tokens, dtype, stream=None):
    _check(lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, S, D, scale,
                      int(causal), window_left, window_right, softcap, _ptr(alibi_slopes),
                      alibi_batch_stride, _ptr(cu_seqlens), total_tokens, dtype, _stream(stream)))


def fa_fwd_fp8(q, k, v, out, lse, B, Hq, Hkv, S, D, scale, q_descale, k_descale, v_descale,
               causal, window_left, window_right, softcap, alibi_slopes, alibi_batch_stride,
               cu_seqlens, total_tokens, out_dtype, stream=None):
    _check(lib.fa_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, S, D, scale,
                          q_descale, k_descale, v_descale, int(causal), window_left, window_right,
                          softcap, _ptr(alibi_slopes), alibi_batch_stride, _ptr(cu_seqlens),
                          total_tokens, out_dtype, _stream(stream)))


def fa_selftest_fwd_timeout(q, k, v, out, lse, B, H, S, scale, wait_limit_ns, dtype, stream=None):
    _check(lib.fa_selftest_fwd_timeout(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, S,
                                       scale, wait_limit_ns, dtype, _stream(stream)))


def fa_selftest_poly(which, x, out_poly, out_ref, n, stream=None):
    _check(lib.fa_selftest_poly(which, _ptr(x), _ptr(out_poly), _ptr(out_ref), n, _stream(stream)))


def fa_fwd_qkvpacked(qkv, out, lse, B, H, S, D, scale, causal, window_left, window_right, softcap,
                     alibi_slopes, alibi_batch_stride, cu_seqlens, total_tokens, dtype, stream=None):
    _check(lib.fa_fwd_qkvpacked(_ptr(qkv), _ptr(out), _ptr(lse), B, H, S, D, scale, int(causal),
                                window_left, window_right, softcap, _ptr(alibi_slopes),
                                alibi_batch_stride, _ptr(cu_seqlens), total_tokens, dtype,
                                _stream(stream)))


def fa_bwd_qkvpacked(qkv, out, lse, dout, dqkv, B, H, S, D, scale, causal, window_left,
                     window_right, softcap, alibi_slopes, alibi_batch_stride, cu_seqlens,
                     total_tokens, dtype, workspace, workspace_bytes, stream=None):
    _check(lib.fa_bwd_qkvpacked(_ptr(qkv), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dqkv), B, H, S, D,
                                scale, int(causal), window_left, window_right, softcap,
                                _ptr(alibi_slopes), alibi_batch_stride, _ptr(cu_seqlens),
                                total_tokens, dtype, _ptr(workspace), workspace_bytes,
                                _stream(stream)))


def fa_bwd_workspace_size(B, Hq, S, D, total_tokens=0) -> int:
    return int(lib.fa_bwd_workspace_size(B, Hq, S, D, total_tokens))


def fa_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv, S, D, scale, causal, window_left,
           window_right, softcap, alibi_slopes, alibi_batch_stride, cu_seqlens, total_tokens, dtype,
           workspace, workspace_bytes, stream=None):
    _check(lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq),
                      _ptr(dk), _ptr(dv), B, Hq, Hkv, S, D, scale, int(causal), window_left,
                      window_right, softcap, _ptr(alibi_slopes), alibi_batch_stride,
                      _ptr(cu_seqlens), total_tokens, dtype, _ptr(workspace), workspace_bytes,
                      _stream(stream)))


def fa_kvcache_workspace_size(B, Sq, Hq, D, num_splits, rotary_dim=0) -> int:
    return int(lib.fa_kvcache_workspace_size(B, Sq, Hq, D, num_splits, rotary_dim))


def fa_fwd_kvcache(q, k_new, v_new, k_cache, v_cache, block_table, cache_seqlens, rotary_cos,
                   rotary_sin, out, lse, B, Sq, Hq, Hkv, D, page_size, max_pages_per_seq,
                   num_pages, rotary_rows, rotary_dim, rotary_interleaved, scale, causal,
                   window_left, window_right, softcap, alibi_slopes, alibi_batch_stride,
                   num_splits, dtype, workspace, workspace_bytes, stream=None):
    _check(lib.fa_fwd_kvcache(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                              _ptr(block_table), _ptr(cache_seqlens), _ptr(rotary_cos),
                              _ptr(rotary_sin), _ptr(out), _ptr(lse), B, Sq, Hq, Hkv, D, page_size,
                              max_pages_per_seq, num_pages, rotary_rows, rotary_dim,
                              int(rotary_interleaved), scale, int(causal), window_left,
                              window_right, softcap, _ptr(alibi_slopes), alibi_batch_stride,
                              num_splits, dtype, _ptr(workspace), workspace_bytes,
                              _stream(stream)))


def fa_fwd_kvcache_int8(q, k_new, v_new, k_cache, v_cache, k_scale, v_scale, block_table,
                        cache_seqlens, rotary_cos, rotary_sin, out, lse, B, Sq, Hq, Hkv, D,
                        page_size, max_pages_per_seq, num_pages, rotary_rows, rotary_dim,
                        rotary_interleaved, scale, causal, window_left, window_right, softcap,
                        alibi_slopes, alibi_batch_stride, num_splits, dtype, workspace,
                        workspace_bytes, stream=None):
    _check(lib.fa_fwd_kvcache_int8(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                   _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), _ptr(block_table),
                                   _ptr(cache_seqlens), _ptr(rotary_cos), _ptr(rotary_sin),
                                   _ptr(out), _ptr(lse), B, Sq, Hq, Hkv, D, page_size,
                                   max_pages_per_seq, num_pages, rotary_rows, rotary_dim,
                                   int(rotary_interleaved), scale, int(causal), window_left,
                                   window_right, softcap, _ptr(alibi_slopes), alibi_batch_stride,
                                   num_splits, dtype, _ptr(workspace), workspace_bytes,
                                   _stream(stream)))


def fa_kv_quantize_int8(src, codes, scales, num_pages, page_size, Hkv, D, dtype, stream=None):
    _check(lib.fa_kv_quantize_int8(_ptr(src), _ptr(codes), _ptr(scales), num_pages, page_size,
                                   Hkv, D, dtype, _stream(stream)))


def fa_fwd_kvcache_int4(q, k_new, v_new, k_cache, v_cache, k_scale, v_scale, block_table,
                        cache_seqlens, rotary_cos, rotary_sin, out, lse, B, Sq, Hq, Hkv, D,
                        page_size, max_pages_per_seq, num_pages, rotary_rows, rotary_dim,
                        rotary_interleaved, scale, causal, window_left, window_right, softcap,
                        alibi_slopes, alibi_batch_stride, num_splits, dtype, workspace,
                        workspace_bytes, stream=None):
    _check(lib.fa_fwd_kvcache_int4(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                   _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), _ptr(block_table),
                                   _ptr(cache_seqlens), _ptr(rotary_cos), _ptr(rotary_sin),
                                   _ptr(out), _ptr(lse), B, Sq, Hq, Hkv, D, page_size,
                                   max_pages_per_seq, num_pages, rotary_rows, rotary_dim,
                                   int(rotary_interleaved), scale, int(causal), window_left,
                                   window_right, softcap, _ptr(alibi_slopes), alibi_batch_stride,
                                   num_splits, dtype, _ptr(workspace), workspace_bytes,
                                   _stream(stream)))


def fa_kv_quantize_int4(src, codes, scales, num_pages, page_size, Hkv, D, dtype, stream=None):
    _check(lib.fa_kv_quantize_int4(_ptr(src), _ptr(codes), _ptr(scales), num_pages, page_size,
                                   Hkv, D, dtype, _stream(stream)))


# size of the library's static scratch array used by fa_fwd_kvcache_noalloc
FA_NOALLOC_SCRATCH_BYTES = 24 * 1024 * 1024


def fa_fwd_kvcache_noalloc(q, k_new, v_new, k_cache, v_cache, block_table, cache_seqlens,
                           rotary_cos, rotary_sin, out, lse, B, Sq, Hq, Hkv, D, page_size,
                           max_pages_per_seq, num_pages, rotary_rows, rotary_dim,
                           rotary_interleaved, scale, causal, window_left, window_right, softcap,
                           alibi_slopes, alibi_batch_stride, num_splits, dtype, stream=None):
    """fa_fwd_kvcache for callers that cannot allocate device memory: no
    workspace argument; the split partials and rotated queries live in the
    library's own static device array (see include/fa.h)."""
    _check(lib.fa_fwd_kvcache_noalloc(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                      _ptr(v_cache), _ptr(block_table), _ptr(cache_seqlens),
                                      _ptr(rotary_cos), _ptr(rotary_sin), _ptr(out), _ptr(lse), B,
                                      Sq, Hq, Hkv, D, page_size, max_pages_per_seq, num_pages,
                                      rotary_rows, rotary_dim, int(rotary_interleaved), scale,
                                      int(causal), window_left, window_right, softcap,
                                      _ptr(alibi_slopes), alibi_batch_stride, num_splits, dtype,
                                      _stream(stream)))


def fa_kernel_timing_enable(enable: bool = True):
    _check(lib.fa_kernel_timing_enable(int(bool(enable))))


def fa_kernel_timing_reset():
    _check(lib.fa_kernel_timing_reset())


def fa_kernel_timing_read(name: str):
    """(total milliseconds, launches) of kernel `name` since the last reset,
    from CUDA events the library recorded around each launch."""
    ms = ctypes.c_float(0.0)
    n = ctypes.c_int(0)
    _check(lib.fa_kernel_timing_read(name.encode(), ctypes.byref(ms), ctypes.byref(n)))
    return float(ms.value), int(n.value)


def fa_get_device_status() -> int:
    v = ctypes.c_int(0)
    _check(lib.fa_get_device_status(ctypes.byref(v)))
    return v.value


# ---------------------------------------------------------------------------
# tensor-level conveniences (allocation through torch only)
# ---------------------------------------------------------------------------
def _scale(scale, D):
    return float(D) ** -0.5 if scale is None else float(scale)


def _alibi(alibi_slopes, Hq):
    """(tensor, batch stride) for the C ABI: None, a float32 (Hq,) vector
    (stride 0) or a float32 (B, Hq) array with contiguous rows."""
    if alibi_slopes is None:
        return None, 0
    _need_cuda(alibi_slopes)
    if alibi_slopes.dtype != torch.float32 or alibi_slopes.shape[-1] != Hq or alibi_slopes.dim() > 2:
        raise FaError(FA_ERR_INVALID_ARG, "alibi_slopes must be float32 (Hq,) or (B, Hq)")
    return alibi_slopes, (0 if alibi_slopes.dim() == 1 else alibi_slopes.stride(0))


def fwd(q, k, v, scale=None, causal=False, window=(-1, -1), softcap=0.0, cu_seqlens=None,
        max_seqlen=None, out=None, lse=None, alibi_slopes=None, stream=None):
    """q (B,S,Hq,D), k/v (B,S,Hkv,D) -> (out, lse (B,Hq,S)); varlen: q (T,Hq,D),
    cu_seqlens int32 (B+1) on the device, lse (Hq,T). alibi_slopes: float32
    (Hq,) or (B, Hq) on the device."""
    _need_cuda(q, k, v, cu_seqlens)
    if cu_seqlens is None:
        B, S, Hq, D = q.shape
        Hkv = k.shape[2]
        T = 0
        lse_shape = (B, Hq, S)
    else:
        T, Hq, D = q.shape
        Hkv = k.shape[1]
        B = cu_seqlens.numel() - 1
        if max_seqlen is None:
            raise FaError(FA_ERR_INVALID_ARG, "max_seqlen is required with cu_seqlens")
        S = int(max_seqlen)
        lse_shape = (Hq, T)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=q.device)
    al, als = _alibi(alibi_slopes, Hq)
    fa_fwd(q, k, v, out, lse, B, Hq, Hkv, S, D, _scale(scale, D), causal, window[0], window[1],
           softcap, al, als, cu_seqlens, T, _dt(q), stream)
    return out, lse


_FP8_IN = (torch.uint8, torch.float8_e4m3fn)


def fwd_fp8(q, k, v, q_descale, k_descale, v_descale, scale=None, causal=False, window=(-1, -1),
            softcap=0.0, cu_seqlens=None, max_seqlen=None, out=None, lse=None, alibi_slopes=None,
            out_dtype=torch.bfloat16, stream=None):
    """FP8 forward: q, k, v are E4M3 codes (uint8 bit patterns or
    torch.float8_e4m3fn) in fwd's layouts, each tensor with a float descale;
    out in out_dtype (bf16 / fp16), lse float32 as in fwd."""
    _need_cuda(q, k, v, cu_seqlens)
    for t in (q, k, v):
        if t.dtype not in _FP8_IN:
            raise FaError(FA_ERR_INVALID_ARG, "fwd_fp8 takes uint8 or float8_e4m3fn q, k, v")
    if cu_seqlens is None:
        B, S, Hq, D = q.shape
        Hkv = k.shape[2]
        T = 0
        lse_shape = (B, Hq, S)
    else:
        T, Hq, D = q.shape
        Hkv = k.shape[1]
        B = cu_seqlens.numel() - 1
        if max_seqlen is None:
            raise FaError(FA_ERR_INVALID_ARG, "max_seqlen is required with cu_seqlens")
        S = int(max_seqlen)
        lse_shape = (Hq, T)
    if out_dtype not in _DTYPE:
        raise FaError(FA_ERR_INVALID_ARG, f"out_dtype {out_dtype} not supported (bf16/fp16)")
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    if lse is None:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=q.device)
    al, als = _alibi(alibi_slopes, Hq)
    fa_fwd_fp8(q, k, v, out, lse, B, Hq, Hkv, S, D, _scale(scale, D), float(q_descale),
               float(k_descale), float(v_descale), causal, window[0], window[1], softcap, al, als,
               cu_seqlens, T, _DTYPE[out.dtype], stream)
    return out, lse


def bwd(q, k, v, out, lse, dout, scale=None, causal=False, window=(-1, -1), softcap=0.0,
        cu_seqlens=None, max_seqlen=None, dq=None, dk=None, dv=None, workspace=None,
        alibi_slopes=None, stream=None):
    """Gradients (dq, dk, dv) of sum(out * dout); layouts as in fwd."""
    _need_cuda(q, k, v, out, lse, dout, cu_seqlens)
    if cu_seqlens is None:
        B, S, Hq, D = q.shape
        Hkv = k.shape[2]
        T = 0
    else:
        T, Hq, D = q.shape
        Hkv = k.shape[1]
        B = cu_seqlens.numel() - 1
        S = int(max_seqlen)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    nbytes = fa_bwd_workspace_size(B, Hq, S, D, T)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    al, als = _alibi(alibi_slopes, Hq)
    fa_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv, S, D, _scale(scale, D), causal,
           window[0], window[1], softcap, al, als, cu_seqlens, T, _dt(q), workspace,
           workspace.numel(), stream)
    return dq, dk, dv


def _packed_dims(qkv, cu_seqlens, max_seqlen):
    if cu_seqlens is None:
        B, S, three, H, D = qkv.shape
        return B, S, H, D, 0
    T, three, H, D = qkv.shape
    if max_seqlen is None:
        raise FaError(FA_ERR_INVALID_ARG, "max_seqlen is required with cu_seqlens")
    return cu_seqlens.numel() - 1, int(max_seqlen), H, D, T


def fwd_qkvpacked(qkv, scale=None, causal=False, window=(-1, -1), softcap=0.0, cu_seqlens=None,
                  max_seqlen=None, out=None, lse=None, alibi_slopes=None, stream=None):
    """qkv (B,S,3,H,D) (varlen: (T,3,H,D)) -> (out (B,S,H,D), lse (B,H,S));
    the three tensors are read in place."""
    _need_cuda(qkv, cu_seqlens)
    B, S, H, D, T = _packed_dims(qkv, cu_seqlens, max_seqlen)
    if out is None:
        out = torch.empty(qkv.shape[:-3] + (H, D), dtype=qkv.dtype, device=qkv.device)
    if lse is None:
        shape = (B, H, S) if cu_seqlens is None else (H, T)
        lse = torch.empty(shape, dtype=torch.float32, device=qkv.device)
    al, als = _alibi(alibi_slopes, H)
    fa_fwd_qkvpacked(qkv, out, lse, B, H, S, D, _scale(scale, D), causal, window[0], window[1],
                     softcap, al, als, cu_seqlens, T, _dt(qkv), stream)
    return out, lse


def bwd_qkvpacked(qkv, out, lse, dout, scale=None, causal=False, window=(-1, -1), softcap=0.0,
                  cu_seqlens=None, max_seqlen=None, dqkv=None, workspace=None, alibi_slopes=None,
                  stream=None):
    """Gradient dqkv, packed like qkv, of sum(out * dout)."""
    _need_cuda(qkv, out, lse, dout, cu_seqlens)
    B, S, H, D, T = _packed_dims(qkv, cu_seqlens, max_seqlen)
    dqkv = torch.empty_like(qkv) if dqkv is None else dqkv
    nbytes = fa_bwd_workspace_size(B, H, S, D, T)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=qkv.device)
    al, als = _alibi(alibi_slopes, H)
    fa_bwd_qkvpacked(qkv, out, lse, dout, dqkv, B, H, S, D, _scale(scale, D), causal, window[0],
                     window[1], softcap, al, als, cu_seqlens, T, _dt(qkv), workspace,
                     workspace.numel(), stream)
    return dqkv


def fwd_kvcache(q, k_cache, v_cache, cache_seqlens, block_table, k_new=None, v_new=None,
                rotary_cos=None, rotary_sin=None, rotary_interleaved=False, scale=None,
                causal=True, window=(-1, -1), softcap=0.0, num_splits=1, out=None, lse=None,
                workspace=None, alibi_slopes=None, stream=None, k_scale=None, v_scale=None):
    """One decode step: q (B,Sq,Hq,D); caches (num_pages, page_size, Hkv, D)
    with block_table int32 (B, max_pages), or block_table None and contiguous
    caches (B, capacity, Hkv, D); cache_seqlens int32 (B). Appends
    k_new/v_new (B,Sq,Hkv,D) in place, then attends. rotary_cos/rotary_sin:
    float32 (rows, rotary_dim/2) tables that rotate q and k_new at their
    positions. int8 caches (codes) and int4 caches (uint8, two codes per
    byte: (num_pages, page_size, Hkv, D / 2)) take their float32 row scales
    k_scale, v_scale (num_pages, Hkv, page_size) and run
    fa_fwd_kvcache_int8 / _int4.
    Returns (out (B,Sq,Hq,D), lse (B,Hq,Sq))."""
    q4 = k_cache.dtype == torch.uint8
    q8 = k_cache.dtype == torch.int8 or q4
    if q8 != (k_scale is not None) or (k_scale is None) != (v_scale is None):
        raise FaError(FA_ERR_INVALID_ARG, "int8 caches take k_scale and v_scale; 16-bit caches take neither")
    if q8:
        npg, ps, hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
        if v_cache.dtype != k_cache.dtype or v_cache.shape != k_cache.shape:
            raise FaError(FA_ERR_INVALID_ARG, "k_cache and v_cache must both be int8 of one shape")
        if q4 and k_cache.shape[3] * 2 != q.shape[3]:
            raise FaError(FA_ERR_INVALID_ARG, "an int4 cache's last dim is D / 2")
        for sc in (k_scale, v_scale):
            if sc.dtype != torch.float32 or tuple(sc.shape) != (npg, hkv, ps):
                raise FaError(FA_ERR_INVALID_ARG,
                              f"int8 cache scales must be float32 {(npg, hkv, ps)} (num_pages, Hkv, page_size)")
    _need_cuda(q, k_cache, v_cache, cache_seqlens, block_table, k_new, v_new, rotary_cos,
               rotary_sin, k_scale, v_scale)
    B, Sq, Hq, D = q.shape
    num_pages, page_size, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    max_pages = 1 if block_table is None else block_table.shape[1]
    if (rotary_cos is None) != (rotary_sin is None):
        raise FaError(FA_ERR_INVALID_ARG, "rotary_cos and rotary_sin go together")
    if rotary_cos is not None and (rotary_cos.dtype != torch.float32 or rotary_sin.dtype != torch.float32
                                   or rotary_cos.shape != rotary_sin.shape or rotary_cos.dim() != 2):
        raise FaError(FA_ERR_INVALID_ARG, "rotary tables must be float32 (rows, rotary_dim/2), same shape")
    rot_rows, rot_dim = (0, 0) if rotary_cos is None else (rotary_cos.shape[0], 2 * rotary_cos.shape[1])
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device) if lse is None else lse
    nbytes = fa_kvcache_workspace_size(B, Sq, Hq, D, num_splits, rot_dim)
    if workspace is None and nbytes > 0:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    args = (block_table, cache_seqlens, rotary_cos, rotary_sin, out, lse, B, Sq, Hq, Hkv, D,
            page_size, max_pages, num_pages, rot_rows, rot_dim, rotary_interleaved,
            _scale(scale, D), causal, window[0], window[1], softcap, *_alibi(alibi_slopes, Hq),
            num_splits, _dt(q), workspace, 0 if workspace is None else workspace.numel(), stream)
    if q4:
        fa_fwd_kvcache_int4(q, k_new, v_new, k_cache, v_cache, k_scale, v_scale, *args)
    elif q8:
        fa_fwd_kvcache_int8(q, k_new, v_new, k_cache, v_cache, k_scale, v_scale, *args)
    else:
        fa_fwd_kvcache(q, k_new, v_new, k_cache, v_cache, *args)
    return out, lse


def kv_quantize_int8(cache, codes=None, scales=None, stream=None):
    """A 16-bit cache (num_pages, page_size, Hkv, D) -> (int8 codes of the
    same shape, float32 scales (num_pages, Hkv, page_size)) in the format of
    fa_fwd_kvcache_int8."""
    num_pages, page_size, Hkv, D = cache.shape
    if codes is not None and (codes.dtype != torch.int8 or codes.shape != cache.shape):
        raise FaError(FA_ERR_INVALID_ARG, "codes must be int8 of the cache's shape")
    if scales is not None and (scales.dtype != torch.float32 or
                               tuple(scales.shape) != (num_pages, Hkv, page_size)):
        raise FaError(FA_ERR_INVALID_ARG, "scales must be float32 (num_pages, Hkv, page_size)")
    _need_cuda(cache, codes, scales)
    if codes is None:
        codes = torch.empty(cache.shape, dtype=torch.int8, device=cache.device)
    if scales is None:
        scales = torch.empty((num_pages, Hkv, page_size), dtype=torch.float32, device=cache.device)
    fa_kv_quantize_int8(cache, codes, scales, num_pages, page_size, Hkv, D, _dt(cache), stream)
    return codes, scales


def kv_quantize_int4(cache, codes=None, scales=None, stream=None):
    """A 16-bit cache (num_pages, page_size, Hkv, D) -> (uint8 codes
    (num_pages, page_size, Hkv, D / 2), two per byte, float32 scales
    (num_pages, Hkv, page_size)) in the format of fa_fwd_kvcache_int4."""
    num_pages, page_size, Hkv, D = cache.shape
    if codes is not None and (codes.dtype != torch.uint8 or tuple(codes.shape) != (num_pages, page_size, Hkv, D // 2)):
        raise FaError(FA_ERR_INVALID_ARG, "codes must be uint8 (num_pages, page_size, Hkv, D / 2)")
    if scales is not None and (scales.dtype != torch.float32 or
                               tuple(scales.shape) != (num_pages, Hkv, page_size)):
        raise FaError(FA_ERR_INVALID_ARG, "scales must be float32 (num_pages, Hkv, page_size)")
    _need_cuda(cache, codes, scales)
    if codes is None:
        codes = torch.empty((num_pages, page_size, Hkv, D // 2), dtype=torch.uint8, device=cache.device)
    if scales is None:
        scales = torch.empty((num_pages, Hkv, page_size), dtype=torch.float32, device=cache.device)
    fa_kv_quantize_int4(cache, codes, scales, num_pages, page_size, Hkv, D, _dt(cache), stream)
    return codes, scales
