"""Python binding of libfa_b200 (exact IO-aware attention on B200, sm_100a).

Argument marshalling only: every step of attention runs in the CUDA kernels of
``libfa_b200.so``; there is no CPU or PyTorch fallback. If the library is
missing this import fails (build it with ``python io_aware_exact_27_b200/build.py``).

Two layers:
  * ``fa_fwd``, ``fa_fwd_varlen``, ``fa_fwd_fp8``, ``fa_bwd``, ``fa_bwd_varlen``,
    ``fa_bwd_workspace_size``, ``fa_get_status`` ... — the C entry points of
    ``include/fa_b200.h`` with the same names and arguments; tensors may be
    passed as torch CUDA tensors (their data pointers are used) or raw ints.
    A non-OK status raises ``FAError``.
  * ``attention_fwd`` / ``attention_fwd_varlen`` / ``attention_bwd`` ... —
    allocate the outputs with torch on the inputs' device and call the above
    on the current stream.
"""

from __future__ import annotations

import ctypes
import math
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfa_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python io_aware_exact_27_b200/build.py` "
                      "(nvcc, sm_100a); there is no fallback implementation")

_lib = ctypes.CDLL(LIB_PATH, mode=ctypes.RTLD_LOCAL)

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_Z = ctypes.c_size_t

_SIGS = {
    "fa_fwd": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P],
    "fa_fwd_varlen": [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P],
    "fa_fwd_fp8": [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P],
    "fa_bwd": [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _I, _I, _I, _I, _I, _I, _F, _P],
    "fa_bwd_varlen": [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P],
    "fa_get_status": [_P],
    "fa_fwd_kvcache": [_P, _P, _P, _P, _P, _P, _P, _Z, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P],
    "fa_attn_merge": [_P, _P, _I, _P, _P, _I, _I, _I, _I, _P],
    "fa_fp8_quantize": [_P, _P, _P, _I, _I, _I, _I, _I, _P],
    "fa_fp8_dequantize": [_P, _P, _P, _I, _I, _I, _I, _I, _P],
    "fa_grad_accumulate": [_P, _P, _P, ctypes.c_longlong, _I, _P],
    "fa_fwd_blocksparse": [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P],
    "fa_bwd_blocksparse": [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _I, _I, _I, _I, _I, _I, _F, _P],
    "fa_bwd_noalloc": [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P],
    "fa_bwd_part": [_I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _I, _I, _I, _I, _I, _I, _F, _P],
    "fa_bwd_fp8": [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _I, _I, _I, _I, _I, _I, _F, _P],
}
for _name, _args in _SIGS.items():
    getattr(_lib, _name).argtypes = _args
    getattr(_lib, _name).restype = _I
_lib.fa_bwd_workspace_size.argtypes = [_I, _I, _I, _I]
_lib.fa_bwd_workspace_size.restype = _Z
_lib.fa_bwd_blocksparse_workspace_size.argtypes = [_I, _I, _I, _I, _I]
_lib.fa_bwd_blocksparse_workspace_size.restype = _Z
_lib.fa_fwd_kvcache_workspace_size.argtypes = [_I, _I, _I, _I, _I]
_lib.fa_fwd_kvcache_workspace_size.restype = _Z
_lib.fa_fwd_kvcache_num_splits.argtypes = [_I, _I, _I, _I]
_lib.fa_fwd_kvcache_num_splits.restype = _I
_lib.fa_status_string.argtypes = [_I]
_lib.fa_status_string.restype = ctypes.c_char_p
_lib.fa_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
_lib.fa_set_wait_timeout_ns.restype = None
_lib.fa_debug_set_inject.argtypes = [_I]
_lib.fa_debug_set_inject.restype = None
_lib.fa_last_device_error_word.argtypes = []
_lib.fa_last_device_error_word.restype = _I

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT, FA_ERR_WORKSPACE = range(6)
FA_BWD_PREPARE, FA_BWD_DKDV, FA_BWD_DQ, FA_BWD_ALL = 1, 2, 4, 7


class FAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {fa_status_string(status)}")


def fa_status_string(status: int) -> str:
    return _lib.fa_status_string(int(status)).decode()


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(st: int, where: str):
    if st != FA_OK:
        raise FAError(st, where)


# ---------------------------------------------------------------- C entry points

def fa_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, scale, stream=None):
    _check(_lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d, int(causal),
                       float(scale), _stream(stream)), "fa_fwd")


def fa_fwd_varlen(q, k, v, o, lse, cu_seqlens, nseq, max_seqlen, total_T, Hq, Hkv, d, causal, scale, stream=None):
    _check(_lib.fa_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens), nseq, max_seqlen,
                              total_T, Hq, Hkv, d, int(causal), float(scale), _stream(stream)), "fa_fwd_varlen")


def fa_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, lse, B, Hq, Hkv, N, d, causal, scale, stream=None):
    _check(_lib.fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale), _ptr(v_scale), _ptr(o),
                           _ptr(lse), B, Hq, Hkv, N, d, int(causal), float(scale), _stream(stream)), "fa_fwd_fp8")


def fa_bwd_workspace_size(tokens, nseq, Hq, d) -> int:
    return int(_lib.fa_bwd_workspace_size(tokens, nseq, Hq, d))


def fa_bwd_blocksparse_workspace_size(B, Hq, Hkv, N, d) -> int:
    return int(_lib.fa_bwd_blocksparse_workspace_size(B, Hq, Hkv, N, d))


def fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, ws_bytes, B, Hq, Hkv, N, d, causal, scale, stream=None):
    _check(_lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                       _ptr(workspace), ws_bytes, B, Hq, Hkv, N, d, int(causal), float(scale), _stream(stream)),
           "fa_bwd")


def fa_bwd_fp8(q8, k8, q_scale, k_scale, q, k, v, o, lse, dout, dq, dk, dv, workspace, ws_bytes, B, Hq, Hkv, N, d,
               causal, scale, stream=None):
    _check(_lib.fa_bwd_fp8(_ptr(q8), _ptr(k8), _ptr(q_scale), _ptr(k_scale), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                           _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), ws_bytes, B, Hq, Hkv,
                           N, d, int(causal), float(scale), _stream(stream)),
           "fa_bwd_fp8")


def fa_fwd_kvcache(q, k_cache, v_cache, cache_seqlens, o, lse, workspace, ws_bytes, B, Nq, Hq, Hkv, Ncache, d,
                   causal, scale, num_splits, stream=None):
    _check(_lib.fa_fwd_kvcache(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_seqlens), _ptr(o), _ptr(lse),
                               _ptr(workspace), ws_bytes, B, Nq, Hq, Hkv, Ncache, d, int(causal), float(scale),
                               int(num_splits), _stream(stream)), "fa_fwd_kvcache")


def fa_attn_merge(o_parts, lse_parts, nparts, o, lse, B, N, H, d, stream=None):
    _check(_lib.fa_attn_merge(_ptr(o_parts), _ptr(lse_parts), int(nparts), _ptr(o), _ptr(lse), B, N, H, d,
                              _stream(stream)), "fa_attn_merge")


def fa_fwd_blocksparse(q, k, v, block_mask, o, lse, B, Hq, Hkv, N, d, causal, scale, stream=None):
    _check(_lib.fa_fwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(block_mask), _ptr(o), _ptr(lse), B, Hq, Hkv, N,
                                   d, int(causal), float(scale), _stream(stream)), "fa_fwd_blocksparse")


def attention_fwd_blocksparse(q, k, v, block_mask, causal=False, scale=None, stream=None):
    """q [B,N,Hq,d], k/v [B,N,Hkv,d] bf16, block_mask uint8 [Hq, ceil(N/128), ceil(N/128)] (CUDA)
    -> (o [B,N,Hq,d] bf16, lse [B,Hq,N] f32)."""
    import torch
    _check_inputs(bf16=dict(q=q, k=k, v=v), u8=dict(block_mask=block_mask))
    B, N, Hq, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    fa_fwd_blocksparse(q, k, v, block_mask, o, lse, B, Hq, k.shape[2], N, d, causal, _default_scale(d, scale), stream)
    return o, lse


def fa_bwd_blocksparse(q, k, v, block_mask, o, lse, dout, dq, dk, dv, workspace, ws_bytes, B, Hq, Hkv, N, d, causal,
                       scale, stream=None):
    _check(_lib.fa_bwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(block_mask), _ptr(o), _ptr(lse), _ptr(dout),
                                   _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), ws_bytes, B, Hq, Hkv, N, d,
                                   int(causal), float(scale), _stream(stream)), "fa_bwd_blocksparse")


def attention_bwd_blocksparse(q, k, v, block_mask, o, lse, dout, causal=False, scale=None, workspace=None,
                              stream=None):
    """Gradients (dq, dk, dv) of sum(o * dout) for attention_fwd_blocksparse with the same block_mask."""
    import torch
    _check_inputs(bf16=dict(q=q, k=k, v=v, o=o, dout=dout), f32=dict(lse=lse), u8=dict(block_mask=block_mask))
    B, N, Hq, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = fa_bwd_blocksparse_workspace_size(B, Hq, k.shape[2], N, d)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    fa_bwd_blocksparse(q, k, v, block_mask, o, lse, dout, dq, dk, dv, workspace, workspace.numel(), B, Hq,
                       k.shape[2], N, d, causal, _default_scale(d, scale), stream)
    return dq, dk, dv


def fa_grad_accumulate(acc, part, out, count, first, stream=None):
    _check(_lib.fa_grad_accumulate(_ptr(acc), _ptr(part), _ptr(out), int(count), int(first), _stream(stream)),
           "fa_grad_accumulate")


def fa_fp8_quantize(x, codes, scales, B, N, H, d, rotate, stream=None):
    _check(_lib.fa_fp8_quantize(_ptr(x), _ptr(codes), _ptr(scales), B, N, H, d, int(rotate), _stream(stream)),
           "fa_fp8_quantize")


def quantize_fp8(x, rotate=False, stream=None):
    """x [B,N,H,d] bf16 (CUDA) -> (codes [B,N,H,d] float8_e4m3fn, scales [B,H,ceil(N/128)] f32)."""
    import torch
    _check_inputs(bf16=dict(x=x))
    B, N, H, d = x.shape
    codes = torch.empty((B, N, H, d), dtype=torch.float8_e4m3fn, device=x.device)
    scales = torch.empty((B, H, (N + 127) // 128), dtype=torch.float32, device=x.device)
    fa_fp8_quantize(x, codes, scales, B, N, H, d, rotate, stream)
    return codes, scales


def fa_fp8_dequantize(codes, scales, x, B, N, H, d, unrotate, stream=None):
    _check(_lib.fa_fp8_dequantize(_ptr(codes), _ptr(scales), _ptr(x), B, N, H, d, int(unrotate), _stream(stream)),
           "fa_fp8_dequantize")


def dequantize_fp8(codes, scales, unrotate=False, stream=None):
    """codes [B,N,H,d] float8_e4m3fn + scales [B,H,ceil(N/128)] f32 (CUDA) -> bf16 [B,N,H,d]
    values in the original space (rotation undone with unrotate=True)."""
    import torch
    _check_inputs(bytes1=dict(codes=codes), f32=dict(scales=scales))
    B, N, H, d = codes.shape
    x = torch.empty((B, N, H, d), dtype=torch.bfloat16, device=codes.device)
    fa_fp8_dequantize(codes, scales, x, B, N, H, d, unrotate, stream)
    return x


def attention_bwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, lse, dout, causal=False, scale=None, rotated=False,
                      workspace=None, stream=None):
    """Gradients (dq, dk, dv) bf16 of sum(o * dout) for the fp8 forward (o, lse from
    attention_fwd_fp8 on these codes), with respect to the original-space inputs:
    the codes are dequantised (Q and K unrotated when they were quantised with the
    rotation) for the 16-bit products, and fa_bwd_fp8 forms the scores on the
    codes themselves, as the forward did."""
    q = dequantize_fp8(q8, q_scale, rotated, stream)
    k = dequantize_fp8(k8, k_scale, rotated, stream)
    v = dequantize_fp8(v8, v_scale, False, stream)
    import torch
    _check_inputs(bf16=dict(q=q, k=k, v=v, o=o, dout=dout), f32=dict(lse=lse, q_scale=q_scale, k_scale=k_scale),
                  bytes1=dict(q8=q8, k8=k8))
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    scale = _default_scale(d, scale)
    if workspace is None:
        nb = fa_bwd_workspace_size(B * N, B, Hq, d)
        workspace = torch.empty(nb, dtype=torch.uint8, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    fa_bwd_fp8(q8, k8, q_scale, k_scale, q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace.numel(), B, Hq, Hkv,
               N, d, causal, scale, stream)
    return dq, dk, dv


def attention_fwd_fp8_rotated(q, k, v, causal=False, scale=None, stream=None):
    """bf16 q [B,N,Hq,d], k/v [B,N,Hkv,d] (CUDA) -> (o bf16, lse f32): Q and K
    rotated by H_d/sqrt(d) and quantised, V quantised, then the fp8 forward."""
    q8, qs = quantize_fp8(q, True, stream)
    k8, ks = quantize_fp8(k, True, stream)
    v8, vs = quantize_fp8(v, False, stream)
    return attention_fwd_fp8(q8, k8, v8, qs, ks, vs, causal=causal, scale=scale, stream=stream)


def fa_fwd_kvcache_workspace_size(B, Nq, Hq, d, num_splits) -> int:
    return int(_lib.fa_fwd_kvcache_workspace_size(B, Nq, Hq, d, num_splits))


def fa_fwd_kvcache_num_splits(B, Hkv, Ncache, d) -> int:
    return int(_lib.fa_fwd_kvcache_num_splits(B, Hkv, Ncache, d))


def fa_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, d, causal, scale, stream=None):
    """fa_bwd with its scratch in the library's built-in device array (no allocation)."""
    _check(_lib.fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                               _ptr(dv), B, Hq, Hkv, N, d, int(causal), float(scale), _stream(stream)),
           "fa_bwd_noalloc")


def fa_bwd_part(parts, q, k, v, o, lse, dout, dq, dk, dv, workspace, ws_bytes, B, Hq, Hkv, N, d, causal, scale,
                stream=None):
    _check(_lib.fa_bwd_part(int(parts), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                            _ptr(dk), _ptr(dv), _ptr(workspace), ws_bytes, B, Hq, Hkv, N, d, int(causal),
                            float(scale), _stream(stream)), "fa_bwd_part")


def fa_bwd_varlen(q, k, v, o, lse, dout, dq, dk, dv, workspace, ws_bytes, cu_seqlens, nseq, max_seqlen, total_T,
                  Hq, Hkv, d, causal, scale, stream=None):
    _check(_lib.fa_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                              _ptr(dv), _ptr(workspace), ws_bytes, _ptr(cu_seqlens), nseq, max_seqlen, total_T, Hq,
                              Hkv, d, int(causal), float(scale), _stream(stream)), "fa_bwd_varlen")


def fa_get_status(stream=None) -> int:
    """Synchronises the stream; returns (and clears) the device status code."""
    return int(_lib.fa_get_status(_stream(stream)))


def fa_last_device_error_word() -> int:
    return int(_lib.fa_last_device_error_word())


def fa_set_wait_timeout_ns(ns: int):
    _lib.fa_set_wait_timeout_ns(int(ns))


def fa_debug_set_inject(mode: int):
    _lib.fa_debug_set_inject(int(mode))


# ---------------------------------------------------------------- torch conveniences

def _default_scale(d, scale):
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def _check_inputs(bf16=None, f32=None, i32=None, u8=None, bytes1=None):
    """The C entry points see only data pointers: every tensor handed to them
    must be dense (contiguous), of the documented element type, and on the
    GPU. Each argument maps names to tensors of one element type (bytes1: any
    1-byte type, the e4m3 codes). Layout and types are checked for all of
    them before residency. Raises ValueError."""
    import torch
    groups = ((bf16, torch.bfloat16, None), (f32, torch.float32, None), (i32, torch.int32, None),
              (u8, torch.uint8, None), (bytes1, None, 1))
    named = []
    for tensors, dtype, itemsize in groups:
        for name, t in (tensors or {}).items():
            if not t.is_contiguous():
                raise ValueError(f"{name} must be contiguous (the library reads it as a dense array)")
            if dtype is not None and t.dtype != dtype:
                raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
            if itemsize is not None and t.element_size() != itemsize:
                raise ValueError(f"{name} must have {itemsize}-byte elements, got {t.element_size()}")
            named.append((name, t))
    for name, t in named:
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")


def attention_fwd(q, k, v, causal=False, scale=None, out=None, lse=None, stream=None):
    """q [B,N,Hq,d], k/v [B,N,Hkv,d] bf16 CUDA tensors -> (o [B,N,Hq,d] bf16, lse [B,Hq,N] f32)."""
    import torch
    _check_inputs(bf16=dict(q=q, k=k, v=v, out=q if out is None else out),
                  f32=None if lse is None else dict(lse=lse))
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    fa_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, _default_scale(d, scale), stream)
    return o, lse


def attention_fwd_varlen(q, k, v, cu_seqlens, max_seqlen, causal=False, scale=None, out=None, lse=None,
                         stream=None):
    """q [T,Hq,d], k/v [T,Hkv,d] bf16, cu_seqlens int32 [nseq+1] (CUDA) -> (o [T,Hq,d], lse [Hq,T])."""
    import torch
    _check_inputs(bf16=dict(q=q, k=k, v=v, out=q if out is None else out),
                  f32=None if lse is None else dict(lse=lse), i32=dict(cu_seqlens=cu_seqlens))
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((Hq, T), dtype=torch.float32, device=q.device) if lse is None else lse
    fa_fwd_varlen(q, k, v, o, lse, cu_seqlens, cu_seqlens.numel() - 1, max_seqlen, T, Hq, Hkv, d, causal,
                  _default_scale(d, scale), stream)
    return o, lse


def attention_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, causal=False, scale=None, stream=None):
    """e4m3 q8 [B,N,Hq,d], k8/v8 [B,N,Hkv,d] + f32 block scales -> (o bf16, lse f32)."""
    import torch
    _check_inputs(bytes1=dict(q8=q8, k8=k8, v8=v8), f32=dict(q_scale=q_scale, k_scale=k_scale, v_scale=v_scale))
    B, N, Hq, d = q8.shape
    Hkv = k8.shape[2]
    o = torch.empty((B, N, Hq, d), dtype=torch.bfloat16, device=q8.device)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q8.device)
    fa_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, lse, B, Hq, Hkv, N, d, causal, _default_scale(d, scale),
               stream)
    return o, lse


def attention_bwd(q, k, v, o, lse, dout, causal=False, scale=None, workspace=None, stream=None):
    """Gradients (dq, dk, dv) of sum(o * dout); inputs as attention_fwd produced them."""
    import torch
    _check_inputs(bf16=dict(q=q, k=k, v=v, o=o, dout=dout), f32=dict(lse=lse))
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = fa_bwd_workspace_size(B * N, B, Hq, d)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace.numel(), B, Hq, Hkv, N, d, causal,
           _default_scale(d, scale), stream)
    return dq, dk, dv


def attention_bwd_varlen(q, k, v, o, lse, dout, cu_seqlens, max_seqlen, causal=False, scale=None, workspace=None,
                         stream=None):
    import torch
    _check_inputs(bf16=dict(q=q, k=k, v=v, o=o, dout=dout), f32=dict(lse=lse), i32=dict(cu_seqlens=cu_seqlens))
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    nseq = cu_seqlens.numel() - 1
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = fa_bwd_workspace_size(T, nseq, Hq, d)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    fa_bwd_varlen(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace.numel(), cu_seqlens, nseq, max_seqlen, T,
                  Hq, Hkv, d, causal, _default_scale(d, scale), stream)
    return dq, dk, dv


def attention_fwd_kvcache(q, k_cache, v_cache, cache_seqlens, causal=True, scale=None, num_splits=None,
                          stream=None):
    """q [B,Nq,Hq,d], caches [B,Ncache,Hkv,d] bf16, cache_seqlens int32 [B] (CUDA)
    -> (o [B,Nq,Hq,d] bf16, lse [B,Hq,Nq] f32). num_splits defaults to the
    library's choice for this device (fa_fwd_kvcache_num_splits)."""
    import torch
    _check_inputs(bf16=dict(q=q, k_cache=k_cache, v_cache=v_cache), i32=dict(cache_seqlens=cache_seqlens))
    B, Nq, Hq, d = q.shape
    Ncache, Hkv = k_cache.shape[1], k_cache.shape[2]
    if num_splits is None:
        num_splits = fa_fwd_kvcache_num_splits(B, Hkv, Ncache, d)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    ws_bytes = fa_fwd_kvcache_workspace_size(B, Nq, Hq, d, num_splits)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    fa_fwd_kvcache(q, k_cache, v_cache, cache_seqlens, o, lse, ws, ws_bytes, B, Nq, Hq, Hkv, Ncache, d, causal,
                   _default_scale(d, scale), num_splits, stream)
    return o, lse
