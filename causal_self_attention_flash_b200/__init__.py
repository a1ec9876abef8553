"""libcattn: fused causal multi-head self-attention for B200 (sm_100a).

Python entry points with the same names as the C ABI (include/cattn.h).
They take torch CUDA tensors, allocate outputs with torch when none are
given, pass raw device pointers and the current CUDA stream to the library
and raise CattnError on a non-zero status.  Nothing here computes: torch
only provides device memory and streams.

Layout: q, k, v, o, do, dq, dk, dv are bf16 (B, H, T, D) contiguous; lse
and delta are fp32 (B, H, T).
"""

from __future__ import annotations

import math

import torch

from ._binding import (ERR_CUDA, ERR_INVALID_ARG, ERR_TIMEOUT, ERR_TOO_LARGE,
                       ERR_UNSUPPORTED, LIB, LIB_PATH, NOALLOC_SCRATCH_BYTES, OK,
                       CattnError)

__all__ = [
    "attn_fwd", "attn_bwd", "attn_fwd_ex", "attn_bwd_ex", "attn_bwd_preprocess",
    "attn_bwd_workspace_bytes",
    "cattn_get_device_status", "cattn_set_wait_timeout_us",
    "cattn_selftest_wait_timeout", "cattn_status_string", "cattn_version",
    "cattn_timing_enable", "cattn_timing_read", "KERNEL_NAMES",
    "CausalAttention", "CattnError", "LIB", "LIB_PATH",
    "OK", "ERR_INVALID_ARG", "ERR_UNSUPPORTED", "ERR_CUDA", "ERR_TIMEOUT", "ERR_TOO_LARGE",
    "attn_bwd_noalloc", "NOALLOC_SCRATCH_BYTES",
]


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(name, st):
    if st != OK:
        raise CattnError(name, st, int(LIB.cattn_last_cuda_error()) if st == ERR_CUDA else 0)


def _shape(q):
    if q.dim() != 4:
        raise ValueError("expected a (B, H, T, D) tensor")
    return tuple(int(x) for x in q.shape)


def _want(t, like, dtype, shape):
    if t is None:
        return torch.empty(shape, dtype=dtype, device=like.device)
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"output must be contiguous {dtype} of shape {shape}")
    return t


def _inputs(*ts):
    for t in ts:
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous bf16 CUDA tensors")


def attn_fwd_ex(q, k, v, scale=None, o=None, lse=None, o_lo=None, want_o_lo=True,
                stream=None):
    """(o, lse, o_lo) = causal attention of bf16 (B,H,T,D) q, k, v, with the
    bf16 rounding residual o_lo = bf16(O - o) of the output (None if not
    wanted)."""
    _inputs(q, k, v)
    B, H, T, D = _shape(q)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    o = _want(o, q, torch.bfloat16, (B, H, T, D))
    lse = _want(lse, q, torch.float32, (B, H, T))
    if want_o_lo:
        o_lo = _want(o_lo, q, torch.bfloat16, (B, H, T, D))
    st = LIB.attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), float(scale), B, H, T, D,
                         o.data_ptr(), lse.data_ptr(),
                         o_lo.data_ptr() if o_lo is not None else None, _stream(stream))
    _check("attn_fwd_ex", st)
    return o, lse, o_lo


def attn_fwd(q, k, v, scale=None, o=None, lse=None, stream=None):
    """(o, lse) = causal attention of bf16 (B,H,T,D) q, k, v."""
    _inputs(q, k, v)
    B, H, T, D = _shape(q)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    o = _want(o, q, torch.bfloat16, (B, H, T, D))
    lse = _want(lse, q, torch.float32, (B, H, T))
    st = LIB.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), float(scale), B, H, T, D,
                      o.data_ptr(), lse.data_ptr(), _stream(stream))
    _check("attn_fwd", st)
    return o, lse


def attn_bwd_workspace_bytes(B, H, T, D):
    return int(LIB.attn_bwd_workspace_bytes(B, H, T, D))


def attn_bwd_preprocess(o, do, delta=None, stream=None):
    """delta = rowsum(do * o), fp32 (B,H,T)."""
    _inputs(o, do)
    B, H, T, D = _shape(o)
    delta = _want(delta, o, torch.float32, (B, H, T))
    st = LIB.attn_bwd_preprocess(o.data_ptr(), do.data_ptr(), B, H, T, D, delta.data_ptr(),
                                 _stream(stream))
    _check("attn_bwd_preprocess", st)
    return delta


def attn_bwd(q, k, v, o, lse, do, scale=None, dq=None, dk=None, dv=None,
             workspace=None, stream=None, o_lo=None, grad_dtype=torch.bfloat16):
    """(dq, dk, dv) of causal attention; workspace allocated with torch if
    not given (a uint8 CUDA tensor of attn_bwd_workspace_bytes bytes).
    With the forward's o_lo or grad_dtype=torch.float32 this calls
    attn_bwd_ex."""
    _inputs(q, k, v, o, do)
    B, H, T, D = _shape(q)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be contiguous fp32 (B, H, T)")
    if grad_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("grad_dtype must be torch.bfloat16 or torch.float32")
    dq = _want(dq, q, grad_dtype, (B, H, T, D))
    dk = _want(dk, q, grad_dtype, (B, H, T, D))
    dv = _want(dv, q, grad_dtype, (B, H, T, D))
    need = attn_bwd_workspace_bytes(B, H, T, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    if o_lo is None and grad_dtype == torch.bfloat16:
        st = LIB.attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                          lse.data_ptr(), do.data_ptr(), float(scale), B, H, T, D,
                          dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                          workspace.numel(), _stream(stream))
        _check("attn_bwd", st)
    else:
        if o_lo is not None:
            _inputs(o_lo)
        st = LIB.attn_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                             o_lo.data_ptr() if o_lo is not None else None, lse.data_ptr(),
                             do.data_ptr(), float(scale), B, H, T, D, dq.data_ptr(),
                             dk.data_ptr(), dv.data_ptr(),
                             1 if grad_dtype == torch.float32 else 0,
                             workspace.data_ptr(), workspace.numel(), _stream(stream))
        _check("attn_bwd_ex", st)
    return dq, dk, dv


attn_bwd_ex = attn_bwd


def attn_bwd_noalloc(q, k, v, o, lse, do, scale=None, dq=None, dk=None, dv=None,
                     stream=None):
    """attn_bwd without a workspace: the library's fixed scratch of
    NOALLOC_SCRATCH_BYTES is used instead (see include/cattn.h; calls that
    overlap on the GPU race).  Only the outputs, if not given, are
    allocated here, by torch; the C call itself allocates nothing."""
    _inputs(q, k, v, o, do)
    B, H, T, D = _shape(q)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = _want(dq, q, torch.bfloat16, (B, H, T, D))
    dk = _want(dk, q, torch.bfloat16, (B, H, T, D))
    dv = _want(dv, q, torch.bfloat16, (B, H, T, D))
    st = LIB.attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              lse.data_ptr(), do.data_ptr(), float(scale), B, H, T, D,
                              dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), _stream(stream))
    _check("attn_bwd_noalloc", st)
    return dq, dk, dv


def cattn_get_device_status(clear=False, stream=None):
    return int(LIB.cattn_get_device_status(1 if clear else 0, _stream(stream)))


def cattn_set_wait_timeout_us(us: int):
    LIB.cattn_set_wait_timeout_us(int(us))


def cattn_selftest_wait_timeout(timeout_us: int, stream=None):
    return int(LIB.cattn_selftest_wait_timeout(int(timeout_us), _stream(stream)))


KERNEL_NAMES = ("fwd_kernel", "bwd_pre_kernel", "bwd_kernel", "dq_convert_kernel")


def cattn_timing_enable(enable: bool = True):
    LIB.cattn_timing_enable(1 if enable else 0)


def cattn_timing_read():
    """{kernel name: (total ms, launches)} since the last read."""
    import ctypes
    n = len(KERNEL_NAMES)
    ms = (ctypes.c_float * n)()
    cnt = (ctypes.c_int * n)()
    _check("cattn_timing_read", LIB.cattn_timing_read(ms, cnt, n))
    return {KERNEL_NAMES[i]: (float(ms[i]), int(cnt[i])) for i in range(n)}


def cattn_status_string(st: int) -> str:
    return LIB.cattn_status_string(int(st)).decode()


def cattn_version() -> int:
    return int(LIB.cattn_version())


class CausalAttention(torch.autograd.Function):
    """autograd wrapper: forward = attn_fwd, backward = attn_bwd."""

    @staticmethod
    def forward(ctx, q, k, v, scale=None):
        o, lse, o_lo = attn_fwd_ex(q, k, v, scale)
        ctx.save_for_backward(q, k, v, o, lse, o_lo)
        ctx.scale = scale
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse, o_lo = ctx.saved_tensors
        dq, dk, dv = attn_bwd(q, k, v, o, lse, do.contiguous(), ctx.scale, o_lo=o_lo)
        return dq, dk, dv, None
