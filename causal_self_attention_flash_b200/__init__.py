"""libcattn: fused causal multi-head self-attention for B200 (sm_100a).

Python entry points with the same names as the C ABI (include/cattn.h).
They take torch CUDA tensors, allocate outputs with torch when none are
given, pass raw device pointers and the current CUDA stream to the library
and raise CattnError on a non-zero status.  Nothing here computes: torch
only provides device memory and streams.

Layout: q, k, v, o, do, dq, dk, dv are bf16 (B, H, T, D) contiguous; lse
and delta are fp32 (B, H, T).  The _strided calls take (B, H, T, D) views
with any strides whose last one is 1 (e.g. the parts of a fused (B, T, 3C)
projection, see split_qkv), and CausalAttentionQKV goes from that fused
projection straight to a (B, T, C) output with no transposes.
"""

from __future__ import annotations

import ctypes
import math

import torch

from ._binding import (ERR_CUDA, ERR_INVALID_ARG, ERR_TIMEOUT, ERR_TOO_LARGE,
                       ERR_UNSUPPORTED, LIB, LIB_PATH, NOALLOC_SCRATCH_BYTES, OK,
                       CattnError, Dropout, Layout)

__all__ = [
    "attn_fwd", "attn_bwd", "attn_fwd_ex", "attn_bwd_ex", "attn_bwd_preprocess",
    "attn_bwd_workspace_bytes",
    "cattn_get_device_status", "cattn_set_wait_timeout_us",
    "cattn_selftest_wait_timeout", "cattn_status_string", "cattn_version",
    "cattn_last_device_status",
    "cattn_timing_enable", "cattn_timing_read", "KERNEL_NAMES",
    "CausalAttention", "CattnError", "LIB", "LIB_PATH",
    "OK", "ERR_INVALID_ARG", "ERR_UNSUPPORTED", "ERR_CUDA", "ERR_TIMEOUT", "ERR_TOO_LARGE",
    "attn_bwd_noalloc", "NOALLOC_SCRATCH_BYTES",
    "attn_fwd_strided", "attn_bwd_strided", "split_qkv", "CausalAttentionQKV", "Layout",
    "Dropout", "dropout_params", "attn_dropout_mask_bytes", "attn_dropout_mask",
    "attn_decode", "attn_decode_workspace_bytes",
    "SUPPORTED_HEAD_SIZES", "padded_head_size", "pad_qkv_projection", "pad_out_projection",
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
    """An output buffer: allocated like `like` if None, else checked (the
    library writes through its pointer, so it must be device memory of the
    right size on like's device)."""
    if t is None:
        return torch.empty(shape, dtype=dtype, device=like.device)
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"output must be contiguous {dtype} of shape {tuple(shape)}")
    if not t.is_cuda or t.device != like.device:
        raise ValueError(f"output must be on {like.device}")
    return t


def _same_device(ref):
    if ref.device.index != torch.cuda.current_device():
        raise ValueError(f"tensors are on {ref.device}, the current device is "
                         f"cuda:{torch.cuda.current_device()}: call under torch.cuda.device")


def _inputs(*ts):
    """Inputs: one (B, H, T, D) shape (the first tensor's), then contiguous
    bf16 tensors on the current CUDA device."""
    ref = ts[0]
    for t in ts:
        if t.dim() != 4 or tuple(t.shape) != tuple(ref.shape):
            raise ValueError(f"inputs must share the (B, H, T, D) shape {tuple(ref.shape)}, "
                             f"got {tuple(t.shape)}")
    for t in ts:
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous bf16 CUDA tensors")
        if t.device != ref.device:
            raise ValueError("inputs must be on one device")
    _same_device(ref)


def _vector(x, like, shape, what):
    """A contiguous fp32 (B, H, T) input such as LSE, on like's device."""
    if tuple(x.shape) != tuple(shape):
        raise ValueError(f"{what} must have shape {tuple(shape)}, got {tuple(x.shape)}")
    if x.dtype != torch.float32 or not x.is_contiguous() or not x.is_cuda or x.device != like.device:
        raise ValueError(f"{what} must be contiguous fp32 on {like.device}")


def _workspace(ws, like, need):
    """A caller-given workspace: device memory on like's device; returns its
    size in bytes (the library checks it against `need`)."""
    if ws is None:
        return torch.empty(max(need, 1), dtype=torch.uint8, device=like.device)
    if not ws.is_cuda or ws.device != like.device or not ws.is_contiguous():
        raise ValueError(f"workspace must be contiguous device memory on {like.device}")
    return ws


def _nbytes(t):
    return t.numel() * t.element_size()


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
    _vector(lse, q, (B, H, T), "lse")
    if grad_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("grad_dtype must be torch.bfloat16 or torch.float32")
    dq = _want(dq, q, grad_dtype, (B, H, T, D))
    dk = _want(dk, q, grad_dtype, (B, H, T, D))
    dv = _want(dv, q, grad_dtype, (B, H, T, D))
    workspace = _workspace(workspace, q, attn_bwd_workspace_bytes(B, H, T, D))
    if o_lo is None and grad_dtype == torch.bfloat16:
        st = LIB.attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                          lse.data_ptr(), do.data_ptr(), float(scale), B, H, T, D,
                          dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                          _nbytes(workspace), _stream(stream))
        _check("attn_bwd", st)
    else:
        if o_lo is not None:
            _inputs(q, o_lo)
        st = LIB.attn_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                             o_lo.data_ptr() if o_lo is not None else None, lse.data_ptr(),
                             do.data_ptr(), float(scale), B, H, T, D, dq.data_ptr(),
                             dk.data_ptr(), dv.data_ptr(),
                             1 if grad_dtype == torch.float32 else 0,
                             workspace.data_ptr(), _nbytes(workspace), _stream(stream))
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
    _vector(lse, q, (B, H, T), "lse")
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


def cattn_selftest_wait_timeout(timeout_us: int, stream=None, workspace=None):
    """The hang guard's self-test; with a workspace (a uint8 CUDA tensor of
    a backward's workspace) it records into that workspace's status words."""
    if workspace is None:
        return int(LIB.cattn_selftest_wait_timeout(int(timeout_us), _stream(stream)))
    if not workspace.is_cuda:
        raise ValueError("workspace must be device memory")
    return int(LIB.cattn_selftest_wait_timeout_ws(int(timeout_us), workspace.data_ptr(),
                                                  _stream(stream)))


def cattn_last_device_status(workspace, stream=None):
    """Status recorded by the last backward call that used this workspace
    (waits for `stream`)."""
    if not workspace.is_cuda:
        raise ValueError("workspace must be device memory")
    return int(LIB.cattn_last_device_status(workspace.data_ptr(), _stream(stream)))


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


def _layout(t, dtype, what, shape=None, device=None):
    """cattn_layout of a (B, H, T, D) view whose last stride is 1 (checked
    against the expected shape and device when given)."""
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError(f"{what}: expected a (B, H, T, D) view with unit last stride")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{what}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype or not t.is_cuda:
        raise ValueError(f"{what}: expected a {dtype} CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{what}: expected a tensor on {device}")
    return Layout(t.stride(0), t.stride(1), t.stride(2))


def split_qkv(qkv, n_head):
    """(q, k, v) as (B, H, T, D) views into a fused (B, T, 3C) projection,
    as the pages' c_attn produces it.  View arithmetic only: no copies."""
    B, T, C3 = qkv.shape
    C = C3 // 3
    D = C // n_head
    parts = qkv.split(C, dim=2)
    return tuple(x.view(B, T, n_head, D).transpose(1, 2) for x in parts)


def dropout_params(p, seed=0, offset=0, mask=None):
    """cattn_dropout for drop probability p (0 <= p < 1), a 64-bit seed and
    a 32-bit counter offset; None for p == 0 (or None).  mask: an optional
    uint8 device tensor of attn_dropout_mask_bytes(B, H, T) bytes that the
    forward fills with its keep bits and the backward then reads (see
    attn_dropout_mask); the tensor must stay alive until the backward."""
    if p is None or p == 0:
        return None
    ptr = None
    if mask is not None:
        if not mask.is_cuda or not mask.is_contiguous() or mask.dtype != torch.uint8:
            raise ValueError("mask must be a contiguous uint8 device tensor")
        ptr = mask.data_ptr()
    return Dropout(float(p), int(seed) & 0xFFFFFFFFFFFFFFFF, int(offset) & 0xFFFFFFFF, ptr)


def attn_dropout_mask_bytes(B, H, T):
    return int(LIB.attn_dropout_mask_bytes(B, H, T))


def attn_dropout_mask(B, H, T, device):
    """A keep-bit cache buffer (uint8, attn_dropout_mask_bytes(B, H, T)
    bytes) for dropout_params(..., mask=...)."""
    n = attn_dropout_mask_bytes(B, H, T)
    if n == 0:
        raise ValueError("empty or invalid shape")
    return torch.empty(n, dtype=torch.uint8, device=device)


def attn_fwd_strided(q, k, v, scale=None, o=None, lse=None, o_lo=None, stream=None,
                     dropout=None):
    """attn_fwd_ex on strided (B, H, T, D) views.  o (and o_lo) may be views
    too, e.g. of a (B, T, C) buffer (o_lo must share o's strides); if not
    given they are allocated contiguous.  dropout: a Dropout (see
    dropout_params) for attention dropout.  Returns (o, lse, o_lo)."""
    B, H, T, D = _shape(q)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    shp = (B, H, T, D)
    lq, lk, lv = (_layout(t, torch.bfloat16, n, shp, q.device)
                  for t, n in ((q, "q"), (k, "k"), (v, "v")))
    _same_device(q)
    if o is None:
        o = torch.empty(shp, dtype=torch.bfloat16, device=q.device)
    lo = _layout(o, torch.bfloat16, "o", shp, q.device)
    if o_lo is not None:
        _layout(o_lo, torch.bfloat16, "o_lo", shp, q.device)
        if o_lo.stride() != o.stride():
            raise ValueError("o_lo must be a bf16 view with o's strides")
    lse = _want(lse, q, torch.float32, (B, H, T))
    olo_ptr = o_lo.data_ptr() if o_lo is not None else None
    if dropout is None:
        st = LIB.attn_fwd_strided(q.data_ptr(), lq, k.data_ptr(), lk, v.data_ptr(), lv,
                                  float(scale), B, H, T, D, o.data_ptr(), lo, lse.data_ptr(),
                                  olo_ptr, _stream(stream))
        _check("attn_fwd_strided", st)
    else:
        st = LIB.attn_fwd_dropout(q.data_ptr(), lq, k.data_ptr(), lk, v.data_ptr(), lv,
                                  float(scale), B, H, T, D, ctypes.byref(dropout), o.data_ptr(),
                                  lo, lse.data_ptr(), olo_ptr, _stream(stream))
        _check("attn_fwd_dropout", st)
    return o, lse, o_lo


def attn_bwd_strided(q, k, v, o, lse, do, scale=None, dq=None, dk=None, dv=None,
                     workspace=None, stream=None, o_lo=None, grad_dtype=torch.bfloat16,
                     dropout=None):
    """attn_bwd_ex on strided (B, H, T, D) views of q, k, v, o (o_lo with o's
    strides), do and the outputs dq, dk, dv (allocated contiguous if not
    given; e.g. the three parts of one (B, T, 3C) gradient buffer).  dropout:
    the forward's Dropout, for attention dropout."""
    B, H, T, D = _shape(q)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    shp = (B, H, T, D)
    if grad_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("grad_dtype must be torch.bfloat16 or torch.float32")
    ins = [_layout(t, torch.bfloat16, n, shp, q.device)
           for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do"))]
    _same_device(q)
    _vector(lse, q, (B, H, T), "lse")
    if o_lo is not None:
        _layout(o_lo, torch.bfloat16, "o_lo", shp, q.device)
        if o_lo.stride() != o.stride():
            raise ValueError("o_lo must be a bf16 view with o's strides")
    outs = []
    for t in (dq, dk, dv):
        outs.append(t if t is not None else torch.empty(shp, dtype=grad_dtype, device=q.device))
    dq, dk, dv = outs
    louts = [_layout(t, grad_dtype, n, shp, q.device)
             for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv"))]
    workspace = _workspace(workspace, q, attn_bwd_workspace_bytes(B, H, T, D))
    olo_ptr = o_lo.data_ptr() if o_lo is not None else None
    f32 = 1 if grad_dtype == torch.float32 else 0
    if dropout is None:
        st = LIB.attn_bwd_strided(q.data_ptr(), ins[0], k.data_ptr(), ins[1], v.data_ptr(),
                                  ins[2], o.data_ptr(), ins[3], olo_ptr, lse.data_ptr(),
                                  do.data_ptr(), ins[4], float(scale), B, H, T, D,
                                  dq.data_ptr(), louts[0], dk.data_ptr(), louts[1],
                                  dv.data_ptr(), louts[2], f32,
                                  workspace.data_ptr(), _nbytes(workspace), _stream(stream))
        _check("attn_bwd_strided", st)
    else:
        st = LIB.attn_bwd_dropout(q.data_ptr(), ins[0], k.data_ptr(), ins[1], v.data_ptr(),
                                  ins[2], o.data_ptr(), ins[3], olo_ptr, lse.data_ptr(),
                                  do.data_ptr(), ins[4], float(scale), B, H, T, D,
                                  ctypes.byref(dropout), dq.data_ptr(), louts[0],
                                  dk.data_ptr(), louts[1], dv.data_ptr(), louts[2], f32,
                                  workspace.data_ptr(), _nbytes(workspace), _stream(stream))
        _check("attn_bwd_dropout", st)
    return dq, dk, dv


def attn_decode_workspace_bytes(B, H, Tq, L, D):
    return int(LIB.attn_decode_workspace_bytes(B, H, Tq, L, D))


def attn_decode(q, k, v, L, scale=None, o=None, lse=None, workspace=None, stream=None):
    """Causal attention of the Tq newest positions against a key/value
    cache: q (B, H, Tq, D) holds the query rows at positions L-Tq .. L-1,
    k and v (B, H, >= L, D) views of the cache whose first L rows are the
    sequence so far (any strides with unit last stride).  Returns (o, lse),
    o (B, H, Tq, D) bf16 and lse (B, H, Tq) fp32."""
    B, H, Tq, D = _shape(q)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    for t, n in ((k, "k"), (v, "v")):
        if t.dim() != 4 or tuple(t.shape[:2]) != (B, H) or t.shape[3] != D:
            raise ValueError(f"{n} must be a (B, H, >= L, D) view matching q")
        if t.shape[2] < L:
            raise ValueError(f"{n}: the cache holds fewer than L positions")
    lq = _layout(q, torch.bfloat16, "q", None, q.device)
    lk = _layout(k, torch.bfloat16, "k", None, q.device)
    lv = _layout(v, torch.bfloat16, "v", None, q.device)
    _same_device(q)
    if o is None:
        o = torch.empty((B, H, Tq, D), dtype=torch.bfloat16, device=q.device)
    lo = _layout(o, torch.bfloat16, "o", (B, H, Tq, D), q.device)
    lse = _want(lse, q, torch.float32, (B, H, Tq))
    need = attn_decode_workspace_bytes(B, H, Tq, L, D)
    if workspace is None and need == 0:
        ws_ptr, ws_n = None, 0
    else:
        workspace = _workspace(workspace, q, need)
        ws_ptr, ws_n = workspace.data_ptr(), _nbytes(workspace)
    st = LIB.attn_decode(q.data_ptr(), lq, k.data_ptr(), lk, v.data_ptr(), lv, float(scale),
                         B, H, Tq, int(L), D, o.data_ptr(), lo, lse.data_ptr(),
                         ws_ptr, ws_n, _stream(stream))
    _check("attn_decode", st)
    return o, lse


SUPPORTED_HEAD_SIZES = (16, 32, 64, 128)


def padded_head_size(d: int) -> int:
    """The smallest head size the kernels take that holds d (e.g. 12 -> 16)."""
    for s in SUPPORTED_HEAD_SIZES:
        if d <= s:
            return s
    raise ValueError(f"head size {d} above {SUPPORTED_HEAD_SIZES[-1]}")


def pad_qkv_projection(weight, bias, n_head, d, d_pad=None):
    """One-time set-up for head sizes the kernels do not take (12, say):
    the c_attn projection (weight (3C, C_in), bias (3C,) or None, rows
    [q heads | k heads | v heads], d rows per head) re-laid so that each
    head gets d_pad rows, the extra ones zero.  Its output is then a
    (B, T, 3 * n_head * d_pad) buffer whose zero-padded heads the d_pad
    kernels process exactly (padded q and k add nothing to the scores;
    padded v columns give zero output columns); pass scale = 1/sqrt(d).
    Not on the per-step path: a model does this once to its weights."""
    d_pad = d_pad or padded_head_size(d)
    w = weight.reshape(3, n_head, d, -1)
    wp = weight.new_zeros(3, n_head, d_pad, w.shape[-1])
    wp[:, :, :d] = w
    bp = None
    if bias is not None:
        bp = bias.new_zeros(3, n_head, d_pad)
        bp[:, :, :d] = bias.reshape(3, n_head, d)
        bp = bp.reshape(-1)
    return wp.reshape(3 * n_head * d_pad, -1), bp


def pad_out_projection(weight, n_head, d, d_pad=None):
    """The matching c_proj weight (C_out, n_head * d) with zero columns for
    the padded head columns, so that y (B, T, n_head * d_pad) from the
    kernels feeds it unchanged (the padded columns of y are zero, and the
    zero columns keep their gradient zero)."""
    d_pad = d_pad or padded_head_size(d)
    w = weight.reshape(weight.shape[0], n_head, d)
    wp = weight.new_zeros(weight.shape[0], n_head, d_pad)
    wp[:, :, :d] = w
    return wp.reshape(weight.shape[0], n_head * d_pad)


class CausalAttentionQKV(torch.autograd.Function):
    """autograd wrapper from the fused projection to the merged output:
    qkv (B, T, 3C) bf16 -> y (B, T, C) bf16 = the heads of causal attention
    side by side, as the pages' CausalSelfAttention glues them together
    before c_proj.  Forward and backward read and write those layouts in
    place (attn_fwd_strided / attn_bwd_strided); dqkv comes back as one
    (B, T, 3C) tensor.  apply(qkv, n_head, scale=None, dropout_p=0.0,
    seed=0, offset=0): with dropout_p > 0, attention dropout with the mask
    of (seed, offset), the same in the backward: the forward keeps its keep
    bits in a cache buffer (attn_dropout_mask, 1 bit per element of the
    causal tiles) that the backward reads instead of drawing them again."""

    @staticmethod
    def forward(ctx, qkv, n_head, scale=None, dropout_p=0.0, seed=0, offset=0):
        B, T, C3 = qkv.shape
        C = C3 // 3
        D = C // n_head
        q, k, v = split_qkv(qkv, n_head)
        y = torch.empty((B, T, C), dtype=torch.bfloat16, device=qkv.device)
        y_lo = torch.empty_like(y)
        o = y.view(B, T, n_head, D).transpose(1, 2)
        o_lo = y_lo.view(B, T, n_head, D).transpose(1, 2)
        mask = attn_dropout_mask(B, n_head, T, qkv.device) if dropout_p else None
        drop = dropout_params(dropout_p, seed, offset, mask)
        _, lse, _ = attn_fwd_strided(q, k, v, scale, o=o, o_lo=o_lo, dropout=drop)
        ctx.save_for_backward(qkv, y, y_lo, lse)
        ctx.n_head, ctx.scale, ctx.drop, ctx.mask = n_head, scale, drop, mask
        return y

    @staticmethod
    def backward(ctx, dy):
        qkv, y, y_lo, lse = ctx.saved_tensors
        n_head = ctx.n_head
        B, T, C = y.shape
        D = C // n_head
        q, k, v = split_qkv(qkv, n_head)
        o = y.view(B, T, n_head, D).transpose(1, 2)
        o_lo = y_lo.view(B, T, n_head, D).transpose(1, 2)
        dy = dy.contiguous()
        do = dy.view(B, T, n_head, D).transpose(1, 2)
        dqkv = torch.empty_like(qkv)
        dq, dk, dv = split_qkv(dqkv, n_head)
        attn_bwd_strided(q, k, v, o, lse, do, ctx.scale, dq=dq, dk=dk, dv=dv, o_lo=o_lo,
                         dropout=ctx.drop)
        return dqkv, None, None, None, None, None


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
