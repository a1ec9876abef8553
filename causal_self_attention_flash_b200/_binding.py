"""ctypes binding of libcattn's C ABI (declared in include/cattn.h).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  There is no fallback; if the shared library is
missing, importing this module raises.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libcattn.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_CUDA = 3
ERR_TIMEOUT = 4
ERR_TOO_LARGE = 5

STATUS_NAMES = {OK: "CATTN_OK", ERR_INVALID_ARG: "CATTN_ERR_INVALID_ARG",
                ERR_UNSUPPORTED: "CATTN_ERR_UNSUPPORTED", ERR_CUDA: "CATTN_ERR_CUDA",
                ERR_TIMEOUT: "CATTN_ERR_TIMEOUT", ERR_TOO_LARGE: "CATTN_ERR_TOO_LARGE"}



class Layout(ctypes.Structure):
    """cattn_layout: element strides (b, h, t) of a (B, H, T, D) tensor."""
    _fields_ = [("b", ctypes.c_longlong), ("h", ctypes.c_longlong), ("t", ctypes.c_longlong)]


class Dropout(ctypes.Structure):
    """cattn_dropout: drop probability p, generator seed, counter offset and
    the optional keep-bit cache (device pointer or None)."""
    _fields_ = [("p", ctypes.c_float), ("seed", ctypes.c_ulonglong), ("offset", ctypes.c_uint),
                ("mask", ctypes.c_void_p)]


# name -> (restype, argtypes), mirroring include/cattn.h
_vp, _i, _f, _sz, _u32 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_float,
                          ctypes.c_size_t, ctypes.c_uint32)
_L = Layout
_DP = ctypes.POINTER(Dropout)
SIGNATURES = {
    "attn_fwd": (_i, [_vp, _vp, _vp, _f, _i, _i, _i, _i, _vp, _vp, _vp]),
    "attn_fwd_ex": (_i, [_vp, _vp, _vp, _f, _i, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "attn_bwd_workspace_bytes": (_sz, [_i, _i, _i, _i]),
    "attn_bwd_preprocess": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp]),
    "attn_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _f, _i, _i, _i, _i,
                      _vp, _vp, _vp, _vp, _sz, _vp]),
    "attn_bwd_ex": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _f, _i, _i, _i, _i,
                         _vp, _vp, _vp, _i, _vp, _sz, _vp]),
    "attn_bwd_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _f, _i, _i, _i, _i,
                              _vp, _vp, _vp, _vp]),
    "attn_fwd_strided": (_i, [_vp, _L, _vp, _L, _vp, _L, _f, _i, _i, _i, _i, _vp, _L, _vp, _vp,
                              _vp]),
    "attn_bwd_strided": (_i, [_vp, _L, _vp, _L, _vp, _L, _vp, _L, _vp, _vp, _vp, _L, _f,
                              _i, _i, _i, _i, _vp, _L, _vp, _L, _vp, _L, _i, _vp, _sz, _vp]),
    "attn_fwd_dropout": (_i, [_vp, _L, _vp, _L, _vp, _L, _f, _i, _i, _i, _i, _DP, _vp, _L, _vp,
                              _vp, _vp]),
    "attn_bwd_dropout": (_i, [_vp, _L, _vp, _L, _vp, _L, _vp, _L, _vp, _vp, _vp, _L, _f,
                              _i, _i, _i, _i, _DP, _vp, _L, _vp, _L, _vp, _L, _i, _vp, _sz, _vp]),
    "attn_decode_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "attn_dropout_mask_bytes": (_sz, [_i, _i, _i]),
    "attn_decode": (_i, [_vp, _L, _vp, _L, _vp, _L, _f, _i, _i, _i, _i, _i, _vp, _L, _vp, _vp,
                         _sz, _vp]),
    "cattn_get_device_status": (_i, [_i, _vp]),
    "cattn_set_wait_timeout_us": (None, [_u32]),
    "cattn_selftest_wait_timeout": (_i, [_u32, _vp]),
    "cattn_last_device_status": (_i, [_vp, _vp]),
    "cattn_selftest_wait_timeout_ws": (_i, [_u32, _vp, _vp]),
    "cattn_timing_enable": (None, [_i]),
    "cattn_timing_read": (_i, [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int), _i]),
    "cattn_status_string": (ctypes.c_char_p, [_i]),
    "cattn_version": (_i, []),
    "cattn_plan_passes": (_i, [_i, _i, _i, _i, ctypes.POINTER(ctypes.c_uint16), _i]),
    "cattn_last_cuda_error": (_i, []),
}


class CattnError(RuntimeError):
    def __init__(self, fn: str, status: int, cuda_error: int = 0):
        self.status = status
        self.cuda_error = cuda_error
        extra = f" (CUDA error {cuda_error})" if status == ERR_CUDA else ""
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}{extra}")


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"libcattn.so not found at {path}; build it with "
            "`python causal_self_attention_flash_b200/build.py`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


# CATTN_NOALLOC_SCRATCH_BYTES of include/cattn.h
NOALLOC_SCRATCH_BYTES = 64 << 20

LIB = load()
