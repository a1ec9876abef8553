"""CPU tests of the C ABI: the library loads, exports every function the
header declares, and rejects bad arguments before touching any device.

Only argument errors that the library detects before its first CUDA call
are exercised here (no GPU on this host): every call below returns without
launching anything and without dereferencing the (fake) pointers.
"""

import ctypes
import math
import os
import re

import pytest
import torch  # noqa: F401  (loads the CUDA runtime libcattn links against)

import causal_self_attention_flash_b200 as cattn
from causal_self_attention_flash_b200 import _binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cattn.h")

ALIGNED = 0x10000  # fake, 16-byte aligned; never dereferenced by these calls


def header_functions():
    with open(HEADER) as f:
        src = f.read()
    return re.findall(r"^CATTN_API\s+[\w\s\*]+?\b(\w+)\s*\(", src, flags=re.M)


def test_header_declares_the_forward_and_backward_calls():
    names = header_functions()
    for n in ("attn_fwd", "attn_bwd", "attn_bwd_workspace_bytes", "attn_bwd_preprocess"):
        assert n in names


def test_every_declared_symbol_is_exported():
    lib = ctypes.CDLL(_binding.LIB_PATH)
    names = header_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
        assert n in _binding.SIGNATURES, n


def test_version_and_strings():
    assert cattn.cattn_version() == 100
    assert cattn.cattn_status_string(0) == "ok"
    assert "invalid" in cattn.cattn_status_string(1)
    assert cattn.cattn_status_string(99) == "unknown status"


def fwd(q=ALIGNED, k=ALIGNED, v=ALIGNED, scale=0.125, B=1, H=1, T=8, D=64,
        o=ALIGNED, lse=ALIGNED):
    return cattn.LIB.attn_fwd(q, k, v, scale, B, H, T, D, o, lse, None)


def bwd(ptrs=None, scale=0.125, B=1, H=1, T=8, D=64, ws=ALIGNED, ws_bytes=1 << 30):
    p = ptrs or [ALIGNED] * 9
    return cattn.LIB.attn_bwd(p[0], p[1], p[2], p[3], p[4], p[5], scale, B, H, T, D,
                              p[6], p[7], p[8], ws, ws_bytes, None)


@pytest.mark.parametrize("D", [0, 8, 48, 96, 256])
def test_unsupported_head_size(D):
    assert fwd(D=D) == cattn.ERR_UNSUPPORTED
    assert bwd(D=D) == cattn.ERR_UNSUPPORTED
    assert cattn.attn_bwd_workspace_bytes(1, 1, 8, D) == 0


@pytest.mark.parametrize("shape", [(-1, 1, 8), (1, -1, 8), (1, 1, -8), (1, 1, (1 << 20) + 1),
                                   (1 << 16, 1 << 16, 8)])
def test_bad_sizes(shape):
    B, H, T = shape
    assert fwd(B=B, H=H, T=T) == cattn.ERR_INVALID_ARG
    assert bwd(B=B, H=H, T=T) == cattn.ERR_INVALID_ARG
    assert cattn.attn_bwd_workspace_bytes(B, H, T, 64) == 0


@pytest.mark.parametrize("scale", [0.0, -1.0, math.nan, math.inf])
def test_bad_scale(scale):
    assert fwd(scale=scale) == cattn.ERR_INVALID_ARG
    assert bwd(scale=scale) == cattn.ERR_INVALID_ARG


@pytest.mark.parametrize("which", range(5))
def test_null_pointer_fwd(which):
    args = dict(q=ALIGNED, k=ALIGNED, v=ALIGNED, o=ALIGNED, lse=ALIGNED)
    args[list(args)[which]] = None
    assert fwd(**args) == cattn.ERR_INVALID_ARG


@pytest.mark.parametrize("which", range(9))
def test_null_pointer_bwd(which):
    p = [ALIGNED] * 9
    p[which] = None
    assert bwd(ptrs=p) == cattn.ERR_INVALID_ARG
    assert bwd(ws=None) == cattn.ERR_INVALID_ARG


@pytest.mark.parametrize("which", range(4))
def test_misaligned_fwd(which):
    args = dict(q=ALIGNED, k=ALIGNED, v=ALIGNED, o=ALIGNED)
    args[list(args)[which]] = ALIGNED + 8     # bf16 tensors need 16 bytes
    assert fwd(**args) == cattn.ERR_INVALID_ARG
    assert fwd(lse=ALIGNED + 2) == cattn.ERR_INVALID_ARG


def test_residual_entry_points_check_alignment():
    args = (ALIGNED, ALIGNED, ALIGNED, 0.125, 1, 1, 8, 64, ALIGNED, ALIGNED)
    assert cattn.LIB.attn_fwd_ex(*args, ALIGNED + 8, None) == cattn.ERR_INVALID_ARG
    assert cattn.LIB.attn_fwd_ex(ALIGNED, ALIGNED, ALIGNED, 0.125, 1, 1, 8, 48, ALIGNED,
                                 ALIGNED, None, None) == cattn.ERR_UNSUPPORTED
    p = [ALIGNED] * 4
    assert cattn.LIB.attn_bwd_ex(*p, ALIGNED + 8, ALIGNED, ALIGNED, 0.125, 1, 1, 8, 64,
                                 ALIGNED, ALIGNED, ALIGNED, 0, ALIGNED, 1 << 30,
                                 None) == cattn.ERR_INVALID_ARG
    for bad_dtype in (-1, 2, 7):
        assert cattn.LIB.attn_bwd_ex(*p, None, ALIGNED, ALIGNED, 0.125, 1, 1, 8, 64,
                                     ALIGNED, ALIGNED, ALIGNED, bad_dtype, ALIGNED, 1 << 30,
                                     None) == cattn.ERR_INVALID_ARG


def test_static_scratch_backward_refuses_oversized_shapes():
    """attn_bwd_noalloc: shapes beyond its fixed scratch are refused before
    any device call (here, on a host without a GPU)."""
    p = [ALIGNED] * 6
    out = [ALIGNED] * 3
    B, H, T, D = 2, 16, 8192, 128          # needs ~135 MB of scratch
    assert cattn.attn_bwd_workspace_bytes(B, H, T, D) > cattn.NOALLOC_SCRATCH_BYTES
    assert cattn.LIB.attn_bwd_noalloc(*p, 0.125, B, H, T, D, *out, None) == cattn.ERR_TOO_LARGE
    assert cattn.attn_bwd_workspace_bytes(8, 25, 1024, 64) <= cattn.NOALLOC_SCRATCH_BYTES
    assert cattn.LIB.attn_bwd_noalloc(*p, 0.125, 1, 1, 8, 48, *out, None) == \
        cattn.ERR_UNSUPPORTED
    assert cattn.LIB.attn_bwd_noalloc(*p[:5], None, 0.125, 1, 1, 8, 64, *out, None) == \
        cattn.ERR_INVALID_ARG
    assert "scratch" in cattn.cattn_status_string(cattn.ERR_TOO_LARGE)


def test_misaligned_or_small_workspace():
    assert bwd(ws=ALIGNED + 128) == cattn.ERR_INVALID_ARG
    need = cattn.attn_bwd_workspace_bytes(1, 1, 8, 64)
    assert bwd(ws_bytes=need - 1) == cattn.ERR_INVALID_ARG


def test_empty_shapes_are_noops():
    for B, H, T in ((0, 4, 8), (2, 0, 8), (2, 4, 0)):
        assert fwd(q=None, k=None, v=None, o=None, lse=None, B=B, H=H, T=T) == cattn.OK
        assert bwd(ptrs=[None] * 9, ws=None, ws_bytes=0, B=B, H=H, T=T) == cattn.OK
        assert cattn.LIB.attn_bwd_preprocess(None, None, B, H, T, 64, None, None) == cattn.OK
        assert cattn.attn_bwd_workspace_bytes(B, H, T, 64) == 0


@pytest.mark.parametrize("B,H,T,D", [(1, 1, 1, 16), (16, 12, 1024, 64), (2, 16, 8192, 128),
                                     (3, 5, 1000, 32)])
def test_workspace_formula(B, H, T, D):
    def r256(x):
        return (x + 255) // 256 * 256
    tpad = (T + 127) // 128 * 128
    # the call's status words (256 bytes), the dQ accumulator, LSE2, Delta
    want = 256 + r256(B * H * T * D * 4) + 2 * r256(B * H * tpad * 4)
    assert cattn.attn_bwd_workspace_bytes(B, H, T, D) == want


def test_last_device_status_checks_its_workspace_pointer():
    """cattn_last_device_status reads the status words at the start of a
    backward workspace; a null or misaligned workspace is refused before
    any device call."""
    assert cattn.LIB.cattn_last_device_status(None, None) == cattn.ERR_INVALID_ARG
    assert cattn.LIB.cattn_last_device_status(ALIGNED + 16, None) == cattn.ERR_INVALID_ARG
    assert cattn.LIB.cattn_selftest_wait_timeout_ws(1000, None, None) == cattn.ERR_INVALID_ARG
    assert cattn.LIB.cattn_selftest_wait_timeout_ws(1000, ALIGNED + 128, None) == \
        cattn.ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors():
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        cattn.attn_fwd(q, q, q)
    with pytest.raises(ValueError):
        cattn.attn_fwd(q.float(), q.float(), q.float())


def test_product_has_no_oracle_dependency():
    """The product package never imports or names the oracle."""
    pkg = os.path.dirname(cattn.__file__)
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                with open(os.path.join(dirpath, f)) as fh:
                    src = fh.read()
                assert "oracle" not in src, f
                assert "workloads" not in src, f


# ------------------------------------------------------------ strided calls

def contiguous(H, T, D):
    return _binding.Layout(H * T * D, T * D, D)


def fwd_strided(lay=None, lo=None, B=1, H=2, T=8, D=64):
    c = contiguous(H, T, D)
    lq = lay or c
    return cattn.LIB.attn_fwd_strided(ALIGNED, lq, ALIGNED, c, ALIGNED, c, 0.125, B, H, T, D,
                                      ALIGNED, lo or c, ALIGNED, None, None)


def bwd_strided(bad_index=None, bad=None, B=1, H=2, T=8, D=64):
    c = contiguous(H, T, D)
    lays = [c] * 8   # q, k, v, o, dout, dq, dk, dv
    if bad_index is not None:
        lays[bad_index] = bad
    return cattn.LIB.attn_bwd_strided(ALIGNED, lays[0], ALIGNED, lays[1], ALIGNED, lays[2],
                                      ALIGNED, lays[3], None, ALIGNED, ALIGNED, lays[4], 0.125,
                                      B, H, T, D, ALIGNED, lays[5], ALIGNED, lays[6],
                                      ALIGNED, lays[7], 0, ALIGNED, 1 << 30, None)


@pytest.mark.parametrize("bad", [(0, 64, 8), (512, 64, 0), (512, -64, 8), (512, 64, 12),
                                 (516, 64, 64), (1 << 38, 64, 64), (512, 3, 64)])
def test_strided_calls_reject_bad_strides(bad):
    lay = _binding.Layout(*bad)
    assert fwd_strided(lay=lay) == cattn.ERR_INVALID_ARG
    assert fwd_strided(lo=lay) == cattn.ERR_INVALID_ARG
    for i in range(8):
        assert bwd_strided(i, lay) == cattn.ERR_INVALID_ARG


def test_self_overlapping_output_layouts_are_refused():
    """An output whose own elements would share addresses (rows closer than
    D, heads closer than a head's span, ...) is refused before anything
    runs; the same strides on an input only read, and pass the check."""
    B, H, T, D = 1, 2, 8, 64
    overlapping = [_binding.Layout(H * T * D, T * D, 8),      # rows overlap
                   _binding.Layout(H * T * D, 64, D),         # heads overlap rows
                   _binding.Layout(T * D, T * D, D),          # batches overlap heads
                   _binding.Layout(H * T * D, 8, 128)]        # heads 8 apart, D = 64 wide
    for lay in overlapping:
        assert fwd_strided(lo=lay, B=2) == cattn.ERR_INVALID_ARG, (lay.b, lay.h, lay.t)
        for i in (5, 6, 7):      # dq, dk, dv
            assert bwd_strided(i, lay, B=2) == cattn.ERR_INVALID_ARG, (i, lay.b, lay.h, lay.t)
        # as an input the layout only reads: the argument check lets it through
        # (what follows is the device check, which fails on a host without a GPU)
        assert fwd_strided(lay=lay, B=2) != cattn.ERR_INVALID_ARG
    C = H * D   # (B, T, C) output: heads interleaved within each row, no overlap
    btc = _binding.Layout(T * C, D, C)
    assert fwd_strided(lo=btc, B=2) != cattn.ERR_INVALID_ARG
    padded = _binding.Layout(H * T * (D + 16), T * (D + 16), D + 16)
    assert fwd_strided(lo=padded, B=2) != cattn.ERR_INVALID_ARG
    # decode: its (B, H, Tq, D) output is checked the same way
    c = _binding.Layout(H * 8 * D, 8 * D, D)
    assert cattn.LIB.attn_decode(ALIGNED, c, ALIGNED, c, ALIGNED, c, 0.125, 1, H, 2, 8, D,
                                 ALIGNED, _binding.Layout(H * 2 * D, 2 * D, 16), ALIGNED,
                                 ALIGNED, 1 << 20, None) == cattn.ERR_INVALID_ARG


def test_strided_calls_check_shapes_and_empty():
    assert fwd_strided(D=48) == cattn.ERR_UNSUPPORTED
    assert bwd_strided(D=48) == cattn.ERR_UNSUPPORTED
    assert fwd_strided(T=0) == cattn.OK
    assert bwd_strided(B=0) == cattn.OK


def test_split_qkv_views_share_the_fused_buffer():
    import torch as t
    B, T, H, D = 2, 16, 4, 32
    qkv = t.arange(B * T * 3 * H * D, dtype=t.float32).view(B, T, 3 * H * D)
    q, k, v = cattn.split_qkv(qkv, H)
    C = H * D
    assert q.shape == (B, H, T, D)
    assert q.stride() == (T * 3 * C, D, 3 * C, 1) == k.stride() == v.stride()
    assert k.data_ptr() - q.data_ptr() == C * qkv.element_size()
    assert v.data_ptr() - q.data_ptr() == 2 * C * qkv.element_size()
    # element (b, h, t, d) of q is qkv[b, t, h*D + d]
    assert float(q[1, 2, 3, 4]) == float(qkv[1, 3, 2 * D + 4])
    assert float(v[0, 3, 5, 1]) == float(qkv[0, 5, 2 * C + 3 * D + 1])


# ------------------------------------------------------------ dropout calls

def fwd_dropout(drop, B=1, H=2, T=8, D=64):
    c = contiguous(H, T, D)
    return cattn.LIB.attn_fwd_dropout(ALIGNED, c, ALIGNED, c, ALIGNED, c, 0.125, B, H, T, D,
                                      drop, ALIGNED, c, ALIGNED, None, None)


def bwd_dropout(drop, B=1, H=2, T=8, D=64):
    c = contiguous(H, T, D)
    return cattn.LIB.attn_bwd_dropout(ALIGNED, c, ALIGNED, c, ALIGNED, c, ALIGNED, c, None,
                                      ALIGNED, ALIGNED, c, 0.125, B, H, T, D, drop,
                                      ALIGNED, c, ALIGNED, c, ALIGNED, c, 0, ALIGNED, 1 << 30,
                                      None)


@pytest.mark.parametrize("p", [1.0, -0.01, float("nan"), float("inf"), 7.0])
def test_dropout_calls_reject_bad_probability(p):
    import ctypes
    d = ctypes.byref(_binding.Dropout(p, 1, 2))
    assert fwd_dropout(d) == cattn.ERR_INVALID_ARG
    assert bwd_dropout(d) == cattn.ERR_INVALID_ARG


def test_dropout_calls_accept_empty_and_null():
    import ctypes
    d = ctypes.byref(_binding.Dropout(0.2, 1, 2))
    assert fwd_dropout(d, T=0) == cattn.OK
    assert bwd_dropout(d, B=0) == cattn.OK
    assert fwd_dropout(d, D=48) == cattn.ERR_UNSUPPORTED
    assert fwd_dropout(None, T=0) == cattn.OK


def test_dropout_params_helper():
    assert cattn.dropout_params(0.0) is None and cattn.dropout_params(None) is None
    d = cattn.dropout_params(0.2, seed=-1, offset=1 << 33)
    assert d.seed == (1 << 64) - 1 and d.offset == 0 and abs(d.p - 0.2) < 1e-7


# ------------------------------------------------------------ decode call

def decode(Tq=1, L=8, B=1, H=2, D=64, lay=None, ws_bytes=1 << 20):
    c = _binding.Layout(H * L * D, L * D, D)
    return cattn.LIB.attn_decode(ALIGNED, lay or c, ALIGNED, c, ALIGNED, c, 0.125, B, H, Tq, L,
                                 D, ALIGNED, c, ALIGNED, ALIGNED, ws_bytes, None)


def test_decode_checks_arguments_before_the_device():
    assert decode(Tq=9) == cattn.ERR_UNSUPPORTED
    assert decode(Tq=0) == cattn.ERR_INVALID_ARG
    assert decode(Tq=4, L=3) == cattn.ERR_INVALID_ARG
    assert decode(D=48) == cattn.ERR_UNSUPPORTED
    assert decode(B=0) == cattn.OK
    assert decode(lay=_binding.Layout(512, 64, 12)) == cattn.ERR_INVALID_ARG


def test_dropout_mask_bytes_formula():
    # 2 KB (128 x 128 bits) per tile on or below the diagonal, per head
    for B, H, T in [(1, 1, 1), (2, 3, 128), (2, 3, 129), (16, 12, 1024), (1, 2, 8192)]:
        n = (T + 127) // 128
        assert cattn.attn_dropout_mask_bytes(B, H, T) == B * H * n * (n + 1) // 2 * 2048
    assert cattn.attn_dropout_mask_bytes(0, 1, 64) == 0
    assert cattn.attn_dropout_mask_bytes(1, 1, 0) == 0
    assert cattn.attn_dropout_mask_bytes(1, 1, (1 << 20) + 1) == 0


def test_dropout_mask_alignment_is_checked_before_the_device():
    c = _binding.Layout(2 * 8 * 64, 8 * 64, 64)
    d = _binding.Dropout(0.5, 1, 2, ALIGNED + 8)     # not 16-byte aligned
    assert cattn.LIB.attn_fwd_dropout(ALIGNED, c, ALIGNED, c, ALIGNED, c, 0.125, 1, 2, 8, 64,
                                      ctypes.byref(d), ALIGNED, c, ALIGNED, None,
                                      None) == cattn.ERR_INVALID_ARG
    assert ctypes.sizeof(_binding.Dropout) == 32


def test_decode_needs_no_workspace():
    # the CTAs of a head (a thread-block cluster) merge their partial
    # results in distributed shared memory: no workspace for any shape
    for B, H, Tq, L, D in [(1, 1, 1, 1, 16), (2, 3, 4, 257, 64), (16, 12, 1, 1024, 64),
                           (1, 2, 8, 4096, 128), (2, 16, 1, 8192, 128), (64, 12, 2, 300, 32),
                           (16, 12, 8, 1024, 64), (1, 1, 9, 16, 64), (1, 1, 2, 1, 64)]:
        assert cattn.attn_decode_workspace_bytes(B, H, Tq, L, D) == 0


# ------------------------------------------------------------ Python checks

def test_python_calls_reject_mismatched_shapes_before_any_launch():
    import torch as t
    q = t.zeros(1, 2, 16, 64, dtype=t.bfloat16)
    short = t.zeros(1, 2, 8, 64, dtype=t.bfloat16)
    with pytest.raises(ValueError, match="share the"):
        cattn.attn_fwd(q, short, q)
    with pytest.raises(ValueError, match="share the"):
        cattn.attn_fwd_ex(q, q, short)
    lse = t.zeros(1, 2, 16)
    with pytest.raises(ValueError, match="share the"):
        cattn.attn_bwd(q, q, q, q, lse, short)
    with pytest.raises(ValueError, match="share the"):
        cattn.attn_bwd_noalloc(q, q, short, q, lse, q)
    with pytest.raises(ValueError, match="share the"):
        cattn.attn_bwd_preprocess(q, short)


def test_python_buffers_must_be_device_memory_of_the_right_shape():
    import torch as t
    like = t.zeros(1, 2, 16, 64, dtype=t.bfloat16)
    with pytest.raises(ValueError, match="output must be on"):
        cattn._want(t.zeros(1, 2, 16, 64, dtype=t.bfloat16), like, t.bfloat16, (1, 2, 16, 64))
    with pytest.raises(ValueError, match="shape"):
        cattn._want(t.zeros(1, 2, 8, 64, dtype=t.bfloat16), like, t.bfloat16, (1, 2, 16, 64))
    with pytest.raises(ValueError, match="workspace"):
        cattn._workspace(t.zeros(1024, dtype=t.uint8), like, 512)
    with pytest.raises(ValueError, match="lse must have shape"):
        cattn._vector(t.zeros(1, 2, 8), like, (1, 2, 16), "lse")
    with pytest.raises(ValueError, match="fp32"):
        cattn._vector(t.zeros(1, 2, 16), like, (1, 2, 16), "lse")   # a CPU tensor
    assert cattn._nbytes(t.zeros(10, dtype=t.float32)) == 40


# ------------------------------------------------------------ the header as C

@pytest.mark.parametrize("lang,std", [("c", "c99"), ("c", "c11"), ("c++", "c++17")])
def test_header_is_plain_c_and_cpp(lang, std, tmp_path):
    """include/cattn.h compiles on its own, warning-free, as C and as C++,
    and a C program can take the address of every entry point (the ABI has
    no C++ types in it)."""
    import re
    import shutil
    import subprocess
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    inc = os.path.join(ROOT, "include")
    names = re.findall(r"CATTN_API\s+[\w\s\*]+?\b(\w+)\s*\(",
                       open(os.path.join(inc, "cattn.h")).read())
    assert "attn_fwd" in names and "attn_decode" in names and "attn_bwd_dropout" in names
    src = tmp_path / ("t.c" if lang == "c" else "t.cpp")
    body = "\n".join(f"  p = (fn)&{n}; (void)p;" for n in names)
    src.write_text(f'#include "cattn.h"\ntypedef void (*fn)(void);\nint main(void) {{\n'
                   f'  fn p;\n{body}\n  return 0;\n}}\n')
    r = subprocess.run([cc, f"-std={std}", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-fsyntax-only", "-I", inc, str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_strided_dropout_and_decode_calls_check_alignment_and_nulls():
    """Every pointer of the newer entry points is checked before anything
    runs: bf16 tensors 16-byte aligned, LSE 4, workspace 256; nulls
    refused."""
    import ctypes
    c = contiguous(2, 8, 64)
    d = ctypes.byref(_binding.Dropout(0.1, 1, 2))
    fwd_args = lambda q=ALIGNED, k=ALIGNED, v=ALIGNED, o=ALIGNED, lse=ALIGNED, olo=None: (  # noqa: E731
        q, c, k, c, v, c, 0.125, 1, 2, 8, 64, d, o, c, lse, olo, None)
    for bad in (dict(q=ALIGNED + 8), dict(k=ALIGNED + 2), dict(v=ALIGNED + 8), dict(o=ALIGNED + 8),
                dict(lse=ALIGNED + 2), dict(olo=ALIGNED + 8), dict(q=None), dict(lse=None)):
        assert cattn.LIB.attn_fwd_dropout(*fwd_args(**bad)) == cattn.ERR_INVALID_ARG, bad
    ptrs = [ALIGNED] * 10   # q k v o o_lo lse do dq dk dv
    for i, bad in ((0, ALIGNED + 8), (3, ALIGNED + 8), (4, ALIGNED + 8), (5, ALIGNED + 2),
                   (6, ALIGNED + 8), (7, ALIGNED + 8), (8, None), (9, ALIGNED + 8)):
        p = list(ptrs)
        p[i] = bad
        r = cattn.LIB.attn_bwd_dropout(p[0], c, p[1], c, p[2], c, p[3], c, p[4], p[5], p[6], c,
                                       0.125, 1, 2, 8, 64, d, p[7], c, p[8], c, p[9], c, 0,
                                       ALIGNED, 1 << 30, None)
        assert r == cattn.ERR_INVALID_ARG, (i, bad)
    r = cattn.LIB.attn_bwd_dropout(*[x for t in zip(ptrs[:4], [c] * 4) for x in t], ALIGNED,
                                   ALIGNED, ALIGNED, c, 0.125, 1, 2, 8, 64, d, ALIGNED, c,
                                   ALIGNED, c, ALIGNED, c, 0, ALIGNED + 128, 1 << 30, None)
    assert r == cattn.ERR_INVALID_ARG    # workspace not 256-byte aligned
    for kw in (dict(q=ALIGNED + 8), dict(k=ALIGNED + 8), dict(o=ALIGNED + 8),
               dict(lse=ALIGNED + 2), dict(v=None)):
        a = dict(q=ALIGNED, k=ALIGNED, v=ALIGNED, o=ALIGNED, lse=ALIGNED, ws=ALIGNED)
        a.update(kw)
        r = cattn.LIB.attn_decode(a["q"], c, a["k"], c, a["v"], c, 0.125, 1, 2, 1, 8, 64,
                                  a["o"], c, a["lse"], a["ws"], 1 << 20, None)
        assert r == cattn.ERR_INVALID_ARG, kw
