"""GPU test of attn_bwd_noalloc, the backward entry point that allocates
nothing and works in the library's fixed scratch array instead of a
caller-provided workspace.  It exists for callers that cannot allocate
device memory (runtimes that hand a plugin only its inputs and outputs,
or code that must avoid cudaMalloc/cudaFree and the synchronisation they
can cause).

Two calls in a row, on different shapes, are compared with the ordinary
workspace-taking attn_bwd on the same inputs, within the tolerance the
parity tests use.  The second call also shows that contents the first call
left in the shared scratch do not leak into its result.  This file is
collected last so that a run stopping at the first failure has already
run every other test.
"""

import math

import pytest
import torch

from parity_util import check_bf16
from workloads import as_f64, bf16_inputs

pytestmark = pytest.mark.gpu


def _noalloc_through_c_abi(lib, q, k, v, o, lse, do, scale):
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    st = lib.LIB.attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  lse.data_ptr(), do.data_ptr(), float(scale), *q.shape,
                                  dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream)
    assert st == lib.OK, lib.cattn_status_string(st)
    return dq, dk, dv


def test_static_scratch_backward_matches_workspace_backward(lib):
    cases = [((2, 3, 300, 64), 4101), ((1, 4, 1000, 64), 4102), ((2, 2, 200, 128), 4103)]
    for (B, H, T, D), seed in cases:
        scale = 1.0 / math.sqrt(D)
        q, k, v, do = (t.cuda() for t in bf16_inputs(B, H, T, D, seed=seed))
        o, lse = lib.attn_fwd(q, k, v, scale)
        want = lib.attn_bwd(q, k, v, o, lse, do, scale)           # existing entry point
        got = _noalloc_through_c_abi(lib, q, k, v, o, lse, do, scale)
        torch.cuda.synchronize()
        assert lib.cattn_get_device_status() == lib.OK
        for name, g, w in zip(("dq", "dk", "dv"), got, want):
            check_bf16(f"{name} B{B} H{H} T{T} D{D}", as_f64(g), as_f64(w))


def test_second_call_allocates_no_device_memory(lib):
    """The call's promise: after the first call on a device (which looks up
    the array's address), a call leaves the device's free memory unchanged.
    The outputs are allocated before the measurement and passed in; this
    goes through the Python wrapper, whose only work is marshalling."""
    B, H, T, D = 2, 3, 300, 64
    scale = 1.0 / math.sqrt(D)
    q, k, v, do = (t.cuda() for t in bf16_inputs(B, H, T, D, seed=4104))
    o, lse = lib.attn_fwd(q, k, v, scale)
    outs = [torch.empty_like(q) for _ in range(3)]
    lib.attn_bwd_noalloc(q, k, v, o, lse, do, scale, dq=outs[0], dk=outs[1], dv=outs[2])
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    got = lib.attn_bwd_noalloc(q, k, v, o, lse, do, scale, dq=outs[0], dk=outs[1], dv=outs[2])
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)
    assert all(g is w for g, w in zip(got, outs))
    want = lib.attn_bwd(q, k, v, o, lse, do, scale)
    torch.cuda.synchronize()
    assert lib.cattn_get_device_status() == lib.OK
    for name, g, w in zip(("dq", "dk", "dv"), got, want):
        check_bf16(f"{name} (Python wrapper)", as_f64(g), as_f64(w))
