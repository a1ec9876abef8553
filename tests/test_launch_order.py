"""GPU checks of the launch mode: the forward, the backward's kernels and
decode are programmatic dependents of the kernel before them on the stream
(each waits for it before touching memory).

* A CUDA graph of forward + backward, replayed, gives the eager calls'
  results bit for bit (the dependency is captured as a graph edge).
* Inputs rewritten by a torch kernel right before the call are what the
  call reads: every call here runs immediately after an in-place torch
  kernel on its inputs, and the results equal those of a fresh call on
  inputs made in advance (dQ to within its run-dependent rounding), with
  and without dropout.
"""

import pytest
import torch

from workloads import bf16_inputs

pytestmark = pytest.mark.gpu


def _dev(*ts):
    return tuple(t.to("cuda:0") for t in ts)


def _same(name, a, b):
    """Bit for bit, except dQ: its fp32 tile sums arrive in a run-dependent
    order, so its bf16 result may differ by one rounding step."""
    if name != "dq":
        assert torch.equal(a, b), name
        return
    a, b = a.float(), b.float()
    assert torch.all((a - b).abs() <= b.abs() / 128 + 1e-6 * b.abs().max()), name


@pytest.mark.parametrize("shape", [(2, 3, 300, 64), (1, 2, 1024, 128), (4, 2, 129, 32)])
def test_graph_replay_matches_eager(lib, shape):
    B, H, T, D = shape
    q, k, v, do = _dev(*bf16_inputs(B, H, T, D, seed=9000 + T))
    scale = D ** -0.5
    o_e, lse_e = lib.attn_fwd(q, k, v, scale)
    dq_e, dk_e, dv_e = lib.attn_bwd(q, k, v, o_e, lse_e, do, scale)
    torch.cuda.synchronize()

    o, lse = torch.empty_like(q), torch.empty(B, H, T, device=q.device)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws = torch.empty(lib.attn_bwd_workspace_bytes(B, H, T, D), dtype=torch.uint8, device=q.device)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up outside the capture
        lib.attn_fwd(q, k, v, scale, o=o, lse=lse)
        lib.attn_bwd(q, k, v, o, lse, do, scale, dq=dq, dk=dk, dv=dv, workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    for t in (o, lse, dq, dk, dv):
        t.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        lib.attn_fwd(q, k, v, scale, o=o, lse=lse)
        lib.attn_bwd(q, k, v, o, lse, do, scale, dq=dq, dk=dk, dv=dv, workspace=ws)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert lib.cattn_get_device_status() == lib.OK
    for name, a, b in (("o", o, o_e), ("lse", lse, lse_e), ("dq", dq, dq_e), ("dk", dk, dk_e),
                       ("dv", dv, dv_e)):
        _same(name, a, b)


def test_inputs_written_just_before_the_call(lib):
    B, H, T, D = 4, 4, 512, 64
    scale = D ** -0.5
    q, k, v, do = _dev(*bf16_inputs(B, H, T, D, seed=77))
    # the expected results, on inputs scaled in advance
    q2, v2, do2 = q * 2, v * 0.5, do * 3
    torch.cuda.synchronize()
    o_ref, lse_ref = lib.attn_fwd(q2, k, v2, scale)
    g_ref = lib.attn_bwd(q2, k, v2, o_ref, lse_ref, do2, scale)
    torch.cuda.synchronize()
    for _ in range(3):
        qa, va, doa = q.clone(), v.clone(), do.clone()
        torch.cuda.synchronize()
        # each call follows the torch kernel that writes its inputs
        qa.mul_(2)
        va.mul_(0.5)
        o, lse = lib.attn_fwd(qa, k, va, scale)
        doa.mul_(3)
        g = lib.attn_bwd(qa, k, va, o, lse, doa, scale)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
        for name, a, b in zip(("dq", "dk", "dv"), g, g_ref):
            _same(name, a, b)


def test_decode_after_cache_write(lib):
    B, H, L, D, Tq = 8, 12, 1024, 64, 2
    g = torch.Generator().manual_seed(5)
    q = torch.randn(B, H, Tq, D, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(B, H, L, D, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, H, L, D, generator=g).to(torch.bfloat16).cuda()
    k_new = torch.randn(B, H, 1, D, generator=g).to(torch.bfloat16).cuda()
    kr, vr = k.clone(), v.clone()
    kr[:, :, L - 1:] = k_new
    vr[:, :, L - 1:] = k_new
    torch.cuda.synchronize()
    o_ref, lse_ref = lib.attn_decode(q, kr, vr, L, D ** -0.5)
    torch.cuda.synchronize()
    for _ in range(3):
        kc, vc = k.clone(), v.clone()
        torch.cuda.synchronize()
        kc[:, :, L - 1:].copy_(k_new)  # the new position's key and value,
        vc[:, :, L - 1:].copy_(k_new)  # written right before the decode
        o, lse = lib.attn_decode(q, kc, vc, L, D ** -0.5)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_dropout_inputs_written_just_before_the_call(lib):
    B, H, T, D = 2, 4, 384, 64
    scale = D ** -0.5
    q, k, v, do = _dev(*bf16_inputs(B, H, T, D, seed=78))
    drop = lib.dropout_params(0.2, seed=11, offset=3)
    q2, v2, do2 = q * 2, v * 0.5, do * 3
    torch.cuda.synchronize()
    o_ref, lse_ref, _ = lib.attn_fwd_strided(q2, k, v2, scale, dropout=drop)
    g_ref = lib.attn_bwd_strided(q2, k, v2, o_ref, lse_ref, do2, scale, dropout=drop)
    torch.cuda.synchronize()
    for _ in range(3):
        qa, va, doa = q.clone(), v.clone(), do.clone()
        torch.cuda.synchronize()
        qa.mul_(2)
        va.mul_(0.5)
        o, lse, _ = lib.attn_fwd_strided(qa, k, va, scale, dropout=drop)
        doa.mul_(3)
        g = lib.attn_bwd_strided(qa, k, va, o, lse, doa, scale, dropout=drop)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
        for name, a, b in zip(("dq", "dk", "dv"), g, g_ref):
            _same(name, a, b)
