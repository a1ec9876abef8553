"""GPU parity of the strided calls: q, k, v read in place from a fused
(B, T, 3C) projection, O written into a (B, T, C) buffer, dO read from and
dQ, dK, dV written into such layouts.

The strided kernels do the same arithmetic as the contiguous ones, only at
other addresses, so O, LSE, dK and dV must match the contiguous calls bit
for bit.  dQ is summed across key tiles in an order that can vary between
runs, so it must match to within a bf16 rounding step.  A sampled subset of
heads is also checked against the fp64 oracle.
"""

import pytest
import torch

import oracle
from parity_util import check_bf16
from workloads import as_f64, bf16_inputs

pytestmark = pytest.mark.gpu


def fused(q, k, v):
    """(B, H, T, D) q, k, v -> one (B, T, 3C) projection holding them."""
    B, H, T, D = q.shape
    return torch.cat([t.transpose(1, 2).reshape(B, T, H * D) for t in (q, k, v)], dim=2)


def merged(x):
    """(B, H, T, D) -> (B, T, H*D)."""
    B, H, T, D = x.shape
    return x.transpose(1, 2).reshape(B, T, H * D)


def close_bf16_steps(a, b, what):
    """a and b equal except for one bf16 rounding step of |b|, plus an fp32
    summation-order slack of 1e-5 of the largest |b| (dQ's fp32 partial sums
    arrive from several key tiles in a run-dependent order)."""
    a, b = a.double(), b.double()
    step = b.abs() * 2.0 ** -7 + 1e-5 * b.abs().max().item()
    bad = (a - b).abs() > step
    assert not bad.any(), f"{what}: {(a - b).abs().max().item()}"


@pytest.mark.parametrize("shape", [(2, 4, 300, 64), (1, 3, 129, 32), (2, 2, 200, 16),
                                   (1, 2, 260, 128)])
@pytest.mark.parametrize("residual", [False, True])
def test_fused_projection_layout_matches_contiguous(lib, shape, residual):
    B, H, T, D = shape
    dev = torch.device("cuda:0")
    q, k, v, do = (t.to(dev) for t in bf16_inputs(B, H, T, D, seed=4242 + D, qk_std=1.0))
    scale = D ** -0.5
    # contiguous reference path
    if residual:
        o_c, lse_c, olo_c = lib.attn_fwd_ex(q, k, v, scale)
        dq_c, dk_c, dv_c = lib.attn_bwd(q, k, v, o_c, lse_c, do, scale, o_lo=olo_c)
    else:
        o_c, lse_c = lib.attn_fwd(q, k, v, scale)
        dq_c, dk_c, dv_c = lib.attn_bwd(q, k, v, o_c, lse_c, do, scale)
    # strided path: views into fused / merged buffers
    qkv = fused(q, k, v)
    qs, ks, vs = lib.split_qkv(qkv, H)
    y = torch.full((B, T, H * D), float("nan"), dtype=torch.bfloat16, device=dev)
    o_s = y.view(B, T, H, D).transpose(1, 2)
    olo_s = None
    if residual:
        y_lo = torch.full_like(y, float("nan"))
        olo_s = y_lo.view(B, T, H, D).transpose(1, 2)
    _, lse_s, _ = lib.attn_fwd_strided(qs, ks, vs, scale, o=o_s, o_lo=olo_s)
    dy = merged(do).contiguous()
    do_s = dy.view(B, T, H, D).transpose(1, 2)
    dqkv = torch.full_like(qkv, float("nan"))
    dqs, dks, dvs = lib.split_qkv(dqkv, H)
    lib.attn_bwd_strided(qs, ks, vs, o_s, lse_s, do_s, scale, dq=dqs, dk=dks, dv=dvs, o_lo=olo_s)
    torch.cuda.synchronize()
    assert lib.cattn_get_device_status() == lib.OK
    assert torch.equal(o_s, o_c)
    assert torch.equal(lse_s, lse_c)
    if residual:
        assert torch.equal(olo_s, olo_c)
    assert torch.equal(dks, dk_c)
    assert torch.equal(dvs, dv_c)
    close_bf16_steps(dqs, dq_c, "dq")
    # every element of the fused gradient was written
    assert not torch.isnan(dqkv).any() and not torch.isnan(y).any()


def test_strided_against_oracle(lib):
    B, H, T, D = 2, 3, 333, 64
    dev = torch.device("cuda:0")
    q, k, v, do = bf16_inputs(B, H, T, D, seed=777, qk_std=1.0)
    scale = D ** -0.5
    qkv = fused(q, k, v).to(dev)
    y = lib.CausalAttentionQKV.apply(qkv.requires_grad_(True), H, scale)
    y.backward(merged(do).to(dev))
    torch.cuda.synchronize()
    dqkv = qkv.grad
    C = H * D
    got_o = y.view(B, T, H, D).transpose(1, 2)
    got = {"o": got_o,
           "dq": dqkv[..., :C].view(B, T, H, D).transpose(1, 2),
           "dk": dqkv[..., C:2 * C].view(B, T, H, D).transpose(1, 2),
           "dv": dqkv[..., 2 * C:].view(B, T, H, D).transpose(1, 2)}
    qn, kn, vn, don = (as_f64(t) for t in (q, k, v, do))
    o, _ = oracle.attention_forward(qn, kn, vn, scale)
    dq, dk, dv = oracle.attention_backward(qn, kn, vn, don, scale)
    for n, ref in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv)):
        check_bf16(n, as_f64(got[n]), ref)


def test_fp32_gradients_strided(lib):
    """grad_dtype fp32 with strided fp32 outputs (the strides count fp32
    elements)."""
    B, H, T, D = 1, 2, 257, 64
    dev = torch.device("cuda:0")
    q, k, v, do = (t.to(dev) for t in bf16_inputs(B, H, T, D, seed=99, qk_std=1.0))
    scale = D ** -0.5
    o, lse, o_lo = lib.attn_fwd_ex(q, k, v, scale)
    ref = lib.attn_bwd(q, k, v, o, lse, do, scale, o_lo=o_lo, grad_dtype=torch.float32)
    g = torch.full((B, T, 3 * H * D), float("nan"), dtype=torch.float32, device=dev)
    dqs, dks, dvs = lib.split_qkv(g, H)
    lib.attn_bwd_strided(q, k, v, o, lse, do, scale, dq=dqs, dk=dks, dv=dvs, o_lo=o_lo,
                         grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(dks, ref[1]) and torch.equal(dvs, ref[2])
    assert torch.allclose(dqs, ref[0], rtol=1e-5, atol=1e-5 * ref[0].abs().max().item())
    assert not torch.isnan(g).any()


def test_plain_and_residual_calls_run_different_kernels(lib):
    """The plain calls (bf16 P, bf16 dS) and the residual calls (hi/lo P
    and dS) are different kernels: their outputs differ in low bits.  Guards
    the dispatch: a plain call that ran the residual kernel would still
    pass every tolerance test."""
    B, H, T, D = 1, 4, 384, 64
    dev = torch.device("cuda:0")
    q, k, v, do = (t.to(dev) for t in bf16_inputs(B, H, T, D, seed=1001, qk_std=1.0))
    scale = D ** -0.5
    for strided in (False, True):
        if strided:
            qkv = fused(q, k, v)
            qs, ks, vs = lib.split_qkv(qkv, H)
            o1, l1, _ = lib.attn_fwd_strided(qs, ks, vs, scale)
            o2, l2, olo = lib.attn_fwd_strided(qs, ks, vs, scale, o_lo=torch.empty_like(q))
            g1 = lib.attn_bwd_strided(qs, ks, vs, o1, l1, do, scale)
            g2 = lib.attn_bwd_strided(qs, ks, vs, o2, l2, do, scale, o_lo=olo)
        else:
            o1, l1 = lib.attn_fwd(q, k, v, scale)
            o2, l2, olo = lib.attn_fwd_ex(q, k, v, scale)
            g1 = lib.attn_bwd(q, k, v, o1, l1, do, scale)
            g2 = lib.attn_bwd(q, k, v, o2, l2, do, scale, o_lo=olo)
        torch.cuda.synchronize()
        assert not torch.equal(o1, o2), strided
        assert not torch.equal(g1[1], g2[1]), strided


@pytest.mark.parametrize("D", [32, 64, 128])
def test_padded_rows_collapse_to_the_flat_kernels(lib, D):
    """(B, H, T, D) views of buffers whose rows are padded to D + 16: the
    batch stride is still H head strides, so the FLAT instances run (3-D
    tensor maps with a row stride other than D, the strided preprocess)."""
    B, H, T = 2, 3, 200
    dev = torch.device("cuda:0")
    q, k, v, do = (t.to(dev) for t in bf16_inputs(B, H, T, D, seed=606 + D, qk_std=1.0))
    scale = D ** -0.5

    def padded(x):
        buf = torch.full((B, H, T, D + 16), float("nan"), dtype=x.dtype, device=dev)
        buf[..., :D] = x
        return buf[..., :D]

    o_c, lse_c, olo_c = lib.attn_fwd_ex(q, k, v, scale)
    g_c = lib.attn_bwd(q, k, v, o_c, lse_c, do, scale, o_lo=olo_c)
    qp, kp, vp, dop = (padded(t) for t in (q, k, v, do))
    o_p = padded(torch.zeros_like(q))
    olo_p = padded(torch.zeros_like(q))
    _, lse_p, _ = lib.attn_fwd_strided(qp, kp, vp, scale, o=o_p, o_lo=olo_p)
    gp = [padded(torch.zeros_like(q)) for _ in range(3)]
    lib.attn_bwd_strided(qp, kp, vp, o_p, lse_p, dop, scale, dq=gp[0], dk=gp[1], dv=gp[2],
                         o_lo=olo_p)
    torch.cuda.synchronize()
    assert lib.cattn_get_device_status() == lib.OK
    assert torch.equal(o_p, o_c) and torch.equal(lse_p, lse_c) and torch.equal(olo_p, olo_c)
    assert torch.equal(gp[1], g_c[1]) and torch.equal(gp[2], g_c[2])
    close_bf16_steps(gp[0], g_c[0], "dq")
