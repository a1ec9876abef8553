"""Head sizes the kernels do not take (12 in the pages' 48-channel,
4-head configuration): zero-padded head layouts set up once in the
projection weights.  CPU tests of the weight helpers (exact, in fp64), and
a check with the fp64 oracle that attention over zero-padded heads is
attention over the original heads."""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import causal_self_attention_flash_b200 as cattn
import oracle


def test_padded_head_size():
    assert [cattn.padded_head_size(d) for d in (1, 12, 16, 17, 33, 64, 100, 128)] == \
        [16, 16, 16, 32, 64, 64, 128, 128]
    with pytest.raises(ValueError):
        cattn.padded_head_size(129)


def test_projection_padding_is_exact():
    g = torch.Generator().manual_seed(3)
    B, T, C, H, d = 2, 5, 48, 4, 12
    W = torch.randn(3 * C, C, generator=g, dtype=torch.float64)
    b = torch.randn(3 * C, generator=g, dtype=torch.float64)
    Wo = torch.randn(C, C, generator=g, dtype=torch.float64)
    x = torch.randn(B, T, C, generator=g, dtype=torch.float64)
    Wp, bp = cattn.pad_qkv_projection(W, b, H, d)
    assert Wp.shape == (3 * H * 16, C) and bp.shape == (3 * H * 16,)
    qkv = x @ W.T + b
    qkvp = (x @ Wp.T + bp).view(B, T, 3, H, 16)
    assert torch.equal(qkvp[..., :d], qkv.view(B, T, 3, H, d))
    assert torch.count_nonzero(qkvp[..., d:]) == 0
    # out projection: padded y columns meet zero weight columns
    y = torch.randn(B, T, H, d, generator=g, dtype=torch.float64)
    yp = torch.zeros(B, T, H, 16, dtype=torch.float64)
    yp[..., :d] = y
    Wop = cattn.pad_out_projection(Wo, H, d)
    assert Wop.shape == (C, H * 16)
    assert torch.allclose(yp.reshape(B, T, -1) @ Wop.T, y.reshape(B, T, -1) @ Wo.T,
                          rtol=0, atol=1e-12)


def test_attention_over_zero_padded_heads_is_the_original():
    """fp64 oracle: padding q, k, v with zero columns and keeping the scale
    of the original head size leaves O (first d columns) and LSE unchanged,
    puts zeros in O's padded columns, and the same holds for the gradients
    when dO's padded columns are zero."""
    rng = np.random.default_rng(5)
    B, H, T, d, dp = 1, 2, 9, 12, 16
    q, k, v, do = (rng.standard_normal((B, H, T, d)) for _ in range(4))
    pad = lambda x: np.concatenate([x, np.zeros(x.shape[:-1] + (dp - d,))], -1)  # noqa: E731
    s = 1 / math.sqrt(d)
    o, lse = oracle.attention_forward(q, k, v, s)
    op, lsep = oracle.attention_forward(pad(q), pad(k), pad(v), s)
    assert np.allclose(op[..., :d], o, rtol=1e-13, atol=1e-13) and np.allclose(lsep, lse)
    assert not op[..., d:].any()
    g = oracle.attention_backward(q, k, v, do, s)
    gp = oracle.attention_backward(pad(q), pad(k), pad(v), pad(do), s)
    for a, b in zip(g, gp):
        assert np.allclose(b[..., :d], a, rtol=1e-12, atol=1e-12) and not b[..., d:].any()


@pytest.mark.gpu
def test_head_size_12_runs_on_the_16_kernels(lib):
    """n_embd 48, 4 heads (head size 12): the padded projection feeds the
    fused-layout autograd call with head size 16 and scale 1/sqrt(12).  The
    real columns match the fp64 oracle on the unpadded heads; the padded
    columns of y and of the gradient are exactly zero."""
    from parity_util import check_bf16
    from workloads import as_f64
    g = torch.Generator().manual_seed(12)
    B, T, C, H, d, dp = 4, 200, 48, 4, 12, 16
    W = torch.randn(3 * C, C, generator=g) / math.sqrt(C)
    x = torch.randn(B, T, C, generator=g)
    Wp, _ = cattn.pad_qkv_projection(W, None, H, d)
    qkvp = (x @ Wp.T).to(torch.bfloat16)                    # (B, T, 3 * H * 16)
    heads = qkvp.float().view(B, T, 3, H, dp)[..., :d]       # the unpadded q, k, v
    q, k, v = (heads[:, :, i].transpose(1, 2) for i in range(3))
    dy = torch.randn(B, T, H, d, generator=g).to(torch.bfloat16)
    dyp = torch.zeros(B, T, H, dp, dtype=torch.bfloat16)
    dyp[..., :d] = dy
    dev = torch.device("cuda:0")
    qkv_dev = qkvp.to(dev).requires_grad_(True)
    y = lib.CausalAttentionQKV.apply(qkv_dev, H, 1 / math.sqrt(d))
    y.backward(dyp.reshape(B, T, H * dp).to(dev))
    torch.cuda.synchronize()
    yv = y.detach().view(B, T, H, dp)
    gv = qkv_dev.grad.view(B, T, 3, H, dp)
    assert bool((yv[..., d:] == 0).all()) and bool((gv[..., d:] == 0).all())
    qn, kn, vn = (as_f64(t) for t in (q, k, v))
    don = as_f64(dy.transpose(1, 2))
    ro, _ = oracle.attention_forward(qn, kn, vn, 1 / math.sqrt(d))
    rq, rk, rv = oracle.attention_backward(qn, kn, vn, don, 1 / math.sqrt(d))
    check_bf16("o", as_f64(yv[..., :d].transpose(1, 2)), ro)
    for i, (n, ref) in enumerate((("dq", rq), ("dk", rk), ("dv", rv))):
        check_bf16(n, as_f64(gv[:, :, i, :, :d].transpose(1, 2)), ref)
