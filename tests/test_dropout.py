"""GPU parity of attention dropout (attn_fwd_dropout / attn_bwd_dropout)
against the fp64 dropout oracle, plus a bit-exact check of the mask.

The mask is read back from the kernels directly: with V = a shifted
identity (V[j, d] = 1 iff j = d + shift) the forward output is
O[i, d] = P~[i, d + shift], whose zeros are exactly the dropped entries;
with dO a shifted identity the backward's dV[j, d] = P~[d + shift, j]
shows the mask the backward derived (its threads hold keys, not queries,
and rebuild the bits by a warp shuffle).  Both must equal the oracle's
Philox mask bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle
import oracle.dropout as odrop
from parity_util import check_bf16, check_lse
from workloads import as_f64, bf16_inputs

pytestmark = pytest.mark.gpu

SEED = 0x0123456789ABCDEF


def run(lib, q, k, v, do, scale, p, seed, offset, residual=False, f32=False):
    dev = torch.device("cuda:0")
    q, k, v, do = (t.to(dev) for t in (q, k, v, do))
    drop = lib.dropout_params(p, seed, offset)
    o = torch.empty_like(q)
    o_lo = torch.empty_like(q) if residual else None
    _, lse, _ = lib.attn_fwd_strided(q, k, v, scale, o=o, o_lo=o_lo, dropout=drop)
    gd = torch.float32 if f32 else torch.bfloat16
    dq, dk, dv = lib.attn_bwd_strided(q, k, v, o, lse, do, scale, o_lo=o_lo, dropout=drop,
                                      grad_dtype=gd)
    torch.cuda.synchronize()
    assert lib.cattn_get_device_status() == lib.OK
    return o, lse, dq, dk, dv


@pytest.mark.parametrize("shape", [(1, 2, 200, 64), (2, 3, 129, 32), (1, 2, 300, 16),
                                   (1, 2, 260, 128), (2, 2, 1024, 64)])
@pytest.mark.parametrize("residual", [False, True])
def test_dropout_against_oracle(lib, shape, residual):
    B, H, T, D = shape
    p, offset = 0.2, 17
    q, k, v, do = bf16_inputs(B, H, T, D, seed=5150 + T + D, qk_std=1.0)
    scale = D ** -0.5
    o, lse, dq, dk, dv = run(lib, q, k, v, do, scale, p, SEED, offset, residual)
    qn, kn, vn, don = (as_f64(t) for t in (q, k, v, do))
    ro, rl = odrop.attention_forward_dropout(qn, kn, vn, scale, p, SEED, offset)
    rq, rk, rv = odrop.attention_backward_dropout(qn, kn, vn, don, scale, p, SEED, offset)
    check_bf16("o", as_f64(o), ro)
    check_lse(as_f64(lse), rl)
    for n, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        check_bf16(n, as_f64(got), ref)


def test_dropout_fp32_gradients(lib):
    B, H, T, D = 1, 2, 333, 64
    p, offset = 0.3, 4
    q, k, v, do = bf16_inputs(B, H, T, D, seed=31337, qk_std=1.0)
    scale = D ** -0.5
    _, _, dq, dk, dv = run(lib, q, k, v, do, scale, p, SEED, offset, residual=True, f32=True)
    qn, kn, vn, don = (as_f64(t) for t in (q, k, v, do))
    rq, rk, rv = odrop.attention_backward_dropout(qn, kn, vn, don, scale, p, SEED, offset)
    for n, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        err = np.abs(as_f64(got) - ref).max()
        assert err < 2e-3, (n, err)


def _identity(T, D, shift):
    x = torch.zeros(T, D)
    for d in range(D):
        if 0 <= d + shift < T:
            x[d + shift, d] = 1.0
    return x


@pytest.mark.parametrize("p", [0.25, 0.9])
@pytest.mark.parametrize("shift", [0, 128])
def test_mask_bits_match_oracle(lib, shift, p):
    B, H, T, D = 2, 3, 256, 128
    offset, seed = 0x9E3779B9, SEED
    q, k, _, _ = bf16_inputs(B, H, T, D, seed=2024, qk_std=0.3)
    eye = _identity(T, D, shift).to(torch.bfloat16)
    v = eye.expand(B, H, T, D).contiguous()
    do = eye.expand(B, H, T, D).contiguous()
    scale = D ** -0.5
    o, _, _, _, dv = run(lib, q, k, v, do, scale, p, seed, offset)
    o, dv = o.float().cpu().numpy(), dv.float().cpu().numpy()
    ii = np.arange(T)[:, None]
    for b in range(B):
        for h in range(H):
            keep = odrop.keep_mask_head(b, h, H, T, p, seed, offset)
            # forward: O[i, d] = P~[i, d + shift], visible where d + shift <= i
            vis = ii >= np.arange(D)[None, :] + shift
            got = o[b, h] != 0
            want = keep[:, shift:shift + D] & vis
            assert np.array_equal(got, want), (b, h, np.argwhere(got != want)[:5])
            # backward: dV[j, d] = P~[d + shift, j], visible where j <= d + shift
            visb = ii <= np.arange(D)[None, :] + shift
            gotb = dv[b, h] != 0
            wantb = keep[shift:shift + D, :].T & visb
            assert np.array_equal(gotb, wantb), (b, h, np.argwhere(gotb != wantb)[:5])
            # the drop rate of the visible entries is near p
            rate = 1.0 - want[vis].mean()
            assert abs(rate - p) < 0.05, rate


def test_p_zero_and_tiny_p_are_the_plain_calls(lib):
    B, H, T, D = 1, 2, 200, 64
    q, k, v, do = bf16_inputs(B, H, T, D, seed=77, qk_std=1.0)
    scale = D ** -0.5
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o0, l0, _ = lib.attn_fwd_strided(qd, kd, vd, scale)
    g0 = lib.attn_bwd_strided(qd, kd, vd, o0, l0, dod, scale)
    for p in (0.0, 1e-6):  # both give a zero threshold
        drop = lib.Dropout(p, 1, 2)
        o1, l1, _ = lib.attn_fwd_strided(qd, kd, vd, scale, dropout=drop)
        g1 = lib.attn_bwd_strided(qd, kd, vd, o1, l1, dod, scale, dropout=drop)
        torch.cuda.synchronize()
        assert torch.equal(o0, o1) and torch.equal(l0, l1)
        assert torch.equal(g0[1], g1[1]) and torch.equal(g0[2], g1[2])


def test_seed_and_offset_select_the_mask(lib):
    B, H, T, D = 1, 2, 256, 64
    q, k, v, do = bf16_inputs(B, H, T, D, seed=78, qk_std=1.0)
    scale = D ** -0.5
    a = run(lib, q, k, v, do, scale, 0.5, 1, 2)
    b = run(lib, q, k, v, do, scale, 0.5, 1, 2)
    c = run(lib, q, k, v, do, scale, 0.5, 1, 3)
    d = run(lib, q, k, v, do, scale, 0.5, 1 + (1 << 32), 2)
    assert torch.equal(a[0], b[0]) and torch.equal(a[3], b[3]) and torch.equal(a[4], b[4])
    assert not torch.equal(a[0], c[0]) and not torch.equal(a[0], d[0])


def test_invalid_probability_is_rejected(lib):
    dev = torch.device("cuda:0")
    q = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16, device=dev)
    for p in (1.0, -0.1, float("nan"), 2.0):
        with pytest.raises(lib.CattnError):
            lib.attn_fwd_strided(q, q, q, 0.125, dropout=lib.Dropout(p, 0, 0))


def test_autograd_qkv_with_dropout(lib):
    B, H, T, D = 2, 3, 190, 64
    p, seed, offset = 0.2, 99, 5
    q, k, v, do = bf16_inputs(B, H, T, D, seed=4321, qk_std=1.0)
    scale = D ** -0.5
    C = H * D
    merged = lambda x: x.transpose(1, 2).reshape(B, T, C)
    qkv = torch.cat([merged(q), merged(k), merged(v)], 2).cuda().requires_grad_(True)
    y = lib.CausalAttentionQKV.apply(qkv, H, scale, p, seed, offset)
    y.backward(merged(do).cuda())
    torch.cuda.synchronize()
    g = qkv.grad
    view = lambda x: x.reshape(B, T, H, D).transpose(1, 2)
    qn, kn, vn, don = (as_f64(t) for t in (q, k, v, do))
    ro, _ = odrop.attention_forward_dropout(qn, kn, vn, scale, p, seed, offset)
    rq, rk, rv = odrop.attention_backward_dropout(qn, kn, vn, don, scale, p, seed, offset)
    check_bf16("o", as_f64(view(y)), ro)
    check_bf16("dq", as_f64(view(g[..., :C])), rq)
    check_bf16("dk", as_f64(view(g[..., C:2 * C])), rk)
    check_bf16("dv", as_f64(view(g[..., 2 * C:])), rv)


def _il_pos(c):
    """Bit position of element c (0..31) of a keep word in the interleaved
    order: c = 16 h + 4 v + k sits at bit 8 k + 4 h + v."""
    return 8 * (c & 3) + 4 * ((c >> 4) & 1) + ((c >> 2) & 3)


def _unpack_mask(buf, B, H, T):
    """The keep-bit cache as a (B, H, T, T) bool array [query, key]: block
    bh * n_pairs + qt (qt + 1) / 2 + kt holds words [kr][w], bit il_pos(c) =
    query 128 qt + 32 w + c, key 128 kt + kr (tiles on or below the
    diagonal)."""
    n = (T + 127) // 128
    n_pairs = n * (n + 1) // 2
    words = buf.view(torch.int32).cpu().numpy().view(np.uint32).reshape(B * H, n_pairs, 128, 4)
    pos = np.array([_il_pos(c) for c in range(32)], dtype=np.uint32)
    bits = (words[..., None] >> pos) & 1  # [bh, blk, kr, w, c]
    full = np.zeros((B * H, n * 128, n * 128), dtype=bool)
    for qt in range(n):
        for kt in range(qt + 1):
            blk = bits[:, qt * (qt + 1) // 2 + kt].reshape(B * H, 128, 128)  # [kr, 32 w + c]
            full[:, qt * 128:(qt + 1) * 128, kt * 128:(kt + 1) * 128] = blk.transpose(0, 2, 1)
    return full[:, :T, :T].reshape(B, H, T, T)


@pytest.mark.parametrize("shape", [(1, 2, 300, 64), (2, 1, 260, 128), (1, 1, 129, 16)])
def test_cached_mask_bits_match_oracle(lib, shape):
    B, H, T, D = shape
    p, seed, offset = 0.3, SEED, 99
    q, k, v, _ = bf16_inputs(B, H, T, D, seed=4242 + T, qk_std=1.0)
    dev = torch.device("cuda:0")
    q, k, v = (t.to(dev) for t in (q, k, v))
    mask = lib.attn_dropout_mask(B, H, T, dev)
    assert mask.numel() == B * H * ((T + 127) // 128) * ((T + 127) // 128 + 1) // 2 * 2048
    lib.attn_fwd_strided(q, k, v, D ** -0.5, dropout=lib.dropout_params(p, seed, offset, mask))
    torch.cuda.synchronize()
    got = _unpack_mask(mask, B, H, T)
    causal = np.tril(np.ones((T, T), dtype=bool))
    for b in range(B):
        for h in range(H):
            want = odrop.keep_mask_head(b, h, H, T, p, seed, offset)
            assert np.array_equal(got[b, h] & causal, want & causal), (b, h)


@pytest.mark.parametrize("shape", [(2, 3, 129, 32), (1, 2, 260, 128), (2, 2, 1024, 64)])
@pytest.mark.parametrize("residual", [False, True])
def test_backward_with_cached_mask_is_bit_identical(lib, shape, residual):
    B, H, T, D = shape
    p, seed, offset = 0.2, SEED, 5
    q, k, v, do = bf16_inputs(B, H, T, D, seed=777 + T + D, qk_std=1.0)
    dev = torch.device("cuda:0")
    q, k, v, do = (t.to(dev) for t in (q, k, v, do))
    scale = D ** -0.5
    mask = lib.attn_dropout_mask(B, H, T, dev)
    drawn = lib.dropout_params(p, seed, offset)
    cached = lib.dropout_params(p, seed, offset, mask)
    res = []
    for drop in (drawn, cached):
        o = torch.empty_like(q)
        o_lo = torch.empty_like(q) if residual else None
        _, lse, _ = lib.attn_fwd_strided(q, k, v, scale, o=o, o_lo=o_lo, dropout=drop)
        res.append((o, lse) + lib.attn_bwd_strided(q, k, v, o, lse, do, scale, o_lo=o_lo,
                                                   dropout=drop))
    torch.cuda.synchronize()
    assert lib.cattn_get_device_status() == lib.OK
    for a, b in zip(*res):
        assert torch.equal(a, b)
