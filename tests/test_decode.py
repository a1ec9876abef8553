"""GPU parity of decode attention (attn_decode) against the fp64 decode
oracle: the Tq newest query rows of a sequence against its first L cached
keys and values, with contiguous and (B, Tmax, H, D) cache layouts."""

import numpy as np
import pytest
import torch

import oracle.decode as odec
from parity_util import check_bf16, check_lse
from workloads import as_f64

pytestmark = pytest.mark.gpu


def draw(seed, *shape):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("B,H,L,Tq,D", [(1, 2, 1, 1, 16), (2, 3, 300, 1, 64), (2, 2, 257, 8, 128),
                                         (1, 4, 513, 2, 32), (2, 2, 64, 8, 16), (3, 2, 1000, 4, 64),
                                         (1, 2, 4096, 1, 128), (16, 12, 1024, 1, 64),
                                         (2, 2, 8, 8, 64), (1, 1, 257, 8, 32),
                                         # many heads: each warp walks several
                                         # chunks of its head
                                         (16, 12, 1024, 4, 64), (8, 25, 1024, 8, 64),
                                         (2, 16, 8192, 2, 128),
                                         # clusters of 8 (one head), 5 and 2 CTAs
                                         (1, 1, 8192, 8, 128), (1, 50, 1000, 3, 64),
                                         (1, 99, 300, 1, 32)])
@pytest.mark.parametrize("cache_layout", ["bhtd", "bthd"])
def test_decode_against_oracle(lib, B, H, L, Tq, D, cache_layout):
    dev = torch.device("cuda:0")
    Tmax = L + 37                       # cache capacity beyond the live length
    q = draw(11 + L, B, H, Tq, D)
    if cache_layout == "bhtd":
        k = draw(12 + L, B, H, Tmax, D)
        v = draw(13 + L, B, H, Tmax, D)
        kd, vd = k.to(dev), v.to(dev)
    else:                               # (B, Tmax, H, D) storage, (B, H, Tmax, D) views
        k = draw(12 + L, B, Tmax, H, D).transpose(1, 2)
        v = draw(13 + L, B, Tmax, H, D).transpose(1, 2)
        kd = k.transpose(1, 2).contiguous().to(dev).transpose(1, 2)
        vd = v.transpose(1, 2).contiguous().to(dev).transpose(1, 2)
        assert kd.stride(2) == H * D
    # poison the rows past L: they must not be read into the result
    kd[:, :, L:] = float("nan")
    vd[:, :, L:] = float("nan")
    scale = D ** -0.5
    o, lse = lib.attn_decode(q.to(dev), kd, vd, L, scale)
    torch.cuda.synchronize()
    ro, rl = odec.decode_attention(as_f64(q), as_f64(k), as_f64(v), scale, L)
    check_bf16("o", as_f64(o), ro)
    check_lse(as_f64(lse), rl)


def test_decode_matches_forward_rows(lib):
    """the decode of the last rows agrees with the full forward's last rows"""
    B, H, T, D, Tq = 2, 3, 700, 64, 5
    dev = torch.device("cuda:0")
    q, k, v = (draw(s, B, H, T, D).to(dev) for s in (21, 22, 23))
    o_full, lse_full = lib.attn_fwd(q, k, v)
    o, lse = lib.attn_decode(q[:, :, T - Tq:].contiguous(), k, v, T)
    torch.cuda.synchronize()
    assert torch.allclose(lse, lse_full[:, :, T - Tq:], atol=1e-4, rtol=0)
    diff = (o.float() - o_full[:, :, T - Tq:].float()).abs().max().item()
    assert diff < 2e-2, diff


def test_decode_argument_errors(lib):
    dev = torch.device("cuda:0")
    q = torch.zeros(1, 1, 9, 64, dtype=torch.bfloat16, device=dev)
    k = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16, device=dev)
    with pytest.raises(lib.CattnError):        # Tq above 8
        lib.attn_decode(q, k, k, 16)
    with pytest.raises(lib.CattnError):        # L < Tq
        lib.attn_decode(q[:, :, :4], k, k, 3)
    # no workspace is needed: an empty one is accepted
    ws = torch.empty(0, dtype=torch.uint8, device=dev)
    lib.attn_decode(q[:, :, :1], k, k, 16, workspace=ws)
    torch.cuda.synchronize()


def test_decode_strided_query_and_output(lib):
    """q and o as (B, Tq, H, D) storage seen as (B, H, Tq, D) views (the
    layout of a fused projection's rows), the cache (B, Tmax, H, D): every
    stride of the call differs from the contiguous one."""
    B, H, Tq, L, D = 3, 5, 6, 700, 64
    dev = torch.device("cuda:0")
    Tmax = L + 5
    qs = draw(31, B, Tq, H, D)
    ks = draw(32, B, Tmax, H, D)
    vs = draw(33, B, Tmax, H, D)
    q = qs.to(dev).transpose(1, 2)
    k = ks.to(dev).transpose(1, 2)
    v = vs.to(dev).transpose(1, 2)
    o_store = torch.full((B, Tq, H, D), float("nan"), dtype=torch.bfloat16, device=dev)
    o = o_store.transpose(1, 2)
    scale = D ** -0.5
    o2, lse = lib.attn_decode(q, k, v, L, scale, o=o)
    torch.cuda.synchronize()
    assert o2.data_ptr() == o.data_ptr()
    ro, rl = odec.decode_attention(as_f64(qs.transpose(1, 2)), as_f64(ks.transpose(1, 2)),
                                   as_f64(vs.transpose(1, 2)), scale, L)
    check_bf16("o", as_f64(o), ro)
    check_lse(as_f64(lse), rl)
