"""CPU checks of how the persistent kernels deal their work items
(cattn_plan_passes, host only): every item goes to exactly one CTA, and the
planned passes never leave a CTA more loaded than plain alternating passes
do.  The dealing rule is restated here from the header's description."""

from __future__ import annotations

import ctypes

import pytest

import causal_self_attention_flash_b200 as cattn


def plan(kind, BH, n_tiles, G):
    buf = (ctypes.c_uint16 * 64)()
    n = cattn.LIB.cattn_plan_passes(kind, BH, n_tiles, G, buf, 64)
    assert n >= 0
    return [buf[k] for k in range(n)]


def costs(kind, BH, n_tiles):
    if kind == 0:
        n_pairs = (n_tiles + 1) // 2
        out = []
        for u in range(BH * n_pairs):
            c = n_pairs - 1 - u // BH
            nlo = 2 * c + 1
            nhi = 2 * c + 2 if 2 * c + 1 < n_tiles else 0
            out.append(nlo + nhi)
        return out
    return [n_tiles - u // BH for u in range(BH * n_tiles)]


def deal(n_items, G, codes):
    """CTA of every item under the header's rule."""
    owner = [-1] * n_items
    passes = (n_items + G - 1) // G
    for k in range(passes):
        for b in range(G):
            if k < len(codes):
                r, d = codes[k] & 0x7FFF, codes[k] >> 15
                j = (r - b) % G if d else (b - r) % G
            else:
                j = G - 1 - b if k & 1 else b
            u = k * G + j
            if u < n_items:
                assert owner[u] == -1, (k, b, u)
                owner[u] = b
    return owner


SHAPES = [(192, 8, 148), (200, 8, 148), (384, 2, 148), (32, 64, 148), (96, 16, 148),
          (576, 8, 148), (2, 1, 2), (3, 5, 15), (7, 9, 148), (1, 1, 1), (5000, 8, 148)]


@pytest.mark.parametrize("kind", [0, 1])
@pytest.mark.parametrize("BH,n_tiles,sms", SHAPES)
def test_every_item_dealt_once_and_balance_not_worse(kind, BH, n_tiles, sms):
    cost = costs(kind, BH, n_tiles)
    G = min(len(cost), sms)
    codes = plan(kind, BH, n_tiles, G)
    owner = deal(len(cost), G, codes)
    assert all(o >= 0 for o in owner)
    load = [0] * G
    for u, b in enumerate(owner):
        load[b] += cost[u]
    snake = [0] * G
    for u, b in enumerate(deal(len(cost), G, [])):
        snake[b] += cost[u]
    assert max(load) <= max(snake)


def test_gpt2_layer_forward_balance():
    # the GPT-2 124M layer (16 x 12 heads, 8 tiles) on 148 SMs: alternating
    # passes leave the busiest CTA at 50 key tiles against a mean of 46.7;
    # the plan reaches the next integer above the mean
    kind, BH, n_tiles, G = 0, 192, 8, 148
    cost = costs(kind, BH, n_tiles)
    owner = deal(len(cost), G, plan(kind, BH, n_tiles, G))
    load = [0] * G
    for u, b in enumerate(owner):
        load[b] += cost[u]
    assert max(load) == 47


def test_backward_passes_alternate():
    assert plan(1, 192, 8, 148) == []


def test_bad_arguments():
    buf = (ctypes.c_uint16 * 4)()
    for args in ((2, 1, 1, 1), (0, 0, 1, 1), (1, 1, 0, 1), (0, 1, 1, 0)):
        assert cattn.LIB.cattn_plan_passes(*args, buf, 4) == -1
