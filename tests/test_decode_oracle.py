"""CPU pins of the decode oracle (oracle/decode.py).

Decode attention is causal attention restricted to the newest Tq rows, so
it is pinned to facts that do not come from its own code: the last rows of
the (separately pinned) full-sequence oracle, the pure-Python brute force,
the closed form of a one-token cache, and invariance to cache rows past L.
A planted mistake in a copy of the module must fail some pin.
"""

from __future__ import annotations

import math
import types

import numpy as np
import pytest

import oracle
import oracle.decode as dec_mod
from oracle import brute


def _rand(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


def pin_last_rows_of_full_attention(dec):
    B, H, L, D, Tq = 2, 3, 37, 8, 5
    q, k, v = (_rand(s, B, H, L, D) for s in (1, 2, 3))
    o_full, lse_full = oracle.attention_forward(q, k, v, 0.4)
    o, lse = dec(q[:, :, L - Tq:], k, v, 0.4, L)
    assert np.allclose(o, o_full[:, :, L - Tq:], rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, lse_full[:, :, L - Tq:], rtol=1e-12, atol=1e-12)


def pin_brute_force(dec):
    L, D, Tq = 6, 3, 2
    q, k, v = (_rand(s, 1, 1, L, D) for s in (4, 5, 6))
    bo, bl = brute.forward_head(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist(), 0.7)
    o, lse = dec(q[:, :, L - Tq:], k, v, 0.7, L)
    assert np.allclose(o[0, 0], np.array(bo)[L - Tq:], rtol=1e-12, atol=1e-12)
    assert np.allclose(lse[0, 0], np.array(bl)[L - Tq:], rtol=1e-12, atol=1e-12)


def pin_single_key(dec):
    q, k, v = (_rand(s, 1, 2, 1, 4) for s in (7, 8, 9))
    o, lse = dec(q, k, v, 0.5, 1)
    assert np.allclose(o, v, rtol=0, atol=0)
    assert np.allclose(lse[..., 0], 0.5 * (q * k).sum(-1)[..., 0], rtol=1e-14)


def pin_ignores_rows_past_L(dec):
    B, H, Tmax, D, L, Tq = 1, 2, 20, 4, 11, 3
    q = _rand(10, B, H, Tq, D)
    k, v = _rand(11, B, H, Tmax, D), _rand(12, B, H, Tmax, D)
    o1, l1 = dec(q, k, v, 1.0, L)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, L:] += 100.0
    v2[:, :, L:] -= 50.0
    o2, l2 = dec(q, k2, v2, 1.0, L)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def pin_row_sees_its_own_key(dec):
    """a large score on the newest key of row r dominates row r only"""
    L, D, Tq = 9, 2, 3
    q = np.zeros((1, 1, Tq, D))
    q[0, 0, :, 0] = 1.0
    k = np.zeros((1, 1, L, D))
    v = np.arange(L * D, dtype=float).reshape(1, 1, L, D)
    k[0, 0, L - 2, 0] = 60.0     # key at position L-2: visible to rows 1, 2 only
    o, _ = dec(q, k, v, 1.0, L)
    assert np.allclose(o[0, 0, 1], v[0, 0, L - 2]) and np.allclose(o[0, 0, 2], v[0, 0, L - 2])
    assert np.allclose(o[0, 0, 0], v[0, 0, :L - 2].mean(0))


ALL_PINS = [pin_last_rows_of_full_attention, pin_brute_force, pin_single_key,
            pin_ignores_rows_past_L, pin_row_sees_its_own_key]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_pin_holds(pin):
    pin(dec_mod.decode_attention)


MUTANTS = [
    ("query position off by one", "pos = L - Tq + r", "pos = L - Tq + r - 1"),
    ("sees one key too many", "k[b, h, :pos + 1] @ q[b, h, r]", "k[b, h, :pos + 2] @ q[b, h, r]"),
    ("scale dropped", "s = scale * (k[b, h, :pos + 1] @ q[b, h, r])",
     "s = (k[b, h, :pos + 1] @ q[b, h, r])"),
    ("max dropped from LSE", "lse[b, h, r] = m + np.log(e.sum())", "lse[b, h, r] = np.log(e.sum())"),
    ("values of the wrong rows", "@ v[b, h, :pos + 1]", "@ v[b, h, 1:pos + 2]"),
]


@pytest.mark.parametrize("desc,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(desc, old, new):
    with open(dec_mod.__file__) as f:
        src = f.read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("decode_mutant")
    exec(compile(src.replace(old, new), "decode_mutant", "exec"), mod.__dict__)
    for pin in ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(mod.decode_attention)
        except (AssertionError, ValueError, IndexError):
            return
    pytest.fail(f"no pin catches: {desc}")
