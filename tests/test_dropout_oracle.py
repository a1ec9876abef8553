"""CPU pins of the dropout oracle (oracle/dropout.py).

* The generator: Philox4x32-10 must reproduce the published known-answer
  vectors (tests/golden/philox4x32_10_kat.txt).
* The mask: drop rate and pair statistics at the requested probability,
  determinism, dependence on seed and offset, and the documented placement
  of each element's 16 bits in the Philox blocks.
* The arithmetic: p = 0 reduces exactly to the dropout-free oracle; the
  dropout output is unbiased (its mean over many masks is the dropout-free
  output, which pins the keep scale); central finite differences of
  L = <O, dO> with the mask held fixed match the backward.
* Planted mistakes in a copy of the module are each caught by some pin.
"""

from __future__ import annotations

import os
import types

import numpy as np
import pytest

import oracle
import oracle.dropout as drop_mod

KAT = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def _rand(seed, B, H, T, D, std=1.0):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((B, H, T, D)) * std for _ in range(4)]


def _impl(mod=drop_mod):
    return types.SimpleNamespace(
        philox=mod.philox4x32_10, mask=mod.keep_mask_head, r16=mod.random16,
        fwd=mod.attention_forward_dropout, bwd=mod.attention_backward_dropout,
        ks=mod.keep_scale)


# ---------------------------------------------------------------- pins

def pin_kat(impl):
    with open(KAT) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        w = [int(x, 16) for x in r]
        got = impl.philox(np.array(w[:4]), (w[4], w[5]))
        assert [int(x) for x in got] == w[6:], (r, [hex(int(x)) for x in got])


def pin_drop_rate(impl):
    T = 1024
    for p in (0.2, 0.5):
        m = impl.mask(1, 2, 3, T, p, 0x1234_5678_9ABC_DEF0, 7)
        n = T * T
        t = round(p * 65536) / 65536
        drop = 1.0 - m.mean()
        sigma = np.sqrt(t * (1 - t) / n)
        assert abs(drop - t) < 5 * sigma, (p, drop)
        # neighbours (same query, keys j and j+1; same key, queries i and i+1)
        for both in ((~m[:, :-1] & ~m[:, 1:]).mean(), (~m[:-1, :] & ~m[1:, :]).mean()):
            assert abs(both - t * t) < 5 * np.sqrt(t * t * (1 - t * t) / n), (p, both)


def pin_uniform_bits(impl):
    """the 16-bit values are uniform: chi-square over the 256 values of
    the high byte and of the low byte."""
    T = 512
    r = impl.r16(0, 0, 1, np.arange(T)[:, None], np.arange(T)[None, :], 99, 3).ravel()
    for byte in (r >> np.uint64(8), r & np.uint64(255)):
        counts = np.bincount(byte.astype(np.int64), minlength=256)
        e = r.size / 256
        chi2 = ((counts - e) ** 2 / e).sum()
        assert 160 < chi2 < 370, chi2     # 255 degrees of freedom, beyond 4.5 sigma


def pin_stream_separation(impl):
    T = 64
    base = impl.mask(0, 1, 2, T, 0.5, 5, 9)
    assert np.array_equal(base, impl.mask(0, 1, 2, T, 0.5, 5, 9))
    for other in (impl.mask(0, 1, 2, T, 0.5, 6, 9), impl.mask(0, 1, 2, T, 0.5, 5, 10),
                  impl.mask(1, 1, 2, T, 0.5, 5, 9), impl.mask(0, 0, 2, T, 0.5, 5, 9),
                  impl.mask(0, 1, 2, T, 0.5, 5 + (1 << 32), 9)):
        agree = (other == base).mean()
        assert 0.4 < agree < 0.6, agree


def pin_bit_placement(impl):
    """element (b, h, i, j): word (j & 7) >> 1, half j & 1 of the block with
    counter (j >> 3, i, b*H + h, offset) and key (seed low, seed high)."""
    seed, offset, H = 0xDEADBEEF_01234567, 11, 5
    for b, h, i, j in ((0, 0, 0, 0), (1, 2, 5, 13), (3, 4, 1000, 999), (0, 3, 77, 64)):
        blk = impl.philox(np.array([j >> 3, i, b * H + h, offset]),
                          (seed & 0xFFFFFFFF, seed >> 32))
        want = (int(blk[(j & 7) >> 1]) >> (16 * (j & 1))) & 0xFFFF
        assert int(impl.r16(b, h, H, i, j, seed, offset)) == want
        # dropped iff the 16 bits are below round(p * 65536)
        for pr in (0.1, 0.5, 0.9):
            m = impl.mask(b, h, H, max(i, j) + 1, pr, seed, offset)
            assert bool(m[i, j]) == (want >= round(pr * 65536)), (b, h, i, j, pr)


def pin_p_zero(impl):
    q, k, v, do = _rand(1, 2, 2, 9, 4)
    o0, l0 = oracle.attention_forward(q, k, v, 0.5)
    o1, l1 = impl.fwd(q, k, v, 0.5, 0.0, 3, 4)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)
    g0 = oracle.attention_backward(q, k, v, do, 0.5)
    g1 = impl.bwd(q, k, v, do, 0.5, 0.0, 3, 4)
    for a, b in zip(g0, g1):
        assert np.allclose(a, b, rtol=1e-13, atol=1e-13)


def pin_unbiased(impl):
    """E over masks of the dropout output is the dropout-free output."""
    q, k, v, _ = _rand(2, 1, 1, 12, 3)
    ref, _ = oracle.attention_forward(q, k, v, 0.7)
    n = 400
    outs = np.stack([impl.fwd(q, k, v, 0.7, 0.3, 77, off)[0] for off in range(n)])
    mean, sd = outs.mean(0), outs.std(0)
    z = np.abs(mean - ref) / (sd / np.sqrt(n) + 1e-12)
    assert z.max() < 6.0, z.max()


def pin_finite_differences(impl):
    q, k, v, do = _rand(3, 1, 2, 6, 3)
    scale, p, seed, off = 0.8, 0.35, 123, 5
    dq, dk, dv = impl.bwd(q, k, v, do, scale, p, seed, off)

    def loss(q_, k_, v_):
        return float((impl.fwd(q_, k_, v_, scale, p, seed, off)[0] * do).sum())

    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [xp if n == name else a for n, a in (("q", q), ("k", k), ("v", v))]
            args_m = [xm if n == name else a for n, a in (("q", q), ("k", k), ("v", v))]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        assert np.allclose(num, g, rtol=1e-6, atol=1e-8), (name, np.abs(num - g).max())


def pin_lse_unchanged(impl):
    q, k, v, _ = _rand(4, 1, 1, 7, 2)
    _, l0 = oracle.attention_forward(q, k, v, 1.0)
    _, l1 = impl.fwd(q, k, v, 1.0, 0.5, 1, 2)
    assert np.array_equal(l0, l1)


ALL_PINS = [pin_kat, pin_drop_rate, pin_uniform_bits, pin_stream_separation,
            pin_bit_placement, pin_p_zero, pin_unbiased, pin_finite_differences,
            pin_lse_unchanged]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_pin_holds(pin):
    pin(_impl())


def test_threshold_and_scale():
    assert drop_mod.drop_threshold(0.2) == 13107
    assert drop_mod.drop_threshold(0.0) == 0
    assert drop_mod.drop_threshold(0.99999999) == 65535
    assert drop_mod.keep_scale(0.5) == 2.0
    with pytest.raises(ValueError):
        drop_mod.drop_threshold(1.0)
    with pytest.raises(ValueError):
        drop_mod.drop_threshold(-0.1)


# (description, exact text in oracle/dropout.py, replacement)
MUTANTS = [
    ("wrong round multiplier", "PHILOX_M1 = 0xCD9E8D57", "PHILOX_M1 = 0xCD9E8D59"),
    ("key not bumped", "k1 = (k1 + PHILOX_W1) & MASK32", "k1 = k1"),
    ("nine rounds", "for rnd in range(10):", "for rnd in range(9):"),
    ("output words swapped", "hi0 ^ c3 ^ np.uint64(k1), lo0)", "lo0, hi0 ^ c3 ^ np.uint64(k1))"),
    ("word chosen by j & 3", "((j & np.uint64(7)) >> np.uint64(1))", "(j & np.uint64(3))"),
    ("high half for even keys", "(np.uint64(16) * (j & np.uint64(1)))",
     "(np.uint64(16) * (np.uint64(1) - (j & np.uint64(1))))"),
    ("counter words i and j swapped", "ctr = np.stack([j >> np.uint64(3), i,",
     "ctr = np.stack([i >> np.uint64(3), j,"),
    ("keep where below the threshold", "return r >= np.uint64(drop_threshold(p))",
     "return r < np.uint64(65536 - drop_threshold(p))"),
    ("keep scale 1/p", "return 65536.0 / (65536.0 - t)", "return 65536.0 / max(t, 1)"),
    ("no rescale in the forward", "o[b, h] = (pr * m * ks) @ v[b, h]", "o[b, h] = (pr * m) @ v[b, h]"),
    ("dP without the mask", "dp = dpd * m * ks", "dp = dpd * ks"),
    ("dP without the keep scale", "dp = dpd * m * ks", "dp = dpd * m"),
    ("dV from the undropped P", "dv[b, h] = pd.T @ do[b, h]", "dv[b, h] = pr.T @ do[b, h]"),
    ("mask transposed in the backward", "pd = pr * m * ks", "pd = pr * m.T * ks"),
    ("Delta from the dropped P", "dlt = (pr * dp).sum(axis=1)", "dlt = (pd * dp).sum(axis=1)"),
]


def _mutant(old, new):
    with open(drop_mod.__file__) as f:
        src = f.read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("oracle.dropout_mutant")
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new), "dropout_mutant", "exec"), mod.__dict__)
    return _impl(mod)


@pytest.mark.parametrize("desc,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(desc, old, new):
    impl = _mutant(old, new)
    for pin in ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(impl)
        except (AssertionError, ValueError, FloatingPointError, IndexError):
            return
    pytest.fail(f"no pin catches: {desc}")
