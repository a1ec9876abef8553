"""CPU pins of the dropout oracle (oracle/dropout.py).

* The generator: Philox4x32-10 must reproduce the published known-answer
  vectors (tests/golden/philox4x32_10_kat.txt).
* The mask: drop rate and pair statistics at the requested probability,
  determinism, dependence on seed and offset, and the documented placement
  of each element's 8 bits in the Philox blocks.
* The arithmetic: p = 0 reduces exactly to the dropout-free oracle; the
  dropout output is unbiased (its mean over many masks is the dropout-free
  output) and the keep scale is exactly 1 / the keep probability of the
  8-bit draw; central finite differences of
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
        philox=mod.philox4x32_10, mask=mod.keep_mask_head, r8=mod.random8,
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
    for p in (0.1, 0.2, 0.5):  # 0.1 is 25.6 / 256: rounded, not truncated
        m = impl.mask(1, 2, 3, T, p, 0x1234_5678_9ABC_DEF0, 7)
        n = T * T
        t = round(p * 256) / 256
        drop = 1.0 - m.mean()
        sigma = np.sqrt(t * (1 - t) / n)
        assert abs(drop - t) < 5 * sigma, (p, drop)
        # neighbours (same query, keys j and j+1; same key, queries i and i+1)
        for both in ((~m[:, :-1] & ~m[:, 1:]).mean(), (~m[:-1, :] & ~m[1:, :]).mean()):
            assert abs(both - t * t) < 5 * np.sqrt(t * t * (1 - t * t) / n), (p, both)


def pin_uniform_bits(impl):
    """the 8-bit values are uniform: chi-square over their 256 values, for
    all keys and for each of the four byte positions j & 3 alone."""
    T = 512
    r = impl.r8(0, 0, 1, np.arange(T)[:, None], np.arange(T)[None, :], 99, 3)
    for sel in (r.ravel(), r[:, 0::4].ravel(), r[:, 1::4].ravel(), r[:, 2::4].ravel(),
                r[:, 3::4].ravel()):
        counts = np.bincount(sel.astype(np.int64), minlength=256)
        e = sel.size / 256
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
    """element (b, h, i, j): word (j & 15) >> 2, byte j & 3 of the block
    with counter (j >> 4, i, b*H + h, offset) and key (seed low, seed high)."""
    seed, offset, H = 0xDEADBEEF_01234567, 11, 5
    for b, h, i, j in ((0, 0, 0, 0), (1, 2, 5, 13), (3, 4, 1000, 999), (0, 3, 77, 64)):
        blk = impl.philox(np.array([j >> 4, i, b * H + h, offset]),
                          (seed & 0xFFFFFFFF, seed >> 32))
        want = (int(blk[(j & 15) >> 2]) >> (8 * (j & 3))) & 0xFF
        assert int(impl.r8(b, h, H, i, j, seed, offset)) == want
        # dropped iff the 8 bits are below round(p * 256)
        for pr in (0.1, 0.5, 0.9):
            m = impl.mask(b, h, H, max(i, j) + 1, pr, seed, offset)
            assert bool(m[i, j]) == (want >= round(pr * 256)), (b, h, i, j, pr)


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


def pin_exact_keep_scale(impl):
    """the keep scale times the exact keep probability is 1: the byte is
    uniform over 256 values, so with the threshold t read off the mask
    (the smallest kept byte, the largest dropped one plus 1) the keep
    probability is (256 - t) / 256."""
    T = 256
    r = impl.r8(0, 1, 2, np.arange(T)[:, None], np.arange(T)[None, :], 5, 6)
    for p in (0.1, 0.3, 0.77):
        m = impl.mask(0, 1, 2, T, p, 5, 6)
        t = int(r[m].min())
        assert t == int(r[~m].max()) + 1, p
        assert abs(impl.ks(p) * (256 - t) / 256 - 1.0) < 1e-12, (p, t, impl.ks(p))


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
            pin_bit_placement, pin_p_zero, pin_unbiased, pin_exact_keep_scale,
            pin_finite_differences, pin_lse_unchanged]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_pin_holds(pin):
    pin(_impl())


def test_threshold_and_scale():
    assert drop_mod.drop_threshold(0.2) == 51
    assert drop_mod.drop_threshold(0.1) == 26
    assert drop_mod.drop_threshold(0.0) == 0
    assert drop_mod.drop_threshold(0.001) == 0
    assert drop_mod.drop_threshold(0.99999999) == 255
    assert drop_mod.keep_scale(0.2) == 256.0 / 205.0
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
    ("word chosen by j & 3", "((j & np.uint64(15)) >> np.uint64(2))", "(j & np.uint64(3))"),
    ("bytes taken high first", "(np.uint64(8) * (j & np.uint64(3)))",
     "(np.uint64(8) * (np.uint64(3) - (j & np.uint64(3))))"),
    ("16 keys per block, counter j >> 3", "ctr = np.stack([j >> np.uint64(4), i,",
     "ctr = np.stack([j >> np.uint64(3), i,"),
    ("counter words i and j swapped", "ctr = np.stack([j >> np.uint64(4), i,",
     "ctr = np.stack([i >> np.uint64(4), j,"),
    ("seven bits drawn", "& np.uint64(0xFF)", "& np.uint64(0x7F)"),
    ("keep where below the threshold", "return r >= np.uint64(drop_threshold(p))",
     "return r < np.uint64(256 - drop_threshold(p))"),
    ("threshold truncated", "min(int(np.rint(p * 256.0)), 255)", "min(int(p * 256.0), 255)"),
    ("keep scale 1/p", "return 256.0 / (256.0 - t)", "return 256.0 / max(t, 1)"),
    ("keep scale from the unrounded p", "return 256.0 / (256.0 - t)", "return 1.0 / (1.0 - p)"),
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
