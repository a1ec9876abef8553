"""CPU tests of the fp64 oracle against facts it cannot set for itself.

Every pin in tests/pins.py must hold for the oracle; then each of a list
of plausible mistakes is planted in a copy of the oracle's source, and at
least one pin must catch it.
"""

import types

import numpy as np
import pytest

import oracle
import oracle.attention as oracle_mod
import pins
from workloads import WORKLOADS, as_f64, bf16_inputs, draw, seed_for

ORACLE = types.SimpleNamespace(fwd=oracle.attention_forward,
                               bwd=oracle.attention_backward)


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin_holds(pin):
    pin(ORACLE)


# (description, exact text in oracle/attention.py, replacement)
MUTANTS = [
    ("mask lets the next future key through", "k=1)", "k=2)"),
    ("mask hides the diagonal", "k=1)", "k=0)"),
    ("scale dropped from scores", "s = scale * (q2 @ k2.T)", "s = (q2 @ k2.T)"),
    ("max dropped from LSE", "lse = (m + np.log(l))[:, 0]", "lse = np.log(l)[:, 0]"),
    ("softmax stabiliser taken per column", "m = s.max(axis=1, keepdims=True)",
     "m = s.max(axis=0, keepdims=True)"),
    ("dV without the transpose", "dv[b, h] = p.T @ do[b, h]", "dv[b, h] = p @ do[b, h]"),
    ("Delta term dropped", "ds = p * (dp - dlt[:, None])", "ds = p * dp"),
    ("Delta summed over the wrong axis", "dlt = (p * dp).sum(axis=1)",
     "dlt = (p * dp).sum(axis=0)"),
    ("dK without the transpose", "dk[b, h] = scale * (ds.T @ q[b, h])",
     "dk[b, h] = scale * (ds @ q[b, h])"),
    ("scale dropped from dQ", "dq[b, h] = scale * (ds @ k[b, h])",
     "dq[b, h] = (ds @ k[b, h])"),
    ("dP with V untransposed", "dp = do[b, h] @ v[b, h].T",
     "dp = do[b, h] @ v[b, h][::-1].T"),
]


def _mutant(old, new):
    with open(oracle_mod.__file__) as f:
        src = f.read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return types.SimpleNamespace(fwd=mod.attention_forward,
                                 bwd=mod.attention_backward)


@pytest.mark.parametrize("desc,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(desc, old, new):
    impl = _mutant(old, new)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(impl)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches: {desc}"


def test_row_and_head_helpers_match_full():
    q, k, v, do = (as_f64(t) for t in bf16_inputs(2, 3, 40, 8, seed=11))
    scale = 0.35
    o, lse = oracle.attention_forward(q, k, v, scale)
    dq, dk, dv, delta = oracle.attention_backward(q, k, v, do, scale,
                                                  return_delta=True)
    rows = [0, 1, 17, 39]
    ro, rl = oracle.attention_rows(q, k, v, scale, 1, 2, rows)
    np.testing.assert_allclose(ro, o[1, 2, rows], rtol=0, atol=1e-13)
    np.testing.assert_allclose(rl, lse[1, 2, rows], rtol=0, atol=1e-13)
    heads = [0, 4, 5]
    ho, hl = oracle.attention_forward_heads(q, k, v, scale, heads)
    hq, hk, hv = oracle.attention_backward_heads(q, k, v, do, scale, heads)
    for n, f in enumerate(heads):
        b, h = divmod(f, 3)
        np.testing.assert_array_equal(ho[n], o[b, h])
        np.testing.assert_array_equal(hl[n], lse[b, h])
        np.testing.assert_allclose(hq[n], dq[b, h], rtol=0, atol=1e-14)
        np.testing.assert_allclose(hk[n], dk[b, h], rtol=0, atol=1e-14)
        np.testing.assert_allclose(hv[n], dv[b, h], rtol=0, atol=1e-14)
    # Delta from (O, dO) equals sum_j P_ij dP_ij
    np.testing.assert_allclose(oracle.delta_from_o(o, do), delta, rtol=0, atol=1e-12)


def _given_o_pins(given_o):
    """Facts outside attention_backward_given_o that pin it:
    (1) given the exact output it is the ordinary backward (the two forms of
    Delta agree, sum_j P_ij dP_ij = sum_d dO_id O_id);
    (2) its change under a perturbation e of the given output is the closed
    form of the chain rule: Delta moves by delta_i = sum_d dO_id e_id, so dS
    moves by -P_ij delta_i, dQ_i by -scale delta_i (P K)_i, dK_j by
    -scale sum_i P_ij delta_i Q_i, and dV not at all;
    (3) it is linear in the output (the perturbation doubled doubles the
    change)."""
    q, k, v, do = (as_f64(t) for t in bf16_inputs(1, 3, 37, 8, seed=21))
    scale = 0.41
    heads = [0, 2]
    o, _ = oracle.attention_forward_heads(q, k, v, scale, heads)
    exact = oracle.attention_backward_heads(q, k, v, do, scale, heads)
    given = given_o(q, k, v, do, o, scale, heads)
    for a, b_ in zip(given, exact):
        np.testing.assert_allclose(a, b_, rtol=0, atol=1e-13)
    rng = np.random.default_rng(5)
    e = rng.standard_normal(o.shape) * 1e-3
    moved = given_o(q, k, v, do, o + e, scale, heads)
    moved2 = given_o(q, k, v, do, o + 2 * e, scale, heads)
    for n, f in enumerate(heads):
        b, h = divmod(f, 3)
        p, _ = oracle.head_probs(q[b, h], k[b, h], scale)
        dlt = (do[b, h] * e[n]).sum(axis=1)
        want_dq = -scale * dlt[:, None] * (p @ k[b, h])
        want_dk = -scale * (p * dlt[:, None]).T @ q[b, h]
        np.testing.assert_allclose(moved[0][n] - exact[0][n], want_dq, rtol=0, atol=1e-12)
        np.testing.assert_allclose(moved[1][n] - exact[1][n], want_dk, rtol=0, atol=1e-12)
        np.testing.assert_array_equal(moved[2][n], exact[2][n])
        np.testing.assert_allclose(moved2[0][n] - exact[0][n], 2 * want_dq, rtol=0, atol=1e-12)


def test_backward_given_o_is_pinned():
    _given_o_pins(oracle.attention_backward_given_o)


GIVEN_O_MUTANTS = [
    ("exact Delta instead of the given output's",
     "dlt_o = (o_heads[n] * do[b, h]).sum(axis=1)", "dlt_o = (p * dp_n).sum(axis=1)"),
    ("given output of the wrong head", "(o_heads[n] * do[b, h])", "(o_heads[-1] * do[b, h])"),
    ("Delta subtracted column-wise", "ds_n = p * (dp_n - dlt_o[:, None])",
     "ds_n = p * (dp_n - dlt_o[None, :])"),
]


@pytest.mark.parametrize("desc,old,new", GIVEN_O_MUTANTS, ids=[m[0] for m in GIVEN_O_MUTANTS])
def test_given_o_planted_mistake_is_caught(desc, old, new):
    with open(oracle_mod.__file__) as f:
        src = f.read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("oracle_given_o_mutant")
    exec(compile(src.replace(old, new), "oracle_given_o_mutant", "exec"), mod.__dict__)
    with pytest.raises(AssertionError):
        _given_o_pins(mod.attention_backward_given_o)


def test_tiny_workload_fp32_and_bf16_inputs():
    """The tiny check runs on its raw fp32 draws as well as on the bf16
    rounding the GPU sees; the two results differ only by input rounding."""
    w = WORKLOADS[0]
    raw = [t.double().numpy() for t in draw(w.B, w.H, w.T, w.D, seed_for(0))]
    rnd = [as_f64(t) for t in bf16_inputs(w.B, w.H, w.T, w.D, seed_for(0))]
    o1, l1 = oracle.attention_forward(*raw[:3], w.scale)
    o2, l2 = oracle.attention_forward(*rnd[:3], w.scale)
    assert np.abs(o1 - o2).max() < 0.05
    assert np.abs(l1 - l2).max() < 0.05
    assert np.isfinite(o1).all() and np.isfinite(l1).all()
    pins.pin_single_token(ORACLE)


def test_long_context_logit_spread():
    """The long-context workload draws q and k with std 2, so that
    scale*q.k has std 4 (a peaked softmax).  Checked on a slice."""
    w = WORKLOADS[4]
    q, k, _, _ = draw(1, 1, 512, w.D, seed_for(4), w.qk_std)
    s = (q[0, 0] @ k[0, 0].T).double() * w.scale
    assert 3.6 < float(s.std()) < 4.4
