"""Pins for the fp64 oracle: facts fixed by the definition of causal
attention or by mathematics, not by the oracle itself.

Each pin takes an implementation ``impl`` with ``impl.fwd(q, k, v, scale)
-> (o, lse)`` and ``impl.bwd(q, k, v, do, scale) -> (dq, dk, dv)`` (numpy
float64, shape (B, H, T, D)) and raises AssertionError when the fact does
not hold.  tests/test_oracle.py runs every pin on the real oracle (all must
hold) and on planted mistakes (some pin must fail for each).

Definition followed ("nanoGPT: a real GPT in two 300-line files",
section 2 "How the code works", CausalSelfAttention; "Words to know":
Causal): softmax(scale * q k^T with future keys at minus infinity) @ v.
"""

from __future__ import annotations

import json
import math
import os

import numpy as np

from oracle import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden",
                      "two_token_worked_example.json")


def _rng(seed):
    return np.random.default_rng(seed)


def _rand(rng, B, H, T, D, std=1.0):
    return [rng.standard_normal((B, H, T, D)) * s for s in (std, std, 1.0, 1.0)]


def pin_golden(impl):
    """Hand-derived two-token example (tests/golden)."""
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        arr = {n: np.array(c[n], dtype=np.float64).reshape(1, 1, 2, 1)
               for n in ("q", "k", "v", "do", "o", "dq", "dk", "dv")}
        o, lse = impl.fwd(arr["q"], arr["k"], arr["v"], c["scale"])
        np.testing.assert_allclose(o, arr["o"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse.reshape(2), c["lse"], rtol=0, atol=1e-12)
        dq, dk, dv = impl.bwd(arr["q"], arr["k"], arr["v"], arr["do"], c["scale"])
        np.testing.assert_allclose(dq, arr["dq"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dk, arr["dk"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dv, arr["dv"], rtol=0, atol=1e-12)


def pin_single_token(impl):
    """T = 1: the only key is the query's own; O = V, LSE = scale q.k,
    dQ = dK = 0, dV = dO."""
    rng = _rng(1)
    B, H, D = 2, 3, 5
    q, k, v, do = _rand(rng, B, H, 1, D)
    scale = 0.37
    o, lse = impl.fwd(q, k, v, scale)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, scale * (q * k).sum(-1), rtol=0, atol=1e-14)
    dq, dk, dv = impl.bwd(q, k, v, do, scale)
    np.testing.assert_allclose(dq, 0, atol=1e-14)
    np.testing.assert_allclose(dk, 0, atol=1e-14)
    np.testing.assert_allclose(dv, do, rtol=0, atol=1e-14)


def pin_constant_keys(impl):
    """All key rows equal: every visible key has the same score, so
    P_ij = 1/(i+1): O_i = mean(V_0..V_i), LSE_i = scale q_i.k + ln(i+1),
    dV_j = sum_{i>=j} dO_i/(i+1), dQ = 0."""
    rng = _rng(2)
    B, H, T, D = 1, 2, 9, 3
    q, _, v, do = _rand(rng, B, H, T, D)
    krow = rng.standard_normal((B, H, 1, D))
    k = np.repeat(krow, T, axis=2)
    scale = 0.8
    o, lse = impl.fwd(q, k, v, scale)
    counts = np.arange(1, T + 1, dtype=np.float64)
    prefix_mean = np.cumsum(v, axis=2) / counts[:, None]
    np.testing.assert_allclose(o, prefix_mean, rtol=0, atol=1e-12)
    want_lse = scale * (q * krow).sum(-1) + np.log(counts)
    np.testing.assert_allclose(lse, want_lse, rtol=0, atol=1e-12)
    dq, dk, dv = impl.bwd(q, k, v, do, scale)
    np.testing.assert_allclose(dq, 0, atol=1e-12)
    w = do / counts[:, None]                       # dO_i / (i+1)
    want_dv = np.flip(np.cumsum(np.flip(w, axis=2), axis=2), axis=2)
    np.testing.assert_allclose(dv, want_dv, rtol=0, atol=1e-12)


def pin_first_row_and_weights(impl):
    """Row 0 sees only key 0, so O_0 = V_0 and LSE_0 = scale q_0.k_0.
    With V = identity columns (D = T), O row i is exactly P row i: it must
    be a probability vector with no weight on future keys."""
    rng = _rng(3)
    B, H, T = 1, 2, 7
    D = T
    q = rng.standard_normal((B, H, T, D))
    k = rng.standard_normal((B, H, T, D))
    v = np.broadcast_to(np.eye(T), (B, H, T, T)).copy()
    scale = 0.6
    o, lse = impl.fwd(q, k, v, scale)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], atol=1e-14)
    np.testing.assert_allclose(lse[:, :, 0], scale * (q[:, :, 0] * k[:, :, 0]).sum(-1),
                               atol=1e-14)
    np.testing.assert_allclose(o.sum(-1), 1.0, atol=1e-13)        # row sums
    assert (o >= 0).all()
    future = np.triu(np.ones((T, T), dtype=bool), k=1)
    assert np.all(o[:, :, future] == 0.0)                         # causal
    # and P_ij = exp(scale q_i.k_j - LSE_i) on the visible part
    s = scale * np.einsum("bhid,bhjd->bhij", q, k)
    p = np.exp(s - lse[..., None])
    np.testing.assert_allclose(o[:, :, ~future], p[:, :, ~future], rtol=1e-12)


def pin_causality(impl):
    """Perturbing q/k/v at positions > i leaves O and LSE rows <= i
    bit-unchanged; perturbing dO at positions < j leaves dK_j, dV_j
    unchanged; dQ_i depends on dO_i only among the dO rows."""
    rng = _rng(4)
    B, H, T, D = 1, 2, 12, 4
    q, k, v, do = _rand(rng, B, H, T, D)
    scale = 0.5
    o, lse = impl.fwd(q, k, v, scale)
    dq, dk, dv = impl.bwd(q, k, v, do, scale)
    for i in (0, 3, 7, T - 2):
        q2, k2, v2 = q.copy(), k.copy(), v.copy()
        for t in (q2, k2, v2):
            t[:, :, i + 1:] += rng.standard_normal(t[:, :, i + 1:].shape) * 3
        o2, lse2 = impl.fwd(q2, k2, v2, scale)
        assert np.array_equal(o2[:, :, :i + 1], o[:, :, :i + 1])
        assert np.array_equal(lse2[:, :, :i + 1], lse[:, :, :i + 1])
        assert not np.allclose(o2[:, :, i + 1:], o[:, :, i + 1:])
    for j in (1, 5, T - 1):
        do2 = do.copy()
        do2[:, :, :j] += rng.standard_normal(do2[:, :, :j].shape)
        dq2, dk2, dv2 = impl.bwd(q, k, v, do2, scale)
        np.testing.assert_allclose(dk2[:, :, j:], dk[:, :, j:], rtol=0, atol=1e-13)
        np.testing.assert_allclose(dv2[:, :, j:], dv[:, :, j:], rtol=0, atol=1e-13)
        np.testing.assert_allclose(dq2[:, :, j:], dq[:, :, j:], rtol=0, atol=1e-13)
        if j >= 2:                                  # dQ_0 is always 0
            assert not np.allclose(dq2[:, :, 1:j], dq[:, :, 1:j])


def pin_key_shift(impl):
    """Adding one vector c to every key multiplies row i's weights by the
    common factor exp(scale q_i.c): P and O are unchanged, LSE_i moves by
    scale q_i.c, and dQ, dK, dV are unchanged (rows of dS sum to 0)."""
    rng = _rng(5)
    B, H, T, D = 2, 1, 10, 3
    q, k, v, do = _rand(rng, B, H, T, D)
    c = rng.standard_normal((B, H, 1, D))
    scale = 0.7
    o, lse = impl.fwd(q, k, v, scale)
    o2, lse2 = impl.fwd(q, k + c, v, scale)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2 - lse, scale * (q * c).sum(-1), rtol=0, atol=1e-12)
    g = impl.bwd(q, k, v, do, scale)
    g2 = impl.bwd(q, k + c, v, do, scale)
    for a, b in zip(g, g2):
        np.testing.assert_allclose(b, a, rtol=0, atol=1e-11)


def pin_finite_differences(impl):
    """Central differences of L = sum(O * dO) match dQ, dK, dV."""
    rng = _rng(6)
    B, H, T, D = 1, 1, 5, 3
    q, k, v, do = _rand(rng, B, H, T, D)
    scale = 0.9
    dq, dk, dv = impl.bwd(q, k, v, do, scale)

    def loss(q_, k_, v_):
        return float((impl.fwd(q_, k_, v_, scale)[0] * do).sum())

    h = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        num = np.zeros_like(grad)
        for idx in np.ndindex(grad.shape):
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.abs(num - grad).max() / max(np.abs(grad).max(), 1e-30)
        assert err <= 1e-6, (which, err)


def pin_brute_force(impl):
    """The pure-Python loop version (oracle/brute.py) agrees to 1e-12."""
    rng = _rng(7)
    for (T, D) in ((1, 1), (2, 3), (5, 2), (8, 4)):
        B, H = 1, 2
        q, k, v, do = _rand(rng, B, H, T, D)
        scale = 1.0 / math.sqrt(D)
        o, lse = impl.fwd(q, k, v, scale)
        dq, dk, dv = impl.bwd(q, k, v, do, scale)
        for b in range(B):
            for h in range(H):
                args = [x[b, h].tolist() for x in (q, k, v)]
                bo, bl = brute.forward_head(*args, scale)
                np.testing.assert_allclose(o[b, h], bo, rtol=0, atol=1e-12)
                np.testing.assert_allclose(lse[b, h], bl, rtol=0, atol=1e-12)
                bq, bk, bv = brute.backward_head(*args, do[b, h].tolist(), scale)
                np.testing.assert_allclose(dq[b, h], bq, rtol=0, atol=1e-12)
                np.testing.assert_allclose(dk[b, h], bk, rtol=0, atol=1e-12)
                np.testing.assert_allclose(dv[b, h], bv, rtol=0, atol=1e-12)


def pin_torch_autograd(impl):
    """Library special case: torch CPU float64 softmax of the masked
    matmul, differentiated by autograd, agrees to 1e-10."""
    import torch
    rng = _rng(8)
    B, H, T, D = 2, 2, 33, 8
    q, k, v, do = _rand(rng, B, H, T, D, std=1.5)
    scale = 1.0 / math.sqrt(D)
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True)
                  for x in (q, k, v))
    s = (tq @ tk.transpose(-1, -2)) * scale
    mask = torch.ones(T, T, dtype=torch.bool).triu(1)
    s = s.masked_fill(mask, float("-inf"))
    to = torch.softmax(s, dim=-1) @ tv
    tlse = torch.logsumexp(s, dim=-1)
    (to * torch.tensor(do)).sum().backward()
    o, lse = impl.fwd(q, k, v, scale)
    dq, dk, dv = impl.bwd(q, k, v, do, scale)
    np.testing.assert_allclose(o, to.detach().numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(lse, tlse.detach().numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=0, atol=1e-10)


ALL_PINS = [pin_golden, pin_single_token, pin_constant_keys,
            pin_first_row_and_weights, pin_causality, pin_key_shift,
            pin_finite_differences, pin_brute_force, pin_torch_autograd]
