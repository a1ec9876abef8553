"""fp64 CPU oracle for causal multi-head self-attention (forward + backward).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
module; only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it.  It shares no code with the CUDA library.

What it computes is the written-out ("slow") attention that
"nanoGPT: a real GPT in two 300-line files", section 2 "How the code works"
(model.py: the GPT, CausalSelfAttention) describes: q @ k transposed, times
1/sqrt(head size), future positions filled with minus infinity, softmax,
then @ v; done independently for every head.  "Causal" means a position
sees itself and earlier positions only (same page, "Words to know" and
section 8 "Self-check"), so key j is visible to query i iff j <= i.

The flash-style kernels reach exactly this result up to rounding (the online
softmax is an exact rewrite), so the oracle is the plain definition: it
materialises the T x T score matrix for one (b, h) at a time in float64.

The gradients are not printed on the pages (there, autograd supplies them:
section 1 "Summary", "Autograd does the calculus").  They are the chain rule
through the definition above, for a scalar loss L with dL/dO = dO:

    dV = P^T dO
    dP = dO V^T
    Delta_i = sum_j P_ij dP_ij          (= sum_d dO_id O_id)
    dS = P * (dP - Delta)               (softmax Jacobian, row-wise)
    dQ = scale * dS K
    dK = scale * dS^T Q

LSE is the natural-log row log-sum-exp of the scaled, masked scores,
computed stably as m + log(sum exp(S - m)).

Every pin of this module lives in tests/test_oracle.py (closed forms for
T = 1 and constant keys, row sums, causality under perturbation, shift
invariance, central finite differences, a pure-Python brute force and the
hand-derived fixture under tests/golden/).
"""

from __future__ import annotations

import numpy as np


def _check(q, k, v):
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if q.ndim != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share shape (B, H, T, D)")
    return q, k, v


def causal_mask(T: int) -> np.ndarray:
    """Boolean (T, T): True where key j is in the future of query i (j > i)."""
    return np.triu(np.ones((T, T), dtype=bool), k=1)


def head_probs(q2, k2, scale):
    """Scores, probabilities and LSE of one head.

    q2, k2: (T, D) float64.  Returns (P (T,T), lse (T,)).
    """
    s = scale * (q2 @ k2.T)                       # q @ k^T times scale
    s = np.where(causal_mask(s.shape[0]), -np.inf, s)   # fill the future
    m = s.max(axis=1, keepdims=True)              # row 0 always sees key 0
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    p = e / l                                     # softmax
    lse = (m + np.log(l))[:, 0]
    return p, lse


def attention_forward(q, k, v, scale):
    """Forward pass: returns (o (B,H,T,D), lse (B,H,T)) in float64."""
    q, k, v = _check(q, k, v)
    B, H, T, D = q.shape
    o = np.empty((B, H, T, D))
    lse = np.empty((B, H, T))
    for b in range(B):
        for h in range(H):
            p, lse[b, h] = head_probs(q[b, h], k[b, h], scale)
            o[b, h] = p @ v[b, h]                 # then @ v
    return o, lse


def attention_backward(q, k, v, do, scale, return_delta=False):
    """Backward pass of L = <O, dO>: returns (dq, dk, dv) in float64.

    With ``return_delta`` also returns Delta (B, H, T).
    """
    q, k, v = _check(q, k, v)
    do = np.asarray(do, dtype=np.float64)
    if do.shape != q.shape:
        raise ValueError("dO must match q's shape")
    B, H, T, D = q.shape
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    delta = np.empty((B, H, T))
    for b in range(B):
        for h in range(H):
            p, _ = head_probs(q[b, h], k[b, h], scale)
            dv[b, h] = p.T @ do[b, h]
            dp = do[b, h] @ v[b, h].T
            dlt = (p * dp).sum(axis=1)
            ds = p * (dp - dlt[:, None])
            dq[b, h] = scale * (ds @ k[b, h])
            dk[b, h] = scale * (ds.T @ q[b, h])
            delta[b, h] = dlt
    if return_delta:
        return dq, dk, dv, delta
    return dq, dk, dv


def attention_forward_heads(q, k, v, scale, heads):
    """Forward for a subset of flat head indices (b*H + h).

    Returns (o (n,T,D), lse (n,T)) for the listed heads, in order.
    """
    q, k, v = _check(q, k, v)
    B, H, T, D = q.shape
    o = np.empty((len(heads), T, D))
    lse = np.empty((len(heads), T))
    for n, f in enumerate(heads):
        b, h = divmod(f, H)
        p, lse[n] = head_probs(q[b, h], k[b, h], scale)
        o[n] = p @ v[b, h]
    return o, lse


def attention_backward_heads(q, k, v, do, scale, heads):
    """Backward for a subset of flat head indices; returns (dq, dk, dv)
    each (n, T, D)."""
    q, k, v = _check(q, k, v)
    do = np.asarray(do, dtype=np.float64)
    B, H, T, D = q.shape
    out = [np.empty((len(heads), T, D)) for _ in range(3)]
    for n, f in enumerate(heads):
        b, h = divmod(f, H)
        sub = [x[b:b + 1, h:h + 1] for x in (q, k, v, do)]
        dq, dk, dv = attention_backward(*sub, scale)
        out[0][n], out[1][n], out[2][n] = dq[0, 0], dk[0, 0], dv[0, 0]
    return tuple(out)


def attention_backward_given_o(q, k, v, do, o_heads, scale, heads):
    """Backward pass with the row term taken from a GIVEN output instead of
    the exact one, for a subset of flat head indices (b*H + h).

    The chain rule above writes Delta either as sum_j P_ij dP_ij or as
    sum_d dO_id O_id; a backward that receives O from the caller (the pages'
    interface passes it in bf16) can only use the second form with the O
    it was given.  Here Delta_i = sum_d dO_id o_id with o from ``o_heads``
    ((n, T, D), one row block per listed head), and then, as in
    attention_backward, dS = P * (dP - Delta), dQ = scale dS K,
    dK = scale dS^T Q, dV = P^T dO.  With o equal to the exact output this
    is attention_backward; with o = bf16(exact output) it is the exact
    gradient reachable through that interface.  Returns (dq, dk, dv), each
    (n, T, D).
    """
    q, k, v = _check(q, k, v)
    do = np.asarray(do, dtype=np.float64)
    o_heads = np.asarray(o_heads, dtype=np.float64)
    B, H, T, D = q.shape
    out = [np.empty((len(heads), T, D)) for _ in range(3)]
    for n, f in enumerate(heads):
        b, h = divmod(f, H)
        p, _ = head_probs(q[b, h], k[b, h], scale)
        dp_n = do[b, h] @ v[b, h].T
        dlt_o = (o_heads[n] * do[b, h]).sum(axis=1)    # Delta from the given O
        ds_n = p * (dp_n - dlt_o[:, None])
        out[0][n] = scale * (ds_n @ k[b, h])
        out[1][n] = scale * (ds_n.T @ q[b, h])
        out[2][n] = p.T @ do[b, h]
    return tuple(out)


def attention_rows(q, k, v, scale, b, h, rows):
    """O and LSE of chosen query rows of one head, one row at a time.

    A row i needs only keys 0..i, so this scales to any T: used to check
    sampled outputs of the full-size workloads.
    """
    q, k, v = (np.asarray(x[b, h], dtype=np.float64) for x in (q, k, v))
    o = np.empty((len(rows), q.shape[1]))
    lse = np.empty(len(rows))
    for n, i in enumerate(rows):
        s = scale * (k[:i + 1] @ q[i])            # visible keys only
        m = s.max()
        e = np.exp(s - m)
        l = e.sum()
        o[n] = (e / l) @ v[:i + 1]
        lse[n] = m + np.log(l)
    return o, lse


def delta_from_o(o, do):
    """Delta_i = sum_d dO_id * O_id for given O and dO (any leading dims)."""
    o = np.asarray(o, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    return (o * do).sum(axis=-1)
