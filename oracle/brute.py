"""Pure-Python brute force of causal attention, for tiny inputs only.

TEST INFRASTRUCTURE ONLY (see oracle/attention.py).  This is a second,
independent statement of the same definition ("nanoGPT: a real GPT in two
300-line files", section 2 "How the code works": scores = q.k times
1/sqrt(head size), future filled with minus infinity, softmax, then a
weighted sum of v), written as explicit loops over Python floats with
``math.exp``/``math.log`` and no numpy, so that a slip in the vectorised
oracle (a transposed operand, a wrong mask diagonal, a dropped term) shows
up as a disagreement.  It takes nested lists [T][D] for one head.

The backward here is *not* the Delta/dS formulation of the vectorised
oracle: it differentiates L = sum_i sum_d O_id dO_id directly through the
quotient O_i = sum_j e_ij v_j / sum_j e_ij with e_ij = exp(s_ij), term by
term, so the two share no algebraic shortcut.
"""

from __future__ import annotations

import math


def forward_head(q, k, v, scale):
    """q, k, v: lists [T][D].  Returns (o [T][D], lse [T])."""
    T = len(q)
    D = len(q[0])
    o, lse = [], []
    for i in range(T):
        s = []
        for j in range(i + 1):                    # visible keys j <= i
            acc = 0.0
            for d in range(D):
                acc += q[i][d] * k[j][d]
            s.append(acc * scale)
        m = max(s)
        w = [math.exp(x - m) for x in s]
        z = sum(w)
        row = []
        for d in range(D):
            acc = 0.0
            for j in range(i + 1):
                acc += w[j] * v[j][d]
            row.append(acc / z)
        o.append(row)
        lse.append(m + math.log(z))
    return o, lse


def backward_head(q, k, v, do, scale):
    """Gradients of L = <O, dO> by the quotient rule, term by term.

    Returns (dq, dk, dv) as lists [T][D].
    """
    T = len(q)
    D = len(q[0])
    dq = [[0.0] * D for _ in range(T)]
    dk = [[0.0] * D for _ in range(T)]
    dv = [[0.0] * D for _ in range(T)]
    for i in range(T):
        s = []
        for j in range(i + 1):
            s.append(scale * sum(q[i][d] * k[j][d] for d in range(D)))
        m = max(s)
        e = [math.exp(x - m) for x in s]
        z = sum(e)
        # numerator N_d = sum_j e_j v_jd ; O_d = N_d / z
        num = [sum(e[j] * v[j][d] for j in range(i + 1)) for d in range(D)]
        # dL/dv_jd = dO_id * e_j / z
        for j in range(i + 1):
            for d in range(D):
                dv[j][d] += do[i][d] * e[j] / z
        # dL/ds_j = sum_d dO_id * (e_j v_jd / z - N_d e_j / z^2)
        for j in range(i + 1):
            g = 0.0
            for d in range(D):
                g += do[i][d] * (e[j] * v[j][d] / z - num[d] * e[j] / (z * z))
            # s_j = scale * q_i . k_j
            for d in range(D):
                dq[i][d] += g * scale * k[j][d]
                dk[j][d] += g * scale * q[i][d]
    return dq, dk, dv
