"""fp64 CPU oracle for decode attention over a key/value cache.

TEST INFRASTRUCTURE ONLY (see oracle/attention.py): nothing on the product
path imports it; it shares no code with the CUDA library.

generate() in "nanoGPT: a real GPT in two 300-line files" (section 2, "How
the code works") runs the model once per new token and keeps the last
position; with a key/value cache only the newest positions need attention.
For a sequence whose first L keys and values are cached, and Tq query rows
at positions L - Tq .. L - 1, row r is the causal attention of that
position (same page, "Words to know": a position sees itself and earlier
ones):

    s_j = scale * q_r . k_j   for j = 0 .. L - Tq + r
    o_r = sum_j softmax(s)_j v_j,   lse_r = log sum_j exp(s_j)

which is the definition of causal attention restricted to those rows.
"""

from __future__ import annotations

import numpy as np


def decode_attention(q, k, v, scale, L):
    """q (B, H, Tq, D); k, v (B, H, >= L, D).  Returns (o (B, H, Tq, D),
    lse (B, H, Tq)) in float64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, H, Tq, D = q.shape
    if not 1 <= Tq <= L <= k.shape[2] or v.shape[2] < L:
        raise ValueError("need 1 <= Tq <= L <= cache length")
    o = np.empty((B, H, Tq, D))
    lse = np.empty((B, H, Tq))
    for b in range(B):
        for h in range(H):
            for r in range(Tq):
                pos = L - Tq + r
                s = scale * (k[b, h, :pos + 1] @ q[b, h, r])   # visible keys only
                m = s.max()
                e = np.exp(s - m)
                o[b, h, r] = (e / e.sum()) @ v[b, h, :pos + 1]
                lse[b, h, r] = m + np.log(e.sum())
    return o, lse
