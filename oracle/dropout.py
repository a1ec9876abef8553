"""fp64 CPU oracle for causal self-attention with attention dropout.

TEST INFRASTRUCTURE ONLY (see oracle/attention.py): nothing on the product
path imports it; it shares no code with the CUDA library.

What is computed.  "nanoGPT: a real GPT in two 300-line files", section 2
"How the code works" (model.py, CausalSelfAttention.forward) passes the
model's dropout rate to PyTorch's fused attention while training, and
section 3 "Run it, tested" gives 0.2 for the character-level Shakespeare
model.  The pages do not spell out what that dropout does; the plain
reading, and the one PyTorch documents for that argument, is inverted
dropout on the attention probabilities after the softmax:

    P   = softmax_row(scale * Q K^T + causal mask)       (as without dropout)
    M_ij in {0, 1}, kept with probability 1 - p
    P~  = P * M / (1 - p)
    O   = P~ V,       LSE unchanged (the log-sum-exp of the undropped scores)

and, for a scalar loss with dL/dO = dO (chain rule through the above, the
mask held fixed):

    dV      = P~^T dO
    dP~     = dO V^T
    dP      = dP~ * M / (1 - p)
    Delta_i = sum_j P_ij dP_ij        (= sum_d dO_id O_id, as without dropout)
    dS      = P * (dP - Delta)
    dQ = scale * dS K,   dK = scale * dS^T Q

The mask.  Random bits come from Philox4x32-10, the counter-based generator
of J. K. Salmon, M. A. Moraes, R. O. Dror and D. E. Shaw, "Parallel random
numbers: as easy as 1, 2, 3" (SC 2011), written here from its definition:
a 4 x 32-bit counter and a 2 x 32-bit key, ten rounds of two 32 x 32 -> 64
bit multiplications whose halves are mixed with the other counter words and
the key, the key advanced by two Weyl constants between rounds.  The kernel
side implements the same generator on its own; the two agree because both
follow the definition, which published known-answer vectors pin
(tests/golden/philox4x32_10_kat.txt).

Element (b, h, i, j) of the mask (query i, key j) takes 8 random bits
from the Philox block with

    counter = (j >> 4, i, b * H + h, offset),   key = (seed low 32, seed high 32)

namely byte j & 3 (bits 8 (j & 3) .. 8 (j & 3) + 7) of output word
(j & 15) >> 2.  The element is dropped iff that byte, as an unsigned
integer, is below t = round(p * 256); so the drop probability is t / 256
(p to within 2^-9) and the kept values are scaled by 256 / (256 - t),
which makes E[P~] = P exactly.  The pages fix the rate, not how finely it
is drawn: 8 bits per element is the reading taken here (flash-attention's
own dropout also draws 8 bits per element), one generator block per 16
elements.
"""

from __future__ import annotations

import numpy as np

from .attention import _check, head_probs

# Philox4x32 round multipliers and key increments (Salmon et al. 2011).
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
MASK32 = 0xFFFFFFFF


def philox4x32_10(ctr, key):
    """Philox4x32 with 10 rounds.

    ctr: uint array (..., 4) of 32-bit counter words; key: (k0, k1) ints.
    Returns uint64 array (..., 4) holding the four 32-bit output words.
    """
    c = np.asarray(ctr, dtype=np.uint64) & np.uint64(MASK32)
    c0, c1, c2, c3 = (c[..., n].copy() for n in range(4))
    k0, k1 = int(key[0]) & MASK32, int(key[1]) & MASK32
    m0, m1 = np.uint64(PHILOX_M0), np.uint64(PHILOX_M1)
    sh, lo = np.uint64(32), np.uint64(MASK32)
    for rnd in range(10):
        if rnd > 0:                                   # bump the key between rounds
            k0 = (k0 + PHILOX_W0) & MASK32
            k1 = (k1 + PHILOX_W1) & MASK32
        p0 = c0 * m0                                  # exact: both factors < 2^32
        p1 = c2 * m1
        hi0, lo0 = p0 >> sh, p0 & lo
        hi1, lo1 = p1 >> sh, p1 & lo
        c0, c1, c2, c3 = (hi1 ^ c1 ^ np.uint64(k0), lo1,
                          hi0 ^ c3 ^ np.uint64(k1), lo0)
    return np.stack([c0, c1, c2, c3], axis=-1)


def drop_threshold(p: float) -> int:
    """t = round(p * 256) for 0 <= p < 1 (at most 255)."""
    if not 0.0 <= p < 1.0:
        raise ValueError("dropout probability must be in [0, 1)")
    return min(int(np.rint(p * 256.0)), 255)


def keep_scale(p: float) -> float:
    """The factor kept probabilities are multiplied by: 1 / (1 - t/256)."""
    t = drop_threshold(p)
    return 256.0 / (256.0 - t)


def random8(b, h, H, i, j, seed: int, offset: int):
    """The 8 random bits of mask element(s) (b, h, i, j); i and j may be
    broadcastable integer arrays."""
    i = np.asarray(i, dtype=np.uint64)
    j = np.asarray(j, dtype=np.uint64)
    i, j = np.broadcast_arrays(i, j)
    ctr = np.stack([j >> np.uint64(4), i,
                    np.full(i.shape, b * H + h, dtype=np.uint64),
                    np.full(i.shape, offset & MASK32, dtype=np.uint64)], axis=-1)
    out = philox4x32_10(ctr, (seed & MASK32, (seed >> 32) & MASK32))
    word = np.take_along_axis(out, ((j & np.uint64(15)) >> np.uint64(2)).astype(np.int64)[..., None],
                              axis=-1)[..., 0]
    return (word >> (np.uint64(8) * (j & np.uint64(3)))) & np.uint64(0xFF)


def keep_mask_head(b, h, H, T, p: float, seed: int, offset: int):
    """Boolean (T, T) keep mask of head (b, h): True where kept (the future
    half is returned too, though it never matters)."""
    r = random8(b, h, H, np.arange(T)[:, None], np.arange(T)[None, :], seed, offset)
    return r >= np.uint64(drop_threshold(p))


def attention_forward_dropout(q, k, v, scale, p, seed, offset):
    """Forward with dropout: returns (o (B,H,T,D), lse (B,H,T)), float64."""
    q, k, v = _check(q, k, v)
    B, H, T, D = q.shape
    ks = keep_scale(p)
    o = np.empty((B, H, T, D))
    lse = np.empty((B, H, T))
    for b in range(B):
        for h in range(H):
            pr, lse[b, h] = head_probs(q[b, h], k[b, h], scale)
            m = keep_mask_head(b, h, H, T, p, seed, offset)
            o[b, h] = (pr * m * ks) @ v[b, h]
    return o, lse


def attention_backward_dropout(q, k, v, do, scale, p, seed, offset):
    """Backward of L = <O, dO> with dropout: returns (dq, dk, dv), float64."""
    q, k, v = _check(q, k, v)
    do = np.asarray(do, dtype=np.float64)
    if do.shape != q.shape:
        raise ValueError("dO must match q's shape")
    B, H, T, D = q.shape
    ks = keep_scale(p)
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    for b in range(B):
        for h in range(H):
            pr, _ = head_probs(q[b, h], k[b, h], scale)
            m = keep_mask_head(b, h, H, T, p, seed, offset)
            pd = pr * m * ks                          # P~
            dv[b, h] = pd.T @ do[b, h]
            dpd = do[b, h] @ v[b, h].T                # dP~
            dp = dpd * m * ks
            dlt = (pr * dp).sum(axis=1)
            ds = pr * (dp - dlt[:, None])
            dq[b, h] = scale * (ds @ k[b, h])
            dk[b, h] = scale * (ds.T @ q[b, h])
    return dq, dk, dv
