"""Softmax attention, plain fp64.

What it computes: for each head, O = softmax(scale * Q K^T) V over the keys a
query may read, and LSE = log sum_k exp(scale * q . k).  This is the
definition of the attention the chunk reads with ([LWI] "How the cache keeps
the world alive": self-attention over the sliding KV cache with sink tokens;
[WiW]: the native block reads 6 anchor + 8 recent + 4 current latent-frame
slots).  Keys that a query may not read do not take part at all; a query
that may read no key gets O = 0 and LSE = -inf (not reachable by any
workload here; defined for robustness).

Parity: pinned (brute-force scalar loops on tiny inputs, Q = 0 -> mean of V
and LSE = ln N, constant V, single key, key permutation invariance).
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import numpy as np


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float
              ) -> Tuple[np.ndarray, np.ndarray]:
    """q [Nq, H, D], k/v [Nk, H, D] -> (O [Nq, H, D] fp64, LSE [H, Nq] fp64)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Nq, H, D = q.shape
    o = np.zeros((Nq, H, v.shape[2]), dtype=np.float64)
    lse = np.full((H, Nq), -np.inf, dtype=np.float64)
    if k.shape[0] == 0:
        return o, lse
    for h in range(H):
        z = scale * (q[:, h, :] @ k[:, h, :].T)           # [Nq, Nk]
        m = z.max(axis=1, keepdims=True)
        p = np.exp(z - m)
        l = p.sum(axis=1, keepdims=True)
        o[:, h, :] = (p @ v[:, h, :]) / l
        lse[h] = (m + np.log(l))[:, 0]
    return o, lse


def masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, allowed: np.ndarray,
                     scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Attention where query i reads key j only if ``allowed[i, j]``.

    Rows are handled one at a time so that disallowed keys never enter the
    arithmetic.
    """
    q = np.asarray(q, dtype=np.float64)
    Nq, H, D = q.shape
    o = np.zeros((Nq, H, v.shape[2]), dtype=np.float64)
    lse = np.full((H, Nq), -np.inf, dtype=np.float64)
    for i in range(Nq):
        keys = np.nonzero(allowed[i])[0]
        if keys.size == 0:
            continue
        oi, li = attention(q[i:i + 1], k[keys], v[keys], scale)
        o[i] = oi[0]
        lse[:, i] = li[:, 0]
    return o, lse


def attention_bruteforce(q, k, v, scale: float, allowed: Optional[np.ndarray] = None):
    """Scalar Python loops (tiny inputs only): the textbook definition
    o_i = sum_j exp(s_ij) v_j / sum_j exp(s_ij), s_ij = scale * q_i . k_j,
    written without max-subtraction or vectorisation."""
    Nq, H, D = len(q), len(q[0]), len(q[0][0])
    Nk = len(k)
    Dv = len(v[0][0]) if Nk else D
    o = [[[0.0] * Dv for _ in range(H)] for _ in range(Nq)]
    lse = [[-math.inf] * Nq for _ in range(H)]
    for i in range(Nq):
        for h in range(H):
            num = [0.0] * Dv
            den = 0.0
            for j in range(Nk):
                if allowed is not None and not allowed[i][j]:
                    continue
                s = scale * sum(float(q[i][h][d]) * float(k[j][h][d]) for d in range(D))
                e = math.exp(s)
                den += e
                for d in range(Dv):
                    num[d] += e * float(v[j][h][d])
            if den > 0.0:
                o[i][h] = [x / den for x in num]
                lse[h][i] = math.log(den)
    return np.array(o, dtype=np.float64), np.array(lse, dtype=np.float64)
