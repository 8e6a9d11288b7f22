"""Backward pass of attention under the MoBA mask, plain fp64.

What it computes (the training step that follows the MoBA forward: "Infinite
Worlds with Versatile Interactions", causal-pretraining paragraph -- the mask
is used to pretrain the model; "Mix Forcing", "Mix the training modes").  For
O = softmax(scale * Q K^T restricted to the allowed keys) V and an upstream
gradient dO, with P the attention probabilities:

    dV = P^T dO
    dP = dO V^T
    D_i = sum_j P_ij dP_ij  ( = sum_d dO_id O_id )
    dS = P o (dP - D)            (elementwise, zero where a key is not allowed)
    dQ = scale * dS K
    dK = scale * dS^T Q

This is the chain rule written out for softmax attention; nothing in it is
approximate.  Rows that may read no key contribute nothing.

Parity: pinned (central finite differences of the forward oracle's loss
sum(O * dO) on tiny inputs; dV against an explicit sum; the identity
D = rowsum(dO o O)).
"""
from __future__ import annotations

from typing import Iterable, Tuple

import numpy as np

from .moba import MobaLayout, moba_allowed


def attention_bwd_masked(q, k, v, do, allowed: np.ndarray, scale: float
                         ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Full-matrix backward for small inputs: q, k, v, do [L, H, D]; allowed [Lq, Lk].
    Returns (dq, dk, dv) in fp64."""
    q, k, v, do = (np.asarray(x, np.float64) for x in (q, k, v, do))
    H = q.shape[1]
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for h in range(H):
        z = scale * (q[:, h] @ k[:, h].T)
        z = np.where(allowed, z, -np.inf)
        m = z.max(axis=1, keepdims=True)
        m = np.where(np.isfinite(m), m, 0.0)
        e = np.exp(z - m)
        l = e.sum(axis=1, keepdims=True)
        p = np.where(l > 0, e / np.where(l > 0, l, 1.0), 0.0)
        o = p @ v[:, h]
        dv[:, h] = p.T @ do[:, h]
        dp = do[:, h] @ v[:, h].T
        d = (do[:, h] * o).sum(axis=1, keepdims=True)
        ds = p * (dp - d)
        dq[:, h] = scale * ds @ k[:, h]
        dk[:, h] = scale * ds.T @ q[:, h]
    return dq, dk, dv


def moba_bwd_dense(q, k, v, do, lay: MobaLayout, scale: float):
    """Backward under the MoBA mask with the explicit [L, L] mask (small layouts)."""
    pos = np.arange(lay.seq_len)
    return attention_bwd_masked(q, k, v, do, moba_allowed(pos[:, None], pos[None, :], lay), scale)


def _row_probs(q, k, lay, rows, h, scale):
    """P rows (over all keys; zeros where not allowed) of the listed query rows, head h."""
    kpos = np.arange(lay.seq_len)
    out = np.zeros((len(rows), lay.seq_len))
    for n, r in enumerate(rows):
        keys = np.nonzero(moba_allowed(r, kpos, lay))[0]
        z = scale * (k[keys, h] @ q[r, h])
        z = z - z.max()
        e = np.exp(z)
        out[n, keys] = e / e.sum()
    return out


def moba_dq_rows(q, k, v, do, lay: MobaLayout, rows: Iterable[int], scale: float) -> np.ndarray:
    """dQ of the listed query rows ([n, H, D]), each from its own row of P."""
    q, k, v, do = (np.asarray(x, np.float64) for x in (q, k, v, do))
    rows = list(rows)
    H = q.shape[1]
    out = np.zeros((len(rows), H, q.shape[2]))
    for h in range(H):
        p = _row_probs(q, k, lay, rows, h, scale)            # [n, L]
        o = p @ v[:, h]
        dp = do[rows, h] @ v[:, h].T
        d = (do[rows, h] * o).sum(axis=1, keepdims=True)
        ds = p * (dp - d)
        out[:, h] = scale * ds @ k[:, h]
    return out


def moba_dkdv_keys(q, k, v, do, lay: MobaLayout, keys: Iterable[int], scale: float):
    """dK and dV of the listed key rows ([n, H, D] each).  Every query that may read
    one of the keys is evaluated in full, so pick keys read by few queries."""
    q, k, v, do = (np.asarray(x, np.float64) for x in (q, k, v, do))
    keys = np.asarray(list(keys))
    qpos = np.arange(lay.seq_len)
    readers = np.nonzero(np.any(moba_allowed(qpos[:, None], keys[None, :], lay), axis=1))[0]
    H = q.shape[1]
    dk = np.zeros((keys.size, H, q.shape[2]))
    dv = np.zeros_like(dk)
    for h in range(H):
        p = _row_probs(q, k, lay, readers, h, scale)          # [nq, L]
        o = p @ v[:, h]
        dp = do[readers, h] @ v[:, h].T
        d = (do[readers, h] * o).sum(axis=1, keepdims=True)
        ds = p * (dp - d)
        dv[:, h] = p[:, keys].T @ do[readers, h]
        dk[:, h] = scale * ds[:, keys].T @ q[readers, h]
    return dk, dv
