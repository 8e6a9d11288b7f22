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

from .moba import MobaLayout, block_of, moba_allowed


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


def _by_query_block(rows: np.ndarray, lay: MobaLayout):
    """Yield (positions into ``rows``, sorted key indices the block may read) for
    each query block the rows fall in; the rule is constant on a block, so its
    first row's allowed keys are every row's."""
    kind, idx = block_of(rows, lay)
    kpos = np.arange(lay.seq_len)
    for kd, ix in sorted(set(zip(kind.tolist(), idx.tolist()))):
        sel = np.nonzero((kind == kd) & (idx == ix))[0]
        keys = np.nonzero(moba_allowed(rows[sel[0]], kpos, lay))[0]
        yield sel, keys


def _rows_bwd(q, k, v, do, rows, keys, h, scale):
    """P, dS of the given query rows over their readable keys (head h)."""
    z = scale * (q[rows, h] @ k[keys, h].T)
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    p = e / e.sum(axis=1, keepdims=True)
    o = p @ v[keys, h]
    dp = do[rows, h] @ v[keys, h].T
    d = (do[rows, h] * o).sum(axis=1, keepdims=True)
    return p, p * (dp - d)


def moba_dq_rows(q, k, v, do, lay: MobaLayout, rows: Iterable[int], scale: float,
                 batch: int = 1024) -> np.ndarray:
    """dQ of the listed query rows ([n, H, D]), each from its own row of P (taken
    over the keys the row may read; every other entry of P is zero)."""
    q, k, v, do = (np.asarray(x, np.float64) for x in (q, k, v, do))
    rows = np.asarray(list(rows), dtype=np.int64)
    out = np.zeros((rows.size, q.shape[1], q.shape[2]))
    for sel, keys in _by_query_block(rows, lay):
        for b in range(0, sel.size, batch):
            part = sel[b:b + batch]
            for h in range(q.shape[1]):
                _, ds = _rows_bwd(q, k, v, do, rows[part], keys, h, scale)
                out[part, h] = scale * ds @ k[keys, h]
    return out


def _rows_p_cols(q, k, v, do, rows, keys, cols, h, scale):
    """P and dS of the given query rows (head h) on the key columns ``cols`` only.  The
    row's normaliser and D = rowsum(dO o O) need the whole row over its readable
    ``keys``; dS_ij = P_ij (dP_ij - D_i) is elementwise in j, so dP is formed on the
    listed columns alone."""
    z = scale * (q[rows, h] @ k[keys, h].T)
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    p = e / e.sum(axis=1, keepdims=True)
    o = p @ v[keys, h]
    d = (do[rows, h] * o).sum(axis=1, keepdims=True)
    p_c = p[:, cols]
    dp_c = do[rows, h] @ v[keys[cols], h].T
    return p_c, p_c * (dp_c - d)


def moba_dkdv_keys(q, k, v, do, lay: MobaLayout, keys: Iterable[int], scale: float,
                   batch: int = 1024):
    """dK and dV of the listed key rows ([n, H, D] each): the sums over every query
    that may read them.  Each such query's row of P is evaluated in full, so pick
    keys read by few queries."""
    q, k, v, do = (np.asarray(x, np.float64) for x in (q, k, v, do))
    keys = np.asarray(list(keys), dtype=np.int64)
    qpos = np.arange(lay.seq_len)
    readers = np.nonzero(np.any(moba_allowed(qpos[:, None], keys[None, :], lay), axis=1))[0]
    H = q.shape[1]
    dk = np.zeros((keys.size, H, q.shape[2]))
    dv = np.zeros_like(dk)
    for sel, ks in _by_query_block(readers, lay):
        col = np.searchsorted(ks, keys)
        hit = (col < ks.size) & (ks[np.minimum(col, ks.size - 1)] == keys)
        for b in range(0, sel.size, batch):
            r = readers[sel[b:b + batch]]
            for h in range(H):
                p_c, ds_c = _rows_p_cols(q, k, v, do, r, ks, col[hit], h, scale)
                dv[hit, h] += p_c.T @ do[r, h]
                dk[hit, h] += scale * ds_c.T @ q[r, h]
    return dk, dv
