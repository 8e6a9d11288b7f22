"""3D rotary position embedding (t, h, w), plain fp64.

What it computes.  The 832x464 workload statement fixes a 3D RoPE over
(latent frame t, patch row h, patch column w) with base 10000, absolute
indices and the rotary split 44/42/42 dims over head_dim 128; the pages only
name RoPE as one of the fused elementwise kernels ([RT], step table, "Kernel
fusion" row).  Readings taken where the statement is silent:

  * head_dim is cut into D/2 consecutive *interleaved* pairs (x[2i], x[2i+1]);
    the first ``pairs_t`` pairs rotate with t, the next ``pairs_h`` with h,
    the last ``pairs_w`` with w.
  * within an axis that owns P pairs, pair j turns by the angle
    pos * base ** (-(2 j) / (2 P)), i.e. ordinary 1D RoPE of width 2P.
  * the rotation of a pair is (x0 cos a - x1 sin a, x0 sin a + x1 cos a).
  * the default split gives h and w floor(D/6) pairs and t the rest
    (22/21/21 pairs = 44/42/42 dims at D = 128; 12/10/10 pairs at D = 64,
    where the stated "22/21/21 dims" cannot be cut into pairs).

Parity: pinned (identity at position 0, pair-norm preservation, relative
position property, reduction to textbook 1D RoPE, axis separation).
"""
from __future__ import annotations

import math
from typing import Tuple

import numpy as np


def rope_pairs_default(head_dim: int) -> Tuple[int, int, int]:
    """(pairs_t, pairs_h, pairs_w) of the default split (see module header)."""
    ph = head_dim // 6
    return head_dim // 2 - 2 * ph, ph, ph


def axis_of_pair(i: int, pairs: Tuple[int, int, int]) -> Tuple[int, int]:
    """Axis (0 = t, 1 = h, 2 = w) and index j within that axis of pair i."""
    pt, ph, pw = pairs
    if i < pt:
        return 0, i
    if i < pt + ph:
        return 1, i - pt
    if i < pt + ph + pw:
        return 2, i - pt - ph
    raise IndexError(i)


def rope_positions(frames, grid_h: int, grid_w: int):
    """Per-token (t, h, w) positions of whole latent frames.

    Tokens of one frame are row-major over the (h, w) patch grid, frames are
    concatenated in the given order.  Returns three int64 arrays of length
    len(frames) * grid_h * grid_w.
    """
    T = grid_h * grid_w
    t = np.repeat(np.asarray(frames, dtype=np.int64), T)
    tok = np.tile(np.arange(T, dtype=np.int64), len(frames))
    return t, tok // grid_w, tok % grid_w


def rope3d(x: np.ndarray, t: np.ndarray, h: np.ndarray, w: np.ndarray,
           pairs: Tuple[int, int, int], base: float = 10000.0) -> np.ndarray:
    """Rotate ``x`` [N, H, D] (any float dtype) at token positions (t, h, w).

    Returns a new float64 array.  Positions are per token (length N); every
    head uses the same rotation.
    """
    x = np.asarray(x, dtype=np.float64)
    N, H, D = x.shape
    if sum(pairs) * 2 != D:
        raise ValueError("pairs must cover head_dim")
    pos = (np.asarray(t, dtype=np.float64), np.asarray(h, dtype=np.float64),
           np.asarray(w, dtype=np.float64))
    # angle of every (token, pair): pair i of axis a (index j in it) turns by pos_a * freq
    ang = np.empty((N, D // 2))
    for i in range(D // 2):
        axis, j = axis_of_pair(i, pairs)
        ang[:, i] = pos[axis] * base ** (-(2.0 * j) / (2.0 * pairs[axis]))
    c = np.cos(ang)[:, None, :]                      # [N, 1, D/2]
    s = np.sin(ang)[:, None, :]
    x0 = x[:, :, 0::2]                               # first element of each pair
    x1 = x[:, :, 1::2]
    out = np.empty_like(x)
    out[:, :, 0::2] = x0 * c - x1 * s
    out[:, :, 1::2] = x0 * s + x1 * c
    return out


def rope_angle(axis_pos: float, j: int, n_pairs: int, base: float = 10000.0) -> float:
    """Angle of pair j of an axis with ``n_pairs`` pairs at position axis_pos."""
    return axis_pos * base ** (-(2.0 * j) / (2.0 * n_pairs))


__all__ = ["rope3d", "rope_positions", "axis_of_pair", "rope_pairs_default", "rope_angle",
           "math"]
