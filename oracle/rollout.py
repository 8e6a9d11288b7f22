"""Chunk-wise autoregressive rollout over the sink + window cache, fp64.

What it computes ([LWI] "The trick: treat video like a causal stream": the
state is anchor tokens plus recent context, old tokens are evicted while the
anchors are kept, each step reads the state and its result is appended;
[WiW]: the block reads 6 anchor + 8 recent + 4 current latent frames; [RT]
setup: 16-frame chunks = 4 latent frames, four denoising steps):

  for each chunk t (frames f0 .. f0+F-1):
      (dynamic window) evict down to the scheduled window W_t
      for each denoising step:
          Q_rot = RoPE3D(Q), K_rot = RoPE3D(K) at the chunk's own positions
          O = attention(Q_rot, [K of cached frames, K_rot], [V cached, V])
      append the last step's rotated K and V of each frame to the cache

Readings: the queries of a chunk read every token of their own chunk (no
causal mask inside a chunk); the cache stores K already rotated at its
absolute frame index; V is not rotated; the finalized K/V are the last
step's; with a dynamic window the eviction to W_t happens before the
chunk's attention and appends use the largest window as capacity.

Auxiliary frames ([WiW] second paragraph: temporary auxiliary attention
blocks carry extra evidence for the current chunk and are removed once it is
finalized): ``aux_for(chunk)`` may give K, V of extra frames (and temporal
positions, at which K is rotated like a cached frame; without positions K is
used as given); every attention call of that chunk reads them besides the
cached frames and the chunk itself, and they are never cached.

Parity: pinned (equals brute-force attention over the whole concatenated
rollout under the set-based visibility rule; a chunk's output does not change
when later chunks change; auxiliary copies of every visible frame leave O
unchanged and add ln 2 to LSE; auxiliary frames change only their own chunk).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np

from . import fp8
from .attn import attention
from .cache import CacheModel
from .rope import rope3d, rope_pairs_default, rope_positions


@dataclasses.dataclass
class RolloutResult:
    outputs: List[np.ndarray]          # per (chunk, step): O of the checked rows [n, H, D]
    lses: List[np.ndarray]             # per (chunk, step): LSE [H, n]
    rows: List[np.ndarray]             # per (chunk, step): checked row indices
    slot_maps: List[List[int]]         # per chunk, after its append
    appended_slots: List[List[int]]    # per chunk: slot of each appended frame
    evicted: List[List[int]]           # per chunk: frames evicted (dynamic evict + append)
    visible: List[List[int]]           # per chunk: cached frames read (ascending)
    n_keys: List[int]                  # per chunk: keys read (cached + current)


def rollout(spec, chunks, rows_for=None, use_rope: bool = True,
            window_schedule: Optional[List[int]] = None, aux_for=None,
            qk_fp8: bool = False) -> RolloutResult:
    """Run the rollout of ``spec`` (a RolloutSpec) over ``chunks``.

    ``chunks`` yields dicts with chunk, step, frames, q, k, v as produced by
    ``workloads.rollout_chunks``.  ``rows_for(chunk, step)`` returns the query
    rows to evaluate (default: all).  ``aux_for(chunk)`` returns None or
    (k_aux, v_aux, positions) with k_aux, v_aux [n * T, H, D] and positions a
    list of n temporal positions or None.  ``qk_fp8``: the QK^T product sees Q
    and K as ``fp8.fp8_operand`` gives them -- blocks of 128 tokens of each
    cached or auxiliary frame, and of the current chunk for its own Q and K.
    """
    T = spec.grid_h * spec.grid_w
    scale = 1.0 / math.sqrt(spec.head_dim)
    pairs = (spec.rope().pairs_t, spec.rope().pairs_h, spec.rope().pairs_w)
    # the workload states the split; it must be the oracle's own pinned default
    if pairs != rope_pairs_default(spec.head_dim):
        raise ValueError(f"RoPE pair split {pairs} differs from the oracle's default "
                         f"{rope_pairs_default(spec.head_dim)} for head_dim {spec.head_dim}")
    cap = spec.window if window_schedule is None else max(spec.window, max(window_schedule))
    cache = CacheModel(spec.sinks, cap)
    store: Dict[int, tuple] = {}     # frame -> (K_rot [T,H,D], V [T,H,D])
    res = RolloutResult([], [], [], [], [], [], [], [])
    pending_evicted: List[int] = []
    for item in chunks:
        c, s, frames = item["chunk"], item["step"], item["frames"]
        q = np.asarray(item["q"], dtype=np.float64)
        k = np.asarray(item["k"], dtype=np.float64)
        v = np.asarray(item["v"], dtype=np.float64)
        if s == 0 and window_schedule is not None:
            pending_evicted = cache.evict(window_schedule[c])
            for f in pending_evicted:
                store.pop(f, None)
        rows = np.arange(q.shape[0]) if rows_for is None else np.asarray(rows_for(c, s))
        if qk_fp8:
            # a query block's scale depends on all of its rows: rotate them all
            if use_rope:
                t, hh, ww = rope_positions(frames, spec.grid_h, spec.grid_w)
                q_rot = fp8.fp8_operand(rope3d(q, t, hh, ww, pairs, spec.rope().base))[rows]
                k_rot = rope3d(k, t, hh, ww, pairs, spec.rope().base)
            else:
                q_rot, k_rot = fp8.fp8_operand(q)[rows], k
        elif use_rope:
            # each token turns by the angles of its own position, so only the
            # evaluated query rows need rotating
            t, hh, ww = rope_positions(frames, spec.grid_h, spec.grid_w)
            q_rot = rope3d(q[rows], t[rows], hh[rows], ww[rows], pairs, spec.rope().base)
            k_rot = rope3d(k, t, hh, ww, pairs, spec.rope().base)
        else:
            q_rot, k_rot = q[rows], k
        vis = cache.cached_frames()
        k_aux, v_aux = [], []
        aux = aux_for(c) if aux_for is not None else None
        if aux is not None and np.asarray(aux[0]).shape[0] > 0:
            ka = np.asarray(aux[0], dtype=np.float64)
            va = np.asarray(aux[1], dtype=np.float64)
            if aux[2] is not None and use_rope:
                ta, ha, wa = rope_positions(list(aux[2]), spec.grid_h, spec.grid_w)
                ka = rope3d(ka, ta, ha, wa, pairs, spec.rope().base)
            k_aux, v_aux = [ka], [va]
        if qk_fp8:
            # per frame for cached and auxiliary keys, over the chunk for its own
            k_cached = [fp8.fp8_operand(store[f][0]) for f in vis]
            k_aux = [fp8.fp8_operand(ka[n * T:(n + 1) * T]) for ka in k_aux
                     for n in range(ka.shape[0] // T)]
            k_all = np.concatenate(k_cached + k_aux + [fp8.fp8_operand(k_rot)], axis=0)
        else:
            k_all = np.concatenate([store[f][0] for f in vis] + k_aux + [k_rot], axis=0)
        v_all = np.concatenate([store[f][1] for f in vis] + v_aux + [v], axis=0)
        o, lse = attention(q_rot, k_all, v_all, scale)
        res.outputs.append(o)
        res.lses.append(lse)
        res.rows.append(rows)
        if s == spec.steps - 1:
            res.visible.append(vis)
            res.n_keys.append(k_all.shape[0])
            slots, ev = cache.append(frames)
            for f in ev:
                store.pop(f, None)
            for n, f in enumerate(frames):
                if slots[n] >= 0:
                    store[f] = (k_rot[n * T:(n + 1) * T], v[n * T:(n + 1) * T])
            res.appended_slots.append(slots)
            res.evicted.append(pending_evicted + ev)
            res.slot_maps.append(cache.slot_map())
            pending_evicted = []
    return res
