"""MoBA (Mixture of Bidirectional and Autoregressive) training mask.

What it computes ([IW] causal-pretraining paragraph; [MF] "Mix the training
modes"): a teacher-forcing mask for causal next-chunk prediction with a fully
bidirectional block appended.  The sequence is

    [ C1 .. Cn | N1 .. Nn | B ]       (clean chunks, noisy chunks, bidir block)

and a query may read a key as follows (the MoBA workload statement spells
the rule out; the pages give its shape):

    query in C_i : keys of C_j for j <= i           (clean history, causal)
    query in N_i : keys of C_j for j <  i, and N_i  (teacher forcing)
    query in B   : every key of B                    (bidirectional block)

and nothing else.  Within one (query chunk, key chunk) pair the rule is all
or nothing, so a square tile of the score matrix is FULL (every in-range
entry allowed), EMPTY (none) or PARTIAL.

Parity: pinned (n = 1 reduces to three independent full attentions;
tile classes by reduction of the explicit boolean mask vs by reduction over
the chunk pairs a tile spans; closed-form count of allowed entries).
"""
from __future__ import annotations

import dataclasses
from typing import Iterable, Tuple

import numpy as np

from .attn import attention

TILE_EMPTY = 0
TILE_PARTIAL = 1
TILE_FULL = 2

BLOCK_C, BLOCK_N, BLOCK_B = 0, 1, 2


@dataclasses.dataclass(frozen=True)
class MobaLayout:
    n_chunks: int
    chunk_tokens: int
    n_bidir_chunks: int

    @property
    def seq_len(self) -> int:
        return (2 * self.n_chunks + self.n_bidir_chunks) * self.chunk_tokens


def block_of(pos: np.ndarray, lay: MobaLayout) -> Tuple[np.ndarray, np.ndarray]:
    """(block kind, chunk index within the kind) of each position."""
    pos = np.asarray(pos, dtype=np.int64)
    nc = lay.n_chunks * lay.chunk_tokens
    kind = np.where(pos < nc, BLOCK_C, np.where(pos < 2 * nc, BLOCK_N, BLOCK_B))
    base = np.where(kind == BLOCK_C, 0, np.where(kind == BLOCK_N, nc, 2 * nc))
    idx = (pos - base) // lay.chunk_tokens
    return kind, idx


def moba_allowed(qpos, kpos, lay: MobaLayout) -> np.ndarray:
    """Boolean: may the query at ``qpos`` read the key at ``kpos`` (broadcasts)."""
    qk, qi = block_of(qpos, lay)
    kk, ki = block_of(kpos, lay)
    c_row = (qk == BLOCK_C) & (kk == BLOCK_C) & (ki <= qi)
    n_row = (qk == BLOCK_N) & (((kk == BLOCK_C) & (ki < qi)) | ((kk == BLOCK_N) & (ki == qi)))
    b_row = (qk == BLOCK_B) & (kk == BLOCK_B)
    return c_row | n_row | b_row


def moba_mask(lay: MobaLayout) -> np.ndarray:
    """Explicit [L, L] boolean mask (small layouts only)."""
    pos = np.arange(lay.seq_len)
    return moba_allowed(pos[:, None], pos[None, :], lay)


def _n_tiles(L: int, tile: int) -> int:
    return (L + tile - 1) // tile


def classify_tiles_mask(lay: MobaLayout, tile: int = 128) -> np.ndarray:
    """Tile classes by reducing the explicit mask over each tile's in-range part."""
    m = moba_mask(lay)
    L = lay.seq_len
    nt = _n_tiles(L, tile)
    out = np.zeros((nt, nt), dtype=np.uint8)
    for i in range(nt):
        for j in range(nt):
            blk = m[i * tile:min((i + 1) * tile, L), j * tile:min((j + 1) * tile, L)]
            out[i, j] = TILE_FULL if blk.all() else (TILE_PARTIAL if blk.any() else TILE_EMPTY)
    return out


def classify_tiles_blocks(lay: MobaLayout, tile: int = 128) -> np.ndarray:
    """Tile classes by reducing the rule over the distinct chunks each tile spans.

    Because the rule is constant on every (query chunk, key chunk) pair, the
    tile's class is decided by the pairs of chunks that occur in it.  Works at
    full size (no [L, L] matrix).
    """
    L = lay.seq_len
    nt = _n_tiles(L, tile)
    # distinct (kind, idx) chunk ids per tile
    spans = []
    for i in range(nt):
        pos = np.arange(i * tile, min((i + 1) * tile, L))
        kind, idx = block_of(pos, lay)
        ids = sorted(set(zip(kind.tolist(), idx.tolist())))
        # a representative position of each distinct chunk
        reps = [int(pos[np.nonzero((kind == a) & (idx == b))[0][0]]) for a, b in ids]
        spans.append(np.array(reps, dtype=np.int64))
    # all key-side representatives in one array, with the tile each belongs to
    krep = np.concatenate(spans)
    starts = np.cumsum([0] + [len(sp) for sp in spans[:-1]])
    out = np.zeros((nt, nt), dtype=np.uint8)
    for i in range(nt):
        a = moba_allowed(spans[i][:, None], krep[None, :], lay)     # [rows reps, all key reps]
        n_ok = np.add.reduceat(a.sum(axis=0), starts)                # allowed pairs per key tile
        n_all = len(spans[i]) * np.diff(np.append(starts, krep.size))
        out[i] = np.where(n_ok == n_all, TILE_FULL, np.where(n_ok > 0, TILE_PARTIAL, TILE_EMPTY))
    return out


def moba_attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, lay: MobaLayout,
                        rows: Iterable[int], scale: float):
    """Masked attention of the listed query rows: ([n, H, D] O, [H, n] LSE)."""
    rows = np.asarray(list(rows), dtype=np.int64)
    kpos = np.arange(lay.seq_len)
    H, D = q.shape[1], q.shape[2]
    o = np.zeros((rows.size, H, v.shape[2]), dtype=np.float64)
    lse = np.full((H, rows.size), -np.inf, dtype=np.float64)
    # rows of the same chunk read the same keys: group them
    kind, idx = block_of(rows, lay)
    groups = {}
    for n, (a, b) in enumerate(zip(kind.tolist(), idx.tolist())):
        groups.setdefault((a, b), []).append(n)
    for members in groups.values():
        rep = rows[members[0]]
        keys = np.nonzero(moba_allowed(rep, kpos, lay))[0]
        if keys.size == 0:
            continue
        sel = rows[members]
        og, lg = attention(q[sel], k[keys], v[keys], scale)
        o[members] = og
        lse[:, members] = lg
    return o, lse
