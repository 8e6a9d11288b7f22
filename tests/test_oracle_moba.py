"""Pins of the oracle's MoBA mask, tile classes and masked attention."""
import numpy as np
import pytest

from oracle.attn import attention, masked_attention
from oracle.moba import (MobaLayout, moba_mask, moba_allowed, classify_tiles_mask,
                         classify_tiles_blocks, moba_attention_rows, TILE_EMPTY,
                         TILE_PARTIAL, TILE_FULL)

# The rule written out as a table of (query chunk -> key chunks it reads) for
# n = 3 clean/noisy chunks and a 2-chunk bidirectional block, read off the
# statement "Ci attends Cj for j <= i; Ni attends Cj for j < i and attends Ni;
# B attends all of B".
TABLE_N3_M2 = {
    "C1": {"C1"}, "C2": {"C1", "C2"}, "C3": {"C1", "C2", "C3"},
    "N1": {"N1"}, "N2": {"C1", "N2"}, "N3": {"C1", "C2", "N3"},
    "B1": {"B1", "B2"}, "B2": {"B1", "B2"},
}
ORDER = ["C1", "C2", "C3", "N1", "N2", "N3", "B1", "B2"]


def test_rule_table():
    c = 5
    lay = MobaLayout(3, c, 2)
    m = moba_mask(lay)
    for a, qa in enumerate(ORDER):
        for b, kb in enumerate(ORDER):
            blk = m[a * c:(a + 1) * c, b * c:(b + 1) * c]
            expect = kb in TABLE_N3_M2[qa]
            assert blk.all() == expect and blk.any() == expect, (qa, kb)


@pytest.mark.parametrize("n,c,mb", [(1, 4, 1), (2, 3, 1), (8, 2, 8), (5, 7, 3)])
def test_allowed_count_closed_form(n, c, mb):
    # allowed chunk pairs: n(n+1)/2 (clean) + n(n-1)/2 + n (noisy) + mb^2 (bidir)
    lay = MobaLayout(n, c, mb)
    assert int(moba_mask(lay).sum()) == (n * (n + 1) // 2 + n * (n - 1) // 2 + n + mb * mb) * c * c


def test_one_chunk_is_three_full_attentions():
    rng = np.random.default_rng(12)
    c = 6
    lay = MobaLayout(1, c, 1)
    L = lay.seq_len
    q, k, v = (rng.standard_normal((L, 2, 8)) for _ in range(3))
    o, lse = masked_attention(q, k, v, moba_mask(lay), 0.35)
    for blk in range(3):
        s = slice(blk * c, (blk + 1) * c)
        ob, lb = attention(q[s], k[s], v[s], 0.35)
        np.testing.assert_allclose(o[s], ob, atol=1e-13)
        np.testing.assert_allclose(lse[:, s], lb, atol=1e-13)


@pytest.mark.parametrize("n,c,mb,tile", [(2, 5, 1, 4), (3, 7, 2, 4), (4, 3, 2, 8), (2, 16, 2, 16),
                                         (3, 20, 1, 16), (5, 6, 3, 4), (2, 9, 0, 4)])
def test_tile_classes_two_ways(n, c, mb, tile):
    lay = MobaLayout(n, c, mb)
    a = classify_tiles_mask(lay, tile)
    b = classify_tiles_blocks(lay, tile)
    assert np.array_equal(a, b)
    assert set(np.unique(a)) <= {TILE_EMPTY, TILE_PARTIAL, TILE_FULL}


def test_tile_classes_cover_allowed_entries():
    """Allowed entries = entries of full tiles + allowed entries inside partial tiles;
    empty tiles hold none."""
    lay = MobaLayout(4, 11, 2)
    tile = 8
    m = moba_mask(lay)
    cls = classify_tiles_blocks(lay, tile)
    L = lay.seq_len
    total = 0
    for i in range(cls.shape[0]):
        for j in range(cls.shape[1]):
            blk = m[i * tile:min(L, (i + 1) * tile), j * tile:min(L, (j + 1) * tile)]
            if cls[i, j] == TILE_EMPTY:
                assert not blk.any()
            elif cls[i, j] == TILE_FULL:
                assert blk.all()
            total += int(blk.sum())
    assert total == int(m.sum())


def test_rows_match_explicit_mask():
    rng = np.random.default_rng(13)
    lay = MobaLayout(3, 5, 2)
    L = lay.seq_len
    q, k, v = (rng.standard_normal((L, 2, 8)) for _ in range(3))
    rows = [0, 4, 5, 9, 14, 15, 19, 24, 29, 30, 39, L - 1]
    o, lse = moba_attention_rows(q, k, v, lay, rows, 0.3)
    ob, lb = masked_attention(q[rows], k, v, moba_mask(lay)[rows], 0.3)
    np.testing.assert_allclose(o, ob, atol=1e-13)
    np.testing.assert_allclose(lse, lb, atol=1e-13)


def test_clean_chunks_causal():
    """A clean chunk's output does not change when any later part changes."""
    rng = np.random.default_rng(14)
    lay = MobaLayout(3, 4, 1)
    L = lay.seq_len
    q, k, v = (rng.standard_normal((L, 1, 4)) for _ in range(3))
    rows = list(range(0, 8))                  # C1, C2
    o1, _ = moba_attention_rows(q, k, v, lay, rows, 0.5)
    k2, v2 = k.copy(), v.copy()
    k2[8:] = rng.standard_normal(k2[8:].shape)
    v2[8:] = rng.standard_normal(v2[8:].shape)
    o2, _ = moba_attention_rows(q, k2, v2, lay, rows, 0.5)
    assert np.array_equal(o1, o2)


def test_allowed_broadcast_shapes():
    lay = MobaLayout(2, 3, 1)
    assert moba_allowed(np.arange(15)[:, None], np.arange(15)[None, :], lay).shape == (15, 15)


def _tile_counts_by_intervals(n, c, mb, tile=128):
    """Independent count of the tile classes: each query row's readable keys written
    as at most two intervals straight from the rule (C_i: [0, (i+1)c); N_i:
    [0, i c) and [nc + i c, nc + (i+1) c); B: [2nc, L)), overlapped with every key
    tile and summed over the rows of each query tile."""
    nc = n * c
    L = (2 * n + mb) * c
    nt = (L + tile - 1) // tile
    kt0 = np.arange(nt) * tile
    kt1 = np.minimum(kt0 + tile, L)
    counts = {TILE_FULL: 0, TILE_PARTIAL: 0, TILE_EMPTY: 0}
    for qt in range(nt):
        r = np.arange(qt * tile, min((qt + 1) * tile, L))
        i = np.where(r < nc, r // c, np.where(r < 2 * nc, (r - nc) // c, 0))
        lo0 = np.where(r < 2 * nc, 0, 2 * nc)
        hi0 = np.where(r < nc, (i + 1) * c, np.where(r < 2 * nc, i * c, L))
        lo1 = np.where((r >= nc) & (r < 2 * nc), nc + i * c, 0)
        hi1 = np.where((r >= nc) & (r < 2 * nc), nc + (i + 1) * c, 0)
        ov = np.zeros(nt, dtype=np.int64)
        for lo, hi in ((lo0, hi0), (lo1, hi1)):
            a = np.clip(np.minimum(hi[:, None], kt1[None, :]) - np.maximum(lo[:, None], kt0[None, :]),
                        0, None)
            ov += a.sum(axis=0)
        area = r.size * (kt1 - kt0)
        counts[TILE_FULL] += int((ov == area).sum())
        counts[TILE_EMPTY] += int((ov == 0).sum())
        counts[TILE_PARTIAL] += int(((ov > 0) & (ov < area)).sum())
    return counts


@pytest.mark.parametrize("n,c,mb,tile", [(3, 7, 2, 4), (5, 6, 3, 4), (2, 16, 2, 16), (3, 50, 2, 128)])
def test_tile_counts_by_intervals_small(n, c, mb, tile):
    ref = classify_tiles_mask(MobaLayout(n, c, mb), tile)
    got = _tile_counts_by_intervals(n, c, mb, tile)
    assert got == {k: int((ref == k).sum()) for k in (TILE_FULL, TILE_PARTIAL, TILE_EMPTY)}


def test_training_sequence_tile_counts():
    """The 144768-token training sequence (8 clean + 8 noisy chunks of 6032 tokens and an
    8-chunk bidirectional block) has 1131 x 1131 tiles of 128: 300713 full, 2629 partial
    and 975819 empty, counted from the row intervals and by the oracle's chunk-pair
    reduction."""
    expect = {TILE_FULL: 300713, TILE_PARTIAL: 2629, TILE_EMPTY: 975819}
    assert sum(expect.values()) == 1131 * 1131
    assert _tile_counts_by_intervals(8, 6032, 8) == expect
    cls = classify_tiles_blocks(MobaLayout(8, 6032, 8), 128)
    assert {k: int((cls == k).sum()) for k in expect} == expect
