"""Pins of the oracle's cache bookkeeping: worked examples, closed forms, invariants."""
import os

import numpy as np
import pytest

from oracle.cache import CacheModel, visible_frames_closed_form

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _read(name):
    out = []
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        cols = [c.strip() for c in line.split("|")]
        ints = lambda s: [] if s == "-" else [int(x) for x in s.split()]  # noqa: E731
        out.append(dict(chunk=int(cols[0]), frames=ints(cols[1]), slots=ints(cols[2]),
                        evicted=ints(cols[3]), slot_map=ints(cols[4]), keys=int(cols[5])))
    return out


@pytest.mark.parametrize("name,S,W,F,T", [
    ("slot_map_2anchor_2window.txt", 2, 2, 2, 16),
    ("slot_map_6anchor_8window.txt", 6, 8, 4, 1508),
])
def test_worked_examples(name, S, W, F, T):
    c = CacheModel(S, W)
    for row in _read(name):
        keys = (c.n_cached() + F) * T
        assert keys == row["keys"]
        slots, ev = c.append(row["frames"])
        assert slots == row["slots"]
        assert ev == row["evicted"]
        assert c.slot_map() == row["slot_map"]


@pytest.mark.parametrize("S,W,F", [(2, 2, 2), (6, 8, 4), (0, 3, 1), (3, 0, 2), (1, 5, 3), (6, 8, 5)])
def test_static_window_ring_closed_form(S, W, F):
    """Static window: frame f sits in slot f if f < S, else S + ((f - S) mod W)."""
    c = CacheModel(S, W)
    for chunk in range(20):
        frames = list(range(chunk * F, (chunk + 1) * F))
        slots, _ = c.append(frames)
        for f, s in zip(frames, slots):
            if f < S:
                assert s == f
            elif W == 0:
                assert s == -1
            else:
                assert s == S + (f - S) % W


@pytest.mark.parametrize("S,W,F", [(2, 2, 2), (6, 8, 4), (0, 4, 3), (4, 0, 2), (3, 5, 4)])
def test_visible_set_closed_form(S, W, F):
    c = CacheModel(S, W)
    for chunk in range(15):
        f0 = chunk * F
        assert c.cached_frames() == visible_frames_closed_form(f0, S, W)
        c.append(range(f0, f0 + F))


def test_invariants_dynamic():
    rng = np.random.default_rng(11)
    S, Wmax, F = 6, 8, 4
    c = CacheModel(S, Wmax)
    f = 0
    all_evicted = []
    for chunk in range(60):
        keep = int(rng.integers(2, 9))
        before = c.cached_frames()
        ev = c.evict(keep)
        all_evicted += ev
        # evicted = oldest non-anchor frames
        non_anchor = [x for x in before if x >= S]
        assert ev == non_anchor[:max(0, len(non_anchor) - keep)]
        assert len([x for x in c.cached_frames() if x >= S]) <= keep
        slots, ev2 = c.append(range(f, f + F))
        all_evicted += ev2
        f += F
        cached = c.cached_frames()
        # anchors never evicted, at most S + W frames, no duplicates
        assert all(a in cached for a in range(min(S, f)))
        assert not any(a < S for a in all_evicted)
        assert len(cached) <= S + Wmax
        sm = [x for x in c.slot_map() if x >= 0]
        assert len(sm) == len(set(sm))
        # the newest min(F, Wmax) frames are cached
        assert all(x in cached for x in range(f - min(F, Wmax), f))


def test_errors():
    c = CacheModel(2, 2)
    c.append([0, 1])
    with pytest.raises(ValueError):
        c.append([1])
    with pytest.raises(ValueError):
        c.evict(3)
    with pytest.raises(ValueError):
        CacheModel(0, 0)
