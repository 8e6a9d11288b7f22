"""Pins of the oracle rollout's auxiliary frames (temporary evidence blocks read by
one chunk and dropped when it is finalized)."""
import math

import numpy as np

from kv_cache_chunk_ring_b200 import workloads as wl
from oracle.rollout import rollout
from oracle.rope import rope3d, rope_positions

SPEC = wl.TINY_F32   # 1 head, d64, 4 x 4 tokens per frame, 2 anchors + 2 window, 2 frames/chunk


def _items():
    return list(wl.rollout_chunks(SPEC))


def test_no_aux_is_the_plain_rollout():
    items = _items()
    a = rollout(SPEC, items)
    b = rollout(SPEC, items, aux_for=lambda c: (np.zeros((0, 1, 64)), np.zeros((0, 1, 64)), []))
    for x, y in zip(a.outputs, b.outputs):
        assert np.array_equal(x, y)


def test_copies_of_every_visible_frame_double_each_key():
    """Auxiliary copies of all visible frames (raw K at their own positions, V) make
    every key appear twice: O unchanged, LSE + ln 2."""
    items = _items()
    T = SPEC.tokens_per_frame
    plain = rollout(SPEC, items)
    raw = {}                                   # frame -> raw (K, V) of its finalized step
    for it in items:
        for n, f in enumerate(it["frames"]):
            raw[f] = (it["k"][n * T:(n + 1) * T], it["v"][n * T:(n + 1) * T])

    def aux_for(c):
        frames = plain.visible[c] + list(SPEC.frames_of_chunk(c))
        return (np.concatenate([raw[f][0] for f in frames]),
                np.concatenate([raw[f][1] for f in frames]), frames)
    dup = rollout(SPEC, items, aux_for=aux_for)
    for c in range(SPEC.n_chunks):
        np.testing.assert_allclose(dup.outputs[c], plain.outputs[c], atol=1e-12)
        np.testing.assert_allclose(dup.lses[c], plain.lses[c] + math.log(2.0), atol=1e-12)


def test_aux_changes_only_its_own_chunk():
    items = _items()
    plain = rollout(SPEC, items)
    k, v, pos = wl.aux_frames(SPEC, 3, 2)
    one = rollout(SPEC, items, aux_for=lambda c: (k, v, pos) if c == 3 else None)
    for c in range(SPEC.n_chunks):
        same = np.array_equal(one.outputs[c], plain.outputs[c])
        assert same == (c != 3), c
    assert one.slot_maps == plain.slot_maps


def test_prerotated_aux_without_positions():
    items = _items()
    k, v, pos = wl.aux_frames(SPEC, 2, 2)
    t, h, w = rope_positions(pos, SPEC.grid_h, SPEC.grid_w)
    r = SPEC.rope()
    k_rot = rope3d(np.asarray(k, np.float64), t, h, w, (r.pairs_t, r.pairs_h, r.pairs_w), r.base)
    a = rollout(SPEC, items, aux_for=lambda c: (k, v, pos) if c == 2 else None)
    b = rollout(SPEC, items, aux_for=lambda c: (k_rot, v, None) if c == 2 else None)
    np.testing.assert_allclose(a.outputs[2], b.outputs[2], atol=1e-12)


def test_aux_is_plain_attention_over_the_extra_keys():
    """One query row, brute force: softmax over [cached, aux, current] keys by a scalar loop."""
    items = _items()
    k, v, pos = wl.aux_frames(SPEC, 4, 1)
    res = rollout(SPEC, items, aux_for=lambda c: (k, v, pos) if c == 4 else None,
                  rows_for=lambda c, s: [5])
    plain = rollout(SPEC, items)
    r = SPEC.rope()
    pairs = (r.pairs_t, r.pairs_h, r.pairs_w)
    T = SPEC.tokens_per_frame
    it = items[4]
    t, h, w = rope_positions(it["frames"], SPEC.grid_h, SPEC.grid_w)
    q = rope3d(np.asarray(it["q"], np.float64), t, h, w, pairs, r.base)[5, 0]
    keys, vals = [], []
    for f in plain.visible[4]:
        src = next(x for x in items if f in x["frames"])
        n = src["frames"].index(f)
        tt, hh, ww = rope_positions([f], SPEC.grid_h, SPEC.grid_w)
        keys.append(rope3d(np.asarray(src["k"][n * T:(n + 1) * T], np.float64), tt, hh, ww,
                           pairs, r.base)[:, 0])
        vals.append(np.asarray(src["v"][n * T:(n + 1) * T], np.float64)[:, 0])
    ta, ha, wa = rope_positions(pos, SPEC.grid_h, SPEC.grid_w)
    keys.append(rope3d(np.asarray(k, np.float64), ta, ha, wa, pairs, r.base)[:, 0])
    vals.append(np.asarray(v, np.float64)[:, 0])
    keys.append(rope3d(np.asarray(it["k"], np.float64), t, h, w, pairs, r.base)[:, 0])
    vals.append(np.asarray(it["v"], np.float64)[:, 0])
    K = np.concatenate(keys)
    V = np.concatenate(vals)
    z = [float(q @ K[j]) / math.sqrt(64) for j in range(K.shape[0])]
    m = max(z)
    e = [math.exp(x - m) for x in z]
    o = sum(e[j] * V[j] for j in range(len(e))) / sum(e)
    np.testing.assert_allclose(res.outputs[4][0, 0], o, atol=1e-12)
