"""Pins of the oracle's rollout against brute-force attention over the whole
concatenated rollout with an explicit visibility mask built from the set-based
rule, and causality properties."""
import math

import numpy as np

from kv_cache_chunk_ring_b200 import workloads as wl
from oracle.attn import masked_attention, attention
from oracle.cache import visible_frames_closed_form
from oracle.rollout import rollout
from oracle.rope import rope3d, rope_positions


def _brute(spec, chunks, schedule=None):
    T = spec.tokens_per_frame
    F = spec.chunk_frames
    last = [c for c in chunks if c["step"] == spec.steps - 1]
    pairs = (spec.rope().pairs_t, spec.rope().pairs_h, spec.rope().pairs_w)
    ks, vs = [], []
    for c in last:
        t, h, w = rope_positions(c["frames"], spec.grid_h, spec.grid_w)
        ks.append(rope3d(c["k"], t, h, w, pairs))
        vs.append(np.asarray(c["v"], np.float64))
    K, V = np.concatenate(ks), np.concatenate(vs)
    outs = []
    for c in chunks:
        ch = c["chunk"]
        f0 = ch * F
        t, h, w = rope_positions(c["frames"], spec.grid_h, spec.grid_w)
        q = rope3d(c["q"], t, h, w, pairs)
        kc = rope3d(c["k"], t, h, w, pairs)
        vc = np.asarray(c["v"], np.float64)
        W = spec.window if schedule is None else schedule[ch]
        vis = visible_frames_closed_form(f0, spec.sinks, W)
        allowed_frames = np.zeros(K.shape[0] // T, dtype=bool)
        allowed_frames[vis] = True
        # keys: [all finalized frames ..., current chunk's own (this step's) K/V]
        keys_k = np.concatenate([K, kc])
        keys_v = np.concatenate([V, vc])
        allowed = np.concatenate([np.repeat(allowed_frames, T), np.ones(F * T, bool)])
        allowed = np.broadcast_to(allowed, (q.shape[0], allowed.size))
        o, lse = masked_attention(q, keys_k, keys_v, allowed, 1 / math.sqrt(spec.head_dim))
        outs.append((o, lse))
    return outs


def test_tiny_rollout_equals_bruteforce():
    spec = wl.shrink(wl.TINY_F32, grid_h=2, grid_w=3, n_chunks=6)
    chunks = list(wl.rollout_chunks(spec))
    res = rollout(spec, chunks)
    ref = _brute(spec, chunks)
    for (o, lse), o2, l2 in zip(ref, res.outputs, res.lses):
        np.testing.assert_allclose(o2, o, atol=1e-12)
        np.testing.assert_allclose(l2, lse, atol=1e-12)
    assert res.n_keys == [12, 24, 36, 36, 36, 36]


def test_multi_step_uses_last_step_kv():
    spec = wl.shrink(wl.TINY_F32, grid_h=2, grid_w=2, n_chunks=4, steps=3, sinks=1, window=2)
    chunks = list(wl.rollout_chunks(spec))
    res = rollout(spec, chunks)
    ref = _brute(spec, chunks)
    for (o, lse), o2 in zip(ref, res.outputs):
        np.testing.assert_allclose(o2, o, atol=1e-12)


def test_dynamic_window_equals_bruteforce():
    spec = wl.shrink(wl.VIDEO_720P_DYN, heads=2, head_dim=16, grid_h=2, grid_w=2, n_chunks=12,
                     dtype="f32", text_env=0, text_local=0)
    sched = spec.window_schedule()
    chunks = list(wl.rollout_chunks(spec))
    res = rollout(spec, chunks, window_schedule=sched)
    ref = _brute(spec, chunks, sched)
    for (o, lse), o2 in zip(ref, res.outputs):
        np.testing.assert_allclose(o2, o, atol=1e-12)
    for ch, vis in enumerate(res.visible):
        assert vis == visible_frames_closed_form(ch * spec.chunk_frames, spec.sinks, sched[ch])


def test_chunk_output_unchanged_by_later_chunks():
    spec = wl.shrink(wl.TINY_F32, grid_h=2, grid_w=2, n_chunks=5)
    chunks = list(wl.rollout_chunks(spec))
    res1 = rollout(spec, chunks)
    rng = np.random.default_rng(99)
    chunks2 = [dict(c) for c in chunks]
    for c in chunks2[3:]:
        for key in ("q", "k", "v"):
            c[key] = rng.standard_normal(c[key].shape).astype(np.float32)
    res2 = rollout(spec, chunks2)
    for a, b in zip(res1.outputs[:3], res2.outputs[:3]):
        assert np.array_equal(a, b)


def test_window_schedule_seeded_range():
    s = wl.VIDEO_720P_DYN.window_schedule()
    assert len(s) == 60 and min(s) >= 2 and max(s) <= 8
    assert s == wl.VIDEO_720P_DYN.window_schedule()


def test_cross_attention_reads_env_and_own_prompt_only():
    """Causal chunk-wise cross-attention: a chunk reads the shared env prompt and
    its own local prompt; changing a future chunk's prompt changes nothing."""
    rng = np.random.default_rng(15)
    env_k, env_v = rng.standard_normal((4, 1, 8)), rng.standard_normal((4, 1, 8))
    loc = [(rng.standard_normal((3, 1, 8)), rng.standard_normal((3, 1, 8))) for _ in range(3)]
    q = rng.standard_normal((5, 1, 8))
    allk = np.concatenate([env_k] + [k for k, _ in loc])
    allv = np.concatenate([env_v] + [v for _, v in loc])
    for t in range(3):
        allowed = np.zeros((5, allk.shape[0]), bool)
        allowed[:, :4] = True
        allowed[:, 4 + 3 * t:4 + 3 * (t + 1)] = True
        ob, _ = masked_attention(q, allk, allv, allowed, 0.3)
        o, _ = attention(q, np.concatenate([env_k, loc[t][0]]), np.concatenate([env_v, loc[t][1]]), 0.3)
        np.testing.assert_allclose(o, ob, atol=1e-13)


def test_checked_rows_equal_the_full_rollout_rows():
    """Evaluating a subset of query rows gives those rows of the full rollout, up to the
    order of fp64 rounding inside the library matmul (RoPE turns each token by its own
    position; attention is row by row)."""
    spec = wl.shrink(wl.VIDEO_832x464, grid_h=3, grid_w=5, heads=2, head_dim=64, chunk_frames=2,
                     sinks=1, window=2, n_chunks=4, seed=41)
    items = list(wl.rollout_chunks(spec))
    full = rollout(spec, items)
    pick = {c: np.array(sorted({0, 7, 29, c + 3})) for c in range(spec.n_chunks)}
    part = rollout(spec, items, rows_for=lambda c, s: pick[c])
    for n, it in enumerate(items):
        rows = pick[it["chunk"]]
        np.testing.assert_allclose(part.outputs[n], full.outputs[n][rows], rtol=0, atol=1e-13)
        np.testing.assert_allclose(part.lses[n], full.lses[n][:, rows], rtol=0, atol=1e-13)
    assert part.slot_maps == full.slot_maps
