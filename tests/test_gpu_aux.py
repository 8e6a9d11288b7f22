"""GPU parity of chunk attention with auxiliary frames (temporary evidence blocks
read by the current chunk and dropped when it is finalized) against the oracle."""
import math

import numpy as np
import pytest

from kv_cache_chunk_ring_b200 import workloads as wl
from oracle.rollout import rollout
from tests.gpu_helpers import TOL_LSE, assert_close, gpu_rollout, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_chunk_ring_b200 import build
    build.build()


def _aux_for(spec, n, skip=()):
    def f(c):
        if c in skip or n == 0:
            return None
        return wl.aux_frames(spec, c, n)
    return f


@pytest.mark.parametrize("spec,n_aux", [
    (wl.shrink(wl.VIDEO_832x464, grid_h=8, grid_w=16, heads=2, chunk_frames=2, sinks=1, window=2,
               n_chunks=5, seed=51), 2),
    (wl.shrink(wl.VIDEO_832x464, grid_h=5, grid_w=9, heads=2, head_dim=64, chunk_frames=3,
               sinks=2, window=3, n_chunks=4, seed=52), 3),
    (wl.TINY_F32, 2),
])
def test_rollout_with_aux_frames(spec, n_aux):
    items = list(wl.rollout_chunks(spec))
    aux_for = _aux_for(spec, n_aux, skip=(0,))
    ref = rollout(spec, items, aux_for=aux_for)
    got = gpu_rollout(spec, items, aux_for=aux_for, aux_frames=n_aux)
    for i, (o, r) in enumerate(zip(got["outputs"], ref.outputs)):
        assert_close(o, r, f"call {i}")
        assert np.abs(got["lses"][i] - ref.lses[i]).max() <= TOL_LSE
    assert got["slot_maps"] == ref.slot_maps
    assert got["cache"].num_aux() == 0           # dropped by the last append


def test_copies_of_every_visible_frame_add_ln2():
    """Auxiliary copies (raw K at their own positions, V) of every frame the chunk reads:
    O unchanged, LSE + ln 2, on the GPU."""
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    spec = wl.shrink(wl.VIDEO_832x464, grid_h=8, grid_w=16, heads=2, chunk_frames=2, sinks=1,
                     window=2, n_chunks=4, seed=53)
    T, F = spec.tokens_per_frame, spec.chunk_frames
    items = list(wl.rollout_chunks(spec))
    cache = kvcr.Cache(spec.sinks, spec.window, T, spec.heads, spec.head_dim, F,
                       rope=spec.rope(), aux_frames=spec.sinks + spec.window + F)
    raw = {}
    for it in items[:3]:
        cache.append(to_dev(it["k"], "bf16"), to_dev(it["v"], "bf16"), it["frames"])
        for n, f in enumerate(it["frames"]):
            raw[f] = (it["k"][n * T:(n + 1) * T], it["v"][n * T:(n + 1) * T])
    it = items[3]
    q, k, v = (to_dev(it[x], "bf16") for x in ("q", "k", "v"))
    o0, l0 = cache.attention(q, k, v, it["frames"], want_lse=True)
    vis = [f for f in cache.slot_map() if f >= 0]
    for n, f in enumerate(it["frames"]):
        raw[f] = (it["k"][n * T:(n + 1) * T], it["v"][n * T:(n + 1) * T])
    frames = sorted(vis) + list(it["frames"])
    cache.set_aux(to_dev(np.concatenate([raw[f][0] for f in frames]), "bf16"),
                  to_dev(np.concatenate([raw[f][1] for f in frames]), "bf16"), frames)
    o1, l1 = cache.attention(q, k, v, it["frames"], want_lse=True)
    torch.cuda.synchronize()
    assert_close(to_np(o1), to_np(o0), "duplicated keys")
    assert np.abs(l1.cpu().numpy() - l0.cpu().numpy() - math.log(2.0)).max() <= TOL_LSE


def test_full_size_832x464_with_four_aux_frames():
    """6 anchors + 8 window + 4 auxiliary frames (33176 keys per steady-state call)."""
    spec = wl.shrink(wl.VIDEO_832x464, n_chunks=6)
    items = list(wl.rollout_chunks(spec))
    aux_for = _aux_for(spec, 4, skip=(0, 1, 2))
    rows = wl.sample_rows(spec.chunk_tokens, 192, 1020, list(range(64)))
    rows_for = lambda c, s: rows
    ref = rollout(spec, items, rows_for=rows_for, aux_for=aux_for)
    got = gpu_rollout(spec, items, rows_for=rows_for, aux_for=aux_for, aux_frames=4)
    for i, (o, r) in enumerate(zip(got["outputs"], ref.outputs)):
        assert_close(o, r, f"call {i}")
        assert np.abs(got["lses"][i] - ref.lses[i]).max() <= TOL_LSE
    assert got["slot_maps"] == ref.slot_maps
    assert ref.n_keys[5] == 27144 + 4 * spec.tokens_per_frame


def test_static_scratch_entry_reads_the_aux_frames():
    """The allocation-free entry point reads the same visible slots (auxiliary ones
    included) as chunk_attention_fwd: bit-identical outputs."""
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    spec = wl.shrink(wl.VIDEO_832x464, grid_h=8, grid_w=16, heads=2, chunk_frames=2, sinks=1,
                     window=2, n_chunks=4, seed=54)
    T, F = spec.tokens_per_frame, spec.chunk_frames
    items = list(wl.rollout_chunks(spec))
    cache = kvcr.Cache(spec.sinks, spec.window, T, spec.heads, spec.head_dim, F,
                       rope=spec.rope(), aux_frames=3)
    for it in items[:3]:
        cache.append(to_dev(it["k"], "bf16"), to_dev(it["v"], "bf16"), it["frames"])
    k_aux, v_aux, pos = wl.aux_frames(spec, 3, 3)
    cache.set_aux(to_dev(k_aux, "bf16"), to_dev(v_aux, "bf16"), pos)
    it = items[3]
    q, k, v = (to_dev(it[x], "bf16") for x in ("q", "k", "v"))
    o1, l1 = cache.attention(q, k, v, it["frames"], want_lse=True)
    o2 = torch.empty_like(q)
    l2 = torch.empty_like(l1)
    kvcr.chunk_attention_fwd_static_scratch(cache.handle, q, k, v, it["frames"], o2, l2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
