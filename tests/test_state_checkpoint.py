"""Checkpoint of a cache's host state: export after any schedule of appends and evictions,
import into a fresh cache of the same configuration, and both caches behave identically
from then on; wrong configurations and damaged states are refused with nothing changed."""
import random

import pytest

from kv_cache_chunk_ring_b200 import kvcr
from kv_cache_chunk_ring_b200 import workloads as wl
from oracle.cache import CacheModel


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kv_cache_chunk_ring_b200 import build
    build.build()


def _mk(S=2, W=4, F=3, aux=0, **kw):
    return kvcr.Cache(S, W, 12, 2, 64, F, rope=None, bookkeeping_only=True, aux_frames=aux, **kw)


@pytest.mark.parametrize("seed", range(12))
def test_restored_cache_continues_like_the_original(seed):
    rng = random.Random(seed)
    S, W, F = rng.randint(0, 3), rng.randint(1, 5), rng.randint(1, 4)
    a, ref = _mk(S, W, F), CacheModel(S, W)
    frame = 0

    def step(cache_list, model):
        nonlocal frame
        if rng.random() < 0.3:
            keep = rng.randint(0, W)
            evs = [c.evict(keep) for c in cache_list]
            ev_ref = model.evict(keep)
            assert all(e == ev_ref for e in evs)
        n = rng.randint(1, F)
        frames = list(range(frame, frame + n))
        frame += n + rng.randint(0, 2)
        outs = [c.append(None, None, frames) for c in cache_list]
        slots, ev = model.append(frames)
        for o in outs:
            assert o == (slots, ev)
        maps = [c.slot_map() for c in cache_list]
        assert all(m == model.slot_map() for m in maps)

    for _ in range(rng.randint(0, 12)):
        step([a], ref)
    state = a.export_state()
    b = _mk(S, W, F)
    b.import_state(state)
    assert b.slot_map() == a.slot_map() and b.num_cached() == a.num_cached()
    assert kvcr.kv_cache_last_append(b.handle, F) == kvcr.kv_cache_last_append(a.handle, F)
    assert b.export_state() == state
    for _ in range(10):
        step([a, b], ref)


def test_configuration_mismatch_and_damage_are_refused():
    a = _mk()
    for frames in ([0, 1, 2], [3, 4, 5]):
        a.append(None, None, frames)
    state = a.export_state()
    for other in (_mk(S=3), _mk(W=5), _mk(F=2), _mk(aux=1)):
        before = other.export_state()
        with pytest.raises(kvcr.KvcrError) as e:
            other.import_state(state)
        assert e.value.code == kvcr.KVCR_ESHAPE
        assert other.export_state() == before
    b = _mk()
    before = b.export_state()
    words = len(state) // 4
    damaged = [state[:-4], state + b"\0\0\0\0", b"XXXX" + state[4:]]
    # a cached frame claimed twice; an anchor count beyond the anchors; a broken permutation
    slot0 = 2 + 18                      # magic, version, 18 configuration words
    damaged.append(state[:4 * (slot0 + 1)] + state[4 * slot0:4 * (slot0 + 1)] +
                   state[4 * (slot0 + 2):])
    damaged.append(state[:4 * (slot0 + 6)] + (7).to_bytes(4, "little", signed=True) +
                   state[4 * (slot0 + 7):])
    damaged.append(state[:4 * (slot0 + 9)] + (1).to_bytes(4, "little", signed=True) +
                   state[4 * (slot0 + 10):])        # physical slot 1 twice
    assert words > slot0 + 10
    for d in damaged:
        with pytest.raises(kvcr.KvcrError) as e:
            b.import_state(d)
        assert e.value.code in (kvcr.KVCR_EINVAL, kvcr.KVCR_ESHAPE)
        assert b.export_state() == before


def test_rope_parameters_are_part_of_the_configuration():
    spec = wl.shrink(wl.VIDEO_832x464, grid_h=3, grid_w=4, heads=2, head_dim=64)
    a = kvcr.Cache(2, 2, 12, 2, 64, 2, rope=spec.rope(), bookkeeping_only=True)
    b = kvcr.Cache(2, 2, 12, 2, 64, 2, rope=None, bookkeeping_only=True)
    with pytest.raises(kvcr.KvcrError) as e:
        b.import_state(a.export_state())
    assert e.value.code == kvcr.KVCR_ESHAPE


def test_export_needs_room():
    import ctypes
    a = _mk()
    n = ctypes.c_size_t()
    assert kvcr.lib().kv_cache_export_state(a.handle, None, 0, ctypes.byref(n)) == kvcr.KVCR_OK
    buf = ctypes.create_string_buffer(n.value)
    assert kvcr.lib().kv_cache_export_state(a.handle, buf, n.value - 4,
                                            ctypes.byref(n)) == kvcr.KVCR_ESTORAGE
