"""CPU tests of the C-ABI library: it loads, exports every declared symbol, and its
host bookkeeping / tile classification match the oracle bit-exactly.  No kernel
runs here (bookkeeping-only caches; classification is host code)."""
import os
import re

import numpy as np
import pytest

from kv_cache_chunk_ring_b200 import kvcr
from kv_cache_chunk_ring_b200 import workloads as wl
from oracle.cache import CacheModel
from oracle.moba import MobaLayout, classify_tiles_blocks, classify_tiles_mask

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from kv_cache_chunk_ring_b200 import build
    build.build()


def _declared():
    text = open(os.path.join(ROOT, "include", "kvcr.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?(?:int|void|size_t|long long|char)\s*\**\s*(\w+)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_header_declares_bound_symbols():
    assert sorted(kvcr.EXPORTS) == _declared()


def test_library_exports_every_declared_symbol():
    L = kvcr.lib()
    for name in _declared():
        assert hasattr(L, name), name


def _bk_cache(S, W, T=4, H=1, D=64, F=4):
    return kvcr.kv_cache_init(S, W, T, H, D, F, None, kvcr.KVCR_BF16, None)


@pytest.mark.parametrize("spec", wl.ALL_ROLLOUTS, ids=lambda s: s.name)
def test_bookkeeping_matches_oracle(spec):
    sched = spec.window_schedule() if spec.window_seed is not None else None
    cap = spec.window
    h = _bk_cache(spec.sinks, cap, spec.tokens_per_frame, spec.heads, spec.head_dim,
                  spec.chunk_frames)
    ref = CacheModel(spec.sinks, cap)
    try:
        for c in range(spec.n_chunks):
            if sched is not None:
                ev_ref = ref.evict(sched[c])
                assert kvcr.kv_cache_evict(h, sched[c]) == ev_ref
            frames = spec.frames_of_chunk(c)
            slots_ref, evicted_ref = ref.append(frames)
            kvcr.kv_cache_append_rope(h, None, None, frames)
            slots, evicted = kvcr.kv_cache_last_append(h, len(frames))
            assert slots == slots_ref
            assert evicted == evicted_ref
            assert kvcr.kv_cache_slot_map(h, spec.sinks + cap) == ref.slot_map()
            assert kvcr.kv_cache_num_cached(h) == ref.n_cached()
    finally:
        kvcr.kv_cache_destroy(h)


def test_random_schedules_match_oracle():
    rng = np.random.default_rng(21)
    for trial in range(40):
        S = int(rng.integers(0, 5))
        W = int(rng.integers(0 if S > 0 else 1, 9))
        F = int(rng.integers(1, 6))
        h = _bk_cache(S, W, F=F)
        ref = CacheModel(S, W)
        f = int(rng.integers(0, 3))
        for step in range(25):
            if W > 0 and rng.random() < 0.3:
                keep = int(rng.integers(0, W + 1))
                assert kvcr.kv_cache_evict(h, keep) == ref.evict(keep)
            n = int(rng.integers(0, F + 1))
            frames = []
            for _ in range(n):
                f += int(rng.integers(1, 3))
                frames.append(f)
            if not frames:
                continue
            s_ref, e_ref = ref.append(frames)
            kvcr.kv_cache_append_rope(h, None, None, frames)
            assert kvcr.kv_cache_last_append(h, n) == (s_ref, e_ref)
            assert kvcr.kv_cache_slot_map(h, S + W) == ref.slot_map()
        kvcr.kv_cache_destroy(h)


def test_errors_leave_state_unchanged():
    h = _bk_cache(2, 2, F=2)
    kvcr.kv_cache_append_rope(h, None, None, [0, 1])
    before = kvcr.kv_cache_slot_map(h, 4)
    with pytest.raises(kvcr.KvcrError) as e:
        kvcr.kv_cache_append_rope(h, None, None, [1, 2])       # not increasing
    assert e.value.code == kvcr.KVCR_ESTATE
    with pytest.raises(kvcr.KvcrError) as e:
        kvcr.kv_cache_append_rope(h, None, None, [5, 4])
    assert e.value.code == kvcr.KVCR_ESTATE
    assert kvcr.kv_cache_slot_map(h, 4) == before
    with pytest.raises(kvcr.KvcrError) as e:
        kvcr.kv_cache_evict(h, 3)
    assert e.value.code == kvcr.KVCR_EINVAL
    with pytest.raises(kvcr.KvcrError) as e:      # attention needs device storage
        kvcr.lib()
        rc = kvcr.lib().chunk_attention_fwd(h, None, 8, None, None, kvcr._i32([7]), 1, 0.0, None,
                                            None, None)
        kvcr._check(rc)
    assert e.value.code == kvcr.KVCR_ESTATE
    kvcr.kv_cache_destroy(h)


def test_init_validation():
    for args, code in [((0, 0), kvcr.KVCR_ESHAPE), ((20, 13), kvcr.KVCR_ESHAPE)]:
        with pytest.raises(kvcr.KvcrError) as e:
            _bk_cache(*args)
        assert e.value.code == code
    with pytest.raises(kvcr.KvcrError) as e:
        kvcr.kv_cache_init(2, 2, 4, 1, 96, 2, None, kvcr.KVCR_BF16, None)
    assert e.value.code == kvcr.KVCR_EUNSUPPORTED
    bad = wl.RopeSpec(2, 3, 10, 10, 10)   # grid 2x3 != 4 tokens
    with pytest.raises(kvcr.KvcrError) as e:
        kvcr.kv_cache_init(2, 2, 4, 1, 64, 2, bad, kvcr.KVCR_BF16, None)
    assert e.value.code == kvcr.KVCR_ESHAPE
    assert kvcr.kv_cache_storage_bytes(0, 0, 4, 1, 64, 2, False, kvcr.KVCR_BF16) == 0


def test_storage_bytes_cover_slots_and_scratch():
    T, H, D, S, W, F = 1508, 12, 128, 6, 8, 4
    frame = T * H * D * 2
    n = kvcr.kv_cache_storage_bytes(S, W, T, H, D, F, True, kvcr.KVCR_BF16)
    assert n >= 2 * (S + W) * frame + 2 * F * frame
    assert n < 2 * (S + W) * frame + 2 * F * frame + 4 * T * D * 8 + 4096


@pytest.mark.parametrize("n,c,m,tile", [(2, 5, 1, 4), (3, 7, 2, 4), (4, 3, 2, 8), (2, 16, 2, 16),
                                        (3, 20, 1, 16), (5, 6, 3, 4), (2, 9, 0, 4), (3, 50, 2, 128),
                                        (4, 200, 3, 128)])
def test_classify_tiles_small_match_oracle(n, c, m, tile):
    got = kvcr.moba_classify_tiles(n, c, m, tile)
    ref = classify_tiles_mask(MobaLayout(n, c, m), tile)
    assert np.array_equal(got, ref)


def test_classify_tiles_full_size_matches_oracle():
    spec = wl.MOBA_8x6032
    got = kvcr.moba_classify_tiles(spec.n_chunks, spec.chunk_tokens, spec.n_bidir_chunks, 128)
    ref = classify_tiles_blocks(MobaLayout(spec.n_chunks, spec.chunk_tokens, spec.n_bidir_chunks), 128)
    assert got.shape == (1131, 1131)
    assert np.array_equal(got, ref)


def test_moba_bwd_workspace_bytes():
    # 8 bytes per (head, row), rows rounded up to a multiple of 128
    assert kvcr.moba_attention_bwd_workspace_bytes(2, 200, 1, 3) == 3 * 1024 * 8   # L = 1000
    assert kvcr.moba_attention_bwd_workspace_bytes(8, 6032, 8, 12) == 12 * 1131 * 128 * 8
    assert kvcr.moba_attention_bwd_workspace_bytes(0, 200, 1, 3) == 0
    assert kvcr.moba_attention_bwd_workspace_bytes(2, 200, 1, 0) == 0


def test_moba_bwd_rejects_bad_arguments_before_launch():
    import ctypes
    L = kvcr.lib()
    lay = kvcr.kvcr_moba_layout(2, 200, 1)
    p = ctypes.c_void_p(1 << 20)                     # aligned, never dereferenced
    args = lambda **kw: [kw.get(n, p) for n in ("q", "k", "v", "o", "do", "lse")]
    call = lambda *a, dtype=kvcr.KVCR_BF16, hd=128, ws_bytes=1 << 30, ws=p, dq=p: \
        L.moba_attention_bwd(*a, ctypes.byref(lay), 2, hd, dtype, 0.0, dq, p, p, ws, ws_bytes,
                             None)
    assert call(*args(), dtype=kvcr.KVCR_F32) == kvcr.KVCR_EUNSUPPORTED
    assert call(*args(), hd=96) == kvcr.KVCR_EUNSUPPORTED
    assert call(*args(q=None)) == kvcr.KVCR_EINVAL
    assert call(*args(), dq=None) == kvcr.KVCR_EINVAL
    assert call(*args(k=ctypes.c_void_p((1 << 20) + 8))) == kvcr.KVCR_EINVAL
    assert call(*args(), ws_bytes=16) == kvcr.KVCR_ESTORAGE
    bad = kvcr.kvcr_moba_layout(0, 200, 1)
    assert L.moba_attention_bwd(p, p, p, p, p, p, ctypes.byref(bad), 2, 128, kvcr.KVCR_BF16, 0.0,
                                p, p, p, p, 1 << 30, None) == kvcr.KVCR_ESHAPE


def test_aux_slots_bookkeeping():
    """Auxiliary frames are visible until the chunk's append drops them; they never
    touch the anchor / window slot table."""
    c = kvcr.Cache(2, 2, 16, 1, 64, 2, dtype="f32", bookkeeping_only=True, aux_frames=3)
    ref = kvcr.Cache(2, 2, 16, 1, 64, 2, dtype="f32", bookkeeping_only=True)
    assert c.num_aux() == 0
    for ch in range(5):
        frames = [2 * ch, 2 * ch + 1]
        n = ch % 4
        if n <= 3:
            c.set_aux(None, None, positions=list(range(n)))
            assert c.num_aux() == n
        c.append(None, None, frames)
        ref.append(None, None, frames)
        assert c.num_aux() == 0
        assert c.slot_map() == ref.slot_map()
    with pytest.raises(kvcr.KvcrError) as e:
        c.set_aux(None, None, positions=[0, 1, 2, 3])        # more than aux_frames
    assert e.value.code == kvcr.KVCR_ESHAPE
    assert c.num_aux() == 0
    with pytest.raises(kvcr.KvcrError) as e:
        c.set_aux(None, None, positions=[0, -1])
    assert e.value.code == kvcr.KVCR_EINVAL
    c.set_aux(None, None, positions=[4, 5])
    c.set_aux(None, None, positions=[])                        # n = 0 drops them now
    assert c.num_aux() == 0


def test_aux_storage_bytes():
    T, H, D, F = 1508, 12, 128, 4
    base = kvcr.kv_cache_storage_bytes(6, 8, T, H, D, F, True, "bf16")
    assert kvcr.kv_cache_storage_bytes_aux(6, 8, 0, T, H, D, F, True, "bf16") == base
    frame = T * H * D * 2
    grown = kvcr.kv_cache_storage_bytes_aux(6, 8, 4, T, H, D, F, True, "bf16")
    assert base + 2 * 4 * frame <= grown <= base + 2 * 4 * frame + 2 * 256
    assert kvcr.kv_cache_storage_bytes_aux(6, 8, 19, T, H, D, F, True, "bf16") == 0  # > 32 slots


def test_batched_append_bookkeeping_matches_single_appends():
    caches = [kvcr.Cache(2, 3, 16, 1, 64, 2, dtype="f32", bookkeeping_only=True) for _ in range(3)]
    twins = [kvcr.Cache(2, 3, 16, 1, 64, 2, dtype="f32", bookkeeping_only=True) for _ in range(3)]
    caches[1].append(None, None, [0])
    twins[1].append(None, None, [0])
    for ch in range(1, 7):
        frames = [2 * ch, 2 * ch + 1]
        if ch == 4:
            caches[2].evict(1)
            twins[2].evict(1)
        kvcr.append_batch(caches, None, None, frames)
        for c, t in zip(caches, twins):
            t.append(None, None, frames)
            assert c.slot_map() == t.slot_map()
            assert kvcr.kv_cache_last_append(c.handle, 2) == kvcr.kv_cache_last_append(t.handle, 2)


def test_batched_append_rejects_before_changing_anything():
    a = kvcr.Cache(2, 2, 16, 1, 64, 2, dtype="f32", bookkeeping_only=True)
    b = kvcr.Cache(2, 2, 16, 1, 64, 2, dtype="f32", bookkeeping_only=True)
    other = kvcr.Cache(2, 2, 25, 1, 64, 2, dtype="f32", bookkeeping_only=True)
    b.append(None, None, [0, 1, 2])
    before = (a.slot_map(), b.slot_map())
    with pytest.raises(kvcr.KvcrError) as e:          # b already holds frame 2
        kvcr.append_batch([a, b], None, None, [1, 2])
    assert e.value.code == kvcr.KVCR_ESTATE
    with pytest.raises(kvcr.KvcrError) as e:
        kvcr.append_batch([a, other], None, None, [5])
    assert e.value.code == kvcr.KVCR_ESHAPE
    with pytest.raises(kvcr.KvcrError) as e:
        kvcr.append_batch([a, a], None, None, [5])
    assert e.value.code == kvcr.KVCR_EINVAL
    assert (a.slot_map(), b.slot_map()) == before


def test_moba_longest_sequence_accepted_and_one_more_rejected():
    """The MoBA calls take sequences of up to 4096 tiles of 128 tokens (524288)."""
    import ctypes
    assert kvcr.moba_attention_bwd_workspace_bytes(16, 16384, 0, 1) == 4096 * 128 * 8
    assert kvcr.moba_attention_bwd_workspace_bytes(16, 16384, 0, 1) > 0
    assert kvcr.moba_attention_bwd_workspace_bytes(16, 16385, 0, 1) == 0
    with pytest.raises(kvcr.KvcrError) as e:
        kvcr.moba_classify_tiles(16, 16385, 0, 128)
    assert e.value.code == kvcr.KVCR_ESHAPE
    cls = kvcr.moba_classify_tiles(16, 16384, 0, 128)
    assert cls.shape == (4096, 4096)


def test_cache_flags():
    F, T, H = 2, 12, 2
    base = kvcr.kv_cache_storage_bytes_ex(2, 3, 0, T, H, 128, F, 1, kvcr.KVCR_BF16, 0)
    fused = kvcr.kv_cache_storage_bytes_ex(2, 3, 0, T, H, 128, F, 1, kvcr.KVCR_BF16,
                                           kvcr.KVCR_CACHE_FUSED_FINALIZE)
    # two spare frame slots of K and V (bf16), each 256-byte aligned
    assert fused - base >= 2 * F * T * H * 128 * 2
    assert fused - base < 2 * F * T * H * 128 * 2 + 2 * 256
    fp8 = kvcr.kv_cache_storage_bytes_ex(2, 3, 0, T, H, 128, F, 1, kvcr.KVCR_BF16,
                                         kvcr.KVCR_CACHE_FP8_K)
    # e4m3 K of 5 slots + their scales + two chunks of e4m3 staging (and scales)
    assert fp8 - base >= 5 * T * H * 128 + 2 * F * T * H * 128
    both = kvcr.KVCR_CACHE_FP8_K | kvcr.KVCR_CACHE_FUSED_FINALIZE
    assert kvcr.kv_cache_storage_bytes_ex(2, 3, 0, T, H, 128, F, 1, kvcr.KVCR_BF16, both) == 0
    assert kvcr.kv_cache_storage_bytes_ex(2, 3, 0, T, H, 128, F, 1, kvcr.KVCR_BF16, 8) == 0
    for flags, dtype, D, code in [(both, kvcr.KVCR_BF16, 128, kvcr.KVCR_EINVAL),
                                  (8, kvcr.KVCR_BF16, 128, kvcr.KVCR_EINVAL),
                                  (kvcr.KVCR_CACHE_FP8_K, kvcr.KVCR_BF16, 64,
                                   kvcr.KVCR_EUNSUPPORTED),
                                  (kvcr.KVCR_CACHE_FP8_K, kvcr.KVCR_F32, 128,
                                   kvcr.KVCR_EUNSUPPORTED),
                                  (kvcr.KVCR_CACHE_FUSED_FINALIZE, kvcr.KVCR_F32, 64,
                                   kvcr.KVCR_EUNSUPPORTED)]:
        with pytest.raises(kvcr.KvcrError) as e:
            kvcr.kv_cache_init_ex(2, 3, 0, T, H, D, F, None, dtype, flags, None)
        assert e.value.code == code, (flags, dtype, D)
    # spare slots count against the 32 frame slots
    with pytest.raises(kvcr.KvcrError) as e:
        kvcr.kv_cache_init_ex(6, 20, 4, T, H, 128, 4, None, kvcr.KVCR_BF16,
                              kvcr.KVCR_CACHE_FUSED_FINALIZE, None)
    assert e.value.code == kvcr.KVCR_ESHAPE
    h = kvcr.kv_cache_init_ex(6, 20, 2, T, H, 128, 4, None, kvcr.KVCR_BF16,
                              kvcr.KVCR_CACHE_FUSED_FINALIZE, None)
    kvcr.kv_cache_destroy(h)


def test_new_entry_points_need_their_cache_kind():
    """Bookkeeping-only caches refuse attention; the e4m3 and fused entry points also
    refuse a cache made without their flag (before any launch)."""
    h = kvcr.kv_cache_init(1, 2, 4, 1, 128, 1, None, kvcr.KVCR_BF16, None)
    L = kvcr.lib()
    for fn in (L.chunk_attention_fwd_fp8, L.chunk_attention_fwd_finalize):
        rc = fn(h, None, 4, None, None, kvcr._i32([3]), 1, 0.0, None, None, None)
        assert rc == kvcr.KVCR_ESTATE
    kvcr.kv_cache_destroy(h)
