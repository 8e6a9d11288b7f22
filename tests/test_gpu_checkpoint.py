"""Restore after a restart on the GPU: a cache's exported host state plus a copy of its device
storage, loaded into a new cache of the same configuration, gives bit-identical attention and
appends from then on -- also for a fused-finalize cache whose slots were relabelled."""
import pytest

from kv_cache_chunk_ring_b200 import workloads as wl
from tests.gpu_helpers import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_chunk_ring_b200 import build
    build.build()


@pytest.mark.parametrize("fused", [False, True])
def test_restore_from_state_and_storage(fused):
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    spec = wl.shrink(wl.VIDEO_832x464, grid_h=6, grid_w=20, heads=2, chunk_frames=2, sinks=1,
                     window=3, n_chunks=7, seed=33)
    items = list(wl.rollout_chunks(spec))

    def mk():
        return kvcr.Cache(spec.sinks, spec.window, spec.tokens_per_frame, spec.heads,
                          spec.head_dim, spec.chunk_frames, rope=spec.rope(), fused_finalize=fused)

    def run(cache, it):
        q, k, v = (to_dev(it[x], "bf16") for x in ("q", "k", "v"))
        if fused:
            o, lse = cache.attention_finalize(q, k, v, it["frames"], want_lse=True)
        else:
            o, lse = cache.attention(q, k, v, it["frames"], want_lse=True)
            cache.append(k, v, it["frames"])
        return o, lse

    a = mk()
    for it in items[:4]:
        run(a, it)
    torch.cuda.synchronize()
    state, storage = a.export_state(), a.storage.clone()
    b = mk()
    b.storage.copy_(storage)
    b.import_state(state)
    for it in items[4:]:
        oa, la = run(a, it)
        ob, lb = run(b, it)
        torch.cuda.synchronize()
        assert torch.equal(oa, ob) and torch.equal(la, lb)
        assert a.slot_map() == b.slot_map()
    for slot, frame in enumerate(a.slot_map()):
        if frame >= 0:
            for x, y in zip(a.slot_tensors(slot), b.slot_tensors(slot)):
                assert torch.equal(x, y)
