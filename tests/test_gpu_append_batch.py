"""The batched all-layer append writes exactly what one append per cache writes."""
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


@pytest.mark.parametrize("spec", [
    wl.shrink(wl.VIDEO_832x464, grid_h=8, grid_w=16, heads=2, chunk_frames=2, sinks=1, window=2,
              n_chunks=5, seed=61, layers=4),
    wl.shrink(wl.VIDEO_832x464, n_chunks=5, seed=62, layers=3),
    wl.shrink(wl.TINY_F32, layers=3, n_chunks=5),
])
def test_batch_equals_single_appends(spec):
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    T, F = spec.tokens_per_frame, spec.chunk_frames
    mk = lambda: kvcr.Cache(spec.sinks, spec.window, T, spec.heads, spec.head_dim, F,
                            rope=spec.rope(), dtype=spec.dtype)
    batch = [mk() for _ in range(spec.layers)]
    single = [mk() for _ in range(spec.layers)]
    per_layer = [list(wl.rollout_chunks(spec, layer)) for layer in range(spec.layers)]
    for c in range(spec.n_chunks):
        if c == 3 and spec.window > 1:           # one layer's window shrinks: states differ
            batch[0].evict(1)
            single[0].evict(1)
        ks = [to_dev(per_layer[l][c]["k"], spec.dtype) for l in range(spec.layers)]
        vs = [to_dev(per_layer[l][c]["v"], spec.dtype) for l in range(spec.layers)]
        frames = per_layer[0][c]["frames"]
        kvcr.append_batch(batch, ks, vs, frames)
        for l in range(spec.layers):
            single[l].append(ks[l], vs[l], frames)
        torch.cuda.synchronize()
        for b, s in zip(batch, single):
            assert b.slot_map() == s.slot_map()
            for slot, f in enumerate(b.slot_map()):
                if f < 0:
                    continue
                kb, vb = b.slot_tensors(slot)
                ksg, vsg = s.slot_tensors(slot)
                assert torch.equal(kb, ksg) and torch.equal(vb, vsg), (c, slot)
