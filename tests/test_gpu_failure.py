"""Failure detection on the GPU without a fault: a wait inside the attention kernel
that nothing satisfies runs out after a short bound, the kernel reports
KVCR_ETIMEOUT through the device status word, and the CUDA context stays usable."""
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


def test_withheld_signal_times_out_and_context_survives():
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    spec = wl.shrink(wl.VIDEO_832x464, grid_h=8, grid_w=16, heads=2, chunk_frames=2, sinks=1,
                     window=2, n_chunks=3, seed=31)
    items = list(wl.rollout_chunks(spec))
    cache = kvcr.Cache(spec.sinks, spec.window, spec.tokens_per_frame, spec.heads,
                       spec.head_dim, spec.chunk_frames, rope=spec.rope())
    for it in items[:2]:
        cache.append(to_dev(it["k"], "bf16"), to_dev(it["v"], "bf16"), it["frames"])
    q, k, v = (to_dev(items[2][x], "bf16") for x in ("q", "k", "v"))
    o_ref, _ = cache.attention(q, k, v, items[2]["frames"])
    torch.cuda.synchronize()
    kvcr.kvcr_check_status()

    kvcr.kvcr_debug_inject(1, 50_000_000)           # withhold one signal, 50 ms bound
    try:
        o_bad = torch.zeros_like(q)
        cache.attention(q, k, v, items[2]["frames"], out=o_bad)
        with pytest.raises(kvcr.KvcrError) as e:
            kvcr.kvcr_check_status()
        assert e.value.code == kvcr.KVCR_ETIMEOUT
        # every CTA gave up (each withholds one signal): its rows are NaN, not stale data
        assert torch.isnan(o_bad.float()).all()
    finally:
        kvcr.kvcr_debug_inject(0, 0)

    # the status was cleared and the same call works again, bit for bit
    o2, _ = cache.attention(q, k, v, items[2]["frames"])
    torch.cuda.synchronize()
    kvcr.kvcr_check_status()
    assert torch.equal(o2, o_ref)


def test_inject_argument_checks():
    from kv_cache_chunk_ring_b200 import kvcr
    with pytest.raises(kvcr.KvcrError):
        kvcr.kvcr_debug_inject(7, 0)
    kvcr.kvcr_debug_inject(0, 0)
