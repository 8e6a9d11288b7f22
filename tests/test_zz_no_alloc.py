"""chunk_attention_fwd_static_scratch: chunk attention that allocates nothing.

It exists for callers that cannot allocate device memory when they call the
library -- hosts whose memory pool owns every allocation and hands the library
only the cache buffer, or real-time loops that cannot take the device
synchronisation of cudaMalloc/cudaFree.  Instead of the cache's scratch region
it stages the rotated queries and keys in a fixed 36 MiB array the library
keeps on the device.

These tests call it through the C ABI and check, on two calls in a row per
chunk, that it returns what chunk_attention_fwd returns (same tolerances as
the other parity tests), at a small size and at the 832x464 chunk size, and
that a chunk larger than the array is refused before anything runs.
"""
import numpy as np
import pytest

from kv_cache_chunk_ring_b200 import workloads as wl
from tests.gpu_helpers import TOL_LSE, assert_close, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_chunk_ring_b200 import build
    build.build()


def _check_against_existing(spec, n_chunks):
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    cache = kvcr.Cache(spec.sinks, spec.window, spec.tokens_per_frame, spec.heads,
                       spec.head_dim, spec.chunk_frames, rope=spec.rope())
    for item in list(wl.rollout_chunks(spec))[:n_chunks]:
        q, k, v = (to_dev(item[x], "bf16") for x in ("q", "k", "v"))
        o_ref, lse_ref = cache.attention(q, k, v, item["frames"], want_lse=True)
        o_ref_np, lse_ref_np = to_np(o_ref), lse_ref.cpu().numpy()
        for _ in range(2):                      # two calls in a row share the array
            o = torch.full_like(q, float("nan"))
            lse = torch.full_like(lse_ref, float("nan"))
            kvcr.chunk_attention_fwd_static_scratch(cache.handle, q, k, v, item["frames"], o, lse)
            torch.cuda.synchronize()
            assert_close(to_np(o), o_ref_np, "static-scratch vs chunk_attention_fwd")
            assert np.abs(lse.cpu().numpy() - lse_ref_np).max() <= TOL_LSE
        cache.append(k, v, item["frames"])
    kvcr.kvcr_check_status()


def test_matches_chunk_attention_small():
    spec = wl.shrink(wl.VIDEO_832x464, grid_h=8, grid_w=16, heads=4, chunk_frames=2, sinks=2,
                     window=2, n_chunks=4, seed=21)
    _check_against_existing(spec, 4)


def test_matches_chunk_attention_832x464_chunk():
    spec = wl.shrink(wl.VIDEO_832x464, sinks=1, window=1, n_chunks=2, seed=22)
    _check_against_existing(spec, 2)


def test_refuses_chunk_larger_than_array():
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    # 8 frames x 1508 tokens x 12 heads x 128 x 2 bytes = 37 MB per staged tensor > 18 MiB
    spec = wl.shrink(wl.VIDEO_832x464, sinks=1, window=1, chunk_frames=8, n_chunks=1)
    cache = kvcr.Cache(spec.sinks, spec.window, spec.tokens_per_frame, spec.heads,
                       spec.head_dim, spec.chunk_frames, rope=spec.rope())
    n = spec.chunk_tokens
    q = torch.zeros((n, spec.heads, spec.head_dim), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    with pytest.raises(kvcr.KvcrError) as e:
        kvcr.chunk_attention_fwd_static_scratch(cache.handle, q, q, q, list(range(8)), o)
    assert e.value.code == kvcr.KVCR_ESHAPE
    assert "bytes of staging" in str(e.value)
