"""The work counts behind bench.py's throughput figures, checked against the oracle:
useful FLOPs = 4 * D * H * (number of allowed (query, key) pairs), algorithmic bytes of the
append = read and write of K and V."""
import numpy as np
import pytest

from kv_cache_chunk_ring_b200 import workloads as wl
from oracle.cache import CacheModel
from oracle.moba import MobaLayout, moba_mask


@pytest.mark.parametrize("n,c,m", [(1, 3, 0), (2, 5, 1), (3, 4, 2), (4, 2, 3)])
def test_moba_useful_flops_is_the_allowed_pair_count(n, c, m):
    import bench
    spec = wl.MobaSpec("t", heads=3, head_dim=16, n_chunks=n, chunk_tokens=c, n_bidir_chunks=m,
                       seed=0)
    pairs = int(moba_mask(MobaLayout(n, c, m)).sum())
    assert bench.moba_useful_flops(spec) == 4.0 * pairs * 3 * 16


def test_moba_workload_useful_tflop():
    import bench
    # 8 + 8 chunks of 6032 tokens + an 8-chunk bidirectional block: 30.40 TFLOP forward
    assert abs(bench.moba_useful_flops(wl.MOBA_8x6032) / 1e12 - 30.40) < 0.01


def test_steady_state_step_flops_counts_every_visible_key():
    """Chunk step: the queries of 4 frames read 6 + 8 cached frames and their own 4."""
    import bench
    spec = wl.VIDEO_832x464
    cache = CacheModel(spec.sinks, spec.window)
    for c in range(bench.STEADY_CHUNK):
        cache.append(spec.frames_of_chunk(c))
    n_keys = (len(cache.cached_frames()) + spec.chunk_frames) * spec.tokens_per_frame
    assert n_keys == 27144
    assert bench.step_flops(spec) == 4.0 * spec.chunk_tokens * n_keys * spec.heads * spec.head_dim
    assert abs(bench.step_flops(spec) / 1e12 - 1.006) < 0.001


def test_append_bytes():
    import bench
    spec = wl.VIDEO_832x464
    # K and V of 4 frames of 1508 tokens x 12 heads x 128, bf16, each read once and written once
    assert bench.append_bytes(spec) == 2 * 2 * 4 * 1508 * 12 * 128 * 2
