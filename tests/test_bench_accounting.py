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


def test_clock_samples_outside_the_timed_window_are_dropped(tmp_path):
    """The clock summary keeps only nvidia-smi samples stamped inside the timed region:
    idle samples before it (the sampler starts early) must not pull the median down,
    and a throttle reason seen only outside it is not reported."""
    import time

    import bench

    def stamp(t):
        return time.strftime("%Y/%m/%d %H:%M:%S", time.localtime(t)) + ".%03d" % int((t % 1) * 1000)

    t0 = time.mktime(time.strptime("2026/12/03 10:00:00", "%Y/%m/%d %H:%M:%S"))
    rows = [  # (time, sm clock, sw_power_cap)
        (t0 - 0.40, 345, "Not Active"),   # idle, before the window
        (t0 - 0.10, 1965, "Active"),      # before the window, power cap
        (t0 + 0.05, 1965, "Not Active"),
        (t0 + 0.10, 1950, "Not Active"),
        (t0 + 0.15, 1935, "Not Active"),
        (t0 + 0.60, 300, "Active"),       # after the window
    ]
    path = tmp_path / "clocks.csv"
    with open(path, "w") as f:
        for t, clk, cap in rows:
            f.write(f"{stamp(t)}, 0, {clk}, 1965, 700.00, 0x0, Not Active, Not Active, "
                    f"Not Active, {cap}\n")

    class _Proc:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    s = bench.ClockSampler(0)
    s.path = str(path)
    s.proc = _Proc()
    s.f = open(path, "a")
    s.window(t0, t0 + 0.2)
    got = s.stop()
    assert got == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 3}
