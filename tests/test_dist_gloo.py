"""The multi-process host logic of bench.py on CPU: two gloo ranks, each with its own
timing, agree on the slowest rank's time and on the whole-job throughput."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        my_ms = 10.0 + 5.0 * rank               # rank 1 is the slow one
        ms = bench.max_over_ranks(my_ms, dist, torch.device("cpu"))
        value = bench.whole_job_throughput(world, 20, 1e12, ms)
        out.put((rank, ms, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_max_time_and_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [15.0, 15.0]
    # 2 ranks x 20 steps x 1 TFLOP in 15 ms
    assert res[0][2] == pytest.approx(2 * 20 * 1.0 / 15e-3)
    assert res[0][2] == res[1][2]


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(3.5, None, None) == 3.5


def _head_split_rank(rank, world, port, out):
    """One rank of the head partition: its heads of every chunk's Q, K, V, the oracle
    rollout on them, and the library's slot table (bookkeeping-only cache)."""
    import dataclasses
    import datetime

    import torch.distributed as dist

    from kv_cache_chunk_ring_b200 import kvcr
    from kv_cache_chunk_ring_b200 import shard as sh
    from kv_cache_chunk_ring_b200 import workloads as wl
    from oracle.rollout import rollout
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        spec = _head_split_spec()
        h0, h1 = sh.head_range(spec.heads, world, rank)
        items = [dict(it, **{x: sh.slice_heads(it[x], h0, h1) for x in ("q", "k", "v")})
                 for it in wl.rollout_chunks(spec)]
        ref = rollout(dataclasses.replace(spec, heads=h1 - h0), items)
        cache = kvcr.Cache(spec.sinks, spec.window, spec.tokens_per_frame, h1 - h0,
                           spec.head_dim, spec.chunk_frames, rope=spec.rope(),
                           bookkeeping_only=True)
        maps = []
        for it in items:
            cache.append(None, None, it["frames"])
            maps.append(cache.slot_map())
        parts = [None] * world
        dist.all_gather_object(parts, (h0, h1, ref.outputs, ref.lses, maps, ref.slot_maps))
        if rank == 0:
            out.put(parts)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _head_split_spec():
    from kv_cache_chunk_ring_b200 import workloads as wl
    return wl.shrink(wl.VIDEO_832x464, grid_h=4, grid_w=6, heads=12, head_dim=64, chunk_frames=2,
                     sinks=1, window=2, n_chunks=4, seed=31)


@pytest.mark.parametrize("world", [2, 3])
def test_head_split_over_gloo_ranks_equals_unsplit(world):
    """12 heads split over gloo ranks: every rank keeps the same slot table as the
    oracle, and the heads the ranks computed, put side by side, are the unsplit
    rollout's outputs and LSEs."""
    import numpy as np

    from kv_cache_chunk_ring_b200 import build
    from kv_cache_chunk_ring_b200 import workloads as wl
    from oracle.rollout import rollout
    build.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_head_split_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    parts = q.get(timeout=300)
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    spec = _head_split_spec()
    full = rollout(spec, list(wl.rollout_chunks(spec)))
    assert parts[0][0] == 0 and parts[-1][1] == spec.heads
    assert all(parts[i][1] == parts[i + 1][0] for i in range(world - 1))
    for _, _, outs, lses, maps, ref_maps in parts:
        assert maps == ref_maps == full.slot_maps
    for n in range(len(full.outputs)):
        o = np.concatenate([p[2][n] for p in parts], axis=1)
        lse = np.concatenate([p[3][n] for p in parts], axis=0)
        np.testing.assert_allclose(o, full.outputs[n], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, full.lses[n], rtol=0, atol=1e-12)


def test_head_range_partition():
    from kv_cache_chunk_ring_b200 import shard as sh
    for heads in (12, 7, 1):
        for world in range(1, heads + 1):
            r = [sh.head_range(heads, world, k) for k in range(world)]
            assert r[0][0] == 0 and r[-1][1] == heads
            assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
            sizes = [b - a for a, b in r]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        sh.head_range(12, 13, 0)
