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
