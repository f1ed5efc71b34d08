"""The N > 1 bench path on CPU: two gloo ranks, one process each.

The layer runs as independent replicas (no collective on the data path);
what crosses ranks is only the timing: every rank reports its timed region,
the job takes the slowest, and throughput counts the units of all ranks.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        my_ms = [12.5, 20.0][rank]
        slow = bench.max_over_ranks(my_ms)
        # a second collective in the same order on every rank
        slow2 = bench.max_over_ranks(100.0 - my_ms)
        rate = bench.whole_job_rate(4096, world, 10, slow)
        q.put((rank, slow, slow2, rate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_takes_the_slowest_and_counts_all_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(2))
    for rank, slow, slow2, rate in out:
        assert slow == 20.0 and slow2 == 87.5
        assert rate == pytest.approx(4096 * 2 * 10 / 20e-3)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.0) == 3.0
    assert bench.whole_job_rate(100, 1, 5, 10.0) == pytest.approx(100 * 5 / 10e-3)
