"""The multi-rank path of bench.py on CPU: two gloo ranks, as torchrun would
launch them.  Every rank runs its own independent call (heads are independent,
so there is no data-path collective); the only exchange is the max-over-ranks
time, and the job's throughput counts every rank's calls."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, times, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    from datetime import timedelta
    r, wsz, local = bench.dist_env()
    assert (r, wsz, local) == (rank, world, rank)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        t_max = bench.max_over_ranks(times[rank], world, torch.device("cpu"))
        results[rank] = (t_max, bench.calls_per_second(t_max, world))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_takes_the_slowest_rank():
    world, times = 2, [12.5, 20.0]
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), times, results), nprocs=world, join=True,
                       start_method="spawn")
    assert len(results) == world
    for r in range(world):
        t_max, value = results[r]
        assert t_max == 20.0
        assert value == pytest.approx(2 * 1000.0 / 20.0)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(7.0, 1, None) == 7.0
    assert bench.calls_per_second(250.0, 1) == pytest.approx(4.0)
