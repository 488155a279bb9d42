"""Multi-rank host logic of bench.py on CPU: two gloo ranks, as torchrun
would start them, agree on the slowest rank's time and on the whole-job
throughput (replicas: every rank's tokens over that time)."""
import os
import socket
from datetime import timedelta

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench

        ms = bench.max_over_ranks(10.0 + 5.0 * rank, "cpu")  # rank r took 10 + 5 r ms
        q.put((rank, ms, bench.job_tokens_per_s(8, 100, world, ms)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_ranks_take_the_slowest_time_and_count_every_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=150) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, *_ in got] == [0, 1]
    for _, ms, value in got:
        assert ms == 15.0  # the slower rank's time on both
        assert value == pytest.approx(8 * 100 * 2 / 15e-3)


def test_single_process_needs_no_process_group():
    import bench

    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.job_tokens_per_s(1, 200, 1, 14.0) == pytest.approx(200 / 14e-3)
