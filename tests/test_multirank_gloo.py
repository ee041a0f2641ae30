"""bench.py's multi-rank host logic on CPU: two gloo ranks, each timing its
own independent problem; the reported time is the slowest rank's, the
value counts every rank's MACs (weak scaling, no data-path collective), and
a re-measurement that one rank asks for is taken by all."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    my_ms = 20.0 + 5.0 * rank  # rank 1 is the slow one
    worst = bench.reduce_max(my_ms, dist, "cpu")
    value = bench.aggregate_value(worst, world)
    # only rank 1 saw a bad clock record: both ranks re-measure together
    remeasure = bench.any_rank(rank == 1, dist, "cpu")
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, worst, value, remeasure))


def test_two_gloo_ranks_max_time_and_weak_scaled_value():
    import bench

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, worst, value, remeasure in got:
        assert worst == 25.0
        assert value == pytest.approx(2 * bench.MACS_PER_STEP / 0.025)
        assert remeasure is True


def test_single_process_identity():
    import bench

    assert bench.reduce_max(3.5) == 3.5
    assert bench.any_rank(True) is True and bench.any_rank(False) is False
    assert bench.aggregate_value(50.0, 1) == pytest.approx(bench.MACS_PER_STEP / 0.05)
