"""The multi-process path of bench.py on CPU: two gloo ranks, each timing its own
copy of the workload (weak scaling, no data-path collective); the job time is the
slowest rank's and the throughput counts every rank's walks."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import sys

    import torch.distributed as dist

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    my_ms = [120.0, 250.0][rank]
    worst = bench.max_over_ranks(my_ms, world)
    qps = bench.job_throughput(256, 100, world, worst)
    dist.barrier()
    out.put((rank, worst, qps))
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, worst, qps in res:
        assert worst == 250.0
        assert qps == pytest.approx(256 * 100 * 2 / 0.25)


def test_single_rank_is_a_no_op():
    import bench

    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(256, 10, 1, 1000.0) == pytest.approx(2560.0)
