"""The replica (N > 1) host logic of bench.py on CPU: world-size-2 gloo process group.

Replicas run independent caches with no data-path collective; the only cross-rank step is the
max over ranks of the timings, which sets the whole-job throughput."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local = [10.0 + rank, 5.0 - rank, 7.0]
        mx = bench.max_over_ranks(local)
        value = bench.throughput(world, 1000, mx[0])
        q.put((rank, mx, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_throughput_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, value in out:
        assert mx == [11.0, 5.0, 7.0]
        assert value == pytest.approx(2 * 1000 / 0.011)


def test_single_process_aggregation_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.throughput(1, 500, 250.0) == pytest.approx(2000.0)


def test_reference_arm_nonzero_rank_does_nothing(capsys):
    import bench

    class A:
        workload, budget, steps, warmup, gpus = "tiny", None, 1, 0, 2
    bench.run_reference(A, rank=1)
    assert capsys.readouterr().out == ""
