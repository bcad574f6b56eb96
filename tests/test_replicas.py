"""The benchmark's multi-rank path on CPU (gloo, world size 2): every rank
runs an independent replica; the job time is the slowest rank's, the value
counts every rank's query tokens, and only collectives on timing are used."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    local_ms = 100.0 + 50.0 * rank
    m = bench.max_over_ranks(local_ms, dist, "cpu")
    v = bench.job_throughput(world, 96, 10, m)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, m, v))


def test_two_rank_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, v in res:
        assert m == 150.0                      # the slowest rank
        assert v == pytest.approx(2 * 96 * 10 / 0.150)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(12.5) == 12.5
    assert bench.job_throughput(1, 96, 10, 1000.0) == pytest.approx(960.0)
