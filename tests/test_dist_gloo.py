"""The multi-GPU path is replicas only: every rank runs the whole layer on its
own batch and the job's time is the slowest rank's.  This checks the host
side of that path -- the max-over-ranks reduction and the whole-job
throughput -- with two gloo ranks on the CPU (no GPU, no collective on the
data path)."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [120.0, 80.0][rank]
        worst = bench.max_over_ranks(local_ms, dist, device="cpu")
        value = bench.replica_throughput(4096, 10, world, worst)
        dist.barrier()
        q.put((rank, worst, value))
    finally:
        dist.destroy_process_group()


def test_replica_timing_is_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, worst, value in res:
        assert worst == 120.0
        assert value == pytest.approx(2 * 4096 * 10 / 0.120)


def test_single_process_is_identity():
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.replica_throughput(100, 2, 1, 1000.0) == pytest.approx(200.0)
