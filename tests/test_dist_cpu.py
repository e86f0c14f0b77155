"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

The scan shards over independent (batch, head) lanes, so N GPUs run N
replicas with no collective on the data path; the only cross-rank step is
the timing aggregation: whole-job value = units of all ranks / max device
time over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    os.environ["RANK"] = str(rank)
    os.environ["WORLD_SIZE"] = str(world)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    elapsed = [0.5, 0.8][rank]
    units = [1000.0, 3000.0][rank]
    value, tmax, total = bench.aggregate(elapsed, units, dist, torch.device("cpu"))
    q.put((rank, value, tmax, total))
    dist.barrier()
    dist.destroy_process_group()


def test_aggregate_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(2))
    for rank, value, tmax, total in res:
        assert tmax == pytest.approx(0.8)
        assert total == pytest.approx(4000.0)
        assert value == pytest.approx(4000.0 / 0.8)


def test_aggregate_single_rank():
    import bench
    v, t, u = bench.aggregate(2.0, 10.0)
    assert v == 5.0 and t == 2.0 and u == 10.0
