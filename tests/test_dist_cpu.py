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


def test_launch_plan():
    import bench
    assert bench.launch_plan(1, {}) == ("run", 1)
    assert bench.launch_plan(2, {}) == ("relaunch", 2)
    assert bench.launch_plan(8, {"WORLD_SIZE": "8"}) == ("run", 8)
    kind, msg = bench.launch_plan(2, {"WORLD_SIZE": "1"})
    assert kind == "error" and "WORLD_SIZE=1" in msg
    kind, _ = bench.launch_plan(1, {"WORLD_SIZE": "4"})
    assert kind == "error"
    assert bench.launch_plan(0, {})[0] == "error"
    cmd = bench.torchrun_command(4, ["--gpus", "4", "--steps", "3"], 29999)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert cmd[cmd.index("--nproc-per-node") + 1] == "4"
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-3:] == ["--gpus", "4", "--steps", "3"][-3:]


def test_bench_refuses_a_world_size_that_disagrees_with_gpus():
    """--gpus 2 under a one-rank WORLD_SIZE exits non-zero before any device work
    (it never prints a line with n_gpus 1)."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--steps", "1"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "WORLD_SIZE=1" in r.stderr
    assert '"n_gpus"' not in r.stdout
