"""Rank logic of the multi-GPU benchmark on two CPU ranks (gloo): every rank
takes the same collective steps, the job's time is the slowest rank's, the
whole-job throughput counts every rank's steps, and only rank 0 reports."""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, times, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        t = bench.max_over_ranks(times[rank], dist, "cpu")
        v = bench.job_throughput(world, 10, t)
        dist.barrier()
        out[rank] = (t, v)
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_job_throughput():
    world = 2
    times = [120.0, 150.0]  # ms for 10 steps on each rank
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), times, out), nprocs=world, start_method="spawn")
    assert out[0][0] == out[1][0] == 150.0           # the job ends with the slowest rank
    assert out[0][1] == pytest.approx(2 * 10 / 0.150)  # all ranks' steps over that time


def test_single_rank_passthrough():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(1, 20, 1000.0) == pytest.approx(20.0)


def test_reference_arm_other_ranks_exit_without_work():
    sys.path.insert(0, ROOT)
    import bench

    class A:
        pass
    # rank 1 of a torchrun launch returns at once (rank 0 alone times the oracle)
    assert bench.run_reference(A(), 1, 2) == 0


def test_replica_launcher_starts_n_ranks(capfd):
    """bench.py --gpus N without a launcher starts N ranks through torchrun; rank 0 alone prints, with
    n_gpus = N and the job's throughput over the slowest rank's time."""
    sys.path.insert(0, ROOT)
    import json
    import bench
    cmd = bench.replica_command(2, "x.py", ["--steps", "3"], 12345)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert cmd[cmd.index("--nproc-per-node") + 1] == "2" and cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-3:] == ["x.py", "--steps", "3"]
    rc = bench.run_replicas(2, [], script=os.path.join(ROOT, "tests", "rank_probe.py"), timeout_s=300)
    assert rc == 0
    lines = [ln for ln in capfd.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["n_gpus"] == 2
    assert rec["ms_per_step"] == pytest.approx(12.5)          # the slower rank: 125 ms over 10 steps
    assert rec["value"] == pytest.approx(2 * 10 / 0.125)
