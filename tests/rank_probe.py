"""One rank of the benchmark's replica launcher, without a GPU (gloo): each rank
reports a fixed per-rank time, the job takes the slowest, and rank 0 alone
prints the benchmark-style JSON line.  Run by tests/test_multi_rank_cpu.py
through bench.run_replicas."""

import datetime
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch.distributed as dist  # noqa: E402

import bench  # noqa: E402


def main():
    rank = int(os.environ["RANK"])
    world = int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        steps = 10
        dist.barrier()
        t = bench.max_over_ranks(100.0 + 25.0 * rank, dist, "cpu")  # ms for `steps` steps
        dist.barrier()
        if rank == 0:
            print(json.dumps({"n_gpus": world, "steps": steps, "ms_per_step": t / steps,
                              "value": bench.job_throughput(world, steps, t)}))
    finally:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
