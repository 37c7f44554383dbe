"""One rank of the two-process CPU check of bench.py's multi-rank plumbing.

Launched by tests/test_bench_dist.py through torch.distributed.run with the
gloo backend; prints one JSON line with what this rank computed."""
import datetime
import json
import os
import sys

import torch
import torch.distributed as dist

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def main():
    world, rank, local = bench.dist_env()
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    # each rank's own "device time" differs; the job's time is the slowest rank's
    mine = 1.5 + rank
    slowest = bench.max_over_ranks(mine, world, torch.device("cpu"))
    value = bench.job_throughput(1e9, slowest, world)
    dist.barrier()
    line = json.dumps({"rank": rank, "world": world, "local": local, "mine": mine, "slowest": slowest,
                       "value": value}) + "\n"
    os.write(1, line.encode())  # one write: the ranks share the pipe, lines must not interleave
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
