"""Worker for the multi-rank host-logic test: run under torchrun with the gloo
backend, every rank reports a different step time; rank 0 prints what the
bench's aggregation makes of them as one JSON line."""
import datetime
import json
import os
import sys

import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def main():
    rank, world, local = bench.dist_env()
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    ms = 10.0 + 5.0 * rank  # rank r took 10 + 5r ms
    slowest = bench.max_over_ranks(ms, dist, "cpu")
    value = bench.job_tflops(1e12, world, slowest)
    got = [None] * world
    dist.all_gather_object(got, {"rank": rank, "local": local, "slowest": slowest})
    dist.barrier()
    dist.destroy_process_group()
    if rank == 0:
        print(json.dumps({"world": world, "per_rank": got, "value": value}), flush=True)


if __name__ == "__main__":
    main()
