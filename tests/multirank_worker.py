"""Worker for test_multirank.py, launched with torch.distributed.run on the
CPU (gloo): each rank reports a different device time and the bench's
max-over-ranks / whole-job throughput logic must agree on every rank."""
import json
import os
import sys

import torch
import torch.distributed as dist

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def main():
    import datetime
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    rank, world = dist.get_rank(), dist.get_world_size()
    ms = 10.0 + 5.0 * rank                        # rank r "took" 10 + 5 r ms
    slowest = bench.max_over_ranks(ms, dist, torch.device("cpu"))
    value, t = bench.combine_ranks([slowest], world, 3.0)  # 3 units per rank
    got = [None] * world
    dist.all_gather_object(got, {"rank": rank, "slowest": slowest, "value": value})
    if rank == 0:
        print(json.dumps({"world": world, "per_rank": got}), flush=True)
    dist.barrier()
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
