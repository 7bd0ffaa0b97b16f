"""One rank of a CPU stand-in for bench.py's device step (used by
test_bench_dist.py to check bench.launch_ranks): every rank joins a gloo
group from the environment the launcher set, does rank-dependent work, and
rank 0 prints the whole-job line the way bench.py does (units summed over
ranks, time = the slowest rank's)."""
import json
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch.distributed as dist  # noqa: E402

import bench  # noqa: E402


def main():
    world, rank, local = bench.dist_env()
    dist.init_process_group("gloo", rank=rank, world_size=world)
    t0 = time.perf_counter()
    units = float(rank + 1)                      # rank r processes r + 1 units
    time.sleep(0.05 * (rank + 1))
    secs = time.perf_counter() - t0
    total, tmax = bench.aggregate(dist, units, secs, "cpu")
    if rank == 0:
        print(json.dumps({"n_gpus": world, "units": total, "seconds": tmax,
                          "value": total / tmax, "local_rank": local}), flush=True)
    dist.barrier()
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
