"""One rank of the launch test (run by bench.relaunch under torchrun, on CPU with gloo).

Each rank times a step of its own (rank r sleeps 20 + 30 r ms), the ranks meet at a barrier,
the step time is the max over ranks (bench.reduce_max) and rank 0 prints one JSON line with
the whole job's value (bench.weak_value), as bench.py does for the decode."""
import argparse
import datetime
import json
import os
import sys
import time

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import torch.distributed as dist  # noqa: E402

import bench  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--units", type=int, required=True)
    args = ap.parse_args()
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        t0 = time.perf_counter()
        time.sleep(0.02 + 0.03 * rank)
        own = (time.perf_counter() - t0) * 1e3
        dist.barrier()
        (ms,) = bench.reduce_max([own], world)
        every = [0.0] * world
        every[rank] = own
        every = bench.reduce_max(every, world)
        if rank == 0:
            print(json.dumps({"n_gpus": world, "ranks_seen": dist.get_world_size(), "ms_per_step": ms,
                              "rank_ms": every, "value": bench.weak_value(world, args.units, ms)}), flush=True)
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
