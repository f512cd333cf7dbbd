"""Run under torch.distributed.run on CPU (gloo): every rank reduces a few
per-rank timings with bench.max_over_ranks and writes what it got to
<out_dir>/rank<r>.json (argv[1])."""
import datetime
import json
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import torch.distributed as dist  # noqa: E402

import bench  # noqa: E402


def main():
    rank = int(os.environ["RANK"])
    world = int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        local = [1.0 + rank, 10.0 - rank, 5.0]
        got = bench.max_over_ranks(local, world)
        with open(os.path.join(sys.argv[1], f"rank{rank}.json"), "w") as f:
            json.dump({"rank": rank, "world": world, "local": local, "max": got,
                       "value": bench.job_throughput(world, 100, got[0])}, f)
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
