"""A rank of the launcher test: joins a gloo process group on the CPU, sums
the ranks with one all-reduce and writes what it saw to <out_dir>/rank<r>.json."""
import json
import os
import sys
from datetime import timedelta

import torch
import torch.distributed as dist


def main():
    out_dir = sys.argv[1]
    rank = int(os.environ["RANK"])
    world = int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    t = torch.tensor([float(rank)])
    dist.all_reduce(t)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"rank": rank, "world": world, "rank_sum": float(t.item()),
                   "local_rank": int(os.environ["LOCAL_RANK"])}, f)
    dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
