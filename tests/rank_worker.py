"""Worker for the world-size-2 tests of bench.py's multi-rank plumbing, run
by torchrun on the CPU (gloo): every rank joins the group, passes the
barrier, and prints its view of the maximum over ranks of a per-rank time."""
import json
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402

world, rank, local = bench.dist_setup("gloo")
bench.barrier(world)
mx = bench.max_over_ranks(1.5 * (rank + 1), world, torch.device("cpu"))
bench.barrier(world)
print(json.dumps({"rank": rank, "world": world, "local": local, "max": mx}), flush=True)
import torch.distributed as dist  # noqa: E402

dist.destroy_process_group()
