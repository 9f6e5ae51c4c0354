"""One rank of the launcher test in test_multirank.py (CPU, gloo): checks the environment that
torch.distributed.run gives each rank, exchanges the expert-parallel group plan of bench.py with the
other ranks and appends what it saw to the file named on the command line."""
import json
import os
import sys

import torch.distributed as dist

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402

out_path, n, E, k = sys.argv[1], int(sys.argv[2]), int(sys.argv[3]), int(sys.argv[4])
world, rank, local = bench._dist()
dist.init_process_group("gloo")
try:
    plan = bench.ep_group_plan(n, E, k, world, rank)
    plans = [None] * world
    dist.all_gather_object(plans, plan)
    ms = bench.reduce_max(10.0 + rank, world, "cpu")
    if rank == 0:
        with open(out_path, "w") as f:
            json.dump(dict(world=world, local=local, master=os.environ.get("MASTER_ADDR"), plans=plans, ms=ms), f)
    dist.barrier()
finally:
    dist.destroy_process_group()
