"""Rank body for the multi-rank CPU test (spawned processes, gloo)."""

import os
import sys
from datetime import timedelta


def rank_main(rank, world, port, ms, out_q):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    import torch
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        t = bench.max_over_ranks([ms[rank], 10.0 * ms[rank]], torch.device("cpu"))
        out_q.put((rank, t, bench.job_rate(2.0e12, world, t[0])))
        dist.barrier()
    finally:
        dist.destroy_process_group()
