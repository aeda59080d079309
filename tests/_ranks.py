"""Rank body for the two-process gloo test of bench.py's multi-rank host logic
(a module of its own so that spawned processes can import it)."""
import datetime
import os
import sys
from pathlib import Path

ROOT = Path(__file__).resolve().parent.parent


def rank_main(rank: int, world: int, port: int, queue) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, str(ROOT))
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, w, local = bench.dist_env()
        bench.barrier(True)
        # each rank's device time differs; every rank must see the slowest
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, True)
        value = bench.aggregate_rate(w, 8192, 20, ms)
        bench.barrier(True)
        queue.put((r, w, local, ms, value))
    finally:
        dist.destroy_process_group()
