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


def gather_rank_main(rank: int, world: int, port: int, queue) -> None:
    """Context-parallel host logic on CPU: every rank's tensor gathered in rank
    order, and the token ranges of the parts."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, str(ROOT))
    import torch
    import torch.distributed as dist

    from kernelized_linear_attention_chunked_b200.context_parallel import (gather_parts,
                                                                           local_range)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        x = torch.full((2, 3), float(rank + 1))
        stacked = gather_parts(x)
        queue.put((rank, stacked.tolist(), local_range(1024, world, rank)))
    finally:
        dist.destroy_process_group()


def cp_rank_main(rank: int, world: int, port: int, queue, d: int, T: int) -> None:
    """Context-parallel prefill on the GPU: this rank's part of one seeded
    sequence (gloo for the one exchange; the ranks' kernels never wait on each
    other)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, str(ROOT))
    import torch
    import torch.distributed as dist

    import kernelized_linear_attention_chunked_b200 as kata
    from kernelized_linear_attention_chunked_b200.context_parallel import (
        local_range, prefill_context_parallel)
    from kernelized_linear_attention_chunked_b200.inputs import prefill_inputs
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v = prefill_inputs(1, 2, T, d, dtype="bf16", seed=77)
        a, b = local_range(T, world, rank)
        part = [x[:, :, a:b].contiguous().cuda() for x in (q, k, v)]
        o, H, s = prefill_context_parallel(*part, chunk=64)
        kata.sync_status()
        queue.put((rank, o.cpu(), H.cpu(), s.cpu()))
    finally:
        dist.destroy_process_group()
