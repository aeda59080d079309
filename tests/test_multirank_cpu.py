"""bench.py's multi-rank path on CPU: two gloo ranks on 127.0.0.1 run its
barrier, the max-over-ranks timing and the weak-scaling aggregate (the path
torchrun takes with one rank per GPU, NCCL replaced by gloo); the reference arm
does no work on ranks other than 0."""
import argparse
import socket
import sys
from pathlib import Path

import pytest
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parent.parent
sys.path.insert(0, str(ROOT))
sys.path.insert(0, str(Path(__file__).resolve().parent))

import _ranks  # noqa: E402
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ranks.rank_main, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(queue.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, (rank, world, local, ms, value) in enumerate(results):
        assert (rank, world, local) == (r, 2, r)
        assert ms == 15.0  # rank 1's time, seen by both ranks
        assert value == pytest.approx(2 * 8192 * 20 / 0.015)


def test_single_rank_helpers():
    assert bench.max_over_ranks(3.5, False) == 3.5
    assert bench.aggregate_rate(1, 100, 10, 1000.0) == pytest.approx(1000.0)
    # weak scaling: N ranks of the same per-rank work and time give N times the rate
    assert bench.aggregate_rate(4, 100, 10, 1000.0) == pytest.approx(4000.0)


def test_reference_arm_is_rank0_only(capsys):
    args = argparse.Namespace(gpus=2, steps=1, warmup=3)
    bench.run_reference(args, rank=1)
    assert capsys.readouterr().out == ""


def test_context_parallel_gather_and_ranges_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ranks.gather_rank_main, args=(r, 2, port, queue))
             for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(queue.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, stacked, rng in results:
        # rank order on every rank: part 0 from rank 0, part 1 from rank 1
        assert stacked == [[[1.0] * 3] * 2, [[2.0] * 3] * 2]
        assert rng == (512 * rank, 512 * (rank + 1))
