"""Context-parallel prefill: one sequence split over the ranks of a process
group, one exchange step.

"Kernelized Linear Attention: Breaking the Capacity Wall with Symmetric Cones",
s2.3: across blocks the state propagates as a prefix sum, so the state before
rank r's part is the sum of the earlier parts' states. Each rank:
  1. computes the final state of its own part from zero (kata_prefill,
     state only);
  2. all-gathers the parts' states (the one collective; NCCL over NVLink for
     GPU ranks);
  3. forms the exclusive prefix over the parts (kata_state_prefix);
  4. runs kata_prefill on its part from that prefix, which gives its outputs
     and the state after its part exactly as one long prefill would.
Every arithmetic step runs in libkata's kernels; this module only moves
tensors and calls the collective.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _binding as kb


def local_range(T: int, world: int, rank: int) -> tuple[int, int]:
    """Token range [start, stop) of rank `rank` when T tokens are split into
    `world` consecutive parts of equal length (T % world == 0)."""
    if T % world:
        raise ValueError(f"T={T} does not split into {world} equal parts")
    n = T // world
    return rank * n, (rank + 1) * n


def gather_parts(x: torch.Tensor, group=None) -> torch.Tensor:
    """[world, *x.shape]: every rank's x stacked in rank order. Backends that
    exchange host tensors only (gloo) get host copies."""
    world = dist.get_world_size(group)
    nccl = dist.get_backend(group) == "nccl"
    src = x.contiguous() if nccl else x.detach().cpu().contiguous()
    parts = [torch.empty_like(src) for _ in range(world)]
    dist.all_gather(parts, src, group=group)
    return torch.stack(parts).to(x.device)


def prefill_context_parallel(q, k, v, chunk: int, eps: float = 1e-6, group=None,
                             output: bool = True, state: bool = True, stream=None):
    """q, k, v [B, H, T_part, d]: this rank's consecutive part of the sequence
    (rank order = sequence order). Returns (o of this part or None, the state
    after this part or None); the last rank's state is the whole sequence's."""
    rank = dist.get_rank(group)
    _, H_loc, s_loc = kb.prefill(q, k, v, chunk, eps, output=False, stream=stream)
    H_pre, s_pre = kb.state_prefix(gather_parts(H_loc, group), gather_parts(s_loc, group),
                                   stream=stream)
    H_in = H_pre[rank] if rank > 0 else None
    s_in = s_pre[rank] if rank > 0 else None
    o, H_out, s_out = kb.prefill(q, k, v, chunk, eps, H_in=H_in, s_in=s_in, output=output,
                                 state=state, stream=stream)
    return o, H_out, s_out
