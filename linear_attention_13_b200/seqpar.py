"""Sequence parallelism across GPUs for the prefill.

A sequence split over the R ranks of a process group (rank r holding tokens
[r N/R, (r+1) N/R) of every (batch, head)) is prefilled in one exchange:

  1. dS_r = K_r^T V_r of the rank's tokens           (la_state_increment)
  2. all-gather of dS over the ranks                  (torch.distributed)
  3. S_in,r = sum of dS_r' over the ranks r' < r      (la_state_prefix)
  4. outputs of the rank's tokens from S_in,r         (la_prefill_from_state)

so only B*H*d*d fp32 values per rank cross the links, once.  The improved
linear-attention sequence parallelism (LASP) that section 2 of the futurefh
page names has no algorithm in the pages; this is the plain reading of it for
the recurrence o_t = q_t S_t.

The three compute steps run in the library's CUDA kernels.  ``compute`` lets
the host tests substitute host implementations, so that the exchange itself can
be checked with CPU ranks over gloo.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional


@dataclass
class ShardCompute:
    """The per-rank steps: increment(k, v) -> dS; prefix(gathered, rank) -> S_in;
    prefill(q, k, v, state_in) -> (o, state_out)."""
    increment: Callable
    prefix: Callable
    prefill: Callable


def cuda_compute(blk: int = 128, flags: int = 0) -> ShardCompute:
    import linear_attention_13_b200 as la

    return ShardCompute(
        increment=lambda k, v: la.state_increment(k, v),
        prefix=lambda gathered, rank: la.state_prefix(gathered, rank),
        prefill=lambda q, k, v, state_in: la.prefill(q, k, v, blk=blk, flags=flags, state_in=state_in),
    )


def prefill_sequence_parallel(q, k, v, group=None, compute: Optional[ShardCompute] = None,
                              blk: int = 128, flags: int = 0):
    """Prefill of this rank's token shard [B,H,N_r,d] of a sequence split over
    the ranks of ``group`` in rank order.  Returns (o_r, state_out_r); the last
    rank's state is the final state of the whole sequence.  Every rank of the
    group must call it (one all-gather)."""
    import torch
    import torch.distributed as dist

    compute = compute or cuda_compute(blk, flags)
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    delta = compute.increment(k, v).contiguous()
    if dist.get_backend(group) == "nccl":
        gathered = torch.empty((world,) + tuple(delta.shape), dtype=delta.dtype, device=delta.device)
        dist.all_gather_into_tensor(gathered, delta, group=group)
    else:
        parts = [torch.empty_like(delta) for _ in range(world)]
        dist.all_gather(parts, delta, group=group)
        gathered = torch.stack(parts)
    state_in = compute.prefix(gathered, rank)
    return compute.prefill(q, k, v, state_in)
