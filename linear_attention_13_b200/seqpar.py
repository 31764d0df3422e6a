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

_DTYPE_CODES = {"torch.bfloat16": 1, "torch.float32": 2, "torch.float64": 3, "torch.float16": 4}


class SequenceParallelError(RuntimeError):
    """Raised on every rank of the group when one rank's local step failed or
    the shards do not describe one sequence (``rank`` = the first rank at
    fault, ``reason`` its description)."""

    def __init__(self, rank: int, reason: str):
        self.rank = rank
        self.reason = reason
        super().__init__(f"sequence-parallel prefill: rank {rank}: {reason}")


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


def _agree(q, k, v, delta, error, group, rank, world):
    """Every rank publishes (ok, B, H, d, dtype, N) of its shard; all ranks
    then see the same table and fail together, before any state is exchanged,
    if one rank's local step failed or the shards do not share B, H, d and the
    dtype (N may differ between ranks)."""
    import torch
    import torch.distributed as dist

    dev = delta.device if delta is not None else q.device
    if dist.get_backend(group) == "nccl" and dev.type != "cuda":
        dev = torch.device("cuda", torch.cuda.current_device())
    shapes_ok = (q.dim() == 4 and k.shape == v.shape and k.dim() == 4
                 and q.shape[:2] == k.shape[:2] and q.shape[2] == k.shape[2]
                 and q.shape[3] == k.shape[3] and q.dtype == k.dtype == v.dtype)
    ok = error is None and shapes_ok
    dims = tuple(q.shape) if q.dim() == 4 else (0, 0, 0, 0)
    mine = torch.tensor([1 if ok else 0, dims[0], dims[1], dims[3],
                         _DTYPE_CODES.get(str(q.dtype), 0), dims[2]], dtype=torch.int64, device=dev)
    table = torch.empty((world, mine.numel()), dtype=torch.int64, device=dev)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(table, mine, group=group)
    else:
        parts = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(parts, mine, group=group)
        table = torch.stack(parts)
    table = table.cpu().tolist()
    for r, row in enumerate(table):
        if row[0] == 0:
            why = repr(error) if r == rank and error is not None else (
                "shard shapes or dtypes disagree" if r == rank else "its local step failed")
            raise SequenceParallelError(r, why)
    ref = table[0][1:5]
    for r, row in enumerate(table):
        if row[1:5] != ref:
            raise SequenceParallelError(r, f"shard (B, H, d, dtype) = {tuple(row[1:5])} differs from "
                                           f"rank 0's {tuple(ref)}")


def prefill_sequence_parallel(q, k, v, group=None, compute: Optional[ShardCompute] = None,
                              blk: int = 128, flags: int = 0):
    """Prefill of this rank's token shard [B,H,N_r,d] of a sequence split over
    the ranks of ``group`` in rank order.  Returns (o_r, state_out_r); the last
    rank's state is the final state of the whole sequence.  Every rank of the
    group must call it: two all-gathers, a 6-integer agreement on the shards
    (a failed local step or a shard of another B, H, d or dtype makes every
    rank raise SequenceParallelError) and the states.  A rank that never
    calls (or has left the group) makes the others fail when the process
    group's timeout expires."""
    import torch
    import torch.distributed as dist

    compute = compute or cuda_compute(blk, flags)
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    delta, error = None, None
    try:
        delta = compute.increment(k, v).contiguous()
    except Exception as e:  # noqa: BLE001 - reported to every rank, then re-raised
        error = e
    _agree(q, k, v, delta, error, group, rank, world)
    if dist.get_backend(group) == "nccl":
        gathered = torch.empty((world,) + tuple(delta.shape), dtype=delta.dtype, device=delta.device)
        dist.all_gather_into_tensor(gathered, delta, group=group)
    else:
        parts = [torch.empty_like(delta) for _ in range(world)]
        dist.all_gather(parts, delta, group=group)
        gathered = torch.stack(parts)
    state_in = compute.prefix(gathered, rank)
    return compute.prefill(q, k, v, state_in)
