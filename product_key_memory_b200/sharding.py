"""Host-side plumbing for running the layer on several GPUs, one process per GPU.

The forward needs no exchange: every (token, head) is independent, so each rank takes
a contiguous range of the batch's tokens against its own replica of the parameters
and writes the matching rows of out, indices and weights ("Large Memory Layers with
Product Keys", gptget.net summary, Methodology: the memory is read per query).

The value backward has one exchange step. A slot's gradient is the sum over every
pick of that slot in the batch, and the picks of one slot come from tokens on any
rank, so the per-rank sums must be added up. Rows are owned in contiguous blocks
(rank r owns rows [r*N/W, (r+1)*N/W) of the n*n-row table): each rank runs
pkm_backward_values on its own tokens into a zeroed fp32 table, then one
reduce-scatter adds the W partial tables and leaves each rank the sum of its own
block. With NCCL the reduce-scatter runs over NVLink; with gloo (tests) on the CPU.

No function here computes any part of the layer; they only split ranges and call
torch.distributed.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist


def token_range(B: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous tokens [start, stop) of rank `rank` out of `world`; the first
    B % world ranks take one token more."""
    if world < 1 or not 0 <= rank < world or B < 0:
        raise ValueError("token_range: need B >= 0 and 0 <= rank < world")
    base, extra = divmod(B, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def row_block(slots: int, world: int, rank: int) -> Tuple[int, int]:
    """Rows [start, stop) of the value table owned by `rank`: equal blocks of
    slots / world rows (slots must be a multiple of world)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("row_block: need 0 <= rank < world")
    if slots % world:
        raise ValueError("row_block: the %d slots do not split into %d equal blocks"
                         % (slots, world))
    per = slots // world
    return rank * per, (rank + 1) * per


def reduce_value_grads(grad_values: torch.Tensor, out: Optional[torch.Tensor] = None,
                       group=None) -> torch.Tensor:
    """Sum the ranks' partial value-gradient tables [n*n][v] (fp32) and return this
    rank's owned block [n*n / world][v] of the sum (row_block). Every rank must call
    it, in the same order as its other collectives."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    slots = grad_values.shape[0]
    start, stop = row_block(slots, world, rank)
    if out is None:
        out = torch.empty((stop - start,) + tuple(grad_values.shape[1:]),
                          dtype=grad_values.dtype, device=grad_values.device)
    dist.reduce_scatter_tensor(out, grad_values.contiguous(), op=dist.ReduceOp.SUM,
                               group=group)
    return out
