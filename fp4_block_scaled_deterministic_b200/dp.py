"""Data-parallel plumbing of the linear-layer passes: one process per GPU, tokens
sharded across ranks, weights replicated.

Fprop and Dgrad need no exchange (each rank's tokens are independent and every rank
quantises the same W identically). Wgrad contracts over the tokens, so each rank
produces a partial dW; the one exchange of the path is the sum of those partials,
issued per projection right after its Wgrad GEMM so that it overlaps the next
projection. Token blocks of the column-wise quantisation (16/32 tokens) never
straddle ranks because every shard is a multiple of 32 tokens.

For NVFP4 the tensor scale of an activation is per rank by default; `allreduce_amax_`
makes it global (a max over ranks of the amax cells) when bit-identical codes across
any world size are wanted.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def token_shard(total_tokens: int, rank: int, world: int, block: int = 32) -> tuple[int, int]:
    """[start, stop) of this rank's tokens; shards are equal and multiples of `block`."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    if total_tokens % (world * block) != 0:
        raise ValueError(f"{total_tokens} tokens do not split into {world} shards of "
                         f"whole {block}-token blocks")
    per = total_tokens // world
    return rank * per, (rank + 1) * per


def allreduce_wgrad(dW: torch.Tensor, group=None, async_op: bool = True):
    """Sum the partial weight gradients of all ranks in place. The sum's rounding
    order is that of the collective's algorithm: NCCL picks it from the message size
    and the topology (ring, tree or in-switch NVLS), the same choice on every run of
    one configuration; NCCL_ALGO=Ring pins one fixed order across configurations."""
    return dist.all_reduce(dW, op=dist.ReduceOp.SUM, group=group, async_op=async_op)


def allreduce_amax_(amax: torch.Tensor, group=None) -> torch.Tensor:
    """Max over ranks of NVFP4 amax cells, in place."""
    dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return amax


def max_over_ranks(value: float, device, group=None) -> float:
    """The slowest rank's time: every multi-rank number is reported as this max."""
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
