"""Data-parallel plumbing of the linear-layer passes: one process per GPU, tokens
sharded across ranks, weights replicated.

Fprop and Dgrad need no exchange (each rank's tokens are independent and every rank
quantises the same W identically). Wgrad contracts over the tokens, so each rank
produces a partial dW; the one exchange of the path is the sum of those partials,
issued per projection right after its Wgrad GEMM so that it overlaps the next
projection. Token blocks of the column-wise quantisation (16/32 tokens) never
straddle ranks because every shard is a multiple of 32 tokens.

The sum is taken in a fixed order. Wgrad is the pass whose numerics the MXFP4
pre-training summary singles out (Findings section 1), so its result should not
depend on which reduction algorithm a collective library picks for a message size
or topology. `allreduce_wgrad` therefore moves data only (an all-to-all of dW chunks
and an all-gather) and adds the P partials of each chunk itself, in rank order
0, 1, ..., P-1, one fp32 addition per element and step: the result is bit-identical
on every run and for every NCCL algorithm, protocol and topology, and equals that
rank-ordered sum computed on one device.

For NVFP4 the tensor scale of an activation is per rank by default; `allreduce_amax_`
makes it global (a max over ranks of the amax cells) when bit-identical codes across
any world size are wanted.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

REDUCTION = ("dW sum in rank order: all-to-all of P chunks, local fp32 sum of the P "
             "partials in rank order 0..P-1, all-gather (independent of the collective "
             "library's algorithm)")

_side_streams: dict = {}


def token_shard(total_tokens: int, rank: int, world: int, block: int = 32) -> tuple[int, int]:
    """[start, stop) of this rank's tokens; shards are equal and multiples of `block`."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    if total_tokens % (world * block) != 0:
        raise ValueError(f"{total_tokens} tokens do not split into {world} shards of "
                         f"whole {block}-token blocks")
    per = total_tokens // world
    return rank * per, (rank + 1) * per


def rank_ordered_sum_(parts: torch.Tensor) -> torch.Tensor:
    """Sum of parts[0], parts[1], ... in that order (elementwise, one rounding per
    addition); parts has the rank as its leading dimension."""
    acc = parts[0].clone()
    for j in range(1, parts.shape[0]):
        acc.add_(parts[j])
    return acc


class _Done:
    """Handle of a finished (or stream-ordered) reduction."""

    def __init__(self, event=None):
        self.event = event

    def wait(self):
        if self.event is not None:
            torch.cuda.current_stream(self.event.device).wait_event(self.event)

    def is_completed(self):
        return self.event is None or self.event.query()


def _reduce_in_place(flat: torch.Tensor, world: int, group) -> None:
    n = flat.numel()
    chunk = n // world
    recv = torch.empty_like(flat)
    dist.all_to_all_single(recv, flat, group=group)  # recv[i] = rank i's copy of my chunk
    acc = rank_ordered_sum_(recv.view(world, chunk))
    dist.all_gather_into_tensor(flat, acc, group=group)  # chunk r of dW from rank r


def allreduce_wgrad(dW: torch.Tensor, group=None, async_op: bool = True):
    """Replace every rank's partial dW (contiguous) by the sum of all ranks' partials,
    added in rank order (see the module docstring). dW.numel() must be a multiple of
    the world size. On CUDA the exchange and the sum run on a side stream that starts
    after the work already queued on the current stream; with async_op the returned
    handle's wait() orders the caller's current stream after it, otherwise the current
    stream is ordered after it before returning."""
    world = dist.get_world_size(group)
    if world == 1:
        return _Done()
    if not dW.is_contiguous():
        raise ValueError("dW must be contiguous")
    flat = dW.view(-1)
    if flat.numel() % world:
        raise ValueError(f"dW of {flat.numel()} elements does not split into {world} chunks")
    if not flat.is_cuda:
        _reduce_in_place(flat, world, group)
        return _Done()
    dev = flat.device
    side = _side_streams.get(dev)
    if side is None:
        side = _side_streams[dev] = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        _reduce_in_place(flat, world, group)
        done = torch.cuda.Event()
        done.record(side)
    flat.record_stream(side)
    handle = _Done(done)
    if not async_op:
        handle.wait()
    return handle


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
