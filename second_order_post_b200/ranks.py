"""A model's sublayers spread over ranks (one process per GPU).

The mixed-precision allocator ranks every sublayer of the model by its
sensitivity tr(H_G)·tr(H_X) [wmrh §六]. Everything else in a sublayer's
quantization is local to it. So each rank quantizes its own share of the
sublayers with its own engine, and the only exchange is the scores. The
greedy allocator needs every sublayer's score and size, so these are
gathered once (one collective of 2 x n_sublayers numbers). Every rank then
runs the same host allocator (kronq_allocate_bits) on the same arrays, and so
gets the same bit widths without a second exchange.

The collectives are torch.distributed calls on whatever process group the
caller set up (NCCL over NVLink for GPUs, gloo on CPU).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import kronq as K


def my_sublayers(n: int, world: int, rank: int) -> range:
    """This rank's contiguous share of the sublayer indices [0, n); the
    shares of all ranks partition [0, n) and differ in size by at most 1."""
    if n < 0 or world <= 0 or not 0 <= rank < world:
        raise ValueError("need n >= 0, world > 0 and 0 <= rank < world")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def _coll_device(group, device):
    if device is not None:
        return torch.device(device)
    if dist.get_backend(group) == "nccl":
        return torch.device("cuda", torch.cuda.current_device())
    return torch.device("cpu")


def gather_scores(local_scores, local_numel, n_total: int, group=None, device=None):
    """All ranks' (score, numel) in global sublayer order. Rank r contributes
    the entries my_sublayers(n_total, world, r); each entry of the result is
    written by exactly one rank, so a sum-reduction of zero-filled fp64
    buffers is an exact gather (sizes up to 2^53)."""
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    mine = my_sublayers(n_total, world, rank)
    if len(local_scores) != len(mine) or len(local_numel) != len(mine):
        raise ValueError(f"rank {rank} holds sublayers {mine.start}..{mine.stop - 1}: "
                         f"expected {len(mine)} scores and sizes")
    buf = torch.zeros(2, n_total, dtype=torch.float64, device=_coll_device(group, device))
    if len(mine):
        buf[0, mine.start:mine.stop] = torch.tensor([float(s) for s in local_scores],
                                                    dtype=torch.float64)
        buf[1, mine.start:mine.stop] = torch.tensor([float(m) for m in local_numel],
                                                    dtype=torch.float64)
    dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
    host = buf.cpu()
    return host[0].tolist(), [int(m) for m in host[1].tolist()]


def allocate_bits_across_ranks(local_scores, local_numel, n_total: int,
                               avg_budget: float, group=None, device=None):
    """Bit widths of all n_total sublayers (global order), the same on every
    rank: the scores are gathered, then kronq_allocate_bits runs locally."""
    scores, numel = gather_scores(local_scores, local_numel, n_total, group, device)
    return K.kronq_allocate_bits(scores, numel, avg_budget)


def max_over_ranks(x: float, group=None, device=None) -> float:
    """The largest x over the ranks of the group (a timing's max over ranks)."""
    t = torch.tensor([float(x)], dtype=torch.float64, device=_coll_device(group, device))
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
