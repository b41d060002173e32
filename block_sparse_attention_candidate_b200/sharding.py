"""Multi-GPU partitioning of one attention layer (one process per GPU).

Every stage of the path is independent per (batch, head): the candidate set
is geometry shared by all heads, the pooled scores and the selection of a
head read only that head's Q and K, and the attention of a head reads only its
own Q, K, V and kept-block lists.  A layer therefore splits over ranks by
heads with no exchange at all: rank r runs the unchanged library calls on its
contiguous range of heads.

When a caller's activations arrive split over the sequence instead (the
sequence parallelism of a multi-GPU video model), one all-to-all regroups
them by heads before the calls and one regroups the outputs afterwards: the
Ulysses-style exchange, through torch.distributed (NCCL over NVLink on GPUs,
gloo in the host tests).  These are collectives around the hot path, not in
it; nothing here computes any part of the method.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist


def head_range(heads: int, world: int, rank: int) -> Tuple[int, int]:
    """[h0, h1) of the heads rank `rank` of `world` owns: contiguous, sizes
    differing by at most one, lower ranks taking the extra heads."""
    if heads < 1 or world < 1 or not 0 <= rank < world:
        raise ValueError("need heads >= 1, world >= 1 and 0 <= rank < world")
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def head_shard(x: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """The heads of `x` ([B, H, N, ...]) that `rank` owns, as a contiguous tensor."""
    h0, h1 = head_range(x.shape[1], world, rank)
    return x[:, h0:h1].contiguous()


def seq_to_head_shards(x: torch.Tensor, group: Optional[dist.ProcessGroup] = None) -> torch.Tensor:
    """[B, H, N/W, D] (this rank's sequence slice, all heads) -> [B, H/W, N, D]
    (this rank's heads, the whole sequence).  H and N must divide by the world
    size W; rank r holds tokens [r N/W, (r+1) N/W) before and heads
    [r H/W, (r+1) H/W) after."""
    world = dist.get_world_size(group)
    B, H, n_loc, D = x.shape
    if H % world:
        raise ValueError("heads must divide by the world size")
    hw = H // world
    # chunk s of the send buffer goes to rank s: this rank's tokens of rank s's heads
    send = x.reshape(B, world, hw, n_loc, D).permute(1, 0, 2, 3, 4).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv chunk s: rank s's tokens of this rank's heads
    return recv.permute(1, 2, 0, 3, 4).reshape(B, hw, world * n_loc, D).contiguous()


def head_to_seq_shards(y: torch.Tensor, group: Optional[dist.ProcessGroup] = None) -> torch.Tensor:
    """Inverse of seq_to_head_shards: [B, H/W, N, ...] (this rank's heads) ->
    [B, H, N/W, ...] (this rank's tokens, all heads).  Works for O ([..., D])
    and for the LSE ([B, H/W, N], given as [B, H/W, N, 1])."""
    world = dist.get_world_size(group)
    B, hw, N, D = y.shape
    if N % world:
        raise ValueError("tokens must divide by the world size")
    n_loc = N // world
    # chunk s goes to rank s: this rank's heads over rank s's tokens
    send = y.reshape(B, hw, world, n_loc, D).permute(2, 0, 1, 3, 4).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv chunk s: rank s's heads over this rank's tokens
    return recv.permute(1, 0, 2, 3, 4).reshape(B, world * hw, n_loc, D).contiguous()
