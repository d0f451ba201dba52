"""One Sol-Attn call split across GPUs by heads.

Every (batch, head) slice of the forward is independent: its pooling, its
routing (Eqs. 4-5) and its attention (Eqs. 9-10) read nothing of any other
head.  So one call is split across the ranks of a process group by heads,
rank r taking the contiguous heads [h0_r, h1_r), and needs no exchange inside
the operation.

Video DiTs that run sequence parallel (the Ulysses layout) hold activations
split by tokens instead: rank r has every head of its contiguous token range
[s_r, e_r).  For them the call is bracketed by two all-to-all exchanges:
seq -> head before (each rank sends every other rank that rank's heads of
its own tokens) and head -> seq after (each rank sends back every other
rank's tokens of its own heads).  Both are plain data movement: the output
equals the single-GPU call on the gathered tensors exactly.

The per-rank compute is the library's call on the rank's own device
(`attend`, by default `api.forward`); this module only moves tensors with
torch.distributed (NCCL on GPUs, gloo on CPU).  No shared-memory multicast or
peer-memory operand is involved.
"""

from __future__ import annotations

from typing import Callable, Sequence

import torch
import torch.distributed as dist


def split_range(n: int, world: int, rank: int) -> tuple[int, int]:
    """[start, end) of part `rank` when n items are cut into `world`
    contiguous parts whose sizes differ by at most one (the first n % world
    parts take one more)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def split_sizes(n: int, world: int) -> list[int]:
    return [e - s for s, e in (split_range(n, world, r) for r in range(world))]


def _world_rank(group):
    return dist.get_world_size(group), dist.get_rank(group)


def _exchange(send: list[torch.Tensor], recv_shapes: list[tuple], group) -> list[torch.Tensor]:
    """One all-to-all: send[p] goes to rank p; returns the tensors received
    from every rank, of the given shapes.  The pieces travel as one flat
    buffer with per-rank split sizes (all_to_all_single, which NCCL and gloo
    both provide, uneven splits included)."""
    flat_in = torch.cat([t.reshape(-1) for t in send])
    sizes_in = [t.numel() for t in send]
    sizes_out = [int(torch.Size(sh).numel()) for sh in recv_shapes]
    flat_out = torch.empty(sum(sizes_out), dtype=flat_in.dtype, device=flat_in.device)
    dist.all_to_all_single(flat_out, flat_in, output_split_sizes=sizes_out, input_split_sizes=sizes_in,
                           group=group)
    return [piece.view(sh) for piece, sh in zip(torch.split(flat_out, sizes_out), recv_shapes)]


def seq_to_head(x: torch.Tensor, heads: int, L: int, group=None) -> torch.Tensor:
    """[b, heads, L_r, d] (this rank's tokens, every head) ->
    [b, H_r, L, d] (every token, this rank's heads), by one all-to-all."""
    world, rank = _world_rank(group)
    b, H, Lr, d = x.shape
    if H != heads or Lr != split_sizes(L, world)[rank]:
        raise ValueError(f"expected [b, {heads}, {split_sizes(L, world)[rank]}, d], got {tuple(x.shape)}")
    hs = split_sizes(heads, world)
    ls = split_sizes(L, world)
    send, off = [], 0
    for p in range(world):  # rank p's heads of my tokens
        send.append(x[:, off:off + hs[p]])
        off += hs[p]
    recv = _exchange(send, [(b, hs[rank], ls[q], d) for q in range(world)], group)
    return torch.cat(recv, dim=2)


def head_to_seq(o: torch.Tensor, heads: int, L: int, group=None) -> torch.Tensor:
    """[b, H_r, L, d] (every token, this rank's heads) ->
    [b, heads, L_r, d] (this rank's tokens, every head): the inverse of
    seq_to_head."""
    world, rank = _world_rank(group)
    b, Hr, Lf, d = o.shape
    hs = split_sizes(heads, world)
    ls = split_sizes(L, world)
    if Hr != hs[rank] or Lf != L:
        raise ValueError(f"expected [b, {hs[rank]}, {L}, d], got {tuple(o.shape)}")
    send, off = [], 0
    for p in range(world):  # my heads of rank p's tokens
        send.append(o[:, :, off:off + ls[p]])
        off += ls[p]
    recv = _exchange(send, [(b, hs[q], ls[rank], d) for q in range(world)], group)
    return torch.cat(recv, dim=1)


def default_attend(q, k, v, beta, block):
    from video_diffusion_b200 import api
    return api.forward(q, k, v, beta, block)


def forward_heads(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, beta: float, block=128,
                  attend: Callable = default_attend) -> torch.Tensor:
    """The rank's share of a head-split call: q, k, v hold this rank's heads
    with every token ([b, H_r, L, d]); returns their output."""
    if q.shape[1] == 0:
        return torch.empty_like(q)
    return attend(q, k, v, beta, block)


def forward_ulysses(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, beta: float, heads: int, L: int,
                    block=128, group=None, attend: Callable = default_attend) -> torch.Tensor:
    """Sequence-parallel call: q, k, v are this rank's token range of every
    head ([b, heads, L_r, d], ranges from split_range(L, world, rank)).
    Exchanges to head shards, runs this rank's heads, exchanges back; returns
    this rank's token range of the output, every head."""
    qh = seq_to_head(q, heads, L, group)
    kh = seq_to_head(k, heads, L, group)
    vh = seq_to_head(v, heads, L, group)
    oh = forward_heads(qh, kh, vh, beta, block, attend)
    return head_to_seq(oh, heads, L, group)


def shard_heads(x: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """This rank's heads of a full [b, H, L, d] tensor (a view)."""
    h0, h1 = split_range(x.shape[1], world, rank)
    return x[:, h0:h1]


def shard_tokens(x: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """This rank's token range of a full [b, H, L, d] tensor (a view)."""
    s0, s1 = split_range(x.shape[2], world, rank)
    return x[:, :, s0:s1]


def exchange_bytes(shape: Sequence[int], element_size: int, world: int, rank: int) -> int:
    """Bytes this rank sends to other ranks in one seq -> head exchange of one
    [b, H, L, d] tensor (the head -> seq exchange of the output moves as many)."""
    b, H, L, d = shape
    hs, ls = split_sizes(H, world), split_sizes(L, world)
    return sum(b * hs[p] * ls[rank] * d * element_size for p in range(world) if p != rank)
