"""Sequence-parallel attention over several GPUs by head sharding (Ulysses).

"Vortex Research Agenda", Novel Architecture (ragged Ulysses) and "H3 Performance
Roadmap", distributed execution: when one sequence is spread over N ranks by tokens,
attention needs every token of a head on one rank.  One all-to-all turns the token
shards of Q, K and V into head shards (every token, H/N heads per rank); each rank runs
the attention of its heads on its own GPU; a second all-to-all turns the output back
into token shards.  The heads are independent problems, so the result is bit for bit
that of one GPU running all heads.

Layout: rank r holds tokens [offsets[r], offsets[r] + counts[r]) of [B, T, H, D], the
consecutive shards of ``token_counts(T, N)`` (the first T mod N ranks one token more:
the ragged split).  H must be a multiple of N; rank r owns heads [r H/N, (r+1) H/N).

The exchanges go through ``torch.distributed.all_to_all_single`` on the process group
(NCCL over NVLink on GPUs; gloo in the CPU tests), moving raw bytes so that any element
type travels unchanged.  Q, K and V share one exchange.  This module holds only the
data movement; the attention itself is the library's (``h3attn_forward_ex``) or a
function the caller passes.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch
import torch.distributed as dist


def token_counts(T: int, world: int) -> list:
    """Tokens of each rank's shard: T // world, the first T % world ranks one more."""
    if T < world:
        raise ValueError(f"{T} tokens cannot be spread over {world} ranks")
    return [T // world + (1 if r < T % world else 0) for r in range(world)]


def _bytes(x: torch.Tensor) -> torch.Tensor:
    return x.contiguous().view(-1).view(torch.uint8)


def _group_info(group):
    return dist.get_world_size(group), dist.get_rank(group)


def seq_to_head(xs: Sequence[torch.Tensor], T: int, group=None) -> list:
    """Token shards -> head shards, for several tensors in one all-to-all.

    xs: tensors [B, T_r, H, D] of this rank (same shape and dtype), T_r = token_counts(T, N)[r].
    Returns, per input, [B, T, H/N, D]: every token of this rank's H/N heads (contiguous).
    """
    world, rank = _group_info(group)
    n = len(xs)
    B, Tr, H, D = xs[0].shape
    counts = token_counts(T, world)
    if Tr != counts[rank]:
        raise ValueError(f"rank {rank} holds {Tr} tokens, its shard of {T} is {counts[rank]}")
    if H % world:
        raise ValueError(f"{H} heads do not split over {world} ranks")
    for x in xs:
        if x.shape != xs[0].shape or x.dtype != xs[0].dtype:
            raise ValueError("the tensors of one exchange need one shape and dtype")
    Hn = H // world
    esz = xs[0].element_size()
    # send buffer [N, n, B, T_r, Hn, D]: the block for rank d holds its heads of every
    # tensor (one strided copy per tensor)
    send = torch.empty((world, n, B, Tr, Hn, D), dtype=xs[0].dtype, device=xs[0].device)
    for i, x in enumerate(xs):
        send[:, i].copy_(x.reshape(B, Tr, world, Hn, D).permute(2, 0, 1, 3, 4))
    recv = torch.empty(n * B * T * Hn * D * esz, dtype=torch.uint8, device=xs[0].device)
    dist.all_to_all_single(recv, _bytes(send), [n * B * c * Hn * D * esz for c in counts],
                           [n * B * Tr * Hn * D * esz] * world, group=group)
    # block from source rank s: [n, B, T_s, Hn, D]; join along the tokens in rank order
    parts = torch.split(recv, [n * B * c * Hn * D * esz for c in counts])
    blocks = [p.view(xs[0].dtype).view(n, B, c, Hn, D) for p, c in zip(parts, counts)]
    full = blocks[0] if world == 1 else torch.cat(blocks, dim=2)     # [n, B, T, Hn, D]
    return [full[i] for i in range(n)]


def head_to_seq(o: torch.Tensor, T: int, group=None) -> torch.Tensor:
    """Head shard -> token shard: o [B, T, H/N, D] (every token of this rank's heads)
    to [B, T_r, H, D] (this rank's tokens of every head)."""
    world, rank = _group_info(group)
    B, T_, Hn, D = o.shape
    if T_ != T:
        raise ValueError(f"head shard holds {T_} tokens, expected {T}")
    counts = token_counts(T, world)
    Tr = counts[rank]
    esz = o.element_size()
    # send buffer: the block for rank d is its token range of every batch item, [B, T_d, Hn, D]
    if B == 1:
        send = _bytes(o)
    else:
        offs = [sum(counts[:d]) for d in range(world)]
        send = torch.cat([_bytes(o[:, a:a + c]) for a, c in zip(offs, counts)])
    recv = torch.empty(world * B * Tr * Hn * D * esz, dtype=torch.uint8, device=o.device)
    dist.all_to_all_single(recv, send, [B * Tr * Hn * D * esz] * world,
                           [B * c * Hn * D * esz for c in counts], group=group)
    # block from source rank s: its heads [s Hn, (s+1) Hn) of this rank's tokens
    blocks = recv.view(o.dtype).view(world, B, Tr, Hn, D)
    return blocks.permute(1, 2, 0, 3, 4).reshape(B, Tr, world * Hn, D)


def _library_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, softmax_scale: float) -> torch.Tensor:
    from . import h3attn_check_status, h3attn_forward_ex, new_workspace, OK, H3AttnError
    B, T, Hn, D = q.shape
    ws = new_workspace(B, T, T, Hn, device=q.device)
    out = torch.empty_like(q)
    h3attn_forward_ex(q, k, v, softmax_scale, out, ws)
    st = h3attn_check_status(ws)
    if st != OK:
        raise H3AttnError(st, "ulysses attention")
    return out


def ulysses_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, T: int, softmax_scale: float,
                      group=None, attend: Optional[Callable] = None) -> torch.Tensor:
    """Attention of one sequence spread over the ranks of ``group`` by tokens.

    q, k, v: this rank's token shard [B, T_r, H, D] of the sequence of T tokens.  The
    attention of this rank's H/N heads runs on its GPU through the library
    (``attend(q, k, v, softmax_scale)`` replaces it, e.g. in CPU tests).  Returns the
    output of this rank's tokens, [B, T_r, H, D].
    """
    qh, kh, vh = seq_to_head([q, k, v], T, group)
    o = (attend or _library_attention)(qh, kh, vh, softmax_scale)
    return head_to_seq(o, T, group)
