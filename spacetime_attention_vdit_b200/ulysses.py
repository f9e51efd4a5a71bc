"""Ulysses sequence parallelism around the single-GPU attention calls.

"Video Diffusion Models, in depth" (Training; Inference; Failure modes): when
one clip's tokens are split over the GPUs of a node, an all-to-all swaps the
split from tokens to heads, every GPU runs ordinary attention over all tokens
for its share of the heads, and a second all-to-all swaps back.  It is limited
by the head count (the heads must divide over the GPUs) and belongs inside one
NVLink domain.

Rank r of a group of P holds the contiguous token shard [r L/P, (r+1) L/P) of
every [B, L, heads, D] tensor.  Between the two exchanges rank r holds all L
tokens of heads [r H/P, (r+1) H/P).  The exchanges are torch.distributed
all_to_all_single calls (NCCL over NVLink/NVSwitch on GPUs, gloo on CPU); the
attention in between is any single-device call taking and returning
[B, L, heads, D] tensors, by default the library's full attention, so the
kernels stay unchanged.  Divided attention works the same way: after the first
exchange every rank holds whole frames and whole sites.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _world(group):
    return dist.get_world_size(group), dist.get_rank(group)


def tokens_to_heads(x: torch.Tensor, group=None) -> torch.Tensor:
    """[B, L/P, H, D] (this rank's tokens, all heads) -> [B, L, H/P, D] (all
    tokens, this rank's heads)."""
    P, _ = _world(group)
    B, Ls, H, D = x.shape
    if H % P != 0:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    # chunk j of the send buffer goes to rank j: heads [j H/P, (j+1) H/P)
    send = x.reshape(B, Ls, P, H // P, D).permute(2, 0, 1, 3, 4).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # chunk i of the receive buffer came from rank i: its tokens [i L/P, (i+1) L/P)
    return recv.permute(1, 0, 2, 3, 4).reshape(B, P * Ls, H // P, D)


def heads_to_tokens(x: torch.Tensor, group=None) -> torch.Tensor:
    """[B, L, H/P, D] (all tokens, this rank's heads) -> [B, L/P, H, D] (this
    rank's tokens, all heads): the inverse of :func:`tokens_to_heads`."""
    P, _ = _world(group)
    B, L, Hp, D = x.shape
    if L % P != 0:
        raise ValueError(f"{L} tokens do not split over {P} ranks")
    Ls = L // P
    # chunk j goes to rank j: tokens [j L/P, (j+1) L/P)
    send = x.reshape(B, P, Ls, Hp, D).permute(1, 0, 2, 3, 4).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # chunk i came from rank i: heads [i H/P, (i+1) H/P)
    return recv.permute(1, 2, 0, 3, 4).reshape(B, Ls, P * Hp, D)


def attention_ulysses(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, attn=None, group=None) -> torch.Tensor:
    """Attention over a token-sharded clip: this rank's [B, L/P, H, D] shards of
    Q, K and V in, this rank's shard of O out.  ``attn(q, k, v)`` runs on the
    head-sharded tensors [B, L, H/P, D]; the default is the library's full
    attention (pass e.g. ``lambda q, k, v: attn_divided_time(q, k, v, T, HW)``
    for a divided pass)."""
    if attn is None:
        from . import attn_full as attn
    qh = tokens_to_heads(q, group)
    kh = tokens_to_heads(k, group)
    vh = tokens_to_heads(v, group)
    return heads_to_tokens(attn(qh, kh, vh), group)
