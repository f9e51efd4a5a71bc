"""Divided attention over a clip whose frames are split across GPUs.

Divided attention ("Video and 3D Generation" cheatsheet, "Divided attention";
"Video as a 3D signal", "Patches and attention") runs a time pass over the T
tokens of each spatial site and a space pass over the HW tokens of each frame.
When one clip is spread over P ranks of a node for sequence parallelism ("Video
Diffusion Models, in depth", Inference: several GPUs working on one clip) by
frames, rank r holding frames [r T/P, (r+1) T/P) of every [B, T*HW, heads, D]
tensor, the space pass needs nothing from the other ranks: each frame is whole.
The time pass needs every frame of a site, so an all-to-all swaps the split
from frames to sites (rank r then holds sites [r HW/P, (r+1) HW/P) of all T
frames), the time pass runs on that shard, and a second all-to-all swaps back.
The exchanges are torch.distributed all_to_all_single calls (NCCL over
NVLink/NVSwitch on GPUs, gloo on CPU); the passes in between are the library's
single-GPU calls, unchanged.  Layouts stay frame-major throughout: a shard of
frames is a contiguous run of tokens, a shard of sites is T frames of HW/P
tokens each.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _split(T: int, HW: int, group):
    P = dist.get_world_size(group)
    if T % P != 0 or HW % P != 0:
        raise ValueError(f"{T} frames and {HW} sites must both split over {P} ranks")
    return P, T // P, HW // P


def frames_to_sites(x: torch.Tensor, T: int, HW: int, group=None) -> torch.Tensor:
    """[B, (T/P)*HW, H, D] (this rank's frames, all sites) -> [B, T*(HW/P), H, D]
    (all frames, this rank's sites), both frame-major."""
    P, Tl, HWl = _split(T, HW, group)
    B, Ls, H, D = x.shape
    if Ls != Tl * HW:
        raise ValueError(f"{Ls} tokens on this rank, expected {Tl} frames x {HW} sites")
    # chunk j of the send buffer goes to rank j: this rank's frames at sites [j HW/P, (j+1) HW/P)
    send = x.reshape(B, Tl, P, HWl, H, D).permute(2, 0, 1, 3, 4, 5).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # chunk i came from rank i: frames [i T/P, (i+1) T/P) at this rank's sites
    return recv.permute(1, 0, 2, 3, 4, 5).reshape(B, T * HWl, H, D)


def sites_to_frames(x: torch.Tensor, T: int, HW: int, group=None) -> torch.Tensor:
    """[B, T*(HW/P), H, D] (all frames, this rank's sites) -> [B, (T/P)*HW, H, D]
    (this rank's frames, all sites): the inverse of :func:`frames_to_sites`."""
    P, Tl, HWl = _split(T, HW, group)
    B, Lx, H, D = x.shape
    if Lx != T * HWl:
        raise ValueError(f"{Lx} tokens on this rank, expected {T} frames x {HWl} sites")
    # chunk j goes to rank j: frames [j T/P, (j+1) T/P) of this rank's sites
    send = x.reshape(B, P, Tl, HWl, H, D).permute(1, 0, 2, 3, 4, 5).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # chunk i came from rank i: this rank's frames at sites [i HW/P, (i+1) HW/P)
    return recv.permute(1, 2, 0, 3, 4, 5).reshape(B, Tl * HW, H, D)


def divided_attention_frame_sharded(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, T: int, HW: int,
                                    time_attn=None, space_attn=None, group=None):
    """Both passes of divided attention for this rank's frames of a clip: Q, K, V
    are [B, (T/P)*HW, heads, D] shards; returns (time-pass output, space-pass
    output), each the same shard of what the single-GPU calls return for the
    whole clip.  ``time_attn(q, k, v, T, sites)`` and ``space_attn(q, k, v,
    frames, HW)`` default to the library's kernels."""
    P, Tl, HWl = _split(T, HW, group)
    if time_attn is None:
        from . import attn_divided_time as time_attn
    if space_attn is None:
        from . import attn_divided_space as space_attn
    o_space = space_attn(q, k, v, Tl, HW)
    qs, ks, vs = (frames_to_sites(x, T, HW, group) for x in (q, k, v))
    o_time = sites_to_frames(time_attn(qs, ks, vs, T, HWl), T, HW, group)
    return o_time, o_space
