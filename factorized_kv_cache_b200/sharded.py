"""Decode of long sequences split across devices by token range.

One process per GPU.  Rank r of a group of G holds, for every sequence, the
contiguous token range ``token_range(L, G, r)`` of its cache, with the tokens'
global positions (B_K is stored rotated at those positions, so nothing about
RoPE changes).  Each rank runs ``tpa_decode_attention_lse`` on its range, the
ranks exchange their (out, lse) pairs (h x (d_h + 1) fp32 per sequence) with
one all-gather, and ``tpa_merge_lse`` combines them: softmax over a disjoint
union of token sets is exact in this form (page "Tensor Product Attention Is
All You Need", section FlashTPA: attention is the softmax over every cached
token; the split-KV reduction applied across devices).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def token_range(length: int, world: int, rank: int) -> tuple[int, int]:
    """[start, end) of rank ``rank``'s share of ``length`` tokens: contiguous, sizes differ by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of {world}")
    base, extra = divmod(length, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def all_gather_partials(out: torch.Tensor, lse: torch.Tensor, group=None):
    """Every rank's (out [..., d_h], lse [...]) stacked in rank order: ([G, ..., d_h], [G, ...])."""
    world = dist.get_world_size(group)
    parts_out = torch.empty((world,) + tuple(out.shape), dtype=out.dtype, device=out.device)
    parts_lse = torch.empty((world,) + tuple(lse.shape), dtype=lse.dtype, device=lse.device)
    dist.all_gather(list(parts_out.unbind(0)), out.contiguous(), group=group)
    dist.all_gather(list(parts_lse.unbind(0)), lse.contiguous(), group=group)
    return parts_out, parts_lse


def decode_token_sharded(cache, q, q_pos, group=None, scale=None, max_len=None, workspace_buf=None):
    """Decode of sequences whose token ranges are spread over the group: this rank's ``cache``
    holds its range; returns the output of the whole range and its lse, on every rank."""
    from . import tpa as T

    out, lse = T.tpa_decode_attention_lse(cache, q, q_pos, scale=scale, max_len=max_len,
                                          workspace_buf=workspace_buf)
    parts_out, parts_lse = all_gather_partials(out, lse, group)
    return T.tpa_merge_lse(parts_out, parts_lse)
