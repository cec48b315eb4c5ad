"""Split-KV across GPUs for long sequences.

A sequence too long for one GPU's cache (or whose attention one GPU reads too slowly) is spread
over the ranks of a process group: rank r holds a contiguous range of the sequence's pages in
its own pool.  Every rank runs mla_decode_attn over its own pages, which yields that part's
normalised o_lat and its lse; the parts are all-gathered and mla_merge_partials weighs them by
exp(lse_r - lse), which is the softmax over all the rows ([LP] "Classic attention and the cost
of the KV cache": the output is a softmax-weighted sum over every cached row).

Plumbing only: the partition is host arithmetic on lengths, the exchange is torch.distributed
(NCCL between GPUs), and every arithmetic step runs in the library's kernels.
"""
from __future__ import annotations

import math

import torch

from . import mla_decode_attn, mla_merge_partials

PAGE = 64


def partition_tokens(seq_len: int, world: int, page: int = PAGE) -> list[tuple[int, int]]:
    """Token range [begin, end) of every rank: contiguous whole pages, the sequence's page count
    divided as evenly as possible (rank r takes pages [r P / W, (r + 1) P / W)).  Ranks past the
    last page get an empty range at the end of the sequence."""
    if world < 1 or seq_len < 0:
        raise ValueError("world >= 1 and seq_len >= 0 required")
    n_pages = math.ceil(seq_len / page)
    out = []
    for r in range(world):
        p0, p1 = r * n_pages // world, (r + 1) * n_pages // world
        out.append((min(p0 * page, seq_len), min(p1 * page, seq_len)))
    return out


def local_view(page_table_row: torch.Tensor, seq_len: int, world: int, rank: int,
               page: int = PAGE) -> tuple[torch.Tensor, int]:
    """The rank's share of one sequence described by the sequence's full page-table row: the
    page ids of its pages (in order) and its token count."""
    b, e = partition_tokens(seq_len, world, page)[rank]
    return page_table_row[b // page:(e + page - 1) // page], e - b


def gather_partials(o_local: torch.Tensor, lse_local: torch.Tensor, group=None):
    """All-gather of every rank's (o_lat, lse), stacked in rank order: [world, ...]."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    o_all = [torch.empty_like(o_local) for _ in range(world)]
    l_all = [torch.empty_like(lse_local) for _ in range(world)]
    dist.all_gather(o_all, o_local.contiguous(), group=group)
    dist.all_gather(l_all, lse_local.contiguous(), group=group)
    return torch.stack(o_all), torch.stack(l_all)


def decode_split_kv(d, q_cat, pool, page_table, seq_lens, ws, o_lat, lse=None, group=None,
                    q_lo=None, stream=None):
    """This rank's part of a split-KV decode: attention over the rank's pages (pool, page_table
    and seq_lens describe only those), the gather of every rank's (o_lat, lse), and the merge
    into o_lat / lse, which every rank then holds."""
    o_loc = torch.empty_like(o_lat)
    l_loc = torch.empty(d.batch, d.n_heads, dtype=torch.float32, device=o_lat.device)
    mla_decode_attn(d, q_cat, pool, page_table, seq_lens, o_loc, ws, lse=l_loc, q_lo=q_lo,
                    stream=stream)
    o_all, l_all = gather_partials(o_loc, l_loc, group)
    mla_merge_partials(d, o_all, l_all, o_lat, lse, stream=stream)
