"""Context split of long sequences over the ranks of a process group.

Plumbing around two C calls (include/mla.h): every rank runs
mla_decode_attn_partial on its window of every sequence's pages, the ranks'
(o_lat, lse) partials are all-gathered (torch.distributed: NCCL between GPUs),
and every rank merges them with mla_merge_ranks.  The partials are the only
data the ranks exchange: d_c + 1 fp32 values per query row and rank.

mla_merge_ranks reads each partial through a plain pointer, so a caller that
maps its peers' partial buffers into the process (NVLink peer access) can hand
it the peers' pointers instead and skip the gather: the exchange then happens
inside the merge kernel.  This module implements the gather form.
"""
from __future__ import annotations

from . import mla_decode_attn_partial, mla_merge_ranks


def gather_partials(o_lat, lse, group=None):
    """All-gather this rank's partials; returns (o_lats, lses), lists indexed by rank."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    o_lats = [torch.empty_like(o_lat) for _ in range(world)]
    lses = [torch.empty_like(lse) for _ in range(world)]
    dist.all_gather(o_lats, o_lat.contiguous(), group=group)
    dist.all_gather(lses, lse.contiguous(), group=group)
    return o_lats, lses


def context_split_decode(dims, q_lat, pool, page_table, seq_lens, w_uv, workspace, out, lse=None,
                         dev_status=None, group=None, stream=None) -> None:
    """mla_decode_attn with the key range of every sequence split over the group's
    ranks: this rank attends over its window, the partials are gathered, and the
    merged result (out, lse) is written on every rank.  Every rank holds the whole
    q_lat, page table and lengths; only the page-table entries of its own window
    are read, so its pool needs to hold only those pages.  The calls run on
    `stream`, which must be torch's current stream when the group uses NCCL (the
    gather is ordered after the partial on that stream)."""
    import torch
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, nq, H = q_lat.shape[0], q_lat.shape[1], q_lat.shape[2]
    o_lat = torch.empty((B, nq, H, dims.d_c), dtype=torch.float32, device=q_lat.device)
    part_lse = torch.empty((B, nq, H), dtype=torch.float32, device=q_lat.device)
    mla_decode_attn_partial(dims, q_lat, pool, page_table, seq_lens, rank, world, workspace, o_lat, part_lse,
                            dev_status=dev_status, stream=stream)
    o_lats, lses = gather_partials(o_lat, part_lse, group)
    mla_merge_ranks(dims, o_lats, lses, w_uv, out, lse, stream=stream)
