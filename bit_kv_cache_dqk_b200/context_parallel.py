"""Context-parallel decode: one sequence's cached pages spread over ranks.

Each rank holds a contiguous range of every sequence's logical pages (its own
pool and page table), decodes them with ``dqk_decode_partial`` into one
(m, l, o) record per (sequence, query head), the ranks all-gather the records
over NCCL, and ``dqk_merge_partials`` forms the output on every rank.  The
pages say nothing about how the context is split or where; the merge is the
log-sum-exp combination of partial softmax results that the single-GPU decode
already uses between its CTAs, carried across GPUs.  The exchange is
B * Hq * (d + 2) * 4 bytes per rank, so it is latency-bound and NCCL's
all-gather is the whole of it.

Host logic only: every step of the decode and the merge runs in libdualqk.
"""
from __future__ import annotations

import numpy as np

from . import dualqk as Q

PAGE = 16


def page_range(num_pages: int, rank: int, world: int) -> tuple[int, int]:
    """Logical pages [p0, p1) of a sequence with num_pages pages that rank
    `rank` of `world` holds: contiguous, sizes differing by at most one."""
    return (rank * num_pages) // world, ((rank + 1) * num_pages) // world


def rank_view(lens: np.ndarray, table: np.ndarray, rank: int, world: int):
    """(token counts [batch] int32, page table [batch][max_pages_r] int32) of
    the part of each sequence rank `rank` holds, from the full lengths and the
    full logical->physical page table.  Only a sequence's last page may be
    partly filled, so a range's token count is its pages' tokens clipped to
    the sequence length."""
    lens = np.asarray(lens, np.int64)
    table = np.asarray(table, np.int32)
    npages = (lens + PAGE - 1) // PAGE
    spans = [page_range(int(n), rank, world) for n in npages]
    width = max([p1 - p0 for p0, p1 in spans] + [1])
    sub = np.full((len(lens), width), -1, np.int32)
    sub_lens = np.zeros(len(lens), np.int32)
    for b, (p0, p1) in enumerate(spans):
        sub[b, :p1 - p0] = table[b, p0:p1]
        sub_lens[b] = max(0, min(int(lens[b]), p1 * PAGE) - p0 * PAGE)
    return sub_lens, sub


def decode(layer, q, q_dtype, batch, hq, head_dim, seq_lens, page_table, max_pages, sparsity_pct, out,
           sel_out, workspace, workspace_bytes, group=None):
    """Context-parallel decode of this rank's share (seq_lens, page_table as
    returned by rank_view, on the device) into out [batch][Hq][d] fp32, the
    same on every rank of `group`.  Runs on the current stream, which NCCL's
    collective orders itself against."""
    import torch
    part = torch.empty((batch, hq, head_dim + 2), dtype=torch.float32, device=out.device)
    Q.dqk_decode_partial(layer, q, q_dtype, batch, seq_lens, page_table, max_pages, sparsity_pct, part,
                         sel_out, workspace, workspace_bytes)
    parts = gather_records(part, group)
    Q.dqk_merge_partials(parts, parts.shape[0], batch, hq, head_dim, out)
    return out


def gather_records(part, group=None):
    """[world][...] stack of every rank's records, in rank order (one flat
    all-gather; the record layout is the same on every rank)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return part.unsqueeze(0)
    world = dist.get_world_size(group)
    flat = torch.empty(world * part.numel(), dtype=part.dtype, device=part.device)
    dist.all_gather_into_tensor(flat, part.contiguous().reshape(-1), group=group)
    return flat.view((world,) + tuple(part.shape))
