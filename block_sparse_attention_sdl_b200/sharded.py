"""Mask selection for a sequence whose heads are split over ranks.

The head-adaptive global budget of the Step-dLLM abstract ranks the block
scores of all heads of a sequence together.  When attention is sharded over
GPUs by heads (rank r holds a contiguous range of whole KV-head groups), every
step of the path stays local except that ranking: the radix select needs the
digit histograms of all ranks (one sum over ranks per pass) and, for the tie
order, the per-rank counts of keys above and at the threshold (one gather).
After that each rank writes its own part of the mask, which is exactly its
part of the single-device selection.

The kernels are the library's (`sdl_select_shard_*`); this module only moves
the small histograms and totals between ranks, by default with
`torch.distributed` (NCCL on GPUs).
"""
from __future__ import annotations

from . import (SDL_SELECT_PASSES, select_shard_count, select_shard_finish, select_shard_hist,
               select_shard_pass, select_shard_workspace_bytes)


def head_range(H: int, H_kv: int, rank: int, world: int) -> tuple[int, int]:
    """[h0, h1) of the query heads rank ``rank`` of ``world`` holds: whole KV-head
    groups, split evenly (H_kv must be a multiple of ``world``)."""
    if H_kv % world or H % H_kv:
        raise ValueError("heads must split into whole KV-head groups per rank")
    per = H // world
    return rank * per, (rank + 1) * per


class CudaStages:
    """The library's staged selection on this rank's scores [B, H_local, nb, nb]."""

    def __init__(self, scores, sparsity: float, block: int, L: int, heads_total: int,
                 workspace=None, stream=None):
        import torch
        self.scores, self.sparsity, self.block, self.L = scores, sparsity, block, L
        self.heads_total, self.stream = heads_total, stream
        n = select_shard_workspace_bytes(scores, block, L)
        if workspace is None:
            workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=scores.device)
        self.ws = workspace

    def hist_pass(self, p: int):
        select_shard_pass(self.scores, self.sparsity, self.block, self.L, self.heads_total, p,
                          self.ws, self.stream)

    def hist(self, p: int):
        return select_shard_hist(self.ws, self.scores, self.block, self.L, p)

    def count(self):
        return select_shard_count(self.scores, self.sparsity, self.block, self.L,
                                  self.heads_total, self.ws, stream=self.stream)

    def finish(self, offsets, row_ptr=None, col_idx=None, want_mask: bool = False):
        return select_shard_finish(self.scores, self.sparsity, self.block, self.L,
                                   self.heads_total, offsets, self.ws, row_ptr=row_ptr,
                                   col_idx=col_idx, want_mask=want_mask, stream=self.stream)


def torch_collectives(group=None):
    """(all_reduce, all_gather) over ``group`` with torch.distributed: the sum in
    place, and the list of every rank's tensor."""
    import torch
    import torch.distributed as dist

    def all_reduce(t):
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)

    def all_gather(t):
        out = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
        dist.all_gather(out, t, group=group)
        return out

    return all_reduce, all_gather


def shard_offsets(gathered, rank: int):
    """int64 [B, 2] for the finishing stage from every rank's totals [B, 2]: keys above
    the threshold over all ranks, and threshold ties held by the ranks before ``rank``."""
    import torch
    g = torch.stack(list(gathered))  # [W, B, 2]
    return torch.stack([g[:, :, 0].sum(0), g[:rank, :, 1].sum(0)], dim=1).contiguous()


def select_mask_sharded(scores, sparsity: float, block: int, L: int, heads_total: int,
                        rank: int, *, group=None, all_reduce=None, all_gather=None, stages=None,
                        row_ptr=None, col_idx=None, want_mask: bool = False, stream=None):
    """This rank's (row_ptr, col_idx, mask) of the global selection over ``heads_total``
    heads, from its scores fp32 [B, H_local, nb, nb] (its heads, in rank order).  Every
    rank of the group calls it with the same sparsity, block, L and heads_total."""
    if all_reduce is None or all_gather is None:
        all_reduce, all_gather = torch_collectives(group)
    st = stages if stages is not None else CudaStages(scores, sparsity, block, L, heads_total,
                                                      stream=stream)
    for p in range(SDL_SELECT_PASSES):
        st.hist_pass(p)
        all_reduce(st.hist(p))
    totals = st.count()
    offsets = shard_offsets(all_gather(totals), rank)
    return st.finish(offsets, row_ptr=row_ptr, col_idx=col_idx, want_mask=want_mask)
