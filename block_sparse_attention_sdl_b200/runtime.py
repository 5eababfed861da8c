"""Step schedules around the library calls (host logic only).

Step-dLLM (abstract) refreshes the block-sparse mask at anchor steps of the
denoising trajectory and reuses it within each interval.  Here step ``s`` is an
anchor when ``s % anchor_every == 0`` (step 0 always is); at an anchor the mask
is rebuilt from that step's Q and K before the step's own sparse attention
runs, so every step, anchors included, attends with the mask of its anchor
``(s // anchor_every) * anchor_every``.

Two variants of the prior methods the abstract compares against (SparseD
abstract) are selectable: a uniform budget per head instead of the
head-adaptive global one (``budget="head"``), and dense attention for the first
``dense_steps`` steps followed by a single mask, built at step
``dense_steps`` and reused for every later step (``anchor_every=None``).

``ColSparseAttention`` is the column-sparse scheme of the PulseCol abstract on
the same schedule: every query head keeps a set of key tokens, refreshed at
anchor steps, gathered and attended to at every step.

With ``heads_total`` the layer is one rank's part of a head-sharded attention
layer: its tensors hold ``H`` of the sequence's ``heads_total`` query heads
(whole KV-head groups, ranks in head order), and the global budget is met with
the staged selection of ``sharded.py`` (histogram sums and totals exchanged
over ``group``); scores, attention and the tile plan stay local.
"""
from __future__ import annotations

import torch

from . import (anchor_refresh, anchor_step, anchor_workspace_bytes, block_scores, col_budget,
               col_gather, col_scores, col_scores_workspace_bytes, col_select, col_sparse_attn,
               dense_attn, make_shape, mask_budget, scores_workspace_bytes, select_mask,
               select_shard_capacity, select_workspace_bytes, sparse_attn, tile_lists,
               tile_lists_bytes, tile_order, tile_plan)
from .sharded import CudaStages, select_mask_sharded, torch_collectives


def is_dense(step: int, dense_steps: int = 0) -> bool:
    return step < dense_steps


def is_anchor(step: int, anchor_every, dense_steps: int = 0) -> bool:
    """Whether the mask is rebuilt at `step` (anchor_every None: only at dense_steps)."""
    if step < dense_steps:
        return False
    if anchor_every is None:
        return step == dense_steps
    return (step - dense_steps) % anchor_every == 0


def anchor_of(step: int, anchor_every, dense_steps: int = 0):
    """The step whose mask `step` attends with, or None for a dense step."""
    if step < dense_steps:
        return None
    if anchor_every is None:
        return dense_steps
    return dense_steps + ((step - dense_steps) // anchor_every) * anchor_every


class StepSparseAttention:
    """One attention layer's block-sparse state across denoising steps.

    All device buffers (scores, workspaces, CSR lists, tile plan) are allocated
    once here, so the per-step calls allocate nothing.
    """

    def __init__(self, B, H, H_kv, L, d, block, sparsity, anchor_every, dtype=torch.bfloat16,
                 device="cuda", budget: str = "sequence", dense_steps: int = 0,
                 heads_total=None, rank: int = 0, group=None, collectives=None):
        if budget not in ("sequence", "head"):
            raise ValueError("budget must be 'sequence' or 'head'")
        # a head-sharded layer needs the exchange only for the budget across heads
        self.sharded = heads_total is not None and budget == "sequence"
        self.heads_total = H if heads_total is None else heads_total
        self.rank, self.group = rank, group
        self.collectives = collectives
        self.B, self.H, self.H_kv, self.L, self.d, self.block = B, H, H_kv, L, d, block
        self.sparsity, self.anchor_every = sparsity, anchor_every
        self.per_head, self.dense_steps = budget == "head", dense_steps
        self.nb = L // block
        probe_q = torch.empty((B, L, H, d), dtype=dtype, device="meta")
        probe_k = torch.empty((B, L, H_kv, d), dtype=dtype, device="meta")
        shape = make_shape(probe_q, probe_k, block)
        full = make_shape(torch.empty((B, L, self.heads_total, d), dtype=dtype, device="meta"),
                          torch.empty((B, L, self.heads_total, d), dtype=dtype, device="meta"),
                          block)
        # kept blocks of the whole sequence (every rank's heads)
        self.budget = mask_budget(full, sparsity, self.per_head)
        if self.budget < 0:
            raise ValueError("sparsity outside [0, 1) or budget below the diagonal blocks")
        dev = torch.device(device)
        self.scores = torch.empty((B, H, self.nb, self.nb), dtype=torch.float32, device=dev)
        if self.sharded:
            capacity = select_shard_capacity(self.scores, sparsity, block, L, self.heads_total)
        else:
            capacity = mask_budget(shape, sparsity, self.per_head)
        self.ws_scores = torch.empty(max(scores_workspace_bytes(shape), 16), dtype=torch.uint8,
                                     device=dev)
        self.ws_select = torch.empty(max(select_workspace_bytes(shape, self.per_head), 16),
                                     dtype=torch.uint8, device=dev)
        self.row_ptr = torch.empty(B * H * self.nb + 1, dtype=torch.int32, device=dev)
        self.col_idx = torch.empty(capacity, dtype=torch.int32, device=dev)
        # 64-token blocks: which two query blocks share a 128-row tile (rebuilt with the mask)
        self.plan = (torch.empty((B, H, (self.nb + 1) // 2, 2), dtype=torch.int32, device=dev)
                     if block == 64 else None)
        # the plan's tiles, costliest first (the attention kernel's take order)
        self.order = (torch.empty(B * H * ((self.nb + 1) // 2), dtype=torch.int32, device=dev)
                      if block == 64 else None)
        # the tiles' kept-block lists in that order (bf16: the tensor-core kernel reads them
        # instead of building each tile's list from the CSR when it takes the tile)
        self.lists = (torch.empty(tile_lists_bytes(B, H, L, block), dtype=torch.uint8,
                                  device=dev)
                      if block == 64 and dtype == torch.bfloat16 else None)
        self.mask_step = None  # anchor step whose mask is current
        # the head-adaptive budget on one device: scores and selection in one launch
        self.fused = not self.sharded and not self.per_head
        self.ws_anchor = (torch.empty(max(anchor_workspace_bytes(probe_q, probe_k, block), 16),
                                      dtype=torch.uint8, device=dev) if self.fused else None)

    def refresh(self, q, k, step: int, stream=None):
        if self.fused and self.plan is not None:
            # the whole step (scores, mask, plan, order, lists) from one C call
            anchor_step(q, k, self.block, self.sparsity, scores=self.scores,
                        row_ptr=self.row_ptr, col_idx=self.col_idx, plan=self.plan,
                        order=self.order, lists=self.lists, want_lists=self.lists is not None,
                        workspace=self.ws_anchor, stream=stream)
            self.mask_step = step
            return
        if self.fused:
            anchor_refresh(q, k, self.block, self.sparsity, scores=self.scores,
                           row_ptr=self.row_ptr, col_idx=self.col_idx, want_plan=False,
                           workspace=self.ws_anchor, stream=stream)
        else:
            block_scores(q, k, self.block, scores=self.scores, workspace=self.ws_scores,
                         stream=stream)
            self.select(stream)
        if self.plan is not None:
            tile_plan(self.row_ptr, self.col_idx, self.B, self.H, self.L, self.block,
                      plan=self.plan, stream=stream)
            tile_order(self.row_ptr, self.plan, self.B, self.H, self.L, self.block,
                       order=self.order, stream=stream)
        if self.lists is not None:
            tile_lists(self.row_ptr, self.col_idx, self.plan, self.order, self.B, self.H, self.L,
                       self.block, lists=self.lists, stream=stream)
        self.mask_step = step

    def select(self, stream=None):
        """The mask from the current scores (every rank of a sharded layer calls it)."""
        if self.sharded:
            if self.collectives is not None:
                all_reduce, all_gather = self.collectives
            elif torch.distributed.is_available() and torch.distributed.is_initialized():
                all_reduce, all_gather = torch_collectives(self.group)
            else:  # a single rank holds every head
                all_reduce, all_gather = (lambda t: None), (lambda t: [t])
            stages = CudaStages(self.scores, self.sparsity, self.block, self.L, self.heads_total,
                                workspace=self.ws_select, stream=stream)
            select_mask_sharded(self.scores, self.sparsity, self.block, self.L,
                                self.heads_total, self.rank, all_reduce=all_reduce,
                                all_gather=all_gather, stages=stages, row_ptr=self.row_ptr,
                                col_idx=self.col_idx)
        else:
            select_mask(self.scores, self.sparsity, self.block, self.L, row_ptr=self.row_ptr,
                        col_idx=self.col_idx, workspace=self.ws_select,
                        per_head=self.per_head, stream=stream)

    def __call__(self, q, k, v, step: int, out=None, lse=None, stream=None):
        if is_dense(step, self.dense_steps):
            return dense_attn(q, k, v, self.block, out=out, lse=lse, stream=stream)
        if is_anchor(step, self.anchor_every, self.dense_steps) or self.mask_step is None:
            self.refresh(q, k, anchor_of(step, self.anchor_every, self.dense_steps), stream)
        return sparse_attn(q, k, v, self.row_ptr, self.col_idx, self.block, out=out, lse=lse,
                           plan=self.plan, order=self.order, lists=self.lists, stream=stream)


class ColSparseAttention:
    """One attention layer's column-sparse state (the PulseCol abstract).

    Every query head keeps Lc key tokens for all of its query rows: chosen from the
    column scores at refresh steps (step 0 and every ``refresh_every`` steps;
    ``None``: step 0 only) and reused in between.  Every step gathers the kept K and
    V tokens of that step's tensors and runs dense attention over them.  Buffers are
    allocated once here.
    """

    def __init__(self, B, H, H_kv, L, d, block, sparsity, refresh_every,
                 dtype=torch.bfloat16, device="cuda"):
        self.B, self.H, self.H_kv, self.L, self.d, self.block = B, H, H_kv, L, d, block
        self.sparsity, self.anchor_every = sparsity, refresh_every
        self.per_head, self.sharded, self.fused, self.dense_steps = True, False, False, 0
        probe_q = torch.empty((B, L, H, d), dtype=dtype, device="meta")
        probe_k = torch.empty((B, L, H_kv, d), dtype=dtype, device="meta")
        self.Lc = col_budget(probe_q, probe_k, block, sparsity)
        # kept work in 64x64-block equivalents (L and Lc are whole 64-token tiles)
        self.budget = B * H * (L // 64) * (self.Lc // 64)
        dev = torch.device(device)
        self.col_scores = torch.empty((B, H, L), dtype=torch.float32, device=dev)
        self.ws = torch.empty(max(col_scores_workspace_bytes(probe_q, probe_k, block), 16),
                              dtype=torch.uint8, device=dev)
        self.cols = torch.empty((B, H, self.Lc), dtype=torch.int32, device=dev)
        self.k_cols = torch.empty((B, self.Lc, H, d), dtype=dtype, device=dev)
        self.v_cols = torch.empty((B, self.Lc, H, d), dtype=dtype, device=dev)
        self.mask_step = None
        self._qk = None  # the tensors of the last refresh (shapes for the selection)

    def refresh(self, q, k, step: int, stream=None):
        col_scores(q, k, self.block, out=self.col_scores, workspace=self.ws, stream=stream)
        self._qk = (q, k)
        self.select(stream)
        self.mask_step = step

    def select(self, stream=None):
        q, k = self._qk
        col_select(self.col_scores, q, k, self.block, self.sparsity, cols=self.cols,
                   stream=stream)

    def attend(self, q, k, v, out=None, lse=None, stream=None):
        """This step's attention over the kept columns (gather, then attention)."""
        col_gather(k, v, self.cols, q, self.block, k_cols=self.k_cols, v_cols=self.v_cols,
                   stream=stream)
        return col_sparse_attn(q, self.k_cols, self.v_cols, self.block, out=out,
                               want_lse=lse is not None, lse=lse, stream=stream)

    def __call__(self, q, k, v, step: int, out=None, lse=None, stream=None):
        if is_anchor(step, self.anchor_every) or self.mask_step is None:
            self.refresh(q, k, anchor_of(step, self.anchor_every), stream)
        return self.attend(q, k, v, out=out, lse=lse, stream=stream)
