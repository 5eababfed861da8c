"""The fused anchor step (one cooperative launch) against the separate calls.

sdl_anchor_refresh runs the bodies of the block-score, selection and tile-plan
kernels in one launch; its scores, CSR lists and plan must equal those of
sdl_block_scores + sdl_select_mask + sdl_tile_plan bit for bit, and its mask the
oracle's selection on those scores.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_sdl_b200 as sdl
import oracle
import synth

pytestmark = pytest.mark.gpu

CASES = [
    # dtype, B, L, H, H_kv, d, bs, sparsity
    ("fp32", 1, 512, 2, 2, 64, 64, 0.5),
    ("bf16", 2, 1024, 4, 2, 128, 64, 0.7),      # two sequences, GQA
    ("bf16", 1, 576, 3, 3, 64, 64, 0.6),        # nb = 9: a tile with one query block
    ("bf16", 1, 2048, 8, 8, 128, 128, 0.8),     # 128-token blocks: no tile plan
    ("bf16", 1, 512, 4, 4, 64, 64, 1 - 1 / 8),  # diagonal only
    ("bf16", 1, 17408, 2, 2, 64, 64, 0.95),     # nb = 272: adjacent pairs
    ("bf16", 1, 8192, 32, 32, 128, 64, 0.9),    # the 8K workload's shape
    ("bf16", 1, 1024, 4, 4, 64, 64, 0.0),       # keep everything: the threshold is the minimum
    ("bf16", 3, 576, 3, 1, 64, 64, 0.5),        # three sequences, nb = 9: one row per chunk
]


@pytest.mark.parametrize("dtype,B,L,H,H_kv,d,bs,s", CASES)
def test_fused_anchor_equals_separate_calls(dtype, B, L, H, H_kv, d, bs, s):
    w = synth.small_workload(dtype=dtype, B=B, H=H, H_kv=H_kv, L=L, d=d, bs=bs, sparsity=s,
                             planted=2)
    x = synth.device_inputs(w, 0)
    q, k = x["q"], x["k"]
    sc1 = sdl.block_scores(q, k, bs)
    rp1, ci1, _ = sdl.select_mask(sc1, s, bs, L)
    plan1 = sdl.tile_plan(rp1, ci1, B, H, L, bs) if bs == 64 else None
    sc2, rp2, ci2, plan2 = sdl.anchor_refresh(q, k, bs, s)
    torch.cuda.synchronize()
    assert sdl.last_device_status() == sdl.SDL_OK
    assert torch.equal(sc1, sc2)
    assert torch.equal(rp1, rp2) and torch.equal(ci1, ci2)
    if bs == 64:
        assert torch.equal(plan1, plan2)
    else:
        assert plan2 is None
    nb = L // bs
    mask = np.zeros((B * H * nb, nb), dtype=np.uint8)
    rp, ci = rp2.cpu().numpy(), ci2.cpu().numpy()
    for r in range(B * H * nb):
        mask[r, ci[rp[r]:rp[r + 1]]] = 1
    want, _, kept = oracle.select(sc2.cpu().numpy().astype(np.float64), s)
    assert np.array_equal(mask.reshape(want.shape), want)
    assert int(rp[-1]) == kept


@pytest.mark.parametrize("B,H,L,s", [(2, 4, 1024, 0.6), (3, 8, 2048, 0.85)])
def test_fused_anchor_hands_out_ties_in_row_order(B, H, L, s):
    """Q = 0: every row's scores are exactly 1/nb, so every off-diagonal score ties
    with the threshold and the quota of ties runs through the row chunks and the
    batch elements in flat row order, as the separate calls and the oracle do."""
    w = synth.small_workload(B=B, H=H, H_kv=H, L=L, d=128, bs=64, sparsity=s, planted=2)
    x = synth.device_inputs(w, 0)
    q = torch.zeros_like(x["q"])
    sc1 = sdl.block_scores(q, x["k"], 64)
    rp1, ci1, _ = sdl.select_mask(sc1, s, 64, L)
    sc2, rp2, ci2, _ = sdl.anchor_refresh(q, x["k"], 64, s, want_plan=False)
    torch.cuda.synchronize()
    assert sdl.last_device_status() == sdl.SDL_OK
    assert torch.equal(sc1, sc2)
    nb = L // 64
    assert bool((sc2 == 1.0 / nb).all())
    assert torch.equal(rp1, rp2) and torch.equal(ci1, ci2)
    want, _, kept = oracle.select(sc2.cpu().numpy().astype(np.float64), s)
    rp, ci = rp2.cpu().numpy(), ci2.cpu().numpy()
    mask = np.zeros((B * H * nb, nb), dtype=np.uint8)
    for r in range(B * H * nb):
        mask[r, ci[rp[r]:rp[r + 1]]] = 1
    assert np.array_equal(mask.reshape(want.shape), want)
    assert int(rp[-1]) == kept


def test_fused_anchor_repeated_launches_on_one_workspace():
    """The barrier counters are reset for every launch: back-to-back refreshes on
    one workspace and distinct inputs stay exact."""
    w = synth.small_workload(B=1, H=8, H_kv=8, L=2048, d=128, bs=64, sparsity=0.8, planted=2)
    ws = torch.empty(sdl.anchor_workspace_bytes(*[torch.empty((1, 2048, 8, 128),
                                                              dtype=torch.bfloat16,
                                                              device="cuda")] * 2, 64),
                     dtype=torch.uint8, device="cuda")
    for step in range(4):
        x = synth.device_inputs(w, step)
        sc, rp, ci, plan = sdl.anchor_refresh(x["q"], x["k"], 64, 0.8, workspace=ws)
        sc1 = sdl.block_scores(x["q"], x["k"], 64)
        rp1, ci1, _ = sdl.select_mask(sc1, 0.8, 64, 2048)
        torch.cuda.synchronize()
        assert sdl.last_device_status() == sdl.SDL_OK
        assert torch.equal(sc, sc1) and torch.equal(rp, rp1) and torch.equal(ci, ci1)


@pytest.mark.parametrize("dtype,B,L,H,H_kv,d,s", [
    ("bf16", 2, 1024, 4, 2, 128, 0.7),
    ("bf16", 1, 576, 3, 3, 64, 0.6),          # nb = 9: a tile with one query block
    ("fp32", 1, 512, 2, 2, 64, 0.5),          # no tile lists for fp32 layers, still buildable
    ("bf16", 1, 17408, 2, 2, 64, 0.95),       # nb = 272: adjacent pairs
    ("bf16", 1, 8192, 32, 32, 128, 0.9),      # the 8K workload's shape
])
def test_anchor_step_equals_separate_calls(dtype, B, L, H, H_kv, d, s):
    """sdl_anchor_step: scores, CSR lists, tile plan, take order and tile lists
    equal the separate calls bit for bit, over two steps on one set of buffers."""
    w = synth.small_workload(dtype=dtype, B=B, H=H, H_kv=H_kv, L=L, d=d, bs=64, sparsity=s,
                             planted=2)
    bufs = None
    for step in range(2):
        x = synth.device_inputs(w, step)
        q, k = x["q"], x["k"]
        sc1, rp1, ci1, _ = sdl.anchor_refresh(q, k, 64, s, want_plan=False)
        plan1 = sdl.tile_plan(rp1, ci1, B, H, L, 64)
        order1 = sdl.tile_order(rp1, plan1, B, H, L, 64)
        lists1 = sdl.tile_lists(rp1, ci1, plan1, order1, B, H, L, 64)
        if bufs is None:
            bufs = sdl.anchor_step(q, k, 64, s)
        else:
            sc, rp, ci, plan, order, lists = bufs
            bufs = sdl.anchor_step(q, k, 64, s, scores=sc, row_ptr=rp, col_idx=ci, plan=plan,
                                   order=order, lists=lists)
        torch.cuda.synchronize()
        assert sdl.last_device_status() == sdl.SDL_OK
        sc, rp, ci, plan, order, lists = bufs
        assert torch.equal(sc, sc1)
        assert torch.equal(rp, rp1) and torch.equal(ci, ci1[:ci.numel()])
        assert torch.equal(plan, plan1) and torch.equal(order, order1)
        assert _lists_used(lists, B, H, L) == _lists_used(lists1, B, H, L)


def _lists_used(lists, B, H, L):
    """The written part of a tile-lists buffer: each record's (item, n_ent, t0, t1)
    and its first n_ent entries (the slack after them is never written)."""
    n_items = B * H * ((L + 127) // 128)
    cap = ((L // 64) + 7) // 8 * 8
    raw = lists.cpu().numpy()
    rec = raw[:n_items * 32].view(np.int32).reshape(n_items, 8)
    ent = raw[n_items * 32:n_items * 32 + n_items * cap * 2].view(np.uint16).reshape(n_items, cap)
    return [(tuple(rec[r, :4]), tuple(ent[r, :max(rec[r, 1], 0)])) for r in range(n_items)]


@pytest.mark.parametrize("B,H,nb,cap", [
    (1, 100, 1024, 1024),   # 51200 tiles: costs recomputed in the second walk; 13 warps count
    (2, 64, 128, 128),      # the 8K block count: all 32 warps count
    (3, 7, 17, 5),          # odd block count, costs in a narrow range (many ties)
])
def test_tile_order_exact_at_scale(B, H, nb, cap):
    """The take order is the stable sort of the tiles by descending cost (a tile's
    two list lengths), checked entry for entry against numpy's stable sort, with
    row offsets only (the order reads no column indices)."""
    rng = np.random.default_rng(B * 1000 + H + nb)
    # skewed list lengths in [1, cap]: many short rows, a few long ones
    lens = np.minimum(cap, 1 + rng.geometric(4.0 / cap, size=B * H * nb)).astype(np.int64)
    rp = np.zeros(B * H * nb + 1, np.int64)
    rp[1:] = np.cumsum(lens)
    n_qt = (nb + 1) // 2
    # a random valid pairing per head
    pl = np.full((B, H, n_qt, 2), -1, np.int32)
    for b in range(B):
        for h in range(H):
            flat = np.full(2 * n_qt, -1)
            flat[:nb] = rng.permutation(nb)
            pl[b, h] = flat.reshape(n_qt, 2)
    rp_d = torch.from_numpy(rp.astype(np.int32)).cuda()
    plan_d = torch.from_numpy(pl).cuda()
    order = sdl.tile_order(rp_d, plan_d, B, H, nb * 64, 64).cpu().numpy()
    assert sdl.last_device_status() == sdl.SDL_OK
    flat = pl.reshape(-1, 2)
    head = np.arange(B * H * n_qt) // n_qt
    cost = np.zeros(B * H * n_qt, np.int64)
    for s_ in range(2):
        qb = flat[:, s_]
        ok = qb >= 0
        cost[ok] += lens[head[ok] * nb + qb[ok]]
    assert np.array_equal(order, np.argsort(-cost, kind="stable"))


@pytest.mark.parametrize("per_head", [False, True])
def test_selection_is_the_same_over_many_back_to_back_calls(per_head):
    """The radix resolution is shared by every block of the count and digit-pass
    kernels; a race there (a thread reading the count left after another thread had
    updated it) made a few selections of long runs write rows out of order.  On the
    8K workload's block scores at four anchors, 40 calls each, queued back to back,
    must all give the oracle's CSR."""
    w = synth.WORKLOADS["bf16-L8192-H32-s90"]
    nb, s = w.nb, w.sparsity
    for step in (0, 32, 64, 96):
        x = synth.device_inputs(w, step)
        scores = sdl.block_scores(x["q"], x["k"], w.bs)
        want, _, kept = oracle.select(scores.cpu().numpy().astype(np.float64), s,
                                      per_head=per_head)
        outs = [sdl.select_mask(scores, s, w.bs, w.L, per_head=per_head)[:2]
                for _ in range(40)]
        torch.cuda.synchronize()
        assert sdl.last_device_status() == sdl.SDL_OK, (step, sdl.last_device_detail())
        rp0, ci0 = outs[0][0].cpu().numpy(), outs[0][1].cpu().numpy()
        mask = np.zeros((w.B * w.H * nb, nb), dtype=np.uint8)
        for r in range(w.B * w.H * nb):
            mask[r, ci0[rp0[r]:rp0[r + 1]]] = 1
        assert np.array_equal(mask.reshape(want.shape), want) and int(rp0[-1]) == kept, step
        for k, (rp, ci) in enumerate(outs[1:]):
            assert torch.equal(rp, outs[0][0]) and torch.equal(ci, outs[0][1]), (step, k)


def test_fused_anchor_is_the_same_over_many_back_to_back_calls():
    """The fused kernel resolves the threshold in its digit-pass and count phases
    with the same shared routine: at four anchors of the 8K workload, 30 queued
    calls each give one result."""
    w = synth.WORKLOADS["bf16-L8192-H32-s90"]
    for step in (0, 32, 64, 96):
        x = synth.device_inputs(w, step)
        outs = [sdl.anchor_refresh(x["q"], x["k"], w.bs, w.sparsity, want_plan=False)[1:3]
                for _ in range(30)]
        torch.cuda.synchronize()
        assert sdl.last_device_status() == sdl.SDL_OK, (step, sdl.last_device_detail())
        for k, (rp, ci) in enumerate(outs[1:]):
            assert torch.equal(rp, outs[0][0]) and torch.equal(ci, outs[0][1]), (step, k)
