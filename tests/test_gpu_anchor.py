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
