"""Mask selection with the heads of a sequence split over ranks (library kernels).

One GPU holds every rank's shard: the ranks' stages run in lockstep in one
process and the exchanges between them are plain tensor sums, so no kernel
waits on another.  The union of the ranks' parts must equal the single-device
selection of all heads bit for bit, and the oracle's global selection.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_sdl_b200 as sdl
import oracle
from block_sparse_attention_sdl_b200.sharded import (CudaStages, head_range,
                                                     select_mask_sharded, shard_offsets)

pytestmark = pytest.mark.gpu


def _scores(B, H, nb, seed, ties=False):
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((B, H, nb, nb)) * rng.uniform(0.3, 4.0, size=(1, H, 1, 1))
    if ties:
        z = np.round(z)
    e = np.exp(z - z.max(-1, keepdims=True))
    return (e / e.sum(-1, keepdims=True)).astype(np.float32)


def _lockstep(scores, s, bs, L, H_kv, W):
    """Every rank's stages of the sharded selection, interleaved as the collectives
    order them; returns each rank's (row_ptr, col_idx, mask)."""
    B, H = scores.shape[:2]
    stages = []
    for r in range(W):
        h0, h1 = head_range(H, H_kv, r, W)
        stages.append(CudaStages(scores[:, h0:h1].contiguous(), s, bs, L, H))
    for p in range(sdl.SDL_SELECT_PASSES):
        for st in stages:
            st.hist_pass(p)
        total = torch.stack([st.hist(p) for st in stages]).sum(0, dtype=torch.int32)
        for st in stages:
            st.hist(p).copy_(total)
    totals = [st.count() for st in stages]
    return [st.finish(shard_offsets(totals, r), want_mask=True) for r, st in enumerate(stages)]


CASES = [
    # B, H, H_kv, nb, W, sparsity, ties
    (1, 8, 8, 8, 2, 0.5, False),
    (2, 8, 8, 32, 4, 0.9, False),
    (1, 16, 16, 16, 4, 0.75, True),
    (2, 4, 4, 9, 2, 0.0, False),           # every block kept
    (1, 8, 8, 16, 8, 1.0 - 1.0 / 16, False),  # diagonal only
    (1, 28, 4, 32, 4, 0.9, False),         # GQA: whole KV-head groups per rank
    (1, 32, 32, 128, 2, 0.9, False),       # the 8K workload's shape
]


@pytest.mark.parametrize("B,H,H_kv,nb,W,s,ties", CASES)
def test_sharded_selection_equals_single_device(B, H, H_kv, nb, W, s, ties):
    L, bs = nb * 64, 64
    P = _scores(B, H, nb, seed=B * 1000 + H * 10 + nb, ties=ties)
    scores = torch.from_numpy(P).cuda()
    rp1, ci1, m1 = sdl.select_mask(scores, s, bs, L, want_mask=True)
    parts = _lockstep(scores, s, bs, L, H_kv, W)
    torch.cuda.synchronize()
    assert sdl.last_device_status() == sdl.SDL_OK
    got = torch.cat([m for _, _, m in parts], dim=1)
    assert torch.equal(got, m1)
    want, _, kept = oracle.select(P.astype(np.float64), s)
    assert np.array_equal(got.cpu().numpy(), want)
    # each rank's CSR agrees with its mask: ascending columns, counts from row_ptr
    total = 0
    for rp, ci, m in parts:
        rp, ci, m = rp.cpu().numpy(), ci.cpu().numpy(), m.cpu().numpy()
        nrows = m.shape[0] * m.shape[1] * nb
        n = int(rp[nrows])
        assert np.array_equal(np.diff(rp), m.reshape(nrows, nb).sum(1))
        cols = np.nonzero(m.reshape(nrows, nb))[1]
        assert np.array_equal(ci[:n], cols)
        total += n
    assert total == kept == int(ci1.numel())


def test_sharded_selection_single_rank_through_the_host_path():
    """World size 1 through select_mask_sharded (identity exchanges) == select_mask."""
    B, H, nb, s = 2, 8, 16, 0.8
    L = nb * 64
    scores = torch.from_numpy(_scores(B, H, nb, seed=5)).cuda()
    rp, ci, m = select_mask_sharded(scores, s, 64, L, H, 0, all_reduce=lambda t: None,
                                    all_gather=lambda t: [t], want_mask=True)
    rp1, ci1, m1 = sdl.select_mask(scores, s, 64, L, want_mask=True)
    torch.cuda.synchronize()
    assert torch.equal(m, m1) and torch.equal(rp, rp1)
    assert torch.equal(ci[:ci1.numel()], ci1)


def test_shard_arguments_are_checked():
    scores = torch.from_numpy(_scores(1, 4, 8, seed=3)).cuda()
    with pytest.raises(sdl.SdlError):
        sdl.select_shard_capacity(scores, 0.5, 64, 512, heads_total=2)  # fewer than local
    st = CudaStages(scores, 0.5, 64, 512, 8)
    with pytest.raises(sdl.SdlError):
        sdl.select_shard_pass(scores, 0.5, 64, 512, 8, 3, st.ws)  # no pass 3
    small = torch.empty(4, dtype=torch.int32, device="cuda")
    offs = torch.zeros((1, 2), dtype=torch.int64, device="cuda")
    with pytest.raises(sdl.SdlError):
        sdl.select_shard_finish(scores, 0.5, 64, 512, 8, offs, st.ws, col_idx=small)
