"""GPU parity of each library call against the fp64 oracle on small shapes.

Shapes span several 128-row tiles and a ragged tail (odd block counts), both
block sizes, both head dims, GQA groups 1/2/7, bf16 and fp32, and strided
(fused-QKV) layouts.  Attention is checked with the GPU's own mask, so mask
parity and attention parity are independent.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_util import (TOL, bf16_to_f64, check_close, check_csr, compare_masks,
                               csr_to_mask, sample_rows)

pytestmark = pytest.mark.gpu

sdl = pytest.importorskip("block_sparse_attention_sdl_b200")


def _inputs(w, step=0):
    host = synth.host_inputs(w, step)
    dev = synth.device_inputs(w, step)
    return host, dev


def _mask_to_csr(mask):
    B, H, nb, _ = mask.shape
    flat = mask.reshape(-1, nb)
    row_ptr = np.zeros(flat.shape[0] + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum(flat.sum(1))
    col_idx = np.concatenate([np.nonzero(r)[0] for r in flat]).astype(np.int32)
    return torch.from_numpy(row_ptr).cuda(), torch.from_numpy(col_idx).cuda()


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("L,H,Hkv,d", [(256, 2, 2, 64), (1024, 4, 2, 128), (640, 7, 1, 128)])
def test_generator_twins_bit_identical(dtype, L, H, Hkv, d):
    w = synth.small_workload(dtype=dtype, L=L, H=H, H_kv=Hkv, d=d, planted=2)
    for step in (0, 3):
        for x in ("q", "k", "v"):
            host = synth.host_tensor(w, x, step)
            dev = synth.device_tensor(w, x, step).cpu()
            if dtype == "bf16":
                dev = dev.view(torch.int16).numpy().view(np.uint16)
            else:
                dev = dev.numpy()
            assert np.array_equal(host, dev), (x, step)


SCORE_CASES = [
    ("bf16", 512, 2, 2, 64, 64),
    ("bf16", 2048, 4, 4, 128, 64),
    ("bf16", 1024, 7, 1, 128, 64),
    ("bf16", 2048, 2, 1, 128, 128),
    ("fp32", 512, 2, 2, 64, 64),
    ("fp32", 1024, 4, 2, 128, 128),
]


@pytest.mark.parametrize("dtype,L,H,Hkv,d,bs", SCORE_CASES)
def test_block_scores(dtype, L, H, Hkv, d, bs):
    w = synth.small_workload(dtype=dtype, L=L, H=H, H_kv=Hkv, d=d, bs=bs, planted=2)
    host, dev = _inputs(w)
    P = sdl.block_scores(dev["q"], dev["k"], bs)
    torch.cuda.synchronize()
    want = oracle.block_scores(host["q"], host["k"], bs)
    got = P.cpu().numpy().astype(np.float64)
    rel = np.abs(got - want) / want
    assert rel.max() < 2e-5, rel.max()
    assert np.allclose(got.sum(-1), 1.0, atol=1e-5)


@pytest.mark.parametrize("B,H,nb,s", [(1, 2, 8, 0.5), (1, 4, 32, 0.8), (2, 3, 16, 0.7),
                                      (1, 32, 128, 0.9), (1, 2, 5, 0.3)])
def test_select_matches_oracle(B, H, nb, s):
    rng = np.random.default_rng(nb * 7 + H)
    logits = rng.standard_normal((B, H, nb, nb)) * rng.uniform(0.2, 3.0, (1, H, 1, 1))
    P = np.exp(logits) / np.exp(logits).sum(-1, keepdims=True)
    P32 = P.astype(np.float32)
    # the oracle sees the same fp32 values the kernel sees
    want, tau, kept = oracle.select(P32.astype(np.float64), s)
    row_ptr, col_idx, mask = sdl.select_mask(torch.from_numpy(P32).cuda(), s, 64, nb * 64,
                                             want_mask=True)
    torch.cuda.synchronize()
    rp, ci = row_ptr.cpu().numpy(), col_idx.cpu().numpy()
    check_csr(rp, ci, B, H, nb, kept)
    got = csr_to_mask(rp, ci, B, H, nb)
    assert np.array_equal(got, mask.cpu().numpy())
    assert np.array_equal(got, want)  # identical fp32 inputs: no excuse needed


@pytest.mark.parametrize("B,H,nb,s", [(1, 4, 16, 0.7), (2, 3, 32, 0.9), (1, 32, 128, 0.9)])
def test_select_per_head_budget_matches_oracle(B, H, nb, s):
    """Uniform per-head budget: the same rule applied to every head alone."""
    rng = np.random.default_rng(nb * 5 + H)
    logits = rng.standard_normal((B, H, nb, nb)) * rng.uniform(0.2, 3.0, (1, H, 1, 1))
    P32 = (np.exp(logits) / np.exp(logits).sum(-1, keepdims=True)).astype(np.float32)
    want, tau, kept = oracle.select(P32.astype(np.float64), s, per_head=True)
    row_ptr, col_idx, mask = sdl.select_mask(torch.from_numpy(P32).cuda(), s, 64, nb * 64,
                                             want_mask=True, per_head=True)
    torch.cuda.synchronize()
    rp, ci = row_ptr.cpu().numpy(), col_idx.cpu().numpy()
    check_csr(rp, ci, B, H, nb, kept)
    got = csr_to_mask(rp, ci, B, H, nb)
    assert np.array_equal(got, mask.cpu().numpy())
    assert np.array_equal(got, want)
    per = got.reshape(B * H, -1).sum(-1)
    assert (per == per[0]).all() and per.sum() == kept


def test_select_exact_ties_follow_flat_index():
    B, H, nb = 1, 3, 16
    P = np.full((B, H, nb, nb), 1.0 / nb, dtype=np.float32)
    P[0, 1, :, 5] = 0.5  # some strictly larger entries
    for s in (0.6, 0.75, 0.9):
        want, _, kept = oracle.select(P.astype(np.float64), s)
        rp, ci, _ = sdl.select_mask(torch.from_numpy(P).cuda(), s, 64, nb * 64)
        got = csr_to_mask(rp.cpu().numpy(), ci.cpu().numpy(), B, H, nb)
        assert np.array_equal(got, want), s


def test_select_extremes():
    P = torch.rand(1, 2, 8, 8).cuda()
    rp, ci, _ = sdl.select_mask(P, 0.0, 64, 512)
    assert ci.numel() == 128 and torch.equal(rp[-1].cpu(), torch.tensor(128, dtype=torch.int32))
    s_diag = 1.0 - 16 / 128
    rp, ci, _ = sdl.select_mask(P, s_diag, 64, 512)
    assert torch.equal(ci.cpu(), torch.arange(8, dtype=torch.int32).repeat(2))


def test_select_reuses_workspace_across_calls():
    """Workspace contents on entry do not matter: a dirty workspace gives the same mask."""
    P = torch.rand(1, 4, 32, 32, device="cuda")
    P = P / P.sum(-1, keepdim=True)
    ws = torch.full((1 << 20,), 0xAB, dtype=torch.uint8, device="cuda")
    a = sdl.select_mask(P, 0.8, 64, 2048, workspace=ws)
    b = sdl.select_mask(P, 0.8, 64, 2048, workspace=ws)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


ATTN_CASES = [
    # dtype, B, L, H, Hkv, d, bs, density
    ("bf16", 1, 256, 2, 2, 128, 64, 0.5),
    ("bf16", 1, 320, 2, 1, 128, 64, 0.5),  # odd block count: ragged last tile
    ("bf16", 2, 1024, 4, 2, 128, 64, 0.3),
    ("bf16", 1, 1024, 7, 1, 128, 64, 0.25),
    ("bf16", 1, 1024, 2, 2, 128, 128, 0.4),
    ("bf16", 1, 512, 2, 2, 64, 64, 0.5),
    ("bf16", 1, 768, 4, 4, 64, 128, 0.5),
    ("fp32", 1, 512, 2, 2, 64, 64, 0.5),
    ("fp32", 1, 512, 2, 1, 128, 128, 0.5),
]


def _random_mask(B, H, nb, density, rng):
    m = (rng.random((B, H, nb, nb)) < density).astype(np.uint8)
    for i in range(nb):
        m[:, :, i, i] = 1
    return m


@pytest.mark.parametrize("dtype,B,L,H,Hkv,d,bs,density", ATTN_CASES)
def test_sparse_attention(dtype, B, L, H, Hkv, d, bs, density):
    w = synth.Workload("t", dtype, B, H, Hkv, L, d, bs, 0.5, 1, 1, 0.02, ("uniform", 0.3, 4.0), 1)
    host, dev = _inputs(w)
    nb = L // bs
    rng = np.random.default_rng(L + H)
    mask = _random_mask(B, H, nb, density, rng)
    rp, ci = _mask_to_csr(mask)
    O, lse = sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, bs, want_lse=True)
    assert sdl.last_device_status() == sdl.SDL_OK
    Ow, lw = oracle.attention(host["q"], host["k"], host["v"], bs, mask=mask)
    got = bf16_to_f64(O).transpose(0, 2, 1, 3)
    check_close(got, Ow, dtype)
    assert np.abs(lse.cpu().numpy() - lw).max() <= TOL[dtype]["lse"]


@pytest.mark.parametrize("kind", ["dense", "sparse"])
def test_sharp_logits_raise_the_reference_within_and_across_tiles(kind):
    """Sharpness 16 to 48 per head: along an item's key blocks the maximum logit
    grows past the running reference by more than the lazy-rescale threshold
    (16 in log2 units), so the raise path runs (the step's weights redone against
    the new reference, O and the row sums rescaled in TMEM), and weights come
    close to 2^16 where the reference lags; O and LSE still match the oracle."""
    B, H, Hkv, L, d, bs = 1, 4, 2, 2048, 128, 64
    w = synth.Workload("sharp", "bf16", B, H, Hkv, L, d, bs, 0.5, 1, 1, 0.02,
                       ("fixed", [16.0, 24.0, 32.0, 48.0]), 1)
    host, dev = _inputs(w)
    nb = L // bs
    if kind == "dense":
        mask = np.ones((B, H, nb, nb), np.uint8)
    else:
        mask = _random_mask(B, H, nb, 0.5, np.random.default_rng(11))
    # the inputs reach the raise path: for rows of query block 0, the logits of
    # the first kept 64-key block against those of the later kept blocks
    q = host["q"][0].astype(np.float64)
    k = host["k"][0].astype(np.float64)
    growth = 0.0
    for h in range(H):
        kept = np.flatnonzero(mask[0, h, 0])
        x = q[:bs, h] @ k[:, h // (H // Hkv)].T / np.sqrt(d) * np.log2(np.e)
        first = x[:, kept[0] * bs:(kept[0] + 1) * bs].max(1)
        later = np.max([x[:, j * bs:(j + 1) * bs].max(1) for j in kept], axis=0)
        growth = max(growth, float((later - first).max()))
    assert growth > 2 * 16.0, growth
    if kind == "dense":
        O, lse = sdl.dense_attn(dev["q"], dev["k"], dev["v"], want_lse=True)
        Ow, lw = oracle.attention(host["q"], host["k"], host["v"], bs)
    else:
        rp, ci = _mask_to_csr(mask)
        O, lse = sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, bs, want_lse=True)
        Ow, lw = oracle.attention(host["q"], host["k"], host["v"], bs, mask=mask)
    assert sdl.last_device_status() == sdl.SDL_OK
    check_close(bf16_to_f64(O).transpose(0, 2, 1, 3), Ow, "bf16")
    assert np.abs(lse.cpu().numpy() - lw).max() <= TOL["bf16"]["lse"]


@pytest.mark.parametrize("kind", ["diag", "ones", "single_far"])
@pytest.mark.parametrize("bs", [64, 128])
def test_sparse_attention_edge_masks(kind, bs):
    w = synth.small_workload(L=1024, H=2, H_kv=2, d=128, bs=bs)
    host, dev = _inputs(w)
    nb = 1024 // bs
    if kind == "diag":
        mask = np.broadcast_to(np.eye(nb, dtype=np.uint8), (1, 2, nb, nb)).copy()
    elif kind == "ones":
        mask = np.ones((1, 2, nb, nb), np.uint8)
    else:  # diagonal plus the farthest block only
        mask = np.broadcast_to(np.eye(nb, dtype=np.uint8), (1, 2, nb, nb)).copy()
        for i in range(nb):
            mask[0, :, i, nb - 1 - i] = 1
    rp, ci = _mask_to_csr(mask)
    O = sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, bs)
    Ow, _ = oracle.attention(host["q"], host["k"], host["v"], bs, mask=mask)
    check_close(bf16_to_f64(O).transpose(0, 2, 1, 3), Ow, "bf16")


@pytest.mark.parametrize("bs", [64, 128])
def test_sparse_attention_empty_rows(bs):
    """A caller's mask may leave rows empty: those rows are zero with LSE -inf.

    Covers a 128-row tile with both query blocks empty, one with only one,
    and empty tiles between non-empty ones in a CTA's schedule.
    """
    w = synth.small_workload(L=1024, H=4, H_kv=2, d=128, bs=bs)
    host, dev = _inputs(w)
    nb = 1024 // bs
    rng = np.random.default_rng(7 + bs)
    mask = (rng.random((1, 4, nb, nb)) < 0.3).astype(np.uint8)
    mask[0, 0, :, :] = 0  # a whole head empty
    mask[0, 1, 0:2, :] = 0  # the first tile of head 1 (both 64-token halves at bs 64)
    mask[0, 2, 3, :] = 0  # one row only
    mask[0, 3, nb - 1, :] = 0  # the last row
    rp, ci = _mask_to_csr(mask)
    O, lse = sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, bs, want_lse=True)
    assert sdl.last_device_status() == sdl.SDL_OK
    Ow, lw = oracle.attention(host["q"], host["k"], host["v"], bs, mask=mask)
    check_close(bf16_to_f64(O).transpose(0, 2, 1, 3), Ow, "bf16")
    lg = lse.cpu().numpy()
    assert np.array_equal(np.isinf(lg), np.isinf(lw))
    fin = np.isfinite(lw)
    assert np.abs(lg[fin] - lw[fin]).max() <= TOL["bf16"]["lse"]


@pytest.mark.parametrize("bs,density", [(64, 0.15), (128, 0.3)])
def test_sparse_attention_many_tiles_per_cta(bs, density):
    """More 128-row tiles than SMs: each persistent CTA walks several tiles,
    reusing both list / Q / O slots; checked on sampled rows of every head."""
    w = synth.Workload("t", "bf16", 2, 12, 4, 4096, 128, bs, 0.5, 1, 1, 0.02,
                       ("uniform", 0.3, 4.0), 1)
    host, dev = _inputs(w)
    nb = 4096 // bs
    rng = np.random.default_rng(11)
    mask = _random_mask(2, 12, nb, density, rng)
    rp, ci = _mask_to_csr(mask)
    O, lse = sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, bs, want_lse=True)
    assert sdl.last_device_status() == sdl.SDL_OK
    rows = sample_rows(2, 12, 4096, bs, mask.sum(-1), n_blocks=6, rows_per_block=6)
    Ow, lw = oracle.attention(host["q"], host["k"], host["v"], bs, mask=mask, rows=rows)
    got = bf16_to_f64(O)[rows[:, 0], rows[:, 2], rows[:, 1]]
    check_close(got, Ow, "bf16")
    lg = lse.cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]]
    assert np.abs(lg - lw).max() <= TOL["bf16"]["lse"]


def _greedy_plan(M):
    """The tile-plan rule restated: blocks by descending list length (ties: lower
    index), each unpaired block paired with the unpaired block of largest list
    intersection (ties: lower index); adjacent pairs above 256 blocks."""
    nb = M.shape[0]
    n_qt = (nb + 1) // 2
    if nb > 256:
        return np.array([[2 * p, 2 * p + 1 if 2 * p + 1 < nb else -1] for p in range(n_qt)])
    ln = M.sum(1)
    ov = (M[:, None, :].astype(np.int64) & M[None, :, :]).sum(-1)
    used = np.zeros(nb, bool)
    pairs = []
    for i in sorted(range(nb), key=lambda i: (-ln[i], i)):
        if used[i]:
            continue
        used[i] = True
        cand = [j for j in range(nb) if not used[j]]
        best = max(cand, key=lambda j: (ov[i, j], -j)) if cand else -1
        if best >= 0:
            used[best] = True
        pairs.append((i, best))
    return np.array(pairs)


@pytest.mark.parametrize("nb,density", [(9, 0.4), (32, 0.2), (128, 0.1), (300, 0.05)])
def test_tile_plan_follows_the_greedy_rule(nb, density):
    B, H = 1, 3
    rng = np.random.default_rng(nb)
    mask = _random_mask(B, H, nb, density, rng)
    rp, ci = _mask_to_csr(mask)
    plan = sdl.tile_plan(rp, ci, B, H, nb * 64, 64).cpu().numpy()
    for h in range(H):
        want = _greedy_plan(mask[0, h].astype(bool))
        assert np.array_equal(plan[0, h], want), h
        got = plan[0, h].ravel()
        assert sorted(got[got >= 0].tolist()) == list(range(nb))  # every block exactly once


@pytest.mark.parametrize("L,H,Hkv,density,kind", [(1024, 4, 2, 0.3, "greedy"),
                                                 (1088, 3, 1, 0.25, "random"),
                                                 (2048, 2, 2, 0.15, "random")])
def test_sparse_attention_with_tile_plan(L, H, Hkv, density, kind):
    """Any pairing of query blocks into tiles gives the oracle's result."""
    w = synth.small_workload(L=L, H=H, H_kv=Hkv, d=128, bs=64)
    host, dev = _inputs(w)
    nb = L // 64
    rng = np.random.default_rng(L + H)
    mask = _random_mask(1, H, nb, density, rng)
    rp, ci = _mask_to_csr(mask)
    if kind == "greedy":
        plan = sdl.tile_plan(rp, ci, 1, H, L, 64)
    else:
        n_qt = (nb + 1) // 2
        pl = np.full((1, H, n_qt, 2), -1, np.int32)
        for h in range(H):
            perm = rng.permutation(nb)
            flat = np.full(2 * n_qt, -1)
            flat[:nb] = perm
            pl[0, h] = flat.reshape(n_qt, 2)
        plan = torch.from_numpy(pl).cuda()
    O, lse = sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, 64, want_lse=True, plan=plan)
    assert sdl.last_device_status() == sdl.SDL_OK
    Ow, lw = oracle.attention(host["q"], host["k"], host["v"], 64, mask=mask)
    check_close(bf16_to_f64(O).transpose(0, 2, 1, 3), Ow, "bf16")
    assert np.abs(lse.cpu().numpy() - lw).max() <= TOL["bf16"]["lse"]


@pytest.mark.parametrize("L,H,density", [(1024, 4, 0.3), (4096, 8, 0.15), (576, 3, 0.5)])
def test_tile_order_is_costliest_first_and_exact(L, H, density):
    """The take order is a permutation of the tiles sorted by the two blocks' list
    lengths (descending), and attention taken in it equals the plan order bit for bit."""
    w = synth.small_workload(L=L, H=H, H_kv=H, d=128, bs=64)
    _, dev = _inputs(w)
    nb = L // 64
    rng = np.random.default_rng(L * 7 + H)
    mask = _random_mask(1, H, nb, density, rng)
    mask[0, H - 1] = 1  # the last head keeps every block: its tiles are the costliest
    rp, ci = _mask_to_csr(mask)
    plan = sdl.tile_plan(rp, ci, 1, H, L, 64)
    order = sdl.tile_order(rp, plan, 1, H, L, 64)
    O1 = sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, 64, plan=plan)
    O2 = sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, 64, plan=plan, order=order)
    assert sdl.last_device_status() == sdl.SDL_OK
    assert torch.equal(O1, O2)
    o = order.cpu().numpy()
    n_qt = (nb + 1) // 2
    assert np.array_equal(np.sort(o), np.arange(H * n_qt))
    lens = mask.sum(-1).reshape(-1).astype(np.int64)  # list length per (h, query block)
    pl = plan.cpu().numpy().reshape(-1, 2)
    cost = np.array([sum(lens[(x // n_qt) * nb + qb] for qb in pl[x] if qb >= 0)
                     for x in range(H * n_qt)])
    assert np.all(np.diff(cost[o]) <= 0)
    assert cost[o[0]] == cost.max()
    # stable: equal costs keep the tile order
    same = np.diff(cost[o]) == 0
    assert np.all(np.diff(o)[same] > 0)


def test_scheduled_attention_two_sequences_gqa():
    """Tile plan and costliest-first take order over two sequences under GQA: the
    oracle's result, LSE included, with tiles of both sequences interleaved."""
    B, L, H, Hkv = 2, 1024, 4, 2
    w = synth.small_workload(B=B, L=L, H=H, H_kv=Hkv, d=128, bs=64)
    host, dev = _inputs(w)
    nb = L // 64
    rng = np.random.default_rng(2024)
    mask = _random_mask(B, H, nb, 0.3, rng)
    mask[1, 0] = 1  # one head of the second sequence keeps every block
    rp, ci = _mask_to_csr(mask)
    plan = sdl.tile_plan(rp, ci, B, H, L, 64)
    order = sdl.tile_order(rp, plan, B, H, L, 64)
    O, lse = sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, 64, want_lse=True,
                             plan=plan, order=order)
    assert sdl.last_device_status() == sdl.SDL_OK
    Ow, lw = oracle.attention(host["q"], host["k"], host["v"], 64, mask=mask)
    check_close(bf16_to_f64(O).transpose(0, 2, 1, 3), Ow, "bf16")
    assert np.abs(lse.cpu().numpy() - lw).max() <= TOL["bf16"]["lse"]


def test_bad_tile_order_entry_is_reported():
    w = synth.small_workload(L=256, H=1, H_kv=1, d=128)
    _, dev = _inputs(w)
    mask = np.ones((1, 1, 4, 4), np.uint8)
    rp, ci = _mask_to_csr(mask)
    plan = sdl.tile_plan(rp, ci, 1, 1, 256, 64)
    order = torch.tensor([1, 5], dtype=torch.int32, device="cuda")  # 5: no such tile
    sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, 64, plan=plan, order=order)
    assert sdl.last_device_status() == sdl.SDL_ERR_BAD_MASK
    assert sdl.last_device_detail() == ("take-order entry (attention)", 5)
    assert sdl.last_device_status() == sdl.SDL_OK and sdl.last_device_detail() is None


def test_bad_tile_plan_entry_is_reported():
    w = synth.small_workload(L=256, H=1, H_kv=1, d=128)
    _, dev = _inputs(w)
    mask = np.ones((1, 1, 4, 4), np.uint8)
    rp, ci = _mask_to_csr(mask)
    plan = torch.tensor([[[[0, 1], [2, 77]]]], dtype=torch.int32, device="cuda")  # 77 >= nb
    sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, 64, plan=plan)
    assert sdl.last_device_status() == sdl.SDL_ERR_BAD_MASK
    assert sdl.last_device_detail() == ("tile plan entry", 1)  # tile 1 holds the 77


def test_repeated_launches_on_two_streams_are_identical():
    """The attention kernel's CTAs take tiles from a per-launch counter that the
    last CTA resets; 150 launches, alternating over two streams, must all give
    the result of the first, bit for bit."""
    w = synth.small_workload(L=2048, H=8, H_kv=2, d=128, bs=64)
    _, dev = _inputs(w)
    mask = _random_mask(1, 8, 32, 0.3, np.random.default_rng(3))
    rp, ci = _mask_to_csr(mask)
    ref = sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, 64)
    ref_dense = sdl.dense_attn(dev["q"], dev["k"], dev["v"])
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [torch.empty_like(ref) for _ in range(4)]
    torch.cuda.synchronize()
    for n in range(150):
        with torch.cuda.stream(streams[n % 2]):
            if n % 3 == 2:
                sdl.dense_attn(dev["q"], dev["k"], dev["v"], out=outs[2 + n % 2])
            else:
                sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, 64, out=outs[n % 2])
    torch.cuda.synchronize()
    assert sdl.last_device_status() == sdl.SDL_OK
    assert torch.equal(outs[0], ref) and torch.equal(outs[1], ref)
    assert torch.equal(outs[2], ref_dense) and torch.equal(outs[3], ref_dense)


@pytest.mark.parametrize("dtype,L,H,Hkv,d", [("bf16", 1024, 4, 2, 128), ("bf16", 640, 2, 2, 64),
                                             ("fp32", 512, 2, 2, 64)])
def test_dense_attention(dtype, L, H, Hkv, d):
    w = synth.small_workload(dtype=dtype, L=L, H=H, H_kv=Hkv, d=d)
    host, dev = _inputs(w)
    O, lse = sdl.dense_attn(dev["q"], dev["k"], dev["v"], want_lse=True)
    Ow, lw = oracle.attention(host["q"], host["k"], host["v"], 64)
    check_close(bf16_to_f64(O).transpose(0, 2, 1, 3), Ow, dtype)
    assert np.abs(lse.cpu().numpy() - lw).max() <= TOL[dtype]["lse"]


def test_strided_fused_qkv_layout():
    """Q, K, V as views into one [B, L, H + 2*H_kv, d] buffer (fused projection)."""
    w = synth.small_workload(L=512, H=4, H_kv=2, d=128)
    host, dev = _inputs(w)
    fused = torch.empty((1, 512, 8, 128), dtype=torch.bfloat16, device="cuda")
    fused[:, :, 0:4] = dev["q"]
    fused[:, :, 4:6] = dev["k"]
    fused[:, :, 6:8] = dev["v"]
    q, k, v = fused[:, :, 0:4], fused[:, :, 4:6], fused[:, :, 6:8]
    o_big = torch.zeros((1, 512, 4, 256), dtype=torch.bfloat16, device="cuda")
    o = o_big[..., 64:192]  # strided output
    mask = _random_mask(1, 4, 8, 0.5, np.random.default_rng(1))
    rp, ci = _mask_to_csr(mask)
    sdl.sparse_attn(q, k, v, rp, ci, 64, out=o)
    Ow, _ = oracle.attention(host["q"], host["k"], host["v"], 64, mask=mask)
    check_close(bf16_to_f64(o).transpose(0, 2, 1, 3), Ow, "bf16")
    assert torch.count_nonzero(o_big[..., :64]) == 0 and torch.count_nonzero(o_big[..., 192:]) == 0
    P = sdl.block_scores(q, k, 64)
    want = oracle.block_scores(host["q"], host["k"], 64)
    assert np.abs(P.cpu().numpy() - want).max() / want.min() < 1e-4


def test_bad_list_entry_is_reported_and_skipped():
    w = synth.small_workload(L=256, H=1, H_kv=1, d=128)
    _, dev = _inputs(w)
    rp = torch.tensor([0, 2, 3, 4, 6], dtype=torch.int32, device="cuda")
    ci = torch.tensor([0, 99, 1, 2, 3, 3], dtype=torch.int32, device="cuda")  # 99 out of range
    sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, 64)
    assert sdl.last_device_status() == sdl.SDL_ERR_BAD_MASK
    assert sdl.last_device_status() == sdl.SDL_OK  # reading clears it


def test_argument_errors_do_not_launch():
    q = torch.zeros((1, 256, 2, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sdl.SdlError) as e:
        sdl.dense_attn(q, q[:, :, :1], q[:, :, :1], block=96)
    assert e.value.status == sdl.SDL_ERR_UNSUPPORTED
    k3 = torch.zeros((1, 256, 3, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sdl.SdlError) as e:
        sdl.dense_attn(q, k3, k3)  # 2 query heads over 3 KV heads
    assert e.value.status == sdl.SDL_ERR_INVALID_ARG
    P = torch.rand(1, 2, 4, 4, device="cuda")
    with pytest.raises(sdl.SdlError) as e:
        sdl.select_mask(P, 0.5, 64, 256, col_idx=torch.empty(3, dtype=torch.int32, device="cuda"))
    assert e.value.status == sdl.SDL_ERR_CAPACITY


def test_bounded_wait_times_out_and_the_context_survives():
    """A wait on a phase nothing completes gives up at its limit and raises the timeout
    bit, which sdl_last_device_status reports once and clears; kernels still run."""
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    sdl.wait_selfcheck(2_000_000)  # 2 ms
    t1.record()
    assert sdl.last_device_status() == sdl.SDL_ERR_TIMEOUT
    assert 1.5 <= t0.elapsed_time(t1) < 100.0
    assert sdl.last_device_status() == sdl.SDL_OK
    with pytest.raises(sdl.SdlError):
        sdl.wait_selfcheck(10)  # below the smallest limit
    w = synth.small_workload(L=256, H=2, H_kv=2, d=64, bs=64, sparsity=0.5)
    host, dev = _inputs(w)
    O = sdl.dense_attn(dev["q"], dev["k"], dev["v"])
    assert sdl.last_device_status() == sdl.SDL_OK
    Ow, _ = oracle.attention(host["q"], host["k"], host["v"], 64)
    check_close(bf16_to_f64(O).transpose(0, 2, 1, 3), Ow, "bf16")


@pytest.mark.parametrize("B,L,H,Hkv,density", [(1, 1024, 4, 2, 0.3), (2, 1024, 4, 2, 0.2),
                                               (1, 576, 3, 1, 0.5), (1, 4096, 8, 8, 0.12)])
def test_listed_attention_equals_scheduled(B, L, H, Hkv, density):
    """Tiles and lists prebuilt once (sdl_tile_lists) give the scheduled path's result
    bit for bit, LSE included, and the records hold the tiles in take order with the
    union of their two query blocks' kept blocks in step order: blocks only the first
    keeps paired with blocks only the second keeps, then the unpaired rest of either,
    then the blocks both keep, each class ascending."""
    w = synth.small_workload(B=B, L=L, H=H, H_kv=Hkv, d=128, bs=64)
    _, dev = _inputs(w)
    nb = L // 64
    rng = np.random.default_rng(B * L + H)
    mask = _random_mask(B, H, nb, density, rng)
    rp, ci = _mask_to_csr(mask)
    plan = sdl.tile_plan(rp, ci, B, H, L, 64)
    order = sdl.tile_order(rp, plan, B, H, L, 64)
    lists = sdl.tile_lists(rp, ci, plan, order, B, H, L, 64)
    O1, l1 = sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, 64, want_lse=True, plan=plan,
                             order=order)
    O2, l2 = sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, 64, want_lse=True,
                             lists=lists)
    assert sdl.last_device_status() == sdl.SDL_OK
    assert torch.equal(O1, O2) and torch.equal(l1, l2)
    # the records, rebuilt on the host
    n_qt = (nb + 1) // 2
    n = B * H * n_qt
    cap = (nb + 7) // 8 * 8
    raw = lists.cpu().numpy()
    rec = raw[:n * 32].view(np.int32).reshape(n, 8)
    ent = raw[n * 32:n * 32 + n * cap * 2].view(np.uint16).reshape(n, cap)
    o = order.cpu().numpy()
    pl = plan.cpu().numpy().reshape(-1, 2)
    assert np.array_equal(rec[:, 0], o)
    for r in range(n):
        item = o[r]
        bh = item // n_qt
        b, h = bh // H, bh % H
        rows = [qb for qb in pl[item]]
        want_t = [qb * 64 if qb >= 0 else L for qb in rows]
        assert list(rec[r, 2:4]) == want_t
        keep = np.zeros((2, nb), bool)
        for s, qb in enumerate(rows):
            if qb >= 0:
                keep[s] = mask[b, h, qb].astype(bool)
        a_only = np.nonzero(keep[0] & ~keep[1])[0]
        b_only = np.nonzero(keep[1] & ~keep[0])[0]
        both = np.nonzero(keep[0] & keep[1])[0]
        npair = min(len(a_only), len(b_only))
        union = np.concatenate([np.stack([a_only[:npair], b_only[:npair]], 1).reshape(-1),
                                a_only[npair:], b_only[npair:], both]).astype(np.int64)
        assert rec[r, 1] == len(union)
        e = ent[r, :len(union)]
        assert np.array_equal(e & 0x3FFF, union)
        assert np.array_equal((e >> 14) & 1, keep[0][union]) and \
            np.array_equal((e >> 15) & 1, keep[1][union])


def test_listed_attention_adjacent_pairs_and_bad_record():
    """Lists built without a plan or order pair adjacent query blocks in tile order,
    which is what the plain call does; a record naming no tile is reported."""
    B, L, H, Hkv = 1, 1024, 4, 2
    w = synth.small_workload(B=B, L=L, H=H, H_kv=Hkv, d=128, bs=64)
    _, dev = _inputs(w)
    nb = L // 64
    mask = _random_mask(B, H, nb, 0.3, np.random.default_rng(5))
    rp, ci = _mask_to_csr(mask)
    lists = sdl.tile_lists(rp, ci, None, None, B, H, L, 64)
    O1 = sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, 64)
    O2 = sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, 64, lists=lists)
    assert sdl.last_device_status() == sdl.SDL_OK
    assert torch.equal(O1, O2)
    bad = lists.clone()
    bad[:4] = torch.tensor(np.array([1 << 20], np.int32).view(np.uint8), device=bad.device)
    sdl.sparse_attn(dev["q"], dev["k"], dev["v"], rp, ci, 64, lists=bad)
    assert sdl.last_device_status() == sdl.SDL_ERR_BAD_MASK
    assert sdl.last_device_status() == sdl.SDL_OK
