"""Pins for the fp64 CPU oracle, independent of the oracle's own code.

Each test checks one oracle function against something fixed outside it: a
closed form, an invariant of the definition, brute force over all masks on a
tiny case, or an independent library routine (torch fp64 on the CPU).  The
definitions follow the Step-dLLM abstract (block-sparse mask rebuilt at anchor
steps under a head-adaptive global budget; block-sparse attention), with the
block score and the selection rule read as: mean-pooled Q and K per block,
pooled QK^T * scale, row softmax; keep every diagonal block and give the rest
of the budget to the largest scores of all heads together.
"""
import itertools
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth

RNG = np.random.default_rng(1234)


def rand_bf16(shape, scale=1.0, rng=RNG):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    bits = x.view(np.uint32)
    return ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16).astype(np.uint16)


def t64(a):
    return torch.from_numpy(oracle.widen(a))


# ----------------------------------------------------------------------- pool


def test_pool_matches_avg_pool1d():
    x = rand_bf16((2, 256, 3, 32))
    got = oracle.pool(x, 64)
    xt = t64(x).permute(0, 2, 3, 1).reshape(6, 32, 256)  # (B*H, d, L)
    want = F.avg_pool1d(xt, 64, 64).reshape(2, 3, 32, 4).permute(0, 1, 3, 2)
    assert np.allclose(got, want.numpy(), rtol=0, atol=1e-14)


def test_pool_constant_blocks_are_fixed_points():
    vals = RNG.standard_normal((1, 4, 2, 16)).astype(np.float32)
    x = np.repeat(vals, 128, axis=1)  # every token of block i equals vals[:, i]
    got = oracle.pool(np.ascontiguousarray(x), 128)
    assert np.array_equal(got, vals.transpose(0, 2, 1, 3).astype(np.float64))


def test_pool_respects_strides():
    big = rand_bf16((1, 128, 4, 64))
    view = big[:, :, 1:3, :]  # non-contiguous head axis
    got = oracle.pool(view, 64)
    want = oracle.pool(np.ascontiguousarray(view), 64)
    assert np.array_equal(got, want)


# --------------------------------------------------------------- block scores


def _torch_scores(q, k, bs, scale):
    B, L, H, d = q.shape
    Hkv = k.shape[2]
    qb = F.avg_pool1d(t64(q).permute(0, 2, 3, 1).reshape(B * H, d, L), bs, bs)
    kb = F.avg_pool1d(t64(k).permute(0, 2, 3, 1).reshape(B * Hkv, d, L), bs, bs)
    qb = qb.reshape(B, H, d, -1).transpose(2, 3)
    kb = kb.reshape(B, Hkv, d, -1).transpose(2, 3).repeat_interleave(H // Hkv, dim=1)
    return torch.softmax(qb @ kb.transpose(2, 3) * scale, dim=-1).numpy()


@pytest.mark.parametrize("H,Hkv,bs", [(4, 4, 64), (6, 2, 64), (2, 1, 128)])
def test_scores_match_torch(H, Hkv, bs):
    q = rand_bf16((1, 512, H, 64), 3.0)
    k = rand_bf16((1, 512, Hkv, 64))
    got = oracle.block_scores(q, k, bs)
    want = _torch_scores(q, k, bs, 1 / 8)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-15)


def test_score_rows_sum_to_one():
    q = rand_bf16((2, 512, 2, 64), 4.0)
    k = rand_bf16((2, 512, 2, 64))
    P = oracle.block_scores(q, k, 64)
    assert np.all(P > 0)
    assert np.allclose(P.sum(-1), 1.0, rtol=0, atol=1e-12)


def test_identical_key_blocks_give_uniform_rows():
    q = rand_bf16((1, 256, 2, 64), 2.0)
    kblk = rand_bf16((1, 64, 2, 64))
    k = np.ascontiguousarray(np.tile(kblk, (1, 4, 1, 1)))
    P = oracle.block_scores(q, k, 64)
    assert np.allclose(P, 0.25, rtol=0, atol=1e-14)


def test_scale_argument():
    q = rand_bf16((1, 256, 1, 64), 2.0)
    k = rand_bf16((1, 256, 1, 64))
    assert np.allclose(oracle.block_scores(q, k, 64, scale=0.0), 0.25, atol=1e-15)
    a = oracle.block_scores(q, k, 64, scale=0.25)
    assert np.allclose(a, _torch_scores(q, k, 64, 0.25), rtol=1e-12)
    assert np.allclose(oracle.block_scores(q, k, 64), _torch_scores(q, k, 64, 1 / 8), rtol=1e-12)


# --------------------------------------------------------------------- budget


def test_budget_values():
    # floor((1 - s) * H * nb^2 + 0.5): 0.2*32768 = 6553.6 -> 6554, 0.1*524288 = 52428.8 ->
    # 52429, 0.1*1835008 = 183500.8 -> 183501, 0.05*8388608 = 419430.4 -> 419430
    assert oracle.budget(2, 8, 0.5) == 64
    assert oracle.budget(32, 32, 0.8) == 6554
    assert oracle.budget(32, 128, 0.9) == 52429
    assert oracle.budget(28, 256, 0.9) == 183501
    assert oracle.budget(32, 512, 0.95) == 419430
    assert oracle.budget(4, 4, 0.0) == 64


def test_budget_invalid():
    assert oracle.budget(2, 8, 1.0) == -1
    assert oracle.budget(2, 8, -0.1) == -1
    assert oracle.budget(2, 8, float("nan")) == -1
    # 0.1 * 128 + 0.5 -> 13 kept, below the 16 diagonal blocks
    assert oracle.budget(2, 8, 0.9) == -1
    assert oracle.budget(2, 8, 0.875) == 16  # exactly the diagonal


# ------------------------------------------------------------------ selection


def _offdiag(mask):
    B, H, nb, _ = mask.shape
    eye = np.eye(nb, dtype=bool)
    return mask[:, :, ~eye]


def test_select_brute_force_all_subsets():
    """Global top-k == the subset of k off-diagonal blocks with the largest total score."""
    rng = np.random.default_rng(7)
    H, nb = 2, 3
    P = rng.random((1, H, nb, nb))
    free = [(h, i, j) for h in range(H) for i in range(nb) for j in range(nb) if i != j]
    for k in range(0, len(free) + 1):
        total = H * nb * nb
        s = 1.0 - (H * nb + k) / total
        mask, tau, kept = oracle.select(P, s)
        assert kept == H * nb + k
        best, best_set = -1.0, None
        for sub in itertools.combinations(range(len(free)), k):
            m = sum(P[0][free[x]] for x in sub)
            if m > best:
                best, best_set = m, set(sub)
        want = np.zeros_like(mask)
        for h in range(H):
            for i in range(nb):
                want[0, h, i, i] = 1
        for x in best_set:
            want[(0,) + free[x]] = 1
        assert np.array_equal(mask, want), k


def test_select_ties_go_to_lower_flat_index():
    H, nb = 2, 4
    P = np.full((1, H, nb, nb), 0.25)
    k = 5
    s = 1.0 - (H * nb + k) / (H * nb * nb)
    mask, tau, kept = oracle.select(P, s)
    flat_free = [f for f in range(H * nb * nb) if (f // nb) % nb != f % nb]
    want = np.zeros(H * nb * nb, dtype=np.uint8)
    want[[f for f in range(H * nb * nb) if (f // nb) % nb == f % nb]] = 1
    want[flat_free[:k]] = 1
    assert np.array_equal(mask.reshape(-1), want)
    assert tau[0] == 0.25


def test_select_matches_lexsort_and_counts():
    rng = np.random.default_rng(11)
    B, H, nb, s = 2, 4, 16, 0.8
    P = rng.random((B, H, nb, nb))
    mask, tau, kept = oracle.select(P, s)
    kb = math.floor((1 - s) * H * nb * nb + 0.5)
    assert kept == B * kb
    for b in range(B):
        assert mask[b].sum() == kb
        assert all(mask[b, h, i, i] == 1 for h in range(H) for i in range(nb))
        flat = np.arange(H * nb * nb)
        off = (flat // nb) % nb != flat % nb
        vals = P[b].reshape(-1)[off]
        idx = flat[off]
        order = np.lexsort((idx, -vals))  # by -P, then by index
        want = np.zeros(H * nb * nb, dtype=np.uint8)
        want[~off] = 1
        want[idx[order[:kb - H * nb]]] = 1
        assert np.array_equal(mask[b].reshape(-1), want)
        assert tau[b] == vals[order[kb - H * nb - 1]]


def test_select_extremes():
    P = RNG.random((1, 3, 8, 8))
    mask, _, kept = oracle.select(P, 0.0)
    assert kept == 3 * 64 and mask.all()
    s = 1.0 - (3 * 8) / (3 * 64)
    mask, tau, kept = oracle.select(P, s)
    assert kept == 24
    assert np.array_equal(mask[0], np.broadcast_to(np.eye(8, dtype=np.uint8), (3, 8, 8)))
    assert tau[0] == math.inf


def test_select_single_head_is_per_head_topk():
    P = RNG.random((1, 1, 16, 16))
    s = 0.7
    mask, _, _ = oracle.select(P, s)
    k = math.floor(0.3 * 256 + 0.5) - 16
    off = ~np.eye(16, dtype=bool)
    top = torch.topk(torch.from_numpy(P[0, 0][off]), k).indices.numpy()
    want = np.zeros(off.sum(), dtype=np.uint8)
    want[top] = 1
    assert np.array_equal(mask[0, 0][off], want)


def test_select_per_head_brute_force_and_counts():
    """Uniform per-head budget (the prior methods' rule): in every head, the kept
    off-diagonal set is the one of largest total score among all subsets of that
    head's per-head size, the diagonal is kept, and each head keeps the same count."""
    rng = np.random.default_rng(11)
    H, nb = 3, 3
    P = rng.random((1, H, nb, nb))
    free_h = [(i, j) for i in range(nb) for j in range(nb) if i != j]
    for k in range(0, len(free_h) + 1):
        s = 1.0 - (nb + k) / (nb * nb)
        mask, tau, kept = oracle.select(P, s, per_head=True)
        assert kept == H * (nb + k)
        for h in range(H):
            assert mask[0, h].sum() == nb + k
            assert all(mask[0, h, i, i] == 1 for i in range(nb))
            best, best_set = -1.0, None
            for sub in itertools.combinations(range(len(free_h)), k):
                tot = sum(P[0, h, free_h[x][0], free_h[x][1]] for x in sub)
                if tot > best:
                    best, best_set = tot, set(sub)
            got = {x for x, (i, j) in enumerate(free_h) if mask[0, h, i, j]}
            assert got == best_set


def test_select_per_head_differs_from_global_on_skewed_heads():
    """A head with a concentrated row distribution gets fewer blocks under the global
    budget than under the per-head one; per head, every head gets the same count."""
    nb = 8
    P = np.full((1, 2, nb, nb), 1.0 / nb)
    P[0, 0] = 1e-3
    np.fill_diagonal(P[0, 0], 1.0)
    mask_g, _, _ = oracle.select(P, 0.5)
    mask_h, _, _ = oracle.select(P, 0.5, per_head=True)
    assert mask_h[0, 0].sum() == mask_h[0, 1].sum()
    assert mask_g[0, 0].sum() < mask_g[0, 1].sum()


def test_select_is_head_adaptive():
    """A concentrated head keeps few blocks; a flat head with larger entries keeps many."""
    nb = 16
    conc = np.full((nb, nb), 0.2 / (nb - 1))
    conc[:, 3] = 0.8  # all mass on one key block
    flat = np.full((nb, nb), 1.0 / nb)
    P = np.stack([conc, flat])[None]
    s = 1.0 - (2 * nb + 40) / (2 * nb * nb)
    mask, _, _ = oracle.select(P, s)
    per_head = _offdiag(mask).reshape(2, -1).sum(-1)
    assert per_head[0] == nb - 1  # only column 3 off the diagonal (0.8 > 1/16 > 0.2/15)
    assert per_head[1] == 40 - (nb - 1)


# ------------------------------------------------------------------ attention


def _expand_mask(mask, bs):
    return torch.from_numpy(mask.astype(bool)).repeat_interleave(bs, 2).repeat_interleave(bs, 3)


def _sdpa(q, k, v, mask=None, bs=64, scale=None):
    B, L, H, d = q.shape
    g = H // k.shape[2]
    qt = t64(q).permute(0, 2, 1, 3)
    kt = t64(k).permute(0, 2, 1, 3).repeat_interleave(g, 1)
    vt = t64(v).permute(0, 2, 1, 3).repeat_interleave(g, 1)
    am = None if mask is None else _expand_mask(mask, bs)
    return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=am, scale=scale).numpy()


def _rand_mask(B, H, nb, p, rng):
    m = (rng.random((B, H, nb, nb)) < p).astype(np.uint8)
    for i in range(nb):
        m[:, :, i, i] = 1
    return m


@pytest.mark.parametrize("H,Hkv", [(2, 2), (4, 1), (6, 3)])
def test_dense_matches_sdpa(H, Hkv):
    q = rand_bf16((1, 256, H, 64), 2.0)
    k = rand_bf16((1, 256, Hkv, 64))
    v = rand_bf16((1, 256, Hkv, 64))
    O, _ = oracle.attention(q, k, v, 64)
    assert np.allclose(O, _sdpa(q, k, v), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("bs,H,Hkv", [(64, 4, 2), (128, 2, 2)])
def test_sparse_matches_masked_sdpa(bs, H, Hkv):
    rng = np.random.default_rng(5)
    q = rand_bf16((2, 512, H, 64), 3.0, rng)
    k = rand_bf16((2, 512, Hkv, 64), 1.0, rng)
    v = rand_bf16((2, 512, Hkv, 64), 1.0, rng)
    mask = _rand_mask(2, H, 512 // bs, 0.3, rng)
    O, _ = oracle.attention(q, k, v, bs, mask=mask)
    assert np.allclose(O, _sdpa(q, k, v, mask, bs), rtol=1e-10, atol=1e-12)


def test_all_ones_mask_is_dense():
    q, k, v = (rand_bf16((1, 256, 2, 64)) for _ in range(3))
    O1, l1 = oracle.attention(q, k, v, 64, mask=np.ones((1, 2, 4, 4), np.uint8))
    O2, l2 = oracle.attention(q, k, v, 64)
    assert np.array_equal(O1, O2) and np.array_equal(l1, l2)


def test_constant_v_gives_constant_output():
    q = rand_bf16((1, 256, 2, 64), 3.0)
    k = rand_bf16((1, 256, 2, 64))
    c = rand_bf16((64,))
    v = np.ascontiguousarray(np.broadcast_to(c, (1, 256, 2, 64)))
    mask = _rand_mask(1, 2, 4, 0.4, np.random.default_rng(2))
    O, _ = oracle.attention(q, k, v, 64, mask=mask)
    assert np.allclose(O, oracle.widen(c), rtol=0, atol=1e-13)


def test_permuting_tokens_inside_a_key_block():
    rng = np.random.default_rng(3)
    q, k, v = (rand_bf16((1, 256, 2, 64), 1.0, rng) for _ in range(3))
    mask = _rand_mask(1, 2, 4, 0.5, rng)
    perm = np.arange(256)
    perm[64:128] = 64 + rng.permutation(64)
    O1, l1 = oracle.attention(q, k, v, 64, mask=mask)
    O2, l2 = oracle.attention(q, np.ascontiguousarray(k[:, perm]), np.ascontiguousarray(v[:, perm]),
                              64, mask=mask)
    assert np.allclose(O1, O2, rtol=1e-12, atol=1e-14) and np.allclose(l1, l2, rtol=1e-13)


def test_diagonal_only_is_blockwise_dense():
    q, k, v = (rand_bf16((1, 256, 2, 64)) for _ in range(3))
    mask = np.broadcast_to(np.eye(4, dtype=np.uint8), (1, 2, 4, 4))
    O, _ = oracle.attention(q, k, v, 64, mask=mask)
    for i in range(4):
        sl = slice(64 * i, 64 * (i + 1))
        want = _sdpa(q[:, sl].copy(), k[:, sl].copy(), v[:, sl].copy())
        assert np.allclose(O[:, :, sl], want, rtol=1e-10, atol=1e-12)


def test_zero_query_closed_form():
    """q = 0: uniform weights over the kept tokens; LSE = log(kept tokens)."""
    q = np.zeros((1, 256, 2, 64), np.uint16)
    k = rand_bf16((1, 256, 2, 64))
    v = rand_bf16((1, 256, 2, 64))
    mask = _rand_mask(1, 2, 4, 0.5, np.random.default_rng(9))
    O, lse = oracle.attention(q, k, v, 64, mask=mask)
    vw = oracle.widen(v)
    for h in range(2):
        for i in range(4):
            cols = np.nonzero(mask[0, h, i])[0]
            toks = np.concatenate([np.arange(64 * j, 64 * j + 64) for j in cols])
            want = vw[0, toks, h].mean(axis=0)
            assert np.allclose(O[0, h, 64 * i:64 * i + 64], want, rtol=0, atol=1e-14)
            assert np.allclose(lse[0, h, 64 * i:64 * i + 64], math.log(len(toks)), atol=1e-14)


def test_weights_are_a_distribution_on_kept_tokens():
    """V = identity (d = L) makes O the attention weights themselves."""
    L = 128
    q = rand_bf16((1, L, 1, L), 0.3)
    k = rand_bf16((1, L, 1, L), 0.3)
    v = np.ascontiguousarray(np.eye(L, dtype=np.float32)[None, :, None, :])
    qf, kf = oracle.widen(q).astype(np.float32), oracle.widen(k).astype(np.float32)
    mask = np.array([[[[1, 0], [1, 1]]]], np.uint8)
    O, lse = oracle.attention(qf, kf, v, 64, mask=mask)
    W = O[0, 0]
    assert np.all(W >= 0)
    assert np.allclose(W.sum(-1), 1.0, atol=1e-13)
    assert np.all(W[:64, 64:] == 0)  # block (0, 1) is not kept
    logits = (oracle.widen(q)[0, :, 0] @ oracle.widen(k)[0, :, 0].T) / math.sqrt(L)
    ref = torch.logsumexp(torch.from_numpy(logits[:64, :64]), -1).numpy()
    assert np.allclose(lse[0, 0, :64], ref, rtol=1e-13)


def test_row_subset_matches_full():
    q, k, v = (rand_bf16((2, 256, 4, 64)) for _ in range(3))
    mask = _rand_mask(2, 4, 4, 0.5, np.random.default_rng(4))
    O, lse = oracle.attention(q, k, v, 64, mask=mask)
    rows = np.array([[0, 0, 0], [1, 3, 255], [0, 2, 100], [1, 1, 64]])
    Os, ls = oracle.attention(q, k, v, 64, mask=mask, rows=rows)
    for r, (b, h, t) in enumerate(rows):
        assert np.array_equal(Os[r], O[b, h, t]) and ls[r] == lse[b, h, t]


def test_oracle_reads_synth_fp32_and_bf16():
    for dt in ("fp32", "bf16"):
        w = synth.small_workload(dtype=dt, L=128, H=2, H_kv=2, d=64)
        x = synth.host_inputs(w, 0)
        O, _ = oracle.attention(x["q"], x["k"], x["v"], 64)
        assert np.allclose(O, _sdpa(x["q"], x["k"], x["v"]), rtol=1e-10, atol=1e-12)
