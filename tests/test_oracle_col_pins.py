"""Pins for the column-sparse (PulseCol) part of the fp64 oracle.

The PulseCol abstract keeps, per query head, a set of key tokens (columns of
the attention matrix) for all of the head's query rows, found at an early step
and refreshed at a few later ones.  The oracle's reading: a column's score is
the mean over query blocks of the softmax of the block-mean query against every
key token; each head keeps its Lc = 64 * floor((1 - s) * L / 64 + 0.5) (at
least 64) best columns, ties to the lower index; attention runs over those
columns only.  Every check here is against something outside the oracle: torch
fp64, NumPy sorting, closed forms and invariants.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

RNG = np.random.default_rng(4321)


def rand_bf16(shape, scale=1.0, rng=RNG):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    bits = x.view(np.uint32)
    return ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16).astype(np.uint16)


def t64(a):
    return torch.from_numpy(oracle.widen(a))


def test_col_budget_values():
    assert oracle.col_budget(8192, 0.9) == 832    # 819.2 -> 12.8 tiles -> 13
    assert oracle.col_budget(2048, 0.8) == 384    # 409.6 -> 6.4 tiles -> 6
    assert oracle.col_budget(256, 0.9) == 64      # at least one tile
    assert oracle.col_budget(1024, 0.0) == 1024
    assert oracle.col_budget(1000, 0.5) == -1     # L not whole tiles
    assert oracle.col_budget(1024, 1.0) == -1


def _torch_col_scores(q, k, bs, scale):
    B, L, H, d = q.shape
    Hkv = k.shape[2]
    qb = F.avg_pool1d(t64(q).permute(0, 2, 3, 1).reshape(B * H, d, L), bs, bs)
    qb = qb.reshape(B, H, d, -1).transpose(2, 3)                      # [B, H, nb, d]
    kt = t64(k).permute(0, 2, 1, 3).repeat_interleave(H // Hkv, 1)    # [B, H, L, d]
    return torch.softmax(qb @ kt.transpose(2, 3) * scale, dim=-1).mean(2).numpy()


@pytest.mark.parametrize("H,Hkv,bs", [(2, 2, 64), (6, 2, 64), (2, 1, 128)])
def test_col_scores_match_torch(H, Hkv, bs):
    q = rand_bf16((2, 512, H, 64), 3.0)
    k = rand_bf16((2, 512, Hkv, 64))
    got = oracle.col_scores(q, k, bs)
    assert np.allclose(got, _torch_col_scores(q, k, bs, 1 / 8), rtol=1e-12, atol=1e-16)


def test_col_scores_are_a_distribution_per_head():
    q = rand_bf16((1, 512, 3, 64), 4.0)
    k = rand_bf16((1, 512, 3, 64))
    S = oracle.col_scores(q, k, 64)
    assert np.all(S > 0)
    assert np.allclose(S.sum(-1), 1.0, rtol=0, atol=1e-12)


def test_identical_keys_give_uniform_columns():
    q = rand_bf16((1, 256, 2, 64), 2.0)
    k = np.ascontiguousarray(np.tile(rand_bf16((1, 1, 2, 64)), (1, 256, 1, 1)))
    assert np.allclose(oracle.col_scores(q, k, 64), 1 / 256, rtol=0, atol=1e-15)


def test_col_select_matches_lexsort():
    S = RNG.random((2, 3, 512))
    for s in (0.3, 0.8, 0.95):
        cols = oracle.col_select(S, s)
        Lc = oracle.col_budget(512, s)
        assert cols.shape == (2, 3, Lc)
        for b in range(2):
            for h in range(3):
                order = np.lexsort((np.arange(512), -S[b, h]))  # score desc, index asc
                assert np.array_equal(cols[b, h], np.sort(order[:Lc]))


def test_col_select_ties_go_to_lower_columns():
    S = np.zeros((1, 1, 256))
    S[0, 0, 200:] = 1.0          # 56 clear winners
    cols = oracle.col_select(S, 0.75)  # Lc = 64: 56 winners + the 8 lowest tied columns
    assert np.array_equal(cols[0, 0], np.r_[np.arange(8), np.arange(200, 256)])


def test_col_select_keeps_the_largest_total():
    S = RNG.random((1, 2, 192))
    for s in (0.5, 0.6):               # Lc = 128 and 64 of 192
        cols = oracle.col_select(S, s)
        Lc = oracle.col_budget(192, s)
        assert cols.shape[2] == Lc
        for h in range(2):
            kept = S[0, h, cols[0, h]].sum()
            assert kept == pytest.approx(np.sort(S[0, h])[-Lc:].sum(), rel=1e-12)


def _sdpa_cols(q, k, v, cols, scale):
    B, L, H, d = q.shape
    g = H // k.shape[2]
    qt = t64(q).permute(0, 2, 1, 3)
    kt = t64(k).permute(0, 2, 1, 3).repeat_interleave(g, 1)
    vt = t64(v).permute(0, 2, 1, 3).repeat_interleave(g, 1)
    am = torch.zeros((B, H, 1, L), dtype=torch.bool)
    for b in range(B):
        for h in range(H):
            am[b, h, 0, torch.from_numpy(cols[b, h].astype(np.int64))] = True
    return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=am, scale=scale).numpy()


@pytest.mark.parametrize("H,Hkv", [(2, 2), (4, 2)])
def test_col_attention_matches_masked_sdpa(H, Hkv):
    q = rand_bf16((1, 256, H, 64), 2.0)
    k = rand_bf16((1, 256, Hkv, 64))
    v = rand_bf16((1, 256, Hkv, 64))
    cols = np.stack([np.stack([np.sort(RNG.choice(256, 64, replace=False)) for _ in range(H)])])
    O, lse = oracle.col_attention(q, k, v, cols.astype(np.int32))
    want = _sdpa_cols(q, k, v, cols, 1 / 8)
    assert np.allclose(O, want, rtol=1e-10, atol=1e-12)
    # LSE by its definition on the kept columns
    qt, kt = oracle.widen(q), oracle.widen(k)
    for h in range(H):
        z = qt[0, :, h, :] @ kt[0, cols[0, h], h // (H // Hkv), :].T / 8
        assert np.allclose(lse[0, h], np.log(np.exp(z).sum(-1)), rtol=1e-12)


def test_all_columns_is_dense_attention():
    q = rand_bf16((1, 128, 2, 64), 2.0)
    k = rand_bf16((1, 128, 2, 64))
    v = rand_bf16((1, 128, 2, 64))
    cols = np.tile(np.arange(128, dtype=np.int32), (1, 2, 1))
    O, lse = oracle.col_attention(q, k, v, cols)
    Od, lsed = oracle.attention(q, k, v, 64)
    assert np.allclose(O, Od, rtol=1e-12, atol=1e-14)
    assert np.allclose(lse, lsed, rtol=1e-12)


def test_constant_v_gives_constant_output_on_any_columns():
    q = rand_bf16((1, 128, 2, 64), 3.0)
    k = rand_bf16((1, 128, 2, 64))
    v = np.ascontiguousarray(np.tile(rand_bf16((1, 1, 2, 64)), (1, 128, 1, 1)))
    cols = np.array([[[3, 9, 64, 100], [0, 1, 2, 127]]], dtype=np.int32)
    O, _ = oracle.col_attention(q, k, v, cols)
    for h in range(2):
        assert np.allclose(O[0, h], oracle.widen(v)[0, 0, h], rtol=1e-12)
