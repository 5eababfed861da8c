"""Comparison helpers shared by the GPU parity tests (host side only)."""
from __future__ import annotations

import numpy as np

# Tolerances: output O in max-abs / mean-abs for bf16 workloads, max-abs for fp32;
# the mask is exact except for entries whose deciding score is within 1e-5
# relative of the oracle's threshold.
TOL = {"bf16": dict(max_abs=1e-2, mean_abs=1e-3, lse=1e-3),
       "fp32": dict(max_abs=1e-4, mean_abs=1e-4, lse=1e-5)}
TIE_REL = 1e-5


def csr_to_mask(row_ptr: np.ndarray, col_idx: np.ndarray, B: int, H: int, nb: int) -> np.ndarray:
    mask = np.zeros((B * H * nb, nb), dtype=np.uint8)
    for r in range(B * H * nb):
        mask[r, col_idx[row_ptr[r]:row_ptr[r + 1]]] = 1
    return mask.reshape(B, H, nb, nb)


def check_csr(row_ptr: np.ndarray, col_idx: np.ndarray, B: int, H: int, nb: int, budget: int):
    """Structural validity: counts, ascending lists, in range, diagonal present."""
    assert row_ptr[0] == 0 and row_ptr[-1] == budget
    assert np.all(np.diff(row_ptr) >= 1)
    for r in range(B * H * nb):
        lst = col_idx[row_ptr[r]:row_ptr[r + 1]]
        assert np.all(np.diff(lst) > 0), f"row {r} not ascending"
        assert lst[0] >= 0 and lst[-1] < nb
        assert (r % nb) in lst, f"row {r} misses its diagonal block"


def compare_masks(gpu_mask, oracle_mask, P_oracle, tau):
    """Returns the number of excused near-threshold differences; fails on any other."""
    diff = gpu_mask != oracle_mask
    if not diff.any():
        return 0
    B = gpu_mask.shape[0]
    excused = 0
    for b in range(B):
        idx = np.argwhere(diff[b])
        for h, i, j in idx:
            p = P_oracle[b, h, i, j]
            assert i != j, "diagonal block differs"
            assert abs(p - tau[b]) <= TIE_REL * tau[b], (
                f"mask differs at b={b} h={h} i={i} j={j}: P={p!r}, threshold={tau[b]!r}")
            excused += 1
    return excused


def bf16_to_f64(t):
    import torch
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def check_close(got: np.ndarray, want: np.ndarray, dtype: str, what: str = "O"):
    tol = TOL[dtype]
    err = np.abs(got - want)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= tol["max_abs"], f"{what}: max abs error {mx:.3e} > {tol['max_abs']}"
    assert mean <= tol["mean_abs"], f"{what}: mean abs error {mean:.3e} > {tol['mean_abs']}"
    return mx, mean


def sample_rows(B, H, L, bs, lists_len, n_blocks=4, rows_per_block=8, seed=0):
    """(b, h, t) triples: for each (b, h) the first and last query block, the block
    with the longest kept list, and random others; a few rows in each."""
    rng = np.random.default_rng(seed)
    nb = L // bs
    out = []
    for b in range(B):
        for h in range(H):
            lens = lists_len[b, h]
            blocks = {0, nb - 1, int(np.argmax(lens))}
            while len(blocks) < min(n_blocks, nb):
                blocks.add(int(rng.integers(nb)))
            for i in sorted(blocks):
                rows = {i * bs, i * bs + bs - 1}
                while len(rows) < min(rows_per_block, bs):
                    rows.add(int(i * bs + rng.integers(bs)))
                out.extend((b, h, t) for t in sorted(rows))
    return np.array(out, dtype=np.int64)
