"""Column-sparse attention (the PulseCol abstract) on the GPU against the oracle.

Column scores within fp32 rounding of the fp64 oracle; the kept columns exactly
the oracle's selection on the GPU's own scores (and on the oracle's scores up to
entries within 1e-5 of the threshold); gathered K/V exact copies; attention over
the GPU's columns within the block-sparse path's output tolerances.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_sdl_b200 as sdl
import oracle
import synth
from parity_util import TOL, bf16_to_f64, check_close

pytestmark = pytest.mark.gpu

CASES = [
    # dtype, B, L, H, H_kv, d, sparsity
    ("fp32", 1, 256, 2, 2, 64, 0.5),
    ("bf16", 1, 512, 4, 2, 128, 0.8),       # GQA
    ("bf16", 2, 1024, 2, 2, 64, 0.9),       # two sequences
    ("bf16", 1, 2048, 4, 4, 128, 0.75),
    ("bf16", 1, 576, 2, 2, 128, 0.7),       # a partial 128-key score tile
]


def _host_dev(w):
    return synth.host_inputs(w, 0), synth.device_inputs(w, 0)


@pytest.mark.parametrize("dtype,B,L,H,H_kv,d,s", CASES)
def test_col_scores_select_gather_attention(dtype, B, L, H, H_kv, d, s):
    w = synth.small_workload(dtype=dtype, B=B, H=H, H_kv=H_kv, L=L, d=d, bs=64, sparsity=s,
                             planted=2)
    host, dev = _host_dev(w)
    q, k, v = dev["q"], dev["k"], dev["v"]
    S = sdl.col_scores(q, k, 64)
    cols = sdl.col_select(S, q, k, 64, s)
    kc, vc = sdl.col_gather(k, v, cols, q, 64)
    O, lse = sdl.col_sparse_attn(q, kc, vc, 64, want_lse=True)
    torch.cuda.synchronize()
    assert sdl.last_device_status() == sdl.SDL_OK
    # scores: fp32 FFMA against the fp64 definition
    Sw = oracle.col_scores(host["q"], host["k"], 64)
    assert np.allclose(S.cpu().numpy(), Sw, rtol=2e-5, atol=1e-9)
    # selection: exactly the oracle's rule on the GPU's own scores
    Lc = oracle.col_budget(L, s)
    assert cols.shape == (B, H, Lc) == tuple(oracle.col_select(Sw, s).shape)
    want_cols = oracle.col_select(S.cpu().numpy().astype(np.float64), s)
    assert np.array_equal(cols.cpu().numpy(), want_cols)
    # and the oracle's own selection, but for entries at the threshold within 1e-5
    oc = oracle.col_select(Sw, s)
    for b in range(B):
        for h in range(H):
            diff = set(oc[b, h]) ^ set(want_cols[b, h])
            tau = np.sort(Sw[b, h])[-Lc]
            for u in diff:
                assert abs(Sw[b, h, u] - tau) <= 1e-5 * tau
    # gather: exact copies
    g = H // H_kv
    idx = cols.long()
    for b in range(B):
        for h in range(H):
            assert torch.equal(kc[b, :, h], k[b, idx[b, h], h // g])
            assert torch.equal(vc[b, :, h], v[b, idx[b, h], h // g])
    # attention over the GPU's columns
    Ow, lw = oracle.col_attention(host["q"], host["k"], host["v"], cols.cpu().numpy())
    got = (bf16_to_f64(O) if dtype == "bf16" else O.double().cpu().numpy()).transpose(0, 2, 1, 3)
    check_close(got, Ow, dtype)
    assert np.abs(lse.cpu().numpy() - lw).max() <= TOL[dtype]["lse"]


def test_all_columns_equal_dense_attention():
    w = synth.small_workload(B=1, H=2, H_kv=2, L=512, d=128, bs=64, sparsity=0.0, planted=1)
    _, dev = _host_dev(w)
    q, k, v = dev["q"], dev["k"], dev["v"]
    cols = torch.arange(512, dtype=torch.int32, device="cuda").repeat(1, 2, 1).contiguous()
    kc, vc = sdl.col_gather(k, v, cols, q, 64)
    O = sdl.col_sparse_attn(q, kc, vc, 64)
    Od = sdl.dense_attn(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(O, Od)


def test_col_arguments_are_checked():
    w = synth.small_workload(B=1, H=2, H_kv=2, L=256, d=64, bs=64, sparsity=0.5)
    _, dev = _host_dev(w)
    q, k = dev["q"], dev["k"]
    with pytest.raises(sdl.SdlError):
        sdl.col_budget(q, k, 64, 1.0)
    S = sdl.col_scores(q, k, 64)
    small = torch.empty((1, 2, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(sdl.SdlError):
        sdl.col_select(S, q, k, 64, 0.5, cols=small)
    kc = torch.empty((1, 96, 2, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sdl.SdlError):
        sdl.col_sparse_attn(q, kc, kc, 64)  # 96 columns: not whole 64-key tiles


def test_col_schedule_refreshes_at_anchors_only():
    """The column set changes only at refresh steps; a step in between attends with
    its anchor's columns over its own inputs."""
    from block_sparse_attention_sdl_b200.runtime import ColSparseAttention
    w = synth.small_workload(B=1, H=4, H_kv=2, L=512, d=128, bs=64, sparsity=0.8, planted=2,
                             steps=4, anchor_every=2)
    att = ColSparseAttention(w.B, w.H, w.H_kv, w.L, w.d, w.bs, w.sparsity, 2)
    seen = []
    for step in range(4):
        x = synth.device_inputs(w, step)
        O = att(x["q"], x["k"], x["v"], step)
        torch.cuda.synchronize()
        seen.append(att.cols.clone())
        assert att.mask_step == (step // 2) * 2
        if step in (1, 3):
            assert torch.equal(seen[step], seen[step - 1])
            host = synth.host_inputs(w, step)
            Ow, _ = oracle.col_attention(host["q"], host["k"], host["v"], att.cols.cpu().numpy())
            check_close(bf16_to_f64(O).transpose(0, 2, 1, 3), Ow, "bf16")
    assert sdl.last_device_status() == sdl.SDL_OK


@pytest.mark.parametrize("heads", [(0, 17), (5, 31)])
def test_col_scores_full_size_sampled_heads(heads):
    """The 8K / 32-head workload that bench.py times (--variant pulsecol): column
    scores of two heads against the oracle, and the kept columns of those heads
    exactly the oracle's rule on the GPU's scores."""
    w = synth.WORKLOADS["bf16-L8192-H32-s90"]
    host, dev = _host_dev(w)
    S = sdl.col_scores(dev["q"], dev["k"], w.bs)
    cols = sdl.col_select(S, dev["q"], dev["k"], w.bs, w.sparsity)
    torch.cuda.synchronize()
    assert sdl.last_device_status() == sdl.SDL_OK
    hs = list(heads)
    Sw = oracle.col_scores(np.ascontiguousarray(host["q"][:, :, hs]),
                           np.ascontiguousarray(host["k"][:, :, hs]), w.bs)
    got = S.cpu().numpy()[:, hs]
    assert np.allclose(got, Sw, rtol=2e-5, atol=1e-9)
    want = oracle.col_select(got.astype(np.float64), w.sparsity)
    assert np.array_equal(cols.cpu().numpy()[:, hs], want)
