"""Host logic of bench.py (no GPU): the launch counts it claims, the whole-job rate,
the per-rank seeds, and the rule that the DRAM traffic it reports comes from the
committed ncu record only while the kernel source it was taken on is unchanged."""
import hashlib
import json
import os

import bench


def test_launches_per_anchor():
    # fused anchor + plan + order + lists (64-token blocks)
    assert bench.launches_per_anchor(64, fused=True, lists=True) == 4
    assert bench.launches_per_anchor(64, fused=True) == 3
    # 128-token blocks: no plan, order or lists
    assert bench.launches_per_anchor(128, fused=True, lists=True) == 1
    # separate calls: pool, score; zero, 3 histograms, count, scan, write; (+ totals)
    assert bench.launches_per_anchor(128) == 9
    assert bench.launches_per_anchor(128, sharded=True) == 10
    assert bench.launches_per_anchor(64, lists=True) == 12


def test_job_rate_and_seeds():
    # 1e12 FLOP per step, 10 steps, 2 ranks, 1 s -> 20 TFLOP/s
    assert bench.job_rate(1e12, 10, 2, 1000.0) == 20.0
    assert [bench.rank_seed(7, r) for r in range(3)] == [7, 8, 9]


def test_traffic_record_follows_the_kernel_source(tmp_path, monkeypatch):
    src_dir = tmp_path / "block_sparse_attention_sdl_b200" / "csrc"
    src_dir.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = src_dir / "attn_tc.cu"
    src.write_bytes(b"// kernel v1\n")
    rec = {"attn_tc_sha256": hashlib.sha256(b"// kernel v1\n").hexdigest(),
           "bytes_per_launch": 123456}
    (tmp_path / "profiles" / "sparse_attn_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record() == 123456
    src.write_bytes(b"// kernel v2\n")  # changed since the capture: no figure
    assert bench.traffic_record() is None
    os.remove(tmp_path / "profiles" / "sparse_attn_traffic.json")
    assert bench.traffic_record() is None


def test_csr_mask_matches_a_dense_mask():
    import numpy as np
    rng = np.random.default_rng(3)
    B, H, nb = 2, 3, 5
    want = (rng.random((B, H, nb, nb)) < 0.4).astype(np.uint8)
    rows = want.reshape(-1, nb)
    row_ptr = np.concatenate([[0], np.cumsum(rows.sum(1))]).astype(np.int32)
    col_idx = np.concatenate([np.flatnonzero(r) for r in rows]).astype(np.int32)
    assert np.array_equal(bench.csr_mask(row_ptr, col_idx, B, H, nb), want)


class _FakeAtt:
    def __init__(self, row_ptr, col_idx):
        import torch
        self.row_ptr, self.col_idx = torch.as_tensor(row_ptr), torch.as_tensor(col_idx)
        self.per_head = False


class _FakeRunner:
    """What parity_check reads from the bench's runner, on the CPU."""

    def __init__(self, att, interval):
        from block_sparse_attention_sdl_b200 import runtime
        self.rt, self.att, self.interval, self.dense_steps = runtime, att, interval, 0
        self.pulsecol, self.shard = False, None


def test_parity_check_passes_the_oracle_output_and_catches_a_wrong_one():
    """The bench's self-check: an output equal to the oracle's (rounded to bf16) with
    the oracle's own mask passes; the same output with one row perturbed fails."""
    import numpy as np
    import torch
    import oracle
    import synth
    w = synth.small_workload(L=512, H=2, H_kv=1, d=64, sparsity=0.5, planted=1, steps=3,
                             anchor_every=2)
    step = 2  # an anchor step: its own mask
    host = synth.host_inputs(w, step)
    P = oracle.block_scores(host["q"], host["k"], w.bs)
    mask, _, kept = oracle.select(P, w.sparsity)
    rows = mask.reshape(-1, w.nb)
    row_ptr = np.concatenate([[0], np.cumsum(rows.sum(1))]).astype(np.int32)
    col_idx = np.concatenate([np.flatnonzero(r) for r in rows]).astype(np.int32)
    O, _ = oracle.attention(host["q"], host["k"], host["v"], w.bs, mask=mask)
    out = torch.as_tensor(O.transpose(0, 2, 1, 3).copy()).to(torch.bfloat16)  # [B, L, H, d]
    runner = _FakeRunner(_FakeAtt(row_ptr, col_idx), w.anchor_every)
    res = bench.parity_check(runner, w, 0, step, out)
    assert res["ok"], res
    assert res["mask_entries_other"] == 0 and res["mask_blocks"] == kept
    assert res["max_abs"] < 1e-2 and res["oracle_mask_max_abs"] == res["max_abs"]
    bad = out.clone()
    bad[0, w.L - 1, 1] += 0.05   # the last row of the last query block is always sampled
    assert not bench.parity_check(runner, w, 0, step, bad)["ok"]


def test_parity_check_reads_the_mask_snapshot_of_the_checked_step():
    """The bench refreshes the layer's mask after the timed loop (separate timings on
    step 0's inputs); the check must judge the mask the checked step used, passed as
    a snapshot, and a stale mask in the layer's buffers must not be read instead."""
    import numpy as np
    import torch
    import oracle
    import synth
    w = synth.small_workload(L=512, H=2, H_kv=1, d=64, sparsity=0.5, planted=1, steps=4,
                             anchor_every=2)
    step = 2

    def csr_of(s):
        h = synth.host_inputs(w, s)
        m, _, _ = oracle.select(oracle.block_scores(h["q"], h["k"], w.bs), w.sparsity)
        r = m.reshape(-1, w.nb)
        rp = np.concatenate([[0], np.cumsum(r.sum(1))]).astype(np.int32)
        ci = np.concatenate([np.flatnonzero(x) for x in r]).astype(np.int32)
        return m, torch.as_tensor(rp), torch.as_tensor(ci)

    mask2, rp2, ci2 = csr_of(step)
    mask0, rp0, ci0 = csr_of(0)
    assert not np.array_equal(mask0, mask2)
    host = synth.host_inputs(w, step)
    O, _ = oracle.attention(host["q"], host["k"], host["v"], w.bs, mask=mask2)
    out = torch.as_tensor(O.transpose(0, 2, 1, 3).copy()).to(torch.bfloat16)
    runner = _FakeRunner(_FakeAtt(rp0, ci0), w.anchor_every)  # refreshed since: step 0's
    assert not bench.parity_check(runner, w, 0, step, out)["ok"]
    res = bench.parity_check(runner, w, 0, step, out, mask=(rp2, ci2))
    assert res["ok"] and res["mask_entries_other"] == 0, res
