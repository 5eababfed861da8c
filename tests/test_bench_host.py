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
