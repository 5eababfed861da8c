"""Multi-rank host logic of bench.py on CPU: two gloo ranks over 127.0.0.1.

bench.py under torchrun gives each rank its own independent sequence (seed +
rank), synchronises with barriers around the timed region and reports the
slowest rank's time; the whole-job rate counts every rank's steps.  These
tests run that logic with the gloo backend (no GPU), world size 2.
"""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import bench
    import synth
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cpu = torch.device("cpu")
        bench.barrier(True)
        # the slowest rank's time is the job's time
        ms = bench.max_over_ranks(10.0 + 3.0 * rank, True, cpu)
        # each rank its own sequence: inputs from its own seed, reproducible
        w = synth.small_workload(L=256, H=2, H_kv=2, d=64)
        seed = bench.rank_seed(7, rank)
        q = synth.host_tensor(w, "q", 0, seed)
        q2 = synth.host_tensor(w, "q", 0, seed)
        digest = torch.tensor([float(np.asarray(q, dtype=np.float64).sum())], dtype=torch.float64)
        all_d = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(all_d, digest)
        rate = bench.job_rate(2.0e9, 4, world, ms)
        # a clock rejection on one rank makes every rank retry the timed loop
        retry = bench.any_rank(rank == 1, True, cpu)
        keep = bench.any_rank(False, True, cpu)
        bench.barrier(True)
        np.save(os.path.join(out_dir, f"rank{rank}.npy"),
                np.array([ms, rate, float(np.array_equal(np.asarray(q), np.asarray(q2)))] +
                         [float(d.item()) for d in all_d] + [float(retry), float(keep)]))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_timing_and_seeds(tmp_path):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    r0 = np.load(tmp_path / "rank0.npy")
    r1 = np.load(tmp_path / "rank1.npy")
    assert r0[0] == r1[0] == 13.0                      # max over ranks, on every rank
    assert r0[1] == r1[1] == pytest.approx(2.0e9 * 4 * 2 / 13.0e-3 / 1e12)
    assert r0[2] == r1[2] == 1.0                       # a rank's inputs are reproducible
    assert r0[3] == r1[3] and r0[4] == r1[4]           # every rank saw the same digests
    assert r0[3] != r0[4]                              # and the two sequences differ
    assert r0[5] == r1[5] == 1.0 and r0[6] == r1[6] == 0.0  # one decision on every rank


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun only rank 0 times the oracle; other ranks exit 0 silently."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def _scores_np(B, H, nb, seed, ties):
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((B, H, nb, nb)) * rng.uniform(0.3, 4.0, size=(1, H, 1, 1))
    if ties:
        z = np.round(z)  # many equal logits, hence equal scores, within a row
    e = np.exp(z - z.max(-1, keepdims=True))
    return (e / e.sum(-1, keepdims=True)).astype(np.float32)


SHARD_CASES = [(2, 8, 16, 0.8, False, 11), (1, 8, 12, 0.6, True, 12),
               (2, 4, 8, 1.0 - 1.0 / 8, False, 13)]  # the last: diagonal only


def _shard_rank_main(rank, world, port, out_dir):
    import datetime

    from block_sparse_attention_sdl_b200.sharded import head_range, select_mask_sharded
    from shard_stages_np import NumpyStages
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        for n, (B, H, nb, s, ties, seed) in enumerate(SHARD_CASES):
            P = _scores_np(B, H, nb, seed, ties)
            h0, h1 = head_range(H, H, rank, world)
            st = NumpyStages(P[:, h0:h1], s, H)
            rp, ci, mask = select_mask_sharded(None, s, 64, nb * 64, H, rank, stages=st)
            parts = [torch.zeros_like(mask) for _ in range(world)]
            dist.all_gather(parts, mask)
            np.save(os.path.join(out_dir, f"shard{n}_rank{rank}.npy"),
                    torch.cat(parts, dim=1).numpy())
            np.save(os.path.join(out_dir, f"shard{n}_csr{rank}.npy"),
                    np.concatenate([rp.numpy(), ci.numpy()]))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_head_sharded_selection(tmp_path):
    """Heads split over two ranks: the histogram sums and tie offsets exchanged with
    gloo reproduce the oracle's global selection exactly, on every rank."""
    import oracle
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_shard_rank_main, args=(r, 2, port, str(tmp_path)))
             for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for n, (B, H, nb, s, ties, seed) in enumerate(SHARD_CASES):
        want, _, kept = oracle.select(_scores_np(B, H, nb, seed, ties).astype(np.float64), s)
        for r in range(2):
            got = np.load(tmp_path / f"shard{n}_rank{r}.npy")
            assert np.array_equal(got, want), (n, r)
        total = sum(int(np.load(tmp_path / f"shard{n}_csr{r}.npy")[B * (H // 2) * nb])
                    for r in range(2))
        assert total == kept
