"""Seeded input generator: Philox known answers, deviate statistics, workload structure."""
import math
import os

import numpy as np
import pytest

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def test_philox_known_answers():
    n = 0
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        w = [int(x, 16) for x in line.split()]
        assert synth.philox(w[:4], w[4:6]) == tuple(w[6:])
        n += 1
    assert n == 3


def test_irwin_hall_moments():
    lib = synth.host_lib()
    z = np.array([lib.synth_normal(i, 7, synth.T_Q, 0, synth.UNIT) for i in range(200000)])
    assert abs(z.mean()) < 0.01
    assert abs(z.var() - 1.0) < 0.01
    assert np.abs(z).max() <= 2 * math.sqrt(3) + 1e-12
    # Irwin-Hall(4) excess kurtosis is -6/(5*4) = -0.3
    k = ((z - z.mean()) ** 4).mean() / z.var() ** 2 - 3
    assert abs(k + 0.3) < 0.03


def test_fill_deterministic_and_step_dependent():
    w = synth.small_workload(L=128, H=2, H_kv=2, d=64)
    a = synth.host_tensor(w, "q", 1)
    b = synth.host_tensor(w, "q", 1)
    c = synth.host_tensor(w, "q", 2)
    assert a.dtype == np.uint16 and a.shape == (1, 128, 2, 64)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c)
    # step noise is small: consecutive steps differ by about noise * sharpness
    qa = (a.astype(np.uint32) << 16).view(np.float32)
    qc = (c.astype(np.uint32) << 16).view(np.float32)
    sharp = synth.sharpness(w)
    for h in range(2):
        diff = (qa[:, :, h] - qc[:, :, h]).std()
        assert diff == pytest.approx(w.noise * math.sqrt(2) * sharp[h], rel=0.15)


def test_fill_value_formula_fp32():
    w = synth.small_workload(dtype="fp32", L=64, H=2, H_kv=2, d=64, planted=0,
                             sharp=("fixed", (0.5, 3.0)))
    q = synth.host_tensor(w, "q", 3)
    lib = synth.host_lib()
    for (t, h, c) in [(0, 0, 0), (5, 1, 17), (63, 1, 63)]:
        elem = (t * 2 + h) * 64 + c
        zb = lib.synth_normal(elem, synth.STEP_BASE, synth.T_Q, 0, synth.UNIT)
        zs = lib.synth_normal(elem, 3, synth.T_Q, 0, synth.UNIT)
        want = np.float32((0.5, 3.0)[h] * (zb + w.noise * zs))
        assert q[0, t, h, c] == want


def test_planted_blocks_and_redraw():
    w = synth.WORKLOADS["bf16-L8192-H32-s90"]
    p0 = synth.planted_blocks(w, 0)
    assert p0.shape == (1, 32, 128)
    assert (p0.sum(-1) == 8).all()
    assert np.array_equal(p0, synth.planted_blocks(w, 63))
    p1 = synth.planted_blocks(w, 64)
    # a quarter (2 of 8) of each head's planted blocks move at the redraw step
    assert ((p0 & p1).sum(-1) == 6).all()
    assert np.array_equal(p1, synth.planted_blocks(w, 159))
    p2 = synth.planted_blocks(w, 160)
    assert ((p1 & p2).sum(-1) == 6).all()
    assert (p2.sum(-1) == 8).all()


def test_planted_keys_shift_along_query_direction():
    w = synth.small_workload(L=512, H=4, H_kv=2, d=64, bs=64, planted=2, noise=0.0)
    k = (synth.host_tensor(w, "k", 0).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    plant = synth.planted_blocks(w, 0)
    u = synth.plant_direction(w)
    assert np.allclose(np.linalg.norm(u, axis=-1), 1.0)
    for kh in range(2):
        blocks = k[0, :, kh].reshape(8, 64, 64).mean(axis=1) @ u[0, kh]
        planted = plant[0, kh].astype(bool)
        # mean projection of planted blocks is about +2, others about 0
        assert np.all(blocks[planted] > 1.5) and np.all(np.abs(blocks[~planted]) < 0.6)


def test_sharpness_range():
    w = synth.WORKLOADS["bf16-L2048-H32-s80"]
    s = synth.sharpness(w)
    assert s.shape == (32,) and (s >= 0.3).all() and (s < 4.0).all()
    assert s.std() > 0.5
    assert list(synth.sharpness(synth.WORKLOADS["fp32-L512-H2-s50"])) == [0.5, 3.0]
