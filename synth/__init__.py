"""Seeded synthetic inputs shaped like the diffusion-LLM attention workloads.

This module is shared by both sides of every parity check: the CPU oracle reads
the host build's output, the GPU library reads the device build's output, and
the two builds produce identical bits (``gen_core.h`` holds the arithmetic).
It contains none of the attention method's arithmetic.

Workloads (from the Step-dLLM abstract, "8K context, 256 denoising steps, 90%
sparsity", and the SparseD abstract, "64k context length with 1,024 denoising
steps"; the other shapes are LLaDA-8B- and Dream-7B-like attention layers):

* ``fp32-L512-H2-s50``     fp32, H=2, L=512, d=64, 64-token blocks, 50 %
* ``bf16-L2048-H32-s80``   LLaDA-8B-like layer, 80 %
* ``bf16-L8192-H32-s90``   the 8K / 256-step / 90 % setting
* ``bf16-L16384-H28kv4-s90`` Dream-7B-like GQA (28 query / 4 KV heads)
* ``bf16-L65536-H32-bs128-s95`` long context, 128-token blocks, 95 %

Construction of step ``s`` of a workload (all readings of the configs):

* Q[b,t,h,:] = sharp_h * (Zq_base + noise * Zq_s)
* K[b,t,kh,:] = Zk_base + amp * u[b,kh] (tokens of planted blocks only) + noise * Zk_s
* V[b,t,kh,:] = Zv_base + noise * Zv_s

Z are unit-variance deviates from Philox-4x32-10 (see ``gen_core.h``), so step
``s`` is regenerable without replaying earlier steps.  ``u[b,kh]`` is the unit
direction of the exact integer sum of the base query draws of the KV head's
query heads (the head group's mean query direction); ``amp`` = 2 (two key
standard deviations).  Sharpness is drawn per query head from U(lo, hi), or
fixed.  Planted blocks are drawn per KV head; at each redraw step a quarter of
them move to fresh block indices and stay there.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_HOST_SO = os.path.join(_HERE, "libsynth_host.so")
_DEV_SO = os.path.join(_HERE, "libsynth_dev.so")

T_Q, T_K, T_V, T_SHARP, T_PLANT = 1, 2, 3, 16, 17
STEP_BASE = 0xFFFFFFFF
UNIT = math.sqrt(3.0) * 2.0 ** -32
PLANT_AMP = 2.0


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str  # "fp32" | "bf16"
    B: int
    H: int
    H_kv: int
    L: int
    d: int
    bs: int
    sparsity: float
    steps: int
    anchor_every: int
    noise: float
    sharp: tuple  # ("fixed", (..)) or ("uniform", lo, hi)
    planted: int  # planted key blocks per KV head
    redraw_steps: tuple = ()
    redraw_frac: float = 0.25
    timed_steps: tuple = field(default=())  # empty: 0..steps-1

    @property
    def nb(self) -> int:
        return self.L // self.bs

    @property
    def group(self) -> int:
        return self.H // self.H_kv

    def is_anchor(self, step: int) -> bool:
        return step % self.anchor_every == 0

    def anchor_of(self, step: int) -> int:
        return (step // self.anchor_every) * self.anchor_every

    def schedule(self):
        return list(self.timed_steps) if self.timed_steps else list(range(self.steps))


WORKLOADS = {
    w.name: w
    for w in [
        Workload("fp32-L512-H2-s50", "fp32", 1, 2, 2, 512, 64, 64, 0.50, 4, 2, 0.05,
                 ("fixed", (0.5, 3.0)), 0),
        Workload("bf16-L2048-H32-s80", "bf16", 1, 32, 32, 2048, 128, 64, 0.80, 16, 4, 0.02,
                 ("uniform", 0.3, 4.0), 4),
        Workload("bf16-L8192-H32-s90", "bf16", 1, 32, 32, 8192, 128, 64, 0.90, 256, 32, 0.02,
                 ("uniform", 0.3, 4.0), 8, redraw_steps=(64, 160)),
        Workload("bf16-L16384-H28kv4-s90", "bf16", 1, 28, 4, 16384, 128, 64, 0.90, 64, 16, 0.02,
                 ("uniform", 0.3, 4.0), 8),
        Workload("bf16-L65536-H32-bs128-s95", "bf16", 1, 32, 32, 65536, 128, 128, 0.95, 1024, 128,
                 0.02, ("uniform", 0.3, 4.0), 16, timed_steps=tuple(range(0, 1024, 32))),
    ]
}
ORDER = list(WORKLOADS)


def small_workload(name: str = "tiny", dtype: str = "bf16", B=1, H=2, H_kv=2, L=256, d=64, bs=64,
                   sparsity=0.5, planted=1, noise=0.02, sharp=("uniform", 0.3, 4.0),
                   steps=4, anchor_every=2) -> Workload:
    """An ad-hoc workload for unit tests (same construction, other sizes)."""
    return Workload(name, dtype, B, H, H_kv, L, d, bs, sparsity, steps, anchor_every, noise, sharp,
                    planted)


# --------------------------------------------------------------------------- build


def _build_host(force=False):
    src = os.path.join(_HERE, "gen_host.c")
    if force or not os.path.exists(_HOST_SO) or os.path.getmtime(_HOST_SO) < max(
            os.path.getmtime(src), os.path.getmtime(os.path.join(_HERE, "gen_core.h"))):
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-o",
                               _HOST_SO, src, "-lpthread"])


def _build_dev(force=False):
    src = os.path.join(_HERE, "gen_dev.cu")
    if force or not os.path.exists(_DEV_SO) or os.path.getmtime(_DEV_SO) < max(
            os.path.getmtime(src), os.path.getmtime(os.path.join(_HERE, "gen_core.h"))):
        subprocess.check_call(["nvcc", "-O3", "-fmad=false", "-gencode",
                               "arch=compute_100a,code=sm_100a", "-Xcompiler", "-fPIC", "-shared",
                               "-o", _DEV_SO, src])


def build(force=False, device=True):
    _build_host(force)
    if device:
        _build_dev(force)


_host = None
_dev = None


def host_lib():
    global _host
    if _host is None:
        _build_host()
        lib = ctypes.CDLL(_HOST_SO)
        lib.synth_philox.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_uint32,
                                     ctypes.c_uint32, ctypes.POINTER(ctypes.c_uint32)]
        lib.synth_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
                                     ctypes.c_uint64, ctypes.c_double]
        lib.synth_normal.restype = ctypes.c_double
        lib.synth_fill.argtypes = [ctypes.c_void_p, ctypes.c_int] + [ctypes.c_int] * 5 + [
            ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_double, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_double, ctypes.c_int]
        lib.synth_qsum.argtypes = [ctypes.c_void_p] + [ctypes.c_int] * 4 + [ctypes.c_uint64,
                                                                              ctypes.c_int]
        _host = lib
    return _host


def dev_lib():
    global _dev
    if _dev is None:
        if not os.path.exists(_DEV_SO):
            raise RuntimeError(f"{_DEV_SO} is missing: run synth.build() or __graft_entry__.build()")
        lib = ctypes.CDLL(_DEV_SO)
        lib.synth_fill_dev.argtypes = [ctypes.c_void_p, ctypes.c_int] + [ctypes.c_int] * 5 + [
            ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_double, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_double, ctypes.c_void_p]
        lib.synth_fill_dev.restype = ctypes.c_int
        _dev = lib
    return _dev


def philox(ctr, key=(0, 0)):
    """Philox-4x32-10 of a 4-word counter and 2-word key (host build)."""
    c = (ctypes.c_uint32 * 4)(*[int(x) & 0xFFFFFFFF for x in ctr])
    o = (ctypes.c_uint32 * 4)()
    host_lib().synth_philox(c, int(key[0]) & 0xFFFFFFFF, int(key[1]) & 0xFFFFFFFF, o)
    return tuple(int(x) for x in o)


def _key(seed):
    return (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)


# ------------------------------------------------------------------ per-head setup


def sharpness(w: Workload, seed: int = 0) -> np.ndarray:
    kind = w.sharp[0]
    if kind == "fixed":
        vals = np.asarray(w.sharp[1], dtype=np.float64)
        assert vals.shape == (w.H,)
        return vals
    lo, hi = w.sharp[1], w.sharp[2]
    out = np.empty(w.H, dtype=np.float64)
    for h in range(w.H):
        r = philox((h, 0, 0, T_SHARP), _key(seed))
        u = (r[0] >> 8) * 2.0 ** -24
        out[h] = lo + (hi - lo) * u
    return out


def _epoch(w: Workload, step: int) -> int:
    return sum(1 for s in w.redraw_steps if step >= s)


def planted_blocks(w: Workload, step: int, seed: int = 0) -> np.ndarray:
    """uint8 [B, H_kv, nb]: 1 where a key block is planted at this step."""
    nb = w.nb
    out = np.zeros((w.B, w.H_kv, nb), dtype=np.uint8)
    if w.planted == 0:
        return out
    epoch = _epoch(w, step)
    nred = max(1, int(round(w.planted * w.redraw_frac)))
    for b in range(w.B):
        for kh in range(w.H_kv):
            cur = []
            n = 0
            while len(cur) < w.planted:
                j = philox((n, kh, b, T_PLANT), _key(seed))[0] % nb
                n += 1
                if j not in cur:
                    cur.append(j)
            for e in range(1, epoch + 1):
                n = 0
                taken = set(cur)  # new blocks avoid every block planted before this redraw
                for i in range(nred):
                    pos = ((e - 1) * nred + i) % w.planted
                    while True:
                        j = philox((n, kh, b, T_PLANT + 256 * e), _key(seed))[0] % nb
                        n += 1
                        if j not in taken:
                            break
                    taken.add(j)
                    cur[pos] = j
            out[b, kh, cur] = 1
    return out


_dir_cache = {}


def plant_direction(w: Workload, seed: int = 0, nthreads: int | None = None) -> np.ndarray:
    """fp64 [B, H_kv, d]: unit direction of the group's summed base queries."""
    key = (w.B, w.H, w.H_kv, w.L, w.d, seed)
    if key in _dir_cache:
        return _dir_cache[key]
    sums = np.zeros((w.B, w.H, w.d), dtype=np.int64)
    host_lib().synth_qsum(sums.ctypes.data, w.B, w.L, w.H, w.d, seed,
                          nthreads or os.cpu_count() or 1)
    g = w.group
    grp = sums.reshape(w.B, w.H_kv, g, w.d).astype(np.float64).sum(axis=2)
    # int64 -> float64 is exact here: |sum| < 7 * 2^49 < 2^53
    norm = np.sqrt((grp * grp).sum(axis=-1, keepdims=True))
    out = grp / norm
    _dir_cache[key] = out
    return out


def _tensor_setup(w: Workload, which: str, step: int, seed: int):
    if which == "q":
        return T_Q, w.H, sharpness(w, seed), None, None
    if which == "k":
        if w.planted:
            return T_K, w.H_kv, None, plant_direction(w, seed), planted_blocks(w, step, seed)
        return T_K, w.H_kv, None, None, None
    return T_V, w.H_kv, None, None, None


def host_tensor(w: Workload, which: str, step: int, seed: int = 0, nthreads=None) -> np.ndarray:
    """Step tensor on the host: uint16 bf16 bits or float32, shape [B, L, Hx, d]."""
    tid, hx, sharp, direc, plant = _tensor_setup(w, which, step, seed)
    dt = np.float32 if w.dtype == "fp32" else np.uint16
    out = np.empty((w.B, w.L, hx, w.d), dtype=dt)
    keep = []

    def ptr(a):
        if a is None:
            return None
        a = np.ascontiguousarray(a)
        keep.append(a)
        return a.ctypes.data

    rc = host_lib().synth_fill(out.ctypes.data, 1 if w.dtype == "fp32" else 0, w.B, w.L, hx, w.d,
                               w.bs, step, tid, seed, UNIT, w.noise, ptr(sharp), ptr(direc),
                               ptr(plant), PLANT_AMP, nthreads or os.cpu_count() or 1)
    if rc != 0:
        raise ValueError("synth_fill rejected its arguments")
    return out


def host_inputs(w: Workload, step: int, seed: int = 0):
    return {x: host_tensor(w, x, step, seed) for x in ("q", "k", "v")}


def to_torch(a: np.ndarray):
    """Host array -> torch CPU tensor of the workload dtype (bf16 bits reinterpreted)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t


def device_tensor(w: Workload, which: str, step: int, seed: int = 0, out=None, device="cuda"):
    """Step tensor generated on the GPU (same bits as :func:`host_tensor`)."""
    import torch
    tid, hx, sharp, direc, plant = _tensor_setup(w, which, step, seed)
    dt = torch.float32 if w.dtype == "fp32" else torch.bfloat16
    if out is None:
        out = torch.empty((w.B, w.L, hx, w.d), dtype=dt, device=device)
    keep = []

    def dptr(a, tdt):
        if a is None:
            return None
        t = torch.as_tensor(np.ascontiguousarray(a)).to(device=device, dtype=tdt)
        keep.append(t)
        return t.data_ptr()

    stream = torch.cuda.current_stream(out.device).cuda_stream
    rc = dev_lib().synth_fill_dev(out.data_ptr(), 1 if w.dtype == "fp32" else 0, w.B, w.L, hx, w.d,
                                  w.bs, step, tid, seed, UNIT, w.noise,
                                  dptr(sharp, torch.float64), dptr(direc, torch.float64),
                                  dptr(plant, torch.uint8), PLANT_AMP, stream)
    if rc != 0:
        raise RuntimeError(f"synth_fill_dev failed with cudaError {rc}")
    torch.cuda.current_stream(out.device).synchronize()  # keep[] outlives the kernel
    return out


def device_inputs(w: Workload, step: int, seed: int = 0, device="cuda"):
    return {x: device_tensor(w, x, step, seed, device=device) for x in ("q", "k", "v")}
