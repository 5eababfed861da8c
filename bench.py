"""Benchmark: block-sparse attention for diffusion-LLM denoising steps on B200.

Workload: one bidirectional attention layer over the 8K / 256-step / 90 %-sparse
denoising schedule of the Step-dLLM abstract (B=1, H=32, L=8192, d=128,
64-token blocks, anchor every 32 steps), synthetic seeded bf16 inputs
regenerated from the seed at every step.

A step is one denoising step of that schedule: at anchor steps the block
scores and the mask are rebuilt (sdl_block_scores + sdl_select_mask), then
block-sparse attention runs (sdl_sparse_attn).  ``--steps K`` times steps
0..K-1 (K=256 is the whole schedule); every step has its own inputs (192 MiB,
larger than L2), all resident in HBM before the timed region starts.

``value`` is the algorithmic sparse-attention throughput of the whole step
loop: 4 * block^2 * d FLOP per kept block, times the kept blocks, over the
device time of the K steps (anchor work included).  The JSON line also carries
the kernel-only rate against the bf16 tensor peak, per-step latency, the dense
baseline and the sparse/dense speedup, the end-to-end figure through host
buffers, and the oracle's CPU time.

Multi-GPU (torchrun): each rank runs its own independent sequence (weak
scaling, no collective on the data path); the time is the max over ranks.
``--impl reference`` times the fp64 CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "bf16-L8192-H32-s90"
METRIC = "sparse attn TFLOPS (% bf16 peak) + per-step latency & speedup vs dense at 8K/90%"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=256)
    p.add_argument("--step-stride", type=int, default=1,
                   help="time steps 0, S, 2S, ... of the schedule (the 64K workload is timed "
                        "at every 32nd step of its 1024, anchors included)")
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="sdl", choices=["sdl", "reference"])
    p.add_argument("--workload", default=WORKLOAD)
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--variant", choices=["step-dllm", "uniform-head", "sparsed", "pulsecol"],
                   default="step-dllm",
                   help="step-dllm: head-adaptive global budget, mask refreshed every anchor "
                        "interval (the headline); uniform-head: the same schedule with a "
                        "uniform per-head budget; sparsed: dense attention for the first "
                        "--dense-steps steps, then one mask reused for every later step; "
                        "pulsecol: column-sparse attention (key tokens kept per head, "
                        "refreshed every anchor interval, same FLOP budget)")
    p.add_argument("--shard", choices=["sequences", "heads"], default="sequences",
                   help="sequences: every rank its own independent sequence (weak scaling, no "
                        "collective); heads: the ranks split the heads of one sequence, the "
                        "mask's global budget met by the staged selection with NCCL "
                        "exchanges (strong scaling)")
    p.add_argument("--dense-steps", type=int, default=32,
                   help="dense warm-up steps of the sparsed variant")
    p.add_argument("--profile", choices=["sparse", "dense", "scores"], default=None,
                   help="launch only this attention kernel, or (scores) the separate block-"
                        "score and selection calls (warmup + steps times, one input), and "
                        "print the event-timed average; for profiler captures")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, index: int):
        self.ok = False
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            pass
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [k for k, v in self.REASONS.items() if self.reasons & v]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}

    def rejected(self):
        bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
        return bool(bad & set(self.summary()["reasons"]))


# ------------------------------------------------------------------- steps


class Runner:
    """The library's step loop over per-step device inputs, with per-launch events."""

    def __init__(self, w, seed, device, variant="step-dllm", dense_steps=0, shard=None,
                 rank=0):
        """shard: None (every head here) or (h0, h1, kv0, kv1), this rank's query- and
        KV-head ranges of a head-sharded sequence."""
        import block_sparse_attention_sdl_b200 as sdl
        from block_sparse_attention_sdl_b200 import runtime
        self.sdl, self.w, self.rt = sdl, w, runtime
        sparsed = variant == "sparsed"
        self.interval = None if sparsed else w.anchor_every
        self.dense_steps = dense_steps if sparsed else 0
        self.shard = shard
        self.H, self.H_kv = (w.H, w.H_kv) if shard is None else (shard[1] - shard[0],
                                                                 shard[3] - shard[2])
        self.pulsecol = variant == "pulsecol"
        if self.pulsecol:
            self.att = runtime.ColSparseAttention(w.B, self.H, self.H_kv, w.L, w.d, w.bs,
                                                  w.sparsity, self.interval, device=device)
        else:
            self.att = runtime.StepSparseAttention(
                w.B, self.H, self.H_kv, w.L, w.d, w.bs, w.sparsity, self.interval,
                device=device, budget="head" if variant == "uniform-head" else "sequence",
                dense_steps=self.dense_steps, heads_total=None if shard is None else w.H,
                rank=rank)
        self.out = torch.empty((w.B, w.L, self.H, w.d), dtype=torch.bfloat16, device=device)
        self.seed = seed
        self.kinds = []  # per attention launch: "sparse" or "dense"

    def make_inputs(self, steps):
        import synth
        xs = [synth.device_inputs(self.w, s, self.seed) for s in steps]
        if self.shard is not None:
            # this rank's heads only, as a head-sharded projection would hand them over
            h0, h1, kv0, kv1 = self.shard
            xs = [{"q": x["q"][:, :, h0:h1].contiguous(), "k": x["k"][:, :, kv0:kv1].contiguous(),
                   "v": x["v"][:, :, kv0:kv1].contiguous()} for x in xs]
        return xs

    def step(self, x, s, ev=None, out=None):
        att, w, rt = self.att, self.w, self.rt
        out = self.out if out is None else out
        dense = rt.is_dense(s, self.dense_steps)
        if not dense and (rt.is_anchor(s, self.interval, self.dense_steps) or
                          att.mask_step is None):
            if ev is not None:
                ev["a0"].append(torch.cuda.Event(enable_timing=True))
                ev["a0"][-1].record()
            att.refresh(x["q"], x["k"], rt.anchor_of(s, self.interval, self.dense_steps))
            if ev is not None:
                ev["a1"].append(torch.cuda.Event(enable_timing=True))
                ev["a1"][-1].record()
        if ev is not None:
            ev["s0"].append(torch.cuda.Event(enable_timing=True))
            ev["s0"][-1].record()
            self.kinds.append("dense" if dense else "sparse")
        if dense:
            self.sdl.dense_attn(x["q"], x["k"], x["v"], w.bs, out=out)
        elif self.pulsecol:
            att.attend(x["q"], x["k"], x["v"], out=out)
        else:
            self.sdl.sparse_attn(x["q"], x["k"], x["v"], att.row_ptr, att.col_idx, w.bs,
                                 out=out, plan=att.plan, order=att.order, lists=att.lists)
        if ev is not None:
            ev["s1"].append(torch.cuda.Event(enable_timing=True))
            ev["s1"][-1].record()

    def prime(self, x):
        """Run the anchor and attention kernels once, untimed (see main)."""
        self.att.refresh(x["q"], x["k"], 0)
        if self.pulsecol:
            self.att.attend(x["q"], x["k"], x["v"], out=self.out)
        else:
            self.sdl.sparse_attn(x["q"], x["k"], x["v"], self.att.row_ptr, self.att.col_idx,
                                 self.w.bs, out=self.out, plan=self.att.plan,
                                 order=self.att.order, lists=self.att.lists)
        self.att.mask_step = None


def barrier(dist_on):
    if dist_on:
        import torch.distributed as dist
        dist.barrier()


def rank_seed(seed: int, rank: int) -> int:
    """Seed of the independent sequence a rank runs (weak scaling over sequences)."""
    return seed + rank


def job_rate(flop_per_step: float, n_steps: int, world: int, ms_max: float) -> float:
    """Whole-job TFLOP/s: every rank's steps over the slowest rank's device time."""
    return flop_per_step * n_steps * world / (ms_max * 1e-3) / 1e12


def any_rank(flag: bool, dist_on, device) -> bool:
    """True on every rank if `flag` is true on any of them."""
    if not dist_on:
        return bool(flag)
    import torch.distributed as dist
    t = torch.tensor([1 if flag else 0], dtype=torch.int32, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return bool(t.item())


def max_over_ranks(x, dist_on, device):
    if not dist_on:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def time_steps(runner, inputs, steps, dist_on, device, with_events=True):
    ev = {"a0": [], "a1": [], "s0": [], "s1": []} if with_events else None
    runner.att.mask_step = None
    barrier(dist_on)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for x, s in zip(inputs, steps):
        runner.step(x, s, ev)
    e1.record()
    torch.cuda.synchronize()
    barrier(dist_on)
    ms = e0.elapsed_time(e1)
    return ms, ev


def launches_per_anchor(block: int, sharded: bool = False, fused: bool = False,
                        lists: bool = False):
    # fused: scores and selection in one launch; else pool, score; select: zero, 3
    # histogram passes, count, scan, write (+ the per-rank totals when the heads are
    # sharded); tile plan and its order (64-token blocks), and the tiles' lists
    plan = (2 + (1 if lists else 0)) if block == 64 else 0
    if fused:
        return 1 + plan
    return 2 + 7 + (1 if sharded else 0) + plan


def e2e_measure(runner, inputs, steps, device):
    """Same step loop with the inputs copied from pinned host memory and the
    output copied back, every step, inside the timed region.  Uploads, the step
    and downloads run on three streams over double-buffered device tensors (the
    upload of step i+1 and the download of step i-1 overlap step i), ordered by
    events, as a serving loop would run them."""
    ring = min(len(inputs), 8)
    host_in = []
    for x in inputs[:ring]:
        host_in.append({k: v.cpu().pin_memory() for k, v in x.items()})
    host_out = [torch.empty_like(runner.out, device="cpu").pin_memory() for _ in range(2)]
    dev_in = [{k: torch.empty_like(v) for k, v in inputs[0].items()} for _ in range(2)]
    dev_out = [torch.empty_like(runner.out) for _ in range(2)]
    bytes_in = sum(v.numel() * v.element_size() for v in dev_in[0].values())
    bytes_out = runner.out.numel() * runner.out.element_size()
    s_c = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def loop(n):
        runner.att.mask_step = None
        s_in.wait_stream(s_c)  # uploads start after whatever the compute stream has queued
        in_done = [torch.cuda.Event() for _ in range(2)]
        c_done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]
        for i in range(n):
            b, h = i % 2, host_in[i % ring]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(c_done[b])  # step i-2 has read this input buffer
                for k in dev_in[b]:
                    dev_in[b][k].copy_(h[k], non_blocking=True)
                in_done[b].record(s_in)
            s_c.wait_event(in_done[b])
            if i >= 2:
                s_c.wait_event(out_done[b])  # step i-2's output has been read back
            runner.step(dev_in[b], steps[i], out=dev_out[b])
            c_done[b].record(s_c)
            with torch.cuda.stream(s_out):
                s_out.wait_event(c_done[b])
                host_out[b].copy_(dev_out[b], non_blocking=True)
                out_done[b].record(s_out)
        for e in out_done:
            s_c.wait_event(e)

    loop(min(3, len(steps)))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    loop(len(steps))
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1), bytes_in, bytes_out


def traffic_record():
    """Per-launch DRAM bytes of the sparse kernel from the committed ncu summary,
    if it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "sparse_attn_traffic.json")
    src = os.path.join(ROOT, "block_sparse_attention_sdl_b200", "csrc", "attn_tc.cu")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    with open(src, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()
    if rec.get("attn_tc_sha256") != digest:
        return None
    return rec.get("bytes_per_launch")


# ------------------------------------------------------------- cpu oracle


def csr_mask(row_ptr: np.ndarray, col_idx: np.ndarray, B: int, H: int, nb: int) -> np.ndarray:
    """uint8 [B, H, nb, nb] block mask of a CSR list."""
    rows = np.repeat(np.arange(B * H * nb), np.diff(row_ptr))
    mask = np.zeros((B * H * nb, nb), dtype=np.uint8)
    mask[rows, col_idx[:row_ptr[-1]]] = 1
    return mask.reshape(B, H, nb, nb)


def parity_check(runner, w, seed, step, out, n_random=2, rows_per_block=4, mask=None):
    """Outside the timed region: the output of timed step `step` (`out`, on the
    device) on sampled query rows against the fp64 oracle with the GPU's own mask
    (all heads; per head the first and last query block, the block with the
    longest kept list and `n_random` others), and the GPU's mask of that step's
    anchor against the oracle's selection (differences allowed only within 1e-5
    relative of the oracle's threshold, and counted).  Attention under the
    oracle's own mask on the same rows is reported beside it, not checked.
    `mask`: (row_ptr, col_idx) as they were at that step, when the layer's own
    buffers have been refreshed since."""
    import oracle
    import synth
    rt = runner.rt
    if runner.pulsecol or runner.shard is not None:
        return None
    nb, H = w.nb, w.H
    host = synth.host_inputs(w, step, seed)
    a_step = rt.anchor_of(step, runner.interval, runner.dense_steps)
    rng = np.random.default_rng(seed + 1)
    res = {"step": step, "anchor_step": a_step}
    if a_step is None:  # a dense step of the sparsed schedule
        gpu_mask = None
        lens = np.full((w.B, H, nb), nb)
    else:
        rp_t, ci_t = mask if mask is not None else (runner.att.row_ptr, runner.att.col_idx)
        rp = rp_t.cpu().numpy()
        ci = ci_t.cpu().numpy()
        gpu_mask = csr_mask(rp, ci, w.B, H, nb)
        lens = np.diff(rp).reshape(w.B, H, nb)
        ha = host if a_step == step else synth.host_inputs(w, a_step, seed)
        P = oracle.block_scores(ha["q"], ha["k"], w.bs)
        want, tau, kept = oracle.select(P, w.sparsity, per_head=runner.att.per_head)
        diff = np.argwhere(gpu_mask != want)
        taus = tau.reshape(w.B, -1)
        near = 0
        for b, h, i, j in diff:
            t_b = taus[b, h if runner.att.per_head else 0]
            if i != j and abs(P[b, h, i, j] - t_b) <= 1e-5 * t_b:
                near += 1
        res.update({"mask_blocks": int(gpu_mask.sum()), "oracle_blocks": kept,
                    "mask_entries_near_threshold": near,
                    "mask_entries_other": int(len(diff) - near)})
    rows = []
    for b in range(w.B):
        for h in range(H):
            blocks = {0, nb - 1, int(np.argmax(lens[b, h]))}
            blocks |= set(int(x) for x in rng.integers(nb, size=n_random))
            for i in sorted(blocks):
                ts = {i * w.bs, i * w.bs + w.bs - 1}
                ts |= set(int(i * w.bs + x) for x in rng.integers(w.bs, size=rows_per_block))
                rows.extend((b, h, t) for t in sorted(ts))
    rows = np.array(rows, dtype=np.int64)
    idx = torch.as_tensor(rows, device=out.device)
    got = out[idx[:, 0], idx[:, 2], idx[:, 1]].float().cpu().numpy().astype(np.float64)
    want_o, _ = oracle.attention(host["q"], host["k"], host["v"], w.bs, mask=gpu_mask, rows=rows)
    err = np.abs(got - want_o)
    tol_max, tol_mean = (1e-2, 1e-3) if w.dtype == "bf16" else (1e-4, 1e-4)
    res.update({"rows": int(len(rows)), "max_abs": float(err.max()),
                "mean_abs": float(err.mean()), "tol_max_abs": tol_max,
                "tol_mean_abs": tol_mean, "finite": bool(np.isfinite(got).all())})
    res["ok"] = bool(res["finite"] and res["max_abs"] <= tol_max and res["mean_abs"] <= tol_mean
                     and res.get("mask_entries_other", 0) == 0)
    if gpu_mask is not None:
        own, _ = oracle.attention(host["q"], host["k"], host["v"], w.bs, mask=want, rows=rows)
        res["oracle_mask_max_abs"] = float(np.abs(got - own).max())
    return res



def cpu_oracle_sample(w, seed, target_s=20.0):
    """Times the fp64 oracle's block-sparse attention on a bounded sample of the
    workload's query rows (all heads, evenly spaced query blocks) of step 0 with
    its anchor mask; returns (TFLOP/s, cores, description, sample seconds, extra)
    with extra = the oracle's anchor work (block scores + selection) in seconds and
    the sample's time scaled linearly to every query block (an extrapolation)."""
    import oracle
    import synth
    host = synth.host_inputs(w, 0, seed)
    ta = time.perf_counter()
    P = oracle.block_scores(host["q"], host["k"], w.bs)
    mask, _, _ = oracle.select(P, w.sparsity)
    anchor_s = time.perf_counter() - ta
    cores = os.cpu_count() or 1
    nb = w.nb

    def rows_for(nblk):
        blocks = np.linspace(0, nb - 1, nblk).round().astype(int)
        r = [(0, h, i * w.bs + t) for h in range(w.H) for i in blocks for t in range(w.bs)]
        return np.array(r, dtype=np.int64)

    def flops(rows):
        kept = mask[rows[:, 0], rows[:, 1], rows[:, 2] // w.bs].sum(-1) * w.bs
        return float((kept * 4 * w.d).sum())

    rows = rows_for(1)
    t0 = time.perf_counter()
    oracle.attention(host["q"], host["k"], host["v"], w.bs, mask=mask, rows=rows, nthreads=cores)
    dt = time.perf_counter() - t0
    nblk = int(min(nb, max(1, target_s / max(dt, 1e-3))))
    rows = rows_for(nblk)
    t0 = time.perf_counter()
    oracle.attention(host["q"], host["k"], host["v"], w.bs, mask=mask, rows=rows, nthreads=cores)
    dt = time.perf_counter() - t0
    what = "one full step" if nblk == nb else f"{nblk} of {nb} query blocks x {w.H} heads"
    desc = (f"block-sparse attention of {len(rows)} query rows ({what}, step 0 with its "
            f"anchor mask), fp64, {cores} threads")
    extra = {"anchor_s": anchor_s}
    if nblk == nb:
        extra["full_step_s"] = dt
    else:
        extra["full_step_s_extrapolated"] = dt * nb / nblk
    return flops(rows) / dt / 1e12, cores, desc, dt, extra


def run_config(args, w, world: int) -> dict:
    """The bench line's `config` for a workload, variant and launch (both arms)."""
    heads = args.shard == "heads"
    sparsed = args.variant == "sparsed"
    cfg = {"workload": args.workload, "global_batch": w.B * (1 if heads else world),
           "seq_len": w.L, "heads": w.H, "kv_heads": w.H_kv, "head_dim": w.d, "block": w.bs,
           "sparsity": w.sparsity, "anchor_every": None if sparsed else w.anchor_every,
           "dense_steps": args.dense_steps if sparsed else 0,
           "budget": ("key columns per head" if args.variant == "pulsecol" else
                      "per head" if args.variant == "uniform-head" else
                      "per sequence, across heads"),
           "parallelism": (f"heads split over {world} ranks" if heads else
                           f"independent sequences x{world}"),
           "l2": l2_note(w)}
    stride = getattr(args, "step_stride", 1)
    if stride > 1:
        cfg["timed_steps"] = f"0, {stride}, ..., {stride * (args.steps - 1)}"
    return cfg


def l2_note(w) -> str:
    """How the timed steps avoid reading their inputs from L2 (126 MB on B200)."""
    mib = w.B * w.L * (w.H + 2 * w.H_kv) * w.d * 2 / 2 ** 20
    if mib * 2 ** 20 > 126e6:
        return f"inputs larger than L2 ({mib:.0f} MiB per step, distinct per step)"
    return f"inputs distinct per step ({mib:.0f} MiB each, generated before timing), none read twice"


def run_reference(args):
    """The reference arm: the fp64 CPU oracle, timed per step on a bounded sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import synth
    w = synth.WORKLOADS[args.workload]
    per_step_target = max(0.5, 60.0 / max(1, args.steps + args.warmup))
    vals, tot = [], 0.0
    for i in range(args.warmup + args.steps):
        v, cores, desc, dt, extra = cpu_oracle_sample(w, args.seed, target_s=per_step_target)
        if i >= args.warmup:
            vals.append(v)
            tot += dt
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded Philox, see synth/)",
        "config": run_config(args, w, int(os.environ.get("WORLD_SIZE", "1"))),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": desc, **extra},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def profile_kernel(runner, args):
    """Only the chosen attention kernel, back to back on one input (mask from one
    anchor refresh): the launch list is warmup + steps launches of that kernel."""
    w, sdl = runner.w, runner.sdl
    x = runner.make_inputs([0])[0]
    runner.att.refresh(x["q"], x["k"], 0)
    torch.cuda.synchronize()
    if args.profile == "scores":
        # the anchor's parts as separate calls: block scores (pool + score kernels),
        # then the selection kernels on those scores
        att = runner.att
        fn = lambda: (sdl.block_scores(x["q"], x["k"], w.bs, scores=att.scores,
                                       workspace=att.ws_scores), att.select())
        flop = 0.0
    elif args.profile == "sparse":
        fn = lambda: sdl.sparse_attn(x["q"], x["k"], x["v"], runner.att.row_ptr,
                                     runner.att.col_idx, w.bs, out=runner.out,
                                     plan=runner.att.plan, order=runner.att.order,
                                     lists=runner.att.lists)
        flop = 4.0 * w.bs * w.bs * w.d * runner.att.budget
    else:
        fn = lambda: sdl.dense_attn(x["q"], x["k"], x["v"], out=runner.out)
        flop = 4.0 * w.B * w.H * w.L * w.L * w.d
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / max(args.steps, 1)
    print(json.dumps({"profile": args.profile, "workload": args.workload, "ms": ms,
                      "tflops": flop / (ms * 1e-3) / 1e12,
                      "status": sdl.last_device_status()}))


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    import synth
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if dist_on:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    w = synth.WORKLOADS[args.workload]
    heads = args.shard == "heads"
    if heads:
        # one sequence, its heads split over the ranks (whole KV-head groups)
        from block_sparse_attention_sdl_b200.sharded import head_range
        h0, h1 = head_range(w.H, w.H_kv, rank, world)
        g = w.H // w.H_kv
        shard, seed = (h0, h1, h0 // g, h1 // g), args.seed
    else:
        shard, seed = None, rank_seed(args.seed, rank)  # each rank: its own sequence
    runner = Runner(w, seed, device, args.variant, args.dense_steps, shard, rank)
    if args.profile:
        profile_kernel(runner, args)
        return
    if args.step_stride < 1:
        raise SystemExit("--step-stride must be at least 1")
    steps = list(range(0, args.steps * args.step_stride, args.step_stride))
    inputs = runner.make_inputs(steps)
    warm = [inputs[i % len(inputs)] for i in range(args.warmup)]
    for x, s in zip(warm, range(args.warmup)):
        runner.step(x, s)
    # A schedule that starts with dense steps launches no anchor or sparse kernel
    # while warming up: run each once, untimed, so that none is loaded inside the
    # timed region.  The timed schedule then builds its own masks.
    runner.prime(inputs[0])
    torch.cuda.synchronize()
    sdl = runner.sdl
    status_warm = sdl.last_device_status()  # warm-up and priming (clears the word)
    detail_warm = sdl.last_device_detail()

    sampler = ClockSampler(local)
    for attempt in range(2):
        with sampler:
            ms, ev = time_steps(runner, inputs, steps, dist_on, device)
        # every rank takes the same decision (a retry runs the timed loop's barriers)
        if not any_rank(sampler.rejected(), dist_on, device):
            break
        sampler = ClockSampler(local)
    ms_max = max_over_ranks(ms, dist_on, device)
    # outside the timed region: the device status word, and the last timed
    # step's output kept for the parity check (later launches reuse the buffer)
    status_timed = sdl.last_device_status()
    detail_timed = sdl.last_device_detail()
    last_out = runner.out.clone()
    # the mask the last timed step used (the separate timings below refresh it)
    last_mask = (None if runner.pulsecol else
                 (runner.att.row_ptr.clone(), runner.att.col_idx.clone()))

    pk, pk_kind = peaks()
    budget = runner.att.budget  # kept blocks of the whole sequence
    flop_step = 4.0 * w.bs * w.bs * w.d * budget
    dense_flop = 4.0 * w.B * w.H * w.L * w.L * w.d
    kinds = runner.kinds[-len(steps):]
    n_dense_steps = kinds.count("dense")
    # sequences counted per rank (weak scaling) or once, split over the ranks (heads)
    seqs = 1 if heads else world
    # algorithmic work of the timed steps: kept blocks on sparse steps, L^2 on dense ones
    value = job_rate((flop_step * (len(steps) - n_dense_steps) + dense_flop * n_dense_steps) /
                     len(steps), len(steps), seqs, ms_max)
    # this rank's launches: its own kept blocks and heads
    local_blocks = int(runner.att.row_ptr[-1].item()) if heads else budget
    flop_local = 4.0 * w.bs * w.bs * w.d * local_blocks
    attn_ms = [a.elapsed_time(b) for a, b in zip(ev["s0"], ev["s1"])]
    sparse_ms = [t for t, k in zip(attn_ms, kinds) if k == "sparse"]
    anchor_ms = [a.elapsed_time(b) for a, b in zip(ev["a0"], ev["a1"])]
    sp_avg = statistics.mean(sparse_ms)
    sp_q = statistics.quantiles(sparse_ms, n=10) if len(sparse_ms) > 1 else [sp_avg] * 9
    kernel_tflops = flop_local / (sp_avg * 1e-3) / 1e12
    peak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])

    # anchor-step kernels, timed apart: scoring bandwidth and selection latency
    x0 = inputs[0]

    def ev_time(fn, n=10):
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    att = runner.att
    if runner.pulsecol:
        sc_ms = ev_time(lambda: sdl.col_scores(x0["q"], x0["k"], w.bs, out=att.col_scores,
                                               workspace=att.ws))
    else:
        sc_ms = ev_time(lambda: sdl.block_scores(x0["q"], x0["k"], w.bs, scores=att.scores,
                                                 workspace=att.ws_scores))
    se_ms = ev_time(att.select)
    # the whole anchor step, launches queued back to back (the GPU's own time for
    # it, with no idle queue in front)
    an_ms = None if runner.pulsecol else ev_time(lambda: att.refresh(x0["q"], x0["k"], 0))
    score_bytes = (2 * w.B * w.L * (runner.H + runner.H_kv) * w.d +
                   4 * w.B * runner.H * w.nb * w.nb)
    # dense baseline on distinct inputs per launch (larger than L2 in total)
    de = []
    for i in range(min(11, len(inputs))):
        x = inputs[i]
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        sdl.dense_attn(x["q"], x["k"], x["v"], out=runner.out)
        b.record()
        de.append((a, b))
    torch.cuda.synchronize()
    dense_ms = statistics.median([a.elapsed_time(b) for a, b in de[1:]] or
                                 [de[0][0].elapsed_time(de[0][1])])
    dense_flop = 4.0 * w.B * runner.H * w.L * w.L * w.d  # this rank's heads

    e2e = None
    if not args.no_e2e:
        e_ms, bi, bo = e2e_measure(runner, inputs, steps, device)
        e_ms = max_over_ranks(e_ms, dist_on, device)
        e2e = {"value": job_rate(flop_step, len(steps), seqs, e_ms), "unit": "TFLOP/s",
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": e_ms / len(steps)}
    status_after = sdl.last_device_status()  # the e2e loop and the separate timings
    detail_after = sdl.last_device_detail()

    parity = None
    if rank == 0 and not heads:
        parity = parity_check(runner, w, seed, steps[-1], last_out, mask=last_mask)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, desc, _, extra = cpu_oracle_sample(w, seed)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc,
               **extra}

    n_anchor = len(anchor_ms)
    # the ncu record covers the block-sparse kernel's launch only
    traffic = None if runner.pulsecol else traffic_record()
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": len(steps), "warmup": args.warmup, "ms_per_step": ms_max / len(steps),
        "higher_is_better": True, "scaling": "strong" if heads else "weak", "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded Philox inputs shaped like the 8K/90% workload, regenerated "
                "per step)",
        "config": run_config(args, w, world),
        "variant": args.variant,
        "sparse_attn_ms": sp_avg, "sparse_attn_tflops": kernel_tflops,
        "sparse_attn_ms_p10_p50_p90": [sp_q[0], statistics.median(sparse_ms), sp_q[-1]],
        "dense_steps_timed": n_dense_steps,
        "pct_bf16_peak": kernel_tflops / peak,
        # against the measured sustained figure (a GEMM back to back under the power
        # cap): the fair denominator when long tensor-bound launches settle at the cap
        "pct_bf16_peak_sustained": kernel_tflops / pk.get(
            "bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]),
        "dense_attn_ms": dense_ms, "dense_attn_tflops": dense_flop / (dense_ms * 1e-3) / 1e12,
        "speedup_vs_dense": dense_ms / sp_avg,
        "speedup_vs_dense_amortized": dense_ms / (ms_max / len(steps)),
        "anchor_ms": statistics.mean(anchor_ms) if anchor_ms else None,
        # the first anchor is issued into an idle queue right after the timing
        # barrier; the later ones behind the previous steps' attention launches
        "anchor_ms_first": anchor_ms[0] if anchor_ms else None,
        "anchor_ms_steady": statistics.mean(anchor_ms[1:]) if len(anchor_ms) > 1 else None,
        "anchor_ms_back_to_back": an_ms,
        "block_scores_ms": sc_ms,
        "block_scores_gbs": None if runner.pulsecol else score_bytes / (sc_ms * 1e-3) / 1e9,
        "select_mask_ms": se_ms, "mask_blocks": budget,
        "columns_per_head": getattr(runner.att, "Lc", None),
        "tokens_steps_per_s": w.B * world * w.L * len(steps) / (ms_max * 1e-3),
        "roofline": {"bound": "tensor", "achieved": kernel_tflops, "peak": peak,
                     "unit": "TFLOP/s", "frac": kernel_tflops / peak,
                     "peak_source": f"bf16_tflops burst, {pk_kind}",
                     "traffic": traffic},
        "cpu_baseline": cpu,
        "e2e": e2e,
        # pulsecol: gather + attention per step; pool, the score statistics, their
        # combination, the score sums and the selection per refresh
        "gpu_launches": (2 * len(steps) + 5 * n_anchor if runner.pulsecol else
                         len(steps) + n_anchor * launches_per_anchor(
                             w.bs, runner.att.sharded, runner.att.fused,
                             runner.att.lists is not None)),
        "clocks": sampler.summary(),
        "device_status": {"warmup": status_warm, "timed": status_timed, "after": status_after,
                          "bad_mask_detail": [detail_warm, detail_timed, detail_after]},
        "parity": parity,
    }
    if rank == 0:
        print(json.dumps(line))
    if dist_on:
        import torch.distributed as dist
        dist.destroy_process_group()
    # a kernel that reported a timeout or a rejected list entry, or an output
    # off the oracle, voids the line's numbers
    if any(st != sdl.SDL_OK for st in (status_warm, status_timed, status_after)):
        sys.exit(3)
    if parity is not None and not parity["ok"]:
        sys.exit(4)


if __name__ == "__main__":
    main()
