#!/usr/bin/env python
"""Benchmark of the fused attention-distillation KL divergence (forward + backward).

One step = the whole hot path on one batch: forward (per-row KL and both
log-sum-exps), the mean loss, and the backward for every requested gradient
(student dQ_s, dK_s and, for the headline workload, teacher dQ_t, dK_t).

Default workload: B=1, H=32, N_Q=N_K=8192, d_t=d_s=128, causal, teacher and
student Q/K drawn independently from N(0,1) in bf16, gradients of the mean
loss for both teacher and student.  Throughput counts 2*N_Q*N_K*(d_t+d_s)
forward FLOPs and 2*N_Q*N_K*(d_t+d_s) + 4*N_Q*N_K*(d_s + d_t) backward FLOPs
per head, halved for causal masks (2.199 TFLOP per step here).

  python bench.py [--gpus N --steps K --warmup W] [--workload NAME]
  python bench.py --impl reference ...    # the fp64 CPU oracle on the same workload
  python bench.py --impl materialised ... # torch eager on the GPU, both N_Q x N_K
                                          # distributions materialised (the
                                          # baseline the fused method replaces)

With N > 1 (torchrun, one process per GPU) every rank solves its own
independent problem of the default size (heads are independent: no data-path
collective); the value is the total FLOPs of all ranks over the slowest rank's
device time.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attn-KL fwd+bwd TFLOP/s and % of B200 bf16 tensor peak (N=8192, d=128, causal)"
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 2**20


# ----------------------------------------------------------------------------- flop accounting

def visible_pairs(w) -> float:
    """Number of (query, key) pairs per head, the causal mask counted as a half."""
    return w.N_Q * w.N_K / (2.0 if w.causal else 1.0)


def step_flops(w) -> float:
    per = 2 * (w.d_t + w.d_s) + 2 * (w.d_t + w.d_s) + 4 * w.d_s + (4 * w.d_t if w.teacher_grads else 0)
    return per * visible_pairs(w) * w.B * w.H


def fwd_flops(w) -> float:
    """The forward's share of step_flops: 2 (d_t + d_s) per visible pair."""
    return 2 * (w.d_t + w.d_s) * visible_pairs(w) * w.B * w.H


def key_owner_kernel(w) -> str:
    """The key-owner kernel the library launches for a workload: the persistent
    form where the CTA's K rows fit in tensor memory beside the two logit
    buffers and the dK accumulators (512 columns), else one CTA per key tile."""
    cols = 256 + w.d_s + (w.d_t if w.teacher_grads else 0) + w.d_t // 2 + w.d_s // 2
    return "streamkl_bwd_dkv_persistent_kernel" if cols <= 512 else "streamkl_bwd_dkv_kernel"


def kernel_names(w) -> list:
    """The step's kernels in launch order: forward, loss mean, key-owner, query-owner."""
    return ["streamkl_fwd_persistent_kernel", "streamkl_mean_kernel", key_owner_kernel(w), "streamkl_bwd_dq_kernel"]


def kernel_flops(w) -> dict:
    """MMA FLOPs each kernel issues per launch (what its tensor pipe executes)."""
    n = visible_pairs(w) * w.B * w.H
    s = 2 * (w.d_t + w.d_s)                      # S_t and S_s
    g = 2 * w.d_s + (2 * w.d_t if w.teacher_grads else 0)
    fwd, mean, dkv, dq = kernel_names(w)
    return {fwd: s * n, dkv: (s + g) * n, dq: (s + g) * n, mean: 0.0}


def kernel_method_flops(w) -> dict:
    """The method's own FLOPs attributed to each kernel per launch (step_flops
    split over the kernels): the forward's logits; for each backward kernel its
    own gradient contraction plus half of the one logit recompute the method
    counts (the second recompute is this design's duplicate, not the method's)."""
    n = visible_pairs(w) * w.B * w.H
    s = 2 * (w.d_t + w.d_s)
    g = 2 * w.d_s + (2 * w.d_t if w.teacher_grads else 0)
    fwd, mean, dkv, dq = kernel_names(w)
    return {fwd: s * n, dkv: (s / 2 + g) * n, dq: (s / 2 + g) * n, mean: 0.0}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle sampling of one GPU while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        import torch
        self.proc = None
        self.lines = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        self.cmd = ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self) -> dict:
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, pw, reasons = [], None, [], set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
                pw.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [s for s, p in zip(sm, pw) if p > 250.0] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "samples_under_load": len(loaded), "power_w_max": max(pw)}


# ----------------------------------------------------------------------------- helpers

def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops_sustained"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS, "fallback"


def kernel_source_hash() -> str:
    """Hash of the device code (the .cuh files that define the kernels)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "attention_kl_divergence_attn_b200", "csrc")
    for fn in sorted(f for f in os.listdir(csrc) if f.endswith(".cuh")):
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary of the current sources, else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    # the counters hold for the sources they were taken from, and for later
    # sources listed with the change that left the captured kernels as they were
    here = kernel_source_hash()
    if rec.get("source_hash") != here and here not in {e.get("hash") for e in rec.get("unchanged_for", [])}:
        return None
    e = rec.get("kernels", {}).get(kernel, {})
    if e.get("workload") != workload:
        return None
    return e.get("dram_bytes_per_launch")


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(w, n_rows: int, seed: int, cores: int, heads: int = 1):
    """Times the fp64 oracle on `n_rows` seeded rows of each of the first
    `heads` (batch, head) slices: forward of those rows plus their full backward
    (dQ rows and dK contributions).  Returns (seconds, metric FLOPs of the
    sampled (query, key) pairs, rows per head)."""
    import numpy as np
    import oracle
    from attention_kl_divergence_attn_b200 import inputs
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(w.N_Q, size=min(n_rows, w.N_Q), replace=False)).astype(np.int64)
    g = 1.0 / w.rows
    dt = 0.0
    for k in range(heads):
        b, h = divmod(k % (w.B * w.H), w.H)
        qt, kt, qs, ks = (oracle._f64(t[None, None]) for t in inputs.head_inputs(w, b, h))
        t0 = time.perf_counter()
        oracle.rows(qt, kt, qs, ks, w.scale_t, w.scale_s, w.causal, rows, nthreads=cores)
        oracle.bwd_rows(qt, kt, qs, ks, w.scale_t, w.scale_s, w.causal, g, rows, teacher=w.teacher_grads,
                        nthreads=cores)
        dt += time.perf_counter() - t0
    if w.causal:
        pairs = float(np.minimum(w.N_K, rows + (w.N_K - w.N_Q) + 1).sum())
    else:
        pairs = float(len(rows) * w.N_K)
    per = step_flops(w) / (visible_pairs(w) * w.B * w.H)
    return dt, per * pairs * heads, len(rows)


def rows_for(w, seconds: float, cores: int) -> int:
    """Rows of one head the oracle processes in about `seconds` (two-point
    calibration, so the fixed per-call cost does not inflate the estimate)."""
    t1, _, n1 = oracle_sample(w, 32, 1, cores)
    t2, _, n2 = oracle_sample(w, 256, 2, cores)
    per_row = max((t2 - t1) / max(n2 - n1, 1), 1e-6)
    fixed = max(t1 - per_row * n1, 0.0)
    return int(min(w.N_Q, max(16, (seconds - fixed) / per_row)))


def cpu_baseline(w, target_s: float = 15.0):
    """The oracle on about `target_s` seconds of the workload: a seeded sample of
    rows of head (0,0), or whole heads (0,0), (0,1), ... when one head takes
    less; the full step's time is extrapolated linearly from the sample."""
    cores = cpu_cores()
    n_rows = rows_for(w, target_s, cores)
    heads = 1
    if n_rows >= w.N_Q:                             # one whole head is quick: take several
        t1, _, _ = oracle_sample(w, w.N_Q, 3, cores)
        heads = int(max(1, min(w.B * w.H, round(target_s / max(t1, 1e-3)))))
    dt, fl, n = oracle_sample(w, n_rows, 3, cores, heads)
    value = fl / dt / 1e12
    return {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} seeded query rows of each of the first {heads} (batch, head) slice(s): forward plus full backward "
                      f"({'teacher and student' if w.teacher_grads else 'student'} gradients) in fp64, "
                      f"{dt:.1f} s wall, metric FLOPs counted over the rows' visible keys",
            "gflops": value * 1e3,
            "extrapolated_full_step_s": step_flops(w) / (value * 1e12)}


# ----------------------------------------------------------------------------- multi-rank helpers

def rank_workload(w, rank: int):
    """The workload one rank solves: the same shape, its own seed (ranks are
    independent problems; no data crosses between them)."""
    return dataclasses.replace(w, seed=w.seed + 7919 * rank)


def max_over_ranks(values, world: int, device):
    """Element-wise maximum of per-rank timings (the slowest rank decides)."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank's FLOPs over the slowest rank's step time."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cores = cpu_cores()
    total = args.steps + args.warmup
    budget = 150.0                                  # seconds for the whole run
    n_rows = rows_for(w, budget / total, cores)
    for k in range(args.warmup):
        oracle_sample(w, n_rows, 200 + k, cores)
    tsum = fsum = 0.0
    for k in range(args.steps):
        dt, fl, n = oracle_sample(w, n_rows, 1000 + k, cores)
        tsum += dt
        fsum += fl
    value = fsum / tsum / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tsum / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: {n_rows} seeded query rows of head (0,0), forward plus full "
                                   f"backward in fp64 on {cores} host threads"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- materialised comparison

_LOGITS_MODE = {}


def materialised_logits(a, b):
    """a [B,H,N,d] @ b[B,H,M,d]^T in fp32 from bf16 inputs: a bf16 GEMM with fp32
    output where torch has it (with autograd) on this device, else an fp32 GEMM of
    the upcast inputs (TF32 off), so the logits are fp32 either way."""
    import torch
    B, H, N, d = a.shape
    M = b.shape[2]
    mode = _LOGITS_MODE.get(a.device)
    if mode is None:
        mode = "fp32 GEMM"
        try:
            t = torch.ones(1, 2, 2, dtype=torch.bfloat16, device=a.device, requires_grad=True)
            torch.bmm(t, t, out_dtype=torch.float32).sum().backward()
            mode = "bf16 GEMM, fp32 output"
        except Exception:
            pass
        _LOGITS_MODE[a.device] = mode
    if mode == "fp32 GEMM":
        return torch.matmul(a.float(), b.float().transpose(-1, -2))
    return torch.bmm(a.reshape(B * H, N, d), b.reshape(B * H, M, d).transpose(1, 2),
                     out_dtype=torch.float32).reshape(B, H, N, M)


def materialised_step(x, w, mask=None):
    """The computation the fused method replaces: both [B, H, N_Q, N_K] logit
    matrices and both log-softmax distributions materialised in fp32, the
    per-row KL(P || Q) reduced from them, and autograd through all of it for
    the gradients of the mean loss (left in x[i].grad).  Returns (kl, loss)."""
    import torch.nn.functional as F
    for t in x:
        t.grad = None
    st = materialised_logits(x[0], x[1]) * w.scale_t
    ss = materialised_logits(x[2], x[3]) * w.scale_s
    if mask is not None:                  # finite fill: P = 0 there, and no inf - inf
        st = st.masked_fill(mask, -1e9)
        ss = ss.masked_fill(mask, -1e9)
    logp, logq = F.log_softmax(st, -1), F.log_softmax(ss, -1)
    kl = F.kl_div(logq, logp, reduction="none", log_target=True).sum(-1)
    loss = kl.mean()
    loss.backward()
    return kl.detach(), loss.detach()


def materialised_mask(w, device):
    """The causal mask (True = hidden) of a workload, or None."""
    import torch
    if not w.causal:
        return None
    i = torch.arange(w.N_Q, device=device)[:, None]
    j = torch.arange(w.N_K, device=device)[None, :]
    return j > i + (w.N_K - w.N_Q)


def run_materialised(args, w):
    """The computation the fused method replaces, in torch eager on one GPU
    (materialised_step).  Same FLOP count, so the value compares directly; the
    peak device memory is reported next to it.  Rank 0 only."""
    import torch
    from attention_kl_divergence_attn_b200 import inputs
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    base = {"impl": "materialised", "metric": METRIC, "unit": "TFLOP/s", "n_gpus": 1,
            "config": workload_config(w), "data": "synthetic"}
    try:
        x = [t.to(dev) for t in inputs.make_inputs(w)]
        for i, t in enumerate(x):
            t.requires_grad_(i >= 2 or w.teacher_grads)
        mask = materialised_mask(w, dev)
        for _ in range(args.warmup):
            materialised_step(x, w, mask)
        torch.cuda.synchronize(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        steps = min(args.steps, 20)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(steps):
            materialised_step(x, w, mask)
        t1.record()
        torch.cuda.synchronize(dev)
        ms = t0.elapsed_time(t1) / steps
    except torch.cuda.OutOfMemoryError as exc:
        print(json.dumps(dict(base, unavailable=f"out of device memory: {str(exc).splitlines()[0]}")), flush=True)
        return 0
    line = dict(base, value=step_flops(w) / (ms * 1e-3) / 1e12, ms_per_step=ms, steps=steps,
                warmup=args.warmup, higher_is_better=True,
                dtype=f"bf16 inputs, logits by {_LOGITS_MODE.get(dev)}, fp32 softmax/KL",
                peak_device_bytes=int(torch.cuda.max_memory_allocated(dev)))
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w) -> dict:
    in_bytes = 2 * w.B * w.H * (w.N_Q * (w.d_t + w.d_s) + w.N_K * (w.d_t + w.d_s))
    return {"workload": w.name, "B": w.B, "H": w.H, "N_Q": w.N_Q, "N_K": w.N_K, "d_t": w.d_t, "d_s": w.d_s,
            "causal": w.causal, "teacher_grads": w.teacher_grads, "student": w.student,
            "flops_per_step": step_flops(w),
            "l2": (f"inputs {in_bytes / 1e6:.0f} MB per step vs 126 MB L2; no flush"
                   if in_bytes > L2_BYTES else
                   "L2 flushed between steps (256 MB write, outside each step's event window)")}


# ----------------------------------------------------------------------------- main arm

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["mine", "reference", "materialised"], default="mine")
    ap.add_argument("--workload", default="causal_8k_d128")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    from attention_kl_divergence_attn_b200 import inputs
    w = inputs.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.impl == "materialised":
        return run_materialised(args, w)

    import torch
    import torch.distributed as dist
    import attention_kl_divergence_attn_b200 as skl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    # each rank solves its own independent problem (its own seed)
    wr = rank_workload(w, rank)
    host = [t.pin_memory() for t in inputs.make_inputs(wr)]
    x = [t.to(dev, non_blocking=True) for t in host]
    B, H, NQ, NK, dt_, ds_ = w.B, w.H, w.N_Q, w.N_K, w.d_t, w.d_s
    f32 = dict(dtype=torch.float32, device=dev)
    kl, lt, ls = (torch.empty(B, H, NQ, **f32) for _ in range(3))
    loss = torch.empty((), **f32)
    dqs, dks = torch.empty(B, H, NQ, ds_, **f32), torch.empty(B, H, NK, ds_, **f32)
    dqt = torch.empty(B, H, NQ, dt_, **f32) if w.teacher_grads else None
    dkt = torch.empty(B, H, NK, dt_, **f32) if w.teacher_grads else None
    flush = None
    if 2 * B * H * (NQ + NK) * (dt_ + ds_) <= L2_BYTES:
        flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    kw = dict(stream=stream)

    names = kernel_names(w)

    outs0 = (kl, lt, ls, loss, dqs, dks, dqt, dkt)

    def step(ev=None, x=x, o=outs0):
        kl, lt, ls, loss, dqs, dks, dqt, dkt = o
        if flush is not None:
            flush.zero_()
        if ev is not None:
            ev[0].record(stream)
        skl.streamkl_fwd(*x, w.scale_t, w.scale_s, w.causal, loss_mean=False, out=(kl, lt, ls), **kw)
        if ev is not None:
            ev[1].record(stream)
        skl.streamkl_loss_mean(kl, out=loss, **kw)
        if ev is not None:
            ev[2].record(stream)
        skl.streamkl_bwd_dk(*x, kl, lt, ls, w.scale_t, w.scale_s, w.causal, teacher_grads=w.teacher_grads,
                            out=(dks, dkt), **kw)
        if ev is not None:
            ev[3].record(stream)
        skl.streamkl_bwd_dq(*x, kl, lt, ls, w.scale_t, w.scale_s, w.causal, teacher_grads=w.teacher_grads,
                            out=(dqs, dqt), **kw)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    skl.streamkl_check(stream)

    # memory proof: one step allocates nothing beyond the buffers above
    torch.cuda.reset_peak_memory_stats(dev)
    alloc0 = torch.cuda.memory_allocated(dev)
    free0 = torch.cuda.mem_get_info(dev)[0]
    step()
    torch.cuda.synchronize(dev)
    memory = {"extra_bytes_during_step": int(torch.cuda.max_memory_allocated(dev) - alloc0),
              "device_free_delta_bytes": int(free0 - torch.cuda.mem_get_info(dev)[0]),
              "workspace_bytes": int(skl.workspace(dev).numel()),
              "materialised_fp32_bytes_per_distribution": B * H * NQ * NK * 4}
    # launches per step: the four kernels, plus the combine kernels when key splits are planned
    split = skl.workspace_size(B, H, NQ, NK, dt_, ds_, w.causal) > 256
    launches_per_step = 4 + ((2 + (1 if w.teacher_grads else 0)) if split else 0)

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    with sampler:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        t0.record(stream)
        for k in range(K):
            step(evs[k])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    ms_total = t0.elapsed_time(t1)
    if flush is not None:
        # the L2 flush runs between steps: time each step from its first to its
        # last event (the flush before it excluded) and sum over the steps
        ms_total = sum(e[0].elapsed_time(e[4]) for e in evs)
    per_kernel = {n: 0.0 for n in names}
    for e in evs:
        for i, n in enumerate(names):
            per_kernel[n] += e[i].elapsed_time(e[i + 1])
    per_kernel = {n: v / K for n, v in per_kernel.items()}
    # forward (with the loss) and backward on their own: medians over the steps
    fwd_ms = statistics.median(e[0].elapsed_time(e[2]) for e in evs)
    bwd_ms = statistics.median(e[2].elapsed_time(e[4]) for e in evs)
    # a plain bf16 GEMM through torch (cuBLAS) in the same run, as a reference rate
    ga = torch.randn(8192, 8192, device=dev).bfloat16()
    gb = torch.randn(8192, 8192, device=dev).bfloat16()
    for _ in range(3):
        torch.matmul(ga, gb)
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(20):
        torch.matmul(ga, gb)
    g1.record(stream)
    torch.cuda.synchronize(dev)
    cublas_tflops = 2 * 8192 ** 3 * 20 / (g0.elapsed_time(g1) * 1e-3) / 1e12
    del ga, gb
    code = skl.streamkl_check(stream)

    # End to end through the public API: every step copies its inputs from pinned
    # host memory to the device and reads its results back to pinned host memory
    # (the loss and all gradients; the per-row KL and LSEs stay on the device as
    # the backward's inputs).  Uploads run on one copy stream into one of two
    # device input sets, downloads on another from one of two device output sets,
    # so step k+1's upload and step k-1's download overlap step k's kernels (all
    # inside the timed region).  A second variant reads back only the loss.
    h2d = sum(t.numel() * t.element_size() for t in host)
    xs = [x, [torch.empty_like(t) for t in x]]
    outs = [outs0, tuple(None if t is None else torch.empty_like(t) for t in outs0)]
    back = [(3, 4, 5, 6, 7), (3,)]                   # output indices read back: everything / the loss only
    host_out = [None if t is None else torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs0]
    up_stream, down_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    copied = [torch.cuda.Event() for _ in range(2)]  # inputs of set i uploaded
    used = [torch.cuda.Event() for _ in range(2)]    # the step on set i is done
    fetched = [torch.cuda.Event() for _ in range(2)] # outputs of set i downloaded
    for e in fetched:
        e.record(down_stream)

    def upload(i):
        with torch.cuda.stream(up_stream):
            up_stream.wait_event(used[i])            # the step that last read set i is done
            for dst, src in zip(xs[i], host):
                dst.copy_(src, non_blocking=True)
            copied[i].record(up_stream)

    def download(i, which):
        with torch.cuda.stream(down_stream):
            down_stream.wait_event(used[i])
            for j in back[which]:
                if outs[i][j] is not None:
                    host_out[j].copy_(outs[i][j], non_blocking=True)
            fetched[i].record(down_stream)

    def d2h_bytes(which):
        return sum(outs0[j].numel() * outs0[j].element_size() for j in back[which] if outs0[j] is not None)

    def e2e_run(n, which, start=None):
        if start is not None:
            up_stream.wait_event(start)
            down_stream.wait_event(start)
        upload(0)
        for k in range(n):
            cur = k & 1
            if k + 1 < n:
                upload(cur ^ 1)
            stream.wait_event(copied[cur])
            stream.wait_event(fetched[cur])          # set cur's previous results are on the host
            step(x=xs[cur], o=outs[cur])
            used[cur].record(stream)
            download(cur, which)
        stream.wait_event(fetched[(n - 1) & 1])      # the last results are on the host

    ms_e2e = []
    for which in range(2):
        e2e_run(args.warmup, which)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        e0.record(stream)
        e2e_run(K, which, start=e0)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e.append(e0.elapsed_time(e1))
    ms_e2e, ms_e2e_loss = ms_e2e

    if world > 1:
        ms_total, ms_e2e, ms_e2e_loss = max_over_ranks([ms_total, ms_e2e, ms_e2e_loss], world, dev)

    ms_step = ms_total / K
    flops = step_flops(w)
    value = job_throughput(flops, world, ms_step)
    e2e_value = job_throughput(flops, world, ms_e2e / K)
    e2e_loss_value = job_throughput(flops, world, ms_e2e_loss / K)

    sustained, burst, peak_src = measured_peak()
    kf, km = kernel_flops(w), kernel_method_flops(w)
    dominant = max((n for n in names if kf[n] > 0), key=lambda n: per_kernel[n])
    # the kernels are timed with CUDA events over millisecond launches, so the
    # burst GEMM rate is the denominator; `achieved` counts the method's own
    # FLOPs in the launch, `achieved_issued` every MMA FLOP it issues
    achieved = km[dominant] / (per_kernel[dominant] * 1e-3) / 1e12
    achieved_issued = kf[dominant] / (per_kernel[dominant] * 1e-3) / 1e12
    traffic = recorded_traffic(dominant, w.name)

    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            try:
                cpu = cpu_baseline(w)
            except Exception as exc:                 # the CPU leg must not hide the GPU number
                cpu = {"value": None, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                       "sample": f"failed: {exc}"}
        total_k = sum(per_kernel.values())
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_config(w), parallelism=f"independent problem per GPU x{world}"),
            "pct_of_nominal_bf16_peak": 100.0 * value / world / NOMINAL_BF16_TFLOPS,
            "pct_of_measured_bf16_peak": 100.0 * value / world / burst,
            "roofline": {"bound": "tensor", "kernel": dominant, "achieved": achieved, "peak": burst,
                         "unit": "TFLOP/s", "frac": achieved / burst, "traffic": traffic,
                         "frac_method": achieved / burst, "frac_issued": achieved_issued / burst,
                         "achieved_issued": achieved_issued,
                         "peak_source": f"bf16_tflops (burst) of {peak_src}",
                         "flops_per_launch": km[dominant], "issued_flops_per_launch": kf[dominant]},
            "kernels": {n: {"ms": per_kernel[n], "share": per_kernel[n] / total_k,
                            "mma_tflops": (kf[n] / (per_kernel[n] * 1e-3) / 1e12) if kf[n] else None}
                        for n in names},
            "phases": {"fwd_ms_median": fwd_ms, "bwd_ms_median": bwd_ms,
                       "fwd_tflops": fwd_flops(w) / (fwd_ms * 1e-3) / 1e12,
                       "bwd_tflops": (flops - fwd_flops(w)) / (bwd_ms * 1e-3) / 1e12},
            "cublas_bf16_gemm_tflops_same_run": cublas_tflops,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h_bytes(0),
                    "reads_back": "loss and every gradient (dQ_s, dK_s" + (", dQ_t, dK_t)" if w.teacher_grads else ")")},
            "e2e_loss_only": {"value": e2e_loss_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                              "d2h_bytes_per_step": d2h_bytes(1)},
            "gpu_launches": launches_per_step * K,
            "memory": memory,
            "clocks": sampler.summary(),
            "device_status": code,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
