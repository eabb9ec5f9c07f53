#!/usr/bin/env python
"""Benchmark of the ZeRO partitioned optimizer step on B200.

One step = the whole hot path on one batch of synthetic gradients: reduce-scatter of
every bucket of W replica gradients (fp32 rank-ordered sum + fp64 sum of squares),
the finalize kernel (overflow, norm, clip, loss scaler, step constants) and the fused
AdamW + half-cast update of every rank's partition (which is also the all-gather).

Default workload: the Llama-7B-shaped tensor list (6,738,415,616 params, 291 tensors),
W = 8 simulated ranks, bf16 gradients, reduce_bucket_size 5e8 (14 buckets). Replica
buffers hold one bucket (2 slots of W x 5e8 bf16, generated before timing); fp32
master / m / v / reduced gradient and the bf16 gathered buffer are resident
(about 137 GB). Each step moves about 337 GB, far more than L2, so no flush is needed.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs an independent replica of the workload on its
own GPU (the single-GPU step has no cross-GPU exchange); the time is the max over
ranks and `value` counts the parameters all ranks updated.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ZeRO step params/s and achieved HBM GB/s vs ~8 TB/s peak, W=8 simulated ranks"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama7b",
                    help="llama7b | gpt2 | enc | tiny | sweep")
    ap.add_argument("--log2n", type=int, default=26, help="sweep: log2 of the parameter count")
    ap.add_argument("--world", type=int, default=8, help="sweep: simulated ranks W")
    ap.add_argument("--dtype", default="bf16", help="sweep: bf16 | fp16")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--sweep", action="store_true",
                    help="roofline sweep: 2^{24,26,28,30} x W in {1,2,4,8,16} x {bf16, fp16}; "
                         "one JSON line per point")
    ap.add_argument("--sweep-log2n", default="24,26,28,30")
    ap.add_argument("--sweep-world", default="1,2,4,8,16")
    ap.add_argument("--sweep-dtype", default="bf16,fp16")
    ap.add_argument("--resident", action="store_true",
                    help="sweep: points with W <= 2 keep whole-model replica buffers and run "
                         "zero_step_resident (4W + 26 bytes per parameter)")
    ap.add_argument("--graph", action="store_true",
                    help="replay each step from a CUDA graph (launch-bound small workloads)")
    ap.add_argument("--micro", type=int, default=1,
                    help="gradient accumulation: micro-batches per step (each reduces every "
                         "bucket; the later ones add into the reduced gradient)")
    ap.add_argument("--overlap", action="store_true",
                    help="overlap_comm: each bucket's gradients are produced (generated) on a "
                         "second stream while the previous bucket is reduced; timed against "
                         "producing and reducing on one stream")
    ap.add_argument("--checkpoint", action="store_true",
                    help="sharded checkpoint save / load (and a resharded load) of the "
                         "optimizer state after one step; workload --checkpoint-workload")
    ap.add_argument("--checkpoint-workload", default="gpt2")
    ap.add_argument("--zero3", action="store_true",
                    help="ZeRO-3 forward gather / release over the 7B tensor list")
    return ap.parse_args()


def get_workload(args):
    import synthgen
    if args.workload == "sweep":
        return synthgen.sweep(args.log2n, args.world, args.dtype)
    wl = synthgen.workload(args.workload)
    return wl


def max_over_ranks(x: float, world_size: int, device) -> float:
    """The largest of every rank's x (the job's time is its slowest rank's). A collective
    of the default process group on `device` (a CUDA device under NCCL, "cpu" under gloo);
    every rank calls it in the same order."""
    if world_size <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step: int, steps: int, world_size: int, seconds: float) -> float:
    """Units processed by all ranks per second of the slowest rank (weak scaling: every
    rank runs the same workload)."""
    return units_per_rank_step * steps * world_size / seconds


def workload_config(wl, n_buckets: int, n_pad: int, world_size: int, micro: int = 1) -> dict:
    """The `config` object of the JSON line (both arms describe the same workload)."""
    step_bytes = (schedule_bytes_per_param(wl.world) + (micro - 1) * (2 * wl.world + 8)) * n_pad
    return {
        "workload": f"{wl.name}_w{wl.world}",
        "params": wl.n,
        "tensors": len(wl.tensors),
        "W": wl.world,
        "reduce_bucket_size": wl.bucket,
        "buckets": n_buckets,
        "grad_dtype": wl.gdtype,
        "replica_buffers": "bucket-sized, 2 slots" if wl.streaming else "resident",
        "micro_batches": micro,
        "l2": f"no flush: each step moves {step_bytes / 1e9:.0f} GB, inputs >> 126 MB L2",
        "parallelism": f"replicas x{world_size} (simulated dp{wl.world} per GPU)",
    }


def schedule_bytes_per_param(W: int) -> int:
    # reduce-scatter: W half reads + fp32 write; update: fp32 R, p, m, v reads, p, m, v
    # writes and the half write
    return 2 * W + 4 + 16 + 14


def model_bytes_per_param(W: int) -> int:
    return 2 * W + 26


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    with open(os.path.join(ROOT, "zero_sharded_mixed_replica_b200", "csrc", "kernels.cu"), "rb") as f:
        h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    src_hash, traffic = None, None
    hash_key, traffic_key = "kernels.cu sha256[:16]:", "dram bytes per launch:"
    with open(path) as f:
        for line in f:
            if line.startswith(hash_key):
                src_hash = line[len(hash_key):].strip()
            if line.startswith(traffic_key):
                traffic = float(line[len(traffic_key):].split()[0])
    if src_hash != kernel_source_hash():
        return None
    return traffic


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 100):
        self.gpu_index = gpu_index
        self.period_ms = period_ms
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 f"-lms", str(self.period_ms), "-i", str(self.gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.reader.join(timeout=2)
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------- our arm

def run_ours(args, rank: int, world_size: int, local_rank: int):
    import torch
    import torch.distributed as dist

    from synthgen import device as sdev
    import zero_sharded_mixed_replica_b200 as zb

    wl = get_workload(args)
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    s = torch.cuda.Stream(dev)
    torch.cuda.set_stream(s)
    sh = s.cuda_stream
    half = {"bf16": torch.bfloat16, "fp16": torch.float16}[wl.gdtype]

    scaler = zb.scaler_cfg(wl.dynamic, wl.init_scale_power, wl.loss_scale_window,
                           wl.hysteresis, wl.min_loss_scale)
    adamw = zb.adamw_cfg(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.max_grad_norm)
    opt = zb.ZeroOptimizer([t.shape for t in wl.tensors], wl.world, wl.bucket, wl.gdtype,
                           wl.align, scaler, adamw, device=str(dev), stream=s)
    plan = opt.plan
    n_pad, W, nb = plan.n_pad, wl.world, plan.n_buckets
    sdev.init_master(wl, opt.master, sh)
    opt.cast_params()
    # replica gradients: streaming workloads use two slots of W bucket-sized buffers
    # (indexed from the bucket start); resident ones whole-model buffers (flat index)
    L = min(wl.bucket, n_pad) if wl.streaming else n_pad
    slots = [[torch.zeros(L, dtype=half, device=dev) for _ in range(W)] for _ in range(2)]
    scale = float(2.0 ** wl.init_scale_power) if wl.dynamic else 1.0
    for k in range(2):
        sdev.fill_grads(wl, slots[k], 0, min(L, wl.n), k + 1, scale, sh)
    torch.cuda.synchronize(dev)

    M = max(1, args.micro)
    ev_k1 = [[torch.cuda.Event(enable_timing=True) for _ in range(2)]
             for _ in range(args.steps * nb * M)]
    ev_k3 = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    ev_k2 = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]

    def one_step(t: int, timed: int = -1):
        bufs = slots[(t - 1) % 2] if wl.streaming else slots[0]
        for k in range(M):  # micro-batches reuse the resident replica slot
            for b in range(nb):
                e = (timed * M + k) * nb + b
                if timed >= 0:
                    ev_k1[e][0].record(s)
                base = b * wl.bucket if wl.streaming else 0
                if M == 1:
                    opt.reduce_scatter_bucket(b, bufs, base_offset=base)
                else:
                    opt.reduce_scatter_bucket_accum(b, k, M, bufs, base_offset=base)
                if timed >= 0:
                    ev_k1[e][1].record(s)
        if timed >= 0:
            ev_k2[timed][0].record(s)
        opt.step_finalize()
        if timed >= 0:
            ev_k2[timed][1].record(s)
            ev_k3[timed][0].record(s)
        opt.step_update()
        if timed >= 0:
            ev_k3[timed][1].record(s)

    graphs = None
    if args.graph and M > 1:
        raise SystemExit("--graph with --micro > 1 is not supported")
    if args.graph:
        # one graph per replica slot; replays keep all step state on the device
        graphs = []
        for k in range(2 if wl.streaming else 1):
            g = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream(dev)
            side.wait_stream(s)
            keep = opt.stream
            opt.stream = side
            with torch.cuda.stream(side), torch.cuda.graph(g, stream=side):
                for b in range(nb):
                    opt.reduce_scatter_bucket(b, slots[k],
                                              base_offset=b * wl.bucket if wl.streaming else 0)
                opt.step()
            opt.stream = keep
            s.wait_stream(side)
            graphs.append(g)

        def one_step(t: int, timed: int = -1):  # noqa: F811  (graph replay)
            graphs[(t - 1) % len(graphs)].replay()

    step_no = 0
    for _ in range(args.warmup):
        step_no += 1
        one_step(step_no)
    torch.cuda.synchronize(dev)
    if world_size > 1:
        dist.barrier()
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    if world_size > 1:
        dist.barrier()
    t_wall0 = time.perf_counter()
    start.record(s)
    for i in range(args.steps):
        step_no += 1
        one_step(step_no, timed=i)
    end.record(s)
    torch.cuda.synchronize(dev)
    t_wall = time.perf_counter() - t_wall0
    if world_size > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms_total = start.elapsed_time(end)
    res = opt.result()

    # Optional all-gather into per-rank copies (not part of the step: the gathered
    # buffer is complete after the update). Timed apart on n_dst destinations that fit
    # next to the resident state.
    free_b, _ = torch.cuda.mem_get_info(dev)
    n_dst = int(min(W, max(0, (free_b - (4 << 30)) // (2 * n_pad))))
    k4 = None
    if n_dst > 0:
        dst = [torch.empty(n_pad, dtype=half, device=dev) for _ in range(n_dst)]
        opt.all_gather(dst)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        opt.all_gather(dst)
        e1.record(s)
        torch.cuda.synchronize(dev)
        k4_ms = e0.elapsed_time(e1)
        k4 = {"n_dst": n_dst, "ms": k4_ms,
              "gbs": (2 + 2 * n_dst) * n_pad / (k4_ms / 1e3) / 1e9}
        del dst

    if graphs is None:
        k1_ms = [a.elapsed_time(b) for a, b in ev_k1]
        k2_ms = [a.elapsed_time(b) for a, b in ev_k2]
        k3_ms = [a.elapsed_time(b) for a, b in ev_k3]
    else:  # no events inside a graph: only whole steps are timed
        k1_ms = k2_ms = k3_ms = [float("nan")]

    ms_max = max_over_ranks(ms_total, world_size, dev)

    out = None
    if rank == 0:
        ms_step = ms_max / args.steps
        params_step = plan.n  # parameters updated per step (padding excluded)
        value = whole_job_rate(params_step, args.steps, world_size, ms_max / 1e3)
        peak, peak_kind = measured_peaks()
        k3_avg = sum(k3_ms) / len(k3_ms)
        k3_bytes = 30 * n_pad  # R, p, m, v read (16 B) + p, m, v write (12 B) + half (2 B)
        k3_gbs = k3_bytes / (k3_avg / 1e3) / 1e9
        # first micro-batch passes (2W + 4 B/param) and accumulate passes (2W + 8)
        first = [i for i in range(len(k1_ms)) if (i // nb) % M == 0]
        later = [i for i in range(len(k1_ms)) if (i // nb) % M != 0]
        full_b = [k1_ms[i] for i in first if plan.bucket(i % nb)[1] == wl.bucket] or \
            [k1_ms[i] for i in first]
        k1_avg = sum(full_b) / len(full_b)
        k1_bytes = (2 * W + 4) * plan.bucket(0)[1]
        acc = None
        if later and graphs is None:
            acc_b = [k1_ms[i] for i in later if plan.bucket(i % nb)[1] == wl.bucket] or \
                [k1_ms[i] for i in later]
            acc_ms = sum(acc_b) / len(acc_b)
            acc = {"ms_per_full_bucket": acc_ms,
                   "gbs": (2 * W + 8) * plan.bucket(0)[1] / (acc_ms / 1e3) / 1e9,
                   "bytes_per_param": 2 * W + 8}
        step_bytes = (schedule_bytes_per_param(W) + (M - 1) * (2 * W + 8)) * n_pad
        sched_gbs = step_bytes / (ms_step / 1e3) / 1e9
        model_gbs = (model_bytes_per_param(W) + (M - 1) * 2 * W) * plan.n / (ms_step / 1e3) / 1e9
        traffic = profiled_traffic("adamw_cast", wl.name)
        out = {
            "metric": METRIC,
            "value": value,
            "unit": "params/s",
            "n_gpus": world_size,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32",  # arithmetic of the step (half inputs, fp64 norm)
            "data": "synthetic (seeded Philox gradients and init; random-init weights of the shape list)",
            "config": workload_config(wl, nb, n_pad, world_size, M),
            "hbm_gbs_schedule": sched_gbs,
            "hbm_gbs_model": model_gbs,
            "frac_of_8tbs_schedule": sched_gbs / 8000.0,
            "frac_of_peak_schedule": sched_gbs / peak,
            "stage_ms": {"reduce_scatter_total": sum(k1_ms) / args.steps,
                         "finalize": sum(k2_ms) / len(k2_ms),
                         "adamw_cast": k3_avg},
            "reduce_scatter_gbs": k1_bytes / (k1_avg / 1e3) / 1e9,
            "accumulate_pass": acc,
            "all_gather_copies": k4,
            "roofline": {
                "kernel": "adamw_cast_kernel",
                "bound": "hbm",
                "achieved": k3_gbs,
                "peak": peak,
                "peak_kind": peak_kind,
                "unit": "GB/s",
                "frac": k3_gbs / peak,
                "traffic": traffic,
                "algorithmic_bytes_per_launch": k3_bytes,
            },
            "gpu_launches": args.steps * (M * nb + 2),
            "cuda_graph": bool(graphs),
            "clocks": clocks,
            "wall_s_timed": t_wall,
            "last_result": {k: res[k] for k in ("global_norm", "clip_coef", "adam_t", "skipped")},
        }
    if rank == 0 and graphs:
        out["stage_ms"] = None
        out["reduce_scatter_gbs"] = None
        out["roofline"] = {"kernel": "whole step (CUDA graph replay)", "bound": "hbm",
                           "achieved": sched_gbs, "peak": peak, "peak_kind": peak_kind,
                           "unit": "GB/s", "frac": sched_gbs / peak, "traffic": None,
                           "algorithmic_bytes_per_launch": schedule_bytes_per_param(W) * n_pad}
    del opt, slots, graphs
    torch.cuda.empty_cache()
    return out


def run_e2e(args, wl, local_rank: int, world_size: int = 1):
    """Same metric through the public C ABI with HOST gradient buffers: every bucket's
    replica slices are copied host -> device (pinned) inside the timed region by
    zero_reduce_scatter_bucket_host, and the step result is read back each step. Timed
    with CUDA events on the stream that carries the copies, the kernels and the result
    read (host waits between steps show up as idle time); max over ranks. With several
    ranks each keeps one pinned slot (every step reuses it) to bound host memory."""
    import torch

    import synthgen
    from synthgen import device as sdev
    import zero_sharded_mixed_replica_b200 as zb

    dev = torch.device("cuda", local_rank)
    s = torch.cuda.Stream(dev)
    torch.cuda.set_stream(s)
    scaler = zb.scaler_cfg(wl.dynamic, wl.init_scale_power, wl.loss_scale_window,
                           wl.hysteresis, wl.min_loss_scale)
    adamw = zb.adamw_cfg(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.max_grad_norm)
    opt = zb.ZeroOptimizer([t.shape for t in wl.tensors], wl.world, wl.bucket, wl.gdtype,
                           wl.align, scaler, adamw, device=str(dev), stream=s)
    plan = opt.plan
    W, nb = wl.world, plan.n_buckets
    sdev.init_master(wl, opt.master, s.cuda_stream)
    opt.cast_params()
    L = min(wl.bucket, plan.n_pad) if wl.streaming else plan.n_pad
    half = {"bf16": torch.bfloat16, "fp16": torch.float16}[wl.gdtype]
    # pinned host gradients: the same recipe as the device-resident run
    n_slots = 2 if world_size == 1 else 1
    host = [[torch.zeros(L, dtype=torch.int16).pin_memory() for _ in range(W)]
            for _ in range(n_slots)]
    # generated on the device (the same bits as the host generator) and copied into the
    # pinned buffers: seconds instead of a minute of host arithmetic per rank
    tmp = torch.zeros(L, dtype=torch.int16, device=dev)
    for k in range(n_slots):
        for r in range(W):
            synthgen.grads_cuda(tmp.data_ptr(), 0, min(L, wl.n), wl.seed, r, wl.slot(k + 1),
                                wl.grad_sigma, wl.spike_frac, 1.0, wl.dtype_code, s.cuda_stream)
            host[k][r].copy_(tmp)
    torch.cuda.synchronize(dev)
    del tmp
    staging = [torch.empty(min(wl.bucket, plan.n_pad), dtype=half, device=dev) for _ in range(W)]
    h2d = 0

    def one(t):
        nonlocal h2d
        hb = host[(t - 1) % n_slots]
        ptrs = [h.data_ptr() for h in hb]
        for b in range(nb):
            opt.reduce_scatter_bucket_host(b, ptrs, b * wl.bucket if wl.streaming else 0, staging)
            h2d += W * plan.bucket(b)[1] * 2
        opt.step()
        return opt.result()  # device -> host read of the step result (synchronises)

    import torch.distributed as dist
    one(1)
    torch.cuda.synchronize(dev)
    if world_size > 1:
        dist.barrier()
    h2d = 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for i in range(args.e2e_steps):
        one(i + 2)
    e1.record(s)
    torch.cuda.synchronize(dev)
    dt = max_over_ranks(e0.elapsed_time(e1) / 1e3, world_size, dev)
    out = {"value": whole_job_rate(plan.n, args.e2e_steps, world_size, dt), "unit": "params/s",
           "h2d_bytes_per_step": h2d // args.e2e_steps,
           "d2h_bytes_per_step": ctypes.sizeof(zb.StepResult),
           "steps": args.e2e_steps,
           "path": "zero_reduce_scatter_bucket_host (pinned host replicas) + zero_step + zero_get_result"}
    del opt, staging, host
    torch.cuda.empty_cache()
    return out


def run_sweep_point(wl, steps: int, local_rank: int, resident: bool = False) -> dict:
    """All steps of one sweep point. Replica slots are regenerated before every step
    (the loss scale in force for fp16, the +inf site at step 5) outside the timed part;
    each step's kernels are timed with CUDA events on the launching stream. With
    `resident` (W <= 2 only) the replicas cover the whole flat space and the step is
    zero_step_resident."""
    import torch

    from synthgen import device as sdev
    import zero_sharded_mixed_replica_b200 as zb

    dev = torch.device("cuda", local_rank)
    s = torch.cuda.Stream(dev)
    torch.cuda.set_stream(s)
    sh = s.cuda_stream
    half = {"bf16": torch.bfloat16, "fp16": torch.float16}[wl.gdtype]
    scaler = zb.scaler_cfg(wl.dynamic, wl.init_scale_power, wl.loss_scale_window,
                           wl.hysteresis, wl.min_loss_scale)
    adamw = zb.adamw_cfg(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.max_grad_norm)
    opt = zb.ZeroOptimizer([t.shape for t in wl.tensors], wl.world, wl.bucket, wl.gdtype,
                           wl.align, scaler, adamw, device=str(dev), stream=s)
    plan = opt.plan
    sdev.init_master(wl, opt.master, sh)
    opt.cast_params()
    resident = resident and wl.world <= 2
    L = plan.n_pad if resident else min(wl.bucket, plan.n_pad)
    slots = [[torch.empty(L, dtype=half, device=dev) for _ in range(wl.world)]
             for _ in range(1 if resident else 2)]
    scale = float(2.0 ** wl.init_scale_power) if wl.dynamic else 1.0
    inf_bits = torch.tensor(0x7C00 if wl.gdtype == "fp16" else 0x7F80,
                            dtype=torch.int32).to(torch.int16)
    applied, skipped = [], []
    for t in range(1, steps + 1):
        bufs = slots[(t - 1) % len(slots)]
        sdev.fill_grads(wl, bufs, 0, L, t, scale, sh)
        if resident:  # the +inf sites at their flat index
            for idx, rep in wl.inf_sites_at(t):
                bufs[rep].view(torch.int16)[idx] = inf_bits
        else:
            sdev.plant_infs(wl, bufs, t, wl.bucket)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        if resident:
            opt.step_resident(bufs)
        else:
            for bk in range(plan.n_buckets):
                opt.reduce_scatter_bucket(bk, bufs, base_offset=bk * wl.bucket)
            opt.step()
        b.record(s)
        res = opt.result()
        (skipped if res["skipped"] else applied).append(a.elapsed_time(b))
        scale = float(res["next_scale"]) if wl.dynamic else 1.0
    ms = statistics.median(applied[1:] if len(applied) > 2 else applied)
    W = wl.world
    sched = 4 * W + 26 if resident else schedule_bytes_per_param(W)
    out = {
        "point": wl.name, "params": plan.n, "W": W, "grad_dtype": wl.gdtype,
        "buckets": plan.n_buckets, "steps": steps,
        "schedule": "resident replicas (4W+26 B/param)" if resident else "stored R (2W+34 B/param)",
        "ms_per_applied_step_median": ms,
        "params_per_s": plan.n / (ms / 1e3),
        "hbm_gbs_schedule": sched * plan.n_pad / (ms / 1e3) / 1e9,
        "hbm_gbs_model": model_bytes_per_param(W) * plan.n / (ms / 1e3) / 1e9,
        "first_step_ms": (applied + skipped)[0],
        "skipped_steps": len(skipped),
        "ms_skipped_step_median": statistics.median(skipped) if skipped else None,
    }
    peak, kind = measured_peaks()
    out["frac_of_8tbs_schedule"] = out["hbm_gbs_schedule"] / 8000.0
    out["frac_of_peak_schedule"] = out["hbm_gbs_schedule"] / peak
    del opt, slots
    torch.cuda.empty_cache()
    return out


def run_zero3_forward(args, local_rank: int) -> dict:
    """The ZeRO-3 parameter side of a forward pass over the Llama-7B-shaped tensor list
    (one layer per transformer block, embedding first, head last), W = 8 partitions of
    the bf16 parameters on one GPU: every FETCH is a zero3_gather into a fresh buffer,
    every RELEASE drops it. Knobs: max live parameters 1e9 and persistence threshold 1e6
    as the pages configure them; the prefetch bucket the pages leave "auto" is taken as
    the reduce bucket, 5e8. Timed with CUDA events around whole passes."""
    import torch

    import synthgen
    import zero_sharded_mixed_replica_b200 as zb
    from zero_sharded_mixed_replica_b200 import zero3

    wl = synthgen.workload("llama7b")
    dev = torch.device("cuda", local_rank)
    layer_of = []
    for t in wl.tensors:
        if t.name.startswith("model.layers."):
            layer_of.append(int(t.name.split(".")[2]) + 1)
        else:
            layer_of.append(0 if t.name.startswith("model.embed") else 33)
    plan = zb.Plan([t.shape for t in wl.tensors], wl.world, wl.bucket, wl.align)
    sched = zb.Zero3Schedule(plan, layer_of, 34, 500_000_000, 1_000_000_000, 1_000_000)
    params = torch.empty(plan.n_pad, dtype=torch.bfloat16, device=dev)
    parts = zero3.partitions_of(params, plan)
    s = torch.cuda.current_stream(dev)
    for _ in range(max(1, args.warmup)):
        zero3.run_forward(plan, sched, parts, torch.bfloat16, lambda l, v: None, device=dev)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    passes = max(1, args.steps // 4)
    for _ in range(passes):
        zero3.run_forward(plan, sched, parts, torch.bfloat16, lambda l, v: None, device=dev)
    e1.record(s)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / passes
    fetched = sched.stats["fetched_elements"]
    peak, kind = measured_peaks()
    gbs = 4 * fetched / (ms / 1e3) / 1e9  # 2 B read + 2 B written per gathered element
    # the gather kernel alone, on the largest fetch of the pass
    big = max((ids for op, _, ids in sched.events if op == zb.ZERO3_FETCH),
              key=lambda ids: sum(plan.tensor_table[t][1] for t in ids))
    n_big = sum(plan.tensor_table[t][1] for t in big)
    dst = torch.empty(n_big, dtype=torch.bfloat16, device=dev)
    zb.zero3_gather(plan, big, parts, dst, s.cuda_stream)
    e0.record(s)
    for _ in range(10):
        zb.zero3_gather(plan, big, parts, dst, s.cuda_stream)
    e1.record(s)
    torch.cuda.synchronize(dev)
    k_ms = e0.elapsed_time(e1) / 10
    k_gbs = 4 * n_big / (k_ms / 1e3) / 1e9
    return {"mode": "zero3_forward_gather", "workload": "llama7b_w8", "passes": passes,
            "ms_per_forward": ms, "gathered_elements": fetched,
            "copy_gbs": gbs, "frac_of_peak": gbs / peak,
            "gather_kernel": {"elements": n_big, "tensors": len(big), "ms": k_ms,
                              "copy_gbs": k_gbs, "frac_of_peak": k_gbs / peak},
            "schedule": sched.stats}


def run_overlap(args, local_rank: int) -> dict:
    """ZeroOptimizer.overlapped_step on the streaming workload: bucket b's W replica
    gradients are generated into one of two bucket-sized slots (the stand-in for the
    backward pass producing them), then reduced. Three timings per step, CUDA events on
    the optimizer's stream: generation and reduction on one stream (serial), on two
    streams ordered by events (overlapped), and generation alone."""
    import torch

    from synthgen import device as sdev
    import zero_sharded_mixed_replica_b200 as zb

    wl = get_workload(args)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cons = torch.cuda.Stream(dev)
    torch.cuda.set_stream(cons)
    scaler = zb.scaler_cfg(wl.dynamic, wl.init_scale_power, wl.loss_scale_window,
                           wl.hysteresis, wl.min_loss_scale)
    adamw = zb.adamw_cfg(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.max_grad_norm)
    opt = zb.ZeroOptimizer([t.shape for t in wl.tensors], wl.world, wl.bucket, wl.gdtype,
                           wl.align, scaler, adamw, device=str(dev), stream=cons)
    sdev.init_master(wl, opt.master, cons.cuda_stream)
    opt.cast_params()
    half = {"bf16": torch.bfloat16, "fp16": torch.float16}[wl.gdtype]
    L = min(wl.bucket, opt.plan.n_pad)
    slots = [[torch.empty(L, dtype=half, device=dev) for _ in range(wl.world)] for _ in range(2)]
    scale = float(2.0 ** wl.init_scale_power) if wl.dynamic else 1.0
    state = {"t": 1}

    def produce(b, bufs, sh):
        sdev.fill_grads(wl, bufs, 0, opt.plan.bucket(b)[1], state["t"], scale, sh)

    def timed(prod, steps, fill_only=False):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(cons)
        prod.wait_stream(cons)
        for _ in range(steps):
            if fill_only:
                for b in range(opt.plan.n_buckets):
                    produce(b, slots[b % 2], cons.cuda_stream)
            else:
                opt.overlapped_step(produce, slots, prod)
            state["t"] += 1
        e1.record(cons)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / steps

    side = torch.cuda.Stream(dev)
    steps = max(2, args.steps // 4)
    timed(side, 1)  # warm-up
    out = {"mode": "overlap_comm", "workload": f"{wl.name}_w{wl.world}", "params": opt.plan.n,
           "buckets": opt.plan.n_buckets, "steps": steps,
           "ms_per_step_serial": timed(cons, steps),
           "ms_per_step_overlapped": timed(side, steps),
           "ms_generation_only": timed(cons, steps, fill_only=True),
           "producer": "seeded gradient generation (Philox + Irwin-Hall), ALU-bound"}
    out["ms_hidden"] = out["ms_per_step_serial"] - out["ms_per_step_overlapped"]
    opt.result()
    del opt, slots
    torch.cuda.empty_cache()
    return out


def run_checkpoint(args, local_rank: int) -> dict:
    """Wall-clock of `checkpoint.save` (device -> host, one file per rank, SHA-256) and
    `checkpoint.load` (read, verify, host -> device, rebuild the half parameters) of the
    fp32 master / exp_avg / exp_avg_sq after one step, and of a load resharded to W/2.
    Host I/O to a temporary directory: a measurement of the host side, not of a kernel."""
    import shutil
    import tempfile

    import torch

    import synthgen
    from synthgen import device as sdev
    import zero_sharded_mixed_replica_b200 as zb
    from zero_sharded_mixed_replica_b200 import checkpoint

    wl = synthgen.workload(args.checkpoint_workload)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    scaler = zb.scaler_cfg(wl.dynamic, wl.init_scale_power, wl.loss_scale_window,
                           wl.hysteresis, wl.min_loss_scale)
    adamw = zb.adamw_cfg(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.max_grad_norm)
    opt = zb.ZeroOptimizer([t.shape for t in wl.tensors], wl.world, wl.bucket, wl.gdtype,
                           wl.align, scaler, adamw, device=str(dev))
    s = torch.cuda.current_stream(dev).cuda_stream
    sdev.init_master(wl, opt.master, s)
    opt.cast_params()
    half = {"bf16": torch.bfloat16, "fp16": torch.float16}[wl.gdtype]
    L = min(wl.bucket, opt.plan.n_pad) if wl.streaming else opt.plan.n_pad
    grads = [torch.zeros(L, dtype=half, device=dev) for _ in range(wl.world)]
    sdev.fill_grads(wl, grads, 0, min(L, wl.n), 1, float(2.0 ** wl.init_scale_power)
                    if wl.dynamic else 1.0, s)
    for b in range(opt.plan.n_buckets):
        opt.reduce_scatter_bucket(b, grads, b * wl.bucket if wl.streaming else 0)
    opt.step()
    opt.result()
    del grads
    state_bytes = 12 * opt.plan.n_pad
    d = tempfile.mkdtemp(prefix="zero_ckpt_")
    try:
        t0 = time.perf_counter()
        checkpoint.save(opt, d)
        t1 = time.perf_counter()
        back = checkpoint.load(d, device=str(dev))
        torch.cuda.synchronize(dev)
        t2 = time.perf_counter()
        same = all(torch.equal(a, b) for a, b in ((opt.master, back.master),
                                                   (opt.exp_avg, back.exp_avg),
                                                   (opt.exp_avg_sq, back.exp_avg_sq),
                                                   (opt.params, back.params)))
        del back
        torch.cuda.empty_cache()
        w2 = max(1, wl.world // 2)
        t3 = time.perf_counter()
        resh = checkpoint.load(d, world_size=w2, device=str(dev))
        torch.cuda.synchronize(dev)
        t4 = time.perf_counter()
        n = opt.plan.n
        same_resh = torch.equal(resh.master[:n], opt.master[:n])
        del resh
    finally:
        shutil.rmtree(d, ignore_errors=True)
    return {"mode": "checkpoint", "workload": f"{wl.name}_w{wl.world}", "params": opt.plan.n,
            "state_bytes": state_bytes, "shards": wl.world,
            "save_s": t1 - t0, "save_gbs": state_bytes / (t1 - t0) / 1e9,
            "load_s": t2 - t1, "load_gbs": state_bytes / (t2 - t1) / 1e9,
            "resharded_load_world": w2, "resharded_load_s": t4 - t3,
            "round_trip_identical": bool(same), "resharded_identical": bool(same_resh),
            "timing": "host wall clock (perf_counter), device synchronised"}


# ---------------------------------------------------------------------------- oracle arm

def oracle_sample_run(wl, seconds: float, max_steps: int = 0, warmup: int = 0):
    """The CPU oracle, as it stands (single-threaded C), on a bounded sample of the
    workload: the first `n` elements of the first bucket, all W replicas, one step of
    reduce + sum of squares + finalize + AdamW/cast per iteration. Inputs are drawn
    before timing. Returns (params/s, sample description, steps, seconds)."""
    import numpy as np

    import oracle
    import synthgen

    n = min(1 << 24, wl.n)
    dt = wl.dtype_code
    grads = [synthgen.grads_host(0, n, wl.seed, r, wl.slot(1), wl.grad_sigma, wl.spike_frac,
                                 1.0, dt) for r in range(wl.world)]
    master = synthgen.master_random_host(0, n, wl.seed, wl.init_sigma)
    m = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32)
    R = np.zeros(n, np.float32)
    params = oracle.f32_to_half(master, dt)
    cfg, hp = oracle.workload_cfg(wl)
    st = oracle.state_init(cfg)
    # the oracle is single-threaded: pin the timed part to one host core
    prev_affinity = os.sched_getaffinity(0)
    core = min(prev_affinity)
    os.sched_setaffinity(0, {core})
    try:
        for _ in range(warmup):
            oracle.step(grads, dt, wl.bucket, R, master, m, v, params, dt, cfg, hp, st)
        steps = 0
        t0 = time.perf_counter()
        while True:
            oracle.step(grads, dt, wl.bucket, R, master, m, v, params, dt, cfg, hp, st)
            steps += 1
            el = time.perf_counter() - t0
            if (max_steps and steps >= max_steps) or (not max_steps and el >= seconds):
                break
    finally:
        os.sched_setaffinity(0, prev_affinity)
    desc = (f"{n} params ({wl.name} flat indices 0..{n - 1}), W={wl.world} {wl.gdtype} replicas, "
            f"{steps} full oracle steps (reduce, sum of squares, finalize, AdamW + cast), "
            f"pinned to host core {core}; params/s of the sample, not extrapolated")
    return n * steps / el, desc, steps, el


def run_reference(args, rank: int, world_size: int = 1):
    if rank != 0:
        return None
    import oracle
    wl = get_workload(args)
    pl = oracle.plan(wl.numels, wl.world, wl.bucket, wl.align)
    val, desc, steps, el = oracle_sample_run(wl, 0, max_steps=args.steps, warmup=args.warmup)
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": val,
        "unit": "params/s",
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": el / steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded Philox gradients and init)",
        "config": workload_config(wl, pl.n_buckets, pl.n_pad, world_size, max(1, args.micro)),
        "cpu_baseline": {"value": val, "unit": "params/s", "cores": 1, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": val, "unit": "params/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world_size = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        out = run_reference(args, rank, world_size)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    if args.zero3:
        print(json.dumps(run_zero3_forward(args, local_rank)), flush=True)
        return

    if args.checkpoint:
        print(json.dumps(run_checkpoint(args, local_rank)), flush=True)
        return

    if args.overlap:
        print(json.dumps(run_overlap(args, local_rank)), flush=True)
        return

    if args.sweep:
        import synthgen
        for log2n in [int(x) for x in args.sweep_log2n.split(",")]:
            for W in [int(x) for x in args.sweep_world.split(",")]:
                for dt in args.sweep_dtype.split(","):
                    wl = synthgen.sweep(log2n, W, dt)
                    print(json.dumps(run_sweep_point(wl, wl.steps, local_rank, args.resident)),
                          flush=True)
        return

    import torch
    import torch.distributed as dist
    if world_size > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    out = run_ours(args, rank, world_size, local_rank)
    wl = get_workload(args)
    if args.micro > 1:  # the end-to-end and oracle legs time the one-micro-batch step
        args.no_e2e = args.no_cpu_baseline = True
    if not args.no_e2e:
        e2e = run_e2e(args, wl, local_rank, world_size)  # every rank takes part
        if rank == 0:
            out["e2e"] = e2e
    if rank == 0:
        if not args.no_cpu_baseline and world_size == 1:
            val, desc, steps, el = oracle_sample_run(wl, args.cpu_seconds)
            out["cpu_baseline"] = {"value": val, "unit": "params/s", "cores": 1, "kind": "oracle",
                                   "sample": desc, "host_cpu_count": os.cpu_count()}
        print(json.dumps(out), flush=True)
    if world_size > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
