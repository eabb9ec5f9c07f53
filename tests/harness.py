"""Test harness: drives synthetic workloads through the CUDA library (C ABI via the
binding) and compares its outputs with the CPU oracle."""
from __future__ import annotations

import os
from typing import Callable, Optional

import numpy as np
import torch

import synthgen
from synthgen import device as sdev
import zero_sharded_mixed_replica_b200 as zb

HALF = {"bf16": torch.bfloat16, "fp16": torch.float16}


def stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def make_opt(wl) -> zb.ZeroOptimizer:
    scaler = zb.scaler_cfg(wl.dynamic, wl.init_scale_power, wl.loss_scale_window,
                           wl.hysteresis, wl.min_loss_scale)
    adamw = zb.adamw_cfg(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.max_grad_norm)
    return zb.ZeroOptimizer([t.shape for t in wl.tensors], wl.world, wl.bucket, wl.gdtype,
                            wl.align, scaler, adamw)


def first_scale(wl) -> float:
    return float(2.0 ** wl.init_scale_power) if wl.dynamic else 1.0


def run_resident(wl, steps: Optional[int] = None, on_step: Optional[Callable] = None):
    """Replica gradients resident over the whole padded space; every bucket reduced from
    them each step. Returns (optimizer, per-step results)."""
    opt = make_opt(wl)
    s = stream()
    sdev.init_master(wl, opt.master, s)
    opt.cast_params()
    n_pad = opt.plan.n_pad
    grads = [torch.zeros(n_pad, dtype=HALF[wl.gdtype], device="cuda") for _ in range(wl.world)]
    scale = first_scale(wl)
    results = []
    for t in range(1, (steps or wl.steps) + 1):
        sdev.fill_grads(wl, grads, 0, wl.n, t, scale, s)
        sdev.plant_infs(wl, grads, t)
        opt.full_step(grads)
        res = opt.result()
        results.append(res)
        scale = float(res["next_scale"]) if wl.dynamic else 1.0
        if on_step is not None:
            on_step(t, res, opt)
    return opt, results


def run_streaming(wl, steps: Optional[int] = None):
    """Replica buffers hold one bucket; two slots alternate by step."""
    opt = make_opt(wl)
    assert opt.plan.n == opt.plan.n_pad, "streaming inputs need an unpadded tensor list"
    s = stream()
    sdev.init_master(wl, opt.master, s)
    opt.cast_params()
    L = min(wl.bucket, opt.plan.n_pad)
    slots = [[torch.empty(L, dtype=HALF[wl.gdtype], device="cuda") for _ in range(wl.world)]
             for _ in range(2)]
    scale = first_scale(wl)
    results = []
    for t in range(1, (steps or wl.steps) + 1):
        bufs = slots[(t - 1) % 2]
        sdev.fill_grads(wl, bufs, 0, L, t, scale, s)
        sdev.plant_infs(wl, bufs, t, wl.bucket)
        for b in range(opt.plan.n_buckets):
            opt.reduce_scatter_bucket(b, bufs, base_offset=b * wl.bucket)
        opt.step()
        res = opt.result()
        results.append(res)
        scale = float(res["next_scale"]) if wl.dynamic else 1.0
    del slots
    return opt, results


# ----------------------------------------------------------------------------- checks

def to_np(x: torch.Tensor) -> np.ndarray:
    if x.dtype in (torch.bfloat16, torch.float16):
        return x.view(torch.int16).cpu().numpy().view(np.uint16)
    return x.cpu().numpy()


def half_ulp_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    def ordered(h):
        h = h.astype(np.int32)
        return np.where(h & 0x8000, -(h & 0x7FFF), h)
    return np.abs(ordered(a) - ordered(b))


# Per test and array: the fraction of bit-identical elements and the largest plain
# relative error |got - want| / |want| (over want != 0), written out at the end of the
# session when ZERO_PARITY_REPORT names a file (see conftest.py).
REPORT: dict = {}


def record(name: str, got: np.ndarray, want: np.ndarray, ulp: Optional[np.ndarray] = None):
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    entry = {"elements": int(want.size)}
    if ulp is not None:
        entry["identical"] = float(np.mean(ulp == 0)) if ulp.size else 1.0
        entry["max_ulp"] = int(ulp.max()) if ulp.size else 0
    else:
        same = got.view(np.uint32) == want.view(np.uint32) \
            if got.dtype == want.dtype == np.float32 else got == want
        entry["identical"] = float(np.mean(same)) if want.size else 1.0
        w = want.astype(np.float64)
        nz = w != 0
        rel = np.abs(got.astype(np.float64)[nz] - w[nz]) / np.abs(w[nz])
        entry["max_rel"] = float(rel.max()) if rel.size else 0.0
    cases = REPORT.setdefault(test, {})
    key, i = name, 1
    while key in cases:  # the same array checked again later in the test
        i += 1
        key = f"{name}#{i}"
    cases[key] = entry


def check_state(name: str, got: np.ndarray, want: np.ndarray, world: int) -> float:
    """fp32 state criterion: |got - want| <= 1e-6 * max(|want|, rms of want over the
    rank's partition). Returns the fraction of bit-identical elements."""
    record(name, got, want)
    assert got.shape == want.shape
    n = want.size
    p = n // world if world and n % world == 0 else n
    w64 = want.astype(np.float64).reshape(-1, p) if p else want.astype(np.float64)
    rms = np.sqrt(np.mean(w64 ** 2, axis=1, keepdims=True)) if p else 0.0
    floor = np.broadcast_to(rms, w64.shape).reshape(-1) if p else 0.0
    err = np.abs(got.astype(np.float64) - want.astype(np.float64)) / \
        np.maximum(np.abs(want.astype(np.float64)), np.maximum(floor, 1e-300))
    worst = float(err.max()) if n else 0.0
    assert worst <= 1e-6, f"{name}: max relative error {worst:.3e} > 1e-6"
    return float(np.mean(got.view(np.uint32) == want.view(np.uint32))) if n else 1.0


def check_scalars(res: dict, sc: dict, exact_k: bool = False) -> None:
    for key in ("overflow", "skipped", "hysteresis", "iter", "adam_t"):
        assert res[key] == sc[key], (key, res[key], sc[key])
    assert res["scale_used"] == sc["scale_used"] and res["next_scale"] == sc["next_scale"]
    if not sc["overflow"]:
        assert abs(res["global_norm"] - sc["norm"]) <= 1e-5 * abs(sc["norm"]), \
            (res["global_norm"], sc["norm"])
        assert abs(res["clip_coef"] - sc["clip_coef"]) <= 2e-7 * abs(sc["clip_coef"])
        if exact_k:
            assert res["k"] == sc["k"]


def check_all(opt: zb.ZeroOptimizer, ref: dict, world: int) -> dict:
    """R bit-exact, fp32 state within tolerance, params within 1 ulp."""
    R = to_np(opt.reduced)
    record("R", R, ref["R"])
    assert np.array_equal(R.view(np.uint32), ref["R"].view(np.uint32)), \
        f"reduced gradient: {np.sum(R.view(np.uint32) != ref['R'].view(np.uint32))} elements differ"
    same = {}
    for name, t in (("master", opt.master), ("m", opt.exp_avg), ("v", opt.exp_avg_sq)):
        same[name] = check_state(name, to_np(t), ref[name], world)
    d = half_ulp_distance(to_np(opt.params), ref["params"])
    record("params", None, ref["params"], ulp=d)
    assert d.max(initial=0) <= 1, f"params: max ulp distance {d.max()}"
    same["params"] = float(np.mean(d == 0)) if d.size else 1.0
    return same
