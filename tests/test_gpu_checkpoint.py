"""Checkpoints of the device optimizer through the C ABI: save after two steps, reload
(same W, then another W), continue, and compare with the uninterrupted run / the
oracle."""
import numpy as np
import pytest
import torch

import oracle
import synthgen
from synthgen import device as sdev
from zero_sharded_mixed_replica_b200 import checkpoint as ck

from harness import HALF, check_all, run_resident, stream

pytestmark = pytest.mark.gpu


def _wl(world=4):
    t = synthgen.TensorSpec
    return synthgen.Workload("ck", [t("a", (50000,), "normal"), t("b", (33, 7), "ones"),
                                    t("c", (9999,), "normal")], world=world, bucket=15000,
                             steps=4, gdtype="fp16", dynamic=True, align=8, grad_sigma=3e-2,
                             inf_sites={2: 1})


def _continue(opt, wl, steps, first_t):
    s = stream()
    grads = [torch.zeros(opt.plan.n_pad, dtype=HALF[wl.gdtype], device="cuda")
             for _ in range(wl.world)]
    scale = float(opt.result()["next_scale"])
    for t in range(first_t, first_t + steps):
        sdev.fill_grads(wl, grads, 0, wl.n, t, scale, s)
        sdev.plant_infs(wl, grads, t)
        opt.full_step(grads)
        scale = float(opt.result()["next_scale"])


def test_save_load_continue_bit_exact(tmp_path):
    wl = _wl()
    full, _ = run_resident(wl, steps=4)
    two, _ = run_resident(wl, steps=2)
    ck.save(two, str(tmp_path))
    back = ck.load(str(tmp_path))
    for a, b in ((back.master, two.master), (back.exp_avg, two.exp_avg),
                 (back.exp_avg_sq, two.exp_avg_sq), (back.params, two.params)):
        assert torch.equal(a, b)
    _continue(back, wl, 2, 3)
    for a, b in ((back.master, full.master), (back.exp_avg, full.exp_avg),
                 (back.exp_avg_sq, full.exp_avg_sq), (back.params, full.params)):
        assert torch.equal(a, b)
    ra, rb = back.result(), full.result()
    for k in ("adam_t", "iter", "next_scale", "hysteresis", "global_norm"):
        assert ra[k] == rb[k], k


def test_reshard_8_to_4_then_step_matches_oracle(tmp_path):
    wl8 = _wl(8)
    two, _ = run_resident(wl8, steps=2)
    ck.save(two, str(tmp_path))
    back = ck.load(str(tmp_path), world_size=4)
    n = wl8.n
    assert back.plan.world_size == 4
    assert torch.equal(back.master[:n], two.master[:n]) and not back.master[n:].any()
    # one more step with W = 4 replicas, against the oracle started from the same state
    wl4 = _wl(4)
    meta, master, m, v = ck.load_flat(str(tmp_path))
    pl = oracle.plan(wl4.numels, 4, wl4.bucket, wl4.align)
    cfg, hp = oracle.workload_cfg(wl4)
    st = oracle.State(**meta["scaler_state"])
    master, m, v = (ck.place(a, pl.n_pad) for a in (master, m, v))
    params = oracle.f32_to_half(master, wl4.dtype_code)
    R = np.zeros(pl.n_pad, np.float32)
    g = oracle.resident_grads(wl4, pl.n_pad, 3, oracle.step_grad_scale(wl4, st))
    oracle.step(g, wl4.dtype_code, wl4.bucket, R, master, m, v, params, wl4.dtype_code,
                cfg, hp, st)
    _continue(back, wl4, 1, 3)
    check_all(back, dict(R=R, master=master, m=m, v=v, params=params), 4)
