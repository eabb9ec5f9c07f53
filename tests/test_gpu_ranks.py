"""The rank-local entry points (zero_reduce_scatter_segment, zero_step_local_sumsq,
zero_step_finalize_ranks, zero_step_update_partition) on one GPU: the W ranks of a
multi-process run are played one after another in one process and one stream (no
kernel waits on another), each with its own plan, workspace and partition buffers; the
update writes every rank's half values into all W gathered buffers, as the fused
all-gather does over NVLink. Results must equal the CPU oracle's whole-model step."""
import numpy as np
import pytest
import torch

import oracle
import synthgen
from synthgen import device as sdev
import zero_sharded_mixed_replica_b200 as zb

from harness import HALF, check_scalars, check_state, half_ulp_distance, stream, to_np

pytestmark = pytest.mark.gpu


def _wl(shapes, W, bucket, align, dtype, dynamic, steps):
    t = [synthgen.TensorSpec(f"t{i}", s, "normal" if i % 2 == 0 else "ones")
         for i, s in enumerate(shapes)]
    return synthgen.Workload("ranks", t, world=W, bucket=bucket, steps=steps, gdtype=dtype,
                             dynamic=dynamic, align=align, grad_sigma=3e-2,
                             inf_sites={2: 1} if dynamic else {})


CASES = [
    ([(100003,), (77, 5)], 2, 30000, 8, "bf16", False, 3),
    ([(1 << 18,), (4097,)], 4, 50000, 128, "fp16", True, 4),
    ([(6000,), (3, 3)], 8, 1001, 1, "bf16", False, 3),
]


@pytest.mark.parametrize("case", CASES, ids=["w2", "w4_fp16", "w8_ragged"])
def test_rank_local_calls_match_oracle(case):
    wl = _wl(*case)
    W = wl.world
    s = stream()
    scaler = zb.scaler_cfg(wl.dynamic, wl.init_scale_power, wl.loss_scale_window,
                           wl.hysteresis, wl.min_loss_scale)
    adamw = zb.adamw_cfg(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.max_grad_norm)
    plans = [zb.Plan([t.shape for t in wl.tensors], W, wl.bucket, wl.align) for _ in range(W)]
    n_pad, p = plans[0].n_pad, plans[0].p
    half = HALF[wl.gdtype]
    master_full = torch.zeros(n_pad, dtype=torch.float32, device="cuda")
    sdev.init_master(wl, master_full, s)
    gathered = [torch.zeros(n_pad, dtype=half, device="cuda") for _ in range(W)]
    init_opt = zb.ZeroOptimizer([t.shape for t in wl.tensors], W, wl.bucket, wl.gdtype, wl.align)
    init_opt.master.copy_(master_full)
    init_opt.cast_params()
    for g in gathered:
        g.copy_(init_opt.params)
    ranks = []
    for r in range(W):
        f32 = dict(dtype=torch.float32, device="cuda")
        rk = dict(plan=plans[r], master=master_full[r * p:(r + 1) * p].clone(),
                  m=torch.zeros(p, **f32), v=torch.zeros(p, **f32), R=torch.zeros(p, **f32),
                  ws=torch.zeros(plans[r].workspace_bytes(), dtype=torch.uint8, device="cuda"))
        zb.zero_state_init(rk["plan"], rk["ws"], scaler, s)
        ranks.append(rk)
    grads = [torch.zeros(n_pad, dtype=half, device="cuda") for _ in range(W)]
    s_all = torch.zeros(W, dtype=torch.float64, device="cuda")
    scale = float(2.0 ** wl.init_scale_power) if wl.dynamic else 1.0
    ref = oracle.run_resident(wl)
    from zero_sharded_mixed_replica_b200.distributed import partition_buckets
    for t in range(1, wl.steps + 1):
        sdev.fill_grads(wl, grads, 0, wl.n, t, scale, s)
        sdev.plant_infs(wl, grads, t)
        for r, rk in enumerate(ranks):
            for b in partition_buckets(n_pad, W, wl.bucket, r):
                zb.zero_reduce_scatter_segment(rk["plan"], b, r, wl.gdtype, grads, 0, rk["R"],
                                               rk["ws"], s)
            zb.zero_step_local_sumsq(rk["plan"], r, rk["ws"], s_all[r:r + 1], s)
        results = []
        for r, rk in enumerate(ranks):
            zb.zero_step_finalize_ranks(rk["plan"], adamw, s_all, rk["ws"], s)
            zb.zero_step_update_partition(rk["plan"], r, rk["master"], rk["m"], rk["v"], rk["R"],
                                          [g[r * p:] for g in gathered], wl.gdtype, rk["ws"], s)
            results.append(zb.zero_get_result(rk["ws"], s))
        sc = ref["scalars"][t - 1] if t == wl.steps else None
        # every rank decided the same
        for res in results[1:]:
            for k in ("global_norm", "k", "skipped", "scale_used", "next_scale", "adam_t"):
                assert res[k] == results[0][k], k
        scale = float(results[0]["next_scale"]) if wl.dynamic else 1.0
        if sc is not None:
            check_scalars(results[0], sc)
    if wl.dynamic:
        assert [r["skipped"] for r in ref["scalars"]] == [0, 1, 0, 0]
    for r, rk in enumerate(ranks):
        sl = slice(r * p, (r + 1) * p)
        assert np.array_equal(to_np(rk["R"]).view(np.uint32), ref["R"][sl].view(np.uint32))
        for name in ("master", "m", "v"):
            check_state(name, to_np(rk[name]), ref[name][sl], 1)
    for g in gathered:
        assert half_ulp_distance(to_np(g), ref["params"]).max() <= 1


def test_rank_calls_out_of_order():
    plan = zb.Plan([(10000,)], 2, 3000)
    ws = torch.zeros(plan.workspace_bytes(), dtype=torch.uint8, device="cuda")
    zb.zero_state_init(plan, ws, zb.scaler_cfg(False))
    g = [torch.zeros(plan.n_pad, dtype=torch.bfloat16, device="cuda")] * 2
    R = torch.zeros(plan.p, dtype=torch.float32, device="cuda")
    out = torch.zeros(1, dtype=torch.float64, device="cuda")
    with pytest.raises(zb.ZeroError) as e:  # bucket 3 lies in rank 1's partition only
        zb.zero_reduce_scatter_segment(plan, 3, 0, "bf16", g, 0, R, ws)
    assert e.value.code == zb.ZERO_EINVAL
    with pytest.raises(zb.ZeroError) as e:  # sum before the segments are reduced
        zb.zero_step_local_sumsq(plan, 0, ws, out)
    assert e.value.code == zb.ZERO_ESTATE
    zb.zero_reduce_scatter_segment(plan, 0, 0, "bf16", g, 0, R, ws)
    with pytest.raises(zb.ZeroError) as e:
        zb.zero_reduce_scatter_segment(plan, 0, 0, "bf16", g, 0, R, ws)
    assert e.value.code == zb.ZERO_ESTATE
    zb.zero_reduce_scatter_segment(plan, 1, 0, "bf16", g, 0, R, ws)
    zb.zero_step_local_sumsq(plan, 0, ws, out)
    s_all = torch.zeros(2, dtype=torch.float64, device="cuda")
    zb.zero_step_finalize_ranks(plan, zb.adamw_cfg(), s_all, ws)
    assert zb.zero_get_result(ws)["adam_t"] == 1
