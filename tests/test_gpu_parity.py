"""Parity of the CUDA path (through the C ABI) with the CPU oracle on the same seeded
inputs: every workload, edge shapes, overflow cases, the loss scaler, the auxiliary
calls. Integer / flag state bit-exact; fp32 master, m, v within 1e-6 relative (floor:
rms of the rank's partition); global norm within 1e-5 relative; half params within
1 ulp; reduced gradient bit-exact."""
import gc
import math

import numpy as np
import pytest
import torch

import oracle
import synthgen
from synthgen import device as sdev
import zero_sharded_mixed_replica_b200 as zb

from harness import (HALF, check_all, check_scalars, check_state, half_ulp_distance, record,
                     make_opt, run_resident, run_streaming, stream, to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _free_memory():
    yield
    gc.collect()
    torch.cuda.empty_cache()


# ----------------------------------------------------------------------------- inputs

def test_device_inputs_match_host_inputs():
    n = (1 << 20) + 13
    for dt, spike, scale in (("bf16", 0.001, 1.0), ("fp16", 0.0, 65536.0), ("bf16", 0.0, 1.0)):
        buf = torch.empty(n, dtype=HALF[dt], device="cuda")
        synthgen.grads_cuda(buf.data_ptr(), 7, n, 0, 3, 2, 1e-3, spike, scale,
                            synthgen.DTYPE_CODE[dt], stream())
        host = synthgen.grads_host(7, n, 0, 3, 2, 1e-3, spike, scale, synthgen.DTYPE_CODE[dt])
        assert np.array_equal(to_np(buf), host)
    m = torch.empty(n, dtype=torch.float32, device="cuda")
    synthgen.master_random_cuda(m.data_ptr(), 5, n, 0, 0.02, stream())
    assert np.array_equal(to_np(m), synthgen.master_random_host(5, n, 0, 0.02))


# ----------------------------------------------------------------------------- workloads

def _per_step_oracle(wl):
    snaps = []

    def keep(t, sc, R, master, m, v, params):
        snaps.append(dict(R=R.copy(), master=master.copy(), m=m.copy(), v=v.copy(),
                          params=params.copy()))
    ref = oracle.run_resident(wl, on_step=keep)
    return ref, snaps


def test_tiny_parity_every_step():
    wl = synthgen.workload("tiny")
    ref, snaps = _per_step_oracle(wl)
    same = []

    def on_step(t, res, opt):
        check_scalars(res, ref["scalars"][t - 1], exact_k=True)
        same.append(check_all(opt, snaps[t - 1], wl.world))
    run_resident(wl, on_step=on_step)
    assert len(same) == wl.steps
    # every config clips: norm ~1.45 for tiny
    assert all(s["norm"] > 1.0 for s in ref["scalars"])
    # the operation order is the same on both sides: expect bit-identical state
    assert all(v == 1.0 for s in same for v in s.values()), same


def test_encoder_layer_fp16_dynamic_scaler():
    wl = synthgen.workload("enc")
    ref = oracle.run_resident(wl)
    opt, results = run_resident(wl)
    for res, sc in zip(results, ref["scalars"]):
        check_scalars(res, sc)
    # hand-derived trace: +inf at steps 3 and 7; the first spends the hysteresis
    # budget, the second halves the scale; 8 steps applied.
    assert [r["scale_used"] for r in results] == [65536.0] * 7 + [32768.0] * 3
    assert [r["skipped"] for r in results] == [0, 0, 1, 0, 0, 0, 1, 0, 0, 0]
    assert results[-1]["adam_t"] == 8 and results[-1]["next_scale"] == 32768.0
    check_all(opt, ref, wl.world)


def test_gpt2_medium_w8_two_buckets():
    wl = synthgen.workload("gpt2")
    ref = oracle.run_resident(wl)
    opt, results = run_resident(wl)
    for res, sc in zip(results, ref["scalars"]):
        check_scalars(res, sc)
        assert sc["clip_coef"] < 1.0  # x8 spikes make every step clip
    same = check_all(opt, ref, wl.world)
    if all(r["k"] == s["k"] for r, s in zip(results, ref["scalars"])):
        # same multiplier and the same operation order on both sides: bit-identical
        assert all(v == 1.0 for v in same.values()), same


def test_llama7b_w8_streaming_full_size_sampled():
    """The 7B-shaped W=8 workload at full size, in the launch configuration the
    benchmark times (14 buckets of 5e8, bucket-sized replica buffers). The oracle
    computes every step's scalars from the full gradient stream and the update of
    sampled elements one by one."""
    wl = synthgen.workload("llama7b")
    scalars = oracle.streaming_scalars(wl)
    opt, results = run_streaming(wl)
    for res, sc in zip(results, scalars):
        check_scalars(res, sc.as_dict())
    pl = opt.plan
    rng = np.random.default_rng(11)
    idx = np.unique(np.concatenate([
        rng.integers(0, pl.n_pad, 4096),
        [0, 1, pl.n_pad - 1, pl.n_pad - 8],
        [r * pl.p + d for r in range(1, wl.world) for d in (-1, 0)],
        [b * wl.bucket + d for b in range(1, pl.n_buckets) for d in (-1, 0)],
    ]).astype(np.int64))
    want = oracle.streaming_samples(wl, idx, scalars)
    it = torch.from_numpy(idx).cuda()
    got_R = opt.reduced[it].cpu().numpy()
    record("R (sampled)", got_R, want["R"])
    assert np.array_equal(got_R.view(np.uint32), want["R"].view(np.uint32))
    for name, t in (("master", opt.master), ("m", opt.exp_avg), ("v", opt.exp_avg_sq)):
        g = t[it].cpu().numpy()
        record(name + " (sampled)", g, want[name])
        w = want[name].astype(np.float64)
        floor = np.sqrt(np.mean(w ** 2))
        err = np.abs(g - w) / np.maximum(np.abs(w), floor)
        assert err.max() <= 1e-6, (name, err.max())
    d = half_ulp_distance(to_np(opt.params[it]), want["params"])
    record("params (sampled)", None, want["params"], ulp=d)
    assert d.max() <= 1
    # the padding-free 7B list: invariants over the whole buffer
    assert torch.isfinite(opt.master).all().item()
    del opt


# ----------------------------------------------------------------------------- edge shapes

EDGE = [
    # (shapes, W, bucket, align, dtype, dynamic)
    ([(1000,), (3, 7), (1,), ()], 3, 37, 1, "bf16", False),        # ragged, odd W, odd buckets
    ([(4097,), (129, 3)], 16, 1001, 128, "fp16", True),             # W=16, padding, bucket % 8 != 0
    ([(2048, 3)], 1, 1 << 20, 128, "bf16", False),                  # W=1, one bucket
    ([(5,), (0, 9), (7, 1)], 4, 8, 2, "fp16", False),               # empty tensor, tiny buckets
    ([(300001,)], 5, 65536, 8, "bf16", False),                      # several full buckets + tail
    ([(1 << 16,)], 8, 1 << 13, 128, "bf16", False),                 # buckets = partitions / 1
]


def _edge_workload(shapes, W, bucket, align, dtype, dynamic, steps=3):
    tensors = [synthgen.TensorSpec(f"t{i}", s, "normal" if i % 2 == 0 else "ones")
               for i, s in enumerate(shapes)]
    return synthgen.Workload("edge", tensors, world=W, bucket=bucket, steps=steps, gdtype=dtype,
                             dynamic=dynamic, align=align, grad_sigma=3e-2,
                             inf_sites={2: 1} if dynamic else {})


@pytest.mark.parametrize("case", EDGE, ids=[f"edge{i}" for i in range(len(EDGE))])
def test_edge_shapes(case):
    wl = _edge_workload(*case)
    ref = oracle.run_resident(wl)
    opt, results = run_resident(wl)
    for res, sc in zip(results, ref["scalars"]):
        check_scalars(res, sc)
    check_all(opt, ref, wl.world)
    # padding stays exactly zero everywhere
    n = opt.plan.n
    for t in (opt.master, opt.exp_avg, opt.exp_avg_sq, opt.reduced):
        assert not t[n:].any().item()
    assert not opt.params[n:].view(torch.int16).any().item()


def test_empty_plan_step():
    opt = zb.ZeroOptimizer([], 4, 100)
    opt.step()
    res = opt.result()
    assert res["global_norm"] == 0.0 and res["adam_t"] == 1 and res["skipped"] == 0


def test_streaming_matches_resident_inputs():
    """Bucket-sized replica buffers with base offset = bucket start give the same
    reduced gradient as whole-model buffers holding the same values."""
    wl = synthgen.sweep(18, 4, "bf16", steps=1)
    wl.bucket = 40000
    opt_s, res_s = run_streaming(wl, steps=1)
    opt_r = make_opt(wl)
    s = stream()
    sdev.init_master(wl, opt_r.master, s)
    opt_r.cast_params()
    n = opt_r.plan.n_pad
    full = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(wl.world)]
    for b in range(opt_r.plan.n_buckets):
        st, ln = opt_r.plan.bucket(b)
        for r in range(wl.world):
            synthgen.grads_cuda(full[r].data_ptr() + 2 * st, 0, ln, wl.seed, r, wl.slot(1),
                                wl.grad_sigma, 0.0, 1.0, 0, s)
    opt_r.full_step(full)
    res_r = opt_r.result()
    assert torch.equal(opt_s.reduced, opt_r.reduced)
    assert res_s[0]["global_norm"] == res_r["global_norm"]
    assert torch.equal(opt_s.master, opt_r.master)


# ----------------------------------------------------------------------------- invariance

def test_partition_invariance_across_world_sizes():
    """Replicas RNE(g/W) for W in {1,2,4,8}: W equal bf16 copies sum exactly in fp32, so
    the reduced gradient is g for every W and every output must be bit-identical."""
    n = 1 << 20
    g = synthgen.grads_host(0, n, 0, 0, 1, 1e-3, 0.0, 1.0, synthgen.BF16)
    g32 = oracle.half_to_f32(g, oracle.BF16)
    outs = []
    for W in (1, 2, 4, 8):
        opt = zb.ZeroOptimizer([(n,)], W, 1 << 18)
        sdev.init_master(synthgen.Workload("inv", [synthgen.TensorSpec("w", (n,), "normal")],
                                           world=W, bucket=1 << 18, steps=1), opt.master, stream())
        opt.cast_params()
        part = torch.from_numpy(g32 / W).cuda().to(torch.bfloat16)
        assert torch.equal(part.float() * W, torch.from_numpy(g32).cuda())
        for _ in range(2):
            opt.full_step([part] * W)
        res = opt.result()
        outs.append((res, [to_np(t).copy() for t in (opt.reduced, opt.master, opt.exp_avg,
                                                      opt.exp_avg_sq, opt.params)]))
    ref_res, ref_arrs = outs[0]
    for res, arrs in outs[1:]:
        assert res["k"] == ref_res["k"]
        assert abs(res["global_norm"] - ref_res["global_norm"]) <= 1e-12 * ref_res["global_norm"]
        for a, b in zip(arrs, ref_arrs):
            assert np.array_equal(a.view(np.uint8), b.view(np.uint8))


# ----------------------------------------------------------------------------- overflow

@pytest.mark.parametrize("kind", ["+inf", "-inf", "nan", "inf-inf"])
def test_overflow_skips_step_and_moves_scaler(kind):
    n = 4096
    wl = synthgen.Workload("ovf", [synthgen.TensorSpec("w", (n,), "normal")], world=2,
                           bucket=1000, steps=1, gdtype="fp16", dynamic=True)
    opt = make_opt(wl)
    sdev.init_master(wl, opt.master, stream())
    opt.cast_params()
    g = [torch.full((n,), 0.25, dtype=torch.float16, device="cuda") for _ in range(2)]
    opt.full_step(g)  # one good step so m, v are non-zero
    before = [t.clone() for t in (opt.master, opt.exp_avg, opt.exp_avg_sq, opt.params)]
    vals = {"+inf": (math.inf, 0.0), "-inf": (-math.inf, 1.0), "nan": (math.nan, 0.0),
            "inf-inf": (math.inf, -math.inf)}[kind]
    g[0][1234] = vals[0]
    g[1][1234] = vals[1]
    opt.full_step(g)
    res = opt.result()
    assert res["overflow"] == 1 and res["skipped"] == 1 and res["adam_t"] == 1
    assert res["hysteresis"] == 1 and res["next_scale"] == 65536.0
    for a, b in zip(before, (opt.master, opt.exp_avg, opt.exp_avg_sq, opt.params)):
        assert torch.equal(a, b)
    opt.full_step(g)  # second overflow in a row halves the scale
    assert opt.result()["next_scale"] == 32768.0


def test_scaler_all_flag_sequences_match_oracle():
    """Every overflow-flag sequence of length 10 (so every shorter one as a prefix), on
    a short window so growth and hysteresis refills happen, device vs oracle."""
    n, L = 1024, 10
    cfg_o = oracle.scaler_cfg(True, 4, 3, 2, 1.0)
    hp = oracle.hparams()
    opt = zb.ZeroOptimizer([(n,)], 1, 1 << 20, "fp16",
                           scaler=zb.scaler_cfg(True, 4, 3, 2, 1.0))
    good = torch.full((n,), 2.0 ** -6, dtype=torch.float16, device="cuda")
    bad = good.clone()
    bad[17] = math.inf
    S_good = n * (2.0 ** -6) ** 2
    for code in range(1 << L):
        zb.zero_state_init(opt.plan, opt.workspace, zb.scaler_cfg(True, 4, 3, 2, 1.0))
        st = oracle.state_init(cfg_o)
        for i in range(L):
            f = (code >> i) & 1
            opt.full_step([bad if f else good])
            res = opt.result()
            sc = oracle.finalize(math.inf if f else S_good, bool(f), cfg_o, hp, st).as_dict()
            check_scalars(res, sc, exact_k=True)


# ----------------------------------------------------------------------------- aux calls

@pytest.mark.parametrize("dt", ["bf16", "fp16"])
def test_cast_params_matches_oracle(dt):
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.normal(0, 0.02, 100000), rng.normal(0, 1e4, 1000),
                        [65504, 65520, 1e-8, -0.0, 3.4e38, 1e-40]]).astype(np.float32)
    pad = (-x.size) % 8
    x = np.concatenate([x, np.zeros(pad + 3, np.float32)])
    opt = zb.ZeroOptimizer([(x.size,)], 1, 1 << 30, dt, align=1)
    opt.master.copy_(torch.from_numpy(x).cuda())
    opt.cast_params()
    assert np.array_equal(to_np(opt.params), oracle.f32_to_half(x, synthgen.DTYPE_CODE[dt]))


def test_all_gather_replicas():
    opt = zb.ZeroOptimizer([(12345,)], 3, 4000, align=1)
    opt.params.copy_(torch.randn(opt.plan.n_pad, device="cuda").to(torch.bfloat16))
    dst = [torch.zeros_like(opt.params) for _ in range(19)]  # more than one launch batch
    opt.all_gather(dst)
    for d in dst:
        assert torch.equal(d.view(torch.int16), opt.params.view(torch.int16))
    opt.all_gather([])  # canonical buffer only: a no-op


def test_host_staging_path_equals_device_path():
    wl = synthgen.sweep(20, 4, "bf16", steps=1)
    wl.bucket = 300000
    n = wl.n
    host = [torch.from_numpy(synthgen.grads_host(0, n, 0, r, 1, 1e-3, 0.0, 1.0, 0)
                             .view(np.int16)).pin_memory() for r in range(4)]
    dev = [h.cuda().view(torch.bfloat16) for h in host]
    a, b = make_opt(wl), make_opt(wl)
    staging = [torch.empty(wl.bucket, dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    for bk in range(a.plan.n_buckets):
        a.reduce_scatter_bucket(bk, dev, 0)
        b.reduce_scatter_bucket_host(bk, [h.data_ptr() for h in host], 0, staging)
    a.step()
    b.step()
    assert torch.equal(a.reduced, b.reduced)
    assert a.result()["global_norm"] == b.result()["global_norm"]


def test_out_of_order_calls_are_rejected():
    opt = zb.ZeroOptimizer([(10000,)], 2, 3000)
    g = [torch.zeros(opt.plan.n_pad, dtype=torch.bfloat16, device="cuda")] * 2
    opt.reduce_scatter_bucket(0, g)
    with pytest.raises(zb.ZeroError) as e:
        opt.reduce_scatter_bucket(0, g)
    assert e.value.code == zb.ZERO_ESTATE
    with pytest.raises(zb.ZeroError) as e:
        opt.step()
    assert e.value.code == zb.ZERO_ESTATE
    for b in range(1, opt.plan.n_buckets):
        opt.reduce_scatter_bucket(b, g)
    opt.step()
    assert opt.result()["adam_t"] == 1


def test_guard_regions_untouched():
    """Buffers that are views of larger allocations: nothing past n_pad is written."""
    wl = _edge_workload([(777,), (33,)], 3, 100, 8, "bf16", False, steps=2)
    opt = make_opt(wl)
    n = opt.plan.n_pad
    big = {k: torch.full((n + 64,), 7.0, device="cuda")
           for k in ("master", "exp_avg", "exp_avg_sq", "reduced")}
    for k, t in big.items():
        setattr(opt, k, t[:n])
    opt.master.zero_()
    opt.exp_avg.zero_()
    opt.exp_avg_sq.zero_()
    pbig = torch.full((n + 64,), 3.0, dtype=torch.bfloat16, device="cuda")
    opt.params = pbig[:n]
    g = [torch.ones(n + 64, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    for _ in range(2):
        opt.full_step([x[:n] for x in g])
    opt.result()
    for t in big.values():
        assert torch.all(t[n:] == 7.0)
    assert torch.all(pbig[n:] == 3.0)


# ----------------------------------------------------------------------------- sweep

def _check_streaming(wl, idx=None, steps=None):
    scalars = oracle.streaming_scalars(wl, steps=steps)
    opt, results = run_streaming(wl, steps=steps)
    for res, sc in zip(results, scalars):
        check_scalars(res, sc.as_dict())
    if idx is None:
        idx = np.arange(opt.plan.n_pad, dtype=np.int64)
    want = oracle.streaming_samples(wl, idx, scalars)
    it = torch.from_numpy(idx).cuda()
    assert np.array_equal(opt.reduced[it].cpu().numpy().view(np.uint32), want["R"].view(np.uint32))
    for name, t in (("master", opt.master), ("m", opt.exp_avg), ("v", opt.exp_avg_sq)):
        check_state(name, t[it].cpu().numpy(), want[name], 1)
    assert half_ulp_distance(to_np(opt.params[it]), want["params"]).max() <= 1
    return results


@pytest.mark.parametrize("world", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_sweep_2_24_every_element(world, dtype):
    """Every 2^24 sweep point (W in {1, 2, 4, 8, 16} x {bf16, fp16}), 10 steps (fp16:
    dynamic scaler with one +inf at step 5), every element compared."""
    wl = synthgen.sweep(24, world, dtype)
    results = _check_streaming(wl)
    if dtype == "fp16":
        assert [r["skipped"] for r in results] == [0, 0, 0, 0, 1, 0, 0, 0, 0, 0]
        assert results[-1]["adam_t"] == 9


def test_sweep_2_30_w16_sampled():
    """The largest sweep point (2^30 params, W=16, 6 buckets of 2e8), 3 steps,
    scalars from the full gradient stream and ~4k sampled elements."""
    wl = synthgen.sweep(30, 16, "bf16", steps=3)
    rng = np.random.default_rng(5)
    n = wl.n
    idx = np.unique(np.concatenate([rng.integers(0, n, 4096), [0, n - 1],
                                    [b * wl.bucket + d for b in range(1, 6) for d in (-1, 0)],
                                    [r * (n // 16) + d for r in range(1, 16) for d in (-1, 0)]]))
    _check_streaming(wl, idx.astype(np.int64))


# ----------------------------------------------------------------------------- accumulation

@pytest.mark.parametrize("dtype,W,M", [("bf16", 8, 4), ("fp16", 4, 3)])
def test_gradient_accumulation(dtype, W, M):
    """M micro-batches per step, reduced bucket by bucket in micro-major order and
    accumulated in the fp32 reduced gradient; fp16 with a +inf in step 2's last
    micro-batch (the whole step is skipped)."""
    t = synthgen.TensorSpec
    wl = synthgen.Workload("accum", [t("a", (300007,), "normal"), t("b", (64, 33), "ones")],
                           world=W, bucket=100000, steps=3, gdtype=dtype,
                           dynamic=dtype == "fp16", align=8, grad_sigma=1e-2,
                           inf_sites={2: 1} if dtype == "fp16" else {}, micro_batches=M)
    ref = oracle.run_resident(wl)
    opt = make_opt(wl)
    s = stream()
    sdev.init_master(wl, opt.master, s)
    opt.cast_params()
    n_pad = opt.plan.n_pad
    grads = [torch.zeros(n_pad, dtype=HALF[dtype], device="cuda") for _ in range(W)]
    scale = float(2.0 ** wl.init_scale_power) if wl.dynamic else 1.0
    for step in range(1, wl.steps + 1):
        for k in range(M):
            sdev.fill_grads(wl, grads, 0, wl.n, step, scale, s, micro=k)
            if k == M - 1:
                sdev.plant_infs(wl, grads, step)
            for b in range(opt.plan.n_buckets):
                opt.reduce_scatter_bucket_accum(b, k, M, grads)
        opt.step()
        res = opt.result()
        check_scalars(res, ref["scalars"][step - 1])
        scale = float(res["next_scale"]) if wl.dynamic else 1.0
    if dtype == "fp16":
        assert [s_["skipped"] for s_ in ref["scalars"]] == [0, 1, 0]
    check_all(opt, ref, W)
    # out of order: micro-batch 1 before 0
    with pytest.raises(zb.ZeroError) as e:
        opt.reduce_scatter_bucket_accum(0, 1, M, grads)
    assert e.value.code == zb.ZERO_ESTATE


# ----------------------------------------------------------------------------- bounded waits

def test_bounded_wait_gives_up_and_reports():
    """A wait that nothing completes ends after about a second with the sticky error
    flag set; zero_get_result reports ZERO_EDEVICE, the context stays usable, and a
    state re-initialisation clears the flag."""
    import time
    opt = zb.ZeroOptimizer([(4096,)], 2, 4096)
    t0 = time.perf_counter()
    zb.zero_selftest_bounded_wait(opt.workspace)
    with pytest.raises(zb.ZeroError) as e:
        opt.result()
    assert e.value.code == zb.ZERO_EDEVICE
    assert 0.5 < time.perf_counter() - t0 < 30
    zb.zero_state_init(opt.plan, opt.workspace, opt.scaler)
    g = [torch.zeros(opt.plan.n_pad, dtype=torch.bfloat16, device="cuda")] * 2
    opt.full_step(g)
    assert opt.result()["device_error"] == 0


# ----------------------------------------------------------------------------- CUDA graphs

def test_captured_step_replays_like_eager_steps():
    """A CUDA graph of one step, replayed 4 times (an overflow in the replica buffers
    before the third replay), equals 4 eager steps bit for bit, scaler state included."""
    wl = synthgen.Workload("graph", [synthgen.TensorSpec("w", (300000,), "normal"),
                                     synthgen.TensorSpec("b", (77,), "zeros")], world=4,
                           bucket=100000, steps=4, gdtype="fp16", dynamic=True, grad_sigma=1e-2)
    outs = []
    for mode in ("eager", "graph"):
        opt = make_opt(wl)
        s = stream()
        sdev.init_master(wl, opt.master, s)
        opt.cast_params()
        g = [torch.zeros(opt.plan.n_pad, dtype=torch.float16, device="cuda") for _ in range(4)]
        sdev.fill_grads(wl, g, 0, wl.n, 1, 2.0 ** 16, s)
        graph = opt.capture_step(g) if mode == "graph" else None
        for t in range(4):
            if t == 2:
                g[1][123] = float("inf")
            if t == 3:
                g[1][123] = 0.0
            if graph is None:
                opt.full_step(g)
            else:
                graph.replay()
        torch.cuda.synchronize()
        outs.append((opt.result(), [to_np(x).copy() for x in (opt.master, opt.exp_avg,
                                                               opt.exp_avg_sq, opt.params)]))
    (re, ae), (rg, ag) = outs
    for k in ("adam_t", "iter", "next_scale", "hysteresis", "global_norm", "skipped"):
        assert re[k] == rg[k], k
    assert re["adam_t"] == 3
    for a, b in zip(ae, ag):
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8))


def test_binding_refuses_short_device_buffers():
    p = zb.Plan([(5000,)], 2, 3000)
    ws = torch.zeros(p.workspace_bytes(), dtype=torch.uint8, device="cuda")
    g = [torch.zeros(p.n_pad, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    R = torch.zeros(p.n_pad, device="cuda")
    for args in ((g, R[:-1], ws), (g, R, ws[:-1]), ([g[0], g[1][:p.bucket(0)[1] - 1]], R, ws)):
        with pytest.raises(zb.ZeroError) as e:
            zb.zero_reduce_scatter_bucket(p, 0, "bf16", args[0], 0, args[1], args[2])
        assert e.value.code == zb.ZERO_EINVAL and "needs" in e.value.message
    zb.zero_state_init(p, ws, zb.scaler_cfg(False))
    zb.zero_reduce_scatter_bucket(p, 0, "bf16", g, 0, R, ws)  # the full-size call goes through


def test_overlapped_production_equals_serial_streaming():
    """overlapped_step: each bucket's gradients are produced on a second stream into one
    of two slots while the previous bucket is reduced; the result must be bit-identical
    to producing the whole step first (the serial streaming run)."""
    wl = synthgen.sweep(20, 4, "bf16", steps=3)
    wl.bucket = 1 << 17  # 8 buckets
    ref_opt, ref_res = run_streaming(wl)
    opt = make_opt(wl)
    s = stream()
    sdev.init_master(wl, opt.master, s)
    opt.cast_params()
    slots = [[torch.empty(wl.bucket, dtype=torch.bfloat16, device="cuda") for _ in range(wl.world)]
             for _ in range(2)]
    prod = torch.cuda.Stream()
    for t in range(1, wl.steps + 1):
        def produce(b, bufs, sh, t=t):
            sdev.fill_grads(wl, bufs, 0, opt.plan.bucket(b)[1], t, 1.0, sh)
        opt.overlapped_step(produce, slots, prod)
        res = opt.result()
        assert res["global_norm"] == ref_res[t - 1]["global_norm"]
    for a, b in ((opt.reduced, ref_opt.reduced), (opt.master, ref_opt.master),
                 (opt.exp_avg, ref_opt.exp_avg), (opt.exp_avg_sq, ref_opt.exp_avg_sq),
                 (opt.params, ref_opt.params)):
        assert torch.equal(a.view(torch.int32 if a.element_size() == 4 else torch.int16),
                           b.view(torch.int32 if b.element_size() == 4 else torch.int16))


def test_all_gather_tma_ring_wraps():
    """Enough 32 KB tiles that every CTA of the copy kernel wraps its 4-stage ring, a
    ragged tail after the last full tile, and two launches of destinations."""
    n = 148 * 16384 * 6 + 12345
    opt = zb.ZeroOptimizer([(n,)], 2, 1 << 30, align=1)
    src = torch.randint(-32768, 32767, (opt.plan.n_pad,), dtype=torch.int16, device="cuda")
    opt.params.view(torch.int16).copy_(src)
    dst = [torch.zeros_like(opt.params) for _ in range(17)]
    opt.all_gather(dst)
    for d in dst:
        assert torch.equal(d.view(torch.int16), src)


# ----------------------------------------------------------------------------- resident W <= 2

RESIDENT = [
    ([(1 << 20,)], 2, 1 << 20, 128, "bf16", False, 3),             # the tiny shape, one bucket
    ([(300001,), (77, 5)], 1, 65536, 8, "bf16", False, 3),         # W=1, several buckets, tail
    ([(4097,), (129, 3), (50000,)], 2, 1001, 1, "fp16", True, 4),  # fp16 scaler, +inf at step 2
]


@pytest.mark.parametrize("case", RESIDENT, ids=["w2_bf16", "w1_ragged", "w2_fp16_overflow"])
def test_step_resident_equals_oracle(case):
    """zero_step_resident (sum of squares only in the bucket kernel; the update sums the
    resident replicas again) against the oracle's step: same bits as the stored-R path."""
    wl = _edge_workload(*case)
    ref = oracle.run_resident(wl)
    opt = make_opt(wl)
    s = stream()
    sdev.init_master(wl, opt.master, s)
    opt.cast_params()
    n_pad = opt.plan.n_pad
    grads = [torch.zeros(n_pad, dtype=HALF[wl.gdtype], device="cuda") for _ in range(wl.world)]
    scale = float(2.0 ** wl.init_scale_power) if wl.dynamic else 1.0
    for t in range(1, wl.steps + 1):
        sdev.fill_grads(wl, grads, 0, wl.n, t, scale, s)
        sdev.plant_infs(wl, grads, t)
        opt.step_resident(grads)
        res = opt.result()
        check_scalars(res, ref["scalars"][t - 1], exact_k=True)
        scale = float(res["next_scale"]) if wl.dynamic else 1.0
    for name, t_ in (("master", opt.master), ("m", opt.exp_avg), ("v", opt.exp_avg_sq)):
        same = check_state(name, to_np(t_), ref[name], wl.world)
        assert same == 1.0, (name, same)
    d = half_ulp_distance(to_np(opt.params), ref["params"])
    record("params", None, ref["params"], ulp=d)
    assert d.max() == 0
    if wl.dynamic:
        assert [r["skipped"] for r in ref["scalars"]] == [0, 1, 0, 0]


def test_step_resident_refusals():
    opt = zb.ZeroOptimizer([(10000,)], 4, 3000)
    g = [torch.zeros(opt.plan.n_pad, dtype=torch.bfloat16, device="cuda")] * 4
    with pytest.raises(zb.ZeroError) as e:
        opt.step_resident(g)
    assert e.value.code == zb.ZERO_EINVAL and "world_size <= 2" in e.value.message
    opt = zb.ZeroOptimizer([(10000,)], 2, 3000)
    g = [torch.zeros(opt.plan.n_pad, dtype=torch.bfloat16, device="cuda")] * 2
    opt.reduce_scatter_bucket(0, g)
    with pytest.raises(zb.ZeroError) as e:
        opt.step_resident(g)
    assert e.value.code == zb.ZERO_ESTATE


@pytest.mark.parametrize("gdt,pdt", [("bf16", "fp16"), ("fp16", "bf16")])
@pytest.mark.parametrize("resident", [False, True], ids=["stored_R", "resident"])
def test_gradient_and_parameter_dtypes_differ(gdt, pdt, resident):
    """Gradients in one half type, the gathered parameters in the other (the kernels'
    mixed instantiations), three buckets and a ragged tail, 2 steps, against the
    oracle's step with the same pair of types: bit-identical."""
    codes = {"bf16": synthgen.BF16, "fp16": synthgen.FP16}
    W, n, bucket = 2, 200003, 70000
    plan = zb.Plan([(n,)], W, bucket, 1)
    n_pad = plan.n_pad
    master0 = synthgen.master_random_host(0, n_pad, 0, 0.02)
    grads = [synthgen.grads_host(0, n_pad, 0, r, 1, 3e-2, 0.0, 1.0, codes[gdt]) for r in range(W)]
    cfg_o, hp = oracle.scaler_cfg(False), oracle.hparams()
    st = oracle.state_init(cfg_o)
    R = np.zeros(n_pad, np.float32)
    master, m, v = master0.copy(), np.zeros(n_pad, np.float32), np.zeros(n_pad, np.float32)
    params = oracle.f32_to_half(master0, codes[pdt])
    for _ in range(2):
        oracle.step(grads, codes[gdt], bucket, R, master, m, v, params, codes[pdt], cfg_o, hp, st)

    s = stream()
    dev = dict(device="cuda")
    g_d = [torch.from_numpy(g.view(np.int16)).cuda() for g in grads]
    M = torch.from_numpy(master0).cuda()
    Mm, Vv = torch.zeros(n_pad, **dev), torch.zeros(n_pad, **dev)
    Rd = torch.zeros(n_pad, **dev)
    P = torch.zeros(n_pad, dtype=torch.int16, **dev)
    ws = torch.zeros(plan.workspace_bytes(), dtype=torch.uint8, **dev)
    cfg = zb.adamw_cfg()
    zb.zero_state_init(plan, ws, zb.scaler_cfg(False), s)
    zb.zero_cast_params(plan, M, P, pdt, s)
    for _ in range(2):
        if resident:
            zb.zero_step_resident(plan, cfg, gdt, g_d, M, Mm, Vv, P, pdt, ws, s)
        else:
            for b in range(plan.n_buckets):
                zb.zero_reduce_scatter_bucket(plan, b, gdt, g_d, 0, Rd, ws, s)
            zb.zero_step(plan, cfg, M, Mm, Vv, Rd, P, pdt, ws, s)
    assert zb.zero_get_result(ws, s)["adam_t"] == 2
    for got, want in ((M, master), (Mm, m), (Vv, v)):
        assert np.array_equal(to_np(got).view(np.uint32), want.view(np.uint32))
    assert np.array_equal(to_np(P).view(np.uint16), params)
    if not resident:
        assert np.array_equal(to_np(Rd).view(np.uint32), R.view(np.uint32))
