"""Host-side checks of the C ABI (no GPU needed): the library loads and exports every
symbol include/zero_b200.h declares, its planner agrees bit for bit with the oracle's
independent planner, and misuse is rejected with the documented codes before any
device work."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import synthgen
import zero_sharded_mixed_replica_b200 as zb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "zero_b200.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"ZERO_API\s+[\w\s\*]*?\b(zero_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _declared_symbols()
    assert len(names) >= 20
    lib = ctypes.CDLL(zb.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert zb.zero_abi_version() == zb.ABI_VERSION == 2


def _shapes_to_numels(shapes):
    return [int(np.prod(s)) if len(s) else 1 for s in shapes]


@pytest.mark.parametrize("seed", range(40))
def test_planner_matches_oracle_planner(seed):
    rng = np.random.default_rng(100 + seed)
    shapes = []
    for _ in range(int(rng.integers(0, 8))):
        nd = int(rng.integers(0, 4))
        shapes.append(tuple(int(x) for x in rng.integers(0, 9, nd)))
    W = int(rng.integers(1, 17))
    A = int(rng.choice([1, 2, 3, 8, 128]))
    B = int(rng.integers(1, 3000))
    plan = zb.Plan(shapes, W, B, A)
    numels = _shapes_to_numels(shapes)
    ref = oracle.plan(numels, W, B, A)
    assert (plan.n, plan.n_pad, plan.p, plan.n_buckets) == (ref.n, ref.n_pad, ref.p, ref.n_buckets)
    for t in range(len(shapes)):
        assert plan.tensor(t) == (int(ref.offsets[t]), numels[t])
    for b in range(plan.n_buckets):
        s, ln = plan.bucket(b)
        assert (s, ln) == ref.bucket_range(b)
    segs = np.array(plan.work_segments(), dtype=np.int64).reshape(-1, 4)
    assert np.array_equal(segs, oracle.work_segments(ref.n_pad, W, B))
    for r in range(W):
        got = np.array(plan.partition(r), dtype=np.int64).reshape(-1, 4)
        assert np.array_equal(got, oracle.partition(numels, ref.n_pad, W, r)), r
    assert plan.info.n_segments == len(segs)


def test_config_plans():
    for name in ("tiny", "enc", "gpt2", "llama7b"):
        wl = synthgen.workload(name)
        plan = zb.Plan([t.shape for t in wl.tensors], wl.world, wl.bucket, wl.align)
        ref = oracle.plan(wl.numels, wl.world, wl.bucket, wl.align)
        assert (plan.n, plan.n_pad, plan.p, plan.n_buckets) == (ref.n, ref.n_pad, ref.p, ref.n_buckets)
        # memory per rank equals the oracle's accounting (no padding in these lists)
        for stage in range(4):
            got = plan.memory(stage)
            want = oracle.memory_per_rank(float(wl.n), wl.world, stage)
            for k in want:
                assert got[k] == want[k]
        assert plan.workspace_bytes() < 1 << 20


def test_memory_saving_87_5_percent_at_w8():
    plan = zb.Plan([(1 << 20,)], 8, 1 << 30)
    ddp, z1 = plan.memory(0), plan.memory(1)
    assert 1 - z1["optimizer_state"] / ddp["optimizer_state"] == 0.875


def _code(fn, *a):
    with pytest.raises(zb.ZeroError) as e:
        fn(*a)
    return e.value.code


def test_plan_errors():
    assert _code(zb.Plan, [(4,)], 0, 10) == zb.ZERO_EINVAL
    assert _code(zb.Plan, [(4,)], 17, 10) == zb.ZERO_EINVAL
    assert _code(zb.Plan, [(4,)], 2, 0) == zb.ZERO_EINVAL
    assert _code(zb.Plan, [(4,)], 2, 10, 0) == zb.ZERO_EINVAL
    assert _code(zb.Plan, [(4, -1)], 2, 10) == zb.ZERO_EINVAL
    assert _code(zb.Plan, [(1 << 40, 1 << 40)], 2, 10) == zb.ZERO_ERANGE
    assert _code(zb.Plan, [(1 << 62,), (1 << 62,)], 2, 10) == zb.ZERO_ERANGE
    p = zb.Plan([(4,)], 2, 10)
    assert _code(p.bucket, p.n_buckets) == zb.ZERO_EINVAL
    assert _code(p.partition, 2) == zb.ZERO_EINVAL
    assert _code(p.memory, 4) == zb.ZERO_EINVAL


def test_empty_plan():
    p = zb.Plan([], 4, 100)
    assert (p.n, p.n_pad, p.n_buckets) == (0, 0, 0)
    assert p.work_segments() == []
    assert p.partition(0) == []
    p = zb.Plan([(0, 5), ()], 2, 100, 1)  # an empty tensor and a scalar
    assert (p.n, p.n_pad) == (1, 2)
    assert p.partition(0) == [(1, 0, 0, 1)] and p.partition(1) == [(-1, 0, 1, 1)]


def test_step_call_errors_before_any_device_work():
    p = zb.Plan([(1024,)], 2, 512)
    ws = 1 << 20  # fake, aligned device addresses: never dereferenced on these paths
    R = 2 << 20
    g = [3 << 20, 4 << 20]
    assert _code(zb.zero_reduce_scatter_bucket, p, 2, "bf16", g, 0, R, ws) == zb.ZERO_EINVAL
    assert _code(zb.zero_reduce_scatter_bucket, p, -1, "bf16", g, 0, R, ws) == zb.ZERO_EINVAL
    assert _code(zb.zero_reduce_scatter_bucket, p, 0, 7, g, 0, R, ws) == zb.ZERO_EINVAL
    assert _code(zb.zero_reduce_scatter_bucket, p, 0, "bf16", [g[0], 0], 0, R, ws) == zb.ZERO_EINVAL
    assert _code(zb.zero_reduce_scatter_bucket, p, 0, "bf16", [g[0], g[1] + 2], 0, R, ws) == zb.ZERO_EALIGN
    assert _code(zb.zero_reduce_scatter_bucket, p, 0, "bf16", g, 0, R + 4, ws) == zb.ZERO_EALIGN
    assert _code(zb.zero_reduce_scatter_bucket, p, 0, "bf16", g, 0, None, ws) == zb.ZERO_EINVAL
    assert _code(zb.zero_reduce_scatter_bucket, p, 1, "bf16", g, 600, R, ws) == zb.ZERO_EINVAL
    cfg = zb.adamw_cfg()
    # a step before every bucket was reduced
    assert _code(zb.zero_step, p, cfg, R, R, R, R, R, "bf16", ws) == zb.ZERO_ESTATE
    assert _code(zb.zero_step_update, p, R, R, R, R, R, "bf16", ws) == zb.ZERO_ESTATE
    for bad in (zb.adamw_cfg(beta1=1.0), zb.adamw_cfg(eps=0.0), zb.adamw_cfg(lr=-1.0),
                zb.adamw_cfg(beta2=float("nan")), zb.adamw_cfg(max_grad_norm=float("nan"))):
        assert _code(zb.zero_step_finalize, p, bad, ws) == zb.ZERO_EINVAL
    assert _code(zb.zero_step, p, cfg, R + 8, R, R, R, R, "bf16", ws) == zb.ZERO_EALIGN
    assert _code(zb.zero_state_init, p, ws, zb.scaler_cfg(True, loss_scale_window=0)) == zb.ZERO_EINVAL
    assert _code(zb.zero_state_init, p, ws, zb.scaler_cfg(True, hysteresis=0)) == zb.ZERO_EINVAL
    assert _code(zb.zero_state_init, p, ws, zb.scaler_cfg(False, static_scale=0.0)) == zb.ZERO_EINVAL
    assert _code(zb.zero_state_init, p, ws + 8, zb.scaler_cfg(False)) == zb.ZERO_EALIGN
    assert _code(zb.zero_all_gather, p, R, [0], "bf16") == zb.ZERO_EINVAL
    assert _code(zb.zero_all_gather, p, R, [R + 2], "bf16") == zb.ZERO_EALIGN
    zb.zero_all_gather(p, R, [], "bf16")  # n_dst = 0: nothing to do


def _msg(fn, *a):
    with pytest.raises(zb.ZeroError) as e:
        fn(*a)
    assert e.value.code == zb.ZERO_EINVAL
    return e.value.message


def test_binding_checks_tensor_arguments():
    """Tensor arguments are checked (dtype, layout, host or device, length) before their
    addresses reach the library; raw integer addresses are passed through."""
    import torch
    p = zb.Plan([(1000,)], 2, 512)
    ws, R = 1 << 20, 2 << 20  # raw addresses: not checked, never dereferenced here
    bf = [torch.zeros(p.n_pad, dtype=torch.bfloat16) for _ in range(2)]
    assert "device memory" in _msg(zb.zero_reduce_scatter_bucket, p, 0, "bf16", bf, 0, R, ws)
    fp = [torch.zeros(p.n_pad, dtype=torch.float16)] * 2
    assert "where bf16" in _msg(zb.zero_reduce_scatter_bucket, p, 0, "bf16", fp, 0, R, ws)
    strided = [torch.zeros(2 * p.n_pad, dtype=torch.bfloat16)[::2]] * 2
    assert "contiguous" in _msg(zb.zero_reduce_scatter_bucket, p, 0, "bf16", strided, 0, R, ws)
    f64 = torch.zeros(p.n_pad, dtype=torch.float64)
    assert "where f32" in _msg(zb.zero_step, p, zb.adamw_cfg(), f64, R, R, R, R, "bf16", ws)
    # the host-staging call wants host replicas that cover the bucket
    b0, len0 = p.bucket(1)
    short = [torch.zeros(b0 + len0 - 1, dtype=torch.int16)] * 2
    assert "needs %d" % (b0 + len0) in _msg(zb.zero_reduce_scatter_bucket_host, p, 1, "bf16",
                                             short, 0, [3 << 20, 4 << 20], R, ws)
    # a replica buffer indexed from the bucket start needs only the bucket's length
    based = [torch.zeros(len0 - 1, dtype=torch.int16)] * 2
    assert "needs %d" % len0 in _msg(zb.zero_reduce_scatter_bucket_host, p, 1, "bf16", based,
                                      b0, [3 << 20, 4 << 20], R, ws)
    ws_host = torch.zeros(p.workspace_bytes(), dtype=torch.uint8)
    assert "device memory" in _msg(zb.zero_state_init, p, ws_host, zb.scaler_cfg(False))


def test_step_resident_refusals_before_any_device_work():
    cfg = zb.adamw_cfg()
    ws, m = 1 << 20, 2 << 20  # fake aligned device addresses, never dereferenced here
    p4 = zb.Plan([(1024,)], 4, 512)
    assert _code(zb.zero_step_resident, p4, cfg, "bf16", [m] * 4, m, m, m, m, "bf16", ws) \
        == zb.ZERO_EINVAL  # world_size > 2
    p2 = zb.Plan([(1024,)], 2, 512)
    assert _code(zb.zero_step_resident, p2, cfg, 7, [m] * 2, m, m, m, m, "bf16", ws) \
        == zb.ZERO_EINVAL  # grad dtype
    assert _code(zb.zero_step_resident, p2, cfg, "bf16", [m, m + 2], m, m, m, m, "bf16", ws) \
        == zb.ZERO_EALIGN
    assert _code(zb.zero_step_resident, p2, cfg, "bf16", [m, 0], m, m, m, m, "bf16", ws) \
        == zb.ZERO_EINVAL
    assert _code(zb.zero_step_resident, p2, cfg, "bf16", [m] * 2, m + 4, m, m, m, "bf16", ws) \
        == zb.ZERO_EALIGN
    assert _code(zb.zero_step_resident, p2, zb.adamw_cfg(beta1=1.0), "bf16", [m] * 2, m, m, m,
                 m, "bf16", ws) == zb.ZERO_EINVAL


def test_step_full_refusals_before_any_device_work():
    cfg = zb.adamw_cfg()
    ws, m = 1 << 20, 2 << 20  # fake aligned device addresses, never dereferenced here
    p = zb.Plan([(1024,)], 2, 512)
    call = zb.zero_step_full
    assert _code(call, p, cfg, "bf16", [m] * 2, 5, m, m, m, m, m, "bf16", ws) == zb.ZERO_EINVAL
    assert _code(call, p, cfg, 7, [m] * 2, 0, m, m, m, m, m, "bf16", ws) == zb.ZERO_EINVAL
    assert _code(call, p, cfg, "bf16", [m, m + 2], 0, m, m, m, m, m, "bf16", ws) == zb.ZERO_EALIGN
    assert _code(call, p, cfg, "bf16", [m, 0], 0, m, m, m, m, m, "bf16", ws) == zb.ZERO_EINVAL
    assert _code(call, p, cfg, "bf16", [m] * 2, 0, m + 4, m, m, m, m, "bf16", ws) == zb.ZERO_EALIGN
    assert _code(call, p, cfg, "bf16", [m] * 2, 0, None, m, m, m, m, "bf16", ws) == zb.ZERO_EINVAL
    assert _code(call, p, zb.adamw_cfg(eps=0.0), "bf16", [m] * 2, 0, m, m, m, m, m, "bf16", ws) \
        == zb.ZERO_EINVAL


@pytest.mark.parametrize("std", ["c99", "c11"])
def test_header_compiles_as_plain_c(tmp_path, std):
    """include/zero_b200.h is a C header: a C program that includes it, links against
    libzero_b200.so and plans a step compiles without warnings under -pedantic and runs."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use.c"
    src.write_text('#include "zero_b200.h"\n'
                   "int main(void) {\n"
                   "  zero_plan* plan = 0;\n"
                   "  const int64_t dims[1] = {1024};\n"
                   "  const int32_t ndims[1] = {1};\n"
                   "  int rc = zero_plan_create(dims, ndims, 1, 2, 512, 128, &plan);\n"
                   "  if (rc == ZERO_OK) zero_plan_destroy(plan);\n"
                   "  return zero_abi_version() == ZERO_ABI_VERSION ? rc : 1;\n"
                   "}\n")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(zb.LIB_PATH)
    exe = tmp_path / "use"
    r = subprocess.run([cc, f"-std={std}", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-I", os.path.join(root, "include"), str(src), "-o", str(exe),
                        "-L", libdir, "-lzero_b200", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    # planning needs no GPU: the program runs here too
    assert subprocess.run([str(exe)]).returncode == 0
