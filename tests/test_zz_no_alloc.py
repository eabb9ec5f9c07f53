"""zero_reduce_sumsq_noalloc: the reduction + sum of squares for callers that cannot
allocate device memory (its scratch is an array built into the library). Checked
through the C ABI against the workspace-based entry points on the same inputs, on two
calls in a row, so a call never sees what the previous one left in the shared array.

This file is collected last on purpose: it must pass alone in a fresh process and
after every other test."""
import ctypes
import math

import numpy as np
import pytest
import torch

import synthgen
import zero_sharded_mixed_replica_b200 as zb

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    lib = ctypes.CDLL(zb.LIB_PATH)
    fn = lib.zero_reduce_sumsq_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_int64,
                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    return fn


def _inputs(world, n, slot, dtype, seed_shift):
    half = torch.bfloat16 if dtype == "bf16" else torch.float16
    scale = 1.0 if dtype == "bf16" else 1024.0
    bufs = []
    for r in range(world):
        b = torch.empty(n, dtype=half, device="cuda")
        synthgen.grads_cuda(b.data_ptr(), seed_shift, n, 0, r, slot, 1e-3, 0.001, scale,
                            synthgen.DTYPE_CODE[dtype], torch.cuda.current_stream().cuda_stream)
        bufs.append(b)
    return bufs


def _reference(world, n, dtype, bufs):
    """The workspace path: a one-bucket plan, zero_reduce_scatter_bucket, then the
    finalize step, whose result carries the sum of squares."""
    opt = zb.ZeroOptimizer([(n,)], world, n, dtype, align=1,
                           scaler=zb.scaler_cfg(False), adamw=zb.adamw_cfg())
    assert opt.plan.n_pad == n and opt.plan.n_buckets == 1
    opt.reduce_scatter_bucket(0, bufs)
    opt.step_finalize()
    res = opt.result()
    return opt.reduced.clone(), res["sumsq"]


@pytest.mark.parametrize("world,n,dtype", [(4, 5_000_004, "bf16"), (3, (1 << 26) + 5, "fp16"),
                                           (8, 8 * 2048, "bf16")])
def test_noalloc_matches_workspace_path_two_calls(world, n, dtype):
    fn = _noalloc_fn()
    stream = torch.cuda.current_stream().cuda_stream
    reduced = torch.empty(n, dtype=torch.float32, device="cuda")
    sumsq = torch.empty(1, dtype=torch.float64, device="cuda")
    for call, (slot, shift) in enumerate(((1, 0), (2, 12345))):
        bufs = _inputs(world, n, slot, dtype, shift)
        want_R, want_S = _reference(world, n, dtype, bufs)
        reduced.fill_(float("nan"))
        sumsq.fill_(float("nan"))
        ptrs = (ctypes.c_void_p * world)(*[b.data_ptr() for b in bufs])
        rc = fn(world, zb.DTYPES[dtype], ptrs, n, reduced.data_ptr(), sumsq.data_ptr(), stream)
        assert rc == 0, zb.lib.zero_last_error()
        torch.cuda.synchronize()
        assert torch.equal(reduced.view(torch.int32), want_R.view(torch.int32)), call
        got_S = float(sumsq.item())
        # the same tolerance as the global norm everywhere else: 1e-5 relative
        assert abs(math.sqrt(got_S) - math.sqrt(want_S)) <= 1e-5 * math.sqrt(want_S), (call, got_S, want_S)


def test_noalloc_rejects_bad_arguments():
    fn = _noalloc_fn()
    x = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    r = torch.zeros(64, dtype=torch.float32, device="cuda")
    s = torch.zeros(1, dtype=torch.float64, device="cuda")
    ptrs = (ctypes.c_void_p * 2)(x.data_ptr(), x.data_ptr())
    assert fn(2, 0, ptrs, (1 << 27) + 1, r.data_ptr(), s.data_ptr(), None) == zb.ZERO_ERANGE
    assert "exceeds the limit" in zb.lib.zero_last_error().decode()
    assert fn(0, 0, ptrs, 64, r.data_ptr(), s.data_ptr(), None) == zb.ZERO_EINVAL
    assert fn(2, 5, ptrs, 64, r.data_ptr(), s.data_ptr(), None) == zb.ZERO_EINVAL
    assert fn(2, 0, ptrs, 64, r.data_ptr() + 4, s.data_ptr(), None) == zb.ZERO_EALIGN
    assert fn(2, 0, ptrs, 0, r.data_ptr(), s.data_ptr(), None) == 0
    torch.cuda.synchronize()
    assert float(s.item()) == 0.0
