"""CPU oracle of the ZeRO partitioned mixed-precision optimizer step.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package. It shares
no code with the CUDA library and never calls it.

The arithmetic lives in ``zero_oracle.c`` (plain single-threaded C, fp32 where the
method is fp32, fp64 for the sum of squares and the norm, -ffp-contract=off). This
module only marshals numpy arrays and drives whole workloads:

* ``run_resident``: every step of a workload whose replica gradients are resident,
  on the full arrays, exactly as ``oracle_step`` defines it.
* ``streaming_scalars`` / ``streaming_samples``: workloads whose replica buffers hold
  one bucket (the 7B-shaped one). The synthetic gradients do not depend on the
  parameters, so pass A runs the reduction and sum of squares bucket by bucket to
  get every step's scalars (norm, overflow, loss scale, clip multiplier), and
  pass B runs the elementwise update of chosen flat indices through all steps with
  those scalars. Per-bucket partial sums are accumulated in flat order inside each
  bucket and added in bucket order, the same definition ``oracle_step`` uses.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

import synthgen

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liboracle.so")

BF16, FP16 = 0, 1


def build() -> None:
    """Compile the oracle: plain C, -O2, no FMA contraction, no fast-math."""
    subprocess.check_call(
        ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-fPIC",
         "-shared", "-o", LIB_PATH, os.path.join(_HERE, "zero_oracle.c"), "-lm"])


class ScalerCfg(ctypes.Structure):
    _fields_ = [("dynamic", ctypes.c_int32), ("init_scale_power", ctypes.c_int32),
                ("window", ctypes.c_int64), ("hysteresis", ctypes.c_int32),
                ("min_scale", ctypes.c_float), ("factor", ctypes.c_float),
                ("static_scale", ctypes.c_float)]


class State(ctypes.Structure):
    _fields_ = [("scale", ctypes.c_float), ("cur_hysteresis", ctypes.c_int32),
                ("iter", ctypes.c_int64), ("last_overflow_iter", ctypes.c_int64),
                ("adam_t", ctypes.c_int64)]

    def copy(self) -> "State":
        s = State()
        ctypes.memmove(ctypes.byref(s), ctypes.byref(self), ctypes.sizeof(State))
        return s


class HParams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double),
                ("beta2", ctypes.c_double), ("eps", ctypes.c_double),
                ("weight_decay", ctypes.c_double), ("max_grad_norm", ctypes.c_double)]


class Scalars(ctypes.Structure):
    _fields_ = [("sumsq", ctypes.c_double), ("norm", ctypes.c_double),
                ("overflow", ctypes.c_int32), ("skipped", ctypes.c_int32),
                ("scale_used", ctypes.c_float), ("next_scale", ctypes.c_float),
                ("clip_coef", ctypes.c_float), ("k", ctypes.c_float),
                ("hysteresis", ctypes.c_int32), ("iter", ctypes.c_int64),
                ("adam_t", ctypes.c_int64),
                ("b1", ctypes.c_float), ("omb1", ctypes.c_float), ("b2", ctypes.c_float),
                ("omb2", ctypes.c_float), ("bc1", ctypes.c_float), ("bc2", ctypes.c_float),
                ("eps", ctypes.c_float), ("lr", ctypes.c_float), ("decay", ctypes.c_float)]

    def as_dict(self) -> dict:
        return {f: getattr(self, f) for f, _ in self._fields_}


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            build()
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        L.oracle_plan_sizes.argtypes = [vp, i32, i32, i64, i32, vp]
        L.oracle_plan_tensor_offsets.argtypes = [vp, i32, vp]
        L.oracle_plan_work_segments.restype = i64
        L.oracle_plan_work_segments.argtypes = [i64, i32, i64, i64, vp, vp, vp, vp]
        L.oracle_plan_partition.restype = i64
        L.oracle_plan_partition.argtypes = [vp, i32, i64, i32, i32, i64, vp, vp, vp, vp]
        L.oracle_half_to_f32.restype = ctypes.c_float
        L.oracle_half_to_f32.argtypes = [ctypes.c_uint16, i32]
        L.oracle_f32_to_half.restype = ctypes.c_uint16
        L.oracle_f32_to_half.argtypes = [ctypes.c_float, i32]
        L.oracle_f32_to_half_array.argtypes = [vp, vp, i64, i32]
        L.oracle_half_to_f32_array.argtypes = [vp, vp, i64, i32]
        L.oracle_state_init.argtypes = [ctypes.POINTER(ScalerCfg), ctypes.POINTER(State)]
        L.oracle_reduce.argtypes = [i32, i32, vp, i64, vp]
        L.oracle_reduce_accumulate.argtypes = [i32, i32, vp, i64, vp]
        L.oracle_sumsq.argtypes = [vp, i64, ctypes.POINTER(ctypes.c_double)]
        L.oracle_any_nonfinite.restype = i32
        L.oracle_any_nonfinite.argtypes = [vp, i64]
        L.oracle_finalize.argtypes = [ctypes.c_double, i32, ctypes.POINTER(ScalerCfg),
                                      ctypes.POINTER(HParams), ctypes.POINTER(State),
                                      ctypes.POINTER(Scalars)]
        L.oracle_adamw.argtypes = [i64, vp, vp, vp, vp, vp, i32, ctypes.POINTER(Scalars)]
        L.oracle_step.argtypes = [i32, i32, vp, i64, i64, vp, vp, vp, vp, vp, i32,
                                  ctypes.POINTER(ScalerCfg), ctypes.POINTER(HParams),
                                  ctypes.POINTER(State), ctypes.POINTER(Scalars)]
        L.oracle_memory_per_rank.argtypes = [ctypes.c_double, i32, i32, vp]
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags.c_contiguous
    return a.ctypes.data


def _ptr_array(arrs: Sequence[np.ndarray]):
    return (ctypes.c_void_p * len(arrs))(*[_ptr(a) for a in arrs])


# ----------------------------------------------------------------------------
# planner
# ----------------------------------------------------------------------------

@dataclass
class Plan:
    n: int
    n_pad: int
    p: int
    n_buckets: int
    bucket: int
    world: int
    offsets: np.ndarray

    def bucket_range(self, b: int) -> Tuple[int, int]:
        s = b * self.bucket
        return s, min(self.bucket, self.n_pad - s)


def plan(numels: Sequence[int], world: int, bucket: int, align: int = 128) -> Plan:
    nums = np.ascontiguousarray(numels, dtype=np.int64)
    out = np.zeros(4, np.int64)
    rc = lib().oracle_plan_sizes(_ptr(nums) if nums.size else None, len(nums), world,
                                 bucket, align, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_plan_sizes rejected the arguments")
    offs = np.zeros(max(len(nums), 1), np.int64)
    if len(nums):
        lib().oracle_plan_tensor_offsets(_ptr(nums), len(nums), _ptr(offs))
    return Plan(int(out[0]), int(out[1]), int(out[2]), int(out[3]), bucket, world,
                offs[:len(nums)])


def work_segments(n_pad: int, world: int, bucket: int) -> np.ndarray:
    cnt = lib().oracle_plan_work_segments(n_pad, world, bucket, 0, None, None, None, None)
    cols = [np.zeros(max(cnt, 1), np.int64) for _ in range(4)]
    lib().oracle_plan_work_segments(n_pad, world, bucket, cnt, *[_ptr(c) for c in cols])
    return np.stack([c[:cnt] for c in cols], axis=1)


def partition(numels: Sequence[int], n_pad: int, world: int, rank: int) -> np.ndarray:
    nums = np.ascontiguousarray(numels, dtype=np.int64)
    npp = _ptr(nums) if nums.size else None
    cnt = lib().oracle_plan_partition(npp, len(nums), n_pad, world, rank, 0,
                                      None, None, None, None)
    cols = [np.zeros(max(cnt, 1), np.int64) for _ in range(4)]
    lib().oracle_plan_partition(npp, len(nums), n_pad, world, rank, cnt,
                                *[_ptr(c) for c in cols])
    return np.stack([c[:cnt] for c in cols], axis=1)


# ----------------------------------------------------------------------------
# conversions and step pieces
# ----------------------------------------------------------------------------

def half_to_f32(h: np.ndarray, dtype: int) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, np.float32)
    lib().oracle_half_to_f32_array(_ptr(h), _ptr(out), h.size, dtype)
    return out


def f32_to_half(x: np.ndarray, dtype: int) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().oracle_f32_to_half_array(_ptr(x), _ptr(out), x.size, dtype)
    return out


def scaler_cfg(dynamic: bool, init_scale_power: int = 16, window: int = 100,
               hysteresis: int = 2, min_scale: float = 1.0, factor: float = 2.0,
               static_scale: float = 1.0) -> ScalerCfg:
    return ScalerCfg(int(dynamic), init_scale_power, window, hysteresis, min_scale, factor,
                     static_scale)


def hparams(lr=6e-5, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01,
            max_grad_norm=1.0) -> HParams:
    return HParams(lr, beta1, beta2, eps, weight_decay, max_grad_norm)


def state_init(cfg: ScalerCfg) -> State:
    st = State()
    lib().oracle_state_init(ctypes.byref(cfg), ctypes.byref(st))
    return st


def reduce(grads: Sequence[np.ndarray], dtype: int) -> np.ndarray:
    n = grads[0].size
    R = np.empty(n, np.float32)
    lib().oracle_reduce(len(grads), dtype, _ptr_array(grads), n, _ptr(R))
    return R


def reduce_accumulate(grads: Sequence[np.ndarray], dtype: int, R: np.ndarray) -> None:
    lib().oracle_reduce_accumulate(len(grads), dtype, _ptr_array(grads), grads[0].size, _ptr(R))


def sumsq(R: np.ndarray, S: float = 0.0) -> float:
    acc = ctypes.c_double(S)
    lib().oracle_sumsq(_ptr(R), R.size, ctypes.byref(acc))
    return acc.value


def any_nonfinite(R: np.ndarray) -> bool:
    return bool(lib().oracle_any_nonfinite(_ptr(R), R.size))


def finalize(S: float, nonfinite: bool, cfg: ScalerCfg, hp: HParams, st: State) -> Scalars:
    out = Scalars()
    lib().oracle_finalize(S, int(nonfinite), ctypes.byref(cfg), ctypes.byref(hp),
                          ctypes.byref(st), ctypes.byref(out))
    return out


def adamw(R, master, m, v, params, pdtype: int, sc: Scalars) -> None:
    lib().oracle_adamw(R.size, _ptr(R), _ptr(master), _ptr(m), _ptr(v), _ptr(params),
                       pdtype, ctypes.byref(sc))


def step(grads: Sequence[np.ndarray], gdtype: int, bucket: int, R, master, m, v, params,
         pdtype: int, cfg: ScalerCfg, hp: HParams, st: State) -> Scalars:
    out = Scalars()
    lib().oracle_step(len(grads), gdtype, _ptr_array(grads), master.size, bucket, _ptr(R),
                      _ptr(master), _ptr(m), _ptr(v), _ptr(params), pdtype,
                      ctypes.byref(cfg), ctypes.byref(hp), ctypes.byref(st),
                      ctypes.byref(out))
    return out


def memory_per_rank(psi: float, world: int, stage: int) -> Dict[str, float]:
    out = np.zeros(4, np.float64)
    if lib().oracle_memory_per_rank(psi, world, stage, _ptr(out)) != 0:
        raise ValueError("bad memory accounting arguments")
    return dict(zip(("params", "grads", "optimizer_state", "total"), out.tolist()))


# ----------------------------------------------------------------------------
# whole workloads
# ----------------------------------------------------------------------------

def workload_cfg(wl) -> Tuple[ScalerCfg, HParams]:
    cfg = scaler_cfg(wl.dynamic, wl.init_scale_power, wl.loss_scale_window, wl.hysteresis,
                     wl.min_loss_scale)
    hp = hparams(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.max_grad_norm)
    return cfg, hp


def initial_master(wl, n_pad: int) -> np.ndarray:
    """Master weights at step 0 (input recipe); the padding is zero."""
    master = np.zeros(n_pad, np.float32)
    off = 0
    for t in wl.tensors:
        if t.init == "normal":
            synthgen.master_random_host(off, t.numel, wl.seed, wl.init_sigma,
                                        out=master[off:off + t.numel])
        elif t.init == "ones":
            master[off:off + t.numel] = 1.0
        off += t.numel
    return master


def initial_master_at(wl, idx: np.ndarray) -> np.ndarray:
    offs = np.cumsum([0] + wl.numels)
    out = np.zeros(idx.size, np.float32)
    tid = np.searchsorted(offs, idx, side="right") - 1
    rnd = np.zeros(idx.size, bool)
    for k, t in enumerate(wl.tensors):
        sel = tid == k
        if t.init == "normal":
            rnd |= sel
        elif t.init == "ones":
            out[sel] = 1.0
    if rnd.any():
        out[rnd] = synthgen.master_random_at_host(idx[rnd], wl.seed, wl.init_sigma)
    return out


def step_grad_scale(wl, st: State) -> float:
    return float(st.scale) if wl.dynamic else 1.0


def resident_grads(wl, n_pad: int, t: int, scale: float,
                   out: Optional[List[np.ndarray]] = None, micro: int = 0) -> List[np.ndarray]:
    """Replica gradients of step t (micro-batch `micro`) over the whole padded space
    (input recipe); +inf sites go into the step's last micro-batch."""
    dt = wl.dtype_code
    if out is None:
        out = [np.zeros(n_pad, np.uint16) for _ in range(wl.world)]
    for r in range(wl.world):
        synthgen.grads_host(0, wl.n, wl.seed, r, wl.micro_slot(t, micro), wl.grad_sigma,
                            wl.spike_frac, scale, dt, out=out[r][:wl.n])
        out[r][wl.n:] = 0
    if micro == wl.micro_batches - 1:
        inf = np.uint16(0x7c00 if dt == FP16 else 0x7f80)
        for idx, rep in wl.inf_sites_at(t):
            out[rep][idx] = inf
    return out


def run_resident(wl, steps: Optional[int] = None, on_step=None) -> dict:
    """All steps of a resident workload on the full arrays; returns final state. With
    micro_batches > 1 the reduced gradient accumulates over the micro-batches of a step
    (bucket by bucket, in micro-batch order) before the norm is taken."""
    pl = plan(wl.numels, wl.world, wl.bucket, wl.align)
    cfg, hp = workload_cfg(wl)
    st = state_init(cfg)
    dt = wl.dtype_code
    master = initial_master(wl, pl.n_pad)
    m = np.zeros(pl.n_pad, np.float32)
    v = np.zeros(pl.n_pad, np.float32)
    R = np.zeros(pl.n_pad, np.float32)
    params = f32_to_half(master, dt)
    grads = None
    scalars = []
    for t in range(1, (steps or wl.steps) + 1):
        scale = step_grad_scale(wl, st)
        if wl.micro_batches == 1:
            grads = resident_grads(wl, pl.n_pad, t, scale, out=grads)
            sc = step(grads, dt, wl.bucket, R, master, m, v, params, dt, cfg, hp, st)
        else:
            for k in range(wl.micro_batches):
                grads = resident_grads(wl, pl.n_pad, t, scale, out=grads, micro=k)
                if k == 0:
                    R[:] = reduce(grads, dt)
                else:
                    reduce_accumulate(grads, dt, R)
            S, bad = 0.0, False
            for b in range(pl.n_buckets):
                s0, ln = pl.bucket_range(b)
                S = S + sumsq(R[s0:s0 + ln])
                bad = bad or any_nonfinite(R[s0:s0 + ln])
            sc = finalize(S, bad, cfg, hp, st)
            adamw(R, master, m, v, params, dt, sc)
        scalars.append(sc.as_dict())
        if on_step is not None:
            on_step(t, sc, R, master, m, v, params)
    return dict(plan=pl, master=master, m=m, v=v, R=R, params=params, scalars=scalars,
                state=st)


# ---------------------------- streaming workloads ----------------------------

def _bucket_effective_len(pl: Plan, n: int, b: int) -> int:
    s, ln = pl.bucket_range(b)
    return max(0, min(ln, n - s))


def streaming_slot_partials(wl, pl: Plan, t: int, scale: float,
                            chunk: int = 1 << 24) -> Dict[int, Tuple[float, bool]]:
    """For step t: {effective bucket length L: (flat-order S over buffer [0, L),
    non-finite flag)} for every distinct L among the buckets."""
    dt = wl.dtype_code
    lengths = sorted({_bucket_effective_len(pl, wl.n, b) for b in range(pl.n_buckets)})
    need = lengths[-1] if lengths else 0
    infs = {}
    for idx, rep in wl.inf_sites_at(t):
        b = idx // pl.bucket
        infs.setdefault(idx - b * pl.bucket, set()).add(rep)
    out = {}
    S, bad = 0.0, False
    if 0 in lengths:
        out[0] = (0.0, False)
    bufs = [np.empty(chunk, np.uint16) for _ in range(wl.world)]
    inf = np.uint16(0x7c00 if dt == FP16 else 0x7f80)
    j0 = 0
    li = 0
    while j0 < need:
        n = min(chunk, need - j0)
        # stop the chunk at the next snapshot length
        while li < len(lengths) and lengths[li] <= j0:
            li += 1
        if li < len(lengths):
            n = min(n, lengths[li] - j0)
        views = []
        for r in range(wl.world):
            synthgen.grads_host(j0, n, wl.seed, r, wl.slot(t), wl.grad_sigma, wl.spike_frac,
                                scale, dt, out=bufs[r][:n])
            views.append(bufs[r][:n])
        for j, reps in infs.items():
            if j0 <= j < j0 + n:
                for rep in reps:
                    views[rep][j - j0] = inf
        R = reduce(views, dt)
        S = sumsq(R, S)
        bad = bad or any_nonfinite(R)
        j0 += n
        if j0 in lengths:
            out[j0] = (S, bad)
    return out


def streaming_scalars(wl, steps: Optional[int] = None, chunk: int = 1 << 24) -> List[Scalars]:
    """Pass A: the scalar decisions of every step of a streaming workload."""
    pl = plan(wl.numels, wl.world, wl.bucket, wl.align)
    cfg, hp = workload_cfg(wl)
    st = state_init(cfg)
    res = []
    cache = {}
    for t in range(1, (steps or wl.steps) + 1):
        # steps that draw the same slot at the same scale with no +inf sites see the
        # same bucket contents: their partial sums are computed once
        key = (wl.slot(t), step_grad_scale(wl, st)) if not wl.inf_sites.get(t) else ("t", t)
        if key not in cache:
            cache[key] = streaming_slot_partials(wl, pl, t, step_grad_scale(wl, st), chunk)
        parts = cache[key]
        S, bad = 0.0, False
        for b in range(pl.n_buckets):
            Sb, badb = parts[_bucket_effective_len(pl, wl.n, b)]
            S = S + Sb
            bad = bad or badb
        res.append(finalize(S, bad, cfg, hp, st))
    return res


def streaming_samples(wl, idx: np.ndarray, scalars: Sequence[Scalars]) -> dict:
    """Pass B: master, m, v, params and the last reduced gradient at flat indices idx
    after every step in `scalars` (from pass A)."""
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    pl = plan(wl.numels, wl.world, wl.bucket, wl.align)
    dt = wl.dtype_code
    master = initial_master_at(wl, idx)
    m = np.zeros(idx.size, np.float32)
    v = np.zeros(idx.size, np.float32)
    params = f32_to_half(master, dt)
    j = (idx - (idx // pl.bucket) * pl.bucket).astype(np.uint64)
    real = idx < wl.n
    R = np.zeros(idx.size, np.float32)
    inf = np.uint16(0x7c00 if dt == FP16 else 0x7f80)
    for t, sc in enumerate(scalars, start=1):
        grads = []
        for r in range(wl.world):
            g = synthgen.grads_at_host(j, wl.seed, r, wl.slot(t), wl.grad_sigma, wl.spike_frac,
                                       float(sc.scale_used) if wl.dynamic else 1.0, dt)
            g[~real] = 0
            grads.append(g)
        for site, rep in wl.inf_sites_at(t):
            js = site - (site // pl.bucket) * pl.bucket
            grads[rep][j == js] = inf
        R = reduce(grads, dt)
        adamw(R, master, m, v, params, dt, sc)
    return dict(master=master, m=m, v=v, params=params, R=R)
