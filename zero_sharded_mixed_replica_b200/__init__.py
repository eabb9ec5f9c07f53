"""Python binding of libzero_b200: the ZeRO partitioned mixed-precision optimizer step
on B200 (sm_100a).

This module only marshals arguments into the C ABI declared in ``include/zero_b200.h``;
every step of the optimizer runs in the library's CUDA kernels. The functions carry
the C names. There is no fallback: if ``libzero_b200.so`` is missing or fails to load,
importing the binding raises.

Device buffers are passed as integer device addresses (``tensor.data_ptr()``) or as
torch tensors; streams as integer ``cudaStream_t`` handles (``stream.cuda_stream``)
or torch streams; ``None`` means the legacy default stream.
"""
from __future__ import annotations

import ctypes
import os
from typing import Iterable, List, Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzero_b200.so")

ZERO_OK = 0
ZERO_EINVAL = -1
ZERO_EALIGN = -2
ZERO_ERANGE = -3
ZERO_ESTATE = -4
ZERO_ECUDA = -5
ZERO_ENOMEM = -6
ZERO_EDEVICE = -7
ZERO_BF16 = 0
ZERO_FP16 = 1
ZERO_MAX_WORLD = 16
DTYPES = {"bf16": ZERO_BF16, "fp16": ZERO_FP16}

_ERR_NAMES = {ZERO_EINVAL: "EINVAL", ZERO_EALIGN: "EALIGN", ZERO_ERANGE: "ERANGE",
              ZERO_ESTATE: "ESTATE", ZERO_ECUDA: "ECUDA", ZERO_ENOMEM: "ENOMEM",
              ZERO_EDEVICE: "EDEVICE"}


class ZeroError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"{_ERR_NAMES.get(code, code)}: {message}")
        self.code = code
        self.message = message


class PlanInfo(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int64), ("n_pad", ctypes.c_int64), ("p", ctypes.c_int64),
                ("n_buckets", ctypes.c_int64), ("n_segments", ctypes.c_int64),
                ("n_tensors", ctypes.c_int64), ("bucket_size", ctypes.c_int64),
                ("world_size", ctypes.c_int32), ("align", ctypes.c_int32)]


class Segment(ctypes.Structure):
    _fields_ = [("tensor", ctypes.c_int64), ("offset_in_tensor", ctypes.c_int64),
                ("flat_offset", ctypes.c_int64), ("length", ctypes.c_int64)]


class WorkSegment(ctypes.Structure):
    _fields_ = [("bucket", ctypes.c_int64), ("rank", ctypes.c_int64),
                ("start", ctypes.c_int64), ("length", ctypes.c_int64)]


class ScalerCfg(ctypes.Structure):
    _fields_ = [("dynamic", ctypes.c_int32), ("initial_scale_power", ctypes.c_int32),
                ("loss_scale_window", ctypes.c_int64), ("hysteresis", ctypes.c_int32),
                ("min_loss_scale", ctypes.c_float), ("scale_factor", ctypes.c_float),
                ("static_scale", ctypes.c_float)]


class AdamWCfg(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double),
                ("beta2", ctypes.c_double), ("eps", ctypes.c_double),
                ("weight_decay", ctypes.c_double), ("max_grad_norm", ctypes.c_double)]


class StepResult(ctypes.Structure):
    _fields_ = [("global_norm", ctypes.c_double), ("sumsq", ctypes.c_double),
                ("clip_coef", ctypes.c_float), ("scale_used", ctypes.c_float),
                ("next_scale", ctypes.c_float), ("k", ctypes.c_float),
                ("overflow", ctypes.c_int32), ("skipped", ctypes.c_int32),
                ("hysteresis", ctypes.c_int32), ("device_error", ctypes.c_int32),
                ("iter", ctypes.c_int64), ("adam_t", ctypes.c_int64)]

    def as_dict(self) -> dict:
        return {f: getattr(self, f) for f, _ in self._fields_}


class ScalerState(ctypes.Structure):
    _fields_ = [("scale", ctypes.c_float), ("cur_hysteresis", ctypes.c_int32),
                ("iter", ctypes.c_int64), ("last_overflow_iter", ctypes.c_int64),
                ("adam_t", ctypes.c_int64)]

    def as_dict(self) -> dict:
        return {f: getattr(self, f) for f, _ in self._fields_}


class Zero3Event(ctypes.Structure):
    _fields_ = [("op", ctypes.c_int32), ("layer", ctypes.c_int32), ("first", ctypes.c_int64),
                ("count", ctypes.c_int64)]


class Zero3Stats(ctypes.Structure):
    _fields_ = [("peak_live_elements", ctypes.c_int64), ("fetched_elements", ctypes.c_int64),
                ("fetch_events", ctypes.c_int64), ("persistent_elements", ctypes.c_int64),
                ("over_budget_layers", ctypes.c_int64)]


class Memory(ctypes.Structure):
    _fields_ = [("params", ctypes.c_double), ("grads", ctypes.c_double),
                ("optimizer_state", ctypes.c_double), ("total", ctypes.c_double)]


ABI_VERSION = 2  # must equal ZERO_ABI_VERSION of include/zero_b200.h


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; "
            f"g.build()'` (nvcc, sm_100a). There is no CPU fallback.")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    P = ctypes.POINTER
    sig = {
        "zero_plan_create": [vp, vp, i32, i32, i64, i32, P(vp)],
        "zero_plan_destroy": [vp],
        "zero_plan_get_info": [vp, P(PlanInfo)],
        "zero_plan_tensor": [vp, i32, P(i64), P(i64)],
        "zero_plan_bucket": [vp, i64, P(i64), P(i64)],
        "zero_plan_work_segments": [vp, vp, i64, P(i64)],
        "zero_plan_partition": [vp, i32, vp, i64, P(i64)],
        "zero_plan_memory": [vp, i32, P(Memory)],
        "zero_workspace_bytes": [vp, P(ctypes.c_size_t)],
        "zero_state_init": [vp, vp, P(ScalerCfg), vp],
        "zero_cast_params": [vp, vp, vp, i32, vp],
        "zero_state_read": [vp, P(ScalerState), vp],
        "zero_state_write": [vp, vp, P(ScalerCfg), P(ScalerState), vp],
        "zero_reduce_scatter_bucket": [vp, i64, i32, vp, i64, vp, vp, vp],
        "zero_reduce_scatter_bucket_host": [vp, i64, i32, vp, i64, vp, vp, vp, vp],
        "zero_reduce_scatter_bucket_accum": [vp, i64, i32, i32, i32, vp, i64, vp, vp, vp],
        "zero_step": [vp, P(AdamWCfg), vp, vp, vp, vp, vp, i32, vp, vp],
        "zero_step_finalize": [vp, P(AdamWCfg), vp, vp],
        "zero_step_resident": [vp, P(AdamWCfg), i32, vp, vp, vp, vp, vp, i32, vp, vp],
        "zero_step_full": [vp, P(AdamWCfg), i32, vp, i64, vp, vp, vp, vp, vp, i32, vp, vp],
        "zero_step_update": [vp, vp, vp, vp, vp, vp, i32, vp, vp],
        "zero_all_gather": [vp, vp, vp, i32, i32, vp],
        "zero_get_result": [vp, P(StepResult), vp],
        "zero_reduce_scatter_segment": [vp, i64, i32, i32, vp, i64, vp, vp, vp],
        "zero_step_local_sumsq": [vp, i32, vp, vp, vp],
        "zero_step_finalize_ranks": [vp, P(AdamWCfg), vp, vp, vp],
        "zero_step_update_partition": [vp, i32, vp, vp, vp, vp, vp, i32, i32, vp, vp],
        "zero_ipc_handle_bytes": [],
        "zero_ipc_get_handle": [vp, vp, P(i64)],
        "zero_ipc_open_handle": [vp, P(vp)],
        "zero_ipc_close": [vp],
        "zero_reduce_sumsq_noalloc": [i32, i32, vp, i64, vp, vp, vp],
        "zero_selftest_bounded_wait": [vp, vp],
        "zero3_schedule_create": [vp, vp, i32, i64, i64, i64, P(vp)],
        "zero3_schedule_events": [vp, vp, i64, P(i64)],
        "zero3_schedule_tensors": [vp, vp, i64, P(i64)],
        "zero3_schedule_stats": [vp, P(Zero3Stats)],
        "zero3_schedule_destroy": [vp],
        "zero3_gather": [vp, vp, i32, vp, vp, vp],
        "zero_last_error": [],
        "zero_abi_version": [],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    L.zero_plan_destroy.restype = None
    L.zero3_schedule_destroy.restype = None
    L.zero_last_error.restype = ctypes.c_char_p
    if L.zero_abi_version() != ABI_VERSION:
        raise ImportError(f"{LIB_PATH} has ABI {L.zero_abi_version()}, this binding wants "
                          f"{ABI_VERSION}: rebuild the library")
    return L


lib = _load()


def _check(rc: int) -> None:
    if rc != ZERO_OK:
        raise ZeroError(rc, (lib.zero_last_error() or b"").decode())


def _addr(x) -> Optional[int]:
    """Device address of an int, a torch tensor, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _ptr_array(ptrs: Sequence) -> ctypes.Array:
    return (ctypes.c_void_p * len(ptrs))(*[_addr(p) for p in ptrs])


# Tensor arguments are checked before their addresses cross the ABI (the library trusts
# the lengths the plan implies, and a short buffer would be read or written out of
# bounds on the device). Plain integers are raw addresses and are not checked.
_HALF_DTYPES = {"bf16": ("torch.bfloat16", "torch.int16", "torch.uint16"),
                "fp16": ("torch.float16", "torch.int16", "torch.uint16")}
_KIND_DTYPES = {"f32": ("torch.float32",), "f64": ("torch.float64",)}


def _buf(x, kind: str, need: int, name: str, host: bool = False) -> Optional[int]:
    """Address of `x` after checking a tensor argument: `kind` is "f32", "f64", "bf16",
    "fp16" or "bytes"; `need` the elements (bytes for "bytes") it must hold."""
    if x is None or isinstance(x, int):
        return x
    dt = str(x.dtype)
    if kind in _HALF_DTYPES:
        ok, unit = dt in _HALF_DTYPES[kind], 2
    elif kind in _KIND_DTYPES:
        ok, unit = dt in _KIND_DTYPES[kind], 1
    else:
        ok, unit = True, 1
    if not ok:
        raise ZeroError(ZERO_EINVAL, f"{name}: dtype {dt} where {kind} is expected")
    if not x.is_contiguous():
        raise ZeroError(ZERO_EINVAL, f"{name}: not contiguous")
    where = x.device.type
    if (where == "cpu") != host:
        raise ZeroError(ZERO_EINVAL, f"{name}: a {where} tensor where "
                                     f"{'host' if host else 'device'} memory is expected")
    have = x.numel() * x.element_size() if kind == "bytes" else \
        x.numel() * x.element_size() // (2 if unit == 2 else x.element_size())
    if have < need:
        raise ZeroError(ZERO_EINVAL, f"{name}: holds {have} {'bytes' if kind == 'bytes' else 'elements'}"
                                     f", needs {need}")
    return x.data_ptr()


def _dtype_name(dt) -> str:
    return dt if isinstance(dt, str) else {v: k for k, v in DTYPES.items()}.get(int(dt), "?")


def _replicas(plan, bucket: int, base: int, grads: Sequence, gdt, name: str, host=False):
    """The replica pointer array of one bucket, each tensor checked to cover it."""
    start, length = plan.bucket(bucket) if 0 <= bucket < plan.n_buckets else (base, 0)
    need = max(0, start + length - int(base))
    kind = _dtype_name(gdt)
    return (ctypes.c_void_p * len(grads))(
        *[_buf(g, kind, need, f"{name}[{r}]", host) for r, g in enumerate(grads)])


def _dtype(dt) -> int:
    return DTYPES[dt] if isinstance(dt, str) else int(dt)


# ---------------------------------------------------------------------------- planning

class Plan:
    """Owns a zero_plan handle (host memory)."""

    def __init__(self, shapes: Iterable[Sequence[int]], world_size: int,
                 reduce_bucket_size: int, align: int = 128):
        shapes = [tuple(int(d) for d in s) for s in shapes]
        dims = [d for s in shapes for d in s]
        ndims = [len(s) for s in shapes]
        dims_arr = (ctypes.c_int64 * max(len(dims), 1))(*dims)
        ndims_arr = (ctypes.c_int32 * max(len(ndims), 1))(*ndims)
        h = ctypes.c_void_p()
        _check(lib.zero_plan_create(dims_arr, ndims_arr, len(shapes), int(world_size),
                                    int(reduce_bucket_size), int(align), ctypes.byref(h)))
        self._h = h
        self._destroy = lib.zero_plan_destroy  # kept for interpreter shutdown
        self.shapes = shapes
        inf = PlanInfo()
        _check(lib.zero_plan_get_info(self._h, ctypes.byref(inf)))
        self.info = inf

    @property
    def handle(self):
        return self._h

    def __del__(self):
        h = getattr(self, "_h", None)
        destroy = getattr(self, "_destroy", None)
        if h is not None and h.value and destroy is not None:
            destroy(h)
            self._h = None

    # convenience views of the info
    n = property(lambda self: self.info.n)
    n_pad = property(lambda self: self.info.n_pad)
    p = property(lambda self: self.info.p)
    n_buckets = property(lambda self: self.info.n_buckets)
    world_size = property(lambda self: self.info.world_size)
    bucket_size = property(lambda self: self.info.bucket_size)

    def tensor(self, t: int):
        off, num = ctypes.c_int64(), ctypes.c_int64()
        _check(lib.zero_plan_tensor(self._h, t, ctypes.byref(off), ctypes.byref(num)))
        return off.value, num.value

    @property
    def tensor_table(self) -> List[tuple]:
        """(flat offset, numel) of every tensor, read once."""
        if getattr(self, "_table", None) is None:
            self._table = [self.tensor(t) for t in range(self.info.n_tensors)]
        return self._table

    def bucket(self, b: int):
        """(start, length) of bucket b (asked of the library once per bucket)."""
        cache = self.__dict__.setdefault("_buckets", {})
        if b not in cache:
            s, ln = ctypes.c_int64(), ctypes.c_int64()
            _check(lib.zero_plan_bucket(self._h, b, ctypes.byref(s), ctypes.byref(ln)))
            cache[b] = (s.value, ln.value)
        return cache[b]

    def work_segments(self) -> List[tuple]:
        cnt = ctypes.c_int64()
        _check(lib.zero_plan_work_segments(self._h, None, 0, ctypes.byref(cnt)))
        arr = (WorkSegment * max(cnt.value, 1))()
        _check(lib.zero_plan_work_segments(self._h, arr, cnt.value, ctypes.byref(cnt)))
        return [(s.bucket, s.rank, s.start, s.length) for s in arr[:cnt.value]]

    def partition(self, rank: int) -> List[tuple]:
        cnt = ctypes.c_int64()
        _check(lib.zero_plan_partition(self._h, rank, None, 0, ctypes.byref(cnt)))
        arr = (Segment * max(cnt.value, 1))()
        _check(lib.zero_plan_partition(self._h, rank, arr, cnt.value, ctypes.byref(cnt)))
        return [(s.tensor, s.offset_in_tensor, s.flat_offset, s.length) for s in arr[:cnt.value]]

    def memory(self, stage: int) -> dict:
        m = Memory()
        _check(lib.zero_plan_memory(self._h, stage, ctypes.byref(m)))
        return {f: getattr(m, f) for f, _ in Memory._fields_}

    def workspace_bytes(self) -> int:
        if getattr(self, "_ws_bytes", None) is None:
            b = ctypes.c_size_t()
            _check(lib.zero_workspace_bytes(self._h, ctypes.byref(b)))
            self._ws_bytes = b.value
        return self._ws_bytes


def zero_plan_create(shapes, world_size, reduce_bucket_size, align=128) -> Plan:
    return Plan(shapes, world_size, reduce_bucket_size, align)


def zero_workspace_bytes(plan: Plan) -> int:
    return plan.workspace_bytes()


def scaler_cfg(dynamic: bool, initial_scale_power: int = 16, loss_scale_window: int = 100,
               hysteresis: int = 2, min_loss_scale: float = 1.0, scale_factor: float = 2.0,
               static_scale: float = 1.0) -> ScalerCfg:
    return ScalerCfg(int(dynamic), initial_scale_power, loss_scale_window, hysteresis,
                     min_loss_scale, scale_factor, static_scale)


def adamw_cfg(lr=6e-5, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01,
              max_grad_norm=1.0) -> AdamWCfg:
    return AdamWCfg(lr, beta1, beta2, eps, weight_decay, max_grad_norm)


# ---------------------------------------------------------------------------- the step

def zero_state_init(plan: Plan, workspace, cfg: ScalerCfg, stream=None) -> None:
    ws = _buf(workspace, "bytes", plan.workspace_bytes(), "workspace")
    _check(lib.zero_state_init(plan.handle, ws, ctypes.byref(cfg), _stream(stream)))


def zero_state_read(workspace, stream=None) -> dict:
    st = ScalerState()
    _check(lib.zero_state_read(_addr(workspace), ctypes.byref(st), _stream(stream)))
    return st.as_dict()


def zero_state_write(plan: Plan, workspace, cfg: ScalerCfg, state: dict, stream=None) -> None:
    st = ScalerState(**{k: state[k] for k, _ in ScalerState._fields_})
    _check(lib.zero_state_write(plan.handle, _buf(workspace, "bytes", plan.workspace_bytes(),
                                                  "workspace"), ctypes.byref(cfg),
                                ctypes.byref(st), _stream(stream)))


def zero_cast_params(plan: Plan, master, params, param_dtype, stream=None) -> None:
    _check(lib.zero_cast_params(plan.handle, _buf(master, "f32", plan.n_pad, "master"),
                                _buf(params, _dtype_name(param_dtype), plan.n_pad, "params"),
                                _dtype(param_dtype), _stream(stream)))


def zero_reduce_scatter_bucket(plan: Plan, bucket: int, grad_dtype, replica_grads: Sequence,
                               replica_base_offset: int, reduced, workspace, stream=None) -> None:
    _check(lib.zero_reduce_scatter_bucket(
        plan.handle, bucket, _dtype(grad_dtype),
        _replicas(plan, bucket, replica_base_offset, replica_grads, grad_dtype, "replica_grads"),
        int(replica_base_offset), _buf(reduced, "f32", plan.n_pad, "reduced"),
        _buf(workspace, "bytes", plan.workspace_bytes(), "workspace"), _stream(stream)))


def zero_reduce_scatter_bucket_host(plan: Plan, bucket: int, grad_dtype,
                                    host_replica_grads: Sequence, host_base_offset: int,
                                    device_staging: Sequence, reduced, workspace,
                                    stream=None) -> None:
    length = plan.bucket(bucket)[1] if 0 <= bucket < plan.n_buckets else 0
    kind = _dtype_name(grad_dtype)
    staging = (ctypes.c_void_p * len(device_staging))(
        *[_buf(b, kind, length, f"device_staging[{r}]") for r, b in enumerate(device_staging)])
    _check(lib.zero_reduce_scatter_bucket_host(
        plan.handle, bucket, _dtype(grad_dtype),
        _replicas(plan, bucket, host_base_offset, host_replica_grads, grad_dtype,
                  "host_replica_grads", host=True),
        int(host_base_offset), staging, _buf(reduced, "f32", plan.n_pad, "reduced"),
        _buf(workspace, "bytes", plan.workspace_bytes(), "workspace"), _stream(stream)))


def zero_reduce_scatter_bucket_accum(plan: Plan, bucket: int, micro: int, n_micro: int,
                                     grad_dtype, replica_grads: Sequence,
                                     replica_base_offset: int, reduced, workspace,
                                     stream=None) -> None:
    _check(lib.zero_reduce_scatter_bucket_accum(
        plan.handle, bucket, micro, n_micro, _dtype(grad_dtype),
        _replicas(plan, bucket, replica_base_offset, replica_grads, grad_dtype, "replica_grads"),
        int(replica_base_offset), _buf(reduced, "f32", plan.n_pad, "reduced"),
        _buf(workspace, "bytes", plan.workspace_bytes(), "workspace"), _stream(stream)))


def zero_step(plan: Plan, cfg: AdamWCfg, master, exp_avg, exp_avg_sq, reduced, params,
              param_dtype, workspace, stream=None) -> None:
    n = plan.n_pad
    _check(lib.zero_step(plan.handle, ctypes.byref(cfg), _buf(master, "f32", n, "master"),
                         _buf(exp_avg, "f32", n, "exp_avg"), _buf(exp_avg_sq, "f32", n, "exp_avg_sq"),
                         _buf(reduced, "f32", n, "reduced"),
                         _buf(params, _dtype_name(param_dtype), n, "params"), _dtype(param_dtype),
                         _buf(workspace, "bytes", plan.workspace_bytes(), "workspace"),
                         _stream(stream)))


def zero_step_full(plan: Plan, cfg: AdamWCfg, grad_dtype, replica_grads: Sequence,
                   replica_base_offset: int, reduced, master, exp_avg, exp_avg_sq, params,
                   param_dtype, workspace, stream=None) -> None:
    n, gk = plan.n_pad, _dtype_name(grad_dtype)
    need = max(0, n - int(replica_base_offset))
    reps = (ctypes.c_void_p * len(replica_grads))(
        *[_buf(g, gk, need, f"replica_grads[{r}]") for r, g in enumerate(replica_grads)])
    _check(lib.zero_step_full(plan.handle, ctypes.byref(cfg), _dtype(grad_dtype), reps,
                              int(replica_base_offset), _buf(reduced, "f32", n, "reduced"),
                              _buf(master, "f32", n, "master"), _buf(exp_avg, "f32", n, "exp_avg"),
                              _buf(exp_avg_sq, "f32", n, "exp_avg_sq"),
                              _buf(params, _dtype_name(param_dtype), n, "params"),
                              _dtype(param_dtype),
                              _buf(workspace, "bytes", plan.workspace_bytes(), "workspace"),
                              _stream(stream)))


def zero_step_resident(plan: Plan, cfg: AdamWCfg, grad_dtype, replica_grads: Sequence, master,
                       exp_avg, exp_avg_sq, params, param_dtype, workspace, stream=None) -> None:
    n, gk = plan.n_pad, _dtype_name(grad_dtype)
    reps = (ctypes.c_void_p * len(replica_grads))(
        *[_buf(g, gk, n, f"replica_grads[{r}]") for r, g in enumerate(replica_grads)])
    _check(lib.zero_step_resident(plan.handle, ctypes.byref(cfg), _dtype(grad_dtype), reps,
                                  _buf(master, "f32", n, "master"),
                                  _buf(exp_avg, "f32", n, "exp_avg"),
                                  _buf(exp_avg_sq, "f32", n, "exp_avg_sq"),
                                  _buf(params, _dtype_name(param_dtype), n, "params"),
                                  _dtype(param_dtype),
                                  _buf(workspace, "bytes", plan.workspace_bytes(), "workspace"),
                                  _stream(stream)))


def zero_step_finalize(plan: Plan, cfg: AdamWCfg, workspace, stream=None) -> None:
    _check(lib.zero_step_finalize(plan.handle, ctypes.byref(cfg),
                                  _buf(workspace, "bytes", plan.workspace_bytes(), "workspace"),
                                  _stream(stream)))


def zero_step_update(plan: Plan, master, exp_avg, exp_avg_sq, reduced, params, param_dtype,
                     workspace, stream=None) -> None:
    n = plan.n_pad
    _check(lib.zero_step_update(plan.handle, _buf(master, "f32", n, "master"),
                                _buf(exp_avg, "f32", n, "exp_avg"),
                                _buf(exp_avg_sq, "f32", n, "exp_avg_sq"),
                                _buf(reduced, "f32", n, "reduced"),
                                _buf(params, _dtype_name(param_dtype), n, "params"),
                                _dtype(param_dtype),
                                _buf(workspace, "bytes", plan.workspace_bytes(), "workspace"),
                                _stream(stream)))


def zero_all_gather(plan: Plan, params, rank_params: Sequence, param_dtype, stream=None) -> None:
    kind, n = _dtype_name(param_dtype), plan.n_pad
    arr = (ctypes.c_void_p * len(rank_params))(
        *[_buf(d, kind, n, f"rank_params[{r}]") for r, d in enumerate(rank_params)]) \
        if rank_params else None
    _check(lib.zero_all_gather(plan.handle, _buf(params, kind, n, "params"), arr,
                               len(rank_params), _dtype(param_dtype), _stream(stream)))


def zero_get_result(workspace, stream=None) -> dict:
    r = StepResult()
    _check(lib.zero_get_result(_addr(workspace), ctypes.byref(r), _stream(stream)))
    return r.as_dict()


def zero_selftest_bounded_wait(workspace, stream=None) -> None:
    _check(lib.zero_selftest_bounded_wait(_addr(workspace), _stream(stream)))


ZERO3_FETCH, ZERO3_COMPUTE, ZERO3_RELEASE = 0, 1, 2


class Zero3Schedule:
    """The ZeRO-3 fetch / compute / release order of one forward pass (host memory)."""

    def __init__(self, plan: Plan, layer_of_tensor: Sequence[int], n_layers: int,
                 prefetch_bucket_size: int, max_live_parameters: int,
                 persistence_threshold: int):
        arr = (ctypes.c_int32 * max(len(layer_of_tensor), 1))(*layer_of_tensor)
        h = ctypes.c_void_p()
        _check(lib.zero3_schedule_create(plan.handle, arr, n_layers, int(prefetch_bucket_size),
                                         int(max_live_parameters), int(persistence_threshold),
                                         ctypes.byref(h)))
        self._h = h
        self._destroy = lib.zero3_schedule_destroy
        cnt = ctypes.c_int64()
        _check(lib.zero3_schedule_events(h, None, 0, ctypes.byref(cnt)))
        ev = (Zero3Event * max(cnt.value, 1))()
        _check(lib.zero3_schedule_events(h, ev, cnt.value, ctypes.byref(cnt)))
        tc = ctypes.c_int64()
        _check(lib.zero3_schedule_tensors(h, None, 0, ctypes.byref(tc)))
        ts = (ctypes.c_int32 * max(tc.value, 1))()
        _check(lib.zero3_schedule_tensors(h, ts, tc.value, ctypes.byref(tc)))
        ids = list(ts[:tc.value])
        self.events = [(e.op, e.layer, ids[e.first:e.first + e.count]) for e in ev[:cnt.value]]
        st = Zero3Stats()
        _check(lib.zero3_schedule_stats(h, ctypes.byref(st)))
        self.stats = {f: getattr(st, f) for f, _ in Zero3Stats._fields_}

    def __del__(self):
        h = getattr(self, "_h", None)
        d = getattr(self, "_destroy", None)
        if h is not None and h.value and d is not None:
            d(h)
            self._h = None


def zero3_gather(plan: Plan, tensors: Sequence[int], partitions: Sequence, dst,
                 stream=None) -> None:
    arr = (ctypes.c_int32 * max(len(tensors), 1))(*tensors)
    if dst is not None and not isinstance(dst, int):  # a tensor: check its length
        table = plan.tensor_table
        need = 2 * sum(table[t][1] for t in tensors if 0 <= t < len(table))  # 2-byte elements
        dst = _buf(dst, "bytes", need, "dst")
    _check(lib.zero3_gather(plan.handle, arr, len(tensors),
                            _ptr_array(partitions) if partitions else None, dst,
                            _stream(stream)))


def zero_abi_version() -> int:
    return lib.zero_abi_version()


# ---------------------------------------------------------------------------- one rank of W

def zero_reduce_scatter_segment(plan: Plan, bucket: int, rank: int, grad_dtype,
                                replica_grads: Sequence, replica_base_offset: int,
                                reduced_local, workspace, stream=None) -> None:
    _check(lib.zero_reduce_scatter_segment(
        plan.handle, bucket, rank, _dtype(grad_dtype),
        _replicas(plan, bucket, replica_base_offset, replica_grads, grad_dtype, "replica_grads"),
        int(replica_base_offset), _buf(reduced_local, "f32", plan.p, "reduced_local"),
        _buf(workspace, "bytes", plan.workspace_bytes(), "workspace"), _stream(stream)))


def zero_step_local_sumsq(plan: Plan, rank: int, workspace, sumsq_out, stream=None) -> None:
    _check(lib.zero_step_local_sumsq(plan.handle, rank,
                                     _buf(workspace, "bytes", plan.workspace_bytes(), "workspace"),
                                     _buf(sumsq_out, "f64", 1, "sumsq_out"), _stream(stream)))


def zero_step_finalize_ranks(plan: Plan, cfg: AdamWCfg, sumsq_ranks, workspace,
                             stream=None) -> None:
    _check(lib.zero_step_finalize_ranks(plan.handle, ctypes.byref(cfg),
                                        _buf(sumsq_ranks, "f64", plan.world_size, "sumsq_ranks"),
                                        _buf(workspace, "bytes", plan.workspace_bytes(),
                                             "workspace"), _stream(stream)))


def zero_step_update_partition(plan: Plan, rank: int, master_local, exp_avg_local,
                               exp_avg_sq_local, reduced_local, params_dst: Sequence,
                               param_dtype, workspace, stream=None) -> None:
    p, kind = plan.p, _dtype_name(param_dtype)
    dst = (ctypes.c_void_p * len(params_dst))(
        *[_buf(d, kind, p, f"params_dst[{i}]") for i, d in enumerate(params_dst)])
    _check(lib.zero_step_update_partition(
        plan.handle, rank, _buf(master_local, "f32", p, "master_local"),
        _buf(exp_avg_local, "f32", p, "exp_avg_local"),
        _buf(exp_avg_sq_local, "f32", p, "exp_avg_sq_local"),
        _buf(reduced_local, "f32", p, "reduced_local"), dst, len(params_dst),
        _dtype(param_dtype), _buf(workspace, "bytes", plan.workspace_bytes(), "workspace"),
        _stream(stream)))


def zero_ipc_get_handle(device_ptr) -> tuple:
    """(handle bytes, byte offset of the pointer in its allocation)."""
    buf = ctypes.create_string_buffer(lib.zero_ipc_handle_bytes())
    off = ctypes.c_int64()
    _check(lib.zero_ipc_get_handle(_addr(device_ptr), buf, ctypes.byref(off)))
    return buf.raw, off.value


def zero_ipc_open_handle(handle: bytes) -> int:
    """Start of the peer's mapped allocation (add the exporter's offset)."""
    p = ctypes.c_void_p()
    _check(lib.zero_ipc_open_handle(ctypes.create_string_buffer(handle, len(handle)),
                                    ctypes.byref(p)))
    return int(p.value)


def zero_ipc_close(base: int) -> None:
    _check(lib.zero_ipc_close(ctypes.c_void_p(base)))


def zero_reduce_sumsq_noalloc(world_size: int, grad_dtype, replica_grads: Sequence, n: int,
                              reduced, sumsq, stream=None) -> None:
    _check(lib.zero_reduce_sumsq_noalloc(world_size, _dtype(grad_dtype), _ptr_array(replica_grads),
                                         int(n), _addr(reduced), _addr(sumsq), _stream(stream)))


from .optimizer import ZeroOptimizer  # noqa: E402  (torch plumbing around the calls above)
