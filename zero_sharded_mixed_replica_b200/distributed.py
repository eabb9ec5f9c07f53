"""The ZeRO step across W processes, one GPU each (rank r owns partition r).

The orders of work and exchange live in `DistributedZeroStep`; what runs on a device
lives in a backend. `CudaRankBackend` is the product backend: peers' gradient and
gathered-parameter buffers are mapped into each process with CUDA IPC, the
reduce-scatter reads them over NVLink inside the bucket kernel (rank-ordered fp32 sum,
as on one GPU), and the update writes this rank's half values into every rank's
gathered buffer (the all-gather fused into the update) -- or, with
`fused_all_gather=False`, into its own buffer followed by a collective all-gather.
The only collectives are one all-gather of the W fp64 sums of squares (rank order, so
every rank computes the same norm, clip and loss-scale decision) and the stream-ordered
barriers that separate writers from peer readers. With `host_exchange=True` those
exchanges go through the host instead (a device synchronize, then a CPU collective, e.g.
gloo): slower, but no device work ever waits on another process's device work, which is
what ranks that share one GPU need.

Sources: [Z1] "ZeRO技术解析" 2.1 (parameters split into N parts, gradients
reduce-scattered, each GPU updates its own partition, parameters gathered with
all-gather) and 2.2 (bucketed communication); [Z3] "ZeRO 和分片优化器" technical
insight (each GPU keeps only its own gradient slice).
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from . import (AdamWCfg, Plan, ScalerCfg, adamw_cfg, scaler_cfg, zero_get_result,
               zero_ipc_close, zero_ipc_get_handle, zero_ipc_open_handle,
               zero_reduce_scatter_segment, zero_state_init, zero_step_finalize_ranks,
               zero_step_local_sumsq, zero_step_update_partition)

_TORCH_HALF = {"bf16": torch.bfloat16, "fp16": torch.float16}


def allgather_chunks(p: int, allgather_bucket_size: Optional[int]) -> List[Tuple[int, int]]:
    """[start, end) ranges of a partition of p elements gathered one bucket at a time
    ([Z2] ds_config allgather_bucket_size, counted in elements like reduce_bucket_size);
    None or a size >= p gathers the partition at once."""
    if p <= 0:
        return []
    b = p if not allgather_bucket_size or allgather_bucket_size >= p else int(allgather_bucket_size)
    return [(c, min(c + b, p)) for c in range(0, p, b)]


def partition_buckets(plan_n_pad: int, world: int, bucket: int, rank: int) -> range:
    """Buckets that meet partition `rank` (each such bucket holds exactly one of the
    rank's work segments)."""
    p = plan_n_pad // world
    if p == 0:
        return range(0)
    lo, hi = rank * p, (rank + 1) * p
    return range(lo // bucket, (hi - 1) // bucket + 1)


class DistributedZeroStep:
    """One optimizer step on this rank. `backend` does the device work; `group` is the
    process group of the W ranks (NCCL for CUDA tensors, gloo for CPU tensors)."""

    def __init__(self, backend, group=None):
        self.backend = backend
        self.group = group
        self.rank = backend.rank
        self.world = backend.world
        self.buckets = partition_buckets(backend.n_pad, self.world, backend.bucket, self.rank)

    def step(self):
        be = self.backend
        # every rank has finished writing this step's gradients before any peer reads them
        be.before_peer_reads(self.group)
        for b in self.buckets:
            be.reduce_segment(b)
        s_local = be.local_sumsq()
        s_all = torch.empty(self.world, dtype=torch.float64, device=s_local.device)
        dist.all_gather_into_tensor(s_all, s_local, group=self.group)
        be.finalize(s_all)
        be.update()
        be.after_update(self.group)
        return be


class CudaRankBackend:
    """Device side of one rank: plan, workspace, the rank's fp32 partition state and
    reduced gradient (p elements each), its whole-model replica gradient buffer and
    gathered half buffer (n_pad each), and IPC mappings of every peer's two buffers."""

    def __init__(self, shapes: Sequence[Sequence[int]], reduce_bucket_size: int, dtype: str,
                 rank: int, world: int, group=None, align: int = 128,
                 scaler: Optional[ScalerCfg] = None, adamw: Optional[AdamWCfg] = None,
                 fused_all_gather: bool = True, device: Optional[torch.device] = None,
                 host_exchange: bool = False, allgather_bucket_size: Optional[int] = None):
        self.rank, self.world, self.dtype = rank, world, dtype
        self.device = device or torch.device("cuda", torch.cuda.current_device())
        self.plan = Plan(shapes, world, reduce_bucket_size, align)
        self.n_pad, self.p, self.bucket = self.plan.n_pad, self.plan.p, reduce_bucket_size
        f32 = dict(dtype=torch.float32, device=self.device)
        self.master = torch.zeros(self.p, **f32)
        self.exp_avg = torch.zeros(self.p, **f32)
        self.exp_avg_sq = torch.zeros(self.p, **f32)
        self.reduced = torch.zeros(self.p, **f32)
        self.grads = torch.zeros(self.n_pad, dtype=_TORCH_HALF[dtype], device=self.device)
        self.params = torch.zeros(self.n_pad, dtype=_TORCH_HALF[dtype], device=self.device)
        self.workspace = torch.zeros(self.plan.workspace_bytes(), dtype=torch.uint8,
                                     device=self.device)
        self.sumsq = torch.zeros(1, dtype=torch.float64, device=self.device)
        self.scaler = scaler if scaler is not None else scaler_cfg(dynamic=(dtype == "fp16"))
        self.adamw = adamw if adamw is not None else adamw_cfg()
        self.fused_all_gather = fused_all_gather
        self.host_exchange = host_exchange
        self.gather_chunks = allgather_chunks(self.p, allgather_bucket_size)
        zero_state_init(self.plan, self.workspace, self.scaler, self._s())
        # peers' buffers, mapped once (IPC handles travel through the process group). A
        # handle names a whole allocation, which may hold both buffers: each distinct
        # allocation is mapped once and the exporter's offset places the buffer in it.
        mine = (zero_ipc_get_handle(self.grads), zero_ipc_get_handle(self.params))
        handles: List = [None] * world
        dist.all_gather_object(handles, mine, group=group)
        self._opened: Dict[bytes, int] = {}

        def peer(h) -> int:
            key, off = h
            if key not in self._opened:
                self._opened[key] = zero_ipc_open_handle(key)
            return self._opened[key] + off

        self.peer_grads, self.peer_params = [], []
        for q in range(world):
            if q == rank:
                self.peer_grads.append(self.grads.data_ptr())
                self.peer_params.append(self.params.data_ptr())
            else:
                self.peer_grads.append(peer(handles[q][0]))
                self.peer_params.append(peer(handles[q][1]))

    def _s(self) -> int:
        return torch.cuda.current_stream(self.device).cuda_stream

    def close(self) -> None:
        """Unmap the peers' allocations (every rank must be done reading and writing
        them, and must call this before any rank frees its buffers)."""
        for base in self._opened.values():
            zero_ipc_close(base)
        self._opened = {}

    def own_slice(self) -> torch.Tensor:
        return self.params[self.rank * self.p:(self.rank + 1) * self.p]

    # ---- the step
    def _host_barrier(self, group) -> None:
        torch.cuda.synchronize(self.device)
        dist.barrier(group=group)

    def before_peer_reads(self, group) -> None:
        if self.host_exchange:
            self._host_barrier(group)
            return
        # stream-ordered barrier: a rank's gradient writes precede its all-reduce, which
        # no rank completes before all have entered it
        flag = torch.zeros(1, device=self.device)
        dist.all_reduce(flag, group=group)

    def reduce_segment(self, b: int) -> None:
        zero_reduce_scatter_segment(self.plan, b, self.rank, self.dtype, self.peer_grads, 0,
                                    self.reduced, self.workspace, self._s())

    def local_sumsq(self) -> torch.Tensor:
        zero_step_local_sumsq(self.plan, self.rank, self.workspace, self.sumsq, self._s())
        return self.sumsq.cpu() if self.host_exchange else self.sumsq

    def finalize(self, s_all: torch.Tensor) -> None:
        if self.host_exchange:
            s_all = s_all.to(self.device)
        zero_step_finalize_ranks(self.plan, self.adamw, s_all, self.workspace, self._s())

    def update(self) -> None:
        off = 2 * self.rank * self.p  # bytes to this rank's slice of a gathered buffer
        base = self.peer_params if self.fused_all_gather else [self.params.data_ptr()]
        dst = [q + off for q in base]
        zero_step_update_partition(self.plan, self.rank, self.master, self.exp_avg,
                                   self.exp_avg_sq, self.reduced, dst, self.dtype,
                                   self.workspace, self._s())

    def after_update(self, group) -> None:
        if self.host_exchange:
            if not self.fused_all_gather:
                # one bucket of every rank's slice at a time; the halves travel as bytes
                # (gloo has no 16-bit float types)
                own = self.own_slice().cpu().view(torch.uint8)
                for c0, c1 in self.gather_chunks:
                    parts = [torch.empty(2 * (c1 - c0), dtype=torch.uint8)
                             for _ in range(self.world)]
                    dist.all_gather(parts, own[2 * c0:2 * c1].contiguous(), group=group)
                    for q, part in enumerate(parts):
                        lo = q * self.p
                        self.params[lo + c0:lo + c1].copy_(
                            part.view(self.params.dtype).to(self.device))
            # the peers' stores into this buffer (or the copies above) have landed, and
            # every rank is done reading the peers' gradients
            self._host_barrier(group)
            return
        if self.fused_all_gather:
            # every rank's stores into the peers' gathered buffers have landed before any
            # rank uses its buffer
            flag = torch.zeros(1, device=self.device)
            dist.all_reduce(flag, group=group)
        elif len(self.gather_chunks) == 1:
            dist.all_gather_into_tensor(self.params, self.own_slice().clone(), group=group)
        else:
            own = self.own_slice().clone()
            for c0, c1 in self.gather_chunks:
                dist.all_gather([self.params[q * self.p + c0:q * self.p + c1]
                                 for q in range(self.world)], own[c0:c1], group=group)

    def result(self) -> dict:
        return zero_get_result(self.workspace, self._s())
