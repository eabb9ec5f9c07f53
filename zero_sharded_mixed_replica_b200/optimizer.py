"""ZeroOptimizer: device buffers for one ZeRO partitioned optimizer (torch allocates them,
the library's kernels do all the work).

Buffers, all flat over the padded parameter space of the plan (n_pad elements):
  master, exp_avg, exp_avg_sq  fp32   rank r owns [r*p, (r+1)*p) of each
  reduced                      fp32   reduce-scattered gradient, same ownership
  params                       half   the gathered parameter buffer
  workspace                    bytes  scaler state, partial sums, step result
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import (AdamWCfg, Plan, ScalerCfg, adamw_cfg, scaler_cfg, zero_all_gather,
               zero_cast_params, zero_get_result, zero_reduce_scatter_bucket,
               zero_reduce_scatter_bucket_accum, zero_reduce_scatter_bucket_host,
               zero_state_init, zero_step, zero_step_finalize, zero_step_full,
               zero_step_resident, zero_step_update)

_TORCH_HALF = {"bf16": torch.bfloat16, "fp16": torch.float16}


class ZeroOptimizer:
    def __init__(self, shapes: Sequence[Sequence[int]], world_size: int,
                 reduce_bucket_size: int, dtype: str = "bf16", align: int = 128,
                 scaler: Optional[ScalerCfg] = None, adamw: Optional[AdamWCfg] = None,
                 device: str = "cuda", stream: Optional[torch.cuda.Stream] = None):
        self.plan = Plan(shapes, world_size, reduce_bucket_size, align)
        self.dtype = dtype
        self.device = torch.device(device)
        self.stream = stream
        n = self.plan.n_pad
        f32 = dict(dtype=torch.float32, device=self.device)
        self.master = torch.zeros(n, **f32)
        self.exp_avg = torch.zeros(n, **f32)
        self.exp_avg_sq = torch.zeros(n, **f32)
        self.reduced = torch.zeros(n, **f32)
        self.params = torch.zeros(n, dtype=_TORCH_HALF[dtype], device=self.device)
        self.workspace = torch.zeros(self.plan.workspace_bytes(), dtype=torch.uint8,
                                     device=self.device)
        self.scaler = scaler if scaler is not None else scaler_cfg(dynamic=(dtype == "fp16"))
        self.adamw = adamw if adamw is not None else adamw_cfg()
        # the buffers allocated here are passed by address (the binding checks tensor
        # arguments, which costs host time on small steps); one that a caller has
        # replaced is passed as a tensor and checked
        self._own = {k: (getattr(self, k), getattr(self, k).data_ptr()) for k in
                     ("master", "exp_avg", "exp_avg_sq", "reduced", "params", "workspace")}
        zero_state_init(self.plan, self.workspace, self.scaler, self._s())

    def _b(self, name: str):
        t = getattr(self, name)
        own = self._own[name]
        return own[1] if own[0] is t else t

    def _s(self):
        return self.stream.cuda_stream if self.stream is not None else \
            torch.cuda.current_stream(self.device).cuda_stream

    # -------------------------------------------------------------- step pieces
    def cast_params(self) -> None:
        """params <- round_to_nearest_even(master): after initialising or loading master."""
        zero_cast_params(self.plan, self._b("master"), self._b("params"), self.dtype, self._s())

    def reduce_scatter_bucket(self, bucket: int, replica_grads: Sequence, base_offset: int = 0):
        zero_reduce_scatter_bucket(self.plan, bucket, self.dtype, replica_grads, base_offset,
                                   self._b("reduced"), self._b("workspace"), self._s())

    def reduce_scatter_bucket_accum(self, bucket: int, micro: int, n_micro: int,
                                    replica_grads: Sequence, base_offset: int = 0):
        """Micro-batch `micro` of `n_micro` (gradient accumulation) for one bucket."""
        zero_reduce_scatter_bucket_accum(self.plan, bucket, micro, n_micro, self.dtype,
                                         replica_grads, base_offset, self._b("reduced"),
                                         self._b("workspace"), self._s())

    def reduce_scatter_bucket_host(self, bucket: int, host_replica_grads: Sequence,
                                   host_base_offset: int, device_staging: Sequence):
        zero_reduce_scatter_bucket_host(self.plan, bucket, self.dtype, host_replica_grads,
                                        host_base_offset, device_staging, self._b("reduced"),
                                        self._b("workspace"), self._s())

    def step(self) -> None:
        zero_step(self.plan, self.adamw, self._b("master"), self._b("exp_avg"),
                  self._b("exp_avg_sq"), self._b("reduced"), self._b("params"), self.dtype,
                  self._b("workspace"), self._s())

    def step_finalize(self) -> None:
        zero_step_finalize(self.plan, self.adamw, self._b("workspace"), self._s())

    def step_update(self) -> None:
        zero_step_update(self.plan, self._b("master"), self._b("exp_avg"),
                         self._b("exp_avg_sq"), self._b("reduced"), self._b("params"),
                         self.dtype, self._b("workspace"), self._s())

    def all_gather(self, rank_params: Sequence = ()) -> None:
        zero_all_gather(self.plan, self._b("params"), list(rank_params), self.dtype, self._s())

    def result(self) -> dict:
        """Step result; synchronises the stream."""
        return zero_get_result(self._b("workspace"), self._s())

    # -------------------------------------------------------------- whole step
    def full_step(self, replica_grads: Sequence, base_offset: int = 0) -> None:
        """Reduce-scatter every bucket from whole-model replica buffers, then step (one
        library call)."""
        zero_step_full(self.plan, self.adamw, self.dtype, replica_grads, base_offset,
                       self._b("reduced"), self._b("master"), self._b("exp_avg"),
                       self._b("exp_avg_sq"), self._b("params"), self.dtype,
                       self._b("workspace"), self._s())

    def step_resident(self, replica_grads: Sequence) -> None:
        """The whole step from whole-model replica buffers that stay resident, for
        world_size <= 2: the update re-reads the replicas instead of a stored reduced
        gradient (4W + 26 instead of 2W + 34 bytes per parameter); results are the same
        bits as full_step. `reduced` is not written."""
        zero_step_resident(self.plan, self.adamw, self.dtype, replica_grads, self._b("master"),
                           self._b("exp_avg"), self._b("exp_avg_sq"), self._b("params"),
                           self.dtype, self._b("workspace"), self._s())

    def overlapped_step(self, produce, slots: Sequence[Sequence], producer_stream) -> None:
        """One step whose reduce-scatter of bucket b overlaps the production of the next
        buckets (the pages' overlap_comm). `produce(b, bufs, stream)` enqueues on `stream`
        (the producer's, a raw handle) the writes of bucket b's W replica gradients into
        `bufs`, one of the `slots` (each a list of W buffers of at least one bucket,
        indexed from the bucket start). Bucket b goes to slot b % len(slots); it is reduced
        on this optimizer's stream as soon as it has been written, and the slot goes back
        to the producer once the reduction has read it. With two slots the reduction of
        bucket b runs while bucket b + 1 is produced. Events order the two streams; the
        host never waits."""
        cons = self.stream if self.stream is not None else torch.cuda.current_stream(self.device)
        n = len(slots)
        ev = getattr(self, "_slot_events", None)
        if ev is None or len(ev) != n:
            ev = self._slot_events = [(torch.cuda.Event(), torch.cuda.Event()) for _ in range(n)]
        for b in range(self.plan.n_buckets):
            ready, free = ev[b % n]
            producer_stream.wait_event(free)  # the slot's previous bucket has been read
            with torch.cuda.stream(producer_stream):
                produce(b, slots[b % n], producer_stream.cuda_stream)
            ready.record(producer_stream)
            cons.wait_event(ready)
            self.reduce_scatter_bucket(b, slots[b % n], base_offset=self.plan.bucket(b)[0])
            free.record(cons)
        self.step()

    def capture_step(self, replica_grads: Sequence, base_offset: int = 0) -> torch.cuda.CUDAGraph:
        """A CUDA graph of one full step over fixed replica buffers (every launch of the
        step, no host work): `graph.replay()` runs a step. The step allocates nothing and
        never synchronises, so it captures as is; the loss-scaler state stays on the device,
        so replays keep skipping, scaling and counting steps like eager calls. Capture on a
        side stream, as CUDA graphs require; the plan's host bookkeeping sees one step."""
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        keep = self.stream
        self.stream = side
        try:
            with torch.cuda.stream(side), torch.cuda.graph(graph, stream=side):
                self.full_step(replica_grads, base_offset)
        finally:
            self.stream = keep
        torch.cuda.current_stream(self.device).wait_stream(side)
        return graph
