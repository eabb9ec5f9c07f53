"""ZeRO-3 forward pass over partitioned half parameters: runs a Zero3Schedule, gathering
each FETCH into a device buffer (zero3_gather), handing every layer views of its full
tensors, and dropping a buffer once all of its tensors are released.

On one GPU the ranks' partitions are the W slices of the gathered buffer the update
writes; in a multi-process run they are the ranks' own partition buffers, mapped over
CUDA IPC.
"""
from __future__ import annotations

from typing import Callable, Dict, List, Sequence

import torch

from . import Plan, ZERO3_COMPUTE, ZERO3_FETCH, ZERO3_RELEASE, Zero3Schedule, zero3_gather


def partitions_of(params: torch.Tensor, plan: Plan) -> List[int]:
    """Device addresses of the W partitions inside a gathered buffer."""
    p, esz = plan.p, params.element_size()
    return [params.data_ptr() + r * p * esz for r in range(plan.world_size)]


def run_forward(plan: Plan, schedule: Zero3Schedule, partitions: Sequence[int],
                dtype: torch.dtype, on_layer: Callable[[int, Dict[int, torch.Tensor]], None],
                device="cuda", stream=None) -> dict:
    """Executes the schedule; `on_layer(layer, {tensor id: flat view})` stands for the
    layer's forward computation. Returns live-memory statistics in elements."""
    table = plan.tensor_table
    live: Dict[int, tuple] = {}      # tensor id -> (buffer id, offset)
    buffers: Dict[int, list] = {}    # buffer id -> [tensor, remaining tensors]
    next_id, live_elems, peak = 0, 0, 0
    s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    for op, layer, ids in schedule.events:
        if op == ZERO3_FETCH:
            sizes = [table[t][1] for t in ids]
            buf = torch.empty(sum(sizes), dtype=dtype, device=device)
            # sized here for exactly these tensors: passed by address, unchecked
            zero3_gather(plan, ids, partitions, buf.data_ptr(), s)
            off = 0
            for t, n in zip(ids, sizes):
                live[t] = (next_id, off)
                off += n
            buffers[next_id] = [buf, len(ids)]
            next_id += 1
            live_elems += sum(sizes)
            peak = max(peak, live_elems)
        elif op == ZERO3_COMPUTE:
            views = {t: buffers[b][0][off:off + table[t][1]] for t, (b, off) in live.items()}
            on_layer(layer, views)
        elif op == ZERO3_RELEASE:
            for t in ids:
                b, _ = live.pop(t)
                live_elems -= table[t][1]
                buffers[b][1] -= 1
                if buffers[b][1] == 0:
                    del buffers[b]
    return {"peak_live_elements": peak, "buffers_left": len(buffers)}
