"""Device-side fills of the seeded synthetic inputs (harness only; before any timed
region). Same recipe and bits as the host fills in ``synthgen``."""
from __future__ import annotations

from typing import Sequence

import torch

from . import (FP16, grads_cuda, master_random_cuda)


def init_master(wl, master: torch.Tensor, stream: int) -> None:
    """master[:] <- the workload's initial fp32 weights (padding zero)."""
    master.zero_()
    off = 0
    for t in wl.tensors:
        if t.init == "normal":
            master_random_cuda(master.data_ptr() + 4 * off, off, t.numel, wl.seed,
                               wl.init_sigma, stream)
        elif t.init == "ones":
            master[off:off + t.numel].fill_(1.0)
        off += t.numel


def fill_grads(wl, bufs: Sequence[torch.Tensor], j0: int, n: int, t: int, scale: float,
               stream: int, micro: int = 0) -> None:
    """bufs[r][0:n] <- replica r's gradient bits at buffer indices j0 .. j0+n-1, step t
    (micro-batch `micro` of a resident workload with gradient accumulation)."""
    slot = wl.micro_slot(t, micro) if not wl.streaming else wl.slot(t)
    for r, b in enumerate(bufs):
        grads_cuda(b.data_ptr(), j0, n, wl.seed, r, slot, wl.grad_sigma, wl.spike_frac,
                   scale, wl.dtype_code, stream)


def plant_infs(wl, bufs: Sequence[torch.Tensor], t: int, bucket: int = 0) -> None:
    """Write +inf at step t's injection sites. Resident buffers are indexed by flat index;
    streaming (bucket-sized) ones by flat index minus its bucket start."""
    bits = 0x7C00 if wl.dtype_code == FP16 else 0x7F80
    for idx, rep in wl.inf_sites_at(t):
        j = idx - (idx // bucket) * bucket if wl.streaming else idx
        bufs[rep].view(torch.int16)[j] = torch.tensor(bits, dtype=torch.int32).to(torch.int16)
