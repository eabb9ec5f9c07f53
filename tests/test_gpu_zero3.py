"""ZeRO-3 gather of layer tensors from the ranks' parameter partitions (one GPU: the W
slices of the gathered buffer) and a forward pass driven by the schedule: every layer
sees exactly its tensors' values, and every buffer is dropped at the end."""
import numpy as np
import pytest
import torch

import synthgen
import zero_sharded_mixed_replica_b200 as zb
from zero_sharded_mixed_replica_b200 import zero3

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world,align", [(1, 1), (3, 1), (8, 8), (16, 128)])
def test_gather_bit_exact(world, align):
    rng = np.random.default_rng(world)
    shapes = [(int(rng.integers(1, 5000)),) for _ in range(90)] + [(70001,), (3,), (1,)]
    plan = zb.Plan(shapes, world, 1 << 20, align)
    params = torch.randint(-32768, 32767, (plan.n_pad,), dtype=torch.int16, device="cuda").view(torch.bfloat16)
    parts = zero3.partitions_of(params, plan)
    for trial in range(4):
        ids = [int(x) for x in rng.choice(len(shapes), size=int(rng.integers(1, 80)), replace=False)]
        total = sum(plan.tensor(t)[1] for t in ids)
        dst = torch.full((total + 1,), 7, dtype=torch.int16, device="cuda")
        zb.zero3_gather(plan, ids, parts, dst[:total].view(torch.bfloat16))
        want = torch.cat([params.view(torch.int16)[o:o + n] for o, n in (plan.tensor(t) for t in ids)])
        assert torch.equal(dst[:total], want)
        assert int(dst[total]) == 7  # nothing written past the end


def test_forward_pass_over_gpt2_layers():
    wl = synthgen.workload("gpt2")
    layer_of = []
    for t in wl.tensors:
        layer_of.append(int(t.name.split(".")[1]) + 1 if t.name.startswith("h.") else
                        (0 if t.name.startswith("w") else 25))
    plan = zb.Plan([t.shape for t in wl.tensors], 8, 200_000_000)
    params = torch.randint(-32768, 32767, (plan.n_pad,), dtype=torch.int16,
                           device="cuda").view(torch.bfloat16)
    sched = zb.Zero3Schedule(plan, layer_of, 26, 50_000_000, 120_000_000, 100_000)
    seen = []

    def on_layer(layer, views):
        for t, v in views.items():
            o, n = plan.tensor(t)
            assert torch.equal(v.view(torch.int16), params.view(torch.int16)[o:o + n])
        mine = {t for t, l in enumerate(layer_of) if l == layer}
        assert mine <= set(views)
        seen.append(layer)

    out = zero3.run_forward(plan, sched, zero3.partitions_of(params, plan), torch.bfloat16,
                            on_layer)
    assert seen == list(range(26))
    assert out["peak_live_elements"] == sched.stats["peak_live_elements"]
    assert out["buffers_left"] == 1  # the persistent tensors' buffer
