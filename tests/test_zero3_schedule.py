"""The ZeRO-3 fetch / release scheduler: the library's C++ scheduler against the oracle's
plain simulation (random layer structures and knobs), a hand-derived golden schedule,
and invariants checked by replaying the events."""
import os

import numpy as np
import pytest

from oracle import zero3 as oz3
import zero_sharded_mixed_replica_b200 as zb

OPS = {zb.ZERO3_FETCH: "FETCH", zb.ZERO3_COMPUTE: "COMPUTE", zb.ZERO3_RELEASE: "RELEASE"}
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "zero3_schedule.txt")


def _lib_schedule(numels, layers, n_layers, pb, ml, pt):
    plan = zb.Plan([(n,) for n in numels], 1, 1 << 30, 1)
    s = zb.Zero3Schedule(plan, layers, n_layers, pb, ml, pt)
    return [(OPS[o], l, ids) for o, l, ids in s.events], s.stats


def test_golden_schedule():
    lines = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    numels = [int(x) for x in lines[0][1:]]
    layers = [int(x) for x in lines[1][1:]]
    pb, ml, pt = (int(x) for x in lines[2][1:])
    want = [(l[0], int(l[1]), [int(x) for x in l[2:]]) for l in lines[3:-1]]
    stats = [int(x) for x in lines[-1][1:]]
    ev, st = _lib_schedule(numels, layers, 3, pb, ml, pt)
    assert ev == want
    assert [st[k] for k in ("peak_live_elements", "fetched_elements", "fetch_events",
                            "persistent_elements", "over_budget_layers")] == stats
    ev2, st2 = oz3.schedule(numels, layers, 3, pb, ml, pt)
    assert ev2 == want and st2 == st


def _replay_invariants(numels, layers, n_layers, pb, ml, pt, events, stats):
    live, fetched = set(), []
    persistent = {t for t in range(len(numels)) if layers[t] >= 0 and numels[t] <= pt}
    computed = []
    for op, l, ids in events:
        if op == "FETCH":
            assert not (set(ids) & live)
            live.update(ids)
            fetched += ids
        elif op == "COMPUTE":
            need = {t for t in range(len(numels)) if layers[t] == l}
            assert need <= live, l  # every tensor of the layer is there
            computed.append(l)
        else:
            assert set(ids) == {t for t in range(len(numels)) if layers[t] == l} - persistent
            live.difference_update(ids)
    assert computed == list(range(n_layers))
    used = [t for t in range(len(numels)) if layers[t] >= 0]
    assert sorted(fetched) == sorted(used)  # each used tensor gathered exactly once
    assert live == persistent
    assert stats["fetched_elements"] == sum(numels[t] for t in used)


@pytest.mark.parametrize("seed", range(60))
def test_scheduler_matches_oracle(seed):
    rng = np.random.default_rng(seed)
    n_layers = int(rng.integers(0, 7))
    nt = int(rng.integers(0, 25))
    numels = [int(x) for x in rng.integers(1, 500, nt)]
    layers = [int(x) for x in rng.integers(-1, max(n_layers, 1), nt)] if n_layers else [-1] * nt
    pb, ml, pt = int(rng.integers(0, 1500)), int(rng.integers(0, 3000)), int(rng.integers(0, 50))
    ev, st = _lib_schedule(numels, layers, n_layers, pb, ml, pt)
    ev2, st2 = oz3.schedule(numels, layers, n_layers, pb, ml, pt)
    assert ev == ev2
    assert st == st2
    _replay_invariants(numels, layers, n_layers, pb, ml, pt, ev, st)


def test_llama_layers_budget():
    # the 7B tensor list, one layer per transformer block (embedding first, head last)
    import synthgen
    wl = synthgen.workload("llama7b")
    layer_of = []
    for t in wl.tensors:
        if t.name.startswith("model.layers."):
            layer_of.append(int(t.name.split(".")[2]) + 1)
        elif t.name.startswith("model.embed"):
            layer_of.append(0)
        else:
            layer_of.append(33)
    plan = zb.Plan([t.shape for t in wl.tensors], 8, 500_000_000)
    s = zb.Zero3Schedule(plan, layer_of, 34, 500_000_000, 1_000_000_000, 1_000_000)
    st = s.stats
    assert st["persistent_elements"] == 65 * 4096  # every RMSNorm weight stays resident
    assert st["fetched_elements"] == wl.n
    assert st["peak_live_elements"] <= 1_000_000_000 + st["persistent_elements"]
    assert st["over_budget_layers"] == 0
