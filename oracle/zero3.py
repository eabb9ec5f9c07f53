"""Oracle of the ZeRO-3 fetch / release schedule (TEST INFRASTRUCTURE).

A plain simulation of the policy the library implements for the stage-3 knobs named on
"ZeRO技术解析" 1.2.3 / 3.1 / 6 (stage3_prefetch_bucket_size, stage3_max_live_parameters,
stage3_param_persistence_threshold) and the per-layer gather-then-release of "ZeRO 和分片优
化器" (technical insight): persistent tensors (numel <= threshold) fetched once first;
before each layer its missing tensors (forced); then later tensors in order while the
elements fetched ahead stay <= the prefetch bucket and the live elements <= the budget;
the layer computes; its tensors are released. Written without the library's cursor: it
rescans the future tensors from the start every time.
"""
from typing import List, Sequence, Tuple


def schedule(numels: Sequence[int], layer_of_tensor: Sequence[int], n_layers: int,
             prefetch: int, max_live: int, persist: int) -> Tuple[List[tuple], dict]:
    layers = [[t for t in range(len(numels)) if layer_of_tensor[t] == l and numels[t] > persist]
              for l in range(n_layers)]
    persistent = [t for t in range(len(numels)) if layer_of_tensor[t] >= 0 and numels[t] <= persist]
    events, live = [], set()
    stats = dict(peak_live_elements=0, fetched_elements=0, fetch_events=0,
                 persistent_elements=sum(numels[t] for t in persistent), over_budget_layers=0)
    if persistent:
        events.append(("FETCH", -1, list(persistent)))
        stats["fetch_events"] += 1
        stats["fetched_elements"] += stats["persistent_elements"]
    for i in range(n_layers):
        need = [t for t in layers[i] if t not in live]
        if need:
            live.update(need)
            events.append(("FETCH", i, need))
            stats["fetch_events"] += 1
            stats["fetched_elements"] += sum(numels[t] for t in need)
            if sum(numels[t] for t in live) > max_live:
                stats["over_budget_layers"] += 1
        pre = []
        future = [t for l in range(i + 1, n_layers) for t in layers[l]]
        for t in future:
            if t in live:
                continue
            ahead = sum(numels[u] for u in future if u in live)
            if ahead + numels[t] > prefetch or sum(numels[u] for u in live) + numels[t] > max_live:
                break
            live.add(t)
            pre.append(t)
        if pre:
            events.append(("FETCH", i, pre))
            stats["fetch_events"] += 1
            stats["fetched_elements"] += sum(numels[t] for t in pre)
        stats["peak_live_elements"] = max(stats["peak_live_elements"],
                                          sum(numels[t] for t in live) + stats["persistent_elements"])
        events.append(("COMPUTE", i, []))
        if layers[i]:
            events.append(("RELEASE", i, list(layers[i])))
        live.difference_update(layers[i])
    return events, stats
