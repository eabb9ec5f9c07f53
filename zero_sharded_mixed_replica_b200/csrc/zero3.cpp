// zero3.cpp -- the ZeRO-3 parameter fetch / release schedule (host only).
//
// [Z1] "ZeRO技术解析" 1.2.3 (parameters themselves partitioned; sub_group_size,
// stage3_prefetch_bucket_size), 3.1 (stage3_max_live_parameters 1e9), 5.1 (lower
// stage3_max_live_parameters on OOM), 5.2 (stage3_prefetch overlaps communication with
// compute), 6 (stage3_param_persistence_threshold 1e6); [Z2] (the other parts are
// all-gathered during the forward pass and released right after use); [Z3] technical
// insight (before a layer's forward its full parameters are all-gathered; afterwards the
// slices a GPU does not own are dropped). The pages name the knobs only; the policy
// below is the reading this library implements.
#include <stdint.h>

#include <new>
#include <string>
#include <vector>

#include "zero_b200.h"
#include "zero_internal.h"

struct zero3_schedule {
  std::vector<zero3_event> events;
  std::vector<int32_t> tensors;  // the tensor ids the events reference
  zero3_stats stats{};
};

using namespace zero;

extern "C" {

int zero3_schedule_create(const zero_plan* plan, const int32_t* layer_of_tensor,
                          int32_t n_layers, int64_t prefetch_bucket_size,
                          int64_t max_live_parameters, int64_t persistence_threshold,
                          zero3_schedule** out) {
  if (!plan || !out || (!layer_of_tensor && !plan->numel.empty()))
    return fail(ZERO_EINVAL, "NULL argument");
  *out = nullptr;
  if (n_layers < 0) return fail(ZERO_EINVAL, "n_layers < 0");
  if (prefetch_bucket_size < 0 || max_live_parameters < 0 || persistence_threshold < 0)
    return fail(ZERO_EINVAL, "knobs must be >= 0");
  const int32_t nt = (int32_t)plan->numel.size();
  for (int32_t t = 0; t < nt; ++t)
    if (layer_of_tensor[t] < -1 || layer_of_tensor[t] >= n_layers)
      return fail(ZERO_EINVAL, "layer_of_tensor[" + std::to_string(t) + "] out of range");
  zero3_schedule* s = new (std::nothrow) zero3_schedule();
  if (!s) return fail(ZERO_ENOMEM, "schedule allocation failed");
  try {
    // tensors of each layer in declared order; persistent ones apart
    std::vector<std::vector<int32_t>> layer(n_layers);
    std::vector<int32_t> persistent;
    for (int32_t t = 0; t < nt; ++t) {
      if (layer_of_tensor[t] < 0) continue;  // not used in the forward pass
      if (plan->numel[t] <= persistence_threshold)
        persistent.push_back(t);
      else
        layer[layer_of_tensor[t]].push_back(t);
    }
    auto emit = [&](int32_t op, int32_t l, const std::vector<int32_t>& ts) {
      if (ts.empty() && op != ZERO3_COMPUTE) return;
      zero3_event e{op, l, (int64_t)s->tensors.size(), (int64_t)ts.size()};
      s->tensors.insert(s->tensors.end(), ts.begin(), ts.end());
      s->events.push_back(e);
    };
    int64_t persistent_elems = 0;
    for (int32_t t : persistent) persistent_elems += plan->numel[t];
    if (!persistent.empty()) {
      emit(ZERO3_FETCH, -1, persistent);
      s->stats.fetch_events += 1;
      s->stats.fetched_elements += persistent_elems;
    }
    s->stats.persistent_elements = persistent_elems;

    std::vector<uint8_t> live(nt, 0);
    int64_t live_total = 0;
    int32_t next_layer = 0;  // prefetch cursor: (layer, index in layer)
    size_t next_index = 0;
    for (int32_t i = 0; i < n_layers; ++i) {
      // demand: this layer's tensors that are not live yet (even over the live budget)
      std::vector<int32_t> need;
      for (int32_t t : layer[i])
        if (!live[t]) need.push_back(t);
      for (int32_t t : need) {
        live[t] = 1;
        live_total += plan->numel[t];
        s->stats.fetched_elements += plan->numel[t];
      }
      if (!need.empty()) {
        emit(ZERO3_FETCH, i, need);
        s->stats.fetch_events += 1;
        if (live_total > max_live_parameters) s->stats.over_budget_layers += 1;
      }
      // prefetch: later layers' tensors in order while both bounds hold
      if (next_layer <= i) {
        next_layer = i + 1;
        next_index = 0;
      }
      int64_t ahead = 0;
      for (int32_t l = i + 1; l < n_layers; ++l)
        for (int32_t t : layer[l])
          if (live[t]) ahead += plan->numel[t];
      std::vector<int32_t> pre;
      while (next_layer < n_layers) {
        if (next_index >= layer[next_layer].size()) {
          ++next_layer;
          next_index = 0;
          continue;
        }
        const int32_t t = layer[next_layer][next_index];
        const int64_t n = plan->numel[t];
        if (ahead + n > prefetch_bucket_size || live_total + n > max_live_parameters) break;
        live[t] = 1;
        live_total += n;
        ahead += n;
        s->stats.fetched_elements += n;
        pre.push_back(t);
        ++next_index;
      }
      if (!pre.empty()) {
        emit(ZERO3_FETCH, i, pre);
        s->stats.fetch_events += 1;
      }
      if (live_total + persistent_elems > s->stats.peak_live_elements)
        s->stats.peak_live_elements = live_total + persistent_elems;
      emit(ZERO3_COMPUTE, i, {});
      // release this layer's tensors
      std::vector<int32_t> rel;
      for (int32_t t : layer[i]) {
        live[t] = 0;
        live_total -= plan->numel[t];
        rel.push_back(t);
      }
      emit(ZERO3_RELEASE, i, rel);
    }
  } catch (const std::bad_alloc&) {
    delete s;
    return fail(ZERO_ENOMEM, "schedule allocation failed");
  }
  *out = s;
  return ZERO_OK;
}

int zero3_schedule_events(const zero3_schedule* s, zero3_event* out, int64_t cap,
                          int64_t* count) {
  if (!s || !count || (cap > 0 && !out)) return fail(ZERO_EINVAL, "NULL argument");
  const int64_t n = (int64_t)s->events.size();
  for (int64_t i = 0; i < n && i < cap; ++i) out[i] = s->events[i];
  *count = n;
  return ZERO_OK;
}

int zero3_schedule_tensors(const zero3_schedule* s, int32_t* out, int64_t cap,
                           int64_t* count) {
  if (!s || !count || (cap > 0 && !out)) return fail(ZERO_EINVAL, "NULL argument");
  const int64_t n = (int64_t)s->tensors.size();
  for (int64_t i = 0; i < n && i < cap; ++i) out[i] = s->tensors[i];
  *count = n;
  return ZERO_OK;
}

int zero3_schedule_stats(const zero3_schedule* s, zero3_stats* out) {
  if (!s || !out) return fail(ZERO_EINVAL, "NULL argument");
  *out = s->stats;
  return ZERO_OK;
}

void zero3_schedule_destroy(zero3_schedule* s) { delete s; }

}  // extern "C"
