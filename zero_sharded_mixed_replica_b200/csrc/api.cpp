// api.cpp -- the C ABI of libzero_b200 (declared in include/zero_b200.h): planner,
// argument checks, host-side step bookkeeping and the launches.
#include <cuda_runtime.h>
#include <math.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>
#include <string.h>

#include <new>
#include <mutex>
#include <string>

#include "zero_b200.h"
#include "zero_internal.h"

namespace zero {

namespace {
thread_local std::string g_last_error;

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int check_dtype(int32_t dt, const char* what) {
  if (dt != ZERO_BF16 && dt != ZERO_FP16)
    return fail(ZERO_EINVAL, std::string(what) + ": dtype must be ZERO_BF16 or ZERO_FP16");
  return ZERO_OK;
}

int64_t bucket_len(const zero_plan* p, int64_t b) {
  const int64_t s = b * p->bucket;
  const int64_t rest = p->n_pad - s;
  return rest < p->bucket ? rest : p->bucket;
}

int32_t* ws_bucket_blocks(const zero_plan* p, void* ws) {
  return (int32_t*)((char*)ws + p->ws_bucket_blocks_off);
}
double* ws_partial(const zero_plan* p, void* ws) {
  return (double*)((char*)ws + p->ws_partial_off);
}

bool bad_real(double x) { return !isfinite(x); }

int check_adamw(const zero_adamw_cfg* c) {
  if (!c) return fail(ZERO_EINVAL, "adamw cfg is NULL");
  if (bad_real(c->lr) || c->lr < 0) return fail(ZERO_EINVAL, "lr must be finite and >= 0");
  if (bad_real(c->beta1) || c->beta1 < 0 || c->beta1 >= 1)
    return fail(ZERO_EINVAL, "beta1 must be in [0, 1)");
  if (bad_real(c->beta2) || c->beta2 < 0 || c->beta2 >= 1)
    return fail(ZERO_EINVAL, "beta2 must be in [0, 1)");
  if (bad_real(c->eps) || c->eps <= 0) return fail(ZERO_EINVAL, "eps must be finite and > 0");
  if (bad_real(c->weight_decay)) return fail(ZERO_EINVAL, "weight_decay must be finite");
  if (isnan(c->max_grad_norm)) return fail(ZERO_EINVAL, "max_grad_norm is NaN");
  return ZERO_OK;
}

// K1 for bucket b with replica pointers already checked
int reduce_bucket(zero_plan* plan, int64_t b, int32_t dt, const uint16_t* const* g_at_start,
                  float* reduced, void* ws, cudaStream_t s, int accumulate = 0,
                  int want_sumsq = 1) {
  const int64_t start = b * plan->bucket, len = bucket_len(plan, b);
  int grid = 1;
  cudaError_t e = rs_grid(len, plan->world, dt, &grid);
  if (e != cudaSuccess) return cuda_fail(e, "reduce-scatter occupancy query");
  e = launch_reduce_scatter(plan->world, dt, g_at_start, reduced + start, len,
                            ws_partial(plan, ws) + b * plan->slots_full,
                            ws_bucket_blocks(plan, ws) + b,
                            &((WsHeader*)ws)->result.device_error, grid, s, accumulate,
                            want_sumsq);
  if (e != cudaSuccess) return cuda_fail(e, "reduce-scatter launch");
  if (want_sumsq) {
    plan->reduced[b] = 1;
    plan->reduced_count += 1;
  }
  return ZERO_OK;
}

// NVTX range for the lifetime of a scope (a no-op unless a profiler is attached)
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

int check_bucket_call(zero_plan* plan, int64_t bucket, int32_t dt, float* reduced,
                      void* ws) {
  if (!plan) return fail(ZERO_EINVAL, "plan is NULL");
  if (int rc = check_dtype(dt, "zero_reduce_scatter_bucket")) return rc;
  if (bucket < 0 || bucket >= plan->n_buckets)
    return fail(ZERO_EINVAL, "bucket " + std::to_string(bucket) + " out of range [0, " +
                                 std::to_string(plan->n_buckets) + ")");
  if (!reduced || !ws) return fail(ZERO_EINVAL, "reduced or workspace is NULL");
  if (!aligned16(reduced) || !aligned16(ws))
    return fail(ZERO_EALIGN, "reduced and workspace must be 16-byte aligned");
  if (plan->reduced[bucket])
    return fail(ZERO_ESTATE, "bucket " + std::to_string(bucket) +
                                 " was already reduce-scattered in this step");
  return ZERO_OK;
}

}  // namespace

void set_error(const std::string& msg) { g_last_error = msg; }

int fail(int code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(ZERO_ECUDA, std::string(what) + ": " + cudaGetErrorName(e) + " (" +
                              cudaGetErrorString(e) + ")");
}

const char* last_error_cstr() { return g_last_error.c_str(); }

}  // namespace zero

using namespace zero;

extern "C" {

const char* zero_last_error(void) { return last_error_cstr(); }

int zero_abi_version(void) { return ZERO_ABI_VERSION; }

// ------------------------------------------------------------------ planning

int zero_plan_create(const int64_t* dims, const int32_t* ndims, int32_t n_tensors,
                     int32_t world_size, int64_t reduce_bucket_size, int32_t align_elems,
                     zero_plan** out) {
  if (!out) return fail(ZERO_EINVAL, "out is NULL");
  *out = nullptr;
  if (n_tensors < 0) return fail(ZERO_EINVAL, "n_tensors < 0");
  if (n_tensors > 0 && !ndims) return fail(ZERO_EINVAL, "ndims is NULL");
  if (world_size < 1 || world_size > ZERO_MAX_WORLD)
    return fail(ZERO_EINVAL, "world_size must be in [1, " + std::to_string(ZERO_MAX_WORLD) + "]");
  if (reduce_bucket_size < 1) return fail(ZERO_EINVAL, "reduce_bucket_size must be >= 1");
  if (align_elems < 1) return fail(ZERO_EINVAL, "align_elems must be >= 1");
  zero_plan* p = new (std::nothrow) zero_plan();
  if (!p) return fail(ZERO_ENOMEM, "plan allocation failed");
  try {
    p->world = world_size;
    p->align = align_elems;
    p->bucket = reduce_bucket_size;
    p->numel.resize(n_tensors);
    p->offset.resize(n_tensors);
    int64_t d = 0, total = 0;
    for (int32_t t = 0; t < n_tensors; ++t) {
      if (ndims[t] < 0) {
        delete p;
        return fail(ZERO_EINVAL, "ndims[" + std::to_string(t) + "] < 0");
      }
      if (ndims[t] > 0 && !dims) {
        delete p;
        return fail(ZERO_EINVAL, "dims is NULL");
      }
      int64_t numel = 1;
      for (int32_t k = 0; k < ndims[t]; ++k, ++d) {
        const int64_t x = dims[d];
        if (x < 0) {
          delete p;
          return fail(ZERO_EINVAL, "negative dim in tensor " + std::to_string(t));
        }
        if (x != 0 && numel > INT64_MAX / x) {
          delete p;
          return fail(ZERO_ERANGE, "numel of tensor " + std::to_string(t) + " overflows int64");
        }
        numel *= x;
      }
      if (numel > INT64_MAX - total) {
        delete p;
        return fail(ZERO_ERANGE, "parameter count overflows int64");
      }
      p->numel[t] = numel;
      p->offset[t] = total;
      total += numel;
    }
    p->n = total;
    const int64_t unit = (int64_t)world_size * align_elems;
    const int64_t units = total / unit + (total % unit != 0);
    if (units > INT64_MAX / unit) {
      delete p;
      return fail(ZERO_ERANGE, "padded parameter count overflows int64");
    }
    p->n_pad = units * unit;
    p->p = p->n_pad / world_size;
    p->n_buckets = p->n_pad / reduce_bucket_size + (p->n_pad % reduce_bucket_size != 0);
    p->slots_full = p->n_buckets ? rs_slots(bucket_len(p, 0)) : 0;
    p->slots_last = p->n_buckets ? rs_slots(bucket_len(p, p->n_buckets - 1)) : 0;
    p->total_slots = p->n_buckets ? (p->n_buckets - 1) * p->slots_full + p->slots_last : 0;
    p->reduced.assign((size_t)p->n_buckets, 0);
    p->next_micro.assign((size_t)p->n_buckets, 0);
    p->ws_bucket_blocks_off = kWsHeaderBytes;
    p->ws_partial_off =
        round_up(p->ws_bucket_blocks_off + sizeof(int32_t) * (size_t)p->n_buckets, 256);
    p->ws_bytes = round_up(p->ws_partial_off + sizeof(double) * (size_t)p->total_slots, 256);
  } catch (const std::bad_alloc&) {
    delete p;
    return fail(ZERO_ENOMEM, "plan allocation failed");
  }
  *out = p;
  return ZERO_OK;
}

void zero_plan_destroy(zero_plan* plan) { delete plan; }

int zero_plan_get_info(const zero_plan* plan, zero_plan_info* out) {
  if (!plan || !out) return fail(ZERO_EINVAL, "plan or out is NULL");
  out->n = plan->n;
  out->n_pad = plan->n_pad;
  out->p = plan->p;
  out->n_buckets = plan->n_buckets;
  int64_t segs = 0;
  zero_plan_work_segments(plan, nullptr, 0, &segs);
  out->n_segments = segs;
  out->n_tensors = (int64_t)plan->numel.size();
  out->bucket_size = plan->bucket;
  out->world_size = plan->world;
  out->align = plan->align;
  return ZERO_OK;
}

int zero_plan_tensor(const zero_plan* plan, int32_t t, int64_t* flat_offset, int64_t* numel) {
  if (!plan || !flat_offset || !numel) return fail(ZERO_EINVAL, "NULL argument");
  if (t < 0 || (size_t)t >= plan->numel.size()) return fail(ZERO_EINVAL, "tensor out of range");
  *flat_offset = plan->offset[t];
  *numel = plan->numel[t];
  return ZERO_OK;
}

int zero_plan_bucket(const zero_plan* plan, int64_t b, int64_t* start, int64_t* length) {
  if (!plan || !start || !length) return fail(ZERO_EINVAL, "NULL argument");
  if (b < 0 || b >= plan->n_buckets) return fail(ZERO_EINVAL, "bucket out of range");
  *start = b * plan->bucket;
  *length = bucket_len(plan, b);
  return ZERO_OK;
}

int zero_plan_work_segments(const zero_plan* plan, zero_work_segment* out, int64_t cap,
                            int64_t* count) {
  if (!plan || !count) return fail(ZERO_EINVAL, "NULL argument");
  if (cap > 0 && !out) return fail(ZERO_EINVAL, "out is NULL");
  int64_t c = 0;
  for (int64_t b = 0; b < plan->n_buckets; ++b) {
    const int64_t s = b * plan->bucket, e = s + bucket_len(plan, b);
    // ranks whose partition meets [s, e)
    for (int64_t r = s / plan->p; r < plan->world && r * plan->p < e; ++r) {
      const int64_t lo = r * plan->p > s ? r * plan->p : s;
      const int64_t hi = (r + 1) * plan->p < e ? (r + 1) * plan->p : e;
      if (hi <= lo) continue;
      if (c < cap) out[c] = zero_work_segment{b, r, lo, hi - lo};
      ++c;
    }
  }
  *count = c;
  return ZERO_OK;
}

int zero_plan_partition(const zero_plan* plan, int32_t rank, zero_segment* out, int64_t cap,
                        int64_t* count) {
  if (!plan || !count) return fail(ZERO_EINVAL, "NULL argument");
  if (rank < 0 || rank >= plan->world) return fail(ZERO_EINVAL, "rank out of range");
  if (cap > 0 && !out) return fail(ZERO_EINVAL, "out is NULL");
  const int64_t lo = (int64_t)rank * plan->p, hi = lo + plan->p;
  int64_t c = 0;
  // tensors are sorted by offset: binary search for the first one ending after lo
  size_t t0 = 0, t1 = plan->numel.size();
  while (t0 < t1) {
    const size_t mid = (t0 + t1) / 2;
    if (plan->offset[mid] + plan->numel[mid] <= lo)
      t0 = mid + 1;
    else
      t1 = mid;
  }
  for (size_t t = t0; t < plan->numel.size() && plan->offset[t] < hi; ++t) {
    const int64_t a = plan->offset[t] > lo ? plan->offset[t] : lo;
    const int64_t end = plan->offset[t] + plan->numel[t];
    const int64_t b = end < hi ? end : hi;
    if (b <= a) continue;
    if (c < cap) out[c] = zero_segment{(int64_t)t, a - plan->offset[t], a, b - a};
    ++c;
  }
  const int64_t pa = plan->n > lo ? plan->n : lo;
  if (hi > pa) {
    if (c < cap) out[c] = zero_segment{-1, pa - plan->n, pa, hi - pa};
    ++c;
  }
  *count = c;
  return ZERO_OK;
}

int zero_plan_memory(const zero_plan* plan, int32_t stage, zero_memory* out) {
  if (!plan || !out) return fail(ZERO_EINVAL, "NULL argument");
  if (stage < 0 || stage > 3) return fail(ZERO_EINVAL, "stage must be 0..3");
  const double full = (double)plan->n_pad, part = (double)plan->p;
  out->optimizer_state = 12.0 * (stage >= 1 ? part : full);
  out->grads = 2.0 * (stage >= 2 ? part : full);
  out->params = 2.0 * (stage >= 3 ? part : full);
  out->total = out->params + out->grads + out->optimizer_state;
  return ZERO_OK;
}

// ------------------------------------------------------------------ device state

int zero_workspace_bytes(const zero_plan* plan, size_t* bytes) {
  if (!plan || !bytes) return fail(ZERO_EINVAL, "NULL argument");
  *bytes = plan->ws_bytes;
  return ZERO_OK;
}

int zero_state_init(zero_plan* plan, void* workspace, const zero_scaler_cfg* cfg,
                    void* stream) {
  if (!plan || !workspace || !cfg) return fail(ZERO_EINVAL, "NULL argument");
  if (!aligned16(workspace)) return fail(ZERO_EALIGN, "workspace must be 16-byte aligned");
  if (cfg->dynamic) {
    if (cfg->loss_scale_window < 1) return fail(ZERO_EINVAL, "loss_scale_window must be >= 1");
    if (cfg->hysteresis < 1) return fail(ZERO_EINVAL, "hysteresis must be >= 1");
    if (!(cfg->min_loss_scale > 0) || !isfinite(cfg->min_loss_scale))
      return fail(ZERO_EINVAL, "min_loss_scale must be finite and > 0");
    if (!(cfg->scale_factor > 1) || !isfinite(cfg->scale_factor))
      return fail(ZERO_EINVAL, "scale_factor must be finite and > 1");
    if (cfg->initial_scale_power < -126 || cfg->initial_scale_power > 127)
      return fail(ZERO_EINVAL, "initial_scale_power out of range");
  } else if (!(cfg->static_scale > 0) || !isfinite(cfg->static_scale)) {
    return fail(ZERO_EINVAL, "static_scale must be finite and > 0");
  }
  cudaError_t e = launch_state_init(workspace, *cfg, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "state init launch");
  plan->reduced.assign((size_t)plan->n_buckets, 0);
  plan->reduced_count = 0;
  plan->next_micro.assign((size_t)plan->n_buckets, 0);
  plan->n_micro = 0;
  plan->finalized = false;
  return ZERO_OK;
}

int zero_state_read(const void* workspace, zero_scaler_state* out, void* stream) {
  if (!workspace || !out) return fail(ZERO_EINVAL, "NULL argument");
  WsHeader h;
  cudaError_t e = cudaMemcpyAsync(&h, workspace, sizeof h, cudaMemcpyDeviceToHost,
                                  (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "state copy");
  e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  if (h.magic != kWsMagic) return fail(ZERO_ESTATE, "workspace was never initialised");
  out->scale = h.scale;
  out->cur_hysteresis = h.cur_hysteresis;
  out->iter = h.iter;
  out->last_overflow_iter = h.last_overflow_iter;
  out->adam_t = h.adam_t;
  return ZERO_OK;
}

int zero_state_write(zero_plan* plan, void* workspace, const zero_scaler_cfg* cfg,
                     const zero_scaler_state* state, void* stream) {
  if (!state) return fail(ZERO_EINVAL, "NULL argument");
  if (!(state->scale > 0) || !isfinite(state->scale))
    return fail(ZERO_EINVAL, "state scale must be finite and > 0");
  if (state->iter < 0 || state->adam_t < 0 || state->adam_t > state->iter ||
      state->last_overflow_iter < -1 || state->last_overflow_iter >= state->iter)
    return fail(ZERO_EINVAL, "inconsistent step counters");
  if (int rc = zero_state_init(plan, workspace, cfg, stream)) return rc;
  cudaError_t e = launch_state_write(workspace, *state, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "state write launch");
  return ZERO_OK;
}

int zero_cast_params(const zero_plan* plan, const float* master, void* params,
                     int32_t param_dtype, void* stream) {
  if (!plan) return fail(ZERO_EINVAL, "NULL argument");
  if (plan->n_pad > 0 && (!master || !params)) return fail(ZERO_EINVAL, "NULL argument");
  if (int rc = check_dtype(param_dtype, "zero_cast_params")) return rc;
  if (!aligned16(master) || !aligned16(params))
    return fail(ZERO_EALIGN, "master and params must be 16-byte aligned");
  cudaError_t e = launch_cast(param_dtype, master, params, plan->n_pad, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cast launch");
  return ZERO_OK;
}

// ------------------------------------------------------------------ the step

int zero_reduce_scatter_bucket(zero_plan* plan, int64_t bucket, int32_t grad_dtype,
                               const void* const* replica_grads, int64_t replica_base_offset,
                               float* reduced, void* workspace, void* stream) {
  NvtxRange nvtx("zero_reduce_scatter_bucket");
  if (int rc = check_bucket_call(plan, bucket, grad_dtype, reduced, workspace)) return rc;
  if (!replica_grads) return fail(ZERO_EINVAL, "replica_grads is NULL");
  const int64_t start = bucket * plan->bucket;
  if (replica_base_offset < 0 || replica_base_offset > start)
    return fail(ZERO_EINVAL, "replica_base_offset must be in [0, bucket start]");
  const uint16_t* g[ZERO_MAX_WORLD];
  for (int r = 0; r < plan->world; ++r) {
    if (!replica_grads[r]) return fail(ZERO_EINVAL, "replica_grads[" + std::to_string(r) + "] is NULL");
    if (!aligned16(replica_grads[r]))
      return fail(ZERO_EALIGN, "replica_grads[" + std::to_string(r) + "] is not 16-byte aligned");
    g[r] = (const uint16_t*)replica_grads[r] + (start - replica_base_offset);
  }
  return reduce_bucket(plan, bucket, grad_dtype, g, reduced, workspace, (cudaStream_t)stream);
}

int zero_reduce_scatter_bucket_host(zero_plan* plan, int64_t bucket, int32_t grad_dtype,
                                    const void* const* host_replica_grads,
                                    int64_t host_base_offset, void* const* device_staging,
                                    float* reduced, void* workspace, void* stream) {
  if (int rc = check_bucket_call(plan, bucket, grad_dtype, reduced, workspace)) return rc;
  if (!host_replica_grads || !device_staging)
    return fail(ZERO_EINVAL, "host_replica_grads or device_staging is NULL");
  const int64_t start = bucket * plan->bucket, len = bucket_len(plan, bucket);
  if (host_base_offset < 0 || host_base_offset > start)
    return fail(ZERO_EINVAL, "host_base_offset must be in [0, bucket start]");
  const uint16_t* g[ZERO_MAX_WORLD];
  for (int r = 0; r < plan->world; ++r) {
    if (!host_replica_grads[r] || !device_staging[r])
      return fail(ZERO_EINVAL, "NULL replica pointer " + std::to_string(r));
    if (!aligned16(device_staging[r]))
      return fail(ZERO_EALIGN, "device_staging[" + std::to_string(r) + "] is not 16-byte aligned");
    const uint16_t* src = (const uint16_t*)host_replica_grads[r] + (start - host_base_offset);
    cudaError_t e = cudaMemcpyAsync(device_staging[r], src, (size_t)len * sizeof(uint16_t),
                                    cudaMemcpyHostToDevice, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy of a replica bucket");
    g[r] = (const uint16_t*)device_staging[r];
  }
  return reduce_bucket(plan, bucket, grad_dtype, g, reduced, workspace, (cudaStream_t)stream);
}

int zero_reduce_scatter_bucket_accum(zero_plan* plan, int64_t bucket, int32_t micro,
                                     int32_t n_micro, int32_t grad_dtype,
                                     const void* const* replica_grads,
                                     int64_t replica_base_offset, float* reduced,
                                     void* workspace, void* stream) {
  if (int rc = check_bucket_call(plan, bucket, grad_dtype, reduced, workspace)) return rc;
  if (!replica_grads) return fail(ZERO_EINVAL, "replica_grads is NULL");
  if (n_micro < 1) return fail(ZERO_EINVAL, "n_micro must be >= 1");
  if (plan->n_micro != 0 && plan->n_micro != n_micro)
    return fail(ZERO_ESTATE, "n_micro changed within a step");
  if (micro != plan->next_micro[bucket])
    return fail(ZERO_ESTATE, "micro-batch " + std::to_string(micro) + " of bucket " +
                                 std::to_string(bucket) + " out of order (expected " +
                                 std::to_string(plan->next_micro[bucket]) + ")");
  const int64_t start = bucket * plan->bucket;
  if (replica_base_offset < 0 || replica_base_offset > start)
    return fail(ZERO_EINVAL, "replica_base_offset must be in [0, bucket start]");
  const uint16_t* g[ZERO_MAX_WORLD];
  for (int r = 0; r < plan->world; ++r) {
    if (!replica_grads[r]) return fail(ZERO_EINVAL, "replica_grads[" + std::to_string(r) + "] is NULL");
    if (!aligned16(replica_grads[r]))
      return fail(ZERO_EALIGN, "replica_grads[" + std::to_string(r) + "] is not 16-byte aligned");
    g[r] = (const uint16_t*)replica_grads[r] + (start - replica_base_offset);
  }
  const bool last = micro == n_micro - 1;
  if (int rc = reduce_bucket(plan, bucket, grad_dtype, g, reduced, workspace,
                             (cudaStream_t)stream, micro > 0 ? 1 : 0, last ? 1 : 0))
    return rc;
  plan->n_micro = n_micro;
  plan->next_micro[bucket] = last ? 0 : micro + 1;
  return ZERO_OK;
}

int zero_step_finalize(zero_plan* plan, const zero_adamw_cfg* cfg, void* workspace,
                       void* stream) {
  NvtxRange nvtx("zero_step_finalize");
  if (!plan || !workspace) return fail(ZERO_EINVAL, "NULL argument");
  if (int rc = check_adamw(cfg)) return rc;
  if (!aligned16(workspace)) return fail(ZERO_EALIGN, "workspace must be 16-byte aligned");
  if (plan->reduced_count != plan->n_buckets)
    return fail(ZERO_ESTATE, "zero_step before every bucket was reduce-scattered (" +
                                 std::to_string(plan->reduced_count) + " of " +
                                 std::to_string(plan->n_buckets) + ")");
  cudaError_t e = launch_finalize(workspace, ws_bucket_blocks(plan, workspace), plan->slots_full,
                                  ws_partial(plan, workspace), plan->n_buckets, *cfg,
                                  (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "finalize launch");
  plan->reduced.assign((size_t)plan->n_buckets, 0);
  plan->reduced_count = 0;
  plan->next_micro.assign((size_t)plan->n_buckets, 0);
  plan->n_micro = 0;
  plan->finalized = true;
  return ZERO_OK;
}

int zero_step_update(zero_plan* plan, float* master, float* exp_avg, float* exp_avg_sq,
                     const float* reduced, void* params, int32_t param_dtype,
                     const void* workspace, void* stream) {
  NvtxRange nvtx("zero_step_update");
  if (!plan || !workspace) return fail(ZERO_EINVAL, "NULL argument");
  if (plan->n_pad > 0 && (!master || !exp_avg || !exp_avg_sq || !reduced || !params))
    return fail(ZERO_EINVAL, "NULL argument");
  if (int rc = check_dtype(param_dtype, "zero_step_update")) return rc;
  if (!aligned16(master) || !aligned16(exp_avg) || !aligned16(exp_avg_sq) ||
      !aligned16(reduced) || !aligned16(params) || !aligned16(workspace))
    return fail(ZERO_EALIGN, "step buffers must be 16-byte aligned");
  if (!plan->finalized)
    return fail(ZERO_ESTATE, "zero_step_update without a zero_step_finalize before it");
  void* dst[1] = {params};
  cudaError_t e = launch_update(param_dtype, reduced, master, exp_avg, exp_avg_sq, dst, 1,
                                plan->n_pad, workspace, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "update launch");
  plan->finalized = false;
  return ZERO_OK;
}

int zero_step(zero_plan* plan, const zero_adamw_cfg* cfg, float* master, float* exp_avg,
              float* exp_avg_sq, const float* reduced, void* params, int32_t param_dtype,
              void* workspace, void* stream) {
  if (!plan || !workspace) return fail(ZERO_EINVAL, "NULL argument");
  if (plan->n_pad > 0 && (!master || !exp_avg || !exp_avg_sq || !reduced || !params))
    return fail(ZERO_EINVAL, "NULL argument");
  if (int rc = check_dtype(param_dtype, "zero_step")) return rc;
  if (!aligned16(master) || !aligned16(exp_avg) || !aligned16(exp_avg_sq) ||
      !aligned16(reduced) || !aligned16(params))
    return fail(ZERO_EALIGN, "step buffers must be 16-byte aligned");
  if (int rc = zero_step_finalize(plan, cfg, workspace, stream)) return rc;
  return zero_step_update(plan, master, exp_avg, exp_avg_sq, reduced, params, param_dtype,
                          workspace, stream);
}

int zero_step_full(zero_plan* plan, const zero_adamw_cfg* cfg, int32_t grad_dtype,
                   const void* const* replica_grads, int64_t replica_base_offset,
                   float* reduced, float* master, float* exp_avg, float* exp_avg_sq,
                   void* params, int32_t param_dtype, void* workspace, void* stream) {
  NvtxRange nvtx("zero_step_full");
  // every check before the first launch, so that a refused call changes nothing
  if (!plan || !workspace) return fail(ZERO_EINVAL, "NULL argument");
  if (int rc = check_dtype(grad_dtype, "zero_step_full")) return rc;
  if (int rc = check_dtype(param_dtype, "zero_step_full")) return rc;
  if (int rc = check_adamw(cfg)) return rc;
  if (plan->n_pad > 0 && (!reduced || !master || !exp_avg || !exp_avg_sq || !params ||
                          !replica_grads))
    return fail(ZERO_EINVAL, "NULL argument");
  if (!aligned16(workspace) ||
      (plan->n_pad > 0 && (!aligned16(reduced) || !aligned16(master) || !aligned16(exp_avg) ||
                           !aligned16(exp_avg_sq) || !aligned16(params))))
    return fail(ZERO_EALIGN, "step buffers and workspace must be 16-byte aligned");
  if (replica_base_offset != 0)
    return fail(ZERO_EINVAL, "replica_base_offset must be 0: the replicas hold every bucket");
  if (plan->reduced_count != 0 || plan->n_micro != 0)
    return fail(ZERO_ESTATE, "zero_step_full after buckets of this step were already reduced");
  for (int r = 0; r < plan->world && plan->n_pad > 0; ++r) {
    if (!replica_grads[r]) return fail(ZERO_EINVAL, "replica_grads[" + std::to_string(r) + "] is NULL");
    if (!aligned16(replica_grads[r]))
      return fail(ZERO_EALIGN, "replica_grads[" + std::to_string(r) + "] is not 16-byte aligned");
  }
  for (int64_t b = 0; b < plan->n_buckets; ++b)
    if (int rc = zero_reduce_scatter_bucket(plan, b, grad_dtype, replica_grads,
                                            replica_base_offset, reduced, workspace, stream))
      return rc;
  return zero_step(plan, cfg, master, exp_avg, exp_avg_sq, reduced, params, param_dtype,
                   workspace, stream);
}

int zero_step_resident(zero_plan* plan, const zero_adamw_cfg* cfg, int32_t grad_dtype,
                       const void* const* replica_grads, float* master, float* exp_avg,
                       float* exp_avg_sq, void* params, int32_t param_dtype, void* workspace,
                       void* stream) {
  NvtxRange nvtx("zero_step_resident");
  if (!plan || !workspace) return fail(ZERO_EINVAL, "NULL argument");
  if (int rc = check_dtype(grad_dtype, "zero_step_resident")) return rc;
  if (int rc = check_dtype(param_dtype, "zero_step_resident")) return rc;
  if (int rc = check_adamw(cfg)) return rc;
  if (plan->world > 2)
    return fail(ZERO_EINVAL,
                "zero_step_resident moves fewer bytes only for world_size <= 2; use "
                "zero_reduce_scatter_bucket and zero_step");
  if (plan->n_pad > 0 && (!master || !exp_avg || !exp_avg_sq || !params || !replica_grads))
    return fail(ZERO_EINVAL, "NULL argument");
  if (!aligned16(workspace) || (plan->n_pad > 0 && (!aligned16(master) || !aligned16(exp_avg) ||
                                                    !aligned16(exp_avg_sq) || !aligned16(params))))
    return fail(ZERO_EALIGN, "step buffers and workspace must be 16-byte aligned");
  if (plan->reduced_count != 0 || plan->n_micro != 0)
    return fail(ZERO_ESTATE, "zero_step_resident after buckets of this step were already reduced");
  const uint16_t* g[ZERO_MAX_WORLD];
  for (int r = 0; r < plan->world && plan->n_pad > 0; ++r) {
    if (!replica_grads[r]) return fail(ZERO_EINVAL, "replica_grads[" + std::to_string(r) + "] is NULL");
    if (!aligned16(replica_grads[r]))
      return fail(ZERO_EALIGN, "replica_grads[" + std::to_string(r) + "] is not 16-byte aligned");
    g[r] = (const uint16_t*)replica_grads[r];
  }
  cudaStream_t s = (cudaStream_t)stream;
  // the sum of squares of every bucket; the reduced gradient is not stored
  for (int64_t b = 0; b < plan->n_buckets; ++b) {
    const int64_t start = b * plan->bucket, len = bucket_len(plan, b);
    const uint16_t* gb[ZERO_MAX_WORLD];
    for (int r = 0; r < plan->world; ++r) gb[r] = g[r] + start;
    int grid = 1;
    cudaError_t e = rs_grid(len, plan->world, grad_dtype, &grid);
    if (e != cudaSuccess) return cuda_fail(e, "reduce-scatter occupancy query");
    e = launch_reduce_scatter(plan->world, grad_dtype, gb, nullptr, len,
                              ws_partial(plan, workspace) + b * plan->slots_full,
                              ws_bucket_blocks(plan, workspace) + b,
                              &((WsHeader*)workspace)->result.device_error, grid, s,
                              /*accumulate=*/0, /*want_sumsq=*/1, /*store=*/0);
    if (e != cudaSuccess) return cuda_fail(e, "sum-of-squares launch");
  }
  cudaError_t e = launch_finalize(workspace, ws_bucket_blocks(plan, workspace), plan->slots_full,
                                  ws_partial(plan, workspace), plan->n_buckets, *cfg, s);
  if (e != cudaSuccess) return cuda_fail(e, "finalize launch");
  e = launch_update_resident(plan->world, grad_dtype, param_dtype, g, master, exp_avg,
                             exp_avg_sq, params, plan->n_pad, workspace, s);
  if (e != cudaSuccess) return cuda_fail(e, "update launch");
  plan->finalized = false;
  return ZERO_OK;
}

int zero_all_gather(const zero_plan* plan, const void* params, void* const* rank_params,
                    int32_t n_dst, int32_t param_dtype, void* stream) {
  if (!plan) return fail(ZERO_EINVAL, "NULL argument");
  if (int rc = check_dtype(param_dtype, "zero_all_gather")) return rc;
  if (n_dst < 0) return fail(ZERO_EINVAL, "n_dst < 0");
  if (n_dst == 0 || plan->n_pad == 0) return ZERO_OK;  // the fused cast wrote the buffer
  if (!params) return fail(ZERO_EINVAL, "NULL argument");
  if (!rank_params) return fail(ZERO_EINVAL, "rank_params is NULL");
  if (!aligned16(params)) return fail(ZERO_EALIGN, "params must be 16-byte aligned");
  for (int d = 0; d < n_dst; ++d) {
    if (!rank_params[d]) return fail(ZERO_EINVAL, "rank_params[" + std::to_string(d) + "] is NULL");
    if (!aligned16(rank_params[d]))
      return fail(ZERO_EALIGN, "rank_params[" + std::to_string(d) + "] is not 16-byte aligned");
  }
  cudaError_t e = launch_replicate(params, rank_params, n_dst, plan->n_pad, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "all-gather copy launch");
  return ZERO_OK;
}

int zero_get_result(const void* workspace, zero_step_result* out, void* stream) {
  if (!workspace || !out) return fail(ZERO_EINVAL, "NULL argument");
  const WsHeader* h = (const WsHeader*)workspace;
  cudaError_t e = cudaMemcpyAsync(out, &h->result, sizeof(zero_step_result),
                                  cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "result copy");
  e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  if (out->device_error)
    return fail(ZERO_EDEVICE, "a kernel gave up on a bounded internal wait (code " +
                                  std::to_string(out->device_error) + "); outputs are incomplete");
  return ZERO_OK;
}

// ------------------------------------------------------------------ one rank of W processes

namespace {
// buckets [b0, b1) that meet partition `rank`
void rank_buckets(const zero_plan* plan, int32_t rank, int64_t* b0, int64_t* b1) {
  if (plan->p == 0 || plan->n_buckets == 0) {
    *b0 = *b1 = 0;
    return;
  }
  const int64_t lo = (int64_t)rank * plan->p, hi = lo + plan->p;
  *b0 = lo / plan->bucket;
  *b1 = (hi - 1) / plan->bucket + 1;
}
}  // namespace

int zero_reduce_scatter_segment(zero_plan* plan, int64_t bucket, int32_t rank,
                                int32_t grad_dtype, const void* const* replica_grads,
                                int64_t replica_base_offset, float* reduced_local,
                                void* workspace, void* stream) {
  if (!plan) return fail(ZERO_EINVAL, "plan is NULL");
  if (rank < 0 || rank >= plan->world) return fail(ZERO_EINVAL, "rank out of range");
  if (int rc = check_bucket_call(plan, bucket, grad_dtype, reduced_local, workspace)) return rc;
  if (!replica_grads) return fail(ZERO_EINVAL, "replica_grads is NULL");
  int64_t b0, b1;
  rank_buckets(plan, rank, &b0, &b1);
  if (bucket < b0 || bucket >= b1)
    return fail(ZERO_EINVAL, "bucket " + std::to_string(bucket) + " does not meet partition " +
                                 std::to_string(rank));
  const int64_t bs = bucket * plan->bucket, be = bs + bucket_len(plan, bucket);
  const int64_t ps = (int64_t)rank * plan->p, pe = ps + plan->p;
  const int64_t lo = bs > ps ? bs : ps, hi = be < pe ? be : pe;
  if (replica_base_offset < 0 || replica_base_offset > lo)
    return fail(ZERO_EINVAL, "replica_base_offset must be in [0, segment start]");
  const uint16_t* g[ZERO_MAX_WORLD];
  for (int r = 0; r < plan->world; ++r) {
    if (!replica_grads[r]) return fail(ZERO_EINVAL, "replica_grads[" + std::to_string(r) + "] is NULL");
    if (!aligned16(replica_grads[r]))
      return fail(ZERO_EALIGN, "replica_grads[" + std::to_string(r) + "] is not 16-byte aligned");
    g[r] = (const uint16_t*)replica_grads[r] + (lo - replica_base_offset);
  }
  const int64_t len = hi - lo;
  int grid = 1;
  cudaError_t e = rs_grid(len, plan->world, grad_dtype, &grid);
  if (e != cudaSuccess) return cuda_fail(e, "reduce-scatter occupancy query");
  e = launch_reduce_scatter(plan->world, grad_dtype, g, reduced_local + (lo - ps), len,
                            ws_partial(plan, workspace) + bucket * plan->slots_full,
                            ws_bucket_blocks(plan, workspace) + bucket,
                            &((WsHeader*)workspace)->result.device_error, grid,
                            (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "reduce-scatter launch");
  plan->reduced[bucket] = 1;
  plan->reduced_count += 1;
  return ZERO_OK;
}

int zero_step_local_sumsq(zero_plan* plan, int32_t rank, void* workspace, double* sumsq_out,
                          void* stream) {
  if (!plan || !workspace || !sumsq_out) return fail(ZERO_EINVAL, "NULL argument");
  if (rank < 0 || rank >= plan->world) return fail(ZERO_EINVAL, "rank out of range");
  if (((uintptr_t)sumsq_out & 7u) != 0) return fail(ZERO_EALIGN, "sumsq_out must be 8-byte aligned");
  int64_t b0, b1;
  rank_buckets(plan, rank, &b0, &b1);
  for (int64_t b = b0; b < b1; ++b)
    if (!plan->reduced[b])
      return fail(ZERO_ESTATE, "segment of bucket " + std::to_string(b) + " not reduced yet");
  if (plan->reduced_count != b1 - b0)
    return fail(ZERO_ESTATE, "buckets outside this rank's partition were reduced");
  cudaError_t e = launch_local_sumsq(ws_bucket_blocks(plan, workspace), plan->slots_full,
                                     ws_partial(plan, workspace), b0, b1, sumsq_out,
                                     (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "local sum launch");
  plan->local_summed = true;
  return ZERO_OK;
}

int zero_step_finalize_ranks(zero_plan* plan, const zero_adamw_cfg* cfg,
                             const double* sumsq_ranks, void* workspace, void* stream) {
  if (!plan || !workspace || !sumsq_ranks) return fail(ZERO_EINVAL, "NULL argument");
  if (int rc = check_adamw(cfg)) return rc;
  if (!plan->local_summed)
    return fail(ZERO_ESTATE, "zero_step_finalize_ranks before zero_step_local_sumsq");
  cudaError_t e = launch_finalize_ranks(workspace, sumsq_ranks, plan->world, *cfg,
                                        (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "finalize launch");
  plan->reduced.assign((size_t)plan->n_buckets, 0);
  plan->reduced_count = 0;
  plan->next_micro.assign((size_t)plan->n_buckets, 0);
  plan->n_micro = 0;
  plan->local_summed = false;
  plan->finalized = true;
  return ZERO_OK;
}

int zero_step_update_partition(zero_plan* plan, int32_t rank, float* master_local,
                               float* exp_avg_local, float* exp_avg_sq_local,
                               const float* reduced_local, void* const* params_dst,
                               int32_t n_dst, int32_t param_dtype, const void* workspace,
                               void* stream) {
  if (!plan || !workspace || !params_dst) return fail(ZERO_EINVAL, "NULL argument");
  if (rank < 0 || rank >= plan->world) return fail(ZERO_EINVAL, "rank out of range");
  if (n_dst < 1 || n_dst > ZERO_MAX_WORLD)
    return fail(ZERO_EINVAL, "n_dst must be in [1, " + std::to_string(ZERO_MAX_WORLD) + "]");
  if (int rc = check_dtype(param_dtype, "zero_step_update_partition")) return rc;
  if (plan->p > 0 && (!master_local || !exp_avg_local || !exp_avg_sq_local || !reduced_local))
    return fail(ZERO_EINVAL, "NULL argument");
  if (!aligned16(master_local) || !aligned16(exp_avg_local) || !aligned16(exp_avg_sq_local) ||
      !aligned16(reduced_local) || !aligned16(workspace))
    return fail(ZERO_EALIGN, "partition buffers must be 16-byte aligned");
  void* dst[ZERO_MAX_WORLD];
  for (int d = 0; d < n_dst; ++d) {
    if (!params_dst[d] && plan->p > 0) return fail(ZERO_EINVAL, "params_dst has a NULL entry");
    dst[d] = params_dst[d];  // where this rank's p half values go in destination d
    if (!aligned16(dst[d]))
      return fail(ZERO_EALIGN, "params_dst[" + std::to_string(d) + "] is not 16-byte aligned");
  }
  if (!plan->finalized)
    return fail(ZERO_ESTATE, "zero_step_update_partition without a finalize before it");
  cudaError_t e = launch_update(param_dtype, reduced_local, master_local, exp_avg_local,
                                exp_avg_sq_local, dst, n_dst, plan->p, workspace,
                                (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "update launch");
  plan->finalized = false;
  return ZERO_OK;
}

// ------------------------------------------------------------------ diagnostics

int zero_selftest_bounded_wait(void* workspace, void* stream) {
  if (!workspace) return fail(ZERO_EINVAL, "NULL argument");
  if (!aligned16(workspace)) return fail(ZERO_EALIGN, "workspace must be 16-byte aligned");
  cudaError_t e = launch_selftest_wait(workspace, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return ZERO_OK;
}

// ------------------------------------------------------------------ peer memory

int zero_ipc_handle_bytes(void) { return (int)sizeof(cudaIpcMemHandle_t); }

// The start of the allocation holding a device pointer, from the driver's
// cuMemGetAddressRange, looked up through the runtime so that the library does not link
// the driver library itself (it must load on machines without one).
typedef int (*MemGetAddressRangeFn)(unsigned long long* base, size_t* size,
                                    unsigned long long ptr);

static int allocation_offset(const void* device_ptr, int64_t* offset) {
  static std::once_flag once;
  static MemGetAddressRangeFn fn = nullptr;
  static cudaError_t lookup = cudaSuccess;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    lookup = cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &q);
    if (lookup == cudaSuccess && q == cudaDriverEntryPointSuccess) fn = (MemGetAddressRangeFn)f;
  });
  if (!fn) return fail(ZERO_ECUDA, "cuMemGetAddressRange unavailable");
  unsigned long long base = 0;
  size_t size = 0;
  const int r = fn(&base, &size, (unsigned long long)(uintptr_t)device_ptr);
  if (r != 0) return fail(ZERO_ECUDA, "cuMemGetAddressRange failed (" + std::to_string(r) + ")");
  *offset = (int64_t)((uintptr_t)device_ptr - (uintptr_t)base);
  return ZERO_OK;
}

int zero_ipc_get_handle(const void* device_ptr, void* handle_out, int64_t* offset_out) {
  if (!device_ptr || !handle_out || !offset_out) return fail(ZERO_EINVAL, "NULL argument");
  int rc = allocation_offset(device_ptr, offset_out);
  if (rc != ZERO_OK) return rc;
  cudaIpcMemHandle_t h;
  cudaError_t e = cudaIpcGetMemHandle(&h, (void*)device_ptr);
  if (e != cudaSuccess) return cuda_fail(e, "cudaIpcGetMemHandle");
  memcpy(handle_out, &h, sizeof h);
  return ZERO_OK;
}

int zero_ipc_open_handle(const void* handle, void** base_out) {
  if (!handle || !base_out) return fail(ZERO_EINVAL, "NULL argument");
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof h);
  cudaError_t e = cudaIpcOpenMemHandle(base_out, h, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) return cuda_fail(e, "cudaIpcOpenMemHandle");
  return ZERO_OK;
}

int zero_ipc_close(void* base) {
  if (!base) return fail(ZERO_EINVAL, "NULL argument");
  cudaError_t e = cudaIpcCloseMemHandle(base);
  if (e != cudaSuccess) return cuda_fail(e, "cudaIpcCloseMemHandle");
  return ZERO_OK;
}

}  // extern "C"
