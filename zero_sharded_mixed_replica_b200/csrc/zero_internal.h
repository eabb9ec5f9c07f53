// zero_internal.h -- plan object, device workspace layout and kernel launchers of
// libzero_b200 (not part of the public ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "zero_b200.h"

namespace zero {

// Reduce-scatter: partial-sum slots are reserved for one block per 256 groups of 8
// elements, at most kRsMaxBlocks per bucket (a launch uses at most that many blocks).
constexpr int kRsThreads = 256;
constexpr int kRsMaxBlocks = 148 * 8;
// Launch shape of the small grid-stride kernels (cast).
constexpr int kUpThreads = 256;
constexpr int kFinalizeThreads = 1024;

constexpr uint32_t kWsMagic = 0x5A45524Fu;  // "ZERO"

// Device workspace header. Written by zero_state_init and by the finalize kernel; read
// by the update kernel. Lives at offset 0 of the caller's workspace.
struct WsHeader {
  uint32_t magic;
  int32_t dynamic;
  int32_t hysteresis_cfg;
  int32_t init_scale_power;
  int64_t window;
  float min_scale;
  float factor;
  float static_scale;
  float pad0;
  // loss-scaler and AdamW state
  float scale;
  int32_t cur_hysteresis;
  int64_t iter;
  int64_t last_overflow_iter;
  int64_t adam_t;
  // constants of this step's elementwise update (written by finalize)
  float k, b1, omb1, b2, omb2, bc1, bc2, eps, lr, decay;
  int32_t skip;
  int32_t pad1;
  zero_step_result result;
};
static_assert(sizeof(WsHeader) <= 512, "workspace header grew past its slot");

constexpr size_t kWsHeaderBytes = 512;

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace zero

struct zero_plan {
  int32_t world = 1;
  int32_t align = 1;
  int64_t bucket = 1;
  int64_t n = 0, n_pad = 0, p = 0, n_buckets = 0;
  std::vector<int64_t> numel, offset;  // per tensor
  // reduce-scatter partial-sum slots: bucket b owns slots [b*slots_full, b*slots_full +
  // slots_of(b)); every bucket but the last has slots_full of them.
  int64_t slots_full = 0, slots_last = 0, total_slots = 0;
  // per-step bookkeeping (host side)
  std::vector<uint8_t> reduced;
  int64_t reduced_count = 0;
  // gradient accumulation: next micro-batch expected per bucket, and the step's count
  std::vector<int32_t> next_micro;
  int32_t n_micro = 0;
  bool finalized = false;  // finalize ran and no update consumed it yet
  bool local_summed = false;  // one rank: its local sum of squares was taken this step
  size_t ws_bucket_blocks_off = 0;  // int32 per bucket: blocks of its last launch
  size_t ws_partial_off = 0;        // double per slot
  size_t ws_bytes = 0;
};

namespace zero {

void set_error(const std::string& msg);
int fail(int code, const std::string& msg);
int cuda_fail(cudaError_t e, const char* what);

// partial-sum slots reserved for a bucket of `len` elements
int64_t rs_slots(int64_t len);
// grid the reduce-scatter kernel uses for a bucket of `len` elements (<= rs_slots(len))
cudaError_t rs_grid(int64_t len, int world, int dtype, int* grid);

// Launchers (kernels.cu). All return cudaSuccess or the launch error.
cudaError_t launch_state_init(void* ws, const zero_scaler_cfg& cfg, cudaStream_t s);
cudaError_t launch_state_write(void* ws, const zero_scaler_state& st, cudaStream_t s);
cudaError_t launch_selftest_wait(void* ws, cudaStream_t s);
// accumulate: R += the pass's sum (micro-batches after the first); want_sumsq: write
// the per-block sums of squares (the last pass of a step)
cudaError_t launch_reduce_scatter(int world, int dtype, const uint16_t* const* g, float* R,
                                  int64_t len, double* partial, int32_t* bucket_blocks,
                                  int32_t* device_error, int grid, cudaStream_t s,
                                  int accumulate = 0, int want_sumsq = 1, int store = 1);
// AdamW + cast with the reduced gradient formed again from W <= 2 resident replicas
// (g[r]: replica r at flat element 0)
cudaError_t launch_update_resident(int world, int gdt, int pdt, const uint16_t* const* g,
                                   float* master, float* m, float* v, void* params, int64_t n,
                                   const void* ws, cudaStream_t s);
cudaError_t launch_finalize(void* ws, const int32_t* bucket_blocks, int64_t slots_full,
                            const double* partial, int64_t n_buckets,
                            const zero_adamw_cfg& cfg, cudaStream_t s);
cudaError_t launch_update(int dtype, const float* R, float* master, float* m, float* v,
                          void* const* params, int n_params, int64_t n, const void* ws,
                          cudaStream_t s);
cudaError_t launch_local_sumsq(const int32_t* bucket_blocks, int64_t slots_full,
                               const double* partial, int64_t b0, int64_t b1, double* out,
                               cudaStream_t s);
cudaError_t launch_finalize_ranks(void* ws, const double* s_ranks, int world,
                                  const zero_adamw_cfg& cfg, cudaStream_t s);
cudaError_t launch_cast(int dtype, const float* master, void* params, int64_t n,
                        cudaStream_t s);
cudaError_t launch_replicate(const void* src, void* const* dst, int n_dst, int64_t n_halves,
                             cudaStream_t s);

}  // namespace zero
