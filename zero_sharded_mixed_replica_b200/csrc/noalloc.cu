// noalloc.cu -- zero_reduce_sumsq_noalloc: the reduce-scatter reduction plus its fp64
// sum of squares, for callers that cannot allocate device memory. The per-block
// partial sums live in a file-scope device array instead of a caller workspace.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <string>

#include "zero_b200.h"
#include "zero_internal.h"

namespace zero {
namespace {

// Elements one block covers: 256 threads x one 8-element group each.
constexpr int64_t kNoallocBlockElems = (int64_t)kRsThreads * 8;
static_assert(ZERO_NOALLOC_MAX_ELEMS == (int64_t)ZERO_NOALLOC_MAX_BLOCKS * kNoallocBlockElems,
              "the element limit must match the scratch slots");

// Scratch: one fp64 partial sum per block, then one slot whose first 4 bytes receive
// the block count the reduction kernel records. Every GPU that loads the library holds
// this array until the process exits.
static __device__ __align__(256) double g_noalloc_scratch[ZERO_NOALLOC_MAX_BLOCKS + 32];

// Device address of g_noalloc_scratch per device, looked up once per device.
std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {nullptr};

cudaError_t scratch_for_current_device(double** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // the current device's copy
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = (double*)g_scratch_ptr[dev];
  return cudaSuccess;
}

// Sums partial[0 .. blocks) in a fixed order (thread-strided, then a block tree) into
// *out.
__global__ void __launch_bounds__(kFinalizeThreads)
    noalloc_sum_kernel(const double* __restrict__ partial, int32_t blocks, double* out) {
  double acc = 0.0;
  for (int32_t j = threadIdx.x; j < blocks; j += kFinalizeThreads) acc = __dadd_rn(acc, partial[j]);
  __shared__ double warp_sums[32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc = __dadd_rn(acc, __shfl_down_sync(0xffffffffu, acc, o));
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) warp_sums[wid] = acc;
  __syncthreads();
  if (wid == 0) {
    acc = lane < kFinalizeThreads / 32 ? warp_sums[lane] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc = __dadd_rn(acc, __shfl_down_sync(0xffffffffu, acc, o));
    if (lane == 0) *out = acc;
  }
}

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace
}  // namespace zero

using namespace zero;

extern "C" int zero_reduce_sumsq_noalloc(int32_t world_size, int32_t grad_dtype,
                                         const void* const* replica_grads, int64_t n,
                                         float* reduced, double* sumsq, void* stream) {
  if (world_size < 1 || world_size > ZERO_MAX_WORLD)
    return fail(ZERO_EINVAL, "world_size must be in [1, " + std::to_string(ZERO_MAX_WORLD) + "]");
  if (grad_dtype != ZERO_BF16 && grad_dtype != ZERO_FP16)
    return fail(ZERO_EINVAL, "grad_dtype must be ZERO_BF16 or ZERO_FP16");
  if (n < 0) return fail(ZERO_EINVAL, "n < 0");
  if (n > ZERO_NOALLOC_MAX_ELEMS)
    return fail(ZERO_ERANGE, "n = " + std::to_string(n) + " exceeds the limit of " +
                                 std::to_string((long long)ZERO_NOALLOC_MAX_ELEMS) +
                                 " elements per zero_reduce_sumsq_noalloc call (its " +
                                 std::to_string(ZERO_NOALLOC_MAX_BLOCKS) +
                                 " built-in partial-sum slots); split the range into calls");
  if (!replica_grads || !sumsq || (n > 0 && !reduced)) return fail(ZERO_EINVAL, "NULL argument");
  if (!aligned(sumsq, 8)) return fail(ZERO_EALIGN, "sumsq must be 8-byte aligned");
  if (n > 0 && !aligned(reduced, 16)) return fail(ZERO_EALIGN, "reduced must be 16-byte aligned");
  const uint16_t* g[ZERO_MAX_WORLD];
  for (int r = 0; r < world_size; ++r) {
    if (!replica_grads[r] && n > 0)
      return fail(ZERO_EINVAL, "replica_grads[" + std::to_string(r) + "] is NULL");
    if (!aligned(replica_grads[r], 16))
      return fail(ZERO_EALIGN, "replica_grads[" + std::to_string(r) + "] is not 16-byte aligned");
    g[r] = (const uint16_t*)replica_grads[r];
  }
  double* scratch = nullptr;
  cudaError_t e = scratch_for_current_device(&scratch);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the no-alloc scratch");
  int64_t blocks = (n + kNoallocBlockElems - 1) / kNoallocBlockElems;
  if (blocks < 1) blocks = 1;
  cudaStream_t s = (cudaStream_t)stream;
  // the reduce-scatter kernel with one block per 2048 elements, its partial sums and
  // block count written into the scratch array
  e = launch_reduce_scatter(world_size, grad_dtype, g, reduced, n, scratch,
                            (int32_t*)(scratch + ZERO_NOALLOC_MAX_BLOCKS), nullptr, (int)blocks, s);
  if (e != cudaSuccess) return cuda_fail(e, "no-alloc reduce launch");
  noalloc_sum_kernel<<<1, kFinalizeThreads, 0, s>>>(scratch, (int32_t)blocks, sumsq);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "no-alloc sum launch");
  return ZERO_OK;
}
