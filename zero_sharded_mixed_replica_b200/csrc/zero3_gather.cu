// zero3_gather.cu -- the ZeRO-3 all-gather of a layer's tensors from the ranks'
// parameter partitions into one contiguous buffer (a pure copy stream).
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "zero_b200.h"
#include "zero_internal.h"

namespace zero {
namespace {

constexpr int kGatherThreads = 256;
constexpr int kGatherMaxPieces = 64;
constexpr int64_t kGatherChunk = 1 << 16;  // elements per block per piece
constexpr int kGatherUnroll = 4;           // 16-byte loads in flight per thread

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

struct GatherArgs {
  const uint16_t* src[kGatherMaxPieces];
  uint16_t* dst[kGatherMaxPieces];
  int64_t len[kGatherMaxPieces];
};

// blockIdx.y: piece; blockIdx.x: a chunk of kGatherChunk elements of that piece.
__global__ void __launch_bounds__(kGatherThreads) gather_kernel(const __grid_constant__ GatherArgs a) {
  const int k = blockIdx.y;
  const int64_t lo = (int64_t)blockIdx.x * kGatherChunk;
  const int64_t len = a.len[k];
  if (lo >= len) return;
  const int64_t hi = lo + kGatherChunk < len ? lo + kGatherChunk : len;
  const uint16_t* s = a.src[k];
  uint16_t* d = a.dst[k];
  // 16-byte vectors when both sides reach alignment at the same element
  const uintptr_t sa = (uintptr_t)(s + lo), da = (uintptr_t)(d + lo);
  if ((sa & 15u) == (da & 15u) && (sa & 1u) == 0) {
    const int64_t head = (int64_t)(((16u - (da & 15u)) & 15u) / 2u);
    const int64_t h = lo + head < hi ? lo + head : hi;
    for (int64_t i = lo + threadIdx.x; i < h; i += kGatherThreads) d[i] = s[i];
    const int64_t nvec = (hi - h) / 8;
    const uint4* vs = (const uint4*)(s + h);
    uint4* vd = (uint4*)(d + h);
    for (int64_t v0 = threadIdx.x; v0 < nvec; v0 += kGatherUnroll * kGatherThreads) {
      uint4 x[kGatherUnroll];
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int64_t v = v0 + (int64_t)u * kGatherThreads;
        if (v < nvec) x[u] = ld_stream(vs + v);
      }
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int64_t v = v0 + (int64_t)u * kGatherThreads;
        if (v < nvec) vd[v] = x[u];
      }
    }
    for (int64_t i = h + 8 * nvec + threadIdx.x; i < hi; i += kGatherThreads) d[i] = s[i];
  } else {
    for (int64_t i = lo + threadIdx.x; i < hi; i += kGatherThreads) d[i] = s[i];
  }
}

}  // namespace
}  // namespace zero

using namespace zero;

extern "C" int zero3_gather(const zero_plan* plan, const int32_t* tensors, int32_t n_tensors,
                            const void* const* partitions, void* dst, void* stream) {
  if (!plan || (n_tensors > 0 && (!tensors || !partitions || !dst)))
    return fail(ZERO_EINVAL, "NULL argument");
  if (n_tensors < 0) return fail(ZERO_EINVAL, "n_tensors < 0");
  for (int r = 0; r < plan->world && n_tensors > 0; ++r)
    if (!partitions[r]) return fail(ZERO_EINVAL, "partitions[" + std::to_string(r) + "] is NULL");
  // pieces: each tensor split at partition boundaries
  std::vector<const uint16_t*> src;
  std::vector<uint16_t*> dd;
  std::vector<int64_t> len;
  int64_t out = 0;
  for (int32_t k = 0; k < n_tensors; ++k) {
    const int32_t t = tensors[k];
    if (t < 0 || (size_t)t >= plan->numel.size())
      return fail(ZERO_EINVAL, "tensor id " + std::to_string(t) + " out of range");
    int64_t i = plan->offset[t];
    const int64_t end = i + plan->numel[t];
    while (i < end) {
      const int64_t r = i / plan->p;
      const int64_t stop = (r + 1) * plan->p < end ? (r + 1) * plan->p : end;
      src.push_back((const uint16_t*)partitions[r] + (i - r * plan->p));
      dd.push_back((uint16_t*)dst + out);
      len.push_back(stop - i);
      out += stop - i;
      i = stop;
    }
  }
  for (size_t p0 = 0; p0 < src.size(); p0 += kGatherMaxPieces) {
    GatherArgs a{};
    int64_t maxlen = 0;
    const size_t np = src.size() - p0 < (size_t)kGatherMaxPieces ? src.size() - p0 : kGatherMaxPieces;
    for (size_t k = 0; k < np; ++k) {
      a.src[k] = src[p0 + k];
      a.dst[k] = dd[p0 + k];
      a.len[k] = len[p0 + k];
      if (a.len[k] > maxlen) maxlen = a.len[k];
    }
    const int64_t gx = (maxlen + kGatherChunk - 1) / kGatherChunk;
    if (gx == 0) continue;
    void* args[] = {&a};
    cudaError_t e = cudaLaunchKernel((const void*)gather_kernel, dim3((unsigned)gx, (unsigned)np),
                                     dim3(kGatherThreads), args, 0, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "gather launch");
  }
  return ZERO_OK;
}
