/*
 * synth_fill.cu -- device fills of the seeded synthetic inputs (zero_synth.h).
 * Harness code: it creates inputs before a timed region and is never part of the
 * optimizer step. Values are bit-identical to synth_host.c for the same arguments.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include "zero_synth.h"

namespace {

__global__ void fill_grads_kernel(uint16_t* __restrict__ out, uint64_t j0, uint64_t n,
                                  uint32_t seed, uint32_t replica, uint32_t slot,
                                  double c_grad, uint32_t spike_threshold, double scale,
                                  int dtype) {
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t k = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride)
    out[k] = synth_grad_bits(seed, replica, slot, j0 + k, c_grad, spike_threshold, scale, dtype);
}

__global__ void fill_master_kernel(float* __restrict__ out, uint64_t i0, uint64_t n,
                                   uint32_t seed, double c_init) {
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t k = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride)
    out[k] = synth_master_value(seed, i0 + k, c_init);
}

int grid_for(uint64_t n) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  uint64_t want = (n + 255) / 256;
  uint64_t cap = (uint64_t)sms * 16;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  return (int)want;
}

}  // namespace

extern "C" {

/* Returns 0 on success, otherwise the cudaError_t of the launch. */
int synth_fill_grads_cuda(void* out, uint64_t j0, uint64_t n, uint32_t seed,
                          uint32_t replica, uint32_t slot, double c_grad,
                          uint32_t spike_threshold, double scale, int dtype,
                          cudaStream_t stream) {
  if (n == 0) return 0;
  fill_grads_kernel<<<grid_for(n), 256, 0, stream>>>((uint16_t*)out, j0, n, seed, replica,
                                                     slot, c_grad, spike_threshold, scale,
                                                     dtype);
  return (int)cudaGetLastError();
}

int synth_fill_master_cuda(float* out, uint64_t i0, uint64_t n, uint32_t seed,
                           double c_init, cudaStream_t stream) {
  if (n == 0) return 0;
  fill_master_kernel<<<grid_for(n), 256, 0, stream>>>(out, i0, n, seed, c_init);
  return (int)cudaGetLastError();
}

}  // extern "C"
