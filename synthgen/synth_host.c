/*
 * synth_host.c -- host fills of the seeded synthetic inputs (zero_synth.h).
 * Used by the CPU-oracle harness; OpenMP only splits index ranges, every value is
 * a pure function of (seed, stream, step, index), so the thread count never changes
 * a result. Holds none of the optimizer-step arithmetic.
 */
#include <stdint.h>
#include "zero_synth.h"

void synth_philox_host(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  synth_u32x4 r = synth_philox4x32_10(ctr[0], ctr[1], ctr[2], ctr[3], key[0], key[1]);
  for (int i = 0; i < 4; ++i) out[i] = r.v[i];
}

uint16_t synth_round_double_host(double x, int dtype) { return synth_to_half_bits(x, dtype); }

void synth_round_double_array_host(const double* x, uint16_t* out, int64_t n, int dtype) {
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < n; ++k) out[k] = synth_to_half_bits(x[k], dtype);
}

void synth_normal_array_host(double* out, uint64_t j0, int64_t n, uint32_t seed,
                             uint32_t stream, uint32_t step, double c) {
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < n; ++k) out[k] = synth_normal(seed, stream, step, j0 + (uint64_t)k, c);
}

void synth_fill_grads_host(uint16_t* out, uint64_t j0, int64_t n, uint32_t seed,
                           uint32_t replica, uint32_t slot, double c_grad,
                           uint32_t spike_threshold, double scale, int dtype) {
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < n; ++k)
    out[k] = synth_grad_bits(seed, replica, slot, j0 + (uint64_t)k, c_grad,
                             spike_threshold, scale, dtype);
}

void synth_fill_master_host(float* out, uint64_t i0, int64_t n, uint32_t seed, double c_init) {
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < n; ++k) out[k] = synth_master_value(seed, i0 + (uint64_t)k, c_init);
}

void synth_inf_site_host(uint32_t seed, uint32_t step, uint32_t k, uint64_t n,
                         uint32_t world, uint64_t* index, uint32_t* replica) {
  synth_inf_site(seed, step, k, n, world, index, replica);
}

/* Gradient bits at an explicit list of buffer indices (sampled checks at full size). */
void synth_grads_at_host(uint16_t* out, const uint64_t* j, int64_t n, uint32_t seed,
                         uint32_t replica, uint32_t slot, double c_grad,
                         uint32_t spike_threshold, double scale, int dtype) {
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < n; ++k)
    out[k] = synth_grad_bits(seed, replica, slot, j[k], c_grad, spike_threshold, scale, dtype);
}

/* Master values at an explicit list of flat indices. */
void synth_master_at_host(float* out, const uint64_t* i, int64_t n, uint32_t seed,
                          double c_init) {
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < n; ++k) out[k] = synth_master_value(seed, i[k], c_init);
}
