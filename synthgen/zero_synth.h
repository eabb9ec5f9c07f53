/*
 * zero_synth.h -- seeded synthetic inputs for the ZeRO optimizer-step workloads.
 *
 * This header is the ONE piece of code shared by the CUDA harness (synth_fill.cu)
 * and the CPU-oracle harness (synth_host.c). It draws numbers and nothing else:
 * no reduction, norm, clipping, loss-scaling, AdamW or cast of the optimizer step
 * lives here. Both sides include it, so a gradient or master value for a given
 * (seed, stream, step, index) is bit-identical on host and device.
 *
 * Generator: Philox4x32-10, the counter-based generator of Salmon, Moraes, Dror and
 * Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11), written from that
 * paper's definition (two 32x32->64 multiplies per round, Weyl key schedule).
 *
 * Normal approximation: Irwin-Hall with four 32-bit uniforms. The integer sum
 * s = u0+u1+u2+u3 - (2^33 - 2) has mean 0 and variance (2^64-1)/3, so
 * z = s * sqrt(3)/2^32 has mean 0 and variance 1 - 2^-64; tails stop at +-2*sqrt(3).
 * The value sigma*z is formed as ONE IEEE double multiply of the exact integer s by
 * a constant c = sigma*sqrt(3)/2^32 that the host computes once and hands to both
 * sides, so host and device results agree bit for bit.
 *
 * Rounding to bf16 / fp16 input bits is done here with integer operations on the
 * double's bit pattern (round to nearest, ties to even), again identical on both sides.
 */
#ifndef ZERO_SYNTH_H
#define ZERO_SYNTH_H

#include <stdint.h>

#ifdef __CUDACC__
#define SYNTH_HD __host__ __device__ __forceinline__
#else
#define SYNTH_HD static inline
#endif

/* Philox4x32 round multipliers and key increments (Salmon et al., SC'11, Philox-4x32). */
#define SYNTH_PHILOX_M0 0xD2511F53u
#define SYNTH_PHILOX_M1 0xCD9E8D57u
#define SYNTH_PHILOX_W0 0x9E3779B9u
#define SYNTH_PHILOX_W1 0xBB67AE85u

/* Stream identifiers (the second key word); the first key word is the seed. */
#define SYNTH_STREAM_INIT 0u          /* master-weight initialisation            */
#define SYNTH_STREAM_GRAD 1u          /* + replica index r: replica r gradients  */
#define SYNTH_STREAM_SPIKE 0x1000u    /* + replica index r: x8 spike selector     */
#define SYNTH_STREAM_INF 0x2000u      /* +inf injection sites                    */

/* Element dtype codes for generated half-precision buffers. */
#define SYNTH_BF16 0
#define SYNTH_FP16 1

typedef struct {
  uint32_t v[4];
} synth_u32x4;

SYNTH_HD synth_u32x4 synth_philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                         uint32_t c3, uint32_t k0, uint32_t k1) {
  for (int round = 0; round < 10; ++round) {
    const uint64_t p0 = (uint64_t)SYNTH_PHILOX_M0 * (uint64_t)c0;
    const uint64_t p1 = (uint64_t)SYNTH_PHILOX_M1 * (uint64_t)c2;
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    const uint32_t n0 = hi1 ^ c1 ^ k0;
    const uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
    k0 += SYNTH_PHILOX_W0;
    k1 += SYNTH_PHILOX_W1;
  }
  synth_u32x4 r;
  r.v[0] = c0;
  r.v[1] = c1;
  r.v[2] = c2;
  r.v[3] = c3;
  return r;
}

/* One Philox block for (seed, stream) at counter (index, step). */
SYNTH_HD synth_u32x4 synth_block(uint32_t seed, uint32_t stream, uint32_t step,
                                 uint64_t index) {
  return synth_philox4x32_10((uint32_t)index, (uint32_t)(index >> 32), step, 0u,
                             seed, stream);
}

/* Irwin-Hall(4) integer: sum of the four words minus their mean. |s| < 2^34. */
SYNTH_HD int64_t synth_irwin_hall4(synth_u32x4 u) {
  return (int64_t)u.v[0] + (int64_t)u.v[1] + (int64_t)u.v[2] + (int64_t)u.v[3] -
         (int64_t)((1ull << 33) - 2ull);
}

/* sigma * z for the block at (seed, stream, step, index); c = sigma*sqrt(3)/2^32. */
SYNTH_HD double synth_normal(uint32_t seed, uint32_t stream, uint32_t step,
                             uint64_t index, double c) {
  return (double)synth_irwin_hall4(synth_block(seed, stream, step, index)) * c;
}

/*
 * Round a double to a binary format with p significand bits (hidden bit included),
 * exponent bias `bias` and `ebits` exponent bits, nearest-even, returning the bits.
 * NaN -> quiet NaN, overflow -> inf, underflow -> subnormal or signed zero.
 */
SYNTH_HD uint16_t synth_round_double(double x, int p, int ebits, int bias) {
  union {
    double d;
    uint64_t u;
  } cv;
  cv.d = x;
  const uint64_t bits = cv.u;
  const uint16_t sign = (uint16_t)((bits >> 63) << (p - 1 + ebits));
  const int dexp = (int)((bits >> 52) & 0x7ff);
  uint64_t mant = bits & ((1ull << 52) - 1);
  const uint16_t exp_all = (uint16_t)(((1u << ebits) - 1u) << (p - 1));
  if (dexp == 0x7ff) {
    if (mant != 0) return (uint16_t)(sign | exp_all | (1u << (p - 2)));
    return (uint16_t)(sign | exp_all);
  }
  if (dexp == 0) return sign; /* double zero or subnormal: far below any half unit */
  const int e = dexp - 1023;  /* x = M * 2^(e-52), M = 2^52 + mant */
  const uint64_t M = (1ull << 52) | mant;
  const int emin = 1 - bias;
  int shift = 53 - p;
  if (e < emin) shift += emin - e;
  uint64_t q;
  if (shift > 54) {
    q = 0;
  } else {
    q = M >> shift;
    const uint64_t rem = M & ((1ull << shift) - 1ull);
    const uint64_t half = 1ull << (shift - 1);
    if (rem > half || (rem == half && (q & 1ull))) q += 1;
  }
  if (e < emin) {
    /* units of 2^(emin-p+1); q == 2^(p-1) encodes the smallest normal correctly */
    return (uint16_t)(sign | (uint16_t)q);
  }
  const int64_t E = (int64_t)e + bias;
  const uint64_t enc = ((uint64_t)E << (p - 1)) + (q - (1ull << (p - 1)));
  if ((enc >> (p - 1)) >= ((1ull << ebits) - 1ull)) return (uint16_t)(sign | exp_all);
  return (uint16_t)(sign | (uint16_t)enc);
}

SYNTH_HD uint16_t synth_to_half_bits(double x, int dtype) {
  return dtype == SYNTH_FP16 ? synth_round_double(x, 11, 5, 15)
                             : synth_round_double(x, 8, 8, 127);
}

SYNTH_HD uint16_t synth_inf_bits(int dtype) {
  return dtype == SYNTH_FP16 ? (uint16_t)0x7c00u : (uint16_t)0x7f80u;
}

/*
 * Gradient recipe. Replica r's gradient at buffer index j of step slot s:
 *   g = sigma_g * z(seed, GRAD + r, s, j)
 *   if spike_threshold > 0 and word0 of Philox(seed, SPIKE + r, s, j) < threshold: g *= 8
 *   g *= scale   (a power of two: the loss scale in force, 1 when loss scaling is off)
 *   bits = RNE(g) in the requested half type
 * c_grad = sigma_g*sqrt(3)/2^32 computed by the host.
 */
SYNTH_HD uint16_t synth_grad_bits(uint32_t seed, uint32_t replica, uint32_t slot,
                                  uint64_t j, double c_grad, uint32_t spike_threshold,
                                  double scale, int dtype) {
  double g = synth_normal(seed, SYNTH_STREAM_GRAD + replica, slot, j, c_grad);
  if (spike_threshold != 0u) {
    const synth_u32x4 h = synth_block(seed, SYNTH_STREAM_SPIKE + replica, slot, j);
    if (h.v[0] < spike_threshold) g *= 8.0;
  }
  g *= scale;
  return synth_to_half_bits(g, dtype);
}

/* Master initialisation for a random tensor: float(sigma_w * z(seed, INIT, 0, i)). */
SYNTH_HD float synth_master_value(uint32_t seed, uint64_t i, double c_init) {
  return (float)synth_normal(seed, SYNTH_STREAM_INIT, 0u, i, c_init);
}

/*
 * +inf injection site k (k = 0, 1, ...) of step t: flat index uniform in [0, n)
 * and replica uniform in [0, W), both by 64-bit / 32-bit modulo of Philox words.
 */
SYNTH_HD void synth_inf_site(uint32_t seed, uint32_t step, uint32_t k, uint64_t n,
                             uint32_t world, uint64_t* index, uint32_t* replica) {
  const synth_u32x4 u = synth_block(seed, SYNTH_STREAM_INF, step, (uint64_t)k);
  const uint64_t w64 = ((uint64_t)u.v[1] << 32) | (uint64_t)u.v[0];
  *index = n ? (w64 % n) : 0u;
  *replica = world ? (u.v[2] % world) : 0u;
}

#endif /* ZERO_SYNTH_H */
