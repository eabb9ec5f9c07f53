/*
 * zero_oracle.c -- CPU oracle of the ZeRO partitioned mixed-precision optimizer step.
 *
 * TEST INFRASTRUCTURE (see zero_oracle.h): plain single-threaded loops in flat order,
 * built with -O2 -ffp-contract=off. Shares no code with the CUDA library.
 */
#include "zero_oracle.h"

#include <math.h>
#include <stddef.h>
#include <string.h>

/* ============================ planner ============================ */
/* [Z1] 2.1: parameters are split automatically into N parts (one per GPU), with a
 * bucket strategy for communication; the FSDP comparison table in [Z1] 4.1 says ZeRO
 * divides by dynamic bucket rather than by module. Reading: tensors are flattened in
 * declared order, padded with zeros to a multiple of W*A, partition r is the r-th
 * contiguous block of P = N_pad/W elements, and buckets are fixed contiguous ranges
 * of reduce_bucket_size ELEMENTS over the padded flat space (the last one shorter). */

int oracle_plan_sizes(const int64_t* numels, int32_t n_tensors, int32_t world,
                      int64_t bucket, int32_t align, int64_t out[4]) {
  if (n_tensors < 0 || world < 1 || bucket < 1 || align < 1) return -1;
  int64_t n = 0;
  for (int32_t t = 0; t < n_tensors; ++t) {
    if (numels[t] < 0) return -1;
    if (numels[t] > INT64_MAX - n) return -1;
    n += numels[t];
  }
  const int64_t unit = (int64_t)world * (int64_t)align;
  const int64_t units = n / unit + (n % unit != 0);
  if (units > INT64_MAX / unit) return -1;
  const int64_t n_pad = units * unit;
  out[0] = n;
  out[1] = n_pad;
  out[2] = n_pad / world;
  out[3] = n_pad / bucket + (n_pad % bucket != 0);
  return 0;
}

int oracle_plan_tensor_offsets(const int64_t* numels, int32_t n_tensors, int64_t* offsets) {
  int64_t off = 0;
  for (int32_t t = 0; t < n_tensors; ++t) {
    offsets[t] = off;
    off += numels[t];
  }
  return 0;
}

static int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
static int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

int64_t oracle_plan_work_segments(int64_t n_pad, int32_t world, int64_t bucket,
                                  int64_t cap, int64_t* seg_bucket, int64_t* seg_rank,
                                  int64_t* seg_start, int64_t* seg_len) {
  const int64_t p = n_pad / world;
  int64_t count = 0;
  for (int64_t b = 0; b * bucket < n_pad; ++b) {
    const int64_t b0 = b * bucket, b1 = min64(b0 + bucket, n_pad);
    for (int32_t r = 0; r < world; ++r) {
      const int64_t lo = max64(b0, (int64_t)r * p), hi = min64(b1, (int64_t)(r + 1) * p);
      if (hi > lo) {
        if (count < cap) {
          seg_bucket[count] = b;
          seg_rank[count] = r;
          seg_start[count] = lo;
          seg_len[count] = hi - lo;
        }
        ++count;
      }
    }
  }
  return count;
}

int64_t oracle_plan_partition(const int64_t* numels, int32_t n_tensors, int64_t n_pad,
                              int32_t world, int32_t rank, int64_t cap, int64_t* tensor,
                              int64_t* off_in_tensor, int64_t* flat_off, int64_t* len) {
  const int64_t p = n_pad / world;
  const int64_t lo = (int64_t)rank * p, hi = lo + p;
  int64_t count = 0, off = 0;
  for (int32_t t = 0; t < n_tensors; ++t) {
    const int64_t a = max64(lo, off), b = min64(hi, off + numels[t]);
    if (b > a) {
      if (count < cap) {
        tensor[count] = t;
        off_in_tensor[count] = a - off;
        flat_off[count] = a;
        len[count] = b - a;
      }
      ++count;
    }
    off += numels[t];
  }
  /* the zero padding [N, N_pad) */
  const int64_t a = max64(lo, off), b = hi;
  if (b > a) {
    if (count < cap) {
      tensor[count] = -1;
      off_in_tensor[count] = a - off;
      flat_off[count] = a;
      len[count] = b - a;
    }
    ++count;
  }
  return count;
}

/* ============================ half conversions ============================ */
/* bf16: 1 sign, 8 exponent (bias 127), 7 fraction bits. fp16: 1, 5 (bias 15), 10. */

float oracle_half_to_f32(uint16_t h, int32_t dtype) {
  uint32_t bits;
  if (dtype == ORACLE_BF16) {
    bits = (uint32_t)h << 16; /* bf16 is the top half of an fp32 */
  } else {
    const uint32_t sign = (uint32_t)(h >> 15) << 31;
    const uint32_t e = (h >> 10) & 0x1f, f = h & 0x3ff;
    if (e == 0) {
      /* zero or subnormal: f * 2^-24 (exact in fp32) */
      float mag = (float)f * (1.0f / 16777216.0f);
      return sign ? -mag : mag;
    }
    if (e == 31)
      bits = sign | 0x7f800000u | (f << 13);
    else
      bits = sign | ((e - 15 + 127) << 23) | (f << 13);
  }
  float out;
  memcpy(&out, &bits, sizeof out);
  return out;
}

/* Round to the nearest representable value, ties to the one with an even last
 * fraction bit; beyond the largest finite value by half a unit or more -> inf.
 * Done by bracketing |x| between two neighbours on the target grid in exact double
 * arithmetic. */
uint16_t oracle_f32_to_half(float x, int32_t dtype) {
  const int p = dtype == ORACLE_BF16 ? 8 : 11;     /* significand bits incl. hidden */
  const int emin = dtype == ORACLE_BF16 ? -126 : -14;
  const int emax = dtype == ORACLE_BF16 ? 127 : 15;
  const int bias = dtype == ORACLE_BF16 ? 127 : 15;
  const int fbits = p - 1;
  const uint16_t sign = signbit(x) ? (uint16_t)0x8000 : (uint16_t)0;
  const uint16_t inf = dtype == ORACLE_BF16 ? (uint16_t)0x7f80 : (uint16_t)0x7c00;
  if (isnan(x)) return (uint16_t)(sign | inf | (1u << (fbits - 1)));
  const double a = fabs((double)x);
  if (isinf(a)) return (uint16_t)(sign | inf);
  if (a == 0.0) return sign;
  int e2;
  frexp(a, &e2); /* a = f * 2^e2, f in [0.5, 1): floor(log2 a) = e2 - 1 */
  int E = e2 - 1;
  if (E < emin) E = emin;
  const double ulp = ldexp(1.0, E - fbits);
  const double q = floor(a / ulp);
  const double dlo = a - q * ulp, dhi = (q + 1.0) * ulp - a;
  double r = q;
  if (dhi < dlo || (dhi == dlo && fmod(q, 2.0) != 0.0)) r = q + 1.0;
  const double value = r * ulp;
  const double max_finite = (2.0 - ldexp(1.0, -fbits)) * ldexp(1.0, emax);
  if (value > max_finite) return (uint16_t)(sign | inf);
  if (value < ldexp(1.0, emin)) /* subnormal: fraction counts units of 2^(emin-fbits) */
    return (uint16_t)(sign | (uint16_t)r);
  int ev;
  frexp(value, &ev);
  const int Ev = ev - 1;
  const double frac = value / ldexp(1.0, Ev - fbits) - ldexp(1.0, fbits);
  return (uint16_t)(sign | (uint16_t)((Ev + bias) << fbits) | (uint16_t)frac);
}

void oracle_f32_to_half_array(const float* x, uint16_t* out, int64_t n, int32_t dtype) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_half(x[i], dtype);
}

void oracle_half_to_f32_array(const uint16_t* h, float* out, int64_t n, int32_t dtype) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_half_to_f32(h[i], dtype);
}

/* ============================ the step ============================ */

/* Loss-scaler start state. [Z1] 3.3 and 5.1 name the knobs (loss_scale_window,
 * hysteresis, initial_scale_power, min_loss_scale) but not the rules; reading: the
 * scale starts at 2^initial_scale_power, the hysteresis budget at `hysteresis`, the
 * iteration counter at 0 and the last overflow at -1. */
void oracle_state_init(const oracle_scaler_cfg* cfg, oracle_state* st) {
  st->scale = cfg->dynamic ? ldexpf(1.0f, cfg->init_scale_power) : cfg->static_scale;
  st->cur_hysteresis = cfg->hysteresis;
  st->iter = 0;
  st->last_overflow_iter = -1;
  st->adam_t = 0;
}

/* [Z1] 2.1 / [Z3] technical insight: gradients are reduce-scattered so each rank keeps
 * the summed slice for its own parameters. Reading: a SUM (no averaging), in fp32,
 * in rank order 0..W-1. */
void oracle_reduce(int32_t world, int32_t gdtype, const uint16_t* const* grads, int64_t n,
                   float* R) {
  for (int64_t i = 0; i < n; ++i) {
    float acc = oracle_half_to_f32(grads[0][i], gdtype);
    for (int32_t r = 1; r < world; ++r) acc = acc + oracle_half_to_f32(grads[r][i], gdtype);
    R[i] = acc;
  }
}

void oracle_reduce_accumulate(int32_t world, int32_t gdtype, const uint16_t* const* grads,
                              int64_t n, float* R) {
  for (int64_t i = 0; i < n; ++i) {
    float acc = oracle_half_to_f32(grads[0][i], gdtype);
    for (int32_t r = 1; r < world; ++r) acc = acc + oracle_half_to_f32(grads[r][i], gdtype);
    R[i] = R[i] + acc;
  }
}

void oracle_sumsq(const float* R, int64_t n, double* S) {
  double acc = *S;
  for (int64_t i = 0; i < n; ++i) {
    const double r = (double)R[i];
    acc = acc + r * r;
  }
  *S = acc;
}

int32_t oracle_any_nonfinite(const float* R, int64_t n) {
  for (int64_t i = 0; i < n; ++i)
    if (!isfinite(R[i])) return 1;
  return 0;
}

/* Steps (2)-(4) of the step's scalar part.
 * - Overflow ([Z1] 3.3, 5.1, fp16 dynamic loss scaling): any non-finite reduced
 *   gradient or a non-finite S. Reading: an overflowing step is skipped whole.
 * - Norm: L2 norm of the unscaled gradient, sqrt(S)/scale in fp64.
 * - Clip ([Z1] 6, gradient_clipping 1.0): c = max_norm/(norm + 1e-6) when that is
 *   below 1, else 1; one fp32 multiplier k = fp32(c/scale) folds unscale and clip.
 * - Scaler transition, reading of loss_scale_window / hysteresis / min_loss_scale:
 *   on overflow, if the hysteresis budget is <= 1 the scale is divided by the factor
 *   (not below min_loss_scale), otherwise the budget drops by one, and the overflow
 *   iteration is recorded; on a good step, when (iter - last_overflow) is a multiple
 *   of the window the scale is multiplied by the factor and the budget is refilled.
 *   The iteration counter then advances.
 * - AdamW ([Z1] 3.1): applied-step counter t, bias corrections 1 - beta^t in fp64. */
void oracle_finalize(double S, int32_t nonfinite, const oracle_scaler_cfg* cfg,
                     const oracle_hparams* hp, oracle_state* st, oracle_scalars* out) {
  const float scale = st->scale;
  const int32_t overflow = (nonfinite || !isfinite(S)) ? 1 : 0;
  const double norm = sqrt(S) / (double)scale;
  double c = 1.0;
  if (!overflow && hp->max_grad_norm > 0.0) {
    const double cc = hp->max_grad_norm / (norm + 1e-6);
    if (cc < 1.0) c = cc;
  }
  out->sumsq = S;
  out->norm = norm;
  out->overflow = overflow;
  out->skipped = overflow;
  out->scale_used = scale;
  out->clip_coef = (float)c;
  out->k = (float)(c / (double)scale);

  if (cfg->dynamic) {
    if (overflow) {
      if (st->cur_hysteresis <= 1) {
        float s = st->scale / cfg->factor;
        st->scale = s > cfg->min_scale ? s : cfg->min_scale;
      } else {
        st->cur_hysteresis -= 1;
      }
      st->last_overflow_iter = st->iter;
    } else if ((st->iter - st->last_overflow_iter) % cfg->window == 0) {
      st->scale = st->scale * cfg->factor;
      st->cur_hysteresis = cfg->hysteresis;
    }
  }
  st->iter += 1;
  if (!overflow) st->adam_t += 1;

  out->next_scale = st->scale;
  out->hysteresis = st->cur_hysteresis;
  out->iter = st->iter;
  out->adam_t = st->adam_t;

  const double t = (double)st->adam_t;
  out->b1 = (float)hp->beta1;
  out->omb1 = (float)(1.0 - hp->beta1);
  out->b2 = (float)hp->beta2;
  out->omb2 = (float)(1.0 - hp->beta2);
  out->bc1 = (float)(1.0 - pow(hp->beta1, t));
  out->bc2 = (float)(1.0 - pow(hp->beta2, t));
  out->eps = (float)hp->eps;
  out->lr = (float)hp->lr;
  out->decay = (float)(1.0 - hp->lr * hp->weight_decay);
}

/* Step (4)-(5): [Z1] 2.1 each GPU updates only its own partition; [Z1] 3.1 AdamW with
 * lr and weight_decay; [Z3] FAQ: first and second moments beside fp32 master weights.
 * Reading: decoupled decay on the pre-update weight, bias-corrected moments, eps
 * outside the square root:
 *   g = R*k; m = b1*m + (1-b1)*g; v = b2*v + (1-b2)*(g*g);
 *   p = p*(1 - lr*wd) - lr * ((m/bc1) / (sqrt(v/bc2) + eps));
 * then the half copy of p goes to the same flat index of the gathered buffer, which
 * is the all-gather ([Z1] 2.1, parameters gathered by allgather). */
void oracle_adamw(int64_t n, const float* R, float* master, float* m, float* v,
                  uint16_t* params, int32_t pdtype, const oracle_scalars* sc) {
  if (sc->skipped) return;
  for (int64_t i = 0; i < n; ++i) {
    const float g = R[i] * sc->k;
    const float mi = sc->b1 * m[i] + sc->omb1 * g;
    const float vi = sc->b2 * v[i] + sc->omb2 * (g * g);
    const float t1 = mi / sc->bc1;
    const float t2 = sqrtf(vi / sc->bc2) + sc->eps;
    const float p = master[i] * sc->decay - sc->lr * (t1 / t2);
    m[i] = mi;
    v[i] = vi;
    master[i] = p;
    params[i] = oracle_f32_to_half(p, pdtype);
  }
}

#define ORACLE_MAX_WORLD 256

void oracle_step(int32_t world, int32_t gdtype, const uint16_t* const* grads, int64_t n_pad,
                 int64_t bucket, float* R, float* master, float* m, float* v,
                 uint16_t* params, int32_t pdtype, const oracle_scaler_cfg* cfg,
                 const oracle_hparams* hp, oracle_state* st, oracle_scalars* out) {
  const uint16_t* g[ORACLE_MAX_WORLD];
  double S = 0.0;
  int32_t nonfinite = 0;
  for (int64_t b0 = 0; b0 < n_pad; b0 += bucket) {
    const int64_t len = min64(bucket, n_pad - b0);
    for (int32_t r = 0; r < world; ++r) g[r] = grads[r] + b0;
    oracle_reduce(world, gdtype, g, len, R + b0);
    double Sb = 0.0;
    oracle_sumsq(R + b0, len, &Sb);
    S = S + Sb;
    nonfinite |= oracle_any_nonfinite(R + b0, len);
  }
  oracle_finalize(S, nonfinite, cfg, hp, st, out);
  oracle_adamw(n_pad, R, master, m, v, params, pdtype, out);
}

/* ============================ memory accounting ============================ */
/* [Z2] memory arithmetic: fp32 weights plus gradient, momentum and variance of the
 * same size; [Z2] stage table (ZeRO-1 ~4x, ZeRO-2 ~8x, ZeRO-3 tens of x); [Z1] 1.2.1
 * (8 GPUs save about 87.5% of optimizer-state memory). Reading (mixed precision, the
 * pages' fp16/bf16 + fp32-master setting): params 2 B, grads 2 B, optimizer state
 * 12 B (fp32 master, m, v) per parameter; stage s partitions the first s of
 * {optimizer state, gradients, parameters} over W ranks. */
int oracle_memory_per_rank(double psi, int32_t world, int32_t stage, double out[4]) {
  if (world < 1 || stage < 0 || stage > 3) return -1;
  const double w = (double)world;
  const double params = 2.0 * psi, grads = 2.0 * psi, optim = 12.0 * psi;
  out[2] = stage >= 1 ? optim / w : optim;
  out[1] = stage >= 2 ? grads / w : grads;
  out[0] = stage >= 3 ? params / w : params;
  out[3] = out[0] + out[1] + out[2];
  return 0;
}
