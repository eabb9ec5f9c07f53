// kernels.cu -- sm_100a kernels of the ZeRO partitioned optimizer step.
//
// All kernels here are HBM-bandwidth bound streams (about 0.3 flop per byte); none is
// a contraction, so none uses tensor cores. The step's kernels (bucket reduction,
// update) and the all-gather copies are persistent grids of one CTA per SM fed by TMA:
// a producer thread moves tiles between global and shared memory with 1-D bulk copies
// through an mbarrier ring while the CTA's other threads compute from shared memory;
// every wait is bounded. The small kernels (cast, state) are grid-stride loops over
// 16-byte vectors. Every byte of a step is touched once, so nothing is kept in L1.
//
// Floating-point operations on the data path use the explicitly rounded intrinsics
// (__fadd_rn, __fmul_rn, __fdiv_rn, __fsqrt_rn and the fp64 ones) so that the compiler
// cannot contract them into fused multiply-adds: every value is the correctly rounded
// result of the operation sequence the step defines.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zero_internal.h"

namespace zero {
namespace {

// ------------------------------------------------------------------ memory helpers

__device__ __forceinline__ uint4 ld_nc_u4(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

__device__ __forceinline__ float4 ld_nc_f4(const float* p) {
  float4 r;
  asm("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
      : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
      : "l"(p));
  return r;
}

// coherent load for data this kernel later overwrites at the same address
__device__ __forceinline__ float4 ld_f4(const float* p) {
  float4 r;
  asm("ld.global.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
      : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
      : "l"(p));
  return r;
}

__device__ __forceinline__ void st_f4(float* p, float a, float b, float c, float d) {
  asm volatile("st.global.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

__device__ __forceinline__ void st_u4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

__device__ __forceinline__ void st_cs_f4(float* p, float a, float b, float c, float d) {
  asm volatile("st.global.cs.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

// ------------------------------------------------------------------ TMA bulk copies

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Programmatic dependent launch. The step kernels are launched with programmatic stream
// serialization: one may be scheduled while its predecessor in the stream is finishing,
// so each sets up its shared memory, lets its own successor be scheduled, and then waits
// (griddepcontrol.wait: every prerequisite grid has completed and its writes are visible)
// before it reads or writes any global memory. Without a programmatic predecessor the
// wait returns at once.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// arrive and announce `bytes` of bulk copies that will complete on this barrier phase
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with the given parity to complete, at most about one second;
// false when the wait gave up.
constexpr uint64_t kWaitLimitNs = 1000000000ull;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity))
    if (global_ns() - t0 > kWaitLimitNs) return false;
  return true;
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar` (addresses and
// size multiples of 16 bytes). No multicast.
__device__ __forceinline__ void bulk_load(void* dst_smem, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst_smem)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// 1-D bulk copy shared -> global (TMA store), tracked by bulk async-groups of this thread
__device__ __forceinline__ void bulk_store(void* dst, const void* src_smem, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_addr(src_smem)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// at most one committed group still reading its shared-memory source
__device__ __forceinline__ void bulk_wait_read_but1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// every committed group complete (its writes performed)
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ------------------------------------------------------------------ half helpers

// dtype 0 = bf16, 1 = fp16
template <int DT>
__device__ __forceinline__ float half_bits_to_float(uint32_t h) {
  if constexpr (DT == ZERO_BF16) {
    return __uint_as_float(h << 16);  // bf16 is the high half of an fp32: exact
  } else {
    return __half2float(__ushort_as_half((unsigned short)h));  // exact widening
  }
}

// Two packed halves (element 2k in the low 16 bits) to two floats.
template <int DT>
__device__ __forceinline__ void unpack2(uint32_t w, float& lo, float& hi) {
  if constexpr (DT == ZERO_BF16) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xffff0000u);
  } else {
    lo = __half2float(__ushort_as_half((unsigned short)(w & 0xffffu)));
    hi = __half2float(__ushort_as_half((unsigned short)(w >> 16)));
  }
}

template <int DT>
__device__ __forceinline__ void unpack8(const uint4& x, float (&f)[8]) {
  unpack2<DT>(x.x, f[0], f[1]);
  unpack2<DT>(x.y, f[2], f[3]);
  unpack2<DT>(x.z, f[4], f[5]);
  unpack2<DT>(x.w, f[6], f[7]);
}

// Round to nearest even.
template <int DT>
__device__ __forceinline__ uint32_t float_to_half_bits(float x) {
  if constexpr (DT == ZERO_BF16) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x));
  } else {
    return (uint32_t)__half_as_ushort(__float2half_rn(x));
  }
}

template <int DT>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  return float_to_half_bits<DT>(lo) | (float_to_half_bits<DT>(hi) << 16);
}

// ------------------------------------------------------------------ reductions

// Sum over the block in a fixed order (shuffle tree per warp, then warp 0 over the
// warp sums); the result is valid in thread 0.
template <int THREADS>
__device__ __forceinline__ double block_sum(double x) {
  static_assert(THREADS % 32 == 0 && THREADS <= 1024, "block shape");
  __shared__ double warp_sums[32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = __dadd_rn(x, __shfl_down_sync(0xffffffffu, x, o));
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) warp_sums[wid] = x;
  __syncthreads();
  if (wid == 0) {
    x = lane < THREADS / 32 ? warp_sums[lane] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = __dadd_rn(x, __shfl_down_sync(0xffffffffu, x, o));
  }
  return x;
}

// ================================================================== K1: reduce-scatter

struct RsArgs {
  const uint16_t* g[ZERO_MAX_WORLD];  // replica r, element 0 of the bucket
  float* R;                           // reduced gradient, element 0 of the bucket
  double* partial;                    // this bucket's partial-sum slots
  int32_t* blocks;                    // where block 0 records the grid size
  int64_t len;                        // elements in the bucket
  int64_t head;                       // scalar elements before the first aligned group
  int64_t nvec;                       // aligned groups of 8 elements
  int32_t* device_error;              // sticky error word, or null
  int32_t accumulate;                 // 1: R += this pass's sum (later micro-batches)
  int32_t want_sumsq;                 // 1: accumulate the sum of squares (last pass)
  int32_t store;                      // 0: R is not written (only the sum of squares)
};

// Pipeline shape of the reduce-scatter: each of kRsStages shared-memory stages holds the
// W replica tiles of one tile (rs_tile<W>() halves each, about 64 KB per stage); one
// producer thread keeps the stages filled with 1-D bulk copies, kRsConsumers threads sum
// from shared memory. One CTA per SM.
constexpr int kRsStages = 3;
constexpr int kRsConsumers = 256;
constexpr int kRsTmaThreads = kRsConsumers + 32;

template <int W>
__host__ __device__ constexpr int rs_tile() {
  // a multiple of 2048 (one 8-element group per consumer thread) near 32768 / W
  return (32768 / W) / 2048 * 2048 < 2048 ? 2048 : (32768 / W) / 2048 * 2048;
}

template <int W>
__host__ __device__ constexpr size_t rs_smem_bytes() {
  return (size_t)kRsStages * W * rs_tile<W>() * sizeof(uint16_t) + 2 * kRsStages * sizeof(uint64_t);
}

// For every element i of the bucket: R[i] = ((g_0[i] + g_1[i]) + ...) + g_{W-1}[i] in
// fp32, and ss += R[i]^2 in fp64 (the square of an fp32 is exact in fp64, so the fused
// multiply-add rounds exactly like the separate add would). Full tiles of the aligned
// body [head, head + 8*nvec) go through the TMA pipeline; the last CTA takes the rest
// (the unaligned head, the groups after the last full tile, the last < 8 elements).
// Each CTA writes its ss to its own slot; the finalize kernel adds the slots in a fixed
// order. A wait that gives up (about one second) ends the CTA's pipeline early and
// records a code in *device_error when that pointer is set.
// The rank-ordered sums acc[0..7] of elements R[0..7]: add what earlier micro-batches
// left in R (accumulate), store, and add the squares of the stored values to ss.
__device__ __forceinline__ void finish8(const RsArgs& a, float* R, float (&acc)[8], double& ss) {
  if (a.accumulate) {
    const float4 o0 = ld_f4(R), o1 = ld_f4(R + 4);
    acc[0] = __fadd_rn(o0.x, acc[0]);
    acc[1] = __fadd_rn(o0.y, acc[1]);
    acc[2] = __fadd_rn(o0.z, acc[2]);
    acc[3] = __fadd_rn(o0.w, acc[3]);
    acc[4] = __fadd_rn(o1.x, acc[4]);
    acc[5] = __fadd_rn(o1.y, acc[5]);
    acc[6] = __fadd_rn(o1.z, acc[6]);
    acc[7] = __fadd_rn(o1.w, acc[7]);
  }
  // R is read back only after every bucket of the step: stream it past the caches
  if (a.store) {
    st_cs_f4(R, acc[0], acc[1], acc[2], acc[3]);
    st_cs_f4(R + 4, acc[4], acc[5], acc[6], acc[7]);
  }
  if (a.want_sumsq) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const double d = (double)acc[j];
      ss = __fma_rn(d, d, ss);
    }
  }
}

template <int W, int DT>
__global__ void __launch_bounds__(kRsTmaThreads, 1)
    rs_bucket_kernel(const __grid_constant__ RsArgs a) {
  constexpr int TILE = rs_tile<W>();
  constexpr uint32_t kStageBytes = (uint32_t)W * TILE * sizeof(uint16_t);
  extern __shared__ __align__(128) unsigned char smem[];
  uint16_t* stage_buf = (uint16_t*)smem;  // [kRsStages][W][TILE]
  uint64_t* full = (uint64_t*)(smem + (size_t)kRsStages * kStageBytes);
  uint64_t* empty = full + kRsStages;
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int st = 0; st < kRsStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kRsConsumers / 32);
    }
    mbar_init_fence();
  }
  __syncthreads();
  pdl_launch_dependents();
  pdl_wait();

  const int64_t n_tiles = (8 * a.nvec) / TILE;
  const int64_t G = gridDim.x;
  double ss = 0.0;

  if (tid >= kRsConsumers) {
    if (tid == kRsConsumers) {  // producer
      int64_t k = 0;
      for (int64_t t = blockIdx.x; t < n_tiles; t += G, ++k) {
        const int st = (int)(k % kRsStages);
        if (k >= kRsStages && !mbar_wait(&empty[st], (uint32_t)((k / kRsStages - 1) & 1))) {
          if (a.device_error) atomicOr(a.device_error, 8);
          break;
        }
        mbar_arrive_expect_tx(&full[st], kStageBytes);
        uint16_t* dst = stage_buf + (size_t)st * W * TILE;
        const int64_t off = a.head + t * TILE;
#pragma unroll
        for (int r = 0; r < W; ++r)
          bulk_load(dst + r * TILE, a.g[r] + off, TILE * sizeof(uint16_t), &full[st]);
      }
      for (int64_t j = k > kRsStages ? k - kRsStages : 0; j < k; ++j)
        if (!mbar_wait(&full[j % kRsStages], (uint32_t)((j / kRsStages) & 1)) && a.device_error)
          atomicOr(a.device_error, 32);
    }
  } else {
    int64_t k = 0;
    for (int64_t t = blockIdx.x; t < n_tiles; t += G, ++k) {
      const int st = (int)(k % kRsStages);
      if (!mbar_wait(&full[st], (uint32_t)((k / kRsStages) & 1))) {
        if (a.device_error) atomicOr(a.device_error, 16);
        break;
      }
      const uint16_t* src = stage_buf + (size_t)st * W * TILE;
      const int64_t off = a.head + t * TILE;
#pragma unroll
      for (int q = 0; q < TILE / (8 * kRsConsumers); ++q) {
        const int e = (q * kRsConsumers + tid) * 8;
        float acc[8];
        unpack8<DT>(*(const uint4*)(src + e), acc);
#pragma unroll
        for (int r = 1; r < W; ++r) {
          float x[8];
          unpack8<DT>(*(const uint4*)(src + r * TILE + e), x);
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[j] = __fadd_rn(acc[j], x[j]);
        }
        finish8(a, a.R + off + e, acc, ss);
      }
      __syncwarp();
      if ((tid & 31) == 0) mbar_arrive(&empty[st]);
    }

    if (blockIdx.x == G - 1) {
      // aligned groups after the last full tile, with plain 16-byte loads
      const int64_t vec_end = a.head + 8 * a.nvec;
      for (int64_t e = a.head + n_tiles * TILE + 8 * (int64_t)tid; e < vec_end;
           e += 8 * kRsConsumers) {
        float acc[8];
        unpack8<DT>(ld_nc_u4(a.g[0] + e), acc);
#pragma unroll
        for (int r = 1; r < W; ++r) {
          float x[8];
          unpack8<DT>(ld_nc_u4(a.g[r] + e), x);
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[j] = __fadd_rn(acc[j], x[j]);
        }
        finish8(a, a.R + e, acc, ss);
      }
      // scalar elements: the unaligned head [0, head) and the last (len - vec_end)
      const int64_t n_scalar = a.head + (a.len - vec_end);
      for (int64_t q = tid; q < n_scalar; q += kRsConsumers) {
        const int64_t i = q < a.head ? q : vec_end + (q - a.head);
        float acc = half_bits_to_float<DT>(a.g[0][i]);
#pragma unroll
        for (int r = 1; r < W; ++r) acc = __fadd_rn(acc, half_bits_to_float<DT>(a.g[r][i]));
        if (a.accumulate) acc = __fadd_rn(a.R[i], acc);
        if (a.store) a.R[i] = acc;
        if (a.want_sumsq) {
          const double d = (double)acc;
          ss = __fma_rn(d, d, ss);
        }
      }
    }
  }
  ss = block_sum<kRsTmaThreads>(ss);
  if (tid == 0) {
    a.partial[blockIdx.x] = ss;
    if (blockIdx.x == 0) *a.blocks = (int32_t)gridDim.x;
  }
}

template <int W, int DT>
const void* rs_kernel_ptr() {
  return (const void*)rs_bucket_kernel<W, DT>;
}

template <int W>
size_t rs_smem_for() {
  return rs_smem_bytes<W>();
}

typedef const void* (*KernelGetter)();

template <int DT, int... Ws>
struct RsTable {
  static const void* get(int w) {
    const void* ptrs[] = {rs_kernel_ptr<Ws, DT>()...};
    return ptrs[w - 1];
  }
  static size_t smem(int w) {
    const size_t bytes[] = {rs_smem_for<Ws>()...};
    return bytes[w - 1];
  }
};

using RsBf16 = RsTable<ZERO_BF16, 1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15, 16>;
using RsFp16 = RsTable<ZERO_FP16, 1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15, 16>;

const void* rs_kernel_for(int world, int dtype) {
  return dtype == ZERO_BF16 ? RsBf16::get(world) : RsFp16::get(world);
}

size_t rs_smem_for_world(int world) { return RsBf16::smem(world); }

// ================================================================== K2: finalize

__device__ double pow_int(double x, int64_t n) {
  // x^n by binary exponentiation, every product rounded (no contraction)
  double result = 1.0, base = x;
  while (n > 0) {
    if (n & 1) result = __dmul_rn(result, base);
    base = __dmul_rn(base, base);
    n >>= 1;
  }
  return result;
}

// Everything the step decides from S, done by one thread: overflow (S not finite), the
// unscaled norm, the clip coefficient, the one fp32 multiplier k, the loss-scaler
// transition, the step counter and the fp32 constants of the update.
__device__ void finalize_scalars(WsHeader* h, double S, const zero_adamw_cfg& cfg) {
  const float scale = h->scale;
  const int32_t overflow = isfinite(S) ? 0 : 1;
  const double norm = __ddiv_rn(__dsqrt_rn(S), (double)scale);
  double c = 1.0;
  if (!overflow && cfg.max_grad_norm > 0.0) {
    const double cc = __ddiv_rn(cfg.max_grad_norm, __dadd_rn(norm, 1e-6));
    if (cc < 1.0) c = cc;
  }
  const float k = __double2float_rn(__ddiv_rn(c, (double)scale));

  // loss-scaler transition
  if (h->dynamic) {
    if (overflow) {
      if (h->cur_hysteresis <= 1) {
        const float s = __fdiv_rn(h->scale, h->factor);
        h->scale = s > h->min_scale ? s : h->min_scale;
      } else {
        h->cur_hysteresis -= 1;
      }
      h->last_overflow_iter = h->iter;
    } else if ((h->iter - h->last_overflow_iter) % h->window == 0) {
      h->scale = __fmul_rn(h->scale, h->factor);
      h->cur_hysteresis = h->hysteresis_cfg;
    }
  }
  h->iter += 1;
  if (!overflow) h->adam_t += 1;
  const int64_t t = h->adam_t;

  h->k = k;
  h->b1 = __double2float_rn(cfg.beta1);
  h->omb1 = __double2float_rn(__dsub_rn(1.0, cfg.beta1));
  h->b2 = __double2float_rn(cfg.beta2);
  h->omb2 = __double2float_rn(__dsub_rn(1.0, cfg.beta2));
  h->bc1 = __double2float_rn(__dsub_rn(1.0, pow_int(cfg.beta1, t)));
  h->bc2 = __double2float_rn(__dsub_rn(1.0, pow_int(cfg.beta2, t)));
  h->eps = __double2float_rn(cfg.eps);
  h->lr = __double2float_rn(cfg.lr);
  h->decay = __double2float_rn(__dsub_rn(1.0, __dmul_rn(cfg.lr, cfg.weight_decay)));
  h->skip = overflow;

  zero_step_result& r = h->result;
  r.global_norm = norm;
  r.sumsq = S;
  r.clip_coef = __double2float_rn(c);
  r.scale_used = scale;
  r.next_scale = h->scale;
  r.k = k;
  r.overflow = overflow;
  r.skipped = overflow;
  r.hysteresis = h->cur_hysteresis;
  r.iter = h->iter;
  r.adam_t = t;  // r.device_error is left as it is: sticky until zero_state_init
}

// Sum of the partial-sum slots of buckets [b0, b1) in a fixed order: each thread walks
// the buckets in order and its own slots in order, then the block tree. Valid in thread 0.
__device__ double sum_bucket_slots(const int32_t* __restrict__ bucket_blocks, int64_t slots_full,
                                   const double* __restrict__ partial, int64_t b0, int64_t b1) {
  double acc = 0.0;
  for (int64_t b = b0; b < b1; ++b) {
    const int32_t nb = bucket_blocks[b];
    const double* p = partial + b * slots_full;
    for (int j = threadIdx.x; j < nb; j += kFinalizeThreads) acc = __dadd_rn(acc, p[j]);
  }
  return block_sum<kFinalizeThreads>(acc);
}

// Single process: S over every bucket, then the scalar step.
__global__ void __launch_bounds__(kFinalizeThreads)
    finalize_kernel(WsHeader* h, const int32_t* __restrict__ bucket_blocks, int64_t slots_full,
                    const double* __restrict__ partial, int64_t n_buckets, zero_adamw_cfg cfg) {
  pdl_launch_dependents();
  pdl_wait();
  const double S = sum_bucket_slots(bucket_blocks, slots_full, partial, 0, n_buckets);
  if (threadIdx.x == 0) finalize_scalars(h, S, cfg);
}

// One rank: the sum over the buckets its partition meets, for the cross-rank exchange.
__global__ void __launch_bounds__(kFinalizeThreads)
    local_sumsq_kernel(const int32_t* __restrict__ bucket_blocks, int64_t slots_full,
                       const double* __restrict__ partial, int64_t b0, int64_t b1,
                       double* out) {
  const double S = sum_bucket_slots(bucket_blocks, slots_full, partial, b0, b1);
  if (threadIdx.x == 0) *out = S;
}

// One rank, after the exchange: S = ((s_0 + s_1) + ...) + s_{W-1} in rank order, so every
// rank computes the same S, then the scalar step.
__global__ void finalize_ranks_kernel(WsHeader* h, const double* __restrict__ s_ranks,
                                      int32_t world, zero_adamw_cfg cfg) {
  double S = s_ranks[0];
  for (int32_t r = 1; r < world; ++r) S = __dadd_rn(S, s_ranks[r]);
  finalize_scalars(h, S, cfg);
}

// ================================================================== K3: AdamW + cast

struct UpArgs {
  const float* R;
  float* p;
  float* m;
  float* v;
  uint16_t* out[ZERO_MAX_WORLD];  // gathered half buffers (element 0 of this range)
  int32_t n_out;
  int64_t n;
  const WsHeader* h;
  int32_t* device_error;  // &h->result.device_error
};

struct AdamConsts {
  float k, b1, omb1, b2, omb2, bc1, bc2, eps, lr, decay;
};

// One element, in the step's operation order, each operation rounded.
__device__ __forceinline__ void adamw1(const AdamConsts& c, float r, float& p, float& m,
                                       float& v) {
  const float g = __fmul_rn(r, c.k);
  m = __fadd_rn(__fmul_rn(c.b1, m), __fmul_rn(c.omb1, g));
  v = __fadd_rn(__fmul_rn(c.b2, v), __fmul_rn(c.omb2, __fmul_rn(g, g)));
  const float t1 = __fdiv_rn(m, c.bc1);
  const float t2 = __fadd_rn(__fsqrt_rn(__fdiv_rn(v, c.bc2)), c.eps);
  p = __fsub_rn(__fmul_rn(p, c.decay), __fmul_rn(c.lr, __fdiv_rn(t1, t2)));
}

// Pipeline shape: tiles of kUpTile elements; each of kUpStages shared-memory stages holds
// the R, p, m, v tiles (4 x 16 KB); one producer thread keeps the stages filled with
// 1-D bulk copies while kUpConsumers threads compute from shared memory and store the
// results straight to global memory. One CTA per SM (128 KB of shared memory). The
// update is heavy per element (three divisions and a square root): 16 consumer warps
// with two stages sustain about 10 % more bandwidth than 8 warps with three stages
// (measured over 2^30 elements: 6.50 against 5.90 TB/s back to back).
constexpr int kUpTile = 4096;
constexpr int kUpStages = 2;
constexpr int kUpConsumers = 512;
constexpr int kUpTmaThreads = kUpConsumers + 32;  // + one producer warp
constexpr size_t kUpStageBytes = 4ull * kUpTile * sizeof(float);
constexpr size_t kUpSmemBytes = kUpStages * kUpStageBytes + 2 * kUpStages * sizeof(uint64_t);

// AdamW + half cast over [0, n): full tiles through the TMA pipeline, the last
// n % kUpTile elements by the last CTA with plain loads. Returns at once (every thread)
// when the finalize step decided to skip. A wait that gives up (about one second)
// records a code in *device_error and ends the CTA's work early.
template <int DT>
__global__ void __launch_bounds__(kUpTmaThreads, 1)
    adamw_cast_kernel(const __grid_constant__ UpArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  float* stage_buf = (float*)smem;  // [kUpStages][R, p, m, v][kUpTile]
  uint64_t* full = (uint64_t*)(smem + kUpStages * kUpStageBytes);
  uint64_t* empty = full + kUpStages;
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int st = 0; st < kUpStages; ++st) {
      mbar_init(&full[st], 1);                   // the producer's expect_tx arrival
      mbar_init(&empty[st], kUpConsumers / 32);  // one arrival per consumer warp
    }
    mbar_init_fence();
  }
  __syncthreads();
  pdl_launch_dependents();
  pdl_wait();

  const WsHeader* h = a.h;
  if (h->skip) return;  // overflow: the whole step is skipped (every thread)
  AdamConsts c;
  c.k = h->k;
  c.b1 = h->b1;
  c.omb1 = h->omb1;
  c.b2 = h->b2;
  c.omb2 = h->omb2;
  c.bc1 = h->bc1;
  c.bc2 = h->bc2;
  c.eps = h->eps;
  c.lr = h->lr;
  c.decay = h->decay;

  const int64_t n_tiles = a.n / kUpTile;
  const int64_t G = gridDim.x;

  if (tid >= kUpConsumers) {
    // producer warp: one thread issues the bulk copies
    if (tid == kUpConsumers) {
      int64_t k = 0;
      for (int64_t t = blockIdx.x; t < n_tiles; t += G, ++k) {
        const int st = (int)(k % kUpStages);
        if (k >= kUpStages &&
            !mbar_wait(&empty[st], (uint32_t)((k / kUpStages - 1) & 1))) {
          atomicOr(a.device_error, 1);
          break;
        }
        if (*(volatile int32_t*)a.device_error) break;
        mbar_arrive_expect_tx(&full[st], (uint32_t)kUpStageBytes);
        const int64_t off = t * kUpTile;
        float* dst = stage_buf + (size_t)st * 4 * kUpTile;
        bulk_load(dst, a.R + off, kUpTile * 4, &full[st]);
        bulk_load(dst + kUpTile, a.p + off, kUpTile * 4, &full[st]);
        bulk_load(dst + 2 * kUpTile, a.m + off, kUpTile * 4, &full[st]);
        bulk_load(dst + 3 * kUpTile, a.v + off, kUpTile * 4, &full[st]);
      }
      // before the CTA exits: the copies of the last stages must have landed
      for (int64_t j = k > kUpStages ? k - kUpStages : 0; j < k; ++j)
        if (!mbar_wait(&full[j % kUpStages], (uint32_t)((j / kUpStages) & 1)))
          atomicOr(a.device_error, 4);
    }
    return;
  }

  // consumers: each thread takes 4 consecutive elements per 1024-element slice
  int64_t k = 0;
  for (int64_t t = blockIdx.x; t < n_tiles; t += G, ++k) {
    const int st = (int)(k % kUpStages);
    if (!mbar_wait(&full[st], (uint32_t)((k / kUpStages) & 1))) {
      atomicOr(a.device_error, 2);
      break;
    }
    const float* src = stage_buf + (size_t)st * 4 * kUpTile;
    const int64_t off = t * kUpTile;
#pragma unroll
    for (int q = 0; q < kUpTile / (4 * kUpConsumers); ++q) {
      const int e = (q * kUpConsumers + tid) * 4;
      const float4 r = *(const float4*)(src + e);
      float4 p = *(const float4*)(src + kUpTile + e);
      float4 m = *(const float4*)(src + 2 * kUpTile + e);
      float4 v = *(const float4*)(src + 3 * kUpTile + e);
      adamw1(c, r.x, p.x, m.x, v.x);
      adamw1(c, r.y, p.y, m.y, v.y);
      adamw1(c, r.z, p.z, m.z, v.z);
      adamw1(c, r.w, p.w, m.w, v.w);
      st_f4(a.p + off + e, p.x, p.y, p.z, p.w);
      st_f4(a.m + off + e, m.x, m.y, m.z, m.w);
      st_f4(a.v + off + e, v.x, v.y, v.z, v.w);
      const uint2 hv = make_uint2(pack2<DT>(p.x, p.y), pack2<DT>(p.z, p.w));
      for (int d = 0; d < a.n_out; ++d) *(uint2*)(a.out[d] + off + e) = hv;
    }
    __syncwarp();
    if ((tid & 31) == 0) mbar_arrive(&empty[st]);
  }

  // the ragged tail after the last full tile
  if (blockIdx.x == G - 1) {
    for (int64_t i = n_tiles * kUpTile + tid; i < a.n; i += kUpConsumers) {
      float p = a.p[i], m = a.m[i], v = a.v[i];
      adamw1(c, a.R[i], p, m, v);
      a.p[i] = p;
      a.m[i] = m;
      a.v[i] = v;
      const uint16_t hb = (uint16_t)float_to_half_bits<DT>(p);
      for (int d = 0; d < a.n_out; ++d) a.out[d][i] = hb;
    }
  }
}

// ================================================================== K3': resident replicas

// AdamW + cast for a step whose W replica gradients are still resident when the update
// runs (worth it for W <= 2): the reduced gradient of every element is formed again from
// the replica tiles -- the same rank-ordered fp32 sum as the bucket kernel, so the same
// bits -- instead of being stored by the bucket kernel and read back. A step then moves
// 4W + 26 bytes per parameter instead of 2W + 34. Pipeline as K3; a stage holds the W
// replica tiles (halves) and the p, m, v tiles (fp32) of kUpTile elements.
constexpr int kResMaxWorld = 2;
struct UpResArgs {
  const uint16_t* g[kResMaxWorld];  // replica r, element 0 of the flat space
  float* p;
  float* m;
  float* v;
  uint16_t* out;  // the gathered half buffer
  int64_t n;
  const WsHeader* h;
  int32_t* device_error;
};

template <int W>
__host__ __device__ constexpr size_t up_res_stage_bytes() {
  return (size_t)kUpTile * (W * sizeof(uint16_t) + 3 * sizeof(float));
}
template <int W>
__host__ __device__ constexpr size_t up_res_smem_bytes() {
  return kUpStages * up_res_stage_bytes<W>() + 2 * kUpStages * sizeof(uint64_t);
}

template <int GD>
__device__ __forceinline__ void unpack4(const uint2& x, float (&f)[4]) {
  unpack2<GD>(x.x, f[0], f[1]);
  unpack2<GD>(x.y, f[2], f[3]);
}

template <int W, int GD, int PD>
__global__ void __launch_bounds__(kUpTmaThreads, 1)
    adamw_resident_kernel(const __grid_constant__ UpResArgs a) {
  constexpr size_t kStage = up_res_stage_bytes<W>();
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = (uint64_t*)(smem + kUpStages * kStage);
  uint64_t* empty = full + kUpStages;
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int st = 0; st < kUpStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kUpConsumers / 32);
    }
    mbar_init_fence();
  }
  __syncthreads();
  pdl_launch_dependents();
  pdl_wait();

  const WsHeader* h = a.h;
  if (h->skip) return;  // overflow: the whole step is skipped (every thread)
  AdamConsts c;
  c.k = h->k;
  c.b1 = h->b1;
  c.omb1 = h->omb1;
  c.b2 = h->b2;
  c.omb2 = h->omb2;
  c.bc1 = h->bc1;
  c.bc2 = h->bc2;
  c.eps = h->eps;
  c.lr = h->lr;
  c.decay = h->decay;

  const int64_t n_tiles = a.n / kUpTile;
  const int64_t G = gridDim.x;

  if (tid >= kUpConsumers) {
    if (tid == kUpConsumers) {  // producer
      int64_t k = 0;
      for (int64_t t = blockIdx.x; t < n_tiles; t += G, ++k) {
        const int st = (int)(k % kUpStages);
        if (k >= kUpStages &&
            !mbar_wait(&empty[st], (uint32_t)((k / kUpStages - 1) & 1))) {
          atomicOr(a.device_error, 1);
          break;
        }
        if (*(volatile int32_t*)a.device_error) break;
        mbar_arrive_expect_tx(&full[st], (uint32_t)kStage);
        const int64_t off = t * kUpTile;
        unsigned char* dst = smem + st * kStage;
#pragma unroll
        for (int r = 0; r < W; ++r)
          bulk_load(dst + (size_t)r * kUpTile * sizeof(uint16_t), a.g[r] + off,
                    kUpTile * sizeof(uint16_t), &full[st]);
        float* f = (float*)(dst + (size_t)W * kUpTile * sizeof(uint16_t));
        bulk_load(f, a.p + off, kUpTile * 4, &full[st]);
        bulk_load(f + kUpTile, a.m + off, kUpTile * 4, &full[st]);
        bulk_load(f + 2 * kUpTile, a.v + off, kUpTile * 4, &full[st]);
      }
      for (int64_t j = k > kUpStages ? k - kUpStages : 0; j < k; ++j)
        if (!mbar_wait(&full[j % kUpStages], (uint32_t)((j / kUpStages) & 1)))
          atomicOr(a.device_error, 4);
    }
    return;
  }

  int64_t k = 0;
  for (int64_t t = blockIdx.x; t < n_tiles; t += G, ++k) {
    const int st = (int)(k % kUpStages);
    if (!mbar_wait(&full[st], (uint32_t)((k / kUpStages) & 1))) {
      atomicOr(a.device_error, 2);
      break;
    }
    const unsigned char* base = smem + st * kStage;
    const uint16_t* gs = (const uint16_t*)base;
    const float* fs = (const float*)(base + (size_t)W * kUpTile * sizeof(uint16_t));
    const int64_t off = t * kUpTile;
#pragma unroll
    for (int q = 0; q < kUpTile / (4 * kUpConsumers); ++q) {
      const int e = (q * kUpConsumers + tid) * 4;
      float r[4];
      unpack4<GD>(*(const uint2*)(gs + e), r);
#pragma unroll
      for (int w = 1; w < W; ++w) {
        float x[4];
        unpack4<GD>(*(const uint2*)(gs + w * kUpTile + e), x);
#pragma unroll
        for (int j = 0; j < 4; ++j) r[j] = __fadd_rn(r[j], x[j]);
      }
      float4 p = *(const float4*)(fs + e);
      float4 m = *(const float4*)(fs + kUpTile + e);
      float4 v = *(const float4*)(fs + 2 * kUpTile + e);
      adamw1(c, r[0], p.x, m.x, v.x);
      adamw1(c, r[1], p.y, m.y, v.y);
      adamw1(c, r[2], p.z, m.z, v.z);
      adamw1(c, r[3], p.w, m.w, v.w);
      st_f4(a.p + off + e, p.x, p.y, p.z, p.w);
      st_f4(a.m + off + e, m.x, m.y, m.z, m.w);
      st_f4(a.v + off + e, v.x, v.y, v.z, v.w);
      *(uint2*)(a.out + off + e) = make_uint2(pack2<PD>(p.x, p.y), pack2<PD>(p.z, p.w));
    }
    __syncwarp();
    if ((tid & 31) == 0) mbar_arrive(&empty[st]);
  }

  // the ragged tail after the last full tile
  if (blockIdx.x == G - 1) {
    for (int64_t i = n_tiles * kUpTile + tid; i < a.n; i += kUpConsumers) {
      float r = half_bits_to_float<GD>(a.g[0][i]);
#pragma unroll
      for (int w = 1; w < W; ++w) r = __fadd_rn(r, half_bits_to_float<GD>(a.g[w][i]));
      float p = a.p[i], m = a.m[i], v = a.v[i];
      adamw1(c, r, p, m, v);
      a.p[i] = p;
      a.m[i] = m;
      a.v[i] = v;
      a.out[i] = (uint16_t)float_to_half_bits<PD>(p);
    }
  }
}

// ================================================================== small kernels

template <int DT>
__global__ void __launch_bounds__(kUpThreads)
    cast_kernel(const float* __restrict__ master, uint16_t* __restrict__ out, int64_t n) {
  const int64_t nthr = (int64_t)gridDim.x * kUpThreads;
  const int64_t tid = (int64_t)blockIdx.x * kUpThreads + threadIdx.x;
  const int64_t nvec = n / 8;
  for (int64_t vi = tid; vi < nvec; vi += nthr) {
    const float4 a = ld_nc_f4(master + vi * 8), b = ld_nc_f4(master + vi * 8 + 4);
    st_u4(out + vi * 8, pack2<DT>(a.x, a.y), pack2<DT>(a.z, a.w), pack2<DT>(b.x, b.y),
          pack2<DT>(b.z, b.w));
  }
  for (int64_t i = nvec * 8 + tid; i < n; i += nthr) out[i] = (uint16_t)float_to_half_bits<DT>(master[i]);
}

constexpr int kReplicateMax = 16;
struct ReplicateArgs {
  const uint16_t* src;
  uint16_t* dst[kReplicateMax];
  int n_dst;
  int64_t n;
};

// K4: copies of the gathered buffer into per-rank buffers, moved by the TMA engine alone.
// Thread 0 of each CTA bulk-loads 32 KB tiles (tile blockIdx + j * gridDim) into a
// 4-stage shared-memory ring and bulk-stores each landed tile to every destination (one
// bulk group per tile); a stage is reloaded once the stores of its previous tile have read
// it. The elements after the last full tile are copied by the last CTA's warp. A load
// wait that gives up (about one second) ends the ring; the CTA then waits (bounded) for
// its copies in flight and copies its remaining tiles with plain loads, so the result
// stays complete. Sources and destinations are 16-byte aligned (checked by the caller).
constexpr int kRepStages = 4;
constexpr int kRepTileBytes = 32768;
constexpr int kRepThreads = 32;
constexpr size_t kRepSmemBytes = (size_t)kRepStages * kRepTileBytes + kRepStages * sizeof(uint64_t);

__global__ void __launch_bounds__(kRepThreads) replicate_kernel(const __grid_constant__ ReplicateArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = (uint64_t*)(smem + (size_t)kRepStages * kRepTileBytes);
  __shared__ int64_t first_plain;  // first of this CTA's tiles left to the plain copy
  constexpr int64_t kTileElems = kRepTileBytes / 2;
  const int64_t n_tiles = a.n / kTileElems;
  const int64_t G = gridDim.x;
  const int64_t my = (int64_t)blockIdx.x < n_tiles ? (n_tiles - blockIdx.x + G - 1) / G : 0;
  if (threadIdx.x == 0) {
    for (int st = 0; st < kRepStages; ++st) mbar_init(&full[st], 1);
    mbar_init_fence();
    int64_t issued = my < kRepStages ? my : kRepStages;
    for (int64_t j = 0; j < issued; ++j) {
      mbar_arrive_expect_tx(&full[j], kRepTileBytes);
      bulk_load(smem + j * kRepTileBytes, a.src + (blockIdx.x + j * G) * kTileElems,
                kRepTileBytes, &full[j]);
    }
    int64_t j = 0;
    for (; j < my; ++j) {
      const int st = (int)(j % kRepStages);
      if (!mbar_wait(&full[st], (uint32_t)((j / kRepStages) & 1))) break;
      const int64_t off = (blockIdx.x + j * G) * kTileElems;
      for (int d = 0; d < a.n_dst; ++d)
        bulk_store(a.dst[d] + off, smem + st * kRepTileBytes, kRepTileBytes);
      bulk_commit();
      if (j >= 1) {
        bulk_wait_read_but1();  // the stores of tile j - 1 have read their stage
        const int64_t jn = j - 1 + kRepStages;
        if (jn < my) {
          const int sp = (int)(jn % kRepStages);
          mbar_arrive_expect_tx(&full[sp], kRepTileBytes);
          bulk_load(smem + sp * kRepTileBytes, a.src + (blockIdx.x + jn * G) * kTileElems,
                    kRepTileBytes, &full[sp]);
          issued = jn + 1;
        }
      }
    }
    // loads still in flight (only after a wait gave up) land before the CTA goes on
    for (int64_t q = j; q < issued; ++q)
      mbar_wait(&full[q % kRepStages], (uint32_t)((q / kRepStages) & 1));
    bulk_wait_all();
    first_plain = j;
  }
  __syncwarp();
  for (int64_t j = first_plain; j < my; ++j) {  // empty unless a wait gave up
    const int64_t off = (blockIdx.x + j * G) * kTileElems;
    for (int64_t v = threadIdx.x; v < kTileElems / 8; v += kRepThreads) {
      const uint4 x = ld_nc_u4(a.src + off + v * 8);
      for (int d = 0; d < a.n_dst; ++d) st_u4(a.dst[d] + off + v * 8, x.x, x.y, x.z, x.w);
    }
  }
  if (blockIdx.x == G - 1) {  // the elements after the last full tile
    const int64_t t0 = n_tiles * kTileElems;
    const int64_t nvec = (a.n - t0) / 8;
    for (int64_t v = threadIdx.x; v < nvec; v += kRepThreads) {
      const uint4 x = ld_nc_u4(a.src + t0 + v * 8);
      for (int d = 0; d < a.n_dst; ++d) st_u4(a.dst[d] + t0 + v * 8, x.x, x.y, x.z, x.w);
    }
    for (int64_t i = t0 + nvec * 8 + threadIdx.x; i < a.n; i += kRepThreads)
      for (int d = 0; d < a.n_dst; ++d) a.dst[d][i] = a.src[i];
  }
}

__global__ void state_init_kernel(WsHeader* h, zero_scaler_cfg cfg) {
  h->magic = kWsMagic;
  h->dynamic = cfg.dynamic;
  h->hysteresis_cfg = cfg.hysteresis;
  h->init_scale_power = cfg.initial_scale_power;
  h->window = cfg.loss_scale_window;
  h->min_scale = cfg.min_loss_scale;
  h->factor = cfg.scale_factor;
  h->static_scale = cfg.static_scale;
  h->pad0 = 0.f;
  h->scale = cfg.dynamic ? ldexpf(1.0f, cfg.initial_scale_power) : cfg.static_scale;
  h->cur_hysteresis = cfg.hysteresis;
  h->iter = 0;
  h->last_overflow_iter = -1;
  h->adam_t = 0;
  h->skip = 1;  // nothing to apply before the first finalize
  h->pad1 = 0;
  zero_step_result& r = h->result;
  r.global_norm = 0.0;
  r.sumsq = 0.0;
  r.clip_coef = 1.f;
  r.scale_used = h->scale;
  r.next_scale = h->scale;
  r.k = 0.f;
  r.overflow = 0;
  r.skipped = 0;
  r.hysteresis = h->cur_hysteresis;
  r.device_error = 0;
  r.iter = 0;
  r.adam_t = 0;
}

// One thread waits on a phase of its own shared-memory barrier that nothing completes
// (no arrivals, no copies in flight): the bounded wait gives up after about one second
// and records code 64 in the sticky error word.
__global__ void selftest_wait_kernel(int32_t* device_error) {
  __shared__ uint64_t bar;
  mbar_init(&bar, 1);
  mbar_init_fence();
  if (!mbar_wait(&bar, 0)) atomicOr(device_error, 64);
}

__global__ void state_write_kernel(WsHeader* h, zero_scaler_state st) {
  h->scale = st.scale;
  h->cur_hysteresis = st.cur_hysteresis;
  h->iter = st.iter;
  h->last_overflow_iter = st.last_overflow_iter;
  h->adam_t = st.adam_t;
  h->result.scale_used = st.scale;
  h->result.next_scale = st.scale;
  h->result.hysteresis = st.cur_hysteresis;
  h->result.iter = st.iter;
  h->result.adam_t = st.adam_t;
}

// ------------------------------------------------------------------ grid sizing

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

cudaError_t persistent_grid(const void* kernel, int threads, int64_t work_items, int* grid) {
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int64_t g = (int64_t)per_sm * sm_count();
  const int64_t need = (work_items + threads - 1) / threads;
  if (g > need) g = need;
  if (g < 1) g = 1;
  *grid = (int)g;
  return cudaSuccess;
}

}  // namespace

// ================================================================== launchers

namespace {

// A launch that may overlap the tail of the previous kernel in the stream (the kernel
// waits for it before touching global memory; see pdl_wait).
cudaError_t launch_chained(const void* kernel, dim3 grid, dim3 block, void** args,
                           size_t smem, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, kernel, args);
}

}  // namespace

int64_t rs_slots(int64_t len) {
  int64_t groups = (len + 7) / 8;
  int64_t blocks = (groups + kRsThreads - 1) / kRsThreads;
  if (blocks < 1) blocks = 1;
  if (blocks > kRsMaxBlocks) blocks = kRsMaxBlocks;
  return blocks;
}

cudaError_t rs_grid(int64_t len, int world, int dtype, int* grid) {
  const void* k = rs_kernel_for(world, dtype);
  const size_t smem = rs_smem_for_world(world);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kRsTmaThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int64_t g = (int64_t)per_sm * sm_count();
  const int64_t cap = rs_slots(len);
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  *grid = (int)g;
  return cudaSuccess;
}

cudaError_t launch_state_init(void* ws, const zero_scaler_cfg& cfg, cudaStream_t s) {
  state_init_kernel<<<1, 1, 0, s>>>((WsHeader*)ws, cfg);
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(void* ws, cudaStream_t s) {
  selftest_wait_kernel<<<1, 1, 0, s>>>(&((WsHeader*)ws)->result.device_error);
  return cudaGetLastError();
}

cudaError_t launch_state_write(void* ws, const zero_scaler_state& st, cudaStream_t s) {
  state_write_kernel<<<1, 1, 0, s>>>((WsHeader*)ws, st);
  return cudaGetLastError();
}

cudaError_t launch_reduce_scatter(int world, int dtype, const uint16_t* const* g, float* R,
                                  int64_t len, double* partial, int32_t* bucket_blocks,
                                  int32_t* device_error, int grid, cudaStream_t s,
                                  int accumulate, int want_sumsq, int store) {
  RsArgs a;
  a.device_error = device_error;
  a.accumulate = accumulate;
  a.want_sumsq = want_sumsq;
  a.store = store;
  for (int r = 0; r < ZERO_MAX_WORLD; ++r) a.g[r] = r < world ? g[r] : nullptr;
  a.R = R;
  a.partial = partial;
  a.blocks = bucket_blocks;
  a.len = len;
  // vector body only if every stream reaches 16-byte alignment at the same element
  int64_t head = -1;
  {
    const uintptr_t rr = (uintptr_t)R;
    bool ok = (rr % 4) == 0;
    int64_t h = ok ? (int64_t)(((16 - rr % 16) % 16) / 4) : 0;  // R wants head % 4 == h
    // candidate heads 0..7 with head % 4 == h
    for (int64_t cand = h; ok && cand < 8; cand += 4) {
      bool all = true;
      for (int r = 0; r < world; ++r) {
        const uintptr_t gr = (uintptr_t)g[r];
        if (gr % 2 != 0 || (gr + 2 * (uintptr_t)cand) % 16 != 0) {
          all = false;
          break;
        }
      }
      if (all) {
        head = cand;
        break;
      }
    }
  }
  if (head < 0 || head > len) {
    a.head = len;
    a.nvec = 0;
  } else {
    a.head = head;
    a.nvec = (len - head) / 8;
  }
  const void* k = rs_kernel_for(world, dtype);
  const size_t smem = rs_smem_for_world(world);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  void* args[] = {&a};
  return launch_chained(k, dim3(grid), dim3(kRsTmaThreads), args, smem, s);
}

cudaError_t launch_finalize(void* ws, const int32_t* bucket_blocks, int64_t slots_full,
                            const double* partial, int64_t n_buckets,
                            const zero_adamw_cfg& cfg, cudaStream_t s) {
  WsHeader* h = (WsHeader*)ws;
  void* args[] = {(void*)&h, (void*)&bucket_blocks, (void*)&slots_full, (void*)&partial,
                  (void*)&n_buckets, (void*)&cfg};
  return launch_chained((const void*)finalize_kernel, dim3(1), dim3(kFinalizeThreads), args, 0, s);
}

cudaError_t launch_local_sumsq(const int32_t* bucket_blocks, int64_t slots_full,
                               const double* partial, int64_t b0, int64_t b1, double* out,
                               cudaStream_t s) {
  local_sumsq_kernel<<<1, kFinalizeThreads, 0, s>>>(bucket_blocks, slots_full, partial, b0, b1,
                                                    out);
  return cudaGetLastError();
}

cudaError_t launch_finalize_ranks(void* ws, const double* s_ranks, int world,
                                  const zero_adamw_cfg& cfg, cudaStream_t s) {
  finalize_ranks_kernel<<<1, 1, 0, s>>>((WsHeader*)ws, s_ranks, world, cfg);
  return cudaGetLastError();
}

cudaError_t launch_update(int dtype, const float* R, float* master, float* m, float* v,
                          void* const* params, int n_params, int64_t n, const void* ws,
                          cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  WsHeader* h = (WsHeader*)ws;
  UpArgs a;
  a.R = R;
  a.p = master;
  a.m = m;
  a.v = v;
  for (int d = 0; d < ZERO_MAX_WORLD; ++d) a.out[d] = d < n_params ? (uint16_t*)params[d] : nullptr;
  a.n_out = n_params;
  a.n = n;
  a.h = h;
  a.device_error = &h->result.device_error;
  const void* k = dtype == ZERO_BF16 ? (const void*)adamw_cast_kernel<ZERO_BF16>
                                     : (const void*)adamw_cast_kernel<ZERO_FP16>;
  // the shared-memory opt-in is per function and device: set it before every launch
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kUpSmemBytes);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kUpTmaThreads, kUpSmemBytes);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int64_t grid = (int64_t)per_sm * sm_count();
  const int64_t n_tiles = n / kUpTile;
  if (grid > n_tiles) grid = n_tiles;
  if (grid < 1) grid = 1;
  void* args[] = {&a};
  return launch_chained(k, dim3((unsigned)grid), dim3(kUpTmaThreads), args, kUpSmemBytes, s);
}

cudaError_t launch_update_resident(int world, int gdt, int pdt, const uint16_t* const* g,
                                   float* master, float* m, float* v, void* params, int64_t n,
                                   const void* ws, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  WsHeader* h = (WsHeader*)ws;
  UpResArgs a;
  for (int r = 0; r < kResMaxWorld; ++r) a.g[r] = r < world ? g[r] : nullptr;
  a.p = master;
  a.m = m;
  a.v = v;
  a.out = (uint16_t*)params;
  a.n = n;
  a.h = h;
  a.device_error = &h->result.device_error;
  const void* table[2][2][2] = {
      {{(const void*)adamw_resident_kernel<1, ZERO_BF16, ZERO_BF16>,
        (const void*)adamw_resident_kernel<1, ZERO_BF16, ZERO_FP16>},
       {(const void*)adamw_resident_kernel<1, ZERO_FP16, ZERO_BF16>,
        (const void*)adamw_resident_kernel<1, ZERO_FP16, ZERO_FP16>}},
      {{(const void*)adamw_resident_kernel<2, ZERO_BF16, ZERO_BF16>,
        (const void*)adamw_resident_kernel<2, ZERO_BF16, ZERO_FP16>},
       {(const void*)adamw_resident_kernel<2, ZERO_FP16, ZERO_BF16>,
        (const void*)adamw_resident_kernel<2, ZERO_FP16, ZERO_FP16>}}};
  const void* k = table[world - 1][gdt == ZERO_FP16][pdt == ZERO_FP16];
  const size_t smem = world == 1 ? up_res_smem_bytes<1>() : up_res_smem_bytes<2>();
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kUpTmaThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int64_t grid = (int64_t)per_sm * sm_count();
  const int64_t n_tiles = n / kUpTile;
  if (grid > n_tiles) grid = n_tiles;
  if (grid < 1) grid = 1;
  void* args[] = {&a};
  return launch_chained(k, dim3((unsigned)grid), dim3(kUpTmaThreads), args, smem, s);
}

cudaError_t launch_cast(int dtype, const float* master, void* params, int64_t n,
                        cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const void* k = dtype == ZERO_BF16 ? (const void*)cast_kernel<ZERO_BF16>
                                     : (const void*)cast_kernel<ZERO_FP16>;
  int grid = 1;
  cudaError_t e = persistent_grid(k, kUpThreads, (n + 7) / 8, &grid);
  if (e != cudaSuccess) return e;
  uint16_t* out = (uint16_t*)params;
  void* args[] = {(void*)&master, (void*)&out, (void*)&n};
  return cudaLaunchKernel(k, dim3(grid), dim3(kUpThreads), args, 0, s);
}

cudaError_t launch_replicate(const void* src, void* const* dst, int n_dst, int64_t n_halves,
                             cudaStream_t s) {
  if (n_halves == 0 || n_dst == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute((const void*)replicate_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kRepSmemBytes);
  if (e != cudaSuccess) return e;
  // one CTA per SM (the ring takes 128 KB of shared memory), never more than the tiles
  const int64_t n_tiles = n_halves / (kRepTileBytes / 2);
  int64_t grid = sm_count();
  if (grid > n_tiles) grid = n_tiles;
  if (grid < 1) grid = 1;
  for (int d0 = 0; d0 < n_dst; d0 += kReplicateMax) {
    ReplicateArgs a;
    a.src = (const uint16_t*)src;
    a.n_dst = n_dst - d0 < kReplicateMax ? n_dst - d0 : kReplicateMax;
    for (int d = 0; d < kReplicateMax; ++d)
      a.dst[d] = d < a.n_dst ? (uint16_t*)dst[d0 + d] : nullptr;
    a.n = n_halves;
    void* args[] = {&a};
    e = cudaLaunchKernel((const void*)replicate_kernel, dim3((unsigned)grid), dim3(kRepThreads),
                         args, kRepSmemBytes, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace zero
