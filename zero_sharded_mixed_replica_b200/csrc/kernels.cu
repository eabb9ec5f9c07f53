// kernels.cu -- sm_100a kernels of the ZeRO partitioned optimizer step.
//
// All kernels here are HBM-bandwidth bound streams (about 0.3 flop per byte); none is
// a contraction, so none uses tensor cores. Each is a persistent grid-stride loop over
// 16-byte vectors, sized from the SM count and the kernel's occupancy, with loads
// marked L1::no_allocate (every byte is touched once per step).
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
};

// For every element i of the bucket: R[i] = ((g_0[i] + g_1[i]) + ...) + g_{W-1}[i] in
// fp32, and ss += R[i]^2 in fp64 (the square of an fp32 is exact in fp64, so the fused
// multiply-add rounds exactly like the separate add would). Each block writes its ss
// to its own slot; the finalize kernel adds the slots in a fixed order.
// U groups per thread per trip keep >= 8 16-byte loads in flight for small W.
template <int W, int DT, int U>
__global__ void __launch_bounds__(kRsThreads) rs_bucket_kernel(const __grid_constant__ RsArgs a) {
  double ss = 0.0;
  const int64_t nthr = (int64_t)gridDim.x * kRsThreads;
  const int64_t tid = (int64_t)blockIdx.x * kRsThreads + threadIdx.x;
  for (int64_t v0 = tid; v0 < a.nvec; v0 += nthr * U) {
    uint4 x[U][W];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t v = v0 + (int64_t)u * nthr;
      if (v < a.nvec) {
        const int64_t e = a.head + v * 8;
#pragma unroll
        for (int r = 0; r < W; ++r) x[u][r] = ld_nc_u4(a.g[r] + e);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t v = v0 + (int64_t)u * nthr;
      if (v < a.nvec) {
        const int64_t e = a.head + v * 8;
        float acc[8];
        unpack8<DT>(x[u][0], acc);
#pragma unroll
        for (int r = 1; r < W; ++r) {
          float t[8];
          unpack8<DT>(x[u][r], t);
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[j] = __fadd_rn(acc[j], t[j]);
        }
        st_f4(a.R + e, acc[0], acc[1], acc[2], acc[3]);
        st_f4(a.R + e + 4, acc[4], acc[5], acc[6], acc[7]);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const double d = (double)acc[j];
          ss = __fma_rn(d, d, ss);
        }
      }
    }
  }
  // scalar elements: the unaligned head [0, head) and the tail after the last group
  const int64_t body_end = a.head + 8 * a.nvec;
  const int64_t n_scalar = a.head + (a.len - body_end);
  for (int64_t q = tid; q < n_scalar; q += nthr) {
    const int64_t i = q < a.head ? q : body_end + (q - a.head);
    float acc = half_bits_to_float<DT>(a.g[0][i]);
#pragma unroll
    for (int r = 1; r < W; ++r) acc = __fadd_rn(acc, half_bits_to_float<DT>(a.g[r][i]));
    a.R[i] = acc;
    const double d = (double)acc;
    ss = __fma_rn(d, d, ss);
  }
  ss = block_sum<kRsThreads>(ss);
  if (threadIdx.x == 0) {
    a.partial[blockIdx.x] = ss;
    if (blockIdx.x == 0) *a.blocks = (int32_t)gridDim.x;
  }
}

template <int W, int DT>
constexpr int rs_unroll() {
  return W >= 8 ? 1 : (W >= 4 ? 2 : 4);
}

template <int W, int DT>
const void* rs_kernel_ptr() {
  return (const void*)rs_bucket_kernel<W, DT, rs_unroll<W, DT>()>;
}

typedef const void* (*KernelGetter)();

template <int DT, int... Ws>
struct RsTable {
  static const void* get(int w) {
    const void* ptrs[] = {rs_kernel_ptr<Ws, DT>()...};
    return ptrs[w - 1];
  }
};

const void* rs_kernel_for(int world, int dtype) {
  if (dtype == ZERO_BF16)
    return RsTable<ZERO_BF16, 1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15, 16>::get(world);
  return RsTable<ZERO_FP16, 1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15, 16>::get(world);
}

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

__global__ void __launch_bounds__(kFinalizeThreads)
    finalize_kernel(WsHeader* h, const int32_t* __restrict__ bucket_blocks, int64_t slots_full,
                    const double* __restrict__ partial, int64_t n_buckets, zero_adamw_cfg cfg) {
  // S: fixed order -- each thread walks buckets in order and its own slots in order,
  // then the block tree.
  double acc = 0.0;
  for (int64_t b = 0; b < n_buckets; ++b) {
    const int32_t nb = bucket_blocks[b];
    const double* p = partial + b * slots_full;
    for (int j = threadIdx.x; j < nb; j += kFinalizeThreads) acc = __dadd_rn(acc, p[j]);
  }
  const double S = block_sum<kFinalizeThreads>(acc);
  if (threadIdx.x != 0) return;

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
  r.reserved = 0;
  r.iter = h->iter;
  r.adam_t = t;
}

// ================================================================== K3: AdamW + cast

struct UpArgs {
  const float* R;
  float* p;
  float* m;
  float* v;
  void* out;  // gathered half buffer
  int64_t n;
  const WsHeader* h;
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

template <int DT>
__global__ void __launch_bounds__(kUpThreads) adamw_cast_kernel(const __grid_constant__ UpArgs a) {
  const WsHeader* h = a.h;
  if (h->skip) return;  // overflow: the whole step is skipped
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
  const int64_t nthr = (int64_t)gridDim.x * kUpThreads;
  const int64_t tid = (int64_t)blockIdx.x * kUpThreads + threadIdx.x;
  const int64_t nvec = a.n / 8;
  uint16_t* out = (uint16_t*)a.out;
  for (int64_t vi = tid; vi < nvec; vi += nthr) {
    const int64_t e = vi * 8;
    const float4 r0 = ld_nc_f4(a.R + e), r1 = ld_nc_f4(a.R + e + 4);
    float4 p0 = ld_f4(a.p + e), p1 = ld_f4(a.p + e + 4);
    float4 m0 = ld_f4(a.m + e), m1 = ld_f4(a.m + e + 4);
    float4 v0 = ld_f4(a.v + e), v1 = ld_f4(a.v + e + 4);
    adamw1(c, r0.x, p0.x, m0.x, v0.x);
    adamw1(c, r0.y, p0.y, m0.y, v0.y);
    adamw1(c, r0.z, p0.z, m0.z, v0.z);
    adamw1(c, r0.w, p0.w, m0.w, v0.w);
    adamw1(c, r1.x, p1.x, m1.x, v1.x);
    adamw1(c, r1.y, p1.y, m1.y, v1.y);
    adamw1(c, r1.z, p1.z, m1.z, v1.z);
    adamw1(c, r1.w, p1.w, m1.w, v1.w);
    st_f4(a.p + e, p0.x, p0.y, p0.z, p0.w);
    st_f4(a.p + e + 4, p1.x, p1.y, p1.z, p1.w);
    st_f4(a.m + e, m0.x, m0.y, m0.z, m0.w);
    st_f4(a.m + e + 4, m1.x, m1.y, m1.z, m1.w);
    st_f4(a.v + e, v0.x, v0.y, v0.z, v0.w);
    st_f4(a.v + e + 4, v1.x, v1.y, v1.z, v1.w);
    st_u4(out + e, pack2<DT>(p0.x, p0.y), pack2<DT>(p0.z, p0.w), pack2<DT>(p1.x, p1.y),
          pack2<DT>(p1.z, p1.w));
  }
  for (int64_t i = nvec * 8 + tid; i < a.n; i += nthr) {
    float p = a.p[i], m = a.m[i], v = a.v[i];
    adamw1(c, a.R[i], p, m, v);
    a.p[i] = p;
    a.m[i] = m;
    a.v[i] = v;
    out[i] = (uint16_t)float_to_half_bits<DT>(p);
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

__global__ void __launch_bounds__(kUpThreads) replicate_kernel(const __grid_constant__ ReplicateArgs a) {
  const int64_t nthr = (int64_t)gridDim.x * kUpThreads;
  const int64_t tid = (int64_t)blockIdx.x * kUpThreads + threadIdx.x;
  const int64_t nvec = a.n / 8;
  for (int64_t vi = tid; vi < nvec; vi += nthr) {
    const uint4 x = ld_nc_u4(a.src + vi * 8);
    for (int d = 0; d < a.n_dst; ++d) st_u4(a.dst[d] + vi * 8, x.x, x.y, x.z, x.w);
  }
  for (int64_t i = nvec * 8 + tid; i < a.n; i += nthr)
    for (int d = 0; d < a.n_dst; ++d) a.dst[d][i] = a.src[i];
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
  r.reserved = 0;
  r.iter = 0;
  r.adam_t = 0;
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

int64_t rs_slots(int64_t len) {
  int64_t groups = (len + 7) / 8;
  int64_t blocks = (groups + kRsThreads - 1) / kRsThreads;
  if (blocks < 1) blocks = 1;
  if (blocks > kRsMaxBlocks) blocks = kRsMaxBlocks;
  return blocks;
}

cudaError_t rs_grid(int64_t len, int world, int dtype, int* grid) {
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      &per_sm, rs_kernel_for(world, dtype), kRsThreads, 0);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int64_t g = (int64_t)per_sm * sm_count();
  const int64_t cap = rs_slots(len);
  if (g > cap) g = cap;
  *grid = (int)g;
  return cudaSuccess;
}

cudaError_t launch_state_init(void* ws, const zero_scaler_cfg& cfg, cudaStream_t s) {
  state_init_kernel<<<1, 1, 0, s>>>((WsHeader*)ws, cfg);
  return cudaGetLastError();
}

cudaError_t launch_reduce_scatter(int world, int dtype, const uint16_t* const* g, float* R,
                                  int64_t /*start*/, int64_t len, double* partial,
                                  int32_t* bucket_blocks, int grid, cudaStream_t s) {
  RsArgs a;
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
  void* args[] = {&a};
  return cudaLaunchKernel(rs_kernel_for(world, dtype), dim3(grid), dim3(kRsThreads), args, 0, s);
}

cudaError_t launch_finalize(void* ws, const int32_t* bucket_blocks, int64_t slots_full,
                            const double* partial, int64_t n_buckets,
                            const zero_adamw_cfg& cfg, cudaStream_t s) {
  finalize_kernel<<<1, kFinalizeThreads, 0, s>>>((WsHeader*)ws, bucket_blocks, slots_full,
                                                 partial, n_buckets, cfg);
  return cudaGetLastError();
}

cudaError_t launch_update(int dtype, const float* R, float* master, float* m, float* v,
                          void* params, int64_t n, const void* ws, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  UpArgs a{R, master, m, v, params, n, (const WsHeader*)ws};
  const void* k = dtype == ZERO_BF16 ? (const void*)adamw_cast_kernel<ZERO_BF16>
                                     : (const void*)adamw_cast_kernel<ZERO_FP16>;
  int grid = 1;
  cudaError_t e = persistent_grid(k, kUpThreads, (n + 7) / 8, &grid);
  if (e != cudaSuccess) return e;
  void* args[] = {&a};
  return cudaLaunchKernel(k, dim3(grid), dim3(kUpThreads), args, 0, s);
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
  int grid = 1;
  cudaError_t e = persistent_grid((const void*)replicate_kernel, kUpThreads,
                                  (n_halves + 7) / 8, &grid);
  if (e != cudaSuccess) return e;
  for (int d0 = 0; d0 < n_dst; d0 += kReplicateMax) {
    ReplicateArgs a;
    a.src = (const uint16_t*)src;
    a.n_dst = n_dst - d0 < kReplicateMax ? n_dst - d0 : kReplicateMax;
    for (int d = 0; d < kReplicateMax; ++d)
      a.dst[d] = d < a.n_dst ? (uint16_t*)dst[d0 + d] : nullptr;
    a.n = n_halves;
    void* args[] = {&a};
    e = cudaLaunchKernel((const void*)replicate_kernel, dim3(grid), dim3(kUpThreads), args, 0, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace zero
