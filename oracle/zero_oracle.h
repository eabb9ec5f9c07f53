/*
 * zero_oracle.h -- CPU oracle of the ZeRO partitioned mixed-precision optimizer step.
 *
 * TEST INFRASTRUCTURE. Only the tests, the package smoke check and the CPU-baseline
 * leg of the benchmark may load this code. The product path (the CUDA library) never
 * links, includes or calls it, and this oracle shares no source with that library.
 *
 * Plain, single-threaded, obviously-correct loops in flat order, compiled with
 * -O2 -ffp-contract=off (no FMA contraction, no fast-math). Precision follows the
 * method: replica gradients are half precision, the reduction and the master / moment
 * state are fp32 (fp32 master weights with first and second moments: "ZeRO and sharded
 * optimizers" FAQ on Adam state), the global sum of squares and the norm are fp64.
 *
 * Sources (web pages; titles and sections):
 *  [Z1] "ZeRO技术解析：大模型分布式训练的革命性突破" (ZeRO explained), section 1.2 (stages),
 *       2.1 (dynamic partitioning: parameters split into N parts, gradients
 *       reduce-scattered, each GPU updates its own partition, bucketed communication),
 *       2.2 (reduce_bucket_size), 3.1 (AdamW lr 6e-5, weight_decay 0.01), 3.3 (fp16
 *       loss_scale_window 100, hysteresis 2), 5.1 (initial_scale_power 16,
 *       min_loss_scale 1), 6 (gradient_clipping 1.0).
 *  [Z2] "大模型分片训练：ZeRO-3策略在PyTorch中的实现" (ZeRO-3 in PyTorch): memory
 *       arithmetic for one TransformerEncoderLayer, the per-stage saving table, the
 *       ds_config with allgather_bucket_size and reduce_scatter.
 *  [Z3] "ZeRO 和分片优化器" (ZeRO and sharded optimizers): technical insight (gradients
 *       are reduce-scattered so each GPU keeps the slice matching its own parameters)
 *       and FAQ (Adam keeps first and second moments beside fp32 master weights).
 * Readings where the pages are silent are stated next to each function.
 */
#ifndef ZERO_ORACLE_H
#define ZERO_ORACLE_H

#include <stdint.h>

#define ORACLE_BF16 0
#define ORACLE_FP16 1

/* ---------------- planner (own implementation, no shared code) ---------------- */

/* Sizes of the flat padded index space. out = {N, N_pad, P, n_buckets}.
 * N = sum of numels in declared order; N_pad = ceil(N / (W*A)) * W*A; P = N_pad / W;
 * buckets are [b*B, min((b+1)*B, N_pad)). Returns 0, or -1 on bad arguments. */
int oracle_plan_sizes(const int64_t* numels, int32_t n_tensors, int32_t world,
                      int64_t bucket, int32_t align, int64_t out[4]);

/* Flat offset of each tensor (prefix sum of numels in declared order). */
int oracle_plan_tensor_offsets(const int64_t* numels, int32_t n_tensors, int64_t* offsets);

/* Work segments = bucket intersect partition, bucket-major then rank.
 * Writes up to cap rows of (bucket, rank, start, len); returns the total count. */
int64_t oracle_plan_work_segments(int64_t n_pad, int32_t world, int64_t bucket,
                                  int64_t cap, int64_t* seg_bucket, int64_t* seg_rank,
                                  int64_t* seg_start, int64_t* seg_len);

/* Partition segments of one rank: pieces of tensors (tensor id, offset inside the
 * tensor, flat offset, length) that fall in [rank*P, (rank+1)*P); the zero padding
 * past N appears as tensor id -1. Returns the count (rows written up to cap). */
int64_t oracle_plan_partition(const int64_t* numels, int32_t n_tensors, int64_t n_pad,
                              int32_t world, int32_t rank, int64_t cap, int64_t* tensor,
                              int64_t* off_in_tensor, int64_t* flat_off, int64_t* len);

/* ---------------- half conversions (own implementation) ---------------- */

float oracle_half_to_f32(uint16_t h, int32_t dtype);
uint16_t oracle_f32_to_half(float x, int32_t dtype);
void oracle_f32_to_half_array(const float* x, uint16_t* out, int64_t n, int32_t dtype);
void oracle_half_to_f32_array(const uint16_t* h, float* out, int64_t n, int32_t dtype);

/* ---------------- the step ---------------- */

typedef struct {
  int32_t dynamic;          /* 1: dynamic loss scaling (fp16); 0: static scale      */
  int32_t init_scale_power; /* initial scale = 2^init_scale_power (dynamic mode)    */
  int64_t window;           /* loss_scale_window                                    */
  int32_t hysteresis;       /* hysteresis                                           */
  float min_scale;          /* min_loss_scale                                       */
  float factor;             /* growth / back-off factor (2)                         */
  float static_scale;       /* scale when dynamic == 0 (1 for bf16)                 */
} oracle_scaler_cfg;

typedef struct {
  float scale;
  int32_t cur_hysteresis;
  int64_t iter;
  int64_t last_overflow_iter;
  int64_t adam_t; /* applied AdamW steps */
} oracle_state;

typedef struct {
  double lr, beta1, beta2, eps, weight_decay, max_grad_norm;
} oracle_hparams;

/* Everything one step decides before the elementwise update. */
typedef struct {
  double sumsq;      /* S: fp64 sum of squares of the reduced (still scaled) gradient */
  double norm;       /* sqrt(S) / scale                                                */
  int32_t overflow;  /* any non-finite reduced gradient, or non-finite S              */
  int32_t skipped;   /* overflow => the whole step is skipped                          */
  float scale_used;  /* loss scale in force for this step                              */
  float next_scale;  /* loss scale after the transition                                */
  float clip_coef;   /* c = min(1, max_norm / (norm + 1e-6)) as fp32                   */
  float k;           /* fp32(c / scale): the one multiplier applied to R               */
  int32_t hysteresis;
  int64_t iter;      /* scaler iteration counter after the step                        */
  int64_t adam_t;    /* applied steps after this one                                   */
  /* fp32 constants of the elementwise update */
  float b1, omb1, b2, omb2, bc1, bc2, eps, lr, decay;
} oracle_scalars;

void oracle_state_init(const oracle_scaler_cfg* cfg, oracle_state* st);

/* Reduce-scatter arithmetic for a range: R[i] = ((g_0[i] + g_1[i]) + ...) + g_{W-1}[i],
 * every term converted exactly from half to fp32, summed in fp32 in rank order. */
void oracle_reduce(int32_t world, int32_t gdtype, const uint16_t* const* grads, int64_t n,
                   float* R);

/* Gradient accumulation over micro-batches ([Z1] 3.1 and [Z2] config:
 * gradient_accumulation_steps): R[i] = R[i] + (((g_0[i] + g_1[i]) + ...) + g_{W-1}[i]),
 * the micro-batch's rank-ordered fp32 sum added to what the earlier micro-batches of
 * the step left in R. */
void oracle_reduce_accumulate(int32_t world, int32_t gdtype, const uint16_t* const* grads,
                              int64_t n, float* R);

/* S += R[0]^2 + R[1]^2 + ... in flat order, each square formed in fp64. */
void oracle_sumsq(const float* R, int64_t n, double* S);

/* 1 if any R[i] is inf or NaN. */
int32_t oracle_any_nonfinite(const float* R, int64_t n);

/* Norm, clip, overflow / skip decision, loss-scaler transition, step counter and the
 * fp32 constants of the update. Updates *st. */
void oracle_finalize(double S, int32_t nonfinite, const oracle_scaler_cfg* cfg,
                     const oracle_hparams* hp, oracle_state* st, oracle_scalars* out);

/* Elementwise AdamW on fp32 master / m / v plus the half cast into the gathered
 * buffer. Does nothing when sc->skipped. */
void oracle_adamw(int64_t n, const float* R, float* master, float* m, float* v,
                  uint16_t* params, int32_t pdtype, const oracle_scalars* sc);

/* One whole step over n_pad resident elements: per bucket reduce + partial sum of
 * squares (S_b in flat order inside bucket b, S = S_0 + S_1 + ... in bucket order),
 * finalize, update. grads[r] holds replica r's n_pad half values. */
void oracle_step(int32_t world, int32_t gdtype, const uint16_t* const* grads, int64_t n_pad,
                 int64_t bucket, float* R, float* master, float* m, float* v,
                 uint16_t* params, int32_t pdtype, const oracle_scaler_cfg* cfg,
                 const oracle_hparams* hp, oracle_state* st, oracle_scalars* out);

/* ---------------- memory accounting ---------------- */

/* Bytes per rank of model state for psi parameters on W data-parallel ranks, with
 * half-precision params and grads and fp32 master + m + v (2 + 2 + 12 bytes/param):
 * stage 0 = plain data parallel, 1 = optimizer state partitioned, 2 = + gradients,
 * 3 = + parameters. out = {params, grads, optimizer_state, total}. */
int oracle_memory_per_rank(double psi, int32_t world, int32_t stage, double out[4]);

#endif /* ZERO_ORACLE_H */
