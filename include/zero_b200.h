/*
 * zero_b200.h -- C ABI of libzero_b200.so: the ZeRO partitioned mixed-precision
 * optimizer step on one B200 (sm_100a), with W data-parallel ranks simulated as W
 * replica gradient buffers and W owned partitions in the same GPU's memory.
 *
 * One step, in order:
 *   1. zero_reduce_scatter_bucket(b) for every bucket b: sum the W replica gradients
 *      of the bucket in fp32 in rank order; each rank's slice of the result is its
 *      reduced gradient partition. Also accumulates the fp64 sum of squares.
 *   2.-4. zero_step: overflow (inf/NaN) detection, dynamic loss-scale update, global
 *      L2-norm clipping, and AdamW on every rank's fp32 master / m / v partition,
 *      writing the rounded half-precision parameters straight into the gathered
 *      buffer (the all-gather of step 5 costs nothing extra on one GPU).
 *   5. zero_all_gather: optional copies of the gathered buffer into per-rank buffers.
 * zero_step_full does 1.-4. in one call; zero_step_resident does them for W <= 2 with
 * fewer bytes when the replicas stay resident. One process per rank: the rank-local
 * calls further down.
 *
 * Sources (web pages; titles and sections):
 *  [Z1] "ZeRO技术解析：大模型分布式训练的革命性突破" (ZeRO explained): 1.2.1-1.2.3 (the three
 *       stages: optimizer state, gradients and parameters partitioned), 2.1 (parameters
 *       split automatically into N parts, gradients reduce-scattered in backward, each
 *       GPU updates only its own partition, bucketed communication), 2.2 (gradient
 *       buckets via reduce_bucket_size; batched all-gather of large matrices), 3.1
 *       (AdamW, lr 6e-5, weight_decay 0.01), 3.3 (fp16 loss_scale_window 100,
 *       hysteresis 2), 5.1 (initial_scale_power 16, min_loss_scale 1), 5.2
 *       (reduce_bucket_size 5e8, contiguous_gradients), 6 (gradient_clipping 1.0,
 *       reduce_bucket_size 2e8).
 *  [Z2] "大模型分片训练：ZeRO-3策略在PyTorch中的实现" (ZeRO-3 in PyTorch): memory arithmetic of
 *       one encoder layer, the per-stage saving table, the ds_config with
 *       allgather_bucket_size and reduce_scatter, deepspeed.initialize.
 *  [Z3] "ZeRO 和分片优化器" (ZeRO and sharded optimizers): gradients are reduce-scattered
 *       so each GPU keeps the slice for its own parameters; Adam keeps first and second
 *       moments beside fp32 master weights (FAQ).
 *
 * Conventions for every call
 *  - Return value: ZERO_OK (0) or a negative ZERO_E* code; zero_last_error() then gives
 *    a message (thread-local, valid until the next call on the same thread). Nothing
 *    throws across this boundary.
 *  - Ownership: the caller allocates and owns every device buffer, the workspace and
 *    the stream. The library owns only the plan (host memory). It never allocates
 *    device memory and never synchronises, except zero_get_result.
 *  - Streams: `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *    stream. All device work of a call is enqueued on that stream, in order. The step
 *    kernels (bucket reduction, finalize, update) are launched with programmatic stream
 *    serialization: one may be scheduled while the kernel before it in the stream is
 *    finishing, but it reads and writes no global memory until that kernel has
 *    completed, so stream order holds exactly as for ordinary launches.
 *  - Device pointers must be 16-byte aligned (ZERO_EALIGN otherwise).
 *  - Conditions found on the device (overflow, a skipped step) are results, not errors.
 *  - Calls on one plan must not run concurrently from several host threads.
 */
#ifndef ZERO_B200_H
#define ZERO_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ZERO_ABI_VERSION 2

#if defined(__GNUC__)
#define ZERO_API __attribute__((visibility("default")))
#else
#define ZERO_API
#endif

/* error codes */
#define ZERO_OK 0
#define ZERO_EINVAL (-1) /* null pointer, W outside [1, ZERO_MAX_WORLD], negative dim, bucket out of range, bad hyperparameter */
#define ZERO_EALIGN (-2) /* a device pointer or replica base offset breaks the alignment rule */
#define ZERO_ERANGE (-3) /* the parameter count overflows int64 */
#define ZERO_ESTATE (-4) /* call out of order: a bucket reduced twice, or a step before every bucket was reduced */
#define ZERO_ECUDA (-5)  /* a CUDA launch or copy failed; the message names the CUDA error */
#define ZERO_ENOMEM (-6) /* host allocation for the plan failed */
#define ZERO_EDEVICE (-7) /* a kernel gave up waiting on its own pipeline (bounded waits of
                             about one second); its output is incomplete */

/* element types of gradients and gathered parameters */
#define ZERO_BF16 0
#define ZERO_FP16 1

#define ZERO_MAX_WORLD 16 /* simulated ranks per reduce-scatter launch */

typedef struct zero_plan zero_plan; /* opaque; host memory owned by the library */

typedef struct {
  int64_t n;          /* parameters: sum of tensor numels in declared order        */
  int64_t n_pad;      /* ceil(n / (W*align)) * W*align                              */
  int64_t p;          /* partition length n_pad / W                                 */
  int64_t n_buckets;  /* ceil(n_pad / bucket_size)                                  */
  int64_t n_segments; /* work segments: bucket intersect partition                  */
  int64_t n_tensors;
  int64_t bucket_size; /* reduce_bucket_size in elements                            */
  int32_t world_size;  /* W                                                         */
  int32_t align;       /* alignment unit A in elements                              */
} zero_plan_info;

/* A piece of one tensor inside one rank's partition; tensor == -1 is zero padding. */
typedef struct {
  int64_t tensor;
  int64_t offset_in_tensor;
  int64_t flat_offset;
  int64_t length;
} zero_segment;

/* bucket intersect partition */
typedef struct {
  int64_t bucket;
  int64_t rank;
  int64_t start; /* flat index */
  int64_t length;
} zero_work_segment;

/* Loss scaler ([Z1] 3.3, 5.1). dynamic=0: a fixed scale `static_scale` (1 for bf16). */
typedef struct {
  int32_t dynamic;
  int32_t initial_scale_power; /* scale starts at 2^initial_scale_power            */
  int64_t loss_scale_window;   /* good steps between growths                        */
  int32_t hysteresis;          /* overflows tolerated before backing off            */
  float min_loss_scale;
  float scale_factor;          /* growth / back-off factor, normally 2              */
  float static_scale;
} zero_scaler_cfg;

/* AdamW ([Z1] 3.1) and clipping ([Z1] 6). max_grad_norm <= 0 disables clipping. */
typedef struct {
  double lr, beta1, beta2, eps, weight_decay, max_grad_norm;
} zero_adamw_cfg;

typedef struct {
  double global_norm; /* L2 norm of the unscaled gradient before clipping           */
  double sumsq;       /* fp64 sum of squares of the scaled reduced gradient         */
  float clip_coef;    /* min(1, max_grad_norm / (global_norm + 1e-6))                */
  float scale_used;   /* loss scale this step's gradients carried                    */
  float next_scale;   /* loss scale after the scaler transition                      */
  float k;            /* fp32 multiplier applied to the reduced gradient: clip/scale */
  int32_t overflow;   /* a reduced gradient was inf or NaN                           */
  int32_t skipped;    /* the update was skipped (overflow)                           */
  int32_t hysteresis; /* hysteresis budget after the step                            */
  int32_t device_error; /* nonzero once a kernel gave up on a bounded wait (sticky until
                           zero_state_init); zero_get_result then returns ZERO_EDEVICE */
  int64_t iter;       /* scaler iterations so far (every step)                       */
  int64_t adam_t;     /* applied AdamW steps so far                                  */
} zero_step_result;

/* Loss-scaler and step-counter state (what a checkpoint must keep besides the tensors). */
typedef struct {
  float scale;
  int32_t cur_hysteresis;
  int64_t iter;
  int64_t last_overflow_iter;
  int64_t adam_t;
} zero_scaler_state;

/* bytes per rank */
typedef struct {
  double params, grads, optimizer_state, total;
} zero_memory;

/* ---------------------------------------------------------------- planning (host only)
 * zero_plan_create: [Z1] 2.1 (parameters split automatically into N = W parts, one per
 * GPU; communication in buckets), [Z1] 4.1 table (ZeRO partitions by dynamic bucket,
 * not by module), [Z1] 2.2 / 5.2 / 6 (reduce_bucket_size).
 * Tensors are flattened in the order given (tensor t has ndims[t] dims read in turn
 * from `dims`; ndims 0 means a scalar), padded with zeros to n_pad, a multiple of
 * W*align_elems; rank r owns the flat range [r*p, (r+1)*p); bucket b is
 * [b*B, min((b+1)*B, n_pad)) with B = reduce_bucket_size ELEMENTS.
 * Errors: EINVAL (null out, world_size outside [1, 16], bucket < 1, align < 1, a
 * negative dim), ERANGE (n overflows), ENOMEM. n_tensors may be 0 (an empty plan). */
ZERO_API int zero_plan_create(const int64_t* dims, const int32_t* ndims, int32_t n_tensors,
                     int32_t world_size, int64_t reduce_bucket_size, int32_t align_elems,
                     zero_plan** out);
ZERO_API void zero_plan_destroy(zero_plan* plan);
ZERO_API int zero_plan_get_info(const zero_plan* plan, zero_plan_info* out);
/* flat offset and numel of tensor t */
ZERO_API int zero_plan_tensor(const zero_plan* plan, int32_t t, int64_t* flat_offset, int64_t* numel);
/* flat start and length of bucket b */
ZERO_API int zero_plan_bucket(const zero_plan* plan, int64_t b, int64_t* start, int64_t* length);
/* Work segments (bucket-major, then rank). Writes min(cap, total) rows; *count = total. */
ZERO_API int zero_plan_work_segments(const zero_plan* plan, zero_work_segment* out, int64_t cap,
                            int64_t* count);
/* Partition table of one rank ([Z3]: each GPU owns one slice). Same cap/count rule. */
ZERO_API int zero_plan_partition(const zero_plan* plan, int32_t rank, zero_segment* out, int64_t cap,
                        int64_t* count);
/* Model-state bytes per rank for ZeRO stage 0..3 on this plan's W ranks, with half
 * params and grads and fp32 master + m + v ([Z2] memory arithmetic and stage table,
 * [Z1] 1.2.1: 8-way optimizer-state partitioning saves 87.5%). Partitioned items take
 * p elements per rank, replicated ones n_pad. */
ZERO_API int zero_plan_memory(const zero_plan* plan, int32_t stage, zero_memory* out);

/* ---------------------------------------------------------------- device state
 * Device workspace: scaler state, step constants, per-block partial sums of squares
 * and the step result. The caller allocates zero_workspace_bytes() of device memory
 * (16-byte aligned) and keeps it for the life of the optimizer. */
ZERO_API int zero_workspace_bytes(const zero_plan* plan, size_t* bytes);
/* Writes the initial scaler state and zero step counters into the workspace
 * ([Z1] 3.3, 5.1): scale 2^initial_scale_power (dynamic) or static_scale, hysteresis
 * budget full. Also resets the plan's per-step bookkeeping. EINVAL on a bad config. */
ZERO_API int zero_state_init(zero_plan* plan, void* workspace, const zero_scaler_cfg* cfg,
                    void* stream);
/* Checkpointing ([Z2]: save through the engine so that the shard information is kept;
 * a plain state_dict save would lose it). zero_state_read copies the scaler and step
 * state out of the workspace (synchronises `stream`); zero_state_write installs a saved
 * state (with its scaler configuration) into a workspace, e.g. after loading shards into
 * a plan of another world size. */
ZERO_API int zero_state_read(const void* workspace, zero_scaler_state* out, void* stream);
ZERO_API int zero_state_write(zero_plan* plan, void* workspace, const zero_scaler_cfg* cfg,
                              const zero_scaler_state* state, void* stream);
/* Writes the half-precision copy of `master` (n_pad fp32) into the gathered buffer
 * `params` (n_pad half): round to nearest even. Used once after initialisation or a
 * load; steps keep the buffer current themselves. */
ZERO_API int zero_cast_params(const zero_plan* plan, const float* master, void* params,
                     int32_t param_dtype, void* stream);

/* ---------------------------------------------------------------- the step
 * zero_reduce_scatter_bucket ([Z1] 2.1 gradients reduce-scattered in backward; [Z1] 2.2
 * reduce_bucket_size; [Z3] each GPU keeps the summed slice for its own parameters):
 *   reduced[i] = ((g_0[i] + g_1[i]) + ...) + g_{W-1}[i]   for i in bucket b,
 * each half converted exactly to fp32 and the sum taken in fp32 in rank order, written
 * at the same flat index of `reduced` (n_pad fp32; rank r's slice [r*p, (r+1)*p) is its
 * reduced gradient partition). The fp64 sum of squares of those values goes to the
 * workspace (it yields both the global norm and the overflow flag).
 *   replica_grads: HOST array of W device pointers; replica_grads[r][j] holds flat index
 *   replica_base_offset + j, so a caller may pass bucket-sized buffers with
 *   replica_base_offset = bucket start, or whole-model buffers with 0. Every replica
 *   pointer and `reduced` must be 16-byte aligned. replica_base_offset must be <= the
 *   bucket start.
 * Each bucket must be reduced exactly once per step (ESTATE on a repeat). */
ZERO_API int zero_reduce_scatter_bucket(zero_plan* plan, int64_t bucket, int32_t grad_dtype,
                               const void* const* replica_grads, int64_t replica_base_offset,
                               float* reduced, void* workspace, void* stream);

/* Same as zero_reduce_scatter_bucket, but the replica gradients are in pinned HOST
 * memory: each replica's bucket slice is first copied (cudaMemcpyAsync, host to device,
 * on `stream`) into device_staging[r] (bucket-sized device buffers, W of them), then
 * reduced. host_replica_grads[r][j] holds flat index host_base_offset + j. */
ZERO_API int zero_reduce_scatter_bucket_host(zero_plan* plan, int64_t bucket, int32_t grad_dtype,
                                    const void* const* host_replica_grads,
                                    int64_t host_base_offset, void* const* device_staging,
                                    float* reduced, void* workspace, void* stream);

/* Gradient accumulation ([Z1] 3.1 and [Z2] config: gradient_accumulation_steps): call
 * once per micro-batch and bucket, micro = 0 .. n_micro-1 in order. Micro-batch 0
 * writes reduced[i] = the rank-ordered fp32 sum as zero_reduce_scatter_bucket does;
 * each later one adds its sum: reduced[i] = reduced[i] + ((g_0[i] + g_1[i]) + ...);
 * the last one also takes the sum of squares of the accumulated values and counts the
 * bucket as reduced for this step. n_micro = 1 is zero_reduce_scatter_bucket. A bucket's
 * micro-batches may interleave with other buckets' (e.g. micro-major order, bucket by
 * bucket as backward produces them). ESTATE on a micro-batch out of order or a change of
 * n_micro within a step. */
ZERO_API int zero_reduce_scatter_bucket_accum(zero_plan* plan, int64_t bucket, int32_t micro,
                                              int32_t n_micro, int32_t grad_dtype,
                                              const void* const* replica_grads,
                                              int64_t replica_base_offset, float* reduced,
                                              void* workspace, void* stream);

/* zero_step = zero_step_finalize + zero_step_update.
 * zero_step_finalize (one CTA): S = sum of the partial sums in a fixed order; overflow
 * = S not finite (any inf/NaN reduced gradient makes S inf or NaN); norm = sqrt(S)/scale
 * in fp64; clip c = max_grad_norm/(norm + 1e-6) when below 1 ([Z1] 6); k = fp32(c/scale)
 * folds unscale and clip into one multiply; loss-scaler transition ([Z1] 3.3, 5.1): on
 * overflow, a hysteresis budget <= 1 divides the scale by the factor (not below
 * min_loss_scale), otherwise the budget drops by one; on a good step the scale grows
 * and the budget refills when (iter - last_overflow_iter) is a multiple of
 * loss_scale_window. An overflowing step is skipped whole (master, m, v, params and
 * adam_t unchanged); otherwise adam_t += 1 and the bias corrections 1 - beta^t are
 * formed in fp64. ESTATE unless every bucket was reduced once since the last step.
 * zero_step_update (AdamW on every owned partition, [Z1] 2.1 and 3.1, [Z3] FAQ), for
 * every flat index i, in fp32 with each operation rounded (no fused multiply-add):
 *   g = reduced[i]*k; m = b1*m + (1-b1)*g; v = b2*v + (1-b2)*(g*g);
 *   p = p*(1 - lr*wd) - lr * ((m/bc1) / (sqrt(v/bc2) + eps));
 *   params[i] = round_to_nearest_even_half(p)   (the fused all-gather write)
 * It does nothing when the finalize step decided to skip. master, exp_avg, exp_avg_sq
 * and reduced are n_pad fp32; params is the n_pad half gathered buffer. */
ZERO_API int zero_step(zero_plan* plan, const zero_adamw_cfg* cfg, float* master, float* exp_avg,
              float* exp_avg_sq, const float* reduced, void* params, int32_t param_dtype,
              void* workspace, void* stream);
ZERO_API int zero_step_finalize(zero_plan* plan, const zero_adamw_cfg* cfg, void* workspace,
                       void* stream);
ZERO_API int zero_step_update(zero_plan* plan, float* master, float* exp_avg, float* exp_avg_sq,
                     const float* reduced, void* params, int32_t param_dtype,
                     const void* workspace, void* stream);

/* zero_step_full: the whole step in one call -- zero_reduce_scatter_bucket for every
 * bucket in order, then zero_step -- for replica buffers that hold every bucket
 * (replica_grads[r][i] is flat element i; replica_base_offset must be 0). Every argument
 * is checked before the first launch, so a refused call changes nothing. Arguments and
 * errors as for those calls; ESTATE when buckets of this step were already
 * reduce-scattered. */
ZERO_API int zero_step_full(zero_plan* plan, const zero_adamw_cfg* cfg, int32_t grad_dtype,
                            const void* const* replica_grads, int64_t replica_base_offset,
                            float* reduced, float* master, float* exp_avg, float* exp_avg_sq,
                            void* params, int32_t param_dtype, void* workspace, void* stream);

/* zero_step_resident: the whole step for W <= 2 ranks whose replica gradients are all
 * still in device memory when the step runs ([Z1] 2.1 the reduce-scatter of gradients
 * and the per-partition update; the schedule is this library's). The bucket kernel
 * computes only the sum of squares of every bucket (no reduced gradient is stored),
 * and the update forms each element's reduced gradient again from the replicas -- the
 * same rank-ordered fp32 sum, so every result is bit-identical to
 * zero_reduce_scatter_bucket for each bucket followed by zero_step. It moves 4W + 26
 * bytes per parameter instead of 2W + 34: 30 against 36 at W = 1, 34 against 38 at
 * W = 2 (equal at W = 4, more above; hence the limit).
 *   replica_grads[r]: replica r's gradients over the whole padded flat space (n_pad
 *       elements of grad_dtype, 16-byte aligned); master / exp_avg / exp_avg_sq: fp32,
 *       n_pad elements; params: the gathered buffer, n_pad elements of param_dtype.
 * Errors: EINVAL (NULL, bad dtype or hyperparameters, world_size > 2), EALIGN, ESTATE
 * when buckets of this step were already reduce-scattered, ECUDA. */
ZERO_API int zero_step_resident(zero_plan* plan, const zero_adamw_cfg* cfg, int32_t grad_dtype,
                                const void* const* replica_grads, float* master,
                                float* exp_avg, float* exp_avg_sq, void* params,
                                int32_t param_dtype, void* workspace, void* stream);

/* zero_all_gather ([Z1] 2.1 parameters gathered by allgather; [Z1] 2.2 batched
 * all-gather; [Z2] allgather_bucket_size): after zero_step the gathered buffer `params`
 * already holds every rank's partition, so n_dst = 0 is a no-op. With n_dst > 0 the
 * full buffer is copied into each rank_params[d] (n_pad halves each, HOST array of
 * device pointers), i.e. the per-rank replicas a multi-process run would hold. */
ZERO_API int zero_all_gather(const zero_plan* plan, const void* params, void* const* rank_params,
                    int32_t n_dst, int32_t param_dtype, void* stream);

/* Copies the step result out of the workspace and synchronises `stream`. Returns
 * ZERO_EDEVICE (with *out filled) if a kernel reported a timed-out internal wait. */
ZERO_API int zero_get_result(const void* workspace, zero_step_result* out, void* stream);

/* ---------------------------------------------------------------- one rank of W processes
 * A real data-parallel run: W processes, one GPU each, the same plan on every rank;
 * rank r owns partition r ([Z1] 2.1: each GPU updates only its own partition; [Z3]: each
 * GPU keeps only the gradient slice for its own parameters) and holds its fp32 master,
 * m, v and reduced gradient for that partition only (p elements each). One step on rank r:
 *   for every bucket b that meets partition r (in order):
 *       zero_reduce_scatter_segment(b, r): reduced_local = rank-ordered fp32 sum of the W
 *       replicas over bucket b ∩ partition r. replica_grads[q] is rank q's gradient
 *       buffer mapped into this process (CUDA IPC, NVLink peer reads; no multicast);
 *       the caller orders it after every rank finished writing bucket b.
 *   zero_step_local_sumsq(r): this rank's fp64 sum of squares into *sumsq_out (device).
 *   exchange: the caller gathers the W sums into sumsq_ranks (device, rank order), e.g.
 *       with an all-gather.
 *   zero_step_finalize_ranks: S = ((s_0 + s_1) + ...) + s_{W-1}, then the same scalar
 *       step as zero_step_finalize -- identical on every rank.
 *   zero_step_update_partition(r): AdamW on the local arrays; the p half results go to
 *       params_dst[d][0 .. p) for every d: where rank r's slice lives in each
 *       destination -- gathered buffer + r*p of this rank and, mapped over CUDA IPC, of
 *       its peers (the all-gather fused into the update as P2P stores), or a buffer
 *       holding only this rank's partition (parameters partitioned as in ZeRO-3).
 *       Each destination must be 16-byte aligned (choose align so that p*2 % 16 == 0).
 * Errors as above; ESTATE when a segment is reduced twice, a bucket outside the rank's
 * partition is reduced, or the calls come out of order. */
ZERO_API int zero_reduce_scatter_segment(zero_plan* plan, int64_t bucket, int32_t rank,
                                         int32_t grad_dtype, const void* const* replica_grads,
                                         int64_t replica_base_offset, float* reduced_local,
                                         void* workspace, void* stream);
ZERO_API int zero_step_local_sumsq(zero_plan* plan, int32_t rank, void* workspace,
                                   double* sumsq_out, void* stream);
ZERO_API int zero_step_finalize_ranks(zero_plan* plan, const zero_adamw_cfg* cfg,
                                      const double* sumsq_ranks, void* workspace, void* stream);
ZERO_API int zero_step_update_partition(zero_plan* plan, int32_t rank, float* master_local,
                                        float* exp_avg_local, float* exp_avg_sq_local,
                                        const float* reduced_local, void* const* params_dst,
                                        int32_t n_dst, int32_t param_dtype,
                                        const void* workspace, void* stream);

/* Peer memory: CUDA IPC handles (zero_ipc_handle_bytes() opaque bytes) so that rank q's
 * buffers can be read and written by the other ranks' kernels over NVLink. The caller
 * moves the handle bytes and the offset between processes (e.g. an all-gather of
 * objects).
 *   zero_ipc_get_handle: a handle to the device allocation that holds device_ptr, and in
 *       *offset_out the byte offset of device_ptr from that allocation's start (a pool
 *       allocator such as torch's places many buffers in one allocation).
 *   zero_ipc_open_handle: maps the peer's whole allocation into this process and returns
 *       its start in *base_out; the peer's buffer is at base + offset. The mapping stays
 *       valid until zero_ipc_close(base) and the exporter must keep the allocation alive
 *       until every peer has closed it. A handle exported by this process cannot be
 *       opened by it (use the pointer itself).
 * Errors: EINVAL for NULL arguments; ECUDA when the runtime refuses (the message names
 * the call). */
ZERO_API int zero_ipc_handle_bytes(void);
ZERO_API int zero_ipc_get_handle(const void* device_ptr, void* handle_out, int64_t* offset_out);
ZERO_API int zero_ipc_open_handle(const void* handle, void** base_out);
ZERO_API int zero_ipc_close(void* base);

/* ---------------------------------------------------------------- ZeRO-3 parameters
 * Stage 3 partitions the half parameters too ([Z1] 1.2.3; [Z2]; [Z3] technical insight):
 * rank r keeps only its partition (p halves; the update writes it with
 * zero_step_update_partition or, on one GPU, into slice r of the gathered buffer), and
 * a layer's tensors are all-gathered before its forward pass and dropped after it.
 *
 * zero3_schedule_create: the fetch / release order for a forward pass over n_layers
 * layers run in order (layer_of_tensor[t] in [0, n_layers), or -1 for a tensor the
 * forward pass does not use), from the knobs of [Z1] 3.1 / 6:
 *   - tensors with numel <= persistence_threshold (stage3_param_persistence_threshold)
 *     are fetched once, first, and never released;
 *   - before layer i: FETCH its tensors that are not live (even past the budget);
 *   - then prefetch the later layers' tensors in order while the live elements fetched
 *     ahead of layer i stay <= prefetch_bucket_size (stage3_prefetch_bucket_size) and
 *     all live elements stay <= max_live_parameters (stage3_max_live_parameters); the
 *     first tensor that does not fit stops the prefetch; the prefetched tensors form one
 *     FETCH (one bucketed all-gather);
 *   - COMPUTE layer i, then RELEASE its tensors.
 * Events reference runs of the tensor-id list (zero3_schedule_tensors). */
#define ZERO3_FETCH 0
#define ZERO3_COMPUTE 1
#define ZERO3_RELEASE 2
typedef struct zero3_schedule zero3_schedule; /* opaque, host memory */
typedef struct {
  int32_t op;    /* ZERO3_FETCH / ZERO3_COMPUTE / ZERO3_RELEASE                        */
  int32_t layer; /* the layer being run (-1: the persistent fetch before layer 0)       */
  int64_t first; /* first index into the tensor-id list                                 */
  int64_t count; /* tensor ids in this event                                            */
} zero3_event;
typedef struct {
  int64_t peak_live_elements;  /* live half elements at the busiest compute, persistent included */
  int64_t fetched_elements;    /* elements all-gathered over the forward pass                    */
  int64_t fetch_events;        /* bucketed all-gathers                                            */
  int64_t persistent_elements; /* elements kept for the whole pass                                */
  int64_t over_budget_layers;  /* layers whose own tensors exceeded max_live_parameters           */
} zero3_stats;
ZERO_API int zero3_schedule_create(const zero_plan* plan, const int32_t* layer_of_tensor,
                                   int32_t n_layers, int64_t prefetch_bucket_size,
                                   int64_t max_live_parameters, int64_t persistence_threshold,
                                   zero3_schedule** out);
ZERO_API int zero3_schedule_events(const zero3_schedule* s, zero3_event* out, int64_t cap,
                                   int64_t* count);
ZERO_API int zero3_schedule_tensors(const zero3_schedule* s, int32_t* out, int64_t cap,
                                    int64_t* count);
ZERO_API int zero3_schedule_stats(const zero3_schedule* s, zero3_stats* out);
ZERO_API void zero3_schedule_destroy(zero3_schedule* s);

/* zero3_gather: the all-gather of a FETCH. dst receives the listed tensors' half values
 * back to back, in the order given; element i of the flat space is read from
 * partitions[i / p][i % p] (partitions[r]: rank r's partition of p halves -- peer memory
 * mapped over CUDA IPC in a multi-process run, read over NVLink; slices of the gathered
 * buffer on one GPU). One launch for up to 64 contiguous pieces, 16-byte vector copies
 * where source and destination share their alignment. */
ZERO_API int zero3_gather(const zero_plan* plan, const int32_t* tensors, int32_t n_tensors,
                          const void* const* partitions, void* dst, void* stream);

/* ---------------------------------------------------------------- no-alloc variant
 * zero_reduce_sumsq_noalloc has no counterpart in the pages. It is for callers that
 * cannot allocate device memory for a workspace: for example a C plugin that its host
 * framework hands only the input and output buffers, with no access to that
 * framework's allocator, or a loop that must not call cudaMalloc because cudaMalloc can
 * synchronise the whole device.
 * Without a plan or a workspace it computes what zero_reduce_scatter_bucket computes for
 * one bucket:
 *   reduced[i] = ((g_0[i] + g_1[i]) + ...) + g_{W-1}[i]   (fp32, rank order), i < n,
 * and writes the fp64 sum of squares of reduced[0 .. n) to *sumsq (device memory).
 * Scratch: the per-block partial sums go to an array of ZERO_NOALLOC_MAX_BLOCKS fp64
 * slots (512 KB) compiled into the library; every GPU that loads the library holds it
 * until the process exits. One block covers 2048 elements, so n may be at most
 * ZERO_NOALLOC_MAX_ELEMS; a larger n returns ZERO_ERANGE (split the range into calls).
 * The first call on a device looks up the array's device address with that device
 * current; make that first call before any stream capture.
 * Every call uses the same array and writes each slot before reading it, so nothing
 * needs clearing between calls; calls that overlap on the GPU (other streams, other
 * host threads) race on the array and return wrong sums, so serialise them.
 * replica_grads is a HOST array of world_size device pointers (16-byte aligned);
 * reduced must be 16-byte aligned and sumsq 8-byte aligned. Errors: EINVAL (W outside
 * [1, 16], bad dtype, NULL pointer, n < 0), EALIGN, ERANGE (n too large), ECUDA. */
#define ZERO_NOALLOC_MAX_BLOCKS 65536
#define ZERO_NOALLOC_MAX_ELEMS ((int64_t)ZERO_NOALLOC_MAX_BLOCKS * 2048)
ZERO_API int zero_reduce_sumsq_noalloc(int32_t world_size, int32_t grad_dtype,
                                       const void* const* replica_grads, int64_t n,
                                       float* reduced, double* sumsq, void* stream);

/* Diagnostics: launches one thread that waits on a barrier phase nothing completes, so
 * the kernels' bounded wait (about one second) runs out; it records its code (64) in the
 * workspace's sticky device_error, as a pipeline wait that gave up would. The next
 * zero_get_result then returns ZERO_EDEVICE and the CUDA context stays usable;
 * zero_state_init clears the flag. */
ZERO_API int zero_selftest_bounded_wait(void* workspace, void* stream);

ZERO_API const char* zero_last_error(void);
ZERO_API int zero_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ZERO_B200_H */
