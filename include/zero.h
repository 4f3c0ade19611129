/*
 * zero.h -- C ABI of the B200 sharded mixed-precision Adam step (ZeRO stages 1, 2 and 3).
 *
 * The library (libzero.so, built from zero_sharded_optimizer_03_b200/csrc) implements the
 * data-parallel hot path of the Zero Redundancy Optimizer as described by
 *   [P1] "ZeRO 优化器的三个阶段深度对比：显存节省与通信开销的量化分析" (wmrh.cn/news/520095)
 *   [P2] "ZeRO 优化器：把显存“分”着用" (5688vip.com course note 03)
 *   [P3] "ZeRO Optimization（零冗余优化）" (ai-master.cc glossary)
 * with its collectives simulated over Nd virtual ranks whose buffers all live in the memory
 * of one GPU: the reduce-scatter is an Nd-way fan-in read and the all-gather an Nd-way
 * fan-out write, inside the same kernels as the optimizer arithmetic.
 *
 * Conventions (every entry point):
 *   - Returns ZERO_OK (0) or a negative error code; zero_last_error() then returns a message
 *     (thread-local, valid until the next call on the same thread).  Nothing aborts.
 *   - The caller owns all memory.  The library never allocates device or host memory.  Device
 *     pointers are plain CUDA device addresses (e.g. torch tensor data_ptr()).
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  Device
 *     work is enqueued on it and runs asynchronously; only zero_read_result synchronizes.
 *   - Element indices are global positions in the flat parameter vector of N elements.  The
 *     fp32 optimizer state (master weights, exp_avg, exp_avg_sq) is stored flat and padded:
 *     Nd*S floats with S = ceil(N/Nd); rank r's shard is the view [r*S, (r+1)*S) and elements
 *     N .. Nd*S-1 are padding that the caller zero-fills once and the library never writes.
 *   - 16-bit values (gradients, bf16 weights) are passed as raw uint16_t bit patterns.
 *   - Pointers that are 16-byte aligned take the vectorised path; any other alignment is
 *     accepted and handled element by element (same results, slower).
 *   - An empty window (lo == hi, N == 0, L == 0) is a valid no-op; its pointers may be NULL.
 *   - An overflow (inf/NaN in the reduced gradient) is not an error: the step is skipped and
 *     reported through the workspace (see zero_read_result).
 *   - Numerics: each update is the element-wise rule written out in zero_adam_shard, one
 *     fp32 round-to-nearest operation at a time, no fused multiply-add; gradient replicas are
 *     summed in rank order 0..Nd-1.  Results do not depend on the launch configuration,
 *     except the last bits of the reported sum of squares (fixed order for a given GPU).
 */
#ifndef ZERO_H
#define ZERO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------ codes and limits */

#define ZERO_OK 0
#define ZERO_EINVAL (-1)   /* an argument is out of range or NULL; the message names it */
#define ZERO_ECUDA (-2)    /* a CUDA runtime call or a kernel launch failed */
#define ZERO_ENOMEM (-3)   /* the fixed scratch memory inside the library is too small for the
                              request (zero_reduce_scatter_noalloc); caller-provided workspaces
                              have a fixed size (zero_workspace_bytes) and cannot run short */
#define ZERO_ETIMEOUT (-4) /* a kernel gave up a bounded internal wait (1 s).  Kernels run
                              asynchronously, so this is recorded in the workspace error word
                              when it happens and returned by the next synchronizing call,
                              zero_read_result, which still fills its output */

#define ZERO_MAX_ND 64   /* largest number of simulated data-parallel ranks */

/* gradient replica element types */
#define ZERO_BF16 0
#define ZERO_FP16 1

/* zero_step flags */
#define ZERO_FUSED 0     /* stages 1/2: one fused pass (default); state copies ping-pong */
#define ZERO_TWO_PASS 1  /* stages 1/2: reduce-scatter into grad_shard, then Adam + all-gather */
#define ZERO_NO_TMA 2    /* ZERO_FUSED: always use the register-pipelined kernel */
#define ZERO_FORCE_TMA 4 /* ZERO_FUSED: use the TMA-pipelined kernel whenever buffers are aligned;
                            stage 3: gather layers with the TMA fan-out instead of the register
                            kernel (the default) */
#define ZERO_BF16_GRAD_SHARD 8 /* ZERO_TWO_PASS / stage 3: keep the reduced gradient as bf16 (see
                                  grad_shard); not described by the pages */
#define ZERO_FUSED_LAYERS 16   /* stage 3: one fused pass per layer (reduce-scatter + AdamW + bf16
                                  shard) writing the other state copy, speculatively, as ZERO_FUSED
                                  does for stages 1/2; needs both state copies, no grad_shard, no
                                  clipping; same results (see zero_step) */

/* zero_allgather gates */
#define ZERO_GATE_ALWAYS 0      /* always cast and write */
#define ZERO_GATE_NO_OVERFLOW 1 /* write nothing if the current step has overflowed so far */

/* ------------------------------------------------------------------ types */

/* Partition of N elements over Nd ranks ([P1] §二: each rank keeps 1/Nd of the optimizer
 * state; [P3] core operations: each process keeps only its own shard). */
typedef struct {
    int64_t N;      /* elements */
    int32_t Nd;     /* ranks */
    int32_t reserved;
    int64_t S;      /* shard length ceil(N/Nd); rank r owns [r*S, min((r+1)*S, N)) */
    int64_t Np;     /* padded length Nd*S */
    int64_t pad;    /* Np - N */
} zero_partition_t;

/* Hyperparameters of one step.  lr may change from call to call (schedules). */
typedef struct {
    double lr;
    double beta1, beta2;
    double eps;
    double weight_decay;  /* decoupled (AdamW); 0 gives Adam */
    double loss_scale;    /* static fp16 loss scale the gradients carry; 1 if none (ignored
                             while the workspace's dynamic loss scaler is on) */
    int32_t grad_average; /* nonzero: g = sum/(Nd*loss_scale) (data-parallel mean); 0: sum/loss_scale */
    int32_t reserved;
    double max_grad_norm; /* > 0: clip the reduced gradient to this global 2-norm before the
                             update, g *= min(1, max_grad_norm/(||g|| + 1e-6)); 0: no clipping.
                             Needs the norm before the update: ZERO_TWO_PASS, stage 3, or the
                             building blocks (the fused one-pass step refuses it) */
} zero_hparams_t;

/* Host copy of the step bookkeeping kept in the workspace. */
typedef struct {
    int64_t step;       /* completed (not skipped) updates t */
    int64_t skipped;    /* steps skipped because of an overflow */
    int32_t overflow;   /* 1 if the last finished step was skipped */
    int32_t live;       /* ZERO_FUSED / ZERO_FUSED_LAYERS: index (0/1) of the state copy that
                           holds the current state */
    double grad_sumsq;  /* sum of squares of the last finished step's reduced gradient */
    int32_t pending_overflow; /* overflow accumulated by the step in progress */
    int32_t reserved;
    double pending_sumsq;     /* sum of squares accumulated by the step in progress */
    int32_t error;            /* nonzero if a kernel gave up a bounded internal wait (1 s); the
                                 step was then skipped.  Sticky until zero_workspace_init. */
    int32_t reserved2;
    double loss_scale;        /* dynamic loss scaler: the scale the next step's gradients must
                                 carry (0 when the scaler is off) */
    int64_t good_steps;       /* dynamic loss scaler: clean steps since the scale last changed */
    int32_t dynamic_scale;    /* 1 when the dynamic loss scaler is on */
    int32_t reserved3;
} zero_step_result_t;

/* Buffers of a whole step (zero_step).  All pointers are device pointers owned by the caller.
 * Unused fields may be NULL. */
typedef struct {
    int32_t grad_dtype;  /* ZERO_BF16 or ZERO_FP16 */
    int32_t flags;       /* ZERO_FUSED or ZERO_TWO_PASS (stages 1/2), plus the ZERO_* options */
    /* stages 1/2: rank r's gradient replica (N elements) and bf16 weight replica (N elements).
     * stage 3: rank r's gradient buffer and gathered-weight buffer for the layer being
     * processed; layer l uses grads[r] + l*grad_layer_stride and params[r] + l*param_layer_stride
     * (a stride of 0 reuses one layer-sized buffer, which is how a backward pass frees them). */
    const uint16_t *grads[ZERO_MAX_ND];
    uint16_t *params[ZERO_MAX_ND];
    /* fp32 state, each padded (stages 1/2: Nd*S floats; stage 3: the padded layers back to back).
     * ZERO_FUSED (stages 1/2) and ZERO_FUSED_LAYERS (stage 3) read copy `live` and write copy
     * 1-live, so both copies must be allocated and zero-initialised in their padding; the other
     * paths use copy 0 in place. */
    float *master[2];
    float *exp_avg[2];
    float *exp_avg_sq[2];
    float *grad_shard;      /* reduced gradient, same padded length (ZERO_TWO_PASS, stage 3 without
                               ZERO_FUSED_LAYERS): fp32,
                               or bf16 (uint16_t storage, cast to float*) with ZERO_BF16_GRAD_SHARD:
                               the reduced mean is then rounded to bf16 (nearest even) before it is
                               stored, and the overflow check, the norm and the update use the
                               rounded value; 2 bytes per element of memory and traffic saved */
    uint16_t *param_shard;  /* stage 3: bf16 weights, the Nd shards of every layer (padded) */
    int64_t grad_layer_stride;
    int64_t param_layer_stride;
    void *workspace;        /* zero_workspace_bytes() bytes, 16-byte aligned, initialised by
                               zero_workspace_init */
} zero_state_t;

/* Per-GPU model-state memory in GiB (2^30 bytes). */
typedef struct {
    double optimizer_states, gradients, parameters, total;
} zero_mem_t;

/* ------------------------------------------------------------------ bookkeeping */

/* Message of the last failed call on this thread ("" if none).  Never NULL. */
const char *zero_last_error(void);

/* Library version string, e.g. "zero-b200 1.0 sm_100a". */
const char *zero_version(void);

/* Fills *out with the partition of N elements over Nd ranks.  N >= 0 (N = 0 gives S = 0),
 * 1 <= Nd <= ZERO_MAX_ND.  Host only. */
int zero_partition(int64_t N, int Nd, zero_partition_t *out);

/* Bytes of device workspace a step needs (a small constant: step counter, overflow flag,
 * sum of squares, per-CTA partials).  One workspace per optimizer (it carries the step count).
 * Every call that takes a workspace refuses, with ZERO_EINVAL and before any device work, a
 * NULL one or one whose address is not a multiple of 16 (the kernels update its doubles and
 * 64-bit counters in place). */
size_t zero_workspace_bytes(void);

/* Sets the workspace to "t completed updates, nothing pending, state copy 0 live".  Async. */
int zero_workspace_init(void *ws, int64_t t, void *stream);

/* Turns on dynamic loss scaling for the optimizer that owns `ws` (mixed precision: the pages
 * only name AMP, [P3] comparisons; this is the usual backoff/growth rule).  From then on the
 * gradients of every step are taken to carry the workspace's current scale (hp->loss_scale is
 * ignored) and the end of each step updates it: after an overflow (the step is skipped) scale *=
 * backoff_factor; after growth_interval clean steps in a row scale *= growth_factor, unless that
 * would leave the finite fp32 range.  Read the scale for the next backward pass from
 * zero_read_result.  zero_workspace_init turns the scaler off.  Async. */
int zero_loss_scaler_init(void *ws, double init_scale, double growth_factor, double backoff_factor,
                          int64_t growth_interval, void *stream);

/* Copies the workspace bookkeeping to *out.  Synchronizes `stream` (waits for queued steps).
 * Returns ZERO_ETIMEOUT, with *out filled, while the workspace error word is set (a bounded
 * internal wait gave up in an earlier step; that step was skipped); ZERO_OK otherwise. */
int zero_read_result(const void *ws, zero_step_result_t *out, void *stream);

/* ------------------------------------------------------------------ building blocks */

/* Starts a step: clears the pending overflow flag and sum of squares.  Async. */
int zero_begin_step(void *ws, void *stream);

/* Reduce-scatter of gradients ([P1] §二 ZeRO-2: gradients are reduced and scattered to the
 * owning ranks; [P3] backward: ReduceScatter).  For every global index i in [lo, hi):
 *     g[i] = (grads[0][i] + grads[1][i] + ... + grads[Nd-1][i]) * inv      (fp32, rank order)
 * with inv = 1/(Nd*loss_scale) (grad_average) or 1/loss_scale, written to grad_out[i] (fp32;
 * element i belongs to rank i/S's shard).  grads: host array of Nd device pointers to replicas
 * of `dtype` (ZERO_BF16 / ZERO_FP16) that cover [lo, hi).  Adds whether any g is inf/NaN and
 * sum(g^2) to the pending values in the workspace.  Only hp->loss_scale and hp->grad_average
 * are read.  0 <= lo <= hi; 1 <= Nd <= ZERO_MAX_ND.  Async. */
int zero_reduce_scatter(const uint16_t *const *grads, int dtype, int Nd, int64_t lo, int64_t hi,
                        const zero_hparams_t *hp, float *grad_out, void *ws, void *stream);

/* Adam/AdamW on a shard ([P1] §二: each rank runs the optimizer step on the parameters it
 * holds; [P2] "ZeRO Stage 1"; [P3] parameter update).  Unless the pending overflow flag is set
 * (then nothing is written), for every i in [lo, hi), in fp32 with t = completed updates + 1:
 *     p = p * (1 - lr*wd)
 *     m = b1*m + (1-b1)*g
 *     v = b2*v + ((1-b2)*g)*g
 *     p = p - (lr/(1-b1^t)) * (m / (sqrt(v)/sqrt(1-b2^t) + eps))
 * on master/exp_avg/exp_avg_sq[i] in place, with g = grad[i].  The scalars in parentheses are
 * evaluated in double and rounded once to fp32.  If param_out is not NULL, param_out[i] =
 * bf16(p) (round to nearest even; the ZeRO-3 weight shard).  Does not advance t (see
 * zero_end_step).  Async. */
int zero_adam_shard(float *master, float *exp_avg, float *exp_avg_sq, const float *grad,
                    int64_t lo, int64_t hi, const zero_hparams_t *hp, uint16_t *param_out,
                    void *ws, void *stream);

/* All-gather of the updated weights ([P1] §二 ZeRO-1: the updated parameters are all-gathered
 * to every rank; [P3] forward: AllGather): replicas[r][i] = bf16(master[i]) for every rank
 * r < Nd and i in [lo, hi).  gate = ZERO_GATE_ALWAYS or ZERO_GATE_NO_OVERFLOW (then nothing
 * is written if the pending overflow flag is set; ws may be NULL with ZERO_GATE_ALWAYS).
 * Async. */
int zero_allgather(const float *master, uint16_t *const *replicas, int Nd, int64_t lo,
                   int64_t hi, int gate, const void *ws, void *stream);

/* Ends a step: if the pending overflow flag is clear, t = t + 1, otherwise the skip count
 * grows; the pending values become the "last step" values of zero_read_result.  Async. */
int zero_end_step(void *ws, void *stream);

/* ZeRO-3 just-in-time gather of one layer ([P1] §三: before a layer runs, its full parameters
 * are all-gathered from the ranks holding the shards and freed after use; [P2] "ZeRO Stage 3";
 * [P3] forward).  shards: Nd device pointers, shard r holds elements [r*S, (r+1)*S) of the
 * layer (S = ceil(L/Nd); the last shards may be partly or wholly padding).  Writes the L
 * elements out[o][j] = shards[j/S][j%S] for every one of the nout (1..ZERO_MAX_ND) output
 * buffers (one per rank that receives the layer).  Async. */
int zero3_gather_layer(const uint16_t *const *shards, int Nd, int64_t L, uint16_t *const *out,
                       int nout, void *stream);

/* ------------------------------------------------------------------ one whole step */

/* One optimizer step of ZeRO stage 1, 2 or 3 ([P1] §二 and §三; [P2] "ZeRO Stage 1/2/3").
 *   stage 1/2, ZERO_FUSED (default): reduce-scatter + unscale + overflow check + Adam + bf16
 *     cast + all-gather in one pass over each bucket [k*bucket, (k+1)*bucket) of [0, N)
 *     (bucket = 0: one bucket).  Two kernels implement the pass with identical results: a
 *     register-pipelined one (16-byte vector loads and stores) and a TMA-pipelined one (bulk
 *     copies through a shared-memory ring, bulk-store fan-out to the replicas).  The TMA one is
 *     chosen for wide fan-in (Nd >= 16) over buckets of at least 2^24 elements when every buffer
 *     is 16-byte aligned; ZERO_NO_TMA / ZERO_FORCE_TMA in flags override the choice.  The pass
 *     reads state copy `live` and writes copy 1-live and the Nd weight replicas; when the step
 *     ends without overflow the copies swap, otherwise the replicas are rewritten from the
 *     unchanged state.  Stages 1 and 2 compute the same values (they differ in what a real
 *     cluster keeps in memory, see zero_memory_estimate).  Buckets after the first, and the
 *     overflow-repair check after the last, are programmatic dependent launches on `stream`
 *     (each may start while the previous kernel of the step finishes; it waits for that kernel
 *     before using its results), so nothing else should be enqueued between them: one
 *     zero_step call enqueues the whole step.  An unbucketed register-pipelined step of at most
 *     2^21 elements has no repair launch: after an overflow the pass's last CTA rewrites the
 *     replicas itself (slower for that skipped step, one launch fewer for every other).  The
 *     first launch of the register-pipelined pass
 *     is a programmatic dependent of whatever precedes it on `stream` and waits for it to
 *     complete before it reads or writes anything, so stream order is kept; after a previous
 *     step's repair check its launch overlaps that kernel.
 *   stage 1/2, ZERO_TWO_PASS: reduce-scatter into grad_shard, then (if no overflow) Adam in
 *     place on copy 0 fused with the cast and the all-gather.
 *   stage 3: N elements in layers of `bucket` elements (the last may be shorter; bucket = 0
 *     means one layer), each padded to a multiple of Nd.  For each layer: gather its bf16
 *     weights from param_shard into params[r] (every rank), reduce-scatter its gradient
 *     replicas into grad_shard; after the last layer, if no overflow, Adam in place on copy 0
 *     and param_shard = bf16(master).
 *   stage 3, ZERO_FUSED_LAYERS: for each layer, one fused pass over the layer that also
 *     gathers it: each element's old bf16 weight goes to every params[r] (the gather above),
 *     then the reduce-scatter of its gradient replicas, unscale, overflow check, Adam from copy
 *     `live` into copy 1-live, and the layer's param_shard = bf16(new master) over the old
 *     weight (with ZERO_FORCE_TMA the gather is a TMA fan-out kernel before the pass).  The
 *     overflow decision needs every layer, so the updates are speculative: the end of the step
 *     swaps the copies if no element overflowed; otherwise param_shard is rewritten from the
 *     unchanged copy.  Same values as the two-phase stage 3, 28 + 4*Nd bytes of traffic per
 *     parameter instead of 36 + 4*Nd, for a second fp32 state copy (12 bytes per parameter);
 *     no grad_shard; refuses max_grad_norm > 0 and ZERO_BF16_GRAD_SHARD (ZERO_EINVAL).
 * Every path skips the whole update (state, weights, t) when any reduced gradient element is
 * inf or NaN.  Every buffer of `st` is memory of the current device (the register-pipelined
 * pass may prefetch a thread's next vector into L2; a pass over other GPUs' memory is
 * zero_fused_window, which never prefetches).  Asynchronous: call zero_read_result to learn
 * whether the step was skipped. */
int zero_step(int stage, int Nd, int64_t N, int64_t bucket, const zero_state_t *st,
              const zero_hparams_t *hp, void *stream);

/* Tracing hook.  Registers two cudaEvent_t handles (passed as void*) for the next zero_step
 * call on this thread: `start_event` is recorded on its stream just before the first kernel
 * that reads gradients and `stop_event` just after the last kernel that writes state (for
 * ZERO_FUSED and ZERO_FUSED_LAYERS: the fused kernels and the overflow-repair check that
 * follows them, which is a no-op unless the step overflowed).  One-shot: the
 * registration is cleared once each event is recorded.  NULL clears.  The events stay owned
 * by the caller.  Always returns ZERO_OK. */
int zero_profile_events(void *start_event, void *stop_event);

/* ------------------------------------------------------------------ no-allocation variant */

/* Result of one zero_reduce_scatter_noalloc window (device memory owned by the caller). */
typedef struct {
    int32_t overflow;  /* 1 if any reduced element of the window is inf or NaN */
    int32_t reserved;
    double sumsq;      /* sum of squares of the window's reduced elements */
} zero_rs_summary_t;

#define ZERO_NOALLOC_MAX_CTAS 16384                                /* scratch slots */
#define ZERO_NOALLOC_MAX_WINDOW ((int64_t)ZERO_NOALLOC_MAX_CTAS * 2048) /* 33,554,432 elements */

/* The pages have no counterpart to this entry point: it exists for callers that cannot
 * allocate device memory.  Some callers cannot hand the library a workspace: a plugin inside a
 * host application that owns all device memory through its own fixed arena has no spare buffer
 * to give, and code on a latency-critical path cannot call cudaMalloc, which may synchronize the
 * whole device.  For them this call computes exactly what zero_reduce_scatter computes (the same
 * grad_out, bit for bit) without a workspace and without allocating anything (no cudaMalloc,
 * cudaFree or allocating library call).
 *
 * Its scratch -- one arrival counter and one partial (flag, sum of squares) per CTA -- is a fixed
 * array inside the library: 256 B + 16 B x ZERO_NOALLOC_MAX_CTAS (about 256 KiB), held by every
 * GPU that loads the library until the process exits.  The call uses one CTA per 2048 elements,
 * so a window [lo, hi) may hold at most ZERO_NOALLOC_MAX_WINDOW elements; a larger window is
 * rejected with ZERO_ENOMEM and a message naming the limit (split it into buckets).
 *
 * grads, dtype, Nd, lo, hi, hp, grad_out: as for zero_reduce_scatter.  summary: device pointer the
 * call writes the window's result to (accumulate = 0), or combines it into (accumulate != 0:
 * overflow |= window's, sumsq += window's; the caller zeroes it before the first window).  The
 * workspace bookkeeping of zero_step is not touched, so a dynamic loss scale kept there does not
 * apply: the unscale factor comes from hp->loss_scale.
 *
 * The first call on each device looks up the scratch array's device address (with that device
 * current) and keeps it; make that first call before any stream capture.  All calls share the one
 * scratch array, which keeps the last call's contents; each call clears the counter before its
 * kernel runs.  Calls that can overlap on the GPU (issued on different streams, or from different
 * host threads without ordering) race on the scratch: issue them on one stream.  Async. */
int zero_reduce_scatter_noalloc(const uint16_t *const *grads, int dtype, int Nd, int64_t lo,
                                int64_t hi, const zero_hparams_t *hp, float *grad_out,
                                zero_rs_summary_t *summary, int accumulate, void *stream);

/* Test hook for the bounded waits inside the TMA-pipelined kernel (failure detection without a
 * GPU fault).  The next TMA-pipelined launch made by zero_step on this thread issues no copies
 * for load unit `unit` of its first CTA, so nothing ever completes that unit's barrier: the
 * CTA's consumers give up after the 1 s bound, the launch drains what it issued, the workspace
 * error word is set (zero_step_result_t.error) and the step is reported as overflowed, so the
 * state and the weight replicas keep their values.  The device stays usable.  One-shot; -1
 * clears.  Units of a CTA are numbered ceil(Nd/8) gradient chunks then one state unit per tile. */
int zero_test_inject_stall(int64_t unit);

/* ------------------------------------------------------------------ one GPU per rank */

/* The fused pass of zero_step (ZERO_FUSED) over the window [lo, hi) only, for a data-parallel
 * rank that owns that window ([P1] §二, [P3] core operations) when the Nd ranks are real GPUs:
 * st->grads[q] and st->params[q] are then the peer-mapped addresses of rank q's gradient and
 * weight buffers (e.g. symmetric memory), so the rank-order fan-in reads the peers' gradients over
 * NVLink and the bf16 results are stored straight into every peer's weight replica -- the
 * reduce-scatter, the update and the all-gather in one kernel over peer memory.  The fp32
 * state pointers are the rank's state indexed by global position (base + lo addresses its
 * first element).  finalize = 0 leaves the step open: the caller combines the pending
 * overflow flag (MAX) and sum of squares (SUM) of every rank in the workspace header (int32 at
 * byte 4, double at byte 8), then calls zero_end_step_flip and zero_repair_window; finalize != 0
 * ends the step here (single GPU) and, after an overflow, rewrites the window of every replica
 * from the unchanged state (a repair check launched after the pass).  No clipping (it needs the
 * global norm first).  Async. */
int zero_fused_window(int Nd, int64_t lo, int64_t hi, const zero_state_t *st,
                      const zero_hparams_t *hp, int finalize, void *stream);

/* zero_end_step for the fused path: ends the step and, if the combined overflow flag is clear,
 * makes the state copy written by the fused pass the live one.  Async. */
int zero_end_step_flip(void *ws, void *stream);

/* After an overflowed (skipped) step, rewrites the window [lo, hi) of every weight replica in
 * st->params from the unchanged live master weights; does nothing after a clean step.  Async. */
int zero_repair_window(int Nd, int64_t lo, int64_t hi, const zero_state_t *st, void *stream);

/* ------------------------------------------------------------------ ZeRO-Offload */

/* Buffers of an offloaded step ([P2] "ZeRO-Offload": optimizer state and gradients in CPU
 * memory, the CPU updates the state, the updated weights go back to the GPU).  Device: the Nd
 * gradient and weight replicas (N elements each), an fp32 staging buffer for the reduced
 * gradient and a bf16 staging buffer for the new weights (N elements each), the workspace.
 * Host: the fp32 master / exp_avg / exp_avg_sq (N elements each; any host memory), and pinned
 * (page-locked) fp32 gradient and bf16 weight buffers (N elements each) for the copies. */
typedef struct {
    int32_t grad_dtype;   /* ZERO_BF16 or ZERO_FP16 */
    int32_t host_threads; /* CPU threads for the host update (0: all hardware threads) */
    const uint16_t *grads[ZERO_MAX_ND];
    uint16_t *params[ZERO_MAX_ND];
    float *grad_dev;
    uint16_t *param_dev;
    float *grad_host;
    uint16_t *param_host;
    float *master_host;
    float *exp_avg_host;
    float *exp_avg_sq_host;
    void *workspace;
    void *upload_stream;  /* cudaStream_t for host->device copies and the fan-out (NULL: `stream`) */
} zero_offload_state_t;

/* AdamW on host memory (the CPU half of ZeRO-Offload).  For i < n, with g = grad[i] * clip_coef,
 * the rule of zero_adam_shard at step t (t >= 1: the update being made), in fp32 with the same
 * operation order, so results are bit-identical to the device kernels; param_out[i] =
 * bf16(master[i]) when param_out is not NULL.  clip_coef in (0, 1] (1: no clipping).  Runs
 * on `nthreads` CPU threads (0: all hardware threads) of a pool kept by the library; blocks
 * until done.  Host pointers only. */
int zero_host_adam(float *master, float *exp_avg, float *exp_avg_sq, const float *grad, int64_t n,
                   const zero_hparams_t *hp, int64_t t, float clip_coef, uint16_t *param_out,
                   int nthreads);

/* One ZeRO-Offload step (stages 1/2 arithmetic, state on the host).  In chunks of `chunk`
 * elements (0: one chunk): the device reduce-scatters the replicas into grad_dev (unscale,
 * overflow flag, sum of squares, dynamic loss scale as in zero_step) and copies each chunk to
 * grad_host on `stream`; once all chunks are reduced the call reads the overflow flag; unless it
 * is set, each chunk is updated on the CPU as soon as it has landed (zero_host_adam, with the
 * clipping factor of hp->max_grad_norm), copied to param_dev and fanned out to the Nd replicas
 * on upload_stream, so copies in both directions overlap the CPU work; finally `stream` waits
 * for the uploads and the step ends on the device (t, skip count, loss scale).  An overflow
 * skips the update: host state and replicas keep their values.  Blocks the calling thread for
 * the CPU part; device work stays queued on the streams. */
int zero_offload_step(int Nd, int64_t N, int64_t chunk, const zero_offload_state_t *st,
                      const zero_hparams_t *hp, void *stream);

/* ------------------------------------------------------------------ accounting (host only) */

/* Per-GPU model-state memory ([P1] §二 code: bytes_per_param for the 16-bit weights and again
 * for the gradients, bytes_per_opt_state for Adam's fp32 copy + m + v).  out[0] plain data
 * parallelism, out[1] ZeRO-1 (optimizer state / Nd), out[2] ZeRO-2 (also gradients / Nd),
 * out[3] ZeRO-3 (everything / Nd).  N >= 0, Nd >= 1, byte counts >= 0, else ZERO_EINVAL. */
int zero_memory_estimate(double N, int Nd, int bytes_per_param, int bytes_per_opt_state,
                         zero_mem_t out[4]);

/* Elements each rank sends per step with ring collectives ([P1] §二, §三; [P3] core
 * operations): stage 0 (plain data parallelism) and stages 1/2 send 2(Nd-1)/Nd*N, stage 3
 * 3(Nd-1)/Nd*N (1.5x).  Returns a negative value for a bad stage or Nd < 1. */
double zero_comm_volume(int stage, double N, int Nd);

#ifdef __cplusplus
}
#endif

#endif /* ZERO_H */
