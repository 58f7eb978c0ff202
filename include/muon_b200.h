/*
 * muon_b200.h -- C ABI of the fused, batched Muon optimizer step and the
 * batched EMA pass for one NVIDIA B200 (sm_100a).
 *
 * What the calls compute (sources are parameter-golf competition pages):
 *  - muon_step_batched: for every matrix weight W (rows x cols, out x in) with
 *    bf16 gradient G and fp32 momentum M, one Muon step:
 *        M' = mu M + G ;  U = G + mu M'   (U = M' without Nesterov)
 *        U_i <- U_i / (||U_i|| + eps_row)            (MuonEq-R, stored rows)
 *        X = U^T if rows > cols else U ;  X <- X / (||X||_F + eps_frob)
 *        K times: A = X X^T ; B = b_k A + c_k A A ; X <- a_k X + B X
 *        O = X^T if transposed else X
 *        W' = W (1 - lr wd) - lr scale O
 *    PR #1584 "Record: Improved Parallel Residuals + Systems Optimization",
 *    section "Summary" (fused Muon kernel, batched EMA); PR #1396 "Record:
 *    Combined 3-Layer Recurrence + Parallel Residuals + Polar Express +
 *    Brotli", table "Techniques Combined" (Polar Express Newton-Schulz with
 *    4 minimax-optimal steps, MuonEq-R row-norm before NS, WD=0.105);
 *    PR #1893 "Record: L_ParallelResiduals_UNetSkips_DepthRecur_Muon_
 *    1.0901", table "Architecture and training stack", row "Optimizer".
 *    The pages name the steps but print no formulas; the formulas above are
 *    the readings this library implements.
 *  - ema_update_batched: E' = d E + (1 - d) P for every parameter tensor
 *    (PR #1893, same table, row "EMA": EMA_DECAY=0.9965).
 *  - muon_step_batched_sched: the Muon step with momentum and learning rate
 *    taken from linear ramps at a step number held in device memory (PR
 *    #1893, same table, row "Optimizer": momentum warm-up from 0.92 over 1500
 *    steps).
 *  - adamw_ema_batched: AdamW of the non-matrix tensors and the EMA of their
 *    new values in one pass (PR #1893, same table, row "Optimizer": AdamW on
 *    embeddings/scalars).
 *
 * Conventions for every call:
 *  - Pointers named device point to device memory; pointers to structs and
 *    arrays of pointers (mats, ema, params, numel, ns_coeffs, hyper) are
 *    HOST memory read during the call only.
 *  - The caller owns every buffer.  No call allocates device memory except
 *    muon_plan_create (a small table owned by the plan until
 *    muon_plan_destroy).
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and the calls return without synchronising, except
 *    muon_get_last_error (synchronises `stream`), muon_plan_timing_read and
 *    muon_plan_destroy (synchronise the device).
 *  - Argument, shape and alignment errors are detected on the host and
 *    returned before anything is enqueued.  A refused launch returns
 *    MUON_ERR_CUDA and nothing after it is enqueued (the call's earlier
 *    launches have run).  A device-side wait that exceeds its time limit (about one
 *    second) makes the kernel record an error word, drain its own copies and
 *    return; muon_get_last_error reports it as MUON_ERR_TIMEOUT.
 */
#ifndef MUON_B200_H
#define MUON_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MUON_OK = 0,
  MUON_ERR_INVALID_ARG = -1, /* null pointer, bad size, non-finite scalar   */
  MUON_ERR_UNSUPPORTED = -2, /* shape or step count beyond the plan         */
  MUON_ERR_ALIGNMENT = -3,   /* a device pointer is not 16-byte aligned      */
  MUON_ERR_CUDA = -4,        /* CUDA runtime/driver error (launch, encode)   */
  MUON_ERR_TIMEOUT = -5,     /* a device-side bounded wait ran out           */
  MUON_ERR_WORKSPACE = -6,   /* workspace null, too small or misaligned      */
  MUON_ERR_DEVICE_CHECK = -7 /* device-checked build: an index out of bounds */
} muon_status_t;

/* Opaque plan: matrix shapes, schedule tables and a small device table. */
typedef struct muon_plan muon_plan_t;

/* A cudaStream_t, passed as an untyped handle. */
typedef void *muon_stream_t;

/* One matrix of the batch.
 *  w          device, fp32, rows x cols row-major; read and updated in place.
 *  momentum   device, fp32, rows x cols row-major; read and updated in place.
 *  grad_bf16  device, bf16 bit patterns, rows x cols row-major; read only.
 *  update_out device, fp32, rows x cols row-major, or NULL.  When set it
 *             receives the orthogonalised update O (before lr and scale).
 *  rows, cols must equal the shape given to muon_plan_create.
 *  update_scale  multiplies lr for this matrix (e.g. sqrt(max(1, rows/cols))).
 *  All non-NULL pointers must be 16-byte aligned. */
typedef struct {
  float *w;
  float *momentum;
  const uint16_t *grad_bf16;
  float *update_out;
  int32_t rows;
  int32_t cols;
  float update_scale;
} muon_matrix_t;

/* Per-call scalars.  momentum in [0, 1); lr, weight_decay finite; eps_row,
 * eps_frob >= 0 (added to the norms); nesterov, eq_r are 0 or 1. */
typedef struct {
  float momentum;
  float lr;
  float weight_decay;
  float eps_row;
  float eps_frob;
  int32_t nesterov;
  int32_t eq_r;
} muon_hyper_t;

/* Builds a plan for n_mats matrices with the given (host) shapes, for up to
 * max_ns_steps Newton-Schulz steps per call.  Allocates the plan's device
 * table on the current device.  rows, cols >= 1; 1 <= n_mats <= 4096;
 * 0 <= max_ns_steps <= 16.  On success *out owns the plan. */
muon_status_t muon_plan_create(const int32_t *rows, const int32_t *cols,
                               int32_t n_mats, int32_t max_ns_steps,
                               muon_plan_t **out);

/* Bytes of device workspace muon_step_batched needs for this plan: two bf16
 * copies of every working matrix X (m x n), the bf16 A and B (m x m) of every
 * matrix, and per-row-block norm partials.  Returns 0 for a NULL plan. */
size_t muon_plan_workspace_bytes(const muon_plan_t *plan);

/* One Muon step over every matrix of the plan (the definition at the top of
 * this file).  mats: host array of n_mats entries in plan order.  ns_coeffs:
 * host array of ns_steps rows (a, b, c); ns_steps in [0, max_ns_steps]; with
 * 0 steps O is the normalised X.  workspace: device, >= workspace_bytes,
 * 256-byte aligned; its contents need not be initialised and are clobbered.
 * Calls on one plan must be ordered (one stream, or synchronised), because
 * the plan's device table and the workspace are shared.  A call is
 * deterministic: same inputs give bitwise-equal outputs. */
muon_status_t muon_step_batched(muon_plan_t *plan, const muon_matrix_t *mats,
                                const muon_hyper_t *hyper,
                                const float *ns_coeffs, int32_t ns_steps,
                                void *workspace, size_t workspace_bytes,
                                muon_stream_t stream);

/* A hyper-parameter that moves linearly from v0 at step t0 to v1 at step t1
 * and holds its end values outside [t0, t1] (t1 <= t0: v0 before t1, v1 from
 * t1 on).  Source: PR #1893 "Record: L_ParallelResiduals_UNetSkips_DepthRecur
 * _Muon_ 1.0901", table "Architecture and training stack", row "Optimizer":
 * Muon momentum 0.99 with a warm-up from 0.92 over 1500 steps, i.e.
 * {0.92, 0.99, 0, 1500}; the page gives the end points and the length, the
 * straight line between them is this library's reading. */
typedef struct {
  float v0;
  float v1;
  int32_t t0;
  int32_t t1;
} muon_ramp_t;

/* Momentum and learning rate of a scheduled step (both finite ramps; the
 * momentum ramp stays in [0, 1)). */
typedef struct {
  muon_ramp_t momentum;
  muon_ramp_t lr;
} muon_schedule_t;

/* muon_step_batched with the momentum and the learning rate taken on the
 * device from `sched` at the step number *step_dev (device int32, owned by
 * the caller, 4-byte aligned, 0 before the first step); the call advances
 * *step_dev by one on the device.  hyper->momentum and hyper->lr are
 * ignored.  Because nothing of the step number passes through the host, a
 * CUDA graph captured from one call (after one uncaptured call with the same
 * buffers and step count, see muon_step_batched) replays every later step
 * with the right schedule values.  Errors as muon_step_batched, plus
 * MUON_ERR_INVALID_ARG for a missing or non-finite schedule or step_dev, and
 * MUON_ERR_ALIGNMENT for a misaligned step_dev. */
muon_status_t muon_step_batched_sched(muon_plan_t *plan, const muon_matrix_t *mats,
                                      const muon_hyper_t *hyper,
                                      const muon_schedule_t *sched, int32_t *step_dev,
                                      const float *ns_coeffs, int32_t ns_steps,
                                      void *workspace, size_t workspace_bytes,
                                      muon_stream_t stream);

/* E' = decay E + (1 - decay) P for n_tensors tensors in one pass.
 *  ema     host array of device fp32 pointers (updated in place).
 *  params  host array of device fp32 pointers (read only).
 *  numel   host array of element counts (>= 0).
 *  Pointers need 4-byte alignment; 16-byte aligned tensors take the
 *  vectorised path.  An ema tensor must not overlap another tensor. */
muon_status_t ema_update_batched(float *const *ema, const float *const *params,
                                 const int64_t *numel, int32_t n_tensors,
                                 float decay, muon_stream_t stream);

/* AdamW settings of the non-matrix parameters.  Source: PR #1893 "Record:
 * L_ParallelResiduals_UNetSkips_DepthRecur_Muon_ 1.0901", table
 * "Architecture and training stack", row "Optimizer": AdamW on embeddings
 * and scalars (the page gives no setting; all are inputs).  lr, weight_decay
 * finite; beta1, beta2 in [0, 1); eps >= 0. */
typedef struct {
  float lr;
  float beta1;
  float beta2;
  float eps;
  float weight_decay;
} adamw_hyper_t;

/* One non-matrix tensor: device fp32 arrays of numel elements (numel >= 0).
 * param, exp_avg (first moment) and exp_avg_sq (second moment) are updated
 * in place, grad is read, ema (may be NULL: no EMA for this tensor) is
 * updated in place.  4-byte alignment required; when all five are 16-byte
 * aligned the tensor takes the vectorised path.  Arrays must not overlap. */
typedef struct {
  float *param;
  const float *grad;
  float *exp_avg;
  float *exp_avg_sq;
  float *ema;
  int64_t numel;
} adamw_tensor_t;

/* AdamW step of every tensor, then the EMA of the updated parameter, in one
 * pass over memory (the other optimizer of the training step, fused into the
 * EMA sweep):
 *   m' = b1 m + (1 - b1) g;  v' = b2 v + (1 - b2) g^2;
 *   p' = p (1 - lr wd) - lr (m' / (1 - b1^t)) / (sqrt(v' / (1 - b2^t)) + eps);
 *   e' = decay e + (1 - decay) p'.
 * t is `step` (>= 1) when step_dev is NULL; otherwise t = *step_dev + 1,
 * *step_dev (device int32, 4-byte aligned) counting the steps already taken,
 * and the call advances *step_dev by one after its kernels, so that a CUDA
 * graph captured from one call serves every step.  Use a counter of its own
 * (muon_step_batched_sched advances its counter too).  Asynchronous on
 * `stream`; argument errors are returned before anything is enqueued. */
muon_status_t adamw_ema_batched(const adamw_tensor_t *tensors, int32_t n_tensors,
                                const adamw_hyper_t *hyper, int32_t step,
                                int32_t *step_dev, float ema_decay,
                                muon_stream_t stream);

/* dst[i] = src[i] rounded to bf16 (nearest, ties to even), i < n: one pass
 * over device memory (src fp32, 4-byte aligned; dst bf16 bit patterns,
 * 2-byte aligned; 16-byte aligned arrays take the vectorised path).  For a
 * gradient reduced in fp32 across data-parallel ranks (PR #1893, table
 * "Architecture and training stack", row "Train context": 8-way training)
 * and handed to the Muon step, which reads bf16 gradients.  Asynchronous on
 * `stream`; MUON_ERR_INVALID_ARG for n < 0 or a NULL array with n > 0,
 * MUON_ERR_ALIGNMENT for misaligned arrays. */
muon_status_t muon_f32_to_bf16(uint16_t *dst, const float *src, int64_t n,
                               muon_stream_t stream);

/* Synchronises `stream`, reads and clears the plan's device error word.
 * Returns MUON_ERR_TIMEOUT if a kernel gave up on a bounded wait since the
 * last call, MUON_ERR_DEVICE_CHECK if a device check of the checked build
 * failed, MUON_ERR_CUDA on a CUDA error, MUON_OK otherwise. */
muon_status_t muon_get_last_error(muon_plan_t *plan, muon_stream_t stream);

/* Enqueues on `stream` a copy of the plan's device error word into
 * *host_word (host memory; pinned for the copy to be asynchronous) without
 * synchronising, for loops that check each step's status a step later.
 * Non-zero means a kernel gave up on a bounded wait (MUON_ERR_TIMEOUT); the
 * word stays set until muon_get_last_error reads and clears it.  Returns
 * MUON_ERR_INVALID_ARG for a NULL argument, MUON_ERR_CUDA if the copy cannot
 * be enqueued. */
muon_status_t muon_plan_error_async(const muon_plan_t *plan, int32_t *host_word,
                                    muon_stream_t stream);

/* Static description of a status code. */
const char *muon_status_string(muon_status_t status);

/* Frees the plan and its device table (synchronises the device first). */
void muon_plan_destroy(muon_plan_t *plan);

/* Per-kernel timing.  While enabled, muon_step_batched records CUDA events on
 * `stream` around each launch.  muon_plan_timing_read synchronises and
 * returns, per launch kind (see muon_kind_t), the number of launches and the
 * summed milliseconds since the last read, then resets the sums. */
typedef enum {
  MUON_KIND_PROLOGUE = 0, /* momentum + MuonEq-R + Frobenius partials      */
  MUON_KIND_GRAM = 1,     /* A = X X^T                                     */
  MUON_KIND_POLY = 2,     /* B = b A + c A A                               */
  MUON_KIND_APPLY = 3,    /* X <- a X + B X (and, last step, W update)     */
  MUON_KIND_FINAL = 4,    /* ns_steps == 0: W update from the normalised X */
  MUON_KIND_NS = 5,       /* all ns_steps Newton-Schulz steps, one launch:
                             gram, poly and apply tiles of every matrix and
                             step, and the weight update of the last step  */
  MUON_KIND_SCALE = 6,    /* per-matrix Frobenius scale from the partials  */
  MUON_KIND_COUNT = 7
} muon_kind_t;
muon_status_t muon_plan_set_timing(muon_plan_t *plan, int32_t enable);
muon_status_t muon_plan_timing_read(muon_plan_t *plan, int32_t *launches,
                                    double *ms, int32_t n_kinds);

/* Kernel launches of one call with ns_steps steps (for launch accounting):
 * muon_step_launches counts a plan whose rows all take the same prologue
 * kernel (one-pass: row length a multiple of 8 and at most 8192; two-pass
 * otherwise); muon_plan_step_launches counts the given plan exactly (0 for
 * a null plan or negative ns_steps). */
int32_t muon_step_launches(int32_t ns_steps);
int32_t muon_plan_step_launches(const muon_plan_t *plan, int32_t ns_steps);
int32_t ema_update_launches(int32_t n_tensors);
/* Launches of adamw_ema_batched (with_step_dev: 1 if a device counter is
 * advanced). */
int32_t adamw_ema_launches(int32_t n_tensors, int32_t with_step_dev);

/* 1 if this library is the device-checked build (compiled with
 * MUON_DEVICE_CHECKS): every work item the kernels decode is checked
 * against its matrix's tile grid and every epilogue store against its
 * buffer before the access; a failure skips the access, records the error
 * word and the offending index, stops the tensor-core kernel like a failed
 * wait, and muon_get_last_error returns MUON_ERR_DEVICE_CHECK.  0 for the
 * default build, which carries none of these checks. */
int32_t muon_device_checks(void);

/* Test hooks.  Fault 1 makes the tensor-core kernel's load warp skip one
 * stage of its first tile in block 0, so that the consumer's bounded wait
 * runs out and the timeout path is exercised (MUON_ERR_TIMEOUT from
 * muon_get_last_error).  Fault 2 asks for more dynamic shared memory than the
 * tensor-core kernel was set up for, so that the runtime refuses its launch
 * and the step call returns MUON_ERR_CUDA (no kernel of it runs; the earlier
 * launches of the call do).  Fault 3, accepted only by the device-checked
 * build (MUON_ERR_UNSUPPORTED otherwise), uploads the work list with its
 * last item moved outside its matrix, which the kernel's checks must catch.
 * 0 turns them off. */
muon_status_t muon_plan_set_fault(muon_plan_t *plan, int32_t fault);

/* ABI version (major * 100 + minor). */
int32_t muon_abi_version(void);

/* Number of device allocations (cudaMalloc) this library has made in the
 * process so far: one per muon_plan_create, none in any other call.  Lets a
 * caller check that a code path allocated nothing. */
int64_t muon_device_allocation_count(void);

/* ---- One batched step without any device allocation ----------------------
 * The pages have no counterpart to this call.  It is for callers that cannot
 * allocate device memory: a framework that owns every device allocation
 * through its own pool and hands a plug-in only its inputs and outputs, or a
 * latency-critical loop that forbids cudaMalloc after start-up (cudaMalloc
 * can synchronise the device and stall other streams).  Such a caller can
 * neither create a plan (muon_plan_create allocates the plan's table) nor
 * provide a workspace.
 *
 * It computes the same step as muon_step_batched on the same kernels.  Its
 * scratch -- the per-matrix table with the TMA descriptors, the work and tile
 * lists, the error word, X, A, B' and the norm partials -- lives in one
 * file-scope device array of MUON_NOALLOC_SCRATCH_BYTES, which every device
 * that loads this library's kernels holds until the process exits.
 *  mats: host array of n_mats matrices (1 <= n_mats <= MUON_NOALLOC_MAX_MATS),
 *        same rules as muon_step_batched; ns_steps in [0, 16].
 *  Returns MUON_ERR_WORKSPACE if the batch needs more scratch than the array
 *  holds (the array fits, e.g., one 11L x 512d layer or any single matrix
 *  up to 1024 x 4096), MUON_ERR_UNSUPPORTED beyond the count limits.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) and sets kernel attributes; make that first call
 * before any stream capture.  Every call re-uploads its tables with
 * cudaMemcpyAsync from pageable host memory (so it cannot be captured), clears
 * the error word with cudaMemsetAsync, and calls no cudaMalloc, cudaFree or
 * other allocating routine.  All calls share the one array: calls that overlap
 * on the GPU (different streams, or different host threads without ordering)
 * race on it; order them on one stream.  A device-side wait that runs out
 * (the step then stops early and leaves W and the momentum partly updated)
 * sets the array's error word, which each call clears at its start and
 * muon_noalloc_error_async reads back.  A refused launch returns
 * MUON_ERR_CUDA at once and enqueues nothing after it. */
#define MUON_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
#define MUON_NOALLOC_MAX_MATS 64
muon_status_t muon_step_batched_noalloc(const muon_matrix_t *mats,
                                        int32_t n_mats,
                                        const muon_hyper_t *hyper,
                                        const float *ns_coeffs,
                                        int32_t ns_steps,
                                        muon_stream_t stream);

/* Enqueues on `stream` a copy of the allocation-free path's error word (of
 * the current device) into *host_word (host memory; pinned for the copy to
 * be asynchronous), without synchronising and without allocating.  Read it
 * after the stream has passed this point: non-zero means a kernel of the last
 * muon_step_batched_noalloc call enqueued before it gave up on a bounded wait
 * (that step is incomplete).  Returns MUON_ERR_INVALID_ARG for a NULL
 * host_word, MUON_ERR_CUDA if the copy cannot be enqueued.  The pages have
 * no counterpart to this call either. */
muon_status_t muon_noalloc_error_async(int32_t *host_word, muon_stream_t stream);

/* Test hook of the allocation-free path, process-wide: the faults of
 * muon_plan_set_fault (1: a bounded wait runs out; 2: the tensor-core
 * kernel's launch is refused) for later muon_step_batched_noalloc calls; 0
 * turns it off. */
muon_status_t muon_noalloc_set_fault(int32_t fault);

#ifdef __cplusplus
}
#endif

#endif /* MUON_B200_H */
