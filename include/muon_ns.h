/*
 * muon_ns.h — C ABI of the B200 (sm_100a) Muon / NorMuon optimizer step.
 *
 * One optimizer step over a set of matrix parameters is four stream-ordered
 * calls:
 *
 *   muon_momentum_norm    momentum + Nesterov look-ahead + per-slice ||U||_F^2
 *   muon_ns_batched       quintic Newton-Schulz, standard form (symmetric
 *                         products computed on one triangle)
 *   muon_gram_ns_batched  quintic Newton-Schulz, Gram form (iterates on the
 *                         small m x m side)
 *   normuon_update        NorMuon per-row variance, normalization and
 *                         norm-preserving rescale (optional), then the
 *                         shape-scaled, decoupled-weight-decay update
 *
 * Sources (page titles):
 *   [dion-121]  microsoft/dion PR #121 "Fix convolution flattening in
 *               megabatches and NorMuon normalization"
 *   [mcore-lsm] Megatron-Core API docs, core.optimizer.layer_sharded_muon
 *   [ds-8437]   DeepSpeed issue #8437 "Muon under AutoTP orthogonalizes each
 *               shard, so the update depends on the TP degree"
 *
 * Data model.  A call takes an array of muon_batch.  A batch is N slices of
 * one shape [rows, cols] (rows = fan_out, cols = fan_in = prod of the
 * parameter's other dims), each slice a row-major matrix.  A megabatch of
 * stacked convolutions [N, out, in, kh, kw] is the batch [N, out, in*kh*kw]
 * ([dion-121] "Problem and fix"); per-head orthogonalization of a
 * head-blocked projection [H*d, cols] is the batch [H, d, cols] with
 * batch_stride d*ld ([ds-8437] "What could be done", option 3).  Every
 * slice is orthogonalized on its own.
 *
 * Ownership.  Every pointer in these structs is DEVICE memory owned by the
 * caller.  The library allocates nothing, frees nothing, keeps no state
 * between calls and does not synchronize the stream; all work is enqueued on
 * the given stream.  Scratch memory is the caller's workspace, sized by
 * muon_workspace_size.
 *
 * Streams and graphs.  A call enqueues only kernels on `stream`, launched
 * with programmatic stream serialization: each may start its prologue while
 * the previous kernel of the stream finishes and waits for it before
 * touching memory.  A whole step
 * can be captured in a CUDA graph; the first call on a device does one-time
 * set-up (kernel attributes, the driver's tensor-map encoder) and must run
 * before any capture on that device.  The set-up is redone when the device's
 * context changes (after cudaDeviceReset); that call, too, must come before
 * any capture.
 *
 * Errors.  Every argument is checked on the host before anything is
 * enqueued.  On any error the call returns a non-zero status and touches no
 * memory ("reject before mutating").  There is no fallback to another
 * precision or kernel.  Device-side waits are bounded: a kernel that waits
 * past its limit writes a non-zero word at workspace offset 0 and returns
 * (see muon_workspace_error).  Empty batches (n == 0, rows == 0 or
 * cols == 0) are accepted and enqueue nothing.
 *
 * Alignment.  Tensor-core operands are read by TMA: slice base pointers must
 * be 16-byte aligned and ld, batch_stride must be multiples of 16 bytes
 * (8 bf16 elements) for ns_in and ns_out; the workspace must be 256-byte
 * aligned.  Violations return MUON_MISALIGNED.
 */
#ifndef MUON_NS_H_
#define MUON_NS_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MUON_API __attribute__((visibility("default")))
#else
#define MUON_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MUON_OK = 0,
  MUON_INVALID_ARG = 1,        /* null pointer where one is required, bad count */
  MUON_BAD_SHAPE = 2,          /* ld < cols, overlapping slices, size limits */
  MUON_UNSUPPORTED_DTYPE = 3,  /* dtype not allowed for that tensor */
  MUON_MISALIGNED = 4,         /* 16-byte TMA rule or 256-byte workspace rule */
  MUON_WORKSPACE_TOO_SMALL = 5,
  MUON_CUDA_ERROR = 6,         /* a CUDA runtime call or launch failed */
  MUON_UNSUPPORTED_DEVICE = 7  /* current device is not sm_100 */
} muon_status;

typedef enum { MUON_F32 = 0, MUON_BF16 = 1, MUON_F16 = 2 } muon_dtype;

/* A strided view of the batch's N slices; element (s, i, j) is at
 * ptr + (s*batch_stride + i*ld + j) elements.  ld >= cols. */
typedef struct {
  void* ptr;
  int64_t ld;
  int64_t batch_stride;
  int32_t dtype;               /* muon_dtype */
  int32_t reserved;
} muon_view;

/* N same-shape slices and every per-slice buffer the step touches.
 * Which fields a call reads or writes is listed at each call. */
typedef struct {
  int64_t n;                   /* slices */
  int64_t rows;                /* fan_out of the slice */
  int64_t cols;                /* fan_in of the slice */
  muon_view grad;              /* G: f32 | bf16, read */
  muon_view momentum;          /* M: f32 | bf16, updated in place */
  muon_view ns_in;             /* U: bf16, the Newton-Schulz input */
  muon_view ns_out;            /* O: bf16, the Newton-Schulz output */
  muon_view weight;            /* W: f32 | bf16, updated in place */
  muon_view weight_copy;       /* optional bf16 copy of an f32 W (ptr NULL: none) */
  float* sumsq;                /* [n] f32: ||U||_F^2 per slice, or NULL */
  float* variance;             /* [n*rows] f32 NorMuon variance, slice-major; NULL without NorMuon */
  float* row_sumsq;            /* [n*rows] f32, slice-major, or NULL: the Newton-Schulz calls
                                  write sum_j O_ij^2 of each stored (bf16) output row here, and
                                  normuon_update takes the NorMuon row statistics from it instead
                                  of reading O a second time */
  int64_t fan_out;             /* the PARAMETER's fan_out = shape[0] and fan_in = prod(shape[1:])  */
  int64_t fan_in;              /* (not the slice's: a head or a megabatch slice takes the whole
                                  parameter's); they set the update's scale (muon_update_scale) */
} muon_batch;

/* Update scale modes ([mcore-lsm] LayerShardedMuon constructor: scale_mode,
 * default 'spectral', times extra_scale_factor).  See muon_update_scale. */
typedef enum { MUON_SCALE_SPECTRAL = 0, MUON_SCALE_RMS_NORM = 1 } muon_scale_mode;

/* Gram form: re-form the Gram matrix from the current iterate every this many
 * iterations (see muon_gram_ns_batched); 0 never. */
#define MUON_GRAM_RESTART_DEFAULT 3

/* Hyperparameters of one step ([mcore-lsm] LayerShardedMuon constructor). */
typedef struct {
  float mu;                    /* momentum, 0.95 */
  int32_t nesterov;            /* 1: U = G + mu*M_new; 0: U = M_new */
  float ns_eps;                /* Frobenius normalization: X0 = U / (||U||_F + ns_eps) */
  float a, b, c;               /* quintic coefficients (3.4445, -4.7750, 2.0315) */
  int32_t ns_steps;            /* iterations, 5; 1..16 */
  float beta2;                 /* NorMuon variance decay, 0.95 */
  float nor_eps;               /* NorMuon: O / (sqrt(v) + nor_eps) */
  float lr;                    /* learning rate */
  float weight_decay;          /* decoupled: W *= 1 - lr*weight_decay before the update */
  const float* abc_schedule;   /* optional HOST array [ns_steps][3] of per-iteration
                                  coefficients; NULL: (a, b, c) at every iteration */
  int32_t scale_mode;          /* muon_scale_mode of the update's shape factor */
  float extra_scale_factor;    /* multiplies the shape factor, 1.0 */
  int32_t gram_restart;        /* Gram form: restart period in iterations, 0 = none;
                                  MUON_GRAM_RESTART_DEFAULT (3) keeps rank-deficient inputs
                                  in band with fp16 m x m iterates */
  int32_t reserved;
} muon_hparams;

/* Bytes of workspace the given call needs for these batches.
 * which: 0 momentum_norm, 1 ns_batched, 2 gram_ns_batched, 3 normuon_update,
 * -1 the maximum over all four.  Returns 0 on invalid arguments. */
MUON_API size_t muon_workspace_size(const muon_batch* batches, int nb, int which);

/*
 * Momentum with Nesterov look-ahead and the squared Frobenius norm.
 * [mcore-lsm] LayerShardedMuon.step(): the elementwise momentum update
 * starts the step; momentum 0.95, nesterov=True.  [ds-8437] "Why it
 * happens": Newton-Schulz first normalizes by the matrix norm.
 *   M <- mu*M + G                   (stored in M's dtype, RN-even)
 *   U  = G + mu*M   (nesterov) or M  (stored to ns_in as bf16, RN-even)
 *   sumsq[s] = sum over slice s of bf16(U)^2   (deterministic order)
 * Reads grad, momentum; writes momentum, ns_in, sumsq (sumsq required).
 */
MUON_API muon_status muon_momentum_norm(const muon_batch* batches, int nb, const muon_hparams* hp,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Standard quintic Newton-Schulz of every slice, fp32 accumulation on the
 * tensor cores; X, A and B are stored in bf16 between products, or in fp16
 * for slices whose short side is at most 128 (the fused path below: with
 * 3 or 4 rows bf16 rounding alone can move the result past 3e-2 of the
 * exact one).  The output is bf16.
 * [ds-8437] "Why it happens": normalize, then iterate on X X^T.
 * [mcore-lsm] use_syrk: A = X X^T and B = b*A + c*A^2 are symmetric, one
 * triangle of each is computed.  Per iteration X <- a*X + B X.  A slice with
 * rows > cols is iterated transposed; the result O is in the slice's own
 * orientation.  X0 = U / (sqrt(sumsq) + ns_eps), with sumsq from
 * muon_momentum_norm when batch.sumsq is non-NULL, else computed here.
 * Batches whose slices have a short side <= 128 run every iteration in one
 * launch (a thread-block cluster per slice, X X^T summed across the cluster
 * in a fixed order): long side <= 2048 (or <= 4096 when not a multiple of 8)
 * with the slice held in shared memory, long side 2049..16384 and a multiple
 * of 8 with its columns streamed from L2 each iteration; tall slices go
 * through a transposed copy in the workspace.  The choice depends on the
 * shape only, so a slice's result does not depend on the rest of the batch.
 * When a call has both such batches and others, the fused batches run on a
 * second stream owned by the calling thread, forked from `stream` after the
 * call's first work and joined back into it before the call returns (event
 * record and wait: legal under stream capture); work enqueued on `stream`
 * afterwards is ordered after all of the call's work.
 * Reads ns_in (left unchanged), sumsq; writes ns_out, and row_sumsq when it
 * is non-NULL (per output row, the sum of squares of the stored bf16 values,
 * summed in a fixed order: tile partials from the last product's epilogue).
 * No batch's ns_out may share a byte with any batch's ns_in or with another
 * batch's ns_out (MUON_INVALID_ARG): ns_out also holds intermediate iterates.
 */
MUON_API muon_status muon_ns_batched(const muon_batch* batches, int nb, const muon_hparams* hp,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Gram Newton-Schulz: the same map iterated on the small side.
 * [ds-8437] "Measurement": the Gram kernel gives the standard kernel's
 * results.  With X0 the normalized slice (m <= n side first) and
 * G = X0 X0^T: A = G, Q = I; per iteration P = a*I + b*A + c*A^2,
 * Q <- P Q, A <- P A P; O = Q X0.  The m x m products use fp16 operands
 * (10-bit mantissa) with fp32 accumulation; X-side products use bf16.
 * Restarts (hp->gram_restart = R > 0): before iterations R, 2R, ... the
 * iterate X = Q X0 is formed (bf16) and the iteration starts again from it
 * (A = X X^T, Q = I).  In exact arithmetic nothing changes (X_k = Q_k X0 and
 * X_k X_k^T = Q_k G Q_k); in fp16, rounding can give A small negative
 * eigenvalues on rank-deficient slices, which A <- P A P amplifies by about
 * a^2 per iteration, and a restart bounds that growth.  Each restart costs
 * one X-sized product and one Gram product (3 m^2 n) and saves three m x m
 * products.
 * Small slices (as for muon_ns_batched) run in one launch: the cluster forms
 * G once (again at each restart) and every CTA iterates on the m x m side.
 * Reads ns_in (left unchanged), sumsq; writes ns_out and row_sumsq (as
 * muon_ns_batched).
 */
MUON_API muon_status muon_gram_ns_batched(const muon_batch* batches, int nb, const muon_hparams* hp,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Newton-Schulz with the form chosen per batch: the Gram form for slices whose
 * long side exceeds the short side by at least `gram_min_ratio` (n >= ratio*m),
 * the standard form otherwise.  By operation count the Gram form
 * (3m^2 n + 17m^3 with one-triangle products) is cheaper than the standard
 * form (5(3m^2 n + m^3)) exactly when n > m; square slices stay standard, the
 * form that keeps rank-deficient inputs in band.  gram_min_ratio <= 1 picks
 * the Gram form for every non-square slice; both forms compute the same map
 * ([ds-8437] "Measurement": the Gram and standard kernels agree).
 * Workspace: max of muon_workspace_size for which = 1 and 2.
 */
MUON_API muon_status muon_ns_auto_batched(const muon_batch* batches, int nb, const muon_hparams* hp,
                                          float gram_min_ratio, void* workspace, size_t workspace_bytes,
                                          cudaStream_t stream);

/*
 * NorMuon normalization and the weight update.
 * [dion-121] follow-on "What it does": one variance per output channel,
 * over the last dim of the flattened [N, out, prod(rest)] view;
 * "Compatibility": norm-preserving rescale, local to the slice.
 * [mcore-lsm] _apply_update: one multiply-add in fp32, one downcast on store.
 * With use_normuon:
 *   v_i <- beta2*v_i + (1-beta2) * mean_j O_ij^2           (per slice row i)
 *   Oh   = O_i / (sqrt(v_i) + nor_eps),  Oh *= ||O||_F / ||Oh||_F (0 stays 0)
 * else Oh = O.  Then W <- W*(1 - lr*weight_decay) - lr*scale*Oh, with
 * scale = muon_update_scale(fan_out, fan_in, hp->scale_mode,
 * hp->extra_scale_factor) of the batch's parameter, and weight_copy <- bf16(W)
 * when given.  With use_normuon and row_sumsq non-NULL, sum_j O_ij^2 is taken
 * from row_sumsq (as the preceding Newton-Schulz call wrote it) and O is read
 * once; a caller whose ns_out did not come from those calls passes NULL.
 * Reads ns_out, variance, row_sumsq; writes variance, weight, weight_copy.
 * MUON_INVALID_ARG if fan_out or fan_in < 1 or the scale mode is unknown.
 */
MUON_API muon_status normuon_update(const muon_batch* batches, int nb, const muon_hparams* hp,
                           int use_normuon, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream);

/*
 * muon_momentum_norm without a workspace argument.  The pages have no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory at the point where they run the step, such as code running
 * under a framework or runtime that owns all device memory and hands out
 * none after start-up, or a real-time or replay loop where allocation is
 * not permitted, and that have nowhere to keep a workspace between calls.
 *
 * It computes exactly what muon_momentum_norm computes (same kernels, same
 * arguments apart from the workspace) and keeps its per-chunk partial sums
 * in a scratch array of MUON_NOALLOC_SCRATCH_FLOATS floats (4 MiB) that the
 * library holds in static device memory on every GPU that loads it, until
 * the process exits.  Nothing is allocated or freed by the call.
 *
 * Limits and sharing:
 *  - the batches may hold at most MUON_NOALLOC_SCRATCH_FLOATS chunks of 8192
 *    elements in total (about 8.6e9 elements); larger calls return
 *    MUON_WORKSPACE_TOO_SMALL and enqueue nothing;
 *  - every call on a device uses the same array, so calls whose kernels can
 *    overlap on the GPU (different streams without ordering between them)
 *    race on it; calls ordered on one stream are safe.  Each call overwrites
 *    every partial it later reads, so nothing needs clearing between calls;
 *  - the first call on a device looks up the array's device address (a
 *    runtime query that does not allocate); make that first call before any
 *    stream capture on that device.
 */
#define MUON_NOALLOC_SCRATCH_FLOATS (1 << 20)
MUON_API muon_status muon_momentum_norm_noalloc(const muon_batch* batches, int nb, const muon_hparams* hp,
                                                cudaStream_t stream);

/* Reads the error word at workspace offset 0 after synchronizing the stream:
 * 0 = no device-side wait timed out since the word was last cleared (each
 * Newton-Schulz call clears it when it starts). */
MUON_API muon_status muon_workspace_error(const void* workspace, cudaStream_t stream, int32_t* error_word);

/*
 * Per-step coefficients for muon_hparams.abc_schedule: the Polar Express
 * schedule.  The pages name a "production Polar Express" schedule but give
 * no coefficients; this computes them by the greedy minimax construction of
 * Amsel, Persson, Musco and Gower, "The Polar Express: Optimal Matrix Sign
 * Methods and Their Application to the Muon Algorithm" (2025).  Step t
 * applies the odd quintic p_t(x) = a x + b x^3 + c x^5 minimizing
 * max |1 - p_t(x)| over the interval [lo_t, hi_t] that holds the singular
 * values of the normalized input after t steps: [lower, 1] for t = 0, then
 * the image of the previous interval under the polynomial applied.  With
 * safety s > 1 the polynomial applied is p_t(x / s) (coefficients a/s,
 * b/s^3, c/s^5); with bf16 Newton-Schulz use s of about 1.01: at s = 1 a
 * value rounded just past the top of the interval meets the steep side of
 * the polynomial and the result drifts (0.13 relative on a Gaussian
 * 128 x 1024 slice, against 0.02 at s = 1.01).
 *
 *   lower   : bound on the smallest normalized singular value, 0 < lower < 1
 *   steps   : 1 .. 16
 *   safety  : 1 <= safety <= 2
 *   abc_out : host array of 3 * steps floats, (a, b, c) per step
 *   err_out : optional host array of `steps` doubles: max |1 - p_t| over
 *             [lo_t, hi_t] of the polynomial applied at step t
 *
 * Host computation only (no device work, no GPU needed).  Returns
 * MUON_INVALID_ARG for arguments out of range and MUON_BAD_SHAPE if the
 * minimax solve fails; nothing is written then.
 */
MUON_API muon_status muon_polar_express_schedule(double lower, int steps, double safety, float* abc_out,
                                                 double* err_out);

/*
 * The update's shape factor of one parameter of shape [fan_out, fan_in]
 * (fan_in = prod of the other dims; [dion-121] review "Correctness —
 * confirmed": a single parameter's shape, never a slice's), times `extra`
 * ([mcore-lsm] extra_scale_factor):
 *   MUON_SCALE_SPECTRAL  sqrt(max(1, fan_out / fan_in))    ([mcore-lsm] default
 *                        'spectral'; the update's RMS-to-RMS operator norm is 1
 *                        when fan_out >= fan_in)
 *   MUON_SCALE_RMS_NORM  0.2 * sqrt(max(fan_out, fan_in))  (the pages name the
 *                        mode, [dion-121] adjust_lr_rms_norm, but not its formula;
 *                        this is the RMS matching of Liu et al., "Muon is Scalable
 *                        for LLM Training" (2025): an orthogonal update then has
 *                        element RMS 0.2, as AdamW's typically does)
 * Host computation (double precision, rounded once to float).
 * MUON_INVALID_ARG for fan_out or fan_in < 1, an unknown mode, a non-finite
 * extra, or a NULL scale_out.
 */
MUON_API muon_status muon_update_scale(int64_t fan_out, int64_t fan_in, int32_t scale_mode, float extra,
                                       float* scale_out);

MUON_API const char* muon_status_string(muon_status status);

/* Kernels this library has enqueued in this process so far (all devices,
 * all threads).  Instrumentation only: lets a caller count the launches of a
 * region without a profiler. */
MUON_API uint64_t muon_kernel_launches(void);

/* Library version, "major.minor.patch". */
MUON_API const char* muon_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MUON_NS_H_ */
