/*
 * muon.h — C ABI of libmuon, a B200 (sm_100a) implementation of the Muon
 * optimizer step for matrix parameters.
 *
 * Method: "Muon is Scalable for LLM Training" (Moonlight technical report,
 * Liu et al. 2025), Section 2:
 *   - Sec. 2.1, Eq. 1 and the paragraph after it: momentum M_t = mu M_{t-1} + G_t
 *     with M_0 = 0, and the Nesterov-style input Y = mu M_t + G_t;
 *   - Sec. 2.1, Eq. 2: Newton-Schulz on X_0 = Y / ||Y||_F with the quintic
 *     iteration X_k = a X + b (X X^T) X + c (X X^T)^2 X;
 *   - Sec. 2.2, Eq. 3 and Eq. 4 (= Sec. 3.1, Eq. 7): the decoupled, shape-scaled
 *     update W_t = W_{t-1} - eta (rms_scale sqrt(max(A,B)) O_t + lambda W_{t-1});
 *   - Sec. 2.3, Algorithm 1, last line: the logged update RMS sqrt(mean(u^2)).
 * Also: the other update scales of Sec. 3.1 (Eq. 5, Eq. 6), the AdamW step
 * of the parameters that are not matrices (Sec. 2.2), and the SVD-entropy
 * diagnostic of Sec. 3.4.
 *
 * Conventions for every entry point:
 *   - All tensors are dense, row-major, contiguous, and live in device memory
 *     of the device that is current when the plan is created.  "Host" arrays
 *     (descriptor lists, coefficient triples) are read before the call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously.  The status and profile
 *     reads synchronize the host, and say so.  A step or compute call whose
 *     device pointers differ from every table the plan keeps may first wait
 *     for the host-to-device copy of an older table to finish, because that
 *     copy reads the pinned buffer the new table is written to.
 *   - Arguments are validated on the host before anything is enqueued; an
 *     error return means nothing was launched and no tensor was modified.
 *   - A plan is not thread-safe: calls on one plan must be serialized by the
 *     caller and enqueued on streams that are ordered with each other.
 */
#ifndef MUON_H_
#define MUON_H_

#include <stddef.h>
#include <stdint.h>

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
  MUON_ERR_INVALID_ARG = 1,    /* null pointer, bad size, bad enum, non-finite hyper-parameter */
  MUON_ERR_SHAPE_MISMATCH = 2, /* descriptor count or shapes differ from the plan */
  MUON_ERR_UNSUPPORTED = 3,    /* request the plan was not built for (e.g. fp32 path without MUON_INIT_FP32_NS) */
  MUON_ERR_NO_MEMORY = 4,      /* device or pinned-host allocation failed in muon_init */
  MUON_ERR_CUDA = 5,           /* a CUDA call or launch failed */
  MUON_ERR_NONFINITE = 6,      /* (muon_get_status) a Frobenius norm was NaN or Inf */
  MUON_ERR_TIMEOUT = 7,        /* (muon_get_status) a device-side wait gave up; results of that call are invalid */
  MUON_ERR_ALIAS = 8,          /* W, G, M (or X_in, O_out) buffers overlap */
  MUON_ERR_NOT_CONVERGED = 9   /* reserved: an iteration hit its limit (the current solvers have none) */
} muon_status_t;

typedef enum { MUON_DT_BF16 = 0, MUON_DT_FP32 = 1 } muon_dtype_t;

/* Arithmetic of the Newton-Schulz products.
 *   MUON_NS_BF16: bf16 operands, fp32 accumulation on the tensor cores (tcgen05),
 *                 iterate X carried between iterations as a bf16 hi/lo pair
 *                 (about 16 significant bits).  The production path.
 *   MUON_NS_FP32: fp32 operands and fp32 products on the CUDA cores; a
 *                 validation path, needs MUON_INIT_FP32_NS at plan creation. */
typedef enum { MUON_NS_BF16 = 0, MUON_NS_FP32 = 1 } muon_ns_precision_t;

/* How the orthogonalised update O is scaled before it is applied ("Muon is
 * Scalable for LLM Training", Sec. 3.1, "Consistent update RMS", which
 * compares the three rules; the method itself uses the first).
 *   MUON_SCALE_MAX_DIM     rms_scale * sqrt(max(rows, cols))   Eq. 4 (= Eq. 7), the default
 *   MUON_SCALE_HIDDEN      rms_scale * sqrt(hidden_dim)        Eq. 5, "Baseline": one H for all
 *   MUON_SCALE_UPDATE_NORM rms_scale / RMS(O), 0 when O = 0    Eq. 6, "Update Norm": every
 *                          matrix's update has RMS exactly rms_scale.  Needs RMS(O) before any
 *                          weight changes, so the step adds one reduction pass over the last
 *                          iterate before the update pass. */
typedef enum { MUON_SCALE_MAX_DIM = 0, MUON_SCALE_HIDDEN = 1, MUON_SCALE_UPDATE_NORM = 2 } muon_scale_mode_t;

/* muon_init flags */
#define MUON_INIT_ZERO_MOMENTUM 0x1u /* zero every M on `stream` (M_0 = 0, Sec. 2.1) */
#define MUON_INIT_FP32_NS       0x2u /* also reserve the workspace of the fp32 path */
#define MUON_INIT_MAX_WORKSPACE 0x4u /* cap the plan's device memory (muon_init_ex only) */

/* One matrix parameter.  Shape [rows, cols]; for muon_init only the shape is
 * kept (pointers may be NULL unless MUON_INIT_ZERO_MOMENTUM is given), for
 * muon_step every pointer is used and may differ from call to call. */
typedef struct {
  float*      W;        /* fp32 [rows, cols], updated in place                     */
  const void* G;        /* gradient [rows, cols], dtype g_dtype, read only          */
  float*      M;        /* fp32 momentum [rows, cols], updated in place            */
  int64_t     rows;     /* A in Lemma 1; 1 <= rows <= 65536                         */
  int64_t     cols;     /* B in Lemma 1; 1 <= cols <= 65536                         */
  int32_t     g_dtype;  /* muon_dtype_t                                              */
  int32_t     reserved; /* must be 0                                                 */
} muon_param_t;

/* Per-call hyper-parameters (all finite). */
typedef struct {
  float   lr;            /* eta_t, the learning rate of this step (schedule is the caller's) */
  float   weight_decay;  /* lambda (Eq. 3)                                                     */
  float   momentum;      /* mu (Eq. 1)                                                         */
  int32_t ns_steps;      /* N, 0..32 (N = 0 gives O = Y / ||Y||_F)                              */
  float   a, b, c;       /* quintic coefficients of Eq. 2                                      */
  float   rms_scale;     /* the 0.2 of Eq. 4                                                   */
  int32_t nesterov;      /* 1: Newton-Schulz input mu M_t + G_t; 0: M_t (plain Eq. 1)          */
  int32_t ns_precision;  /* muon_ns_precision_t                                                */
  int32_t scale_mode;    /* muon_scale_mode_t                                                  */
  float   hidden_dim;    /* H of Eq. 5 (> 0 with MUON_SCALE_HIDDEN, ignored otherwise)          */
} muon_hparams_t;

typedef struct muon_plan_s* muon_plan_t;

/* Fill `hp` with the pages' values: lr 4.2e-4 (Sec. 3.3 peak), weight_decay 0.1
 * (Sec. 3.3), momentum 0.95, ns_steps 5 (Sec. 2.2), (a, b, c) =
 * (3.4445, -4.7750, 2.0315) (Sec. 2.1), rms_scale 0.2 (Eq. 4), nesterov 1,
 * ns_precision MUON_NS_BF16, scale_mode MUON_SCALE_MAX_DIM, hidden_dim 0.
 * Errors: MUON_ERR_INVALID_ARG if hp is NULL. */
MUON_API muon_status_t muon_hparams_default(muon_hparams_t* hp);

/* Build a plan for `n` matrices with the shapes in params[0..n).  The plan
 * owns its device workspace (see muon_workspace_bytes), tile and chunk
 * schedules and TMA descriptors; shapes and count are fixed for its lifetime.
 * With MUON_INIT_ZERO_MOMENTUM the M buffers are zeroed on `stream`.
 * The current CUDA device must be an sm_100 part.
 * Errors: INVALID_ARG (out/params NULL, n < 1, shape out of range, reserved != 0,
 * M NULL with ZERO_MOMENTUM, MUON_INIT_MAX_WORKSPACE without a budget: use
 * muon_init_ex), UNSUPPORTED (device is not sm_100), NO_MEMORY, CUDA.
 * On error *out is set to NULL and nothing is allocated. */
MUON_API muon_status_t muon_init(muon_plan_t* out, const muon_param_t* params, int32_t n, uint32_t flags,
                        void* stream);

/* muon_init with a cap on the plan's device memory.  With
 * MUON_INIT_MAX_WORKSPACE in `flags` (and only then) max_workspace_bytes > 0
 * bounds muon_workspace_bytes(plan): the matrices are packed, largest
 * Newton-Schulz work first, into waves whose iterate and Gram/polynomial
 * buffers are resident one wave at a time, and every call runs the waves one
 * after another on its stream (momentum and normalisation, the N iterations
 * and the update pass of one wave, then the next).  Each matrix's arithmetic
 * does not depend on the wave that holds it, so results are bitwise those of
 * an uncapped plan; only the launch count grows.  Without the flag
 * max_workspace_bytes must be 0 and the call equals muon_init (one wave).
 * For scale: 1624 matrices of an 8-layer, 64+2-expert MoE at hidden 2048
 * need about 41 GB uncapped; a cap trades that for more, smaller launches.
 * Errors: as muon_init, plus INVALID_ARG (flag and budget disagree) and
 * NO_MEMORY (the cap cannot hold the plan's fixed structures and the largest
 * matrix's buffers). */
MUON_API muon_status_t muon_init_ex(muon_plan_t* out, const muon_param_t* params, int32_t n, uint32_t flags,
                                    size_t max_workspace_bytes, void* stream);

/* Number of waves of the plan (1 unless capped); -1 for NULL. */
MUON_API int32_t muon_num_waves(muon_plan_t plan);

/* One Muon step over all n matrices of the plan (n and every shape must equal
 * the plan's):  M <- mu M + G;  Y = mu M + G (or M);  O = Newton-Schulz(Y) with
 * N = hp->ns_steps in the wide orientation (a matrix with rows > cols is
 * treated as its transpose; no data is transposed);  W <- W - lr (scale O +
 * weight_decay W) with scale rms_scale sqrt(max(rows, cols)) (Eq. 4), or as
 * hp->scale_mode selects.  A matrix whose Y is exactly 0 gets O = 0 (pure
 * weight decay).  If update_rms is not NULL it receives, on
 * the device, n floats sqrt(mean(O^2)) in descriptor order.
 * W, G, M of all descriptors must be pairwise disjoint.
 * The plan keeps the device copies of the last few distinct pointer tables,
 * so alternating between buffer sets (double-buffered gradients) issues no
 * copy once each set has been seen; after such a warm-up call a step
 * enqueues kernels only and can be captured in a CUDA graph.
 * Errors: INVALID_ARG, SHAPE_MISMATCH, ALIAS, UNSUPPORTED, CUDA.  Non-finite
 * norms and device-side timeouts are reported later by muon_get_status. */
MUON_API muon_status_t muon_step(muon_plan_t plan, const muon_param_t* params, int32_t n, const muon_hparams_t* hp,
                        float* update_rms, void* stream);

/* Newton-Schulz only (no momentum, no weight update) for all n matrices of
 * the plan: O_out[i] = Newton-Schulz(X_in[i]) with ns_steps iterations of
 * Eq. 2 and coefficients abc[0..2].  X_in[i] has the plan's i-th shape and
 * dtype in_dtype; O_out[i] is fp32 of the same shape.  X_in and O_out are
 * host arrays of n device pointers; no input may overlap an output.
 * Errors: INVALID_ARG, ALIAS, UNSUPPORTED, CUDA. */
MUON_API muon_status_t muon_orthogonalize(muon_plan_t plan, const void* const* X_in, float* const* O_out, int32_t n,
                                 int32_t in_dtype, int32_t ns_steps, const float abc[3], int32_t ns_precision,
                                 void* stream);

/* Device bytes owned by the plan (workspace, schedules, descriptors). 0 for NULL. */
MUON_API size_t muon_workspace_bytes(muon_plan_t plan);

/* Failure-detection test hook (host-side injection; nothing faults).  The
 * first Newton-Schulz launch of the next bf16-path muon_step or
 * muon_orthogonalize call on this plan makes one thread of every CTA wait on
 * a barrier that nothing arrives at, for at most wait_ns nanoseconds
 * (1 .. 10^9), before any operand load or tensor-core instruction is issued.
 * The wait runs out, the launch records MUON_ERR_TIMEOUT in the plan's status
 * and does no work, and the call's results are invalid, as after any
 * device-side timeout; later launches and calls run normally.  This exercises
 * the bounded device waits' error path: muon_get_status must report
 * MUON_ERR_TIMEOUT and the context must stay usable.
 * Errors: INVALID_ARG (NULL plan, wait_ns out of range). */
MUON_API muon_status_t muon_inject_wait_timeout(muon_plan_t plan, uint32_t wait_ns);

/* Synchronizes the plan's last stream, returns the sticky device status of all
 * calls since the previous muon_get_status (MUON_OK, MUON_ERR_TIMEOUT or
 * MUON_ERR_NONFINITE; TIMEOUT wins) and clears it.  CUDA errors: MUON_ERR_CUDA. */
MUON_API muon_status_t muon_get_status(muon_plan_t plan);

/* Release everything the plan owns.  Synchronizes the plan's last stream
 * first.  NULL is a no-op. */
MUON_API void muon_destroy(muon_plan_t plan);

/* Static English text for a status code (never NULL). */
MUON_API const char* muon_status_string(muon_status_t s);

/* Phase timing, for measurement.  Phases: 0 momentum/normalise, 1 Gram
 * (X X^T), 2 polynomial (b A + c A^2), 3 X update (a X + B X), 4 the update
 * pass over the last iterate (weight update or O output), the Eq. 6
 * reduction and the RMS finalisation, 5 Newton-Schulz (phases 1-3 together,
 * split-K reductions included).
 *
 * enable = MUON_PROFILE_LAUNCHES (1): every step/orthogonalize call records a
 * CUDA event on its stream after every launch; each launch's time goes to its
 * phase, and the product launches' time also to phase 5.
 * enable = MUON_PROFILE_SPANS (2): events only where the kernel class
 * changes (after the momentum pass, after the last product launch of each
 * wave, after each update pass).  Phases 1-3 then count launches but get no
 * time and phase 5 gets each wave's whole Newton-Schulz span.  The product
 * launches overlap by their set-up (programmatic dependent launch), which an
 * event between two of them prevents, so this mode times the chain as it
 * runs unprofiled.
 * enable = 0 stops recording.  Other values: MUON_ERR_INVALID_ARG. */
#define MUON_NUM_PHASES 6
#define MUON_PROFILE_LAUNCHES 1
#define MUON_PROFILE_SPANS 2
MUON_API muon_status_t muon_profile_enable(muon_plan_t plan, int32_t enable);

/* Synchronizes, then adds the elapsed milliseconds of every recorded call
 * since the last read into phase_ms[MUON_NUM_PHASES] and the launch counts
 * into launches[MUON_NUM_PHASES] (both zeroed by the caller), writes the
 * number of calls into *calls, and resets the record. */
MUON_API muon_status_t muon_profile_read(muon_plan_t plan, double* phase_ms, int64_t* launches, int32_t* calls);

/* Allocation-free Newton-Schulz of ONE matrix, for callers that cannot call
 * cudaMalloc (device memory owned by a framework allocator or a fixed budget,
 * or loops that must not allocate after start-up).  The paper has no
 * counterpart; this is a deployment convenience around the same kernels as
 * muon_orthogonalize on the bf16 tensor-core path.
 *   O_out = Newton-Schulz(X_in), ns_steps iterations with coefficients abc.
 *   X_in: device [rows, cols] in in_dtype; O_out: device fp32 [rows, cols];
 *   they must not overlap.  Limits: rows, cols <= 8192, rows * cols <= 2^20,
 *   min(rows, cols) <= 1024; larger requests return MUON_ERR_UNSUPPORTED.
 * No device memory is allocated or freed: all scratch lives in one static
 * device array of about 10.7 MB that every GPU loading this library holds
 * until the process exits.  The first call on a device resolves that array's
 * address (cudaGetSymbolAddress); make that first call before any stream
 * capture.  Each call copies its small descriptors (tile lists, TMA
 * descriptors) from pageable host memory, so it may wait on the host until
 * the driver has staged them; a call on a stream that is being captured
 * returns MUON_ERR_UNSUPPORTED and enqueues nothing.  Every call shares the
 * array: calls that can overlap on the GPU (different streams, or several
 * host threads) race and must be serialized by the caller.  Non-finite
 * inputs give non-finite outputs; no status is recorded.
 * Errors: INVALID_ARG, ALIAS, UNSUPPORTED, CUDA. */
MUON_API muon_status_t muon_orthogonalize_noalloc(const void* X_in, float* O_out, int64_t rows, int64_t cols,
                                                  int32_t in_dtype, int32_t ns_steps, const float abc[3],
                                                  void* stream);

/* ------------------------------------------------------------------------
 * Packing for data-parallel Muon ("Muon is Scalable for LLM Training",
 * Sec. 2.3, Algorithm 1): the gradients of many matrices go into one flat
 * buffer before the reduce-scatter, and the updated weights into and out of
 * the flat buffers of the all-gather.  A pack plan holds a fixed list of
 * segments; each run copies all of them in one launch (dst[k] = src[k],
 * converted between bf16 and fp32 with round-to-nearest-even when the dtypes
 * differ), so a step issues a constant number of launches whatever its
 * matrix count.  HBM-bound: source plus destination bytes per element.
 * ------------------------------------------------------------------------ */
typedef struct {
  const void* src;       /* device, numel elements of src_dtype                   */
  void*       dst;       /* device, numel elements of dst_dtype                   */
  int64_t     numel;     /* 1 <= numel <= 2^40                                    */
  int32_t     src_dtype; /* muon_dtype_t                                          */
  int32_t     dst_dtype; /* muon_dtype_t                                          */
} muon_segment_t;

typedef struct muon_pack_plan_s* muon_pack_plan_t;

/* Plan for n >= 1 segments on the current device (the pointers are kept;
 * the caller keeps the buffers alive).  Destinations must be pairwise
 * disjoint and no source may overlap a destination (sources may overlap each
 * other).  Uploads the segment table with a synchronous copy.
 * Errors: INVALID_ARG (NULL, bad count, size or dtype), ALIAS, NO_MEMORY, CUDA.
 * On error *out is NULL. */
MUON_API muon_status_t muon_pack_init(muon_pack_plan_t* out, const muon_segment_t* segs, int32_t n, void* stream);

/* Copy every segment of the plan, asynchronously on `stream` (one launch).
 * Errors: INVALID_ARG (NULL plan, or another device is current), CUDA. */
MUON_API muon_status_t muon_pack_run(muon_pack_plan_t plan, void* stream);

/* Waits for the plan's last stream and frees it; NULL is ignored. */
MUON_API void muon_pack_destroy(muon_pack_plan_t plan);

/* ------------------------------------------------------------------------
 * AdamW companion for the parameters that are not matrices.  The pages
 * update RMSNorm gains, the embedding and the LM head with AdamW, sharing the
 * learning rate and weight decay with Muon (Sec. 2.2, "Matching update RMS of
 * AdamW"; decay on the RMSNorm gains, Appendix D).  The algorithm is AdamW as
 * the pages cite it (Loshchilov and Hutter 2019), per element:
 *   m <- beta1 m + (1 - beta1) g;   v <- beta2 v + (1 - beta2) g^2
 *   P <- P - lr ( m / (1 - beta1^t) / (sqrt(v / (1 - beta2^t)) + eps) + wd P )
 * with wd = weight_decay for tensors with decay = 1 and 0 otherwise.  One
 * fused launch streams every tensor of the plan (fp32 arithmetic, about
 * 26 bytes of HBM traffic per element with a bf16 gradient).
 * ------------------------------------------------------------------------ */
typedef struct {
  float*      P;        /* fp32 parameter [numel], updated in place                      */
  const void* G;        /* gradient [numel], dtype g_dtype, read only                    */
  float*      m;        /* fp32 first moment [numel], updated in place                   */
  float*      v;        /* fp32 second moment [numel], updated in place                  */
  int64_t     numel;    /* 1 <= numel <= 2^31 - 1                                        */
  int32_t     g_dtype;  /* muon_dtype_t                                                   */
  int32_t     decay;    /* 1: decoupled weight decay on this tensor, 0: none             */
} muon_adamw_param_t;

typedef struct {
  float   lr;            /* eta_t, shared with Muon                                        */
  float   beta1, beta2;  /* moment decay rates, each in [0, 1) (not given by the pages)    */
  float   eps;           /* > 0                                                            */
  float   weight_decay;  /* lambda, shared with Muon                                       */
  int32_t step;          /* t >= 1 of this update, for the bias corrections                */
} muon_adamw_hparams_t;

typedef struct muon_adamw_plan_s* muon_adamw_plan_t;

/* lr 4.2e-4, beta1 0.9, beta2 0.95, eps 1e-8, weight_decay 0.1, step 1.
 * Errors: MUON_ERR_INVALID_ARG if hp is NULL. */
MUON_API muon_status_t muon_adamw_hparams_default(muon_adamw_hparams_t* hp);

/* Plan for a fixed list of n >= 1 tensors (only numel and g_dtype are kept;
 * MUON_INIT_ZERO_MOMENTUM zeroes every m and v on `stream`, the usual
 * m_0 = v_0 = 0).  Errors: INVALID_ARG, NO_MEMORY, CUDA, UNSUPPORTED (not an
 * sm_100 device). */
MUON_API muon_status_t muon_adamw_init(muon_adamw_plan_t* out, const muon_adamw_param_t* params, int32_t n,
                                       uint32_t flags, void* stream);

/* One AdamW step over every tensor, asynchronous on `stream`.  params must
 * match the plan (count, numel, g_dtype); P, m and v of all tensors and every
 * G must not overlap.  Validated before anything is enqueued: INVALID_ARG
 * (bad pointer, hyper-parameter or step), SHAPE_MISMATCH, ALIAS; launch
 * failures give MUON_ERR_CUDA. */
MUON_API muon_status_t muon_adamw_step(muon_adamw_plan_t plan, const muon_adamw_param_t* params, int32_t n,
                                       const muon_adamw_hparams_t* hp, void* stream);

/* Waits for the plan's last stream and frees it; NULL is ignored. */
MUON_API void muon_adamw_destroy(muon_adamw_plan_t plan);

/* ------------------------------------------------------------------------
 * SVD-entropy diagnostic ("Muon is Scalable for LLM Training", Sec. 3.4,
 * the SVD-entropy equation and Fig. 4).  For a weight matrix with singular
 * values sigma_1 .. sigma_n, n = min(rows, cols):
 *   H = -(1 / log n) sum_i p_i log p_i,   p_i = sigma_i^2 / sum_j sigma_j^2
 * with 0 log 0 = 0.  H is NaN for a zero matrix, for n = 1 (both 0 / 0) and
 * for a matrix with non-finite entries.
 * sigma_i^2 are the eigenvalues of the Gram matrix of the wide orientation,
 * formed in fp64 from the fp32 entries, reduced to tridiagonal form by
 * Householder reflections (fp64, one CTA per matrix) and found by bisection
 * on Sturm counts (fp64, to 2 eps of the largest); the entropy sums run in
 * fp64 too.
 * ------------------------------------------------------------------------ */
typedef struct muon_entropy_plan_s* muon_entropy_plan_t;

/* Plan for n >= 1 fp32 matrices: shapes[2 i] = rows, shapes[2 i + 1] = cols,
 * each >= 1 with rows * cols < 2^31.  min(rows, cols) <= 8192, else
 * MUON_ERR_UNSUPPORTED.  Allocates the fp64 Gram workspace (about 8 m^2 bytes
 * per matrix, m = min(rows, cols)) and a panel store of 512 m bytes per
 * matrix.  Errors:
 * INVALID_ARG, UNSUPPORTED, NO_MEMORY, CUDA. */
MUON_API muon_status_t muon_entropy_init(muon_entropy_plan_t* out, const int64_t* shapes, int32_t n, void* stream);

/* Entropy of every planned matrix, asynchronous on `stream`.
 * W[i]: device pointer to matrix i, fp32 row-major [rows, cols], read only
 *   (W is a host array of n device pointers).
 * H_out: device fp32 [n], H of each matrix.
 * sigma_out: NULL, or device fp32 [muon_entropy_num_singular_values(plan)]:
 *   the singular values of matrix i, descending, follow those of matrices
 *   0 .. i-1.
 * The outputs must not overlap the inputs or each other.  Everything is
 * validated before anything is enqueued: INVALID_ARG, SHAPE_MISMATCH,
 * ALIAS; launch failures give MUON_ERR_CUDA.  Results are bitwise
 * reproducible. */
MUON_API muon_status_t muon_entropy_compute(muon_entropy_plan_t plan, const float* const* W, int32_t n, float* H_out,
                                            float* sigma_out, void* stream);

/* Total number of singular values of the plan (sum of min(rows, cols)); -1 for NULL. */
MUON_API int64_t muon_entropy_num_singular_values(muon_entropy_plan_t plan);

/* CTAs per matrix of the plan's tridiagonal reduction (one thread-block
 * cluster per matrix: 16, 8, 4 or 2 when all the plan's clusters fit on the
 * GPU at once with one CTA per SM, else 1), chosen by muon_entropy_init;
 * -1 for NULL.  The partial dot products of a column are summed over the
 * cluster's CTAs in rank order, so results are bitwise reproducible for a
 * given plan and may differ in the last bits between plans whose cluster
 * sizes differ. */
MUON_API int32_t muon_entropy_cluster_size(muon_entropy_plan_t plan);

/* Synchronises the plan's last stream, then returns and clears the sticky
 * status of the calls since the previous read: MUON_OK or
 * MUON_ERR_NONFINITE (a matrix had non-finite entries; its H and singular
 * values are NaN).
 * computed_out: NULL or a host int32 array [n] that receives, for the last
 * call, 1 for each matrix whose eigenvalues were computed (one reduction and
 * bisection pass) and 0 for a non-finite one.
 * CUDA errors: MUON_ERR_CUDA. */
MUON_API muon_status_t muon_entropy_get_status(muon_entropy_plan_t plan, int32_t* computed_out);

/* Per-phase timing of the next calls with CUDA events when enable != 0.
 * ms_out: NULL, or a host double array [4] that receives the Gram,
 * tridiagonal reduction, bisection and entropy phase times of the last
 * profiled call (waits for its events; MUON_ERR_INVALID_ARG if no call was
 * profiled). */
MUON_API muon_status_t muon_entropy_profile(muon_entropy_plan_t plan, int32_t enable, double* ms_out);

/* Waits for the plan's last stream and frees it; NULL is ignored. */
MUON_API void muon_entropy_destroy(muon_entropy_plan_t plan);

#ifdef __cplusplus
}
#endif

#endif /* MUON_H_ */
