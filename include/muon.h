/*
 * muon.h -- C ABI of the B200 (sm_100a) Muon optimizer step.
 *
 * The operation, by source:
 *
 *   "Muon: An optimizer for the hidden layers of neural networks" (README of
 *   the KellerJordan/Muon repository), sections "Usage" and "Hyperparameter
 *   tuning": hidden 2-D weights are stepped by Muon (lr 0.02, weight decay
 *   0.01, momentum 0.95, Nesterov, 5 Newton-Schulz steps); every other
 *   parameter by AdamW (lr 3e-4, betas (0.9, 0.95), weight decay 0.01).
 *
 *   "Muon: when the LLM optimizer treats weight matrices as matrices" (blog),
 *   section 3: X = G / ||G||_F, then X <- a X + b (X X^T) X + c (X X^T)^2 X
 *   with a, b, c = 3.4445, -4.7750, 2.0315; PyTorch set-up after section 4:
 *   shape-dependent scaling conventions and decoupled weight decay.
 *
 *   "The Newton-Muon Optimizer" (README of zhehangdu/Newton-Muon), section
 *   "What Is Newton-Muon?": the gradient is right-multiplied by an inverse
 *   activation second moment S^-1 (one d x d estimate, or four d x d blocks
 *   for the MLP contraction) before the standard Muon step.
 *
 * Conventions for every entry point:
 *
 *   - Tensors are caller-owned, contiguous, row-major, on the device the
 *     context was created for, and 16-byte aligned.  Arrays of tensor
 *     pointers (the `weights`, `grads`, ... fields) are HOST arrays whose
 *     elements are DEVICE pointers.  Descriptor structs are read on the host
 *     during the call only; nothing is retained after the call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued on it asynchronously; a call returns before
 *     the GPU finishes.  Calls sharing one context must be ordered (one
 *     stream, or externally synchronised streams): the context's workspace
 *     and descriptor tables are reused from call to call.
 *   - Errors are status codes; nothing throws across the ABI.  Argument
 *     errors are detected on the host before anything is enqueued and leave
 *     every tensor untouched.  muon_last_error() then describes the error.
 *     CUDA errors of earlier asynchronous work surface as MUON_ERR_CUDA on a
 *     later call.  A kernel whose internal wait runs past its limit records
 *     MUON_ERR_TIMEOUT in a device flag read by muon_check_device().
 */
#ifndef MUON_B200_H
#define MUON_B200_H

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
  MUON_ERR_INVALID_ARG = 1,   /* bad shape, count, pointer, alignment or hyper-parameter */
  MUON_ERR_UNSUPPORTED = 2,   /* valid request this build does not implement */
  MUON_ERR_WORKSPACE = 3,     /* a caller-given workspace is too small for one matrix */
  MUON_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed (also earlier async faults) */
  MUON_ERR_NONFINITE = 5,     /* check_finite was set and a gradient held NaN/Inf */
  MUON_ERR_TIMEOUT = 6        /* a bounded device-side wait gave up */
} muon_status;

typedef enum { MUON_F32 = 0, MUON_BF16 = 1 } muon_dtype;

/* Shape-dependent factor multiplying the learning rate (blog, PyTorch
 * set-up after section 4).  ORIGINAL: max(1, rows/cols)^0.5, the convention
 * of the first page's lr 0.02.  MATCH_RMS_ADAMW: 0.2 * sqrt(max(rows, cols)).
 * NONE: 1. */
typedef enum {
  MUON_SCALE_ORIGINAL = 0,
  MUON_SCALE_MATCH_RMS_ADAMW = 1,
  MUON_SCALE_NONE = 2
} muon_scale_mode;

/* Hyper-parameters of one Muon step; muon_default_hparams() fills the
 * sources' defaults.  momentum in [0, 1); ns_steps >= 0; eps > 0 guards the
 * Frobenius normalisation; check_finite != 0 scans the gradients first and,
 * when one holds NaN/Inf, leaves every weight and momentum buffer untouched
 * and returns MUON_ERR_NONFINITE (this synchronises the stream). */
typedef struct {
  float lr;
  float momentum;
  float weight_decay;
  float eps;
  float ns_a, ns_b, ns_c;
  int32_t nesterov;
  int32_t ns_steps;
  int32_t scale_mode;   /* muon_scale_mode */
  int32_t check_finite;
} muon_hparams;

/* A group of `count` hidden weights of one shape rows x cols.
 *   weights[i]   fp32 rows x cols, updated in place.
 *   grads[i]     grad_dtype rows x cols, read only.
 *   momentum[i]  fp32 rows x cols, updated in place (EMA convention:
 *                buf <- beta buf + (1 - beta) g).
 *   update_out   optional (NULL = off): update_out[i] receives the
 *                orthogonalised update O (fp32 rows x cols) before scale and
 *                learning rate, for inspection and staged checking.
 *   precond      optional (NULL = plain Muon): precond[i] points at
 *                precond_blocks consecutive fp32 d x d matrices S_b^-1,
 *                d = cols / precond_blocks; the gradient is right-multiplied
 *                block-diagonally by them before momentum (Newton-Muon).
 *                Several matrices may share one S^-1 (the shared QKV
 *                estimate).  Requires grad_dtype == MUON_BF16.
 *   precond_split  optional (NULL = off; only read with precond, by
 *                muon_step): precond_split[i] is the bf16 high/low split of
 *                precond[i] that muon_newton_refresh wrote to an activation's
 *                s_inv_split (layout there), 16-byte aligned.  The step then
 *                uses it instead of splitting precond[i] again; the caller
 *                keeps the two consistent (both written by the same
 *                refresh).  Individual entries may be NULL. */
typedef struct {
  int64_t rows;
  int64_t cols;
  int32_t count;
  int32_t grad_dtype;              /* muon_dtype */
  float* const* weights;
  const void* const* grads;
  float* const* momentum;
  float* const* update_out;
  const float* const* precond;
  int32_t precond_blocks;
  int32_t reserved;
  const void* const* precond_split;
} muon_group;

/* Newton-Schulz only: outputs[i] (fp32 rows x cols) = NS(inputs[i]). */
typedef struct {
  int64_t rows;
  int64_t cols;
  int32_t count;
  int32_t in_dtype;                /* muon_dtype */
  const void* const* inputs;
  float* const* outputs;
} muon_ns_group;

/* One non-2-D parameter for the aux AdamW step; all buffers have numel
 * elements. */
typedef struct {
  int64_t numel;
  int32_t grad_dtype;              /* muon_dtype */
  int32_t reserved;
  float* param;
  const void* grad;
  float* exp_avg;
  float* exp_avg_sq;
} muon_adamw_tensor;

typedef struct {
  float lr, beta1, beta2, eps, weight_decay;
} muon_adamw_hparams;

/* One activation matrix feeding a Newton-Muon refresh: acts is tokens x
 * width (act_dtype), split into nblocks column blocks of d = width / nblocks;
 * s_inv receives nblocks consecutive fp32 d x d matrices
 * (X_b^T X_b / tokens + damping I)^-1.  s_inv_split, optional (NULL = off,
 * 16-byte aligned), receives their bf16 high/low split for the tensor-core
 * preconditioning: per block, S_hi = bf16(S^-1) as d rows of d, then S_lo =
 * bf16(S^-1 - S_hi) as d more rows (nblocks * 2d * d bf16 in all); pass it to
 * muon_step as the group's precond_split so that steps until the next
 * refresh do not split S^-1 again. */
typedef struct {
  const void* acts;
  int32_t act_dtype;               /* muon_dtype: MUON_BF16 or MUON_F32 */
  int32_t nblocks;
  int64_t tokens;
  int64_t width;
  float* s_inv;
  void* s_inv_split;
} muon_act_desc;

typedef struct muon_ctx muon_ctx;

/* Source: "Muon: An optimizer for the hidden layers of neural networks",
 * sections "Usage" and "Hyperparameter tuning" (lr 0.02, momentum 0.95,
 * weight decay 0.01, Nesterov, 5 steps); "Muon: when the LLM optimizer
 * treats weight matrices as matrices", section 3 (a b c = 3.4445 -4.7750
 * 2.0315).  Fills *hp with those defaults, eps 1e-7 and the ORIGINAL scale;
 * hp NULL: no effect. */
MUON_API void muon_default_hparams(muon_hparams* hp);
/* Source: "Muon: An optimizer for the hidden layers of neural networks",
 * section "Usage" (AdamW for the non-hidden parameters: lr 3e-4, betas 0.9 /
 * 0.95, weight decay 0.01).  Fills *hp with those and eps 1e-8. */
MUON_API void muon_default_adamw_hparams(muon_adamw_hparams* hp);

/* Source: "Muon: An optimizer for the hidden layers of neural networks",
 * section "Usage" (the optimizer is constructed once over the parameter
 * groups and stepped every iteration); the context is that optimizer's
 * device-side state.
 * Create a context on CUDA device `device`.  workspace_bytes == 0: the
 * library allocates and grows its own workspace as needed.  Otherwise the
 * library allocates exactly that much once and splits larger requests into
 * chunks that fit; a single matrix that does not fit returns
 * MUON_ERR_WORKSPACE.  *ctx is NULL on failure.  Errors: ctx NULL or a bad
 * device -> MUON_ERR_INVALID_ARG; a device that is not sm_100 ->
 * MUON_ERR_UNSUPPORTED; a failed CUDA call -> MUON_ERR_CUDA. */
MUON_API muon_status muon_init(muon_ctx** ctx, int device, size_t workspace_bytes);

/* No counterpart on the pages (resource management).  Release the context,
 * its workspace and tables (synchronises the device).  NULL: no effect. */
MUON_API void muon_destroy(muon_ctx* ctx);

/* No counterpart on the pages (error reporting).  Human-readable
 * description of the context's last error ("" if none); the string is owned
 * by the context and valid until its next call. */
MUON_API const char* muon_last_error(const muon_ctx* ctx);
/* No counterpart on the pages (error reporting).  Static name of a status
 * code ("MUON_OK", ...). */
MUON_API const char* muon_status_string(muon_status s);

/* No counterpart on the pages (memory planning).  Workspace bytes a
 * muon_step / muon_orthogonalize over these groups needs to run in one
 * chunk, written to *bytes; host only.  Errors as muon_step's argument
 * checks. */
MUON_API muon_status muon_query_workspace(const muon_group* groups, int32_t ngroups, size_t* bytes);

/* No counterpart on the pages (memory planning).
 * Hand the context a caller-owned device workspace (e.g. a torch tensor).
 * It is used instead of the library's own until replaced; the caller keeps
 * it alive and unmodified while work enqueued with it may run.  ptr must be
 * 256-byte aligned.  ptr == NULL returns to library-owned workspace. */
MUON_API muon_status muon_set_workspace(muon_ctx* ctx, void* ptr, size_t bytes);

/* Source: "Muon: An optimizer for the hidden layers of neural networks",
 * sections "Usage" and "Hyperparameter tuning"; "Muon: when the LLM
 * optimizer treats weight matrices as matrices", section 1 (the moving-
 * average form of momentum), section 3 (Frobenius normalisation and the
 * quintic iteration in bf16) and the PyTorch set-up after section 4 (shape
 * scale, decoupled weight decay).
 * One Muon step over ngroups groups: for every matrix, Nesterov momentum,
 * Frobenius normalisation, hp->ns_steps quintic Newton-Schulz iterations in
 * bf16 with fp32 accumulation (on the transpose when rows > cols), then
 * W <- W (1 - lr wd) - lr scale O.
 *
 * When no group asks for update_out and every width is a multiple of 4, the
 * weight step is applied inside the last Newton-Schulz product, with O in
 * fp32 (never rounded to bf16 or written out); otherwise O is the bf16
 * result of the last product, written to update_out when requested and
 * applied by a separate pass.  Both agree to bf16 rounding of O.
 *
 * The kernels are enqueued on `stream` (NULL: the legacy default stream)
 * with programmatic stream serialization: each may be scheduled while its
 * predecessor drains and waits for it (griddepcontrol.wait) before touching
 * global memory, so stream order holds as for ordinary launches. */
MUON_API muon_status muon_step(muon_ctx* ctx, const muon_group* groups, int32_t ngroups,
                      const muon_hparams* hp, void* stream);

/* Source: "Muon: when the LLM optimizer treats weight matrices as
 * matrices", section 3 (X = G / ||G||_F, then the quintic iteration).
 * Frobenius normalisation plus hp->ns_steps Newton-Schulz iterations only
 * (uses hp->eps, ns_a/b/c, ns_steps): outputs[i] (fp32) = NS(inputs[i]),
 * computed as in muon_step.  Errors as muon_step. */
MUON_API muon_status muon_orthogonalize(muon_ctx* ctx, const muon_ns_group* groups, int32_t ngroups,
                               const muon_hparams* hp, void* stream);

/* Source: "Muon: An optimizer for the hidden layers of neural networks",
 * section "Usage" (every parameter that is not a hidden 2-D weight goes to
 * AdamW); "Muon: when the LLM optimizer treats weight matrices as
 * matrices", section 1 (the first and second moments).  Bias-corrected
 * AdamW with decoupled weight decay over n tensors, in place on param,
 * exp_avg, exp_avg_sq; step counts from 1.  Errors: step < 1, betas outside
 * [0, 1), eps <= 0, NULL pointers -> MUON_ERR_INVALID_ARG, before any
 * launch. */
MUON_API muon_status muon_adamw_step(muon_ctx* ctx, const muon_adamw_tensor* tensors, int32_t n,
                            const muon_adamw_hparams* hp, int64_t step, void* stream);

/* Source: "The Newton-Muon Optimizer", section "What Is Newton-Muon?" (the
 * refresh half of the refresh/apply step: the activation second moment,
 * one d x d estimate per layer input, four d x d blocks for the MLP
 * contraction, and its inverse).
 * For each descriptor, S_b = X_b^T X_b / tokens (+ damping I) of every
 * d-wide column block b and S_b^-1 (fp32 Cholesky, fp32 inverse) into
 * s_inv.  The signature takes an array of activation descriptors and one
 * damping instead of a single activation, so that every layer input of a
 * model refreshes in one call and same-shape blocks share one batched
 * second-moment launch.  bf16 activations are read in place when every
 * width and block width is a multiple of 8 (else through transposed
 * copies); fp32 activations are split into bf16 high and low parts whose
 * three significant cross products are accumulated in fp32.  Errors: NULL
 * or unaligned pointers, a bad shape, damping < 0 -> MUON_ERR_INVALID_ARG;
 * a block width above 4096 -> MUON_ERR_UNSUPPORTED; all before any launch.
 * A second moment that is not positive definite is reported by
 * muon_check_device(). */
MUON_API muon_status muon_newton_refresh(muon_ctx* ctx, const muon_act_desc* acts, int32_t n,
                                float damping, void* stream);

/* Source: "The Newton-Muon Optimizer", section "What Is Newton-Muon?".
 * Newton-Muon right-preconditioning on its own ("What Is Newton-Muon?",
 * the update rule with the gradient replaced by G S^-1, block-diagonal over
 * precond_blocks column blocks): for every matrix of every group,
 *   update_out[i] (fp32 rows x cols) = grads[i] [S_1^-1, ..., S_nb^-1]
 * with S_b^-1 = precond[i] + b d d (fp32 d x d, row-major, d = cols / nb).
 * Each group needs grads (MUON_BF16), precond, precond_blocks and
 * update_out; weights and momentum are ignored and may be NULL.  muon_step
 * does the same product internally when a group carries precond; this call
 * exposes it for callers that precondition and orthogonalise in separate
 * stages.  Block widths that are multiples of 64 run on the tensor cores
 * (S^-1 split into bf16 hi + lo, G in bf16, fp32 accumulation); others on an
 * fp32 tile kernel.  The tensor cores read G in place; each distinct S^-1
 * is split once into bf16 hi/lo stacks in workspace (nb x 2 d^2 x 2 bytes,
 * 256-byte aligned), in batches that fit a capped or caller-owned
 * workspace; MUON_ERR_WORKSPACE if one S^-1 does not fit.  Argument errors
 * are reported before any launch. */
MUON_API muon_status muon_newton_precondition(muon_ctx* ctx, const muon_group* groups, int32_t ngroups,
                                     void* stream);

/* No counterpart on the pages (failure detection).
 * Failure-detection self test: enqueues one kernel whose single bounded
 * wait (an mbarrier that nothing completes) runs out after its 2 s limit,
 * records the timeout in the context's device flags and returns; nothing
 * faults or hangs and the context stays usable.  The next
 * muon_check_device() returns MUON_ERR_TIMEOUT and clears the flag. */
MUON_API muon_status muon_selftest_wait(muon_ctx* ctx, void* stream);

/* No counterpart on the pages (failure detection).
 * Failure-detection self test of the Newton-Schulz engine: one Gram launch
 * (a single tile of a zero 256 x 640 matrix in the context's workspace)
 * whose MMA thread takes the operand stages but never issues a product or
 * releases a stage.  The TMA producer, the MMA thread and the epilogue warps
 * of both CTAs of the pair each give up after their 2 s limit, run their
 * abort sequence (let issued copies land, release TMEM after the cluster
 * barrier) and return; nothing faults or hangs.  The next
 * muon_check_device() returns MUON_ERR_TIMEOUT and clears the flag; the
 * context stays usable.  Needs 458752 bytes of workspace
 * (MUON_ERR_WORKSPACE if a capped or caller-owned one is smaller). */
MUON_API muon_status muon_selftest_gemm(muon_ctx* ctx, void* stream);

/* No counterpart on the pages (failure detection).
 * Synchronise the device and report the context's device-side flags:
 * MUON_ERR_TIMEOUT if a bounded wait gave up since the last check,
 * MUON_ERR_INVALID_ARG if a refreshed second moment was not positive
 * definite, MUON_ERR_CUDA on an asynchronous CUDA error, else MUON_OK.  The
 * flags are cleared.  While a flag is set, every kernel of later muon_step,
 * muon_orthogonalize, muon_adamw_step and muon_newton_precondition calls on
 * this context returns without writing, so a step that lost a product
 * part-way never applies a half-computed update; call this function to
 * learn of the error and resume. */
MUON_API muon_status muon_check_device(muon_ctx* ctx);

/* No counterpart on the pages (instrumentation).  Number of kernels this
 * context has launched since creation. */
MUON_API uint64_t muon_launch_count(const muon_ctx* ctx);

/* No counterpart on the pages (multi-GPU placement; the pages train on one
 * GPU).
 * Owner-computes sharding across `world` ranks (host only, no GPU needed):
 * every matrix i of shape rows[i] x cols[i] is an independent unit of the
 * step, so each goes to one owner rank, which alone keeps its momentum and
 * runs its Muon step; owners then send the updated weights to the other
 * ranks (the caller's collective).  Assignment: longest-processing-time
 * first on the nominal cost 5 (4 m^2 n + 2 m^3) + 5600 rows cols (Newton-
 * Schulz FLOPs plus elementwise bytes weighted by the B200 FLOP/byte
 * ratio), largest unit to the least-loaded rank, ties to the lower index
 * and the lower rank; deterministic, so every rank computes the same
 * owners.  owner[i] receives the rank of matrix i.  Errors: n < 0,
 * world < 1, NULL arrays or non-positive shapes -> MUON_ERR_INVALID_ARG. */
MUON_API muon_status muon_partition(const int64_t* rows, const int64_t* cols, int32_t n, int32_t world,
                                    int32_t* owner);

/* Kernel classes timed by the context's profiler. */
typedef enum {
  MUON_K_MOMENTUM = 0,   /* momentum + cast + Frobenius partial sums      */
  MUON_K_GRAM = 1,       /* A = X X^T                                     */
  MUON_K_POLY = 2,       /* B = b A + c A A                               */
  MUON_K_UPDATE = 3,     /* X <- a X + B X                                */
  MUON_K_APPLY = 4,      /* decay + scaled update of the weights          */
  MUON_K_ADAMW = 5,
  MUON_K_NEWTON_REFRESH = 6,
  MUON_K_PRECONDITION = 7,
  MUON_K_OTHER = 8,      /* finite scan                                    */
  MUON_K_UPDATE_APPLY = 9, /* last update with the weight step in its epilogue */
  MUON_K_NS_SMALL = 10,  /* every iteration of matrices up to 256 x 256 in one launch */
  MUON_K_COUNT = 11
} muon_kernel_kind;

typedef struct {
  double ms[MUON_K_COUNT];          /* summed device time of the launches  */
  uint64_t launches[MUON_K_COUNT];
} muon_kernel_times;

/* No counterpart on the pages (instrumentation).
 * enable != 0: bracket every launch with CUDA events on its stream (a few
 * microseconds of host time per launch; the GPU work is unchanged). */
MUON_API muon_status muon_profile_enable(muon_ctx* ctx, int enable);
/* No counterpart on the pages (instrumentation).
 * Wait for the recorded launches, add their event-measured durations into
 * *out (zeroed first) and reset the accumulators. */
MUON_API muon_status muon_profile_read(muon_ctx* ctx, muon_kernel_times* out);

/* No counterpart on the pages (an allocation-free variant).
 * Newton-Schulz of ONE matrix for callers that cannot allocate device
 * memory -- code running where cudaMalloc is off limits, such as inside a
 * host that manages every device byte itself, a custom allocator's
 * callback, or a process whose memory pool must not grow.  The sources have
 * no counterpart of this entry point; it computes what muon_orthogonalize
 * computes for a one-matrix group, without a context.
 *
 *   input   rows x cols, in_dtype (MUON_F32 or MUON_BF16), device, 16-byte
 *           aligned, read only.
 *   output  rows x cols fp32, device, 16-byte aligned: the orthogonalised
 *           matrix (Frobenius normalisation + hp->ns_steps iterations).
 *   hp      read on the host during the call (eps, ns_a/b/c, ns_steps).
 *   stream  cudaStream_t as void* (NULL = legacy default stream).
 *
 * Scratch is a fixed 32 MiB device array inside this library (every GPU that
 * loads the library holds it until the process exits); no call allocates.
 * A matrix fits when, with m = min(rows, cols), n = max(rows, cols),
 * ld_n = n rounded up to 8 and ld_m = m rounded up to 8, the bf16 buffers
 * (4 m ld_n + 4 m ld_m bytes) plus one float per 64 x 64 tile and about
 * 1 KiB of bookkeeping stay within it (e.g. 1024 x 4096 fits, 2048 x 2048
 * does not); a larger one returns MUON_ERR_WORKSPACE before anything is
 * enqueued.  Bad pointers, shapes, dtypes or hyper-parameters return
 * MUON_ERR_INVALID_ARG.
 *
 * The first call on a device looks the array's device address up (once, with
 * that device current); make that first call before any stream capture.
 * Each device has its own copy of the array, shared by every call on that
 * device: calls whose work overlaps on one GPU (different streams, or
 * threads without ordering) race and corrupt each other's results, so order
 * them on one stream.  The array keeps the last call's contents; each call
 * clears the parts that must start at zero.  The call copies nothing from
 * the host: its one descriptor travels as a kernel parameter.  If a bounded
 * device-side wait gives up during the call, its remaining kernels do
 * nothing and the output is filled with NaN, so the caller can tell a
 * result that is not valid from the output alone. */
MUON_API muon_status muon_orthogonalize_noalloc(const void* input, int32_t in_dtype, int64_t rows,
                                                int64_t cols, float* output, const muon_hparams* hp,
                                                void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MUON_B200_H */
