/*
 * shampoo.h -- C-ABI of the B200 (sm_100a) Shampoo optimizer step.
 *
 * Shampoo preconditions each 2-D weight W (m x n) with two small matrices,
 * L (rows) and R (columns), whose Kronecker product stands in for the full-
 * matrix-Adagrad preconditioner ("Scalable Second Order Optimization for Deep
 * Learning", Anil et al.; podcast transcript, segments 6-8).  One optimizer
 * step is three pieces of extra work (same transcript, segment 10):
 *
 *   shampoo_update_stats   L <- beta2 L + G G^T,  R <- beta2 R + G^T G
 *   shampoo_compute_roots  L^{-1/p}, R^{-1/p} by coupled Newton in float64
 *                          (segment 12), only every so many steps (segment 14)
 *   shampoo_apply          P = L^{-1/p} G R^{-1/p}, grafted to the norm of the
 *                          diagonal-Adagrad step, momentum, weight update
 *
 * Large weights are split into <= b x b blocks, each with its own L and R
 * (segment 16, Lemma 2).  A 1-D parameter keeps one statistic per segment of
 * <= b entries, S <- beta2 S + g g^T, rooted at exponent -2/p (full-matrix
 * Adagrad on the segment when p = 4).
 *
 * Conventions for every call below:
 *  - All work is enqueued, in order, on the CUDA stream given at create time
 *    and is asynchronous with respect to the host unless a call says that it
 *    synchronises.
 *  - Parameters and gradients are CALLER-OWNED device pointers to contiguous
 *    row-major arrays; the library never frees or keeps them past the call's
 *    stream work.  Optimizer state (statistics, roots, Adagrad accumulator,
 *    momentum, work space) is LIBRARY-OWNED device memory, allocated by
 *    shampoo_create and freed by shampoo_destroy.
 *  - Errors are returned as a shampoo_status, never by aborting;
 *    shampoo_last_error() gives a one-line reason.  A context is not
 *    thread-safe: call it from one host thread at a time.
 */
#ifndef SHAMPOO_B200_H
#define SHAMPOO_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct shampoo_ctx shampoo_ctx;   /* opaque, library-owned */

typedef enum {
  SHAMPOO_OK = 0,
  SHAMPOO_EINVAL = 1,         /* bad shape, size, option or null pointer      */
  SHAMPOO_ENOMEM = 2,         /* device allocation failed                      */
  SHAMPOO_ECUDA = 3,          /* a CUDA call or kernel launch failed           */
  SHAMPOO_ENONFINITE = 4,     /* a gradient held NaN/Inf (parameter skipped)   */
  SHAMPOO_ENOTCONVERGED = 5,  /* some roots did not converge (old roots kept)  */
  SHAMPOO_ESTATE = 6,         /* call out of order (e.g. apply before roots)   */
  SHAMPOO_EBUSY = 7           /* an asynchronous root job is still running     */
} shampoo_status;

typedef enum {
  SHAMPOO_GRAFT_NONE = 0,     /* U = P                                         */
  SHAMPOO_GRAFT_ADAGRAD = 1   /* U = (||D||_F / ||P||_F) P per parameter,
                                 D = g / sqrt(a + eps), a <- beta2 a + g*g     */
} shampoo_graft;

typedef enum {
  SHAMPOO_SIDES_BOTH = 0,     /* L and R (the default)                         */
  SHAMPOO_SIDE_LEFT = 1,      /* L only: P = L^{-2/p} G                        */
  SHAMPOO_SIDE_RIGHT = 2      /* R only: P = G R^{-2/p}                        */
} shampoo_side;

typedef enum {
  SHAMPOO_ROOTS_FP64 = 0,          /* Newton products in float64 (mma f64)     */
  SHAMPOO_ROOTS_INT8_EMULATED = 1  /* the same products emulated on the int8
                                      tensor cores (Ozaki scheme)              */
} shampoo_root_method;

typedef enum {
  SHAMPOO_F32 = 0,            /* gradients are float32                         */
  SHAMPOO_BF16 = 1            /* gradients are bfloat16 (statistics in fp32)   */
} shampoo_dtype;

/*
 * shampoo_create -- build the block table and allocate the state.
 *
 *  out         receives the new context (set to NULL on failure).
 *  nparams     number of parameters, >= 1.
 *  shapes      host array [nparams][2] of (rows, cols), each >= 1.  For a 1-D
 *              parameter of length n pass (1, n) and set ndims[i] = 1.
 *  ndims       host array [nparams] of 1 or 2, or NULL for all 2-D.
 *  block_size  b, the largest block side (segment 16): 64, 128, ..., 1024 (a
 *              multiple of 64, the tile side of the kernels).  Blocks form a row-major grid from the top-left
 *              corner; the last block row / column is ragged.
 *  beta2       statistics decay, 0 < beta2 <= 1 (1 = plain accumulation).
 *  epsilon     ridge added at root time, (A + eps I)^{-1/p}, and inside the
 *              graft's sqrt; > 0.
 *  p           root order for the two factors of a 2-D block (4 in the paper,
 *              segment 14); 1-D segments use p/2.  p must be 2 or 4.
 *  graft       SHAMPOO_GRAFT_NONE or SHAMPOO_GRAFT_ADAGRAD (layer-wise).
 *  momentum    heavy-ball factor mu in [0, 1): m <- mu m + U, W <- W - lr m.
 *  grad_dtype  element type of every gradient passed later.
 *  cuda_stream caller-owned cudaStream_t (NULL = legacy default stream).
 * Statistics, accumulator and momentum start at zero.  Roots start unset;
 * shampoo_apply fails with SHAMPOO_ESTATE until shampoo_compute_roots ran.
 * Synchronises the stream once (state zeroing).
 */
shampoo_status shampoo_create(shampoo_ctx** out, int nparams,
                              const int64_t* shapes, const int32_t* ndims,
                              int block_size, float beta2, float epsilon,
                              int p, shampoo_graft graft, float momentum,
                              shampoo_dtype grad_dtype, void* cuda_stream);

/*
 * shampoo_update_stats -- accumulate gradient outer products (segment 10,
 * first piece): per block L <- beta2 L + G G^T and R <- beta2 R + G^T G, per
 * 1-D segment S <- beta2 S + g g^T, and, with grafting, a <- beta2 a + g*g.
 *  grads  host array [nparams] of device pointers, each to rows*cols
 *         elements of grad_dtype, row-major.
 * A parameter whose gradient holds a NaN or Inf is skipped for this step
 * (statistics, accumulator and, in the next apply, weights and momentum are
 * left unchanged); the count is read with shampoo_nonfinite_status.
 */
shampoo_status shampoo_update_stats(shampoo_ctx* ctx, const void* const* grads);

/*
 * shampoo_compute_roots -- inverse p-th roots of every statistic (segment
 * 10, second piece), by the coupled Newton iteration in float64 on the device
 * (segment 12): X -> (A + eps I)^{-1/p}, stopping per matrix when
 * max|X^p (A + eps I) - I| <= tol (default 1e-6), giving up on a non-finite
 * or non-decreasing residual or at the iteration cap (default 100).
 * The caller picks the interval (segment 14: recompute only now and then).
 * Synchronises with the host while it runs (it polls the number of matrices
 * still iterating).  SHAMPOO_ESTATE before the first shampoo_update_stats.
 * Returns SHAMPOO_ENOTCONVERGED when some matrix gave up:
 * those keep their previous root (or c^{-1} I, c^p = the eigenvalue bound
 * the iteration started from, if they never had one); the others are updated.
 */
shampoo_status shampoo_compute_roots(shampoo_ctx* ctx);

/*
 * shampoo_compute_roots_async -- the same root computation, pipelined behind
 * the training steps (podcast transcript, segment 16: the statistics and the
 * preconditioned step keep running on the current roots while the next roots
 * are computed elsewhere and take over once ready; segment 14: roots a few steps old
 * cost next to nothing in quality).
 *
 * Enqueues on the context's stream a copy of the statistics as they stand
 * after every call made so far, and returns without waiting.  A library-owned
 * host thread then runs the coupled Newton iteration on that copy on a
 * library-owned stream of the lowest priority, writing into a second set of
 * roots; the roots in use are untouched until the job is installed.  The
 * first shampoo_apply (or shampoo_install_roots) that finds the job finished
 * swaps the new roots in; matrices that did not converge keep their previous
 * root, as with shampoo_compute_roots.
 *
 * For the steps to run ahead of the root work on the GPU, give the context a
 * stream of higher priority than the default (the library's stream has the
 * lowest).  The second set of roots, its bf16 copy and the statistics copy
 * (3 x 4 b^2 bytes per matrix) are allocated on the first call.
 * Returns SHAMPOO_ESTATE before the first shampoo_update_stats, and
 * SHAMPOO_EBUSY (nothing enqueued) while the previous job still runs; a
 * finished, not yet installed job is installed first.
 * While a job is in flight, shampoo_compute_roots returns SHAMPOO_EBUSY.
 */
shampoo_status shampoo_compute_roots_async(shampoo_ctx* ctx);

/*
 * shampoo_install_roots -- swap in the roots of a finished asynchronous job.
 *  wait       0: install only if the job has finished; 1: block the host
 *             until it finishes, then install.
 *  installed  receives 1 if roots were installed by this call, else 0 (may
 *             be NULL).
 * Returns the job's status when it installs (SHAMPOO_OK, or
 * SHAMPOO_ENOTCONVERGED with the counts in shampoo_root_status and
 * shampoo_root_iterations), SHAMPOO_ECUDA if the job failed (nothing is
 * swapped), and SHAMPOO_OK when there is nothing to install.
 */
shampoo_status shampoo_install_roots(shampoo_ctx* ctx, int wait, int* installed);

/*
 * shampoo_roots_generation -- how many root sets have been put in use: each
 * shampoo_compute_roots that returns SHAMPOO_OK or SHAMPOO_ENOTCONVERGED and
 * each install of an asynchronous job adds one.  Tells a caller at which call
 * new roots took effect.  Host value; -1 for a NULL ctx.
 */
int64_t shampoo_roots_generation(const shampoo_ctx* ctx);

/*
 * shampoo_apply -- precondition and update (segment 10, third piece):
 * per block P = L^{-1/p} G R^{-1/p} (per 1-D segment P = S^{-2/p} g), then
 * per parameter U = s P with the graft scale s, m <- mu m + U, W <- W - lr m.
 *  params  host array [nparams] of device float32 pointers, updated in place.
 *  grads   as for shampoo_update_stats; pass this step's gradients.
 *  lr      learning rate.
 * Returns SHAMPOO_ESTATE if roots were never computed.  First installs the
 * roots of a finished asynchronous job, if there is one (never waits for
 * one); a failed job's SHAMPOO_ECUDA is returned here, before any work.
 */
shampoo_status shampoo_apply(shampoo_ctx* ctx, float* const* params,
                             const void* const* grads, float lr);

/*
 * shampoo_root_status -- result of the last shampoo_compute_roots, or of
 * the last installed asynchronous job.
 *  n_not_converged  number of matrices that kept their previous root.
 *  max_iters        largest Newton iteration count over the matrices.
 * Either pointer may be NULL.  Host values; synchronises the stream.
 */
shampoo_status shampoo_root_status(shampoo_ctx* ctx, int* n_not_converged,
                                   int* max_iters);

/*
 * shampoo_nonfinite_status -- number of parameters skipped by the last
 * shampoo_update_stats because their gradient was not finite.  Synchronises.
 */
shampoo_status shampoo_nonfinite_status(shampoo_ctx* ctx, int* n_params_skipped);

/*
 * shampoo_set_root_options -- Newton stopping rule for later root calls:
 * tol > 0 on max|M - I|, 1 <= max_iters <= 1000.
 */
shampoo_status shampoo_set_root_options(shampoo_ctx* ctx, double tol, int max_iters);

/*
 * shampoo_set_root_method -- how later root calls multiply matrices inside
 * the coupled Newton iteration (the iteration, its stopping rule and its
 * float64 state are the same for both).
 *  method  SHAMPOO_ROOTS_FP64: float64 products (the default).
 *          SHAMPOO_ROOTS_INT8_EMULATED: each float64 operand row is cut into
 *          `slices` signed 7-bit digits below a per-row power of two, and a
 *          product is the exact int32 sum of the digit products whose weights
 *          reach 2^{-7 (slices+1)} (Ozaki scheme), run on the int8 tensor
 *          cores.  Per entry the error is of order n 2^{-7 slices} times the
 *          row and column scales (2^-42 n for 6 slices), against 2^-53 for a
 *          float64 product.
 *  slices  4..6 for the emulated method (6 recommended); ignored otherwise.
 * The emulated method allocates 30 int8 planes of b x b bytes (5 iterates x 6
 * slices) per matrix of a Newton chunk on first use.  SHAMPOO_EBUSY while an
 * asynchronous root job runs.
 */
shampoo_status shampoo_set_root_method(shampoo_ctx* ctx, int method, int slices);

/*
 * shampoo_set_one_sided -- keep only one factor for every block of 2-D
 * parameter `param` (podcast transcript, segment 16: for a layer too large
 * even when blocked, such as a big embedding or softmax, only L or only R is
 * used, Lemma 1).  The kept factor is accumulated as usual and rooted at
 * exponent -2/p (-1/2 for p = 4: full-matrix Adagrad along that dimension);
 * the dropped factor is never accumulated, never rooted, and its root slot
 * holds the identity, so the apply computes P = L^{-1/2} G (side LEFT) or
 * P = G R^{-1/2} (side RIGHT).  SHAMPOO_SIDES_BOTH restores the default.
 * Call between shampoo_create and the first shampoo_update_stats
 * (SHAMPOO_ESTATE later).  SHAMPOO_EINVAL for a 1-D parameter, a bad index
 * or side, or a context created with p != 4.  Synchronises the stream.
 * shampoo_matrix_info reports root_p = 0 for a dropped factor.
 */
shampoo_status shampoo_set_one_sided(shampoo_ctx* ctx, int param, int side);

/*
 * shampoo_num_matrices -- number of statistics matrices: 2 per 2-D block
 * (L then R, blocks in parameter order, row-major within a parameter), then
 * 1 per 1-D segment (parameter order).  Each lives in a b x b slot.
 */
int shampoo_num_matrices(const shampoo_ctx* ctx);

/*
 * shampoo_matrix_info -- for statistic `index`: its valid side (the block's
 * rows for L, columns for R, the segment length for S) and its root exponent
 * denominator (p, or p/2 for a segment or a one-sided block's kept factor,
 * 0 for its dropped factor).  Host values.
 */
shampoo_status shampoo_matrix_info(const shampoo_ctx* ctx, int index,
                                   int* size, int* root_p);

/*
 * shampoo_read_matrix -- copy the b x b float32 slot of statistic `index`
 * (which = 0) or of its root (which = 1) into dst (host or device memory,
 * b*b floats, row-major).  Only the top-left size x size corner is the
 * matrix; the rest is zero.  Synchronises the stream.
 */
shampoo_status shampoo_read_matrix(shampoo_ctx* ctx, int which, int index,
                                   float* dst);

/*
 * shampoo_root_iterations -- per-matrix Newton iteration counts of the last
 * shampoo_compute_roots, in statistic order: k >= 0 when matrix i converged
 * after k steps, -1-k when it gave up at step k.
 *  out  host array of shampoo_num_matrices(ctx) int32 values.
 * SHAMPOO_ESTATE before the first shampoo_compute_roots.
 */
shampoo_status shampoo_root_iterations(shampoo_ctx* ctx, int32_t* out);

/*
 * Kernel profiling.  The library counts every kernel it launches, per
 * kernel name.  With profiling enabled it also records a pair of CUDA events
 * on the context's stream around each launch and sums their elapsed times.
 *  shampoo_profile_enable  clears the counters; on != 0 turns event timing on.
 *  shampoo_profile_count   number of kernel names seen since the last enable.
 *  shampoo_profile_entry   for name `index`: the name (copied into name, at
 *                          most name_len bytes with the terminating NUL), the
 *                          launch count and the summed milliseconds (0 when
 *                          timing was off).  Synchronises on pending events.
 */
shampoo_status shampoo_profile_enable(shampoo_ctx* ctx, int on);
int shampoo_profile_count(const shampoo_ctx* ctx);
shampoo_status shampoo_profile_entry(shampoo_ctx* ctx, int index, char* name, int name_len,
                                     int64_t* launches, double* ms);

/*
 * shampoo_last_error -- one-line reason for the last failed call on ctx
 * (empty string if none).  ctx may be NULL for a create failure.
 */
const char* shampoo_last_error(const shampoo_ctx* ctx);

/* shampoo_destroy -- free all library-owned memory.  NULL is a no-op. */
void shampoo_destroy(shampoo_ctx* ctx);

/*
 * shampoo_batched_inverse_root -- the root kernel on its own (segment 12):
 * X_i = (A_i + eps I)^{-1/p} for `batch` symmetric PSD n x n matrices, by
 * coupled Newton in float64 on the device.
 *  A       device float32 [batch][n][n], row-major, symmetric (read only).
 *  X       device float32 [batch][n][n] output (caller-owned).
 *  batch   >= 1;  n in [1, 1024];  p in {2, 4};  eps > 0;  tol > 0;
 *  max_iters in [1, 1000].
 *  iters   device int32 [batch] or NULL: per-matrix iteration count k, or
 *          -1-k when the matrix gave up at iteration k.  On give-up X_i holds
 *          c^{-1} I (c^p = the starting eigenvalue bound).
 *  stream  caller-owned cudaStream_t.
 * Allocates its float64 work space (7 n' x n' doubles per matrix in flight,
 * n' = n rounded up to 64, at most 2 GiB) in stream order on `stream` from a
 * memory pool the library keeps per device, and frees it back to that pool
 * before returning: the pool keeps the memory (it is not returned to the
 * driver), so calls after the first allocate without the driver.  The
 * three pinned host ints and two events it polls the iteration with are made
 * on a host thread's first call on a device and kept for that thread's later
 * calls there (made again if a device reset released them).
 * Synchronises while it runs, like shampoo_compute_roots.  Returns
 * SHAMPOO_ENOTCONVERGED if any matrix gave up.
 */
shampoo_status shampoo_batched_inverse_root(const float* A, float* X, int batch,
                                            int n, int p, float eps, double tol,
                                            int max_iters, int32_t* iters,
                                            void* stream);

/*
 * shampoo_batched_inverse_root_ex -- shampoo_batched_inverse_root with the
 * product method of shampoo_set_root_method (method, slices).  The emulated
 * method also allocates its int8 slice planes (30 n' x n' bytes per matrix in
 * flight, n' = n rounded up to 64) and frees them before returning.
 */
shampoo_status shampoo_batched_inverse_root_ex(const float* A, float* X, int batch,
                                               int n, int p, float eps, double tol,
                                               int max_iters, int32_t* iters,
                                               void* stream, int method, int slices);

/*
 * shampoo_batched_inverse_root_noalloc -- shampoo_batched_inverse_root for
 * callers that cannot allocate device memory.  (The paper has no counterpart:
 * this is a deployment variant of the same root computation.)
 *
 * Who needs it: code whose device memory is owned by a framework's pooling
 * allocator (a raw cudaMalloc there fragments the pool or fails once the pool
 * has reserved the GPU), code on a path where an allocation's implicit
 * synchronisation is not acceptable, and hosts that forbid allocating after
 * start-up.  This call allocates nothing -- no cudaMalloc, cudaFree, pinned
 * host memory, CUDA events or library allocator.  Its float64 work space is
 * one 64 MiB array compiled into the library, present on every GPU that loads
 * the library until the process exits.
 *
 * Arguments, outputs and results are those of shampoo_batched_inverse_root
 * (A, X and iters are caller-owned device memory).  Limits: n <= 1024; larger
 * n is rejected with SHAMPOO_EINVAL and a message from shampoo_last_error(NULL).
 * Any batch size is accepted; matrices are processed in chunks that fit the
 * work space (7 n' x n' doubles each, n' = n rounded up to 64).
 * Sharing: every call uses the same work space, so calls that overlap on the
 * GPU (from other streams or host threads) race; serialise them.  Every call
 * looks up the work space's device address on the current device (nothing is
 * kept between calls, so a device reset cannot leave a stale address); the
 * first lookup in a process may load the library's device code.
 * Synchronises with the host while it runs.
 */
shampoo_status shampoo_batched_inverse_root_noalloc(const float* A, float* X, int batch, int n,
                                                    int p, float eps, double tol, int max_iters,
                                                    int32_t* iters, void* stream);

/*
 * shampoo_plan_shards -- which rank owns each parameter in the block-sharded
 * data-parallel step.  The blocks of a weight are independent (podcast
 * transcript, segment 16, Lemma 2), so ranks split the optimizer work by
 * whole parameter: each owner receives the summed gradients of its
 * parameters, runs statistics, roots and apply on them alone (the
 * layer-wise graft stays local) and sends the updated weights to the others.
 *  nparams, shapes, ndims, block_size  as for shampoo_create (host arrays).
 *  root_interval  steps between root computations (>= 1), to weigh the
 *                 root work against the per-step work.
 *  nranks   >= 1.
 *  owner    host int32 [nparams] output: the owning rank of each parameter.
 *  rank_cost  host double [nranks] output or NULL: the planned work per
 *             rank, in the planner's flop-like units.
 * Longest-processing-time-first over a per-parameter cost model (statistics
 * and apply GEMMs per step, root products per root interval, elementwise
 * passes); deterministic, so every rank computes the same plan.  Host only:
 * touches no GPU.  SHAMPOO_EINVAL on bad arguments (message from
 * shampoo_last_error(NULL)).
 */
shampoo_status shampoo_plan_shards(int nparams, const int64_t* shapes,
                                   const int32_t* ndims, int block_size,
                                   int root_interval, int nranks, int32_t* owner,
                                   double* rank_cost);

/*
 * shampoo_set_gemm_tiles -- the tiling of the statistics and apply GEMMs.
 *  pair = 1 (the default): where the block side is a multiple of 256, the two
 *    apply GEMMs run 256 x 256 output tiles on pairs of CTAs (tcgen05
 *    cta_group::2: each CTA of a pair loads half of each operand tile, one
 *    MMA reads both), which halves the operand bytes each SM reads per
 *    output.
 *  pair = 0: 128 x 128 tiles on single CTAs.
 * The statistics GEMM always runs single-CTA 128 x 128 tiles (its two-level
 * accumulation keeps 128 running sums per thread).  Both tilings compute the
 * same products in the same precision scheme (results agree to rounding
 * order).  Takes effect from the next call.  SHAMPOO_EINVAL for any other
 * value.
 */
shampoo_status shampoo_set_gemm_tiles(shampoo_ctx* ctx, int pair);

/*
 * shampoo_selftest_stalled_wait -- failure-path check: launches one warp
 * that waits, through the same bounded mbarrier wait every tensor-core
 * pipeline of the library uses, on a barrier phase that nothing completes.
 * The wait gives up after about 2^31 clock cycles (about a second), records
 * the timeout the way a stalled pipeline does and the kernel returns, so the
 * call ends with SHAMPOO_ECUDA ("timed out waiting on its pipeline") and the
 * CUDA context stays usable.  A test of the error path: no fault, no hang.
 * stream: caller-owned cudaStream_t.  Allocates and frees 4 bytes.
 */
shampoo_status shampoo_selftest_stalled_wait(void* stream);

/*
 * shampoo_selftest_stall_next_stats -- failure-path check inside the product
 * kernels: the next shampoo_update_stats of `ctx` launches its statistics
 * GEMM with the MMA issuer first waiting, through the pipelines' bounded
 * wait, on a barrier phase that nothing completes.  That wait runs out (about
 * a second) exactly as a stalled pipeline would: the launch aborts, lets the
 * loads it has in flight land, frees its tensor memory, sets the context's
 * error word and returns.  update_stats itself returns SHAMPOO_OK (it does not
 * wait for its kernels); the next call that synchronises --
 * shampoo_compute_roots, shampoo_install_roots with wait, shampoo_root_status,
 * shampoo_nonfinite_status -- returns SHAMPOO_ECUDA, and so does every step
 * call after an apply has copied the error word back.  The context's
 * statistics are then half-updated: destroy it.  A test of the error path:
 * no fault, no hang.  SHAMPOO_EINVAL if ctx is NULL.
 */
shampoo_status shampoo_selftest_stall_next_stats(shampoo_ctx* ctx);

/*
 * shampoo_selftest_stall_next_apply -- the same failure-path check for the
 * apply GEMMs: the next shampoo_apply launches its first GEMM (Y = G R^{-1/p},
 * on CTA pairs where the block side is a multiple of 256) with the MMA issuer
 * first waiting on a barrier phase that nothing completes; the launch aborts
 * as above (both CTAs of a pair together), the weights of that step are not
 * valid, and the next synchronising call -- or the next step call, once the
 * error word has been copied back -- returns SHAMPOO_ECUDA.  SHAMPOO_EINVAL if
 * ctx is NULL.
 */
shampoo_status shampoo_selftest_stall_next_apply(shampoo_ctx* ctx);

/* Library version, "MAJOR.MINOR.PATCH". */
const char* shampoo_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SHAMPOO_B200_H */
