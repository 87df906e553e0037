/*
 * psgd.h - C ABI of the B200 PowerSGD compression-step library (libpsgd.so).
 *
 * What it computes.  For every gradient matrix M (m x n, row-major, leading
 * dimension n; convolution weights are passed already viewed as
 * out x (in*k*k), "anthology-of-the-sota" note-152 on PowerSGD, section
 * "Method", per-layer approximation with reshaped conv tensors) and W
 * workers, one call of psgd_step performs one PowerSGD compression step in
 * the order the same section gives:
 *
 *   M_w   = G_w + E_w                         error feedback ("Concepts")
 *   P_bar = (1/W) sum_w M_w Q                 right multiply + all-reduce
 *   P_hat = P_bar R^-1  (Gram-Schmidt QR)     orthogonalisation of P
 *   Q_bar = (1/W) sum_w M_w^T P_hat           left multiply + all-reduce
 *   E'_w  = M_w - P_hat Q_bar^T               new error memory
 *   G_hat = P_hat Q_bar^T                     decompressed mean gradient
 *
 * and Q (the warm start, "Concepts", warm-start subspace iteration) is
 * replaced by Q_bar.  The W workers are replica buffers in this GPU's memory;
 * the "all-reduce" is an on-device mean, computed in a fixed order so that
 * results are bitwise reproducible run to run.
 *
 * Orthogonalisation: P_hat is the Q factor of the thin QR of P_bar with a
 * positive diagonal (what Gram-Schmidt produces).  The library computes it
 * as a Cholesky QR: the r x r Gram matrix of P_bar is accumulated in
 * float64, factored (Cholesky, float64), and P_hat = P_bar T with T the
 * inverse of the factor.  A column whose squared norm after projection on
 * the previous ones is <= 1e-12 * max_k ||pbar_k||^2 becomes zero (the
 * pages say nothing about rank deficiency; this is the rule the float64
 * oracle uses too).  NaN inputs propagate; they are not trapped.
 *
 * Precision: G is float32 or bfloat16; E, Q, P_hat, Q_bar and G_hat are
 * float32.  Products are float32 (ranks 16 and 32: tf32 tensor-core
 * products of hi/lo-split factors, relative error below 2^-21), summed in
 * float32 over short runs and then in float64; P_bar, the Gram matrix, its
 * Cholesky factor and every partial sum across CTAs are float64.
 *
 * Ownership: the caller owns every tensor passed in (device memory, e.g.
 * PyTorch tensors).  The library owns its workspace and pointer tables,
 * allocated in psgd_create and released in psgd_destroy.  E and Q are
 * updated in place.
 *
 * Alignment: every device pointer passed must be 16-byte aligned
 * (PSGD_ERR_ALIGN otherwise).  Rows need not be: n may be odd.
 *
 * Streams and ordering: every call enqueues work on `stream` (a
 * cudaStream_t passed as void*, NULL = legacy default stream) and returns
 * without synchronising.  Calls on one context must be ordered (one stream,
 * or synchronised by the caller): they share workspace and counters.
 * Pointer tables are re-uploaded (on `stream`) only when the pointers
 * passed differ from the previous call's.
 *
 * Errors: argument checks are synchronous and return a code; a failed CUDA
 * call returns PSGD_ERR_CUDA.  psgd_last_error gives a message.  Device-side
 * problems are reported through psgd_status.  No call spins on the device.
 */
#ifndef PSGD_H
#define PSGD_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PSGD_API __attribute__((visibility("default")))
#else
#define PSGD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
    PSGD_OK = 0,
    PSGD_ERR_ARG = 1,    /* null pointer, bad shape, rank or worker count */
    PSGD_ERR_ALIGN = 2,  /* a device pointer is not 16-byte aligned */
    PSGD_ERR_CUDA = 3,   /* a CUDA runtime call failed */
    PSGD_ERR_OOM = 4,    /* workspace allocation failed */
    PSGD_ERR_STATE = 5,  /* call not valid in this context's mode */
    PSGD_ERR_DEVICE = 6, /* a kernel found a reduction counter inconsistent (psgd_status) */
    PSGD_ERR_TIMEOUT = 7 /* a bounded wait in a kernel ran out (psgd_status) */
};

typedef enum { PSGD_F32 = 0, PSGD_BF16 = 1 } psgd_dtype; /* dtype of G only */

enum {
    /* Keep M_w (not E'_w) in the error buffers between steps and rebuild
     * E'_w = M_w - P_hat Q_bar^T on the fly in the next step's first pass
     * (saves one read and one write of every worker element per step).  The
     * error buffers then hold M_w after psgd_step; psgd_materialize_errors
     * turns them into E'_w. */
    PSGD_FLAG_LAZY_ERRORS = 1u,
    /* Sum the W workers' M_w element-wise before multiplying by Q or P_hat
     * (one product per matrix element instead of one per worker element).
     * Same result up to rounding, by linearity (note-152, "Concepts"). */
    PSGD_FLAG_SUM_FIRST = 2u,
    /* No warm start (the ablation of note-152, "Claims" C4): every step
     * first overwrites q[l] with a fresh N(0, 1) draw, the psgd_init_q
     * generator with draw index = step number (1, 2, ...; psgd_init_q is
     * draw 0).  One extra launch per step. */
    PSGD_FLAG_NO_WARM_START = 4u
};

typedef struct { int64_t m, n; } psgd_layer;   /* one gradient matrix */
typedef struct psgd_ctx psgd_ctx;              /* opaque */

/* Create a context on the current CUDA device (the pages define no
 * interface; a context holds what note-152 "Method" keeps between steps
 * besides the caller's E and Q: P_hat and Q_bar of the last step).
 * layers[num_layers]: matrix shapes, m >= 1, n >= 1 (num_layers may be 0:
 *   every step is then a no-op).
 * rank: 1 <= rank <= 32 and rank <= min(m, n) for every layer.
 * workers: 1 <= workers <= 256.
 * seed: key of the initial-Q draw (psgd_init_q).
 * grad_dtype: PSGD_F32 or PSGD_BF16.  flags: PSGD_FLAG_*.
 * Allocates the workspace (see psgd_workspace_bytes).  On error *out is
 * NULL. */
PSGD_API int psgd_create(psgd_ctx **out, const psgd_layer *layers, int num_layers, int rank, int workers,
                uint64_t seed, int grad_dtype, unsigned flags);

/* Release the context's workspace, tables and staging (NULL is a no-op);
 * waits for the device first. */
PSGD_API void psgd_destroy(psgd_ctx *ctx);

/* Draw Q0 ~ N(0, 1) for every layer into q[l] (device, n x rank float32,
 * row-major).  Philox4x64-10 (Salmon et al., SC'11) keyed by (seed, l),
 * counter (b, 0, 0, 0) for element block b = e / 4 (e = j*rank + k), then
 * Box-Muller on the word pairs (0,1), (2,3) in float64, rounded to float32.
 * The initial Q is not orthogonalised and is shared by all workers. */
PSGD_API int psgd_init_q(psgd_ctx *ctx, float *const *q, void *stream);

/* One compression step for all layers and workers: the sequence of
 * note-152 "Method" listed at the top of this file.
 * grads[w*L + l]:  device, m x n, grad dtype, read only.
 * errors[w*L + l]: device, m x n float32, E_w in, E'_w out (in place).  With
 *                  PSGD_FLAG_LAZY_ERRORS: M_w out (see the flag).
 * q[l]:            device, n x rank float32, warm start in, Q_bar out.
 * p_hat[l]:        device, m x rank float32 out, or p_hat == NULL, or an
 *                  entry NULL to skip that layer's copy.
 * recon[l]:        device, m x n float32 out (G_hat), or NULL / NULL entry.
 * The last P_hat and Q_bar are also kept inside the context (for
 * psgd_momentum_step and the lazy representation). */
PSGD_API int psgd_step(psgd_ctx *ctx, const void *const *grads, float *const *errors, float *const *q,
              float *const *p_hat, float *const *recon, void *stream);

/* The same step with HOST gradients (an interface variant of psgd_step; no
 * counterpart in the pages): grads_host[w*L + l] are host pointers
 * (pinned for asynchronous copies; pageable works but serialises).  The
 * library copies them into a device staging area it owns (allocated on
 * first use), runs psgd_step, and copies P_hat and Q_bar back to
 * p_hat_host[l] (m x rank) and q_host[l] (n x rank) if those are non-NULL.
 * errors and q stay device pointers (they are state).
 * Upload and step overlap: the layers are split into at most 8 contiguous
 * groups of about equal size; the copies run on a stream of the context's
 * own, which starts after everything already queued on `stream`, and
 * group g's passes start on `stream` as soon as group g's copies are done
 * (one launch of each pass per group).  Steps with power iterations, an SVD
 * refresh or profiling on wait for the whole upload and launch as
 * psgd_step does.  Everything the call enqueues is ordered before later
 * work on `stream`, as for psgd_step. */
PSGD_API int psgd_step_host(psgd_ctx *ctx, const void *const *grads_host, float *const *errors, float *const *q,
                   float *const *p_hat_host, float *const *q_host, void *stream);

/* psgd_step_host for gradients packed into one host buffer per worker (a
 * flat gradient bucket): layer l of worker w starts at element
 * layer_offset[l] of grads_host[w] (grad dtype).  Per layer group (see
 * psgd_step_host) the library uploads each worker's layers with one copy
 * per run of layers that follow one another in the buffer (gaps holding no
 * layer's elements are copied and ignored), so the caller guarantees that
 * elements [0, max_l(layer_offset[l] + m_l * n_l)) of each worker are one
 * allocation (pinned for asynchronous copies).  layer_offset[l] *
 * sizeof(grad dtype) must be a multiple of 16 (PSGD_ERR_ALIGN otherwise),
 * offsets must be >= 0.  Otherwise as psgd_step_host. */
PSGD_API int psgd_step_host_flat(psgd_ctx *ctx, const void *const *grads_host, const int64_t *layer_offset,
                                 float *const *errors, float *const *q, float *const *p_hat_host,
                                 float *const *q_host, void *stream);

/* PSGD_FLAG_LAZY_ERRORS only: write E'_w = M_w - P_hat Q_bar^T (from the
 * last step; the residual of note-152 "Concepts") into errors[w*L + l] in
 * place.  The next step then starts from E'_w as in the eager mode.
 * PSGD_ERR_STATE for a context without the flag. */
PSGD_API int psgd_materialize_errors(psgd_ctx *ctx, float *const *errors, void *stream);

/* Post-compression momentum (note-152, "Concepts"): for every layer, with
 * G_hat = P_hat Q_bar^T of the last step (recomputed on the fly, never read
 * from memory): mom = beta*mom + G_hat; params = params - lr*mom.
 * params[l], mom[l]: device m x n float32, updated in place. */
PSGD_API int psgd_momentum_step(psgd_ctx *ctx, float *const *params, float *const *mom, float lr, float beta,
                       void *stream);

/* Small tensors travel uncompressed (note-152, "Method"): out[k] = mean over
 * the ctx's W workers of vecs[w*count + k] (len[k] float32 elements each,
 * summed in worker order).  After psgd_set_global_workers the sum is
 * divided by the global worker count instead: pass vectors already summed
 * over the ranks (an all-reduce of every local worker's vector) to get the
 * global mean.  Vectors of length 0 may have null pointers.  If params and mom are non-NULL, also applies
 * the momentum update above with out[k] as the gradient. */
PSGD_API int psgd_vec_mean(psgd_ctx *ctx, const float *const *vecs, float *const *out, const int64_t *len, int count,
                  float *const *params, float *const *mom, float lr, float beta, void *stream);

/* Service calls (no counterpart in the pages).
 * Synchronise the last stream used and read the device status word:
 * PSGD_OK; PSGD_ERR_TIMEOUT if a bounded wait of a tensor-core pass ran out
 * (about one second; that tile wrote nothing; bit 0x2 of the word);
 * PSGD_ERR_DEVICE if a reduction counter held an impossible value (bit 0x1,
 * e.g. steps overlapping on one context); or PSGD_ERR_CUDA if a launch
 * failed.  psgd_last_error gives the word.  A set word is reported once and
 * then cleared, so the steps that follow report their own state (the
 * context's counters stay consistent either way).  Either error means the
 * results of the step(s) since the last clean report are not valid. */
PSGD_API int psgd_status(psgd_ctx *ctx);

/* For testing the bounded waits (no counterpart in the pages): with on != 0
 * the tensor-core second pass (ranks 16 and 32, 16-byte rows) of later
 * steps issues no products and commits none, so each of its tiles waits
 * out its one-second limit, sets bit 0x2 of the status word (psgd_status:
 * PSGD_ERR_TIMEOUT), releases its tensor memory and writes no partial; that
 * step's results are not valid.
 * on = 0 (the default) restores normal steps. */
PSGD_API int psgd_test_stall_products(psgd_ctx *ctx, int on);

/* Bytes of device workspace the context holds (excluding host staging). */
PSGD_API int psgd_workspace_bytes(const psgd_ctx *ctx, size_t *bytes);

/* Number of kernel launches one regular psgd_step makes for this context
 * (for launch accounting): per power iteration the first pass, the P_hat
 * kernel and the second pass, + 1 for the third pass in eager mode, + 1
 * with PSGD_FLAG_NO_WARM_START.  An SVD-refresh step makes the launches
 * stated at psgd_set_svd_refresh.  The host-buffer steps launch each pass
 * once per layer group (psgd_step_host). */
PSGD_API int psgd_step_launches(const psgd_ctx *ctx);

/* Allocation-free step for one layer.  No counterpart in the pages: this
 * entry point exists for callers that cannot allocate device memory, for
 * example code whose device memory is owned by another allocator (a
 * framework's caching pool that must account for every byte), code that
 * must not pay for cudaMalloc's implicit device synchronisation inside a
 * training loop, or code running where allocation is not permitted.
 *
 * It runs the same kernels and computes the same eager step as psgd_step
 * for a single m x n layer, with no context: every piece of scratch (layer
 * descriptor, pointer table, P and Q partials, P_bar, P_hat, Q_bar, Gram
 * partials, T, counters) lives in one file-scope static device array of
 * PSGD_STATIC_SCRATCH_BYTES (16 MiB).  Every GPU that loads the library
 * holds that array until the process exits.  The call allocates no device
 * memory and calls no allocating routine: a small set-up kernel, launched
 * on `stream` with the layer descriptor and the pointer table passed by
 * value, writes them into the array and clears the counters and the status
 * word; only a failed call stores its message in thread-local host memory
 * for psgd_last_error(NULL).
 *
 * grads[w], errors[w]: HOST arrays of W device pointers (m x n, grad dtype
 * and float32); q: device n x rank (warm start in, Q_bar out); p_hat:
 * device m x rank or NULL; recon: device m x n or NULL.  Same argument
 * rules as psgd_create / psgd_step (1 <= rank <= min(m, n, 32),
 * 1 <= workers <= 256, 16-byte aligned pointers).  A layer whose scratch
 * does not fit in the static array is rejected with PSGD_ERR_ARG before
 * any device work (psgd_last_error(NULL) says how much it needs).
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) once for that device; make that first call before
 * any stream capture.  All calls share the one array and it keeps the last
 * call's contents (the counters are cleared at the start of every call):
 * calls that overlap on the GPU - on two streams, or from two threads -
 * race and corrupt each other; order them. */
#define PSGD_STATIC_SCRATCH_BYTES (16u << 20)
PSGD_API int psgd_step_static(int64_t m, int64_t n, int rank, int workers, int grad_dtype,
                              const void *const *grads, float *const *errors, float *q, float *p_hat,
                              float *recon, void *stream);

/* Status of the last psgd_step_static call on the current device (no
 * counterpart in the pages): synchronises `stream`, then reads the status
 * word at the head of the static array.  PSGD_OK, PSGD_ERR_TIMEOUT when a
 * bounded wait of a kernel of that call ran out, PSGD_ERR_DEVICE when one
 * found a reduction counter inconsistent (what calls that overlap on the
 * GPU produce: their results are then wrong), or PSGD_ERR_CUDA.  Allocates
 * nothing. */
PSGD_API int psgd_step_static_status(void *stream);

/* Distributed step.  On a real data-parallel job every rank (GPU) holds
 * its own workers (the context's `workers`, usually 1) and the two means of
 * the step are all-reduces ("anthology-of-the-sota" note-152, "Method": P
 * and then Q are all-reduced across workers).  The step is split at those
 * two points so that the caller can run any all-reduce (e.g. NCCL, SUM over
 * float64) between the calls:
 *
 *   psgd_dist_p:      M_w = G_w + E_w for the local workers; p_send =
 *                     sum over local workers of M_w Q (per layer m x R rows,
 *                     float64, R = rank rounded up to a power of two).
 *   (caller)          p_sum = all-reduce(p_send, SUM)
 *   psgd_dist_q:      P_bar = p_sum / W_global, Gram + Cholesky, P_hat;
 *                     q_send = sum over local workers of M_w^T P_hat (n x R rows).
 *   (caller)          q_sum = all-reduce(q_send, SUM)
 *   psgd_dist_finish: Q_bar = q_sum / W_global into q; E'_w for the local
 *                     workers (eager mode) and recon if it was given.
 *
 * psgd_dist_p takes the step's pointers (same meaning as psgd_step); the
 * other two only the reduced buffers.  psgd_dist_sizes gives the float64
 * element counts of p_send/p_sum and q_send/q_sum; psgd_set_global_workers
 * sets W_global (default: the context's own worker count).  Calls out of
 * order return PSGD_ERR_STATE; power iterations > 1 and SVD refresh are
 * not available in the distributed step.  p_sum may alias p_send and q_sum
 * q_send (in-place all-reduce). */
PSGD_API int psgd_set_global_workers(psgd_ctx *ctx, int total_workers);
PSGD_API int psgd_dist_sizes(const psgd_ctx *ctx, size_t *p_elems, size_t *q_elems);
PSGD_API int psgd_dist_p(psgd_ctx *ctx, const void *const *grads, float *const *errors, float *const *q,
                         float *const *p_hat, float *const *recon, double *p_send, void *stream);
PSGD_API int psgd_dist_q(psgd_ctx *ctx, const double *p_sum, double *q_send, void *stream);
PSGD_API int psgd_dist_finish(psgd_ctx *ctx, const double *q_sum, void *stream);

/* Power (subspace) iterations per step, 1 <= iters <= 8 (default 1; the
 * "PowerSGD" glossary page: one or two suffice).  Every iteration repeats
 * P = M Q, mean, orthogonalisation, Q = M^T P_hat, mean, the next one
 * starting from the Q_bar just formed; the residual uses the last
 * iteration's factors.  Later iterations read M (already formed) instead of
 * G and E, so each costs one more read of M for P and one for Q. */
PSGD_API int psgd_set_power_iters(psgd_ctx *ctx, int iters);

/* PowerSGD+ periodic SVD refresh ("From PowerSGD to PowerSGD+", Abstract:
 * the projection subspace is periodically re-aligned with the optimal one
 * through a singular value decomposition).  With every > 0, every step
 * whose number (1, 2, ...) is a multiple of `every` replaces the step's
 * factors by the rank-r truncated SVD of the worker mean M_bar:
 * P_hat = U_r, Q_bar = V_r Sigma_r (singular vectors up to sign), and the
 * residual is taken against it.  The SVD is computed by subspace iteration
 * on an oversampled block of r' = r + p columns (p from
 * psgd_set_svd_oversampling, default 8; r' capped by 32 and by the smallest
 * side of every layer; Halko, Martinsson and Tropp, SIAM Review 2011,
 * section 4.5), started from [warm-start Q | fresh N(0, 1) draws] (the
 * psgd_init_q generator with draw index 2^62 + step number), followed by a
 * Rayleigh-Ritz rotation: C = Q_bar^T Q_bar = W Lambda W^T (Jacobi, float64,
 * eigenvalues descending, each column of W signed so that its
 * largest-magnitude entry is positive), of which the top r directions are
 * kept.  The top-r subspace converges as (sigma_{r'+1} / sigma_r)^(2 J) in
 * J iterations; each layer stops once the estimate of that factor from the
 * orthogonalisation's Cholesky diagonal, (lambda_{r'} / lambda_r)^(J - 1),
 * is at most 1e-10, and after `iters` iterations at most (1 <= iters <= 64).
 * every = 0 turns refresh off (the default).  A refresh step makes
 * 3 * iters + 2 launches, + 1 for the residual pass (eager mode, or when
 * G_hat is wanted), + 1 in lazy mode to write out the previous E' first; a
 * converged layer's later iterations return at once.  With oversampling 0
 * (or when no column can be added) the block is the rank-r factors
 * themselves: `iters` iterations from the warm start, the rotation in
 * place, 3 * (iters - power_iters) + 1 more launches than a regular step. */
PSGD_API int psgd_set_svd_refresh(psgd_ctx *ctx, int every, int iters);

/* Oversampling p of the refresh block above, 0 <= p <= 31 (default 8).  The
 * context holds a second workspace of rank r + p while refresh is on. */
PSGD_API int psgd_set_svd_oversampling(psgd_ctx *ctx, int extra);

/* Per-kernel timing of psgd_step, for measurement: with enable != 0 every
 * later psgd_step records CUDA events (on its stream) around each of its
 * kernel launches.  psgd_profile_read synchronises on those events, writes
 * the summed device milliseconds of the first pass (error feedback + P),
 * the second pass (P_hat and Q, plus every later power iteration) and the third pass
 * (residual / decompression, 0 in lazy mode) to ms[0..2] and the number of recorded steps to *steps, and
 * clears the record.  Recording adds six event records per step.  The
 * distributed calls are recorded too (pass A in psgd_dist_p; the
 * orthogonalisation and pass B in psgd_dist_q; Q_bar and pass C in
 * psgd_dist_finish; the caller's all-reduces in between are not counted). */
PSGD_API int psgd_profile_enable(psgd_ctx *ctx, int enable);
PSGD_API int psgd_profile_read(psgd_ctx *ctx, double *ms, int *steps);

/* Last error message of the context ("" if none); ctx may be NULL for
 * errors of psgd_create. */
PSGD_API const char *psgd_last_error(const psgd_ctx *ctx);

#ifdef __cplusplus
}
#endif

#endif /* PSGD_H */
