/*
 * shampoo.h - C ABI of the blocked Shampoo optimizer step on one NVIDIA B200
 * (sm_100a).  Library: libshampoo.so (shampoo_family_second_b200/).
 *
 * What it computes ("Shampoo optimizer" notes, "Key Components" and the
 * simplified matrix-case listing; podcast transcript "Preconditioned
 * optimization without the full matrix cost", cues 20-28; DASH abstract):
 * every weight W (m x n) is cut into B x B blocks (ragged edges zero-padded),
 * and for every block, each step,
 *     L <- beta L + G G^T,   R <- beta R + G^T G              (statistics)
 *     XL = (L + eps I)^{-1/p},  XR = (R + eps I)^{-1/p}      (every refresh_every steps)
 *     W <- W - lr * XL G XR                                  (update)
 * with p = 4 by default (the notes' -1/4 powers) and p = 2 allowed (SOAP
 * abstract: Shampoo with the 1/2 power).  The roots come from an iterative
 * solver (coupled Newton with a first- or second-degree correction, Newton-DB
 * or Chebyshev) on scaled, damped statistics (coupled Newton: the smaller of the
 * Frobenius norm and 1.25 x a power-iteration estimate of the largest
 * eigenvalue; the others: the Frobenius norm).  All products run on the tensor cores as 3xTF32 (fp32-accurate)
 * tcgen05 MMAs.
 *
 * Conventions (all entry points):
 *  - Ownership: the caller owns every device buffer (weights, gradients,
 *    state, scratch, inputs, outputs).  The library never allocates device
 *    memory; it owns only the small host-side handle.
 *  - Streams: work is enqueued on the caller's cudaStream_t, passed as void*
 *    (NULL = legacy default stream).  shampoo_step and inv_root_batched never
 *    synchronise the host.
 *  - Errors: argument errors return a negative SHAMPOO_ERR_* code before any
 *    work is enqueued; shampoo_last_error() describes the last one on the
 *    calling thread.  Conditions found on the device (non-finite values,
 *    no convergence, a bounded wait that timed out) are OR-ed as
 *    SHAMPOO_DEVFLAG_* bits into a device status word (see shampoo_get_status
 *    and the d_status argument of inv_root_batched).
 *  - Layout: matrices are row-major fp32 unless stated.  Stacks are
 *    (batch, n, n), matrices back to back.
 *  - Thread safety: a handle is not thread-safe; separate handles are
 *    independent.  The profiling counters are process-wide.
 */
#ifndef SHAMPOO_B200_H
#define SHAMPOO_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SHAMPOO_API __attribute__((visibility("default")))
#else
#define SHAMPOO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
enum {
  SHAMPOO_OK = 0,
  SHAMPOO_ERR_INVALID_ARG = -1, /* bad pointer, size, shape or config value */
  SHAMPOO_ERR_UNSUPPORTED = -2, /* valid but not supported (e.g. alignment) */
  SHAMPOO_ERR_WORKSPACE = -3,   /* state or scratch smaller than required */
  SHAMPOO_ERR_CUDA = -4,        /* a CUDA runtime call failed */
  SHAMPOO_ERR_DEVICE = -5       /* get_status: the device status word is non-zero */
};

/* Device status bits (OR-ed into the status word by the kernels). */
enum {
  SHAMPOO_DEVFLAG_NONFINITE = 1,     /* a NaN or Inf was produced */
  SHAMPOO_DEVFLAG_NOT_CONVERGED = 2, /* tol > 0 and a residual stayed above tol after iters */
  SHAMPOO_DEVFLAG_TIMEOUT = 4,       /* a bounded on-chip wait gave up (kernel unwound) */
  SHAMPOO_DEVFLAG_STAGNATED = 8      /* tol > 0 and a residual stopped improving above tol once every
                                        eigenvalue above fp32 resolution had converged (the fp32 floor
                                        of a rank-deficient or ill-conditioned matrix); stopped there */
};

/* Inverse-root solvers (DASH abstract names Newton-DB and Chebyshev). */
enum {
  SHAMPOO_SOLVER_NEWTON = 0,    /* coupled Newton for A^{-1/p} (Guo & Higham 2006) */
  SHAMPOO_SOLVER_NEWTON_DB = 1, /* coupled Y/Z square-root iteration, twice for p = 4 */
  SHAMPOO_SOLVER_CHEBYSHEV = 2, /* Chebyshev interpolant of x^{-1/p}, Clenshaw evaluation */
  SHAMPOO_SOLVER_NEWTON_CUBIC = 3, /* coupled Newton with the degree-2 binomial correction
                                     T = I + (I-M)/p + (p+1)(I-M)^2/(2p^2) after a plain first
                                     step: one more GEMM per iteration, cubic local convergence,
                                     about a third fewer iterations */
  SHAMPOO_SOLVER_NEWTON_CUBIC_F64 = 4 /* the same iteration (scale, damping, stopping rule) with
                                     fp64 iterates on the fp64 tensor-core instruction: the
                                     root of the damped input to the last fp32 bit of the
                                     output, for statistics whose condition number puts the
                                     fp32 iterates' error ((1/p) 2^-24 kappa) above tolerance;
                                     scratch holds fp64 stacks (twice the bytes), and the
                                     products run at the fp64 rate.  In the blocked step it
                                     also keeps L and R in fp64 (their products on the fp64
                                     MMA, the gradients widened exactly; Frobenius scaling;
                                     damping floor n 2^-53 ||L + eps I||_F): with fp32
                                     statistics the update's error floor would stay that of
                                     fp32 rounding whatever the iterates' precision */
};

/* Gradient element types. */
enum { SHAMPOO_F32 = 0, SHAMPOO_BF16 = 1 };

/* Profiler kernel kinds (shampoo_profile_read). */
enum {
  SHAMPOO_KERNEL_GEMM = 0,     /* tensor-core GEMM (stats, roots, apply) */
  SHAMPOO_KERNEL_STACK = 1,    /* partition / stack of the gradient blocks */
  SHAMPOO_KERNEL_NORM = 2,     /* Frobenius norms of the damped statistics */
  SHAMPOO_KERNEL_PROLOGUE = 3, /* damping + scaling + first iterate */
  SHAMPOO_KERNEL_CHECK = 4,    /* residual check */
  SHAMPOO_KERNEL_FINALIZE = 5, /* unscale + output */
  SHAMPOO_KERNEL_CHEB_COEF = 6,/* Chebyshev coefficients */
  SHAMPOO_KERNEL_SCALE = 7,    /* power-iteration spectral scale (coupled Newton) */
  SHAMPOO_KERNEL_MIRROR = 8,   /* lower triangle of symmetric statistics from the upper */
  SHAMPOO_KERNEL_EIGEN = 9,    /* Jacobi sweeps of the eigensolver */
  SHAMPOO_KERNEL_GEMM_F64 = 10,/* fp64 GEMM of the fp64-iterate solver */
  SHAMPOO_KERNEL_PERMUTE = 11, /* tensor Shampoo: unfoldings and mode products' permutes */
  SHAMPOO_KERNEL_GRAM = 12,    /* tensor Shampoo: split-K statistics of short modes */
  SHAMPOO_KERNEL_DIAG = 13,    /* tensor Shampoo: the diagonal variant's sums, roots and scaling */
  SHAMPOO_KERNEL_SOAP = 14,    /* SOAP: Adam in the eigenbasis, basis transposes, carry-over */
  SHAMPOO_KERNEL_KINDS = 15
};

/* Hyper-parameters of the blocked step.
 *  block          B: multiple of 32 in [32, 1024].
 *  beta           statistics decay (beta = 1: plain running sum as in the notes' listing).
 *  eps            damping: roots of (L + eps I); >= 0.
 *  lr             learning rate eta.
 *  root_p         2 or 4.
 *  solver         SHAMPOO_SOLVER_*.
 *  iters          iterations (tol = 0) or iteration cap (tol > 0) per Newton / Newton-DB
 *                 stage, >= 1; ignored by Chebyshev.  NEWTON_CUBIC behaves as NEWTON here.
 *  tol            0: fixed iteration count; > 0: stop a matrix once
 *                 |tr(I - M)|/n (Newton) or |tr(I - Z Y)|/n (Newton-DB) <= tol.  The
 *                 iterations keep every eigenvalue of M (or Z Y) at or below 1, so this trace
 *                 bounds the largest eigenvalue error (times n).  A matrix whose residual
 *                 stops improving once every eigenvalue above fp32 resolution has converged
 *                 stops there (SHAMPOO_DEVFLAG_STAGNATED).
 *  refresh_every  roots recomputed at steps t with t % refresh_every == 0 (t from 0), >= 1.
 *  cheb_degree    Chebyshev degree d in [2, 64].
 *  cheb_lo        Chebyshev interval: [lo / s, 1] with lo = cheb_lo if > 0 else eps,
 *                 s = ||A + eps I||_F.
 *  grad_dtype     SHAMPOO_F32 or SHAMPOO_BF16 (weights and statistics are always fp32).
 *  momentum       alpha in [0, 1): 0 = off (the update uses the raw gradient); > 0 keeps a
 *                 per-block momentum M <- alpha M + G (from M = 0) ahead of the preconditioner,
 *                 and the update becomes W <- W - lr XL M XR, while the statistics still take
 *                 the raw G (podcast transcript, cue 28: momentum 0.9 before preconditioning).
 *  diag_threshold tensor Shampoo only (the blocked step's blocks never exceed 1024): a
 *                 dimension longer than this keeps only the diagonal of its statistic
 *                 (podcast transcript, cue 28: diagonal variant past a size threshold,
 *                 decided per dimension).  <= 0: 1024, the largest root the solvers
 *                 compute; at most 1024. */
typedef struct {
  int32_t block;
  float beta;
  float eps;
  float lr;
  int32_t root_p;
  int32_t solver;
  int32_t iters;
  float tol;
  int32_t refresh_every;
  int32_t cheb_degree;
  float cheb_lo;
  int32_t grad_dtype;
  float momentum;
  int32_t diag_threshold;
} shampoo_config;

typedef struct shampoo_ctx* shampoo_handle;

/* Human-readable name of a return code or device status word.  Never NULL. */
SHAMPOO_API const char* shampoo_status_string(int code);

/* Description of the last error returned on the calling thread ("" if none). */
SHAMPOO_API const char* shampoo_last_error(void);

/* Sizes of the caller-owned device buffers for a parameter set.
 * rows[i] x cols[i] is the shape of weight i (nparams in [1, 1024]).
 * state_bytes: persistent state (statistics, roots, block table, status word).
 * scratch_bytes: per-step scratch (stacked gradient blocks, solver iterates).
 * Host-only; no CUDA call.  Source: the notes' "Key Components" (one m x m and
 * one n x n preconditioner per block: O(m^2 + n^2) memory). */
SHAMPOO_API int shampoo_query_sizes(const shampoo_config* cfg, int32_t nparams, const int64_t* rows, const int64_t* cols,
                        size_t* state_bytes, size_t* scratch_bytes);

/* Create a handle over caller-owned state and scratch (device pointers,
 * 256-byte aligned, at least the queried sizes).  Zeroes the statistics
 * (the notes' listing initialises L and R; eps enters as damping, see
 * shampoo_config.eps), uploads the block table (stream-ordered on `stream`)
 * and sets the step counter to 0. */
SHAMPOO_API int shampoo_init(const shampoo_config* cfg, int32_t nparams, const int64_t* rows, const int64_t* cols,
                 void* d_state, size_t state_bytes, void* d_scratch, size_t scratch_bytes, void* stream,
                 shampoo_handle* out);

/* One optimizer step (the notes' loop body, for every block): accumulate the
 * statistics from the gradients, recompute the roots if step % refresh_every
 * == 0, then W <- W - lr XL G XR in place.  d_weights[i]: fp32 row-major
 * rows[i] x cols[i]; d_grads[i]: same shape, grad_dtype.  Both are host arrays
 * of nparams device pointers.  Enqueued on `stream`; no host sync. */
SHAMPOO_API int shampoo_step(shampoo_handle h, float* const* d_weights, const void* const* d_grads, void* stream);

/* shampoo_step on strided views: ld (host, nparams entries; NULL = cols) gives
 * the row stride, in elements, of d_weights[i] and d_grads[i] alike (cols[i] <=
 * ld[i] < 2^31).  A parameter can then be a sub-matrix of a larger weight, e.g.
 * the blocks one rank owns when the blocks are sharded across ranks.
 * SHAMPOO_ERR_INVALID_ARG for a stride out of range; rows need no alignment
 * (unaligned rows take the scalar load path). */
SHAMPOO_API int shampoo_step_strided(shampoo_handle h, float* const* d_weights, const void* const* d_grads,
                                     const int64_t* ld, void* stream);

/* Synchronises the handle's last stream, reads the device status word into
 * *status (0 = clean; else SHAMPOO_DEVFLAG_* bits) and returns SHAMPOO_OK, or
 * SHAMPOO_ERR_CUDA if the device reported an error.  reset != 0 clears the word. */
SHAMPOO_API int shampoo_get_status(shampoo_handle h, int32_t* status, int32_t reset);

/* Block table: *nb blocks; if table != NULL it receives nb rows of
 * {param, row0, col0, rows, cols} (int64, host memory), in stack order
 * (param, block row, block column).  DASH abstract: blocks stacked into 3D tensors. */
SHAMPOO_API int shampoo_block_table(shampoo_handle h, int32_t* nb, int64_t* table);

/* Device pointers into the state (owned by the caller's state buffer):
 * L: plain stack (nb, B, B) of left statistics; R: (nb, B, B) right statistics
 * (fp32; fp64 values behind the float pointers when cfg.solver is
 * SHAMPOO_SOLVER_NEWTON_CUBIC_F64); rootL / rootR: (nb, B, B) fp32 stacks of
 * XL and XR; *step: steps taken.
 * Ragged blocks hold zeros outside their r x r / c x c valid region.
 * The statistics are symmetric, and a step updates only their tiles on or
 * above the diagonal (every element (i, j) with j >= i, and the diagonal
 * tiles whole); the rest is copied from its transpose on refresh steps only,
 * since only the roots read it.  Between refreshes, call
 * shampoo_sync_statistics before reading L or R as full matrices.  A saved
 * and restored state needs no sync: the next refresh fills the rest again.
 * The apply products read the roots in split forms derived from them after
 * every refresh (XL as bf16 planes, XR as tf32 hi and lo parts, in the
 * scratch); roots written through these pointers take effect after
 * shampoo_set_step, which has the forms derived again before the next
 * apply. */
SHAMPOO_API int shampoo_state_views(shampoo_handle h, float** L, float** R, float** rootL, float** rootR, int64_t* step);

/* Fills the part of every statistics matrix below its diagonal tiles from
 * the transpose of the part above (one pass over the L and R stacks),
 * enqueued on `stream`: reads of L and R ordered after it see the full
 * symmetric matrices.  No-op where every tile is computed: fp32 statistics
 * with B <= 256 (one tile column of 256), fp64 statistics with B <= 64 (one
 * tile of 64).  Statistics as in the
 * notes' matrix-case listing (L = sum G G^T, R = sum G^T G, both symmetric).
 * SHAMPOO_ERR_INVALID_ARG for a NULL handle; SHAMPOO_ERR_CUDA if the launch
 * fails. */
SHAMPOO_API int shampoo_sync_statistics(shampoo_handle h, void* stream);

/* Device pointer to the momentum stack (nb, B, B) fp32 in the state (zero
 * outside each block's r x c region), or NULL when momentum is off. */
SHAMPOO_API int shampoo_momentum_view(shampoo_handle h, float** M);

/* Sets the step counter (checkpoint resume: restore the state buffer bytes,
 * then the counter).  The next step first derives the apply products' split
 * forms of the roots again (see shampoo_state_views). */
SHAMPOO_API int shampoo_set_step(shampoo_handle h, int64_t step);

/* Frees the host-side handle (the caller's device buffers are untouched). */
SHAMPOO_API void shampoo_destroy(shampoo_handle h);

/* Scratch bytes inv_root_batched needs to solve all `batch` matrices in one
 * pass, for p = 2 or 4.  Less (but at least the size for one matrix plus
 * 64 KiB) makes it work through the batch in chunks.  Host-only. */
SHAMPOO_API int inv_root_scratch_bytes(int64_t batch, int32_t n, int32_t solver, size_t* bytes);

/* inv_root_scratch_bytes for a given root order p in {2, 4, 6, 8}: coupled
 * Newton with p = 6 or 8 keeps one more n x n iterate per matrix (T^p).
 * Host-only. */
SHAMPOO_API int inv_root_scratch_bytes_p(int64_t batch, int32_t n, int32_t solver, int32_t p, size_t* bytes);

/* Batched inverse p-th roots: X_i ~ (A_i + eps I)^{-1/p} for symmetric
 * positive semi-definite A_i (the notes' L^{-1/4}, R^{-1/4}; SOAP abstract's
 * p = 2).  DASH abstract: batched inverse-root solvers with matrix scaling.
 *  d_A, d_X      device plain stacks (batch, n, n); n a multiple of 32 in [32, 1024].
 *                A is symmetrised ((A + A^T)/2) before use.
 *  p             2 or 4; also 6 or 8 (order-3 and order-4 tensor Shampoo's -1/(2k)
 *                powers, podcast cue 26) with coupled Newton and Chebyshev.
 *                eps  damping >= 0.
 *  solver, iters, tol, cheb_degree, cheb_lo   as in shampoo_config.
 *  d_scratch     device scratch, 256-byte aligned (see inv_root_scratch_bytes).
 *  d_iters_used  nullable device int32[batch]: iterations run per matrix
 *                (Newton-DB p = 4: both stages; Chebyshev: the degree); negative
 *                when tol > 0 and the residual did not reach tol (cap reached:
 *                SHAMPOO_DEVFLAG_NOT_CONVERGED; stagnated: SHAMPOO_DEVFLAG_STAGNATED).
 *  d_status      nullable device int32: OR of SHAMPOO_DEVFLAG_* (not cleared).
 *  stream        cudaStream_t as void*.  Enqueued; no host sync. */
SHAMPOO_API int inv_root_batched(const float* d_A, float* d_X, int64_t batch, int32_t n, int32_t p, float eps, int32_t solver,
                     int32_t iters, float tol, int32_t cheb_degree, float cheb_lo, void* d_scratch,
                     size_t scratch_bytes, int32_t* d_iters_used, int32_t* d_status, void* stream);

/* inv_root_batched for callers that cannot allocate device memory (no
 * counterpart on the pages: an addition of this library).  Some callers may
 * not call cudaMalloc at all, e.g. code running inside a memory-pool region
 * that forbids allocation, a real-time loop that must not block on the
 * allocator, or an embedding without an allocator.  This entry point takes the
 * solver's scratch from a fixed 32 MiB device array inside the library (held
 * on every GPU that loads the library until the process exits) and allocates
 * nothing; inputs and outputs are still the caller's, with the same meaning as
 * in inv_root_batched.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress) and should come before any stream capture.
 * All calls share the array: calls whose work overlaps on the GPU (other
 * streams or host threads on the same device) race on it.  The solver clears
 * what must start at zero on every call.  Batches larger than the array are
 * solved in chunks (the largest need of the fp32 solvers at p <= 4, coupled
 * Newton at n = 1024, is 28 MiB per matrix); a size whose scratch for one
 * matrix exceeds the array (p = 6, 8 at n = 1024; fp64 iterates from n = 800)
 * returns SHAMPOO_ERR_UNSUPPORTED.  With tol > 0 the iterations are plain
 * kernel launches up to the cap (tiles of finished matrices exit at once),
 * never a CUDA graph, whose instantiation may take device memory; results
 * equal inv_root_batched's. */
SHAMPOO_API int inv_root_batched_noalloc(const float* d_A, float* d_X, int64_t batch, int32_t n, int32_t p, float eps,
                                         int32_t solver, int32_t iters, float tol, int32_t cheb_degree,
                                         float cheb_lo, int32_t* d_iters_used, int32_t* d_status, void* stream);

/* Order-k tensor Shampoo (podcast transcript "Preconditioned optimization
 * without the full matrix cost", cue 26): for a parameter of order k in
 * [2, 4] with dimensions d_0 .. d_{k-1} (each in [1, 2^20]), one statistic per
 * dimension,
 *     H_i <- beta H_i + G_(i) G_(i)^T      (G_(i): mode-i unfolding of G, the
 *                                           other indices in row-major order)
 *     X_i = (H_i + eps I)^{-1/(2k)}        (every refresh_every steps)
 *     W <- W - lr  G x_0 X_0 x_1 X_1 ... x_{k-1} X_{k-1}
 * (x_i: contraction along dimension i).  The parameters are not blocked.  A
 * dimension longer than cfg.diag_threshold keeps the diagonal h_i of H_i
 * (cue 28's diagonal variant) and scales its dimension by
 * d_i = (h_i + eps)^{-1/(2k)} (0 where h_i + eps = 0).
 * Config fields used: beta, eps, lr, solver (coupled Newton either degree,
 * Chebyshev; Newton-DB for order 2 only), iters, tol, refresh_every,
 * cheb_degree, cheb_lo, grad_dtype, diag_threshold; block and root_p are
 * ignored, momentum must be 0.  orders[j] is the order of parameter j; dims holds all
 * parameters' dimensions back to back.  Weights are fp32 and gradients
 * grad_dtype, both row-major (natural layout), device pointers in host
 * arrays.  Ownership, streams and errors as for shampoo_init / shampoo_step;
 * nparams in [1, 256]. */
typedef struct shampoo_tensor_ctx* shampoo_tensor_handle;
SHAMPOO_API int shampoo_tensor_query_sizes(const shampoo_config* cfg, int32_t nparams, const int32_t* orders,
                                           const int64_t* dims, size_t* state_bytes, size_t* scratch_bytes);
SHAMPOO_API int shampoo_tensor_init(const shampoo_config* cfg, int32_t nparams, const int32_t* orders,
                                    const int64_t* dims, void* d_state, size_t state_bytes, void* d_scratch,
                                    size_t scratch_bytes, void* stream, shampoo_tensor_handle* out);
SHAMPOO_API int shampoo_tensor_step(shampoo_tensor_handle h, float* const* d_weights, const void* const* d_grads,
                                    void* stream);
/* Device pointers to the statistic H_i and root X_i of mode `mode` of
 * parameter `param`: npad x npad fp32 (npad = d_i rounded up to 32; zero /
 * identity-scaled beyond d_i), or, when *diagonal = 1, the d_i-vectors h_i and
 * d_i of the diagonal variant (then *npad = d_i); *step: steps taken. */
SHAMPOO_API int shampoo_tensor_views(shampoo_tensor_handle h, int32_t param, int32_t mode, float** H, float** X,
                                     int32_t* npad, int32_t* diagonal, int64_t* step);
/* As shampoo_get_status, for a tensor handle. */
SHAMPOO_API int shampoo_tensor_get_status(shampoo_tensor_handle h, int32_t* status, int32_t reset);
SHAMPOO_API void shampoo_tensor_destroy(shampoo_tensor_handle h);

/* SOAP: Adam run in the eigenbasis of Shampoo's preconditioner (pith.science
 * record of "SOAP: Improving and Stabilizing Shampoo using Adam": abstract
 * and claims; the basis is recomputed every refresh_every steps and kept in
 * between), on the blocks and statistics of the blocked step.  Per block,
 * step t (from 0):
 *     G' = QL^T G QR,  m <- beta1 m + (1 - beta1) G,  v <- beta2 v + (1 - beta2) G'^2,
 *     W <- W - lr QL [ (QL^T m QR / (1 - beta1^{t+1})) / (sqrt(v / (1 - beta2^{t+1})) + eps) ] QR^T,
 *     L <- beta L + G G^T,  R <- beta R + G^T G,
 *     if t % refresh_every == 0: QL, QR <- eigenbases of L, R (the identity before the
 *     first refresh), v carried over as (PL o PL) v (PR o PR)^T, P = Q_new^T Q_old.
 * The current gradient never enters its own projection (its rotation would have
 * exact zeros that fp32 turns into rounding noise, which Adam's normalisation
 * amplifies).  The bases come from eigh_batched's method (cyclic Jacobi
 * warm-started from the previous basis, then refine_iters orthogonalisation
 * steps).
 * shampoo_config fields used: block, beta, lr, refresh_every, grad_dtype. */
typedef struct {
  float beta1;            /* Adam first-moment decay, [0, 1) */
  float beta2;            /* Adam second-moment decay, [0, 1) */
  float eps;              /* Adam epsilon, > 0 */
  int32_t jacobi_sweeps;  /* eigensolver: Jacobi sweep cap per refresh, [1, 100] */
  int32_t refine_iters;   /* eigensolver: orthogonalisation steps per refresh, [0, 100] */
} shampoo_soap_config;
typedef struct shampoo_soap_ctx* shampoo_soap_handle;
SHAMPOO_API int shampoo_soap_query_sizes(const shampoo_config* cfg, const shampoo_soap_config* sc, int32_t nparams,
                                         const int64_t* rows, const int64_t* cols, size_t* state_bytes,
                                         size_t* scratch_bytes);
SHAMPOO_API int shampoo_soap_init(const shampoo_config* cfg, const shampoo_soap_config* sc, int32_t nparams,
                                  const int64_t* rows, const int64_t* cols, void* d_state, size_t state_bytes,
                                  void* d_scratch, size_t scratch_bytes, void* stream, shampoo_soap_handle* out);
/* One SOAP step over every block; weights fp32, gradients grad_dtype, both
 * contiguous row-major.  Enqueued on `stream`; no host sync. */
SHAMPOO_API int shampoo_soap_step(shampoo_soap_handle h, float* const* d_weights, const void* const* d_grads,
                                  void* stream);
/* Device views of the state: statistics L, R; bases QL, QR (eigenvectors as
 * columns); m (original coordinates) and v (eigenbasis), each (nb, B, B);
 * *step: steps taken. */
SHAMPOO_API int shampoo_soap_views(shampoo_soap_handle h, float** L, float** R, float** QL, float** QR, float** m,
                                   float** v, int64_t* step);
SHAMPOO_API int shampoo_soap_get_status(shampoo_soap_handle h, int32_t* status, int32_t reset);
SHAMPOO_API void shampoo_soap_destroy(shampoo_soap_handle h);

/* Block packing for blocks sharded across ranks (DASH abstract: the
 * preconditioner blocks are distributed across devices): one launch moves
 * nblocks r x c blocks between row-strided matrices and one packed fp32
 * buffer holding the blocks back to back, each row-major.
 *  d_table     device int64 [nblocks x 6]: {param, row0, col0, r, c, offset},
 *              offset = the block's first float in d_packed.  Every block must
 *              lie inside its matrix and the packed buffer (not checked on the
 *              device).
 *  d_params    host array of nparams device pointers; ld host array of their
 *              row strides in elements (>= 1).
 *  dtype       element type of the matrices: SHAMPOO_F32, or SHAMPOO_BF16 for
 *              a gather (widened exactly).
 *  direction   0: gather, d_packed = scale * block; 1: scatter, block = d_packed
 *              (scale unused; fp32 matrices only).
 *  max_rows, max_cols   largest r and c in the table (they size the grid).
 * nblocks in [0, 65535], nparams in [1, 1024].  Enqueued on `stream`. */
SHAMPOO_API int shampoo_pack_blocks(const int64_t* d_table, int32_t nblocks, int32_t nparams, void* const* d_params,
                                    const int64_t* ld, int32_t dtype, float* d_packed, int32_t direction, float scale,
                                    int32_t max_rows, int32_t max_cols, void* stream);

/* Batched symmetric eigendecomposition A_i = Q_i diag(lam_i) Q_i^T (the
 * eigenbasis SOAP runs Adam in: pith.science SOAP record; the pages name no
 * method).  warm_start = 0: cyclic Jacobi with the round-robin parallel
 * ordering (Golub & Van Loan sec. 8.5) from A_i, at most jacobi_sweeps sweeps
 * (SHAMPOO_DEVFLAG_NOT_CONVERGED if the off-diagonal mass stays above 1e-5 of
 * ||A_i||_F); warm_start = 1: d_Q holds an approximate basis X on entry (e.g.
 * the previous one): Jacobi runs on the nearly diagonal X^T A X and X is
 * rotated by its eigenvectors.  Then refine_iters Newton-Schulz steps toward
 * the nearest orthogonal matrix (Bjorck & Bowie 1971), X <- 1.5 X - 0.5 X X^T X,
 * each squaring X's departure from orthogonality.
 *  d_A       device stack (batch, n, n), symmetrised before use; n a multiple
 *            of 32 in [32, 1024].
 *  d_Q       device stack (batch, n, n): eigenvectors as columns, in no
 *            particular order (Jacobi's); in/out with warm_start = 1.
 *  d_lam     nullable device (batch, n): eigenvalues, matching Q's columns, as
 *            Rayleigh quotients q_j^T A q_j of the final basis.
 *  d_scratch 256-byte aligned, eigh_scratch_bytes(batch, n) for one pass
 *            (less, but at least one matrix's share, works in chunks).
 *  d_status  nullable device int32: OR of SHAMPOO_DEVFLAG_*.
 * Enqueued on `stream`; no host sync. */
SHAMPOO_API int eigh_scratch_bytes(int64_t batch, int32_t n, size_t* bytes);
SHAMPOO_API int eigh_batched(const float* d_A, float* d_Q, float* d_lam, int64_t batch, int32_t n,
                             int32_t warm_start, int32_t jacobi_sweeps, int32_t refine_iters, void* d_scratch,
                             size_t scratch_bytes, int32_t* d_status, void* stream);

/* The batched fp32-accurate product every stage uses, as a utility:
 * D_i = alpha A_i op(B_i) + beta C_i + gamma I for plain stacks (batch, n, n),
 * op(B) = B^T (op_b = 0) or B (op_b = 1);
 * d_C may be NULL (then beta is ignored) and may equal d_D; d_D must not
 * overlap d_A or d_B.  n a multiple of 32 in [32, 4096]; all four 16-byte
 * aligned.  The kernel splits operand tiles into tf32 hi/lo parts on chip and
 * multiplies them as 3xTF32 on the tensor cores.  No scratch is needed
 * (shampoo_gemm_scratch_bytes returns 0; d_scratch may be NULL).  Enqueued on
 * `stream`; no host sync. */
SHAMPOO_API int shampoo_gemm_scratch_bytes(int64_t batch, int32_t n, size_t* bytes);
SHAMPOO_API int shampoo_gemm_batched(const float* d_A, const float* d_B, const float* d_C, float* d_D, int64_t batch, int32_t n,
                         int32_t op_b, float alpha, float beta, float gamma, void* d_scratch, size_t scratch_bytes,
                         int32_t* d_status, void* stream);

/* The fp64 product of the fp64-iterate solver (SHAMPOO_SOLVER_NEWTON_CUBIC_F64),
 * as a utility: D_i = alpha A_i B_i + beta C_i + gamma I for row-major fp64
 * stacks (batch, n, n) on the fp64 tensor-core instruction (mma m8n8k4).
 * d_C may be NULL (then beta is ignored) and may equal d_D; d_D must not
 * overlap d_A or d_B.  n a multiple of 16 in [16, 4096], batch <= 65535, all
 * four 16-byte aligned.  Enqueued on `stream`; no host sync; non-finite outputs
 * raise SHAMPOO_DEVFLAG_NONFINITE in d_status (nullable). */
SHAMPOO_API int shampoo_dgemm_batched(const double* d_A, const double* d_B, const double* d_C, double* d_D,
                                      int64_t batch, int32_t n, double alpha, double beta, double gamma,
                                      int32_t* d_status, void* stream);

/* Profiling (process-wide).  When enabled, every kernel launch of the library
 * is bracketed by CUDA events on its own stream and tallied per kind with its
 * algorithmic flops (GEMM: executed tiles only) and bytes.
 * shampoo_profile_read synchronises the recorded events. */
SHAMPOO_API void shampoo_profile_enable(int32_t on);
SHAMPOO_API void shampoo_profile_reset(void);
SHAMPOO_API int shampoo_profile_read(int32_t kind, int64_t* launches, double* total_ms, double* alg_flops, double* alg_bytes);

/* Number of kernels this library has launched in this process, including
 * the kernels that residual-checked solver loops ran inside CUDA graphs
 * (counted on the device; once such a loop has run, this call waits for the
 * device). */
SHAMPOO_API uint64_t shampoo_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SHAMPOO_B200_H */
