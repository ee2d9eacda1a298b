/*
 * libmuon -- the Muon weight update on NVIDIA B200 (sm_100a).
 *
 * What is computed (per 2-D weight matrix W of shape rows x cols):
 *   M <- beta*M + G                      momentum buffer, fp32, updated in place
 *                                        (G pre-scaled by hparams.grad_scale)
 *   U  = G + beta*M                      Nesterov look-ahead (U = M without it)
 *   X0 = U / (||U||_F + eps)             Frobenius normalisation
 *   X  = X0 or X0^T so that X is wide    (m = min(rows, cols) rows)
 *   k times:  A = X X^T;  B = b_i A + c_i A A;  X <- a_i X + B X
 *   O  = X (transposed back if needed)
 *   W <- W (1 - lr*wd) - lr * s(rows, cols) * O     decoupled weight decay
 *
 * Source: "Muon Meets Mamba: Spectral Optimization for State Space Models"
 * (arXiv 2608.03941), abstract: Muon orthogonalises the update to each weight
 * matrix with a Newton-Schulz iteration (steepest descent under the spectral
 * norm) and is applied per weight group (input / output projection) of
 * Mamba-2 130M.  "MuonSSM: Orthogonalizing State Space Models", section on the
 * lightweight Newton-Schulz step: no explicit SVD, matrix products only.
 * The pages leave the coefficients, iteration count, momentum convention,
 * normalisation, shape scale and decay order open; this library takes the
 * readings above and makes the coefficients and k a runtime table.
 *
 * Conventions for every entry point:
 *   - Matrices are dense, row-major (PyTorch contiguous), on the context's
 *     device.  Pointer ARRAYS (W, G, M, X, Out) are HOST arrays of `batch`
 *     DEVICE pointers; every matrix of one call has the same rows x cols.
 *   - The caller owns W, G, M, X and Out and the stream.  The context owns its
 *     workspace (grown on first use of a larger shape, then reused), a device
 *     status word and per-matrix flags.
 *   - Calls are asynchronous and stream-ordered on `stream` (a cudaStream_t;
 *     NULL = legacy default stream).  Argument errors are returned
 *     synchronously before anything is enqueued; device-side conditions
 *     (non-finite norm, a kernel wait that ran out) are reported by
 *     muon_get_status() after the stream has been synchronised.
 *   - Two calls on the same context must not run concurrently on different
 *     streams: they share the workspace.  A context is used from one host
 *     thread at a time; separate contexts are independent.
 *   - Work a call puts on the context's internal streams (the uploads of
 *     muon_step_groups_host) starts after what is already queued on `stream`
 *     and joins back into `stream` before the call's last kernel.
 *   - CUDA graphs: muon_step_groups, muon_step_capped, muon_ns_orthogonalize,
 *     muon_power_iteration and muon_min_singular queue only memsets and
 *     kernel launches once the context's buffers are large enough, so they
 *     may be captured on `stream` and the graph replayed, as long as the
 *     pointers and sizes stay the same.  The first call of a shape grows
 *     them, which synchronises the device: made while `stream` is capturing,
 *     such a call returns MUON_ERR_ALLOC before queuing anything and leaves
 *     the capture intact (muon_last_cuda_error says why).  (One exception:
 *     when the device refuses a spectral call's cooperative launch, e.g. with
 *     another client holding SMs, a counter reset may already be queued
 *     before its fallback finds it must grow.)  Make the same call once
 *     before capture.  A graph keeps the addresses of the
 *     context's buffers, so once any call of a context has been captured the
 *     context never grows again: a later call that would need more returns
 *     MUON_ERR_ALLOC (use another context for it).  muon_step_groups_host
 *     and muon_get_status synchronise and cannot be captured.
 *   - No C++ exception crosses this interface.
 */
#ifndef LIBMUON_MUON_H
#define LIBMUON_MUON_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MUON_ABI_VERSION 2

/* Largest number of Newton-Schulz iterations a coefficient table may hold. */
#define MUON_MAX_ITERS 32
/* Largest batch handled by one group descriptor; larger groups are split by the caller. */
#define MUON_MAX_BATCH 256
/* Largest number of groups in one muon_step_groups call. */
#define MUON_MAX_GROUPS 8

typedef enum {
  MUON_OK = 0,
  MUON_ERR_INVALID_ARG = 1,      /* null pointer, batch/rows/cols out of range, bad hparams   */
  MUON_ERR_UNSUPPORTED_SHAPE = 2,/* min(rows, cols) or max(rows, cols) beyond the limits      */
  MUON_ERR_DTYPE = 3,            /* dtype not MUON_BF16 / MUON_F32                            */
  MUON_ERR_CUDA = 4,             /* a CUDA runtime call failed (see muon_last_cuda_error)     */
  MUON_ERR_NONFINITE = 5,        /* device: ||U||_F was not finite for >= 1 matrix            */
  MUON_ERR_TIMEOUT = 6,          /* device: a bounded wait inside a kernel ran out            */
  MUON_ERR_NO_DEVICE = 7,        /* no usable CUDA device / device is not sm_100              */
  MUON_ERR_ALLOC = 8             /* workspace allocation failed, or refused while capturing  */
} muon_status;

typedef enum { MUON_BF16 = 0, MUON_F32 = 1 } muon_dtype;

typedef enum {
  MUON_SCALE_SQRT_RATIO = 0, /* s = sqrt(max(1, rows/cols))  (default)  */
  MUON_SCALE_NONE = 1,       /* s = 1                                   */
  MUON_SCALE_RMS_MATCH = 2   /* s = 0.2 * sqrt(max(rows, cols))         */
} muon_scale_mode;

/* Per-matrix flag bits reported by muon_get_status. */
#define MUON_FLAG_NONFINITE 1 /* ||U||_F or 1/(||U||_F+eps) not finite: W left unchanged, M updated */

typedef struct {
  float lr;           /* learning rate (> 0 not required; any finite value)          */
  float beta;         /* momentum coefficient, finite                                  */
  float weight_decay; /* decoupled decay, applied as W *= (1 - lr*weight_decay)        */
  float eps;          /* added to ||U||_F before dividing, >= 0                        */
  int nesterov;       /* 1: U = G + beta*M (after the buffer update); 0: U = M         */
  int scale_mode;     /* muon_scale_mode                                               */
  float grad_scale;   /* G is read as grad_scale*G (finite, > 0; 1 = as given).  A data- */
                      /* parallel caller that reduce-scattered the SUM of N ranks'      */
                      /* gradients passes 1/N to step on their average, with no extra   */
                      /* pass over G.  0 (a struct from an older caller) is rejected.   */
} muon_hparams;

/* One group of same-shape matrices for muon_step_groups. */
typedef struct {
  void* const* W;       /* host array of `batch` device pointers, rows x cols, `dtype` */
  const void* const* G; /* host array of `batch` pointers (device, or pinned host for   */
                        /*   muon_step_groups_host), rows x cols, `dtype`               */
  float* const* M;      /* host array of `batch` device pointers, rows x cols, fp32     */
  int batch;            /* 1 .. MUON_MAX_BATCH                                          */
  int rows, cols;       /* 1 .. 32768 each, min(rows, cols) <= 8192                     */
  int dtype;            /* muon_dtype of W and G                                        */
} muon_group;

typedef struct muon_ctx muon_ctx;

/* Version of this interface (MUON_ABI_VERSION of the build). */
int muon_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* muon_status_string(muon_status s);

/* Text of the last CUDA error seen by any context in this process (static buffer). */
const char* muon_last_cuda_error(void);

/* Create a context on CUDA device `device` (must be compute capability 10.x).
 * The default coefficient table is 5 quintic iterations (3.4445, -4.7750, 2.0315). */
muon_status muon_create(muon_ctx** ctx, int device);

/* Free the context and its workspace.  Synchronises the device first.  NULL is accepted. */
muon_status muon_destroy(muon_ctx* ctx);

/* Set the Newton-Schulz coefficient table: `abc` is a HOST array of k triples
 * (a_i, b_i, c_i), iteration i uses triple i.  1 <= k <= MUON_MAX_ITERS.
 * Values must be finite.  Takes effect for calls enqueued afterwards. */
muon_status muon_set_coeffs(muon_ctx* ctx, const float* abc, int k);

/* Copy the current table into `abc` (capacity 3*MUON_MAX_ITERS floats) and its length into *k. */
muon_status muon_get_coeffs(const muon_ctx* ctx, float* abc, int* k);

/* One Muon step for `batch` same-shape matrices (see the top of this file).
 * W: rows x cols of `dtype` (bf16 or fp32), updated in place.
 * G: rows x cols of `dtype`, read only.
 * M: rows x cols fp32, updated in place (start from zeros).
 * bf16: operands of the matrix products are bf16 with fp32 accumulation.
 * fp32: operands are split into three bf16 planes (hi + mid + lo, ~24-bit
 *       mantissa) and six plane products are accumulated in fp32. */
muon_status muon_step(muon_ctx* ctx, void* const* W, const void* const* G, float* const* M,
                      int batch, int rows, int cols, int dtype, const muon_hparams* hp,
                      void* stream);

/* muon_step over several groups (e.g. every in_proj and every out_proj of a
 * model) in one call; the matrix products of all groups share launches. */
muon_status muon_step_groups(muon_ctx* ctx, const muon_group* groups, int ngroups,
                             const muon_hparams* hp, void* stream);

/* End-to-end variant for callers whose gradients live in (preferably pinned)
 * HOST memory: each group's G entries are HOST pointers.  The gradients are
 * uploaded to a context-owned device staging buffer in slabs of about 32 MB on
 * an internal copy stream (ordered after the work already queued on `stream`);
 * each slab is stepped on `stream` as soon as its upload has landed, so the
 * transfer of the next slab overlaps the step of this one.  Results equal
 * muon_step_groups on the same gradients bit for bit.  The per-matrix ||U||_F
 * (nu_host, may be NULL) and flags (flags_host, may be NULL), in group order,
 * are copied back.  Returns after the stream has been synchronised; the return
 * value includes device-side status.  With pageable host memory the uploads do
 * not overlap; pin the gradients. */
muon_status muon_step_groups_host(muon_ctx* ctx, const muon_group* groups, int ngroups,
                                  const muon_hparams* hp, float* nu_host, int* flags_host,
                                  void* stream);

/* Newton-Schulz orthogonalisation only: Out_l = NS_k(X_l / (||X_l||_F + eps)),
 * oriented like X_l (no momentum, no scale, no decay).  X and Out are device
 * matrices rows x cols of `dtype`; Out may not alias X. */
muon_status muon_ns_orthogonalize(muon_ctx* ctx, const void* const* X, void* const* Out,
                                  int batch, int rows, int cols, int dtype, float eps,
                                  void* stream);

/* Device-side status of the most recent call on this context.  Synchronises
 * the stream of that call, then copies up to `capacity` per-matrix flag words
 * (MUON_FLAG_*) into `flags` (may be NULL) and the number of matrices into
 * *count (may be NULL).  Returns MUON_ERR_TIMEOUT if any kernel wait ran out,
 * else MUON_ERR_NONFINITE if any matrix was flagged, else MUON_OK. */
muon_status muon_get_status(muon_ctx* ctx, int* flags, int capacity, int* count);

/* ||U||_F per matrix of the most recent call (same order as the flags). */
muon_status muon_get_norms(muon_ctx* ctx, float* nu, int capacity, int* count);

/* Bytes of device workspace the context currently holds. */
size_t muon_workspace_bytes(const muon_ctx* ctx);

/* Per-launch timing.  While enabled, every kernel launch of the context is
 * bracketed by two CUDA events recorded on the launch stream (device time of
 * that launch alone).  muon_profile_read synchronises on those events and
 * sums durations per kernel kind since the last reset. */
typedef enum {
  MUON_KERNEL_MOMENTUM = 0, /* momentum + Nesterov + norm pass        */
  MUON_KERNEL_GRAM = 1,     /* A = X X^T                                */
  MUON_KERNEL_POLY = 2,     /* B = b A + c A A                          */
  MUON_KERNEL_UPDATE = 3,   /* X <- s B' X  with B' = aI + bA + cAA     */
  MUON_KERNEL_APPLY = 4,    /* W <- (1 - lr wd) W - lr s O              */
  MUON_KERNEL_NS_FUSED = 5, /* several phases (and iterations) in one persistent launch */
  MUON_KERNEL_KINDS = 6
} muon_kernel_kind;

typedef struct {
  int launches[MUON_KERNEL_KINDS];
  double ms[MUON_KERNEL_KINDS];
} muon_profile;

muon_status muon_profile_enable(muon_ctx* ctx, int on);
muon_status muon_profile_read(muon_ctx* ctx, muon_profile* out, int reset);

/* Top singular triplet of each matrix by power iteration (Muon Meets Mamba:
 * Spectral Optimization for State Space Models, abstract: Muon lowers the
 * condition number of the projection it trains; the top singular value is the
 * quantity to watch).  Starting from v_l (any nonzero vector; the previous
 * step's v warm-starts it), `iters` times:
 *   u = W v / |W v| ;  v = W^T u / |W^T u| ;  sigma = |W^T u|.
 * W: host array of device pointers, rows x cols of `dtype`, read only.
 * u: device pointers, `rows` floats each, written; v: `cols` floats each, in/out.
 * sigma: DEVICE array of `batch` floats, written.  Uses context scratch. */
muon_status muon_power_iteration(muon_ctx* ctx, const void* const* W, float* const* u, float* const* v,
                                 float* sigma, int batch, int rows, int cols, int dtype, int iters,
                                 void* stream);

/* Smallest singular value of each matrix by shifted power iteration, so that
 * the condition number sigma_max / sigma_min can be tracked (Muon Meets Mamba:
 * Spectral Optimization for State Space Models, abstract: the condition number
 * falls under Muon).  On the wide view X (W, or W^T when rows > cols; m =
 * min(rows, cols)), with s = sigma_max[l]^2, `iters` times
 *   y <- (s y - X X^T y) / |s y - X X^T y|,
 * then sigma_min[l] = |X^T y|, an upper bound on the true value for every y
 * that tightens as y turns toward the bottom singular vector.
 * W: host array of device pointers (rows x cols, `dtype`), read only.
 * y: device pointers, m floats each: start vector in, iterate out.
 * sigma_max: DEVICE array of `batch` floats (e.g. from muon_power_iteration);
 * sigma_min: DEVICE array of `batch` floats, written.  iters may be 0. */
muon_status muon_min_singular(muon_ctx* ctx, const void* const* W, float* const* y, const float* sigma_max,
                              float* sigma_min, int batch, int rows, int cols, int dtype, int iters, void* stream);

/* muon_step with the spectral cap (An Isotropy-Preserving Spectral Cap for
 * Muon: each update loses the direction that contributes most to the growth
 * of the top eigenvalue).  With (u_l, v_l) the top singular pair of the
 * PRE-step W_l (e.g. from muon_power_iteration before this call), the
 * orthogonalised update O_l is replaced by O_l - alpha_l u_l v_l^T,
 * alpha_l = u_l^T O_l v_l, before the scale and decay are applied, so the
 * update does not grow sigma_max(W_l) to first order.  u: `rows` floats,
 * v: `cols` floats per matrix (device); alpha: DEVICE array of `batch`
 * floats, written.  Other arguments as muon_step. */
muon_status muon_step_capped(muon_ctx* ctx, void* const* W, const void* const* G, float* const* M,
                             const float* const* u, const float* const* v, int batch, int rows, int cols,
                             int dtype, const muon_hparams* hp, float* alpha, void* stream);

/* AdamW for the parameters Muon does not take (Muon Meets Mamba: Spectral
 * Optimization for State Space Models, abstract: every weight group not
 * trained with Muon is trained with AdamW).  For each of `count` tensors t:
 *   m <- b1 m + (1 - b1) g ;  v <- b2 v + (1 - b2) g^2
 *   W <- W (1 - lr wd) - lr (m / (1 - b1^step)) / (sqrt(v / (1 - b2^step)) + eps)
 * W: host array of device pointers, numel[t] elements of `dtype`, updated in place.
 * G: same, read only.  m, v: fp32, numel[t] elements, updated in place (start at 0).
 * numel: HOST array of element counts.  Tensors may have any shape (flattened).
 * No context and no allocation; asynchronous on `stream`. */
typedef struct {
  float lr, beta1, beta2, eps, weight_decay;
  int step; /* 1-based step count used for bias correction */
} muon_adamw_hparams;

muon_status muon_adamw_step(void* const* W, const void* const* G, float* const* m, float* const* v,
                            const long long* numel, int count, int dtype,
                            const muon_adamw_hparams* hp, void* stream);

/* Bytes of the library's static device scratch used by muon_momentum_norm_noalloc. */
#define MUON_NOALLOC_SCRATCH_BYTES (256u * 1024u)

/* Momentum, look-ahead and Frobenius norm for callers that cannot allocate
 * device memory (a caller-owned memory pool, an allocator-free runtime, a
 * hook running during CUDA graph capture).  No counterpart in the pages: it
 * is the first pass of muon_step (M <- beta*M + G; U = G + beta*M, or U = M
 * when nesterov == 0; nu_l = ||U_l||_F) without a context and without any
 * allocation, and it does not materialise U.
 * G: host array of `batch` device pointers, rows x cols of `dtype`, read only.
 * M: host array of `batch` device pointers, rows x cols fp32, updated in place.
 * nu: DEVICE array of `batch` floats, written.
 * Scratch: a static device array of MUON_NOALLOC_SCRATCH_BYTES that every GPU
 * loading the library holds until exit.  It must hold one float per 8192
 * elements of each matrix: batch * ceil(rows*cols / 8192) <= 65280, else
 * MUON_ERR_UNSUPPORTED_SHAPE.  The first call on a device looks the scratch
 * address up (cudaGetSymbolAddress), so make it before any stream capture.
 * That address is kept for the life of the process: after cudaDeviceReset
 * (or any destruction of the device's primary context) this entry point must
 * not be called again on that device.
 * Every call shares the scratch: calls that overlap on the GPU race on it.
 * Asynchronous on `stream`; argument errors return before anything is queued. */
muon_status muon_momentum_norm_noalloc(const void* const* G, float* const* M, float* nu, int batch,
                                       int rows, int cols, int dtype, float beta, int nesterov,
                                       void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LIBMUON_MUON_H */
