/*
 * gauss.h -- C ABI of the B200 (sm_100a) fused Gaussian kernel reduction library.
 *
 * The operation (Gaussian kernel sum with signed weights, "Kernel matrix
 * reduction", Implementation sketch, eq. 1; output s_m of "Fast Gauss Sums via
 * Flash Attention", Algorithm 1, step 2, with inputs q = x, k = y, v = w and
 * tau > 0 as in its step 1):
 *
 *     out[b,i,c] = sum_j exp(-tau/2 * |x[b,i,:] - y[b,j,:]|^2) * w[b,j,c]
 *
 * is evaluated without ever forming the M x N kernel matrix: every kernel value
 * is produced on chip and consumed at once.  The weights are called b on the
 * pages; here they are w, to keep b for the batch index.
 *
 * Layouts (all row-major, contiguous, no strides):
 *     x    [B, M, D]   query points, dtype dt
 *     y    [B, N, D]   source points, dtype dt
 *     w    [B, N, C]   weights, dtype dt
 *     out  [B, M, C]   float32
 *     g    [B, M, C]   float32 upstream gradient (backward only)
 *
 * Supported shapes and types:
 *     GS_F32           : 1 <= D <= 8 (CUDA-core path), any C >= 1;
 *                        9 <= D <= 128 (tensor-core path at fp32 accuracy:
 *                        every operand split into two fp16 parts of 11
 *                        significant bits under power-of-two scales, three
 *                        MMAs per product) for the sums, their gradients,
 *                        the diffusion operator and the log-sum-exp.
 *     GS_F16 / GS_BF16 : 1 <= D <= 128 (tensor-core path), any C >= 1.
 *                        Arithmetic: x.y on the tensor cores with fp32
 *                        accumulation; with C > 1 (per pass of value
 *                        channels) kernel values rounded to fp16 for the
 *                        second product and weights converted to fp16 (for
 *                        bf16 weights exact for |w| in [2^-14, 65504]); with
 *                        one channel the products are summed in fp32 from the
 *                        fp32 kernel value and the exact weight.
 *                        The log-sum-exp runs on the tf32 tensor-core path
 *                        (fp16 / bf16 values are exact in tf32).
 *     The log-sum-exp backward and the k-nearest reduction: every dtype,
 *     1 <= D <= 128 (fp16 / bf16 inputs are widened, exactly, to fp32 copies
 *     in the workspace and take the fp32 implementation).
 *   Anything else returns GS_ERR_UNSUPPORTED; there is no CPU fallback.
 *
 * Ownership and synchronisation: the caller owns every buffer, allocates the
 * workspace (size from gs_workspace_bytes) and keeps all of them alive until
 * the work queued on `stream` has finished.  The library allocates no device
 * memory, never synchronises, and enqueues its kernels on `stream` (NULL = the
 * legacy default stream).  All pointers are device pointers that must be
 * 16-byte aligned (GS_ERR_ALIGNMENT otherwise); a pointer may be NULL only when
 * the tensor it names is empty.  Results are deterministic: no floating-point
 * atomics, and every partial sum is combined in a fixed order.
 *
 * Errors: arguments are validated on the host before anything is enqueued; a
 * rejected call enqueues nothing.  Device-side faults the library can detect
 * (a wait on an on-chip barrier that exceeds its time limit) set a device error
 * word instead of trapping; gs_last_device_error() reads and clears it.
 */
#ifndef GAUSS_B200_H
#define GAUSS_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The same object as cudaStream_t / CUstream. */
typedef struct CUstream_st *gs_stream_t;

typedef enum { GS_F32 = 0, GS_F16 = 1, GS_BF16 = 2 } gs_dtype;

typedef enum {
    GS_OP_SUM = 0,
    GS_OP_LSE = 1,
    GS_OP_SUM_BWD = 2,
    GS_OP_LSE_BWD = 3,
    GS_OP_KNN = 4,      /* gs_workspace_bytes: pass K as C */
    GS_OP_DIFFUSION = 5, /* gs_workspace_bytes: M = N, C = columns of V (1 for the scales) */
    GS_OP_SUM_FWD_BWD = 6,
    GS_OP_DIFFUSION_BLOCK = 7
} gs_op;

typedef enum {
    GS_OK = 0,
    GS_ERR_INVALID_ARG = 1, /* NULL pointer for a non-empty tensor, negative size, tau not finite > 0 */
    GS_ERR_UNSUPPORTED = 2, /* a (dtype, D) combination with no kernel */
    GS_ERR_ALIGNMENT = 3,   /* a pointer not 16-byte aligned */
    GS_ERR_WORKSPACE = 4,   /* workspace smaller than gs_workspace_bytes() */
    GS_ERR_TIMEOUT = 5,     /* a device-side wait gave up (reported by gs_last_device_error) */
    GS_ERR_CUDA = 6         /* a CUDA runtime call failed */
} gs_status;

/*
 * Workspace, in bytes, that a call of `op` with these sizes needs on the
 * current device (0 when none; the workspace pointer may then be NULL).  It
 * holds packed operand copies, per-row norms and split-j partial results; the
 * library never reads it before writing it, so it need not be initialised.
 * Returns (size_t)-1 for arguments the corresponding call would reject.
 */
size_t gs_workspace_bytes(gs_op op, int64_t B, int64_t M, int64_t N, int64_t D, int64_t C,
                          gs_dtype dt);

/*
 * Gaussian kernel sum (defined above; "Kernel matrix reduction", Implementation
 * sketch, eq. 1 and eq. 2).  N == 0 writes zeros; M == 0 or B == 0 does nothing.
 */
gs_status gauss_sum_fwd(const void *x, const void *y, const void *w, float *out, int64_t B,
                        int64_t M, int64_t N, int64_t D, int64_t C, float tau, gs_dtype dt,
                        void *ws, size_t ws_bytes, gs_stream_t stream);

/*
 * Log-sum-exp reduction ("Kernel matrix reduction", Overview, the log-sum-exp
 * reduction; the .logsumexp() reduction of the LazyTensor API in "KeOps: a
 * symbolic tensor that never materialises the matrix it represents"), with the
 * weights entering as their logarithm:
 *
 *     out[b,i,c] = log sum_j w[b,j,c] * exp(-tau/2 * |x_i - y_j|^2)
 *
 * computed with a shift so that rows whose every kernel value underflows fp32
 * still get a finite result.  Requires w > 0 (not checked: a non-positive
 * weight gives NaN or -inf, as log does).  N == 0 writes -inf.
 * Supported for 1 <= D <= 128 in every dtype: GS_F32 with D <= 8 on the
 * CUDA-core path (power-of-two weight shifts), the rest on the tensor-core
 * path (split fp16 parts for fp32, tf32 for fp16 / bf16; a running maximum
 * per row).
 */
gs_status gauss_lse_fwd(const void *x, const void *y, const void *w, float *out, int64_t B,
                        int64_t M, int64_t N, int64_t D, int64_t C, float tau, gs_dtype dt,
                        void *ws, size_t ws_bytes, gs_stream_t stream);

/*
 * Forward sum that also keeps what the x-gradient needs, for a forward pass
 * followed by a backward pass on the same inputs.  The gradient formula of
 * gauss_sum_bwd splits as
 *
 *     grad_x[b,i,k] = -tau * sum_c g[b,i,c] ((x_ik - z_k) s0[b,i,c] - s1[b,i,c,k])
 *     s0[b,i,c]   = sum_j K_ij w[b,j,c]                 (= out[b,i,c])
 *     s1[b,i,c,k] = sum_j K_ij w[b,j,c] (y_jk - z_k),   z = x[b,0,:]
 *
 * and neither s0 nor s1 depends on the upstream gradient g, so one fused pass
 * computes them with the forward result.  `saved` [B, M, C * (1 + D)] float32
 * receives [s0 (C) | s1 (C x D, channel c's D values together)] per row;
 * `out` [B, M, C] receives s0.  The pages keep no such sums (they recompute
 * every reduction from scratch): this is a reuse of the same reductions, no
 * approximation.  Workspace: gs_workspace_bytes(GS_OP_SUM_BWD, ...) is enough.
 */
gs_status gauss_sum_fwd_saved(const void *x, const void *y, const void *w, float *out,
                              float *saved, int64_t B, int64_t M, int64_t N, int64_t D,
                              int64_t C, float tau, gs_dtype dt, void *ws, size_t ws_bytes,
                              gs_stream_t stream);

/*
 * The backward of gauss_sum_bwd from the sums gauss_sum_fwd_saved kept for the
 * same x, y, w, tau: grad_x from `saved` and g (a per-row epilogue, no pair
 * work) and grad_w by one fused pass (rows y, columns x, values g).  Either
 * output may be NULL.  Workspace: gs_workspace_bytes(GS_OP_SUM_BWD, ...).
 */
gs_status gauss_sum_bwd_saved(const void *x, const void *y, const void *w, const float *g,
                              const float *saved, float *grad_x, float *grad_w, int64_t B,
                              int64_t M, int64_t N, int64_t D, int64_t C, float tau, gs_dtype dt,
                              void *ws, size_t ws_bytes, gs_stream_t stream);

/*
 * Forward and backward in one call, for an upstream gradient g [B, M, C]
 * (float32) known before the forward (a loss linear in the output, or a
 * cotangent fixed in advance): out = gauss_sum_fwd(x, y, w) and, of
 * L = sum g * out, grad_x [B, M, D] and grad_w [B, N, C] exactly as
 * gauss_sum_bwd defines them ("Kernel matrix reduction", Variants: the
 * gradient is the same fused reduction, its tiles recomputed).  With fp16 /
 * bf16 inputs, C = 1 and D <= 47 every kernel value is computed once: one
 * tensor-core sweep forms the forward sum, the x-gradient sums of
 * gauss_sum_fwd_saved and the column sums grad_w = sum_i K_ij g_i together
 * (g enters the tensor cores as fp16 hi + lo parts under a per-batch power of
 * two, ~22 significant bits; grad_w is then a fixed-order sum of per-128-row-
 * tile partials).  Otherwise the call runs gauss_sum_fwd_saved's pass and
 * gauss_sum_bwd_saved's.  `out` must not be NULL; grad_x and grad_w may be
 * NULL (without grad_w there is nothing to fuse).  Workspace:
 * gs_workspace_bytes(GS_OP_SUM_FWD_BWD, ...); errors as gauss_sum_fwd.
 */
gs_status gauss_sum_fwd_bwd(const void *x, const void *y, const void *w, const float *g, float *out,
                            float *grad_x, float *grad_w, int64_t B, int64_t M, int64_t N,
                            int64_t D, int64_t C, float tau, gs_dtype dt, void *ws,
                            size_t ws_bytes, gs_stream_t stream);

/*
 * Gradient of L = sum_{b,i,c} g[b,i,c] * out[b,i,c] for the Gaussian kernel sum
 * ("Kernel matrix reduction", Variants: gradients through the same fused
 * reduction; the torch.autograd.grad example of the LazyTensor API):
 *
 *     grad_w[b,j,c] = sum_i K_ij g[b,i,c]                                 [B, N, C]
 *     grad_x[b,i,k] = -tau * sum_j K_ij (sum_c g[b,i,c] w[b,j,c]) (x_ik - y_jk)   [B, M, D]
 *
 * with K_ij = exp(-tau/2 |x_i - y_j|^2), recomputed tile by tile, never stored.
 * Either output may be NULL to skip it.  Both outputs are float32.  Same as
 * gauss_sum_vjp with grad_y = grad_tau = NULL.
 */
gs_status gauss_sum_bwd(const void *x, const void *y, const void *w, const float *g,
                        float *grad_x, float *grad_w, int64_t B, int64_t M, int64_t N, int64_t D,
                        int64_t C, float tau, gs_dtype dt, void *ws, size_t ws_bytes,
                        gs_stream_t stream);

/*
 * Every first-order gradient of L = sum_{b,i,c} g[b,i,c] * out[b,i,c] for the
 * Gaussian kernel sum ("Kernel matrix reduction", Variants: derivatives through
 * the fused reduction, for every input):
 *
 *     grad_x[b,i,k] = -tau sum_j K_ij (g_i . w_j) (x_ik - y_jk)            [B, M, D]
 *     grad_y[b,j,k] = -tau sum_i K_ij (g_i . w_j) (y_jk - x_ik)            [B, N, D]
 *     grad_w[b,j,c] = sum_i K_ij g[b,i,c]                                  [B, N, C]
 *     grad_tau[0]   = -1/2 sum_b sum_ij K_ij |x_i - y_j|^2 (g_i . w_j)     one float
 *
 * Any output may be NULL to skip it (grad_tau needs no alignment).  Two passes
 * of the fused kernels at most (rows y for grad_w / grad_y, rows x for grad_x /
 * grad_tau), tiles recomputed, never stored; coordinates in the augmented
 * values are centred at the first row point of each batch.  Workspace:
 * gs_workspace_bytes(GS_OP_SUM_BWD, ...).  grad_tau is a fixed-order reduction.
 */
gs_status gauss_sum_vjp(const void *x, const void *y, const void *w, const float *g,
                        float *grad_x, float *grad_y, float *grad_w, float *grad_tau, int64_t B,
                        int64_t M, int64_t N, int64_t D, int64_t C, float tau, gs_dtype dt,
                        void *ws, size_t ws_bytes, gs_stream_t stream);

/*
 * Every first-order gradient of L = sum_{b,i,c} g[b,i,c] * lse[b,i,c] for the
 * log-sum-exp reduction of gauss_lse_fwd ("Kernel matrix reduction", Overview
 * and Variants: the log-sum-exp reduction and gradients through it).  With the
 * normalised weights p_ijc = w_jc K_ij exp(-lse_ic):
 *
 *     grad_x[b,i,k] = -tau sum_c g_ic sum_j p_ijc (x_ik - y_jk)            [B, M, D]
 *     grad_y[b,j,k] = -tau sum_i sum_c g_ic p_ijc (y_jk - x_ik)            [B, N, D]
 *     grad_w[b,j,c] = sum_i g_ic K_ij exp(-lse_ic)                          [B, N, C]
 *     grad_tau[0]   = -1/2 sum_ic g_ic sum_j p_ijc |x_i - y_j|^2             one float
 *
 * lse [B, M, C] float32 is the forward's output for the same inputs.  The
 * shift -lse is folded into every kernel exponent, so the passes sum p
 * directly (no overflow, no separate normalisation).  1 <= D <= 128 (fp32:
 * D > 8 on split tensor-core passes; fp16 / bf16: exact fp32 copies first),
 * w > 0; any output may be NULL.  Workspace:
 * gs_workspace_bytes(GS_OP_LSE_BWD, ...).
 */
gs_status gauss_lse_bwd(const void *x, const void *y, const void *w, const float *lse,
                        const float *g, float *grad_x, float *grad_y, float *grad_w,
                        float *grad_tau, int64_t B, int64_t M, int64_t N, int64_t D, int64_t C,
                        float tau, gs_dtype dt, void *ws, size_t ws_bytes, gs_stream_t stream);

/*
 * k-nearest reduction ("Kernel matrix reduction", Overview: minima and the
 * indices of the K smallest entries per row; the .argmin() reduction of the
 * LazyTensor API): for every row i, the K smallest squared distances
 * |x[b,i] - y[b,j]|^2 over j, ascending, and their indices j; equal distances
 * are ordered by the lower j.  Rows with fewer than K sources get +inf and
 * index -1 in the missing places.  The row maximum of the Gaussian kernel is
 * exp(-tau/2 * out_sqdist[b,i,0]), attained at out_index[b,i,0].
 * Distances are computed in fp32 as e_k = x_k - y_k, d = e_0^2, then
 * d = fma(e_k, e_k, d) for k = 1 .. D-1 (round to nearest), and every
 * comparison is made on those fp32 values.
 *     out_sqdist [B, M, K] float32, out_index [B, M, K] int64.
 * 1 <= D <= 128, 1 <= K <= 32; fp16 / bf16 inputs are widened (exactly) to
 * fp32 copies in the workspace.  Workspace:
 * gs_workspace_bytes(GS_OP_KNN, B, M, N, D, K, GS_F32).
 */
gs_status gauss_knn(const void *x, const void *y, float *out_sqdist, int64_t *out_index, int64_t B,
                    int64_t M, int64_t N, int64_t D, int64_t K, gs_dtype dt, void *ws,
                    size_t ws_bytes, gs_stream_t stream);

/*
 * Diffusion operator of "FlashDiffusion: Fused Tiled Kernel Spectral
 * Decomposition" (section 2.2, XGEMM: diag(s) K diag(s) applied to a block V;
 * the q and d normalisation passes are kernel applications with V replaced by
 * 1 and by q^-alpha; the right scaling is applied to V, the left one to the
 * rows of the result).  Over one point set x [B, N, D], K_ij =
 * exp(-tau/2 |x_i - x_j|^2).  The page's section 2.1, defining s, did not
 * survive extraction; the reading implemented is the alpha-normalised diffusion
 * map those passes compute:
 *     q = K 1,  d = q^-alpha (K q^-alpha),  s = q^-alpha d^-1/2,
 * so that diag(s) K diag(s) is the symmetric form of the Markov matrix of
 * K_ij / (q_i q_j)^alpha (eigenvalues in [0, 1], sqrt(d) its fixed point).
 *   gauss_diffusion_scales: s_out [B, N] (q_out, d_out optional, may be NULL)
 *   gauss_diffusion_apply:  out [B, N, C] = diag(s) K diag(s) v, v [B, N, C]
 * All of s, q, d, v, out are float32; x has dtype dt (the paths of
 * gauss_sum_fwd).  Workspace: gs_workspace_bytes(GS_OP_DIFFUSION, B, N, N, D, C, dt)
 * with C = 1 for the scales.
 */
/*
 * The kernel application those passes are made of, between a block of rows and
 * a set of columns of the point set:
 *     out[b,i,c] = sum_j exp(-tau/2 |x_rows[b,i] - x_cols[b,j]|^2) v[b,j,c]
 * x_rows [B, M, D] and x_cols [B, N, D] of dtype dt, v [B, N, C] and out
 * [B, M, C] float32 whatever dt (the Gauss sum with float32 values).  With the
 * rows of one rank and the columns of every rank it gives that rank's rows of
 * q = K 1, of K q^-alpha and of K (s v): "FlashDiffusion" (section 3) runs its
 * operator sharded over rows this way.  Workspace:
 * gs_workspace_bytes(GS_OP_DIFFUSION_BLOCK, B, M, N, D, C, dt).
 */
gs_status gauss_diffusion_block(const void *x_rows, const void *x_cols, const float *v, float *out,
                                int64_t B, int64_t M, int64_t N, int64_t D, int64_t C, float tau,
                                gs_dtype dt, void *ws, size_t ws_bytes, gs_stream_t stream);
gs_status gauss_diffusion_scales(const void *x, float *q_out, float *d_out, float *s_out,
                                 int64_t B, int64_t N, int64_t D, float tau, float alpha,
                                 gs_dtype dt, void *ws, size_t ws_bytes, gs_stream_t stream);
gs_status gauss_diffusion_apply(const void *x, const float *s, const float *v, float *out,
                                int64_t B, int64_t N, int64_t D, int64_t C, float tau, gs_dtype dt,
                                void *ws, size_t ws_bytes, gs_stream_t stream);

/*
 * Allocation-free variant of gauss_sum_fwd (no counterpart on the pages: it
 * exists for callers of this library that cannot allocate device memory for a
 * workspace -- a plugin whose host application owns the device-memory budget,
 * a latency-critical loop that must not block in the CUDA allocator, a process
 * under a hard memory cap).  Same arguments, results and kernels as
 * gauss_sum_fwd, without ws / ws_bytes: the scratch comes from a fixed 32 MiB
 * device array inside the library, held per device context until the process
 * exits: on every device context the process creates when CUDA loads modules
 * eagerly (CUDA_MODULE_LOADING=EAGER), and only on devices where this call has
 * been made under lazy loading (the default).  Calls whose scratch need (gs_workspace_bytes of
 * GS_OP_SUM) exceeds 32 MiB return GS_ERR_WORKSPACE.  All calls on a device
 * share the array: calls that overlap on the GPU race (order them on one
 * stream).  The array keeps the last call's contents; nothing in it needs to
 * start at zero.  The first call on a device looks up the array's device
 * address with that device current; make that first call before any stream
 * capture.  The library allocates nothing in this call.
 */
gs_status gauss_sum_fwd_noalloc(const void *x, const void *y, const void *w, float *out, int64_t B,
                                int64_t M, int64_t N, int64_t D, int64_t C, float tau, gs_dtype dt,
                                gs_stream_t stream);

/* A static, human-readable name for a status code. */
const char *gs_status_string(gs_status status);

/*
 * Synchronises `stream`, then reads and clears the device error word of the
 * current device: GS_OK, GS_ERR_TIMEOUT (a kernel gave up on a wait and
 * returned early; its outputs are not valid), or GS_ERR_CUDA if the
 * synchronisation itself failed.
 */
gs_status gs_last_device_error(gs_stream_t stream);

/* Library version, major * 10000 + minor * 100 + patch. */
int gs_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GAUSS_B200_H */
