/*
 * nq.h -- C ABI of the B200 (sm_100a) NanoQuant hot path.
 *
 * Two operations, from the NanoQuant pages (arXiv 2602.06694 summaries):
 *
 *   1. Calibration preconditioners.  NanoQuant summary page (paper.rainbus.top),
 *      "Method steps" (方法步骤详情), stage one: per-linear-layer statistics z_in,
 *      z_out collected over 128 x 2048 calibration tokens are regularised by
 *      Ledoit-Wolf shrinkage into diagonal preconditioners D_in, D_out.  Here
 *      z_in / z_out are the per-channel second moments of the input activations
 *      and of the output gradients (the diagonals of the K-FAC factors, same page,
 *      "Prerequisites" (前置知识), K-FAC paragraph).
 *
 *   2. LB-ADMM initialisation.  Same page, "Core method" (核心方法) and "Method
 *      steps" stage two: the preconditioned target W~ = D_out W D_in is factorised
 *      as diag(s1) U+-1 V+-1^T diag(s2) by an ADMM over continuous latents U, V
 *      with (a) a Cholesky-solved regularised U (V) step, (b) an SVID projection
 *      to a binary proxy Z, (c) a dual update; then magnitude balancing, channel
 *      scale extraction and packing of the signs into integer words.
 *
 * Conventions for every entry point
 *   - Matrices are row-major.  W is m x n (out x in features, the PyTorch layout).
 *   - Pointers named "device" must be CUDA device (or managed) memory of the
 *     current device; "host" pointers are ordinary host memory.
 *   - The caller owns every buffer.  The library allocates no device memory:
 *     all scratch lives in the caller's workspace ``ws`` (size from the matching
 *     *_workspace_size function; 256-byte alignment required).  One exception:
 *     nq_calib_stats_noalloc takes no workspace and keeps its scratch in a fixed
 *     4 MiB array inside the library image (see its declaration).
 *   - All device work is enqueued on ``stream``.  Entry points that fill host
 *     outputs synchronise ``stream`` before returning; the others return as soon
 *     as the work is enqueued.
 *   - Argument errors are reported before anything is launched.  Errors detected
 *     on the device (non-finite values, a non-positive Cholesky pivot, a wait that
 *     ran out) are reported by the next synchronising call on the same workspace.
 *     On error, outputs are unspecified.
 *   - Not thread-safe per workspace: two calls that share a workspace must be
 *     ordered on the same stream.
 */
#ifndef NQ_H
#define NQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *nq_stream_t; /* == cudaStream_t; NULL = legacy default stream */

typedef enum {
    NQ_OK = 0,
    NQ_ERR_INVALID_ARG = 1,  /* bad size, null pointer, misaligned buffer, bad dtype       */
    NQ_ERR_WORKSPACE = 2,    /* workspace too small                                       */
    NQ_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed                          */
    NQ_ERR_NONFINITE = 4,    /* NaN or Inf found in an input                               */
    NQ_ERR_NOT_SPD = 5,      /* non-positive pivot in a Cholesky factorisation             */
    NQ_ERR_TIMEOUT = 6,      /* a bounded device-side wait ran out                         */
    NQ_ERR_UNSUPPORTED = 7   /* no sm_100a device, or a size beyond the supported range    */
} nq_status;

typedef enum { NQ_F32 = 0, NQ_BF16 = 1 } nq_dtype;

/* Arithmetic of the LB-ADMM tensor-core contractions (W^ X, the Grams X^T X):
 *   NQ_PREC_BF16  W^ and the latent factor are rounded to BF16 (RNE) as MMA operands;
 *   NQ_PREC_FP32  both are split into BF16 hi + lo parts and each contraction runs as
 *                 three MMA passes (hi.hi + lo.hi + hi.lo): FP32-level accuracy at three
 *                 times the tensor work.
 * Accumulation is FP32 in both; the solve with G^-1 is always split (FP32-level).
 * nq_lbadmm uses NQ_PREC_BF16 for BF16 weights and NQ_PREC_FP32 for FP32 weights. */
typedef enum { NQ_PREC_BF16 = 0, NQ_PREC_FP32 = 1 } nq_precision;

/* Human-readable name of a status code (static string, never NULL). */
const char *nq_status_string(nq_status s);

/* Library version as major*10000 + minor*100 + patch. */
int32_t nq_version(void);

/* ------------------------------------------------------------------------- */
/* Bits-per-weight accounting.  NanoQuant summary page, "Motivation" (研究动机)  */
/* and "Results" (实验结果): BPW counts one bit per sign of U (m x r) and V      */
/* (n x r) and 16 bits per entry of s1 (m) and s2 (n).                         */
/* ------------------------------------------------------------------------- */

/* ((m+n) r + 16 (m+n)) / (m n).  Returns -1 for m <= 0, n <= 0 or r < 0. */
double nq_bpw(int64_t m, int64_t n, int32_t r);

/* Largest r with nq_bpw(m, n, r) <= bpw: floor((bpw m n - 16 (m+n)) / (m+n)),
 * clamped at 0.  bpw is read as a decimal (a result within 1e-9 of an integer is
 * taken as that integer).  Returns -1 for m <= 0 or n <= 0 or bpw < 0. */
int32_t nq_rank_for_bpw(int64_t m, int64_t n, double bpw);

/* ------------------------------------------------------------------------- */
/* 1. Calibration preconditioners                                              */
/* ------------------------------------------------------------------------- */

/* Workspace bytes for nq_calib_stats / nq_calib_precond on streams of at most
 * T tokens and C channels (either stream). */
size_t nq_calib_workspace_size(int64_t T, int64_t C);

/*
 * Per-channel moments of one token-major stream X (T x C, dtype dt):
 *     s_j = (1/T) sum_t X_tj^2,   q_j = (1/T) sum_t X_tj^4.
 * X: device, row stride C elements.  s, q: device, C doubles each.
 * Accumulation: FP32 within a slab of tokens, FP64 across slabs, fixed order
 * (bit-identical from run to run).  Enqueue only.
 */
nq_status nq_calib_stats(const void *X, int64_t T, int64_t C, nq_dtype dt, double *s, double *q,
                         void *ws, size_t ws_bytes, nq_stream_t stream);

/*
 * nq_calib_stats without a workspace.  The paper has no counterpart: this entry point
 * exists for callers that cannot allocate device memory or pass a workspace -- a plugin
 * inside a host program that owns the device memory pool and refuses new allocations,
 * a process whose device-memory budget is fixed at launch, or a path that must not call
 * cudaMalloc / cudaFree because they may synchronise the device.
 * Same arguments, arithmetic and results as nq_calib_stats.  Its scratch is a fixed
 * 4 MiB array inside the library image, held on every GPU that loads the library until
 * the process exits.  Limit: C <= 32768 channels (any T); larger C returns
 * NQ_ERR_UNSUPPORTED.  The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call before any
 * stream capture.  All calls share the array, so calls whose GPU work may overlap
 * (other streams, other threads) race and must be ordered by the caller.  Nothing in the
 * array needs clearing between calls.  Allocates nothing.  Enqueue only.
 */
nq_status nq_calib_stats_noalloc(const void *X, int64_t T, int64_t C, nq_dtype dt, double *s,
                                 double *q, nq_stream_t stream);

/*
 * Diagonal preconditioners from the activation stream (T_in x n) and the output
 * gradient stream (T_out x m):
 *     mu = mean(s), delta^2 = sum_j (s_j - mu)^2, beta_bar^2 = (1/T) sum_j (q_j - s_j^2),
 *     alpha = min(beta_bar^2, delta^2) / delta^2 (1 if delta^2 = 0),
 *     d~ = (1 - alpha) s + alpha mu,   d = sqrt(max(d~, 1e-12 mu))
 * (Ledoit & Wolf 2004 with target mu I, restricted to the diagonal).
 * alpha_override >= 0 replaces alpha by that value; < 0 selects Ledoit-Wolf.
 * acts, grads: device.  d_in (n), d_out (m): device float.
 * alpha_out: host double[2] {alpha_in, alpha_out}, or NULL.  When non-NULL the call
 * synchronises the stream; otherwise it only enqueues.
 */
nq_status nq_calib_precond(const void *acts, int64_t T_in, int64_t n, const void *grads,
                           int64_t T_out, int64_t m, nq_dtype dt, double alpha_override,
                           float *d_in, float *d_out, double *alpha_out, void *ws,
                           size_t ws_bytes, nq_stream_t stream);

/* ------------------------------------------------------------------------- */
/* 2. LB-ADMM                                                                  */
/* ------------------------------------------------------------------------- */

/* Supported sizes: 1 <= m, n <= 65536; 1 <= r <= min(m, n, 4096). */

/* Workspace bytes for an m x n layer at rank r (holds the whole ADMM state). */
size_t nq_lbadmm_workspace_size(int64_t m, int64_t n, int32_t r);

/*
 * How the inverse G^-1 = (X^T X + (lambda + rho) I)^-1 of each half step is formed.
 * NQ_INV_CHOLESKY: the Cholesky factorisation and triangular inverse (FP32), then
 *   G^-1 = L^-T L^-1 (split-BF16 tensor-core GEMM).
 * NQ_INV_NEWTON: first a Newton-Schulz update of the inverse this side used in its
 *   previous half step, X_{k+1} = X_k + (I - X_k G) X_k (two r x r tensor-core GEMMs per
 *   step: the residual I - X_k G with BF16 operands in the first two steps and split BF16
 *   in the later ones, the correction with BF16 operands), at most 6 steps; the iterate
 *   after the step whose ||I - X_k G||_F is <= 1e-2 is taken (so
 *   ||I - X G||_2 <= 1e-4 up to rounding).  An update whose residual does not shrink,
 *   or that reaches no such step, is dropped and the Cholesky path runs instead, decided
 *   on the device (no synchronisation).
 * NQ_INV_AUTO (default): NQ_INV_NEWTON for r >= 256 once the workspace has run 3
 *   iterations (4 above r = 1536) since its nq_lbadmm_prepare (the first iterations move
 *   G too far), NQ_INV_CHOLESKY otherwise.
 * Process-wide; read when a half step is enqueued.  Returns NQ_ERR_INVALID_ARG for an
 * unknown mode.
 */
typedef enum { NQ_INV_AUTO = 0, NQ_INV_CHOLESKY = 1, NQ_INV_NEWTON = 2 } nq_inverse_mode;
nq_status nq_set_inverse_mode(nq_inverse_mode mode);

/*
 * The latent update of each half step (a measured variant; community blog page, to-do
 * section: a gradient-descent solver in place of the Cholesky solves).
 * NQ_SOLVER_EXACT (default): X = R G^-1, the exact minimiser (G^-1 as nq_set_inverse_mode).
 * NQ_SOLVER_GD: gd_steps (1..1000) gradient steps on the same objective from the side's
 *   current latent, X <- X - eta (X G - R) with eta = 1 / max_i sum_j |G_ij|, each a
 *   split-BF16 tensor-core GEMM X G whose epilogue takes the step.  An inexact update: the
 *   iterates differ from the exact LB-ADMM's (equal as gd_steps grows).
 * Process-wide; read when a half step is enqueued.  NQ_ERR_INVALID_ARG for an unknown
 * solver or a step count out of range.
 */
typedef enum { NQ_SOLVER_EXACT = 0, NQ_SOLVER_GD = 1 } nq_latent_solver;
nq_status nq_set_latent_solver(nq_latent_solver solver, int32_t gd_steps);

/*
 * Scheduling settings of the LB-ADMM iterations (process-wide; none changes what is
 * computed, though a tile width can regroup the objective's partial sums and so its last
 * bits):
 * NQ_TUNE_FACTOR_CTAS: CTAs given to forming G^-1 (factorisation or update) while the
 *   RHS GEMM runs on the other SMs: -1 (default) half of the SMs up to r = 1536, else no
 *   overlap; 0 no overlap; n >= 1: n CTAs (at least 3, at most all SMs but one).
 * NQ_TUNE_NEWTON_BN: tile width of the update's GEMMs: 0 (default) the fewest waves x
 *   width on the CTAs it gets, or 64, 128, 256.
 * NQ_TUNE_SVID_BESIDE: 1 (default) the SVID passes of a side run on an auxiliary stream
 *   beside the next half step's GEMMs; 0: right after the side's solve.
 * NQ_TUNE_NFAST: 1 (default) the RHS GEMM and the solve walk their output tiles column
 *   tile fastest (the large row operand is read once while its few column tiles run
 *   together); 0: row tile fastest.
 * NQ_TUNE_RHS_BN, NQ_TUNE_SOLVE_BN: tile width of the RHS GEMM / of the solve: 0 (default:
 *   RHS 256 for r > 128, solve 128 for 128 < r <= 1024 and 256 above; narrower for small
 *   r), or 128, 256.
 * NQ_TUNE_NEWTON_FUSED: 0 (default) two launches per step of the Newton-Schulz update;
 *   1: all its steps in one cooperative launch on 128 x 128 tiles (grid-wide barriers
 *   between its GEMMs; the update itself is shorter, but its CTAs stay resident through
 *   the barriers and the GEMMs and SVID passes beside it slow down by as much at r = 1000,
 *   more at other ranks).  NQ_TUNE_NEWTON_BN applies to the two-launch form only.
 * Returns NQ_ERR_INVALID_ARG for an unknown key or value.
 */
typedef enum {
    NQ_TUNE_FACTOR_CTAS = 0, NQ_TUNE_NEWTON_BN = 1, NQ_TUNE_SVID_BESIDE = 2, NQ_TUNE_NFAST = 3,
    NQ_TUNE_RHS_BN = 4, NQ_TUNE_SOLVE_BN = 5, NQ_TUNE_NEWTON_FUSED = 6, NQ_TUNE_COUNT = 7
} nq_tuning;
nq_status nq_set_tuning(nq_tuning key, int32_t value);

/*
 * Full LB-ADMM initialisation of one layer.
 *
 * Form of the iteration (the pages give no equations; this is the concrete form
 * implemented, step for step the same as the library's FP64 reference):
 *   W^ = W~ / gamma, gamma = ||W~||_F / (2 sqrt(r)), stored as BF16 (RNE);
 *   V_0[j][k] = sqrt(2/n) * (-1 if bit 63 of SplitMix64(seed, j*r+k) else +1);
 *   Z_U = L_U = Z_V = L_V = 0;
 *   repeat iters times:
 *     U = (W^ V + rho (Z_U - L_U)) (V^T V + (lambda + rho) I)^-1
 *     S = U + L_U;  A = |S|;  b = 1;  K times { a = A b / ||A b||;  b = A^T a }
 *     Z_U = sign(S) * a b^T;   L_U = L_U + U - Z_U
 *     the same for V with W^^T and U
 *     objective[t] = ||W^ - U V^T||_F^2 / ||W^||_F^2   (of W^ and the latents as the
 *                    tensor-core operands hold them: BF16, or split BF16 for FP32)
 *   g_k = sqrt(||V_:k|| / ||U_:k||);  U_:k *= g_k;  V_:k /= g_k
 *   s1_i = gamma mean_k |U_ik|,  s2_j = mean_k |V_jk|
 *   sign bit = (latent < 0), LSB-first along k, row-major uint32[rows][(r+31)/32]
 * Tensor-core operands (W^ and the latent factor of the contraction) are BF16 for BF16
 * weights and split BF16 (FP32-accurate, see nq_precision) for FP32 weights;
 * accumulation and every other quantity is FP32 (reductions FP64 where noted).
 * (V^T V + (lambda + rho) I)^-1 is formed explicitly and applied as a split-BF16 GEMM;
 * how it is formed is set by nq_set_inverse_mode (Cholesky, or a Newton-Schulz update
 * of the previous iteration's inverse that falls back to Cholesky on the device).
 *
 * W: device, m x n, dtype dt.  d_in (n), d_out (m): device float, or NULL for 1.
 * U_packed: device uint32 [m][(r+31)/32];  V_packed: device uint32 [n][(r+31)/32].
 * s1 (m), s2 (n): device float; scales of W~ (for the raw W use s1/d_out, s2/d_in).
 * objective: host float[iters] or NULL.  final_rel_err: host, or NULL:
 *     ||W~ - diag(s1) U+- V+-^T diag(s2)||_F / ||W~||_F.
 * Synchronises the stream when objective or final_rel_err is non-NULL.
 * Requires rho > 0, lambda >= 0, iters >= 1, K >= 1.
 */
nq_status nq_lbadmm(const void *W, nq_dtype dt, int64_t m, int64_t n, const float *d_in,
                    const float *d_out, int32_t r, float rho, float lambda, int32_t iters,
                    int32_t K, uint64_t seed, uint32_t *U_packed, uint32_t *V_packed, float *s1,
                    float *s2, float *objective, float *final_rel_err, void *ws,
                    size_t ws_bytes, nq_stream_t stream);

/*
 * Reconstruction error of a packed factorisation against W~ = D_out W D_in:
 *     ||W~ - diag(s1) U+- V+-^T diag(s2)||_F / ||W~||_F   (0 if both norms vanish).
 * All array arguments are device pointers as in nq_lbadmm; rel_err is host.
 * Uses a +-1 tensor-core GEMM (exact for r <= 4096) with a fused squared-error
 * reduction.  Synchronises the stream.
 */
size_t nq_recon_workspace_size(int64_t m, int64_t n, int32_t r);
nq_status nq_recon_error(const void *W, nq_dtype dt, int64_t m, int64_t n, const float *d_in,
                         const float *d_out, const uint32_t *U_packed, const uint32_t *V_packed,
                         int32_t r, const float *s1, const float *s2, double *rel_err, void *ws,
                         size_t ws_bytes, nq_stream_t stream);

/*
 * Sign packing alone: bits[i][k/32] bit (k%32) = (X[i][k] < 0); -0.0 packs as 0.
 * X: device float rows x r.  bits: device uint32 rows x (r+31)/32.  Enqueue only.
 */
nq_status nq_pack_signs(const float *X, int64_t rows, int32_t r, uint32_t *bits,
                        nq_stream_t stream);

/*
 * Least-squares refit of the channel scales with the signs fixed.  NanoQuant summary
 * page, "Method steps" stage two and "Technical novelty": the scales s1, s2 of
 * W~ ~ diag(s1) U+- V+-^T diag(s2) are extracted after magnitude balancing; this refines
 * them for the fixed packed signs by alternating exact minimisations (P = U+- V+-^T):
 *     s1_i <- sum_j W~_ij P_ij s2_j / sum_j P_ij^2 s2_j^2,   then
 *     s2_j <- sum_i W~_ij P_ij s1_i / sum_i P_ij^2 s1_i^2,   ``sweeps`` times
 * (a scale whose denominator vanishes keeps its value), so the error never increases.
 * Each half sweep is one +-1 tensor-core GEMM (exact) with the sums fused into its
 * epilogue (FP32 within a 64-256 column tile, FP64 across tiles).  W, d_in, d_out,
 * U_packed, V_packed as for nq_recon_error; s1 (m), s2 (n): device float, updated in
 * place.  rel_err: host, or NULL: the reconstruction error after the refit
 * (synchronises when non-NULL).  sweeps >= 1.
 */
size_t nq_ls_refit_workspace_size(int64_t m, int64_t n, int32_t r);
nq_status nq_ls_refit(const void *W, nq_dtype dt, int64_t m, int64_t n, const float *d_in,
                      const float *d_out, const uint32_t *U_packed, const uint32_t *V_packed,
                      int32_t r, float *s1, float *s2, int32_t sweeps, double *rel_err,
                      void *ws, size_t ws_bytes, nq_stream_t stream);

/* ------------------------------------------------------------------------- */
/* 3. Inference with the packed factors.  NanoQuant summary page, "Technical    */
/* novelty" (技术新颖性) and "Limitations" (局限与改进): the compressed layer     */
/* is applied by binary GEMV/GEMM kernels that read the packed signs.          */
/* ------------------------------------------------------------------------- */

/* Batches of at most this many rows take the packed-bit (GEMV) path. */
#define NQ_BINARY_GEMV_MAX_BATCH 16

/* Workspace bytes of nq_binary_matmul for an m x n layer at rank r and batch B. */
size_t nq_binary_workspace_size(int64_t m, int64_t n, int32_t r, int64_t B);

/*
 * Y = X diag(s2) V+- U+-^T diag(s1), i.e. for each of the B input rows x (length n)
 *     y_i = s1_i sum_k U+-[i][k] sum_j V+-[j][k] s2_j x_j      (i < m)
 * with U+-, V+- decoded from the packed words of nq_lbadmm (bit 1 = -1, LSB-first).
 * Apply it to W~-space inputs; for the raw layer pass s1/d_out and s2/d_in as scales.
 *   U_packed [m][(r+31)/32], V_packed [n][(r+31)/32] (uint32), s1 (m), s2 (n) float,
 *   X [B][n] (dtype dt, row stride n), Y [B][m] float: all device.
 * B <= NQ_BINARY_GEMV_MAX_BATCH: SIMT kernels on the packed bits (FP32 sums, fixed
 * order).  Larger B: the signs are expanded once per call into BF16 +-1 tensor-core
 * operands in the workspace and both products run as tcgen05 GEMMs with split (hi + lo)
 * BF16 operands for the scaled inputs, FP32 accumulation.  Enqueue only.
 */
nq_status nq_binary_matmul(const uint32_t *U_packed, const uint32_t *V_packed, const float *s1,
                           const float *s2, int64_t m, int64_t n, int32_t r, const void *X,
                           nq_dtype dt, int64_t B, float *Y, void *ws, size_t ws_bytes,
                           nq_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Step-level interface over the ADMM state held in the workspace.             */
/* nq_lbadmm is nq_lbadmm_prepare + nq_lbadmm_iterate + nq_lbadmm_finish.      */
/* The state fields can be read and written (checkpoint / resume, tests).      */
/* ------------------------------------------------------------------------- */

/* Form W^ (and its transpose) from W, d_in, d_out; set V = V_0(seed) and zero the
 * dual state.  ``prec`` selects the operand precision of the following iterations (the
 * split low parts are formed for NQ_PREC_FP32 and zeroed otherwise).
 * gamma_out: host double or NULL (synchronises when non-NULL). */
nq_status nq_lbadmm_prepare(const void *W, nq_dtype dt, int64_t m, int64_t n, const float *d_in,
                            const float *d_out, int32_t r, uint64_t seed, nq_precision prec,
                            double *gamma_out, void *ws, size_t ws_bytes, nq_stream_t stream);

/* Run ``iters`` full iterations (U side then V side) at precision ``prec`` (use the one
 * given to nq_lbadmm_prepare).  objective: host float[iters] or NULL (synchronises when
 * non-NULL). */
nq_status nq_lbadmm_iterate(int64_t m, int64_t n, int32_t r, float rho, float lambda,
                            int32_t iters, int32_t K, nq_precision prec, float *objective,
                            void *ws, size_t ws_bytes, nq_stream_t stream);

/* One half iteration: side 0 updates U from V, side 1 updates V from U. */
nq_status nq_lbadmm_half_step(int64_t m, int64_t n, int32_t r, float rho, float lambda, int32_t K,
                              int32_t side, nq_precision prec, void *ws, size_t ws_bytes,
                              nq_stream_t stream);

/* Balance, extract s1/s2, pack, and (when final_rel_err != NULL) the reconstruction
 * error against W~ formed from W, d_in, d_out (synchronises then). */
nq_status nq_lbadmm_finish(const void *W, nq_dtype dt, int64_t m, int64_t n, const float *d_in,
                           const float *d_out, int32_t r, uint32_t *U_packed, uint32_t *V_packed,
                           float *s1, float *s2, float *final_rel_err, void *ws, size_t ws_bytes,
                           nq_stream_t stream);

/* State fields.  X = latent after its last step (rows x r, float); S = X + L, the
 * SVID input, from which the dual state is Z = sign(S) a b^T, L = S - Z (rows x r,
 * float); A = a (rows, float); B = b (r, float); WHAT = W^ (m x n, bf16, row
 * stride ld elements); WHAT_LO = its low part in NQ_PREC_FP32 (zero otherwise);
 * GAMMA = gamma (1 double); INV_STATS = the inverse update's counters (11 x 8 bytes:
 * [0] half steps whose G^-1 came from the Newton-Schulz update, [1] attempts that fell
 * back to Cholesky (uint64), [2] steps of the last accepted update (int64), [3..10]
 * ||I - X_k G||_F of the last attempt's steps (double)); GINV_U / GINV_V = G^-1 of the
 * last U / V solve, hi part (r x r, bf16, row stride ld), GINV_U_LO / GINV_V_LO its low
 * part (G^-1 = hi + lo). */
typedef enum {
    NQ_FIELD_U = 0, NQ_FIELD_V = 1, NQ_FIELD_SU = 2, NQ_FIELD_SV = 3, NQ_FIELD_AU = 4,
    NQ_FIELD_AV = 5, NQ_FIELD_BU = 6, NQ_FIELD_BV = 7, NQ_FIELD_WHAT = 8, NQ_FIELD_GAMMA = 9,
    NQ_FIELD_WHAT_LO = 10, NQ_FIELD_INV_STATS = 11, NQ_FIELD_GINV_U = 12,
    NQ_FIELD_GINV_U_LO = 13, NQ_FIELD_GINV_V = 14, NQ_FIELD_GINV_V_LO = 15
} nq_field;

/* Device address, element count, element size and row stride (elements) of a
 * state field inside the workspace.  The address is valid while ws is. */
nq_status nq_lbadmm_state_field(int64_t m, int64_t n, int32_t r, nq_field f, void *ws,
                                size_t ws_bytes, void **dev_ptr, int64_t *count,
                                int32_t *elem_bytes, int64_t *ld);

/* Re-derive the BF16 operand copies (transposes of U and V, with their low parts at
 * NQ_PREC_FP32, and W^^T) after a caller has written NQ_FIELD_U / NQ_FIELD_V /
 * NQ_FIELD_WHAT (/ NQ_FIELD_WHAT_LO) directly.  A warm start from a similar layer is
 * nq_lbadmm_prepare, then the other layer's V written into NQ_FIELD_V, then this call,
 * then nq_lbadmm_iterate. */
nq_status nq_lbadmm_sync_operands(int64_t m, int64_t n, int32_t r, nq_precision prec, void *ws,
                                  size_t ws_bytes, nq_stream_t stream);

/* Device error word of a workspace: 0 if clean, else the first nq_status raised
 * on the device since the last reset; resets it.  Synchronises the stream. */
nq_status nq_lbadmm_check(int64_t m, int64_t n, int32_t r, void *ws, size_t ws_bytes,
                          nq_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Measurement helpers (not steps of the method).  When enabled, the library   */
/* records a pair of CUDA events on the launching stream around every kernel   */
/* launch and attributes the elapsed device time to the kernel's class.  Each  */
/* class's launches are also wrapped in an NVTX range named "nq.<class>".      */
/* Off by default; recording costs one event pair per launch.  Not for use     */
/* while the stream is being captured into a CUDA graph.                       */
/* ------------------------------------------------------------------------- */
typedef enum {
    NQ_K_CALIB = 0,     /* calibration moment reduction (both streams)              */
    NQ_K_CALIB_FIN = 1, /* moments finalize + Ledoit-Wolf                            */
    NQ_K_PREP = 2,      /* target preparation, V_0                                   */
    NQ_K_GRAM = 3,      /* tcgen05 Gram X^T X + (lambda + rho) I                     */
    NQ_K_CHOL = 4,      /* Cholesky factorisation + triangular inverse (FP32 SIMT)   */
    NQ_K_RHS = 5,       /* tcgen05 W^ X + rho (Z - L)                                */
    NQ_K_SOLVE = 6,     /* tcgen05 R G^-1 with the dual-state epilogue               */
    NQ_K_SVID = 7,      /* SVID power passes                                         */
    NQ_K_OBJ = 8,       /* per-iteration objective                                   */
    NQ_K_FINISH = 9,    /* balancing, scales, packing                                */
    NQ_K_RECON = 10,    /* tcgen05 +-1 reconstruction error                          */
    NQ_K_GINV = 11,     /* tcgen05 G^-1 = L^-T L^-1 (symmetric, split BF16)          */
    NQ_K_BINARY = 12,   /* binary GEMV/GEMM on the packed factors                    */
    NQ_K_REFIT = 13,    /* least-squares scale refit                                 */
    NQ_K_NEWTON = 14,   /* tcgen05 Newton-Schulz update of G^-1                      */
    NQ_K_GD = 15,       /* gradient-descent latent update (solver variant)           */
    NQ_K_COUNT = 16
} nq_kernel_class;

/* Number of kernel launches the library has issued in this process. */
int64_t nq_launch_count(void);

/* Enable (1) or disable (0) recording; enabling also clears previous records. */
nq_status nq_profile_enable(int32_t enable);
/* Launch count and summed device milliseconds of one class since enabling.
 * Synchronises with the recorded events. */
nq_status nq_profile_get(int32_t kernel_class, int64_t *launches, double *total_ms);

/* ------------------------------------------------------------------------- */
/* Diagnostics (no counterpart in the pages): run a device-side error path on  */
/* purpose so that a test can check it ends with a status and leaves the       */
/* context usable.                                                             */
/* ------------------------------------------------------------------------- */
typedef enum {
    NQ_SELFTEST_WAIT_TIMEOUT = 0, /* the bounded counter wait of the Cholesky dataflow, on a
                                     word nothing sets, with a poll budget of a few ms:
                                     returns NQ_ERR_TIMEOUT */
    NQ_SELFTEST_NOT_SPD = 1       /* the cooperative Cholesky + inverse kernel on G = -I
                                     (64 x 64): returns NQ_ERR_NOT_SPD */
} nq_selftest_kind;

/* Bytes of device workspace nq_selftest needs (256-byte aligned). */
size_t nq_selftest_workspace_size(void);

/* Run one diagnostic; the workspace (device, caller-owned, 256-byte aligned) is cleared
 * first.  Returns the device status the run raised (NQ_OK if none), NQ_ERR_INVALID_ARG /
 * NQ_ERR_WORKSPACE for bad arguments, NQ_ERR_UNSUPPORTED off sm_100.  Synchronises. */
nq_status nq_selftest(int32_t kind, void *ws, size_t ws_bytes, nq_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* NQ_H */
