// Launchers of the non-GEMM kernels (SIMT, sm_100a).
#pragma once
#include "common.cuh"
#include "layout.h"

namespace nq {

// ---- calibration -----------------------------------------------------------------
// Partial sums of x^2 and x^4 per (token slab, channel) in FP64.
cudaError_t calib_partials(const void *X, int64_t T, int64_t C, int dt_bf16, int nslab,
                           double *ps, double *pq, cudaStream_t s);
// s_c, q_c = sum over slabs / T.
cudaError_t calib_moments(const double *ps, const double *pq, int nslab, int64_t T, int64_t C,
                          double *s_out, double *q_out, cudaStream_t st);
// Ledoit-Wolf diagonal shrinkage -> d (float), alpha (double, device).
cudaError_t calib_ledoit_wolf(const double *s, const double *q, int64_t T, int64_t C,
                              double alpha_override, float *d, double *alpha, int *err,
                              cudaStream_t st);
int calib_num_slabs(int64_t T, int64_t C);

// ---- preconditioned target -----------------------------------------------------
// part[b] = partial sums of (d_out_i W_ij d_in_j)^2; non-finite -> NQ_ERR_NONFINITE.
cudaError_t wt_norm_partials(const void *W, int w_bf16, int64_t m, int64_t n, const float *d_in,
                             const float *d_out, double *part, int *err, cudaStream_t s);
// sum of ``count`` partials in fixed order; writes *sum and, when gamma != null,
// *gamma = sqrt(sum) / (2 sqrt(r)).
cudaError_t reduce_partials(const double *part, int count, double *sum, double *gamma, int r,
                            cudaStream_t s);
// W^ = bf16(d_out W d_in / gamma) into What [m][ldn] and WhatT [n][ldm] (zero padded);
// with WhatL / WhatTL non-null also the low parts bf16(x - bf16(x)) of a split operand.
// part[b] = partial sums of W^^2 (of hi + lo when split).
cudaError_t what_cast(const void *W, int w_bf16, int64_t m, int64_t n, const float *d_in,
                      const float *d_out, const double *gamma, __nv_bfloat16 *What, int64_t ldn,
                      __nv_bfloat16 *WhatT, int64_t ldm, __nv_bfloat16 *WhatL,
                      __nv_bfloat16 *WhatTL, double *part, cudaStream_t s);
// V_0 = sqrt(2/n) * splitmix64 signs into X [n][ldr] (float) and Xt [r][ldn] (bf16; XtL,
// when non-null, the low part).
cudaError_t init_v0(int64_t n, int32_t r, uint64_t seed, float *X, int64_t ldr,
                    __nv_bfloat16 *Xt, __nv_bfloat16 *XtL, int64_t ldn, cudaStream_t s);
// Xt[k][i] = bf16(X[i][k]) for i < rows, k < r (XtL, when non-null: the low part).
cudaError_t transpose_to_bf16(const float *X, int64_t rows, int32_t r, int64_t ldx,
                              __nv_bfloat16 *Xt, __nv_bfloat16 *XtL, int64_t ldt, cudaStream_t s);
// B[j][i] = A[i][j] (bf16), A rows x cols with row stride lda, B row stride ldb.
cudaError_t transpose_bf16(const __nv_bfloat16 *A, int64_t rows, int64_t cols, int64_t lda,
                           __nv_bfloat16 *B, int64_t ldb, cudaStream_t s);

// ---- Cholesky + inverse (cooperative, FP32) -------------------------------------
// G = L L^T for the SPD r x r matrix G (row stride r); writes (L^-1)^T as hi + lo bf16
// [r][ldr] (LiT_hi, LiT_lo).  A, Li: rp x rp FP32 scratch; flags: 2 (rp/64)^2 counters.
// max_ctas > 0 limits the cooperative grid (at least 3 CTAs); 0: one CTA per SM.
// gate: optional device word; the launch does nothing when bit (*gate) of gate_skip is
// set at its start.  zero_state: zero the flags and the grid barrier first (else the
// caller has zeroed the flags, and the barrier words are as a completed barrier left them).
cudaError_t chol_inverse(const float *G, int32_t r, int64_t rp, float *A, float *Li,
                         __nv_bfloat16 *LiT_hi, __nv_bfloat16 *LiT_lo, int64_t ldr,
                         unsigned int *flags, int *err, unsigned int *bar, int max_ctas,
                         const int *gate, int gate_skip, bool zero_state, cudaStream_t s);

// ---- SVID -------------------------------------------------------------------------
// K power steps on |S| (S rows x r, row stride ldf): a = t/||t||, b = A^T t / ||t||.
cudaError_t svid(const float *S, int64_t rows, int32_t r, int64_t ldf, int K, int nsv,
                 float *bcur, float *tvec, float *partb, double *partn, float *a, float *b,
                 cudaStream_t s);

// ---- inference with the packed factors (binary.cu) --------------------------------
// Row chunks of the GEMV path's z pass (partials: chunks x B x r floats).
int bin_gemv_chunks(int64_t n, int32_t r, int64_t B);
// Y = X diag(s2) V+- U+-^T diag(s1) for B <= NQ_BINARY_GEMV_MAX_BATCH on the packed bits;
// P: partials, z: B x r floats.
cudaError_t bin_gemv(const uint32_t *Up, const uint32_t *Vp, const float *s1, const float *s2,
                     int64_t m, int64_t n, int32_t r, const void *X, int x_bf16, int64_t B,
                     float *Y, float *P, float *z, cudaStream_t s);
// Tensor-path operands: Vt hi/lo [r][ldt] (scaled signs of V), Um [m][ldr] (+-1), X split
// into BF16 hi (and lo for FP32 X) rows of stride ldx.
cudaError_t bin_expand(const uint32_t *Up, const uint32_t *Vp, const float *s2, int64_t m,
                       int64_t n, int32_t r, const void *X, int x_bf16, int64_t B,
                       __nv_bfloat16 *Vh, __nv_bfloat16 *Vl, int64_t ldt, __nv_bfloat16 *Um,
                       int64_t ldr, __nv_bfloat16 *Xh, __nv_bfloat16 *Xl, int64_t ldx,
                       cudaStream_t s);

// ---- split-K Gram reduction ------------------------------------------------------
// ---- gradient-descent latent update (solver variant) --------------------------------
// *maxbits = bits of max_i sum_j |G_ij| (non-negative floats order as their bits; the word
// must be zero before the launch).
cudaError_t gd_rowabs_max(const float *G, int32_t r, unsigned int *maxbits, cudaStream_t s);
// Ph/Pl[i][k] = hi / lo BF16 split of X[i][k] (rows x r, X stride ldf, P stride ldp).
cudaError_t split_rows(const float *X, int64_t rows, int32_t r, int64_t ldf,
                       __nv_bfloat16 *Ph, __nv_bfloat16 *Pl, int64_t ldp, cudaStream_t s);
// The solve epilogue's state update for a latent X formed elsewhere: S <- X + S - sign(S) a b^T,
// Xt[k][i] = bf16(X[i][k]) (+ XtL the low part when set), and, when ``objective`` is set,
// nparts FP64 partial sums of (R - rho (2 Z - S_old)) . xo into part (xo: X as the operands
// hold it, R = Rhi + Rlo).  A non-finite X raises NQ_ERR_NONFINITE.
cudaError_t gd_finalize(const float *X, float *S, const float *a, const float *b, int64_t rows,
                        int32_t r, int64_t ldf, float rho, const __nv_bfloat16 *Rhi,
                        const __nv_bfloat16 *Rlo, int64_t ldr, __nv_bfloat16 *Xt,
                        __nv_bfloat16 *XtL, int64_t ldxt, int objective, double *part,
                        int nparts, int *err, cudaStream_t s);

// G (r x r) = sum_{s < S} P[s * T + t] (raw 128 x 128 lower-triangular tiles t < T) +
// diag I, each off-diagonal tile also stored mirrored.
// Gh/Gl (optional, ld ldg): the same Gram split into hi + lo BF16.
cudaError_t gram_reduce(const float *P, int T, int S, int r, float diag, float *G,
                        __nv_bfloat16 *Gh, __nv_bfloat16 *Gl, int64_t ldg, cudaStream_t s);

// ---- objective --------------------------------------------------------------------
// obj[slot] = (what_n2 - 2 sum(px) + <GU - cI, GV - cI>) / what_n2
cudaError_t objective(const float *GU, const float *GV, int32_t r, float c, const double *px,
                      int npx, double *part, const Scalars *sc, float *obj_slot,
                      cudaStream_t s);

// ---- balancing, scales, packing ---------------------------------------------------
cudaError_t column_sumsq(const float *X, int64_t rows, int32_t r, int64_t ldf, int nblk,
                         float *partb, cudaStream_t s);
cudaError_t balance_gains(const float *partU, const float *partV, int nblk, int32_t r, float *gk,
                          cudaStream_t s);
// s_i = scale * mean_k |X_ik g_k^e| (e = +1 for U, -1 for V); sign bits; +-1 bf16 copy.
cudaError_t extract_pack(const float *X, int64_t rows, int32_t r, int64_t ldf, const float *gk,
                         int invert, const double *gamma, float *s_out, uint32_t *bits,
                         __nv_bfloat16 *pm, int64_t ldpm, cudaStream_t s);
cudaError_t pack_signs(const float *X, int64_t rows, int32_t r, int64_t ldx, uint32_t *bits,
                       cudaStream_t s);
// +-1 bf16 [rows][ldpm] from packed bits.
cudaError_t unpack_pm(const uint32_t *bits, int64_t rows, int32_t r, __nv_bfloat16 *pm,
                      int64_t ldpm, cudaStream_t s);
// s_i = sum_t num[t][i] / sum_t den[t][i] over ntiles partial rows (kept when den = 0)
cudaError_t refit_scales(const double *num, const double *den, int ntiles, int64_t M, float *s,
                         cudaStream_t st);
// *out = sqrt(sum(part) / wt_norm2) (0 when both vanish)
cudaError_t recon_finalize(const double *part, int count, const Scalars *sc, double *out,
                           cudaStream_t s);

}  // namespace nq
