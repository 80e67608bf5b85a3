// tcgen05 / TMEM / TMA GEMM for sm_100a with fused LB-ADMM epilogues.
//
// D[M x N] = sum over K-segments s of A_s[M x K_s] . B_s[N x K_s]^T, all operands BF16
// and K-major (row-major with K contiguous), accumulation FP32 in tensor memory.  With
// split3 the three products of split operands (hi.hi + lo.hi + hi.lo) share one stage of
// four tiles per k-block, so each operand tile is loaded once.
// Persistent: one CTA per SM walks 128 x BN output tiles round-robin.  Per CTA:
//   warp 0     one elected thread issues TMA tile loads into a STAGES-deep ring
//   warp 1     allocates TMEM (two accumulator stages of BN columns); one elected thread
//              issues tcgen05.mma (M=128, N=BN, K=16 per instruction, 4 per 64-wide K
//              block) and commits to mbarriers
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (warp w owns TMEM lanes
//              32*(w%4) .. +31, i.e. those tile rows), fused element-wise work, stores
// Every mbarrier wait is bounded; a wait that runs out raises NQ_ERR_TIMEOUT.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "layout.h"

namespace nq {
namespace tc {

constexpr int BM = 128;
constexpr int BK = 64;                 // 64 bf16 = 128 B = one 128B-swizzle atom row
constexpr int A_TILE_BYTES = BM * BK * 2;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;

enum Epi : int { EPI_GRAM = 0, EPI_RHS = 1, EPI_SOLVE = 2, EPI_RECON = 3, EPI_SPLIT = 4,
                 EPI_SCALE = 5, EPI_REFIT = 6, EPI_NS1 = 7, EPI_NS2 = 8, EPI_GD = 9 };

struct Maps {
    CUtensorMap a[3];
    CUtensorMap b[3];
};

struct EpiParams {
    int M, N;
    int nseg;
    int kblocks[3];
    int split3;         // split (hi + lo) operands in one pass over K: A_hi = maps.a[0],
                        // A_lo = maps.a[1], B_hi = maps.b[0], B_lo = maps.b[1]; D = the sum of
                        // hi.hi + lo.hi + hi.lo over kblocks[0] k-blocks
    int tri_k;          // operands zero for k < row index: start each tile's K at max(m0, n0)
    int sym;            // symmetric result (EPI_SPLIT / EPI_GRAM, BN == BM, M == N): lower-
                        // triangular tiles only, each off-diagonal tile also written mirrored
    int nfast;          // tiles in n-fastest order (see tile_origin)
    int max_ctas;       // 0: one CTA per SM; else at most this many CTAs (SMs left free for
                        // kernels running beside this one on another stream)
    int ksplit;         // EPI_GRAM only: > 1 splits the K range into ksplit parts; unit u
                        // (tile u % T, part u / T) writes its raw 128 x 128 tile to
                        // out + u * 128 * 128 (row-major, ld 128) for a later reduction.
                        // Every part must get at least one k-block.
    int *err;
    // Gate: when set, the whole launch returns at once if bit (*gate) of gate_skip is set
    // (the word is read once by every thread before any other work)
    const int *gate;
    int gate_skip;
    // EPI_GRAM: out[row*ldo + col] = acc + (row == col ? diag : 0); when Rhi is set, the
    // same value also split into hi + lo BF16 (Rhi/Rlo, ld ldr); when ns is set, CTA 0
    // opens the Newton-Schulz gate of the half step (ns->gate = NS_RUNNING)
    float *out;
    int64_t ldo;
    float diag;
    // EPI_RHS / EPI_SOLVE: dual state of the side being updated
    float *S;            // [M][ldf]
    const float *a;      // [M]
    const float *b;      // [N]
    int64_t ldf;
    float rho;
    // EPI_SPLIT: Rhi/Rlo[row * ldr + col] = hi + lo bf16 split of acc
    // EPI_RHS: R = acc + rho (2 sign(S) a b^T - S) split into hi + lo bf16
    __nv_bfloat16 *Rhi, *Rlo;  // [M][ldr]
    int64_t ldr;
    // EPI_SOLVE: X = acc; S <- X + S - sign(S) a b^T; Xt[col][row] = bf16(X) and, when XtL
    // is set, XtL[col][row] = bf16(X - Xt) (the low part of a split-BF16 operand).  The
    // objective partial takes X as the operands hold it (Xt, + XtL), so that it belongs
    // to the same latents as the Grams of the operands.
    float *X;                  // [M][ldf]
    __nv_bfloat16 *Xt, *XtL;   // [N][ldxt]
    int64_t ldxt;
    int objective;             // also sum (R - rho (2Z - S_old)) . X into part[tile]
    double *part;              // per-tile partial sums (EPI_SOLVE objective, EPI_RECON)
    // EPI_SCALE: out[row * ldo + col] = acc * s1[col]
    // EPI_RECON: sum_ij (d_out_i W_ij d_in_j - s1_i acc s2_j)^2
    const void *W;
    int w_bf16;
    int w_vec;                 // W rows 16-byte aligned: vector loads in the epilogue
    int cvec;                  // EPI_RECON / EPI_REFIT: the per-column vectors (d_in or d_out,
                               // s2 or sv) start 16-byte aligned: vector loads
    int64_t ldw;
    const float *d_in, *d_out, *s1, *s2;
    // EPI_REFIT: acc = P (row, col) of the +-1 product; with w = W~ of the pair (W read as
    // W[col][row] when refit_trans, i.e. the GEMM's rows are W's columns), accumulate
    // num[tn][row] = sum_col w acc sv[col] and den[tn][row] = sum_col acc^2 sv[col]^2 over
    // the tile's BN columns (tn = the tile's column index)
    int refit_trans;
    const float *sv;
    double *num, *den;
    // Newton-Schulz step k (ns_step) towards G^-1 from X_k, in the form
    // X_{k+1} = X_k (2I - G X_k) = X_k + E_k X_k with E_k = I - X_k G:
    // EPI_NS1: acc = (X_k G)(row, col); E_k = delta - acc split into Rhi/Rlo; the tile's
    //   sum of E_k entries squared goes to part[tile]; the CTA finishing the last tile
    //   forms ||E_k||_F and moves ns->gate: NS_FINAL if k >= ns_min_final and it is
    //   <= ns_tau; NS_FAIL if it is not finite, if k == ns_last without NS_FINAL, if it
    //   grew above 1.5 x the previous step's during the BF16 steps (k < ns_min_final),
    //   or did not fall below 0.9 x the previous step's after the first split step
    //   (k > ns_min_final).
    // EPI_NS2: acc = (E_k X_k)(row, col); X_{k+1} = (Ph + Pl) + acc split into hi + lo,
    //   written to Rhi/Rlo, or to Fhi/Flo when the gate reads NS_FINAL (then the CTA
    //   finishing the last tile sets NS_DONE).
    // EPI_GD (a gradient step of the latent update): acc = (X G)(row, col); with R = Ph + Pl
    // (ld ldr) and eta = 1 / *gd_max: X[row][col] <- X - eta (acc - R) (X: FP32, ld ldf, in
    // place) and its hi + lo split to Fhi/Flo (ld ldr), the next step's operand
    const float *gd_max;
    NsState *ns;
    unsigned int *zero;   // EPI_GRAM: zero_words words zeroed before the tiles (counters
    int zero_words;       // of the factorisation that follows on another stream)
    int ns_step, ns_last, ns_min_final;
    float ns_tau;
    const __nv_bfloat16 *Ph, *Pl;   // X_k (hi, lo), ld ldr
    __nv_bfloat16 *Fhi, *Flo;       // destination of the final iterate, ld ldr
};

// Host: encode a 2-D BF16 tensor map over rows x cols (row stride ld elements) with
// a box of 64 x box_rows and 128-byte swizzle.  Returns false on failure.
bool make_map_bf16(CUtensorMap *map, const void *base, int64_t rows, int64_t cols, int64_t ld,
                   int box_rows);

// Host: launch one GEMM.  BN in {64, 128, 256}.
cudaError_t launch_gemm(const Maps &maps, const EpiParams &p, int epi, int BN, cudaStream_t s);

// Newton-Schulz update of G^-1 (all steps) in one cooperative launch on 128 x 128 tiles.
// X buffers (hi + lo BF16, r x r, ld ldr): 0 holds X_0 on entry and receives the accepted
// iterate; 1 and 2 hold the iterates between steps.  E: the residual I - X_k G.
struct NsMaps {
    CUtensorMap xh[3], xl[3];   // box 64 x 128
    CUtensorMap gh, gl;         // the Gram, split (box 64 x 128)
    CUtensorMap eh;             // E hi (box 64 x 128)
};
struct NsArgs {
    int r;
    int64_t ldr;
    int nsteps, bf16_steps;     // steps enqueued; the first bf16_steps residuals in BF16
    float tau;                  // ||E_k||_F that makes X_{k+1} final
    int *err;
    NsState *ns;                // gate, ticket and grid_count reset by the Gram
    double *part;               // per-tile partials of ||E_k||_F^2
    __nv_bfloat16 *xh[3], *xl[3];
    __nv_bfloat16 *eh, *el;
};
cudaError_t launch_newton(const NsMaps &maps, const NsArgs &a, int max_ctas, cudaStream_t s);

// Host: number of output tiles of a launch (size of the per-tile partial array).
inline int64_t num_tiles(int M, int N, int BN) { return ceil_div(M, BM) * ceil_div(N, BN); }

}  // namespace tc
}  // namespace nq
