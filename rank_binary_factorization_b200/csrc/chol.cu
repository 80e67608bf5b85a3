// Cholesky G = L L^T of the r x r SPD system matrix of the U (V) step and L^-1;
// (L^-1)^T is emitted as BF16 hi + lo for the tensor-core product G^-1 = L^-T L^-1.
// NanoQuant summary page, "Core method" (核心方法), step (a): the regularised linear
// system is solved through a Cholesky factorisation.
//
// One cooperative launch (one CTA of 256 threads per SM) of FP32 SIMT work on 64 x 64
// tiles, scheduled as a dataflow with per-tile completion counters (bounded waits):
//   * CTA 0 runs the critical chain of the blocked right-looking factorisation: tile
//     Cholesky of the diagonal tile, its inverse, the panel tile below it (one tile
//     product A L_jj^-T) and the look-ahead update of the next diagonal tile;
//   * every panel tile L_ij is also stored transposed in the unused upper tile (j, i) of
//     A, and L_jj^-T in the unused upper tile (j, j+1) of L^-1, so all operand tiles are
//     plain cp.async copies;
//   * CTA 1 takes the tasks CTA 0 needs next (panel (j+2, j), updates of (j+2, j+1) and
//     (j+2, j+2)); CTAs 2.. take the other panel tiles and the trailing updates
//     round-robin in a topological order, so every wait ends;
//   * the 64 x 64 tile Cholesky works in 16-column blocks factored by one warp with
//     shuffles (no CTA barrier per column); while that warp sweeps a block, three warps
//     prepare the next block's update (including its share of the look-ahead update) and
//     four warps invert the blocks already finished, so the tile's inverse and update
//     cost little beyond the column sweeps;
//   * L^-1 in the same dataflow: block column m is a forward substitution advanced one
//     block row per factorisation step (X_jm = -L_jj^-1 sum_k L_jk X_km), so the inverse
//     trails the factorisation instead of following it;
//   * (L^-1)^T is written as bf16 hi + lo; G^-1 = L^-T L^-1 is then one split-BF16
//     tensor-core GEMM (see gemm_tc.cu, EPI_SPLIT).
#include "kernels.cuh"

namespace nq {
namespace {

constexpr int TB = 64;      // tile edge
constexpr int LDS = 68;     // shared-memory row stride (floats): float4 aligned, fewer conflicts

using Tile = float[TB][LDS];

struct Chol2Args {
    const float *G;
    int r;
    int nb;
    int64_t rp;
    float *A;     // rp x rp working copy -> L (lower tiles)
    float *Li;    // rp x rp: L^-1 (lower tiles), scratch T in upper tiles
    __nv_bfloat16 *hi, *lo;
    int64_t ldr;
    unsigned int *cnt;  // 2 x nb x nb: operations completed on tile (i, k) of L, of L^-1
    int *err;
    unsigned int *bar;
    const int *gate;    // when set, the launch returns at once if bit (*gate) of
    int gate_skip;      // gate_skip is set
};

// ---- tile movement (L2-coherent loads: other CTAs write the tiles between tasks) -----
__device__ __forceinline__ void load_n(Tile &d, const float *M, int64_t ld, int ti, int tj) {
    const float *base = M + (int64_t)ti * TB * ld + (int64_t)tj * TB;
    for (int f = threadIdx.x; f < TB * TB / 4; f += blockDim.x) {
        const int row = f >> 4, c4 = (f & 15) * 4;
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(base + (int64_t)row * ld + c4));
        *reinterpret_cast<float4 *>(&d[row][c4]) = v;
    }
}
__device__ __forceinline__ void store_n(float *M, int64_t ld, int ti, int tj, const Tile &s) {
    float *base = M + (int64_t)ti * TB * ld + (int64_t)tj * TB;
    for (int f = threadIdx.x; f < TB * TB / 4; f += blockDim.x) {
        const int row = f >> 4, c4 = (f & 15) * 4;
        __stcg(reinterpret_cast<float4 *>(base + (int64_t)row * ld + c4),
               *reinterpret_cast<const float4 *>(&s[row][c4]));
    }
}

// Asynchronous plain tile load (cp.async, L2 only): completes at cp_async_wait.
__device__ __forceinline__ void load_n_async(Tile &d, const float *M, int64_t ld, int ti, int tj) {
    const float *base = M + (int64_t)ti * TB * ld + (int64_t)tj * TB;
    for (int f = threadIdx.x; f < TB * TB / 4; f += blockDim.x) {
        const int row = f >> 4, c4 = (f & 15) * 4;
        const uint32_t sa = (uint32_t)__cvta_generic_to_shared(&d[row][c4]);
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa),
                     "l"(base + (int64_t)row * ld + c4)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Thread's 4 x 4 block of a 64 x 64 tile: rows a0..a0+3, columns b0..b0+3.
__device__ __forceinline__ int blk_a0() { return (threadIdx.x >> 4) * 4; }
__device__ __forceinline__ int blk_b0() { return (threadIdx.x & 15) * 4; }

// acc[i][j] += sum_c X[a0+i][c] * Y[c][b0+j]  (both tiles in plain layout)
__device__ __forceinline__ void mac_n(float (&acc)[4][4], const Tile &X, const Tile &Y) {
    const int a0 = blk_a0(), b0 = blk_b0();
#pragma unroll 2
    for (int c = 0; c < TB; c += 4) {
        float x[4][4], y[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 v = *reinterpret_cast<const float4 *>(&X[a0 + i][c]);
            x[i][0] = v.x;
            x[i][1] = v.y;
            x[i][2] = v.z;
            x[i][3] = v.w;
            const float4 w = *reinterpret_cast<const float4 *>(&Y[c + i][b0]);
            y[i][0] = w.x;
            y[i][1] = w.y;
            y[i][2] = w.z;
            y[i][3] = w.w;
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(x[i][cc], y[cc][j], acc[i][j]);
    }
}

__device__ __forceinline__ void zero(float (&acc)[4][4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
}

// Write the 4 x 4 register block (times sgn) straight to a global tile.
__device__ __forceinline__ void put(float *M, int64_t ld, int ti, int tj, const float (&acc)[4][4],
                                   float sgn) {
    const int a0 = blk_a0(), b0 = blk_b0();
    float *base = M + ((int64_t)ti * TB + a0) * ld + (int64_t)tj * TB + b0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        __stcg(reinterpret_cast<float4 *>(base + (int64_t)i * ld),
               make_float4(sgn * acc[i][0], sgn * acc[i][1], sgn * acc[i][2], sgn * acc[i][3]));
}

// Write the transpose of the thread's 4 x 4 block (of a tile product) into tile (ti, tj):
// entry (a0 + i, b0 + q) of the product goes to row b0 + q, column a0 + i.
__device__ __forceinline__ void put_t(float *M, int64_t ld, int ti, int tj,
                                      const float (&acc)[4][4]) {
    const int a0 = blk_a0(), b0 = blk_b0();
    float *base = M + ((int64_t)ti * TB + b0) * ld + (int64_t)tj * TB + a0;
#pragma unroll
    for (int q = 0; q < 4; ++q)
        __stcg(reinterpret_cast<float4 *>(base + (int64_t)q * ld),
               make_float4(acc[0][q], acc[1][q], acc[2][q], acc[3][q]));
}

// ---- the chain CTA's tile step: factorisation, look-ahead update and inverse ----------
// The column sweep of a 16-column block (warp 0) is a latency chain; the update of the
// next block column that does not depend on the block being swept - including its share
// of the pending rank-64 update with the panel P when FUSE - is formed meanwhile by warps
// 1-3 and 5-7 (warps share an SM sub-partition by warp % 4, so warp 4 stays idle and
// leaves warp 0's sub-partition to it).  After the sweeps, L^-1 is formed block-wise in
// four levels by all warps and lit = li^T.
//   warp 0        factors block b column by column (lane l holds rows 16b + l and
//                 16b + l + 32; column k's multipliers are broadcast by shuffles; every
//                 lane tracks the block's diagonal, so the next pivot needs no shuffle; a
//                 non-positive pivot is recorded and replaced, without a branch);
//   warps 1-3,5-7 sum_m P[i][m] P[c][m] + sum over finished blocks < b of s[i][m] s[c][m]
//                 for block b+1's entries (four pairs at a time), then, after the sweep,
//                 block b's share, and store block b+1's updated columns.
// s: the tile (lower triangle read; L on return); P: the panel L_{j+1,j} in natural layout
// (FUSE only); tmp: scratch of the inverse's block products.
// Warp-level 16 x 16 x 16 product c (+)= A_blk B_blk: lane = row (lane & 15), 8 columns.
__device__ __forceinline__ void blk_acc(float (&c)[8], const Tile &A, int ar, int ac,
                                        const Tile &B, int br, int bc) {
    const int lane = threadIdx.x & 31, row = lane & 15, col0 = (lane >> 4) * 8;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float a = A[ar + row][ac + k];
        const float4 y0 = *reinterpret_cast<const float4 *>(&B[br + k][bc + col0]);
        const float4 y1 = *reinterpret_cast<const float4 *>(&B[br + k][bc + col0 + 4]);
        c[0] = fmaf(a, y0.x, c[0]);
        c[1] = fmaf(a, y0.y, c[1]);
        c[2] = fmaf(a, y0.z, c[2]);
        c[3] = fmaf(a, y0.w, c[3]);
        c[4] = fmaf(a, y1.x, c[4]);
        c[5] = fmaf(a, y1.y, c[5]);
        c[6] = fmaf(a, y1.z, c[6]);
        c[7] = fmaf(a, y1.w, c[7]);
    }
}

__device__ __forceinline__ void blk_store(Tile &D, int dr, int dc, const float (&c)[8], float sgn) {
    const int lane = threadIdx.x & 31, row = lane & 15, col0 = (lane >> 4) * 8;
    *reinterpret_cast<float4 *>(&D[dr + row][dc + col0]) =
        make_float4(sgn * c[0], sgn * c[1], sgn * c[2], sgn * c[3]);
    *reinterpret_cast<float4 *>(&D[dr + row][dc + col0 + 4]) =
        make_float4(sgn * c[4], sgn * c[5], sgn * c[6], sgn * c[7]);
}

// Dot products of four (row i_u, row c_u) pairs over columns [m0, m1) of one tile, summed
// into acc[u] (four independent chains).
__device__ __forceinline__ void dot4(float (&acc)[4], const Tile &X, const int (&i)[4],
                                     const int (&c)[4], int m0, int m1) {
#pragma unroll 2
    for (int m = m0; m < m1; m += 4) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float4 x = *reinterpret_cast<const float4 *>(&X[i[u]][m]);
            const float4 y = *reinterpret_cast<const float4 *>(&X[c[u]][m]);
            acc[u] = fmaf(x.x, y.x, fmaf(x.y, y.y, fmaf(x.z, y.z, fmaf(x.w, y.w, acc[u]))));
        }
    }
}

template <bool FUSE>
__device__ void chain_tile(Tile &s, const Tile &P, float *rdiag, Tile &li, Tile &lit, Tile &tmp,
                           int *err) {
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    // update workers: warps 1-3 and 5-7, thread index tw in [0, 192)
    const bool upd = warp != 0 && warp != 4;
    const int tw = (warp < 4 ? warp - 1 : warp - 2) * 32 + lane;
    bool bad = false;
    // block 0's share of the pending update, by all warps: pairs (i, c), i < 64, c < 16
    if (FUSE) {
        int ii[4], cc[4];
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int pr = u * 256 + t;
            ii[u] = pr >> 4;
            cc[u] = pr & 15;
        }
        dot4(acc, P, ii, cc, 0, TB);
#pragma unroll
        for (int u = 0; u < 4; ++u) s[ii[u]][cc[u]] -= acc[u];
    }
    __syncthreads();
#pragma unroll 1
    for (int b = 0; b < 4; ++b) {
        const int c0 = 16 * b;
        // block b+1's pairs: (i, c), i in [c0+16, 64), c in [c0+16, c0+32); pair
        // pr = u * 192 + tw, u < 4 (pairs past np are clamped onto a valid one, not stored)
        const int np = (48 - c0) * 16;
        int ii[4], cc[4];
        float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int pr = min(u * 192 + tw, np - 1);
            ii[u] = c0 + 16 + (pr >> 4);
            cc[u] = c0 + 16 + (pr & 15);
        }
        if (warp == 0) {
            const int r0 = c0 + lane, r1 = r0 + 32;
            float a0[16], a1[16], d[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                a0[c] = (r0 < TB) ? s[r0][c0 + c] : 0.f;
                a1[c] = (r1 < TB) ? s[r1][c0 + c] : 0.f;
                d[c] = s[c0 + c][c0 + c];
            }
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                bad |= !(d[k] > 0.f);
                const float il = rsqrtf(fmaxf(d[k], 1e-30f));
                if (lane == 0) rdiag[c0 + k] = il;
                const float l0 = a0[k] * il, l1 = a1[k] * il;
                a0[k] = l0;
                a1[k] = l1;
#pragma unroll
                for (int c = k + 1; c < 16; ++c) {
                    const float lc = __shfl_sync(0xffffffffu, l0, c);  // L_{c0+c, c0+k}
                    a0[c] = fmaf(-l0, lc, a0[c]);
                    a1[c] = fmaf(-l1, lc, a1[c]);
                    d[c] = fmaf(-lc, lc, d[c]);
                }
            }
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                if (r0 < TB) s[r0][c0 + c] = (lane >= c) ? a0[c] : 0.f;
                if (r1 < TB) s[r1][c0 + c] = a1[c];
            }
        } else if (upd && b < 3) {
            if (FUSE) dot4(part, P, ii, cc, 0, TB);
            dot4(part, s, ii, cc, 0, c0);
        }
        __syncthreads();
        if (b < 3) {
            if (upd) {   // block b's share; store block b+1's columns
                dot4(part, s, ii, cc, c0, c0 + 16);
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (u * 192 + tw < np) s[ii[u]][cc[u]] -= part[u];
            }
            __syncthreads();
        }
    }
    // L^-1 by 16 x 16 blocks: X_aa by forward substitution, then
    // X_ak = -X_aa sum_{l=k}^{a-1} L_al X_lk by distance a - k = 1, 2, 3
    if (warp < 4 && lane < 16) {
        const int o = 16 * warp;
        float x[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) x[c] = (c == lane) ? 1.f : 0.f;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            x[c] *= rdiag[o + c];
#pragma unroll
            for (int k = c + 1; k < 16; ++k) x[k] = fmaf(-s[o + k][o + c], x[c], x[k]);
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) li[o + k][o + lane] = x[k];
    } else if (warp >= 4) {   // zero the six blocks above the diagonal blocks
        for (int e = t - 128; e < 6 * 256; e += 128) {
            const int blk = e >> 8, q = e & 255;
            const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);           // (0,1..3), (1,2..3), (2,3)
            const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
            li[16 * bi + (q >> 4)][16 * bj + (q & 15)] = 0.f;
        }
    }
    __syncthreads();
#pragma unroll 1
    for (int dist = 1; dist < 4; ++dist) {
        const int a = dist + warp, k = warp;   // warp w < 4 - dist: block (dist + w, w)
        const bool act = warp < 4 - dist;
        if (act) {
            float c[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int l = k; l < a; ++l) blk_acc(c, s, 16 * a, 16 * l, li, 16 * l, 16 * k);
            blk_store(tmp, 16 * a, 16 * k, c, 1.f);
        }
        __syncthreads();
        if (act) {
            float c[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            blk_acc(c, li, 16 * a, 16 * a, tmp, 16 * a, 16 * k);
            blk_store(li, 16 * a, 16 * k, c, -1.f);
        }
        __syncthreads();
    }
    for (int e = t; e < TB * TB; e += blockDim.x) {
        const int c = e >> 6, b = e & 63;
        lit[b][c] = li[c][b];
    }
    __syncthreads();
    if (bad) raise_error(err, NQ_ERR_NOT_SPD);
}

// lower-triangular enumeration idx -> (ii >= kk)
__device__ __forceinline__ void tri_index(int64_t idx, int &ii, int &kk) {
    int a = (int)((sqrt(8.0 * (double)idx + 1.0) - 1.0) * 0.5);
    while ((int64_t)(a + 1) * (a + 2) / 2 <= idx) ++a;
    while ((int64_t)a * (a + 1) / 2 > idx) --a;
    ii = a;
    kk = (int)(idx - (int64_t)a * (a + 1) / 2);
}

// Bounded poll of one counter by the calling thread (null: nothing to wait for).
__device__ __forceinline__ void poll_count(const unsigned int *c, unsigned int v, int *err) {
    if (!c || *(volatile int *)err == NQ_ERR_TIMEOUT) return;
    if (!wait_geq(c, v, kGridSpinLimit)) raise_error(err, NQ_ERR_TIMEOUT);
}

// Several counters at once: warp w < 3 polls counter w (null: none), then a CTA barrier.
__device__ __forceinline__ void wait_counts(const unsigned int *c0, unsigned int v0,
                                            const unsigned int *c1, unsigned int v1,
                                            const unsigned int *c2, unsigned int v2, int *err) {
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0 && w < 3)
        poll_count((w == 0) ? c0 : ((w == 1) ? c1 : c2), (w == 0) ? v0 : ((w == 1) ? v1 : v2),
                   err);
    __syncthreads();
}

// ---- tile counters of the factorisation ------------------------------------------
// cnt(i, k) counts the operations finished on tile (i, k): the k updates of steps
// 0 .. k-1, then its Cholesky (i == k) or panel solve (i > k).  A task waits until the
// counters of its operands reach the required values; waits are bounded and, once one
// has timed out, skipped.
__device__ __forceinline__ void signal_count(unsigned int *c, unsigned int inc) {
    __syncthreads();
    if (threadIdx.x == 0) release_add(c, inc);
}

__global__ void __launch_bounds__(256, 1) chol2_kernel(Chol2Args p) {
    // every CTA reads the same word before any wait: all return, or none
    if (p.gate) {
        const int g = *reinterpret_cast<const volatile int *>(p.gate);
        if ((unsigned)g < 32u && ((p.gate_skip >> g) & 1)) return;
    }
    extern __shared__ __align__(16) float smem_f[];
    Tile &t0 = *reinterpret_cast<Tile *>(smem_f);
    Tile &t1 = *reinterpret_cast<Tile *>(smem_f + TB * LDS);
    Tile &t2 = *reinterpret_cast<Tile *>(smem_f + 2 * TB * LDS);
    const int nb = p.nb;
    const int64_t rp = p.rp;

    // phase 0: A = G padded with the identity
    for (int i = blockIdx.x; i < rp; i += gridDim.x) {
        float *dst = p.A + (int64_t)i * rp;
        const float *src = p.G + (int64_t)i * p.r;
#pragma unroll 4
        for (int j = threadIdx.x; j < rp; j += blockDim.x)
            dst[j] = (i < p.r && j < p.r) ? __ldg(src + j) : (i == j ? 1.f : 0.f);
    }
    grid_barrier(p.bar, p.err);
    Tile &t3 = *reinterpret_cast<Tile *>(smem_f + 3 * TB * LDS);
    Tile &t4 = *reinterpret_cast<Tile *>(smem_f + 4 * TB * LDS);
    float *rdiag = smem_f + 5 * TB * LDS;  // 1 / L_cc of the tile just factored
    // Dataflow factorisation.  CTA 0 runs the critical chain: Cholesky of the diagonal
    // tile and its inverse (kept in shared memory), the panel tile below it as one tile
    // product, the look-ahead update of the next diagonal tile.  CTA 1 takes the tasks CTA 0
    // needs next; CTAs 2.. take the other panel tiles (A_ij L_jj^-T, with L_jj^-T from the
    // upper tile (j, j+1) of Li), the trailing updates and the L^-1 tasks round-robin in a
    // topological order (step by step), so every wait ends.
    auto CNT = [&](int i, int k) { return p.cnt + (int64_t)i * nb + k; };
    auto ICNT = [&](int i, int k) { return p.cnt + (int64_t)(nb + i) * nb + k; };  // L^-1 tiles
    if (blockIdx.x == 0) {
        // t2: L_jj, t3: L_jj^-1, t4: (L_jj^-1)^T, t0: panel operand, t1: panel^T
        load_n(t2, p.A, rp, 0, 0);
        __syncthreads();
        chain_tile<false>(t2, t1, rdiag, t3, t4, t0, p.err);
        store_n(p.A, rp, 0, 0, t2);
        store_n(p.Li, rp, 0, 0, t3);
        if (nb > 1) store_n(p.Li, rp, 0, 1, t4);      // L_00^-T in an unused upper tile
        signal_count(CNT(0, 0), 1);
        for (int j = 0; j + 1 < nb; ++j) {
            wait_counts(CNT(j + 1, j), j, CNT(j + 1, j + 1), j, nullptr, 0, p.err);
            load_n_async(t0, p.A, rp, j + 1, j);       // panel tile, all j updates applied
            load_n_async(t2, p.A, rp, j + 1, j + 1);   // next diagonal tile
            cp_async_wait<1>();
            __syncthreads();
            float acc[4][4];
            zero(acc);
            mac_n(acc, t0, t4);                        // L_{j+1,j} = A_{j+1,j} L_jj^-T
            put(p.A, rp, j + 1, j, acc, 1.f);
            put_t(p.A, rp, j, j + 1, acc);             // L_{j+1,j}^T in the upper tile
            {
                const int a0 = blk_a0(), b0 = blk_b0();
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    *reinterpret_cast<float4 *>(&t1[a0 + i][b0]) =
                        make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
            }
            signal_count(CNT(j + 1, j), 1);
            cp_async_wait<0>();
            __syncthreads();
            // factorisation of the next diagonal tile with its look-ahead update
            // t2 -= L_{j+1,j} L_{j+1,j}^T and its inverse, in one pass
            chain_tile<true>(t2, t1, rdiag, t3, t4, t0, p.err);
            store_n(p.A, rp, j + 1, j + 1, t2);
            store_n(p.Li, rp, j + 1, j + 1, t3);
            if (j + 2 < nb) store_n(p.Li, rp, j + 1, j + 2, t4);  // L^-T, unused upper tile
            signal_count(CNT(j + 1, j + 1), 2);
        }
    } else if (blockIdx.x == 1) {
        // CTA 1 takes the tasks CTA 0 needs next: panel (j+2, j) and the step-j updates of
        // (j+2, j+1) and (j+2, j+2), keeping the panel in shared memory.
        for (int j = 0; j + 2 < nb; ++j) {
            float acc[4][4];
            zero(acc);
            wait_counts(CNT(j, j), j + 1, CNT(j + 2, j), j, nullptr, 0, p.err);
            load_n_async(t0, p.A, rp, j + 2, j);
            load_n_async(t4, p.Li, rp, j, j + 1);    // L_jj^-T
            cp_async_wait<0>();
            __syncthreads();
            mac_n(acc, t0, t4);                        // L_{j+2,j} = A_{j+2,j} L_jj^-T
            put(p.A, rp, j + 2, j, acc, 1.f);
            put_t(p.A, rp, j, j + 2, acc);
            {
                const int a0 = blk_a0(), b0 = blk_b0();
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        t1[a0 + i][b0 + q] = acc[i][q];   // L_{j+2,j}
                        t3[b0 + q][a0 + i] = acc[i][q];   // L_{j+2,j}^T
                    }
            }
            signal_count(CNT(j + 2, j), 1);
            wait_counts(CNT(j + 1, j), j + 1, CNT(j + 2, j + 1), j, CNT(j + 2, j + 2), j, p.err);
            load_n_async(t0, p.A, rp, j, j + 1);      // L_{j+1,j}^T
            cp_async_wait<0>();
            __syncthreads();
            for (int h = 0; h < 2; ++h) {              // h = 0: tile (j+2, j+1); 1: (j+2, j+2)
                zero(acc);
                mac_n(acc, t1, h ? t3 : t0);
                const int a0 = blk_a0(), b0 = blk_b0();
                float *bp = p.A + ((int64_t)(j + 2) * TB + a0) * rp + (int64_t)(j + 1 + h) * TB + b0;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float4 v = __ldcg(reinterpret_cast<const float4 *>(bp + (int64_t)q * rp));
                    v.x -= acc[q][0];
                    v.y -= acc[q][1];
                    v.z -= acc[q][2];
                    v.w -= acc[q][3];
                    __stcg(reinterpret_cast<float4 *>(bp + (int64_t)q * rp), v);
                }
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                release_add(CNT(j + 2, j + 1), 1u);
                release_add(CNT(j + 2, j + 2), 1u);
            }
            __syncthreads();
        }
    } else {
        // Worker tasks of step j, in this order: panel tiles (i, j), i >= j+3; trailing
        // updates of step j; L^-1 tasks: finalise X_jm = -L_jj^-1 acc_jm (m < j), then
        // acc_im += L_ij X_jm for m <= j < i (block column m of L^-1 is a forward
        // substitution, advanced one block row per step of the factorisation).  The L^-1
        // tasks of step j are placed after the factorisation tasks of step j + 1 (still a
        // topological order), so the tasks CTA 0 waits for come first.  One tile per task:
        // grouping tiles that share an operand serialises them on one CTA and was slower.
        const int64_t W = gridDim.x - 2, w = blockIdx.x - 2;
        int64_t base = 0;
        for (int sj = 0; sj <= nb; ++sj) {
            const int jf = sj < nb ? sj : -1;       // factorisation tasks of step jf
            const int ji = sj - 1;                  // L^-1 tasks of step ji
            const int Tf = jf >= 0 ? nb - 1 - jf : 0;
            // panels i >= jf + 3; updates except (jf+1, jf+1) [CTA 0], (jf+2, jf+1) and
            // (jf+2, jf+2) [CTA 1]
            const int P = Tf > 1 ? Tf - 2 : 0;
            const int64_t U = Tf > 1 ? (int64_t)Tf * (Tf + 1) / 2 - 3 : 0;
            const int Ti = ji >= 0 ? nb - 1 - ji : 0;
            const int F = ji >= 0 ? ji : 0;                              // finalise (ji, m)
            const int64_t V = ji >= 0 ? (int64_t)(ji + 1) * Ti : 0;      // L^-1 updates
            const int64_t n = P + U + F + V;
            for (int64_t idx = base + ((w - base % W) % W + W) % W; idx < base + n; idx += W) {
                const int64_t loc = idx - base;
                const int a0 = blk_a0(), b0 = blk_b0();
                float acc[4][4];
                zero(acc);
                const int j = (loc < P + U) ? jf : ji;
                if (loc < P) {  // panel tile (i, j) = A_ij L_jj^-T
                    const int i = j + 3 + (int)loc;
                    wait_counts(CNT(j, j), j + 1, CNT(i, j), j, nullptr, 0, p.err);
                    load_n_async(t0, p.A, rp, i, j);
                    load_n_async(t4, p.Li, rp, j, j + 1);  // L_jj^-T
                    cp_async_wait<0>();
                    __syncthreads();
                    mac_n(acc, t0, t4);
                    put(p.A, rp, i, j, acc, 1.f);
                    put_t(p.A, rp, j, i, acc);
                    signal_count(CNT(i, j), 1);
                } else if (loc < P + U) {  // update of tile (i, k): A_ik -= L_ij L_kj^T
                    int ii, kk;
                    tri_index(loc - P + 3, ii, kk);
                    const int i = j + 1 + ii, k = j + 1 + kk;
                    wait_counts(CNT(i, j), j + 1, CNT(k, j), j + 1, CNT(i, k), j, p.err);
                    load_n_async(t0, p.A, rp, i, j);   // L_ij
                    load_n_async(t1, p.A, rp, j, k);   // L_kj^T (upper-tile copy)
                    cp_async_wait<0>();
                    __syncthreads();
                    mac_n(acc, t0, t1);
                    float *bp = p.A + ((int64_t)i * TB + a0) * rp + (int64_t)k * TB + b0;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float4 v = __ldcg(reinterpret_cast<const float4 *>(bp + (int64_t)q * rp));
                        v.x -= acc[q][0];
                        v.y -= acc[q][1];
                        v.z -= acc[q][2];
                        v.w -= acc[q][3];
                        __stcg(reinterpret_cast<float4 *>(bp + (int64_t)q * rp), v);
                    }
                    signal_count(CNT(i, k), 1);
                } else if (loc < P + U + F) {  // finalise X_jm = -L_jj^-1 acc_jm
                    const int m = (int)(loc - P - U);
                    wait_counts(ICNT(j, m), j - m, CNT(j, j), j + 1, nullptr, 0, p.err);
                    load_n_async(t0, p.Li, rp, j, j);
                    load_n_async(t1, p.Li, rp, j, m);
                    cp_async_wait<0>();
                    __syncthreads();
                    mac_n(acc, t0, t1);
                    put(p.Li, rp, j, m, acc, -1.f);
                    signal_count(ICNT(j, m), 1);
                } else {  // acc_im += L_ij X_jm
                    const int64_t v = loc - P - U - F;
                    const int m = (int)(v / Ti), i = j + 1 + (int)(v % Ti);
                    if (m < j)
                        wait_counts(CNT(i, j), j + 1, ICNT(j, m), j - m + 1, ICNT(i, m), j - m,
                                    p.err);
                    else
                        wait_counts(CNT(i, j), j + 1, CNT(j, j), j + 1, nullptr, 0, p.err);
                    load_n_async(t0, p.A, rp, i, j);   // L_ij
                    load_n_async(t1, p.Li, rp, j, m);  // X_jm (L_jj^-1 when m == j)
                    cp_async_wait<0>();
                    __syncthreads();
                    mac_n(acc, t0, t1);
                    if (m == j) {
                        put(p.Li, rp, i, m, acc, 1.f);
                    } else {
                        float *bp = p.Li + ((int64_t)i * TB + a0) * rp + (int64_t)m * TB + b0;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            float4 x = __ldcg(reinterpret_cast<const float4 *>(bp + (int64_t)q * rp));
                            x.x += acc[q][0];
                            x.y += acc[q][1];
                            x.z += acc[q][2];
                            x.w += acc[q][3];
                            __stcg(reinterpret_cast<float4 *>(bp + (int64_t)q * rp), x);
                        }
                    }
                    signal_count(ICNT(i, m), 1);
                }
                __syncthreads();  // shared tiles free for the next task
            }
            base += n;
        }
    }
    grid_barrier(p.bar, p.err);

    // (L^-1)^T as bf16 hi + lo: LiT[x][y] = Li[y][x] (zero for y < x), all r x r entries,
    // the operand of the tensor-core product G^-1 = Li^T Li.  Thread: 8 consecutive y.
    const int64_t nt2 = (int64_t)nb * nb;
    const bool vec_ok = (p.ldr % 8) == 0;
    for (int64_t idx = blockIdx.x; idx < nt2; idx += gridDim.x) {
        const int ta = (int)(idx / nb), tc = (int)(idx % nb);  // LiT tile (ta, tc)
        __syncthreads();
        if (tc >= ta) load_n(t0, p.Li, rp, tc, ta);              // t0[y][x] = Li_tile(tc,ta)
        __syncthreads();
        for (int e = threadIdx.x; e < TB * TB / 8; e += blockDim.x) {
            const int x = e & 63, y8 = (e >> 6) * 8;
            const int64_t gi = (int64_t)ta * TB + x, gj = (int64_t)tc * TB + y8;
            if (gi >= p.r || gj >= p.r) continue;
            uint32_t h[4], l[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float v0 = (tc >= ta) ? t0[y8 + 2 * k][x] : 0.f;
                const float v1 = (tc >= ta) ? t0[y8 + 2 * k + 1][x] : 0.f;
                const __nv_bfloat162 hh = __floats2bfloat162_rn(v0, v1);
                const __nv_bfloat162 ll = __floats2bfloat162_rn(v0 - __low2float(hh),
                                                                v1 - __high2float(hh));
                h[k] = *reinterpret_cast<const uint32_t *>(&hh);
                l[k] = *reinterpret_cast<const uint32_t *>(&ll);
            }
            __nv_bfloat16 *ph = p.hi + gi * p.ldr + gj, *pl = p.lo + gi * p.ldr + gj;
            if (vec_ok && gj + 8 <= p.r) {
                *reinterpret_cast<uint4 *>(ph) = make_uint4(h[0], h[1], h[2], h[3]);
                *reinterpret_cast<uint4 *>(pl) = make_uint4(l[0], l[1], l[2], l[3]);
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (gj + k >= p.r) break;
                    const uint32_t hw = h[k >> 1], lw = l[k >> 1];
                    const unsigned short hs = (k & 1) ? (unsigned short)(hw >> 16) : (unsigned short)hw;
                    const unsigned short ls = (k & 1) ? (unsigned short)(lw >> 16) : (unsigned short)lw;
                    ph[k] = __ushort_as_bfloat16(hs);
                    pl[k] = __ushort_as_bfloat16(ls);
                }
            }
        }
    }
}

}  // namespace

cudaError_t chol_inverse(const float *G, int32_t r, int64_t rp, float *A, float *Li,
                         __nv_bfloat16 *Gi_hi, __nv_bfloat16 *Gi_lo, int64_t ldr,
                         unsigned int *flags, int *err, unsigned int *bar, int max_ctas,
                         const int *gate, int gate_skip, bool zero_state, cudaStream_t s) {
    if (rp % TB != 0 || rp < r) return cudaErrorInvalidValue;
    constexpr int smem = (5 * TB * LDS + TB) * sizeof(float);
    // grid of the cooperative launch (one CTA per SM), per device
    static std::atomic<int> grids[kMaxDevices];
    const int dev = current_device();
    if (dev < 0) return cudaErrorInvalidDevice;
    int grid = grids[dev].load();
    if (!grid) {
        cudaError_t e = cudaFuncSetAttribute(chol2_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, chol2_kernel, 256, smem);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) return cudaErrorLaunchOutOfResources;
        grid = device_sm_count();
        if (grid < 3) return cudaErrorLaunchOutOfResources;
        grids[dev].store(grid);
    }
    if (max_ctas > 0 && max_ctas < grid) grid = max_ctas < 3 ? 3 : max_ctas;
    const int nb = (int)(rp / TB);
    if (zero_state) {
        cudaError_t e = cudaMemsetAsync(bar, 0, 2 * sizeof(unsigned int), s);
        if (e != cudaSuccess) return e;
        e = cudaMemsetAsync(flags, 0, (size_t)2 * nb * nb * sizeof(unsigned int), s);
        if (e != cudaSuccess) return e;
    }
    Chol2Args args{G, r, nb, rp, A, Li, Gi_hi, Gi_lo, ldr, flags, err, bar, gate, gate_skip};
    void *params[] = {&args};
    count_launch();
    return cudaLaunchCooperativeKernel((const void *)chol2_kernel, dim3(grid), dim3(256), params,
                                       smem, s);
}

}  // namespace nq
