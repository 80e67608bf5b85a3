// G^-1 for the r x r SPD system matrix of the U (V) step: Cholesky G = L L^T, L^-1 by
// recursive doubling, G^-1 = L^-T L^-1, written as BF16 hi + lo for the split-BF16
// tensor-core solve.  NanoQuant summary page, "Core method" (核心方法), step (a): the
// regularised linear system is solved through a Cholesky factorisation.
//
// One cooperative launch of FP32 SIMT work on 64 x 64 tiles (4 x 4 register blocks per
// thread, float4 traffic) with bounded grid barriers:
//   * right-looking blocked Cholesky with look-ahead: while CTAs 1.. apply the trailing
//     update of step j, CTA 0 updates the next diagonal tile and factors it, so a step
//     costs two barriers and the diagonal factorisation overlaps the update;
//   * the diagonal 64 x 64 factorisation and its inverse keep each thread's 16 entries
//     in registers and broadcast the current column / row with one barrier per step;
//   * (L^-1)_21 = -L22^-1 L21 L11^-1 level by level (log2(r/64) levels, two barriers each);
//   * G^-1 tiles (a >= b) = sum_{c >= a} Li(c,a)^T Li(c,b), mirrored.
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
    int *err;
    unsigned int *bar;
};

// ---- tile movement (L2-coherent loads: tiles change between grid barriers) ----------
__device__ __forceinline__ void load_n(Tile &d, const float *M, int64_t ld, int ti, int tj) {
    const float *base = M + (int64_t)ti * TB * ld + (int64_t)tj * TB;
    for (int f = threadIdx.x; f < TB * TB / 4; f += blockDim.x) {
        const int row = f >> 4, c4 = (f & 15) * 4;
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(base + (int64_t)row * ld + c4));
        *reinterpret_cast<float4 *>(&d[row][c4]) = v;
    }
}
// d[c][r] = M_tile[r][c]
__device__ __forceinline__ void load_t(Tile &d, const float *M, int64_t ld, int ti, int tj) {
    const float *base = M + (int64_t)ti * TB * ld + (int64_t)tj * TB;
    for (int f = threadIdx.x; f < TB * TB / 4; f += blockDim.x) {
        const int row = f >> 4, c4 = (f & 15) * 4;
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(base + (int64_t)row * ld + c4));
        d[c4][row] = v.x;
        d[c4 + 1][row] = v.y;
        d[c4 + 2][row] = v.z;
        d[c4 + 3][row] = v.w;
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

// Thread's 4 x 4 block of a 64 x 64 tile: rows a0..a0+3, columns b0..b0+3.
__device__ __forceinline__ int blk_a0() { return (threadIdx.x >> 4) * 4; }
__device__ __forceinline__ int blk_b0() { return (threadIdx.x & 15) * 4; }

// acc[i][j] += sum_{c in [c0, c1)} XT[c][a0+i] * Y[c][b0+j]
__device__ __forceinline__ void mac(float (&acc)[4][4], const Tile &XT, const Tile &Y,
                                   int c0 = 0, int c1 = TB) {
    const int a0 = blk_a0(), b0 = blk_b0();
#pragma unroll 4
    for (int c = c0; c < c1; ++c) {
        const float4 x = *reinterpret_cast<const float4 *>(&XT[c][a0]);
        const float4 y = *reinterpret_cast<const float4 *>(&Y[c][b0]);
        const float xs[4] = {x.x, x.y, x.z, x.w};
        const float ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xs[i], ys[j], acc[i][j]);
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

// ---- 64 x 64 diagonal tile: Cholesky and triangular inverse -------------------------
// Thread t owns row i = t / 4 and the columns 4p + g (g = t % 4, p = 0..15) in
// registers.  Column k (Cholesky) and row k of L^-1 (inverse) are broadcast through a
// double-buffered shared array; the owners of the next column / row publish it in the
// same step, so each of the 2 x 64 steps costs a single CTA barrier.  The loops are
// compact: this code runs once per block step.  The register window is shifted by one
// column quad per four steps so that the current column always sits in a[0].
// On entry s holds A_jj; on exit s holds L_jj (zero above the diagonal), inv holds L_jj^-1.
// cb: 2 x 64 floats of shared scratch.
__device__ void factor_diag(Tile &s, Tile &inv, float *cb, int *err) {
    const int t = threadIdx.x, i = t >> 2, g = t & 3;
    float a[16];
#pragma unroll
    for (int p = 0; p < 16; ++p) a[p] = s[i][4 * p + g];
    bool bad = false;
    if (g == 0) cb[i] = a[0];  // column 0 (its owners have g == 0)
    __syncthreads();
#pragma unroll 1
    for (int q = 0; q < 16; ++q) {
#pragma unroll
        for (int g2 = 0; g2 < 4; ++g2) {
            const int k = 4 * q + g2;
            const float *col = cb + 64 * (k & 1);
            float *nxt = cb + 64 * ((k + 1) & 1);
            float piv = col[k];
            if (!(piv > 0.f)) {
                bad = true;
                piv = 1e-30f;
            }
            const float l = sqrtf(piv);
            const float il = 1.f / l;
            const float lik = (i == k) ? l : col[i] * il;
#pragma unroll
            for (int p = 0; p < 16; ++p) {
                const int j = 4 * (q + p) + g;
                if (j > k && j <= i && j < 64) a[p] = fmaf(-lik, col[j] * il, a[p]);
            }
            if (g == g2) s[i][k] = (i >= k) ? lik : 0.f;
            // publish column k + 1: its owners hold it in a[0] (g2 < 3) or a[1] (g2 == 3)
            if (k + 1 < 64 && g == ((g2 + 1) & 3) && i >= k + 1) nxt[i] = (g2 == 3) ? a[1] : a[0];
            __syncthreads();
        }
#pragma unroll
        for (int p = 0; p < 15; ++p) a[p] = a[p + 1];
    }
    if (bad && t == 0) raise_error(err, NQ_ERR_NOT_SPD);
    // X = L^-1, thread owns x[p] = X[i][4p + g]; row k final = (row k after updates) / L_kk
    float x[16];
#pragma unroll
    for (int p = 0; p < 16; ++p) x[p] = (4 * p + g == i) ? 1.f : 0.f;
    if (i == 0) {
        const float il0 = 1.f / s[0][0];
#pragma unroll
        for (int p = 0; p < 16; ++p) {
            x[p] *= il0;
            cb[4 * p + g] = x[p];
        }
    }
    __syncthreads();
#pragma unroll 1
    for (int k = 0; k < 64; ++k) {
        const float *rowk = cb + 64 * (k & 1);
        float *nxt = cb + 64 * ((k + 1) & 1);
        if (i > k) {
            const float lik = s[i][k];
#pragma unroll
            for (int p = 0; p < 16; ++p)
                if (4 * p + g <= k) x[p] = fmaf(-lik, rowk[4 * p + g], x[p]);
            if (i == k + 1) {  // row k + 1 is now final: scale and publish
                const float il = 1.f / s[i][i];
#pragma unroll
                for (int p = 0; p < 16; ++p) {
                    x[p] *= il;
                    nxt[4 * p + g] = x[p];
                }
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int p = 0; p < 16; ++p) inv[i][4 * p + g] = x[p];
    __syncthreads();
}

// lower-triangular enumeration idx -> (ii >= kk)
__device__ __forceinline__ void tri_index(int64_t idx, int &ii, int &kk) {
    int a = (int)((sqrt(8.0 * (double)idx + 1.0) - 1.0) * 0.5);
    while ((int64_t)(a + 1) * (a + 2) / 2 <= idx) ++a;
    while ((int64_t)a * (a + 1) / 2 > idx) --a;
    ii = a;
    kk = (int)(idx - (int64_t)a * (a + 1) / 2);
}

__global__ void __launch_bounds__(256, 1) chol2_kernel(Chol2Args p) {
    extern __shared__ __align__(16) float smem_f[];
    Tile &t0 = *reinterpret_cast<Tile *>(smem_f);
    Tile &t1 = *reinterpret_cast<Tile *>(smem_f + TB * LDS);
    Tile &t2 = *reinterpret_cast<Tile *>(smem_f + 2 * TB * LDS);
    const int nb = p.nb;
    const int64_t rp = p.rp;

    // phase 0: A = G padded with the identity
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < rp * rp;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / rp, j = e % rp;
        p.A[e] = (i < p.r && j < p.r) ? p.G[i * p.r + j] : (i == j ? 1.f : 0.f);
    }
    grid_barrier(p.bar, p.err);
    if (blockIdx.x == 0) {
        load_n(t0, p.A, rp, 0, 0);
        __syncthreads();
        factor_diag(t0, t1, &t2[0][0], p.err);
        store_n(p.A, rp, 0, 0, t0);
        store_n(p.Li, rp, 0, 0, t1);
    }
    grid_barrier(p.bar, p.err);

    for (int j = 0; j < nb; ++j) {
        // panel: L_ij = A_ij L_jj^-T
        for (int i = j + 1 + blockIdx.x; i < nb; i += gridDim.x) {
            __syncthreads();
            load_t(t0, p.A, rp, i, j);
            load_t(t1, p.Li, rp, j, j);
            __syncthreads();
            float acc[4][4];
            zero(acc);
            mac(acc, t0, t1);
            put(p.A, rp, i, j, acc, 1.f);
        }
        grid_barrier(p.bar, p.err);
        if (j == nb - 1) break;
        const int T = nb - 1 - j;
        if (blockIdx.x == 0) {
            // look-ahead: next diagonal tile, updated then factored
            __syncthreads();
            load_t(t0, p.A, rp, j + 1, j);
            load_n(t2, p.A, rp, j + 1, j + 1);
            __syncthreads();
            float acc[4][4];
            zero(acc);
            mac(acc, t0, t0);  // L_{j+1,j} L_{j+1,j}^T with t0 holding L^T: XT = Y = t0
            __syncthreads();
            {
                const int a0 = blk_a0(), b0 = blk_b0();
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int q = 0; q < 4; ++q) t2[a0 + i][b0 + q] -= acc[i][q];
            }
            __syncthreads();
            factor_diag(t2, t1, &t0[0][0], p.err);
            store_n(p.A, rp, j + 1, j + 1, t2);
            store_n(p.Li, rp, j + 1, j + 1, t1);
        } else {
            const int64_t ntl = (int64_t)T * (T + 1) / 2;
            for (int64_t idx = 1 + (blockIdx.x - 1); idx < ntl; idx += gridDim.x - 1) {
                int ii, kk;
                tri_index(idx, ii, kk);
                const int i = j + 1 + ii, k = j + 1 + kk;
                __syncthreads();
                load_t(t0, p.A, rp, i, j);
                load_t(t1, p.A, rp, k, j);
                __syncthreads();
                float acc[4][4];
                zero(acc);
                mac(acc, t0, t1);
                // A_ik -= acc (read-modify-write of the thread's own block)
                const int a0 = blk_a0(), b0 = blk_b0();
                float *base = p.A + ((int64_t)i * TB + a0) * rp + (int64_t)k * TB + b0;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float4 v = __ldcg(reinterpret_cast<const float4 *>(base + (int64_t)q * rp));
                    v.x -= acc[q][0];
                    v.y -= acc[q][1];
                    v.z -= acc[q][2];
                    v.w -= acc[q][3];
                    __stcg(reinterpret_cast<float4 *>(base + (int64_t)q * rp), v);
                }
            }
        }
        grid_barrier(p.bar, p.err);
    }

    // L^-1 by recursive doubling; T(a, b) = L21 Li11 kept in the unused upper tile (b, a)
    for (int s = 1; s < nb; s *= 2) {
        const int npairs = (int)ceil_div(nb, 2 * s);
        const int64_t jobs = (int64_t)npairs * s * s;
        for (int64_t q = blockIdx.x; q < jobs; q += gridDim.x) {
            const int pr = (int)(q / ((int64_t)s * s));
            const int a = 2 * pr * s + s + (int)((q % ((int64_t)s * s)) / s);
            const int b = 2 * pr * s + (int)(q % s);
            if (a >= nb) continue;
            const int top_end = 2 * pr * s + s;
            float acc[4][4];
            zero(acc);
            for (int c = b; c < top_end; ++c) {
                __syncthreads();
                load_t(t0, p.A, rp, a, c);   // L21(a, c)
                load_n(t1, p.Li, rp, c, b);  // Li11(c, b)
                __syncthreads();
                mac(acc, t0, t1);
            }
            put(p.Li, rp, b, a, acc, 1.f);
        }
        grid_barrier(p.bar, p.err);
        for (int64_t q = blockIdx.x; q < jobs; q += gridDim.x) {
            const int pr = (int)(q / ((int64_t)s * s));
            const int bot0 = 2 * pr * s + s;
            const int a = bot0 + (int)((q % ((int64_t)s * s)) / s);
            const int b = 2 * pr * s + (int)(q % s);
            if (a >= nb) continue;
            float acc[4][4];
            zero(acc);
            for (int c = bot0; c <= a; ++c) {
                __syncthreads();
                load_t(t0, p.Li, rp, a, c);  // Li22(a, c)
                load_n(t1, p.Li, rp, b, c);  // T(c, b) lives at tile (b, c)
                __syncthreads();
                mac(acc, t0, t1);
            }
            put(p.Li, rp, a, b, acc, -1.f);
        }
        grid_barrier(p.bar, p.err);
    }

    // G^-1 = Li^T Li, tiles a >= b, largest sums first; split into bf16 hi + lo
    const int64_t ngi = (int64_t)nb * (nb + 1) / 2;
    for (int64_t idx = blockIdx.x; idx < ngi; idx += gridDim.x) {
        int a, b;
        tri_index(idx, a, b);
        // idx enumerates a ascending: small a = long sums come first
        float acc[4][4];
        zero(acc);
        for (int c = a; c < nb; ++c) {
            __syncthreads();
            load_n(t0, p.Li, rp, c, a);
            load_n(t1, p.Li, rp, c, b);
            __syncthreads();
            mac(acc, t0, t1);
        }
        const int a0 = blk_a0(), b0 = blk_b0();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t gi = (int64_t)a * TB + a0 + i;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int64_t gj = (int64_t)b * TB + b0 + q;
                if (gi < p.r && gj < p.r) {
                    const float v = acc[i][q];
                    const __nv_bfloat16 h = __float2bfloat16_rn(v);
                    const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
                    p.hi[gi * p.ldr + gj] = h;
                    p.lo[gi * p.ldr + gj] = l;
                    p.hi[gj * p.ldr + gi] = h;
                    p.lo[gj * p.ldr + gi] = l;
                }
            }
        }
    }
}

}  // namespace

int64_t chol_padded(int32_t r) { return (int64_t)(r + TB - 1) / TB * TB; }

cudaError_t chol_inverse(const float *G, int32_t r, int64_t rp, float *A, float *Li,
                         __nv_bfloat16 *Gi_hi, __nv_bfloat16 *Gi_lo, int64_t ldr, int *err,
                         unsigned int *bar, cudaStream_t s) {
    if (rp % TB != 0 || rp < r) return cudaErrorInvalidValue;
    constexpr int smem = 3 * TB * LDS * sizeof(float);
    static int grid = 0;
    if (!grid) {
        cudaError_t e = cudaFuncSetAttribute(chol2_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, chol2_kernel, 256, smem);
        if (e != cudaSuccess) return e;
        int dev = 0, sms = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        grid = sms * (per_sm < 1 ? per_sm : 1);
        if (grid < 2) return cudaErrorLaunchOutOfResources;
    }
    cudaError_t e = cudaMemsetAsync(bar, 0, 2 * sizeof(unsigned int), s);
    if (e != cudaSuccess) return e;
    Chol2Args args{G, r, (int)(rp / TB), rp, A, Li, Gi_hi, Gi_lo, ldr, err, bar};
    void *params[] = {&args};
    count_launch();
    return cudaLaunchCooperativeKernel((const void *)chol2_kernel, dim3(grid), dim3(256), params,
                                       smem, s);
}

}  // namespace nq
