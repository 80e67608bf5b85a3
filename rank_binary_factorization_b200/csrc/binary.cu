// Inference with the packed binary factors (sm_100a):
//     Y = X diag(s2) V+- U+-^T diag(s1)      X: B x n,  Y: B x m
// NanoQuant summary page, "Technical novelty" (技术新颖性) and "Limitations" (局限与改进):
// the compressed layer is applied by binary GEMV/GEMM kernels that read the packed signs.
//
// Small batches (GEMV path): two passes over the packed words, one warp per 32-bit word
// and one lane per bit, so every sign is decoded by the lane that uses it:
//   z[b][k] = sum_j (+-1)_{jk} s2_j X[b][j]   per row chunk, then summed over chunks;
//   Y[b][i] = s1_i sum_k (+-1)_{ik} z[b][k]    one warp per output row.
// Large batches: the signs are expanded into BF16 +-1 tensor-core operands (exact) and
// both products run on the tcgen05 GEMM (see binary_* in api.cu).
#include "kernels.cuh"

namespace nq {

// ---- GEMV path ----------------------------------------------------------------------
// z pass: CTA = one chunk of rows of V; its packed words (contiguous in memory) and the
// scaled inputs s2_j X[b][j] are staged in shared memory with coalesced copies, then warp
// w takes words w, w + 8, ... (lane = bit) and walks the chunk's rows.
__global__ void __launch_bounds__(256)
    bin_z_kernel(const uint32_t *__restrict__ Vp, const float *__restrict__ s2,
                 const void *__restrict__ X, int x_bf16, int64_t n, int r, int64_t B,
                 int64_t rows_per_chunk, float *__restrict__ P) {
    extern __shared__ __align__(16) float smz[];
    const int nw = (r + 31) >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t j0 = (int64_t)blockIdx.x * rows_per_chunk;
    const int64_t j1 = min(n, j0 + rows_per_chunk);
    const int64_t nj = j1 - j0;
    float *xs = smz;                                                   // [B][rows_per_chunk]
    uint32_t *vw = reinterpret_cast<uint32_t *>(smz + B * rows_per_chunk);  // [nj][nw]
    for (int64_t e = threadIdx.x; e < B * nj; e += blockDim.x) {
        const int64_t b = e / nj, jj = e % nj, j = j0 + jj;
        const float x = x_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(X)[b * n + j])
                               : reinterpret_cast<const float *>(X)[b * n + j];
        xs[b * rows_per_chunk + jj] = s2[j] * x;
    }
    const uint32_t *src = Vp + j0 * nw;
    for (int64_t e = threadIdx.x; e < nj * nw; e += blockDim.x) vw[e] = __ldg(src + e);
    __syncthreads();
    for (int wd = warp; wd < nw; wd += 8) {
        float z[NQ_BINARY_GEMV_MAX_BATCH];
#pragma unroll
        for (int b = 0; b < NQ_BINARY_GEMV_MAX_BATCH; ++b) z[b] = 0.f;
        for (int64_t jj = 0; jj < nj; ++jj) {
            const bool neg = (vw[jj * nw + wd] >> lane) & 1u;
#pragma unroll
            for (int b = 0; b < NQ_BINARY_GEMV_MAX_BATCH; ++b) {
                if (b >= B) break;
                const float w = xs[b * rows_per_chunk + jj];
                z[b] += neg ? -w : w;
            }
        }
        const int k = 32 * wd + lane;
        if (k < r)
            for (int b = 0; b < B; ++b) P[((int64_t)blockIdx.x * B + b) * r + k] = z[b];
    }
}

// z[b][k] = sum over chunks of P[chunk][b][k]: four interleaved partial sums (chunks
// c = 4q + u into sum u), combined in a fixed order, so the loads stay in flight.
__global__ void bin_zreduce_kernel(const float *__restrict__ P, int chunks, int64_t Br,
                                   float *__restrict__ z) {
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < Br;
         e += (int64_t)gridDim.x * blockDim.x) {
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        int c = 0;
#pragma unroll 2
        for (; c + 4 <= chunks; c += 4) {
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] += P[(int64_t)(c + u) * Br + e];
        }
        for (; c < chunks; ++c) v[c & 3] += P[(int64_t)c * Br + e];
        z[e] = (v[0] + v[1]) + (v[2] + v[3]);
    }
}

// y pass: CTA = 32 output rows; their packed words and (when it fits) z are staged in
// shared memory; warp w takes rows w, w + 8, ... with lane = bit of each word.
constexpr int kBinRowsPerCta = 32;
__global__ void __launch_bounds__(256)
    bin_y_kernel(const uint32_t *__restrict__ Up, const float *__restrict__ s1,
                 const float *__restrict__ z, int64_t m, int r, int64_t B, int z_in_smem,
                 float *__restrict__ Y) {
    extern __shared__ __align__(16) float smy[];
    const int nw = (r + 31) >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t i0 = (int64_t)blockIdx.x * kBinRowsPerCta;
    const int64_t ni = min((int64_t)kBinRowsPerCta, m - i0);
    uint32_t *uw = reinterpret_cast<uint32_t *>(smy);              // [ni][nw]
    float *zs = smy + kBinRowsPerCta * nw;                           // [B][r] when staged
    const uint32_t *src = Up + i0 * nw;
    for (int64_t e = threadIdx.x; e < ni * nw; e += blockDim.x) uw[e] = __ldg(src + e);
    if (z_in_smem)
        for (int64_t e = threadIdx.x; e < B * r; e += blockDim.x) zs[e] = __ldg(z + e);
    __syncthreads();
    const float *zz = z_in_smem ? zs : z;
    for (int ii = warp; ii < ni; ii += 8) {
        float acc[NQ_BINARY_GEMV_MAX_BATCH];
#pragma unroll
        for (int b = 0; b < NQ_BINARY_GEMV_MAX_BATCH; ++b) acc[b] = 0.f;
        for (int wd = 0; wd < nw; ++wd) {
            const int k = 32 * wd + lane;
            if (k >= r) break;
            const bool neg = (uw[ii * nw + wd] >> lane) & 1u;
#pragma unroll
            for (int b = 0; b < NQ_BINARY_GEMV_MAX_BATCH; ++b) {
                if (b >= B) break;
                const float v = zz[(int64_t)b * r + k];
                acc[b] += neg ? -v : v;
            }
        }
        const float sc = s1[i0 + ii];
        for (int b = 0; b < B; ++b) {
            const float t = warp_sum(acc[b]);
            if (lane == 0) Y[(int64_t)b * m + i0 + ii] = sc * t;
        }
    }
}

// Row chunks of the z pass: about two CTAs per SM, at least 32 rows per chunk, and the
// chunk's staged inputs and words within 192 KB of shared memory.
int bin_gemv_chunks(int64_t n, int32_t r, int64_t B) {
    const int64_t nw = (r + 31) / 32;
    int64_t c = 2 * kNumSMsB200;
    if (c > (n + 31) / 32) c = (n + 31) / 32;
    const int64_t max_rows = (192 * 1024) / (4 * ((B > 0 ? B : 1) + nw));
    if (c < (n + max_rows - 1) / max_rows) c = (n + max_rows - 1) / max_rows;
    return c < 1 ? 1 : (int)c;
}

cudaError_t bin_gemv(const uint32_t *Up, const uint32_t *Vp, const float *s1, const float *s2,
                     int64_t m, int64_t n, int32_t r, const void *X, int x_bf16, int64_t B,
                     float *Y, float *P, float *z, cudaStream_t s) {
    const int chunks = bin_gemv_chunks(n, r, B);
    const int64_t rpc = (n + chunks - 1) / chunks;
    const int nw = (r + 31) / 32;
    const size_t smem_z = (size_t)rpc * (B + nw) * sizeof(float);
    if (smem_z > 48 * 1024) {
        static std::atomic<uint64_t> configured{0};
        cudaError_t e = ensure_smem_limit((const void *)bin_z_kernel, 192 * 1024, configured);
        if (e != cudaSuccess) return e;
    }
    bin_z_kernel<<<(unsigned)chunks, 256, smem_z, s>>>(Vp, s2, X, x_bf16, n, r, B, rpc, P);
    count_launch();
    bin_zreduce_kernel<<<(unsigned)ceil_div(B * r, 256), 256, 0, s>>>(P, chunks, B * r, z);
    count_launch();
    // z staged in shared memory when it fits beside the words (at most 96 KB)
    const int z_in_smem = (size_t)B * r * sizeof(float) <= 96 * 1024;
    const size_t smem_y = (size_t)kBinRowsPerCta * nw * sizeof(uint32_t) +
                          (z_in_smem ? (size_t)B * r * sizeof(float) : 0);
    if (smem_y > 48 * 1024) {
        static std::atomic<uint64_t> configured{0};
        cudaError_t e = ensure_smem_limit((const void *)bin_y_kernel, 192 * 1024, configured);
        if (e != cudaSuccess) return e;
    }
    bin_y_kernel<<<(unsigned)ceil_div(m, kBinRowsPerCta), 256, smem_y, s>>>(Up, s1, z, m, r, B,
                                                                           z_in_smem, Y);
    count_launch();
    return cudaGetLastError();
}

// ---- tensor path: operand expansion ---------------------------------------------------
// Vt_hi[k][j] = +-bf16(s2_j), Vt_lo[k][j] = +-bf16(s2_j - bf16(s2_j)): the B operand of
// Z = X diag(s2) V+- (split, so that X V' sums FP32-accurate scaled signs).  [r][ldt]
__global__ void bin_expand_v_kernel(const uint32_t *__restrict__ Vp, const float *__restrict__ s2,
                                    int64_t n, int r, int64_t ldt, __nv_bfloat16 *Vh,
                                    __nv_bfloat16 *Vl) {
    __shared__ __nv_bfloat16 th[32][34], tl[32][34];
    const int nw = (r + 31) >> 5;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8
    const int64_t j0 = (int64_t)blockIdx.y * 32;              // rows j of V
    const int wd = blockIdx.x;                                // word: columns k = 32 wd + tx
    for (int a = ty; a < 32; a += 8) {
        const int64_t j = j0 + a;
        __nv_bfloat16 h = __float2bfloat16_rn(0.f), l = h;
        if (j < n) {
            const float sj = s2[j];
            const bool neg = (Vp[j * nw + wd] >> tx) & 1u;
            h = __float2bfloat16_rn(sj);
            l = __float2bfloat16_rn(sj - __bfloat162float(h));
            if (neg) {
                h = __hneg(h);
                l = __hneg(l);
            }
        }
        th[a][tx] = h;
        tl[a][tx] = l;
    }
    __syncthreads();
    for (int a = ty; a < 32; a += 8) {
        const int k = 32 * wd + a;
        const int64_t j = j0 + tx;
        if (k < r && j < n) {
            Vh[(int64_t)k * ldt + j] = th[tx][a];
            Vl[(int64_t)k * ldt + j] = tl[tx][a];
        }
    }
}

// Um[i][k] = +-1 (bf16), [m][ldr]: the B operand of Y = Z U+-^T.
__global__ void bin_expand_u_kernel(const uint32_t *__restrict__ Up, int64_t m, int r, int64_t ldr,
                                    __nv_bfloat16 *Um) {
    const int nw = (r + 31) >> 5;
    const int64_t total = m * (int64_t)r;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / r;
        const int k = (int)(e % r);
        const bool neg = (Up[i * nw + (k >> 5)] >> (k & 31)) & 1u;
        Um[i * ldr + k] = __float2bfloat16_rn(neg ? -1.f : 1.f);
    }
}

// X (B x n, FP32 or BF16) into BF16 hi (and, for FP32 X, lo) rows of stride ldx.
__global__ void bin_split_x_kernel(const void *__restrict__ X, int x_bf16, int64_t B, int64_t n,
                                   int64_t ldx, __nv_bfloat16 *Xh, __nv_bfloat16 *Xl) {
    const int64_t total = B * n;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = e / n, j = e % n;
        if (x_bf16) {
            Xh[b * ldx + j] = reinterpret_cast<const __nv_bfloat16 *>(X)[e];
        } else {
            const float x = reinterpret_cast<const float *>(X)[e];
            const __nv_bfloat16 h = __float2bfloat16_rn(x);
            Xh[b * ldx + j] = h;
            Xl[b * ldx + j] = __float2bfloat16_rn(x - __bfloat162float(h));
        }
    }
}

cudaError_t bin_expand(const uint32_t *Up, const uint32_t *Vp, const float *s2, int64_t m,
                       int64_t n, int32_t r, const void *X, int x_bf16, int64_t B,
                       __nv_bfloat16 *Vh, __nv_bfloat16 *Vl, int64_t ldt, __nv_bfloat16 *Um,
                       int64_t ldr, __nv_bfloat16 *Xh, __nv_bfloat16 *Xl, int64_t ldx,
                       cudaStream_t s) {
    const int nw = (r + 31) / 32;
    bin_expand_v_kernel<<<dim3((unsigned)nw, (unsigned)ceil_div(n, 32)), 256, 0, s>>>(
        Vp, s2, n, r, ldt, Vh, Vl);
    count_launch();
    bin_expand_u_kernel<<<4 * kNumSMsB200, 256, 0, s>>>(Up, m, r, ldr, Um);
    count_launch();
    bin_split_x_kernel<<<4 * kNumSMsB200, 256, 0, s>>>(X, x_bf16, B, n, ldx, Xh, Xl);
    count_launch();
    return cudaGetLastError();
}

}  // namespace nq
