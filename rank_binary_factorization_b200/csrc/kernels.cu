// SIMT kernels of the NanoQuant hot path (sm_100a): calibration reduction, target
// preparation, V_0, SVID power passes, objective,
// balancing / scale extraction / sign packing.
#include <cooperative_groups.h>

#include "kernels.cuh"

namespace nq {

// =================================================================================
// Calibration statistics.  NanoQuant summary page, "Method steps" (方法步骤详情),
// stage one: per-channel statistics over the calibration tokens.
// =================================================================================
template <bool BF16>
__device__ __forceinline__ void unpack16(const uint4 &raw, float (&x)[BF16 ? 8 : 4]) {
    if constexpr (BF16) {
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __bfloat1622float2(h[i]);
            x[2 * i] = f.x;
            x[2 * i + 1] = f.y;
        }
    } else {
        x[0] = __uint_as_float(raw.x);
        x[1] = __uint_as_float(raw.y);
        x[2] = __uint_as_float(raw.z);
        x[3] = __uint_as_float(raw.w);
    }
}

// Streaming 16-byte load that is not kept in L1 (each byte is read once).
__device__ __forceinline__ uint4 ld_stream16(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// CTA = 8 warps over one slab of 32*VEC channels; warp w takes tokens w, w+8, ...
// of the CTA's token slab; each lane owns VEC consecutive channels (one 16-byte load
// per token) and keeps 8 loads in flight.  FP32 sums over 16 tokens are added into the
// warp's FP64 accumulators in shared memory (laid out [v][lane]: no bank conflicts),
// which keeps the register count low enough for 4 CTAs (32 warps) per SM.
template <bool BF16>
__global__ void __launch_bounds__(256, 4) calib_partial_vec(const void *__restrict__ Xv, int64_t T,
                                                            int64_t C, int64_t tok_per_slab,
                                                            double *__restrict__ ps,
                                                            double *__restrict__ pq) {
    constexpr int VEC = BF16 ? 8 : 4;
    constexpr int ESZ = BF16 ? 2 : 4;
    constexpr int U = 8;  // loads in flight per thread
    __shared__ double sh_s[8][VEC][32];
    __shared__ double sh_q[8][VEC][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t cbase = (int64_t)blockIdx.x * 32 * VEC;
    const int64_t c0 = cbase + lane * VEC;
    const int64_t t_begin = (int64_t)blockIdx.y * tok_per_slab;
    const int64_t t_end = min(T, t_begin + tok_per_slab);
#pragma unroll
    for (int v = 0; v < VEC; ++v) sh_s[warp][v][lane] = sh_q[warp][v][lane] = 0.0;
    if (c0 < C) {
        const char *base = reinterpret_cast<const char *>(Xv) + c0 * ESZ;
        const int64_t row_bytes = C * ESZ;
        int64_t t = t_begin + warp;
        while (t < t_end) {
            float fs[VEC], fq[VEC];
#pragma unroll
            for (int v = 0; v < VEC; ++v) fs[v] = fq[v] = 0.f;
            int cnt = 0;
            for (; cnt < 16 && t + 8 * (U - 1) < t_end; cnt += U, t += 8 * U) {
                uint4 raw[U];
#pragma unroll
                for (int u = 0; u < U; ++u) raw[u] = ld_stream16(base + (t + 8 * u) * row_bytes);
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    float x[VEC];
                    unpack16<BF16>(raw[u], x);
#pragma unroll
                    for (int v = 0; v < VEC; ++v) {
                        const float x2 = x[v] * x[v];
                        fs[v] += x2;
                        fq[v] = fmaf(x2, x2, fq[v]);
                    }
                }
            }
            for (; cnt < 16 && t < t_end; ++cnt, t += 8) {
                float x[VEC];
                unpack16<BF16>(ld_stream16(base + t * row_bytes), x);
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    const float x2 = x[v] * x[v];
                    fs[v] += x2;
                    fq[v] = fmaf(x2, x2, fq[v]);
                }
            }
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                sh_s[warp][v][lane] += fs[v];
                sh_q[warp][v][lane] += fq[v];
            }
        }
    }
    __syncthreads();
    for (int c = threadIdx.x; c < 32 * VEC; c += blockDim.x) {
        if (cbase + c >= C) continue;
        const int v = c % VEC, l = c / VEC;
        double a = 0.0, b = 0.0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            a += sh_s[w][v][l];
            b += sh_q[w][v][l];
        }
        ps[(int64_t)blockIdx.y * C + cbase + c] = a;
        pq[(int64_t)blockIdx.y * C + cbase + c] = b;
    }
}

// Scalar path (C not a multiple of the vector width): thread per channel.
template <bool BF16>
__global__ void __launch_bounds__(256) calib_partial_scalar(const void *__restrict__ Xv, int64_t T,
                                                            int64_t C, int64_t tok_per_slab,
                                                            double *__restrict__ ps,
                                                            double *__restrict__ pq) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= C) return;
    const int64_t t_begin = (int64_t)blockIdx.y * tok_per_slab;
    const int64_t t_end = min(T, t_begin + tok_per_slab);
    double ds = 0.0, dq = 0.0;
    for (int64_t t0 = t_begin; t0 < t_end; t0 += 16) {
        float fs = 0.f, fq = 0.f;
        const int64_t t1 = min(t_end, t0 + 16);
        for (int64_t t = t0; t < t1; ++t) {
            float x;
            if constexpr (BF16)
                x = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(Xv)[t * C + c]);
            else
                x = reinterpret_cast<const float *>(Xv)[t * C + c];
            const float x2 = x * x;
            fs += x2;
            fq = fmaf(x2, x2, fq);
        }
        ds += fs;
        dq += fq;
    }
    ps[(int64_t)blockIdx.y * C + c] = ds;
    pq[(int64_t)blockIdx.y * C + c] = dq;
}

// Token slabs: as many CTAs as fit in one wave (4 CTAs of 256 channels per SM) without
// spilling a partial second wave.
int calib_num_slabs(int64_t T, int64_t C) {
    const int64_t cx = ceil_div(C, 256);
    int64_t ns = (4 * kNumSMsB200) / cx;
    const int64_t max_by_T = ceil_div(T, 256);
    if (ns > max_by_T) ns = max_by_T;
    if (ns < 1) ns = 1;
    if (ns > 4096) ns = 4096;
    return (int)ns;
}

cudaError_t calib_partials(const void *X, int64_t T, int64_t C, int dt_bf16, int nslab,
                           double *ps, double *pq, cudaStream_t s) {
    const int64_t tps = ceil_div(T, nslab);
    const int vec = dt_bf16 ? 8 : 4;
    const bool aligned = (reinterpret_cast<uintptr_t>(X) % 16 == 0) && (C % vec == 0);
    if (aligned) {
        dim3 grid((unsigned)ceil_div(C, 32 * vec), (unsigned)nslab);
        if (dt_bf16)
            calib_partial_vec<true><<<grid, 256, 0, s>>>(X, T, C, tps, ps, pq);
        else
            calib_partial_vec<false><<<grid, 256, 0, s>>>(X, T, C, tps, ps, pq);
    } else {
        dim3 grid((unsigned)ceil_div(C, 256), (unsigned)nslab);
        if (dt_bf16)
            calib_partial_scalar<true><<<grid, 256, 0, s>>>(X, T, C, tps, ps, pq);
        else
            calib_partial_scalar<false><<<grid, 256, 0, s>>>(X, T, C, tps, ps, pq);
    }
    count_launch();
    return cudaGetLastError();
}

__global__ void calib_moments_kernel(const double *__restrict__ ps, const double *__restrict__ pq,
                                     int nslab, int64_t T, int64_t C, double *s_out,
                                     double *q_out) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= C) return;
    double a = 0.0, b = 0.0;
    for (int k = 0; k < nslab; ++k) {
        a += ps[(int64_t)k * C + c];
        b += pq[(int64_t)k * C + c];
    }
    s_out[c] = a / (double)T;
    q_out[c] = b / (double)T;
}

cudaError_t calib_moments(const double *ps, const double *pq, int nslab, int64_t T, int64_t C,
                          double *s_out, double *q_out, cudaStream_t st) {
    calib_moments_kernel<<<(unsigned)ceil_div(C, 256), 256, 0, st>>>(ps, pq, nslab, T, C, s_out,
                                                                     q_out);
    count_launch();
    return cudaGetLastError();
}

// Deterministic block sum (fixed order) of one double per thread; blockDim = 1024.
__device__ double block_sum_1024(double v, double *sh) {
    sh[threadIdx.x] = v;
    __syncthreads();
    for (int o = 512; o > 0; o >>= 1) {
        if (threadIdx.x < o) sh[threadIdx.x] += sh[threadIdx.x + o];
        __syncthreads();
    }
    const double r = sh[0];
    __syncthreads();
    return r;
}

// Ledoit-Wolf 2004 with target mu I restricted to the diagonal (see nq_calib_precond).
__global__ void __launch_bounds__(1024)
    calib_lw_kernel(const double *__restrict__ s, const double *__restrict__ q, int64_t T,
                    int64_t C, double alpha_override, float *d, double *alpha_out, int *err) {
    __shared__ double sh[1024];
    double a = 0.0;
    for (int64_t c = threadIdx.x; c < C; c += blockDim.x) a += s[c];
    const double sum_s = block_sum_1024(a, sh);
    const double mu = sum_s / (double)C;
    double dd = 0.0, bb = 0.0;
    for (int64_t c = threadIdx.x; c < C; c += blockDim.x) {
        const double e = s[c] - mu;
        dd += e * e;
        bb += q[c] - s[c] * s[c];
    }
    const double delta2 = block_sum_1024(dd, sh);
    const double beta_bar2 = block_sum_1024(bb, sh) / (double)T;
    if (!isfinite(sum_s) || !isfinite(beta_bar2)) {
        if (threadIdx.x == 0) raise_error(err, NQ_ERR_NONFINITE);
    }
    double alpha;
    if (alpha_override >= 0.0)
        alpha = alpha_override;
    else
        alpha = delta2 == 0.0 ? 1.0 : fmin(beta_bar2, delta2) / delta2;
    for (int64_t c = threadIdx.x; c < C; c += blockDim.x) {
        double dt = (1.0 - alpha) * s[c] + alpha * mu;
        dt = fmax(dt, 1e-12 * mu);
        d[c] = (float)sqrt(dt);
    }
    if (threadIdx.x == 0 && alpha_out) *alpha_out = alpha;
}

cudaError_t calib_ledoit_wolf(const double *s, const double *q, int64_t T, int64_t C,
                              double alpha_override, float *d, double *alpha, int *err,
                              cudaStream_t st) {
    calib_lw_kernel<<<1, 1024, 0, st>>>(s, q, T, C, alpha_override, d, alpha, err);
    count_launch();
    return cudaGetLastError();
}

// =================================================================================
// Preconditioned, normalised target.  Same page, "Method steps", stage two:
// W~ = D_out W D_in.
// =================================================================================
__device__ __forceinline__ float load_wf(const void *W, int w_bf16, int64_t idx) {
    return w_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(W)[idx])
                  : reinterpret_cast<const float *>(W)[idx];
}

__device__ double block_sum_256(double v, double *sh) {
    sh[threadIdx.x] = v;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if (threadIdx.x < o) sh[threadIdx.x] += sh[threadIdx.x + o];
        __syncthreads();
    }
    const double r = sh[0];
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(256)
    wt_norm_kernel(const void *__restrict__ W, int w_bf16, int64_t m, int64_t n,
                   const float *__restrict__ d_in, const float *__restrict__ d_out, double *part,
                   int *err) {
    __shared__ double sh[256];
    double acc = 0.0;
    bool bad = false;
    for (int64_t i = blockIdx.x; i < m; i += gridDim.x) {
        const float dro = d_out ? d_out[i] : 1.f;
        float f = 0.f;
        for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
            const float w = dro * load_wf(W, w_bf16, i * n + j) * (d_in ? d_in[j] : 1.f);
            bad |= !isfinite(w);
            f = fmaf(w, w, f);
        }
        acc += f;
    }
    if (bad) raise_error(err, NQ_ERR_NONFINITE);
    const double t = block_sum_256(acc, sh);
    if (threadIdx.x == 0) part[blockIdx.x] = t;
}

cudaError_t wt_norm_partials(const void *W, int w_bf16, int64_t m, int64_t n, const float *d_in,
                             const float *d_out, double *part, int *err, cudaStream_t s) {
    wt_norm_kernel<<<kRedBlocks, 256, 0, s>>>(W, w_bf16, m, n, d_in, d_out, part, err);
    count_launch();
    return cudaGetLastError();
}

__global__ void __launch_bounds__(256)
    reduce_partials_kernel(const double *part, int count, double *sum, double *gamma, int r) {
    __shared__ double sh[256];
    double a = 0.0;
    for (int i = threadIdx.x; i < count; i += blockDim.x) a += part[i];
    const double t = block_sum_256(a, sh);
    if (threadIdx.x == 0) {
        if (sum) *sum = t;
        if (gamma) *gamma = sqrt(t) / (2.0 * sqrt((double)r));
    }
}

cudaError_t reduce_partials(const double *part, int count, double *sum, double *gamma, int r,
                            cudaStream_t s) {
    reduce_partials_kernel<<<1, 256, 0, s>>>(part, count, sum, gamma, r);
    count_launch();
    return cudaGetLastError();
}

// 32 x 32 tiles, grid-stride over all tiles of the padded (ldm x ldn) index space.
__global__ void __launch_bounds__(256)
    what_cast_kernel(const void *__restrict__ W, int w_bf16, int64_t m, int64_t n,
                     const float *__restrict__ d_in, const float *__restrict__ d_out,
                     const double *__restrict__ gamma, __nv_bfloat16 *What, int64_t ldn,
                     __nv_bfloat16 *WhatT, int64_t ldm, __nv_bfloat16 *WhatL,
                     __nv_bfloat16 *WhatTL, double *part) {
    __shared__ __nv_bfloat16 tile[32][34];
    __shared__ __nv_bfloat16 tile_lo[32][34];
    __shared__ double sh[256];
    const bool split = WhatL != nullptr;
    const double g = *gamma;
    const float inv = g > 0.0 ? (float)(1.0 / g) : 0.f;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
    const int64_t ntx = ceil_div(ldn, 32), nty = ceil_div(ldm, 32);
    double acc = 0.0;
    for (int64_t t = blockIdx.x; t < ntx * nty; t += gridDim.x) {
        const int64_t i0 = (t / ntx) * 32, j0 = (t % ntx) * 32;
        float f = 0.f;
        for (int k = ty; k < 32; k += 8) {
            const int64_t i = i0 + k, j = j0 + tx;
            __nv_bfloat16 h = __float2bfloat16_rn(0.f), l = h;
            if (i < m && j < n) {
                const float w = (d_out ? d_out[i] : 1.f) * load_wf(W, w_bf16, i * n + j) *
                                (d_in ? d_in[j] : 1.f);
                const float x = w * inv;
                h = __float2bfloat16_rn(x);
                float hv = __bfloat162float(h);
                if (split) {
                    l = __float2bfloat16_rn(x - hv);
                    hv += __bfloat162float(l);
                }
                f = fmaf(hv, hv, f);
            }
            if (i < m && j < ldn) {
                What[i * ldn + j] = h;
                if (split) WhatL[i * ldn + j] = l;
            }
            tile[k][tx] = h;
            tile_lo[k][tx] = l;
        }
        acc += f;
        __syncthreads();
        for (int k = ty; k < 32; k += 8) {
            const int64_t j = j0 + k, i = i0 + tx;
            if (j < n && i < ldm) {
                WhatT[j * ldm + i] = tile[tx][k];
                if (split) WhatTL[j * ldm + i] = tile_lo[tx][k];
            }
        }
        __syncthreads();
    }
    const double s = block_sum_256(acc, sh);
    if (threadIdx.x == 0) part[blockIdx.x] = s;
}

cudaError_t what_cast(const void *W, int w_bf16, int64_t m, int64_t n, const float *d_in,
                      const float *d_out, const double *gamma, __nv_bfloat16 *What, int64_t ldn,
                      __nv_bfloat16 *WhatT, int64_t ldm, __nv_bfloat16 *WhatL,
                      __nv_bfloat16 *WhatTL, double *part, cudaStream_t s) {
    what_cast_kernel<<<kRedBlocks, 256, 0, s>>>(W, w_bf16, m, n, d_in, d_out, gamma, What, ldn,
                                                WhatT, ldm, WhatL, WhatTL, part);
    count_launch();
    return cudaGetLastError();
}

// SplitMix64 (Steele, Lea, Flood 2014), evaluated as a function of a counter.
__device__ __forceinline__ uint64_t splitmix64(uint64_t seed, uint64_t idx) {
    uint64_t z = seed + (idx + 1ull) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__global__ void init_v0_kernel(int64_t n, int32_t r, uint64_t seed, float c, float *X,
                               int64_t ldr, __nv_bfloat16 *Xt, __nv_bfloat16 *XtL, int64_t ldn) {
    const int64_t total = n * (int64_t)r;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        // row-major pass over X (k fastest)
        const int64_t j = e / r, k = e % r;
        const float v = (splitmix64(seed, (uint64_t)e) >> 63) ? -c : c;
        X[j * ldr + k] = v;
        // column-major pass over Xt (j fastest): element (k2, j2)
        const int64_t k2 = e / n, j2 = e % n;
        const float v2 = (splitmix64(seed, (uint64_t)(j2 * r + k2)) >> 63) ? -c : c;
        const __nv_bfloat16 h = __float2bfloat16_rn(v2);
        Xt[k2 * ldn + j2] = h;
        if (XtL) XtL[k2 * ldn + j2] = __float2bfloat16_rn(v2 - __bfloat162float(h));
    }
}

cudaError_t init_v0(int64_t n, int32_t r, uint64_t seed, float *X, int64_t ldr,
                    __nv_bfloat16 *Xt, __nv_bfloat16 *XtL, int64_t ldn, cudaStream_t s) {
    const float c = sqrtf(2.0f / (float)n);
    init_v0_kernel<<<4 * kNumSMsB200, 256, 0, s>>>(n, r, seed, c, X, ldr, Xt, XtL, ldn);
    count_launch();
    return cudaGetLastError();
}

__global__ void __launch_bounds__(256)
    transpose_to_bf16_kernel(const float *__restrict__ X, int64_t rows, int32_t r, int64_t ldx,
                             __nv_bfloat16 *Xt, __nv_bfloat16 *XtL, int64_t ldt) {
    __shared__ float tile[32][33];
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int64_t i0 = (int64_t)blockIdx.y * 32, k0 = (int64_t)blockIdx.x * 32;
    for (int a = ty; a < 32; a += 8) {
        const int64_t i = i0 + a, k = k0 + tx;
        tile[a][tx] = (i < rows && k < r) ? X[i * ldx + k] : 0.f;
    }
    __syncthreads();
    for (int a = ty; a < 32; a += 8) {
        const int64_t k = k0 + a, i = i0 + tx;
        if (k < r && i < rows) {
            const float x = tile[tx][a];
            const __nv_bfloat16 h = __float2bfloat16_rn(x);
            Xt[k * ldt + i] = h;
            if (XtL) XtL[k * ldt + i] = __float2bfloat16_rn(x - __bfloat162float(h));
        }
    }
}

cudaError_t transpose_to_bf16(const float *X, int64_t rows, int32_t r, int64_t ldx,
                              __nv_bfloat16 *Xt, __nv_bfloat16 *XtL, int64_t ldt, cudaStream_t s) {
    dim3 grid((unsigned)ceil_div(r, 32), (unsigned)ceil_div(rows, 32));
    transpose_to_bf16_kernel<<<grid, 256, 0, s>>>(X, rows, r, ldx, Xt, XtL, ldt);
    count_launch();
    return cudaGetLastError();
}

__global__ void __launch_bounds__(256)
    transpose_bf16_kernel(const __nv_bfloat16 *__restrict__ A, int64_t rows, int64_t cols,
                          int64_t lda, __nv_bfloat16 *B, int64_t ldb) {
    __shared__ __nv_bfloat16 tile[32][34];
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int64_t i0 = (int64_t)blockIdx.y * 32, j0 = (int64_t)blockIdx.x * 32;
    for (int a = ty; a < 32; a += 8) {
        const int64_t i = i0 + a, j = j0 + tx;
        tile[a][tx] = (i < rows && j < cols) ? A[i * lda + j] : __float2bfloat16_rn(0.f);
    }
    __syncthreads();
    for (int a = ty; a < 32; a += 8) {
        const int64_t j = j0 + a, i = i0 + tx;
        if (j < cols && i < rows) B[j * ldb + i] = tile[tx][a];
    }
}

cudaError_t transpose_bf16(const __nv_bfloat16 *A, int64_t rows, int64_t cols, int64_t lda,
                           __nv_bfloat16 *B, int64_t ldb, cudaStream_t s) {
    dim3 grid((unsigned)ceil_div(cols, 32), (unsigned)ceil_div(rows, 32));
    transpose_bf16_kernel<<<grid, 256, 0, s>>>(A, rows, cols, lda, B, ldb);
    count_launch();
    return cudaGetLastError();
}

// =================================================================================
// SVID power steps.  Same page, "Core method", step (b): the continuous U is mapped
// to the binary proxy Z = sign(S) * a b^T, a b^T the rank-1 fit of |S| by K power
// steps from b = 1.  One pass over S per power step: t = |S| b row by row and
// b' = |S|^T t / ||t|| column by column, from the same shared-memory copy of S.
// =================================================================================
// Each CTA stages tiles of rows of S in shared memory (16-byte cp.async copies); warp w
// forms the row dot t_w = |S_w.| b, then every thread accumulates its columns' share of
// |S|^T t.  Partial sums per CTA go to partb / partn (fixed order).
// Each CTA walks its tiles of ROWS rows with a two-buffer cp.async ring, so the copy of
// the next tile overlaps the arithmetic on the current one.
__device__ __forceinline__ void cp_async16(float *dst, const float *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(float *dst, const float *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}

template <int ROWS>
__global__ void __launch_bounds__(256)
    svid_pass2_kernel(const float *__restrict__ S, int64_t rows, int r, int64_t ldf,
                      const float *__restrict__ b_in, float *tvec, int write_t, float *partb,
                      double *partn) {
    extern __shared__ __align__(16) float sm[];
    float *sb = sm + 2 * ROWS * ldf;     // b (r)
    __shared__ float st[ROWS];
    __shared__ double sn[ROWS];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int k = threadIdx.x; k < r; k += blockDim.x) sb[k] = b_in ? b_in[k] : 1.f;
    float acc[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) acc[u] = 0.f;
    double nacc = 0.0;
    const int r4 = r >> 2, rt = r - 4 * r4;
    const int64_t ntile = ceil_div(rows, ROWS);
    // copy tile `tile` (ROWS rows of S, zero rows past the end) into buffer `buf`
    auto issue = [&](int64_t tile, float *buf) {
        const int64_t row0 = tile * ROWS;
        for (int e = threadIdx.x; e < ROWS * r4; e += blockDim.x) {
            const int w = e / r4, k4 = e - w * r4;
            const int64_t i = row0 + w;
            float *dst = buf + w * ldf + 4 * k4;
            if (i < rows)
                cp_async16(dst, S + i * ldf + 4 * k4);
            else
                *reinterpret_cast<float4 *>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int e = threadIdx.x; e < ROWS * rt; e += blockDim.x) {
            const int w = e / rt, k = 4 * r4 + e % rt;
            const int64_t i = row0 + w;
            if (i < rows)
                cp_async4(buf + w * ldf + k, S + i * ldf + k);
            else
                buf[w * ldf + k] = 0.f;
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    int64_t tile = blockIdx.x;
    if (tile < ntile) issue(tile, sm);
    int cur = 0;
    for (; tile < ntile; tile += gridDim.x, cur ^= 1) {
        float *bc = sm + cur * ROWS * ldf;
        const int64_t next = tile + gridDim.x;
        if (next < ntile) {
            issue(next, sm + (cur ^ 1) * ROWS * ldf);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        const int64_t row0 = tile * ROWS;
        if (warp < ROWS) {
            float t = 0.f;
            for (int k = lane; k < r; k += 32) t = fmaf(fabsf(bc[warp * ldf + k]), sb[k], t);
            t = warp_sum(t);
            if (lane == 0) {
                st[warp] = t;
                nacc += (double)t * (double)t;
                if (write_t && row0 + warp < rows) tvec[row0 + warp] = t;
            }
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int k = threadIdx.x + 256 * u;
            if (k < r) {
                float v = 0.f;
#pragma unroll
                for (int w = 0; w < ROWS; ++w) v = fmaf(fabsf(bc[w * ldf + k]), st[w], v);
                acc[u] += v;
            }
        }
        __syncthreads();   // bc may be refilled by the next-but-one tile's copy
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        const int k = threadIdx.x + 256 * u;
        if (k < r) partb[(int64_t)blockIdx.x * r + k] = acc[u];
    }
    if (lane == 0 && warp < ROWS) sn[warp] = nacc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double v = 0.0;
        for (int w = 0; w < ROWS; ++w) v += sn[w];
        partn[blockIdx.x] = v;
    }
}

// Row-streaming pass for r <= 32 NPL: lane l of a warp holds columns l, l + 32, ... of one
// row of S in registers; the warp forms t = |S_i.| b with a shuffle sum and adds
// |S_i.| t to its column partials, row after row, with no CTA barrier per row.  At the
// end the 8 warps' partials are summed in a fixed order.
template <int NPL>
__global__ void __launch_bounds__(256, 2)
    svid_rows_kernel(const float *__restrict__ S, int64_t rows, int r, int64_t ldf,
                     const float *__restrict__ b_in, float *tvec, int write_t, float *partb,
                     double *partn) {
    // 16 KB of partial rows (the warps' column sums are combined in two rounds), so that a
    // CTA fits on an SM beside a GEMM CTA of the half step it runs beside
    __shared__ float red[4][32 * NPL];
    __shared__ double sn[8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // b is read from shared memory (its registers go to the next row's prefetch)
    float *sb = red[0];
    for (int k = threadIdx.x; k < 32 * NPL; k += blockDim.x)
        sb[k] = k < r ? (b_in ? b_in[k] : 1.f) : 0.f;
    __syncthreads();
    float acc[NPL];
#pragma unroll
    for (int u = 0; u < NPL; ++u) acc[u] = 0.f;
    double nacc = 0.0;
    const int64_t nw = (int64_t)gridDim.x * 8;
    // two rows in flight per warp: the next row's loads are issued before this row's sums
    float cur[NPL], nxt[NPL];
    int64_t i = (int64_t)blockIdx.x * 8 + warp;
    if (i < rows) {
        const float *row = S + i * ldf;
#pragma unroll
        for (int u = 0; u < NPL; ++u) {
            const int k = lane + 32 * u;
            cur[u] = k < r ? __ldcg(row + k) : 0.f;
        }
    }
    for (; i < rows; i += nw) {
        const int64_t in = i + nw;
        if (in < rows) {
            const float *row = S + in * ldf;
#pragma unroll
            for (int u = 0; u < NPL; ++u) {
                const int k = lane + 32 * u;
                nxt[u] = k < r ? __ldcg(row + k) : 0.f;
            }
        }
        float t = 0.f;
#pragma unroll
        for (int u = 0; u < NPL; ++u) t = fmaf(fabsf(cur[u]), sb[lane + 32 * u], t);
        t = warp_sum(t);
#pragma unroll
        for (int u = 0; u < NPL; ++u) acc[u] = fmaf(fabsf(cur[u]), t, acc[u]);
        if (lane == 0) {
            nacc += (double)t * (double)t;
            if (write_t) tvec[i] = t;
        }
#pragma unroll
        for (int u = 0; u < NPL; ++u) cur[u] = nxt[u];
    }
    __syncthreads();   // every warp is done with sb (it aliases red[0])
    if (warp >= 4) {
#pragma unroll
        for (int u = 0; u < NPL; ++u) red[warp - 4][lane + 32 * u] = acc[u];
    }
    if (lane == 0) sn[warp] = nacc;
    __syncthreads();
    if (warp < 4) {
#pragma unroll
        for (int u = 0; u < NPL; ++u) red[warp][lane + 32 * u] += acc[u];
    }
    __syncthreads();
    for (int k = threadIdx.x; k < r; k += blockDim.x) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) v += red[w][k];
        partb[(int64_t)blockIdx.x * r + k] = v;
    }
    if (threadIdx.x == 0) {
        double v = 0.0;
        for (int w = 0; w < 8; ++w) v += sn[w];
        partn[blockIdx.x] = v;
    }
}

// b'_k = sum over CTAs of partb[.][k] / ||t||: CTA = 32 columns x 32 groups of partial
// rows; each group walks every 32nd partial row, then the 32 group sums are combined in a
// fixed order (deterministic).  The last pass also writes a = t / ||t||.
__global__ void __launch_bounds__(1024)
    svid_reduce_kernel(const float *__restrict__ partb, const double *__restrict__ partn, int nblk,
                       int r, int64_t rows, int last, const float *__restrict__ tvec,
                       float *b_out, float *a_out) {
    __shared__ double s_inv;
    __shared__ double sg[32][33];
    if (threadIdx.x < 32) {
        double n2 = 0.0;
        for (int k = threadIdx.x; k < nblk; k += 32) n2 += partn[k];
        n2 = warp_sum(n2);
        if (threadIdx.x == 0) {
            const double nt = sqrt(n2);
            s_inv = nt > 0.0 ? 1.0 / nt : 0.0;
        }
    }
    const int c = threadIdx.x & 31, grp = threadIdx.x >> 5;
    const int64_t col = (int64_t)blockIdx.x * 32 + c;
    double v = 0.0;
    if (col < r) {
        double w[4] = {0.0, 0.0, 0.0, 0.0};   // interleaved sums keep the loads in flight
        int k = grp, u = 0;
#pragma unroll 4
        for (; k < nblk; k += 32, u = (u + 1) & 3) w[u] += partb[(int64_t)k * r + col];
        v = (w[0] + w[1]) + (w[2] + w[3]);
    }
    sg[grp][c] = v;
    __syncthreads();
    const double inv = s_inv;
    if (grp == 0 && col < r) {
        double t = 0.0;
#pragma unroll
        for (int g = 0; g < 32; ++g) t += sg[g][c];
        b_out[col] = (float)(t * inv);
    }
    if (last) {
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows;
             i += (int64_t)gridDim.x * blockDim.x)
            a_out[i] = (float)((double)tvec[i] * inv);
    }
}

// Rows per pipelined tile: two buffers of ROWS x ldf floats stay near 64 KB, so that
// several CTAs fit on an SM.
static int svid_tile_rows(int64_t ldf) { return ldf <= 1024 ? 8 : (ldf <= 2048 ? 4 : 2); }

template <int ROWS>
static cudaError_t svid_passes(const float *S, int64_t rows, int32_t r, int64_t ldf, int K,
                               int nsv, float *bcur, float *tvec, float *partb, double *partn,
                               float *a, float *b, cudaStream_t s) {
    const size_t smem = (size_t)(2 * ROWS * ldf + r) * sizeof(float);
    // largest dynamic shared-memory limit set so far, per device
    static std::atomic<size_t> configured[kMaxDevices];
    const int dev = current_device();
    if (dev < 0) return cudaErrorInvalidDevice;
    if (smem > 48 * 1024 && smem > configured[dev].load()) {
        cudaError_t e = cudaFuncSetAttribute(svid_pass2_kernel<ROWS>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        size_t prev = configured[dev].load();
        while (prev < smem && !configured[dev].compare_exchange_weak(prev, smem)) {
        }
    }
    // two CTAs per SM (the partial arrays hold nsv >= this many rows)
    int64_t grid = ceil_div(rows, ROWS);
    const int64_t cap = 2 * (int64_t)device_sm_count();
    if (grid > cap) grid = cap;
    if (grid > nsv) grid = nsv;
    for (int pass = 1; pass <= K; ++pass) {
        const float *b_in = pass == 1 ? nullptr : bcur + (size_t)((pass - 1) & 1) * r;
        const bool last = pass == K;
        float *b_out = last ? b : bcur + (size_t)(pass & 1) * r;
        svid_pass2_kernel<ROWS><<<(unsigned)grid, 256, smem, s>>>(S, rows, r, ldf, b_in, tvec,
                                                                 last ? 1 : 0, partb, partn);
        count_launch();
        svid_reduce_kernel<<<(unsigned)ceil_div(r, 32), 1024, 0, s>>>(
            partb, partn, (int)grid, r, rows, last ? 1 : 0, tvec, b_out, a);
        count_launch();
    }
    return cudaGetLastError();
}

template <int NPL>
static cudaError_t svid_row_passes(const float *S, int64_t rows, int32_t r, int64_t ldf, int K,
                                   int nsv, float *bcur, float *tvec, float *partb,
                                   double *partn, float *a, float *b, cudaStream_t s) {
    int64_t grid = ceil_div(rows, 8);
    const int64_t cap = 2 * (int64_t)device_sm_count();
    if (grid > cap) grid = cap;
    if (grid > nsv) grid = nsv;
    for (int pass = 1; pass <= K; ++pass) {
        const float *b_in = pass == 1 ? nullptr : bcur + (size_t)((pass - 1) & 1) * r;
        const bool last = pass == K;
        float *b_out = last ? b : bcur + (size_t)(pass & 1) * r;
        svid_rows_kernel<NPL><<<(unsigned)grid, 256, 0, s>>>(S, rows, r, ldf, b_in, tvec,
                                                            last ? 1 : 0, partb, partn);
        count_launch();
        svid_reduce_kernel<<<(unsigned)ceil_div(r, 32), 1024, 0, s>>>(
            partb, partn, (int)grid, r, rows, last ? 1 : 0, tvec, b_out, a);
        count_launch();
    }
    return cudaGetLastError();
}

cudaError_t svid(const float *S, int64_t rows, int32_t r, int64_t ldf, int K, int nsv,
                 float *bcur, float *tvec, float *partb, double *partn, float *a, float *b,
                 cudaStream_t s) {
    // rows of at most 1024 columns stream through registers; longer rows through tiles
    if (r <= 256) return svid_row_passes<8>(S, rows, r, ldf, K, nsv, bcur, tvec, partb, partn, a, b, s);
    if (r <= 512) return svid_row_passes<16>(S, rows, r, ldf, K, nsv, bcur, tvec, partb, partn, a, b, s);
    if (r <= 1024) return svid_row_passes<32>(S, rows, r, ldf, K, nsv, bcur, tvec, partb, partn, a, b, s);
    switch (svid_tile_rows(ldf)) {
        case 8: return svid_passes<8>(S, rows, r, ldf, K, nsv, bcur, tvec, partb, partn, a, b, s);
        case 4: return svid_passes<4>(S, rows, r, ldf, K, nsv, bcur, tvec, partb, partn, a, b, s);
        default: return svid_passes<2>(S, rows, r, ldf, K, nsv, bcur, tvec, partb, partn, a, b, s);
    }
}

// =================================================================================
// Split-K Gram: G = sum over the parts of the raw 128 x 128 tiles + diag I, mirrored.
// Unit u = part * T + t of the partial array holds lower-triangular tile t (row by row:
// (0,0), (1,0), (1,1), ...) of one K part.  Parts are summed in index order, so the
// result does not depend on the order in which the GEMM's CTAs finished.
// =================================================================================
__global__ void __launch_bounds__(256)
    gram_reduce_kernel(const float *__restrict__ P, int T, int S, int r, float diag, float *G,
                       __nv_bfloat16 *Gh, __nv_bfloat16 *Gl, int64_t ldg) {
    __shared__ float tr[32][33];
    const int t = blockIdx.x;
    int a = (int)((sqrtf(8.f * (float)t + 1.f) - 1.f) * 0.5f);
    while ((a + 1) * (a + 2) / 2 <= t) ++a;
    while (a * (a + 1) / 2 > t) --a;
    const int b = t - a * (a + 1) / 2;
    const int m0 = a * 128, n0 = b * 128;
    const int si = (blockIdx.y >> 2) * 32, sj = (blockIdx.y & 3) * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    for (int k = ty; k < 32; k += 8) {
        const int li = si + k, lj = sj + tx;
        float v = 0.f;
        for (int sp = 0; sp < S; ++sp) v += P[((int64_t)(sp * T + t) * 128 + li) * 128 + lj];
        const int gi = m0 + li, gj = n0 + lj;
        if (gi == gj) v += diag;
        if (gi < r && gj < r) {
            G[(int64_t)gi * r + gj] = v;
            if (Gh) split_bf16(v, Gh + (int64_t)gi * ldg + gj, Gl + (int64_t)gi * ldg + gj);
        }
        tr[k][tx] = v;
    }
    if (a != b) {
        __syncthreads();
        for (int k = ty; k < 32; k += 8) {
            const int gi = n0 + sj + k, gj = m0 + si + tx;   // mirror of tile entry (si+tx, sj+k)
            if (gi < r && gj < r) {
                G[(int64_t)gi * r + gj] = tr[tx][k];
                if (Gh)
                    split_bf16(tr[tx][k], Gh + (int64_t)gi * ldg + gj,
                               Gl + (int64_t)gi * ldg + gj);
            }
        }
    }
}

// =================================================================================
// Gradient-descent latent update (solver variant): step size, operand split, and the
// state update that the solve epilogue performs on the exact path.
// =================================================================================
__global__ void __launch_bounds__(256)
    gd_rowabs_max_kernel(const float *__restrict__ G, int r, unsigned int *maxbits) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + warp;
    if (row >= r) return;
    float v = 0.f;
    for (int j = lane; j < r; j += 32) v += fabsf(G[(int64_t)row * r + j]);
    v = warp_sum(v);
    if (lane == 0) atomicMax(maxbits, __float_as_uint(v));
}

cudaError_t gd_rowabs_max(const float *G, int32_t r, unsigned int *maxbits, cudaStream_t s) {
    gd_rowabs_max_kernel<<<(unsigned)ceil_div(r, 8), 256, 0, s>>>(G, r, maxbits);
    count_launch();
    return cudaGetLastError();
}

__global__ void __launch_bounds__(256)
    split_rows_kernel(const float *__restrict__ X, int64_t rows, int r, int64_t ldf,
                      __nv_bfloat16 *Ph, __nv_bfloat16 *Pl, int64_t ldp) {
    const int64_t total = rows * r;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / r;
        const int k = (int)(e - i * r);
        split_bf16(X[i * ldf + k], Ph + i * ldp + k, Pl + i * ldp + k);
    }
}

cudaError_t split_rows(const float *X, int64_t rows, int32_t r, int64_t ldf,
                       __nv_bfloat16 *Ph, __nv_bfloat16 *Pl, int64_t ldp, cudaStream_t s) {
    split_rows_kernel<<<kRedBlocks, 256, 0, s>>>(X, rows, r, ldf, Ph, Pl, ldp);
    count_launch();
    return cudaGetLastError();
}

__global__ void __launch_bounds__(256)
    gd_finalize_kernel(const float *__restrict__ X, float *S, const float *__restrict__ a,
                       const float *__restrict__ b, int64_t rows, int r, int64_t ldf, float rho,
                       const __nv_bfloat16 *__restrict__ Rhi, const __nv_bfloat16 *__restrict__ Rlo,
                       int64_t ldr, __nv_bfloat16 *Xt, __nv_bfloat16 *XtL, int64_t ldxt,
                       int objective, double *part, int *err) {
    __shared__ double sh[256];
    const int64_t total = rows * r;
    double acc = 0.0;
    bool bad = false;
    // row-major walk: the reads of X, S and R and the store of S are coalesced, the
    // transposed stores of the operand copy are not
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / r;
        const int k = (int)(e - i * r);
        const float x = X[i * ldf + k];
        bad |= !isfinite(x);
        const float so = S[i * ldf + k];
        const float z = (so < 0.f ? -1.f : 1.f) * a[i] * b[k];
        S[i * ldf + k] = x + so - z;
        const __nv_bfloat16 h = __float2bfloat16_rn(x);
        float xo = __bfloat162float(h);
        Xt[(int64_t)k * ldxt + i] = h;
        if (XtL) {
            const __nv_bfloat16 l = __float2bfloat16_rn(x - xo);
            XtL[(int64_t)k * ldxt + i] = l;
            xo += __bfloat162float(l);
        }
        if (objective) {
            const float rr = __bfloat162float(Rhi[i * ldr + k]) + __bfloat162float(Rlo[i * ldr + k]);
            acc += (double)((rr - rho * (2.f * z - so)) * xo);
        }
    }
    if (bad) raise_error(err, NQ_ERR_NONFINITE);
    if (!objective) return;
    sh[threadIdx.x] = acc;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) sh[threadIdx.x] += sh[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) part[blockIdx.x] = sh[0];
}

cudaError_t gd_finalize(const float *X, float *S, const float *a, const float *b, int64_t rows,
                        int32_t r, int64_t ldf, float rho, const __nv_bfloat16 *Rhi,
                        const __nv_bfloat16 *Rlo, int64_t ldr, __nv_bfloat16 *Xt,
                        __nv_bfloat16 *XtL, int64_t ldxt, int objective, double *part,
                        int nparts, int *err, cudaStream_t s) {
    gd_finalize_kernel<<<(unsigned)nparts, 256, 0, s>>>(X, S, a, b, rows, r, ldf, rho, Rhi, Rlo,
                                                         ldr, Xt, XtL, ldxt, objective, part, err);
    count_launch();
    return cudaGetLastError();
}

cudaError_t gram_reduce(const float *P, int T, int S, int r, float diag, float *G,
                        __nv_bfloat16 *Gh, __nv_bfloat16 *Gl, int64_t ldg, cudaStream_t s) {
    gram_reduce_kernel<<<dim3((unsigned)T, 16), 256, 0, s>>>(P, T, S, r, diag, G, Gh, Gl, ldg);
    count_launch();
    return cudaGetLastError();
}

// =================================================================================
// Objective ||W^ - U V^T||^2 / ||W^||^2 = (||W^||^2 - 2 <W^^T U, V> + <U^T U, V^T V>)
// / ||W^||^2 from by-products: <W^^T U, V> from the V-step epilogue, the Gram
// matrices (less the ridge) of both steps.  All three terms are of the latents as the
// tensor-core operands hold them (BF16, or split BF16 at NQ_PREC_FP32), so the identity
// is exact for those matrices and only accumulation rounding enters the difference.
// =================================================================================
__global__ void __launch_bounds__(256)
    gram_dot_kernel(const float *__restrict__ GU, const float *__restrict__ GV, int r, float c,
                    double *part) {
    __shared__ double sh[256];
    const int64_t total = (int64_t)r * r;
    double acc = 0.0;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const bool dg = (e / r) == (e % r);
        acc += (double)(GU[e] - (dg ? c : 0.f)) * (double)(GV[e] - (dg ? c : 0.f));
    }
    const double t = block_sum_256(acc, sh);
    if (threadIdx.x == 0) part[blockIdx.x] = t;
}

__global__ void __launch_bounds__(256)
    objective_kernel(const double *__restrict__ px, int npx, const double *__restrict__ part,
                     int npart, const Scalars *sc, float *obj_slot) {
    __shared__ double sh[256];
    double a = 0.0, b = 0.0;
    for (int i = threadIdx.x; i < npx; i += blockDim.x) a += px[i];
    for (int i = threadIdx.x; i < npart; i += blockDim.x) b += part[i];
    const double spx = block_sum_256(a, sh);
    const double sgg = block_sum_256(b, sh);
    if (threadIdx.x == 0) {
        const double w2 = sc->what_norm2;
        *obj_slot = w2 > 0.0 ? (float)((w2 - 2.0 * spx + sgg) / w2) : 0.f;
    }
}

cudaError_t objective(const float *GU, const float *GV, int32_t r, float c, const double *px,
                      int npx, double *part, const Scalars *sc, float *obj_slot,
                      cudaStream_t s) {
    gram_dot_kernel<<<kRedBlocks, 256, 0, s>>>(GU, GV, r, c, part);
    count_launch();
    objective_kernel<<<1, 256, 0, s>>>(px, npx, part, kRedBlocks, sc, obj_slot);
    count_launch();
    return cudaGetLastError();
}

// =================================================================================
// Magnitude balancing, scale extraction, sign packing.  Same page, "Method steps",
// stage two (after convergence: balance, extract s1 and s2, pack the signs into
// integers) and "Technical novelty" (技术新颖性).
// =================================================================================
__global__ void __launch_bounds__(256)
    column_sumsq_kernel(const float *__restrict__ X, int64_t rows, int r, int64_t ldf,
                        float *partb) {
    float acc[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) acc[u] = 0.f;
    for (int64_t i = blockIdx.x; i < rows; i += gridDim.x) {
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int k = threadIdx.x + 256 * u;
            if (k < r) {
                const float x = X[i * ldf + k];
                acc[u] = fmaf(x, x, acc[u]);
            }
        }
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        const int k = threadIdx.x + 256 * u;
        if (k < r) partb[(int64_t)blockIdx.x * r + k] = acc[u];
    }
}

cudaError_t column_sumsq(const float *X, int64_t rows, int32_t r, int64_t ldf, int nblk,
                         float *partb, cudaStream_t s) {
    column_sumsq_kernel<<<nblk, 256, 0, s>>>(X, rows, r, ldf, partb);
    count_launch();
    return cudaGetLastError();
}

__global__ void balance_gains_kernel(const float *__restrict__ pu, const float *__restrict__ pv,
                                     int nblk, int r, float *gk) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= r) return;
    double su = 0.0, sv = 0.0;
    for (int b = 0; b < nblk; ++b) {
        su += pu[(int64_t)b * r + k];
        sv += pv[(int64_t)b * r + k];
    }
    const double nu = sqrt(su), nv = sqrt(sv);
    gk[k] = (nu > 0.0 && nv > 0.0) ? (float)sqrt(nv / nu) : 1.f;
}

cudaError_t balance_gains(const float *partU, const float *partV, int nblk, int32_t r, float *gk,
                          cudaStream_t s) {
    balance_gains_kernel<<<(unsigned)ceil_div(r, 256), 256, 0, s>>>(partU, partV, nblk, r, gk);
    count_launch();
    return cudaGetLastError();
}

// Warp per row: ballot of (x < 0) over 32 consecutive rank columns -> one word.
__global__ void __launch_bounds__(256)
    extract_pack_kernel(const float *__restrict__ X, int64_t rows, int r, int64_t ldf,
                        const float *__restrict__ gk, int invert, const double *gamma,
                        float *s_out, uint32_t *bits, __nv_bfloat16 *pm, int64_t ldpm) {
    const int lane = threadIdx.x & 31;
    const int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (i >= rows) return;
    const int nw = (r + 31) / 32;
    float sum = 0.f;
    for (int w = 0; w < nw; ++w) {
        const int k = 32 * w + lane;
        const bool in = k < r;
        const float x = in ? X[i * ldf + k] : 0.f;
        if (in) {
            const float g = gk ? gk[k] : 1.f;
            sum += fabsf(invert ? x / g : x * g);
        }
        const unsigned word = __ballot_sync(0xffffffffu, in && x < 0.f);
        if (lane == 0 && bits) bits[i * nw + w] = word;
        if (in && pm) pm[i * ldpm + k] = __float2bfloat16_rn(x < 0.f ? -1.f : 1.f);
    }
    sum = warp_sum(sum);
    if (lane == 0 && s_out) s_out[i] = (float)((double)sum / (double)r * (gamma ? *gamma : 1.0));
}

cudaError_t extract_pack(const float *X, int64_t rows, int32_t r, int64_t ldf, const float *gk,
                         int invert, const double *gamma, float *s_out, uint32_t *bits,
                         __nv_bfloat16 *pm, int64_t ldpm, cudaStream_t s) {
    extract_pack_kernel<<<(unsigned)ceil_div(rows * 32, 256), 256, 0, s>>>(
        X, rows, r, ldf, gk, invert, gamma, s_out, bits, pm, ldpm);
    count_launch();
    return cudaGetLastError();
}

cudaError_t pack_signs(const float *X, int64_t rows, int32_t r, int64_t ldx, uint32_t *bits,
                       cudaStream_t s) {
    return extract_pack(X, rows, r, ldx, nullptr, 0, nullptr, nullptr, bits, nullptr, 0, s);
}

__global__ void unpack_pm_kernel(const uint32_t *__restrict__ bits, int64_t rows, int r,
                                 __nv_bfloat16 *pm, int64_t ldpm) {
    const int nw = (r + 31) / 32;
    const int64_t total = rows * (int64_t)r;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / r;
        const int k = (int)(e % r);
        const uint32_t w = bits[i * nw + k / 32];
        pm[i * ldpm + k] = __float2bfloat16_rn(((w >> (k & 31)) & 1u) ? -1.f : 1.f);
    }
}

cudaError_t unpack_pm(const uint32_t *bits, int64_t rows, int32_t r, __nv_bfloat16 *pm,
                      int64_t ldpm, cudaStream_t s) {
    unpack_pm_kernel<<<4 * kNumSMsB200, 256, 0, s>>>(bits, rows, r, pm, ldpm);
    count_launch();
    return cudaGetLastError();
}

__global__ void __launch_bounds__(256)
    recon_finalize_kernel(const double *part, int count, const Scalars *sc, double *out) {
    __shared__ double sh[256];
    double a = 0.0;
    for (int i = threadIdx.x; i < count; i += blockDim.x) a += part[i];
    const double t = block_sum_256(a, sh);
    if (threadIdx.x == 0) {
        const double w2 = sc->wt_norm2;
        *out = w2 > 0.0 ? sqrt(t / w2) : (t == 0.0 ? 0.0 : INFINITY);
    }
}

// Least-squares scale update: s_i = sum_t num[t][i] / sum_t den[t][i] (tiles in order);
// a scale whose denominator vanishes keeps its value.
__global__ void refit_scales_kernel(const double *__restrict__ num, const double *__restrict__ den,
                                    int ntiles, int64_t M, float *s) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < M;
         i += (int64_t)gridDim.x * blockDim.x) {
        double a = 0.0, b = 0.0;
        for (int t = 0; t < ntiles; ++t) {
            a += num[(int64_t)t * M + i];
            b += den[(int64_t)t * M + i];
        }
        if (b > 0.0) s[i] = (float)(a / b);
    }
}

cudaError_t refit_scales(const double *num, const double *den, int ntiles, int64_t M, float *s,
                         cudaStream_t st) {
    refit_scales_kernel<<<(unsigned)ceil_div(M, 256), 256, 0, st>>>(num, den, ntiles, M, s);
    count_launch();
    return cudaGetLastError();
}

cudaError_t recon_finalize(const double *part, int count, const Scalars *sc, double *out,
                           cudaStream_t s) {
    recon_finalize_kernel<<<1, 256, 0, s>>>(part, count, sc, out);
    count_launch();
    return cudaGetLastError();
}

}  // namespace nq
