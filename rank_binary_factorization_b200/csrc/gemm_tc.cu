// tcgen05 / TMEM / TMA GEMM kernel (sm_100a) and its fused LB-ADMM epilogues.
#include <cudaTypedefs.h>

#include "gemm_tc.cuh"

namespace nq {
namespace tc {

// ---------------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// Bounded wait for the completion of the phase with parity ``parity``.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *err) {
    const uint32_t addr = smem_u32(bar);
    for (uint32_t spin = 0; spin < kMbarSpinLimit; ++spin) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(addr), "r"(parity)
            : "memory");
        if (done) return true;
    }
    raise_error(err, NQ_ERR_TIMEOUT);
    return false;
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), version 1 (sm_100), leading offset unused for this layout.
__device__ __forceinline__ uint64_t smem_desc_sw128(const void *tile) {
    const uint64_t addr = smem_u32(tile);
    uint64_t d = 0;
    d |= (addr & 0x3FFFFull) >> 4;          // start address  [0,14)
    d |= (uint64_t)1 << 16;                 // LBO (ignored)  [16,30)
    d |= (uint64_t)(1024 >> 4) << 32;       // SBO            [32,46)
    d |= (uint64_t)1 << 46;                 // version        [46,48)
    d |= (uint64_t)2 << 61;                 // SWIZZLE_128B   [61,64)
    return d;
}

// Instruction descriptor, kind::f16: D=F32, A=B=BF16, both K-major, N>>3, M>>4.
__host__ __device__ constexpr uint32_t instr_desc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Named barrier among the epilogue warps only (barrier 0 is __syncthreads).
__device__ __forceinline__ void epilogue_bar() {
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kEpiWarps) : "memory");
}

// ---------------------------------------------------------------------------------
// Epilogues: thread owns tile row ``row`` and columns col0 .. col0+15.
// ---------------------------------------------------------------------------------
__device__ __forceinline__ float sgn(float x) { return x < 0.f ? -1.f : 1.f; }

__device__ __forceinline__ float load_w(const EpiParams &p, int64_t i, int64_t j) {
    if (p.w_bf16)
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p.W)[i * p.ldw + j]);
    return reinterpret_cast<const float *>(p.W)[i * p.ldw + j];
}

__device__ __forceinline__ void ld16(float (&d)[16], const float *src) {
#pragma unroll
    for (int j = 0; j < 16; j += 4)
        *reinterpret_cast<float4 *>(&d[j]) = *reinterpret_cast<const float4 *>(src + j);
}
__device__ __forceinline__ void st16(float *dst, const float (&v)[16]) {
#pragma unroll
    for (int j = 0; j < 16; j += 4)
        *reinterpret_cast<float4 *>(dst + j) = *reinterpret_cast<const float4 *>(&v[j]);
}
__device__ __forceinline__ void ld16_bf16(float (&d)[16], const __nv_bfloat16 *src) {
    __align__(16) __nv_bfloat16 h[16];
    reinterpret_cast<uint4 *>(h)[0] = reinterpret_cast<const uint4 *>(src)[0];
    reinterpret_cast<uint4 *>(h)[1] = reinterpret_cast<const uint4 *>(src)[1];
#pragma unroll
    for (int j = 0; j < 16; ++j) d[j] = __bfloat162float(h[j]);
}

// Mirrored store of a symmetric result (EPI_SPLIT): entry (row, col0 + j) also goes to
// (col0 + j, row); consecutive lanes hold consecutive rows, so each store is coalesced.
__device__ __forceinline__ void split_mirror(const EpiParams &p, int row, int col0,
                                             const float (&v)[16]) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        if (col0 + j >= p.N) break;
        const __nv_bfloat16 h = __float2bfloat16_rn(v[j]);
        const int64_t o = (int64_t)(col0 + j) * p.ldr + row;
        p.Rhi[o] = h;
        p.Rlo[o] = __float2bfloat16_rn(v[j] - __bfloat162float(h));
    }
}

// Mirrored store of a symmetric Gram tile (EPI_GRAM with sym): entry (row, col0 + j) also
// goes to (col0 + j, row), and to its hi + lo split when Rhi is set.  Off-diagonal tiles
// only, so no ridge term is added here.
__device__ __forceinline__ void gram_mirror(const EpiParams &p, int row, int col0,
                                            const float (&v)[16]) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        if (col0 + j >= p.N) break;
        p.out[(int64_t)(col0 + j) * p.ldo + row] = v[j];
    }
    if (p.Rhi) split_mirror(p, row, col0, v);
}

// Row segment (row, col0 .. col0 + 15) of a split (hi + lo BF16) output; ``full``: all 16
// columns are inside the matrix (then two 32-byte stores per part).
__device__ __forceinline__ void split_store(__nv_bfloat16 *hi, __nv_bfloat16 *lo, bool full,
                                            int ncols, const float (&v)[16]) {
    if (full) {
        __align__(16) __nv_bfloat16 h[16], l[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            h[j] = __float2bfloat16_rn(v[j]);
            l[j] = __float2bfloat16_rn(v[j] - __bfloat162float(h[j]));
        }
        reinterpret_cast<uint4 *>(hi)[0] = reinterpret_cast<uint4 *>(h)[0];
        reinterpret_cast<uint4 *>(hi)[1] = reinterpret_cast<uint4 *>(h)[1];
        reinterpret_cast<uint4 *>(lo)[0] = reinterpret_cast<uint4 *>(l)[0];
        reinterpret_cast<uint4 *>(lo)[1] = reinterpret_cast<uint4 *>(l)[1];
    } else {
        for (int j = 0; j < 16 && j < ncols; ++j) {
            const __nv_bfloat16 h = __float2bfloat16_rn(v[j]);
            hi[j] = h;
            lo[j] = __float2bfloat16_rn(v[j] - __bfloat162float(h));
        }
    }
}

template <int EPI>
__device__ __forceinline__ void epilogue_chunk(const EpiParams &p, int row, int col0,
                                               const float (&v)[16], float &acc_sum,
                                               float &acc_aux, bool fin) {
    const bool full = (col0 + 16 <= p.N);
    if constexpr (EPI == EPI_GRAM) {
        float *o = p.out + (int64_t)row * p.ldo + col0;
        float w[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) w[j] = v[j] + ((row == col0 + j) ? p.diag : 0.f);
        if (full && (p.ldo & 3) == 0) {
            st16(o, w);
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (full || col0 + j < p.N) o[j] = w[j];
        }
        if (p.Rhi) {
            const int64_t so = (int64_t)row * p.ldr + col0;
            split_store(p.Rhi + so, p.Rlo + so, full, p.N - col0, w);
        }
    } else if constexpr (EPI == EPI_NS1) {
        const int64_t so = (int64_t)row * p.ldr + col0;
        float e[16];
        float part = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            e[j] = (row == col0 + j ? 1.f : 0.f) - v[j];
            if (full || col0 + j < p.N) part += e[j] * e[j];
        }
        split_store(p.Rhi + so, p.Rlo + so, full, p.N - col0, e);
        acc_sum += part;
    } else if constexpr (EPI == EPI_GD) {
        const int64_t so = (int64_t)row * p.ldr + col0;
        float *Xrow = p.X + (int64_t)row * p.ldf + col0;
        const float eta = 1.f / *p.gd_max;
        float rh[16], rl[16], x[16];
        bool bad = false;
        if (full) {
            ld16_bf16(rh, p.Ph + so);
            ld16_bf16(rl, p.Pl + so);
            ld16(x, Xrow);
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const bool in = col0 + j < p.N;
                rh[j] = in ? __bfloat162float(p.Ph[so + j]) : 0.f;
                rl[j] = in ? __bfloat162float(p.Pl[so + j]) : 0.f;
                x[j] = in ? Xrow[j] : 0.f;
            }
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            x[j] = x[j] - eta * (v[j] - (rh[j] + rl[j]));
            bad |= !isfinite(x[j]);
        }
        if (full) {
            st16(Xrow, x);
        } else {
            for (int j = 0; j < 16 && col0 + j < p.N; ++j) Xrow[j] = x[j];
        }
        split_store(p.Fhi + so, p.Flo + so, full, p.N - col0, x);
        if (bad) raise_error(p.err, NQ_ERR_NONFINITE);
    } else if constexpr (EPI == EPI_NS2) {
        const int64_t so = (int64_t)row * p.ldr + col0;
        float xh[16], xl[16], xn[16];
        if (full) {
            ld16_bf16(xh, p.Ph + so);
            ld16_bf16(xl, p.Pl + so);
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const bool in = col0 + j < p.N;
                xh[j] = in ? __bfloat162float(p.Ph[so + j]) : 0.f;
                xl[j] = in ? __bfloat162float(p.Pl[so + j]) : 0.f;
            }
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) xn[j] = (xh[j] + xl[j]) + v[j];
        if (fin)
            split_store(p.Fhi + so, p.Flo + so, full, p.N - col0, xn);
        else
            split_store(p.Rhi + so, p.Rlo + so, full, p.N - col0, xn);
    } else if constexpr (EPI == EPI_SCALE) {
        float *o = p.out + (int64_t)row * p.ldo + col0;
        for (int j = 0; j < 16 && col0 + j < p.N; ++j) o[j] = v[j] * p.s1[col0 + j];
    } else if constexpr (EPI == EPI_SPLIT) {
        __nv_bfloat16 *hi = p.Rhi + (int64_t)row * p.ldr + col0;
        __nv_bfloat16 *lo = p.Rlo + (int64_t)row * p.ldr + col0;
        if (full) {
            __align__(16) __nv_bfloat16 h[16], l[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                h[j] = __float2bfloat16_rn(v[j]);
                l[j] = __float2bfloat16_rn(v[j] - __bfloat162float(h[j]));
            }
            reinterpret_cast<uint4 *>(hi)[0] = reinterpret_cast<uint4 *>(h)[0];
            reinterpret_cast<uint4 *>(hi)[1] = reinterpret_cast<uint4 *>(h)[1];
            reinterpret_cast<uint4 *>(lo)[0] = reinterpret_cast<uint4 *>(l)[0];
            reinterpret_cast<uint4 *>(lo)[1] = reinterpret_cast<uint4 *>(l)[1];
        } else {
            for (int j = 0; j < 16 && col0 + j < p.N; ++j) {
                const __nv_bfloat16 h = __float2bfloat16_rn(v[j]);
                hi[j] = h;
                lo[j] = __float2bfloat16_rn(v[j] - __bfloat162float(h));
            }
        }
    } else if constexpr (EPI == EPI_RHS) {
        const float ai = p.a[row];
        const float *Srow = p.S + (int64_t)row * p.ldf + col0;
        __nv_bfloat16 *hi = p.Rhi + (int64_t)row * p.ldr + col0;
        __nv_bfloat16 *lo = p.Rlo + (int64_t)row * p.ldr + col0;
        if (full) {
            float s[16], bb[16];
            ld16(s, Srow);
            ld16(bb, p.b + col0);
            __align__(16) __nv_bfloat16 h[16], l[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float z = sgn(s[j]) * ai * bb[j];
                const float r = v[j] + p.rho * (2.f * z - s[j]);
                h[j] = __float2bfloat16_rn(r);
                l[j] = __float2bfloat16_rn(r - __bfloat162float(h[j]));
            }
            reinterpret_cast<uint4 *>(hi)[0] = reinterpret_cast<uint4 *>(h)[0];
            reinterpret_cast<uint4 *>(hi)[1] = reinterpret_cast<uint4 *>(h)[1];
            reinterpret_cast<uint4 *>(lo)[0] = reinterpret_cast<uint4 *>(l)[0];
            reinterpret_cast<uint4 *>(lo)[1] = reinterpret_cast<uint4 *>(l)[1];
        } else {
            for (int j = 0; j < 16 && col0 + j < p.N; ++j) {
                const float sj = Srow[j];
                const float z = sgn(sj) * ai * p.b[col0 + j];
                const float r = v[j] + p.rho * (2.f * z - sj);
                const __nv_bfloat16 h = __float2bfloat16_rn(r);
                hi[j] = h;
                lo[j] = __float2bfloat16_rn(r - __bfloat162float(h));
            }
        }
    } else if constexpr (EPI == EPI_SOLVE) {
        const float ai = p.a[row];
        float *Srow = p.S + (int64_t)row * p.ldf + col0;
        float *Xrow = p.X + (int64_t)row * p.ldf + col0;
        bool bad = false;
        float part = 0.f;
        if (full) {
            float so[16], bb[16], sn[16], rr[16];
            ld16(so, Srow);
            ld16(bb, p.b + col0);
            if (p.objective) {
                float lo_[16];
                const int64_t o = (int64_t)row * p.ldr + col0;
                ld16_bf16(rr, p.Rhi + o);
                ld16_bf16(lo_, p.Rlo + o);
#pragma unroll
                for (int j = 0; j < 16; ++j) rr[j] += lo_[j];
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float x = v[j];
                bad |= !isfinite(x);
                const float z = sgn(so[j]) * ai * bb[j];
                sn[j] = x + so[j] - z;
                // the latent as the next contractions see it: bf16(x) (+ its low part)
                const __nv_bfloat16 h = __float2bfloat16_rn(x);
                float xo = __bfloat162float(h);
                p.Xt[(int64_t)(col0 + j) * p.ldxt + row] = h;
                if (p.XtL) {
                    const __nv_bfloat16 l = __float2bfloat16_rn(x - xo);
                    p.XtL[(int64_t)(col0 + j) * p.ldxt + row] = l;
                    xo += __bfloat162float(l);
                }
                if (p.objective) part += (rr[j] - p.rho * (2.f * z - so[j])) * xo;
            }
            st16(Xrow, v);
            st16(Srow, sn);
        } else {
            for (int j = 0; j < 16 && col0 + j < p.N; ++j) {
                const float x = v[j];
                bad |= !isfinite(x);
                const float sold = Srow[j];
                const float z = sgn(sold) * ai * p.b[col0 + j];
                Xrow[j] = x;
                Srow[j] = x + sold - z;
                const __nv_bfloat16 h = __float2bfloat16_rn(x);
                float xo = __bfloat162float(h);
                p.Xt[(int64_t)(col0 + j) * p.ldxt + row] = h;
                if (p.XtL) {
                    const __nv_bfloat16 l = __float2bfloat16_rn(x - xo);
                    p.XtL[(int64_t)(col0 + j) * p.ldxt + row] = l;
                    xo += __bfloat162float(l);
                }
                if (p.objective) {
                    const int64_t o = (int64_t)row * p.ldr + col0 + j;
                    const float r = __bfloat162float(p.Rhi[o]) + __bfloat162float(p.Rlo[o]);
                    part += (r - p.rho * (2.f * z - sold)) * xo;
                }
            }
        }
        if (bad) raise_error(p.err, NQ_ERR_NONFINITE);
        acc_sum += part;
    } else if constexpr (EPI == EPI_REFIT) {
        float pn = 0.f, pd = 0.f;
        const float *dcol = p.refit_trans ? p.d_out : p.d_in;
        const float *drow = p.refit_trans ? p.d_in : p.d_out;
        const float dr = drow ? drow[row] : 1.f;
        float dc[16], sv[16], w[16];
        const bool cv = full && p.cvec;
        if (cv) {
            if (dcol) ld16(dc, dcol + col0);
            ld16(sv, p.sv + col0);
        }
        if (full && !p.refit_trans && p.w_vec) {
            if (p.w_bf16)
                ld16_bf16(w, reinterpret_cast<const __nv_bfloat16 *>(p.W) + (int64_t)row * p.ldw + col0);
            else
                ld16(w, reinterpret_cast<const float *>(p.W) + (int64_t)row * p.ldw + col0);
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int c = col0 + j;
                w[j] = (full || c < p.N) ? (p.refit_trans ? load_w(p, c, row) : load_w(p, row, c)) : 0.f;
            }
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int c = col0 + j;
            if (!(full || c < p.N)) continue;
            const float dcj = cv ? (dcol ? dc[j] : 1.f) : (dcol ? dcol[c] : 1.f);
            const float svj = cv ? sv[j] : p.sv[c];
            const float sc = svj * v[j];
            pn = fmaf(dr * dcj * w[j], sc, pn);
            pd = fmaf(sc, sc, pd);
        }
        acc_sum += pn;
        acc_aux += pd;
    } else if constexpr (EPI == EPI_RECON) {
        const float dro = p.d_out ? p.d_out[row] : 1.f;
        const float s1 = p.s1[row];
        float w[16];
        if (full && p.w_vec) {
            if (p.w_bf16)
                ld16_bf16(w, reinterpret_cast<const __nv_bfloat16 *>(p.W) + (int64_t)row * p.ldw + col0);
            else
                ld16(w, reinterpret_cast<const float *>(p.W) + (int64_t)row * p.ldw + col0);
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) w[j] = (full || col0 + j < p.N) ? load_w(p, row, col0 + j) : 0.f;
        }
        float part = 0.f;
        float di[16], s2v[16];
        const bool cv = full && p.cvec;
        if (cv) {
            if (p.d_in) ld16(di, p.d_in + col0);
            ld16(s2v, p.s2 + col0);
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int c = col0 + j;
            if (!(full || c < p.N)) continue;
            const float dij = cv ? (p.d_in ? di[j] : 1.f) : (p.d_in ? p.d_in[c] : 1.f);
            const float s2j = cv ? s2v[j] : p.s2[c];
            const float wt = dro * w[j] * dij;
            const float d = wt - s1 * v[j] * s2j;
            part += d * d;
        }
        acc_sum += part;
    }
}

// Newton-Schulz bookkeeping, run by one epilogue warp per finished tile.  NS1: the tile's
// sum of squared residual entries goes to part[tile]; the warp that finishes the last tile
// of the launch (ticket) sums the partials in a fixed order and moves the gate.  NS2: the
// last tile closes an accepted update.
template <int EPI>
__device__ __forceinline__ void ns_tile_done(const EpiParams &p, int tile, int num_tiles,
                                             int lane, const double *red, bool fin) {
    NsState *ns = p.ns;
    unsigned last = 0;
    if (lane == 0) {
        if constexpr (EPI == EPI_NS1) {
            double t = 0.0;
            for (int e = 0; e < kEpiWarps; ++e) t += red[e];
            p.part[tile] = t;
        }
        __threadfence();
        last = atomicAdd(&ns->ticket, 1u) == (unsigned)(num_tiles - 1) ? 1u : 0u;
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) return;
    __threadfence();
    if constexpr (EPI == EPI_NS1) {
        double t = 0.0;
        for (int i = lane; i < num_tiles; i += 32) t += __ldcg(p.part + i);
        t = warp_sum(t);
        if (lane == 0) {
            const int k = p.ns_step;
            const double ef = t >= 0.0 ? sqrt(t) : -1.0;   // a timed-out tile left NaN/-1
            ns->ef[k] = ef;
            // the first split step (k == ns_min_final) starts from an iterate at the BF16
            // steps' rounding floor, so its residual is not compared with theirs; within
            // the BF16 steps only growth is a failure (a floor may already be reached)
            const double prev = k > 0 ? ns->ef[k - 1] : 0.0;
            int g = NS_RUNNING;
            if (!(ef >= 0.0 && ef < 1e30))
                g = NS_FAIL;
            else if (k >= p.ns_min_final && ef <= (double)p.ns_tau)
                g = NS_FINAL;
            else if (k >= p.ns_last || (k > p.ns_min_final && ef > 0.9 * prev) ||
                     (k > 0 && k < p.ns_min_final && ef > 1.5 * prev))
                g = NS_FAIL;
            if (g == NS_FAIL) ns->fallbacks += 1;
            ns->ticket = 0;
            __threadfence();
            *reinterpret_cast<volatile int *>(&ns->gate) = g;
        }
    } else {
        if (lane == 0) {
            if (fin) {
                ns->accepted += 1;
                ns->steps = p.ns_step + 1;
            }
            ns->ticket = 0;
            __threadfence();
            if (fin) *reinterpret_cast<volatile int *>(&ns->gate) = NS_DONE;
        }
    }
}

// Output tile -> (m0, n0).  Plain: m fastest (consecutive CTAs share the B tile), or n
// fastest with nfast (they share the A tile: A is the large operand, read from HBM once
// while its row block's few column tiles run at the same time).  Symmetric (BN == BM):
// the lower-triangular tiles (tm >= tn) row by row, so tiles come in order of decreasing
// K range under tri_k.
template <int BN>
__device__ __forceinline__ void tile_origin(const EpiParams &p, int tile, int num_m, int &m0,
                                            int &n0) {
    if (p.sym) {
        int a = (int)((sqrtf(8.f * (float)tile + 1.f) - 1.f) * 0.5f);
        while ((a + 1) * (a + 2) / 2 <= tile) ++a;
        while (a * (a + 1) / 2 > tile) --a;
        m0 = a * BM;
        n0 = (tile - a * (a + 1) / 2) * BN;
    } else if (p.nfast) {
        const int num_n = (p.N + BN - 1) / BN;
        m0 = (tile / num_n) * BM;
        n0 = (tile % num_n) * BN;
    } else {
        m0 = (tile % num_m) * BM;
        n0 = (tile / num_m) * BN;
    }
}

// ---------------------------------------------------------------------------------
// The kernel: persistent, one CTA per SM, tiles assigned round-robin (m fastest, so
// consecutive CTAs share the B tile).  Two TMEM accumulator stages let the epilogue
// of one tile run while the MMAs of the next are issued.
// ---------------------------------------------------------------------------------
template <int BN, int STAGES, int EPI, bool F3>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ Maps maps, const EpiParams p) {
    constexpr int B_TILE_BYTES = BN * BK * 2;
    // F3 (split3): a stage holds A_hi, A_lo, B_hi, B_lo of one k-block and takes the three
    // products hi.hi, lo.hi, hi.lo; otherwise one A and one B tile of one segment
    constexpr int STAGE_BYTES = (F3 ? 2 : 1) * (A_TILE_BYTES + B_TILE_BYTES);
    constexpr uint32_t TMEM_COLS = 2 * BN;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
    uint64_t *empty_bar = full_bar + STAGES;
    uint64_t *tfull = empty_bar + STAGES;
    uint64_t *tempty = tfull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
    __shared__ double red[2][kEpiWarps];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_m = (int)ceil_div(p.M, BM);
    const int num_tiles = p.sym ? num_m * (num_m + 1) / 2 : num_m * (int)ceil_div(p.N, BN);
    const int total_kb = F3 ? p.kblocks[0]
                            : p.kblocks[0] + (p.nseg > 1 ? p.kblocks[1] : 0) +
                                  (p.nseg > 2 ? p.kblocks[2] : 0);
    // split-K: work unit u = (split u / num_tiles, tile u % num_tiles); split s covers the
    // k-blocks [s * kchunk, (s + 1) * kchunk) of the concatenated segments
    const int ksplit = p.ksplit > 1 ? p.ksplit : 1;
    const int num_units = num_tiles * ksplit;
    const int kchunk = (total_kb + ksplit - 1) / ksplit;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&tfull[s], 1);
            mbar_init(&tempty[s], kEpiWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        const int nmaps = F3 ? 2 : p.nseg;
        for (int g = 0; g < nmaps; ++g) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.a[g])) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.b[g])) : "memory");
        }
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // launched with programmatic stream serialization: the set-up above touches no global
    // memory; everything below may read what the previous kernel of the stream wrote, so
    // wait for its completion first, then let the next kernel's launch begin (it waits the
    // same way).  No other GEMM CTA can share this SM (shared memory), so the TMEM
    // allocation above does not wait on the previous kernel.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // gate: the whole launch is skipped on the gate values in gate_skip
    int gate_v = 0;
    bool skip = false;
    if (p.gate) {
        gate_v = *reinterpret_cast<const volatile int *>(p.gate);
        skip = (unsigned)gate_v < 32u && ((p.gate_skip >> gate_v) & 1);
    }
    const bool fin = (EPI == EPI_NS2) && gate_v == NS_FINAL;
    if (EPI == EPI_GRAM && p.ns && blockIdx.x == 0 && threadIdx.x == 0) {
        p.ns->ticket = 0;
        p.ns->grid_count = 0;
        *reinterpret_cast<volatile int *>(&p.ns->gate) = NS_RUNNING;
    }
    if (EPI == EPI_GRAM && p.zero)   // counters of a later kernel, zeroed here
        for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < p.zero_words;
             i += gridDim.x * blockDim.x)
            p.zero[i] = 0u;

    if (!skip) {

        if (warp == 0) {
            if (lane == 0) {
                // TMA producer
                uint32_t it = 0;
                bool ok = true;
                for (int unit = blockIdx.x; unit < num_units && ok; unit += gridDim.x) {
                    const int tile = unit % num_tiles, ks = unit / num_tiles;
                    const int kb0 = ks * kchunk, kb1 = min(total_kb, kb0 + kchunk);
                    int m0, n0;
                    tile_origin<BN>(p, tile, num_m, m0, n0);
                    for (int kb = kb0; kb < kb1; ++kb) {
                        int seg = 0, k = kb;
                        if (!F3)
                            while (seg < p.nseg - 1 && k >= p.kblocks[seg]) k -= p.kblocks[seg++];
                        if (p.tri_k && k < (m0 > n0 ? m0 : n0) / BK) continue;
                        const int s = it % STAGES;
                        if (it >= STAGES &&
                            !mbar_wait(&empty_bar[s], ((it / STAGES) - 1) & 1, p.err)) {
                            ok = false;
                            break;
                        }
                        uint8_t *a_dst = smem + s * STAGE_BYTES;
                        mbar_expect_tx(&full_bar[s], STAGE_BYTES);
                        if constexpr (F3) {
                            uint8_t *b_dst = a_dst + 2 * A_TILE_BYTES;
                            tma_load_2d(a_dst, &maps.a[0], k * BK, m0, &full_bar[s]);
                            tma_load_2d(a_dst + A_TILE_BYTES, &maps.a[1], k * BK, m0, &full_bar[s]);
                            tma_load_2d(b_dst, &maps.b[0], k * BK, n0, &full_bar[s]);
                            tma_load_2d(b_dst + B_TILE_BYTES, &maps.b[1], k * BK, n0, &full_bar[s]);
                        } else {
                            tma_load_2d(a_dst, &maps.a[seg], k * BK, m0, &full_bar[s]);
                            tma_load_2d(a_dst + A_TILE_BYTES, &maps.b[seg], k * BK, n0,
                                        &full_bar[s]);
                        }
                        ++it;
                    }
                }
            }
        } else if (warp == 1) {
            if (lane == 0) {
                // MMA issuer
                constexpr uint32_t idesc = instr_desc_bf16(BM, BN);
                uint32_t it = 0;
                bool ok = true;
                int lt = 0;
                for (int unit = blockIdx.x; unit < num_units && ok; unit += gridDim.x, ++lt) {
                    const int tile = unit % num_tiles, ks = unit / num_tiles;
                    const int kb0 = ks * kchunk, kb1 = min(total_kb, kb0 + kchunk);
                    const int as = lt & 1;
                    int m0, n0;
                    tile_origin<BN>(p, tile, num_m, m0, n0);
                    if (lt >= 2 && !mbar_wait(&tempty[as], ((lt >> 1) - 1) & 1, p.err)) break;
                    tc_fence_after();
                    const uint32_t d = tmem + (uint32_t)(as * BN);
                    bool first = true;
                    for (int kb = kb0; kb < kb1; ++kb) {
                        if (p.tri_k) {
                            int seg = 0, k = kb;
                            if (!F3)
                                while (seg < p.nseg - 1 && k >= p.kblocks[seg])
                                    k -= p.kblocks[seg++];
                            if (k < (m0 > n0 ? m0 : n0) / BK) continue;
                        }
                        const int s = it % STAGES;
                        if (!mbar_wait(&full_bar[s], (it / STAGES) & 1, p.err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint8_t *a_src = smem + s * STAGE_BYTES;
                        if constexpr (F3) {
                            const uint64_t ah = smem_desc_sw128(a_src);
                            const uint64_t al = smem_desc_sw128(a_src + A_TILE_BYTES);
                            const uint64_t bh = smem_desc_sw128(a_src + 2 * A_TILE_BYTES);
                            const uint64_t bl = smem_desc_sw128(a_src + 2 * A_TILE_BYTES + B_TILE_BYTES);
    #pragma unroll
                            for (int k = 0; k < BK / 16; ++k)
                                mma_bf16(d, ah + 2 * k, bh + 2 * k, idesc, (first && k == 0) ? 0u : 1u);
    #pragma unroll
                            for (int k = 0; k < BK / 16; ++k) mma_bf16(d, al + 2 * k, bh + 2 * k, idesc, 1u);
    #pragma unroll
                            for (int k = 0; k < BK / 16; ++k) mma_bf16(d, ah + 2 * k, bl + 2 * k, idesc, 1u);
                        } else {
                            const uint64_t adesc = smem_desc_sw128(a_src);
                            const uint64_t bdesc = smem_desc_sw128(a_src + A_TILE_BYTES);
    #pragma unroll
                            for (int k = 0; k < BK / 16; ++k)
                                mma_bf16(d, adesc + 2 * k, bdesc + 2 * k, idesc,
                                         (first && k == 0) ? 0u : 1u);
                        }
                        mma_commit(&empty_bar[s]);
                        first = false;
                        ++it;
                    }
                    if (ok) mma_commit(&tfull[as]);
                }
            }
        } else {
            // epilogue warps.  Every epilogue warp walks the same tiles and reaches the same
            // named barriers, also after a timed-out wait (then it only skips the work).
            const int q = warp & 3;
            int lt = 0;
            bool dead = false;
            for (int unit = blockIdx.x; unit < num_units; unit += gridDim.x, ++lt) {
                const int tile = unit % num_tiles;
                const int as = lt & 1;
                int m0, n0;
                tile_origin<BN>(p, tile, num_m, m0, n0);
                const int row = m0 + 32 * q + lane;
                float acc_sum = 0.f, acc_aux = 0.f;
                if (!dead) {
                    // one lane waits; the outcome is broadcast so that the warp-collective
                    // tcgen05.ld below is executed by all 32 lanes or by none
                    int ok = 0;
                    if (lane == 0) ok = mbar_wait(&tfull[as], (lt >> 1) & 1, p.err) ? 1 : 0;
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    dead = !ok;
                }
                if (!dead) {
                    tc_fence_after();
                    const uint32_t tbase = tmem + (uint32_t)(as * BN) + ((uint32_t)(32 * q) << 16);
    #pragma unroll 1
                    for (int c = 0; c < BN; c += 16) {
                        float v[16];
                        tmem_ld16(tbase + c, v);  // warp-collective: every lane takes part
                        if (EPI == EPI_GRAM && ksplit > 1) {
                            // split-K partial: the unit's raw 128 x 128 tile, reduced later
                            st16(p.out + ((int64_t)unit * BM + 32 * q + lane) * BM + c, v);
                        } else if (row < p.M && n0 + c < p.N) {
                            epilogue_chunk<EPI>(p, row, n0 + c, v, acc_sum, acc_aux, fin);
                            if constexpr (EPI == EPI_SPLIT)
                                if (p.sym && m0 != n0) split_mirror(p, row, n0 + c, v);
                            if constexpr (EPI == EPI_GRAM)
                                if (p.sym && m0 != n0) gram_mirror(p, row, n0 + c, v);
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[as]);
                }
                if constexpr (EPI == EPI_REFIT) {
                    // one thread owns (row, this tile's columns): its sums are the partials
                    if (!dead && row < p.M) {
                        const int64_t o = (int64_t)(n0 / BN) * p.M + row;
                        p.num[o] = (double)acc_sum;
                        p.den[o] = (double)acc_aux;
                    }
                }
                if constexpr (EPI == EPI_NS1 || EPI == EPI_NS2) {
                    if constexpr (EPI == EPI_NS1) {
                        const double w = warp_sum((double)acc_sum);
                        if (lane == 0) red[as][warp - 2] = dead ? __longlong_as_double(-1ll) : w;
                        epilogue_bar();
                    }
                    if (warp == 2) ns_tile_done<EPI>(p, tile, num_tiles, lane, red[as], fin);
                }
                if constexpr (EPI == EPI_SOLVE || EPI == EPI_RECON) {
                    if (p.part && (EPI == EPI_RECON || p.objective)) {
                        const double w = warp_sum((double)acc_sum);
                        if (lane == 0) red[as][warp - 2] = w;
                        epilogue_bar();
                        if (warp == 2 && lane == 0) {
                            double t = 0.0;
                            for (int e = 0; e < kEpiWarps; ++e) t += red[as][e];
                            p.part[tile] = t;
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------------
// Newton-Schulz update of G^-1 in one cooperative launch.  Phases 2k and 2k+1 are the two
// GEMMs of step k (E_k = I - X_k G; X_{k+1} = X_k + E_k X_k) on 128 x 128 tiles; between
// phases every CTA's epilogue stores are made visible (proxy fence, release) and the next
// phase's loads wait on a grid-wide arrival count (bounded).  The gate decides at each
// phase start, read once per CTA after the barrier: an E phase runs while the gate is
// RUNNING; an X phase runs while RUNNING, and writes the final iterate to X buffer 0 when
// it is FINAL.  The operand pipeline, the TMEM stages and their barriers carry across
// phases; each stage holds four tiles (split phases use all four, BF16 phases two).
// ---------------------------------------------------------------------------------
constexpr int kNsBN = 128;
constexpr int kNsStages = 3;

__device__ __forceinline__ void ns_decide(const NsArgs &a, int k, int lane, int num_tiles) {
    // called by the warp that finished the last E tile of phase 2k
    NsState *ns = a.ns;
    double t = 0.0;
    for (int i = lane; i < num_tiles; i += 32) t += __ldcg(a.part + i);
    t = warp_sum(t);
    if (lane == 0) {
        const double ef = t >= 0.0 ? sqrt(t) : -1.0;
        ns->ef[k] = ef;
        const double prev = k > 0 ? ns->ef[k - 1] : 0.0;
        int g = NS_RUNNING;
        if (!(ef >= 0.0 && ef < 1e30))
            g = NS_FAIL;
        else if (k >= a.bf16_steps && ef <= (double)a.tau)
            g = NS_FINAL;
        else if (k >= a.nsteps - 1 || (k > a.bf16_steps && ef > 0.9 * prev) ||
                 (k > 0 && k < a.bf16_steps && ef > 1.5 * prev))
            g = NS_FAIL;
        if (g == NS_FAIL) ns->fallbacks += 1;
        if (g == NS_FINAL) ns->steps = k + 1;
        ns->ticket = 0;
        __threadfence();
        *reinterpret_cast<volatile int *>(&ns->gate) = g;
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    newton_kernel(const __grid_constant__ NsMaps maps, const NsArgs a) {
    constexpr int BN = kNsBN, STAGES = kNsStages;
    constexpr int B_TILE_BYTES = BN * BK * 2;
    constexpr int STAGE_BYTES = 2 * (A_TILE_BYTES + B_TILE_BYTES);
    constexpr uint32_t TMEM_COLS = 2 * BN;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
    uint64_t *empty_bar = full_bar + STAGES;
    uint64_t *tfull = empty_bar + STAGES;
    uint64_t *tempty = tfull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
    __shared__ double red[2][kEpiWarps];
    __shared__ int s_gate;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_m = (int)ceil_div(a.r, BM);
    const int num_tiles = num_m * (int)ceil_div(a.r, BN);
    const int kbs = (int)ceil_div(a.r, BK);
    const unsigned G = gridDim.x;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&tfull[s], 1);
            mbar_init(&tempty[s], kEpiWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    uint32_t it = 0;       // operand stages issued (producer) / consumed (MMA)
    int lt = 0;            // tiles through the accumulator stages (MMA and epilogue)
    bool ok = true;        // this thread's waits all completed
    const int nphases = 2 * a.nsteps;
    for (int ph = 0; ph < nphases; ++ph) {
        __syncthreads();
        if (threadIdx.x == 0) {
            // (after a wait ran out anywhere, later barriers are not waited for)
            if (ph > 0 && *reinterpret_cast<volatile int *>(a.err) != NQ_ERR_TIMEOUT &&
                !wait_geq(&a.ns->grid_count, (unsigned)ph * G, kGridSpinLimit))
                raise_error(a.err, NQ_ERR_TIMEOUT);
            asm volatile("fence.proxy.async.global;" ::: "memory");
            int g = *reinterpret_cast<volatile int *>(&a.ns->gate);
            if (blockIdx.x == 0 && (ph & 1) == 0 && g == NS_FINAL) {
                // the previous step's X phase wrote the final iterate: close the update
                a.ns->accepted += 1;
                *reinterpret_cast<volatile int *>(&a.ns->gate) = NS_DONE;
            }
            s_gate = g;
        }
        __syncthreads();
        const int k = ph >> 1;
        const bool eph = (ph & 1) == 0;   // E phase (else X phase)
        const int g = s_gate;
        const bool run = eph ? g == NS_RUNNING : (g == NS_RUNNING || g == NS_FINAL);
        const bool fin = !eph && g == NS_FINAL;
        const bool split = eph && k >= a.bf16_steps;
        const int xi = k == 0 ? 0 : 1 + (k & 1);         // X_k
        const int di = 1 + ((k + 1) & 1);                  // X_{k+1} when not final
        // producer and MMA issuer stop after a wait that ran out; the epilogue warps walk
        // every tile of a phase that runs (they meet at named barriers per tile)
        if (run) {
            if (warp == 0) {
                if (lane == 0 && ok) {
                    const CUtensorMap *ma = eph ? &maps.xh[xi] : &maps.eh;
                    const CUtensorMap *mal = &maps.xl[xi];
                    const CUtensorMap *mb = eph ? &maps.gh : &maps.xh[xi];
                    const CUtensorMap *mbl = &maps.gl;
                    const uint32_t bytes = split ? STAGE_BYTES : A_TILE_BYTES + B_TILE_BYTES;
                    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += G) {
                        const int m0 = (tile % num_m) * BM, n0 = (tile / num_m) * BN;
                        for (int kb = 0; kb < kbs; ++kb) {
                            const int s = it % STAGES;
                            if (it >= STAGES &&
                                !mbar_wait(&empty_bar[s], ((it / STAGES) - 1) & 1, a.err)) {
                                ok = false;
                                break;
                            }
                            uint8_t *a_dst = smem + s * STAGE_BYTES;
                            uint8_t *b_dst = a_dst + 2 * A_TILE_BYTES;
                            mbar_expect_tx(&full_bar[s], bytes);
                            tma_load_2d(a_dst, ma, kb * BK, m0, &full_bar[s]);
                            tma_load_2d(b_dst, mb, kb * BK, n0, &full_bar[s]);
                            if (split) {
                                tma_load_2d(a_dst + A_TILE_BYTES, mal, kb * BK, m0, &full_bar[s]);
                                tma_load_2d(b_dst + B_TILE_BYTES, mbl, kb * BK, n0, &full_bar[s]);
                            }
                            ++it;
                        }
                    }
                }
            } else if (warp == 1) {
                if (lane == 0 && ok) {
                    constexpr uint32_t idesc = instr_desc_bf16(BM, BN);
                    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += G, ++lt) {
                        const int as = lt & 1;
                        if (lt >= 2 && !mbar_wait(&tempty[as], ((lt >> 1) - 1) & 1, a.err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d = tmem + (uint32_t)(as * BN);
                        for (int kb = 0; kb < kbs; ++kb) {
                            const int s = it % STAGES;
                            if (!mbar_wait(&full_bar[s], (it / STAGES) & 1, a.err)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            const uint8_t *src = smem + s * STAGE_BYTES;
                            const uint64_t ah = smem_desc_sw128(src);
                            const uint64_t bh = smem_desc_sw128(src + 2 * A_TILE_BYTES);
#pragma unroll
                            for (int q = 0; q < BK / 16; ++q)
                                mma_bf16(d, ah + 2 * q, bh + 2 * q, idesc, (kb == 0 && q == 0) ? 0u : 1u);
                            if (split) {
                                const uint64_t al = smem_desc_sw128(src + A_TILE_BYTES);
                                const uint64_t bl = smem_desc_sw128(src + 2 * A_TILE_BYTES + B_TILE_BYTES);
#pragma unroll
                                for (int q = 0; q < BK / 16; ++q) mma_bf16(d, al + 2 * q, bh + 2 * q, idesc, 1u);
#pragma unroll
                                for (int q = 0; q < BK / 16; ++q) mma_bf16(d, ah + 2 * q, bl + 2 * q, idesc, 1u);
                            }
                            mma_commit(&empty_bar[s]);
                            ++it;
                        }
                        if (ok) mma_commit(&tfull[as]);
                    }
                }
            } else {
                const int qw = warp & 3;
                __nv_bfloat16 *dh = fin ? a.xh[0] : a.xh[di];
                __nv_bfloat16 *dl = fin ? a.xl[0] : a.xl[di];
                const __nv_bfloat16 *ph_ = a.xh[xi], *pl_ = a.xl[xi];
                for (int tile = blockIdx.x; tile < num_tiles; tile += G, ++lt) {
                    const int as = lt & 1;
                    const int m0 = (tile % num_m) * BM, n0 = (tile / num_m) * BN;
                    const int row = m0 + 32 * qw + lane;
                    float acc_sum = 0.f;
                    if (ok) {
                        int w = 0;
                        if (lane == 0) w = mbar_wait(&tfull[as], (lt >> 1) & 1, a.err) ? 1 : 0;
                        w = __shfl_sync(0xffffffffu, w, 0);
                        ok = w != 0;
                    }
                    if (ok) {
                        tc_fence_after();
                        const uint32_t tbase = tmem + (uint32_t)(as * BN) + ((uint32_t)(32 * qw) << 16);
#pragma unroll 1
                        for (int c = 0; c < BN; c += 16) {
                            float v[16];
                            tmem_ld16(tbase + c, v);
                            const int col0 = n0 + c;
                            if (row < a.r && col0 < a.r) {
                                const bool full = col0 + 16 <= a.r;
                                const int64_t so = (int64_t)row * a.ldr + col0;
                                float o[16];
                                if (eph) {
#pragma unroll
                                    for (int j = 0; j < 16; ++j) {
                                        o[j] = (row == col0 + j ? 1.f : 0.f) - v[j];
                                        if (full || col0 + j < a.r) acc_sum += o[j] * o[j];
                                    }
                                    split_store(a.eh + so, a.el + so, full, a.r - col0, o);
                                } else {
                                    float xh[16], xl[16];
                                    if (full) {
                                        ld16_bf16(xh, ph_ + so);
                                        ld16_bf16(xl, pl_ + so);
                                    } else {
#pragma unroll
                                        for (int j = 0; j < 16; ++j) {
                                            const bool in = col0 + j < a.r;
                                            xh[j] = in ? __bfloat162float(ph_[so + j]) : 0.f;
                                            xl[j] = in ? __bfloat162float(pl_[so + j]) : 0.f;
                                        }
                                    }
#pragma unroll
                                    for (int j = 0; j < 16; ++j) o[j] = (xh[j] + xl[j]) + v[j];
                                    split_store(dh + so, dl + so, full, a.r - col0, o);
                                }
                            }
                        }
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&tempty[as]);
                    }
                    if (eph) {
                        // the tile's sum of E^2; the warp finishing the last tile decides
                        const double wsum = warp_sum((double)acc_sum);
                        if (lane == 0) red[as][warp - 2] = ok ? wsum : __longlong_as_double(-1ll);
                        epilogue_bar();
                        if (warp == 2) {
                            unsigned last = 0;
                            if (lane == 0) {
                                double t = 0.0;
                                for (int e = 0; e < kEpiWarps; ++e) t += red[as][e];
                                a.part[tile] = t;
                                __threadfence();
                                last = atomicAdd(&a.ns->ticket, 1u) == (unsigned)(num_tiles - 1) ? 1u : 0u;
                            }
                            last = __shfl_sync(0xffffffffu, last, 0);
                            if (last) {
                                __threadfence();
                                ns_decide(a, k, lane, num_tiles);
                            }
                        }
                    }
                }
            }
        }
        // arrival: this CTA's outputs of the phase are written (every phase, run or not)
        if (warp >= 2) {
            asm volatile("fence.proxy.async.global;" ::: "memory");
            epilogue_bar();
            if (warp == 2 && lane == 0) {
                __threadfence();
                atomicAdd(&a.ns->grid_count, 1u);
            }
        }
    }
    __syncthreads();
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        // an update accepted in the last step: close it once every CTA has arrived
        if (*reinterpret_cast<volatile int *>(a.err) != NQ_ERR_TIMEOUT &&
            !wait_geq(&a.ns->grid_count, (unsigned)nphases * G, kGridSpinLimit))
            raise_error(a.err, NQ_ERR_TIMEOUT);
        if (*reinterpret_cast<volatile int *>(&a.ns->gate) == NS_FINAL) {
            a.ns->accepted += 1;
            *reinterpret_cast<volatile int *>(&a.ns->gate) = NS_DONE;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

bool make_map_bf16(CUtensorMap *map, const void *base, int64_t rows, int64_t cols, int64_t ld,
                   int box_rows) {
    auto encode = get_encode();
    if (!encode) return false;
    if ((reinterpret_cast<uintptr_t>(base) & 15) || (ld * 2) % 16) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int BN, int STAGES, int EPI, bool F3>
static cudaError_t launch_t(const Maps &maps, const EpiParams &p, cudaStream_t s) {
    constexpr int smem = STAGES * (F3 ? 2 : 1) * (A_TILE_BYTES + BN * BK * 2) + 1024 + 256;
    static_assert(smem <= 227 * 1024, "shared memory of a GEMM stage ring");
    auto kern = gemm_kernel<BN, STAGES, EPI, F3>;
    static std::atomic<uint64_t> configured{0};   // devices whose smem limit is set
    cudaError_t e = ensure_smem_limit((const void *)kern, smem, configured);
    if (e != cudaSuccess) return e;
    int sms = device_sm_count();
    if (p.max_ctas > 0 && p.max_ctas < sms) sms = p.max_ctas;
    const int64_t tiles = (p.sym ? ceil_div(p.M, BM) * (ceil_div(p.M, BM) + 1) / 2
                                 : num_tiles(p.M, p.N, BN)) *
                          (p.ksplit > 1 ? p.ksplit : 1);
    const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
    // programmatic dependent launch: the launch overlaps the tail of the previous kernel
    // of the stream; the kernel waits for that kernel's completion before any memory access
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    count_launch();
    return cudaLaunchKernelEx(&cfg, kern, maps, p);
}

template <int EPI>
static cudaError_t launch_bn(const Maps &maps, const EpiParams &p, int BN, cudaStream_t s) {
    if (p.split3) {
        if constexpr (EPI == EPI_RECON || EPI == EPI_SCALE || EPI == EPI_REFIT) {
            return cudaErrorInvalidValue;
        } else {
            switch (BN) {
                case 64: return launch_t<64, 4, EPI, true>(maps, p, s);
                case 128: return launch_t<128, 3, EPI, true>(maps, p, s);
                case 256: return launch_t<256, 2, EPI, true>(maps, p, s);
                default: return cudaErrorInvalidValue;
            }
        }
    }
    switch (BN) {
        case 64: return launch_t<64, 8, EPI, false>(maps, p, s);
        case 128: return launch_t<128, 6, EPI, false>(maps, p, s);
        case 256: return launch_t<256, 4, EPI, false>(maps, p, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gemm(const Maps &maps, const EpiParams &p, int epi, int BN, cudaStream_t s) {
    if (p.M <= 0 || p.N <= 0) return cudaSuccess;
    switch (epi) {
        case EPI_GRAM: return launch_bn<EPI_GRAM>(maps, p, BN, s);
        case EPI_RHS: return launch_bn<EPI_RHS>(maps, p, BN, s);
        case EPI_SOLVE: return launch_bn<EPI_SOLVE>(maps, p, BN, s);
        case EPI_RECON: return launch_bn<EPI_RECON>(maps, p, BN, s);
        case EPI_SPLIT: return launch_bn<EPI_SPLIT>(maps, p, BN, s);
        case EPI_SCALE: return launch_bn<EPI_SCALE>(maps, p, BN, s);
        case EPI_REFIT: return launch_bn<EPI_REFIT>(maps, p, BN, s);
        case EPI_NS1: return launch_bn<EPI_NS1>(maps, p, BN, s);
        case EPI_NS2: return launch_bn<EPI_NS2>(maps, p, BN, s);
        case EPI_GD: return launch_bn<EPI_GD>(maps, p, BN, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_newton(const NsMaps &maps, const NsArgs &a, int max_ctas, cudaStream_t s) {
    constexpr int smem = kNsStages * 2 * (A_TILE_BYTES + kNsBN * BK * 2) + 1024 + 256;
    static_assert(smem <= 227 * 1024, "shared memory of the update's stage ring");
    static std::atomic<uint64_t> configured{0};
    cudaError_t e = ensure_smem_limit((const void *)newton_kernel, smem, configured);
    if (e != cudaSuccess) return e;
    int sms = device_sm_count();
    if (max_ctas > 0 && max_ctas < sms) sms = max_ctas;
    const int64_t tiles = ceil_div(a.r, BM) * ceil_div(a.r, kNsBN);
    const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
    // cooperative: the phases wait on one another across CTAs (one CTA per SM fits)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    count_launch();
    return cudaLaunchKernelEx(&cfg, newton_kernel, maps, a);
}

}  // namespace tc
}  // namespace nq
