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

// ---------------------------------------------------------------------------------
// Epilogues: thread owns tile row ``row`` and columns col0 .. col0+15.
// ---------------------------------------------------------------------------------
__device__ __forceinline__ float sgn(float x) { return x < 0.f ? -1.f : 1.f; }

__device__ __forceinline__ float load_w(const EpiParams &p, int64_t i, int64_t j) {
    if (p.w_bf16)
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p.W)[i * p.ldw + j]);
    return reinterpret_cast<const float *>(p.W)[i * p.ldw + j];
}

template <int EPI>
__device__ __forceinline__ void epilogue_chunk(const EpiParams &p, int row, int col0,
                                               const float (&v)[16], float &acc_sum) {
    const bool full = (col0 + 16 <= p.N);
    if constexpr (EPI == EPI_GRAM) {
        float *o = p.out + (int64_t)row * p.ldo + col0;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (full || col0 + j < p.N) o[j] = v[j] + ((row == col0 + j) ? p.diag : 0.f);
    } else if constexpr (EPI == EPI_RHS) {
        const float ai = p.a[row];
        const float *Srow = p.S + (int64_t)row * p.ldf + col0;
        __nv_bfloat16 *hi = p.Rhi + (int64_t)row * p.ldr + col0;
        __nv_bfloat16 *lo = p.Rlo + (int64_t)row * p.ldr + col0;
        if (full) {
            float s[16], bb[16];
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
                *reinterpret_cast<float4 *>(&s[j]) = *reinterpret_cast<const float4 *>(Srow + j);
                *reinterpret_cast<float4 *>(&bb[j]) =
                    *reinterpret_cast<const float4 *>(p.b + col0 + j);
            }
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
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            if (!(full || col0 + j < p.N)) continue;
            const float x = v[j];
            bad |= !isfinite(x);
            const float sold = Srow[j];
            const float z = sgn(sold) * ai * p.b[col0 + j];
            Xrow[j] = x;
            Srow[j] = x + sold - z;
            p.Xt[(int64_t)(col0 + j) * p.ldxt + row] = __float2bfloat16_rn(x);
            if (p.objective) {
                const int64_t o = (int64_t)row * p.ldr + col0 + j;
                const float r = __bfloat162float(p.Rhi[o]) + __bfloat162float(p.Rlo[o]);
                part += (r - p.rho * (2.f * z - sold)) * x;
            }
        }
        if (bad) raise_error(p.err, NQ_ERR_NONFINITE);
        acc_sum += part;
    } else if constexpr (EPI == EPI_RECON) {
        const float dro = p.d_out ? p.d_out[row] : 1.f;
        const float s1 = p.s1[row];
        float part = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int c = col0 + j;
            if (!(full || c < p.N)) continue;
            const float wt = dro * load_w(p, row, c) * (p.d_in ? p.d_in[c] : 1.f);
            const float d = wt - s1 * v[j] * p.s2[c];
            part += d * d;
        }
        acc_sum += part;
    }
}

// ---------------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------------
template <int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ Maps maps, const EpiParams p) {
    constexpr int B_TILE_BYTES = BN * BK * 2;
    constexpr int STAGE_BYTES = A_TILE_BYTES + B_TILE_BYTES;
    constexpr uint32_t TMEM_COLS = BN < 32 ? 32 : BN;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
    uint64_t *empty_bar = full_bar + STAGES;
    uint64_t *acc_bar = empty_bar + STAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_bar + 1);
    __shared__ double red[kEpiWarps];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * BM;
    const int n0 = blockIdx.y * BN;
    const int total_kb = p.kblocks[0] + (p.nseg > 1 ? p.kblocks[1] : 0) +
                         (p.nseg > 2 ? p.kblocks[2] : 0);

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(acc_bar, 1);
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

    if (warp == 0) {
        if (lane == 0) {
            // TMA producer
            for (int kb = 0; kb < total_kb; ++kb) {
                const int s = kb % STAGES;
                if (kb >= STAGES && !mbar_wait(&empty_bar[s], ((kb / STAGES) - 1) & 1, p.err))
                    break;
                int seg = 0, k = kb;
                while (seg < p.nseg - 1 && k >= p.kblocks[seg]) k -= p.kblocks[seg++];
                uint8_t *a_dst = smem + s * STAGE_BYTES;
                uint8_t *b_dst = a_dst + A_TILE_BYTES;
                mbar_expect_tx(&full_bar[s], STAGE_BYTES);
                tma_load_2d(a_dst, &maps.a[seg], k * BK, m0, &full_bar[s]);
                tma_load_2d(b_dst, &maps.b[seg], k * BK, n0, &full_bar[s]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // MMA issuer
            constexpr uint32_t idesc = instr_desc_bf16(BM, BN);
            bool ok = true;
            for (int kb = 0; kb < total_kb; ++kb) {
                const int s = kb % STAGES;
                if (!mbar_wait(&full_bar[s], (kb / STAGES) & 1, p.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint8_t *a_src = smem + s * STAGE_BYTES;
                const uint64_t adesc = smem_desc_sw128(a_src);
                const uint64_t bdesc = smem_desc_sw128(a_src + A_TILE_BYTES);
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)
                    mma_bf16(tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0);
                mma_commit(&empty_bar[s]);
            }
            if (ok) mma_commit(acc_bar);
        }
    } else {
        // epilogue warps
        const int q = warp & 3;
        const int row = m0 + 32 * q + lane;
        float acc_sum = 0.f;
        // one lane waits; the outcome is broadcast so that the warp-collective
        // tcgen05.ld below is executed by all 32 lanes or by none
        int ok = 0;
        if (lane == 0) ok = mbar_wait(acc_bar, 0, p.err) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (ok) {
            tc_fence_after();
            const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
            for (int c = 0; c < BN; c += 16) {
                float v[16];
                tmem_ld16(tbase + c, v);  // warp-collective: every lane takes part
                if (row < p.M && n0 + c < p.N) epilogue_chunk<EPI>(p, row, n0 + c, v, acc_sum);
            }
        }
        if constexpr (EPI == EPI_SOLVE || EPI == EPI_RECON) {
            double w = warp_sum((double)acc_sum);
            if (lane == 0) red[warp - 2] = w;
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (EPI == EPI_SOLVE || EPI == EPI_RECON) {
        if (threadIdx.x == 0 && p.part && (EPI == EPI_RECON || p.objective))
            p.part[blockIdx.y * gridDim.x + blockIdx.x] = red[0] + red[1] + red[2] + red[3];
    }
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

template <int BN, int STAGES, int EPI>
static cudaError_t launch_t(const Maps &maps, const EpiParams &p, cudaStream_t s) {
    constexpr int smem = STAGES * (A_TILE_BYTES + BN * BK * 2) + 1024 + 256;
    auto kern = gemm_kernel<BN, STAGES, EPI>;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    dim3 grid((unsigned)ceil_div(p.M, BM), (unsigned)ceil_div(p.N, BN));
    kern<<<grid, kThreads, smem, s>>>(maps, p);
    count_launch();
    return cudaGetLastError();
}

template <int EPI>
static cudaError_t launch_bn(const Maps &maps, const EpiParams &p, int BN, cudaStream_t s) {
    switch (BN) {
        case 64: return launch_t<64, 8, EPI>(maps, p, s);
        case 128: return launch_t<128, 6, EPI>(maps, p, s);
        case 256: return launch_t<256, 4, EPI>(maps, p, s);
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
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tc
}  // namespace nq
