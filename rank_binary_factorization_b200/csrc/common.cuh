// Shared device/host helpers of the sm_100a NanoQuant library.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/nq.h"

#define NQ_HD __host__ __device__ __forceinline__

namespace nq {

constexpr int kNumSMsB200 = 148;

// Host-side count of kernel launches issued by the library (nq_launch_count).
void count_launch(int n = 1);

// ---- per-device launch state (host) ------------------------------------------------
// Launch settings depend on the device a call runs on, so every cache is kept per
// device ordinal; one process may drive several GPUs, from several host threads.
constexpr int kMaxDevices = 64;
// Ordinal of the current device, or -1 if it cannot be read or is >= kMaxDevices.
int current_device();
// SM count of the current device (cached per device; kNumSMsB200 if unknown).
int device_sm_count();
// Set the dynamic shared-memory limit of ``func`` to ``bytes`` once per device; ``done``
// is the caller's per-kernel bit set of configured devices.
cudaError_t ensure_smem_limit(const void *func, int bytes, std::atomic<uint64_t> &done);

NQ_HD int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
NQ_HD int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

// Device error word: the first non-OK status raised on the device wins.
__device__ __forceinline__ void raise_error(int *err, int code) {
    if (err) atomicCAS(err, 0, code);
}

// Spin budgets for every device-side wait.  A wait that runs out raises
// NQ_ERR_TIMEOUT on the workspace's error word and returns instead of hanging.
constexpr uint32_t kMbarSpinLimit = 1u << 26;   // polls of mbarrier.try_wait (each may suspend)
constexpr uint32_t kGridSpinLimit = 1u << 24;   // polls of a grid-barrier flag (~50 ns apart)

__device__ __forceinline__ float bf16_round(float x) {
    return __bfloat162float(__float2bfloat16_rn(x));
}

// x as hi + lo BF16 (hi = RNE of x, lo = RNE of the remainder).
__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16 *hi, __nv_bfloat16 *lo) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    *hi = h;
    *lo = __float2bfloat16_rn(x - __bfloat162float(h));
}

// Warp-level sum.
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Publish: *c += inc with release semantics at GPU scope.  Called by one thread after a
// CTA barrier, it makes the CTA's earlier writes visible to any thread that then reads
// the counter with an acquire load (wait_geq).
__device__ __forceinline__ void release_add(unsigned int *c, unsigned int inc) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(c), "r"(inc) : "memory");
}

// Bounded wait until *c >= v (acquire loads, short sleeps after the first polls).
// Returns false when ``limit`` polls ran out; the caller raises NQ_ERR_TIMEOUT.
__device__ __forceinline__ bool wait_geq(const unsigned int *c, unsigned int v, uint32_t limit) {
    uint32_t spins = 0;
    while (ld_acquire_gpu(c) < v) {
        if (++spins > limit) return false;
        if (spins > 64) __nanosleep(32);
    }
    return true;
}

// Grid-wide barrier for kernels launched cooperatively (all CTAs co-resident).
// ``bar`` points at two words: [0] arrival count, [1] generation.  Bounded: a
// barrier that does not complete within the spin budget raises NQ_ERR_TIMEOUT and
// lets the CTA continue (results are then garbage but nothing hangs); after a
// timeout every later barrier is skipped, so at most one budget is spent.
__device__ __forceinline__ void grid_barrier(unsigned int *bar, int *err) {
    __syncthreads();
    if (threadIdx.x == 0 && !(err && *(volatile int *)err == NQ_ERR_TIMEOUT)) {
        const unsigned int gen = ld_acquire_gpu(bar + 1);
        __threadfence();
        const unsigned int arrived = atomicAdd(bar, 1u) + 1u;
        if (arrived == gridDim.x * gridDim.y * gridDim.z) {
            atomicExch(bar, 0u);
            __threadfence();
            atomicAdd(bar + 1, 1u);
        } else {
            uint32_t spins = 0;
            while (ld_acquire_gpu(bar + 1) == gen) {
                if (++spins > kGridSpinLimit) {
                    raise_error(err, NQ_ERR_TIMEOUT);
                    break;
                }
                if (spins > 256) __nanosleep(32);
            }
        }
        __threadfence();
    }
    __syncthreads();
}

}  // namespace nq
