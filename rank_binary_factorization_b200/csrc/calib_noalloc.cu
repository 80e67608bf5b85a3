// nq_calib_stats_noalloc: the calibration moment reduction without a caller workspace.
//
// Some callers cannot hand the library a workspace or allocate device memory at all:
// a plugin or callback running inside a host program that owns the whole device memory
// pool and refuses new allocations after start-up, a process with a device-memory
// budget fixed at launch, or a code path that must not call cudaMalloc / cudaFree
// because those calls may synchronise the device.  For them this entry point keeps
// its scratch (the per-slab partial sums) in a fixed array that is part of the loaded
// library image instead of a workspace.
//
// Cost and limits:
//   * kNoAllocScratchDoubles doubles (4 MiB) of device memory are reserved on every GPU
//     that loads the library, until the process exits;
//   * the scratch bounds the problem: token slabs x channels must fit (every C up to
//     kNoAllocMaxChannels fits for any T); larger calls return NQ_ERR_UNSUPPORTED;
//   * all calls share the one array: calls whose GPU work overlaps (different streams,
//     different host threads) race on it and must be ordered by the caller;
//   * the array keeps the previous call's contents; nothing needs clearing because
//     every partial sum read by a call was written by the same call.
#include <mutex>

#include "kernels.cuh"

namespace nq {
namespace {

constexpr int64_t kNoAllocScratchDoubles = 2 * 262144;   // two partial arrays
constexpr int64_t kNoAllocMaxChannels = 32768;

static __device__ __align__(256) double g_noalloc_scratch[kNoAllocScratchDoubles];

// Host code cannot use g_noalloc_scratch as a device address (on the host it names a
// stand-in object).  The device address is looked up once per device, with that device
// current, and cached.
std::mutex g_mu;
double *g_dev_ptr[64] = {nullptr};

nq_status scratch_for_current_device(double **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NQ_ERR_CUDA;
    if (dev < 0 || dev >= 64) return NQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_dev_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
            return NQ_ERR_CUDA;
        g_dev_ptr[dev] = static_cast<double *>(p);
    }
    *out = g_dev_ptr[dev];
    return NQ_OK;
}

}  // namespace
}  // namespace nq

extern "C" nq_status nq_calib_stats_noalloc(const void *X, int64_t T, int64_t C, nq_dtype dt,
                                            double *s, double *q, nq_stream_t stream) {
    using namespace nq;
    if (!X || !s || !q || T < 1 || C < 1 || (dt != NQ_F32 && dt != NQ_BF16))
        return NQ_ERR_INVALID_ARG;
    const int nslab = calib_num_slabs(T, C);
    if (C > kNoAllocMaxChannels || 2 * (int64_t)nslab * C > kNoAllocScratchDoubles)
        return NQ_ERR_UNSUPPORTED;
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return NQ_ERR_CUDA;
    if (major != 10) return NQ_ERR_UNSUPPORTED;
    double *scratch = nullptr;
    nq_status st = scratch_for_current_device(&scratch);
    if (st != NQ_OK) return st;
    double *ps = scratch;
    double *pq = scratch + (int64_t)nslab * C;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (calib_partials(X, T, C, dt == NQ_BF16, nslab, ps, pq, cs) != cudaSuccess)
        return NQ_ERR_CUDA;
    if (calib_moments(ps, pq, nslab, T, C, s, q, cs) != cudaSuccess) return NQ_ERR_CUDA;
    return NQ_OK;
}
