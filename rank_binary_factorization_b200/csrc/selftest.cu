// nq_selftest: runs the library's device-side error paths on purpose, so that a test can
// check that they end with a status the host reads and leave the context usable.
//
//   NQ_SELFTEST_WAIT_TIMEOUT  one CTA runs the bounded counter wait that the Cholesky
//                             dataflow uses (wait_geq) on a word that nothing sets, with
//                             a short poll budget; the wait gives up and raises
//                             NQ_ERR_TIMEOUT.
//   NQ_SELFTEST_NOT_SPD       the cooperative Cholesky + inverse kernel of the LB-ADMM
//                             step on G = -I (64 x 64): the first pivot is negative and
//                             the kernel raises NQ_ERR_NOT_SPD (it still runs every task
//                             of its dataflow, so every wait ends).
//
// Nothing here can fault or hang: the poll budget is bounded and every address is
// inside the caller's workspace.
#include "kernels.cuh"
#include "layout.h"

namespace nq {
namespace {

constexpr int kR = 64;                               // system size of the NOT_SPD case
constexpr uint32_t kSelftestPolls = 1u << 16;        // a few milliseconds

struct SelftestLayout {
    size_t scal = 0, flag = 0, G = 0, A = 0, Li = 0, hi = 0, lo = 0, cnt = 0, total = 0;
    SelftestLayout() {
        size_t off = 0;
        auto take = [&](size_t bytes) {
            size_t o = off;
            off = align_up(off + bytes);
            return o;
        };
        scal = take(sizeof(Scalars));
        flag = take(sizeof(unsigned int));
        G = take((size_t)kR * kR * 4);
        A = take((size_t)kR * kR * 4);
        Li = take((size_t)kR * kR * 4);
        hi = take((size_t)kR * kR * 2);
        lo = take((size_t)kR * kR * 2);
        cnt = take(2 * sizeof(unsigned int));
        total = off;
    }
};

__global__ void selftest_wait_kernel(const unsigned int *flag, uint32_t polls, int *err) {
    if (threadIdx.x == 0 && !wait_geq(flag, 1u, polls)) raise_error(err, NQ_ERR_TIMEOUT);
}

__global__ void minus_identity_kernel(float *G, int r) {
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < r * r; e += gridDim.x * blockDim.x)
        G[e] = (e / r == e % r) ? -1.f : 0.f;
}

}  // namespace
}  // namespace nq

using namespace nq;

extern "C" size_t nq_selftest_workspace_size(void) { return SelftestLayout().total; }

extern "C" nq_status nq_selftest(int32_t kind, void *ws, size_t ws_bytes, nq_stream_t stream) {
    if (kind != NQ_SELFTEST_WAIT_TIMEOUT && kind != NQ_SELFTEST_NOT_SPD) return NQ_ERR_INVALID_ARG;
    const SelftestLayout L;
    if (!ws || reinterpret_cast<uintptr_t>(ws) % kAlign != 0) return NQ_ERR_INVALID_ARG;
    if (ws_bytes < L.total) return NQ_ERR_WORKSPACE;
    int dev = 0;
    cudaDeviceProp prop;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaGetDeviceProperties(&prop, dev) != cudaSuccess)
        return NQ_ERR_CUDA;
    if (prop.major != 10) return NQ_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char *base = static_cast<char *>(ws);
    Scalars *sc = reinterpret_cast<Scalars *>(base + L.scal);
    if (cudaMemsetAsync(ws, 0, L.total, s) != cudaSuccess) return NQ_ERR_CUDA;
    if (kind == NQ_SELFTEST_WAIT_TIMEOUT) {
        selftest_wait_kernel<<<1, 32, 0, s>>>(reinterpret_cast<unsigned int *>(base + L.flag),
                                              kSelftestPolls, &sc->err);
        count_launch();
    } else {
        float *G = reinterpret_cast<float *>(base + L.G);
        minus_identity_kernel<<<8, 256, 0, s>>>(G, kR);
        count_launch();
        if (chol_inverse(G, kR, kR, reinterpret_cast<float *>(base + L.A),
                         reinterpret_cast<float *>(base + L.Li),
                         reinterpret_cast<__nv_bfloat16 *>(base + L.hi),
                         reinterpret_cast<__nv_bfloat16 *>(base + L.lo), kR,
                         reinterpret_cast<unsigned int *>(base + L.cnt), &sc->err, sc->bar,
                         0, nullptr, 0, true, s) != cudaSuccess)
            return NQ_ERR_CUDA;
    }
    if (cudaGetLastError() != cudaSuccess) return NQ_ERR_CUDA;
    int h = 0;
    if (cudaMemcpyAsync(&h, &sc->err, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return NQ_ERR_CUDA;
    return static_cast<nq_status>(h);
}
