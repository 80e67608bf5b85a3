// C ABI of the library (declared in include/nq.h): argument checks, workspace
// carving and the launch sequence of each entry point.  No device allocation.
#include <math.h>
#include <string.h>

#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "layout.h"

using namespace nq;

namespace nq {
static std::atomic<long long> g_launches{0};
void count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    return dev;
}

int device_sm_count() {
    static std::atomic<int> cache[kMaxDevices];
    const int dev = current_device();
    if (dev < 0) return kNumSMsB200;
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v < 1)
        v = kNumSMsB200;
    cache[dev].store(v, std::memory_order_relaxed);
    return v;
}

cudaError_t ensure_smem_limit(const void *func, int bytes, std::atomic<uint64_t> &done) {
    const int dev = current_device();
    if (dev < 0) return cudaErrorInvalidDevice;
    const uint64_t bit = 1ull << dev;
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}
}  // namespace nq

namespace {

#define NQ_CK(call)                                  \
    do {                                             \
        cudaError_t e_ = (call);                     \
        if (e_ != cudaSuccess) return NQ_ERR_CUDA;   \
    } while (0)

inline cudaStream_t cs(nq_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// ---- optional per-launch device timing (nq_profile_*) ------------------------------
struct ProfRec {
    int cls;
    cudaEvent_t a, b;
};
std::mutex g_prof_mu;
std::vector<ProfRec> g_prof;
size_t g_prof_used = 0;
bool g_prof_on = false;

// NVTX range names of the kernel classes (nq_kernel_class order)
const char *const kClassNames[NQ_K_COUNT] = {
    "nq.calib", "nq.calib_finalize", "nq.prep", "nq.gram", "nq.chol", "nq.rhs",
    "nq.solve", "nq.svid", "nq.objective", "nq.finish", "nq.recon", "nq.ginv", "nq.binary",
    "nq.refit", "nq.newton", "nq.gd"};

// Scope of one kernel class's launches: an NVTX range on the host timeline (seen by
// profilers; inert otherwise) and, when recording is on, a CUDA event pair on the stream.
struct ProfScope {
    ProfRec *rec = nullptr;
    cudaStream_t s;
    ProfScope(int cls, cudaStream_t st) : s(st) {
        nvtxRangePushA(kClassNames[cls]);
        if (!g_prof_on) return;
        std::lock_guard<std::mutex> lk(g_prof_mu);
        if (g_prof_used == g_prof.size()) {
            ProfRec r{cls, nullptr, nullptr};
            if (cudaEventCreate(&r.a) != cudaSuccess || cudaEventCreate(&r.b) != cudaSuccess)
                return;
            g_prof.push_back(r);
        }
        rec = &g_prof[g_prof_used++];
        rec->cls = cls;
        cudaEventRecord(rec->a, s);
    }
    ~ProfScope() {
        if (rec) cudaEventRecord(rec->b, s);
        nvtxRangePop();
    }
};

template <class T>
inline T *at(void *ws, size_t off) {
    return reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}

// The library only runs on sm_100 devices (the kernels are built for sm_100a).
nq_status check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NQ_ERR_CUDA;
    static std::atomic<int> cached[kMaxDevices];
    if (dev >= 0 && dev < kMaxDevices) {
        const int c = cached[dev].load(std::memory_order_relaxed);
        if (c) return c == 1 ? NQ_OK : NQ_ERR_UNSUPPORTED;
    }
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return NQ_ERR_CUDA;
    const bool ok = major == 10;
    if (dev >= 0 && dev < kMaxDevices) cached[dev].store(ok ? 1 : 2, std::memory_order_relaxed);
    return ok ? NQ_OK : NQ_ERR_UNSUPPORTED;
}

inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
// a vector that is absent (identity) or starts on a 16-byte boundary
inline bool vec16(const void *p) { return !p || aligned(p, 16); }

nq_status check_lb_args(int64_t m, int64_t n, int32_t r) {
    if (m < 1 || n < 1 || m > kMaxDim || n > kMaxDim) return NQ_ERR_INVALID_ARG;
    if (r < 1 || r > kMaxRank || r > m || r > n) return NQ_ERR_INVALID_ARG;
    return NQ_OK;
}

nq_status check_ws(void *ws, size_t ws_bytes, size_t need) {
    if (!ws) return NQ_ERR_INVALID_ARG;
    if (!aligned(ws, kAlign)) return NQ_ERR_INVALID_ARG;
    if (ws_bytes < need) return NQ_ERR_WORKSPACE;
    return NQ_OK;
}

int pick_bn(int64_t N) { return N <= 64 ? 64 : (N <= 128 ? 128 : 256); }

inline bool valid_prec(int prec) { return prec == NQ_PREC_BF16 || prec == NQ_PREC_FP32; }

// Tile width for skinny products (few 128-row tiles): the widest BN whose tile count still
// fills the SMs, else the narrowest.
int pick_bn_fill(int64_t M, int64_t N, int sms) {
    for (int bn : {256, 128}) {
        if (N > bn / 2 && ceil_div(M, 128) * ceil_div(N, bn) >= sms) return bn;
    }
    return N <= 64 ? 64 : (ceil_div(M, 128) * ceil_div(N, 128) >= sms ? 128 : 64);
}

nq_status read_err(int *dev_err, cudaStream_t s, bool reset) {
    int h = 0;
    NQ_CK(cudaMemcpyAsync(&h, dev_err, sizeof(int), cudaMemcpyDeviceToHost, s));
    NQ_CK(cudaStreamSynchronize(s));
    if (reset && h) NQ_CK(cudaMemsetAsync(dev_err, 0, sizeof(int), s));
    return static_cast<nq_status>(h);
}

size_t calib_ws_bytes(int64_t C) {
    // token slabs * channels is at most 4 * 148 * 256 + C + 256 (see calib_num_slabs);
    // the partial arrays are sized with headroom above that
    const size_t pd = (size_t)(6 * kNumSMsB200 * 256 + C + 256);
    return align_up(sizeof(Scalars)) + 2 * align_up(pd * 8) + 2 * align_up((size_t)C * 8);
}

struct CalibCarve {
    Scalars *sc;
    double *ps, *pq, *s, *q;
};
CalibCarve carve_calib(void *ws, int64_t C) {
    const size_t pd = (size_t)(6 * kNumSMsB200 * 256 + C + 256);
    size_t off = 0;
    CalibCarve c;
    c.sc = at<Scalars>(ws, off);
    off += align_up(sizeof(Scalars));
    c.ps = at<double>(ws, off);
    off += align_up(pd * 8);
    c.pq = at<double>(ws, off);
    off += align_up(pd * 8);
    c.s = at<double>(ws, off);
    off += align_up((size_t)C * 8);
    c.q = at<double>(ws, off);
    return c;
}

nq_status enqueue_stats(const void *X, int64_t T, int64_t C, int bf16, double *s_out,
                        double *q_out, const CalibCarve &cv, cudaStream_t st) {
    const int nslab = calib_num_slabs(T, C);
    {
        ProfScope ps(NQ_K_CALIB, st);
        NQ_CK(calib_partials(X, T, C, bf16, nslab, cv.ps, cv.pq, st));
    }
    ProfScope ps(NQ_K_CALIB_FIN, st);
    NQ_CK(calib_moments(cv.ps, cv.pq, nslab, T, C, s_out, q_out, st));
    return NQ_OK;
}

// ---- side stream of the r x r factorisation ---------------------------------------
// Per host thread and device: a library-owned stream on which the Cholesky + inverse and
// the G^-1 GEMM of a half step run beside the RHS GEMM, and the two events that fork it
// from, and join it back into, the caller's stream.  Created by the first call of a host
// thread on a device; never destroyed (they live until the process exits).
// The same context also holds the auxiliary stream of the SVID passes, which run beside
// the next half step's RHS GEMM and solve (see lb_iterate), with its events.
struct SideCtx {
    cudaStream_t side = nullptr, aux = nullptr, obj = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr, pre_rhs = nullptr, obj_done = nullptr,
                svid_done[2] = {nullptr, nullptr};
};

nq_status side_ctx(SideCtx **out) {
    thread_local SideCtx ctx[kMaxDevices];
    const int dev = current_device();
    if (dev < 0) return NQ_ERR_CUDA;
    SideCtx &c = ctx[dev];
    if (!c.side) {
        // default priority: raising either stream above the caller's was measured slower
        NQ_CK(cudaStreamCreateWithFlags(&c.side, cudaStreamNonBlocking));
        NQ_CK(cudaStreamCreateWithFlags(&c.aux, cudaStreamNonBlocking));
        NQ_CK(cudaStreamCreateWithFlags(&c.obj, cudaStreamNonBlocking));
        for (cudaEvent_t *e :
             {&c.fork, &c.join, &c.pre_rhs, &c.obj_done, &c.svid_done[0], &c.svid_done[1]})
            NQ_CK(cudaEventCreateWithFlags(e, cudaEventDisableTiming));
    }
    *out = &c;
    return NQ_OK;
}

// CTAs given to the factorisation while the RHS GEMM runs on the others (0: no overlap,
// the factorisation takes the whole GPU before the GEMM).  The factorisation is a chain
// of nb = r/64 dependent tile steps plus ~nb^3/3 tile tasks for its workers; up to
// nb = 24 half of the SMs keep the workers ahead of the chain, so the chain's latency,
// not the SM count, sets its time, and the GEMM runs on the other half meanwhile.
// Beyond that the workers need the whole GPU.
int chol_ctas(int32_t r, int sms) {
    const int nb = (r + 63) / 64;
    return nb <= 24 ? sms / 2 : 0;
}

// ---- LB-ADMM internals ------------------------------------------------------------
struct Lb {
    LbLayout L;
    void *ws;
    Scalars *sc;
    template <class T>
    T *p(size_t off) const {
        return at<T>(ws, off);
    }
};

nq_status lb_open(Lb &lb, int64_t m, int64_t n, int32_t r, void *ws, size_t ws_bytes) {
    nq_status st = check_lb_args(m, n, r);
    if (st) return st;
    lb.L.build(m, n, r);
    st = check_ws(ws, ws_bytes, lb.L.total);
    if (st) return st;
    lb.ws = ws;
    lb.sc = at<Scalars>(ws, lb.L.scal);
    return check_device();
}

// Gram of the operand of side ``other`` (its BF16 transpose) into g[other]; the result is
// symmetric, so only its lower-triangular 128 x 128 tiles are computed and mirrored.  In
// the FP32-accurate mode the operand is split (hi + lo) and the Gram takes three passes.
// With ``ns_prep`` the Gram is also written split (hi + lo BF16) for the Newton-Schulz
// update, and the update's gate is opened; with ``zero_chol`` it also zeroes the tile
// counters of the factorisation that follows it.
nq_status lb_gram(const Lb &lb, int other, float diag, int prec, cudaStream_t s,
                  bool ns_prep = false, bool zero_chol = false) {
    const LbLayout &L = lb.L;
    const int64_t K = L.rows(other), ld = L.ld_rows(other);
    const __nv_bfloat16 *xt = lb.p<__nv_bfloat16>(L.xt[other]);
    const __nv_bfloat16 *xl = lb.p<__nv_bfloat16>(L.xtl[other]);
    constexpr int BN = tc::BM;
    tc::Maps maps;
    memset(&maps, 0, sizeof(maps));
    const int split = prec == NQ_PREC_FP32 ? 1 : 0;
    const void *parts[2] = {xt, xl};
    for (int g = 0; g <= split; ++g)
        if (!tc::make_map_bf16(&maps.a[g], parts[g], L.r, K, ld, tc::BM) ||
            !tc::make_map_bf16(&maps.b[g], parts[g], L.r, K, ld, BN))
            return NQ_ERR_CUDA;
    tc::EpiParams ep;
    memset(&ep, 0, sizeof(ep));
    ep.M = L.r;
    ep.N = L.r;
    ep.nseg = 1;
    ep.split3 = split;
    ep.kblocks[0] = (int)ceil_div(K, tc::BK);
    ep.sym = 1;
    ep.err = &lb.sc->err;
    ep.out = lb.p<float>(L.g[other]);
    ep.ldo = L.r;
    ep.diag = diag;
    __nv_bfloat16 *gh = ns_prep ? lb.p<__nv_bfloat16>(L.gsh) : nullptr;
    __nv_bfloat16 *gl = ns_prep ? lb.p<__nv_bfloat16>(L.gsl) : nullptr;
    ep.Rhi = gh;
    ep.Rlo = gl;
    ep.ldr = L.ldr;
    ep.ns = ns_prep ? lb.p<NsState>(L.ns) : nullptr;
    if (zero_chol) {   // tile counters of the factorisation that follows
        ep.zero = lb.p<unsigned int>(L.chF);
        ep.zero_words = (int)(2 * (L.rp / 64) * (L.rp / 64));
    }
    // few tiles (small r): split K so that the (tile, part) units fill the SMs; the parts
    // are summed in a fixed order by gram_reduce
    const int S = gram_ksplit(L.r, K, 1, device_sm_count());
    ProfScope ps(NQ_K_GRAM, s);
    if (S > 1) {
        ep.ksplit = S;
        ep.out = lb.p<float>(L.gpart);
        NQ_CK(tc::launch_gemm(maps, ep, tc::EPI_GRAM, BN, s));
        NQ_CK(gram_reduce(lb.p<float>(L.gpart), gram_tiles(L.r), S, L.r, diag,
                          lb.p<float>(L.g[other]), gh, gl, L.ldr, s));
        return NQ_OK;
    }
    NQ_CK(tc::launch_gemm(maps, ep, tc::EPI_GRAM, BN, s));
    return NQ_OK;
}

nq_status lb_svid(const Lb &lb, int side, int K, cudaStream_t s) {
    const LbLayout &L = lb.L;
    ProfScope ps(NQ_K_SVID, s);
    NQ_CK(svid(lb.p<float>(L.s[side]), L.rows(side), L.r, L.ldr, K, L.nsv, lb.p<float>(L.bcur),
               lb.p<float>(L.tvec), lb.p<float>(L.partb), lb.p<double>(L.partn),
               lb.p<float>(L.a[side]), lb.p<float>(L.b[side]), s));
    return NQ_OK;
}

// ---- Newton-Schulz update of G^-1 --------------------------------------------------
// The Gram of a side changes little from one iteration to the next, so the inverse used
// by that side's previous solve is a close start for the next one: the Newton-Schulz
// (Schulz 1933; Ben-Israel 1965) iteration X_{k+1} = X_k (2I - G X_k), written as
// X_{k+1} = X_k + E_k X_k with E_k = I - X_k G, converges quadratically (E_{k+1} = E_k^2)
// whenever the spectral radius of E_0 is below 1.  Each step is two r x r tensor-core
// GEMMs: E_k = I - X_k G in plain BF16 for the first kNsBf16Steps steps and split
// (hi + lo) after them, E_k X_k always in plain BF16 (a correction of size |E_k|).  The
// device decides: a step whose ||E_k||_F falls to ns_tau makes the next iterate final
// (written to the side's G^-1); a residual that does not shrink, or no final iterate
// after kNsMaxSteps, falls back to the Cholesky path, which then runs (gated).
constexpr int32_t kNsMinRank = 256;  // below this the factorisation is as fast
// iterations since prepare before the first attempt (3; 4 above r = 1536, where the
// Grams of the fourth iteration still move too far)
inline int ns_first_iter(int32_t r) { return r > 1536 ? 4 : 3; }
constexpr float kNsTau = 1e-2f;      // ||E_k||_F that makes X_{k+1} final (||E||_2 <= 1e-4)

std::atomic<int> g_inverse_mode{NQ_INV_AUTO};

// Latent update: the exact solve (default) or gradient-descent steps (nq_set_latent_solver).
std::atomic<int> g_solver{NQ_SOLVER_EXACT};
std::atomic<int> g_gd_steps{8};

// Performance settings of nq_set_tuning (none changes what is computed).
std::atomic<int> g_tune[NQ_TUNE_COUNT] = {{-1}, {0}, {1}, {1}, {0}, {0}, {0}};

// Tile widths of the RHS GEMM and of the solve (the objective's partials follow the solve's).
int rhs_bn(int32_t r) {
    const int v = g_tune[NQ_TUNE_RHS_BN].load(std::memory_order_relaxed);
    return v ? v : pick_bn(r);
}
int solve_bn(int32_t r) {
    // 128-wide tiles up to r = 1024 (twice the tiles, so the heavy epilogue of one tile
    // overlaps the next tile's MMAs on more CTAs; measured 1 % faster at r = 1000)
    const int v = g_tune[NQ_TUNE_SOLVE_BN].load(std::memory_order_relaxed);
    return v ? v : (r > 128 && r <= 1024 ? 128 : pick_bn(r));
}

// Iterations run on each workspace since its last prepare (host side; AUTO mode).
std::mutex g_iter_mu;
std::unordered_map<const void *, long long> g_iter_count;
long long iters_since_prepare(const void *ws) {
    std::lock_guard<std::mutex> g(g_iter_mu);
    auto it = g_iter_count.find(ws);
    return it == g_iter_count.end() ? 0 : it->second;
}
void add_iters(const void *ws, long long k) {
    std::lock_guard<std::mutex> g(g_iter_mu);
    // bounded: a process that prepares very many distinct workspaces forgets the older
    // counts (their next updates start a few iterations later; results do not change)
    if (g_iter_count.size() >= 4096 && g_iter_count.find(ws) == g_iter_count.end())
        g_iter_count.clear();
    if (k < 0)
        g_iter_count[ws] = 0;
    else
        g_iter_count[ws] += k;
}

// Tile width of the r x r products on ``ctas`` CTAs: the fewest waves x tile width.
int pick_bn_square(int32_t r, int ctas) {
    int best = 64;
    int64_t best_cost = INT64_MAX;
    for (int bn : {256, 128, 64}) {
        const int64_t tiles = ceil_div(r, 128) * ceil_div(r, bn);
        const int64_t cost = ceil_div(tiles, ctas) * bn;
        if (cost < best_cost) {
            best_cost = cost;
            best = bn;
        }
    }
    return best;
}

// All steps in one cooperative launch (see tc::newton_kernel).
nq_status lb_newton_fused(const Lb &lb, int side, int max_ctas, cudaStream_t s) {
    const LbLayout &L = lb.L;
    const int r = L.r;
    tc::NsMaps maps;
    memset(&maps, 0, sizeof(maps));
    tc::NsArgs a;
    memset(&a, 0, sizeof(a));
    const size_t xh[3] = {L.gih[side], L.nqh[0], L.nqh[1]};
    const size_t xl[3] = {L.gil[side], L.nql[0], L.nql[1]};
    for (int i = 0; i < 3; ++i) {
        a.xh[i] = lb.p<__nv_bfloat16>(xh[i]);
        a.xl[i] = lb.p<__nv_bfloat16>(xl[i]);
        if (!tc::make_map_bf16(&maps.xh[i], a.xh[i], r, r, L.ldr, tc::BM) ||
            !tc::make_map_bf16(&maps.xl[i], a.xl[i], r, r, L.ldr, tc::BM))
            return NQ_ERR_CUDA;
    }
    a.eh = lb.p<__nv_bfloat16>(L.nth);
    a.el = lb.p<__nv_bfloat16>(L.ntl);
    if (!tc::make_map_bf16(&maps.gh, lb.p<void>(L.gsh), r, r, L.ldr, tc::BM) ||
        !tc::make_map_bf16(&maps.gl, lb.p<void>(L.gsl), r, r, L.ldr, tc::BM) ||
        !tc::make_map_bf16(&maps.eh, a.eh, r, r, L.ldr, tc::BM))
        return NQ_ERR_CUDA;
    a.r = r;
    a.ldr = L.ldr;
    a.nsteps = kNsMaxSteps;
    a.bf16_steps = kNsBf16Steps;
    a.tau = kNsTau;
    a.err = &lb.sc->err;
    a.ns = lb.p<NsState>(L.ns);
    a.part = lb.p<double>(L.nspart);
    ProfScope ps(NQ_K_NEWTON, s);
    NQ_CK(tc::launch_newton(maps, a, max_ctas, s));
    return NQ_OK;
}

nq_status lb_newton(const Lb &lb, int side, int max_ctas, cudaStream_t s) {
    if (g_tune[NQ_TUNE_NEWTON_FUSED].load(std::memory_order_relaxed))
        return lb_newton_fused(lb, side, max_ctas, s);
    const LbLayout &L = lb.L;
    NsState *ns = lb.p<NsState>(L.ns);
    const int r = L.r;
    const int ctas = max_ctas > 0 ? max_ctas : device_sm_count();
    const int bn_set = g_tune[NQ_TUNE_NEWTON_BN].load(std::memory_order_relaxed);
    const int BN = bn_set ? bn_set : pick_bn_square(r, ctas);
    const int kb = (int)ceil_div(r, tc::BK);
    const void *gh = lb.p<void>(L.gsh), *gl = lb.p<void>(L.gsl);
    const void *eh = lb.p<void>(L.nth), *el = lb.p<void>(L.ntl);
    ProfScope ps(NQ_K_NEWTON, s);
    for (int k = 0; k < kNsMaxSteps; ++k) {
        // X_0: the side's previous G^-1; X_k: iterate buffer k % 2
        const size_t xo_h = k == 0 ? L.gih[side] : L.nqh[k % 2];
        const size_t xo_l = k == 0 ? L.gil[side] : L.nql[k % 2];
        const void *xh = lb.p<void>(xo_h), *xl = lb.p<void>(xo_l);
        const int split = k < kNsBf16Steps ? 0 : 1;
        tc::EpiParams ep;
        memset(&ep, 0, sizeof(ep));
        ep.M = r;
        ep.N = r;
        ep.nseg = 1;
        ep.split3 = split;
        ep.kblocks[0] = kb;
        ep.max_ctas = max_ctas;
        ep.err = &lb.sc->err;
        ep.gate = &ns->gate;
        ep.gate_skip = (1 << NS_DONE) | (1 << NS_FAIL);
        ep.ns = ns;
        ep.ns_step = k;
        ep.ns_last = kNsMaxSteps - 1;
        ep.ns_min_final = kNsBf16Steps;
        ep.ns_tau = kNsTau;
        ep.ldr = L.ldr;
        {   // E_k = I - X_k G: A = X_k, B = G (symmetric: its rows are its columns)
            tc::Maps maps;
            memset(&maps, 0, sizeof(maps));
            const void *as[2] = {xh, xl}, *bs[2] = {gh, gl};
            for (int g = 0; g <= split; ++g)
                if (!tc::make_map_bf16(&maps.a[g], as[g], r, r, L.ldr, tc::BM) ||
                    !tc::make_map_bf16(&maps.b[g], bs[g], r, r, L.ldr, BN))
                    return NQ_ERR_CUDA;
            ep.part = lb.p<double>(L.nspart);
            ep.Rhi = lb.p<__nv_bfloat16>(L.nth);
            ep.Rlo = lb.p<__nv_bfloat16>(L.ntl);
            NQ_CK(tc::launch_gemm(maps, ep, tc::EPI_NS1, BN, s));
        }
        {   // X_{k+1} = X_k + E_k X_k: A = E_k, B = X_k (symmetric).  One BF16 pass: the
            // correction's rounding (2^-8 |E_k| |X_k|) is removed by the next step, and in
            // the final one |E_k| <= 1e-2 keeps it below the split products' floor
            tc::Maps maps;
            memset(&maps, 0, sizeof(maps));
            if (!tc::make_map_bf16(&maps.a[0], eh, r, r, L.ldr, tc::BM) ||
                !tc::make_map_bf16(&maps.b[0], xh, r, r, L.ldr, BN))
                return NQ_ERR_CUDA;
            (void)el;
            ep.split3 = 0;
            ep.part = nullptr;
            ep.Ph = static_cast<const __nv_bfloat16 *>(xh);
            ep.Pl = static_cast<const __nv_bfloat16 *>(xl);
            ep.Rhi = lb.p<__nv_bfloat16>(L.nqh[(k + 1) % 2]);
            ep.Rlo = lb.p<__nv_bfloat16>(L.nql[(k + 1) % 2]);
            ep.Fhi = lb.p<__nv_bfloat16>(L.gih[side]);
            ep.Flo = lb.p<__nv_bfloat16>(L.gil[side]);
            NQ_CK(tc::launch_gemm(maps, ep, tc::EPI_NS2, BN, s));
        }
    }
    return NQ_OK;
}

// One half step: X_side from X_other (Gram, factorisation, G^-1, RHS, solve), then the
// SVID of this side on ``s`` when ``ov`` is null.  Inside lb_iterate ``ov`` is the side
// context and the SVIDs run on its auxiliary stream instead: ``pending`` (>= 0) is the
// side solved by the previous half step, whose SVID is started once this half step's
// G^-1 is formed, beside its RHS GEMM and solve; ``wait_own`` makes the RHS GEMM wait for
// the SVID of ``side`` started by the previous half step (the RHS and the solve read the
// dual state a, b it writes).
nq_status lb_objective(const Lb &lb, float c, int slot, cudaStream_t s);

// Gradient-descent latent update (solver variant): X <- X - eta (X G - R), g_gd_steps steps
// from the side's current latent, each one split-BF16 GEMM X G (K = r) whose epilogue
// takes the step and writes the next operand; then the state update of the exact path's
// solve epilogue (dual state, transposed operand copy, objective partials on the V side).
nq_status lb_gd_steps(const Lb &lb, int side, float rho, int prec, cudaStream_t s) {
    const LbLayout &L = lb.L;
    const int64_t rows = L.rows(side);
    const int BN = solve_bn(L.r);
    const int steps = g_gd_steps.load(std::memory_order_relaxed);
    ProfScope ps(NQ_K_GD, s);
    NQ_CK(split_rows(lb.p<float>(L.x[side]), rows, L.r, L.ldr, lb.p<__nv_bfloat16>(L.gdh[0]),
                     lb.p<__nv_bfloat16>(L.gdl[0]), L.ldr, s));
    for (int j = 0; j < steps; ++j) {
        const int a = j & 1, w = 1 - a;
        tc::Maps maps;
        memset(&maps, 0, sizeof(maps));
        if (!tc::make_map_bf16(&maps.a[0], lb.p<void>(L.gdh[a]), rows, L.r, L.ldr, tc::BM) ||
            !tc::make_map_bf16(&maps.a[1], lb.p<void>(L.gdl[a]), rows, L.r, L.ldr, tc::BM) ||
            !tc::make_map_bf16(&maps.b[0], lb.p<void>(L.gsh), L.r, L.r, L.ldr, BN) ||
            !tc::make_map_bf16(&maps.b[1], lb.p<void>(L.gsl), L.r, L.r, L.ldr, BN))
            return NQ_ERR_CUDA;
        tc::EpiParams ep;
        memset(&ep, 0, sizeof(ep));
        ep.M = (int)rows;
        ep.N = L.r;
        ep.nseg = 1;
        ep.split3 = 1;
        ep.kblocks[0] = (int)ceil_div(L.r, tc::BK);
        ep.nfast = 1;
        ep.err = &lb.sc->err;
        ep.X = lb.p<float>(L.x[side]);
        ep.ldf = L.ldr;
        ep.Ph = lb.p<__nv_bfloat16>(L.rhi);
        ep.Pl = lb.p<__nv_bfloat16>(L.rlo);
        ep.ldr = L.ldr;
        ep.Fhi = lb.p<__nv_bfloat16>(L.gdh[w]);
        ep.Flo = lb.p<__nv_bfloat16>(L.gdl[w]);
        ep.gd_max = lb.p<float>(L.gdmax);
        NQ_CK(tc::launch_gemm(maps, ep, tc::EPI_GD, BN, s));
    }
    const int npx = (int)tc::num_tiles((int)L.n, L.r, solve_bn(L.r));
    NQ_CK(gd_finalize(lb.p<float>(L.x[side]), lb.p<float>(L.s[side]), lb.p<float>(L.a[side]),
                      lb.p<float>(L.b[side]), rows, L.r, L.ldr, rho, lb.p<__nv_bfloat16>(L.rhi),
                      lb.p<__nv_bfloat16>(L.rlo), L.ldr, lb.p<__nv_bfloat16>(L.xt[side]),
                      prec == NQ_PREC_FP32 ? lb.p<__nv_bfloat16>(L.xtl[side]) : nullptr,
                      L.ld_rows(side), side == 1, lb.p<double>(L.part),
                      side == 1 ? npx : kRedBlocks, &lb.sc->err, s));
    return NQ_OK;
}

nq_status lb_half_step(const Lb &lb, int side, float rho, float lambda, int K, int prec,
                       cudaStream_t s, SideCtx *ov = nullptr, int pending = -1,
                       bool wait_own = false, int obj_slot = -1, bool wait_obj = false) {
    const LbLayout &L = lb.L;
    // the Gram below overwrites the Gram of U that the previous objective reads
    if (ov && wait_obj) NQ_CK(cudaStreamWaitEvent(s, ov->obj_done, 0));
    const int other = 1 - side;
    const int64_t rows = L.rows(side), Kd = L.rows(other);
    const int BN = rhs_bn(L.r), BNs = solve_bn(L.r);
    const bool gd = g_solver.load(std::memory_order_relaxed) == NQ_SOLVER_GD;
    const int mode = g_inverse_mode.load(std::memory_order_relaxed);
    const bool newton = !gd && (mode == NQ_INV_NEWTON ||
                                (mode == NQ_INV_AUTO && L.r >= kNsMinRank &&
                                 iters_since_prepare(lb.ws) >= ns_first_iter(L.r)));
    NsState *ns = lb.p<NsState>(L.ns);
    // the update and the gradient steps take the Gram split into hi + lo as their operand
    nq_status st = lb_gram(lb, other, lambda + rho, prec, s, newton || gd, !gd);
    if (st) return st;
    if (gd) {   // step size 1 / max_i sum_j |G_ij|
        ProfScope ps(NQ_K_GD, s);
        NQ_CK(cudaMemsetAsync(lb.p<void>(L.gdmax), 0, sizeof(unsigned int), s));
        NQ_CK(gd_rowabs_max(lb.p<float>(L.g[other]), L.r, lb.p<unsigned int>(L.gdmax), s));
    }
    // The factorisation of G and the G^-1 GEMM depend only on the Gram; the RHS GEMM only
    // on the other side's operand and this side's dual state.  With overlap they run at
    // once: the factorisation on ``cc`` CTAs of a side stream, the RHS GEMM on the rest.
    const int sms = device_sm_count();
    const int fc = g_tune[NQ_TUNE_FACTOR_CTAS].load(std::memory_order_relaxed);
    const int cc = gd ? 0
                      : (fc < 0 ? chol_ctas(L.r, sms)
                                : (fc == 0 ? 0 : std::min(std::max(fc, 3), sms - 1)));
    SideCtx *sc = nullptr;
    if (cc > 0 && (st = side_ctx(&sc))) return st;
    cudaStream_t fs = s;   // stream of the factorisation
    if (cc > 0) {
        NQ_CK(cudaEventRecord(sc->fork, s));
        NQ_CK(cudaStreamWaitEvent(sc->side, sc->fork, 0));
        fs = sc->side;
    }
    if (newton && (st = lb_newton(lb, side, cc, fs))) return st;
    // with the update, the factorisation and the G^-1 GEMM run only if it failed
    const int *gate = newton ? &ns->gate : nullptr;
    const int gate_skip = newton ? (1 << NS_DONE) : 0;
    if (!gd) {
        ProfScope ps(NQ_K_CHOL, fs);
        NQ_CK(chol_inverse(lb.p<float>(L.g[other]), L.r, L.rp, lb.p<float>(L.chA),
                           lb.p<float>(L.chLi), lb.p<__nv_bfloat16>(L.lth),
                           lb.p<__nv_bfloat16>(L.ltl), L.ldr, lb.p<unsigned int>(L.chF),
                           &lb.sc->err, lb.sc->bar, cc, gate, gate_skip, false, fs));
    }
    if (!gd) {
        ProfScope ps(NQ_K_GINV, fs);
        // G^-1 = Li^T Li = LiT LiT^T as three split-BF16 passes, written as hi + lo; G^-1 is
        // symmetric, so only its lower-triangular tiles are computed and mirrored
        tc::Maps maps;
        memset(&maps, 0, sizeof(maps));
        const void *th = lb.p<void>(L.lth), *tl = lb.p<void>(L.ltl);
        const int BNg = tc::BM;  // square tiles: only the lower triangle is computed
        if (!tc::make_map_bf16(&maps.a[0], th, L.r, L.r, L.ldr, tc::BM) ||
            !tc::make_map_bf16(&maps.a[1], tl, L.r, L.r, L.ldr, tc::BM) ||
            !tc::make_map_bf16(&maps.b[0], th, L.r, L.r, L.ldr, BNg) ||
            !tc::make_map_bf16(&maps.b[1], tl, L.r, L.r, L.ldr, BNg))
            return NQ_ERR_CUDA;
        tc::EpiParams ep;
        memset(&ep, 0, sizeof(ep));
        ep.M = L.r;
        ep.N = L.r;
        ep.nseg = 1;
        ep.split3 = 1;
        ep.kblocks[0] = (int)ceil_div(L.r, tc::BK);
        ep.tri_k = 1;
        ep.sym = 1;
        ep.max_ctas = cc;
        ep.err = &lb.sc->err;
        ep.gate = gate;
        ep.gate_skip = gate_skip;
        ep.Rhi = lb.p<__nv_bfloat16>(L.gih[side]);
        ep.Rlo = lb.p<__nv_bfloat16>(L.gil[side]);
        ep.ldr = L.ldr;
        NQ_CK(tc::launch_gemm(maps, ep, tc::EPI_SPLIT, BNg, fs));
    }
    if (cc > 0) NQ_CK(cudaEventRecord(sc->join, fs));
    if (ov && pending >= 0) {   // the previous half step's SVID, beside this RHS and solve
        NQ_CK(cudaEventRecord(ov->pre_rhs, s));
        NQ_CK(cudaStreamWaitEvent(ov->aux, ov->pre_rhs, 0));
        if (obj_slot >= 0) {    // the previous iteration's objective: both Grams are formed
            // (its own stream: behind the SVID passes it could hold up the next Gram)
            NQ_CK(cudaStreamWaitEvent(ov->obj, ov->pre_rhs, 0));
            if ((st = lb_objective(lb, lambda + rho, obj_slot, ov->obj))) return st;
            NQ_CK(cudaEventRecord(ov->obj_done, ov->obj));
        }
        if ((st = lb_svid(lb, pending, K, ov->aux))) return st;
        NQ_CK(cudaEventRecord(ov->svid_done[pending], ov->aux));
    }
    if (ov && wait_own) NQ_CK(cudaStreamWaitEvent(s, ov->svid_done[side], 0));

    // R = W^ X_other + rho (Z - L), split into hi + lo bf16.  FP32-accurate mode: both
    // operands split, three passes [W^_hi, W^_lo, W^_hi] . [X_hi, X_hi, X_lo].
    {
        tc::Maps maps;
        memset(&maps, 0, sizeof(maps));
        const void *A = side == 0 ? lb.p<void>(L.what) : lb.p<void>(L.whatT);
        const void *Al = side == 0 ? lb.p<void>(L.whatL) : lb.p<void>(L.whatTL);
        const int64_t lda = side == 0 ? L.ldn : L.ldm;
        const void *B = lb.p<void>(L.xt[other]), *Bl = lb.p<void>(L.xtl[other]);
        const int split = prec == NQ_PREC_FP32 ? 1 : 0;
        const void *as[2] = {A, Al}, *bs[2] = {B, Bl};
        for (int g = 0; g <= split; ++g)
            if (!tc::make_map_bf16(&maps.a[g], as[g], rows, Kd, lda, tc::BM) ||
                !tc::make_map_bf16(&maps.b[g], bs[g], L.r, Kd, L.ld_rows(other), BN))
                return NQ_ERR_CUDA;
        tc::EpiParams ep;
        memset(&ep, 0, sizeof(ep));
        ep.M = (int)rows;
        ep.N = L.r;
        ep.nseg = 1;
        ep.split3 = split;
        ep.kblocks[0] = (int)ceil_div(Kd, tc::BK);
        ep.err = &lb.sc->err;
        ep.S = lb.p<float>(L.s[side]);
        ep.a = lb.p<float>(L.a[side]);
        ep.b = lb.p<float>(L.b[side]);
        ep.ldf = L.ldr;
        ep.rho = rho;
        ep.Rhi = lb.p<__nv_bfloat16>(L.rhi);
        ep.Rlo = lb.p<__nv_bfloat16>(L.rlo);
        ep.ldr = L.ldr;
        ep.max_ctas = cc > 0 ? sms - cc : 0;
        ep.nfast = g_tune[NQ_TUNE_NFAST].load(std::memory_order_relaxed);
        ProfScope ps(NQ_K_RHS, s);
        NQ_CK(tc::launch_gemm(maps, ep, tc::EPI_RHS, BN, s));
    }
    if (cc > 0) NQ_CK(cudaStreamWaitEvent(s, sc->join, 0));
    if (gd) {
        if ((st = lb_gd_steps(lb, side, rho, prec, s))) return st;
        if (ov) return NQ_OK;
        return lb_svid(lb, side, K, s);
    }
    // X = R G^-1 = [R_hi, R_lo, R_hi] [Gi_hi; Gi_hi; Gi_lo]; S <- X + L; Xt = bf16(X)^T
    {
        tc::Maps maps;
        memset(&maps, 0, sizeof(maps));
        const void *rh = lb.p<void>(L.rhi), *rl = lb.p<void>(L.rlo);
        const void *gh = lb.p<void>(L.gih[side]), *gl = lb.p<void>(L.gil[side]);
        if (!tc::make_map_bf16(&maps.a[0], rh, rows, L.r, L.ldr, tc::BM) ||
            !tc::make_map_bf16(&maps.a[1], rl, rows, L.r, L.ldr, tc::BM) ||
            !tc::make_map_bf16(&maps.b[0], gh, L.r, L.r, L.ldr, BNs) ||
            !tc::make_map_bf16(&maps.b[1], gl, L.r, L.r, L.ldr, BNs))
            return NQ_ERR_CUDA;
        tc::EpiParams ep;
        memset(&ep, 0, sizeof(ep));
        ep.M = (int)rows;
        ep.N = L.r;
        ep.nseg = 1;
        ep.split3 = 1;
        ep.kblocks[0] = (int)ceil_div(L.r, tc::BK);
        ep.err = &lb.sc->err;
        ep.S = lb.p<float>(L.s[side]);
        ep.a = lb.p<float>(L.a[side]);
        ep.b = lb.p<float>(L.b[side]);
        ep.ldf = L.ldr;
        ep.rho = rho;
        ep.Rhi = lb.p<__nv_bfloat16>(L.rhi);
        ep.Rlo = lb.p<__nv_bfloat16>(L.rlo);
        ep.ldr = L.ldr;
        ep.X = lb.p<float>(L.x[side]);
        ep.Xt = lb.p<__nv_bfloat16>(L.xt[side]);
        ep.XtL = prec == NQ_PREC_FP32 ? lb.p<__nv_bfloat16>(L.xtl[side]) : nullptr;
        ep.ldxt = L.ld_rows(side);
        ep.objective = side == 1;
        ep.part = lb.p<double>(L.part);
        ep.nfast = g_tune[NQ_TUNE_NFAST].load(std::memory_order_relaxed);
        ProfScope ps(NQ_K_SOLVE, s);
        NQ_CK(tc::launch_gemm(maps, ep, tc::EPI_SOLVE, BNs, s));
    }
    if (ov) return NQ_OK;
    return lb_svid(lb, side, K, s);
}

nq_status lb_objective(const Lb &lb, float c, int slot, cudaStream_t s) {
    const LbLayout &L = lb.L;
    const int npx = (int)tc::num_tiles((int)L.n, L.r, solve_bn(L.r));
    ProfScope ps(NQ_K_OBJ, s);
    NQ_CK(objective(lb.p<float>(L.g[0]), lb.p<float>(L.g[1]), L.r, c, lb.p<double>(L.part), npx,
                    lb.p<double>(L.partg), lb.sc, lb.p<float>(L.obj) + slot, s));
    return NQ_OK;
}

nq_status lb_prepare(const Lb &lb, const void *W, int bf16, const float *d_in,
                     const float *d_out, uint64_t seed, int prec, cudaStream_t s) {
    const bool split = prec == NQ_PREC_FP32;
    const LbLayout &L = lb.L;
    ProfScope ps(NQ_K_PREP, s);
    NQ_CK(cudaMemsetAsync(lb.sc, 0, sizeof(Scalars), s));
    NQ_CK(wt_norm_partials(W, bf16, L.m, L.n, d_in, d_out, lb.p<double>(L.part), &lb.sc->err, s));
    NQ_CK(reduce_partials(lb.p<double>(L.part), kRedBlocks, &lb.sc->wt_norm2, &lb.sc->gamma, L.r,
                          s));
    NQ_CK(what_cast(W, bf16, L.m, L.n, d_in, d_out, &lb.sc->gamma, lb.p<__nv_bfloat16>(L.what),
                    L.ldn, lb.p<__nv_bfloat16>(L.whatT), L.ldm,
                    split ? lb.p<__nv_bfloat16>(L.whatL) : nullptr,
                    split ? lb.p<__nv_bfloat16>(L.whatTL) : nullptr, lb.p<double>(L.part), s));
    NQ_CK(reduce_partials(lb.p<double>(L.part), kRedBlocks, &lb.sc->what_norm2, nullptr, L.r, s));
    for (int sd = 0; sd < 2; ++sd) {
        const int64_t rw = L.rows(sd);
        NQ_CK(cudaMemsetAsync(lb.p<void>(L.s[sd]), 0, (size_t)rw * L.ldr * 4, s));
        NQ_CK(cudaMemsetAsync(lb.p<void>(L.a[sd]), 0, (size_t)rw * 4, s));
        NQ_CK(cudaMemsetAsync(lb.p<void>(L.b[sd]), 0, (size_t)L.r * 4, s));
        NQ_CK(cudaMemsetAsync(lb.p<void>(L.xt[sd]), 0, (size_t)L.r * L.ld_rows(sd) * 2, s));
        NQ_CK(cudaMemsetAsync(lb.p<void>(L.xtl[sd]), 0, (size_t)L.r * L.ld_rows(sd) * 2, s));
    }
    if (!split) {   // the low parts read as zero (state fields, precision switches)
        NQ_CK(cudaMemsetAsync(lb.p<void>(L.whatL), 0, (size_t)L.m * L.ldn * 2, s));
        NQ_CK(cudaMemsetAsync(lb.p<void>(L.whatTL), 0, (size_t)L.n * L.ldm * 2, s));
    }
    NQ_CK(cudaMemsetAsync(lb.p<void>(L.x[0]), 0, (size_t)L.m * L.ldr * 4, s));
    NQ_CK(cudaMemsetAsync(lb.p<void>(L.x[1]), 0, (size_t)L.n * L.ldr * 4, s));
    // no previous G^-1 yet: zero (a Newton-Schulz start of 0 fails at once)
    for (int sd = 0; sd < 2; ++sd) {
        NQ_CK(cudaMemsetAsync(lb.p<void>(L.gih[sd]), 0, (size_t)L.r * L.ldr * 2, s));
        NQ_CK(cudaMemsetAsync(lb.p<void>(L.gil[sd]), 0, (size_t)L.r * L.ldr * 2, s));
    }
    NQ_CK(cudaMemsetAsync(lb.p<void>(L.ns), 0, sizeof(NsState), s));
    add_iters(lb.ws, -1);
    NQ_CK(init_v0(L.n, L.r, seed, lb.p<float>(L.x[1]), L.ldr, lb.p<__nv_bfloat16>(L.xt[1]),
                  split ? lb.p<__nv_bfloat16>(L.xtl[1]) : nullptr, L.ldn, s));
    return NQ_OK;
}

// After the iterations: the objective of the last one (it needs the Gram of the last V)
// and the copy of the objectives not copied yet.
nq_status lb_iterate_tail(const Lb &lb, float rho, float lambda, int iters, int prec,
                          float *objective_h, cudaStream_t s) {
    nq_status st = lb_gram(lb, 1, lambda + rho, prec, s);
    if (st) return st;
    if ((st = lb_objective(lb, lambda + rho, (iters - 1) % kObjRing, s))) return st;
    if (objective_h) {
        const int done = (iters - 1) / kObjRing * kObjRing;
        NQ_CK(cudaMemcpyAsync(objective_h + done, lb.p<float>(lb.L.obj),
                              (size_t)(iters - done) * 4, cudaMemcpyDeviceToHost, s));
    }
    return NQ_OK;
}

// The iterations.  The SVID of the side just solved is needed only by that side's next
// RHS GEMM, one half step later, so it runs on the auxiliary stream beside the next half
// step's RHS GEMM and solve; the last one runs on ``s`` before returning.  The objective of
// iteration t - 1 needs both Grams, the second formed at the start of iteration t: it runs
// on a stream of its own beside the U half step, before the next Gram of U overwrites the
// first.
nq_status lb_iterate(const Lb &lb, float rho, float lambda, int iters, int K, int prec,
                     float *objective_h, cudaStream_t s) {
    SideCtx *ov = nullptr;
    nq_status st = side_ctx(&ov);
    if (st) return st;
    if (!g_tune[NQ_TUNE_SVID_BESIDE].load(std::memory_order_relaxed)) {
        // every SVID right after its solve, on ``s``
        for (int t = 0; t < iters; ++t) {
            if ((st = lb_half_step(lb, 0, rho, lambda, K, prec, s))) return st;
            if (t > 0 && (st = lb_objective(lb, lambda + rho, (t - 1) % kObjRing, s))) return st;
            if ((st = lb_half_step(lb, 1, rho, lambda, K, prec, s))) return st;
            add_iters(lb.ws, 1);
            if (objective_h && t > 0 && (t % kObjRing) == 0)
                NQ_CK(cudaMemcpyAsync(objective_h + (t - kObjRing), lb.p<float>(lb.L.obj),
                                      (size_t)kObjRing * 4, cudaMemcpyDeviceToHost, s));
        }
        return lb_iterate_tail(lb, rho, lambda, iters, prec, objective_h, s);
    }
    for (int t = 0; t < iters; ++t) {
        // U side: starts the objective of the previous iteration and the SVID of V (solved
        // by the previous half step; none at t = 0) on the auxiliary stream
        st = lb_half_step(lb, 0, rho, lambda, K, prec, s, ov, t > 0 ? 1 : -1, t > 0,
                          t > 0 ? (t - 1) % kObjRing : -1);
        if (st) return st;
        // V side: starts the SVID of U, waits for its own from the previous iteration; its
        // Gram waits for that objective
        if ((st = lb_half_step(lb, 1, rho, lambda, K, prec, s, ov, 0, t > 0, -1, t > 0)))
            return st;
        add_iters(lb.ws, 1);
        if (objective_h && t > 0 && (t % kObjRing) == 0) {
            // the ring holds the objectives of iterations t - kObjRing .. t - 1; the copy is
            // stream-ordered before the next write to slot 0
            NQ_CK(cudaMemcpyAsync(objective_h + (t - kObjRing), lb.p<float>(lb.L.obj),
                                  (size_t)kObjRing * 4, cudaMemcpyDeviceToHost, s));
        }
    }
    // join the auxiliary stream (the last SVID of U; the SVID scratch is shared) and the
    // objective stream, then the last SVID of V
    NQ_CK(cudaStreamWaitEvent(s, ov->svid_done[0], 0));
    if (iters > 1) NQ_CK(cudaStreamWaitEvent(s, ov->obj_done, 0));
    if ((st = lb_svid(lb, 1, K, s))) return st;
    return lb_iterate_tail(lb, rho, lambda, iters, prec, objective_h, s);
}

nq_status lb_finish(const Lb &lb, const void *W, int bf16, const float *d_in, const float *d_out,
                    uint32_t *Up, uint32_t *Vp, float *s1, float *s2, bool want_err,
                    cudaStream_t s) {
    const LbLayout &L = lb.L;
    float *pu = lb.p<float>(L.partb);
    float *pv = pu + (size_t)L.nsv * L.r;
    {
    ProfScope ps(NQ_K_FINISH, s);
    NQ_CK(column_sumsq(lb.p<float>(L.x[0]), L.m, L.r, L.ldr, L.nsv, pu, s));
    NQ_CK(column_sumsq(lb.p<float>(L.x[1]), L.n, L.r, L.ldr, L.nsv, pv, s));
    NQ_CK(balance_gains(pu, pv, L.nsv, L.r, lb.p<float>(L.gk), s));
    NQ_CK(extract_pack(lb.p<float>(L.x[0]), L.m, L.r, L.ldr, lb.p<float>(L.gk), 0, &lb.sc->gamma,
                       s1, Up, lb.p<__nv_bfloat16>(L.rhi), L.ldr, s));
    NQ_CK(extract_pack(lb.p<float>(L.x[1]), L.n, L.r, L.ldr, lb.p<float>(L.gk), 1, nullptr, s2, Vp,
                       lb.p<__nv_bfloat16>(L.rlo), L.ldr, s));
    }
    if (!want_err) return NQ_OK;
    ProfScope ps(NQ_K_RECON, s);
    const int BN = pick_bn(L.n);
    tc::Maps maps;
    memset(&maps, 0, sizeof(maps));
    if (!tc::make_map_bf16(&maps.a[0], lb.p<void>(L.rhi), L.m, L.r, L.ldr, tc::BM) ||
        !tc::make_map_bf16(&maps.b[0], lb.p<void>(L.rlo), L.n, L.r, L.ldr, BN))
        return NQ_ERR_CUDA;
    tc::EpiParams ep;
    memset(&ep, 0, sizeof(ep));
    ep.M = (int)L.m;
    ep.N = (int)L.n;
    ep.nseg = 1;
    ep.kblocks[0] = (int)ceil_div(L.r, tc::BK);
    ep.err = &lb.sc->err;
    ep.part = lb.p<double>(L.part);
    ep.W = W;
    ep.w_bf16 = bf16;
    ep.w_vec = (reinterpret_cast<uintptr_t>(W) % 16 == 0) && ((L.n * (bf16 ? 2 : 4)) % 16 == 0);
    ep.ldw = L.n;
    ep.d_in = d_in;
    ep.d_out = d_out;
    ep.s1 = s1;
    ep.s2 = s2;
    ep.cvec = vec16(d_in) && vec16(s2);
    NQ_CK(tc::launch_gemm(maps, ep, tc::EPI_RECON, BN, s));
    NQ_CK(recon_finalize(lb.p<double>(L.part), (int)tc::num_tiles((int)L.m, (int)L.n, BN), lb.sc,
                         &lb.sc->recon2, s));
    return NQ_OK;
}

}  // namespace

// =====================================================================================
// Public entry points
// =====================================================================================
extern "C" {

const char *nq_status_string(nq_status s) {
    switch (s) {
        case NQ_OK: return "NQ_OK";
        case NQ_ERR_INVALID_ARG: return "NQ_ERR_INVALID_ARG";
        case NQ_ERR_WORKSPACE: return "NQ_ERR_WORKSPACE";
        case NQ_ERR_CUDA: return "NQ_ERR_CUDA";
        case NQ_ERR_NONFINITE: return "NQ_ERR_NONFINITE";
        case NQ_ERR_NOT_SPD: return "NQ_ERR_NOT_SPD";
        case NQ_ERR_TIMEOUT: return "NQ_ERR_TIMEOUT";
        case NQ_ERR_UNSUPPORTED: return "NQ_ERR_UNSUPPORTED";
        default: return "NQ_ERR_UNKNOWN";
    }
}

int32_t nq_version(void) { return 100; }

double nq_bpw(int64_t m, int64_t n, int32_t r) {
    if (m <= 0 || n <= 0 || r < 0) return -1.0;
    return ((double)(m + n) * r + 16.0 * (double)(m + n)) / ((double)m * (double)n);
}

int32_t nq_rank_for_bpw(int64_t m, int64_t n, double bpw) {
    if (m <= 0 || n <= 0 || !(bpw >= 0.0)) return -1;
    const long double x =
        ((long double)bpw * (long double)m * (long double)n - 16.0L * (long double)(m + n)) /
        (long double)(m + n);
    long double f = floorl(x);
    if (x - f > 1.0L - 1e-9L) f += 1.0L;  // a decimal bpw landing just below an integer
    if (f < 0) return 0;
    if (f > 2147483647.0L) return 2147483647;
    return (int32_t)f;
}

size_t nq_calib_workspace_size(int64_t T, int64_t C) {
    if (T < 1 || C < 1) return 0;
    return calib_ws_bytes(C);
}

nq_status nq_calib_stats(const void *X, int64_t T, int64_t C, nq_dtype dt, double *s, double *q,
                         void *ws, size_t ws_bytes, nq_stream_t stream) {
    if (!X || !s || !q || T < 1 || C < 1 || (dt != NQ_F32 && dt != NQ_BF16))
        return NQ_ERR_INVALID_ARG;
    nq_status st = check_ws(ws, ws_bytes, calib_ws_bytes(C));
    if (st) return st;
    if ((st = check_device())) return st;
    CalibCarve cv = carve_calib(ws, C);
    return enqueue_stats(X, T, C, dt == NQ_BF16, s, q, cv, cs(stream));
}

nq_status nq_calib_precond(const void *acts, int64_t T_in, int64_t n, const void *grads,
                           int64_t T_out, int64_t m, nq_dtype dt, double alpha_override,
                           float *d_in, float *d_out, double *alpha_out, void *ws,
                           size_t ws_bytes, nq_stream_t stream) {
    if (!acts || !grads || !d_in || !d_out || T_in < 1 || T_out < 1 || n < 1 || m < 1 ||
        (dt != NQ_F32 && dt != NQ_BF16) || !(alpha_override <= 1.0) || isnan(alpha_override))
        return NQ_ERR_INVALID_ARG;
    const int64_t C = n > m ? n : m;
    nq_status st = check_ws(ws, ws_bytes, calib_ws_bytes(C));
    if (st) return st;
    if ((st = check_device())) return st;
    cudaStream_t s = cs(stream);
    CalibCarve cv = carve_calib(ws, C);
    NQ_CK(cudaMemsetAsync(cv.sc, 0, sizeof(Scalars), s));
    const int bf16 = dt == NQ_BF16;
    if ((st = enqueue_stats(acts, T_in, n, bf16, cv.s, cv.q, cv, s))) return st;
    {
        ProfScope ps(NQ_K_CALIB_FIN, s);
        NQ_CK(calib_ledoit_wolf(cv.s, cv.q, T_in, n, alpha_override, d_in, &cv.sc->alpha[0],
                                &cv.sc->err, s));
    }
    if ((st = enqueue_stats(grads, T_out, m, bf16, cv.s, cv.q, cv, s))) return st;
    {
        ProfScope ps(NQ_K_CALIB_FIN, s);
        NQ_CK(calib_ledoit_wolf(cv.s, cv.q, T_out, m, alpha_override, d_out, &cv.sc->alpha[1],
                                &cv.sc->err, s));
    }
    if (alpha_out) {
        Scalars h;
        NQ_CK(cudaMemcpyAsync(&h, cv.sc, sizeof(Scalars), cudaMemcpyDeviceToHost, s));
        NQ_CK(cudaStreamSynchronize(s));
        alpha_out[0] = h.alpha[0];
        alpha_out[1] = h.alpha[1];
        if (h.err) return static_cast<nq_status>(h.err);
    }
    return NQ_OK;
}

nq_status nq_set_tuning(nq_tuning key, int32_t value) {
    switch (key) {
        case NQ_TUNE_FACTOR_CTAS:
            if (value < -1) return NQ_ERR_INVALID_ARG;
            break;
        case NQ_TUNE_NEWTON_BN:
            if (value != 0 && value != 64 && value != 128 && value != 256) return NQ_ERR_INVALID_ARG;
            break;
        case NQ_TUNE_RHS_BN:
        case NQ_TUNE_SOLVE_BN:
            if (value != 0 && value != 128 && value != 256) return NQ_ERR_INVALID_ARG;
            break;
        case NQ_TUNE_SVID_BESIDE:
        case NQ_TUNE_NFAST:
        case NQ_TUNE_NEWTON_FUSED:
            if (value != 0 && value != 1) return NQ_ERR_INVALID_ARG;
            break;
        default: return NQ_ERR_INVALID_ARG;
    }
    g_tune[key].store(value, std::memory_order_relaxed);
    return NQ_OK;
}

nq_status nq_set_latent_solver(nq_latent_solver solver, int32_t gd_steps) {
    if (solver != NQ_SOLVER_EXACT && solver != NQ_SOLVER_GD) return NQ_ERR_INVALID_ARG;
    if (solver == NQ_SOLVER_GD && (gd_steps < 1 || gd_steps > 1000)) return NQ_ERR_INVALID_ARG;
    if (solver == NQ_SOLVER_GD) g_gd_steps.store(gd_steps, std::memory_order_relaxed);
    g_solver.store(solver, std::memory_order_relaxed);
    return NQ_OK;
}

nq_status nq_set_inverse_mode(nq_inverse_mode mode) {
    if (mode != NQ_INV_AUTO && mode != NQ_INV_CHOLESKY && mode != NQ_INV_NEWTON)
        return NQ_ERR_INVALID_ARG;
    g_inverse_mode.store(mode, std::memory_order_relaxed);
    return NQ_OK;
}

size_t nq_lbadmm_workspace_size(int64_t m, int64_t n, int32_t r) {
    if (check_lb_args(m, n, r)) return 0;
    LbLayout L;
    L.build(m, n, r);
    return L.total;
}

nq_status nq_lbadmm_prepare(const void *W, nq_dtype dt, int64_t m, int64_t n, const float *d_in,
                            const float *d_out, int32_t r, uint64_t seed, nq_precision prec,
                            double *gamma_out, void *ws, size_t ws_bytes, nq_stream_t stream) {
    if (!W || (dt != NQ_F32 && dt != NQ_BF16) || !valid_prec(prec)) return NQ_ERR_INVALID_ARG;
    Lb lb;
    nq_status st = lb_open(lb, m, n, r, ws, ws_bytes);
    if (st) return st;
    cudaStream_t s = cs(stream);
    if ((st = lb_prepare(lb, W, dt == NQ_BF16, d_in, d_out, seed, prec, s))) return st;
    if (gamma_out) {
        NQ_CK(cudaMemcpyAsync(gamma_out, &lb.sc->gamma, sizeof(double), cudaMemcpyDeviceToHost, s));
        return read_err(&lb.sc->err, s, false);
    }
    return NQ_OK;
}

nq_status nq_lbadmm_iterate(int64_t m, int64_t n, int32_t r, float rho, float lambda,
                            int32_t iters, int32_t K, nq_precision prec, float *objective,
                            void *ws, size_t ws_bytes, nq_stream_t stream) {
    if (!(rho > 0.f) || !(lambda >= 0.f) || iters < 1 || K < 1 || !isfinite(rho) ||
        !isfinite(lambda) || !valid_prec(prec))
        return NQ_ERR_INVALID_ARG;
    Lb lb;
    nq_status st = lb_open(lb, m, n, r, ws, ws_bytes);
    if (st) return st;
    cudaStream_t s = cs(stream);
    if ((st = lb_iterate(lb, rho, lambda, iters, K, prec, objective, s))) return st;
    if (objective) return read_err(&lb.sc->err, s, false);
    return NQ_OK;
}

nq_status nq_lbadmm_half_step(int64_t m, int64_t n, int32_t r, float rho, float lambda, int32_t K,
                              int32_t side, nq_precision prec, void *ws, size_t ws_bytes,
                              nq_stream_t stream) {
    if (!(rho > 0.f) || !(lambda >= 0.f) || K < 1 || (side != 0 && side != 1) ||
        !valid_prec(prec))
        return NQ_ERR_INVALID_ARG;
    Lb lb;
    nq_status st = lb_open(lb, m, n, r, ws, ws_bytes);
    if (st) return st;
    return lb_half_step(lb, side, rho, lambda, K, prec, cs(stream));
}

nq_status nq_lbadmm_finish(const void *W, nq_dtype dt, int64_t m, int64_t n, const float *d_in,
                           const float *d_out, int32_t r, uint32_t *U_packed, uint32_t *V_packed,
                           float *s1, float *s2, float *final_rel_err, void *ws, size_t ws_bytes,
                           nq_stream_t stream) {
    if (!U_packed || !V_packed || !s1 || !s2 || (final_rel_err && !W) ||
        (dt != NQ_F32 && dt != NQ_BF16))
        return NQ_ERR_INVALID_ARG;
    Lb lb;
    nq_status st = lb_open(lb, m, n, r, ws, ws_bytes);
    if (st) return st;
    cudaStream_t s = cs(stream);
    if ((st = lb_finish(lb, W, dt == NQ_BF16, d_in, d_out, U_packed, V_packed, s1, s2,
                        final_rel_err != nullptr, s)))
        return st;
    if (final_rel_err) {
        double e = 0.0;
        NQ_CK(cudaMemcpyAsync(&e, &lb.sc->recon2, sizeof(double), cudaMemcpyDeviceToHost, s));
        st = read_err(&lb.sc->err, s, false);
        *final_rel_err = (float)e;
        return st;
    }
    return NQ_OK;
}

nq_status nq_lbadmm(const void *W, nq_dtype dt, int64_t m, int64_t n, const float *d_in,
                    const float *d_out, int32_t r, float rho, float lambda, int32_t iters,
                    int32_t K, uint64_t seed, uint32_t *U_packed, uint32_t *V_packed, float *s1,
                    float *s2, float *objective, float *final_rel_err, void *ws,
                    size_t ws_bytes, nq_stream_t stream) {
    if (!W || !U_packed || !V_packed || !s1 || !s2 || (dt != NQ_F32 && dt != NQ_BF16) ||
        !(rho > 0.f) || !(lambda >= 0.f) || iters < 1 || K < 1 || !isfinite(rho) ||
        !isfinite(lambda))
        return NQ_ERR_INVALID_ARG;
    Lb lb;
    nq_status st = lb_open(lb, m, n, r, ws, ws_bytes);
    if (st) return st;
    cudaStream_t s = cs(stream);
    const int bf16 = dt == NQ_BF16;
    // precision follows the weights: BF16 operands for BF16 weights, split (FP32-accurate)
    // operands for FP32 weights
    const int prec = bf16 ? NQ_PREC_BF16 : NQ_PREC_FP32;
    if ((st = lb_prepare(lb, W, bf16, d_in, d_out, seed, prec, s))) return st;
    if ((st = lb_iterate(lb, rho, lambda, iters, K, prec, objective, s))) return st;
    if ((st = lb_finish(lb, W, bf16, d_in, d_out, U_packed, V_packed, s1, s2,
                        final_rel_err != nullptr, s)))
        return st;
    if (final_rel_err || objective) {
        double e = 0.0;
        NQ_CK(cudaMemcpyAsync(&e, &lb.sc->recon2, sizeof(double), cudaMemcpyDeviceToHost, s));
        st = read_err(&lb.sc->err, s, false);
        if (final_rel_err) *final_rel_err = (float)e;
        return st;
    }
    return NQ_OK;
}

size_t nq_recon_workspace_size(int64_t m, int64_t n, int32_t r) {
    if (check_lb_args(m, n, r)) return 0;
    ReconLayout L;
    L.build(m, n, r);
    return L.total;
}

// ||W~ - diag(s1) U+- V+-^T diag(s2)|| / ||W~|| into sc->recon2 from the +-1 BF16
// operands up (m x r) and vp (n x r), row stride ldr.
static nq_status enqueue_recon(const void *W, nq_dtype dt, int64_t m, int64_t n,
                               const float *d_in, const float *d_out, const __nv_bfloat16 *up,
                               const __nv_bfloat16 *vp, int64_t ldr, int32_t r, const float *s1,
                               const float *s2, Scalars *sc, double *part, cudaStream_t s) {
    NQ_CK(wt_norm_partials(W, dt == NQ_BF16, m, n, d_in, d_out, part, &sc->err, s));
    NQ_CK(reduce_partials(part, kRedBlocks, &sc->wt_norm2, nullptr, r, s));
    const int BN = pick_bn(n);
    tc::Maps maps;
    memset(&maps, 0, sizeof(maps));
    if (!tc::make_map_bf16(&maps.a[0], up, m, r, ldr, tc::BM) ||
        !tc::make_map_bf16(&maps.b[0], vp, n, r, ldr, BN))
        return NQ_ERR_CUDA;
    tc::EpiParams ep;
    memset(&ep, 0, sizeof(ep));
    ep.M = (int)m;
    ep.N = (int)n;
    ep.nseg = 1;
    ep.kblocks[0] = (int)ceil_div(r, tc::BK);
    ep.err = &sc->err;
    ep.part = part;
    ep.W = W;
    ep.w_bf16 = dt == NQ_BF16;
    ep.w_vec = (reinterpret_cast<uintptr_t>(W) % 16 == 0) && ((n * (dt == NQ_BF16 ? 2 : 4)) % 16 == 0);
    ep.ldw = n;
    ep.d_in = d_in;
    ep.d_out = d_out;
    ep.s1 = s1;
    ep.s2 = s2;
    ep.cvec = vec16(d_in) && vec16(s2);
    NQ_CK(tc::launch_gemm(maps, ep, tc::EPI_RECON, BN, s));
    NQ_CK(recon_finalize(part, (int)tc::num_tiles((int)m, (int)n, BN), sc, &sc->recon2, s));
    return NQ_OK;
}

nq_status nq_recon_error(const void *W, nq_dtype dt, int64_t m, int64_t n, const float *d_in,
                         const float *d_out, const uint32_t *U_packed, const uint32_t *V_packed,
                         int32_t r, const float *s1, const float *s2, double *rel_err, void *ws,
                         size_t ws_bytes, nq_stream_t stream) {
    if (!W || !U_packed || !V_packed || !s1 || !s2 || !rel_err ||
        (dt != NQ_F32 && dt != NQ_BF16))
        return NQ_ERR_INVALID_ARG;
    nq_status st = check_lb_args(m, n, r);
    if (st) return st;
    ReconLayout L;
    L.build(m, n, r);
    if ((st = check_ws(ws, ws_bytes, L.total))) return st;
    if ((st = check_device())) return st;
    cudaStream_t s = cs(stream);
    Scalars *sc = at<Scalars>(ws, L.scal);
    double *part = at<double>(ws, L.part);
    __nv_bfloat16 *up = at<__nv_bfloat16>(ws, L.up), *vp = at<__nv_bfloat16>(ws, L.vp);
    NQ_CK(cudaMemsetAsync(sc, 0, sizeof(Scalars), s));
    NQ_CK(unpack_pm(U_packed, m, r, up, L.ldr, s));
    NQ_CK(unpack_pm(V_packed, n, r, vp, L.ldr, s));
    if ((st = enqueue_recon(W, dt, m, n, d_in, d_out, up, vp, L.ldr, r, s1, s2, sc, part, s)))
        return st;
    NQ_CK(cudaMemcpyAsync(rel_err, &sc->recon2, sizeof(double), cudaMemcpyDeviceToHost, s));
    return read_err(&sc->err, s, false);
}

size_t nq_ls_refit_workspace_size(int64_t m, int64_t n, int32_t r) {
    if (check_lb_args(m, n, r)) return 0;
    RefitLayout L;
    L.build(m, n, r);
    return L.total;
}

nq_status nq_ls_refit(const void *W, nq_dtype dt, int64_t m, int64_t n, const float *d_in,
                      const float *d_out, const uint32_t *U_packed, const uint32_t *V_packed,
                      int32_t r, float *s1, float *s2, int32_t sweeps, double *rel_err,
                      void *ws, size_t ws_bytes, nq_stream_t stream) {
    if (!W || !U_packed || !V_packed || !s1 || !s2 || sweeps < 1 ||
        (dt != NQ_F32 && dt != NQ_BF16))
        return NQ_ERR_INVALID_ARG;
    nq_status st = check_lb_args(m, n, r);
    if (st) return st;
    RefitLayout L;
    L.build(m, n, r);
    if ((st = check_ws(ws, ws_bytes, L.total))) return st;
    if ((st = check_device())) return st;
    cudaStream_t s = cs(stream);
    Scalars *sc = at<Scalars>(ws, L.scal);
    __nv_bfloat16 *up = at<__nv_bfloat16>(ws, L.up), *vp = at<__nv_bfloat16>(ws, L.vp);
    double *num = at<double>(ws, L.num), *den = at<double>(ws, L.den);
    ProfScope ps(NQ_K_REFIT, s);
    NQ_CK(cudaMemsetAsync(sc, 0, sizeof(Scalars), s));
    NQ_CK(unpack_pm(U_packed, m, r, up, L.ldr, s));
    NQ_CK(unpack_pm(V_packed, n, r, vp, L.ldr, s));
    const bool wv = (reinterpret_cast<uintptr_t>(W) % 16 == 0) && ((n * (dt == NQ_BF16 ? 2 : 4)) % 16 == 0);
    for (int sw = 0; sw < sweeps; ++sw) {
        for (int pass = 0; pass < 2; ++pass) {
            // pass 0: rows i of W (s1, sums over j with s2); pass 1: columns j (s2, over i)
            const int64_t M = pass == 0 ? m : n, N = pass == 0 ? n : m;
            const __nv_bfloat16 *A = pass == 0 ? up : vp, *Bm = pass == 0 ? vp : up;
            const int BN = pick_bn(N) < 64 ? 64 : pick_bn(N);
            tc::Maps maps;
            memset(&maps, 0, sizeof(maps));
            if (!tc::make_map_bf16(&maps.a[0], A, M, r, L.ldr, tc::BM) ||
                !tc::make_map_bf16(&maps.b[0], Bm, N, r, L.ldr, BN))
                return NQ_ERR_CUDA;
            tc::EpiParams ep;
            memset(&ep, 0, sizeof(ep));
            ep.M = (int)M;
            ep.N = (int)N;
            ep.nseg = 1;
            ep.kblocks[0] = (int)ceil_div(r, tc::BK);
            ep.err = &sc->err;
            ep.W = W;
            ep.w_bf16 = dt == NQ_BF16;
            ep.w_vec = wv;
            ep.ldw = n;
            ep.d_in = d_in;
            ep.d_out = d_out;
            ep.refit_trans = pass;
            ep.sv = pass == 0 ? s2 : s1;
            ep.cvec = vec16(pass == 0 ? d_in : d_out) && vec16(ep.sv);
            ep.num = num;
            ep.den = den;
            NQ_CK(tc::launch_gemm(maps, ep, tc::EPI_REFIT, BN, s));
            NQ_CK(refit_scales(num, den, (int)ceil_div(N, BN), M, pass == 0 ? s1 : s2, s));
        }
    }
    if (!rel_err) return NQ_OK;
    if ((st = enqueue_recon(W, dt, m, n, d_in, d_out, up, vp, L.ldr, r, s1, s2, sc,
                            at<double>(ws, L.part), s)))
        return st;
    NQ_CK(cudaMemcpyAsync(rel_err, &sc->recon2, sizeof(double), cudaMemcpyDeviceToHost, s));
    return read_err(&sc->err, s, false);
}

static bool binary_args_ok(int64_t m, int64_t n, int32_t r, int64_t B) {
    return m >= 1 && n >= 1 && m <= kMaxDim && n <= kMaxDim && r >= 1 && r <= kMaxRank &&
           B >= 1 && B <= kMaxDim;
}

size_t nq_binary_workspace_size(int64_t m, int64_t n, int32_t r, int64_t B) {
    if (!binary_args_ok(m, n, r, B)) return 0;
    BinLayout L;
    L.build(m, n, r, B, NQ_BINARY_GEMV_MAX_BATCH, bin_gemv_chunks(n, r, B));
    return L.total;
}

nq_status nq_binary_matmul(const uint32_t *U_packed, const uint32_t *V_packed, const float *s1,
                           const float *s2, int64_t m, int64_t n, int32_t r, const void *X,
                           nq_dtype dt, int64_t B, float *Y, void *ws, size_t ws_bytes,
                           nq_stream_t stream) {
    if (!U_packed || !V_packed || !s1 || !s2 || !X || !Y || (dt != NQ_F32 && dt != NQ_BF16) ||
        !binary_args_ok(m, n, r, B))
        return NQ_ERR_INVALID_ARG;
    BinLayout L;
    L.build(m, n, r, B, NQ_BINARY_GEMV_MAX_BATCH, bin_gemv_chunks(n, r, B));
    nq_status st = check_ws(ws, ws_bytes, L.total);
    if (st) return st;
    if ((st = check_device())) return st;
    cudaStream_t s = cs(stream);
    const int xb = dt == NQ_BF16;
    Scalars *sc = at<Scalars>(ws, L.scal);
    ProfScope ps(NQ_K_BINARY, s);
    if (B <= NQ_BINARY_GEMV_MAX_BATCH) {
        NQ_CK(bin_gemv(U_packed, V_packed, s1, s2, m, n, r, X, xb, B, Y, at<float>(ws, L.P),
                       at<float>(ws, L.z), s));
        return NQ_OK;
    }
    __nv_bfloat16 *vh = at<__nv_bfloat16>(ws, L.vh), *vl = at<__nv_bfloat16>(ws, L.vl),
                  *um = at<__nv_bfloat16>(ws, L.um), *xh = at<__nv_bfloat16>(ws, L.xh),
                  *xl = at<__nv_bfloat16>(ws, L.xl), *zh = at<__nv_bfloat16>(ws, L.zh),
                  *zl = at<__nv_bfloat16>(ws, L.zl);
    NQ_CK(cudaMemsetAsync(sc, 0, sizeof(Scalars), s));
    NQ_CK(bin_expand(U_packed, V_packed, s2, m, n, r, X, xb, B, vh, vl, L.ldt, um, L.ldr, xh, xl,
                     L.ldt, s));
    // Z = X diag(s2) V+- (B x r) with split operands, written as BF16 hi + lo
    {
        tc::Maps maps;
        memset(&maps, 0, sizeof(maps));
        const int nseg = xb ? 2 : 3;
        const void *as[3] = {xh, xb ? xh : xl, xh}, *bs[3] = {vh, xb ? vl : vh, vl};
        const int BN = pick_bn_fill(B, r, device_sm_count());
        for (int g = 0; g < nseg; ++g)
            if (!tc::make_map_bf16(&maps.a[g], as[g], B, n, L.ldt, tc::BM) ||
                !tc::make_map_bf16(&maps.b[g], bs[g], r, n, L.ldt, BN))
                return NQ_ERR_CUDA;
        tc::EpiParams ep;
        memset(&ep, 0, sizeof(ep));
        ep.M = (int)B;
        ep.N = r;
        ep.nseg = nseg;
        for (int g = 0; g < nseg; ++g) ep.kblocks[g] = (int)ceil_div(n, tc::BK);
        ep.err = &sc->err;
        ep.Rhi = zh;
        ep.Rlo = zl;
        ep.ldr = L.ldr;
        NQ_CK(tc::launch_gemm(maps, ep, tc::EPI_SPLIT, BN, s));
    }
    // Y = (Z_hi + Z_lo) U+-^T diag(s1) (B x m)
    {
        tc::Maps maps;
        memset(&maps, 0, sizeof(maps));
        const int BN = pick_bn_fill(B, m, device_sm_count());
        if (!tc::make_map_bf16(&maps.a[0], zh, B, r, L.ldr, tc::BM) ||
            !tc::make_map_bf16(&maps.a[1], zl, B, r, L.ldr, tc::BM) ||
            !tc::make_map_bf16(&maps.b[0], um, m, r, L.ldr, BN) ||
            !tc::make_map_bf16(&maps.b[1], um, m, r, L.ldr, BN))
            return NQ_ERR_CUDA;
        tc::EpiParams ep;
        memset(&ep, 0, sizeof(ep));
        ep.M = (int)B;
        ep.N = (int)m;
        ep.nseg = 2;
        ep.kblocks[0] = ep.kblocks[1] = (int)ceil_div(r, tc::BK);
        ep.err = &sc->err;
        ep.out = Y;
        ep.ldo = m;
        ep.s1 = s1;
        NQ_CK(tc::launch_gemm(maps, ep, tc::EPI_SCALE, BN, s));
    }
    return NQ_OK;
}

nq_status nq_pack_signs(const float *X, int64_t rows, int32_t r, uint32_t *bits,
                        nq_stream_t stream) {
    if (!X || !bits || rows < 1 || r < 1) return NQ_ERR_INVALID_ARG;
    nq_status st = check_device();
    if (st) return st;
    NQ_CK(pack_signs(X, rows, r, r, bits, cs(stream)));
    return NQ_OK;
}

nq_status nq_lbadmm_state_field(int64_t m, int64_t n, int32_t r, nq_field f, void *ws,
                                size_t ws_bytes, void **dev_ptr, int64_t *count,
                                int32_t *elem_bytes, int64_t *ld) {
    if (!dev_ptr || !count || !elem_bytes || !ld) return NQ_ERR_INVALID_ARG;
    nq_status st = check_lb_args(m, n, r);
    if (st) return st;
    LbLayout L;
    L.build(m, n, r);
    if ((st = check_ws(ws, ws_bytes, L.total))) return st;
    size_t off = 0;
    int64_t cnt = 0, l = 0;
    int32_t eb = 4;
    switch (f) {
        case NQ_FIELD_U: off = L.x[0]; cnt = m * L.ldr; l = L.ldr; break;
        case NQ_FIELD_V: off = L.x[1]; cnt = n * L.ldr; l = L.ldr; break;
        case NQ_FIELD_SU: off = L.s[0]; cnt = m * L.ldr; l = L.ldr; break;
        case NQ_FIELD_SV: off = L.s[1]; cnt = n * L.ldr; l = L.ldr; break;
        case NQ_FIELD_AU: off = L.a[0]; cnt = m; l = 1; break;
        case NQ_FIELD_AV: off = L.a[1]; cnt = n; l = 1; break;
        case NQ_FIELD_BU: off = L.b[0]; cnt = r; l = 1; break;
        case NQ_FIELD_BV: off = L.b[1]; cnt = r; l = 1; break;
        case NQ_FIELD_WHAT: off = L.what; cnt = m * L.ldn; l = L.ldn; eb = 2; break;
        case NQ_FIELD_WHAT_LO: off = L.whatL; cnt = m * L.ldn; l = L.ldn; eb = 2; break;
        case NQ_FIELD_GAMMA: off = L.scal + offsetof(Scalars, gamma); cnt = 1; l = 1; eb = 8; break;
        case NQ_FIELD_INV_STATS: off = L.ns; cnt = 3 + kNsMaxSteps + 2; l = 1; eb = 8; break;
        case NQ_FIELD_GINV_U: off = L.gih[0]; cnt = (int64_t)r * L.ldr; l = L.ldr; eb = 2; break;
        case NQ_FIELD_GINV_U_LO: off = L.gil[0]; cnt = (int64_t)r * L.ldr; l = L.ldr; eb = 2; break;
        case NQ_FIELD_GINV_V: off = L.gih[1]; cnt = (int64_t)r * L.ldr; l = L.ldr; eb = 2; break;
        case NQ_FIELD_GINV_V_LO: off = L.gil[1]; cnt = (int64_t)r * L.ldr; l = L.ldr; eb = 2; break;
        default: return NQ_ERR_INVALID_ARG;
    }
    *dev_ptr = static_cast<char *>(ws) + off;
    *count = cnt;
    *elem_bytes = eb;
    *ld = l;
    return NQ_OK;
}

nq_status nq_lbadmm_sync_operands(int64_t m, int64_t n, int32_t r, nq_precision prec, void *ws,
                                  size_t ws_bytes, nq_stream_t stream) {
    if (!valid_prec(prec)) return NQ_ERR_INVALID_ARG;
    Lb lb;
    nq_status st = lb_open(lb, m, n, r, ws, ws_bytes);
    if (st) return st;
    cudaStream_t s = cs(stream);
    const LbLayout &L = lb.L;
    const bool split = prec == NQ_PREC_FP32;
    NQ_CK(transpose_to_bf16(lb.p<float>(L.x[0]), L.m, L.r, L.ldr, lb.p<__nv_bfloat16>(L.xt[0]),
                            split ? lb.p<__nv_bfloat16>(L.xtl[0]) : nullptr, L.ldm, s));
    NQ_CK(transpose_to_bf16(lb.p<float>(L.x[1]), L.n, L.r, L.ldr, lb.p<__nv_bfloat16>(L.xt[1]),
                            split ? lb.p<__nv_bfloat16>(L.xtl[1]) : nullptr, L.ldn, s));
    NQ_CK(transpose_bf16(lb.p<__nv_bfloat16>(L.what), L.m, L.n, L.ldn,
                         lb.p<__nv_bfloat16>(L.whatT), L.ldm, s));
    if (split)
        NQ_CK(transpose_bf16(lb.p<__nv_bfloat16>(L.whatL), L.m, L.n, L.ldn,
                             lb.p<__nv_bfloat16>(L.whatTL), L.ldm, s));
    return NQ_OK;
}

nq_status nq_lbadmm_check(int64_t m, int64_t n, int32_t r, void *ws, size_t ws_bytes,
                          nq_stream_t stream) {
    Lb lb;
    nq_status st = lb_open(lb, m, n, r, ws, ws_bytes);
    if (st) return st;
    return read_err(&lb.sc->err, cs(stream), true);
}

int64_t nq_launch_count(void) { return (int64_t)nq::g_launches.load(); }

nq_status nq_profile_enable(int32_t enable) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_used = 0;
    g_prof_on = enable != 0;
    return NQ_OK;
}

nq_status nq_profile_get(int32_t kernel_class, int64_t *launches, double *total_ms) {
    if (!launches || !total_ms || kernel_class < 0 || kernel_class >= NQ_K_COUNT)
        return NQ_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    int64_t n = 0;
    double ms = 0.0;
    for (size_t i = 0; i < g_prof_used; ++i) {
        const ProfRec &r = g_prof[i];
        if (r.cls != kernel_class) continue;
        NQ_CK(cudaEventSynchronize(r.b));
        float t = 0.f;
        NQ_CK(cudaEventElapsedTime(&t, r.a, r.b));
        ms += t;
        ++n;
    }
    *launches = n;
    *total_ms = ms;
    return NQ_OK;
}

}  // extern "C"
