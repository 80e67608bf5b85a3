// Workspace layouts of the library (host and device visible).
#pragma once
#include <stddef.h>
#include <stdint.h>

namespace nq {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

constexpr int kSvidRows = 4;          // rows of S staged in shared memory per SVID tile
constexpr int kSvidCtas = 4 * 148;     // CTAs of an SVID pass (4 per SM)
constexpr int kRedBlocks = 592;       // CTAs of grid-stride reduction kernels (4 per SM)
constexpr int kObjRing = 4096;        // per-iteration objective slots kept on the device
constexpr int kMaxRank = 4096;
constexpr int kGramMaxUnits = 2 * 148;  // split-K Gram: most (tile, part) work units

// Lower-triangular 128 x 128 tiles of an r x r Gram.
inline int gram_tiles(int32_t r) {
    const int nm = (r + 127) / 128;
    return nm * (nm + 1) / 2;
}
// Split-K parts of a Gram over K rows (nseg concatenated K segments) on ``sms`` SMs: enough
// (tile, part) units to fill the SMs, at most 8 parts, at least 8 k-blocks of 64 per part.
inline int gram_ksplit(int32_t r, int64_t K, int nseg, int sms) {
    const int T = gram_tiles(r);
    if (T >= sms) return 1;
    int S = sms / T;
    if (S > 8) S = 8;
    const int64_t kb = nseg * ((K + 63) / 64);
    if (S > kb / 8) S = (int)(kb / 8);
    if (S * T > kGramMaxUnits) S = kGramMaxUnits / T;
    return S < 1 ? 1 : S;
}
constexpr int64_t kMaxDim = 65536;

// Newton-Schulz update of G^-1 (see NsState): at most kNsMaxSteps steps, the first
// kNsBf16Steps of them with plain BF16 operands, the rest split (hi + lo).
constexpr int kNsMaxSteps = 6;
constexpr int kNsBf16Steps = 2;
enum NsGate : int { NS_RUNNING = 0, NS_FINAL = 1, NS_DONE = 2, NS_FAIL = 3 };

// State of the Newton-Schulz inverse update of one half step (8-byte words first: the
// first 11 words are readable as a state field).
struct NsState {
    unsigned long long accepted;   // half steps whose inverse came from the update
    unsigned long long fallbacks;  // attempts that fell back to the Cholesky factorisation
    long long steps;               // steps of the last accepted update
    double ef[kNsMaxSteps + 2];    // ||I - X_k G||_F of the last attempt, step by step
    int gate;                      // NsGate of the running half step
    unsigned int ticket;           // finished tiles of the running launch
    unsigned int grid_count;       // phases x CTAs arrived (one-launch update's grid barrier)
    int pad;
};

// Scalars block at the start of every workspace.
struct Scalars {
    double gamma;        // ||W~||_F / (2 sqrt r)
    double wt_norm2;     // ||W~||_F^2 (W~ formed in FP32 from W, d_in, d_out)
    double what_norm2;   // ||W^||_F^2 of the BF16 target
    double alpha[2];     // Ledoit-Wolf intensities (calibration)
    double recon2;       // sum of squared reconstruction errors
    int err;             // first device-side error status
    unsigned int bar[2]; // grid barrier (count, generation)
    int pad;
};

struct LbLayout {
    int64_t m = 0, n = 0;
    int32_t r = 0;
    int64_t ldr = 0;   // leading dim of every [rows][r] array (FP32 and BF16)
    int64_t ldn = 0;   // leading dim of W^ rows (n padded) and of Vt
    int64_t ldm = 0;   // leading dim of W^^T rows (m padded) and of Ut
    int64_t rp = 0;    // r padded to 64 (Cholesky tiles)
    int nsv = 0;       // CTAs of an SVID pass (rows of its partial array)
    size_t scal = 0, what = 0, whatT = 0, whatL = 0, whatTL = 0, x[2] = {0, 0}, s[2] = {0, 0},
           a[2] = {0, 0}, b[2] = {0, 0}, xt[2] = {0, 0}, xtl[2] = {0, 0}, rhi = 0, rlo = 0, g[2] = {0, 0}, chA = 0, chLi = 0,
           gih[2] = {0, 0}, gil[2] = {0, 0}, gsh = 0, gsl = 0, nqh[2] = {0, 0}, nql[2] = {0, 0},
           nth = 0, ntl = 0, nspart = 0, ns = 0, gdh[2] = {0, 0}, gdl[2] = {0, 0}, gdmax = 0,
           lth = 0, ltl = 0, chF = 0, tvec = 0, bcur = 0, gk = 0, part = 0, partn = 0, partg = 0,
           partb = 0, obj = 0, gpart = 0, total = 0;
    size_t part_doubles = 0;   // capacity of ``part`` (doubles): one per GEMM tile

    int64_t rows(int side) const { return side == 0 ? m : n; }
    int64_t ld_rows(int side) const { return side == 0 ? ldm : ldn; }

    void build(int64_t m_, int64_t n_, int32_t r_) {
        m = m_;
        n = n_;
        r = r_;
        ldr = (r + 7) / 8 * 8;
        ldn = (n + 7) / 8 * 8;
        ldm = (m + 7) / 8 * 8;
        rp = (r + 63) / 64 * 64;
        const int64_t maxrows = m > n ? m : n;
        int64_t tiles_rows = (maxrows + kSvidRows - 1) / kSvidRows;
        nsv = (int)(tiles_rows < kSvidCtas ? tiles_rows : kSvidCtas);
        size_t off = 0;
        auto take = [&](size_t bytes) {
            size_t o = off;
            off = align_up(off + bytes);
            return o;
        };
        scal = take(sizeof(Scalars));
        what = take((size_t)m * ldn * 2);
        whatT = take((size_t)n * ldm * 2);
        // low BF16 parts (split operands of the FP32-accurate precision mode)
        whatL = take((size_t)m * ldn * 2);
        whatTL = take((size_t)n * ldm * 2);
        for (int sd = 0; sd < 2; ++sd) {
            const int64_t rw = sd == 0 ? m : n;
            x[sd] = take((size_t)rw * ldr * 4);
            s[sd] = take((size_t)rw * ldr * 4);
            a[sd] = take((size_t)rw * 4);
            b[sd] = take((size_t)r * 4);
            xt[sd] = take((size_t)r * (sd == 0 ? ldm : ldn) * 2);
            xtl[sd] = take((size_t)r * (sd == 0 ? ldm : ldn) * 2);
            g[sd] = take((size_t)r * r * 4);
        }
        rhi = take((size_t)maxrows * ldr * 2);
        rlo = take((size_t)maxrows * ldr * 2);
        chA = take((size_t)rp * rp * 4);
        chLi = take((size_t)rp * rp * 4);
        // G^-1 of each side's solve (hi + lo), kept as the start of that side's next
        // Newton-Schulz update; the Gram split into hi + lo; the update's iterates and its
        // products X G
        for (int sd = 0; sd < 2; ++sd) {
            gih[sd] = take((size_t)r * ldr * 2);
            gil[sd] = take((size_t)r * ldr * 2);
            nqh[sd] = take((size_t)r * ldr * 2);
            nql[sd] = take((size_t)r * ldr * 2);
        }
        gsh = take((size_t)r * ldr * 2);
        gsl = take((size_t)r * ldr * 2);
        nth = take((size_t)r * ldr * 2);
        ntl = take((size_t)r * ldr * 2);
        nspart = take((size_t)((r + 127) / 128) * ((r + 63) / 64) * 8);
        ns = take(sizeof(NsState));
        // gradient-descent variant: the latent split into hi + lo (two buffers, the GEMM of
        // a step reads one and its epilogue writes the other) and the step size's bound
        for (int sd = 0; sd < 2; ++sd) {
            gdh[sd] = take((size_t)maxrows * ldr * 2);
            gdl[sd] = take((size_t)maxrows * ldr * 2);
        }
        gdmax = take(sizeof(unsigned int));
        lth = take((size_t)r * ldr * 2);   // (L^-1)^T, bf16 hi
        ltl = take((size_t)r * ldr * 2);   // (L^-1)^T, bf16 lo
        chF = take((size_t)2 * (rp / 64) * (rp / 64) * 4);  // Cholesky / inverse tile counters
        tvec = take((size_t)maxrows * 4);
        bcur = take((size_t)2 * r * 4);
        gk = take((size_t)r * 4);
        // per-tile partials: GEMM tiles at BN = 64 for the objective (n x r) and the
        // reconstruction error (m x n); grid-stride reductions use kRedBlocks
        const int64_t t_obj = ((n + 127) / 128) * ((r + 63) / 64);
        const int64_t t_rec = ((m + 127) / 128) * ((n + 63) / 64);
        int64_t pd = t_obj > t_rec ? t_obj : t_rec;
        if (pd < kRedBlocks) pd = kRedBlocks;
        part_doubles = (size_t)pd;
        part = take(part_doubles * 8);        // per-tile partials / grid-stride partials
        partn = take((size_t)nsv * 8);        // SVID norm partials
        partg = take((size_t)kRedBlocks * 8); // Gram dot-product partials
        partb = take((size_t)2 * nsv * r * 4);  // column partials (SVID; U and V norms)
        obj = take((size_t)kObjRing * 4);
        // split-K Gram partial tiles (128 x 128 FP32 per unit)
        const int gu = gram_tiles(r) * 8 < kGramMaxUnits ? gram_tiles(r) * 8 : kGramMaxUnits;
        gpart = take((size_t)gu * 128 * 128 * 4);
        total = off;
    }
};

struct CalibLayout {
    int64_t T = 0, C = 0;
    int nslab = 0;     // token slabs
    size_t scal = 0, ps = 0, pq = 0, s = 0, q = 0, total = 0;
    void build(int64_t T_, int64_t C_, int nslab_) {
        T = T_;
        C = C_;
        nslab = nslab_;
        size_t off = 0;
        auto take = [&](size_t bytes) {
            size_t o = off;
            off = align_up(off + bytes);
            return o;
        };
        scal = take(sizeof(Scalars));
        ps = take((size_t)nslab * C * 8);
        pq = take((size_t)nslab * C * 8);
        s = take((size_t)C * 8);
        q = take((size_t)C * 8);
        total = off;
    }
};

// Workspace of nq_binary_matmul.  B <= gemv_max: partials of the z pass (chunks x B x r)
// and z (B x r); larger B: the expanded tensor-core operands.
struct BinLayout {
    int64_t ldt = 0, ldr = 0;   // leading dims (elements) of the n- and r-long BF16 rows
    size_t scal = 0, P = 0, z = 0, vh = 0, vl = 0, um = 0, xh = 0, xl = 0, zh = 0, zl = 0,
           total = 0;
    void build(int64_t m, int64_t n, int32_t r, int64_t B, int gemv_max, int chunks) {
        ldt = (n + 7) / 8 * 8;
        ldr = (r + 7) / 8 * 8;
        size_t off = 0;
        auto take = [&](size_t bytes) {
            size_t o = off;
            off = align_up(off + bytes);
            return o;
        };
        scal = take(sizeof(Scalars));
        if (B <= gemv_max) {
            P = take((size_t)chunks * B * r * 4);
            z = take((size_t)B * r * 4);
        } else {
            vh = take((size_t)r * ldt * 2);
            vl = take((size_t)r * ldt * 2);
            um = take((size_t)m * ldr * 2);
            xh = take((size_t)B * ldt * 2);
            xl = take((size_t)B * ldt * 2);
            zh = take((size_t)B * ldr * 2);
            zl = take((size_t)B * ldr * 2);
        }
        total = off;
    }
};

// Workspace of nq_ls_refit: the +-1 operands, the per-(row, tile) partial sums of both
// passes (tiles of 64 columns at most: the narrowest tile width) and the reduction
// partials of the final reconstruction error.
struct RefitLayout {
    int64_t ldr = 0;
    size_t scal = 0, up = 0, vp = 0, num = 0, den = 0, part = 0, total = 0;
    void build(int64_t m, int64_t n, int32_t r) {
        ldr = (r + 7) / 8 * 8;
        size_t off = 0;
        auto take = [&](size_t bytes) {
            size_t o = off;
            off = align_up(off + bytes);
            return o;
        };
        const int64_t a = ((n + 63) / 64) * m, b = ((m + 63) / 64) * n;
        const int64_t np = a > b ? a : b;
        scal = take(sizeof(Scalars));
        up = take((size_t)m * ldr * 2);
        vp = take((size_t)n * ldr * 2);
        num = take((size_t)np * 8);
        den = take((size_t)np * 8);
        int64_t t_rec = ((m + 127) / 128) * ((n + 63) / 64);
        if (t_rec < kRedBlocks) t_rec = kRedBlocks;
        part = take((size_t)t_rec * 8);
        total = off;
    }
};

struct ReconLayout {
    int64_t m = 0, n = 0;
    int32_t r = 0;
    int64_t ldr = 0;
    size_t scal = 0, up = 0, vp = 0, part = 0, total = 0;
    size_t part_doubles = 0;
    void build(int64_t m_, int64_t n_, int32_t r_) {
        m = m_;
        n = n_;
        r = r_;
        ldr = (r + 7) / 8 * 8;
        size_t off = 0;
        auto take = [&](size_t bytes) {
            size_t o = off;
            off = align_up(off + bytes);
            return o;
        };
        scal = take(sizeof(Scalars));
        up = take((size_t)m * ldr * 2);
        vp = take((size_t)n * ldr * 2);
        int64_t t_rec = ((m + 127) / 128) * ((n + 63) / 64);
        if (t_rec < kRedBlocks) t_rec = kRedBlocks;
        part_doubles = (size_t)t_rec;
        part = take(part_doubles * 8);
        total = off;
    }
};

}  // namespace nq
