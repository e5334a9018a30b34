// C ABI of the Fast LapSum library: argument checks, workspace layout, solver
// dispatch.  Every entry point is declared and documented in include/lapsum.h.
//
// Solver choice follows "Fast LapSum: Exact Differentiable Top-k at Million
// Scale" (gist.science explainer pages), section 2.2: the full-sort solver
// where sorting is affordable, probabilistic bracketing for n > 10^6.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "lapsum_common.cuh"
#include "lapsum_kernels.h"

namespace lapsum {
namespace {

constexpr size_t kAlign = 256;
constexpr int64_t kOnchipMax = 4096;
constexpr int64_t kRowBracketAuto = int64_t(1) << 18;  // AUTO: one CTA per row up to here
constexpr int64_t kRowBracketMax = int64_t(1) << 20;
constexpr int kFoldGridMax = 4096;
constexpr int64_t kGridYMax = 65535;
constexpr double kBracketAlpha = 1e-6;  // miss probability allowed per bracket end

size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Solver for per-row budgets: as for a shared budget; the bracketing solvers
// compute each row's sample size and binomial ranks on the device.
int resolve_path_rowk(int64_t n, int path) {
    switch (path & 0xff) {
        case LAPSUM_PATH_AUTO:
            return n <= kOnchipMax ? LAPSUM_PATH_FULLSORT
                   : n <= kRowBracketAuto ? LAPSUM_PATH_ROWBRACKET
                                          : LAPSUM_PATH_BRACKET;
        case LAPSUM_PATH_FULLSORT:
            return n <= kOnchipMax ? LAPSUM_PATH_FULLSORT : LAPSUM_PATH_RADIX;
        case LAPSUM_PATH_RADIX: return LAPSUM_PATH_RADIX;
        case LAPSUM_PATH_ROWBRACKET: return n <= kRowBracketMax ? LAPSUM_PATH_ROWBRACKET : -1;
        case LAPSUM_PATH_BRACKET: return LAPSUM_PATH_BRACKET;
        default: return -1;
    }
}

int resolve_path(int64_t n, int path) {
    switch (path & 0xff) {
        case LAPSUM_PATH_AUTO:
            return n <= kOnchipMax ? LAPSUM_PATH_FULLSORT
                   : n <= kRowBracketAuto ? LAPSUM_PATH_ROWBRACKET
                                          : LAPSUM_PATH_BRACKET;
        case LAPSUM_PATH_ROWBRACKET: return n <= kRowBracketMax ? LAPSUM_PATH_ROWBRACKET : -1;
        case LAPSUM_PATH_FULLSORT:
            return n <= kOnchipMax ? LAPSUM_PATH_FULLSORT : LAPSUM_PATH_RADIX;
        case LAPSUM_PATH_BRACKET: return LAPSUM_PATH_BRACKET;
        case LAPSUM_PATH_RADIX: return LAPSUM_PATH_RADIX;
        default: return -1;
    }
}

struct Layout {
    size_t header, rows, partials, row_R, tickets, wlist, wtab, wflag;
    size_t keys0, keys1, seg_hist, tile_hist, plan;
    size_t sample, band0, band1, bins, fold_part, fold_ticket, budgets, cand;
    size_t total;
};

Layout make_layout(int64_t B, int64_t n, int rpath) {
    Layout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += up(bytes);
        return o;
    };
    const int64_t tiles = stream_tiles(n);
    L.header = take(sizeof(WsHeader));
    // per-row emit/backward tickets, then the fold and sample tickets and the
    // sample kernel's 2048-bin key histogram (all self-clearing)
    L.tickets = take((size_t)B * 2 * sizeof(uint32_t) + (2 + 2048) * sizeof(uint32_t));
    L.fold_ticket = L.tickets + (size_t)B * 2 * sizeof(uint32_t);
    L.rows = take((size_t)B * sizeof(RowState));
    L.partials = take((size_t)B * (size_t)(tiles > 2 ? tiles : 2) * 4 * sizeof(double));
    L.row_R = take((size_t)B * sizeof(double));
    if (n > kOnchipMax) {  // windowed backward of long rows
        // the pass CTAs of a row split the capacity evenly (rounded up per CTA)
        L.wlist = take((size_t)B * ((size_t)window_capacity(n) + 8192) * sizeof(WinEntry));
        L.wtab = take((size_t)B * (size_t)window_tiles(n) * sizeof(uint2));
        L.wflag = take((size_t)B * sizeof(uint32_t));
    }
    if (rpath == LAPSUM_PATH_RADIX) {
        const int64_t rt = radix_tiles(n);
        L.keys0 = take((size_t)B * (size_t)n * sizeof(uint32_t));
        L.keys1 = take((size_t)B * (size_t)n * sizeof(uint32_t));
        L.seg_hist = take((size_t)B * 1024 * sizeof(uint32_t));
        // per-tile digit histograms (legacy passes) or look-back words, plus
        // the pass's tile counter (8 bytes) right after them
        L.tile_hist = take((size_t)B * 256 * (size_t)rt * sizeof(uint32_t) + 256);
        L.plan = take((size_t)B * 8 * sizeof(int32_t));
    }
    if (rpath == LAPSUM_PATH_ROWBRACKET) {
        L.band0 = take((size_t)B * (size_t)n * sizeof(float));
        L.band1 = take((size_t)B * (size_t)n * sizeof(float));
        L.budgets = take((size_t)B * sizeof(RowBudget));  // per-row budgets' ladders
    }
    if (rpath == LAPSUM_PATH_BRACKET) {
        L.sample = take((size_t)B * kSampleMax * sizeof(float));
        L.band0 = take((size_t)n * sizeof(float));
        L.band1 = take((size_t)n * sizeof(float));
        L.bins = take((size_t)3 * kBins * sizeof(unsigned long long));
        L.fold_part = take((size_t)kFoldGridMax * 4 * sizeof(double));
        L.cand = take((size_t)4096 * sizeof(uint32_t));
        L.budgets = take((size_t)B * sizeof(RowBudget));  // per-row budgets' ladders
    }
    L.total = off;
    return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_dtype(int dtype) {
    return dtype == LAPSUM_DTYPE_F32 || dtype == LAPSUM_DTYPE_BF16 || dtype == LAPSUM_DTYPE_F16;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? LAPSUM_OK : LAPSUM_ECUDA; }

// Binomial(m, q) order-statistic ranks (descending, 1-based) for one bracket:
// l = largest with P(C < l) <= alpha, h = smallest with P(C >= h) <= alpha.
// The upper tail is accumulated downward from mq + 40 sd + 64, past which every
// probability is below 1e-300; results are cached per (m, q, alpha).
void binomial_ranks(int64_t m, double q, double alpha, int64_t* l, int64_t* h) {
    struct Entry {
        int64_t m;
        double q, alpha;
        int64_t l, h;
    };
    static std::mutex mu;
    static std::vector<Entry> cache;
    {
        std::lock_guard<std::mutex> g(mu);
        for (const Entry& e : cache)
            if (e.m == m && e.q == q && e.alpha == alpha) {
                *l = e.l;
                *h = e.h;
                return;
            }
    }
    const double lgm = std::lgamma((double)m + 1.0), lq = std::log(q), l1q = std::log1p(-q);
    auto logpmf = [&](int64_t c) {
        return lgm - std::lgamma((double)c + 1.0) - std::lgamma((double)(m - c) + 1.0) +
               (double)c * lq + (double)(m - c) * l1q;
    };
    double cdf = 0.0;
    int64_t lo = 0;
    for (int64_t c = 0; c <= m; ++c) {
        cdf += std::exp(logpmf(c));
        if (cdf <= alpha) lo = c + 1;
        else break;
    }
    const double mean = (double)m * q, sd = std::sqrt((double)m * q * (1.0 - q));
    int64_t top = (int64_t)std::ceil(mean + 40.0 * sd + 64.0);
    if (top > m) top = m;
    double sf = 0.0;
    int64_t hi = top + 1 <= m ? top + 1 : m + 1;
    for (int64_t c = top; c >= 0; --c) {
        sf += std::exp(logpmf(c));
        if (sf <= alpha) hi = c;
        else break;
    }
    *l = lo;
    *h = hi;
    std::lock_guard<std::mutex> g(mu);
    if (cache.size() < 64) cache.push_back(Entry{m, q, alpha, lo, hi});
}

// Ranks of the bracket ladder: the binomial ranks, then each end moved out by
// a factor of 4 per rung, the last rung open.
void bracket_ladder(int m, double q, int64_t rl[kLadder], int64_t rh[kLadder]) {
    int64_t l0, h0;
    binomial_ranks(m, q, kBracketAlpha, &l0, &h0);
    for (int i = 0; i < kLadder - 1; ++i) {
        rl[i] = l0 >> (2 * i);
        rh[i] = h0 << (2 * i);
        if (rh[i] > m) rh[i] = m + 1;
    }
    rl[kLadder - 1] = 0;
    rh[kLadder - 1] = m + 1;
}

int sample_size(int64_t n, double k) {
    const double q = k / (double)n;
    double want = 64.0 / q;
    int m = 4096;
    while (m < kSampleMax && m < want) m <<= 1;
    return m;
}

// --- optional per-kernel event timing ---------------------------------------
struct ProfRec {
    const char* name;
    cudaEvent_t a, b;
};
struct Profiler {
    std::mutex mu;
    bool on = false;
    std::vector<ProfRec> recs;
    std::vector<cudaEvent_t> pool;
    int open = -1;
    cudaEvent_t get() {
        if (!pool.empty()) {
            cudaEvent_t e = pool.back();
            pool.pop_back();
            return e;
        }
        cudaEvent_t e = nullptr;
        cudaEventCreate(&e);
        return e;
    }
    void recycle() {
        for (auto& r : recs) {
            pool.push_back(r.a);
            pool.push_back(r.b);
        }
        recs.clear();
        open = -1;
    }
};
Profiler& profiler() {
    static Profiler p;
    return p;
}

}  // namespace

int device_sm_count() {
    constexpr int kMaxDevices = 64;
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    if (dev >= 0 && dev < kMaxDevices) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        sms = 1;
    if (dev >= 0 && dev < kMaxDevices) cache[dev].store(sms, std::memory_order_relaxed);
    return sms;
}

void prof_begin(const char* name, cudaStream_t st) {
    Profiler& p = profiler();
    if (!p.on) return;
    std::lock_guard<std::mutex> g(p.mu);
    ProfRec r{name, p.get(), p.get()};
    cudaEventRecord(r.a, st);
    p.recs.push_back(r);
    p.open = (int)p.recs.size() - 1;
}

void prof_end(cudaStream_t st) {
    Profiler& p = profiler();
    if (!p.on) return;
    std::lock_guard<std::mutex> g(p.mu);
    if (p.open >= 0) cudaEventRecord(p.recs[p.open].b, st);
    p.open = -1;
}

}  // namespace lapsum

using namespace lapsum;

extern "C" {

int lapsum_abi_version(void) { return 1; }

const char* lapsum_status_string(int status) {
    switch (status) {
        case LAPSUM_OK: return "ok";
        case LAPSUM_EINVAL: return "invalid argument";
        case LAPSUM_EWORKSPACE: return "workspace missing, misaligned or too small";
        case LAPSUM_ENONFINITE: return "non-finite score";
        case LAPSUM_EBRACKET: return "bracketing retries exhausted";
        case LAPSUM_ECUDA: return "CUDA runtime error";
        default: return "unknown status";
    }
}

size_t lapsum_workspace_bytes(int64_t B, int64_t n, double k, int path) {
    (void)k;
    if (B < 1 || n < 1) return 0;
    const int rp = resolve_path(n, path);
    if (rp < 0) return 0;
    return make_layout(B, n, rp).total;
}

size_t lapsum_workspace_bytes_rowk(int64_t B, int64_t n, int path) {
    if (B < 1 || n < 1) return 0;
    const int rp = resolve_path_rowk(n, path);
    if (rp < 0) return 0;
    return make_layout(B, n, rp).total;
}

size_t lapsum_backward_workspace_bytes(int64_t B, int64_t n) {
    if (B < 1 || n < 1) return 0;
    return make_layout(B, n, LAPSUM_PATH_FULLSORT).total;
}

int lapsum_workspace_init(void* ws, size_t ws_bytes, void* stream) {
    if (ws == nullptr || ws_bytes < sizeof(WsHeader) ||
        (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0)
        return LAPSUM_EWORKSPACE;
    return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream));
}

size_t lapsum_support_bytes(int64_t B, int64_t n) {
    if (B < 1 || n <= kOnchipMax) return 0;
    return support_bytes(B, n);
}

}  // extern "C"

namespace {

// The forward of lapsum_forward and lapsum_forward_support; `support` is null
// for the former.
int forward_impl(const float* r, int64_t ld, float* p, double* b, double* sum_f, int64_t B,
                 int64_t n, double k, const double* k_rows, double t, int path, uint64_t seed,
                 void* ws, size_t ws_bytes, void* support, size_t support_size, void* stream) {
    if (r == nullptr || p == nullptr || b == nullptr) return LAPSUM_EINVAL;
    if (B < 1 || n < 1 || ld < n) return LAPSUM_EINVAL;
    if (k_rows == nullptr && (!(k > 0.0) || !(k < (double)n) || !std::isfinite(k)))
        return LAPSUM_EINVAL;
    if (!(t > 0.0) || !std::isfinite(t)) return LAPSUM_EINVAL;
    const int rp = k_rows != nullptr ? resolve_path_rowk(n, path) : resolve_path(n, path);
    if (rp < 0 || (path & ~0x7ff) != 0) return LAPSUM_EINVAL;
    if (n > INT32_MAX && rp != LAPSUM_PATH_BRACKET) return LAPSUM_EINVAL;
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return LAPSUM_EWORKSPACE;
    const Layout L = make_layout(B, n, rp);
    if (ws_bytes < L.total) return LAPSUM_EWORKSPACE;
    const bool want_sup = support != nullptr && n > kOnchipMax;
    if (want_sup && ((reinterpret_cast<uintptr_t>(support) % kAlign) != 0 ||
                     support_size < support_bytes(B, n)))
        return LAPSUM_EWORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    char* w = static_cast<char*>(ws);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(w + L.header);
    RowState* rows = reinterpret_cast<RowState*>(w + L.rows);
    uint32_t* tickets = reinterpret_cast<uint32_t*>(w + L.tickets);
    double* partials = reinterpret_cast<double*>(w + L.partials);
    const int vec = (aligned16(r) && aligned16(p) && (ld % 4) == 0) ? 1 : 0;
    cudaError_t e = cudaSuccess;
    // the gradient support's per-row flags are cleared by the first kernel of
    // the bracketing paths, and here for the radix path
    const SupportView sv_all = want_sup ? support_view(support, B, n) : SupportView{};

    if (rp == LAPSUM_PATH_FULLSORT) {
        // AUTO: the segment search on rows of n <= 256 (FORCE_MISS sends every
        // row on to the sort inside the same kernel)
        const int search = (path & 0xff) != LAPSUM_PATH_AUTO ? 0
                           : (path & LAPSUM_FLAG_FORCE_MISS) ? 2
                                                             : 1;
        e = launch_onchip_forward(r, ld, p, b, sum_f, B, (int)n, k, k_rows, t, hdr, vec, search,
                                  st);
        return cuda_status(e);
    }
    if (rp == LAPSUM_PATH_RADIX) {
        e = cudaMemsetAsync(rows, 0, (size_t)B * sizeof(RowState), st);
        if (e == cudaSuccess && want_sup)
            e = cudaMemsetAsync(sv_all.flags, 0, (size_t)B * sizeof(uint32_t), st);
        if (e != cudaSuccess) return LAPSUM_ECUDA;
        RadixBuffers rb;
        rb.keys[0] = reinterpret_cast<uint32_t*>(w + L.keys0);
        rb.keys[1] = reinterpret_cast<uint32_t*>(w + L.keys1);
        rb.seg_hist = reinterpret_cast<uint32_t*>(w + L.seg_hist);
        rb.tile_hist = reinterpret_cast<uint32_t*>(w + L.tile_hist);
        rb.plan = reinterpret_cast<int32_t*>(w + L.plan);
        for (int64_t r0 = 0; r0 < B && e == cudaSuccess; r0 += kGridYMax) {
            const int64_t nb = (B - r0 < kGridYMax) ? B - r0 : kGridYMax;
            RadixBuffers sub = rb;
            sub.keys[0] += r0 * n;
            sub.keys[1] += r0 * n;
            sub.seg_hist += r0 * 1024;
            sub.tile_hist += r0 * 256 * radix_tiles(n);
            sub.plan += r0 * 8;
            e = launch_radix_sort_rows(r + r0 * ld, ld, nb, n, sub, rows + r0, hdr, st);
            if (e == cudaSuccess)
                e = launch_rowsolve_sorted_keys(sub, nb, n, k, k_rows ? k_rows + r0 : nullptr, t,
                                                b + r0, rows + r0, hdr, st);
        }
    } else if (rp == LAPSUM_PATH_ROWBRACKET) {
        int64_t rl[kLadder], rh[kLadder];
        RowBudget* budgets = nullptr;
        int m = kSampleMax;
        if (k_rows != nullptr) {
            budgets = reinterpret_cast<RowBudget*>(w + L.budgets);
            for (int i = 0; i < kLadder; ++i) rl[i] = rh[i] = 0;
            e = launch_row_budgets(k_rows, B, n, kBracketAlpha, budgets, st);
            if (e != cudaSuccess) return LAPSUM_ECUDA;
        } else {
            m = sample_size(n, k);
            bracket_ladder(m, k / (double)n, rl, rh);
        }
        e = launch_rowbracket(r, ld, B, n, k, t, seed, m, rl, rh, path, rows,
                              reinterpret_cast<float*>(w + L.band0),
                              reinterpret_cast<float*>(w + L.band1), b, hdr,
                              (aligned16(r) && (ld % 4) == 0) ? 1 : 0, st, budgets,
                              want_sup ? sv_all.flags : nullptr);
    } else {
        BracketBuffers bb;
        bb.sample = reinterpret_cast<float*>(w + L.sample);
        bb.band[0] = reinterpret_cast<float*>(w + L.band0);
        bb.band[1] = reinterpret_cast<float*>(w + L.band1);
        bb.bins = reinterpret_cast<unsigned long long*>(w + L.bins);
        bb.fold_part = reinterpret_cast<double*>(w + L.fold_part);
        bb.cand = reinterpret_cast<uint32_t*>(w + L.cand);
        bb.ticket = reinterpret_cast<uint32_t*>(w + L.fold_ticket);
        bb.fold_grid = bracket_fold_grid();
        if (bb.fold_grid > kFoldGridMax) bb.fold_grid = kFoldGridMax;
        int m = kSampleMax;
        int64_t rl[kLadder], rh[kLadder];
        RowBudget* budgets = nullptr;
        if (k_rows != nullptr) {
            // each row's sample size and ladder, on the device
            budgets = reinterpret_cast<RowBudget*>(w + L.budgets);
            for (int i = 0; i < kLadder; ++i) rl[i] = rh[i] = 0;
            e = launch_row_budgets(k_rows, B, n, kBracketAlpha, budgets, st);
        } else {
            m = sample_size(n, k);
            bracket_ladder(m, k / (double)n, rl, rh);
        }
        for (int64_t row = 0; row < B && e == cudaSuccess; ++row) {
            e = launch_bracket_row(r + row * ld, n, k, t, seed, row, m, rl, rh, path, bb,
                                   rows + row, b + row, hdr,
                                   want_sup ? sv_all.flags + row : nullptr,
                                   budgets != nullptr ? budgets + row : nullptr, st);
        }
    }
    if (e != cudaSuccess) return LAPSUM_ECUDA;
    for (int64_t r0 = 0; r0 < B && e == cudaSuccess; r0 += kGridYMax) {
        const int64_t nb = (B - r0 < kGridYMax) ? B - r0 : kGridYMax;
        const SupportView sv = want_sup ? support_rows(sv_all, r0, n) : SupportView{};
        e = launch_emit(r + r0 * ld, ld, p + r0 * ld, b + r0, sum_f ? sum_f + r0 : nullptr, nb, n,
                        t, partials + r0 * stream_tiles(n), tickets + r0, vec, hdr, r0 == 0 ? 1 : 0,
                        B, rp, want_sup ? &sv : nullptr, st);
    }
    return cuda_status(e);
}

}  // namespace

extern "C" {

int lapsum_forward(const float* r, int64_t ld, float* p, double* b, double* sum_f, int64_t B,
                   int64_t n, double k, double t, int path, uint64_t seed, void* ws,
                   size_t ws_bytes, void* stream) {
    return forward_impl(r, ld, p, b, sum_f, B, n, k, nullptr, t, path, seed, ws, ws_bytes,
                        nullptr, 0, stream);
}

int lapsum_forward_hard(const float* r, int64_t ld, float* p, double* b, int64_t B, int64_t n,
                        double k, int path, void* ws, size_t ws_bytes, void* stream) {
    if (r == nullptr || p == nullptr || b == nullptr) return LAPSUM_EINVAL;
    if (B < 1 || n < 2 || ld < n || n > INT32_MAX) return LAPSUM_EINVAL;
    if (!(k > 0.0) || !(k < (double)n) || !std::isfinite(k)) return LAPSUM_EINVAL;
    const int pc = path & 0xff;
    if ((path & ~0x1ff) != 0 || pc == LAPSUM_PATH_ROWBRACKET || pc > LAPSUM_PATH_ROWBRACKET)
        return LAPSUM_EINVAL;
    // long rows: bracketing for AUTO and BRACKET (when both bracket ranks fit
    // the sample CTAs' candidate lists), the radix full sort otherwise; the
    // workspace is the full-sort one either way
    int rp = n <= kOnchipMax && (pc == LAPSUM_PATH_AUTO || pc == LAPSUM_PATH_FULLSORT)
                 ? LAPSUM_PATH_FULLSORT
                 : LAPSUM_PATH_RADIX;
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return LAPSUM_EWORKSPACE;
    const Layout L = make_layout(B, n, rp);
    if (ws_bytes < L.total) return LAPSUM_EWORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    char* w = static_cast<char*>(ws);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(w + L.header);
    RowState* rows = reinterpret_cast<RowState*>(w + L.rows);
    const int vec = (aligned16(r) && aligned16(p) && (ld % 4) == 0) ? 1 : 0;
    if (rp == LAPSUM_PATH_FULLSORT)
        return cuda_status(launch_onchip_hard(r, ld, p, b, B, (int)n, k, hdr, vec, st));
    if (n > kOnchipMax && (pc == LAPSUM_PATH_AUTO || pc == LAPSUM_PATH_BRACKET)) {
        const int m = sample_size(n, k);
        int64_t rl[kLadder], rh[kLadder];
        bracket_ladder(m, k / (double)n, rl, rh);
        const int64_t need = rh[0] <= m ? rh[0] : (rl[0] >= 1 ? rl[0] : 0);
        const int sgrid = m / 1024;
        if (need >= 1 && need <= 1024 && (int64_t)sgrid * need <= 4096) {
            const int64_t lo = rl[0] >= 1 ? rl[0] : 0;
            const int64_t hi = rh[0] <= m ? rh[0] : 0;
            cudaError_t e = cudaSuccess;
            for (int64_t r0 = 0; r0 < B && e == cudaSuccess; r0 += kGridYMax) {
                const int64_t nb = (B - r0 < kGridYMax) ? B - r0 : kGridYMax;
                e = launch_hard_bracket(
                    r + r0 * ld, ld, p + r0 * ld, b + r0, nb, n, k, 0, m, lo, hi, (int)need,
                    (path & LAPSUM_FLAG_FORCE_MISS) ? 1 : 0, rows + r0,
                    reinterpret_cast<float*>(w + L.keys0) + r0 * n,
                    reinterpret_cast<uint32_t*>(w + L.keys1) + r0 * 4096,
                    reinterpret_cast<uint32_t*>(w + L.tickets) + r0, hdr, B, vec, st);
            }
            return cuda_status(e);
        }
    }
    cudaError_t e = cudaMemsetAsync(rows, 0, (size_t)B * sizeof(RowState), st);
    if (e != cudaSuccess) return LAPSUM_ECUDA;
    RadixBuffers rb;
    rb.keys[0] = reinterpret_cast<uint32_t*>(w + L.keys0);
    rb.keys[1] = reinterpret_cast<uint32_t*>(w + L.keys1);
    rb.seg_hist = reinterpret_cast<uint32_t*>(w + L.seg_hist);
    rb.tile_hist = reinterpret_cast<uint32_t*>(w + L.tile_hist);
    rb.plan = reinterpret_cast<int32_t*>(w + L.plan);
    for (int64_t r0 = 0; r0 < B && e == cudaSuccess; r0 += kGridYMax) {
        const int64_t nb = (B - r0 < kGridYMax) ? B - r0 : kGridYMax;
        RadixBuffers sub = rb;
        sub.keys[0] += r0 * n;
        sub.keys[1] += r0 * n;
        sub.seg_hist += r0 * 1024;
        sub.tile_hist += r0 * 256 * radix_tiles(n);
        sub.plan += r0 * 8;
        e = launch_radix_sort_rows(r + r0 * ld, ld, nb, n, sub, rows + r0, hdr, st);
        if (e == cudaSuccess)
            e = launch_rowhard_sorted_keys(sub, nb, n, k, r + r0 * ld, ld, p + r0 * ld, b + r0,
                                           rows + r0, vec, st);
    }
    return cuda_status(e);
}

int lapsum_bracket_plan(int64_t n, double k, int32_t* m, int64_t* rank_l, int64_t* rank_h) {
    if (m == nullptr || rank_l == nullptr || rank_h == nullptr || n < 1) return LAPSUM_EINVAL;
    if (!(k > 0.0) || !(k < (double)n) || !std::isfinite(k)) return LAPSUM_EINVAL;
    *m = sample_size(n, k);
    bracket_ladder(*m, k / (double)n, rank_l, rank_h);
    return LAPSUM_OK;
}

size_t lapsum_shard_workspace_bytes(int64_t n_shard) {
    if (n_shard < 1) return 0;
    return up(shard_fold_workspace_bytes()) + up(vjp_shard_workspace_bytes());
}

size_t lapsum_shard_band_bytes(int64_t n_band_total) {
    if (n_band_total < 0) return 0;
    return 2 * up((size_t)(n_band_total > 0 ? n_band_total : 1) * sizeof(float));
}

int lapsum_shard_sample(const float* r, int64_t n_shard, int64_t offset, int64_t n, double t,
                        uint64_t seed, int32_t m, float* y, void* stream) {
    if (r == nullptr || y == nullptr || n_shard < 1 || offset < 0 || offset + n_shard > n)
        return LAPSUM_EINVAL;
    if (m < 1 || m > kSampleMax || !(t > 0.0) || !std::isfinite(t)) return LAPSUM_EINVAL;
    return cuda_status(launch_shard_sample(r, n_shard, offset, n, t, seed, m, y,
                                           (cudaStream_t)stream));
}

int lapsum_sample_bracket(const float* y, int32_t m, int64_t rank_l, int64_t rank_h, float* ends,
                          void* stream) {
    if (y == nullptr || ends == nullptr || m < 1 || m > kSampleMax) return LAPSUM_EINVAL;
    if (rank_l < 0 || rank_h < 0 || (rank_l >= 1 && rank_h >= 1 && rank_l > rank_h))
        return LAPSUM_EINVAL;
    return cuda_status(launch_sample_bracket(y, m, rank_l, rank_h, ends, (cudaStream_t)stream));
}

int lapsum_shard_fold(const float* r, int64_t n_shard, const float* ends, double t, double* rec,
                      float* band, void* ws, size_t ws_bytes, void* stream) {
    if (r == nullptr || ends == nullptr || rec == nullptr || band == nullptr || n_shard < 1)
        return LAPSUM_EINVAL;
    if (!(t > 0.0) || !std::isfinite(t)) return LAPSUM_EINVAL;
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 ||
        ws_bytes < lapsum_shard_workspace_bytes(n_shard))
        return LAPSUM_EWORKSPACE;
    return cuda_status(launch_shard_fold(r, n_shard, ends, t, rec, band, ws, (cudaStream_t)stream));
}

int lapsum_shard_band_solve(const float* bands, int64_t stride, const double* recs, int32_t world,
                            const float* ends, double k, double t, double* out, void* scratch,
                            size_t scratch_bytes, void* stream) {
    if (bands == nullptr || recs == nullptr || ends == nullptr || out == nullptr || world < 1 ||
        stride < 0)
        return LAPSUM_EINVAL;
    if (!(k > 0.0) || !std::isfinite(k) || !(t > 0.0) || !std::isfinite(t)) return LAPSUM_EINVAL;
    const size_t half = scratch_bytes / 2 / kAlign * kAlign;
    if (scratch == nullptr || (reinterpret_cast<uintptr_t>(scratch) % kAlign) != 0 ||
        scratch_bytes < lapsum_shard_band_bytes((int64_t)world * stride))
        return LAPSUM_EWORKSPACE;
    float* cur = static_cast<float*>(scratch);
    float* nxt = reinterpret_cast<float*>(static_cast<char*>(scratch) + half);
    return cuda_status(launch_shard_band_solve(bands, stride, recs, world, ends, k, t, cur, nxt, out,
                                               (cudaStream_t)stream));
}

int lapsum_shard_emit(const float* r, int64_t n_shard, const double* b, double t, float* p,
                      void* stream) {
    if (r == nullptr || b == nullptr || p == nullptr || n_shard < 1) return LAPSUM_EINVAL;
    if (!(t > 0.0) || !std::isfinite(t)) return LAPSUM_EINVAL;
    return cuda_status(launch_emit_p(r, p, b, n_shard, t, (cudaStream_t)stream));
}

int lapsum_shard_vjp_partial(const float* r, const float* v, int64_t n_shard, const double* b,
                             double t, double* rec, void* ws, size_t ws_bytes, void* stream) {
    if (r == nullptr || v == nullptr || b == nullptr || rec == nullptr || n_shard < 1)
        return LAPSUM_EINVAL;
    if (!(t > 0.0) || !std::isfinite(t)) return LAPSUM_EINVAL;
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 ||
        ws_bytes < lapsum_shard_workspace_bytes(n_shard))
        return LAPSUM_EWORKSPACE;
    void* vws = static_cast<char*>(ws) + up(shard_fold_workspace_bytes());
    return cuda_status(launch_vjp_partial(r, b, v, n_shard, t, rec, vws, (cudaStream_t)stream));
}

int lapsum_shard_vjp_apply(const float* r, const float* v, int64_t n_shard, const double* b,
                           double t, const double* recs, int32_t world, float* g, void* ws,
                           size_t ws_bytes, void* stream) {
    if (r == nullptr || v == nullptr || b == nullptr || recs == nullptr || g == nullptr ||
        n_shard < 1 || world < 1)
        return LAPSUM_EINVAL;
    if (!(t > 0.0) || !std::isfinite(t)) return LAPSUM_EINVAL;
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 ||
        ws_bytes < lapsum_shard_workspace_bytes(n_shard))
        return LAPSUM_EWORKSPACE;
    void* vws = static_cast<char*>(ws) + up(shard_fold_workspace_bytes());
    return cuda_status(launch_vjp_apply(r, b, v, g, n_shard, t, recs, world, vws,
                                        (cudaStream_t)stream));
}

int lapsum_forward_router(const void* r, int dtype, int64_t ld, float* p, double* b, int64_t B,
                          int64_t n, double k, double t, float eps, int32_t cap, int32_t* sel_idx,
                          float* sel_p, int32_t* sel_cnt, void* ws, size_t ws_bytes,
                          void* stream) {
    if (r == nullptr || p == nullptr || b == nullptr) return LAPSUM_EINVAL;
    if (!valid_dtype(dtype)) return LAPSUM_EINVAL;
    if (B < 1 || n < 1 || n > kOnchipMax || ld < n) return LAPSUM_EINVAL;
    if (!(k > 0.0) || !(k < (double)n) || !std::isfinite(k)) return LAPSUM_EINVAL;
    if (!(t > 0.0) || !std::isfinite(t)) return LAPSUM_EINVAL;
    const bool want_sel = sel_cnt != nullptr;
    if (want_sel != (sel_idx != nullptr) || want_sel != (sel_p != nullptr)) return LAPSUM_EINVAL;
    if (want_sel && (cap < 1 || !(eps >= 0.f) || !std::isfinite(eps))) return LAPSUM_EINVAL;
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return LAPSUM_EWORKSPACE;
    const Layout L = make_layout(B, n, LAPSUM_PATH_FULLSORT);
    if (ws_bytes < L.total) return LAPSUM_EWORKSPACE;
    WsHeader* hdr = reinterpret_cast<WsHeader*>(static_cast<char*>(ws) + L.header);
    const int vec =
        (aligned16(r) && aligned16(p) && (ld % (dtype == LAPSUM_DTYPE_F32 ? 4 : 8)) == 0) ? 1 : 0;
    return cuda_status(launch_onchip_router(r, dtype, ld, p, b, nullptr, B, (int)n, k, t, hdr, vec,
                                            sel_idx, sel_p, sel_cnt, want_sel ? cap : 0, eps, 1,
                                            (cudaStream_t)stream));
}

int lapsum_backward_router(const void* r, int dtype, int64_t ld, const double* b, const float* v,
                           float* g, int64_t B, int64_t n, double t, void* stream) {
    if (r == nullptr || b == nullptr || v == nullptr || g == nullptr) return LAPSUM_EINVAL;
    if (!valid_dtype(dtype)) return LAPSUM_EINVAL;
    if (B < 1 || n < 1 || n > kOnchipMax || ld < n) return LAPSUM_EINVAL;
    if (!(t > 0.0) || !std::isfinite(t)) return LAPSUM_EINVAL;
    const int vec = (aligned16(r) && aligned16(v) && aligned16(g) &&
                     (ld % (dtype == LAPSUM_DTYPE_F32 ? 4 : 8)) == 0)
                        ? 1
                        : 0;
    return cuda_status(launch_onchip_backward_router(r, dtype, ld, b, v, g, B, (int)n, t, vec,
                                                     (cudaStream_t)stream));
}

size_t lapsum_workspace_bytes_lowp(int64_t B, int64_t n, int64_t ld, double k, int path) {
    if (B < 1 || n < 1 || ld < n) return 0;
    const size_t base = lapsum_workspace_bytes(B, n, k, path);
    if (base == 0) return 0;
    return up(base) + up((size_t)B * (size_t)ld * sizeof(float));
}

size_t lapsum_backward_workspace_bytes_lowp(int64_t B, int64_t n, int64_t ld) {
    if (B < 1 || n < 1 || ld < n) return 0;
    return up(lapsum_backward_workspace_bytes(B, n)) + up((size_t)B * (size_t)ld * sizeof(float));
}

int lapsum_forward_lowp(const void* r, int dtype, int64_t ld, float* p, double* b, double* sum_f,
                        int64_t B, int64_t n, double k, double t, int path, uint64_t seed,
                        void* ws, size_t ws_bytes, void* support, size_t support_size,
                        void* stream) {
    if (r == nullptr || p == nullptr || b == nullptr || !valid_dtype(dtype)) return LAPSUM_EINVAL;
    if (B < 1 || n < 1 || ld < n) return LAPSUM_EINVAL;
    if (!(k > 0.0) || !(k < (double)n) || !std::isfinite(k)) return LAPSUM_EINVAL;
    if (!(t > 0.0) || !std::isfinite(t)) return LAPSUM_EINVAL;
    if (dtype == LAPSUM_DTYPE_F32)
        return forward_impl(static_cast<const float*>(r), ld, p, b, sum_f, B, n, k, nullptr, t,
                            path, seed, ws, ws_bytes, support, support_size, stream);
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return LAPSUM_EWORKSPACE;
    const int pc = path & 0xff;
    if (n <= kOnchipMax && (pc == LAPSUM_PATH_AUTO || pc == LAPSUM_PATH_FULLSORT)) {
        // the on-chip kernels read the 16-bit scores themselves
        const Layout L = make_layout(B, n, LAPSUM_PATH_FULLSORT);
        if (ws_bytes < L.total) return LAPSUM_EWORKSPACE;
        WsHeader* hdr = reinterpret_cast<WsHeader*>(static_cast<char*>(ws) + L.header);
        const int vec = (aligned16(r) && aligned16(p) && (ld % 8) == 0) ? 1 : 0;
        return cuda_status(launch_onchip_router(r, dtype, ld, p, b, sum_f, B, (int)n, k, t, hdr,
                                                vec, nullptr, nullptr, nullptr, 0, 0.f,
                                                pc == LAPSUM_PATH_AUTO ? 1 : 0,
                                                (cudaStream_t)stream));
    }
    const size_t base = lapsum_workspace_bytes(B, n, k, path);
    if (base == 0) return LAPSUM_EINVAL;
    if (ws_bytes < up(base) + up((size_t)B * (size_t)ld * sizeof(float))) return LAPSUM_EWORKSPACE;
    float* wide = reinterpret_cast<float*>(static_cast<char*>(ws) + up(base));
    if (launch_widen(r, dtype, ld, B, n, wide, (cudaStream_t)stream) != cudaSuccess)
        return LAPSUM_ECUDA;
    return forward_impl(wide, ld, p, b, sum_f, B, n, k, nullptr, t, path, seed, ws, up(base),
                        support, support_size, stream);
}

int lapsum_backward_lowp(const void* r, int dtype, int64_t ld, const double* b, const float* v,
                         float* g, int64_t B, int64_t n, double t, const void* support,
                         size_t support_size, void* ws, size_t ws_bytes, void* stream) {
    if (r == nullptr || b == nullptr || v == nullptr || g == nullptr || !valid_dtype(dtype))
        return LAPSUM_EINVAL;
    if (B < 1 || n < 1 || ld < n) return LAPSUM_EINVAL;
    if (!(t > 0.0) || !std::isfinite(t)) return LAPSUM_EINVAL;
    if (dtype == LAPSUM_DTYPE_F32 || n <= kOnchipMax) {
        if (n <= kOnchipMax)
            return lapsum_backward_router(r, dtype, ld, b, v, g, B, n, t, stream);
        const float* rf = static_cast<const float*>(r);
        return support != nullptr
                   ? lapsum_backward_support(rf, ld, b, v, g, B, n, t, support, support_size, ws,
                                             ws_bytes, stream)
                   : lapsum_backward(rf, ld, b, v, g, B, n, t, ws, ws_bytes, stream);
    }
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return LAPSUM_EWORKSPACE;
    const size_t base = up(lapsum_backward_workspace_bytes(B, n));
    if (ws_bytes < base + up((size_t)B * (size_t)ld * sizeof(float))) return LAPSUM_EWORKSPACE;
    float* wide = reinterpret_cast<float*>(static_cast<char*>(ws) + base);
    if (launch_widen(r, dtype, ld, B, n, wide, (cudaStream_t)stream) != cudaSuccess)
        return LAPSUM_ECUDA;
    return support != nullptr
               ? lapsum_backward_support(wide, ld, b, v, g, B, n, t, support, support_size, ws,
                                         base, stream)
               : lapsum_backward(wide, ld, b, v, g, B, n, t, ws, base, stream);
}

int lapsum_forward_rowk(const float* r, int64_t ld, float* p, double* b, double* sum_f, int64_t B,
                        int64_t n, const double* k, double t, int path, void* ws, size_t ws_bytes,
                        void* support, size_t support_size, void* stream) {
    if (k == nullptr) return LAPSUM_EINVAL;
    return forward_impl(r, ld, p, b, sum_f, B, n, 0.0, k, t, path, 0, ws, ws_bytes, support,
                        support_size, stream);
}

int lapsum_forward_support(const float* r, int64_t ld, float* p, double* b, double* sum_f,
                           int64_t B, int64_t n, double k, double t, int path, uint64_t seed,
                           void* ws, size_t ws_bytes, void* support, size_t support_size,
                           void* stream) {
    if (support == nullptr && n > kOnchipMax) return LAPSUM_EWORKSPACE;
    return forward_impl(r, ld, p, b, sum_f, B, n, k, nullptr, t, path, seed, ws, ws_bytes, support,
                        support_size, stream);
}

int lapsum_backward_support(const float* r, int64_t ld, const double* b, const float* v, float* g,
                            int64_t B, int64_t n, double t, const void* support,
                            size_t support_size, void* ws, size_t ws_bytes, void* stream) {
    if (r == nullptr || b == nullptr || v == nullptr || g == nullptr) return LAPSUM_EINVAL;
    if (B < 1 || n < 1 || ld < n) return LAPSUM_EINVAL;
    if (!(t > 0.0) || !std::isfinite(t)) return LAPSUM_EINVAL;
    cudaStream_t st = (cudaStream_t)stream;
    const int vec = (aligned16(r) && aligned16(v) && aligned16(g) && (ld % 4) == 0) ? 1 : 0;
    if (n <= kOnchipMax) {
        return cuda_status(launch_onchip_backward(r, ld, b, v, g, B, (int)n, t, vec, st));
    }
    if (support == nullptr || (reinterpret_cast<uintptr_t>(support) % kAlign) != 0 ||
        support_size < support_bytes(B, n))
        return LAPSUM_EWORKSPACE;
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return LAPSUM_EWORKSPACE;
    const Layout L = make_layout(B, n, LAPSUM_PATH_FULLSORT);  // the streaming buffers only
    if (ws_bytes < L.total) return LAPSUM_EWORKSPACE;
    char* w = static_cast<char*>(ws);
    uint32_t* tickets = reinterpret_cast<uint32_t*>(w + L.tickets);
    double* partials = reinterpret_cast<double*>(w + L.partials);
    double* row_R = reinterpret_cast<double*>(w + L.row_R);
    uint32_t* dflag = reinterpret_cast<uint32_t*>(w + L.wflag);
    const SupportView sv_all = support_view(const_cast<void*>(support), B, n);
    cudaError_t e = cudaSuccess;
    for (int64_t r0 = 0; r0 < B && e == cudaSuccess; r0 += kGridYMax) {
        const int64_t nb = (B - r0 < kGridYMax) ? B - r0 : kGridYMax;
        e = launch_backward_support(r + r0 * ld, ld, b + r0, v + r0 * ld, g + r0 * ld, nb, n, t,
                                    support_rows(sv_all, r0, n), B, partials + r0 * stream_tiles(n) * 4,
                                    row_R + r0, tickets + B + r0, dflag + r0, vec, st);
    }
    return cuda_status(e);
}

int lapsum_backward(const float* r, int64_t ld, const double* b, const float* v, float* g,
                    int64_t B, int64_t n, double t, void* ws, size_t ws_bytes, void* stream) {
    if (r == nullptr || b == nullptr || v == nullptr || g == nullptr) return LAPSUM_EINVAL;
    if (B < 1 || n < 1 || ld < n) return LAPSUM_EINVAL;
    if (!(t > 0.0) || !std::isfinite(t)) return LAPSUM_EINVAL;
    cudaStream_t st = (cudaStream_t)stream;
    const int vec = (aligned16(r) && aligned16(v) && aligned16(g) && (ld % 4) == 0) ? 1 : 0;
    if (n <= kOnchipMax) {
        return cuda_status(launch_onchip_backward(r, ld, b, v, g, B, (int)n, t, vec, st));
    }
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return LAPSUM_EWORKSPACE;
    const Layout L = make_layout(B, n, LAPSUM_PATH_FULLSORT);  // the streaming buffers only
    if (ws_bytes < L.total) return LAPSUM_EWORKSPACE;
    char* w = static_cast<char*>(ws);
    uint32_t* tickets = reinterpret_cast<uint32_t*>(w + L.tickets);
    double* partials = reinterpret_cast<double*>(w + L.partials);
    double* row_R = reinterpret_cast<double*>(w + L.row_R);
    cudaError_t e = cudaSuccess;
    const bool windowed = n <= (int64_t)0xffffffffll;  // window entries index rows with 32 bits
    for (int64_t r0 = 0; r0 < B && e == cudaSuccess; r0 += kGridYMax) {
        const int64_t nb = (B - r0 < kGridYMax) ? B - r0 : kGridYMax;
        if (windowed) {
            WindowBuffers wb;
            wb.list = reinterpret_cast<WinEntry*>(w + L.wlist);
            wb.tab = reinterpret_cast<uint2*>(w + L.wtab) + r0 * window_tiles(n);
            wb.flag = reinterpret_cast<uint32_t*>(w + L.wflag) + r0;
            e = launch_backward_window(r + r0 * ld, ld, b + r0, v + r0 * ld, g + r0 * ld, nb, n,
                                       t, wb, partials + r0 * stream_tiles(n) * 4, row_R + r0,
                                       tickets + B + r0, vec, st);
        } else {
            e = launch_backward_stream(r + r0 * ld, ld, b + r0, v + r0 * ld, g + r0 * ld, nb, n,
                                       t, partials + r0 * stream_tiles(n) * 4, row_R + r0,
                                       tickets + B + r0, vec, st);
        }
    }
    return cuda_status(e);
}

int lapsum_backward_kt(const float* r, int64_t ld, const double* b, const float* v, int64_t B,
                       int64_t n, double t, double* g_k, double* g_t, void* ws, size_t ws_bytes,
                       void* stream) {
    if (r == nullptr || b == nullptr || v == nullptr || (g_k == nullptr && g_t == nullptr))
        return LAPSUM_EINVAL;
    if (B < 1 || n < 1 || ld < n) return LAPSUM_EINVAL;
    if (!(t > 0.0) || !std::isfinite(t)) return LAPSUM_EINVAL;
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return LAPSUM_EWORKSPACE;
    const Layout L = make_layout(B, n, LAPSUM_PATH_FULLSORT);
    if (ws_bytes < L.total) return LAPSUM_EWORKSPACE;
    char* w = static_cast<char*>(ws);
    uint32_t* tickets = reinterpret_cast<uint32_t*>(w + L.tickets);
    double* partials = reinterpret_cast<double*>(w + L.partials);
    const int vec = (aligned16(r) && aligned16(v) && (ld % 4) == 0) ? 1 : 0;
    const int64_t slots = stream_tiles(n) > 2 ? stream_tiles(n) : 2;
    cudaError_t e = cudaSuccess;
    for (int64_t r0 = 0; r0 < B && e == cudaSuccess; r0 += kGridYMax) {
        const int64_t nb = (B - r0 < kGridYMax) ? B - r0 : kGridYMax;
        e = launch_backward_kt(r + r0 * ld, ld, b + r0, v + r0 * ld, nb, n, t,
                               partials + r0 * slots * 4, tickets + B + r0,
                               g_k ? g_k + r0 : nullptr, g_t ? g_t + r0 : nullptr, vec,
                               static_cast<cudaStream_t>(stream));
    }
    return cuda_status(e);
}

int lapsum_read_status(void* ws, void* stream, int* device_status) {
    if (ws == nullptr || device_status == nullptr) return LAPSUM_EINVAL;
    cudaStream_t st = (cudaStream_t)stream;
    WsHeader* hdr = static_cast<WsHeader*>(ws);
    uint32_t bits = 0;
    cudaError_t e = cudaMemcpyAsync(&bits, &hdr->status, sizeof(bits), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaMemsetAsync(&hdr->status, 0, sizeof(uint32_t), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return LAPSUM_ECUDA;
    *device_status = (bits & kDevWaitTimeout) ? LAPSUM_ECUDA
                     : (bits & kDevNonFinite) ? LAPSUM_ENONFINITE
                     : (bits & kDevBadBudget) ? LAPSUM_EINVAL
                     : (bits & kDevBracketExhausted) ? LAPSUM_EBRACKET
                                                     : LAPSUM_OK;
    return LAPSUM_OK;
}

int lapsum_row_info_get(void* ws, int64_t row, lapsum_row_info* out, void* stream) {
    if (ws == nullptr || out == nullptr || row < 0) return LAPSUM_EINVAL;
    cudaStream_t st = (cudaStream_t)stream;
    // The record's offset depends on (B, n, path) of the last forward call,
    // which that call left in the workspace header.
    RowState rs;
    WsHeader h;
    cudaError_t e = cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return LAPSUM_ECUDA;
    if (h.last_B <= 0 || row >= h.last_B || h.last_path == LAPSUM_PATH_FULLSORT)
        return LAPSUM_EINVAL;
    const Layout L = make_layout(h.last_B, h.last_n, (int)h.last_path);
    const char* base = static_cast<const char*>(ws) + L.rows + (size_t)row * sizeof(RowState);
    e = cudaMemcpyAsync(&rs, base, sizeof(rs), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return LAPSUM_ECUDA;
    std::memset(out, 0, sizeof(*out));
    out->b = rs.b;
    out->sum_f = rs.sum_f;
    out->S_L = rs.S_L;
    out->S_R = rs.S_R;
    out->a_L = rs.a_L;
    out->a_R = rs.a_R;
    out->cnt_R = (int64_t)rs.cnt_R;
    out->n_band = (int64_t)rs.n_band;
    out->path = rs.path;
    out->attempts = rs.attempts;
    out->sample_m = rs.sample_m;
    out->rank_l = rs.rank_l;
    out->rank_h = rs.rank_h;
    out->refine_levels = rs.refine_levels;
    out->status = (int32_t)rs.status;
    return LAPSUM_OK;
}

int lapsum_profile_enable(int on) {
    Profiler& p = profiler();
    std::lock_guard<std::mutex> g(p.mu);
    p.recycle();
    p.on = on != 0;
    return LAPSUM_OK;
}

int lapsum_profile_read(lapsum_kernel_time* out, int max_entries, int* n_entries) {
    if (n_entries == nullptr || (out == nullptr && max_entries > 0)) return LAPSUM_EINVAL;
    Profiler& p = profiler();
    std::lock_guard<std::mutex> g(p.mu);
    std::vector<lapsum_kernel_time> acc;
    for (auto& r : p.recs) {
        if (cudaEventSynchronize(r.b) != cudaSuccess) return LAPSUM_ECUDA;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) return LAPSUM_ECUDA;
        size_t i = 0;
        for (; i < acc.size(); ++i)
            if (std::strncmp(acc[i].name, r.name, sizeof(acc[i].name)) == 0) break;
        if (i == acc.size()) {
            lapsum_kernel_time kt;
            std::memset(&kt, 0, sizeof(kt));
            std::strncpy(kt.name, r.name, sizeof(kt.name) - 1);
            acc.push_back(kt);
        }
        acc[i].launches += 1;
        acc[i].total_ms += (double)ms;
    }
    *n_entries = (int)acc.size();
    for (int i = 0; i < (int)acc.size() && i < max_entries; ++i) out[i] = acc[i];
    return LAPSUM_OK;
}

int lapsum_sample_get(void* ws, int64_t row, float* out, int64_t m, void* stream) {
    if (ws == nullptr || out == nullptr || row < 0 || m < 1 || m > kSampleMax) return LAPSUM_EINVAL;
    cudaStream_t st = (cudaStream_t)stream;
    WsHeader h;
    cudaError_t e = cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return LAPSUM_ECUDA;
    if (h.last_path != LAPSUM_PATH_BRACKET || row >= h.last_B) return LAPSUM_EINVAL;
    const Layout L = make_layout(h.last_B, h.last_n, LAPSUM_PATH_BRACKET);
    const char* base = static_cast<const char*>(ws) + L.sample + (size_t)row * kSampleMax * 4;
    e = cudaMemcpyAsync(out, base, (size_t)m * sizeof(float), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return cuda_status(e);
}

}  // extern "C"
