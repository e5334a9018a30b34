// Backward of long rows from the gradient support left by the forward.
//
// The VJP of "Fast LapSum: Exact Differentiable Top-k at Million Scale"
// (gist.science explainer pages), section 2.1, is g_i = (f_i/t)(v_i - R) with
// f_i = 0.5 exp(-|x_i|), x_i = (r_i - b)/t and R = sum v f / sum f.  f_i is 0
// in fp32 once |x_i| > 87.4, so only the scores with |x| <= 90 carry gradient.
// The forward's emit pass already computes every x_i; with the support output
// it also lists those scores (position in the tile and x) per warp share of
// each 4096-score tile.  The backward then never reads r:
//
// Pass A (sup_reduce_kernel): one wave of resident CTAs; each walks groups of
//   up to 32 tiles, scans the shares' counts, and works through the listed
//   entries with all its threads: v is gathered at each entry (and kept next
//   to it for pass B), the terms go into an online (mu, sum w, sum w v),
//   w = exp(-(|x| - mu)).  The last CTA of the row combines the CTA records in
//   a fixed order into R and decides whether the list serves the row.
// Pass B (sup_write_kernel): one CTA per tile, one warp per share; the share is
//   zeroed in shared memory, its entries are placed, and it is written out
//   with coalesced 16-byte stores, so every g value is written exactly once.
//
// A row is computed densely (v and r read everywhere) by the same two kernels
// when its list overflowed, was written for another (n, B) or another b, or
// no score of the row has |x| <= 50 (then scores outside the list could weigh
// in R); the forward's emit pass records the first and the last of these per
// row, so every CTA knows the row's mode before it starts.
#include <atomic>

#include "lapsum_common.cuh"
#include "lapsum_kernels.h"
#include "stream_common.cuh"

namespace lapsum {
namespace {

using stream_detail::online_add;
using stream_detail::online_add4;
constexpr int kThreads = 256;
constexpr int kTile = kStreamTile;
constexpr int kShares = kSupWarps;
constexpr int kGroupMax = kThreads / kShares;  // tiles per pass-A CTA (one share per thread)
constexpr size_t kAlignSup = 256;

size_t up256(size_t x) { return (x + kAlignSup - 1) / kAlignSup * kAlignSup; }

// L2 eviction-priority hints: the list (entries and gathered v, a few percent
// of the row) is read again by pass B, so pass A keeps it with evict_last
// while the gathers of v stream through.
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint2 ld_keep(const uint2* p, uint64_t pol) {
    uint2 v;
    asm volatile("ld.global.L2::cache_hint.v2.u32 {%0, %1}, [%2], %3;"
                 : "=r"(v.x), "=r"(v.y)
                 : "l"(p), "l"(pol));
    return v;
}
__device__ __forceinline__ void st_keep(float* p, float v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(pol)
                 : "memory");
}

// Merges a record (m, s, sv) -- sums of weights relative to e^{-m} -- into
// the running (mu, S, Sv); a smaller m rescales the running sums.
__device__ __forceinline__ void online_merge(float m, double s, double sv, float& mu, double& S,
                                             double& Sv) {
    if (m == INFINITY) return;
    if (m < mu) {
        const double sc = (mu == INFINITY) ? 0.0 : exp((double)m - (double)mu);
        S *= sc;
        Sv *= sc;
        mu = m;
    }
    const double f = exp((double)mu - (double)m);
    S += s * f;
    Sv += sv * f;
}

// The online sums of every thread of the CTA combined into thread 0 (one
// barrier): warp shuffles, then thread 0 merges the warps in order.
__device__ __forceinline__ void cta_online_combine(float& mu, double& s, double& sv, float* wmu,
                                                   double* ws, double* wsv) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const float mw = warp_min_f(mu);
    const double sc = (mu == INFINITY) ? 0.0 : exp((double)mw - (double)mu);
    const double s_w = warp_sum_d(s * sc), sv_w = warp_sum_d(sv * sc);
    if (lane == 0) {
        wmu[w] = mw;
        ws[w] = s_w;
        wsv[w] = sv_w;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = INFINITY;
        double a = 0.0, av = 0.0;
        for (int u = 0; u < kThreads / 32; ++u) online_merge(wmu[u], ws[u], wsv[u], m, a, av);
        mu = m;
        s = a;
        sv = av;
    }
}

__device__ __forceinline__ void sup_add(float ax, float vv, float& mu, double& s, double& sv) {
    if (ax < mu) {
        const double sc = (mu == INFINITY) ? 0.0 : (double)__expf(ax - mu);
        s *= sc;
        sv *= sc;
        mu = ax;
    }
    const float w = __expf(mu - ax);
    s += (double)w;
    sv += (double)(w * vv);
}

// The row's mode: the list serves it unless it was written for another call
// shape or threshold, overflowed, or no score has |x| <= 50.
__device__ __forceinline__ bool row_is_dense(const SupportView& sup, const double* b,
                                             int64_t row, int64_t n, int64_t B_total) {
    const bool match = sup.hdr[0] == n && sup.hdr[1] == B_total &&
                       __double_as_longlong(sup.b[row]) == __double_as_longlong(b[row]);
    const uint32_t fl = sup.flags[row];
    return !match || (fl & kSupOverflow) != 0u || (fl & kSupNear) == 0u;
}

template <bool VEC>
__global__ void __launch_bounds__(kThreads, 5) sup_reduce_kernel(
    const float* __restrict__ r, const double* __restrict__ b, const float* __restrict__ v,
    int64_t ld, int64_t n, double t, int64_t B_total, int group, SupportView sup,
    double* __restrict__ partials, double* __restrict__ row_R, uint32_t* __restrict__ tickets,
    uint32_t* __restrict__ dense_flag) {
    pdl_wait();
    __shared__ uint32_t pre[kThreads + 1];  // exclusive prefix of the group's share counts
    __shared__ uint32_t wtot[kThreads / 32];
    __shared__ float wmu[kThreads / 32];
    __shared__ double ws[kThreads / 32], wsv[kThreads / 32];
    __shared__ int flag;
    const int64_t row = blockIdx.y;
    const int64_t nblk = gridDim.x;
    const int64_t tiles = (n + kTile - 1) / kTile;
    const int64_t ngroups = (tiles + group - 1) / group;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float* vr = v + row * ld;
    const bool dense = row_is_dense(sup, b, row, n, B_total);
    float mu = INFINITY;
    double s = 0.0, sv = 0.0;
    if (dense) {
        // every score of the row: this CTA's strided share of it
        const Thr th = make_thr(b[row], t);
        const float* rr = r + row * ld;
        const int64_t stride = nblk * kThreads;
        const int64_t gt = (int64_t)blockIdx.x * kThreads + threadIdx.x;
        if (VEC) {
            const int64_t n4 = n >> 2;
            const float4* r4 = reinterpret_cast<const float4*>(rr);
            const float4* v4 = reinterpret_cast<const float4*>(vr);
            for (int64_t i = gt; i < n4; i += stride) {
                const float4 x0 = __ldcs(r4 + i), y0 = __ldcs(v4 + i);
                online_add4(fabsf(scaled_margin(x0.x, th)), fabsf(scaled_margin(x0.y, th)),
                            fabsf(scaled_margin(x0.z, th)), fabsf(scaled_margin(x0.w, th)), y0.x,
                            y0.y, y0.z, y0.w, mu, s, sv);
            }
            for (int64_t j = (n4 << 2) + gt; j < n; j += stride)
                online_add(fabsf(scaled_margin(rr[j], th)), vr[j], mu, s, sv);
        } else {
            for (int64_t j = gt; j < n; j += stride)
                online_add(fabsf(scaled_margin(rr[j], th)), vr[j], mu, s, sv);
        }
    }
    const uint64_t keep = l2_evict_last_policy();
    // count of share i of group gi: (tile gi * group + i / 8, share i % 8), or 0
    // (the buffer holds a list for this (n, B) whatever it was written for,
    // so the counts load without waiting for the match test)
    auto share_count = [&](int64_t gi) -> uint32_t {
        const int64_t t0 = gi * group;
        const int64_t t1 = t0 + group < tiles ? t0 + group : tiles;
        if (gi >= ngroups || t0 + (int64_t)threadIdx.x / kShares >= t1) return 0u;
        return __ldcs(sup.cnt + (row * tiles + t0) * kShares + threadIdx.x);
    };
    // persistent over groups of tiles; the next group's counts load while
    // the current group's entries are gathered
    uint32_t c_next = dense ? 0u : share_count(blockIdx.x);
    for (int64_t gi = dense ? ngroups : blockIdx.x; gi < ngroups; gi += nblk) {
        const int64_t t0 = gi * group;
        uint32_t c = c_next;
        if (c > (uint32_t)kSupCap) c = 0;  // an overflowed row is dense (not reached)
        // block exclusive scan of the counts
        uint32_t inc = c;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t o = __shfl_up_sync(0xffffffffu, inc, d);
            if (lane >= d) inc += o;
        }
        __syncthreads();  // the previous group is done with pre[] and wtot[]
        if (lane == 31) wtot[warp] = inc;
        __syncthreads();
        uint32_t wpre = 0;
        for (int u = 0; u < warp; ++u) wpre += wtot[u];
        pre[threadIdx.x] = wpre + inc - c;
        if (threadIdx.x == kThreads - 1) pre[kThreads] = wpre + inc;
        __syncthreads();
        c_next = share_count(gi + nblk);
        const uint32_t total = pre[kThreads];
        const uint2* ent = sup.ent + (row * tiles + t0) * kShares * kSupCap;
        float* val = sup.val + (row * tiles + t0) * kShares * kSupCap;
        const float* vg = vr + t0 * kTile;                  // v of the group's first tile
        const int64_t lim = n - t0 * kTile;                 // scores of the row from there on
        constexpr int U = 4;  // entries per thread in flight
        for (uint32_t j0 = 0; j0 < total; j0 += U * kThreads) {
            uint2 e[U];
            int32_t slot[U];
            int32_t gpos[U];  // position from the group's first score
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t j = j0 + u * kThreads + threadIdx.x;
                ok[u] = j < total;
                slot[u] = 0;
                gpos[u] = 0;
                if (ok[u]) {
                    // share holding entry j: the last with pre[share] <= j
                    int lo = 0, hi = kThreads - 1;
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if (pre[mid] <= j) lo = mid;
                        else hi = mid - 1;
                    }
                    slot[u] = lo * kSupCap + (int32_t)(j - pre[lo]);
                    e[u] = ld_keep(ent + slot[u], keep);
                    gpos[u] = (lo / kShares) * kTile;
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (!ok[u]) continue;
                gpos[u] += (int32_t)(e[u].x & (kTile - 1));
                if (gpos[u] >= lim) ok[u] = false;  // never past the row
            }
            float vv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) vv[u] = ok[u] ? __ldcs(vg + gpos[u]) : 0.f;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (!ok[u]) continue;
                const float ax = fabsf(__uint_as_float(e[u].y));
                sup_add(ax, vv[u], mu, s, sv);
                st_keep(val + slot[u], vv[u], keep);
            }
        }
    }
    // CTA record (mu, S, Sv): one barrier
    cta_online_combine(mu, s, sv, wmu, ws, wsv);
    if (threadIdx.x == 0) {
        double* pr = partials + (row * nblk + blockIdx.x) * 4;
        pr[0] = (double)mu;
        pr[1] = s;
        pr[2] = sv;
        __threadfence();
        const uint32_t prev = atomicAdd(&tickets[row], 1u);
        flag = (prev == (uint32_t)nblk - 1u);
        if (flag) tickets[row] = 0u;
    }
    __syncthreads();
    if (!flag) return;
    __threadfence();
    // the row's records in CTA order, each thread's share combined online
    float mloc = INFINITY;
    double a = 0.0, av = 0.0;
    for (int64_t k = threadIdx.x; k < nblk; k += kThreads) {
        const double* pr = partials + (row * nblk + k) * 4;
        online_merge((float)__ldcg(pr), __ldcg(pr + 1), __ldcg(pr + 2), mloc, a, av);
    }
    cta_online_combine(mloc, a, av, wmu, ws, wsv);
    if (threadIdx.x == 0) {
        row_R[row] = dense ? av / a : (a > 0.0 ? av / a : 0.0);
        dense_flag[row] = dense ? 1u : 0u;
    }
}

// g for one tile per CTA: zeroed in shared memory, the listed entries placed,
// then written with 16-byte streaming stores.
// g from the list, one CTA per tile.  Each warp owns one share of the tile,
// the same 512 scores the emit kernel's warp listed (four runs of 128 at
// q * 1024 + warp * 128), so no warp needs another's entries and there is no
// block barrier.  The share's count and its first 32 entries are loaded
// together (the entries speculatively), so a tile costs one memory round
// trip; the share is zeroed in the warp's 2 KB of shared memory, its entries
// are placed, and it is written with 16-byte streaming stores.
// Rows computed densely take g = (f/t)(v - R) from r and v over the tile.
template <bool VEC>
__global__ void __launch_bounds__(kThreads) sup_write_kernel(
    SupportView sup, const uint32_t* __restrict__ dense_flag, const double* __restrict__ row_R,
    const float* __restrict__ r, const double* __restrict__ b, const float* __restrict__ v,
    float* __restrict__ g, int64_t ld, int64_t n, double t) {
    pdl_wait();
    __shared__ __align__(16) float stage[kShares][kTile / kShares];
    const int64_t row = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t tiles = (n + kTile - 1) / kTile;
    const int64_t T = blockIdx.x;
    const int64_t base = T * kTile;
    const int64_t share = (row * tiles + T) * kShares + warp;
    const uint2* ent = sup.ent + share * kSupCap;
    const float* val = sup.val + share * kSupCap;
    // independent loads, issued together
    const uint32_t dflag = dense_flag[row];
    const double R = row_R[row];
    const uint32_t c = __ldcs(sup.cnt + share);  // <= kSupCap: checked by pass A
    const uint2 e0 = __ldcs(ent + lane);
    const float v0 = __ldcs(val + lane);
    if (dflag) {
        // four scores at a time, in the striped order of the other tile kernels
        const Thr th = make_thr(b[row], t);
        const float* rr = r + row * ld;
        const float* vr = v + row * ld;
        float* gr = g + row * ld;
        auto g_of = [&](float x, float vv) {
            const float f = 0.5f * neg_abs_exp(scaled_margin(x, th));
            return f * th.inv_t * (float)((double)vv - R);
        };
#pragma unroll 1
        for (int q = 0; q < kTile / (4 * kThreads); ++q) {
            const int64_t i0 = base + ((int64_t)q * kThreads + threadIdx.x) * 4;
            if (VEC && i0 + 4 <= n) {
                const float4 x = __ldcs(reinterpret_cast<const float4*>(rr + i0));
                const float4 y = __ldcs(reinterpret_cast<const float4*>(vr + i0));
                __stcs(reinterpret_cast<float4*>(gr + i0),
                       make_float4(g_of(x.x, y.x), g_of(x.y, y.y), g_of(x.z, y.z), g_of(x.w, y.w)));
            } else {
                for (int c = 0; c < 4; ++c)
                    if (i0 + c < n) gr[i0 + c] = g_of(rr[i0 + c], vr[i0 + c]);
            }
        }
        return;
    }
    const float hinv = (float)(0.5 / t);
    float* st = stage[warp];
    float4* s4 = reinterpret_cast<float4*>(st);
    constexpr int kRun = kTile / kShares / 4;  // 128 scores per run, four runs per share
    const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q = 0; q < 4; ++q) s4[q * 32 + lane] = z4;
    __syncwarp();
    auto place = [&](uint2 en, float vv) {
        const uint32_t p = en.x & (kTile - 1);
        const uint32_t li = (p >> 10) * kRun + (p & (kRun - 1));  // run q = p / 1024
        st[li] = hinv * __expf(-fabsf(__uint_as_float(en.y))) * (float)((double)vv - R);
    };
    if ((uint32_t)lane < c) place(e0, v0);
    for (uint32_t e = 32 + lane; e < c; e += 32) place(__ldcs(ent + e), __ldcs(val + e));
    __syncwarp();
    float* gs = g + row * ld + base + warp * kRun;
    if (VEC && base + kTile <= n) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
            __stcs(reinterpret_cast<float4*>(gs + q * 1024) + lane, s4[q * 32 + lane]);
    } else {
        for (int q = 0; q < 4; ++q)
            for (int e = lane; e < kRun; e += 32)
                if (base + warp * kRun + q * 1024 + e < n) gs[q * 1024 + e] = st[q * kRun + e];
    }
}

struct SupOffsets {
    size_t hdr, b, flags, cnt, ent, val, total;
};

SupOffsets sup_offsets(int64_t B, int64_t n) {
    const size_t tiles = (size_t)stream_tiles(n);
    SupOffsets o{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += up256(bytes);
        return at;
    };
    o.hdr = take(2 * sizeof(int64_t));
    o.b = take((size_t)B * sizeof(double));
    o.flags = take((size_t)B * sizeof(uint32_t));
    o.cnt = take((size_t)B * tiles * kShares * sizeof(uint32_t));
    o.ent = take((size_t)B * tiles * kShares * kSupCap * sizeof(uint2));
    o.val = take((size_t)B * tiles * kShares * kSupCap * sizeof(float));
    o.total = off;
    return o;
}

}  // namespace

size_t support_bytes(int64_t B, int64_t n) { return sup_offsets(B, n).total; }

SupportView support_view(void* base, int64_t B, int64_t n) {
    const SupOffsets o = sup_offsets(B, n);
    char* p = static_cast<char*>(base);
    SupportView s;
    s.hdr = reinterpret_cast<int64_t*>(p + o.hdr);
    s.b = reinterpret_cast<double*>(p + o.b);
    s.flags = reinterpret_cast<uint32_t*>(p + o.flags);
    s.cnt = reinterpret_cast<uint32_t*>(p + o.cnt);
    s.ent = reinterpret_cast<uint2*>(p + o.ent);
    s.val = reinterpret_cast<float*>(p + o.val);
    return s;
}

SupportView support_rows(const SupportView& s, int64_t r0, int64_t n) {
    const int64_t per_row = stream_tiles(n) * kShares;
    SupportView o = s;
    o.b += r0;
    o.flags += r0;
    o.cnt += r0 * per_row;
    o.ent += r0 * per_row * kSupCap;
    o.val += r0 * per_row * kSupCap;
    return o;
}

cudaError_t launch_backward_support(const float* r, int64_t ld, const double* b, const float* v,
                                    float* g, int64_t B, int64_t n, double t,
                                    const SupportView& sup, int64_t B_total, double* partials,
                                    double* row_R, uint32_t* tickets, uint32_t* dense_flag,
                                    int vec, cudaStream_t st) {
    const int64_t tiles = stream_tiles(n);
    // pass A: one wave of resident CTAs walking groups of up to 32 tiles;
    // pass B: one CTA per tile
    // resident CTAs per SM of pass A, per device
    constexpr int kMaxDevices = 64;
    static std::atomic<int> per_sm[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    int per_sm_a = (dev >= 0 && dev < kMaxDevices) ? per_sm[dev].load(std::memory_order_relaxed) : 0;
    if (per_sm_a == 0) {
        int pa = 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&pa, sup_reduce_kernel<true>, kThreads, 0);
        per_sm_a = pa > 0 ? pa : 1;
        if (dev >= 0 && dev < kMaxDevices) per_sm[dev].store(per_sm_a, std::memory_order_relaxed);
    }
    const int cap_a = per_sm_a * device_sm_count();
    int64_t want = cap_a / B;
    if (want < 1) want = 1;
    // groups of at most 32 tiles, as many per CTA as it takes, all CTAs alike
    const int64_t rounds = (tiles + kGroupMax * want - 1) / (kGroupMax * want);
    int64_t group = (tiles + rounds * want - 1) / (rounds * want);
    if (group < 1) group = 1;
    if (group > kGroupMax) group = kGroupMax;
    const int64_t ngroups = (tiles + group - 1) / group;
    const int64_t per_row = ngroups < want ? ngroups : want;
    {
        ProfScope ps_("sup_reduce", st);
        const dim3 grid((unsigned)per_row, (unsigned)B);
        if (vec)
            launch_pdl(sup_reduce_kernel<true>, grid, dim3(kThreads), 0, st, r, b, v, ld, n, t,
                       B_total, (int)group, sup, partials, row_R, tickets, dense_flag);
        else
            launch_pdl(sup_reduce_kernel<false>, grid, dim3(kThreads), 0, st, r, b, v, ld, n, t,
                       B_total, (int)group, sup, partials, row_R, tickets, dense_flag);
    }
    {
        ProfScope ps_("sup_write", st);
        const dim3 grid((unsigned)tiles, (unsigned)B);
        if (vec)
            launch_pdl(sup_write_kernel<true>, grid, dim3(kThreads), 0, st, sup, dense_flag, row_R,
                       r, b, v, g, ld, n, t);
        else
            launch_pdl(sup_write_kernel<false>, grid, dim3(kThreads), 0, st, sup, dense_flag, row_R,
                       r, b, v, g, ld, n, t);
    }
    return cudaGetLastError();
}

}  // namespace lapsum
