// The zero-temperature limit of long rows through probabilistic bracketing,
// with no full sort ("Fast LapSum: Exact Differentiable Top-k at Million
// Scale", gist.science explainer pages: section 2.3 names DFTopK's midpoint
// threshold as LapSum's t -> 0 limit; section 2.2 gives the bracketing steps).
//
// The limit needs the ceil(k)-th largest score c, the number a of scores above
// it and m equal to it, and, when k = a + m, the next lower score.  Rows run in
// parallel (blockIdx.y = row):
//   hard_sample_kernel  m plain samples r[I] per row (no noise at t = 0); each
//                       CTA keeps its top h keys, the row's last CTA sorts the
//                       candidates and takes the binomial order statistics as
//                       the bracket [a_L, a_R);
//   hard_fold_kernel    one pass: the count above a_R, the band [a_L, a_R)
//                       appended to the row's band buffer, the largest score
//                       below a_L;
//   hard_solve_kernel   one CTA per row: when the bracket holds the rank, c, a,
//                       m and the next lower score come from the band (sorted
//                       on chip, or by an exact radix selection when it is
//                       large); otherwise from an exact selection over the
//                       whole row (rare); then b and the share of the boundary
//                       group;
// and the tile emit shared with the full-sort path writes p.
// -0 and +0 are one value throughout (the key of -0 is read as that of +0).
#include <cmath>

#include "bitonic.cuh"
#include "lapsum_common.cuh"
#include "lapsum_kernels.h"

namespace lapsum {
namespace {

constexpr int kBlk = 1024;
constexpr int kFoldThreads = 256;
constexpr int kTile = 4096;

__device__ __forceinline__ float canon(float x) { return x + 0.f; }  // -0 + 0 = +0
__device__ __forceinline__ uint32_t hkey(float x) { return to_key(canon(x)); }

__global__ void __launch_bounds__(kBlk) hard_sample_kernel(const float* __restrict__ r,
                                                           int64_t ld, int64_t n, uint64_t seed,
                                                           int m, int top_h, int64_t rank_l,
                                                           int64_t rank_h, int force_miss,
                                                           uint32_t* __restrict__ cand,
                                                           uint32_t* __restrict__ tickets,
                                                           RowState* rows) {
    __shared__ uint32_t xch[4 * kBlk];
    __shared__ uint32_t bcast[4];
    __shared__ int flag;
    const int64_t row = blockIdx.y;
    RowState* st = rows + row;
    const float* rr = r + row * ld;
    uint32_t* cr = cand + row * (int64_t)(4 * kBlk);
    if (blockIdx.x == 0) {
        for (int i = threadIdx.x; i < (int)(sizeof(RowState) / 4); i += kBlk)
            reinterpret_cast<uint32_t*>(st)[i] = 0u;
    }
    // the same index stream as the soft sample (counter 2s of the row's
    // stream), without the noise
    const int s = blockIdx.x * kBlk + threadIdx.x;
    uint32_t key[1] = {0u};
    if (s < m) {
        const int64_t I = sample_index(seed, (uint64_t)row << 32, s, n);
        key[0] = hkey(__ldg(rr + I));
    }
    bitonic_sort_row<1, kBlk, kBlk>(key, threadIdx.x, xch);
    if (threadIdx.x >= kBlk - top_h)
        cr[blockIdx.x * top_h + (threadIdx.x - (kBlk - top_h))] = key[0];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t prev = atomicAdd(&tickets[row], 1u);
        flag = (prev == gridDim.x - 1);
        if (flag) tickets[row] = 0u;
    }
    __syncthreads();
    if (!flag) return;
    __threadfence();
    const int c = (int)gridDim.x * top_h;
    auto pick = [&](auto e_tag) {
        constexpr int E = decltype(e_tag)::value;
        uint32_t kk[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int j = threadIdx.x * E + e;
            kk[e] = j < c ? __ldcg(cr + j) : 0u;
        }
        bitonic_sort_row<E, kBlk, kBlk>(kk, threadIdx.x, xch);
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int j = threadIdx.x * E + e;
            if (rank_l >= 1 && j == E * kBlk - rank_l) bcast[0] = kk[e];
            if (rank_h >= 1 && j == E * kBlk - rank_h) bcast[1] = kk[e];
            if (j == E * kBlk - 1) bcast[2] = kk[e];
        }
    };
    if (c <= kBlk) pick(std::integral_constant<int, 1>{});
    else if (c <= 2 * kBlk) pick(std::integral_constant<int, 2>{});
    else pick(std::integral_constant<int, 4>{});
    __syncthreads();
    if (threadIdx.x == 0) {
        float aR = rank_l >= 1 ? from_key(bcast[0]) : INFINITY;
        float aL = rank_h >= 1 ? from_key(bcast[1]) : -INFINITY;
        if (force_miss) {
            // above every sample: the bracket misses unless the row's top
            // scores are all equal to the largest sample
            const float top = from_key(bcast[2]);
            aL = top + fabsf(top) + 1.f;
            aR = INFINITY;
        }
        st->a_L = aL;
        st->a_R = aR;
        st->sample_m = m;
        st->rank_l = (int32_t)rank_l;
        st->rank_h = (int32_t)rank_h;
        st->path = LAPSUM_PATH_BRACKET;
        st->force_miss = force_miss;
    }
}

// One 4096-score tile per CTA: counts above a_R, the band appended (staged in
// shared memory, one global atomic per CTA), the largest key below a_L.
__global__ void __launch_bounds__(kFoldThreads) hard_fold_kernel(const float* __restrict__ r,
                                                                 int64_t ld, int64_t n,
                                                                 float* __restrict__ band,
                                                                 RowState* rows, WsHeader* hdr) {
    __shared__ float stage[kTile];
    __shared__ int scount;
    __shared__ unsigned long long sbase;
    __shared__ uint32_t wmax[kFoldThreads / 32];
    __shared__ uint32_t wcnt[kFoldThreads / 32];
    const int64_t row = blockIdx.y;
    RowState* st = rows + row;
    const float aL = st->a_L, aR = st->a_R;
    const float* rr = r + row * ld;
    float* bd = band + row * n;
    const int64_t base = (int64_t)blockIdx.x * kTile;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    if (threadIdx.x == 0) scount = 0;
    __syncthreads();
    uint32_t cnt = 0u, lmax = 0u;
    bool bad = false;
    for (int q = 0; q < kTile / kFoldThreads; ++q) {
        const int64_t i = base + q * kFoldThreads + threadIdx.x;
        const bool ok = i < n;
        const float x = ok ? canon(__ldcs(rr + i)) : 0.f;
        bad |= ok && !finite_f(x);
        const bool above = ok && x >= aR, below = ok && x < aL;
        const bool inb = ok && !above && !below && finite_f(x);
        cnt += above ? 1u : 0u;
        if (below) lmax = max(lmax, to_key(x));
        const unsigned ball = __ballot_sync(0xffffffffu, inb);
        if (ball != 0u) {
            int at = 0;
            if (lane == __ffs(ball) - 1) at = atomicAdd(&scount, __popc(ball));
            at = __shfl_sync(0xffffffffu, at, __ffs(ball) - 1);
            if (inb) stage[at + __popc(ball & ((1u << lane) - 1u))] = x;
        }
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) {
        cnt += __shfl_xor_sync(0xffffffffu, cnt, d);
        lmax = max(lmax, __shfl_xor_sync(0xffffffffu, lmax, d));
    }
    if (lane == 0) {
        wcnt[w] = cnt;
        wmax[w] = lmax;
    }
    const int any_bad = __syncthreads_or(bad);
    if (threadIdx.x == 0) {
        uint32_t c = 0u, mx = 0u;
        for (int u = 0; u < kFoldThreads / 32; ++u) {
            c += wcnt[u];
            mx = max(mx, wmax[u]);
        }
        if (c != 0u) atomicAdd(&st->cnt_R, (unsigned long long)c);
        if (mx != 0u) atomicMax(&st->bin_kmin, mx);  // the largest key below a_L
        if (any_bad) {
            atomicOr(&st->status, kDevNonFinite);
            set_status(hdr, kDevNonFinite);
        }
        sbase = scount > 0 ? atomicAdd(&st->n_band, (unsigned long long)scount) : 0ull;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < scount; j += kFoldThreads) bd[sbase + j] = stage[j];
}

struct RowKeyGet {
    const float* r;
    __device__ __forceinline__ uint32_t operator()(int64_t i) const { return hkey(r[i]); }
};

// Key of the rho-th largest (1-based) of n keys read through `get`, by three
// radix levels (11, 11, 10 bits) over the whole input; every thread gets it.
template <class Get>
__device__ uint32_t select_desc(Get get, int64_t n, int64_t rho, uint32_t* hist, uint32_t* wsum,
                                uint32_t* bcast) {
    uint32_t prefix = 0u, mask = 0u;
    int64_t remaining = rho;
    const int shifts[3] = {21, 10, 0};
    const int widths[3] = {11, 11, 10};
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int lev = 0; lev < 3; ++lev) {
        const int sh = shifts[lev];
        const uint32_t nbin = 1u << widths[lev];
        for (uint32_t i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0u;
        __syncthreads();
        for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
            const uint32_t kk = get(i);
            if ((kk & mask) == prefix) atomicAdd(&hist[(kk >> sh) & (nbin - 1u)], 1u);
        }
        __syncthreads();
        // exclusive suffix counts over bins (two bins per thread, 1024 threads)
        const int i0 = 2 * threadIdx.x;
        const uint32_t c0 = hist[i0], c1 = hist[i0 + 1];
        uint32_t incl = c0 + c1;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t o = __shfl_down_sync(0xffffffffu, incl, d);
            if (lane + d < 32) incl += o;
        }
        if (lane == 0) wsum[w] = incl;
        __syncthreads();
        int64_t above = (int64_t)incl - (int64_t)(c0 + c1);
        for (int u = w + 1; u < (int)(blockDim.x >> 5); ++u) above += wsum[u];
        const int64_t s1 = above, s0 = above + c1;
        if (s1 < remaining && remaining <= s1 + c1) {
            bcast[0] = i0 + 1;
            bcast[1] = (uint32_t)s1;
        }
        if (s0 < remaining && remaining <= s0 + c0) {
            bcast[0] = i0;
            bcast[1] = (uint32_t)s0;
        }
        __syncthreads();
        remaining -= bcast[1];
        prefix |= bcast[0] << sh;
        mask |= (nbin - 1u) << sh;
        __syncthreads();
    }
    return prefix;
}

struct HardSmem {
    uint32_t xch[4 * kBlk];
    uint32_t sorted[kBandSortMax];
    uint32_t hist[2048];
    uint32_t wsum[32];
    uint32_t bcast[4];
    unsigned long long cnt[3];
};

__global__ void __launch_bounds__(kBlk) hard_solve_kernel(const float* __restrict__ r, int64_t ld,
                                                          int64_t n, double k, int64_t rank,
                                                          const float* __restrict__ band,
                                                          double* __restrict__ b_out,
                                                          RowState* rows, WsHeader* hdr,
                                                          int64_t B_total) {
    extern __shared__ __align__(16) unsigned char dsm[];
    HardSmem* sm = reinterpret_cast<HardSmem*>(dsm);
    const int64_t row = blockIdx.x;
    RowState* st = rows + row;
    const float* rr = r + row * ld;
    const float* bd = band + row * n;
    const int64_t cntR = (int64_t)st->cnt_R, nb = (int64_t)st->n_band;
    const uint32_t below_key = st->bin_kmin;  // 0: no score below a_L
    const bool nonfinite = (st->status & kDevNonFinite) != 0u;
    uint32_t ck;            // key of the boundary score c
    int64_t a, mm;          // scores above c, scores equal to c
    uint32_t lower_key;     // key of the largest score below c (0: none)
    int attempts = 1;
    const bool certified = !nonfinite && cntR < rank && rank <= cntR + nb;
    if (certified && nb <= kBandSortMax) {
        // the band, sorted ascending in shared memory (padding keys last)
        auto sort_into = [&](auto e_tag) {
            constexpr int E = decltype(e_tag)::value;
            uint32_t kk[E];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int64_t j = (int64_t)e * kBlk + threadIdx.x;
                kk[e] = j < nb ? to_key(bd[j]) : 0xffffffffu;
            }
            bitonic_sort_row<E, kBlk, kBlk>(kk, threadIdx.x, sm->xch);
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int64_t j = (int64_t)threadIdx.x * E + e;
                if (j < nb) sm->sorted[j] = kk[e];
            }
        };
        if (nb <= kBlk) sort_into(std::integral_constant<int, 1>{});
        else if (nb <= 2 * kBlk) sort_into(std::integral_constant<int, 2>{});
        else sort_into(std::integral_constant<int, 4>{});
        __syncthreads();
        ck = sm->sorted[nb - (rank - cntR)];
        // the group of keys equal to ck: [lo, hi) in the sorted band
        if (threadIdx.x == 0) {
            sm->cnt[0] = 0ull;
            sm->cnt[1] = 0ull;
            sm->bcast[2] = 0u;
        }
        __syncthreads();
        uint32_t lo_max = 0u;
        unsigned long long gt = 0ull, eq = 0ull;
        for (int64_t j = threadIdx.x; j < nb; j += kBlk) {
            const uint32_t kk = sm->sorted[j];
            gt += kk > ck ? 1ull : 0ull;
            eq += kk == ck ? 1ull : 0ull;
            if (kk < ck) lo_max = max(lo_max, kk);
        }
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) {
            gt += __shfl_xor_sync(0xffffffffu, gt, d);
            eq += __shfl_xor_sync(0xffffffffu, eq, d);
            lo_max = max(lo_max, __shfl_xor_sync(0xffffffffu, lo_max, d));
        }
        if ((threadIdx.x & 31) == 0) {
            atomicAdd(&sm->cnt[0], gt);
            atomicAdd(&sm->cnt[1], eq);
            atomicMax(&sm->bcast[2], lo_max);
        }
        __syncthreads();
        a = cntR + (int64_t)sm->cnt[0];
        mm = (int64_t)sm->cnt[1];
        lower_key = sm->bcast[2] != 0u ? sm->bcast[2] : below_key;
    } else {
        // a band too large for the on-chip sort: an exact selection within the
        // band; a bracket that missed the rank: an exact selection over the
        // whole row (rare)
        const float* src = certified ? bd : rr;
        const int64_t cnt = certified ? nb : n;
        const int64_t rho = certified ? rank - cntR : rank;
        attempts = certified ? 1 : 2;
        ck = select_desc(RowKeyGet{src}, cnt, rho, sm->hist, sm->wsum, sm->bcast);
        if (threadIdx.x == 0) {
            sm->cnt[0] = 0ull;
            sm->cnt[1] = 0ull;
            sm->bcast[2] = 0u;
        }
        __syncthreads();
        uint32_t lo_max = 0u;
        unsigned long long gt = 0ull, eq = 0ull;
        for (int64_t j = threadIdx.x; j < cnt; j += kBlk) {
            const uint32_t kk = hkey(src[j]);
            gt += kk > ck ? 1ull : 0ull;
            eq += kk == ck ? 1ull : 0ull;
            if (kk < ck) lo_max = max(lo_max, kk);
        }
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) {
            gt += __shfl_xor_sync(0xffffffffu, gt, d);
            eq += __shfl_xor_sync(0xffffffffu, eq, d);
            lo_max = max(lo_max, __shfl_xor_sync(0xffffffffu, lo_max, d));
        }
        if ((threadIdx.x & 31) == 0) {
            atomicAdd(&sm->cnt[0], gt);
            atomicAdd(&sm->cnt[1], eq);
            atomicMax(&sm->bcast[2], lo_max);
        }
        __syncthreads();
        a = (int64_t)sm->cnt[0] + (certified ? cntR : 0);
        mm = (int64_t)sm->cnt[1];
        lower_key = sm->bcast[2] != 0u ? sm->bcast[2] : (certified ? below_key : 0u);
    }
    if (threadIdx.x == 0) {
        const float c = from_key(ck);
        double b, frac;
        if (k < (double)(a + mm)) {
            b = (double)c;
            frac = (k - (double)a) / (double)mm;
        } else {  // k = a + m < n: some score lies below c
            b = 0.5 * ((double)c + (double)from_key(lower_key));
            frac = 1.0;
        }
        if (nonfinite) b = nan("");
        st->b = b;
        st->hard_c = c;
        st->hard_frac = frac;
        st->attempts = attempts;
        st->certified = attempts == 1 ? 1 : 0;
        b_out[row] = b;
        if (row == 0) {  // the call shape, for lapsum_row_info_get
            hdr->last_B = B_total;
            hdr->last_n = n;
            hdr->last_path = LAPSUM_PATH_BRACKET;
        }
    }
}

}  // namespace

cudaError_t launch_hard_bracket(const float* r, int64_t ld, float* p, double* b, int64_t B,
                                int64_t n, double k, uint64_t seed, int m, int64_t rank_l,
                                int64_t rank_h, int top_h, int force_miss, RowState* rows,
                                float* band, uint32_t* cand, uint32_t* tickets, WsHeader* hdr,
                                int64_t B_total, int vec, cudaStream_t st) {
    const int64_t rank = (int64_t)std::ceil(k);
    {
        ProfScope ps_("hard_sample", st);
        hard_sample_kernel<<<dim3((unsigned)(m / kBlk), (unsigned)B), kBlk, 0, st>>>(
            r, ld, n, seed, m, top_h, rank_l, rank_h, force_miss, cand, tickets, rows);
    }
    {
        ProfScope ps_("hard_fold", st);
        hard_fold_kernel<<<dim3((unsigned)((n + kTile - 1) / kTile), (unsigned)B), kFoldThreads, 0,
                           st>>>(r, ld, n, band, rows, hdr);
    }
    {
        static std::atomic<unsigned long long> attr_devices{0ull};
        once_per_device(attr_devices, [&]() {
            cudaFuncSetAttribute(hard_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sizeof(HardSmem));
        });
        ProfScope ps_("hard_solve", st);
        hard_solve_kernel<<<(unsigned)B, kBlk, sizeof(HardSmem), st>>>(r, ld, n, k, rank, band, b,
                                                                       rows, hdr, B_total);
    }
    return launch_hard_emit(r, ld, p, B, n, rows, vec, st);
}

}  // namespace lapsum
