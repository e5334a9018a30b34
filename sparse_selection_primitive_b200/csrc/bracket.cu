// Probabilistic bracketing for very long rows.
//
// "Fast LapSum: Exact Differentiable Top-k at Million Scale" (gist.science
// explainer pages), section 2.2, probabilistic bracketing:
//   1. localization: draw a small sample of Laplace-noised scores and take two
//      binomial order statistics as a bracket [a_L, a_R) holding b with high
//      probability;
//   2. streaming and filtering: one pass over the row folds the scores outside
//      the bracket into stable tail sums and keeps the in-bracket middle band;
//   3. exact solution: the exact solver runs on the band only;
//   4. verification: a certification step checks the bracket and widens it
//      when it fails, so the budget always holds exactly.
//
// Kernels (per row, stream-ordered, no host round trip):
//   sample_kernel   1 CTA: counter-based sample y_s = r[I_s] + eps_s, radix
//                   select of the descending ranks l and h -> (a_L, a_R);
//   fold_kernel     grid: one pass over r (float4 loads); tail counts/sums per
//                   thread in fp64, band compaction by warp ballot; per-CTA
//                   partials combined in CTA order by the last CTA;
//   solve_kernel    1 CTA: certify F(a_L) >= k >= F(a_R) from the tails and the
//                   band; narrow a large band with exact histogram levels; sort
//                   the final band (<= 4096) with the register bitonic network;
//                   solve with the tails as virtual end anchors.  A failed
//                   bracket moves the failing end to the next rung of its
//                   ladder (4x the rank, then open) and the same CTA re-folds r.
#include <atomic>
#include <type_traits>

#include "bitonic.cuh"
#include "lapsum_common.cuh"
#include "lapsum_kernels.h"
#include "solve_sorted.cuh"

namespace lapsum {
namespace {

constexpr int kBlk = 1024;
constexpr int kWarpSortMax = 256;  // bands up to this size are sorted and solved by one warp
constexpr int kFoldThreads = 256;
constexpr int kFoldGridMaxShard = 4096;  // fold records of the split-row pieces

struct Ladder {
    int64_t l[kLadder];  // descending ranks for a_R (0 = open)
    int64_t h[kLadder];  // descending ranks for a_L (> m = open)
};

// ----------------------------------------------------------------------------
// Block radix select: key of the rho-th largest (1-based) of m keys read via
// `get`.  Levels of 11, 11 and 10 bits; the histogram lives in `hist` (2048
// words of shared memory).  Every thread gets the result.
// ----------------------------------------------------------------------------
template <class Get>
__device__ uint32_t block_select_desc(Get get, int m, int64_t rho, uint32_t* hist,
                                      uint32_t* wsum, uint32_t* bcast) {
    uint32_t prefix = 0, mask = 0;
    int64_t remaining = rho;
    const int shifts[3] = {21, 10, 0};
    const int widths[3] = {11, 11, 10};
    for (int lev = 0; lev < 3; ++lev) {
        const int sh = shifts[lev];
        const uint32_t nb = 1u << widths[lev];
        for (uint32_t i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        for (int i0 = 0; i0 < m; i0 += blockDim.x) {
            const int i = i0 + threadIdx.x;
            const uint32_t key = i < m ? get(i) : 0u;
            const bool in = i < m && (key & mask) == prefix;
            const uint32_t bn = in ? ((key >> sh) & (nb - 1)) : 0xffffffffu;
            const unsigned peers = __match_any_sync(0xffffffffu, bn);
            if (in && (threadIdx.x & 31) == __ffs(peers) - 1)
                atomicAdd(&hist[bn], (uint32_t)__popc(peers));
        }
        __syncthreads();
        // Suffix counts over bins: thread i owns bins 2i, 2i+1 (1024 threads).
        const int i0 = 2 * threadIdx.x;
        const uint32_t c0 = hist[i0], c1 = hist[i0 + 1];
        uint32_t mine = c0 + c1;
        // exclusive suffix over threads (higher threads first)
        uint32_t incl = mine;
        const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t o = __shfl_down_sync(0xffffffffu, incl, d);
            if (lane + d < 32) incl += o;
        }
        if (lane == 0) wsum[w] = incl;
        __syncthreads();
        uint32_t above = incl - mine;
        for (int u = w + 1; u < (int)(blockDim.x >> 5); ++u) above += wsum[u];
        // bins in descending order: bin i0+1 then i0
        const int64_t s1 = above, s0 = above + c1;  // counts strictly above bin i0+1 / i0
        if (s1 < remaining && remaining <= s1 + c1) {
            bcast[0] = i0 + 1;
            bcast[1] = (uint32_t)s1;
        }
        if (s0 < remaining && remaining <= s0 + c0) {
            bcast[0] = i0;
            bcast[1] = (uint32_t)s0;
        }
        __syncthreads();
        const uint32_t bin = bcast[0];
        remaining -= bcast[1];
        prefix |= bin << sh;
        mask |= (nb - 1) << sh;
        __syncthreads();
    }
    return prefix;
}

struct GlobalSampleKeyGet {
    const float* y;
    __device__ __forceinline__ uint32_t operator()(int i) const { return to_key(y[i]); }
};

// For two ranks at once (1-based, descending; 0 = not wanted): the bin of
// hist_a holding the ra-th largest and the bin of hist_b holding the rb-th
// largest (hist_b may be hist_a), with the counts in higher bins.  Bins
// 0..2047 in descending order; 1024 threads, two bins each; every thread gets
// the results.  bcast: 4 words.
__device__ void rank_bins2(const uint32_t* hist_a, const uint32_t* hist_b, int64_t ra, int64_t rb,
                           uint32_t* wsum /*64*/, uint32_t* bcast, uint32_t* bin_a,
                           uint32_t* above_a, uint32_t* bin_b, uint32_t* above_b) {
    const int i0 = 2 * threadIdx.x;
    const uint32_t a0 = hist_a[i0], a1 = hist_a[i0 + 1];
    const uint32_t b0 = hist_b[i0], b1 = hist_b[i0 + 1];
    uint32_t ia = a0 + a1, ib = b0 + b1;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t oa = __shfl_down_sync(0xffffffffu, ia, d);
        const uint32_t ob = __shfl_down_sync(0xffffffffu, ib, d);
        if (lane + d < 32) {
            ia += oa;
            ib += ob;
        }
    }
    if (lane == 0) {
        wsum[w] = ia;
        wsum[32 + w] = ib;
    }
    __syncthreads();
    uint32_t xa = ia - (a0 + a1), xb = ib - (b0 + b1);  // counts above this thread's bins
    for (int u = w + 1; u < (int)(blockDim.x >> 5); ++u) {
        xa += wsum[u];
        xb += wsum[32 + u];
    }
    auto find = [&](int64_t rho, uint32_t above, uint32_t c0, uint32_t c1, int slot) {
        const int64_t s1 = above, s0 = (int64_t)above + c1;  // above bin i0+1 / bin i0
        if (s1 < rho && rho <= s1 + c1) {
            bcast[slot] = i0 + 1;
            bcast[slot + 1] = (uint32_t)s1;
        }
        if (s0 < rho && rho <= s0 + c0) {
            bcast[slot] = i0;
            bcast[slot + 1] = (uint32_t)s0;
        }
    };
    if (ra >= 1) find(ra, xa, a0, a1, 0);
    if (rb >= 1) find(rb, xb, b0, b1, 2);
    __syncthreads();
    *bin_a = bcast[0];
    *above_a = bcast[1];
    *bin_b = bcast[2];
    *above_b = bcast[3];
    __syncthreads();
}

// Keys of the ra-th and rb-th largest (1-based; 0 = not wanted) of m sample
// keys staged in shared memory, by a radix select whose first level (the
// keys' top 11 bits) is the histogram hist1 the sample kernel already built;
// levels two and three (11 and 10 bits) count, for each rank, only the keys
// sharing its prefix (a few percent of the sample, so most warps skip the
// counting).  h2: 2 x 2048 words.  Needs blockDim.x == 1024.
__device__ void select_two_ranks(const uint32_t* keys, int m, const uint32_t* hist1, int64_t ra,
                                 int64_t rb, uint32_t* h2, uint32_t* wsum, uint32_t* bcast,
                                 uint32_t* key_a, uint32_t* key_b) {
    const int lane = threadIdx.x & 31;
    const bool wa = ra >= 1, wb = rb >= 1;
    if (!wa && !wb) {  // both ends open
        *key_a = 0u;
        *key_b = 0u;
        return;
    }
    uint32_t pa, pb, xa, xb;
    rank_bins2(hist1, hist1, ra, rb, wsum, bcast, &pa, &xa, &pb, &xb);
    // Keys in the lowest wanted bin or above: when there are few (the usual
    // case for a small budget) one warp sorts them all and reads both ranks off.
    const uint32_t low = wb ? pb : pa;
    const uint32_t ncand = wb ? xb + hist1[pb] : xa + hist1[pa];
    // A long sample whose candidates fit one block-wide sort (two keys per
    // thread): the sort takes less time than two radix levels, each a pass
    // over all m keys.
    const bool warp_sort = ncand <= (uint32_t)kWarpSortMax;
    const bool block_sort = !warp_sort && ncand <= 2u * kBlk && m >= 8 * kBlk;
    if (warp_sort || block_sort) {
        const uint32_t cap = warp_sort ? (uint32_t)kWarpSortMax : 2u * kBlk;
        uint32_t* cand = h2;  // cap words; the block sort exchanges through h2 + 2 kBlk
        if (threadIdx.x == 0) bcast[0] = 0u;
        __syncthreads();
        for (int s0 = 0; s0 < m; s0 += blockDim.x) {  // same trip count in every lane
            const int s = s0 + threadIdx.x;
            const uint32_t k = s < m ? keys[s] : 0u;
            const bool take = s < m && (k >> 21) >= low;
            const unsigned ball = __ballot_sync(0xffffffffu, take);
            if (ball == 0u) continue;
            const int leader = __ffs(ball) - 1;
            uint32_t base = 0;
            if (lane == leader) base = atomicAdd(&bcast[0], (uint32_t)__popc(ball));
            base = __shfl_sync(0xffffffffu, base, leader);
            const uint32_t pos = base + __popc(ball & ((1u << lane) - 1u));
            if (take && pos < cap) cand[pos] = k;
        }
        __syncthreads();
        if (block_sort) {
            uint32_t key[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const uint32_t j = threadIdx.x * 2 + e;
                key[e] = j < ncand ? cand[j] : 0u;  // padding sorts first
            }
            bitonic_sort_row<2, kBlk, kBlk>(key, threadIdx.x, h2 + 2 * kBlk);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int j = threadIdx.x * 2 + e;
                if (wa && j == 2 * kBlk - ra) bcast[2] = key[e];
                if (wb && j == 2 * kBlk - rb) bcast[3] = key[e];
            }
        } else if (threadIdx.x < 32) {
            constexpr int E = kWarpSortMax / 32;
            uint32_t key[E];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const uint32_t j = threadIdx.x * E + e;
                key[e] = j < ncand ? cand[j] : 0u;  // padding sorts first
            }
            bitonic_sort_row<E, 32, 32>(key, threadIdx.x, nullptr);
            // ascending: the r-th largest sits at position kWarpSortMax - r
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int j = threadIdx.x * E + e;
                if (wa && j == kWarpSortMax - ra) bcast[2] = key[e];
                if (wb && j == kWarpSortMax - rb) bcast[3] = key[e];
            }
        }
        __syncthreads();
        *key_a = bcast[2];
        *key_b = bcast[3];
        __syncthreads();
        return;
    }
    int64_t rema = ra - xa, remb = rb - xb;
#pragma unroll 1
    for (int lev = 0; lev < 2; ++lev) {
        const int sh = lev == 0 ? 10 : 0;          // position of this level's digit
        const int psh = lev == 0 ? 21 : 10;        // the prefix is key >> psh
        const uint32_t dmask = lev == 0 ? 2047u : 1023u;
        for (int i = threadIdx.x; i < 2 * 2048; i += blockDim.x) h2[i] = 0u;
        __syncthreads();
        for (int s0 = 0; s0 < m; s0 += blockDim.x) {  // same trip count in every lane
            const int s = s0 + threadIdx.x;
            const uint32_t k = s < m ? keys[s] : 0u;
            const bool ina = s < m && wa && (k >> psh) == pa;
            const bool inb = s < m && wb && (k >> psh) == pb;
            // (the digits below the prefix spread over the bins, so plain
            // shared-memory atomics rarely collide)
            if (ina) atomicAdd(&h2[(k >> sh) & dmask], 1u);
            if (inb) atomicAdd(&h2[2048 + ((k >> sh) & dmask)], 1u);
        }
        __syncthreads();
        uint32_t ba, bb;
        rank_bins2(h2, h2 + 2048, wa ? rema : 0, wb ? remb : 0, wsum, bcast, &ba, &xa, &bb, &xb);
        const int width = lev == 0 ? 11 : 10;
        pa = (pa << width) | ba;
        pb = (pb << width) | bb;
        rema -= xa;
        remb -= xb;
    }
    *key_a = pa;
    *key_b = pb;
}

// ----------------------------------------------------------------------------
// 1. Localization sample.
// ----------------------------------------------------------------------------
// Sample s of a row: r[I] plus Laplace(0, t) noise (sample_index, sample_noise).
__device__ __forceinline__ float draw_sample(const float* __restrict__ r, int64_t n, double t,
                                             uint64_t seed, uint64_t c0, int s) {
    const int64_t I = sample_index(seed, c0, s, n);
    const float rv = __ldg(r + I);
    return rv + sample_noise(seed, c0, s, t);
}
// Grid of m / 1024 CTAs: every thread draws one sample.  The order statistics
// of the bracket are found in one of two ways:
//  - top_h > 0 (both ranks at most top_h, and (m / 1024) * top_h <= 4096): each
//    CTA sorts its 1024 keys and keeps its top_h largest, which must hold every
//    sample of global rank <= top_h; the last CTA to finish (atomic ticket)
//    sorts those candidates and reads the two ranks off;
//  - otherwise every CTA adds its samples to a global histogram of the keys'
//    top 11 bits, and the last CTA stages the whole sample in shared memory and
//    selects the two order statistics by radix levels, then clears the
//    histogram for the next call.
__global__ void __launch_bounds__(kBlk) sample_kernel(const float* __restrict__ r, int64_t n,
                                                      double t, uint64_t seed, uint64_t c0, int m,
                                                      Ladder lad, int force_miss, int max_attempts,
                                                      float* __restrict__ sample_out,
                                                      unsigned long long* __restrict__ bins,
                                                      uint32_t* __restrict__ ghist,
                                                      uint32_t* __restrict__ ticket,
                                                      RowState* st, int top_h,
                                                      uint32_t* __restrict__ cand, int clear_bins,
                                                      uint32_t* __restrict__ sup_flag,
                                                      const RowBudget* __restrict__ bud,
                                                      WsHeader* hdr) {
    pdl_wait();
    if (bud != nullptr) {
        // the row's own budget: sample size, ranks and the candidate mode
        // (every CTA of the grid of kSampleMax / kBlk takes part in the ticket)
        m = bud->m;
        for (int i = 0; i < kLadder; ++i) {
            lad.l[i] = bud->l[i];
            lad.h[i] = bud->h[i];
        }
        const int64_t need = lad.h[0] <= m ? lad.h[0] : (lad.l[0] >= 1 ? lad.l[0] : 0);
        top_h = (need >= 1 && need <= kBlk && (int64_t)gridDim.x * need <= 4 * kBlk) ? (int)need
                                                                                      : 0;
    }
    const bool bad_budget = bud != nullptr && !bud->ok;
    if (blockIdx.x == 0) {
        // this kernel starts the row's forward: clear its record, histogram
        // and gradient-support flags
        for (int i = threadIdx.x; i < (int)(sizeof(RowState) / 4); i += kBlk)
            reinterpret_cast<uint32_t*>(st)[i] = 0u;
        if (sup_flag != nullptr && threadIdx.x == 0) *sup_flag = 0u;
        if (clear_bins)
            for (int i = threadIdx.x; i < 3 * kBins; i += kBlk) bins[i] = 0ull;
        __syncthreads();
        phase_mark(st, 14);
    }
    extern __shared__ uint32_t dyn[];
    __shared__ uint32_t hist[2048];
    __shared__ uint32_t wsum[64];
    __shared__ uint32_t bcast[4];
    __shared__ int flag;
    const int s = blockIdx.x * kBlk + threadIdx.x;
    uint32_t key = 0u;  // samples past m sort first
    if (s < m && !bad_budget) {
        const float y = draw_sample(r, n, t, seed, c0, s);
        sample_out[s] = y;
        key = to_key(y);
    }
    if (top_h > 0) {
        uint32_t kk[1] = {key};
        bitonic_sort_row<1, kBlk, kBlk>(kk, threadIdx.x, hist);
        if (threadIdx.x >= kBlk - top_h)
            cand[blockIdx.x * top_h + (threadIdx.x - (kBlk - top_h))] = kk[0];
    } else {
        for (int i = threadIdx.x; i < 2048; i += kBlk) hist[i] = 0u;
        __syncthreads();
        const uint32_t bn = (s < m && !bad_budget) ? key >> 21 : 0xffffffffu;
        // lanes with the same bin add once (samples crowd into few top bins)
        const unsigned peers = __match_any_sync(0xffffffffu, bn);
        if (bn != 0xffffffffu && (threadIdx.x & 31) == __ffs(peers) - 1)
            atomicAdd(&hist[bn], (uint32_t)__popc(peers));
        __syncthreads();
        for (int i = threadIdx.x; i < 2048; i += kBlk)
            if (hist[i] != 0u) atomicAdd(&ghist[i], hist[i]);
    }
    if (blockIdx.x == 0) phase_mark(st, 15);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t prev = atomicAdd(ticket, 1u);
        flag = (prev == gridDim.x - 1);
        if (flag) *ticket = 0u;
    }
    __syncthreads();
    if (!flag) return;
    __threadfence();
    phase_mark(st, 0);
    if (bad_budget) {
        // a budget outside (0, n): b = NaN and a status bit; the later kernels
        // of the row see the bit and return
        for (int i = threadIdx.x; i < 2048; i += kBlk) ghist[i] = 0u;
        if (threadIdx.x == 0) {
            st->status |= kDevBadBudget;
            set_status(hdr, kDevBadBudget);
            st->path = LAPSUM_PATH_BRACKET;
            st->b = nan("");
        }
        return;
    }
    const int64_t ra = lad.l[0] >= 1 ? lad.l[0] : 0;
    const int64_t rb = lad.h[0] <= m ? lad.h[0] : 0;
    uint32_t ka = 0u, kb = 0u, kmax = 0u;
    if (top_h > 0) {
        // the candidates, sorted ascending: the r-th largest sits at npad - r
        const int c = (int)gridDim.x * top_h;
        auto pick = [&](auto e_tag) {
            constexpr int E = decltype(e_tag)::value;
            uint32_t kk[E];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int j = threadIdx.x * E + e;
                kk[e] = j < c ? __ldcg(cand + j) : 0u;
            }
            bitonic_sort_row<E, kBlk, kBlk>(kk, threadIdx.x, dyn);
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int j = threadIdx.x * E + e;
                if (ra >= 1 && j == E * kBlk - ra) bcast[0] = kk[e];
                if (rb >= 1 && j == E * kBlk - rb) bcast[1] = kk[e];
                if (j == E * kBlk - 1) bcast[2] = kk[e];
            }
        };
        if (c <= kBlk) pick(std::integral_constant<int, 1>{});
        else if (c <= 2 * kBlk) pick(std::integral_constant<int, 2>{});
        else pick(std::integral_constant<int, 4>{});
        __syncthreads();
        ka = bcast[0];
        kb = bcast[1];
        kmax = bcast[2];
    } else {
        uint32_t* skeys = dyn;               // the sample's keys, kSampleMax words
        uint32_t* h2 = skeys + kSampleMax;   // select histograms, 2 x 2048 words
        for (int i = threadIdx.x; i < 2048; i += kBlk) {
            hist[i] = __ldcg(ghist + i);
            ghist[i] = 0u;  // ready for the next call
        }
        // the sample's keys into shared memory, eight loads in flight per thread
        for (int s0 = 0; s0 < m; s0 += 8 * kBlk) {
            float yv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int sq = s0 + q * kBlk + threadIdx.x;
                yv[q] = sq < m ? __ldcg(sample_out + sq) : 0.f;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int sq = s0 + q * kBlk + threadIdx.x;
                if (sq < m) skeys[sq] = to_key(yv[q]);
            }
        }
        __syncthreads();
        select_two_ranks(skeys, m, hist, ra, rb, h2, wsum, bcast, &ka, &kb);
        if (force_miss) {
            for (int sq = threadIdx.x; sq < m; sq += kBlk) kmax = max(kmax, skeys[sq]);
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, d));
            if (threadIdx.x == 0) bcast[3] = 0u;
            __syncthreads();
            if ((threadIdx.x & 31) == 0) atomicMax(&bcast[3], kmax);
            __syncthreads();
            kmax = bcast[3];
        }
    }
    const float aR = ra >= 1 ? from_key(ka) : INFINITY;
    const float aL = rb >= 1 ? from_key(kb) : -INFINITY;
    phase_mark(st, 1);
    if (threadIdx.x == 0) {
        st->ladder_R[0] = aR;
        st->ladder_L[0] = aL;
        st->rung_L = 0;
        st->rung_R = 0;
        if (force_miss) {
            // A bracket above every sample value: F(a_L) < k, so it must fail.
            const float top = from_key(kmax);
            st->a_L = top + fabsf(top) + 1.f;
            st->a_R = INFINITY;
            st->rung_L = -1;
        } else {
            st->a_L = aL;
            st->a_R = aR;
        }
        bracket_key_range(st->a_L, st->a_R, &st->bin_kmin, &st->bin_kmax);
        st->sample_m = m;
        st->rank_l = (int32_t)lad.l[0];
        st->rank_h = (int32_t)lad.h[0];
        st->n_band = 0;
        st->attempts = 1;
        st->max_attempts = max_attempts;
        st->force_miss = force_miss;
        st->path = LAPSUM_PATH_BRACKET;
        st->refine_levels = 0;
    }
}

// ----------------------------------------------------------------------------
// 2. Streaming fold.
// ----------------------------------------------------------------------------
struct FoldAcc {
    uint32_t cntR;  // per thread: at most n / (grid threads)
    double SL, SR;
    bool bad;
};

// One score: right tail (count and e^{-(x - aR)/t}), left tail (e^{(x - aL)/t})
// or band.  The tail terms go to fp32 partials that the caller flushes into
// the fp64 accumulators every few scores.
__device__ __forceinline__ void fold_one(float x, float aL, float aR, float inv_t, FoldAcc& acc,
                                         float& sl, float& sr, bool& in_band) {
    acc.bad |= !finite_f(x);
    const bool right = x >= aR, left = x < aL;
    // one exponential serves whichever tail the score is in (band scores are
    // masked out; their argument is a finite dummy)
    const float e = __expf((right ? (aR - x) : (left ? (x - aL) : 0.f)) * inv_t);
    acc.cntR += right ? 1u : 0u;
    sr += right ? e : 0.f;
    sl += left ? e : 0.f;
    in_band = !(right | left);
}
__device__ __forceinline__ void fold_one(float x, float aL, float aR, float inv_t, FoldAcc& acc,
                                         bool& in_band) {
    float sl = 0.f, sr = 0.f;
    fold_one(x, aL, aR, inv_t, acc, sl, sr, in_band);
    acc.SL += (double)sl;
    acc.SR += (double)sr;
}

// The same on a soft row (40 t >= |b|, where every score can carry weight):
// the tail term in fp64, from an fp64 margin, so that the tail sums of 10^6
// soft scores keep the budget (fp32 margins and exponentials leave errors of
// a fraction of an ulp that do not average out).
__device__ __forceinline__ void fold_one_soft(float x, float aL, float aR, double inv_td,
                                              FoldAcc& acc, bool& in_band) {
    acc.bad |= !finite_f(x);
    const bool right = x >= aR, left = x < aL;
    const double a = right ? ((double)x - (double)aR) * inv_td
                           : (left ? ((double)aL - (double)x) * inv_td : 0.0);
    const double e = exp(-a);
    acc.cntR += right ? 1u : 0u;
    acc.SR += right ? e : 0.0;
    acc.SL += left ? e : 0.0;
    in_band = !(right | left);
}

// Adds one band score to the fixed-point band histogram (global atomics).
__device__ __forceinline__ void bin_add(float x, const BinLayout& BL, float inv_t,
                                        unsigned long long* bins) {
    const int j = bin_of(BL, to_key(x));
    const float lo = bin_edge(BL, j), hi = bin_edge(BL, j + 1);
    atomicAdd(&bins[j], 1ull);
    atomicAdd(&bins[kBins + j], __float2ull_rn(__expf((lo - x) * inv_t) * (float)kFixScale));
    atomicAdd(&bins[2 * kBins + j], __float2ull_rn(__expf((x - hi) * inv_t) * (float)kFixScale));
}

constexpr int kStage = 1024;  // band scores staged per CTA before one global append

// Warp-aggregated append of the lanes with `take` to the CTA's staging buffer;
// lanes past its capacity go straight to the global band (rare).
__device__ __forceinline__ void band_stage(bool take, float x, float* sband, int* scount,
                                           float* band, unsigned long long* counter,
                                           unsigned long long cap, const BinLayout& BL,
                                           float inv_t, unsigned long long* bins) {
    const unsigned ball = __ballot_sync(0xffffffffu, take);
    if (ball == 0) return;
    const int lane = threadIdx.x & 31;
    const int leader = __ffs(ball) - 1;
    int base = 0;
    if (lane == leader) base = atomicAdd(scount, __popc(ball));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (take) {
        const int pos = base + __popc(ball & ((1u << lane) - 1u));
        if (pos < kStage) {
            sband[pos] = x;
        } else {
            const unsigned long long g = atomicAdd(counter, 1ull);
            if (g < cap) band[g] = x;
            if (bins != nullptr) bin_add(x, BL, inv_t, bins);
        }
    }
}

// Moves the staged band scores to the global band and histogram.
__device__ __forceinline__ void band_flush(const float* sband, int scount, float* band,
                                           unsigned long long* counter, unsigned long long cap,
                                           const BinLayout& BL, float inv_t,
                                           unsigned long long* bins,
                                           unsigned long long* gbase_sh) {
    const int ns = scount < kStage ? scount : kStage;
    if (threadIdx.x == 0) *gbase_sh = ns > 0 ? atomicAdd(counter, (unsigned long long)ns) : 0ull;
    __syncthreads();
    const unsigned long long gb = *gbase_sh;
    for (int i = threadIdx.x; i < ns; i += blockDim.x) {
        const float x = sband[i];
        if (gb + i < cap) band[gb + i] = x;
        if (bins != nullptr) bin_add(x, BL, inv_t, bins);
    }
}

constexpr int kQ = 1024;  // per-warp circular queue of near scores (power of two)
constexpr size_t kFoldDynSmem = (size_t)(kFoldThreads / 32) * (kQ + 32 * 16) * sizeof(float);

// Swizzled slot of value j (0..15) in a lane's 16-float staging row, so that a
// warp's 16-byte stores of the four float4 groups hit distinct banks.
__device__ __forceinline__ int stage_slot(int lane, int j) {
    return lane * 16 + ((((j >> 2) ^ (lane >> 1)) & 3) << 2) + (j & 3);
}

__global__ void __launch_bounds__(kFoldThreads, 4) fold_kernel(const float* __restrict__ r, int64_t n,
                                                            double t, RowState* st,
                                                            float* __restrict__ band,
                                                            unsigned long long* __restrict__ bins,
                                                            double* __restrict__ part,
                                                            int vec, int hist) {
    pdl_wait();
    __shared__ double red4[kFoldThreads / 32][4];
    __shared__ float sband[kStage];
    // dynamic: per-warp queues (kQ floats each), then per-warp staging rows
    extern __shared__ __align__(16) float fold_dyn[];
    __shared__ int scount;
    __shared__ unsigned long long gbase;
    if (st->status & kDevBadBudget) return;
    const float aL = st->a_L, aR = st->a_R;
    // Scores more than 90 t below the bracket add exactly 0 to the left tail
    // sum in fp32, and scores more than 90 t above it add 1 to the right count
    // and 0 to its sum; only the scores between these limits ("near") need
    // the full fold.  Each trip classifies 16 scores per thread with two
    // compares each (a 16-bit near mask and the far-right count); a warp with
    // near scores stages the trip's values in shared memory, and each lane
    // copies its near ones into the warp's circular queue at its scan offset.
    // The queue is folded 32 scores at a time, so the lanes stay busy on the
    // near scores however sparse they are.  Non-finite scores are caught by a
    // running sum (checked exactly if it overflows).
    const float aLf = aL - (float)(90.0 * t), aRf = aR + (float)(90.0 * t);
    // the band histogram only when the solve will use it (a band expected too
    // large for the on-chip sort)
    const BinLayout BL = make_bins(st->bin_kmin, st->bin_kmax);
    if (!hist) bins = nullptr;
    const float inv_t = (float)(1.0 / t);
    const double inv_td = 1.0 / t;
    // soft row: 40 t >= |b|, b judged by the bracket's finite ends (uniform)
    const double bc = isfinite(aL) ? (isfinite(aR) ? 0.5 * ((double)aL + (double)aR) : (double)aL)
                                   : (isfinite(aR) ? (double)aR : 0.0);
    const bool soft = 40.0 * t >= fabs(bc);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float* q = fold_dyn + warp * kQ;
    float* stg = fold_dyn + (kFoldThreads / 32) * kQ + warp * (32 * 16);
    uint32_t head = 0, tail = 0;  // warp-uniform; tail - head = queued scores
    if (threadIdx.x == 0) scount = 0;
    if (blockIdx.x == 0) phase_mark(st, 16);
    __syncthreads();
    FoldAcc acc{0u, 0.0, 0.0, false};
    uint32_t far_right = 0u;
    float far_right_f = 0.f;  // full trips' count (exact: at most 2^24 per thread)
    float xsum = 0.f;
    bool bad = false;
    unsigned long long* counter = &st->n_band;
    const unsigned long long cap = (unsigned long long)n;
    const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
    const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    auto drain = [&](int cnt) {  // fold `cnt` (<= 32) queued scores, one per lane
        const bool ok = lane < cnt;
        const float x = ok ? q[(head + lane) & (kQ - 1)] : 0.f;
        bool inb = false;
        if (ok) {
            if (soft) fold_one_soft(x, aL, aR, inv_td, acc, inb);
            else fold_one(x, aL, aR, inv_t, acc, inb);
        }
        band_stage(inb, x, sband, &scount, band, counter, cap, BL, inv_t, bins);
        head += cnt;
    };
    // appends the near values of a staged trip (16 per lane, mask m) to the queue
    auto push_staged = [&](uint32_t m) {
        const int c = __popc(m);
        int incl = c;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += o;
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        __syncwarp();
        uint32_t off = tail + (uint32_t)(incl - c);
        while (m != 0u) {
            const int j = __ffs(m) - 1;
            m &= m - 1u;
            q[(off++) & (kQ - 1)] = stg[stage_slot(lane, j)];
        }
        tail += (uint32_t)total;
        __syncwarp();
        while (tail - head >= 32u) drain(32);
    };
    // the generic path for short or ragged parts: values in registers
    auto push = [&](const float* xs, uint32_t m, int cnt_max) {
        __syncwarp();
        const int c = __popc(m);
        int incl = c;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += o;
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        uint32_t off = tail + (uint32_t)(incl - c);
        for (int j = 0; j < cnt_max; ++j)
            if (m & (1u << j)) q[(off++) & (kQ - 1)] = xs[j];
        tail += (uint32_t)total;
        __syncwarp();
        while (tail - head >= 32u) drain(32);
    };
    auto classify = [&](float x, bool valid, uint32_t& m, int j) {
        const bool ge_l = valid && x >= aLf, ge_r = valid && x >= aRf;
        m |= (uint32_t)(ge_l && !ge_r) << j;
        far_right += ge_r ? 1u : 0u;
        if (valid) xsum += x;
    };
    if (vec) {
        const int64_t n4 = n >> 2;
        const float4* r4 = reinterpret_cast<const float4*>(r);
        // Main part: full trips only (every load in range for every thread);
        // the loads run one trip ahead of the processing.
        constexpr int U = 4;
        const int64_t step = (int64_t)U * nthreads;
        const int64_t full = n4 / step;
        const float4* p = r4 + gtid;
        // The last partial trip (at most U vectors per thread, a grid-uniform
        // count) is loaded with bounds checks into the prefetch registers
        // while the last full trip is processed, so that a short row has all
        // its loads in flight at once.
        const int64_t rem_iters = (n4 - full * step + nthreads - 1) / nthreads;
        float4 nv[U];
        auto load_rem = [&]() {
#pragma unroll
            for (int qq = 0; qq < U; ++qq) {
                const int64_t i = full * step + (int64_t)qq * nthreads + gtid;
                nv[qq] = (qq < rem_iters && i < n4) ? __ldcs(r4 + i)
                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        };
        if (full > 0) {
#pragma unroll
            for (int qq = 0; qq < U; ++qq) nv[qq] = __ldcs(p + (int64_t)qq * nthreads);
        } else {
            load_rem();
        }
        for (int64_t it = 0; it < full; ++it, p += step) {
            float4 cur[U];
#pragma unroll
            for (int qq = 0; qq < U; ++qq) cur[qq] = nv[qq];
            if (it + 1 < full) {
#pragma unroll
                for (int qq = 0; qq < U; ++qq) nv[qq] = __ldcs(p + step + (int64_t)qq * nthreads);
            } else {
                load_rem();
            }
            // full trips: the compares give 1.0 / 0.0, the near mask is built
            // exactly in fp32 (16 bits) and the far-right count in a float
            // (exact to 2^24 per thread), all on the floating-point pipes
            float mf = 0.f;
#pragma unroll
            for (int qq = 0; qq < U; ++qq) {
                const float xv[4] = {cur[qq].x, cur[qq].y, cur[qq].z, cur[qq].w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float gl = xv[c] >= aLf ? 1.f : 0.f;
                    const float gr = xv[c] >= aRf ? 1.f : 0.f;
                    mf = fmaf(gl - gr, (float)(1u << (4 * qq + c)), mf);
                    far_right_f += gr;
                    xsum += xv[c];
                }
            }
            const uint32_t m = (uint32_t)mf;
            if (__any_sync(0xffffffffu, m != 0u)) {
#pragma unroll
                for (int qq = 0; qq < U; ++qq)
                    *reinterpret_cast<float4*>(stg + stage_slot(lane, 4 * qq)) = cur[qq];
                push_staged(m);
            }
        }
        // Remainder: the last partial trip, loaded above.
        {
#pragma unroll
            for (int qq = 0; qq < U; ++qq) {
                if (qq >= rem_iters) break;
                const int64_t i = full * step + (int64_t)qq * nthreads + gtid;
                const bool ok = i < n4;
                const float xs[4] = {nv[qq].x, nv[qq].y, nv[qq].z, nv[qq].w};
                uint32_t m = 0u;
#pragma unroll
                for (int j = 0; j < 4; ++j) classify(xs[j], ok, m, j);
                if (__any_sync(0xffffffffu, m != 0u)) push(xs, m, 4);
            }
        }
        // tail elements (n not a multiple of 4)
        const int64_t rem0 = n4 << 2;
        if (blockIdx.x == 0 && threadIdx.x < 32) {
            const int64_t i = rem0 + threadIdx.x;
            const float xs[1] = {i < n ? r[i] : 0.f};
            uint32_t m = 0u;
            classify(xs[0], i < n, m, 0);
            if (__any_sync(0xffffffffu, m != 0u)) push(xs, m, 1);
        }
    } else {
        const int64_t iters = (n + nthreads - 1) / nthreads;
        for (int64_t it = 0; it < iters; ++it) {
            const int64_t i = it * nthreads + gtid;
            const float xs[1] = {i < n ? r[i] : 0.f};
            uint32_t m = 0u;
            classify(xs[0], i < n, m, 0);
            if (__any_sync(0xffffffffu, m != 0u)) push(xs, m, 1);
        }
    }
    if (!(fabsf(xsum) <= 3.402823466e38f)) {
        // a NaN or an infinity, or only an overflowing sum: check this
        // thread's scores one by one (rare)
        if (vec) {
            const int64_t n4 = n >> 2;
            for (int64_t i = gtid; i < n4; i += nthreads) {
                const float4 v = reinterpret_cast<const float4*>(r)[i];
                bad |= !finite_f(v.x) || !finite_f(v.y) || !finite_f(v.z) || !finite_f(v.w);
            }
            if (blockIdx.x == 0 && threadIdx.x < 32 && (n4 << 2) + threadIdx.x < n)
                bad |= !finite_f(r[(n4 << 2) + threadIdx.x]);
        } else {
            for (int64_t i = gtid; i < n; i += nthreads) bad |= !finite_f(r[i]);
        }
    }
    while (tail != head) drain((int)min(32u, tail - head));
    acc.cntR += far_right + (uint32_t)far_right_f;
    acc.bad |= bad;
    __syncthreads();
    band_flush(sband, scount, band, counter, cap, BL, inv_t, bins, &gbase);
    // the CTA's record (count, left sum, right sum, non-finite flag), summed
    // into thread 0 in a fixed order
    // the CTA's record (count, left sum, right sum, non-finite flag), summed
    // into thread 0 in a fixed order; the solve kernel combines the records
    double rec[4] = {(double)acc.cntR, acc.SL, acc.SR, acc.bad ? 1.0 : 0.0};
    block_sum4_to0(rec, red4);
    if (threadIdx.x == 0) {
        double2* pr = reinterpret_cast<double2*>(part) + 2 * blockIdx.x;
        pr[0] = make_double2(rec[0], rec[1]);
        pr[1] = make_double2(rec[2], rec[3]);
    }
    if (blockIdx.x == 0) phase_mark(st, 17);
}

struct FloatGet {
    const float* s;
    __device__ __forceinline__ float operator()(long long j) const { return s[j]; }
};
struct ConstGet {
    float v;
    __device__ __forceinline__ float operator()(long long) const { return v; }
};

struct SolveSmemAll {
    SolveScratch ss;
    SolveResult res;
    Tails sub;          // tails of a histogram sub-bracket
    double binF[2];     // F at the first and last histogram edge
    double red[32];
    float fred[32];
    long long lred[32];
    uint32_t wsum[32];
    uint32_t bcast[8];
    unsigned long long cnt;
    double sred[32][8];  // per-warp partial sums of block_sums
    double sres[8];      // and their totals
    int flag;
    union {
        struct {
            uint32_t xch[4 * kBlk];
            float sorted[kBandSortMax];
        } sort;
        struct {
            uint32_t cnt[kRefineBins];
            float U[kRefineBins];
            float L[kRefineBins];
        } hist;
        uint32_t sel_hist[2048];
    } u;
};

// Band of size <= 4096: sort on chip and solve with the tails.  The network
// size follows the band: 1, 2 or 4 keys per thread.
template <int E>
__device__ void sort_band_into(const float* band, long long nb, SolveSmemAll* sm) {
    uint32_t key[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const long long j = (long long)threadIdx.x * E + e;
        key[e] = j < nb ? to_key(band[j]) : 0xffffffffu;
    }
    bitonic_sort_row<E, kBlk, kBlk>(key, threadIdx.x, sm->u.sort.xch);
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const long long j = (long long)threadIdx.x * E + e;
        if (j < nb) sm->u.sort.sorted[j] = from_key(key[e]);
    }
    __syncthreads();
}
__device__ void solve_small_band(const float* band, long long nb, const Tails& tl, double k,
                                 double t, SolveSmemAll* sm) {
    if (nb <= kBlk) sort_band_into<1>(band, nb, sm);
    else if (nb <= 2 * kBlk) sort_band_into<2>(band, nb, sm);
    else sort_band_into<4>(band, nb, sm);
    solve_sorted_block(FloatGet{sm->u.sort.sorted}, nb, tl, k, t, &sm->ss, &sm->res);
}

// Exact F at the ends of [tl.aL, tl.aR) from a band in global memory (any size),
// plus the band's key range.
__device__ void certify_big_band(const float* band, long long nb, const Tails& tl, double t,
                                 SolveSmemAll* sm, double* F_aL, double* F_aR, uint32_t* kmin,
                                 uint32_t* kmax) {
    double wl = 0.0, vr = 0.0;
    uint32_t lo = 0xffffffffu, hi = 0u;
    const double inv_t = 1.0 / t;
    for (long long j = threadIdx.x; j < nb; j += blockDim.x) {
        const float s = band[j];
        if (tl.hasL) wl += (double)exp_neg((float)((s - tl.aL) * inv_t));
        if (tl.hasR) vr += (double)exp_neg((float)((tl.aR - s) * inv_t));
        const uint32_t kk = to_key(s);
        lo = min(lo, kk);
        hi = max(hi, kk);
    }
    wl = block_sum_d(wl, sm->red);
    vr = block_sum_d(vr, sm->red);
    // key min/max through the float reductions' shared slots
    {
        const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) {
            lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, d));
            hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, d));
        }
        __syncthreads();
        if (lane == 0) {
            sm->wsum[w] = lo;
            sm->u.sel_hist[w] = hi;
        }
        __syncthreads();
        lo = 0xffffffffu;
        hi = 0u;
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
            lo = min(lo, sm->wsum[i]);
            hi = max(hi, sm->u.sel_hist[i]);
        }
        __syncthreads();
    }
    const double lnw = (tl.hasL && tl.hasR) ? ((double)tl.aL - (double)tl.aR) / t : -INFINITY;
    *F_aL = tl.hasL ? tl.cntR + (double)nb - 0.5 * (wl + tl.SR * cold_exp(lnw)) + 0.5 * tl.SL : INFINITY;
    *F_aR = tl.hasR ? tl.cntR - 0.5 * tl.SR + 0.5 * (vr + tl.SL * cold_exp(lnw)) : -INFINITY;
    *kmin = lo;
    *kmax = hi;
}

// One narrowing level of a certified band in `in` (nb > 4096, kmin < kmax):
// histogram the band over <= 2048 key bins with per-bin exponential sums,
// evaluate F at every bin edge by two affine scans, pick the edge pair that
// straddles k, verify it with exact fp64 sums (moving one bin if rounding in
// the histogram picked the wrong one), and compact that bin into `out`.
// Returns the new band size; updates the tails in place.
__device__ long long refine_level(const float* in, long long nb, float* out, Tails& tl,
                                  uint32_t kmin, uint32_t kmax, double k, double t,
                                  SolveSmemAll* sm, uint32_t* nkmin, uint32_t* nkmax) {
    const float inv_t = (float)(1.0 / t);
    const double inv_td = 1.0 / t;  // the exact checks' arguments, in fp64
    const uint32_t range = kmax - kmin;
    int sh = 0;
    while ((range >> sh) >= (uint32_t)kRefineBins) ++sh;
    const int nbin = (int)(range >> sh) + 1;
    auto edge_key = [&](int j) -> uint32_t {
        const unsigned long long e = (unsigned long long)kmin + ((unsigned long long)j << sh);
        const unsigned long long top = (unsigned long long)kmax + 1ull;
        return (uint32_t)(e < top ? e : top);
    };
    auto edge = [&](int j) -> float { return from_key(edge_key(j)); };

    for (int j = threadIdx.x; j < kRefineBins; j += blockDim.x) {
        sm->u.hist.cnt[j] = 0;
        sm->u.hist.U[j] = 0.f;
        sm->u.hist.L[j] = 0.f;
    }
    __syncthreads();
    for (long long i = threadIdx.x; i < nb; i += blockDim.x) {
        const float s = in[i];
        const int j = (int)((to_key(s) - kmin) >> sh);
        atomicAdd(&sm->u.hist.cnt[j], 1u);
        atomicAdd(&sm->u.hist.U[j], __expf((edge(j) - s) * inv_t));
        atomicAdd(&sm->u.hist.L[j], __expf((s - edge(j + 1)) * inv_t));
    }
    __syncthreads();
    // F at every bin edge e_0..e_nbin from the bin aggregates, by two affine
    // scans over the bins (thread i owns bins 2i and 2i+1; bins past nbin are
    // empty and their edges coincide, so their maps are the identity).
    //   Q_j = U_j + g_j Q_{j+1}, Q_nbin = SR e^{(e_nbin - aR)/t}    (weights above e_j)
    //   P_j = L_{j-1} + g_{j-1} P_{j-1}, P_0 = SL e^{(aL - e_0)/t}  (weights below e_j)
    //   F(e_j) = cntR + #{scores in bins >= j} - Q_j/2 + P_j/2,   g_j = e^{(e_j - e_{j+1})/t}
    {
        const int b0 = 2 * threadIdx.x, b1 = b0 + 1;
        const double e0 = (double)edge(b0), e1 = (double)edge(b1), e2 = (double)edge(b1 + 1);
        const double g0 = cold_exp((e0 - e1) / t), g1 = cold_exp((e1 - e2) / t);
        const double U0 = sm->u.hist.U[b0], U1 = sm->u.hist.U[b1];
        const double L0 = sm->u.hist.L[b0], L1 = sm->u.hist.L[b1];
        const long long c01 = (long long)sm->u.hist.cnt[b0] + (long long)sm->u.hist.cnt[b1];
        const Aff mb = aff_then(Aff{g1, U1}, Aff{g0, U0});      // apply bin b1, then b0
        const Aff mf = aff_then(Aff{g0, L0}, Aff{g1, L1});      // edge b0+1, then b0+2
        const Aff eb = block_excl_scan_bwd(mb, sm->ss.wb);
        const Aff ef = block_excl_scan_fwd(mf, sm->ss.wf);
        const long long above = block_excl_suffix_ll(c01, sm->lred);
        const double Qend = tl.hasR ? tl.SR * cold_exp(((double)edge(kRefineBins) - (double)tl.aR) / t) : 0.0;
        const double Pstart = tl.hasL ? tl.SL * cold_exp(((double)tl.aL - (double)edge(0)) / t) : 0.0;
        const double Q2 = fma(eb.a, Qend, eb.c);                // Q at edge b0+2
        const double Q1 = fma(g1, Q2, U1);
        const double Q0 = fma(g0, Q1, U0);
        const double P0 = fma(ef.a, Pstart, ef.c);              // P at edge b0
        const double P1 = fma(g0, P0, L0);
        const double F0 = tl.cntR + (double)(above + c01) - 0.5 * Q0 + 0.5 * P0;
        const double F1 = tl.cntR + (double)(above + (long long)sm->u.hist.cnt[b1]) - 0.5 * Q1 +
                          0.5 * P1;
        int c = 0;
        if (b0 <= nbin && F0 >= k) ++c;
        if (b1 <= nbin && F1 >= k) ++c;
        // Edge e_2048 itself is not evaluated; when b lies above every edge
        // evaluated here, the exact check below moves the bracket up to it.
        const int tot = __syncthreads_count(c >= 1) + __syncthreads_count(c >= 2);
        if (threadIdx.x == 0) sm->bcast[0] = (uint32_t)(tot - 1);
    }
    __syncthreads();
    int jc = (int)sm->bcast[0];
    long long cnt = 0;
    for (int guard = 0; guard < nbin + 2; ++guard) {
        const bool useL = jc < 0, useR = jc + 1 > nbin;
        const float Elo = useL ? tl.aL : edge(jc);
        const float Ehi = useR ? tl.aR : edge(jc + 1);
        const bool hasLo = useL ? tl.hasL : true;
        const bool hasHi = useR ? tl.hasR : true;
        if (threadIdx.x == 0) sm->cnt = 0ull;
        __syncthreads();
        double sl = 0.0, sr = 0.0, w = 0.0, v = 0.0;
        long long cr = 0;
        uint32_t lo = 0xffffffffu, hi = 0u;
        for (long long i = threadIdx.x; i < nb; i += blockDim.x) {
            const float s = in[i];
            bool take = false;
            if (hasHi && s >= Ehi) {
                cr += 1;
                sr += (double)exp_neg((float)(((double)s - (double)Ehi) * inv_td));
            } else if (hasLo && s < Elo) {
                sl += (double)exp_neg((float)(((double)Elo - (double)s) * inv_td));
            } else {
                take = true;
                if (hasLo) w += (double)exp_neg((float)(((double)s - (double)Elo) * inv_td));
                if (hasHi) v += (double)exp_neg((float)(((double)Ehi - (double)s) * inv_td));
                const uint32_t kk = to_key(s);
                lo = min(lo, kk);
                hi = max(hi, kk);
            }
            if (take) {
                const unsigned long long pos = atomicAdd(&sm->cnt, 1ull);
                out[pos] = s;
            }
        }
        sl = block_sum_d(sl, sm->red);
        sr = block_sum_d(sr, sm->red);
        w = block_sum_d(w, sm->red);
        v = block_sum_d(v, sm->red);
        cr = block_sum_ll(cr, sm->lred);
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) {
            lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, d));
            hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, d));
        }
        if ((threadIdx.x & 31) == 0) {
            atomicMin(&sm->bcast[2], lo);
            atomicMax(&sm->bcast[3], hi);
        }
        __syncthreads();
        cnt = (long long)sm->cnt;
        // new tails
        Tails nt;
        nt.hasL = hasLo;
        nt.aL = Elo;
        nt.SL = (useL ? tl.SL : (tl.hasL ? tl.SL * cold_exp(((double)tl.aL - (double)Elo) / t) : 0.0)) + sl;
        nt.hasR = hasHi;
        nt.aR = Ehi;
        nt.SR = (useR ? tl.SR : (tl.hasR ? tl.SR * cold_exp(((double)Ehi - (double)tl.aR) / t) : 0.0)) + sr;
        nt.cntR = tl.cntR + (double)cr;
        const double lnw = (hasLo && hasHi) ? ((double)Elo - (double)Ehi) / t : -INFINITY;
        const double FL = hasLo ? nt.cntR + (double)cnt - 0.5 * (w + nt.SR * cold_exp(lnw)) + 0.5 * nt.SL
                                : INFINITY;
        const double FR = hasHi ? nt.cntR - 0.5 * nt.SR + 0.5 * (v + nt.SL * cold_exp(lnw)) : -INFINITY;
        const uint32_t klo = sm->bcast[2], khi = sm->bcast[3];
        __syncthreads();
        if (threadIdx.x == 0) {
            sm->bcast[2] = 0xffffffffu;
            sm->bcast[3] = 0u;
        }
        if (FL < k && jc >= 0) {
            --jc;
        } else if (FR > k && jc + 1 <= nbin) {
            ++jc;
        } else {
            tl = nt;
            *nkmin = klo;
            *nkmax = khi;
            __syncthreads();
            return cnt;
        }
        __syncthreads();
    }
    return -1;  // unreachable for a certified input band
}

// F at every edge of the fold's band histogram, by two affine scans over the
// bins (thread i owns bins 2i and 2i+1; bins past nbin are empty with equal
// edges, so their maps are the identity):
//   Q_j = U_j + g_j Q_{j+1}   (weights of scores >= e_j),  Q at the top edge = S_R
//   P_j = L_{j-1} + g_{j-1} P_{j-1}  (weights of scores < e_j),  P_0 = S_L
//   F(e_j) = #{scores >= e_j} - Q_j/2 + P_j/2,   g_j = e^{(e_j - e_{j+1})/t}.
// Returns #{edges 0..nbin with F >= k}; F at edge 0 and edge nbin go to
// sm->binF.  With want >= 0 the tails of the sub-bracket [e_want, e_want+1)
// go to sm->sub.  Every thread of the (1024-thread) block must call it.
// With want == -2 the thread that sees the straddle locally (F >= k at edge j,
// F < k at edge j + 1) leaves j in sm->bcast[7] and the sub-bracket tails in
// sm->sub; sm->bcast[6] counts such claims (one when F is monotone).
__device__ int bin_scan(const BinLayout& BL, const unsigned long long* __restrict__ bins,
                        const Tails& tl, double k, double t, SolveSmemAll* sm, int want) {
    const int b0 = 2 * threadIdx.x, b1 = b0 + 1;
    if (want == -2 && threadIdx.x == 0) sm->bcast[6] = 0u;  // read after the scans' barriers
    const double e0 = (double)bin_edge(BL, b0), e1 = (double)bin_edge(BL, b1);
    const double e2 = (double)bin_edge(BL, b1 + 1);
    const double g0 = (e1 > e0) ? cold_exp((e0 - e1) / t) : 1.0;
    const double g1 = (e2 > e1) ? cold_exp((e1 - e2) / t) : 1.0;
    const long long c0 = (long long)bins[b0], c1 = (long long)bins[b1];
    const double U0 = (double)bins[kBins + b0] / kFixScale, U1 = (double)bins[kBins + b1] / kFixScale;
    const double L0 = (double)bins[2 * kBins + b0] / kFixScale;
    const double L1 = (double)bins[2 * kBins + b1] / kFixScale;
    const Aff mb = aff_then(Aff{g1, U1}, Aff{g0, U0});  // bin b1 first, then b0
    const Aff mf = aff_then(Aff{g0, L0}, Aff{g1, L1});  // edge b0+1, then b0+2
    const Aff eb = block_excl_scan_bwd(mb, sm->ss.wb);
    const Aff ef = block_excl_scan_fwd(mf, sm->ss.wf);
    const long long above = block_excl_suffix_ll(c0 + c1, sm->lred);
    const double etop = (double)bin_edge(BL, kBins), efirst = (double)bin_edge(BL, 0);
    const double Qend = (tl.hasR && tl.SR > 0.0) ? tl.SR * cold_exp((etop - (double)tl.aR) / t) : 0.0;
    const double Pst = (tl.hasL && tl.SL > 0.0) ? tl.SL * cold_exp(((double)tl.aL - efirst) / t) : 0.0;
    const double Q2 = fma(eb.a, Qend, eb.c), Q1 = fma(g1, Q2, U1), Q0 = fma(g0, Q1, U0);
    const double P0 = fma(ef.a, Pst, ef.c), P1 = fma(g0, P0, L0), P2 = fma(g1, P1, L1);
    const double A2 = tl.cntR + (double)above, A1 = A2 + (double)c1, A0 = A1 + (double)c0;
    const double F0 = A0 - 0.5 * Q0 + 0.5 * P0, F1 = A1 - 0.5 * Q1 + 0.5 * P1;
    const double F2 = A2 - 0.5 * Q2 + 0.5 * P2;
    const int nb = BL.nbin;
    int c = 0;
    if (b0 <= nb && F0 >= k) ++c;
    if (b1 <= nb && F1 >= k) ++c;
    if (b1 + 1 == kBins && kBins <= nb && F2 >= k) ++c;
    if (b0 == 0) sm->binF[0] = F0;
    if (b0 == nb) sm->binF[1] = F0;
    if (b1 == nb) sm->binF[1] = F1;
    if (b1 + 1 == nb) sm->binF[1] = F2;
    if (want == -2) {
        auto claim = [&](int j, double SL, double SR, double cR) {
            if (atomicAdd(&sm->bcast[6], 1u) == 0u) {
                sm->bcast[7] = (uint32_t)j;
                sm->sub.SL = SL;
                sm->sub.SR = SR;
                sm->sub.cntR = cR;
            }
        };
        if (b0 < nb && F0 >= k && F1 < k) claim(b0, P0, Q1, A1);
        if (b1 < nb && F1 >= k && F2 < k) claim(b1, P1, Q2, A2);
    }
    if (want >= 0) {
        // lower end e_want: weights below it; upper end e_want+1: weights and count above it
        if (b0 == want) sm->sub.SL = P0;
        if (b1 == want) sm->sub.SL = P1;
        if (b0 == want + 1) { sm->sub.SR = Q0; sm->sub.cntR = A0; }
        if (b1 == want + 1) { sm->sub.SR = Q1; sm->sub.cntR = A1; }
        if (b1 + 1 == want + 1) { sm->sub.SR = Q2; sm->sub.cntR = A2; }
        if (threadIdx.x == 0) {
            sm->sub.hasL = true;
            sm->sub.aL = bin_edge(BL, want);
            const float hi = bin_edge(BL, want + 1);
            sm->sub.hasR = isfinite(hi);
            sm->sub.aR = hi;
        }
    }
    const int tot = __syncthreads_count(c >= 1) + __syncthreads_count(c >= 2) +
                    __syncthreads_count(c >= 3);
    return tot;
}

// Copies the band scores that fall in histogram bin `j` into sm->u.sort.sorted
// (at most kBandSortMax of them); returns how many there were.
__device__ long long extract_bin(const float* __restrict__ band, long long nb, const BinLayout& BL,
                                 int j, SolveSmemAll* sm) {
    if (threadIdx.x == 0) sm->cnt = 0ull;
    __syncthreads();
    const long long n4 = nb >> 2;
    const float4* b4 = reinterpret_cast<const float4*>(band);
    // eight 16-byte loads per thread in flight per trip (the band sits in L2)
    constexpr int G = 8;
    for (long long i0 = 0; i0 < n4; i0 += (long long)G * blockDim.x) {
        float4 v[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const long long i = i0 + (long long)g * blockDim.x + threadIdx.x;
            v[g] = i < n4 ? __ldcg(b4 + i) : make_float4(NAN, NAN, NAN, NAN);
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float xs[4] = {v[g].x, v[g].y, v[g].z, v[g].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (xs[q] == xs[q] && bin_of(BL, to_key(xs[q])) == j) {
                    const unsigned long long pos = atomicAdd(&sm->cnt, 1ull);
                    if (pos < (unsigned long long)kBandSortMax) sm->u.sort.sorted[pos] = xs[q];
                }
            }
        }
    }
    for (long long i = (n4 << 2) + threadIdx.x; i < nb; i += blockDim.x) {
        const float x = band[i];
        if (bin_of(BL, to_key(x)) == j) {
            const unsigned long long pos = atomicAdd(&sm->cnt, 1ull);
            if (pos < (unsigned long long)kBandSortMax) sm->u.sort.sorted[pos] = x;
        }
    }
    __syncthreads();
    return (long long)sm->cnt;
}

// Solve through the fold's histogram: certify the bracket from the bin sums,
// pick the bin whose edges straddle k, and solve exactly on that bin's scores
// with the other bins folded into its tails.  A bin picked wrongly by the
// fixed-point rounding fails its own end check and the neighbour is tried.
// Returns 1 (solved, b in sm->res), 0 (bracket failed: F at the ends in
// sm->res), or -1 (the bin is too full for the on-chip sort: use the exact
// narrowing path).
__device__ int solve_with_bins(const float* __restrict__ band, long long nb,
                               const unsigned long long* __restrict__ bins, const BinLayout& BL,
                               const Tails& tl, double k, double t, SolveSmemAll* sm,
                               RowState* probe) {
    const int cntF = bin_scan(BL, bins, tl, k, t, sm, -1);
    const double FL = tl.hasL ? sm->binF[0] : INFINITY;
    const double FR = tl.hasR ? sm->binF[1] : -INFINITY;
    if (!(FL >= k && FR <= k)) {
        __syncthreads();
        if (threadIdx.x == 0) {
            sm->res.F_aL = FL;
            sm->res.F_aR = FR;
        }
        __syncthreads();
        return 0;
    }
    int jc = cntF - 1;
    if (jc < 0) jc = 0;
    if (jc > BL.nbin - 1) jc = BL.nbin - 1;
    for (int guard = 0; guard < 8; ++guard) {
        __syncthreads();
        bin_scan(BL, bins, tl, k, t, sm, jc);
        if ((long long)bins[jc] > kBandSortMax) return -1;
        if (probe) phase_mark(probe, 6 + 3 * min(guard, 1));
        const long long c = extract_bin(band, nb, BL, jc, sm);
        if (probe) phase_mark(probe, 7 + 3 * min(guard, 1));
        Tails sub = sm->sub;
        solve_small_band(sm->u.sort.sorted, c, sub, k, t, sm);
        if (probe) phase_mark(probe, 8 + 3 * min(guard, 1));
        if (sm->res.F_aL < k && jc > 0) {
            --jc;
        } else if (sm->res.F_aR > k && jc < BL.nbin - 1) {
            ++jc;
        } else {
            return 1;
        }
    }
    return -1;
}

// Exact solve of a band too large for the on-chip sort: certify the bracket,
// then narrow by key histograms (ping-ponging between cur and nxt) until the
// band fits on chip or holds a single value.  Returns 1 (solved, b in
// sm->res), 0 (the bracket failed: F at the ends in sm->res) or -1 (no bin
// certified while narrowing; not expected, reported as a failure).
__device__ int solve_exact(float* cur, float* nxt, long long nb, Tails tl, double k,
                           double t, SolveSmemAll* sm, int* levels) {
    double FL, FR;
    uint32_t kmin, kmax;
    certify_big_band(cur, nb, tl, t, sm, &FL, &FR, &kmin, &kmax);
    if (!(FL >= k && FR <= k)) {
        // F at the ends is enough to know which end failed
        if (threadIdx.x == 0) {
            sm->res.F_aL = FL;
            sm->res.F_aR = FR;
        }
        __syncthreads();
        return 0;
    }
    while (nb > kBandSortMax && kmin < kmax) {
        uint32_t nkmin = 0, nkmax = 0;
        nb = refine_level(cur, nb, nxt, tl, kmin, kmax, k, t, sm, &nkmin, &nkmax);
        if (nb < 0) return -1;
        ++*levels;
        float* tmp = cur;
        cur = nxt;
        nxt = tmp;
        kmin = nkmin;
        kmax = nkmax;
    }
    if (nb <= kBandSortMax)
        solve_small_band(cur, nb, tl, k, t, sm);
    else
        solve_sorted_block(ConstGet{from_key(kmin)}, nb, tl, k, t, &sm->ss, &sm->res);
    return 1;
}

// First half of the histogram solve: certify the bracket from the bin sums and
// choose the bin whose edges straddle k, leaving its tails in the row record
// for the extract and final solve kernels.  Returns 1 (bin chosen), 0 (the
// bracket failed: F at the ends in sm->res) or -1 (that bin is too full for
// the on-chip sort: use the exact narrowing path).
__device__ int plan_with_bins(const unsigned long long* __restrict__ bins, const BinLayout& BL,
                              const Tails& tl, double k, double t, SolveSmemAll* sm,
                              RowState* st) {
    const int cntF = bin_scan(BL, bins, tl, k, t, sm, -2);
    const double FL = tl.hasL ? sm->binF[0] : INFINITY;
    const double FR = tl.hasR ? sm->binF[1] : -INFINITY;
    if (!(FL >= k && FR <= k)) {
        __syncthreads();
        if (threadIdx.x == 0) {
            sm->res.F_aL = FL;
            sm->res.F_aR = FR;
        }
        __syncthreads();
        return 0;
    }
    int jc = cntF - 1;
    if (jc < 0) jc = 0;
    if (jc > BL.nbin - 1) jc = BL.nbin - 1;
    __syncthreads();
    if (sm->bcast[6] == 1u && (int)sm->bcast[7] == jc) {
        // the first scan already left this bin's tails
        if (threadIdx.x == 0) {
            sm->sub.hasL = true;
            sm->sub.aL = bin_edge(BL, jc);
            const float hi = bin_edge(BL, jc + 1);
            sm->sub.hasR = isfinite(hi);
            sm->sub.aR = hi;
        }
        __syncthreads();
    } else {
        bin_scan(BL, bins, tl, k, t, sm, jc);
    }
    if ((long long)bins[jc] > kBandSortMax) return -1;
    if (threadIdx.x == 0) {
        st->sub_bin = jc;
        st->sub_aL = sm->sub.aL;
        st->sub_aR = sm->sub.aR;
        st->sub_hasR = sm->sub.hasR ? 1 : 0;
        st->sub_SL = sm->sub.SL;
        st->sub_SR = sm->sub.SR;
        st->sub_cntR = sm->sub.cntR;
        st->n_sub = 0ull;
    }
    return 1;
}

// Single-CTA fold (kBlk threads) of one row: the tail sums and right count of [aL, aR), the
// band scores appended to `band` (capacity n; order depends on timing, the
// solve sorts it).  Four 16-byte loads per thread in flight per trip; every
// score takes one exponential (masked inside the band).  Sets *bad when a
// score is NaN or infinite.
// SOFT: a soft row (40 t >= |b|, b judged by the bracket's finite ends), whose
// tail terms are taken in fp64 so that sums of very many soft scores keep the
// budget; refold_row picks the instance once per call.
template <bool SOFT>
__device__ __noinline__ void refold_row_t(const float* __restrict__ r, int64_t n, int vec, float aL,
                                          float aR, double t, float* band, SolveSmemAll* sm,
                                          Tails& tl, long long* nb, bool* bad) {
    const float k2 = (float)(kLog2e / t);
    const double inv_td = 1.0 / t;
    constexpr bool soft = SOFT;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) sm->cnt = 0ull;
    __syncthreads();
    double SL = 0.0, SR = 0.0;
    uint32_t cR = 0u;
    float probe = 0.f;  // NaN once a score is NaN or infinite
    // One score (ok = in range): the tail terms; returns whether it is in the band.
    auto fold1 = [&](float x, bool ok, float& sl, float& sr) -> bool {
        const bool right = ok && x >= aR, left = ok && x < aL;
        if constexpr (soft) {
            const double a = right ? ((double)x - (double)aR) * inv_td
                                   : (left ? ((double)aL - (double)x) * inv_td : 0.0);
            const double e = exp(-a);
            SR += right ? e : 0.0;
            SL += left ? e : 0.0;
        } else {
            const float e = ex2_ftz((right ? aR - x : (left ? x - aL : 0.f)) * k2);
            sr += right ? e : 0.f;
            sl += left ? e : 0.f;
        }
        cR += right ? 1u : 0u;
        if (ok) probe = fmaf(x, 0.f, probe);
        return ok && !right && !left;
    };
    // Band scores are staged per warp (128 slots of the sort's exchange
    // buffer, free during the fold) and moved to the band with one atomic per
    // 96 or more, so the warps do not queue on one shared counter.
    constexpr uint32_t kWarpStage = 128;
    float* stg = reinterpret_cast<float*>(sm->u.sort.xch) + (threadIdx.x >> 5) * kWarpStage;
    uint32_t wc = 0u;  // warp-uniform: scores staged
    auto flush = [&]() {
        unsigned long long base = 0ull;
        if (lane == 0 && wc != 0u) base = atomicAdd(&sm->cnt, (unsigned long long)wc);
        base = __shfl_sync(0xffffffffu, base, 0);
        __syncwarp();
        for (uint32_t i = lane; i < wc; i += 32)
            if (base + i < (unsigned long long)n) band[base + i] = stg[i];
        __syncwarp();
        wc = 0u;
    };
    // Every lane of the warp calls it together.
    auto append = [&](bool take, float x) {
        const unsigned ball = __ballot_sync(0xffffffffu, take);
        if (ball != 0u) {
            if (take) stg[wc + __popc(ball & ((1u << lane) - 1u))] = x;
            wc += (uint32_t)__popc(ball);
            if (wc > kWarpStage - 32u) flush();
        }
    };
    if (vec) {
        const int64_t n4 = n >> 2;
        constexpr int U = 4;
        constexpr int64_t per_trip = (int64_t)U * kBlk;
        const float4* p4 = reinterpret_cast<const float4*>(r) + threadIdx.x;
        for (int64_t i0 = 0; i0 < n4; i0 += per_trip, p4 += per_trip) {  // same trip count in every lane
            const int64_t rem = n4 - i0 - (int64_t)threadIdx.x;  // this thread's vectors left
            float4 v[U];
#pragma unroll
            for (int q = 0; q < U; ++q)
                v[q] = (int64_t)q * kBlk < rem ? __ldcg(p4 + q * kBlk) : make_float4(0.f, 0.f, 0.f, 0.f);
            // the tails first, with the trip's band scores marked in bm (bit 4q + c);
            // the appends stay off this path, so it holds no more than the loads
            float sl = 0.f, sr = 0.f;
            uint32_t bm = 0u;
#pragma unroll
            for (int q = 0; q < U; ++q) {
                const bool ok = (int64_t)q * kBlk < rem;
                bm |= (uint32_t)fold1(v[q].x, ok, sl, sr) << (4 * q);
                bm |= (uint32_t)fold1(v[q].y, ok, sl, sr) << (4 * q + 1);
                bm |= (uint32_t)fold1(v[q].z, ok, sl, sr) << (4 * q + 2);
                bm |= (uint32_t)fold1(v[q].w, ok, sl, sr) << (4 * q + 3);
            }
            SL += (double)sl;
            SR += (double)sr;
            if (__any_sync(0xffffffffu, bm != 0u)) {
#pragma unroll
                for (int q = 0; q < U; ++q) {
                    append((bm >> (4 * q)) & 1u, v[q].x);
                    append((bm >> (4 * q + 1)) & 1u, v[q].y);
                    append((bm >> (4 * q + 2)) & 1u, v[q].z);
                    append((bm >> (4 * q + 3)) & 1u, v[q].w);
                }
            }
        }
        if (threadIdx.x < 32) {  // the last n mod 4 scores, by warp 0
            const int64_t i = (n4 << 2) + threadIdx.x;
            const bool ok = i < n;
            const float x = ok ? r[i] : 0.f;
            float sl = 0.f, sr = 0.f;
            append(fold1(x, ok, sl, sr), x);
            SL += (double)sl;
            SR += (double)sr;
        }
    } else {
        for (int64_t i0 = 0; i0 < n; i0 += kBlk) {  // same trip count in every lane
            const int64_t i = i0 + threadIdx.x;
            const bool ok = i < n;
            const float x = ok ? r[i] : 0.f;
            float sl = 0.f, sr = 0.f;
            append(fold1(x, ok, sl, sr), x);
            SL += (double)sl;
            SR += (double)sr;
        }
    }
    flush();
    const double sL = block_sum_d(SL, sm->red);
    const double sR = block_sum_d(SR, sm->red);
    const long long cnt = block_sum_ll((long long)cR, sm->lred);
    const int any_bad = __syncthreads_or(!(probe == 0.f));
    tl.hasL = isfinite(aL);
    tl.aL = aL;
    tl.SL = sL;
    tl.hasR = isfinite(aR);
    tl.aR = aR;
    tl.SR = sR;
    tl.cntR = (double)cnt;
    *nb = (long long)sm->cnt;
    if (bad) *bad = any_bad != 0;
}

__device__ void refold_row(const float* __restrict__ r, int64_t n, int vec, float aL, float aR,
                           double t, float* band, SolveSmemAll* sm, Tails& tl, long long* nb,
                           bool* bad) {
    const double bc = isfinite(aL) ? (isfinite(aR) ? 0.5 * ((double)aL + (double)aR) : (double)aL)
                                   : (isfinite(aR) ? (double)aR : 0.0);
    if (40.0 * t >= fabs(bc)) refold_row_t<true>(r, n, vec, aL, aR, t, band, sm, tl, nb, bad);
    else refold_row_t<false>(r, n, vec, aL, aR, t, band, sm, tl, nb, bad);
}

// The attempt loop of the band solve, shared by the grid pipeline's solve
// kernel and the one-CTA-per-row kernel.  Solves the current band exactly
// once its bracket certifies; otherwise widens the failing end by one rung of
// the ladder (select_key(rank) gives the key of that sample order statistic)
// and folds the row again.  On the first attempt a band too large for the
// on-chip sort goes through the fold's histogram (`bins`, when given; with
// `split` the chosen bin is left for the extract and second solve kernels and
// the function returns true at once).  Otherwise writes b, the record and the
// status, and returns false.
template <class SelectKey>
__device__ __noinline__ bool bracket_attempts(const float* __restrict__ r, int64_t n, int vec, double k,
                                 double t, RowState* st, float* band0, float* band1,
                                 const unsigned long long* __restrict__ bins, int split, int m,
                                 const Ladder& lad, SelectKey select_key, Tails tl, long long nb,
                                 SolveSmemAll* sm, double* b_out, WsHeader* hdr) {
    int rungL = st->rung_L, rungR = st->rung_R;
    const int max_attempts = st->max_attempts;
    int attempt = 1;
    int levels = 0;
    bool done = false;
    double b = nan("");
    Tails cert = tl;
    long long nb_cert = nb;
    while (true) {
        float* cur = band0;
        float* nxt = band1;
        bool certified;
        cert = tl;
        nb_cert = nb;
        int via_bins = -1;
        if (bins != nullptr && nb > kBandSortMax && attempt == 1) {
            // the fold built the band histogram for this first bracket; the
            // chosen bin is extracted and solved by the next two kernels when
            // they were launched (split), else here
            const BinLayout BL = make_bins(st->bin_kmin, st->bin_kmax);
            if (!split) {
                via_bins = solve_with_bins(cur, nb, bins, BL, tl, k, t, sm, nullptr);
                if (via_bins == 1) {
                    b = sm->res.b;
                    done = true;
                    certified = true;
                } else if (via_bins == 0) {
                    certified = false;
                }
            } else {
                via_bins = plan_with_bins(bins, BL, tl, k, t, sm, st);
            }
            if (split && via_bins == 1) {
                phase_mark(st, 3);
                if (threadIdx.x == 0) {
                    st->stage = 1;
                    st->attempts = attempt;
                    st->refine_levels = 0;
                    st->certified = 1;
                }
                return true;
            } else if (via_bins == 0) {
                certified = false;
            }
        }
        if (via_bins >= 0) {
            // handled through the histogram
        } else if (nb <= kBandSortMax) {
            phase_mark(st, 19);
            if (nb <= kBlk) sort_band_into<1>(cur, nb, sm);
            else if (nb <= 2 * kBlk) sort_band_into<2>(cur, nb, sm);
            else sort_band_into<4>(cur, nb, sm);
            phase_mark(st, 20);
            solve_sorted_block(FloatGet{sm->u.sort.sorted}, nb, tl, k, t, &sm->ss, &sm->res);
            phase_mark(st, 21);
            certified = sm->res.F_aL >= k && sm->res.F_aR <= k;
            if (certified) {
                b = sm->res.b;
                done = true;
            }
        } else {
            const int e = solve_exact(cur, nxt, nb, tl, k, t, sm, &levels);
            certified = e != 0;
            if (e < 0) break;
            if (e > 0) {
                b = sm->res.b;
                done = true;
            }
        }
        if (done || attempt >= max_attempts) break;
        // widen the failing end to its next rung and fold again
        const bool fail_left = sm->res.F_aL < k;
        float aL = tl.aL, aR = tl.aR;
        if (!tl.hasL) aL = -INFINITY;
        if (!tl.hasR) aR = INFINITY;
        if (fail_left) {
            ++rungL;
            if (rungL >= kLadder - 1 || lad.h[rungL] > m) aL = -INFINITY;
            else aL = from_key(select_key(lad.h[rungL]));
        } else {
            ++rungR;
            if (rungR >= kLadder - 1 || lad.l[rungR] < 1) aR = INFINITY;
            else aR = from_key(select_key(lad.l[rungR]));
        }
        ++attempt;
        refold_row(r, n, vec, aL, aR, t, band0, sm, tl, &nb, nullptr);
    }
    phase_mark(st, 12);
    if (threadIdx.x == 0) {
        st->attempts = attempt;
        st->refine_levels = levels;
        st->rung_L = rungL;
        st->rung_R = rungR;
        st->a_L = cert.hasL ? cert.aL : -INFINITY;
        st->a_R = cert.hasR ? cert.aR : INFINITY;
        st->S_L = cert.SL;
        st->S_R = cert.SR;
        st->cnt_R = (unsigned long long)cert.cntR;
        st->n_band = (unsigned long long)nb_cert;
        st->certified = done ? 1 : 0;
        if (!done) {
            b = nan("");
            st->status |= kDevBracketExhausted;
            set_status(hdr, kDevBracketExhausted);
        }
        st->b = b;
        *b_out = b;
    }
    __syncthreads();
    return false;
}

// ----------------------------------------------------------------------------
// Exact solve of a band of at most kBandSortMax scores without sorting it (the
// usual first attempt).  Every thread holds up to four band scores.
//  1. Certification: F(a_L) >= k >= F(a_R) from the tails and the band.
//  2. Multisection on the band's own values: the segment (lo, hi) of the
//     threshold curve that holds b starts as the bracket; each round takes
//     three band scores strictly inside it as candidates, evaluates F at them
//     (exact counts, fp32 exponentials, fp64 sums) and keeps the tightest
//     candidates with F >= k and F < k, until no band score lies strictly
//     inside.  lo and hi are then neighbouring values of the sorted order (or
//     a bracket end).
//  3. Confirmation in fp64: with P = sum over scores <= lo of e^{(s-lo)/t},
//     Q = sum over scores >= hi of e^{-(s-hi)/t}, m scores >= hi and
//     delta = e^{(lo-hi)/t},  F(lo) = m - delta Q/2 + P/2 and
//     F(hi) = m - Q/2 + delta P/2; when rounding in step 2 picked a neighbour
//     of the right segment, the segment moves by one value.  The root is then
//     the closed form of the segment, as after the sorted scan.
// Returns 1 (b in sm->res), 0 (the bracket failed: F at its ends in sm->res)
// or -1 (not settled within the round limits: the caller sorts instead).
// ----------------------------------------------------------------------------
// Sums of up to eight doubles over the block, fixed order; the result is
// valid in every thread.
template <int N>
__device__ __forceinline__ void block_sums(double (&v)[N], SolveSmemAll* sm) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = warp_sum_d(v[i]);
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < N; ++i) sm->sred[w][i] = v[i];
    }
    __syncthreads();
    if (w == 0) {  // the 32 warp sums, one per lane, summed by warp 0
#pragma unroll
        for (int i = 0; i < N; ++i) {
            const double a = warp_sum_d(sm->sred[lane][i]);
            if (lane == 0) sm->sres[i] = a;
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = sm->sres[i];
}

// The first attempt on a band small enough for the on-chip sort (the usual
// case): sort, scan and root in a function of its own, so that this path keeps
// its registers and its code compact, apart from the widening and narrowing
// machinery.  pre[e] holds band score e * kBlk + threadIdx.x (loaded early by
// the caller; the sort does not care where each key starts).  Returns true
// when the bracket certifies (b in sm->res).
template <int E>
__device__ void sort_preloaded(const float (&pre)[4], long long nb, SolveSmemAll* sm) {
    uint32_t key[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const long long j = (long long)e * kBlk + threadIdx.x;
        key[e] = j < nb ? to_key(pre[e]) : 0xffffffffu;
    }
    bitonic_sort_row<E, kBlk, kBlk>(key, threadIdx.x, sm->u.sort.xch);
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const long long j = (long long)threadIdx.x * E + e;
        if (j < nb) sm->u.sort.sorted[j] = from_key(key[e]);
    }
    __syncthreads();
}
__device__ __noinline__ bool first_small_band(const float (&pre)[4], long long nb, Tails tl,
                                              double k, double t, SolveSmemAll* sm) {
    if (nb <= kBlk) sort_preloaded<1>(pre, nb, sm);
    else if (nb <= 2 * kBlk) sort_preloaded<2>(pre, nb, sm);
    else sort_preloaded<4>(pre, nb, sm);
    solve_sorted_block(FloatGet{sm->u.sort.sorted}, nb, tl, k, t, &sm->ss, &sm->res);
    return sm->res.F_aL >= k && sm->res.F_aR <= k;
}

// One CTA of 1024 threads; 64 registers each (the whole register file) keeps
// the fp64 scans' spills down.
__global__ void __maxnreg__(64) solve_kernel(const float* __restrict__ r, int64_t n, int vec,
                                             double k, double t, RowState* st,
                                             float* __restrict__ band0,
                                             float* __restrict__ band1,
                                             const unsigned long long* __restrict__ bins,
                                             const float* __restrict__ sample, int m,
                                             Ladder lad, double* __restrict__ b_out,
                                             WsHeader* hdr, int split,
                                             const double* __restrict__ fold_part, int nfold,
                                             const RowBudget* __restrict__ bud) {
    pdl_wait();
    extern __shared__ __align__(16) unsigned char dsm[];
    SolveSmemAll* sm = reinterpret_cast<SolveSmemAll*>(dsm);
    if (bud != nullptr) {
        if (!bud->ok) {
            if (threadIdx.x == 0) *b_out = nan("");
            return;
        }
        k = bud->k;
        m = bud->m;
        for (int i = 0; i < kLadder; ++i) {
            lad.l[i] = bud->l[i];
            lad.h[i] = bud->h[i];
        }
    }
    phase_mark(st, 2);
    if (threadIdx.x == 0) {
        sm->bcast[2] = 0xffffffffu;
        sm->bcast[3] = 0u;
    }
    // every load this kernel needs first is issued at once: the row record,
    // the fold CTAs' records and the first 4096 band scores (read as far as
    // the row is long; only the first n_band are used)
    const float aL0 = st->a_L, aR0 = st->a_R;
    const long long nb = (long long)st->n_band;
    float pre[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int64_t j = (int64_t)e * kBlk + threadIdx.x;
        pre[e] = j < n ? __ldcg(band0 + j) : 0.f;
    }
    Tails tl;
    {
        // the fold CTAs' records, combined in CTA order: right count, tail
        // sums and the non-finite flag of the row
        double tot[4] = {0.0, 0.0, 0.0, 0.0};
        for (int i = threadIdx.x; i < nfold; i += kBlk) {
            const double2 p0 = __ldcg(reinterpret_cast<const double2*>(fold_part) + 2 * i);
            const double2 p1 = __ldcg(reinterpret_cast<const double2*>(fold_part) + 2 * i + 1);
            tot[0] += p0.x;
            tot[1] += p0.y;
            tot[2] += p1.x;
            tot[3] += p1.y;
        }
        block_sums<4>(tot, sm);
        if (threadIdx.x == 0) {
            st->cnt_R = (unsigned long long)tot[0];
            st->S_L = tot[1];
            st->S_R = tot[2];
            if (tot[3] > 0.0) {
                st->status |= kDevNonFinite;
                set_status(hdr, kDevNonFinite);
            }
        }
        if (tot[3] > 0.0) {
            if (threadIdx.x == 0) {
                st->b = nan("");
                *b_out = nan("");
            }
            return;
        }
        tl.hasL = isfinite(aL0);
        tl.aL = aL0;
        tl.SL = tot[1];
        tl.hasR = isfinite(aR0);
        tl.aR = aR0;
        tl.SR = tot[2];
        tl.cntR = tot[0];
    }
    if (nb <= kBandSortMax) {
        phase_mark(st, 19);
        const bool ok = first_small_band(pre, nb, tl, k, t, sm);
        phase_mark(st, 21);
        if (ok) {
            if (threadIdx.x == 0) {
                const double b = sm->res.b;
                st->attempts = 1;
                st->refine_levels = 0;
                st->a_L = tl.hasL ? tl.aL : -INFINITY;
                st->a_R = tl.hasR ? tl.aR : INFINITY;
                st->n_band = (unsigned long long)nb;
                st->certified = 1;
                st->b = b;
                *b_out = b;
            }
            phase_mark(st, 12);
            return;
        }
        __syncthreads();
    }
    auto select_key = [&](int64_t rank) {
        return block_select_desc(GlobalSampleKeyGet{sample}, m, rank, sm->u.sel_hist, sm->wsum,
                                 sm->bcast + 4);
    };
    bracket_attempts(r, n, vec, k, t, st, band0, band1, bins, split, m, lad, select_key, tl, nb,
                     sm, b_out, hdr);
}

// ----------------------------------------------------------------------------
// The whole bracketing pipeline for one row in one CTA (rows of moderate
// length, many rows per call): the sample is drawn straight into shared
// memory, its two order statistics are selected there, the CTA folds the row
// (four 16-byte loads per thread in flight), and the attempt loop solves the
// band with the same widening ladder as the grid pipeline.  Rows run in
// parallel, one CTA each; no kernel boundary separates the steps.
// ----------------------------------------------------------------------------
struct RowBracketSmem {
    uint32_t hist1[2048];  // sample keys by their top 11 bits
    uint32_t h2[2 * 2048];
    uint32_t wsum[64];
    uint32_t bcast[4];
};
constexpr size_t kRowBracketFixedSmem = sizeof(SolveSmemAll) + sizeof(RowBracketSmem);

__global__ void __maxnreg__(64) rowbracket_kernel(const float* __restrict__ r, int64_t ld,
                                                  int64_t n, double k0, double t, uint64_t seed,
                                                  int m0, Ladder lad0, int force_miss,
                                                  int max_attempts, int vec, RowState* rows,
                                                  float* __restrict__ band0_all,
                                                  float* __restrict__ band1_all,
                                                  double* __restrict__ b_all, WsHeader* hdr,
                                                  const RowBudget* __restrict__ budgets,
                                                  uint32_t* __restrict__ sup_flags) {
    pdl_wait();
    extern __shared__ __align__(16) unsigned char dsm[];
    SolveSmemAll* sm = reinterpret_cast<SolveSmemAll*>(dsm);
    RowBracketSmem* rb = reinterpret_cast<RowBracketSmem*>(dsm + sizeof(SolveSmemAll));
    uint32_t* keys = reinterpret_cast<uint32_t*>(dsm + kRowBracketFixedSmem);  // m words
    const int64_t row = blockIdx.x;
    const float* rr = r + row * ld;
    RowState* st = rows + row;
    float* band0 = band0_all + row * n;
    float* band1 = band1_all + row * n;
    double* b_out = b_all + row;
    for (int i = threadIdx.x; i < (int)(sizeof(RowState) / 4); i += blockDim.x)
        reinterpret_cast<uint32_t*>(st)[i] = 0u;
    if (sup_flags != nullptr && threadIdx.x == 0) sup_flags[row] = 0u;
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) rb->hist1[i] = 0u;
    __syncthreads();
    // the row's budget, sample size and ladder: shared, or its own entry
    double k = k0;
    int m = m0;
    Ladder lad = lad0;
    if (budgets != nullptr) {
        const RowBudget& bg = budgets[row];
        if (!bg.ok) {  // a budget outside (0, n): b = NaN and a status bit
            if (threadIdx.x == 0) {
                st->status |= kDevBadBudget;
                set_status(hdr, kDevBadBudget);
                st->path = LAPSUM_PATH_ROWBRACKET;
                st->b = nan("");
                *b_out = nan("");
            }
            return;
        }
        k = bg.k;
        m = bg.m;
#pragma unroll
        for (int i = 0; i < kLadder; ++i) {
            lad.l[i] = bg.l[i];
            lad.h[i] = bg.h[i];
        }
    }
    phase_mark(st, 14);
    // 1. the sample, as keys, with its level-1 histogram
    const uint64_t c0 = (uint64_t)row << 32;
    for (int s = threadIdx.x; s < m; s += blockDim.x) {
        const uint32_t key = to_key(draw_sample(rr, n, t, seed, c0, s));
        keys[s] = key;
        atomicAdd(&rb->hist1[key >> 21], 1u);
    }
    __syncthreads();
    phase_mark(st, 15);
    // 2. the bracket's order statistics
    float aR = INFINITY, aL = -INFINITY;
    {
        const int64_t ra = lad.l[0] >= 1 ? lad.l[0] : 0;
        const int64_t rbk = lad.h[0] <= m ? lad.h[0] : 0;
        uint32_t ka = 0u, kb = 0u;
        select_two_ranks(keys, m, rb->hist1, ra, rbk, rb->h2, rb->wsum, rb->bcast, &ka, &kb);
        if (ra >= 1) aR = from_key(ka);
        if (rbk >= 1) aL = from_key(kb);
    }
    phase_mark(st, 0);
    if (force_miss) {
        // a bracket above every sample value: F(a_L) < k, so it must fail
        uint32_t kmax = 0u;
        for (int s = threadIdx.x; s < m; s += blockDim.x) kmax = max(kmax, keys[s]);
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, d));
        if (threadIdx.x == 0) rb->bcast[3] = 0u;
        __syncthreads();
        if ((threadIdx.x & 31) == 0) atomicMax(&rb->bcast[3], kmax);
        __syncthreads();
        const float top = from_key(rb->bcast[3]);
        aL = top + fabsf(top) + 1.f;
        aR = INFINITY;
    }
    if (threadIdx.x == 0) {
        st->ladder_R[0] = aR;
        st->ladder_L[0] = aL;
        st->rung_L = force_miss ? -1 : 0;
        st->rung_R = 0;
        st->sample_m = m;
        st->rank_l = (int32_t)lad.l[0];
        st->rank_h = (int32_t)lad.h[0];
        st->max_attempts = max_attempts;
        st->force_miss = force_miss;
        st->path = LAPSUM_PATH_ROWBRACKET;
    }
    // 3. the fold
    Tails tl;
    long long nb = 0;
    bool bad = false;
    refold_row(rr, n, vec, aL, aR, t, band0, sm, tl, &nb, &bad);
    phase_mark(st, 16);
    if (bad) {
        if (threadIdx.x == 0) {
            st->status |= kDevNonFinite;
            set_status(hdr, kDevNonFinite);
            st->b = nan("");
            *b_out = nan("");
        }
        return;
    }
    // 4. certification, exact solve and widening
    auto select_key = [&](int64_t rank) {
        uint32_t ka = 0u, kb = 0u;
        select_two_ranks(keys, m, rb->hist1, rank, 0, rb->h2, rb->wsum, rb->bcast, &ka, &kb);
        return ka;
    };
    bracket_attempts(rr, n, vec, k, t, st, band0, band1, nullptr, 0, m, lad, select_key, tl, nb,
                     sm, b_out, hdr);
}

// Scores of the chosen histogram bin, gathered from the band by the whole
// grid (the band is large; the bin holds at most 4096 scores).
__global__ void __launch_bounds__(256) extract_kernel(const float* __restrict__ band,
                                                      RowState* st, float* __restrict__ sub) {
    pdl_wait();
    if (st->stage != 1) return;
    if (blockIdx.x == 0) phase_mark(st, 18);
    const long long nb = (long long)st->n_band;
    const BinLayout BL = make_bins(st->bin_kmin, st->bin_kmax);
    const int j = st->sub_bin;
    const long long n4 = nb >> 2;
    const float4* b4 = reinterpret_cast<const float4*>(band);
    const long long stride = (long long)gridDim.x * blockDim.x;
    const int lane = threadIdx.x & 31;
    auto take = [&](bool hit, float x) {
        const unsigned ball = __ballot_sync(0xffffffffu, hit);
        if (ball == 0u) return;
        const int leader = __ffs(ball) - 1;
        unsigned long long base = 0;
        if (lane == leader) base = atomicAdd(&st->n_sub, (unsigned long long)__popc(ball));
        base = __shfl_sync(0xffffffffu, base, leader);
        const unsigned long long pos = base + __popc(ball & ((1u << lane) - 1u));
        if (hit && pos < (unsigned long long)kBandSortMax) sub[pos] = x;
    };
    const long long trips = (n4 + stride - 1) / stride;  // same in every lane
    for (long long tr = 0; tr < trips; ++tr) {
        const long long i = tr * stride + (long long)blockIdx.x * blockDim.x + threadIdx.x;
        const bool ok = i < n4;
        const float4 v = ok ? __ldcg(b4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        take(ok && bin_of(BL, to_key(v.x)) == j, v.x);
        take(ok && bin_of(BL, to_key(v.y)) == j, v.y);
        take(ok && bin_of(BL, to_key(v.z)) == j, v.z);
        take(ok && bin_of(BL, to_key(v.w)) == j, v.w);
    }
    if (blockIdx.x == 0 && threadIdx.x < 32) {
        const long long i = (n4 << 2) + threadIdx.x;
        const bool ok = i < nb;
        const float x = ok ? band[i] : 0.f;
        take(ok && bin_of(BL, to_key(x)) == j, x);
    }
}

// Exact solve on the extracted bin with the rest of the row folded into its
// tails.  If rounding in the fixed-point histogram chose the wrong bin (its own
// end check fails), the single-CTA histogram solve walks to the right one.
__global__ void __maxnreg__(64) solve2_kernel(double k, double t, RowState* st,
                                                      float* __restrict__ band0,
                                                      float* __restrict__ sub,
                                                      const unsigned long long* __restrict__ bins,
                                                      double* __restrict__ b_out, WsHeader* hdr,
                                                      const RowBudget* __restrict__ bud) {
    pdl_wait();
    extern __shared__ __align__(16) unsigned char dsm[];
    SolveSmemAll* sm = reinterpret_cast<SolveSmemAll*>(dsm);
    if (st->stage != 1) return;
    if (bud != nullptr) k = bud->k;
    phase_mark(st, 4);
    const long long ns = (long long)st->n_sub;
    Tails s;
    s.hasL = true;
    s.aL = st->sub_aL;
    s.SL = st->sub_SL;
    s.hasR = st->sub_hasR != 0;
    s.aR = st->sub_aR;
    s.SR = st->sub_SR;
    s.cntR = st->sub_cntR;
    double b = nan("");
    bool ok = false;
    if (ns <= kWarpSortMax) {
        // a small bin (the usual case): one warp sorts it in registers and
        // solves it, with no block barrier on the way
        if (threadIdx.x < 32) {
            uint32_t key[kWarpSortMax / 32];
#pragma unroll
            for (int e = 0; e < kWarpSortMax / 32; ++e) {
                const long long j = (long long)threadIdx.x * (kWarpSortMax / 32) + e;
                key[e] = j < ns ? to_key(sub[j]) : 0xffffffffu;
            }
            bitonic_sort_row<kWarpSortMax / 32, 32, 32>(key, threadIdx.x, nullptr);
#pragma unroll
            for (int e = 0; e < kWarpSortMax / 32; ++e) {
                const long long j = (long long)threadIdx.x * (kWarpSortMax / 32) + e;
                if (j < ns) sm->u.sort.sorted[j] = from_key(key[e]);
            }
            __syncwarp();
            phase_mark(st, 13);
            solve_sorted_block<FloatGet, true>(FloatGet{sm->u.sort.sorted}, ns, s, k, t, &sm->ss,
                                               &sm->res);
        }
        __syncthreads();
        ok = sm->res.F_aL >= k && sm->res.F_aR <= k;
        b = sm->res.b;
    } else if (ns <= kBandSortMax) {
        if (ns <= kBlk) sort_band_into<1>(sub, ns, sm);
        else if (ns <= 2 * kBlk) sort_band_into<2>(sub, ns, sm);
        else sort_band_into<4>(sub, ns, sm);
        phase_mark(st, 13);
        solve_sorted_block(FloatGet{sm->u.sort.sorted}, ns, s, k, t, &sm->ss, &sm->res);
        ok = sm->res.F_aL >= k && sm->res.F_aR <= k;
        b = sm->res.b;
    }
    phase_mark(st, 5);
    if (!ok) {
        Tails tl;
        tl.hasL = isfinite(st->a_L);
        tl.aL = st->a_L;
        tl.SL = st->S_L;
        tl.hasR = isfinite(st->a_R);
        tl.aR = st->a_R;
        tl.SR = st->S_R;
        tl.cntR = (double)st->cnt_R;
        const long long nb = (long long)st->n_band;
        const BinLayout BL = make_bins(st->bin_kmin, st->bin_kmax);
        int v = solve_with_bins(band0, nb, bins, BL, tl, k, t, sm, nullptr);
        if (v < 0) {
            // a neighbouring bin too full for the on-chip sort: exact narrowing,
            // with the extracted bin's buffer as the second band
            int levels = 0;
            v = solve_exact(band0, sub, nb, tl, k, t, sm, &levels);
            if (threadIdx.x == 0) st->refine_levels = levels;
        }
        b = v == 1 ? sm->res.b : nan("");
        ok = v == 1;
    }
    if (threadIdx.x == 0) {
        st->stage = 0;
        if (!ok) {
            st->status |= kDevBracketExhausted;
            st->certified = 0;
            set_status(hdr, kDevBracketExhausted);
        }
        st->b = b;
        *b_out = b;
    }
}

// ----------------------------------------------------------------------------
// Pieces of the bracketing pipeline for one row split over several devices
// (each holds a contiguous shard; the host exchanges the small results
// between them).  The sample is the single-device row's sample: draw s is
// taken by the shard that holds its index.
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256) shard_sample_kernel(const float* __restrict__ r,
                                                           int64_t n_shard, int64_t offset,
                                                           int64_t n, double t, uint64_t seed,
                                                           int m, float* __restrict__ y) {
    const int s = blockIdx.x * 256 + threadIdx.x;
    if (s >= m) return;
    const int64_t I = sample_index(seed, 0ull, s, n);
    const int64_t j = I - offset;
    y[s] = (j >= 0 && j < n_shard) ? __ldg(r + j) + sample_noise(seed, 0ull, s, t) : 0.f;
}

// The two order statistics of a complete sample (ranks counted from the top;
// 0 = open end): ends[0] = a_L (rank_h), ends[1] = a_R (rank_l).
__global__ void __launch_bounds__(kBlk) sample_bracket_kernel(const float* __restrict__ y, int m,
                                                              int64_t rank_l, int64_t rank_h,
                                                              float* __restrict__ ends) {
    __shared__ uint32_t hist[2048];
    __shared__ uint32_t wsum[32];
    __shared__ uint32_t bcast[4];
    float aL = -INFINITY, aR = INFINITY;
    if (rank_h >= 1 && rank_h <= m)
        aL = from_key(block_select_desc(GlobalSampleKeyGet{y}, m, rank_h, hist, wsum, bcast));
    if (rank_l >= 1 && rank_l <= m)
        aR = from_key(block_select_desc(GlobalSampleKeyGet{y}, m, rank_l, hist, wsum, bcast));
    if (threadIdx.x == 0) {
        ends[0] = aL;
        ends[1] = aR;
    }
}

__global__ void shard_fold_setup_kernel(const float* __restrict__ ends, RowState* st) {
    for (int i = 0; i < (int)(sizeof(RowState) / 4); ++i) reinterpret_cast<uint32_t*>(st)[i] = 0u;
    st->a_L = ends[0];
    st->a_R = ends[1];
}

// The fold CTAs' records combined in CTA order into rec = (right count, left
// sum, right sum, non-finite flag, band size).
__global__ void __launch_bounds__(kBlk) shard_fold_records_kernel(
    const double* __restrict__ part, int nfold, const RowState* st, double* __restrict__ rec) {
    extern __shared__ __align__(16) unsigned char dsm[];
    SolveSmemAll* sm = reinterpret_cast<SolveSmemAll*>(dsm);
    double tot[4] = {0.0, 0.0, 0.0, 0.0};
    for (int i = threadIdx.x; i < nfold; i += kBlk) {
        tot[0] += part[4 * i];
        tot[1] += part[4 * i + 1];
        tot[2] += part[4 * i + 2];
        tot[3] += part[4 * i + 3];
    }
    block_sums<4>(tot, sm);
    if (threadIdx.x == 0) {
        rec[0] = tot[0];
        rec[1] = tot[1];
        rec[2] = tot[2];
        rec[3] = tot[3];
        rec[4] = (double)st->n_band;
    }
}

// The exact solve on the gathered band: the shards' records are combined in
// shard order into the tails, the shards' band segments are copied into one
// array, and the band is solved with the tails as virtual anchors (sorted on
// chip, or narrowed by exact histogram levels when large).  out = (b, F(a_L),
// F(a_R), certified).
__global__ void __maxnreg__(64) shard_band_solve_kernel(
    const float* __restrict__ bands, int64_t stride, const double* __restrict__ recs, int world,
    const float* __restrict__ ends, double k, double t, float* __restrict__ cur,
    float* __restrict__ nxt, double* __restrict__ out) {
    extern __shared__ __align__(16) unsigned char dsm[];
    SolveSmemAll* sm = reinterpret_cast<SolveSmemAll*>(dsm);
    Tails tl;
    tl.aL = ends[0];
    tl.aR = ends[1];
    tl.hasL = isfinite(tl.aL);
    tl.hasR = isfinite(tl.aR);
    double cr = 0.0, sl = 0.0, sr = 0.0, bad = 0.0;
    long long nb = 0;
    for (int w = 0; w < world; ++w) {
        cr += recs[5 * w];
        sl += recs[5 * w + 1];
        sr += recs[5 * w + 2];
        bad += recs[5 * w + 3];
        const long long nw = (long long)recs[5 * w + 4];
        for (long long j = threadIdx.x; j < nw; j += kBlk) cur[nb + j] = bands[w * stride + j];
        nb += nw;
    }
    tl.cntR = cr;
    tl.SL = sl;
    tl.SR = sr;
    __syncthreads();
    if (bad > 0.0) {
        if (threadIdx.x == 0) {
            out[0] = nan("");
            out[1] = INFINITY;
            out[2] = -INFINITY;
            out[3] = 1.0;  // settled: the row has a non-finite score
        }
        return;
    }
    int certified = 1;
    if (nb <= kBandSortMax) {
        solve_small_band(cur, nb, tl, k, t, sm);
        certified = sm->res.F_aL >= k && sm->res.F_aR <= k;
    } else {
        int levels = 0;
        certified = solve_exact(cur, nxt, nb, tl, k, t, sm, &levels) == 1;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        out[0] = certified ? sm->res.b : nan("");
        out[1] = sm->res.F_aL;
        out[2] = sm->res.F_aR;
        out[3] = certified ? 1.0 : 0.0;
    }
}

}  // namespace

cudaError_t launch_shard_sample(const float* r, int64_t n_shard, int64_t offset, int64_t n,
                                double t, uint64_t seed, int m, float* y, cudaStream_t st) {
    shard_sample_kernel<<<(unsigned)((m + 255) / 256), 256, 0, st>>>(r, n_shard, offset, n, t, seed,
                                                                   m, y);
    return cudaGetLastError();
}

cudaError_t launch_sample_bracket(const float* y, int m, int64_t rank_l, int64_t rank_h,
                                  float* ends, cudaStream_t st) {
    sample_bracket_kernel<<<1, kBlk, 0, st>>>(y, m, rank_l, rank_h, ends);
    return cudaGetLastError();
}

size_t shard_fold_workspace_bytes() {
    return 512 + (size_t)kFoldGridMaxShard * 4 * sizeof(double);
}

cudaError_t launch_shard_fold(const float* r, int64_t n_shard, const float* ends, double t,
                              double* rec, float* band, void* ws, cudaStream_t st) {
    RowState* rs = static_cast<RowState*>(ws);
    double* part = reinterpret_cast<double*>(static_cast<char*>(ws) + 512);
    int grid = bracket_fold_grid();
    if (grid > kFoldGridMaxShard) grid = kFoldGridMaxShard;
    static std::atomic<unsigned long long> attr_devices{0ull};
    once_per_device(attr_devices, [&]() {
        cudaFuncSetAttribute(fold_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kFoldDynSmem);
        cudaFuncSetAttribute(shard_fold_records_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(SolveSmemAll));
        cudaFuncSetAttribute(shard_band_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(SolveSmemAll));
    });
    shard_fold_setup_kernel<<<1, 1, 0, st>>>(ends, rs);
    const int vec = ((reinterpret_cast<uintptr_t>(r) & 15u) == 0) ? 1 : 0;
    fold_kernel<<<grid, kFoldThreads, kFoldDynSmem, st>>>(r, n_shard, t, rs, band, nullptr, part,
                                                          vec, 0);
    shard_fold_records_kernel<<<1, kBlk, sizeof(SolveSmemAll), st>>>(part, grid, rs, rec);
    return cudaGetLastError();
}

cudaError_t launch_shard_band_solve(const float* bands, int64_t stride, const double* recs,
                                    int world, const float* ends, double k, double t, float* cur,
                                    float* nxt, double* out, cudaStream_t st) {
    static std::atomic<unsigned long long> attr_devices{0ull};
    once_per_device(attr_devices, [&]() {
        cudaFuncSetAttribute(shard_band_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(SolveSmemAll));
    });
    shard_band_solve_kernel<<<1, kBlk, sizeof(SolveSmemAll), st>>>(bands, stride, recs, world,
                                                                  ends, k, t, cur, nxt, out);
    return cudaGetLastError();
}

size_t rowbracket_smem(int m) { return kRowBracketFixedSmem + (size_t)m * sizeof(uint32_t); }

cudaError_t launch_rowbracket(const float* r, int64_t ld, int64_t B, int64_t n, double k, double t,
                              uint64_t seed, int m, int64_t rank_l[kLadder],
                              int64_t rank_h[kLadder], int flags, RowState* rows, float* band0,
                              float* band1, double* b, WsHeader* hdr, int vec, cudaStream_t st,
                              const RowBudget* budgets, uint32_t* sup_flags) {
    static std::atomic<unsigned long long> attr_devices{0ull};
    once_per_device(attr_devices, [&]() {
        cudaFuncSetAttribute(rowbracket_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)rowbracket_smem(kSampleMax));
    });
    Ladder lad;
    for (int i = 0; i < kLadder; ++i) {
        lad.l[i] = rank_l[i];
        lad.h[i] = rank_h[i];
    }
    const int force_miss = (flags & LAPSUM_FLAG_FORCE_MISS) ? 1 : 0;
    const int max_attempts = (flags & LAPSUM_FLAG_NO_RETRY) ? 1 : kMaxAttempts;
    ProfScope ps_("rowbracket", st);
    launch_pdl(rowbracket_kernel, dim3((unsigned)B), dim3(kBlk), rowbracket_smem(m), st, 
        r, ld, n, k, t, seed, m, lad, force_miss, max_attempts, vec, rows, band0, band1, b, hdr,
        budgets, sup_flags);
    return cudaGetLastError();
}

namespace {
// One warp per row: the sample size (4096 doubled up to 32768 while below 64/q)
// and the binomial order-statistic ranks of the bracket (the largest l with
// P(C < l) <= alpha and the smallest h with P(C >= h) <= alpha, C ~ Bin(m, q),
// q = k/n), then the ladder: each end moved out by 4x per rung, the last open.
// The tails are summed 32 terms at a time with a warp prefix sum, in the same
// order as a sequential sum up from 0 and down from mq + 40 sd + 64.
__global__ void __launch_bounds__(256) row_budget_kernel(const double* __restrict__ k_rows,
                                                         int64_t B, int64_t n, double alpha,
                                                         RowBudget* __restrict__ out) {
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= B) return;  // the whole warp
    const double k = k_rows[row];
    RowBudget* o = out + row;
    if (!(k > 0.0 && k < (double)n)) {
        if (lane == 0) {
            o->k = k;
            o->m = 0;
            o->ok = 0;
        }
        return;
    }
    const double q = k / (double)n;
    int m = 4096;
    while (m < kSampleMax && (double)m < 64.0 / q) m <<= 1;
    const double lgm = lgamma((double)m + 1.0), lq = log(q), l1q = log1p(-q);
    auto pmf = [&](int64_t c) {
        return exp(lgm - lgamma((double)c + 1.0) - lgamma((double)(m - c) + 1.0) +
                   (double)c * lq + (double)(m - c) * l1q);
    };
    auto inclusive = [&](double v) {
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const double u = __shfl_up_sync(0xffffffffu, v, d);
            if (lane >= d) v += u;
        }
        return v;
    };
    // lower tail: lo = the first c whose cumulative probability exceeds alpha
    int64_t lo = m + 1;
    double carry = 0.0;
    for (int64_t base = 0; base <= m; base += 32) {
        const int64_t c = base + lane;
        const double cdf = carry + inclusive(c <= m ? pmf(c) : 0.0);
        const unsigned over = __ballot_sync(0xffffffffu, c <= m && cdf > alpha);
        if (over != 0u) {
            lo = base + (__ffs(over) - 1);
            break;
        }
        carry = __shfl_sync(0xffffffffu, cdf, 31);
    }
    // upper tail, summed down from top: hi = one above the first c whose
    // cumulative probability exceeds alpha (0 when none does)
    const double mean = (double)m * q, sd = sqrt((double)m * q * (1.0 - q));
    int64_t top = (int64_t)ceil(mean + 40.0 * sd + 64.0);
    if (top > m) top = m;
    int64_t hi = 0;
    carry = 0.0;
    for (int64_t base = 0; base <= top; base += 32) {
        const int64_t c = top - base - lane;
        const double sf = carry + inclusive(c >= 0 ? pmf(c) : 0.0);
        const unsigned over = __ballot_sync(0xffffffffu, c >= 0 && sf > alpha);
        if (over != 0u) {
            hi = top - base - (__ffs(over) - 1) + 1;
            break;
        }
        carry = __shfl_sync(0xffffffffu, sf, 31);
    }
    if (hi > m) hi = m + 1;
    if (lane == 0) {
        o->k = k;
        o->m = m;
        o->ok = 1;
        for (int i = 0; i < kLadder - 1; ++i) {
            o->l[i] = lo >> (2 * i);
            const int64_t h = hi << (2 * i);
            o->h[i] = h > m ? (int64_t)m + 1 : h;
        }
        o->l[kLadder - 1] = 0;
        o->h[kLadder - 1] = (int64_t)m + 1;
    }
}
}  // namespace

cudaError_t launch_row_budgets(const double* k_rows, int64_t B, int64_t n, double alpha,
                               RowBudget* out, cudaStream_t st) {
    ProfScope ps_("row_budgets", st);
    row_budget_kernel<<<(unsigned)((B + 7) / 8), 256, 0, st>>>(k_rows, B, n, alpha, out);
    return cudaGetLastError();
}

int bracket_fold_grid() {
    // one resident wave of fold CTAs, per device
    constexpr int kMaxDevices = 64;
    static std::atomic<int> per_sm[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    const bool cached = dev >= 0 && dev < kMaxDevices;
    int per = cached ? per_sm[dev].load(std::memory_order_relaxed) : 0;
    if (per == 0) {
        cudaFuncSetAttribute(fold_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kFoldDynSmem);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, fold_kernel, kFoldThreads,
                                                      kFoldDynSmem);
        if (per < 1) per = 1;
        if (cached) per_sm[dev].store(per, std::memory_order_relaxed);
    }
    return device_sm_count() * per;
}

cudaError_t launch_bracket_row(const float* r_row, int64_t n, double k, double t, uint64_t seed,
                               int64_t row, int m, int64_t rank_l[kLadder],
                               int64_t rank_h[kLadder], int flags, const BracketBuffers& buf,
                               RowState* st_row, double* b_out, WsHeader* hdr,
                               uint32_t* sup_flag, const RowBudget* bud, cudaStream_t st) {
    // dynamic shared memory limits, set once per device (they belong to the
    // device's copy of the module)
    static std::atomic<unsigned long long> attr_devices{0ull};
    const size_t solve_smem = sizeof(SolveSmemAll);
    const size_t sample_smem = ((size_t)kSampleMax + 2 * 2048) * sizeof(uint32_t);
    once_per_device(attr_devices, [&]() {
        cudaFuncSetAttribute(solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)solve_smem);
        cudaFuncSetAttribute(solve2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)solve_smem);
        cudaFuncSetAttribute(sample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sample_smem);
        cudaFuncSetAttribute(fold_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kFoldDynSmem);
    });
    Ladder lad;
    for (int i = 0; i < kLadder; ++i) {
        lad.l[i] = rank_l[i];
        lad.h[i] = rank_h[i];
    }
    const int force_miss = (flags & LAPSUM_FLAG_FORCE_MISS) ? 1 : 0;
    const int max_attempts = (flags & LAPSUM_FLAG_NO_RETRY) ? 1 : kMaxAttempts;
    float* sample = buf.sample + row * (int64_t)kSampleMax;
    const uint64_t c0 = (uint64_t)row << 32;
    // With a per-row budget (bud) the sample size and ranks are on the device:
    // the sample grid covers the largest sample, and the split solve kernels
    // are always launched (they return at once when the band was small).
    const int sgrid = bud != nullptr ? kSampleMax / kBlk : (m + kBlk - 1) / kBlk;
    // The band of the first bracket holds about n (h - l) / m scores.  When it
    // should fit the on-chip sort with some room to spare, the solve kernel
    // finishes by itself, the fold builds no band histogram, and the grid-wide
    // extraction and second solve are not launched; a band that turns out
    // larger is still solved exactly, inside the solve kernel.
    const int64_t lo_rank = rank_l[0] > 0 ? rank_l[0] : 0;
    const int64_t hi_rank = rank_h[0] < m ? rank_h[0] : m;
    const double expect_band = (double)n * (double)(hi_rank - lo_rank) / (double)m;
    const int split =
        ((flags & LAPSUM_FLAG_ONE_CTA_SOLVE) == 0 &&
         (bud != nullptr || force_miss || expect_band > 0.75 * kBandSortMax))
            ? 1
            : 0;
    // the fold builds the band histogram for the split solve, and for the
    // one-CTA histogram solve when that is asked for
    const int hist = (split || (flags & LAPSUM_FLAG_ONE_CTA_SOLVE) != 0) ? 1 : 0;
    // both bracket ranks among each sample CTA's top_h keys: candidate selection
    const int64_t need = rank_h[0] <= m ? rank_h[0] : (rank_l[0] >= 1 ? rank_l[0] : 0);
    const int top_h = (bud == nullptr && need >= 1 && need <= kBlk &&
                       (int64_t)sgrid * need <= 4 * kBlk)
                          ? (int)need
                          : 0;
    const size_t smem = (bud == nullptr && top_h > 0) ? (size_t)4 * kBlk * sizeof(uint32_t)
                                                      : sample_smem;
    {
        ProfScope ps_("bracket_sample", st);
        launch_pdl(sample_kernel, dim3(sgrid), dim3(kBlk), smem, st, r_row, n, t, seed, c0, m,
                   lad, force_miss, max_attempts, sample, buf.bins, buf.ticket + 2,
                   buf.ticket + 1, st_row, top_h, buf.cand, hist, sup_flag, bud, hdr);
    }
    const int vec = ((reinterpret_cast<uintptr_t>(r_row) & 15u) == 0) ? 1 : 0;
    {
        ProfScope ps_("bracket_fold", st);
        launch_pdl(fold_kernel, dim3(buf.fold_grid), dim3(kFoldThreads), kFoldDynSmem, st, r_row,
                   n, t, st_row, buf.band[0], buf.bins, buf.fold_part, vec, hist);
    }
    {
        ProfScope ps_("bracket_solve", st);
        launch_pdl(solve_kernel, dim3(1), dim3(kBlk), solve_smem, st, r_row, n, vec, k, t, st_row,
                   buf.band[0], buf.band[1], hist ? buf.bins : nullptr, sample, m, lad, b_out,
                   hdr, split, (const double*)buf.fold_part, buf.fold_grid, bud);
    }
    if (split) {
        {
            ProfScope ps_("bracket_extract", st);
            const int xgrid = bracket_fold_grid() / 2 > 0 ? bracket_fold_grid() / 2 : 1;
            launch_pdl(extract_kernel, dim3(xgrid), dim3(256), 0, st, buf.band[0], st_row, buf.band[1]);
        }
        {
            ProfScope ps_("bracket_solve2", st);
            launch_pdl(solve2_kernel, dim3(1), dim3(kBlk), solve_smem, st, k, t, st_row,
                       buf.band[0], buf.band[1], buf.bins, b_out, hdr, bud);
        }
    }
    return cudaGetLastError();
}

}  // namespace lapsum
