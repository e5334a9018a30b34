// Block-level solve of the budget equation over a sorted array with optional
// folded tails: the stable prefix/suffix scan, the index lookup of the
// balancing segment and the closed-form root ("Fast LapSum: Exact
// Differentiable Top-k at Million Scale", gist.science explainer pages,
// section 2.2, full-sort solver; the tails implement step 3 of the bracketing
// pipeline, the exact solve on the middle band).
//
// Sorted scores s_0 <= ... <= s_{nb-1} may sit between two virtual anchors:
// a left anchor aL carrying SL = sum_{r < aL} e^{(r - aL)/t} (the folded left
// tail) and a right anchor aR carrying SR = sum_{r >= aR} e^{-(r - aR)/t} and
// cntR scores (the folded right tail).  With gap factors gap(j) between
// neighbours (the anchors count as positions -1 and nb), the prefix and
// suffix weights obey P_j = 1 + gap(j) P_{j-1} (P_{-1} = SL) and
// Q_j = 1 + gap(j+1) Q_{j+1} (Q_nb = SR), and the threshold curve is
//     F(s_j) = cntR + (nb - j) - Q_j / 2 + (P_j - 1) / 2.
// The balancing segment is found with counts of F(s_j) >= k taken over thread
// chunks, then recursively over 32 warp lanes, so no per-element storage is
// needed at any n.
#pragma once

#include "lapsum_common.cuh"

namespace lapsum {

struct Tails {
    bool hasL;
    float aL;
    double SL;
    bool hasR;
    float aR;
    double SR;
    double cntR;
};

struct SolveResult {
    double b;
    double F_aL, F_aR;  // budget sum at the bracket ends (+inf / -inf for open ends)
    long long jstar;    // number of sorted band scores with F(s_j) >= k
};

struct SolveScratch {
    Aff wf[32], wb[32];
    double d[8];
    long long ll[4];
};

// HOT: a long array (a whole sorted row): factors are taken with the inlined
// exponential, and each thread's chunk is summarised in closed form (see
// solve_sorted_block); otherwise one out-of-line copy of the exponential
// serves the single-CTA band solves.
template <class Get, bool HOT = false>
struct GapFn {
    Get get;
    long long nb;
    Tails tl;
    double inv_t;
    __device__ __forceinline__ double factor(float lo, float hi) const {
        return HOT ? gap_factor(lo, hi, inv_t) : gap_factor_cold(lo, hi, inv_t);
    }
    // factor between positions j-1 and j (anchors at -1 and nb)
    __device__ __forceinline__ double operator()(long long j) const {
        if (j <= 0) return (j == 0 && tl.hasL && nb > 0) ? factor(tl.aL, get(0)) : 0.0;
        if (j >= nb) return (j == nb && tl.hasR) ? factor(get(nb - 1), tl.aR) : 0.0;
        return factor(get(j - 1), get(j));
    }
};

// One warp narrows [lo, hi) -- whose first element satisfies F >= k -- to the
// last element with F >= k.  P_before = P_{lo-1}, Q_after = Q_hi.  Lane 0
// returns j* and the anchor weights through the out-parameters.
template <class Get, bool HOT>
__device__ void warp_find_crossing(const GapFn<Get, HOT>& gap, long long lo, long long hi,
                                   double P_before, double Q_after, double k, long long* jstar,
                                   double* P_left, double* Q_right) {
    const int lane = threadIdx.x & 31;
    const long long nb = gap.nb;
    const double cntR = gap.tl.cntR;
    while (hi - lo > 32) {
        const long long sc = (hi - lo + 31) / 32;
        const long long l0 = min(hi, lo + lane * sc), l1 = min(hi, l0 + sc);
        Aff af = aff_id(), ab = aff_id();
        double g_first = 0.0;
        for (long long j = l0; j < l1; ++j) {
            const double gj = gap(j);
            if (j == l0) g_first = gj;
            af = aff_then(af, Aff{gj, 1.0});
            if (j > l0) ab = aff_then(Aff{gj, 1.0}, ab);
        }
        if (l1 > l0) ab = aff_then(Aff{gap(l1), 1.0}, ab);
        Aff ef = shfl_up_aff(warp_scan_fwd(af, lane), 1);
        Aff eb = shfl_down_aff(warp_scan_bwd(ab, lane), 1);
        if (lane == 0) ef = aff_id();
        if (lane == 31) eb = aff_id();
        const double pb = fma(ef.a, P_before, ef.c);   // P_{l0-1}
        const double qa = fma(eb.a, Q_after, eb.c);    // Q_{l1}
        const double P0 = fma(g_first, pb, 1.0);
        const double Q0 = fma(ab.a, qa, ab.c);
        const double G0 = cntR + (double)(nb - l0) - 0.5 * Q0 + 0.5 * (P0 - 1.0);
        const unsigned ball = __ballot_sync(0xffffffffu, l0 < l1 && G0 >= k);
        const int L = max(0, __popc(ball) - 1);
        lo = __shfl_sync(0xffffffffu, l0, L);
        hi = __shfl_sync(0xffffffffu, l1, L);
        P_before = __shfl_sync(0xffffffffu, pb, L);
        Q_after = __shfl_sync(0xffffffffu, qa, L);
    }
    // At most 32 elements: one per lane.
    const long long j = lo + lane;
    const bool valid = j < hi;
    const double gj = valid ? gap(j) : 1.0;
    const double gn = valid ? gap(j + 1) : 1.0;
    const Aff mf = valid ? Aff{gj, 1.0} : aff_id();
    const Aff mb = valid ? Aff{gn, 1.0} : aff_id();
    const Aff inf_ = warp_scan_fwd(mf, lane);
    const Aff inb = warp_scan_bwd(mb, lane);
    const double Pj = fma(inf_.a, P_before, inf_.c);
    const double Qj = fma(inb.a, Q_after, inb.c);
    const double Gj = cntR + (double)(nb - j) - 0.5 * Qj + 0.5 * (Pj - 1.0);
    const unsigned ball = __ballot_sync(0xffffffffu, valid && Gj >= k);
    const int c = __popc(ball);  // >= 1 by the invariant on lo
    const long long js = lo + c;
    const double Pl = __shfl_sync(0xffffffffu, Pj, max(0, c - 1));
    const double Qr_in = __shfl_sync(0xffffffffu, Qj, min(31, c));
    if (lane == 0) {
        *jstar = js;
        *P_left = Pl;
        *Q_right = (js < hi) ? Qr_in : Q_after;  // Q_hi when the right anchor opens the next range
    }
}

// Team barrier and count: the whole block, or (WARP) a single warp.
template <bool WARP>
__device__ __forceinline__ void team_sync() {
    if (WARP) __syncwarp();
    else __syncthreads();
}
template <bool WARP>
__device__ __forceinline__ int team_count(bool pred) {
    if (WARP) return __popc(__ballot_sync(0xffffffffu, pred));
    return __syncthreads_count(pred);
}

// Whole-team solve: every thread of the block (or, with WARP, every lane of
// the one calling warp) must call it; the result is valid in `out` for every
// thread of the team after return.  The warp form serves small bands without
// any block barrier.
template <class Get, bool WARP = false, bool HOT = false>
__device__ void solve_sorted_block(Get get, long long nb, const Tails& tl, double k, double t,
                                   SolveScratch* sm, SolveResult* out) {
    const int tid = WARP ? (int)(threadIdx.x & 31) : (int)threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int nthreads = WARP ? 32 : (int)blockDim.x, nwarps = nthreads >> 5;
    GapFn<Get, HOT> gap{get, nb, tl, 1.0 / t};
    const double P_start = tl.hasL ? tl.SL : 0.0;
    const double Q_end = tl.hasR ? tl.SR : 0.0;

    if (nb == 0) {
        if (tid < 32) {  // one warp takes the root
            const double b = segment_root(tl.hasL, tl.aL, tl.SL, tl.hasR, tl.aR, tl.SR,
                                          tl.cntR - k, t);
            if (tid == 0) {
                out->jstar = 0;
                out->b = b;
                const double lnw =
                    (tl.hasL && tl.hasR) ? ((double)tl.aL - (double)tl.aR) / t : -INFINITY;
                out->F_aL = tl.hasL ? tl.cntR - 0.5 * tl.SR * cold_exp(lnw) + 0.5 * tl.SL
                                    : INFINITY;
                out->F_aR = tl.hasR ? tl.cntR - 0.5 * tl.SR + 0.5 * tl.SL * cold_exp(lnw)
                                    : -INFINITY;
            }
        }
        team_sync<WARP>();
        return;
    }

    const long long chunk = (nb + nthreads - 1) / nthreads;
    const long long lo = min(nb, (long long)tid * chunk), hi = min(nb, lo + chunk);
    const bool valid = lo < hi;
    Aff af = aff_id(), ab = aff_id();
    double g_first = 0.0;
    if constexpr (HOT) {
        // A long chunk's maps in closed form: the product of its gap factors
        // telescopes, P_{hi-1} = gap(lo) e^{(s_lo - s_{hi-1})/t} P_{lo-1}
        // + sum_{i in chunk} e^{(s_i - s_{hi-1})/t}, and likewise Q_lo from
        // Q_hi; the sums take unbiased fp32 exponentials (every term at most
        // 1) added in fp64, so three fp64 exponentials serve the whole chunk
        // and no rounding compounds along it.
        if (valid) {
            const float s_first = get(lo), s_last = get(hi - 1);
            const double it = 1.0 / t;
            double cf = 0.0, cb = 0.0;
            for (long long j0 = lo; j0 < hi; j0 += 16) {
                // the loads of 16 positions first, so that they overlap
                float xs[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) xs[u] = j0 + u < hi ? get(j0 + u) : s_last;
                float cf8 = 0.f, cb8 = 0.f;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    if (j0 + u < hi) {
                        // arguments in fp64: an fp32 difference of scores in
                        // different binades rounds the same way for all of them
                        cf8 += exp_neg((float)(((double)s_last - (double)xs[u]) * it));
                        cb8 += exp_neg((float)(((double)xs[u] - (double)s_first) * it));
                    }
                }
                cf += (double)cf8;
                cb += (double)cb8;
            }
            const double span = exp(((double)s_first - (double)s_last) / t);
            g_first = gap(lo);
            af = Aff{g_first * span, cf};
            ab = Aff{gap(hi) * span, cb};
        }
    } else {
        for (long long j = lo; j < hi; ++j) {
            const double gj = gap(j);
            if (j == lo) g_first = gj;
            af = aff_then(af, Aff{gj, 1.0});
            if (j > lo) ab = aff_then(Aff{gj, 1.0}, ab);
        }
        if (valid) ab = aff_then(Aff{gap(hi), 1.0}, ab);
    }

    const Aff inc_f = warp_scan_fwd(af, lane);
    const Aff inc_b = warp_scan_bwd(ab, lane);
    Aff ef = shfl_up_aff(inc_f, 1);
    Aff eb = shfl_down_aff(inc_b, 1);
    if (lane == 0) ef = aff_id();
    if (lane == 31) eb = aff_id();
    if (!WARP && nwarps > 1) {
        // the warps' aggregates, scanned by warp 0 (both directions)
        if (lane == 31) sm->wf[warp] = inc_f;
        if (lane == 0) sm->wb[warp] = inc_b;
        team_sync<WARP>();
        if (warp == 0) {
            const Aff a = lane < nwarps ? sm->wf[lane] : aff_id();
            const Aff c = lane < nwarps ? sm->wb[lane] : aff_id();
            const Aff sa = warp_scan_fwd(a, lane);
            const Aff sc = warp_scan_bwd(c, lane);
            Aff ea = shfl_up_aff(sa, 1);
            Aff ec = shfl_down_aff(sc, 1);
            if (lane == 0) ea = aff_id();
            if (lane == 31) ec = aff_id();
            if (lane < nwarps) {
                sm->wf[lane] = ea;
                sm->wb[lane] = ec;
            }
        }
        team_sync<WARP>();
        ef = aff_then(sm->wf[warp], ef);
        eb = aff_then(sm->wb[warp], eb);
    }
    const double P_before = fma(ef.a, P_start, ef.c);  // P_{lo-1}
    const double Q_after = fma(eb.a, Q_end, eb.c);     // Q_hi
    const double P_lo = fma(g_first, P_before, 1.0);
    const double Q_lo = fma(ab.a, Q_after, ab.c);
    const double G_lo = tl.cntR + (double)(nb - lo) - 0.5 * Q_lo + 0.5 * (P_lo - 1.0);
    const double P_end = fma(af.a, P_before, af.c);    // P_{hi-1}
    const int count = team_count<WARP>(valid && G_lo >= k);
    const int T = count - 1;
    if (tid == 0) sm->d[0] = Q_lo;                      // Q_0
    if (valid && hi == nb) sm->d[1] = P_end;            // P_{nb-1}
    if (tid == T) {
        sm->ll[0] = lo;
        sm->ll[1] = hi;
        sm->d[2] = P_before;
        sm->d[3] = Q_after;
    }
    team_sync<WARP>();

    if (count > 0 && warp == 0) {
        long long js;
        double Pl, Qr;
        warp_find_crossing(gap, sm->ll[0], sm->ll[1], sm->d[2], sm->d[3], k, &js, &Pl, &Qr);
        if (lane == 0) {
            sm->ll[2] = js;
            sm->d[4] = Pl;
            sm->d[5] = Qr;
        }
    }
    team_sync<WARP>();
    if (tid < 32) {  // one warp takes the root; lane 0 writes the result
        double b;
        long long js;
        if (count == 0) {
            js = 0;
            b = segment_root(tl.hasL, tl.aL, tl.hasL ? tl.SL : 0.0, true, get(0), sm->d[0],
                             tl.cntR + (double)nb - k, t);
        } else {
            js = sm->ll[2];
            const bool hasR = js < nb || tl.hasR;
            const double sR = js < nb ? (double)get(js) : (double)tl.aR;
            const double Ah = js < nb ? sm->d[5] : (tl.hasR ? tl.SR : 0.0);
            b = segment_root(true, get(js - 1), sm->d[4], hasR, sR, Ah,
                             tl.cntR + (double)(nb - js) - k, t);
        }
        // the end gap factors, one lane each
        const double g_end = lane == 1 ? gap(nb) : (lane == 0 ? gap(0) : 0.0);
        const double g_nb = __shfl_sync(0xffffffffu, g_end, 1);
        if (lane == 0) {
            out->b = b;
            out->jstar = js;
            const double Q0 = sm->d[0], Pl = sm->d[1];
            out->F_aL = tl.hasL ? tl.cntR + (double)nb - 0.5 * g_end * Q0 + 0.5 * tl.SL
                                : INFINITY;
            out->F_aR = tl.hasR ? tl.cntR - 0.5 * tl.SR + 0.5 * g_nb * Pl : -INFINITY;
        }
    }
    team_sync<WARP>();
}

}  // namespace lapsum
