// Shared device-side building blocks of the Fast LapSum kernels (sm_100a).
//
// Method: "Fast LapSum: Exact Differentiable Top-k at Million Scale"
// (gist.science explainer pages).  Section 2.1 defines p_i = sigma((r_i-b)/t)
// with sigma the Laplace(0,1) CDF and sum_i p_i = k; section 2.2 solves for b
// after a sort with one stable prefix/suffix scan, an index lookup and a
// closed-form root in the balancing segment.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/lapsum.h"

namespace lapsum {

// ---------------------------------------------------------------------------
// Device status bits (sticky, OR-ed into the workspace header).
// ---------------------------------------------------------------------------
enum : uint32_t {
    kDevNonFinite = 1u << 0,
    kDevBracketExhausted = 1u << 1,
    kDevBadBudget = 1u << 2,  // a per-row budget outside (0, n)
    kDevWaitTimeout = 1u << 3,  // a bounded wait on another CTA ran out (results invalid)
};

constexpr int kMaxAttempts = 7;     // 1 + 3 widenings per side; the last rungs are open
constexpr int kLadder = 4;          // rungs per side: ranks r, 4r, 16r, open
constexpr int kBandSortMax = 4096;  // band solved on chip once it is this small
constexpr int kRefineBins = 2048;   // histogram bins per narrowing level

// Workspace header (first 256 bytes of the workspace).
struct WsHeader {
    uint32_t status;       // sticky device status bits
    uint32_t last_path;    // path of the last forward call
    int64_t last_B, last_n;
    uint32_t fold_ticket;  // last-block counters (reset by the block that wins them)
    uint32_t emit_ticket;
    uint32_t bwd_ticket;
    uint32_t pad0;
    uint64_t reserved[27];
};
static_assert(sizeof(WsHeader) == 256, "header is one 256-byte slot");

// Per-row record (radix and bracketing paths), 512 bytes.
struct RowState {
    double b;
    double sum_f;
    double S_L, S_R;      // tail sums of the current bracket
    double R;             // backward ratio sum v f / sum f
    double mu;            // backward shift: min |x|
    float a_L, a_R;       // current bracket
    unsigned long long cnt_R;   // scores >= a_R
    unsigned long long n_band;  // scores in [a_L, a_R) (fold counter)
    int32_t path;
    int32_t attempts;
    int32_t sample_m;
    int32_t rank_l, rank_h;
    int32_t refine_levels;
    uint32_t status;
    int32_t certified;
    int32_t rung_L, rung_R;
    int32_t force_miss;
    int32_t max_attempts;
    float ladder_L[kLadder];  // a_L rungs (descending ranks h, 4h, 16h, open)
    float ladder_R[kLadder];  // a_R rungs (ranks l, l/4, l/16, open)
    uint32_t bin_kmin, bin_kmax;  // key range of the band histogram of the current bracket
    int32_t stage;            // 1: the histogram bin `sub_bin` is left for extract + solve2
    int32_t sub_bin;
    unsigned long long n_sub;  // scores extracted from that bin
    float sub_aL, sub_aR;      // sub-bracket [sub_aL, sub_aR) = that bin's edges
    int32_t sub_hasR, pad1;
    double sub_SL, sub_SR, sub_cntR;  // tails of the sub-bracket
    float hard_c;             // zero-temperature mode: the boundary score c and
    int32_t pad2;             //   the share p of the scores equal to c
    double hard_frac;
    double scratch[35];       // kernel-to-kernel scalars (phase timestamps)
};
static_assert(sizeof(RowState) == 512, "row records are 512-byte slots of the workspace");
static_assert(sizeof(RowState) <= 512, "row record fits its slot");

// ---------------------------------------------------------------------------
// Order-preserving fp32 <-> u32 keys: flip every bit of a negative float,
// only the sign bit of a non-negative one.  Unsigned key order is value order.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t to_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_key(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

__device__ __forceinline__ bool finite_f(float x) { return fabsf(x) <= 3.402823466e38f; }

// ---------------------------------------------------------------------------
// Threshold carried as two floats b = hi + lo, so that per element the scaled
// margin x = (r - b)/t is formed in fp32 with the accuracy of an fp64 b: the
// subtraction r - hi is exact near the threshold (Sterbenz), lo is tiny.
// ---------------------------------------------------------------------------
struct Thr {
    float hi, lo, inv_t;
    float inv_lo;  // 1/t - inv_t
};
__device__ __forceinline__ Thr make_thr(double b, double t) {
    Thr h;
    h.hi = (float)b;
    h.lo = (float)(b - (double)h.hi);
    h.inv_t = (float)(1.0 / t);
    h.inv_lo = (float)(1.0 / t - (double)h.inv_t);
    return h;
}
__device__ __forceinline__ float scaled_margin(float r, const Thr& h) {
    return __fmul_rn(__fsub_rn(__fsub_rn(r, h.hi), h.lo), h.inv_t);
}
// The fast margin with 1/t as a two-float pair (its rounding is common to all
// scores of a row).
__device__ __forceinline__ float scaled_margin_it(float r, const Thr& h) {
    const float d = __fsub_rn(__fsub_rn(r, h.hi), h.lo);
    return fmaf(d, h.inv_t, __fmul_rn(d, h.inv_lo));
}
// Soft rows: t not small against |b|.  On sharp rows (40 t < |b|) every score
// that carries weight (|x| <= 20, beyond which e^{-|x|} < 2.1e-9) lies within
// a factor of two of b, where r - hi is exact, and the fast margin's one
// rounding stays below 2^-24 |x|.
__device__ __forceinline__ bool soft_row(double b, double t) { return 40.0 * t >= fabs(b); }

// 2^y with flush-to-zero for results below the smallest normal float (the
// hardware ex2 approximation; about 2 ulp).  Flushing is harmless here: every
// exponential feeds a probability, a weight or a sum in which a term below
// 1.2e-38 is negligible.
__device__ __forceinline__ float ex2_ftz(float y) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(y));
    return r;
}
constexpr float kLog2e = 1.4426950408889634f;

// e^{-a} for a >= 0 without the hardware approximation's bias: Cody and
// Waite's reduction a = j ln2 + r, |r| <= ln2/2 (ln2 split into a head whose
// product with any j < 512 is exact and a small tail), the Taylor polynomial
// of e^{-r} to degree 7 (truncation below 6e-9 relative) by Horner's rule
// with fused multiply-adds, and 2^{-j} from the exponent field.  About one ulp
// with rounding errors of both signs, so that sums of many p stay on budget;
// results below the smallest normal float are flushed to 0.
__device__ __forceinline__ float exp_neg(float a) {
    const float j = rintf(a * 1.44269504f);
    if (j > 126.f) return 0.f;
    float r = fmaf(-j, 0.693145751953125f, a);
    r = fmaf(-j, 1.428606765330187e-6f, r);
    const float s = -r;
    float q = 1.0f / 5040.0f;
    q = fmaf(q, s, 1.0f / 720.0f);
    q = fmaf(q, s, 1.0f / 120.0f);
    q = fmaf(q, s, 1.0f / 24.0f);
    q = fmaf(q, s, 1.0f / 6.0f);
    q = fmaf(q, s, 0.5f);
    q = fmaf(q, s, 1.0f);
    q = fmaf(q, s, 1.0f);
    const float scale = __int_as_float((127 - (int)j) << 23);
    const float e = q * scale;
    return e >= 1.17549435e-38f ? e : 0.f;
}

// e = exp(-|x|); p = sigma(x) = x < 0 ? e/2 : 1 - e/2; f = e/2.  One exp.
__device__ __forceinline__ float neg_abs_exp(float x) { return ex2_ftz(-fabsf(x) * kLog2e); }
__device__ __forceinline__ float cdf_from(float x, float e) { return x < 0.f ? 0.5f * e : 1.f - 0.5f * e; }

// Gap factor e^{(lo - hi)/t} between two neighbouring sorted scores lo <= hi.
// The difference of two fp32 values is exact in fp64 and the exponential is
// taken in fp64: the scans chain these factors over up to n positions, and an
// fp32 factor's rounding would build up along the chain whenever t is large
// compared with the gaps (weights that barely decay).
__device__ __forceinline__ double gap_factor(float lo, float hi, double inv_t) {
    return exp(((double)lo - (double)hi) * inv_t);
}

// Out-of-line fp64 exponential and logarithms for the single-CTA solve steps.
// Those steps run most of their code once, so every inlined copy of a libm
// routine is fetched cold into the instruction cache; one shared copy per
// routine is fetched once and then stays hot.
static __device__ __noinline__ double cold_exp(double x) { return exp(x); }
static __device__ __noinline__ double cold_log(double x) { return log(x); }
__device__ __forceinline__ double gap_factor_cold(float lo, float hi, double inv_t) {
    return cold_exp(((double)lo - (double)hi) * inv_t);
}

// ---------------------------------------------------------------------------
// Affine maps x -> a x + c, the element of the stable prefix/suffix scans.
// The prefix sum P_j = sum_{i<=j} e^{(s_i - s_j)/t} obeys P_j = 1 + g_j P_{j-1}
// with the gap factor g_j = e^{(s_{j-1} - s_j)/t} in (0, 1]; the suffix sum Q_j
// obeys Q_j = 1 + g_{j+1} Q_{j+1}.  Every factor is at most 1, so nothing
// overflows, and composing maps is associative.
// ---------------------------------------------------------------------------
struct Aff {
    double a, c;
};
__device__ __forceinline__ Aff aff_id() { return {1.0, 0.0}; }
// Apply `first`, then `second`.
__device__ __forceinline__ Aff aff_then(const Aff& first, const Aff& second) {
    return {second.a * first.a, fma(second.a, first.c, second.c)};
}

__device__ __forceinline__ Aff shfl_up_aff(const Aff& v, int d) {
    return {__shfl_up_sync(0xffffffffu, v.a, d), __shfl_up_sync(0xffffffffu, v.c, d)};
}
__device__ __forceinline__ Aff shfl_down_aff(const Aff& v, int d) {
    return {__shfl_down_sync(0xffffffffu, v.a, d), __shfl_down_sync(0xffffffffu, v.c, d)};
}

// Inclusive warp scan in lane order (lane 0 applied first).
__device__ __forceinline__ Aff warp_scan_fwd(Aff v, int lane) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        Aff o = shfl_up_aff(v, d);
        if (lane >= d) v = aff_then(o, v);
    }
    return v;
}
// Inclusive warp scan in reverse lane order (lane 31 applied first).
__device__ __forceinline__ Aff warp_scan_bwd(Aff v, int lane) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        Aff o = shfl_down_aff(v, d);
        if (lane + d < 32) v = aff_then(o, v);
    }
    return v;
}

// Block-wide exclusive scans of affine maps (every thread calls; `wt` holds
// blockDim.x/32 maps of shared memory).  Forward: composition of the maps of
// all lower threads (thread 0 applied first).  Backward: of all higher
// threads (the last thread applied first).  Two levels of warp scans: the
// warps' aggregates are scanned by warp 0, not walked one by one.
__device__ inline Aff block_excl_scan_fwd(const Aff& v, Aff* wt) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const Aff inc = warp_scan_fwd(v, lane);
    Aff ex = shfl_up_aff(inc, 1);
    if (lane == 0) ex = aff_id();
    __syncthreads();
    if (lane == 31) wt[w] = inc;
    __syncthreads();
    if (w == 0) {
        const Aff a = lane < nw ? wt[lane] : aff_id();
        const Aff sc = warp_scan_fwd(a, lane);
        Aff e = shfl_up_aff(sc, 1);
        if (lane == 0) e = aff_id();
        if (lane < nw) wt[lane] = e;
    }
    __syncthreads();
    return aff_then(wt[w], ex);
}
__device__ inline Aff block_excl_scan_bwd(const Aff& v, Aff* wt) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const Aff inc = warp_scan_bwd(v, lane);
    Aff ex = shfl_down_aff(inc, 1);
    if (lane == 31) ex = aff_id();
    __syncthreads();
    if (lane == 0) wt[w] = inc;
    __syncthreads();
    if (w == 0) {
        // aggregates of warps lane..nw-1, the last applied first; lanes past
        // nw hold the identity
        const Aff a = lane < nw ? wt[lane] : aff_id();
        const Aff sc = warp_scan_bwd(a, lane);
        Aff e = shfl_down_aff(sc, 1);
        if (lane == 31) e = aff_id();
        if (lane < nw) wt[lane] = e;
    }
    __syncthreads();
    return aff_then(wt[w], ex);
}
// Block-wide exclusive suffix sum of a count (sum over higher threads).
__device__ inline long long block_excl_suffix_ll(long long v, long long* wt) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    long long inc = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const long long o = __shfl_down_sync(0xffffffffu, inc, d);
        if (lane + d < 32) inc += o;
    }
    __syncthreads();
    if (lane == 0) wt[w] = inc;
    __syncthreads();
    if (w == 0) {  // suffix sums of the warps' totals, exclusive
        long long a = lane < nw ? wt[lane] : 0ll;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const long long o = __shfl_down_sync(0xffffffffu, a, d);
            if (lane + d < 32) a += o;
        }
        const long long own = lane < nw ? wt[lane] : 0ll;
        __syncwarp();
        if (lane < nw) wt[lane] = a - own;
    }
    __syncthreads();
    return inc - v + wt[w];
}

// ---------------------------------------------------------------------------
// Closed-form root of the budget equation inside one segment of the sorted
// order (section 2.2, "closed-form root").  Let the segment lie between a left
// anchor sL (prefix weight Bh = sum over scores <= sL of e^{(s - sL)/t}) and a
// right anchor sR (suffix weight Ah = sum over scores >= sR of e^{-(s - sR)/t}),
// with m scores at or above sR and c = m - k.  With y = e^{(b - sR)/t} and
// delta = e^{(sL - sR)/t} the equation F(b) = k reads
//     Ah y^2 - 2 c y - Bh delta = 0,
// whose positive root is taken in the log domain (delta underflows when t is
// far below the gap):
//     c = 0:  ln y = (ln Bh + ln delta - ln Ah)/2
//     c > 0:  ln y = ln(c + S) - ln Ah
//     c < 0:  ln y = ln Bh + ln delta - ln(S - c),      S = sqrt(c^2 + Ah Bh delta).
// A missing anchor (no scores on that side, weight 0) leaves a single
// exponential:  Bh = 0: b = sR + t ln(2c/Ah);  Ah = 0: b = sL + t ln(Bh/(-2c)).
// segment_root clamps the result into [sL, sR]; segment_root_raw returns the
// root of this segment's formula wherever it lies (outside the segment when
// the balancing segment is another one).
//
// With rho = Ah Bh delta / c^2 the larger magnitude |c| + S is |c| (1 + sqrt(1
// + rho)), or sqrt(Ah Bh delta) (sqrt(1/rho) + sqrt(1 + 1/rho)) when rho > 1,
// so that ln(|c| + S) costs one exponential and one logarithm after ln Ah,
// ln Bh and ln |c|, and ln(S - c) for c < 0 is ln(Ah Bh delta) - ln(|c| + S).
// Every lane of one warp calls it with the same arguments: lanes 0, 1 and 2
// take the three first logarithms at once, and all lanes return b.
// ---------------------------------------------------------------------------
// The body, inlined where it runs many times per warp (the on-chip search); the
// single-CTA solvers call the out-of-line copy below.
template <bool kInline>
__device__ __forceinline__ double segment_root_body(bool hasL, double sL, double Bh, bool hasR,
                                                    double sR, double Ah, double c, double t) {
    auto lg = [](double v) { return kInline ? log(v) : cold_log(v); };
    auto ex = [](double v) { return kInline ? exp(v) : cold_exp(v); };
    const int lane = threadIdx.x & 31;
    hasL = hasL && Bh > 0.0;
    hasR = hasR && Ah > 0.0;
    if (!hasL && !hasR) return nan("");
    double arg = 1.0;
    if (!hasL) arg = 2.0 * c / Ah;
    else if (!hasR) arg = Bh / (-2.0 * c);
    else arg = lane == 0 ? Ah : (lane == 1 ? Bh : fabs(c));
    if (lane > 2) arg = 1.0;
    const double lgv = lg(arg);
    const double l0 = __shfl_sync(0xffffffffu, lgv, 0);
    if (!hasL) return sR + t * l0;
    if (!hasR) return sL + t * l0;
    const double l1 = __shfl_sync(0xffffffffu, lgv, 1);
    const double l2 = __shfl_sync(0xffffffffu, lgv, 2);
    const double lnd = (sL - sR) / t, lnA = l0, lnB = l1;
    double ln_y;
    if (c == 0.0) {
        ln_y = 0.5 * (lnB + lnd - lnA);
    } else {
        const double lnc = l2;
        const double lnrho = lnA + lnB + lnd - 2.0 * lnc;
        double L;  // ln(|c| + S)
        if (lnrho <= 0.0) {
            const double rho = ex(lnrho);
            L = lnc + lg(1.0 + sqrt(1.0 + rho));
        } else {
            const double sg = ex(-lnrho);
            L = 0.5 * (lnA + lnB + lnd) + lg(sqrt(sg) + sqrt(1.0 + sg));
        }
        ln_y = c > 0.0 ? L - lnA : lnB + lnd - L;
    }
    return sR + t * ln_y;
}
static __device__ __noinline__ double segment_root_raw(bool hasL, double sL, double Bh,
                                                       bool hasR, double sR, double Ah, double c,
                                                       double t) {
    return segment_root_body<false>(hasL, sL, Bh, hasR, sR, Ah, c, t);
}
__device__ __forceinline__ double segment_root(bool hasL, double sL, double Bh, bool hasR,
                                               double sR, double Ah, double c, double t) {
    double b = segment_root_raw(hasL, sL, Bh, hasR, sR, Ah, c, t);
    if (hasL && Bh > 0.0 && hasR && Ah > 0.0) {
        if (b < sL) b = sL;
        if (b > sR) b = sR;
    }
    return b;
}

// ---------------------------------------------------------------------------
// Band histogram layout: the key range [kmin, kmax] of a bracket [a_L, a_R)
// split into nbin <= 2048 bins of 2^sh consecutive keys.  Edge j is the float
// with key kmin + j 2^sh (the last edge is kmax + 1, the key of a_R), so bin j
// holds the scores e_j <= s < e_{j+1}.  Per-bin sums are kept in fixed point
// (2^-32 units, every term is at most 1) so that atomic accumulation in any
// order gives the same bits.
// ---------------------------------------------------------------------------
constexpr int kBins = 2048;
constexpr double kFixScale = 4294967296.0;  // 2^32

struct BinLayout {
    uint32_t kmin, kmax;
    int sh, nbin;
};
__device__ __forceinline__ BinLayout make_bins(uint32_t kmin, uint32_t kmax) {
    BinLayout B;
    B.kmin = kmin;
    B.kmax = kmax < kmin ? kmin : kmax;
    B.sh = 0;
    while (((B.kmax - B.kmin) >> B.sh) >= (uint32_t)kBins) ++B.sh;
    B.nbin = (int)((B.kmax - B.kmin) >> B.sh) + 1;
    return B;
}
__device__ __forceinline__ uint32_t bin_edge_key(const BinLayout& B, int j) {
    const unsigned long long e = (unsigned long long)B.kmin + ((unsigned long long)j << B.sh);
    const unsigned long long top = (unsigned long long)B.kmax + 1ull;
    const unsigned long long v = e < top ? e : top;
    return v > 0xffffffffull ? 0xffffffffu : (uint32_t)v;
}
__device__ __forceinline__ float bin_edge(const BinLayout& B, int j) {
    return from_key(bin_edge_key(B, j));
}
__device__ __forceinline__ int bin_of(const BinLayout& B, uint32_t key) {
    if (key <= B.kmin) return 0;
    const uint32_t j = (key - B.kmin) >> B.sh;
    return j >= (uint32_t)B.nbin ? B.nbin - 1 : (int)j;
}
// Key range of the histogram of bracket [aL, aR) (open ends: the finite range).
__device__ __forceinline__ void bracket_key_range(float aL, float aR, uint32_t* kmin,
                                                  uint32_t* kmax) {
    *kmin = (aL >= -3.402823466e38f) ? to_key(aL) : 0x00800000u;  // key of -FLT_MAX
    *kmax = (aR <= 3.402823466e38f) ? to_key(aR) - 1u : 0xff7fffffu;  // key of +FLT_MAX
}

// ---------------------------------------------------------------------------
// Small block utilities.
// ---------------------------------------------------------------------------
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
    return v;
}
__device__ __forceinline__ float warp_min_f(float v) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, d));
    return v;
}
__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, d));
    return v;
}
__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
    return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
    return v;
}
__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
    return v;
}

// Block-wide sum of a double; every thread gets the result.  `red` needs
// blockDim.x/32 doubles.  Fixed tree order, so the result is deterministic.
__device__ inline double block_sum_d(double v, double* red) {
    int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_sum_d(v);
    __syncthreads();
    if (lane == 0) red[w] = v;
    __syncthreads();
    double s = 0.0;
    for (int i = 0; i < nw; ++i) s += red[i];
    return s;
}
__device__ inline float block_min_f(float v, float* red) {
    int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_min_f(v);
    __syncthreads();
    if (lane == 0) red[w] = v;
    __syncthreads();
    float s = red[0];
    for (int i = 1; i < nw; ++i) s = fminf(s, red[i]);
    return s;
}
__device__ inline float block_max_f(float v, float* red) {
    int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_max_f(v);
    __syncthreads();
    if (lane == 0) red[w] = v;
    __syncthreads();
    float s = red[0];
    for (int i = 1; i < nw; ++i) s = fmaxf(s, red[i]);
    return s;
}
// Block-wide sums of four doubles at once, valid in thread 0 only (one
// barrier); `red` needs blockDim.x/32 rows.  Fixed order, deterministic.
__device__ inline void block_sum4_to0(double (&v)[4], double (*red)[4]) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = warp_sum_d(v[i]);
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) red[w][i] = v[i];
    }
    __syncthreads();
    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            double s = 0.0;
            for (int u = 0; u < nw; ++u) s += red[u][i];
            v[i] = s;
        }
    }
}
__device__ inline long long block_sum_ll(long long v, long long* red) {
    int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
    __syncthreads();
    if (lane == 0) red[w] = v;
    __syncthreads();
    long long s = 0;
    for (int i = 0; i < nw; ++i) s += red[i];
    return s;
}

// ---------------------------------------------------------------------------
// SplitMix64 (Steele, Lea and Flood 2014) as a counter-based generator:
// output c of the stream seeded with `seed` is mix(seed + (c+1) * golden gamma).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t splitmix64_at(uint64_t seed, uint64_t c) {
    uint64_t z = seed + (c + 1ull) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// Draw s of a row's localization sample (section 2.2 of the pages): the index
// I = high half of z1 * n and Laplace(0, t) noise by the inverse CDF from 24
// bits of z2, u centred in (-1/2, 1/2); z1, z2 are SplitMix64 outputs 2s and
// 2s + 1 of the stream (seed, counters from c0).
__device__ __forceinline__ int64_t sample_index(uint64_t seed, uint64_t c0, int64_t s, int64_t n) {
    const uint64_t z1 = splitmix64_at(seed, c0 + 2ull * (uint64_t)s);
    return (int64_t)__umul64hi(z1, (uint64_t)n);
}
__device__ __forceinline__ float sample_noise(uint64_t seed, uint64_t c0, int64_t s, double t) {
    const uint64_t z2 = splitmix64_at(seed, c0 + 2ull * (uint64_t)s + 1ull);
    const double u = ((double)(z2 >> 40) + 0.5) * (1.0 / 16777216.0) - 0.5;
    const float a = (float)(1.0 - 2.0 * fabs(u));  // exact: a multiple of 2^-24 in (0, 1]
    return (u < 0.0 ? 1.f : -1.f) * (float)t * logf(a);
}

// Phase timestamps (ns, global timer) of the single-CTA bracketing steps, kept
// in the row record's scratch words for diagnostics.
__device__ __forceinline__ void phase_mark(RowState* st, int slot) {
    if (threadIdx.x == 0) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        reinterpret_cast<unsigned long long*>(st->scratch)[slot] = t;
    }
}

// Programmatic dependent launch: kernels of the long-row pipelines are
// launched so that they may be scheduled while the previous kernel on the
// stream drains; each calls pdl_wait() before it touches any memory, which
// returns once the previous grid has finished and its writes are visible.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void set_status(WsHeader* hdr, uint32_t bits) {
    atomicOr(&hdr->status, bits);
}

}  // namespace lapsum
