// On-chip full-sort solver for rows of n <= 4096 scores, fused with p emission,
// and the fused one-pass VJP for the same rows.
//
// "Fast LapSum: Exact Differentiable Top-k at Million Scale" (gist.science
// explainer pages), section 2.2, full-sort solver: sort the row, run one
// numerically stable prefix/suffix scan over the sorted scores to obtain the
// threshold curve F(s_j), look up the segment where F crosses k, and take the
// closed-form root there.  Section 2.1 gives p and the analytic VJP.
//
// Layout: a row of NPAD = E * RT keys (n padded with +inf keys) is held by RT
// threads, E consecutive elements each, entirely in registers.  Bitonic stages
// with a partner in the same thread swap registers, partners in the same warp
// exchange through shuffles, and only partners in another warp go through
// shared memory.  The scan carries fp64 affine maps (gap factor, 1) whose
// composition is a warp shuffle scan plus one shared-memory step across warps.
#include <cuda_fp16.h>

#include "lapsum_common.cuh"
#include "lapsum_kernels.h"
#include "bitonic.cuh"

namespace lapsum {
namespace {

constexpr uint32_t kPadKey = 0xffffffffu;

template <int E, int RT, int CTA>
struct Shape {
    static constexpr int NPAD = E * RT;
    static constexpr int ROWS = CTA / RT;
    static constexpr int WPR = RT / 32;  // warps per row
    static constexpr int NW = CTA / 32;
    static_assert(RT % 32 == 0 && CTA % RT == 0, "rows are whole warps");
    static_assert(NPAD <= 4096, "on-chip rows hold at most 4096 keys");
};

// Load E consecutive elements of a row (idx = tid*E + e), padding past n.
template <int E>
__device__ __forceinline__ void load_row(const float* __restrict__ row, int n, int tid, bool vec,
                                         bool row_ok, float (&x)[E], bool (&valid)[E]) {
    const int base = tid * E;
    if constexpr (E % 4 == 0) {
        if (vec && row_ok && base + E <= n) {
#pragma unroll
            for (int q = 0; q < E / 4; ++q) {
                float4 v4 = __ldg(reinterpret_cast<const float4*>(row + base) + q);
                x[4 * q + 0] = v4.x;
                x[4 * q + 1] = v4.y;
                x[4 * q + 2] = v4.z;
                x[4 * q + 3] = v4.w;
            }
#pragma unroll
            for (int e = 0; e < E; ++e) valid[e] = true;
            return;
        }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
        valid[e] = row_ok && (base + e < n);
        x[e] = valid[e] ? __ldg(row + base + e) : 0.f;
    }
}

// The same for bf16 scores (bit patterns; bf16 is the upper half of fp32, so
// the widening is exact): eight per 16-byte load.
__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }
template <int E>
__device__ __forceinline__ void load_row(const uint16_t* __restrict__ row, int n, int tid, bool vec,
                                         bool row_ok, float (&x)[E], bool (&valid)[E]) {
    const int base = tid * E;
    if constexpr (E % 8 == 0) {
        if (vec && row_ok && base + E <= n) {
#pragma unroll
            for (int q = 0; q < E / 8; ++q) {
                const uint4 u = __ldg(reinterpret_cast<const uint4*>(row + base) + q);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    x[8 * q + 2 * h] = __uint_as_float(w[h] << 16);
                    x[8 * q + 2 * h + 1] = __uint_as_float(w[h] & 0xffff0000u);
                }
            }
#pragma unroll
            for (int e = 0; e < E; ++e) valid[e] = true;
            return;
        }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
        valid[e] = row_ok && (base + e < n);
        x[e] = valid[e] ? bf16_to_f32(__ldg(row + base + e)) : 0.f;
    }
}

// The same for fp16 scores (IEEE half bit patterns, widened exactly to fp32).
struct F16Bits {
    uint16_t bits;
};
__device__ __forceinline__ float f16_to_f32(uint16_t h) { return __half2float(__ushort_as_half(h)); }
template <int E>
__device__ __forceinline__ void load_row(const F16Bits* __restrict__ row_in, int n, int tid,
                                         bool vec, bool row_ok, float (&x)[E], bool (&valid)[E]) {
    const uint16_t* row = reinterpret_cast<const uint16_t*>(row_in);
    const int base = tid * E;
    if constexpr (E % 8 == 0) {
        if (vec && row_ok && base + E <= n) {
#pragma unroll
            for (int q = 0; q < E / 8; ++q) {
                const uint4 u = __ldg(reinterpret_cast<const uint4*>(row + base) + q);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    x[8 * q + 2 * h] = f16_to_f32((uint16_t)(w[h] & 0xffffu));
                    x[8 * q + 2 * h + 1] = f16_to_f32((uint16_t)(w[h] >> 16));
                }
            }
#pragma unroll
            for (int e = 0; e < E; ++e) valid[e] = true;
            return;
        }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
        valid[e] = row_ok && (base + e < n);
        x[e] = valid[e] ? f16_to_f32(__ldg(row + base + e)) : 0.f;
    }
}

template <int E>
__device__ __forceinline__ void store_row(float* __restrict__ row, int n, int tid, bool vec,
                                          bool row_ok, const float (&y)[E]) {
    if (!row_ok) return;
    const int base = tid * E;
    if constexpr (E % 4 == 0) {
        if (vec && base + E <= n) {
#pragma unroll
            for (int q = 0; q < E / 4; ++q)
                reinterpret_cast<float4*>(row + base)[q] =
                    make_float4(y[4 * q], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]);
            return;
        }
    }
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (base + e < n) row[base + e] = y[e];
}

// Sum of an int over the threads of one row.
template <int E, int RT, int CTA>
__device__ __forceinline__ int row_sum_i(int v, int* red) {
    using S = Shape<E, RT, CTA>;
    v = warp_sum_i(v);
    if constexpr (S::WPR == 1) {
        return v;
    } else {
        const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
        if (lane == 0) red[w] = v;
        __syncthreads();
        const int w0 = (w / S::WPR) * S::WPR;
        int s = 0;
#pragma unroll
        for (int i = 0; i < S::WPR; ++i) s += red[w0 + i];
        __syncthreads();
        return s;
    }
}
template <int E, int RT, int CTA>
__device__ __forceinline__ double row_sum_d(double v, double* red) {
    using S = Shape<E, RT, CTA>;
    v = warp_sum_d(v);
    if constexpr (S::WPR == 1) {
        return v;
    } else {
        const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
        if (lane == 0) red[w] = v;
        __syncthreads();
        const int w0 = (w / S::WPR) * S::WPR;
        double s = 0.0;
#pragma unroll
        for (int i = 0; i < S::WPR; ++i) s += red[w0 + i];
        __syncthreads();
        return s;
    }
}
template <int E, int RT, int CTA>
__device__ __forceinline__ float row_min_f(float v, float* red) {
    using S = Shape<E, RT, CTA>;
    v = warp_min_f(v);
    if constexpr (S::WPR == 1) {
        return v;
    } else {
        const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
        if (lane == 0) red[w] = v;
        __syncthreads();
        const int w0 = (w / S::WPR) * S::WPR;
        float s = red[w0];
#pragma unroll
        for (int i = 1; i < S::WPR; ++i) s = fminf(s, red[w0 + i]);
        __syncthreads();
        return s;
    }
}

// Exclusive prefix of an int over the threads of one row (thread order);
// *total gets the row's sum.
template <int E, int RT, int CTA>
__device__ __forceinline__ int row_excl_scan_i(int v, int* red, int* total) {
    using S = Shape<E, RT, CTA>;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, inc, d);
        if (lane >= d) inc += o;
    }
    if constexpr (S::WPR == 1) {
        *total = __shfl_sync(0xffffffffu, inc, 31);
        return inc - v;
    } else {
        if (lane == 31) red[w] = inc;
        __syncthreads();
        const int w0 = (w / S::WPR) * S::WPR;
        int before = 0, all = 0;
#pragma unroll
        for (int i = 0; i < S::WPR; ++i) {
            const int c = red[w0 + i];
            before += (w0 + i < w) ? c : 0;
            all += c;
        }
        __syncthreads();
        *total = all;
        return before + inc - v;
    }
}

// Barrier over the threads of one row: a row held by one warp needs only the
// warp's own barrier, so the rows of a CTA run their steps independently.
template <int E, int RT, int CTA>
__device__ __forceinline__ void row_sync() {
    if constexpr (Shape<E, RT, CTA>::WPR == 1) __syncwarp();
    else __syncthreads();
}

// Selection list of the router form: per row, the positions (ascending) and
// values of the scores with p > eps, at most cap of them, and their count.
struct SelectOut {
    int32_t* idx;
    float* val;
    int32_t* cnt;
    int cap;
    float eps;
};

// Shared memory of the sort-and-scan solve of one CTA's rows.
template <int E, int RT, int CTA>
struct SortSmem {
    uint32_t xch[(RT > 32) ? CTA * E : 1];
    uint32_t last_key[CTA];
    double first_gap[CTA];
    Aff wf[CTA / 32], wb[CTA / 32];
    int ired[CTA / 32];
    double anchor[CTA / RT][4];
};

// Sort-and-scan solve of one row (section 2.2, full-sort solver): bitonic sort
// of the keys (E per thread, pads last), gap factors, the prefix and suffix
// scans of the threshold curve, the count of F(s_j) >= k and the closed-form
// root in that segment.  Every thread of the CTA calls it when a row spans
// several warps (the CTA synchronises); a row of one warp may call it alone.
// The row's first warp returns b (NaN when `ok` is false); other threads
// return 0.
template <int E, int RT, int CTA>
__device__ __forceinline__ double sort_solve_row(uint32_t (&key)[E], int n, double kr, double t,
                                                 bool ok, SortSmem<E, RT, CTA>& sm) {
    using S = Shape<E, RT, CTA>;
    const int rloc = threadIdx.x / RT;
    const int tid = threadIdx.x % RT;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const double inv_t = 1.0 / t;

    bitonic_sort_row<E, RT, CTA>(key, tid, sm.xch);

    // Sorted values and gap factors g_j = exp((s_{j-1} - s_j)/t), 0 at j = 0 and past n.
    float s[E];
    double g[E];
#pragma unroll
    for (int e = 0; e < E; ++e) s[e] = from_key(key[e]);
    sm.last_key[threadIdx.x] = key[E - 1];
    row_sync<E, RT, CTA>();
    const float s_prev = (tid > 0) ? from_key(sm.last_key[threadIdx.x - 1]) : 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int j = tid * E + e;
        const float sp = (e == 0) ? s_prev : s[e - 1];
        g[e] = (j >= 1 && j < n) ? gap_factor(sp, s[e], inv_t) : 0.0;
    }
    sm.first_gap[threadIdx.x] = g[0];
    row_sync<E, RT, CTA>();
    const double g_next = (tid + 1 < RT) ? sm.first_gap[threadIdx.x + 1] : 0.0;

    // Thread aggregates of the forward (prefix) and backward (suffix) maps.
    Aff af = aff_id(), ab = aff_id();
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int j = tid * E + e;
        const Aff m = (j < n) ? Aff{g[e], 1.0} : aff_id();
        af = aff_then(af, m);
    }
#pragma unroll
    for (int e = E - 1; e >= 0; --e) {
        const int j = tid * E + e;
        const double gn = (e + 1 < E) ? g[e + 1] : g_next;
        const Aff m = (j < n) ? Aff{gn, 1.0} : Aff{0.0, 0.0};
        ab = aff_then(ab, m);
    }
    // Exclusive prefix (maps of earlier threads) and suffix (later threads).
    Aff inc_f = warp_scan_fwd(af, lane);
    Aff inc_b = warp_scan_bwd(ab, lane);
    Aff ex_f = shfl_up_aff(inc_f, 1);
    Aff ex_b = shfl_down_aff(inc_b, 1);
    if (lane == 0) ex_f = aff_id();
    if (lane == 31) ex_b = aff_id();
    if constexpr (S::WPR > 1) {
        if (lane == 31) sm.wf[warp] = inc_f;
        if (lane == 0) sm.wb[warp] = inc_b;
        __syncthreads();
        const int w0 = (warp / S::WPR) * S::WPR;
        Aff pre = aff_id();
        for (int w = w0; w < warp; ++w) pre = aff_then(pre, sm.wf[w]);
        ex_f = aff_then(pre, ex_f);
        Aff suf = aff_id();
        for (int w = w0 + S::WPR - 1; w > warp; --w) suf = aff_then(suf, sm.wb[w]);
        ex_b = aff_then(suf, ex_b);
    }

    // Threshold curve G_j = F(s_j) = (n - j) - Q_j/2 + (P_j - 1)/2 and its count.
    double P[E], Q[E];
    double x = ex_f.c;  // P just before this thread's first element
#pragma unroll
    for (int e = 0; e < E; ++e) {
        x = fma(g[e], x, 1.0);
        P[e] = x;
    }
    double y = ex_b.c;  // Q just after this thread's last element
    int cnt = 0;
#pragma unroll
    for (int e = E - 1; e >= 0; --e) {
        const int j = tid * E + e;
        const double gn = (e + 1 < E) ? g[e + 1] : g_next;
        y = (j < n) ? fma(gn, y, 1.0) : 0.0;
        Q[e] = y;
        const double G = (double)(n - j) - 0.5 * Q[e] + 0.5 * (P[e] - 1.0);
        cnt += (j < n && G >= kr) ? 1 : 0;
    }
    const int jstar = row_sum_i<E, RT, CTA>(cnt, sm.ired);

    // Anchors of the balancing segment: left = sorted position j*-1, right = j*.
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int j = tid * E + e;
        if (j == jstar - 1) {
            sm.anchor[rloc][0] = s[e];
            sm.anchor[rloc][1] = P[e];
        }
        if (j == jstar && j < n) {
            sm.anchor[rloc][2] = s[e];
            sm.anchor[rloc][3] = Q[e];
        }
    }
    row_sync<E, RT, CTA>();
    double bb = 0.0;
    if (tid < 32) {  // the row's first warp takes the root together
        if (!ok) {
            bb = nan("");
        } else {
            const bool hasL = jstar >= 1, hasR = jstar < n;
            bb = segment_root(hasL, sm.anchor[rloc][0], hasL ? sm.anchor[rloc][1] : 0.0, hasR,
                              sm.anchor[rloc][2], hasR ? sm.anchor[rloc][3] : 0.0,
                              (double)(n - jstar) - kr, t);
        }
    }
    return bb;
}

// Emit p_i = sigma((r_i - b)/t) in the original order; optionally the row's
// sum of f and the router list of p > eps.  Every thread of the row calls it.
template <int E, int RT, int CTA>
__device__ __forceinline__ void emit_row(const float (&orig)[E], const bool (&valid)[E],
                                         double bb, double t, float* __restrict__ prow, int n,
                                         int tid, bool vec, bool row_ok, int64_t row,
                                         double* __restrict__ sumf_out, const SelectOut& sel,
                                         int* ired, double* dred) {
    const Thr th = make_thr(bb, t);
    float pv[E];
    double sf = 0.0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const float xs = scaled_margin(orig[e], th);
        const float ex = neg_abs_exp(xs);
        pv[e] = cdf_from(xs, ex);
        if (valid[e]) sf += 0.5 * (double)ex;
    }
    store_row<E>(prow, n, tid, vec, row_ok, pv);
    if (sumf_out != nullptr) {
        const double tot = row_sum_d<E, RT, CTA>(sf, dred);
        if (tid == 0 && row_ok) sumf_out[row] = tot;
    }
    if (sel.cnt != nullptr) {  // the same for every thread of the grid
        int c = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) c += (valid[e] && pv[e] > sel.eps) ? 1 : 0;
        int total = 0;
        int o = row_excl_scan_i<E, RT, CTA>(c, ired, &total);
        if (row_ok) {
#pragma unroll
            for (int e = 0; e < E; ++e) {
                if (valid[e] && pv[e] > sel.eps) {
                    if (o < sel.cap) {
                        sel.idx[row * sel.cap + o] = tid * E + e;
                        sel.val[row * sel.cap + o] = pv[e];
                    }
                    ++o;
                }
            }
            if (tid == 0) sel.cnt[row] = total;
        }
    }
}

template <int E, int RT, int CTA, class In>
__global__ void __launch_bounds__(CTA, CTA == 256 ? 4 : 1) onchip_forward_kernel(
    const In* __restrict__ r, int64_t ld, float* __restrict__ p, double* __restrict__ b_out,
    double* __restrict__ sumf_out, int64_t B, int n, double k, const double* __restrict__ k_rows,
    double t, WsHeader* hdr, int vec, SelectOut sel) {
    using S = Shape<E, RT, CTA>;
    __shared__ SortSmem<E, RT, CTA> sm;
    __shared__ double dred[S::NW];
    __shared__ int row_flag[S::ROWS];
    __shared__ double row_b[S::ROWS];

    const int rloc = threadIdx.x / RT;
    const int tid = threadIdx.x % RT;
    const int64_t row = (int64_t)blockIdx.x * S::ROWS + rloc;
    const bool row_ok = row < B;
    const In* rrow = r + (row_ok ? row : 0) * ld;
    // the row's budget: the shared k, or its own entry of k_rows (checked here: a
    // budget outside (0, n) gives b = NaN and a status bit)
    const double kr = (k_rows != nullptr && row_ok) ? k_rows[row] : k;
    const bool k_ok = kr > 0.0 && kr < (double)n;

    if (tid == 0) row_flag[rloc] = 0;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        hdr->last_B = B;
        hdr->last_n = n;
        hdr->last_path = LAPSUM_PATH_FULLSORT;
    }

    float orig[E];
    bool valid[E];
    load_row<E>(rrow, n, tid, vec != 0, row_ok, orig, valid);
    uint32_t key[E];
    bool bad = false;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        key[e] = valid[e] ? to_key(orig[e]) : kPadKey;
        bad |= valid[e] && !finite_f(orig[e]);
    }
    row_sync<E, RT, CTA>();
    if (bad) atomicOr(&row_flag[rloc], 1);
    if (tid == 0 && !k_ok) atomicOr(&row_flag[rloc], 2);
    row_sync<E, RT, CTA>();
    const int flag = row_flag[rloc];

    const double bb = sort_solve_row<E, RT, CTA>(key, n, kr, t, flag == 0 && row_ok, sm);
    if (tid == 0) {
        if (flag && row_ok)
            set_status(hdr, ((flag & 1) ? kDevNonFinite : 0u) | ((flag & 2) ? kDevBadBudget : 0u));
        row_b[rloc] = bb;
        if (row_ok) b_out[row] = bb;
    }
    row_sync<E, RT, CTA>();
    emit_row<E, RT, CTA>(orig, valid, row_b[rloc], t, p + (row_ok ? row : 0) * ld, n, tid,
                         vec != 0, row_ok, row, sumf_out, sel, sm.ired, dred);
}

// ---------------------------------------------------------------------------
// Rows of at most 256 scores, one warp each, solved without a sort (AUTO).
//
// F(c) = sum_i sigma((r_i - c)/t) is continuous and decreasing.  Between two
// neighbouring scores sA <= c < sB it has the closed form of section 2.2's
// root step: with m scores at or above sB, Bh = sum_{r <= sA} e^{(r - sA)/t}
// and Ah = sum_{r >= sB} e^{-(r - sB)/t},
//     F(c) = m - (Ah/2) e^{(c - sB)/t} + (Bh/2) e^{(sA - c)/t},
// so the neighbours of one point c, a count and two sums of exponentials (each
// term at most 1) give that segment's root.  When the root lies in the
// segment it is b.  When it lies beyond sB, then F(sB) > k and b > sB; read
// past sB, the formula keeps the crossed scores at 1 - e^{|x|}/2 where F has
// e^{-|x|}/2, never more, so the formula's root lies in (sB, b]: moving c
// there never overshoots, and each step leaves at least one score behind;
// symmetrically on the left.  A move back across the score just crossed can
// only come from rounding at a boundary where F = k, and that score is then
// b.  The start is a point whose count of larger scores is close to k, found
// by interpolating the count between the row's extremes.  Rows that do not
// settle in kSearchSteps steps are sorted and solved by the full-sort solver
// in the same warp.
//
// Accuracy: every exponential is fp32 and every term is at most 1, so Ah and
// Bh carry a relative error of about 1e-6 and b one of about 1e-6 t.
// ---------------------------------------------------------------------------
constexpr int kSearchRounds = 6;  // count-interpolation rounds for the start
constexpr int kSearchSteps = 8;   // segment steps before the row is sorted instead

// The closed-form root of one segment (the log-domain form of section 2.2's
// root step, as in segment_root), unclamped, in mixed precision: the
// logarithms, exponentials and square roots of quantities of moderate size
// (Ah, Bh, |c| in [1e-38, 256], rho or 1/rho in (0, 1]) use the hardware
// approximations (about 2^-22 relative, or 2^-21 absolute for a logarithm near
// 0), which move b by a few 1e-7 t; the scaled gap ln delta = (sL - sR)/t,
// which can be large, and every sum that contains it stay in fp64, so b keeps
// fp64 accuracy relative to the anchors.  Every lane of the warp calls it with
// the same arguments; lanes 0, 1 and 2 take the three logarithms.
// sqrt of x >= 0 from the hardware reciprocal square root (about 2^-22 relative)
__device__ __forceinline__ float fast_sqrt(float x) { return x > 0.f ? x * rsqrtf(x) : 0.f; }

__device__ __forceinline__ double search_root(bool hasL, float sL, float Bh, bool hasR, float sR,
                                              float Ah, float c, double t, double inv_t) {
    const int lane = threadIdx.x & 31;
    if (!hasL && !hasR) return nan("");
    float arg = 1.f;
    if (!hasL) arg = 2.f * c / Ah;
    else if (!hasR) arg = Bh / (-2.f * c);
    else arg = lane == 0 ? Ah : (lane == 1 ? Bh : fabsf(c));
    if (lane > 2) arg = 1.f;
    const float lg = __logf(arg);
    const double l0 = (double)__shfl_sync(0xffffffffu, lg, 0);
    if (!hasL) return (double)sR + t * l0;
    if (!hasR) return (double)sL + t * l0;
    const double lnA = l0, lnB = (double)__shfl_sync(0xffffffffu, lg, 1);
    const double lnd = ((double)sL - (double)sR) * inv_t;
    double ln_y;
    if (c == 0.f) {
        ln_y = 0.5 * (lnB + lnd - lnA);
    } else {
        const double lnc = (double)__shfl_sync(0xffffffffu, lg, 2);
        const double lnrho = lnA + lnB + lnd - 2.0 * lnc;
        double L;  // ln(|c| + S)
        if (lnrho <= 0.0) {
            const float rho = __expf((float)lnrho);
            L = lnc + (double)__logf(1.f + fast_sqrt(1.f + rho));
        } else {
            const float sg = __expf((float)-lnrho);
            L = 0.5 * (lnA + lnB + lnd) + (double)__logf(fast_sqrt(sg) + fast_sqrt(1.f + sg));
        }
        ln_y = c > 0.f ? L - lnA : lnB + lnd - L;
    }
    return (double)sR + t * ln_y;
}

template <int E, bool FULL>
__device__ __forceinline__ bool search_row(const float (&x)[E], const bool (&valid)[E], int n,
                                           double k, double t, int max_steps, double* b_out) {
    constexpr unsigned kFull = 0xffffffffu;
    // FULL: every element of the warp is a score of the row (n = 32 E)
    auto ok = [&](int e) { return FULL || valid[e]; };
    float vmin = INFINITY, vmax = -INFINITY;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        if (ok(e)) {
            vmin = fminf(vmin, x[e]);
            vmax = fmaxf(vmax, x[e]);
        }
    }
    // order-preserving keys carry the float extremes through the integer reductions
    float lo = from_key(__reduce_min_sync(kFull, to_key(vmin)));
    float hi = from_key(__reduce_max_sync(kFull, to_key(vmax)));

    // Start: interpolate the count of larger scores between the extremes.
    int nlo = n, nhi = 0;
    const float kf = (float)k;
    for (int round = 0; round < kSearchRounds && nlo - nhi > 2; ++round) {
        float f = __fdividef((float)nlo - kf, (float)(nlo - nhi));
        f = fminf(fmaxf(f, 0.0625f), 0.9375f);
        const float c = fmaf(hi - lo, f, lo);
        if (!(c > lo && c < hi)) break;
        unsigned m = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) m += (ok(e) && x[e] > c) ? 1u : 0u;
        m = __reduce_add_sync(kFull, m);
        if ((double)m >= k) {
            lo = c;
            nlo = (int)m;
        } else {
            hi = c;
            nhi = (int)m;
        }
    }
    float c = ((double)nlo - k <= k - (double)nhi) ? lo : hi;

    const float sc = (float)(1.0 / t) * kLog2e;
    const double inv_t = 1.0 / t;
    int dir = 0;  // last move: +1 right, -1 left
    for (int step = 0; step < max_steps; ++step) {
        // neighbours of c: sA = the largest score <= c, sB = the smallest above
        float a = -INFINITY, bb = INFINITY;
        unsigned m = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            if (ok(e)) {
                if (x[e] <= c) {
                    a = fmaxf(a, x[e]);
                } else {
                    bb = fminf(bb, x[e]);
                    ++m;
                }
            }
        }
        const uint32_t ka = __reduce_max_sync(kFull, to_key(a));
        const uint32_t kb = __reduce_min_sync(kFull, to_key(bb));
        m = __reduce_add_sync(kFull, m);
        const bool hasL = ka != to_key(-INFINITY), hasR = kb != to_key(INFINITY);
        const float sA = from_key(ka), sB = from_key(kb);
        float Bh = 0.f, Ah = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            if (ok(e)) {
                if (x[e] <= c) Bh += ex2_ftz((x[e] - sA) * sc);
                else Ah += ex2_ftz((sB - x[e]) * sc);
            }
        }
        Bh = warp_sum_f(Bh);
        Ah = warp_sum_f(Ah);
        const double rt =
            search_root(hasL, sA, Bh, hasR, sB, Ah, (float)((double)m - k), t, inv_t);
        if (!(rt == rt)) return false;
        const bool right = hasR && rt > (double)sB;
        const bool left = hasL && rt < (double)sA;
        if (!right && !left) {
            *b_out = rt;
            return true;
        }
        const int d = right ? 1 : -1;
        if (dir == -d) {  // back across the score just crossed: F = k there within rounding
            *b_out = right ? (double)sB : (double)sA;
            return true;
        }
        dir = d;
        c = right ? fmaxf((float)rt, sB) : fminf((float)rt, nextafterf(sA, -INFINITY));
    }
    return false;
}

// The sort-and-scan solve for a row the search left, out of line so that the
// search keeps its registers; it reloads the row.
template <int E, class In>
__device__ __noinline__ double search_fallback_row(const In* rrow, int n, int vec, double k,
                                                   double t, SortSmem<E, 32, 256>* sm) {
    float x[E];
    bool valid[E];
    load_row<E>(rrow, n, threadIdx.x & 31, vec != 0, true, x, valid);
    uint32_t key[E];
#pragma unroll
    for (int e = 0; e < E; ++e) key[e] = valid[e] ? to_key(x[e]) : kPadKey;
    return sort_solve_row<E, 32, 256>(key, n, k, t, true, *sm);
}

template <int E, class In>
__global__ void __launch_bounds__(256, 6) onchip_search_kernel(
    const In* __restrict__ r, int64_t ld, float* __restrict__ p, double* __restrict__ b_out,
    double* __restrict__ sumf_out, int64_t B, int n, double k, const double* __restrict__ k_rows,
    double t, WsHeader* hdr, int vec, SelectOut sel, int max_steps) {
    constexpr int RT = 32, CTA = 256;
    __shared__ SortSmem<E, RT, CTA> sm;  // for rows the search leaves to the sort
    __shared__ double dred[CTA / 32];
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (CTA / RT) + (threadIdx.x >> 5);
    const bool row_ok = row < B;
    const In* rrow = r + (row_ok ? row : 0) * ld;
    const double kr = (k_rows != nullptr && row_ok) ? k_rows[row] : k;
    const bool k_ok = kr > 0.0 && kr < (double)n;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        hdr->last_B = B;
        hdr->last_n = n;
        hdr->last_path = LAPSUM_PATH_FULLSORT;
    }

    float orig[E];
    bool valid[E];
    load_row<E>(rrow, n, lane, vec != 0, row_ok, orig, valid);
    bool bad = false;
#pragma unroll
    for (int e = 0; e < E; ++e) bad |= valid[e] && !finite_f(orig[e]);
    bad = __any_sync(0xffffffffu, bad);

    double bb = nan("");
    if (row_ok) {  // uniform over the warp
        if (bad || !k_ok) {
            if (lane == 0)
                set_status(hdr, (bad ? kDevNonFinite : 0u) | (!k_ok ? kDevBadBudget : 0u));
        } else if (!(n == 32 * E ? search_row<E, true>(orig, valid, n, kr, t, max_steps, &bb)
                                  : search_row<E, false>(orig, valid, n, kr, t, max_steps, &bb))) {
            bb = search_fallback_row<E, In>(rrow, n, vec, kr, t, &sm);
        }
        if (lane == 0) b_out[row] = bb;
    }
    emit_row<E, RT, CTA>(orig, valid, bb, t, p + (row_ok ? row : 0) * ld, n, lane, vec != 0,
                         row_ok, row, sumf_out, sel, sm.ired, dred);
}

// Zero-temperature limit ("Fast LapSum: Exact Differentiable Top-k at Million
// Scale", gist.science explainer pages, section 2.3: DFTopK's midpoint
// threshold is LapSum at t -> 0).  After the sort, c is the rank-th largest
// score (rank = ceil(k)), a = #{r > c}, m = #{r = c}: when k < a + m the
// scores equal to c share the remaining budget, p = (k - a)/m, and b = c;
// otherwise (k = a + m) b is the midpoint of c and the largest score below c,
// and p is the 0/1 mask.  -0 is read as +0, so equal values are one group.
template <int E, int RT, int CTA>
__global__ void __launch_bounds__(CTA) onchip_hard_kernel(
    const float* __restrict__ r, int64_t ld, float* __restrict__ p, double* __restrict__ b_out,
    int64_t B, int n, double k, int rank, WsHeader* hdr, int vec) {
    using S = Shape<E, RT, CTA>;
    __shared__ uint32_t xch[(RT > 32) ? CTA * E : 1];
    __shared__ int ired[S::NW];
    __shared__ uint32_t row_key[S::ROWS][2];  // c, then the largest key below c
    __shared__ int row_flag[S::ROWS];
    __shared__ double row_val[S::ROWS][2];    // b, share of the scores equal to c
    const int rloc = threadIdx.x / RT;
    const int tid = threadIdx.x % RT;
    const int64_t row = (int64_t)blockIdx.x * S::ROWS + rloc;
    const bool row_ok = row < B;
    if (tid == 0) row_flag[rloc] = 0;
    float orig[E];
    bool valid[E];
    load_row<E>(r + (row_ok ? row : 0) * ld, n, tid, vec != 0, row_ok, orig, valid);
    uint32_t key[E];
    bool bad = false;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        orig[e] += 0.f;  // -0 -> +0
        key[e] = valid[e] ? to_key(orig[e]) : kPadKey;
        bad |= valid[e] && !finite_f(orig[e]);
    }
    row_sync<E, RT, CTA>();
    if (bad) atomicOr(&row_flag[rloc], 1);
    bitonic_sort_row<E, RT, CTA>(key, tid, xch);
    const int q = n - rank;  // ascending position of c
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (tid * E + e == q) row_key[rloc][0] = key[e];
    row_sync<E, RT, CTA>();
    const uint32_t ck = row_key[rloc][0];
    int lt = 0, eq = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const bool in = tid * E + e < n;
        lt += (in && key[e] < ck) ? 1 : 0;
        eq += (in && key[e] == ck) ? 1 : 0;
    }
    lt = row_sum_i<E, RT, CTA>(lt, ired);
    eq = row_sum_i<E, RT, CTA>(eq, ired);
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (tid * E + e == lt - 1) row_key[rloc][1] = key[e];
    row_sync<E, RT, CTA>();
    if (tid == 0) {
        const float c = from_key(ck);
        const double a = (double)(n - lt - eq), m = (double)eq;
        double bb, frac;
        if (k < a + m) {
            bb = (double)c;
            frac = (k - a) / m;
        } else {
            bb = 0.5 * ((double)c + (double)from_key(row_key[rloc][1]));
            frac = 1.0;
        }
        if (row_flag[rloc] || !row_ok) {
            bb = nan("");
            if (row_ok) set_status(hdr, kDevNonFinite);
        }
        row_val[rloc][0] = bb;
        row_val[rloc][1] = frac;
        if (row_ok) b_out[row] = bb;
    }
    row_sync<E, RT, CTA>();
    const double bb = row_val[rloc][0];
    const float c = from_key(ck), share = (float)row_val[rloc][1];
    float pv[E];
#pragma unroll
    for (int e = 0; e < E; ++e)
        pv[e] = isnan(bb) ? bb : (orig[e] > c ? 1.f : (orig[e] == c ? share : 0.f));
    store_row<E>(p + (row_ok ? row : 0) * ld, n, tid, vec != 0, row_ok, pv);
}

template <int E, int RT, int CTA, class In>
__global__ void __launch_bounds__(CTA) onchip_backward_kernel(
    const In* __restrict__ r, int64_t ld, const double* __restrict__ b,
    const float* __restrict__ v, float* __restrict__ g, int64_t B, int n, double t, int vec) {
    using S = Shape<E, RT, CTA>;
    __shared__ float fred[S::NW];
    __shared__ double dred[S::NW];
    const int rloc = threadIdx.x / RT;
    const int tid = threadIdx.x % RT;
    const int64_t row = (int64_t)blockIdx.x * S::ROWS + rloc;
    const bool row_ok = row < B;
    const int64_t off = (row_ok ? row : 0) * ld;

    float rv[E], vv[E];
    bool valid[E];
    load_row<E>(r + off, n, tid, vec != 0, row_ok, rv, valid);
    load_row<E>(v + off, n, tid, vec != 0, row_ok, vv, valid);  // (same validity)
    const Thr th = make_thr(row_ok ? b[row] : 0.0, t);
    float ax[E];
    float mloc = INFINITY;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        ax[e] = valid[e] ? fabsf(scaled_margin(rv[e], th)) : INFINITY;
        mloc = fminf(mloc, ax[e]);
    }
    const float mu = row_min_f<E, RT, CTA>(mloc, fred);
    // R = sum v f / sum f with weights w = exp(-(|x| - mu)) <= 1, in fp64 (v - R
    // cancels when one weight dominates, and every g is then that small);
    // f = e^{-mu} w / 2 takes the same exponential.
    float wv[E];
    double sw = 0.0, swv = 0.0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        wv[e] = valid[e] ? __expf(mu - ax[e]) : 0.f;
        sw += (double)wv[e];
        swv += (double)wv[e] * (double)vv[e];
    }
    sw = row_sum_d<E, RT, CTA>(sw, dred);
    swv = row_sum_d<E, RT, CTA>(swv, dred);
    const double R = swv / sw;
    const float scale = 0.5f * __expf(-mu) * th.inv_t;
    float gv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) gv[e] = scale * wv[e] * (float)((double)vv[e] - R);
    store_row<E>(g + off, n, tid, vec != 0, row_ok, gv);
}

template <int E, int RT, int CTA, class In>
cudaError_t launch_fwd(const In* r, int64_t ld, float* p, double* b, double* sumf, int64_t B,
                       int n, double k, const double* k_rows, double t, WsHeader* hdr, int vec,
                       const SelectOut& sel, cudaStream_t st) {
    using S = Shape<E, RT, CTA>;
    const int64_t grid = (B + S::ROWS - 1) / S::ROWS;
    {
        ProfScope ps_("onchip_fwd", st);
        onchip_forward_kernel<E, RT, CTA, In>
        <<<(unsigned)grid, CTA, 0, st>>>(r, ld, p, b, sumf, B, n, k, k_rows, t, hdr, vec, sel);
    }
    return cudaGetLastError();
}

template <int E, int RT, int CTA, class In>
cudaError_t launch_bwd(const In* r, int64_t ld, const double* b, const float* v, float* g,
                       int64_t B, int n, double t, int vec, cudaStream_t st) {
    using S = Shape<E, RT, CTA>;
    const int64_t grid = (B + S::ROWS - 1) / S::ROWS;
    {
        ProfScope ps_("onchip_bwd", st);
        onchip_backward_kernel<E, RT, CTA, In><<<(unsigned)grid, CTA, 0, st>>>(r, ld, b, v, g, B, n, t, vec);
    }
    return cudaGetLastError();
}

template <int E, class In>
cudaError_t launch_search(const In* r, int64_t ld, float* p, double* b, double* sumf, int64_t B,
                          int n, double k, const double* k_rows, double t, WsHeader* hdr, int vec,
                          const SelectOut& sel, int search, cudaStream_t st) {
    const int64_t grid = (B + 7) / 8;
    {
        ProfScope ps_("onchip_search", st);
        // search == 2: no segment steps, every row goes to the sort (a test switch)
        onchip_search_kernel<E, In><<<(unsigned)grid, 256, 0, st>>>(
            r, ld, p, b, sumf, B, n, k, k_rows, t, hdr, vec, sel, search == 2 ? 0 : kSearchSteps);
    }
    return cudaGetLastError();
}

template <class In>
cudaError_t onchip_forward_any(const In* r, int64_t ld, float* p, double* b, double* sumf,
                               int64_t B, int n, double k, const double* k_rows, double t,
                               WsHeader* hdr, int vec, const SelectOut& sel, int search,
                               cudaStream_t st) {
    if (search) {
        switch (onchip_npad(n)) {
            case 32: return launch_search<1, In>(r, ld, p, b, sumf, B, n, k, k_rows, t, hdr, vec, sel, search, st);
            case 64: return launch_search<2, In>(r, ld, p, b, sumf, B, n, k, k_rows, t, hdr, vec, sel, search, st);
            case 128: return launch_search<4, In>(r, ld, p, b, sumf, B, n, k, k_rows, t, hdr, vec, sel, search, st);
            case 256: return launch_search<8, In>(r, ld, p, b, sumf, B, n, k, k_rows, t, hdr, vec, sel, search, st);
            default: break;  // longer rows: the sort
        }
    }
    switch (onchip_npad(n)) {
        case 32: return launch_fwd<1, 32, 256, In>(r, ld, p, b, sumf, B, n, k, k_rows, t, hdr, vec, sel, st);
        case 64: return launch_fwd<2, 32, 256, In>(r, ld, p, b, sumf, B, n, k, k_rows, t, hdr, vec, sel, st);
        case 128: return launch_fwd<4, 32, 256, In>(r, ld, p, b, sumf, B, n, k, k_rows, t, hdr, vec, sel, st);
        case 256: return launch_fwd<8, 32, 256, In>(r, ld, p, b, sumf, B, n, k, k_rows, t, hdr, vec, sel, st);
        case 512: return launch_fwd<8, 64, 256, In>(r, ld, p, b, sumf, B, n, k, k_rows, t, hdr, vec, sel, st);
        case 1024: return launch_fwd<8, 128, 256, In>(r, ld, p, b, sumf, B, n, k, k_rows, t, hdr, vec, sel, st);
        case 2048: return launch_fwd<8, 256, 256, In>(r, ld, p, b, sumf, B, n, k, k_rows, t, hdr, vec, sel, st);
        case 4096: return launch_fwd<8, 512, 512, In>(r, ld, p, b, sumf, B, n, k, k_rows, t, hdr, vec, sel, st);
        default: return cudaErrorInvalidValue;
    }
}

template <int E, int RT, int CTA>
cudaError_t launch_hard(const float* r, int64_t ld, float* p, double* b, int64_t B, int n,
                        double k, int rank, WsHeader* hdr, int vec, cudaStream_t st) {
    using S = Shape<E, RT, CTA>;
    const int64_t grid = (B + S::ROWS - 1) / S::ROWS;
    {
        ProfScope ps_("onchip_hard", st);
        onchip_hard_kernel<E, RT, CTA><<<(unsigned)grid, CTA, 0, st>>>(r, ld, p, b, B, n, k, rank,
                                                                       hdr, vec);
    }
    return cudaGetLastError();
}

template <class In>
cudaError_t onchip_backward_any(const In* r, int64_t ld, const double* b, const float* v, float* g,
                                int64_t B, int n, double t, int vec, cudaStream_t st) {
    switch (onchip_npad(n)) {
        case 32: return launch_bwd<1, 32, 256, In>(r, ld, b, v, g, B, n, t, vec, st);
        case 64: return launch_bwd<2, 32, 256, In>(r, ld, b, v, g, B, n, t, vec, st);
        case 128: return launch_bwd<4, 32, 256, In>(r, ld, b, v, g, B, n, t, vec, st);
        case 256: return launch_bwd<8, 32, 256, In>(r, ld, b, v, g, B, n, t, vec, st);
        case 512: return launch_bwd<8, 64, 256, In>(r, ld, b, v, g, B, n, t, vec, st);
        case 1024: return launch_bwd<8, 128, 256, In>(r, ld, b, v, g, B, n, t, vec, st);
        case 2048: return launch_bwd<8, 256, 256, In>(r, ld, b, v, g, B, n, t, vec, st);
        case 4096: return launch_bwd<8, 512, 512, In>(r, ld, b, v, g, B, n, t, vec, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

int onchip_npad(int64_t n) {
    int np = 32;
    while (np < n) np <<= 1;
    return np;
}

cudaError_t launch_onchip_forward(const float* r, int64_t ld, float* p, double* b, double* sumf,
                                  int64_t B, int n, double k, const double* k_rows, double t,
                                  WsHeader* hdr, int vec, int search, cudaStream_t st) {
    return onchip_forward_any<float>(r, ld, p, b, sumf, B, n, k, k_rows, t, hdr, vec,
                                     SelectOut{nullptr, nullptr, nullptr, 0, 0.f}, search, st);
}

cudaError_t launch_onchip_backward(const float* r, int64_t ld, const double* b, const float* v,
                                   float* g, int64_t B, int n, double t, int vec, cudaStream_t st) {
    return onchip_backward_any<float>(r, ld, b, v, g, B, n, t, vec, st);
}

cudaError_t launch_onchip_hard(const float* r, int64_t ld, float* p, double* b, int64_t B, int n,
                               double k, WsHeader* hdr, int vec, cudaStream_t st) {
    const int rank = (int)ceil(k);
    switch (onchip_npad(n)) {
        case 32: return launch_hard<1, 32, 256>(r, ld, p, b, B, n, k, rank, hdr, vec, st);
        case 64: return launch_hard<2, 32, 256>(r, ld, p, b, B, n, k, rank, hdr, vec, st);
        case 128: return launch_hard<4, 32, 256>(r, ld, p, b, B, n, k, rank, hdr, vec, st);
        case 256: return launch_hard<8, 32, 256>(r, ld, p, b, B, n, k, rank, hdr, vec, st);
        case 512: return launch_hard<8, 64, 256>(r, ld, p, b, B, n, k, rank, hdr, vec, st);
        case 1024: return launch_hard<8, 128, 256>(r, ld, p, b, B, n, k, rank, hdr, vec, st);
        case 2048: return launch_hard<8, 256, 256>(r, ld, p, b, B, n, k, rank, hdr, vec, st);
        case 4096: return launch_hard<8, 512, 512>(r, ld, p, b, B, n, k, rank, hdr, vec, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_onchip_router(const void* r, int dtype, int64_t ld, float* p, double* b,
                                 double* sumf, int64_t B, int n, double k, double t, WsHeader* hdr,
                                 int vec, int32_t* sel_idx, float* sel_val, int32_t* sel_cnt,
                                 int cap, float eps, int search, cudaStream_t st) {
    const SelectOut sel{sel_idx, sel_val, sel_cnt, cap, eps};
    if (dtype == LAPSUM_DTYPE_BF16)
        return onchip_forward_any<uint16_t>(static_cast<const uint16_t*>(r), ld, p, b, sumf, B,
                                            n, k, nullptr, t, hdr, vec, sel, search, st);
    if (dtype == LAPSUM_DTYPE_F16)
        return onchip_forward_any<F16Bits>(static_cast<const F16Bits*>(r), ld, p, b, sumf, B, n,
                                           k, nullptr, t, hdr, vec, sel, search, st);
    return onchip_forward_any<float>(static_cast<const float*>(r), ld, p, b, sumf, B, n, k,
                                     nullptr, t, hdr, vec, sel, search, st);
}

cudaError_t launch_onchip_backward_router(const void* r, int dtype, int64_t ld, const double* b,
                                          const float* v, float* g, int64_t B, int n, double t,
                                          int vec, cudaStream_t st) {
    if (dtype == LAPSUM_DTYPE_BF16)
        return onchip_backward_any<uint16_t>(static_cast<const uint16_t*>(r), ld, b, v, g, B, n, t,
                                             vec, st);
    if (dtype == LAPSUM_DTYPE_F16)
        return onchip_backward_any<F16Bits>(static_cast<const F16Bits*>(r), ld, b, v, g, B, n, t,
                                            vec, st);
    return onchip_backward_any<float>(static_cast<const float*>(r), ld, b, v, g, B, n, t, vec, st);
}

}  // namespace lapsum
