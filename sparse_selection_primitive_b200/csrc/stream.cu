// Streaming elementwise kernels over long rows: emission of p and the VJP.
//
// "Fast LapSum: Exact Differentiable Top-k at Million Scale" (gist.science
// explainer pages), section 2.1: p_i = sigma((r_i - b)/t) and an analytic
// VJP.  The VJP used is g_i = (f_i/t)(v_i - R), R = sum_j v_j f_j / sum_j f_j,
// f_i = 0.5 exp(-|r_i - b|/t) (implicit differentiation of sum_i p_i = k).
//
// Each CTA owns a 4096-element tile of one row (256 threads, 16 elements per
// thread as 4 striped float4 accesses, so every warp access is 512 contiguous
// bytes).  Per-row reductions go through per-tile partials in the workspace;
// the last CTA of a row (atomic ticket) combines them in tile order, so the
// row results are deterministic.  No CTA ever waits for another.
#include <cuda_fp16.h>

#include <type_traits>

#include "lapsum_common.cuh"
#include "lapsum_kernels.h"
#include "stream_common.cuh"

namespace lapsum {
namespace {

using namespace stream_detail;

// p = sigma((r - b)/t) for one 4096-score tile per CTA; sum f per row when
// asked for (per-tile partials, combined in tile order by the row's last CTA).
// Full tiles take unchecked 16-byte accesses.
//
// With SUP, every score with |x| <= 90 (the only ones whose f is not 0 in
// fp32) is also listed in the gradient support: each warp appends
// (position in the tile, x) to its own share of the tile's list, in a fixed
// order, and records how many it found (a count above the share's capacity
// marks an overflow; the backward then recomputes the row densely).
template <bool VEC, bool SUMF, bool SUP>
__global__ void __launch_bounds__(kThreads, SUP ? 6 : 1) emit_kernel(const float* __restrict__ r, int64_t ld,
                                                        float* __restrict__ p,
                                                        const double* __restrict__ b,
                                                        double* __restrict__ sumf, int64_t n,
                                                        double t, double* __restrict__ partials,
                                                        uint32_t* __restrict__ tickets,
                                                        WsHeader* hdr, int record_call,
                                                        int64_t B_total, int path_code,
                                                        SupportView sup) {
    pdl_wait();
    __shared__ double red[kThreads / 32];
    __shared__ int flag;
    const int64_t row = blockIdx.y;
    if (record_call && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
        hdr->last_B = B_total;
        hdr->last_n = n;
        hdr->last_path = (uint32_t)path_code;
        if (SUP) {
            sup.hdr[0] = n;
            sup.hdr[1] = B_total;
        }
    }
    const int64_t tiles = gridDim.x;
    const int64_t base = (int64_t)blockIdx.x * kStreamTile;
    const double brow = b[row];
    const Thr th = make_thr(brow, t);
    const float* rr = r + row * ld;
    float* pr = p + row * ld;
    double sf = 0.0;
    // gradient support of this warp's share of the tile: the margins are
    // staged in shared memory with a near mask per thread; a warp with near
    // scores then writes them (lane by lane, at scan offsets) to its share
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __shared__ __align__(16) float mstage[SUP ? kThreads * kPer : 1];
    float* stg = mstage + (SUP ? warp * 32 * kPer : 0);
    const int64_t share = (row * tiles + blockIdx.x) * kSupWarps + warp;
    uint32_t nm = 0u;  // near mask of this thread's 16 scores
    bool near50 = false;  // some score with |x| <= 50 (the support serves the row)
    if (SUP && blockIdx.x == 0 && threadIdx.x == 0) sup.b[row] = brow;
    // Soft rows (t not small against |b|) form p in fp64 and round it once,
    // so that sums of very many soft p stay on budget (fp32 margins and
    // exponentials leave errors of a fraction of an ulp that do not average
    // out over 10^6 scores); sharp rows keep the fp32 forms.  Two copies of
    // the tile loop, chosen once per row.
    const double inv_td = 1.0 / t;
    auto tile = [&](auto soft_tag) {
        constexpr bool SOFT = decltype(soft_tag)::value;
        // margin, e^{-|margin|} and p of one score
        auto mep = [&](float x, float& e, float& pv) {
            if (SOFT) {
                const double xd = ((double)x - brow) * inv_td;
                const double ed = exp(-fabs(xd));
                e = (float)ed;
                pv = (float)(xd < 0.0 ? 0.5 * ed : 1.0 - 0.5 * ed);
                return (float)xd;
            }
            const float m = scaled_margin_it(x, th);
            e = neg_abs_exp(m);
            pv = cdf_from(m, e);
            return m;
        };
        if (VEC && base + kStreamTile <= n) {
            const float4* r4 = reinterpret_cast<const float4*>(rr + base);
            float4* p4 = reinterpret_cast<float4*>(pr + base);
            float4 x[kPer / 4];
#pragma unroll
            for (int q = 0; q < kPer / 4; ++q) x[q] = __ldcs(r4 + q * kThreads + threadIdx.x);
#pragma unroll
            for (int q = 0; q < kPer / 4; ++q) {
                float e0, e1, e2, e3;
                float4 pq;
                const float m0 = mep(x[q].x, e0, pq.x), m1 = mep(x[q].y, e1, pq.y);
                const float m2 = mep(x[q].z, e2, pq.z), m3 = mep(x[q].w, e3, pq.w);
                __stcs(p4 + q * kThreads + threadIdx.x, pq);
                if (SUMF) sf += 0.5 * (double)((e0 + e1) + (e2 + e3));
                if (SUP) {
                    near50 |= fminf(fminf(fabsf(m0), fabsf(m1)), fminf(fabsf(m2), fabsf(m3))) <= 50.f;
                    nm |= (fabsf(m0) <= kSupWindow ? 1u : 0u) << (4 * q);
                    nm |= (fabsf(m1) <= kSupWindow ? 1u : 0u) << (4 * q + 1);
                    nm |= (fabsf(m2) <= kSupWindow ? 1u : 0u) << (4 * q + 2);
                    nm |= (fabsf(m3) <= kSupWindow ? 1u : 0u) << (4 * q + 3);
                    *reinterpret_cast<float4*>(stg + stage_slot16(lane, 4 * q)) =
                        make_float4(m0, m1, m2, m3);
                }
            }
        } else {
            float x[kPer], y[kPer];
            bool ok[kPer];
            load_tile<VEC>(rr, n, base, x, ok);
#pragma unroll
            for (int q = 0; q < kPer; ++q) {
                float e;
                const float xs = mep(x[q], e, y[q]);
                if (SUMF && ok[q]) sf += 0.5 * (double)e;
                if (SUP) {
                    near50 |= ok[q] && fabsf(xs) <= 50.f;
                    nm |= ((ok[q] && fabsf(xs) <= kSupWindow) ? 1u : 0u) << q;
                    stg[stage_slot16(lane, q)] = xs;
                }
            }
            store_tile<VEC>(pr, n, base, y);
        }
    };
    if (soft_row(brow, t)) tile(std::true_type{});
    else tile(std::false_type{});
    uint32_t cnt = 0;  // warp-uniform: entries found in this warp's share
    if (SUP && __any_sync(0xffffffffu, nm != 0u)) {
        const int c = __popc(nm);
        int incl = c;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += o;
        }
        cnt = (uint32_t)__shfl_sync(0xffffffffu, incl, 31);
        __syncwarp();
        uint2* ent = sup.ent + share * kSupCap;
        uint32_t at = (uint32_t)(incl - c);
        uint32_t mm = nm;
        while (mm != 0u) {  // this lane's near scores, in element order
            const int j = __ffs(mm) - 1;
            mm &= mm - 1u;
            // load_tile's element order (the same with and without float4)
            const uint32_t pos = (uint32_t)(4 * ((j >> 2) * kThreads + threadIdx.x) + (j & 3));
            if (at < (uint32_t)kSupCap)
                ent[at] = make_uint2(pos, __float_as_uint(stg[stage_slot16(lane, j)]));
            ++at;
        }
    }
    if (SUP) {
        // the row's flags for the backward (set once: a read before each OR)
        const bool any50 = __any_sync(0xffffffffu, near50);
        if (lane == 0) {
            sup.cnt[share] = cnt;
            const uint32_t want = (any50 ? kSupNear : 0u) | (cnt > (uint32_t)kSupCap ? kSupOverflow : 0u);
            if (want != 0u && (__ldcg(sup.flags + row) & want) != want) atomicOr(sup.flags + row, want);
        }
    }
    if (!SUMF) return;
    sf = block_sum_d(sf, red);
    if (threadIdx.x == 0) partials[row * tiles + blockIdx.x] = sf;
    if (last_block_of_row(&tickets[row], (uint32_t)tiles, &flag)) {
        double s = 0.0;
        for (int64_t i = threadIdx.x; i < tiles; i += kThreads) s += partials[row * tiles + i];
        s = block_sum_d(s, red);
        if (threadIdx.x == 0) sumf[row] = s;
    }
}

// Pass 1 of the VJP.  Each CTA walks a strided share of the row's float4
// groups with the online sums (mu, S, Sv); the CTA then reduces to one record,
// and the last CTA of the row combines the records in CTA order into
// R = Sv / S.
template <bool VEC>
__global__ void __launch_bounds__(kThreads) bwd_reduce_kernel(
    const float* __restrict__ r, int64_t ld, const double* __restrict__ b,
    const float* __restrict__ v, int64_t n, double t, double* __restrict__ partials,
    double* __restrict__ row_R, uint32_t* __restrict__ tickets,
    const uint32_t* __restrict__ need, double* __restrict__ rec_out) {
    pdl_wait();
    __shared__ double red[kThreads / 32];
    __shared__ float fred[kThreads / 32];
    __shared__ int flag;
    const int64_t row = blockIdx.y;
    if (need != nullptr && need[row] == 0u) return;  // the whole row skips
    const int64_t nblk = gridDim.x;
    const Thr th = make_thr(b[row], t);
    const float* rr = r + row * ld;
    const float* vr = v + row * ld;
    float mu = INFINITY;
    double s = 0.0, sv = 0.0;
    const int64_t stride = nblk * kThreads;
    const int64_t gt = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if constexpr (VEC) {
        const int64_t n4 = n >> 2;
        const float4* r4 = reinterpret_cast<const float4*>(rr);
        const float4* v4 = reinterpret_cast<const float4*>(vr);
        int64_t i = gt;
        // four (r, v) float4 pairs in flight per thread
        for (; i + 3 * stride < n4; i += 4 * stride) {
            float4 x[4], y[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                x[q] = __ldcs(r4 + i + q * stride);
                y[q] = __ldcs(v4 + i + q * stride);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
                online_add4(fabsf(scaled_margin(x[q].x, th)), fabsf(scaled_margin(x[q].y, th)),
                            fabsf(scaled_margin(x[q].z, th)), fabsf(scaled_margin(x[q].w, th)),
                            y[q].x, y[q].y, y[q].z, y[q].w, mu, s, sv);
        }
        for (; i < n4; i += stride) {
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
    // CTA record: rescale every thread to the CTA minimum, then sum.
    const float mb = block_min_f(mu, fred);
    const double sc = (mu == INFINITY) ? 0.0 : exp((double)mb - (double)mu);
    s = block_sum_d(s * sc, red);
    sv = block_sum_d(sv * sc, red);
    if (threadIdx.x == 0) {
        double* pr = partials + (row * nblk + blockIdx.x) * 4;
        pr[0] = (double)mb;
        pr[1] = s;
        pr[2] = sv;
    }
    if (last_block_of_row(&tickets[row], (uint32_t)nblk, &flag)) {
        float mloc = INFINITY;
        for (int64_t i = threadIdx.x; i < nblk; i += kThreads)
            mloc = fminf(mloc, (float)partials[(row * nblk + i) * 4]);
        const double mrow = (double)block_min_f(mloc, fred);
        double a = 0.0, av = 0.0;
        for (int64_t i = threadIdx.x; i < nblk; i += kThreads) {
            const double* pr = partials + (row * nblk + i) * 4;
            if (pr[0] == INFINITY) continue;
            const double f = exp(mrow - pr[0]);
            a += pr[1] * f;
            av += pr[2] * f;
        }
        a = block_sum_d(a, red);
        av = block_sum_d(av, red);
        if (threadIdx.x == 0) {
            row_R[row] = av / a;
            if (rec_out != nullptr) {  // the row's record (min |x|, S, Sv), unreduced
                rec_out[0] = mrow;
                rec_out[1] = a;
                rec_out[2] = av;
            }
        }
    }
}

// Pass 2 of the VJP: g = (f/t)(v - R), persistent CTAs striding over tiles.
template <bool VEC>
__global__ void __launch_bounds__(kThreads) bwd_apply_kernel(
    const float* __restrict__ r, int64_t ld, const double* __restrict__ b,
    const float* __restrict__ v, float* __restrict__ g, int64_t n, double t,
    const double* __restrict__ row_R, const uint32_t* __restrict__ need) {
    pdl_wait();
    const int64_t row = blockIdx.y;
    if (need != nullptr && need[row] == 0u) return;
    const Thr th = make_thr(b[row], t);
    const double R = row_R[row];
    const int64_t tiles = (n + kStreamTile - 1) / kStreamTile;
    for (int64_t T = blockIdx.x; T < tiles; T += gridDim.x) {
        const int64_t base = T * kStreamTile;
        float x[kPer], vv[kPer], y[kPer];
        bool ok[kPer];
        load_tile<VEC>(r + row * ld, n, base, x, ok);
        load_tile<VEC>(v + row * ld, n, base, vv, ok);
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const float f = 0.5f * neg_abs_exp(scaled_margin(x[q], th));
            y[q] = f * th.inv_t * (float)((double)vv[q] - R);
        }
        store_tile<VEC>(g + row * ld, n, base, y);
    }
}

// Gradients of L = sum v p with respect to k and t, per row (implicit
// derivatives of the budget equation, "Fast LapSum" pages section 2.1):
//   dL/dk = sum v f / sum f,   dL/dt = -(1/t) sum_i v_i f_i (x_i - xbar),
//   xbar = sum f x / sum f,  x = (r - b)/t,  f = 0.5 exp(-|x|).
// One pass over (r, v): each thread keeps (mu, S, Sv, Sx, Svx) with weights
// w = exp(-(|x| - mu)), mu its smallest |x| so far (a smaller one rescales the
// sums once); CTA records of 8 doubles are combined in CTA order by the row's
// last CTA.
__device__ __forceinline__ void kt_add(float a, float x, float vv, float& mu, double& s0,
                                       double& s1, double& s2, double& s3) {
    if (a < mu) {
        const double sc = (mu == INFINITY) ? 0.0 : (double)__expf(a - mu);
        s0 *= sc;
        s1 *= sc;
        s2 *= sc;
        s3 *= sc;
        mu = a;
    }
    const float w = __expf(mu - a);
    s0 += (double)w;
    s1 += (double)(w * vv);
    s2 += (double)(w * x);
    s3 += (double)(w * vv * x);
}

template <bool VEC>
__global__ void __launch_bounds__(kThreads) bwd_kt_kernel(
    const float* __restrict__ r, int64_t ld, const double* __restrict__ b,
    const float* __restrict__ v, int64_t n, double t, double* __restrict__ partials,
    uint32_t* __restrict__ tickets, double* __restrict__ g_k, double* __restrict__ g_t) {
    pdl_wait();
    __shared__ double red[kThreads / 32];
    __shared__ float fred[kThreads / 32];
    __shared__ int flag;
    const int64_t row = blockIdx.y;
    const int64_t nblk = gridDim.x;
    const Thr th = make_thr(b[row], t);
    const float* rr = r + row * ld;
    const float* vr = v + row * ld;
    float mu = INFINITY;
    double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
    const int64_t stride = nblk * kThreads;
    const int64_t gt0 = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    auto one = [&](float rv, float vv) {
        const float x = scaled_margin(rv, th);
        kt_add(fabsf(x), x, vv, mu, s0, s1, s2, s3);
    };
    if constexpr (VEC) {
        const int64_t n4 = n >> 2;
        const float4* r4 = reinterpret_cast<const float4*>(rr);
        const float4* v4 = reinterpret_cast<const float4*>(vr);
        for (int64_t i = gt0; i < n4; i += stride) {
            const float4 x = __ldcs(r4 + i), y = __ldcs(v4 + i);
            one(x.x, y.x);
            one(x.y, y.y);
            one(x.z, y.z);
            one(x.w, y.w);
        }
        for (int64_t j = (n4 << 2) + gt0; j < n; j += stride) one(rr[j], vr[j]);
    } else {
        for (int64_t j = gt0; j < n; j += stride) one(rr[j], vr[j]);
    }
    const float mb = block_min_f(mu, fred);
    const double sc = (mu == INFINITY) ? 0.0 : exp((double)mb - (double)mu);
    s0 = block_sum_d(s0 * sc, red);
    s1 = block_sum_d(s1 * sc, red);
    s2 = block_sum_d(s2 * sc, red);
    s3 = block_sum_d(s3 * sc, red);
    if (threadIdx.x == 0) {
        double* pr = partials + (row * nblk + blockIdx.x) * 8;
        pr[0] = (double)mb;
        pr[1] = s0;
        pr[2] = s1;
        pr[3] = s2;
        pr[4] = s3;
    }
    if (last_block_of_row(&tickets[row], (uint32_t)nblk, &flag)) {
        float mloc = INFINITY;
        for (int64_t i = threadIdx.x; i < nblk; i += kThreads)
            mloc = fminf(mloc, (float)partials[(row * nblk + i) * 8]);
        const double mrow = (double)block_min_f(mloc, fred);
        double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
        for (int64_t i = threadIdx.x; i < nblk; i += kThreads) {
            const double* pr = partials + (row * nblk + i) * 8;
            if (pr[0] == INFINITY) continue;
            const double f = exp(mrow - pr[0]);
            a0 += pr[1] * f;
            a1 += pr[2] * f;
            a2 += pr[3] * f;
            a3 += pr[4] * f;
        }
        a0 = block_sum_d(a0, red);
        a1 = block_sum_d(a1, red);
        a2 = block_sum_d(a2, red);
        a3 = block_sum_d(a3, red);
        if (threadIdx.x == 0) {
            if (g_k) g_k[row] = a1 / a0;
            if (g_t) g_t[row] = -(1.0 / t) * 0.5 * exp(-mrow) * (a3 - a1 * a2 / a0);
        }
    }
}

// Exact widening of 16-bit scores to fp32: 8 scores per thread per trip
// (16-byte loads, two 16-byte stores) where the row allows, else one by one.
template <int DT>
__device__ __forceinline__ float widen1(uint16_t h) {
    if constexpr (DT == LAPSUM_DTYPE_BF16) return __uint_as_float((uint32_t)h << 16);
    else return __half2float(__ushort_as_half(h));
}
template <int DT>
__global__ void __launch_bounds__(kThreads) widen_kernel(const uint16_t* __restrict__ src,
                                                         int64_t ld, int64_t n, int vec,
                                                         float* __restrict__ dst) {
    const int64_t row = blockIdx.y;
    const uint16_t* s = src + row * ld;
    float* d = dst + row * ld;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    const int64_t gt = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (vec) {
        const int64_t n8 = n >> 3;
        for (int64_t i = gt; i < n8; i += stride) {
            const uint4 u = __ldcs(reinterpret_cast<const uint4*>(s) + i);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
            float y[8];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                y[2 * h] = widen1<DT>((uint16_t)(w[h] & 0xffffu));
                y[2 * h + 1] = widen1<DT>((uint16_t)(w[h] >> 16));
            }
            float4* d4 = reinterpret_cast<float4*>(d) + 2 * i;
            __stcs(d4, make_float4(y[0], y[1], y[2], y[3]));
            __stcs(d4 + 1, make_float4(y[4], y[5], y[6], y[7]));
        }
        for (int64_t j = (n8 << 3) + gt; j < n; j += stride) d[j] = widen1<DT>(s[j]);
    } else {
        for (int64_t j = gt; j < n; j += stride) d[j] = widen1<DT>(s[j]);
    }
}

// R of a row split over devices: the shards' records (min |x|, S, Sv)
// merged in shard order.
__global__ void vjp_combine_kernel(const double* __restrict__ recs, int world,
                                   double* __restrict__ R) {
    double mrow = INFINITY;
    for (int w = 0; w < world; ++w) mrow = fmin(mrow, recs[3 * w]);
    double a = 0.0, av = 0.0;
    for (int w = 0; w < world; ++w) {
        if (recs[3 * w] == INFINITY) continue;
        const double f = exp(mrow - recs[3 * w]);
        a += recs[3 * w + 1] * f;
        av += recs[3 * w + 2] * f;
    }
    *R = av / a;
}

}  // namespace

int64_t stream_tiles(int64_t n) { return (n + kStreamTile - 1) / kStreamTile; }

size_t vjp_shard_workspace_bytes() {
    return 256 + (size_t)device_sm_count() * 8 * 4 * sizeof(double) + 256;
}

cudaError_t launch_vjp_partial(const float* r, const double* b, const float* v, int64_t n,
                               double t, double* rec, void* ws, cudaStream_t st) {
    char* w = static_cast<char*>(ws);
    uint32_t* ticket = reinterpret_cast<uint32_t*>(w);
    double* row_R = reinterpret_cast<double*>(w + 64);
    double* partials = reinterpret_cast<double*>(w + 256);
    int64_t per_row = (int64_t)device_sm_count() * 8;
    if (per_row > stream_tiles(n)) per_row = stream_tiles(n);
    if (per_row < 1) per_row = 1;
    const int vec = ((reinterpret_cast<uintptr_t>(r) | reinterpret_cast<uintptr_t>(v)) & 15u) == 0;
    if (vec)
        bwd_reduce_kernel<true><<<(unsigned)per_row, kThreads, 0, st>>>(
            r, n, b, v, n, t, partials, row_R, ticket, nullptr, rec);
    else
        bwd_reduce_kernel<false><<<(unsigned)per_row, kThreads, 0, st>>>(
            r, n, b, v, n, t, partials, row_R, ticket, nullptr, rec);
    return cudaGetLastError();
}

cudaError_t launch_vjp_apply(const float* r, const double* b, const float* v, float* g, int64_t n,
                             double t, const double* recs, int world, void* ws, cudaStream_t st) {
    double* R = reinterpret_cast<double*>(static_cast<char*>(ws) + 128);
    vjp_combine_kernel<<<1, 1, 0, st>>>(recs, world, R);
    int64_t grid = (int64_t)device_sm_count() * 16;
    if (grid > stream_tiles(n)) grid = stream_tiles(n);
    if (grid < 1) grid = 1;
    const int vec = ((reinterpret_cast<uintptr_t>(r) | reinterpret_cast<uintptr_t>(v) |
                      reinterpret_cast<uintptr_t>(g)) & 15u) == 0;
    if (vec)
        bwd_apply_kernel<true><<<(unsigned)grid, kThreads, 0, st>>>(r, n, b, v, g, n, t, R, nullptr);
    else
        bwd_apply_kernel<false><<<(unsigned)grid, kThreads, 0, st>>>(r, n, b, v, g, n, t, R,
                                                                    nullptr);
    return cudaGetLastError();
}

cudaError_t launch_emit_p(const float* r, float* p, const double* b, int64_t n, double t,
                          cudaStream_t st) {
    const int vec = ((reinterpret_cast<uintptr_t>(r) | reinterpret_cast<uintptr_t>(p)) & 15u) == 0;
    const dim3 grid((unsigned)stream_tiles(n), 1u);
    if (vec)
        emit_kernel<true, false, false><<<grid, kThreads, 0, st>>>(
            r, n, p, b, nullptr, n, t, nullptr, nullptr, nullptr, 0, 1, 0, SupportView{});
    else
        emit_kernel<false, false, false><<<grid, kThreads, 0, st>>>(
            r, n, p, b, nullptr, n, t, nullptr, nullptr, nullptr, 0, 1, 0, SupportView{});
    return cudaGetLastError();
}

cudaError_t launch_widen(const void* src, int dtype, int64_t ld, int64_t B, int64_t n, float* dst,
                         cudaStream_t st) {
    // 16-byte accesses when both rows start on 16-byte boundaries throughout
    const int vec = ((reinterpret_cast<uintptr_t>(src) & 15u) == 0 &&
                     (reinterpret_cast<uintptr_t>(dst) & 15u) == 0 && (ld % 8) == 0)
                        ? 1
                        : 0;
    int64_t per_row = ((int64_t)device_sm_count() * 8 + B - 1) / B;
    const int64_t need = (n / 8 + kThreads - 1) / kThreads;
    if (per_row > need) per_row = need;
    if (per_row < 1) per_row = 1;
    const dim3 grid((unsigned)per_row, (unsigned)B);
    ProfScope ps_("widen", st);
    const uint16_t* s = static_cast<const uint16_t*>(src);
    if (dtype == LAPSUM_DTYPE_BF16)
        widen_kernel<LAPSUM_DTYPE_BF16><<<grid, kThreads, 0, st>>>(s, ld, n, vec, dst);
    else
        widen_kernel<LAPSUM_DTYPE_F16><<<grid, kThreads, 0, st>>>(s, ld, n, vec, dst);
    return cudaGetLastError();
}

cudaError_t launch_emit(const float* r, int64_t ld, float* p, double* b, double* sumf,
                        int64_t B, int64_t n, double t, double* partials, uint32_t* tickets,
                        int vec, WsHeader* hdr, int record_call, int64_t B_total, int path_code,
                        const SupportView* sup, cudaStream_t st) {
    const dim3 grid((unsigned)stream_tiles(n), (unsigned)B);
    ProfScope ps_("emit", st);
    const SupportView sv = sup ? *sup : SupportView{};
#define LAPSUM_EMIT(V, S, U)                                                                  \
    launch_pdl(emit_kernel<V, S, U>, grid, dim3(kThreads), 0, st, r, ld, p, b, sumf, n, t,    \
               partials, tickets, hdr, record_call, B_total, path_code, sv)
    if (sup) {
        if (vec) {
            if (sumf) LAPSUM_EMIT(true, true, true);
            else LAPSUM_EMIT(true, false, true);
        } else {
            if (sumf) LAPSUM_EMIT(false, true, true);
            else LAPSUM_EMIT(false, false, true);
        }
    } else if (vec) {
        if (sumf) LAPSUM_EMIT(true, true, false);
        else LAPSUM_EMIT(true, false, false);
    } else {
        if (sumf) LAPSUM_EMIT(false, true, false);
        else LAPSUM_EMIT(false, false, false);
    }
#undef LAPSUM_EMIT
    return cudaGetLastError();
}

cudaError_t launch_backward_stream_if(const float* r, int64_t ld, const double* b,
                                      const float* v, float* g, int64_t B, int64_t n, double t,
                                      double* partials, double* row_R, uint32_t* tickets, int vec,
                                      const uint32_t* need, cudaStream_t st) {
    // pass 1 runs persistent CTAs: about 8 per SM over all rows, at most one per tile
    const int sms = device_sm_count();
    // As a fallback (need != nullptr) it usually has nothing to do: one CTA
    // per SM keeps the cost of launching it small.
    const int64_t cta_per_sm = need != nullptr ? 1 : 8;
    int64_t per_row = ((int64_t)sms * cta_per_sm + B - 1) / B;
    if (per_row > stream_tiles(n)) per_row = stream_tiles(n);
    if (per_row < 1) per_row = 1;
    const dim3 rgrid((unsigned)per_row, (unsigned)B);
    int64_t apply_row = ((int64_t)sms * (need != nullptr ? 1 : 16) + B - 1) / B;
    if (apply_row > stream_tiles(n)) apply_row = stream_tiles(n);
    if (apply_row < 1) apply_row = 1;
    const dim3 grid_apply((unsigned)apply_row, (unsigned)B);
    if (vec) {
        {
            ProfScope ps_("bwd_reduce", st);
            launch_pdl(bwd_reduce_kernel<true>, dim3(rgrid), dim3(kThreads), 0, st, r, ld, b, v, n,
                       t, partials, row_R, tickets, need, (double*)nullptr);
        }
        {
            ProfScope ps_("bwd_apply", st);
            launch_pdl(bwd_apply_kernel<true>, dim3(grid_apply), dim3(kThreads), 0, st, r, ld, b, v, g, n, t, row_R,
                                                                    need);
        }
    } else {
        {
            ProfScope ps_("bwd_reduce", st);
            launch_pdl(bwd_reduce_kernel<false>, dim3(rgrid), dim3(kThreads), 0, st, r, ld, b, v,
                       n, t, partials, row_R, tickets, need, (double*)nullptr);
        }
        {
            ProfScope ps_("bwd_apply", st);
            launch_pdl(bwd_apply_kernel<false>, dim3(grid_apply), dim3(kThreads), 0, st, r, ld, b, v, g, n, t, row_R,
                                                                     need);
        }
    }
    return cudaGetLastError();
}

cudaError_t launch_backward_stream(const float* r, int64_t ld, const double* b, const float* v,
                                   float* g, int64_t B, int64_t n, double t, double* partials,
                                   double* row_R, uint32_t* tickets, int vec, cudaStream_t st) {
    return launch_backward_stream_if(r, ld, b, v, g, B, n, t, partials, row_R, tickets, vec,
                                     nullptr, st);
}

}  // namespace lapsum

namespace lapsum {

cudaError_t launch_backward_kt(const float* r, int64_t ld, const double* b, const float* v,
                               int64_t B, int64_t n, double t, double* partials,
                               uint32_t* tickets, double* g_k, double* g_t, int vec,
                               cudaStream_t st) {
    const int sms = device_sm_count();
    // records of 8 doubles: at most half as many CTAs per row as the partials
    // region has 4-double slots per row (max(tiles, 2))
    int64_t cap = stream_tiles(n) > 2 ? stream_tiles(n) / 2 : 1;
    int64_t per_row = ((int64_t)sms * 8 + B - 1) / B;
    if (per_row > cap) per_row = cap;
    if (per_row < 1) per_row = 1;
    const dim3 grid((unsigned)per_row, (unsigned)B);
    ProfScope ps_("bwd_kt", st);
    if (vec)
        launch_pdl(bwd_kt_kernel<true>, dim3(grid), dim3(kThreads), 0, st, r, ld, b, v, n, t, partials, tickets, g_k,
                                                       g_t);
    else
        launch_pdl(bwd_kt_kernel<false>, dim3(grid), dim3(kThreads), 0, st, r, ld, b, v, n, t, partials, tickets, g_k,
                                                        g_t);
    return cudaGetLastError();
}

}  // namespace lapsum
