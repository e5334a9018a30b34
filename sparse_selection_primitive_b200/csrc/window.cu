// Windowed backward for long rows.
//
// The VJP of "Fast LapSum: Exact Differentiable Top-k at Million Scale"
// (gist.science explainer pages), section 2.1, is g_i = (f_i/t)(v_i - R) with
// f_i = 0.5 exp(-|x_i|), x_i = (r_i - b)/t and R = sum v f / sum f.  In fp32,
// f_i is exactly 0 once |x_i| > 87.4 (the exponential flushes), so g_i = 0
// there and v_i is never needed.  Only the scores inside the window
// |x| <= 90 -- a few percent of a long row -- carry any gradient.
//
// Pass A (window_pass_kernel): one read of r, tile by tile (4096 scores).
//   Where a float4 group holds window scores, that group of v is read, the
//   window terms go into an online (mu, sum w, sum w v), w = exp(-(|x| - mu)),
//   and (index, x, v) of each window score is appended to the CTA's own region
//   of the window list; a per-tile table records where each tile's entries
//   start.  The last CTA of the row forms R and decides whether the window
//   was enough.
// Pass B (window_write_kernel): g, tile by tile: the tile is zeroed in shared
//   memory, its window entries are placed, and the tile is written out with
//   coalesced 16-byte stores, so every g value is written exactly once.
//
// The window answer equals the dense one whenever the row's smallest |x| is at
// most 50: every score left out has weight below e^-40 of the largest.  When
// it is larger (t far below the gaps around b), or a CTA's list region
// overflows, the row is flagged and the dense two-pass kernels recompute it.
#include "lapsum_common.cuh"
#include "lapsum_kernels.h"

namespace lapsum {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 4096;          // scores per tile: 256 threads x 4 float4
constexpr float kWin = 90.f;         // f == 0 in fp32 beyond this |x|
constexpr float kDenseAbove = 50.f;  // row min |x| above which the dense path recomputes

__device__ __forceinline__ void win_add(float ax, float vv, float& mu, double& s, double& sv) {
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

template <bool VEC>
__global__ void __launch_bounds__(kThreads) window_pass_kernel(
    const float* __restrict__ r, int64_t ld, const double* __restrict__ b,
    const float* __restrict__ v, int64_t n, double t, WinEntry* __restrict__ list,
    uint32_t cap_cta, uint2* __restrict__ tab, uint32_t* __restrict__ wflag,
    double* __restrict__ partials, double* __restrict__ row_R, uint32_t* __restrict__ tickets) {
    pdl_wait();
    __shared__ int scnt, ovf, tstart;
    __shared__ double red[kThreads / 32];
    __shared__ float fred[kThreads / 32];
    __shared__ float qx[kThreads / 32][64];     // per-warp queue of window scores: x ...
    __shared__ uint32_t qi[kThreads / 32][64];  // ... and their positions
    __shared__ int flag;
    const int64_t row = blockIdx.y;
    const int64_t nblk = gridDim.x;
    const int64_t ntiles = (n + kTile - 1) / kTile;
    const Thr th = make_thr(b[row], t);
    const float* rr = r + row * ld;
    const float* vr = v + row * ld;
    WinEntry* region = list + (row * nblk + blockIdx.x) * (int64_t)cap_cta;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    float mu = INFINITY, amin = INFINITY;
    double s = 0.0, sv = 0.0;
    int qn = 0;  // warp-uniform queue length
    if (threadIdx.x == 0) {
        scnt = 0;
        ovf = 0;
    }
    // Window scores are a few percent of a long row: they are queued per warp
    // and handled 32 at a time (v gather, weight, list entry), so the warp's
    // lanes stay busy on them however sparse they are.
    auto drain = [&](int cnt) {
        const bool ok = lane < cnt;
        const uint32_t idx = ok ? qi[warp][lane] : 0u;
        const float x = ok ? qx[warp][lane] : 0.f;
        const float vv = ok ? __ldcs(vr + idx) : 0.f;
        if (ok) win_add(fabsf(x), vv, mu, s, sv);
        int bse = 0;
        if (lane == 0) bse = atomicAdd(&scnt, cnt);
        bse = __shfl_sync(0xffffffffu, bse, 0);
        if (ok) {
            if ((uint32_t)(bse + lane) < cap_cta) region[bse + lane] = WinEntry{idx, x, vv};
            else ovf = 1;
        }
    };
    auto slot = [&](float rv, uint32_t idx, bool valid) {
        const float x = scaled_margin(rv, th);
        const float a = fabsf(x);
        if (valid) amin = fminf(amin, a);
        const bool near = valid && a <= kWin;
        const unsigned ball = __ballot_sync(0xffffffffu, near);
        if (ball) {
            if (near) {
                const int pos = qn + __popc(ball & lt);
                qx[warp][pos] = x;
                qi[warp][pos] = idx;
            }
            qn += __popc(ball);
            if (qn >= 32) {
                __syncwarp();
                drain(32);
                const float kx = lane < qn - 32 ? qx[warp][lane + 32] : 0.f;
                const uint32_t ki = lane < qn - 32 ? qi[warp][lane + 32] : 0u;
                __syncwarp();
                if (lane < qn - 32) {
                    qx[warp][lane] = kx;
                    qi[warp][lane] = ki;
                }
                __syncwarp();
                qn -= 32;
            }
        }
    };
    // full tiles' r is loaded one tile ahead, so the next loads are in flight
    // while the current tile is processed
    float4 nx4[4];
    auto load_full = [&](int64_t T, float4 (&dst)[4]) {
        const int64_t bs = T * kTile;
        if (VEC && T < ntiles && bs + kTile <= n) {
            const float4* r4 = reinterpret_cast<const float4*>(rr + bs);
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[q] = __ldcs(r4 + q * kThreads + threadIdx.x);
        }
    };
    load_full(blockIdx.x, nx4);
    for (int64_t T = blockIdx.x; T < ntiles; T += nblk) {
        __syncthreads();
        if (threadIdx.x == 0) tstart = scnt;
        const int64_t base = T * kTile;
        if (VEC && base + kTile <= n) {
            float4 x4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) x4[q] = nx4[q];
            load_full(T + nblk, nx4);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t i0 = (uint32_t)(base + 4 * (q * kThreads + threadIdx.x));
                slot(x4[q].x, i0, true);
                slot(x4[q].y, i0 + 1, true);
                slot(x4[q].z, i0 + 2, true);
                slot(x4[q].w, i0 + 3, true);
            }
        } else {
            for (int kk = 0; kk < kTile / kThreads; ++kk) {  // same trip count in every lane
                const int64_t j = base + kk * kThreads + threadIdx.x;
                const bool ok = j < n;
                slot(ok ? rr[j] : 0.f, (uint32_t)j, ok);
            }
        }
        __syncwarp();
        if (qn > 0) {
            drain(qn);
            qn = 0;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            const int end = scnt < (int)cap_cta ? scnt : (int)cap_cta;
            const int st = tstart < (int)cap_cta ? tstart : (int)cap_cta;
            tab[row * ntiles + T] = make_uint2((uint32_t)st, (uint32_t)(end - st));
        }
    }
    // CTA record (mu, S, Sv, min |x|), then the row's last CTA combines them
    const float mb = block_min_f(mu, fred);
    const double sc = (mu == INFINITY) ? 0.0 : exp((double)mb - (double)mu);
    s = block_sum_d(s * sc, red);
    sv = block_sum_d(sv * sc, red);
    const float am = block_min_f(amin, fred);
    if (threadIdx.x == 0) {
        double* pr = partials + (row * nblk + blockIdx.x) * 4;
        pr[0] = (double)mb;
        pr[1] = s;
        pr[2] = sv;
        pr[3] = ovf ? -1.0 : (double)am;  // -1 marks an overflowed region
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t prev = atomicAdd(&tickets[row], 1u);
        flag = (prev == (uint32_t)nblk - 1u);
        if (flag) tickets[row] = 0u;
    }
    __syncthreads();
    if (!flag) return;
    __threadfence();
    float mloc = INFINITY, aloc = INFINITY;
    int bad = 0;
    for (int64_t k = threadIdx.x; k < nblk; k += kThreads) {
        const double* pr = partials + (row * nblk + k) * 4;
        mloc = fminf(mloc, (float)pr[0]);
        if (pr[3] < 0.0) bad = 1;
        else aloc = fminf(aloc, (float)pr[3]);
    }
    const double mrow = (double)block_min_f(mloc, fred);
    const float arow = block_min_f(aloc, fred);
    const int anybad = __syncthreads_or(bad);
    double a = 0.0, av = 0.0;
    for (int64_t k = threadIdx.x; k < nblk; k += kThreads) {
        const double* pr = partials + (row * nblk + k) * 4;
        if (pr[0] == INFINITY) continue;
        const double f = exp(mrow - pr[0]);
        a += pr[1] * f;
        av += pr[2] * f;
    }
    a = block_sum_d(a, red);
    av = block_sum_d(av, red);
    if (threadIdx.x == 0) {
        row_R[row] = a > 0.0 ? av / a : 0.0;
        wflag[row] = (anybad || arow > kDenseAbove) ? 1u : 0u;
    }
}

// g tile by tile: zeros with coalesced 16-byte stores, then (after a block
// barrier, so they land last) the tile's window values.
template <bool VEC>
__global__ void __launch_bounds__(kThreads) window_write_kernel(
    const WinEntry* __restrict__ list, uint32_t cap_cta, int64_t pass_blocks,
    const uint2* __restrict__ tab, const uint32_t* __restrict__ wflag,
    const double* __restrict__ row_R, float* __restrict__ g, int64_t ld, int64_t n, double t) {
    pdl_wait();
    const int64_t row = blockIdx.y;
    if (wflag[row]) return;  // the dense kernels own this row
    const int64_t ntiles = (n + kTile - 1) / kTile;
    const double R = row_R[row];
    const float hinv = (float)(0.5 / t);
    float* gr = g + row * ld;
    const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t T = blockIdx.x; T < ntiles; T += gridDim.x) {
        const int64_t base = T * kTile;
        if (VEC && base + kTile <= n) {
            float4* g4 = reinterpret_cast<float4*>(gr + base);
            // plain (cache-resident) stores: the window values scattered below
            // then merge into the same L2 lines before they go to memory
#pragma unroll
            for (int q = 0; q < 4; ++q) g4[q * kThreads + threadIdx.x] = z4;
        } else {
            for (int e = threadIdx.x; e < kTile && base + e < n; e += kThreads) gr[base + e] = 0.f;
        }
        const uint2 se = tab[row * ntiles + T];
        const WinEntry* reg = list + (row * pass_blocks + T % pass_blocks) * (int64_t)cap_cta;
        __syncthreads();
        for (uint32_t k = threadIdx.x; k < se.y; k += kThreads) {
            const WinEntry e = reg[se.x + k];
            gr[e.idx] = hinv * __expf(-fabsf(e.x)) * (float)((double)e.v - R);
        }
    }
}


}  // namespace

uint32_t window_capacity(int64_t n) {
    int64_t c = n / 8;
    if (c < 4096) c = 4096;
    if (c > n) c = n;
    if (c > 0xffffffffll) c = 0xffffffffll;
    return (uint32_t)c;
}

int64_t window_tiles(int64_t n) { return (n + kTile - 1) / kTile; }

cudaError_t launch_backward_window(const float* r, int64_t ld, const double* b, const float* v,
                                   float* g, int64_t B, int64_t n, double t,
                                   const WindowBuffers& wb, double* partials, double* row_R,
                                   uint32_t* tickets, int vec, cudaStream_t st) {
    const int64_t ntiles = window_tiles(n);
    int64_t per_row = ((int64_t)device_sm_count() * 8 + B - 1) / B;
    if (per_row > ntiles) per_row = ntiles;
    if (per_row < 1) per_row = 1;
    // each pass CTA owns an equal share of the row's list capacity
    const uint32_t cap_cta = (uint32_t)(((int64_t)window_capacity(n) + per_row - 1) / per_row);
    const dim3 grid((unsigned)per_row, (unsigned)B);
    int64_t wr = ntiles < (int64_t)device_sm_count() * 8 ? ntiles : (int64_t)device_sm_count() * 8;
    const dim3 wgrid((unsigned)wr, (unsigned)B);
    {
        ProfScope ps_("window_pass", st);
        if (vec)
            launch_pdl(window_pass_kernel<true>, dim3(grid), dim3(kThreads), 0, st, r, ld, b, v, n, t, wb.list, cap_cta,
                                                                wb.tab, wb.flag, partials, row_R,
                                                                tickets);
        else
            launch_pdl(window_pass_kernel<false>, dim3(grid), dim3(kThreads), 0, st, r, ld, b, v, n, t, wb.list,
                                                                 cap_cta, wb.tab, wb.flag,
                                                                 partials, row_R, tickets);
    }
    {
        ProfScope ps_("window_write", st);
        if (vec)
            launch_pdl(window_write_kernel<true>, dim3(wgrid), dim3(kThreads), 0, st, wb.list, cap_cta, per_row, wb.tab,
                                                                  wb.flag, row_R, g, ld, n, t);
        else
            launch_pdl(window_write_kernel<false>, dim3(wgrid), dim3(kThreads), 0, st, wb.list, cap_cta, per_row,
                                                                   wb.tab, wb.flag, row_R, g, ld,
                                                                   n, t);
    }
    // rows the window could not serve: dense recompute (exits at once otherwise)
    return launch_backward_stream_if(r, ld, b, v, g, B, n, t, partials, row_R, tickets, vec,
                                     wb.flag, st);
}

}  // namespace lapsum
