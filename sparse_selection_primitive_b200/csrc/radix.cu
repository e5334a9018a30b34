// Segmented LSD radix sort of fp32 scores (as order-preserving u32 keys, no
// payload) and the per-row solve over the sorted keys.
//
// "Fast LapSum: Exact Differentiable Top-k at Million Scale" (gist.science
// explainer pages), section 2.2: the full-sort solver sorts the scores, after
// which all remaining work is linear.  p and g are elementwise in (r_i, b), so
// only the keys are sorted; no index permutation is carried.
//
// Sort structure, per 8-bit digit pass (4 passes for 32-bit keys):
//   upsweep   one CTA per 4096-key tile: digit histogram of the tile;
//   scan      exclusive scan of (digit, tile) counts per row -> scatter bases;
//   downsweep one CTA per tile: stable rank of every key inside the tile
//             (warp match + per-warp digit counters), a local reorder in
//             shared memory, then coalesced runs written to the bases.
// A prep pass converts r into keys and histograms all four digits of every
// row at once (those histograms do not depend on the key order), so a digit
// that is the same for every key of a row is known up front and its pass is
// skipped for that row.  Each row tracks which ping-pong buffer holds it.
#include "lapsum_common.cuh"
#include "lapsum_kernels.h"
#include "solve_sorted.cuh"

namespace lapsum {
namespace {

constexpr int kThreads = 256;
constexpr int kPerThread = kRadixTile / kThreads;  // 16
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// r (row stride ld) -> keys (row stride n); all-digit histograms per row.
__global__ void __launch_bounds__(kThreads) radix_prep_kernel(const float* __restrict__ r,
                                                              int64_t ld, int64_t n,
                                                              uint32_t* __restrict__ keys,
                                                              uint32_t* __restrict__ seg_hist,
                                                              RowState* rows, WsHeader* hdr) {
    __shared__ uint32_t h[4][256];
    const int64_t row = blockIdx.y;
    const int64_t base = (int64_t)blockIdx.x * kRadixTile;
    for (int i = threadIdx.x; i < 4 * 256; i += kThreads) (&h[0][0])[i] = 0;
    __syncthreads();
    bool bad = false;
    const float* rr = r + row * ld;
    uint32_t* kk = keys + row * n;
    for (int i = threadIdx.x; i < kRadixTile; i += kThreads) {
        const int64_t idx = base + i;
        if (idx < n) {
            const float x = __ldg(rr + idx);
            bad |= !finite_f(x);
            const uint32_t key = to_key(x);
            kk[idx] = key;
#pragma unroll
            for (int d = 0; d < 4; ++d) atomicAdd(&h[d][(key >> (8 * d)) & 255u], 1u);
        }
    }
    if (bad) {
        atomicOr(&rows[row].status, kDevNonFinite);
        set_status(hdr, kDevNonFinite);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 4 * 256; i += kThreads) {
        const uint32_t c = (&h[0][0])[i];
        if (c) atomicAdd(&seg_hist[row * 1024 + i], c);
    }
}

// Per row: which digits are trivial, and which buffer holds the data before
// each pass (plan[row][d], d = 0..4), plus the trivial mask in plan[row][5].
// One CTA per row, one thread per digit value.
__global__ void __launch_bounds__(256) radix_plan_kernel(const uint32_t* __restrict__ seg_hist,
                                                         int64_t B, int64_t n,
                                                         int32_t* __restrict__ plan) {
    const int64_t row = blockIdx.x;
    const uint32_t* h = seg_hist + row * 1024;
    int mask = 0;
#pragma unroll
    for (int d = 0; d < 4; ++d)
        if (__syncthreads_or((int64_t)h[d * 256 + threadIdx.x] == n)) mask |= 1 << d;
    if (threadIdx.x == 0) {
        int par = 0;
        for (int d = 0; d < 4; ++d) {
            plan[row * 8 + d] = par;
            if (!(mask & (1 << d))) par ^= 1;
        }
        plan[row * 8 + 4] = par;
        plan[row * 8 + 5] = mask;
    }
}

__global__ void __launch_bounds__(kThreads) radix_upsweep_kernel(
    const uint32_t* __restrict__ k0, const uint32_t* __restrict__ k1, int64_t n, int64_t tiles,
    int d, const int32_t* __restrict__ plan, uint32_t* __restrict__ tile_hist) {
    __shared__ uint32_t h[256];
    const int64_t row = blockIdx.y;
    if (plan[row * 8 + 5] & (1 << d)) return;
    const uint32_t* src = (plan[row * 8 + d] ? k1 : k0) + row * n;
    const int64_t base = (int64_t)blockIdx.x * kRadixTile;
    h[threadIdx.x] = 0;
    __syncthreads();
    const int shift = 8 * d;
    for (int i = threadIdx.x; i < kRadixTile; i += kThreads) {
        const int64_t idx = base + i;
        if (idx < n) atomicAdd(&h[(src[idx] >> shift) & 255u], 1u);
    }
    __syncthreads();
    tile_hist[(row * 256 + threadIdx.x) * tiles + blockIdx.x] = h[threadIdx.x];
}

// Exclusive scan over (digit, tile) of one row; one thread per digit walks the
// tiles.  Rows with many tiles use radix_scan_wide_kernel instead.
__global__ void __launch_bounds__(256) radix_scan_kernel(const uint32_t* __restrict__ seg_hist,
                                                         int64_t tiles, int d,
                                                         const int32_t* __restrict__ plan,
                                                         uint32_t* __restrict__ tile_hist) {
    __shared__ uint32_t base[256];
    const int64_t row = blockIdx.x;
    if (plan[row * 8 + 5] & (1 << d)) return;
    const int v = threadIdx.x;
    // digit bases from the row histogram (exclusive scan over 256 digits)
    uint32_t c = seg_hist[row * 1024 + d * 256 + v];
    base[v] = c;
    __syncthreads();
    for (int off = 1; off < 256; off <<= 1) {
        uint32_t add = v >= off ? base[v - off] : 0u;
        __syncthreads();
        base[v] += add;
        __syncthreads();
    }
    uint32_t run = base[v] - c;
    uint32_t* th = tile_hist + (row * 256 + v) * tiles;
    for (int64_t tI = 0; tI < tiles; ++tI) {
        const uint32_t x = th[tI];
        th[tI] = run;
        run += x;
    }
}

// Same scan for rows with many tiles: one CTA per (row, digit).
__global__ void __launch_bounds__(256) radix_scan_wide_kernel(const uint32_t* __restrict__ seg_hist,
                                                              int64_t tiles, int d,
                                                              const int32_t* __restrict__ plan,
                                                              uint32_t* __restrict__ tile_hist) {
    __shared__ uint32_t part[256];
    const int64_t row = blockIdx.y;
    const int v = blockIdx.x;
    if (plan[row * 8 + 5] & (1 << d)) return;
    uint32_t dbase = 0;
    for (int u = threadIdx.x; u < v; u += 256) dbase += seg_hist[row * 1024 + d * 256 + u];
    part[threadIdx.x] = dbase;
    __syncthreads();
    for (int off = 128; off > 0; off >>= 1) {
        if (threadIdx.x < off) part[threadIdx.x] += part[threadIdx.x + off];
        __syncthreads();
    }
    uint32_t carry = part[0];
    __syncthreads();
    uint32_t* th = tile_hist + (row * 256 + v) * tiles;
    for (int64_t c0 = 0; c0 < tiles; c0 += 256) {
        const int64_t i = c0 + threadIdx.x;
        const uint32_t x = i < tiles ? th[i] : 0u;
        part[threadIdx.x] = x;
        __syncthreads();
        for (int off = 1; off < 256; off <<= 1) {
            uint32_t add = threadIdx.x >= off ? part[threadIdx.x - off] : 0u;
            __syncthreads();
            part[threadIdx.x] += add;
            __syncthreads();
        }
        if (i < tiles) th[i] = carry + part[threadIdx.x] - x;
        carry += part[255];
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kThreads, 4) radix_downsweep_kernel(
    uint32_t* __restrict__ k0, uint32_t* __restrict__ k1, int64_t n, int64_t tiles, int d,
    const int32_t* __restrict__ plan, const uint32_t* __restrict__ tile_hist) {
    __shared__ uint32_t wcnt[kWarps][256];
    __shared__ uint32_t tstart[256];
    __shared__ uint32_t gbase[256];
    __shared__ uint32_t sorted[kRadixTile];
    const int64_t row = blockIdx.y;
    if (plan[row * 8 + 5] & (1 << d)) return;
    const int par = plan[row * 8 + d];
    const uint32_t* src = (par ? k1 : k0) + row * n;
    uint32_t* dst = (par ? k0 : k1) + row * n;
    const int64_t base = (int64_t)blockIdx.x * kRadixTile;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int shift = 8 * d;

    for (int i = threadIdx.x; i < kWarps * 256; i += kThreads) (&wcnt[0][0])[i] = 0;
    gbase[threadIdx.x] = tile_hist[(row * 256 + threadIdx.x) * tiles + blockIdx.x];
    __syncthreads();

    // Striped ownership keeps the rank stable: warp w owns keys
    // [w*512, (w+1)*512) of the tile, visited 32 at a time in index order.
    uint32_t key[kPerThread], lrank[kPerThread];
    const uint32_t lt = lanemask_lt();
    // all loads first: the warp barriers of the ranking loop below would
    // otherwise hold each load back until the previous key is ranked
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
        const int64_t idx = base + warp * (32 * kPerThread) + e * 32 + lane;
        key[e] = idx < n ? src[idx] : 0u;
    }
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
        const int64_t idx = base + warp * (32 * kPerThread) + e * 32 + lane;
        const bool ok = idx < n;
        const uint32_t dig = (key[e] >> shift) & 255u;
        const uint32_t peers = __match_any_sync(0xffffffffu, ok ? dig : 256u + lane);
        const int leader = __ffs(peers) - 1;
        uint32_t bse = 0;
        if (ok && lane == leader) {
            bse = wcnt[warp][dig];
            wcnt[warp][dig] = bse + __popc(peers);
        }
        bse = __shfl_sync(0xffffffffu, bse, leader);
        lrank[e] = bse + __popc(peers & lt);
        __syncwarp();
    }
    __syncthreads();
    // per digit: exclusive over warps, and the tile count of the digit
    {
        const int v = threadIdx.x;
        uint32_t run = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const uint32_t c = wcnt[w][v];
            wcnt[w][v] = run;
            run += c;
        }
        tstart[v] = run;
    }
    __syncthreads();
    // exclusive scan of tile digit counts -> local start of each digit
    {
        const int v = threadIdx.x;
        const uint32_t c = tstart[v];
        for (int off = 1; off < 256; off <<= 1) {
            uint32_t add = v >= off ? tstart[v - off] : 0u;
            __syncthreads();
            tstart[v] += add;
            __syncthreads();
        }
        tstart[v] -= c;
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
        const int64_t idx = base + warp * (32 * kPerThread) + e * 32 + lane;
        if (idx < n) {
            const uint32_t dig = (key[e] >> shift) & 255u;
            sorted[tstart[dig] + wcnt[warp][dig] + lrank[e]] = key[e];
        }
    }
    __syncthreads();
    const int valid = (int)min((int64_t)kRadixTile, n - base);
    for (int i = threadIdx.x; i < valid; i += kThreads) {
        const uint32_t kv = sorted[i];
        const uint32_t dig = (kv >> shift) & 255u;
        dst[gbase[dig] + (uint32_t)i - tstart[dig]] = kv;
    }
}

// One digit pass in one kernel (for rows of fewer than 2^30 keys): each CTA
// takes the next tile id from a counter, so every tile before it is already
// running; it ranks its tile as the downsweep does, publishes its digit counts
// (word = flag << 30 | count: 1 = the tile's own count, 2 = inclusive prefix
// over the row's tiles so far) and walks back over its predecessors' words
// until an inclusive one, which gives its scatter bases without an upsweep or
// a scan.  Tile 0 publishes its inclusive counts at once, so every walk ends;
// each wait is bounded and sets kDevWaitTimeout if it runs out.
constexpr uint32_t kLbAgg = 1u << 30, kLbInc = 2u << 30, kLbMask = (1u << 30) - 1u;
constexpr int kLbSpinMax = 1 << 22;

__global__ void __launch_bounds__(kThreads, 4) radix_onesweep_kernel(
    uint32_t* __restrict__ k0, uint32_t* __restrict__ k1, int64_t n, int64_t tiles, int d,
    const int32_t* __restrict__ plan, const uint32_t* __restrict__ seg_hist,
    uint32_t* __restrict__ lb, unsigned long long* __restrict__ counter, WsHeader* hdr) {
    __shared__ uint32_t wcnt[kWarps][256];
    __shared__ uint32_t tstart[256];
    __shared__ uint32_t gbase[256];
    __shared__ uint32_t sorted[kRadixTile];
    __shared__ unsigned long long s_id;
    if (threadIdx.x == 0) s_id = atomicAdd(counter, 1ull);
    __syncthreads();
    const int64_t id = (int64_t)s_id;
    const int64_t row = id / tiles, tile = id % tiles;
    if (plan[row * 8 + 5] & (1 << d)) return;  // the whole row skips this digit
    const int par = plan[row * 8 + d];
    const uint32_t* src = (par ? k1 : k0) + row * n;
    uint32_t* dst = (par ? k0 : k1) + row * n;
    const int64_t base = tile * kRadixTile;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int shift = 8 * d;
    const int v = threadIdx.x;

    for (int i = threadIdx.x; i < kWarps * 256; i += kThreads) (&wcnt[0][0])[i] = 0;
    // the row's digit bases: exclusive scan of its digit histogram
    const uint32_t hc = seg_hist[row * 1024 + d * 256 + v];
    tstart[v] = hc;
    __syncthreads();
    for (int off = 1; off < 256; off <<= 1) {
        const uint32_t add = v >= off ? tstart[v - off] : 0u;
        __syncthreads();
        tstart[v] += add;
        __syncthreads();
    }
    const uint32_t dbase = tstart[v] - hc;
    __syncthreads();

    uint32_t key[kPerThread], lrank[kPerThread];
    const uint32_t lt = lanemask_lt();
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
        const int64_t idx = base + warp * (32 * kPerThread) + e * 32 + lane;
        key[e] = idx < n ? src[idx] : 0u;
    }
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
        const int64_t idx = base + warp * (32 * kPerThread) + e * 32 + lane;
        const bool ok = idx < n;
        const uint32_t dig = (key[e] >> shift) & 255u;
        const uint32_t peers = __match_any_sync(0xffffffffu, ok ? dig : 256u + lane);
        const int leader = __ffs(peers) - 1;
        uint32_t bse = 0;
        if (ok && lane == leader) {
            bse = wcnt[warp][dig];
            wcnt[warp][dig] = bse + __popc(peers);
        }
        bse = __shfl_sync(0xffffffffu, bse, leader);
        lrank[e] = bse + __popc(peers & lt);
        __syncwarp();
    }
    __syncthreads();
    uint32_t cnt = 0;  // this tile's count of digit v
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        const uint32_t c = wcnt[w][v];
        wcnt[w][v] = cnt;
        cnt += c;
    }
    // publish, then walk back to the first inclusive word
    volatile uint32_t* words = lb + row * tiles * 256;
    words[tile * 256 + v] = (tile == 0 ? kLbInc : kLbAgg) | cnt;
    uint32_t excl = 0;
    bool timed_out = false;
    if (tile > 0) {
        int64_t j = tile - 1;
        int spins = 0;
        for (;;) {
            const uint32_t w = words[j * 256 + v];
            if ((w & ~kLbMask) == 0u) {
                if (++spins > kLbSpinMax) {
                    timed_out = true;
                    break;
                }
                continue;
            }
            excl += w & kLbMask;
            if ((w & ~kLbMask) == kLbInc || j == 0) break;
            --j;
        }
        if (!timed_out) words[tile * 256 + v] = kLbInc | (excl + cnt);
    }
    if (__syncthreads_or(timed_out)) {  // the bases are unknown: write nothing
        if (threadIdx.x == 0) set_status(hdr, kDevWaitTimeout);
        return;
    }
    gbase[v] = dbase + excl;
    tstart[v] = cnt;
    __syncthreads();
    // exclusive scan of the tile's digit counts -> local start of each digit
    for (int off = 1; off < 256; off <<= 1) {
        const uint32_t add = v >= off ? tstart[v - off] : 0u;
        __syncthreads();
        tstart[v] += add;
        __syncthreads();
    }
    tstart[v] -= cnt;
    __syncthreads();
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
        const int64_t idx = base + warp * (32 * kPerThread) + e * 32 + lane;
        if (idx < n) {
            const uint32_t dig = (key[e] >> shift) & 255u;
            sorted[tstart[dig] + wcnt[warp][dig] + lrank[e]] = key[e];
        }
    }
    __syncthreads();
    const int valid = (int)min((int64_t)kRadixTile, n - base);
    for (int i = threadIdx.x; i < valid; i += kThreads) {
        const uint32_t kv = sorted[i];
        const uint32_t dig = (kv >> shift) & 255u;
        const uint32_t pos = gbase[dig] + (uint32_t)i - tstart[dig];
        if ((int64_t)pos < n) dst[pos] = kv;
    }
}

struct KeyGet {
    const uint32_t* k;
    __device__ __forceinline__ float operator()(long long j) const { return from_key(k[j]); }
};

__global__ void __launch_bounds__(1024) rowsolve_keys_kernel(const uint32_t* __restrict__ k0,
                                                              const uint32_t* __restrict__ k1,
                                                              int64_t n, double k,
                                                              const double* __restrict__ k_rows,
                                                              double t,
                                                              const int32_t* __restrict__ plan,
                                                              double* __restrict__ b_out,
                                                              RowState* rows, WsHeader* hdr) {
    __shared__ SolveScratch sm;
    __shared__ SolveResult res;
    const int64_t row = blockIdx.x;
    const uint32_t* keys = (plan[row * 8 + 4] ? k1 : k0) + row * n;
    Tails tl{false, 0.f, 0.0, false, 0.f, 0.0, 0.0};
    // the row's budget: the shared k or its own entry of k_rows (outside (0, n): b = NaN)
    const double kr = k_rows != nullptr ? k_rows[row] : k;
    const bool k_ok = kr > 0.0 && kr < (double)n;
    solve_sorted_block<KeyGet, false, true>(KeyGet{keys}, (long long)n, tl,
                                             k_ok ? kr : 0.5 * (double)n, t, &sm, &res);
    if (threadIdx.x == 0) {
        if (!k_ok) {
            rows[row].status |= kDevBadBudget;
            set_status(hdr, kDevBadBudget);
        }
        const double b = ((rows[row].status & kDevNonFinite) || !k_ok) ? nan("") : res.b;
        rows[row].b = b;
        rows[row].path = LAPSUM_PATH_RADIX;
        rows[row].attempts = 1;
        b_out[row] = b;
    }
}

// Zero-temperature limit of a sorted row (section 2.3 of the pages: DFTopK's
// midpoint threshold is LapSum at t -> 0): c = the rank-th largest key, its
// group of equal scores [lo, hi) found by two 1024-way searches of the sorted
// keys (-0 and +0 read as one value), then b and the share of the group as in
// the on-chip kernel.  One CTA per row.
__device__ __forceinline__ uint32_t canon_key(uint32_t kk) {
    return kk == 0x7fffffffu ? 0x80000000u : kk;  // the key of -0 as the key of +0
}
// First index in [lo, hi) whose canonical key is >= target (strict: > target),
// or hi.  Every thread of the CTA calls it.
__device__ int64_t block_lower_bound(const uint32_t* __restrict__ keys, int64_t lo, int64_t hi,
                                     uint32_t target, bool strict) {
    while (hi > lo) {
        const int64_t step = (hi - lo + blockDim.x - 1) / blockDim.x;
        const int64_t pos = lo + (int64_t)threadIdx.x * step;
        bool below = false;
        if (pos < hi) {
            const uint32_t kk = canon_key(keys[pos]);
            below = strict ? kk <= target : kk < target;
        }
        const int cnt = __syncthreads_count(below);  // probes before the answer
        const int64_t nlo = cnt > 0 ? lo + (int64_t)(cnt - 1) * step + 1 : lo;
        int64_t nhi = lo + (int64_t)cnt * step;
        if (nhi > hi) nhi = hi;
        lo = nlo;
        hi = nhi;
    }
    return lo;
}

__global__ void __launch_bounds__(1024) rowhard_keys_kernel(const uint32_t* __restrict__ k0,
                                                             const uint32_t* __restrict__ k1,
                                                             int64_t n, double k, int64_t rank,
                                                             const int32_t* __restrict__ plan,
                                                             double* __restrict__ b_out,
                                                             RowState* rows) {
    const int64_t row = blockIdx.x;
    const uint32_t* keys = (plan[row * 8 + 4] ? k1 : k0) + row * n;
    const int64_t q = n - rank;
    const uint32_t ck = canon_key(keys[q]);
    const int64_t lo = block_lower_bound(keys, 0, q + 1, ck, false);
    const int64_t hi = block_lower_bound(keys, q, n, ck, true);
    if (threadIdx.x == 0) {
        const float c = from_key(ck);
        const double a = (double)(n - hi), m = (double)(hi - lo);
        double b, frac;
        if (k < a + m) {
            b = (double)c;
            frac = (k - a) / m;
        } else {  // lo >= 1 here: k = a + m < n
            b = 0.5 * ((double)c + (double)from_key(canon_key(keys[lo - 1])));
            frac = 1.0;
        }
        if (rows[row].status & kDevNonFinite) b = nan("");
        rows[row].b = b;
        rows[row].hard_c = c;
        rows[row].hard_frac = frac;
        rows[row].path = LAPSUM_PATH_RADIX;
        rows[row].attempts = 1;
        b_out[row] = b;
    }
}

// p of the zero-temperature limit: 1 above c, the share at c, 0 below; NaN rows
// stay NaN.  One CTA per 4096-score tile.
template <bool VEC>
__global__ void __launch_bounds__(kThreads) hard_emit_kernel(const float* __restrict__ r,
                                                             int64_t ld, float* __restrict__ p,
                                                             int64_t n, const RowState* rows) {
    const int64_t row = blockIdx.y;
    const RowState& rs = rows[row];
    const float c = rs.hard_c, share = (float)rs.hard_frac;
    const bool nan_row = isnan(rs.b);
    const float* rr = r + row * ld;
    float* pr = p + row * ld;
    auto one = [&](float x) {
        x += 0.f;
        return nan_row ? __int_as_float(0x7fc00000) : (x > c ? 1.f : (x == c ? share : 0.f));
    };
    const int64_t base = (int64_t)blockIdx.x * 4096;
    if (VEC && base + 4096 <= n) {
        const float4* r4 = reinterpret_cast<const float4*>(rr + base);
        float4* p4 = reinterpret_cast<float4*>(pr + base);
        for (int i = threadIdx.x; i < 1024; i += kThreads) {
            const float4 v = __ldcs(r4 + i);
            __stcs(p4 + i, make_float4(one(v.x), one(v.y), one(v.z), one(v.w)));
        }
    } else {
        for (int64_t i = base + threadIdx.x; i < base + 4096 && i < n; i += kThreads)
            pr[i] = one(rr[i]);
    }
}

}  // namespace

cudaError_t launch_rowhard_sorted_keys(const RadixBuffers& buf, int64_t B, int64_t n, double k,
                                       const float* r, int64_t ld, float* p, double* b,
                                       RowState* rows, int vec, cudaStream_t st) {
    const int64_t rank = (int64_t)ceil(k);
    {
        ProfScope ps_("rowhard", st);
        rowhard_keys_kernel<<<(unsigned)B, 1024, 0, st>>>(buf.keys[0], buf.keys[1], n, k, rank,
                                                          buf.plan, b, rows);
    }
    return launch_hard_emit(r, ld, p, B, n, rows, vec, st);
}

cudaError_t launch_hard_emit(const float* r, int64_t ld, float* p, int64_t B, int64_t n,
                             const RowState* rows, int vec, cudaStream_t st) {
    const dim3 grid((unsigned)((n + 4095) / 4096), (unsigned)B);
    ProfScope ps_("hard_emit", st);
    if (vec) hard_emit_kernel<true><<<grid, kThreads, 0, st>>>(r, ld, p, n, rows);
    else hard_emit_kernel<false><<<grid, kThreads, 0, st>>>(r, ld, p, n, rows);
    return cudaGetLastError();
}

int64_t radix_tiles(int64_t n) { return (n + kRadixTile - 1) / kRadixTile; }

cudaError_t launch_radix_sort_rows(const float* r, int64_t ld, int64_t B, int64_t n,
                                   const RadixBuffers& buf, RowState* rows, WsHeader* hdr,
                                   cudaStream_t st) {
    const int64_t tiles = radix_tiles(n);
    cudaError_t e = cudaMemsetAsync(buf.seg_hist, 0, (size_t)B * 1024 * sizeof(uint32_t), st);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)tiles, (unsigned)B);
    {
        ProfScope ps_("radix_prep", st);
        radix_prep_kernel<<<grid, kThreads, 0, st>>>(r, ld, n, buf.keys[0], buf.seg_hist, rows, hdr);
    }
    {
        ProfScope ps_("radix_plan", st);
        radix_plan_kernel<<<(unsigned)B, 256, 0, st>>>(buf.seg_hist, B, n, buf.plan);
    }
    if (n < (int64_t)kLbMask) {
        // one kernel per digit pass: look-back words instead of upsweep + scan
        const size_t words = (size_t)B * 256 * (size_t)tiles * sizeof(uint32_t);
        unsigned long long* counter =
            reinterpret_cast<unsigned long long*>(reinterpret_cast<char*>(buf.tile_hist) + words);
        for (int d = 0; d < 4; ++d) {
            e = cudaMemsetAsync(buf.tile_hist, 0, words + sizeof(unsigned long long), st);
            if (e != cudaSuccess) return e;
            ProfScope ps_("radix_onesweep", st);
            radix_onesweep_kernel<<<(unsigned)(tiles * B), kThreads, 0, st>>>(
                buf.keys[0], buf.keys[1], n, tiles, d, buf.plan, buf.seg_hist, buf.tile_hist, counter,
                hdr);
        }
        return cudaGetLastError();
    }
    for (int d = 0; d < 4; ++d) {
        {
            ProfScope ps_("radix_upsweep", st);
            radix_upsweep_kernel<<<grid, kThreads, 0, st>>>(buf.keys[0], buf.keys[1], n, tiles, d,
                                                        buf.plan, buf.tile_hist);
        }
        if (tiles <= 64)
            {
                ProfScope ps_("radix_scan", st);
                radix_scan_kernel<<<(unsigned)B, 256, 0, st>>>(buf.seg_hist, tiles, d, buf.plan,
                                                           buf.tile_hist);
            }
        else
            {
                ProfScope ps_("radix_scan", st);
                radix_scan_wide_kernel<<<dim3(256, (unsigned)B), 256, 0, st>>>(
                buf.seg_hist, tiles, d, buf.plan, buf.tile_hist);
            }
        {
            ProfScope ps_("radix_downsweep", st);
            radix_downsweep_kernel<<<grid, kThreads, 0, st>>>(buf.keys[0], buf.keys[1], n, tiles, d,
                                                          buf.plan, buf.tile_hist);
        }
    }
    return cudaGetLastError();
}

cudaError_t launch_rowsolve_sorted_keys(const RadixBuffers& buf, int64_t B, int64_t n, double k,
                                        const double* k_rows, double t, double* b, RowState* rows,
                                        WsHeader* hdr, cudaStream_t st) {
    {
        ProfScope ps_("rowsolve", st);
        rowsolve_keys_kernel<<<(unsigned)B, 1024, 0, st>>>(buf.keys[0], buf.keys[1], n, k, k_rows,
                                                       t, buf.plan, b, rows, hdr);
    }
    return cudaGetLastError();
}

}  // namespace lapsum
