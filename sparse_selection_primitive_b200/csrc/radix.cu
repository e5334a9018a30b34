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
#include <type_traits>

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
    float xs[kPerThread];
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
        const int64_t idx = base + e * kThreads + threadIdx.x;
        xs[e] = idx < n ? __ldg(rr + idx) : 0.f;
    }
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
        const int64_t idx = base + e * kThreads + threadIdx.x;
        const bool ok = idx < n;
        const uint32_t key = to_key(xs[e]);
        if (ok) {
            bad |= !finite_f(xs[e]);
            kk[idx] = key;
        }
        if (ok) {
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

// Exclusive scan of one count per thread of a 256-thread block, in thread
// order: warp shuffles, then the warps' totals through `wsum` (8 words).
// Every thread calls it; `wsum` must not be reused before a block barrier.
__device__ __forceinline__ uint32_t block256_excl_scan(uint32_t x, uint32_t* wsum) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    uint32_t inc = x;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, inc, d);
        if (lane >= d) inc += o;
    }
    if (lane == 31) wsum[w] = inc;
    __syncthreads();
    uint32_t pre = 0;
#pragma unroll
    for (int i = 0; i < kWarps; ++i) pre += i < w ? wsum[i] : 0u;
    return pre + inc - x;
}

__global__ void __launch_bounds__(kThreads, 4) radix_onesweep_kernel(
    uint32_t* __restrict__ k0, uint32_t* __restrict__ k1, int64_t n, int64_t tiles, int d,
    const int32_t* __restrict__ plan, const uint32_t* __restrict__ seg_hist,
    uint32_t* __restrict__ lb, unsigned long long* __restrict__ counter, WsHeader* hdr) {
    __shared__ uint32_t wcnt[kWarps][256];
    __shared__ uint32_t tstart[256];
    __shared__ uint32_t sorted[kRadixTile];
    __shared__ uint32_t wsum[2][kWarps];
    __shared__ unsigned long long s_id;
    if (threadIdx.x == 0) s_id = atomicAdd(counter, 1ull);
    __syncthreads();
    // ids run tile-major over the rows, so a tile's predecessor in its row
    // started B ids earlier and has usually published its inclusive counts
    const int64_t id = (int64_t)s_id;
    const int64_t B = (int64_t)gridDim.x / tiles;
    const int64_t tile = id / B, row = id % B;
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
    const uint32_t dbase = block256_excl_scan(seg_hist[row * 1024 + d * 256 + v], wsum[0]);

    uint32_t key[kPerThread], lrank[kPerThread];
    const uint32_t lt = lanemask_lt();
    // tile-local 32-bit positions: warp w owns [w*512, (w+1)*512), visited 32
    // at a time in index order, which keeps the rank stable
    const int valid = (int)min((int64_t)kRadixTile, n - base);
    const uint32_t* tsrc = src + base;
    const int off0 = warp * (32 * kPerThread) + lane;
    auto rank = [&](auto full_tag) {
        constexpr bool FULL = decltype(full_tag)::value;
#pragma unroll
        for (int e = 0; e < kPerThread; ++e) {
            const int li = off0 + e * 32;
            key[e] = (FULL || li < valid) ? tsrc[li] : 0u;
        }
#pragma unroll
        for (int e = 0; e < kPerThread; ++e) {
            const bool ok = FULL || off0 + e * 32 < valid;
            const uint32_t dig = (key[e] >> shift) & 255u;
            const uint32_t peers =
                __match_any_sync(0xffffffffu, ok ? dig : 256u + (uint32_t)lane);
            // every peer reads the digit's count before the lowest peer adds
            // the group (one warp's shared accesses stay in program order)
            const uint32_t old = ok ? wcnt[warp][dig] : 0u;
            if (ok && (peers & lt) == 0u) wcnt[warp][dig] = old + __popc(peers);
            lrank[e] = old + __popc(peers & lt);
            __syncwarp();
        }
    };
    if (valid == kRadixTile) rank(std::true_type{});
    else rank(std::false_type{});
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
        // read four predecessors per round trip, nearest first; stop at the
        // first inclusive word, re-read from the first one not yet published
        int64_t j = tile - 1;
        int spins = 0;
        bool done = false;
        while (!done) {
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) w[q] = j - q >= 0 ? (uint32_t)words[(j - q) * 256 + v] : (uint32_t)kLbInc;
            int adv = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (done || adv < q) continue;
                const uint32_t f = w[q] & ~kLbMask;
                if (f == 0u) continue;  // not published yet
                excl += w[q] & kLbMask;
                ++adv;
                if (f == kLbInc) done = true;
            }
            j -= adv;
            if (!done && adv == 0) {
                if (++spins > kLbSpinMax) {
                    timed_out = true;
                    break;
                }
                // a predecessor still ranking: yield the issue slots to the
                // warps that are doing work
                __nanosleep(100);
            }
        }
        if (!timed_out) words[tile * 256 + v] = kLbInc | (excl + cnt);
    }
    if (__syncthreads_or(timed_out)) {  // the bases are unknown: write nothing
        if (threadIdx.x == 0) set_status(hdr, kDevWaitTimeout);
        return;
    }
    // exclusive scan of the tile's digit counts -> local start of each digit;
    // then per (warp, digit) the local slot base, and per digit the shift
    // from a local slot to the global position
    const uint32_t ts = block256_excl_scan(cnt, wsum[1]);
    tstart[v] = dbase + excl - ts;  // global position of local slot 0 of digit v
#pragma unroll
    for (int w = 0; w < kWarps; ++w) wcnt[w][v] += ts;
    __syncthreads();
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
        if (off0 + e * 32 < valid) {
            const uint32_t dig = (key[e] >> shift) & 255u;
            sorted[wcnt[warp][dig] + lrank[e]] = key[e];
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < valid; i += kThreads) {
        const uint32_t kv = sorted[i];
        const uint32_t pos = tstart[(kv >> shift) & 255u] + (uint32_t)i;
        if ((int64_t)pos < n) dst[pos] = kv;
    }
}

struct KeyGet {
    const uint32_t* k;
    __device__ __forceinline__ float operator()(long long j) const { return from_key(k[j]); }
};

__global__ void __launch_bounds__(512, 2) rowsolve_keys_kernel(const uint32_t* __restrict__ k0,
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

// Long sorted rows: the same solve over the whole GPU.  The row is cut into G
// chunks; one CTA per chunk writes the chunk's prefix and suffix maps in
// closed form (the product of its gap factors telescopes to gap(lo)
// e^{(s_lo - s_{hi-1})/t}, and the sums take fp32 exponentials of terms at
// most 1, added in fp64), and one CTA per row composes the G maps in chunk
// order, takes the chunk where F crosses k, and solves that chunk with
// everything before and after it folded into two anchors.
constexpr int64_t kSolveChunkMin = 65536;
constexpr int kSolveRecMax = 8192;  // chunks per row

struct ChunkRec {
    double fa, fc;  // P_{hi-1} = fa P_{lo-1} + fc
    double ba, bc;  // Q_lo = ba Q_hi + bc
    double g_lo;    // gap factor between positions lo-1 and lo (0 at the row's start)
    double pad[3];
};

__global__ void __launch_bounds__(256) rowsolve_chunk_kernel(const uint32_t* __restrict__ k0,
                                                              const uint32_t* __restrict__ k1,
                                                              int64_t n, int64_t chunk, double t,
                                                              const int32_t* __restrict__ plan,
                                                              ChunkRec* __restrict__ rec) {
    __shared__ double red[2][8];
    const int64_t row = blockIdx.y, c = blockIdx.x;
    const uint32_t* keys = (plan[row * 8 + 4] ? k1 : k0) + row * n;
    const int64_t lo = c * chunk, hi = min(n, lo + chunk);
    const float s_first = from_key(keys[lo]), s_last = from_key(keys[hi - 1]);
    const float it = (float)(1.0 / t);  // 1/t as a two-float pair
    const float it_lo = (float)(1.0 / t - (double)it);
    float cf = 0.f, cb = 0.f;
    double df = 0.0, db = 0.0;
    int cnt = 0;
    for (int64_t j = lo + threadIdx.x; j < hi; j += 256) {
        const float x = from_key(__ldcs(keys + j));
        cf += exp_neg(fmaf(s_last - x, it, (s_last - x) * it_lo));
        cb += exp_neg(fmaf(x - s_first, it, (x - s_first) * it_lo));
        if (++cnt == 16) {  // fp32 partial sums of 16 terms (each at most 1), then fp64
            df += (double)cf;
            db += (double)cb;
            cf = cb = 0.f;
            cnt = 0;
        }
    }
    df += (double)cf;
    db += (double)cb;
    df = warp_sum_d(df);
    db = warp_sum_d(db);
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    if (lane == 0) {
        red[0][w] = df;
        red[1][w] = db;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double sf = 0.0, sb = 0.0;
        for (int i = 0; i < 8; ++i) {
            sf += red[0][i];
            sb += red[1][i];
        }
        const double inv_t = 1.0 / t;
        const double span = exp(((double)s_first - (double)s_last) * inv_t);
        const double g_lo = lo > 0 ? gap_factor(from_key(keys[lo - 1]), s_first, inv_t) : 0.0;
        const double g_hi = hi < n ? gap_factor(s_last, from_key(keys[hi]), inv_t) : 0.0;
        ChunkRec r;
        r.fa = g_lo * span;
        r.fc = sf;
        r.ba = g_hi * span;
        r.bc = sb;
        r.g_lo = g_lo;
        r.pad[0] = r.pad[1] = r.pad[2] = 0.0;
        rec[row * gridDim.x + c] = r;
    }
}

__global__ void __launch_bounds__(1024) rowsolve_combine_kernel(
    const uint32_t* __restrict__ k0, const uint32_t* __restrict__ k1, int64_t n, int64_t chunk,
    int G, double k, const double* __restrict__ k_rows, double t, const int32_t* __restrict__ plan,
    const ChunkRec* __restrict__ recs, double* __restrict__ b_out, RowState* rows, WsHeader* hdr) {
    __shared__ SolveScratch sm;
    __shared__ SolveResult res;
    __shared__ Aff wt[32];
    __shared__ double sP, sQ;
    __shared__ int wc[32];
    const int64_t row = blockIdx.x;
    const uint32_t* keys = (plan[row * 8 + 4] ? k1 : k0) + row * n;
    const ChunkRec* rec = recs + row * G;
    const double kr = k_rows != nullptr ? k_rows[row] : k;
    const bool k_ok = kr > 0.0 && kr < (double)n;
    const double kk = k_ok ? kr : 0.5 * (double)n;
    // each thread composes a run of consecutive chunks
    const int per = (G + (int)blockDim.x - 1) / (int)blockDim.x;
    const int c0 = min(G, (int)threadIdx.x * per), c1 = min(G, c0 + per);
    Aff af = aff_id(), ab = aff_id();
    for (int c = c0; c < c1; ++c) af = aff_then(af, Aff{rec[c].fa, rec[c].fc});
    for (int c = c1 - 1; c >= c0; --c) ab = aff_then(Aff{rec[c].ba, rec[c].bc}, ab);
    const Aff ef = block_excl_scan_fwd(af, wt);  // chunks before this run
    const Aff eb = block_excl_scan_bwd(ab, wt);  // chunks after this run
    // F at each chunk's first score: P_lo = 1 + g_lo P_{lo-1}, Q_lo = ba Q_hi + bc
    double P = ef.c;   // P_{lo-1} of chunk c0 (P before the row is 0)
    double Qs[kSolveRecMax / 1024];
    double Q = eb.c;   // Q_hi of chunk c1 - 1 (Q after the row is 0)
    for (int c = c1 - 1; c >= c0; --c) {
        Q = fma(rec[c].ba, Q, rec[c].bc);
        Qs[c - c0] = Q;  // Q_lo of chunk c
    }
    int cnt = 0;
    for (int c = c0; c < c1; ++c) {
        const double P_lo = fma(rec[c].g_lo, P, 1.0);
        const double G_lo = (double)(n - (int64_t)c * chunk) - 0.5 * Qs[c - c0] + 0.5 * (P_lo - 1.0);
        cnt += G_lo >= kk ? 1 : 0;
        P = fma(rec[c].fa, P, rec[c].fc);  // P_{hi-1}
    }
    // the number of chunks with F(first score) >= k (F decreases along the row)
    int total = warp_sum_i(cnt);
    if ((threadIdx.x & 31) == 0) wc[threadIdx.x >> 5] = total;
    __syncthreads();
    total = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) total += wc[i];
    const int T = total > 0 ? total - 1 : 0;
    // anchors of chunk T: P_{lo_T - 1} and Q_{hi_T}, from the thread that owns T
    if (T >= c0 && T < c1) {
        double Pb = ef.c;
        for (int c = c0; c < T; ++c) Pb = fma(rec[c].fa, Pb, rec[c].fc);
        double Qa = eb.c;
        for (int c = c1 - 1; c > T; --c) Qa = fma(rec[c].ba, Qa, rec[c].bc);
        sP = Pb;
        sQ = Qa;
    }
    __syncthreads();
    const int64_t lo = (int64_t)T * chunk, hi = min(n, lo + chunk);
    Tails tl;
    tl.hasL = lo > 0;
    tl.aL = lo > 0 ? from_key(keys[lo - 1]) : 0.f;
    tl.SL = lo > 0 ? sP : 0.0;
    tl.hasR = hi < n;
    tl.aR = hi < n ? from_key(keys[hi]) : 0.f;
    tl.SR = hi < n ? sQ : 0.0;
    tl.cntR = (double)(n - hi);
    solve_sorted_block<KeyGet, false, true>(KeyGet{keys + lo}, hi - lo, tl, kk, t, &sm, &res);
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
    if (n > 4 * kSolveChunkMin) {
        // chunks of at least 65536 keys (a multiple of 4096), at most 8192 per row;
        // the records take the look-back words' space, free once the sort is done
        int64_t chunk = (n + kSolveRecMax - 1) / kSolveRecMax;
        chunk = ((chunk + 4095) / 4096) * 4096;
        if (chunk < kSolveChunkMin) chunk = kSolveChunkMin;
        const int G = (int)((n + chunk - 1) / chunk);
        ChunkRec* rec = reinterpret_cast<ChunkRec*>(buf.tile_hist);
        {
            ProfScope ps_("rowsolve_chunks", st);
            rowsolve_chunk_kernel<<<dim3((unsigned)G, (unsigned)B), 256, 0, st>>>(
                buf.keys[0], buf.keys[1], n, chunk, t, buf.plan, rec);
        }
        {
            ProfScope ps_("rowsolve", st);
            rowsolve_combine_kernel<<<(unsigned)B, 1024, 0, st>>>(buf.keys[0], buf.keys[1], n, chunk,
                                                               G, k, k_rows, t, buf.plan, rec, b,
                                                               rows, hdr);
        }
        return cudaGetLastError();
    }
    {
        ProfScope ps_("rowsolve", st);
        rowsolve_keys_kernel<<<(unsigned)B, 512, 0, st>>>(buf.keys[0], buf.keys[1], n, k, k_rows,
                                                       t, buf.plan, b, rows, hdr);
    }
    return cudaGetLastError();
}

}  // namespace lapsum
