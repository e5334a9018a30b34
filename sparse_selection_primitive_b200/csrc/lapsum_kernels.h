// Host-side launchers of the Fast LapSum kernels (internal to the library).
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

#include "lapsum_common.cuh"

namespace lapsum {

// Number of SMs of the current device (looked up once per device).
int device_sm_count();

// Optional per-kernel CUDA-event timing (lapsum_profile_enable).  A ProfScope
// records an event pair around the launches in its lifetime when enabled.
void prof_begin(const char* name, cudaStream_t st);
void prof_end(cudaStream_t st);
struct ProfScope {
    cudaStream_t st;
    ProfScope(const char* name, cudaStream_t s) : st(s) { prof_begin(name, s); }
    ~ProfScope() { prof_end(st); }
};

// Launch with programmatic stream serialization (see pdl_wait): the kernel may
// start while the previous kernel on the stream finishes.  Every kernel
// launched this way calls pdl_wait() before its first memory access.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Runs `set` (kernel attributes, which are per device) the first time a
// process reaches this point on the current device; `done` holds one bit per
// device (devices past 63 set it every time).  Thread-safe: a race only sets
// the same attribute twice.
template <class F>
inline void once_per_device(std::atomic<unsigned long long>& done, F set) {
    int dev = 0;
    cudaGetDevice(&dev);
    const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
    if (bit == 0ull || (done.load(std::memory_order_acquire) & bit) == 0ull) {
        set();
        done.fetch_or(bit, std::memory_order_acq_rel);
    }
}

// --- on-chip full sort (n <= 4096) -------------------------------------------
int onchip_npad(int64_t n);
// k_rows (device, B entries) when not null gives each row its own budget.
// search != 0 solves rows of n <= 256 by the segment search (no sort; rows it
// leaves are sorted in the same kernel; 2 leaves every row to the sort);
// otherwise, and for longer rows, the bitonic sort and scans.
cudaError_t launch_onchip_forward(const float* r, int64_t ld, float* p, double* b, double* sumf,
                                  int64_t B, int n, double k, const double* k_rows, double t,
                                  WsHeader* hdr, int vec, int search, cudaStream_t st);
cudaError_t launch_onchip_backward(const float* r, int64_t ld, const double* b, const float* v,
                                   float* g, int64_t B, int n, double t, int vec, cudaStream_t st);
// Zero-temperature limit (hard top-k) of rows of n <= 4096: sort, boundary group, p.
cudaError_t launch_onchip_hard(const float* r, int64_t ld, float* p, double* b, int64_t B, int n,
                               double k, WsHeader* hdr, int vec, cudaStream_t st);
// The router form: scores of any lapsum_dtype (16-bit types as bit patterns,
// widened exactly), optional sum f per row, and optionally (sel_cnt != null)
// the per-row list of positions and values of p > eps (at most cap per row)
// with its count.
cudaError_t launch_onchip_router(const void* r, int dtype, int64_t ld, float* p, double* b,
                                 double* sumf, int64_t B, int n, double k, double t, WsHeader* hdr,
                                 int vec, int32_t* sel_idx, float* sel_val, int32_t* sel_cnt,
                                 int cap, float eps, int search, cudaStream_t st);
cudaError_t launch_onchip_backward_router(const void* r, int dtype, int64_t ld, const double* b,
                                          const float* v, float* g, int64_t B, int n, double t,
                                          int vec, cudaStream_t st);
// Rows of 16-bit scores (bf16 or fp16 bit patterns) widened exactly to fp32:
// dst[row * ld + i] for i < n (the same row stride as the source).
cudaError_t launch_widen(const void* src, int dtype, int64_t ld, int64_t B, int64_t n, float* dst,
                         cudaStream_t st);

// --- radix full sort (segmented LSD, keys only) ------------------------------
constexpr int kRadixTile = 4096;
struct RadixBuffers {
    uint32_t* keys[2];     // ping-pong key buffers, B*n each (rows dense, stride n)
    uint32_t* seg_hist;    // [B][4][256] digit counts of every segment
    uint32_t* tile_hist;   // [B][256][tiles] per-tile digit counts, scanned into offsets
    int32_t* plan;         // [B][8]: parity before pass d (d=0..4), trivial-pass mask
};
int64_t radix_tiles(int64_t n);
cudaError_t launch_radix_sort_rows(const float* r, int64_t ld, int64_t B, int64_t n,
                                   const RadixBuffers& buf, RowState* rows, WsHeader* hdr,
                                   cudaStream_t st);
// Solve every row from its sorted keys (one CTA per row); writes b and RowState.
cudaError_t launch_rowsolve_sorted_keys(const RadixBuffers& buf, int64_t B, int64_t n, double k,
                                        const double* k_rows, double t, double* b, RowState* rows,
                                        WsHeader* hdr, cudaStream_t st);
// p of the zero-temperature limit from each row's record (boundary score c
// and its share): one CTA per 4096-score tile.
cudaError_t launch_hard_emit(const float* r, int64_t ld, float* p, int64_t B, int64_t n,
                             const RowState* rows, int vec, cudaStream_t st);
// The zero-temperature limit through bracketing (rows of n > 4096, in
// parallel): plain samples, their binomial order statistics as the bracket,
// one pass for the count above it, the band and the largest score below it,
// and one CTA per row for the boundary group (an exact selection over the row
// when the bracket misses); then p.  band: B * n floats; cand: B * 4096 keys;
// tickets: B self-resetting counters; top_h as in the soft sample kernel.
cudaError_t launch_hard_bracket(const float* r, int64_t ld, float* p, double* b, int64_t B,
                                int64_t n, double k, uint64_t seed, int m, int64_t rank_l,
                                int64_t rank_h, int top_h, int force_miss, RowState* rows,
                                float* band, uint32_t* cand, uint32_t* tickets, WsHeader* hdr,
                                int64_t B_total, int vec, cudaStream_t st);
// Zero-temperature limit of every row from its sorted keys (one CTA per row),
// then p from r (one CTA per tile); b, the boundary score and its share go to
// the row records.
cudaError_t launch_rowhard_sorted_keys(const RadixBuffers& buf, int64_t B, int64_t n, double k,
                                       const float* r, int64_t ld, float* p, double* b,
                                       RowState* rows, int vec, cudaStream_t st);

// --- streaming kernels over long rows ----------------------------------------
constexpr int kStreamTile = 4096;  // elements per CTA tile of the streaming kernels
int64_t stream_tiles(int64_t n);

// Gradient support of long rows, written by the forward and read by the
// backward: every score with |x| <= kSupWindow, listed per warp share of each
// 4096-score tile (8 shares of 512 scores, kSupCap entries each).
constexpr int kSupWarps = 8;
constexpr int kSupCap = 256;
constexpr float kSupWindow = 90.f;  // f == 0 in fp32 beyond this |x|
constexpr uint32_t kSupOverflow = 1u;  // a share held more scores than its capacity
constexpr uint32_t kSupNear = 2u;      // some score of the row has |x| <= 50
struct SupportView {
    int64_t* hdr;    // [0] n and [1] B of the forward that wrote the list
    double* b;       // [B] threshold of each row at that forward
    uint32_t* flags; // [B] kSupOverflow | kSupNear, cleared by the forward's first kernel
    uint32_t* cnt;   // [B][tiles][8] entries found per share (> kSupCap: overflow)
    uint2* ent;      // [B][tiles][8][kSupCap] (position in the tile, x bits)
    float* val;      // [B][tiles][8][kSupCap] v at each entry (written by the backward)
};
size_t support_bytes(int64_t B, int64_t n);
SupportView support_view(void* base, int64_t B, int64_t n);
SupportView support_rows(const SupportView& s, int64_t r0, int64_t n);  // rows from r0 on

// p = sigma((r - b)/t) and sum f per row; partials: [B][tiles] doubles.
// With sup != nullptr the gradient support is written as well.
cudaError_t launch_emit(const float* r, int64_t ld, float* p, double* b, double* sumf,
                        int64_t B, int64_t n, double t, double* partials, uint32_t* tickets,
                        int vec, WsHeader* hdr, int record_call, int64_t B_total, int path_code,
                        const SupportView* sup, cudaStream_t st);
// Backward from the gradient support: v is read only at the listed scores.
// Rows whose list overflowed, does not match (n, b), or whose smallest |x| is
// above 50 are recomputed by the dense kernels.
// B_total: the rows of the whole call (checked against the forward's).
cudaError_t launch_backward_support(const float* r, int64_t ld, const double* b, const float* v,
                                    float* g, int64_t B, int64_t n, double t,
                                    const SupportView& sup, int64_t B_total, double* partials,
                                    double* row_R, uint32_t* tickets, uint32_t* dense_flag,
                                    int vec, cudaStream_t st);
// Backward for long rows: reduce (mu, sum w, sum w v) per row, then g.
// partials: 4 doubles per CTA record.
cudaError_t launch_backward_stream(const float* r, int64_t ld, const double* b, const float* v,
                                   float* g, int64_t B, int64_t n, double t, double* partials,
                                   double* row_R, uint32_t* tickets, int vec, cudaStream_t st);
// Same, but rows with need[row] == 0 are skipped by every CTA (need on the device).
cudaError_t launch_backward_stream_if(const float* r, int64_t ld, const double* b,
                                      const float* v, float* g, int64_t B, int64_t n, double t,
                                      double* partials, double* row_R, uint32_t* tickets, int vec,
                                      const uint32_t* need, cudaStream_t st);

// The VJP of one shard of a row split over devices: its record (min |x|, S,
// Sv) of the online sums, then g from the shards' records merged in shard
// order (ws: vjp_shard_workspace_bytes(), the ticket at its start cleared
// once); and p of a shard from b.
size_t vjp_shard_workspace_bytes();
cudaError_t launch_vjp_partial(const float* r, const double* b, const float* v, int64_t n,
                               double t, double* rec, void* ws, cudaStream_t st);
cudaError_t launch_vjp_apply(const float* r, const double* b, const float* v, float* g, int64_t n,
                             double t, const double* recs, int world, void* ws, cudaStream_t st);
cudaError_t launch_emit_p(const float* r, float* p, const double* b, int64_t n, double t,
                          cudaStream_t st);

// Gradients of sum v p with respect to k and t, per row; partials: the
// backward partials region (max(tiles, 2) * 4 doubles per row).
cudaError_t launch_backward_kt(const float* r, int64_t ld, const double* b, const float* v,
                               int64_t B, int64_t n, double t, double* partials,
                               uint32_t* tickets, double* g_k, double* g_t, int vec,
                               cudaStream_t st);

// --- windowed backward (scores with |x| <= 90 only) ----------------------------
struct WinEntry {
    uint32_t idx;  // position in the row
    float x;       // (r - b)/t
    float v;       // upstream gradient
};
struct WindowBuffers {
    WinEntry* list;   // [B][window_capacity(n)], split evenly between the pass CTAs
    uint2* tab;       // [B][window_tiles(n)]: (start, count) of each tile's entries
    uint32_t* flag;   // [B] 1 = the dense kernels recompute this row
};
uint32_t window_capacity(int64_t n);
int64_t window_tiles(int64_t n);
cudaError_t launch_backward_window(const float* r, int64_t ld, const double* b, const float* v,
                                   float* g, int64_t B, int64_t n, double t,
                                   const WindowBuffers& wb, double* partials, double* row_R,
                                   uint32_t* tickets, int vec, cudaStream_t st);

// --- probabilistic bracketing --------------------------------------------------
constexpr int kSampleMax = 32768;
struct BracketBuffers {
    float* sample;       // [B][m]
    float* band[2];      // capacity n each
    unsigned long long* bins;  // band histogram of the first bracket: [3][2048]
    double* fold_part;   // fold partials, one record per CTA
    uint32_t* ticket;    // last-block counters: [0] fold, [1] sample; [2..2050) sample histogram
    uint32_t* cand;      // the sample CTAs' top keys (at most 4096)
    int fold_grid;
};
int bracket_fold_grid();
// Pieces of the bracketing for one row split over several devices (contiguous
// shards; the host exchanges the results between the steps).
// y[s] = draw s of the row's sample when its index lies in this shard, else 0.
cudaError_t launch_shard_sample(const float* r, int64_t n_shard, int64_t offset, int64_t n,
                                double t, uint64_t seed, int m, float* y, cudaStream_t st);
// ends = (a_L, a_R): the rank_h-th and rank_l-th largest of the complete sample.
cudaError_t launch_sample_bracket(const float* y, int m, int64_t rank_l, int64_t rank_h,
                                  float* ends, cudaStream_t st);
// One shard folded with the bracket: rec = (count above a_R, left tail sum,
// right tail sum, non-finite flag, band size), the band into `band` (capacity
// n_shard); ws: shard_fold_workspace_bytes().
size_t shard_fold_workspace_bytes();
cudaError_t launch_shard_fold(const float* r, int64_t n_shard, const float* ends, double t,
                              double* rec, float* band, void* ws, cudaStream_t st);
// The exact solve on the shards' bands (bands[w * stride + j], j < rec_w band
// size) with their tails: out = (b, F(a_L), F(a_R), certified); cur and nxt
// hold the total band twice.
cudaError_t launch_shard_band_solve(const float* bands, int64_t stride, const double* recs,
                                    int world, const float* ends, double k, double t, float* cur,
                                    float* nxt, double* out, cudaStream_t st);
// Sample size and bracket ladder of one row with its own budget (filled on the
// device from k[row]); ok = 0 for a budget outside (0, n).
struct RowBudget {
    double k;
    int32_t m, ok;
    int64_t l[kLadder], h[kLadder];
};
cudaError_t launch_row_budgets(const double* k_rows, int64_t B, int64_t n, double alpha,
                               RowBudget* out, cudaStream_t st);
// The whole bracketing pipeline with one CTA per row (rows up to 2^20 scores):
// b[row] and rows[row] for every row; band0/band1: B * n floats each.  With
// `budgets` (not null) each row takes k, m and its ladder from its entry, and m
// is the shared-memory capacity for the sample.
cudaError_t launch_rowbracket(const float* r, int64_t ld, int64_t B, int64_t n, double k, double t,
                              uint64_t seed, int m, int64_t rank_l[kLadder],
                              int64_t rank_h[kLadder], int flags, RowState* rows, float* band0,
                              float* band1, double* b, WsHeader* hdr, int vec, cudaStream_t st,
                              const RowBudget* budgets = nullptr, uint32_t* sup_flags = nullptr);
cudaError_t launch_bracket_row(const float* r_row, int64_t n, double k, double t, uint64_t seed,
                               int64_t row, int m, int64_t rank_l[kLadder],
                               int64_t rank_h[kLadder], int flags, const BracketBuffers& buf,
                               RowState* st_row, double* b_out, WsHeader* hdr,
                               uint32_t* sup_flag, const RowBudget* bud, cudaStream_t st);

}  // namespace lapsum
