/*
 * lapsum.h -- C ABI of the B200 (sm_100a) Fast LapSum soft top-k library.
 *
 * The operator, from "Fast LapSum: Exact Differentiable Top-k at Million Scale"
 * (gist.science explainer pages), section 2.1 "The LapSum operator": for each
 * row of scores r[0..n), a budget k (0 < k < n) and a temperature t > 0,
 *
 *     p_i = sigma((r_i - b) / t),   sigma = CDF of Laplace(0,1),
 *     sum_i p_i = k                 (b is the unique scalar threshold),
 *
 * and the backward pass is the analytic vector-Jacobian product
 *
 *     g_i = (f_i / t) (v_i - sum_j v_j f_j / sum_j f_j),   f_i = 0.5 exp(-|r_i - b| / t).
 *
 * Section 2.2 "Fast LapSum: the GPU solver" gives the two solvers built here:
 * a full-sort solver (sort, one numerically stable prefix/suffix scan, an
 * index lookup of the balancing segment, a closed-form root) and, for rows
 * with n > 10^6, probabilistic bracketing (sample, binomial order-statistic
 * bracket, one streaming fold, exact solve on the middle band, certification
 * with widening).
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or retains device memory.
 *   - Rows are row-major with leading dimension ld >= n (elements): element i
 *     of row j of r, p, v and g is at [j * ld + i].  Vectorised loads are used
 *     when the base pointers are 16-byte aligned and ld is a multiple of 4
 *     (of 8 for bf16 scores).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All work is ordered on it; no call synchronises the host except
 *     lapsum_read_status and lapsum_row_info.
 *   - Argument errors are detected on the host, returned at once, and launch
 *     nothing.  Conditions found on the device (non-finite scores, exhausted
 *     bracket retries, per-row budgets outside (0, n)) are OR-ed into a
 *     sticky status word inside the workspace and reported by
 *     lapsum_read_status, which also clears it.
 *   - Calls that share a workspace must be ordered on one stream (or be
 *     otherwise serialised); concurrent calls on one workspace race.
 */
#ifndef LAPSUM_H
#define LAPSUM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes and device status bits. */
enum lapsum_status {
    LAPSUM_OK = 0,
    LAPSUM_EINVAL = 1,     /* B < 1, n < 1, ld < n, !(0 < k < n), !(t > 0), NULL pointer, bad path;
                              device: a per-row budget outside (0, n); b of that row is NaN */
    LAPSUM_EWORKSPACE = 2, /* ws NULL, not 256-byte aligned, or smaller than lapsum_workspace_bytes */
    LAPSUM_ENONFINITE = 3, /* device: a score was NaN or infinite; b of that row is NaN */
    LAPSUM_EBRACKET = 4,   /* device: every allowed bracket failed certification; b is NaN */
    LAPSUM_ECUDA = 5       /* a CUDA runtime call failed (launch error, bad stream, ...) */
};

/* Solver selection (low byte of `path`). */
enum lapsum_path {
    LAPSUM_PATH_AUTO = 0,     /* n <= 256: segment search without a sort (one warp per row;
                                 a row it does not settle is sorted in the same kernel);
                                 n <= 4096: bitonic; n <= 2^18: bracketing, one CTA per row;
                                 else bracketing over the whole GPU */
    LAPSUM_PATH_FULLSORT = 1, /* full sort: bitonic for n <= 4096, radix above */
    LAPSUM_PATH_BRACKET = 2,  /* probabilistic bracketing (any n >= 2) */
    LAPSUM_PATH_RADIX = 3,    /* full sort with the radix sorter at any n */
    LAPSUM_PATH_ROWBRACKET = 4 /* probabilistic bracketing with one CTA per row: sample, order
                                  statistics, fold and band solve in one kernel (n <= 2^20) */
};

/* Score element types of the router entry points. */
enum lapsum_dtype {
    LAPSUM_DTYPE_F32 = 0,  /* float */
    LAPSUM_DTYPE_BF16 = 1, /* bfloat16, passed as its 16-bit patterns (uint16_t) */
    LAPSUM_DTYPE_F16 = 2   /* IEEE half, passed as its 16-bit patterns (uint16_t) */
};

/* Test and diagnostic flags, OR-ed into `path`. */
enum lapsum_flags {
    LAPSUM_FLAG_FORCE_MISS = 0x100, /* bracketing: start from a bracket that excludes b;
                                       AUTO with n <= 256: skip the segment search, so
                                       every row takes the in-kernel sort */
    LAPSUM_FLAG_NO_RETRY = 0x200,   /* bracketing: allow no widening (a miss => LAPSUM_EBRACKET) */
    LAPSUM_FLAG_ONE_CTA_SOLVE = 0x400 /* bracketing: solve every band inside the single-CTA
                                         solve kernel, without the grid-wide extraction that
                                         large first bands otherwise use */
};

/* Version of this ABI (incremented on any incompatible change). */
int lapsum_abi_version(void);

/* Static, human-readable name of a return code or status bit set. */
const char* lapsum_status_string(int status);

/*
 * Bytes of device workspace that lapsum_forward and lapsum_backward need for
 * this problem size and path (the same buffer serves both).  Returns 0 for
 * invalid sizes.  The workspace must be 256-byte aligned and must be cleared
 * once with lapsum_workspace_init before first use.
 */
size_t lapsum_workspace_bytes(int64_t B, int64_t n, double k, int path);

/*
 * Bytes of workspace lapsum_backward needs on its own (a prefix of any forward
 * workspace for the same B and n, so the forward's buffer can be reused).
 * Returns 0 for invalid sizes.
 */
size_t lapsum_backward_workspace_bytes(int64_t B, int64_t n);

/* Zero the workspace's status word and bookkeeping (stream-ordered). */
int lapsum_workspace_init(void* ws, size_t ws_bytes, void* stream);

/*
 * Forward: for every row, the exact threshold b[row] (fp64) and
 * p[row*ld + i] = sigma((r_i - b)/t) (fp32).  sum_f (may be NULL) receives
 * sum_i f_i per row in fp64.  `seed` drives the bracketing sample (a
 * counter-based SplitMix64 stream); results do not depend on it except for
 * rounding in the last bits.  r and p must not overlap.
 */
int lapsum_forward(const float* r, int64_t ld, float* p, double* b, double* sum_f, int64_t B,
                   int64_t n, double k, double t, int path, uint64_t seed, void* ws,
                   size_t ws_bytes, void* stream);

/*
 * Backward: g[row*ld + i] = (f_i/t)(v_i - R_row), R_row = sum_j v_j f_j / sum_j f_j,
 * with f_i = 0.5 exp(-|r_i - b_row|/t) and b from lapsum_forward.  R is formed
 * with weights shifted by the row's smallest |r_i - b|/t, so it stays finite
 * when every f_i underflows.  g must not overlap r or v.
 */
int lapsum_backward(const float* r, int64_t ld, const double* b, const float* v, float* g,
                    int64_t B, int64_t n, double t, void* ws, size_t ws_bytes, void* stream);

/*
 * Zero-temperature limit (hard top-k).  "Fast LapSum: Exact Differentiable
 * Top-k at Million Scale" (gist.science explainer pages), section 2.3, names
 * DFTopK's threshold -- the midpoint of the k-th and (k+1)-th largest scores
 * -- as LapSum's limit at t -> 0.  For each row, with c the ceil(k)-th largest
 * score, a = #{r > c} and m = #{r = c} (-0 and +0 are one value):
 *   k < a + m:  b = c, p = 1 above c, (k - a)/m at c, 0 below;
 *   k = a + m:  b = (c + d)/2 with d the largest score below c, p the 0/1
 *               mask of the scores above b.
 * So sum p = k, as at every t > 0 (ties at the boundary share the remaining
 * budget instead of a fixed 1/2).  k is real in (0, n); n >= 2.  Solvers: the
 * on-chip sort for n <= 4096 (LAPSUM_PATH_AUTO or LAPSUM_PATH_FULLSORT); for
 * longer rows LAPSUM_PATH_AUTO and LAPSUM_PATH_BRACKET use bracketing without
 * a full sort (section 2.2's steps with plain samples: their binomial order
 * statistics bracket the ceil(k)-th largest score, one pass counts the scores
 * above the bracket, keeps the band inside it and the largest score below it,
 * and the boundary group is read off the sorted band; an exact selection over
 * the row takes over when the bracket misses; LAPSUM_FLAG_FORCE_MISS forces
 * that case for tests), falling back to the radix sort when the bracket ranks
 * are too large for the sample's candidate lists (budgets near n/2);
 * LAPSUM_PATH_FULLSORT and LAPSUM_PATH_RADIX take the radix full sort;
 * LAPSUM_PATH_ROWBRACKET returns LAPSUM_EINVAL.  ws: lapsum_workspace_bytes(B,
 * n, k, LAPSUM_PATH_FULLSORT) for AUTO and FULLSORT, or with LAPSUM_PATH_RADIX
 * for the other paths.  Rows with a non-finite score get b = NaN and p = NaN
 * (status LAPSUM_ENONFINITE).  The limit has no useful gradient (p is
 * piecewise constant in r); there is no backward.
 */
int lapsum_forward_hard(const float* r, int64_t ld, float* p, double* b, int64_t B, int64_t n,
                        double k, int path, void* ws, size_t ws_bytes, void* stream);

/*
 * Router form for short rows (n <= 4096, on chip: the segment search for
 * n <= 256, the sort above), e.g. the scores of
 * a mixture-of-experts router: scores r of type `dtype` (fp32, or bf16 or fp16
 * bit patterns widened exactly to fp32), p (fp32) and b (fp64) as lapsum_forward,
 * and, when sel_cnt is not NULL, the sparse support of each row next to p:
 * sel_idx[row*cap + j] and sel_p[row*cap + j], j < min(cap, sel_cnt[row]),
 * are the positions (ascending) and values of the scores with p > eps, and
 * sel_cnt[row] is their number (it may exceed cap; the list then holds the
 * first cap).  The decision p > eps is taken on the fp32 p that is written.
 * sel_idx/sel_p/sel_cnt are device arrays of B*cap, B*cap and B entries, all
 * NULL or all given; cap >= 1 and eps >= 0 when given.  ws as lapsum_forward
 * with LAPSUM_PATH_FULLSORT.  The pages state the problem for real-valued
 * scores; a narrower score type and the support list are this library's
 * additions for that use.  lapsum_backward_router: g (fp32) from scores of
 * `dtype` and fp32 v, as lapsum_backward (no workspace).  Errors: LAPSUM_EINVAL
 * for n > 4096, an unknown dtype or inconsistent selection arguments, else as
 * lapsum_forward / lapsum_backward.
 */
int lapsum_forward_router(const void* r, int dtype, int64_t ld, float* p, double* b, int64_t B,
                          int64_t n, double k, double t, float eps, int32_t cap, int32_t* sel_idx,
                          float* sel_p, int32_t* sel_cnt, void* ws, size_t ws_bytes,
                          void* stream);
int lapsum_backward_router(const void* r, int dtype, int64_t ld, const double* b, const float* v,
                           float* g, int64_t B, int64_t n, double t, void* stream);

/*
 * Scores of a 16-bit type at any row length: lapsum_forward_lowp and
 * lapsum_backward_lowp take r as `dtype` (LAPSUM_DTYPE_BF16 or _F16 bit
 * patterns, or LAPSUM_DTYPE_F32) with row stride ld, and otherwise behave as
 * lapsum_forward_support / lapsum_backward_support (support may be NULL: then
 * as lapsum_forward / lapsum_backward).  The values solved for are the exact
 * fp32 widenings of the scores (section 2.1 of the pages states the problem
 * for real scores; a narrower storage type is this library's addition).
 * Rows of n <= 4096 with LAPSUM_PATH_AUTO or LAPSUM_PATH_FULLSORT read the
 * 16-bit scores directly in the on-chip kernels; longer rows (or another
 * path) first widen the rows into the tail of ws (one streaming pass, 2 bytes
 * read and 4 written per score) and then run the fp32 solvers on the copy.
 * p, b, sum_f, v and g are as in the fp32 calls (g is fp32).  Workspace:
 * lapsum_workspace_bytes_lowp(B, n, ld, k, path) and
 * lapsum_backward_workspace_bytes_lowp(B, n, ld) bytes (0: invalid sizes or
 * path; the backward of rows with n <= 4096 needs none, ws may then be NULL).
 * Errors: LAPSUM_EINVAL for an unknown dtype, else as the fp32 calls.
 */
size_t lapsum_workspace_bytes_lowp(int64_t B, int64_t n, int64_t ld, double k, int path);
size_t lapsum_backward_workspace_bytes_lowp(int64_t B, int64_t n, int64_t ld);
int lapsum_forward_lowp(const void* r, int dtype, int64_t ld, float* p, double* b, double* sum_f,
                        int64_t B, int64_t n, double k, double t, int path, uint64_t seed,
                        void* ws, size_t ws_bytes, void* support, size_t support_bytes,
                        void* stream);
int lapsum_backward_lowp(const void* r, int dtype, int64_t ld, const double* b, const float* v,
                         float* g, int64_t B, int64_t n, double t, const void* support,
                         size_t support_bytes, void* ws, size_t ws_bytes, void* stream);

/*
 * Forward with a budget per row: as lapsum_forward, with k[row] (fp64, DEVICE
 * memory, B entries, read in stream order) in place of the shared k.  The
 * pages fix one budget per operator call; a budget per row is the next step
 * the same equation allows (every row is solved on its own).  Solvers:
 * LAPSUM_PATH_AUTO gives the on-chip segment search for n <= 256 and the
 * on-chip sort for n <= 4096, the one-CTA-per-row
 * bracketing for n <= 2^18 and the whole-GPU bracketing above (both compute
 * each row's sample size and binomial ranks on the device from its budget);
 * LAPSUM_PATH_FULLSORT, LAPSUM_PATH_RADIX, LAPSUM_PATH_ROWBRACKET (n <= 2^20)
 * and LAPSUM_PATH_BRACKET select one.  The workspace
 * is lapsum_workspace_bytes_rowk(B, n, path) bytes (0 for an invalid size or
 * path).  `support` (may be NULL; see the gradient support below, same
 * rules when not NULL) receives the gradient support of rows with n > 4096.
 * A row whose k[row] is not in (0, n) gets b = NaN and p = NaN, and the
 * workspace status reads LAPSUM_EINVAL (lapsum_read_status); the other rows
 * are unaffected.  Host-side errors as lapsum_forward, plus LAPSUM_EINVAL for
 * k == NULL.
 */
size_t lapsum_workspace_bytes_rowk(int64_t B, int64_t n, int path);
int lapsum_forward_rowk(const float* r, int64_t ld, float* p, double* b, double* sum_f, int64_t B,
                        int64_t n, const double* k, double t, int path, void* ws, size_t ws_bytes,
                        void* support, size_t support_bytes, void* stream);

/*
 * Gradient support: a forward-to-backward hand-over for rows with n > 4096.
 * The pages define only the VJP itself (section 2.1); this pair is a layout
 * choice of this library.  f_i = 0.5 exp(-|x_i|) is exactly 0 in fp32 once
 * |x_i| = |r_i - b|/t exceeds 87.4, so only the scores with |x| <= 90 carry
 * gradient.  lapsum_forward_support computes everything lapsum_forward does
 * and, in the same pass that writes p, lists those scores (position and x)
 * in the caller's `support` buffer.  lapsum_backward_support then produces
 * the same g as lapsum_backward while reading v only at the listed scores and
 * not reading r at all: its traffic is the g write plus the list.
 *
 * lapsum_support_bytes: size of `support` for B rows of n scores (0 when
 * n <= 4096: those rows need no support and `support` may be NULL).  The
 * buffer is owned by the caller, must be 256-byte aligned, needs no
 * initialisation, and is written only by lapsum_forward_support (the backward
 * also keeps the gathered v beside each entry).  It stays valid until the
 * next forward into it; r and b must not change in between.
 *
 * The backward checks (on the device) that the list was written for the same
 * n and B and for this b of each row, and that no list share overflowed (at
 * most half of every 512 consecutive scores inside the window); rows that
 * fail any check, or whose smallest |x| is above 50 (then scores outside the
 * window could weigh in R), are recomputed from r and v by the dense
 * kernels, so the result never depends on the list being usable.
 * Errors: as lapsum_forward / lapsum_backward, plus LAPSUM_EWORKSPACE when
 * n > 4096 and `support` is NULL, misaligned or smaller than
 * lapsum_support_bytes(B, n).  The backward's `ws` is a lapsum_backward
 * workspace (lapsum_backward_workspace_bytes).
 */
size_t lapsum_support_bytes(int64_t B, int64_t n);
int lapsum_forward_support(const float* r, int64_t ld, float* p, double* b, double* sum_f,
                           int64_t B, int64_t n, double k, double t, int path, uint64_t seed,
                           void* ws, size_t ws_bytes, void* support, size_t support_bytes,
                           void* stream);
int lapsum_backward_support(const float* r, int64_t ld, const double* b, const float* v, float* g,
                            int64_t B, int64_t n, double t, const void* support,
                            size_t support_bytes, void* ws, size_t ws_bytes, void* stream);

/*
 * Gradients of L = sum_i v_i p_i with respect to each row's budget k and
 * temperature t, for learning them.  The pages give only the analytic VJP in
 * the scores (section 2.1); these follow from the same implicit
 * differentiation of the budget equation: with x_i = (r_i - b)/t and
 * f_i = 0.5 exp(-|x_i|),
 *     g_k[row] = dL/dk = sum_i v_i f_i / sum_i f_i,
 *     g_t[row] = dL/dt = -(1/t) sum_i v_i f_i (x_i - xbar),  xbar = sum f x / sum f.
 * One pass over r and v (8 bytes per score); weights shifted by the row's
 * smallest |x| as in lapsum_backward.  g_k and g_t are device arrays of B
 * doubles (either may be NULL, not both); ws is a lapsum_backward workspace.
 */
int lapsum_backward_kt(const float* r, int64_t ld, const double* b, const float* v, int64_t B,
                       int64_t n, double t, double* g_k, double* g_t, void* ws, size_t ws_bytes,
                       void* stream);

/*
 * Synchronises `stream`, copies the sticky device status word to
 * *device_status (LAPSUM_OK, or a LAPSUM_E* code for the first condition
 * seen) and clears it.  Returns LAPSUM_OK or LAPSUM_ECUDA.
 */
int lapsum_read_status(void* ws, void* stream, int* device_status);

/* Per-row record of the last forward call (diagnostics; host copy, syncs `stream`). */
typedef struct lapsum_row_info {
    double b;          /* threshold */
    double sum_f;      /* sum_i f_i at b */
    double S_L, S_R;   /* bracketing tail sums of the certified bracket */
    float a_L, a_R;    /* certified bracket (+-inf for an open side) */
    int64_t cnt_R;     /* scores >= a_R */
    int64_t n_band;    /* scores in [a_L, a_R) after the fold */
    int32_t path;      /* solver that ran (LAPSUM_PATH_*) */
    int32_t attempts;  /* brackets tried (1 = first bracket held) */
    int32_t sample_m;  /* bracketing sample size */
    int32_t rank_l;    /* first-attempt order-statistic ranks (descending, 1-based) */
    int32_t rank_h;
    int32_t refine_levels; /* histogram narrowing levels used on the band */
    int32_t status;    /* device status bits of this row */
    int32_t reserved;
} lapsum_row_info;

int lapsum_row_info_get(void* ws, int64_t row, lapsum_row_info* out, void* stream);

/*
 * Copies the bracketing sample of the last forward call on row `row`
 * (m values y_s = r[I_s] + eps_s, in draw order) to host memory `out`.
 * Syncs `stream`.  Returns LAPSUM_EINVAL if the last call did not bracket.
 */
int lapsum_sample_get(void* ws, int64_t row, float* out, int64_t m, void* stream);

/*
 * Optional per-kernel timing: while enabled, every kernel the library launches
 * is bracketed by a pair of CUDA events recorded on the launch stream.
 * lapsum_profile_enable(1) starts a fresh record, lapsum_profile_enable(0)
 * stops and clears it.  lapsum_profile_read waits for the recorded events and
 * returns, per kernel name, the number of launches and their summed device
 * time (first max_entries names; *n_entries gets the total count).  The
 * switch is process-wide and host-thread-safe; it is meant for benchmarks.
 */
typedef struct lapsum_kernel_time {
    char name[48];
    int64_t launches;
    double total_ms;
} lapsum_kernel_time;

int lapsum_profile_enable(int on);
int lapsum_profile_read(lapsum_kernel_time* out, int max_entries, int* n_entries);

/*
 * One row split over several devices (section 2.2's bracketing, with the row's
 * scores in contiguous shards, one per device and process).  Each device holds
 * the shard [offset, offset + n_shard) of a row of n scores; the caller moves
 * the small results between the steps (e.g. NCCL all-reduce / all-gather) and
 * every device then takes the same decisions:
 *   1. lapsum_bracket_plan (host): the sample size m and the rank ladders
 *      rank_l[4], rank_h[4] of the row (as the single-device bracketing);
 *   2. lapsum_shard_sample: y[s] (m floats, device) = draw s of the row's
 *      sample (the single-device sample, seed as lapsum_forward) when its
 *      index lies in this shard, else 0; summing y over the devices gives the
 *      whole sample exactly;
 *   3. lapsum_sample_bracket: ends = (a_L, a_R) (2 floats, device) from the
 *      whole sample: the rank_h-th and rank_l-th largest (0 = open end);
 *   4. lapsum_shard_fold: this shard folded with the bracket: rec (5 doubles,
 *      device) = (scores >= a_R, sum e^{(r - a_L)/t} below a_L, sum
 *      e^{-(r - a_R)/t} at or above a_R, non-finite flag, band size) and the
 *      band scores into band (capacity n_shard floats);
 *   5. lapsum_shard_band_solve: with every device's rec (recs[w * 5 + i]) and
 *      band (bands[w * stride + j], j < its band size): out (4 doubles,
 *      device) = (b, F(a_L), F(a_R), certified 1/0); when not certified the
 *      caller widens the failing end to its next rung (F(a_L) < k: rank_h,
 *      else rank_l) and repeats from step 3; b is NaN for a non-finite row;
 *   6. lapsum_shard_emit: p of this shard from b (device);
 *   backward: lapsum_shard_vjp_partial gives rec (3 doubles, device: the
 *   shard's smallest |x| and shifted sums of f and v f) and
 *   lapsum_shard_vjp_apply g of this shard from every device's rec (recs[w *
 *   3 + i], merged in device order).
 * The records are combined in device order, so every device computes the same
 * b bit for bit.  Workspace: lapsum_shard_workspace_bytes(n_shard) bytes
 * (cleared once with lapsum_workspace_init; steps 4 and the backward), and for
 * step 5 a scratch of lapsum_shard_band_bytes(world * stride) bytes, 256-byte
 * aligned.  Errors: LAPSUM_EINVAL for bad sizes, ranks or parameters,
 * LAPSUM_EWORKSPACE, LAPSUM_ECUDA.  All pointers are device pointers except
 * the outputs of lapsum_bracket_plan.
 */
int lapsum_bracket_plan(int64_t n, double k, int32_t* m, int64_t* rank_l, int64_t* rank_h);
size_t lapsum_shard_workspace_bytes(int64_t n_shard);
size_t lapsum_shard_band_bytes(int64_t n_band_total);
int lapsum_shard_sample(const float* r, int64_t n_shard, int64_t offset, int64_t n, double t,
                        uint64_t seed, int32_t m, float* y, void* stream);
int lapsum_sample_bracket(const float* y, int32_t m, int64_t rank_l, int64_t rank_h, float* ends,
                          void* stream);
int lapsum_shard_fold(const float* r, int64_t n_shard, const float* ends, double t, double* rec,
                      float* band, void* ws, size_t ws_bytes, void* stream);
int lapsum_shard_band_solve(const float* bands, int64_t stride, const double* recs, int32_t world,
                            const float* ends, double k, double t, double* out, void* scratch,
                            size_t scratch_bytes, void* stream);
int lapsum_shard_emit(const float* r, int64_t n_shard, const double* b, double t, float* p,
                      void* stream);
int lapsum_shard_vjp_partial(const float* r, const float* v, int64_t n_shard, const double* b,
                             double t, double* rec, void* ws, size_t ws_bytes, void* stream);
int lapsum_shard_vjp_apply(const float* r, const float* v, int64_t n_shard, const double* b,
                           double t, const double* recs, int32_t world, float* g, void* ws,
                           size_t ws_bytes, void* stream);

/*
 * lapsum_backward_noalloc: the same result as lapsum_backward, for callers
 * that cannot allocate device memory (no workspace argument).  The pages have
 * no counterpart of this call; it exists for code that must not allocate at
 * the point it needs the gradient: work recorded during a CUDA graph capture
 * under a no-allocation rule, hosts that reserve all device memory up front,
 * and plugin hosts that own every allocation.
 *
 * Scratch: a fixed 140 KiB array inside the library (one per GPU that loads
 * it, held until the process exits).  Limits: B <= 1024 rows, and for rows
 * longer than 4096 scores also 8 * (SM count) + B <= 4096 (true for every
 * B <= 1024 on a 148-SM B200); other calls return LAPSUM_EINVAL and launch
 * nothing.
 * The first call on each device looks up the array's device address (one
 * cudaGetSymbolAddress); make that first call before any stream capture.
 * Calls made outside a capture look the address up again (a device reset
 * reloads the library's device code and may move the array); calls made
 * while a capture records the stream use the address of the last lookup.
 * Every call on a device shares the one array and clears the part that must
 * start at zero itself, so calls that overlap on the GPU (different streams
 * without ordering between them) race and give wrong results; order them.
 * Never allocates or frees memory.  Returns LAPSUM_OK, LAPSUM_EINVAL or
 * LAPSUM_ECUDA.
 */
int lapsum_backward_noalloc(const float* r, int64_t ld, const double* b, const float* v, float* g,
                            int64_t B, int64_t n, double t, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LAPSUM_H */
