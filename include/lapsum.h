/*
 * lapsum.h -- C ABI of the B200 (sm_100a) Fast LapSum exact-budget soft top-k.
 *
 * The operator ("Fast LapSum: Exact Differentiable Top-k at Million Scale",
 * technical summary section 2.1): for each row of scores r (length n), a
 * temperature t > 0 and a budget 0 < k < n, find the scalar threshold b with
 *
 *     sum_i F((r_i - b)/t) = k,      F = standard Laplace CDF,
 *
 * return p_i = F((r_i - b)/t), and give the analytic vector-Jacobian product
 *
 *     grad_i = (f_i/t) (g_i - <g,f>/sum f),   f_i = exp(-|r_i - b|/t)/2.
 *
 * Two solvers sit behind lapsum_forward (same page, section 2.2, and the
 * abstract): the full-sort solver (sort, stable prefix/suffix scan, interval
 * search, closed-form root) and, for long rows, probabilistic bracketing
 * (kernel-noised sample, binomial order-statistic bracket [a_L, a_R), one
 * streaming pass folding out-of-band scores into tail sums, an exact solve on
 * the band only -- narrowed by a radix select steered by the threshold curve,
 * then the closed-form root -- a certification pass, and a full-sort fallback
 * when the certification fails).  Every step runs in this library's CUDA
 * kernels.
 *
 * Conventions for every entry point:
 *  - Pointers named *_dev are DEVICE memory, owned by the caller, on the
 *    current CUDA device; rows are contiguous, row-major [rows][n] with row
 *    stride n elements.  Nothing is retained after the call returns except the
 *    library's own workspace.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *    enqueued on it; no entry point synchronises the host except
 *    lapsum_get_stats* / lapsum_profile_read (documented) and a call that
 *    grows the stream's workspace (the first on a stream, or one needing more
 *    room): cudaMalloc, and cudaFree of what it replaces, which waits for the
 *    device.  New workspace is zeroed on `stream` itself, so any stream,
 *    non-blocking ones included, sees it ready.
 *  - Return value: LAPSUM_OK (0) or a negative LAPSUM_ERR_* code.  Argument
 *    errors are detected on the host before anything is enqueued.  Errors
 *    found on the device (non-finite scores, a grid-barrier wait that gave
 *    up) are reported by lapsum_get_stats / lapsum_get_stats_rows.
 *  - The library keeps one workspace per (device, stream); calls on the same
 *    stream are ordered, calls on different streams use different
 *    workspaces.  Not thread-safe for concurrent calls on the same stream.
 */
#ifndef LAPSUM_H
#define LAPSUM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                       /* cudaStream_t == struct CUstream_st* */

#if defined(__GNUC__)
#define LAPSUM_API __attribute__((visibility("default")))
#else
#define LAPSUM_API
#endif

#define LAPSUM_OK                   0
#define LAPSUM_ERR_ARG             -1     /* bad size, budget, temperature or null pointer */
#define LAPSUM_ERR_NONFINITE       -2     /* a score is NaN or +-inf (device-detected)      */
#define LAPSUM_ERR_ALLOC           -3     /* workspace allocation failed                    */
#define LAPSUM_ERR_DEVICE_TIMEOUT  -4     /* an inter-block wait gave up (spin cap)         */
#define LAPSUM_ERR_CUDA            -5     /* a CUDA runtime call failed                     */
#define LAPSUM_ERR_NO_ROOT         -6     /* solver found no crossing (internal)            */
#define LAPSUM_ERR_BOUNDS          -7     /* checked build only: an index or guard word failed */

/* Temperatures accepted by every entry point: LAPSUM_T_MIN <= t <= LAPSUM_T_MAX.
 * The kernels form x = (r - b)/t in fp32 with the scale log2(e)/t; outside this
 * range that scale (or its inverse) is not a finite, normal fp32 number. */
#define LAPSUM_T_MIN 1e-36
#define LAPSUM_T_MAX 1e36

/* Certification modes (lapsum_options.certify) */
#define LAPSUM_CERTIFY_PASS  0
#define LAPSUM_CERTIFY_FUSED 1

/* Solver paths */
#define LAPSUM_PATH_AUTO     0
#define LAPSUM_PATH_FULLSORT 1
#define LAPSUM_PATH_BRACKET  2

/*
 * Tuning of lapsum_forward_ex.  Zero in any field selects its default.
 *   seed        key of the Philox4x64-10 stream that draws the bracketing
 *               sample (default 0).
 *   sample_size s, the number of kernel-noised samples (default
 *               min(65536, max(4096, 2^floor(log2(n/64))))).
 *   delta       bracket miss probability bound (default 1e-6).
 *   band_cap    capacity of the band buffer in scores (default
 *               max(65536, 4 n (jL - jR + 2)/s), at most n).  A larger band
 *               fails certification and takes the full-sort fallback.
 *   spin_cap    polls before a grid-barrier wait of the device-wide sort gives up
 *               (default 2^20).  -1: give up at the first poll that finds the
 *               barrier still closed -- a way to exercise the timeout path, which then
 *               reports LAPSUM_ERR_DEVICE_TIMEOUT through lapsum_get_stats and
 *               leaves the library ready for the next call.
 *   force_path  LAPSUM_PATH_* (default AUTO: bracketing when n >= 2^20, else
 *               full sort).  Bracketing solves the rows of a batch together:
 *               every kernel takes one slice of its grid per row (rows <=
 *               65535), each row with its own sample (Philox counter word =
 *               row), bracket, band, certification and fallback.
 *   certify     LAPSUM_CERTIFY_PASS (default): the certification is its own
 *               linear pass over the row (the abstract's "one additional linear
 *               pass"); LAPSUM_CERTIFY_FUSED: the streaming pass also adds the
 *               band scores' certification terms and decides the verdict, so the
 *               row is read once less.
 *   widen       0 (default): a bracket that fails certification goes straight to
 *               the full-sort fallback.  1: first one widening round ("Fast
 *               LapSum", technical summary section 2.2 step 4, the bracket
 *               "iteratively widened"): when the failure is a miss -- the counts
 *               agree, the band fits, but G(a_R) >= k (b at or above a_R) or
 *               G(a_L) < k (b below a_L) -- the same sample is re-selected at the
 *               ranks of confidence delta^2 and the missed side becomes the new
 *               bracket: [a_R, y_(jR2)) or [y_(jL2), a_L).  The row is streamed,
 *               the band solved and the bracket certified again; the full sort
 *               runs only if that round fails too.  Every decision is taken on
 *               the device (the round's kernels return at once when it is not
 *               needed).
 */
typedef struct {
    uint64_t seed;
    int64_t  sample_size;
    double   delta;
    int64_t  band_cap;
    int32_t  spin_cap;
    int32_t  force_path;
    int32_t  certify;
    int32_t  widen;
    int32_t  reserved[2];
} lapsum_options;

/*
 * Diagnostics of one row of the last lapsum_forward* call on a stream: row 0
 * with lapsum_get_stats, every row with lapsum_get_stats_rows (the one-CTA
 * full-sort path of rows <= 32768 scores keeps row 0's only).
 *   path      LAPSUM_PATH_FULLSORT or LAPSUM_PATH_BRACKET
 *   verdict   bracketing: 1 certified, 0 not certified (fallback ran); -1 n/a
 *   status    device error bits: 1 non-finite score, 2 wait timeout,
 *             4 band overflow, 8 no crossing found, 16 index out of bounds
 *             (checked build)
 *   s, jR, jL sample size and order-statistic ranks of the bracket
 *   a_L, a_R  bracket ends (fp32, rounded outward)
 *   c_L, c_band, c_R   scores below a_L, in [a_L, a_R), at or above a_R
 *   S_L, S_R  tail sums sum_{r<a_L} e^{(r-a_L)/t}, sum_{r>=a_R} e^{-(r-a_R)/t}
 *   G_aL, G_aR  certification values G(a_L), G(a_R)
 *   b         the threshold of row 0
 *   sum_p     sum of the fp32 p of row 0, accumulated in fp64
 *   widened   1 if the widening round ran (then s..G_aR describe its bracket)
 *   flags     rare routes taken: 1 = more than 8192 sample keys shared a target's
 *             16-bit prefix, so the bracket select walked the whole sample
 */
typedef struct {
    int32_t path, verdict, status, fallback;
    int64_t s, jR, jL;
    int64_t c_L, c_band, c_R;
    float   a_L, a_R;
    double  S_L, S_R;
    double  G_aL, G_aR;
    double  b;
    double  sum_p;
    int64_t j_star;
    int64_t widened;
    int64_t flags;
    int64_t reserved[2];
} lapsum_stats;

/*
 * Forward: p_out_dev[rows][n] = F((scores - b)/t), b_out_dev[rows] = b (fp64).
 *   scores_dev  fp32 [rows][n], finite
 *   rows >= 1, n >= 1, 0 < k < n (real), LAPSUM_T_MIN <= t <= LAPSUM_T_MAX
 *   p_out_dev   fp32 [rows][n] (may not alias scores_dev)
 *   b_out_dev   fp64 [rows]
 * Path: "Fast LapSum", technical summary section 2.2 (full-sort solver;
 * probabilistic bracketing for n > 1e6) and abstract (certification, fallback).
 */
LAPSUM_API int lapsum_forward(const float *scores_dev, int64_t rows, int64_t n, double k, double t,
                   float *p_out_dev, double *b_out_dev, struct CUstream_st *stream);

/* As lapsum_forward, with tuning options (opt may be NULL: defaults). */
LAPSUM_API int lapsum_forward_ex(const float *scores_dev, int64_t rows, int64_t n, double k, double t,
                      float *p_out_dev, double *b_out_dev, const lapsum_options *opt,
                      struct CUstream_st *stream);

/*
 * Backward (analytic VJP, technical summary section 2.1):
 *   grad_out_dev[i] = (f_i/t)(g_i - <g,f>/sum f),  f_i = exp(-|scores_i - b|/t)/2,
 * per row, with b_dev[rows] the thresholds returned by the forward.
 * Pure function of (scores, b, g).  grad_out_dev may alias g_dev.
 */
LAPSUM_API int lapsum_backward(const float *scores_dev, const double *b_dev, const float *g_dev,
                    int64_t rows, int64_t n, double t, float *grad_out_dev,
                    struct CUstream_st *stream);

/*
 * One forward + VJP step on HOST buffers: copies the scores and g to the
 * device, runs lapsum_forward_ex and lapsum_backward, and copies p, b and grad
 * back, the copies overlapping the work where the data allow ("Fast LapSum",
 * technical summary sections 2.1-2.2):
 *
 *   scores in -> forward -> [p, b out  |  g in] -> backward -> grad out
 *
 * Host buffers (fp32 [rows][n], b fp64 [rows]): scores_h, g_h read; p_h, b_h,
 * grad_h written.  Page-locked host memory (cudaHostAlloc / pinned tensors)
 * lets the copies run asynchronously and in both directions at once; pageable
 * memory works, with synchronous copies.
 * Device buffers, caller-owned, of the same shapes: scores_dev, g_dev, p_dev,
 * grad_dev, b_dev (grad_dev may alias g_dev; nothing else may alias).
 * Enqueued on `stream` (the copies on two side streams of the library, ordered
 * against `stream` by events): the call returns at once, and the host buffers
 * hold the results once `stream` has been synchronised; until then they must
 * stay valid and untouched.
 * Returns: LAPSUM_ERR_ARG for a null pointer or the forward's argument and
 * option errors (all checked before anything is enqueued), LAPSUM_ERR_CUDA if a
 * copy, stream or event call fails, else the forward's and backward's own
 * codes; a forward or backward that fails once the copies are queued still
 * leaves `stream` waiting for every copy queued, so the buffers may be reused
 * once `stream` has been synchronised.
 */
LAPSUM_API int lapsum_step_host(const float *scores_h, const float *g_h, int64_t rows, int64_t n, double k,
                                double t, float *p_h, double *b_h, float *grad_h, const lapsum_options *opt,
                                float *scores_dev, float *g_dev, float *p_dev, double *b_dev, float *grad_dev,
                                struct CUstream_st *stream);

/* Copies the last forward's diagnostics to *out. Synchronises `stream`.
 * Returns the device error as a LAPSUM_ERR_* code (LAPSUM_OK if none). */
LAPSUM_API int lapsum_get_stats(lapsum_stats *out, struct CUstream_st *stream);

/*
 * Per-row diagnostics of the last lapsum_forward* call on a stream: fills
 * out[0 .. min(rows, max_rows)) (out: host array of max_rows entries), sets
 * *rows_out to the number filled.  Synchronises the stream.  Returns the first
 * device-found error over all rows (as lapsum_get_stats does for row 0), else 0;
 * LAPSUM_ERR_ARG for a null pointer or max_rows < 1.
 */
LAPSUM_API int lapsum_get_stats_rows(lapsum_stats *out, int64_t max_rows, int64_t *rows_out,
                                     struct CUstream_st *stream);

/* Static string for a return code. */
LAPSUM_API const char *lapsum_strerror(int code);

/* Frees every workspace of the current device (synchronises the device first).
 * No other host thread may be inside a call on that device meanwhile; the
 * stats of earlier calls are gone, and the next call on a stream allocates its
 * workspace again. */
LAPSUM_API int lapsum_release(void);

/*
 * Per-kernel timing.  lapsum_profile_enable(1) makes every later launch record
 * a CUDA event pair on its stream; lapsum_profile_read synchronises the device,
 * folds the pending pairs and copies up to `max` entries (kernel name, number
 * of launches, total milliseconds) into the arrays; it returns the number of
 * distinct kernels.  lapsum_profile_enable(0) stops recording; (2) also clears.
 */
LAPSUM_API int lapsum_profile_enable(int mode);
/* Record only launches whose kernel name contains `substring` (NULL or "": all). */
LAPSUM_API int lapsum_profile_filter(const char *substring);
LAPSUM_API int lapsum_profile_read(const char **names, int64_t *launches, double *total_ms, int max);

/*
 * Plan of the bracketing path for one row of n scores (host only, no device
 * work): the sample size s, the order-statistic ranks jR, jL and the band
 * capacity that lapsum_forward_ex would use with `opt` (NULL: defaults).
 * The ranks follow the binomial bound of the abstract / technical summary
 * section 2.2 step 1: X = #{y_j > b} ~ Binomial(s, k/n),
 *   jR = max{j : P(X < j) <= delta/2},  jL = min{j : P(X >= j) <= delta/2}.
 */
LAPSUM_API int lapsum_bracket_plan(int64_t n, double k, const lapsum_options *opt, int64_t *s,
                                   int64_t *jR, int64_t *jL, int64_t *band_cap);

/*
 * Self-test of two device math helpers against the CUDA math library, on n
 * device doubles (no other state touched; synchronous on `stream`):
 *   which = 0: out = 2^{-in} by the table-driven near-tier exponential used in
 *              the tail sums (valid for 0 <= in <= 1000), ref = exp2(-in);
 *   which = 1: out = the sampler's own ln(in) (in > 0, normal), ref = log(in).
 */
LAPSUM_API int lapsum_selftest_math(int which, const double *in_dev, double *out_dev,
                                    double *ref_dev, int64_t n, struct CUstream_st *stream);

/*
 * Backward without any device allocation.  The method's pages have no
 * counterpart of this entry point: it exists for callers that may not call
 * cudaMalloc while they run -- for instance a plugin inside a host framework
 * that owns all device memory, or a process held to a fixed memory budget.  lapsum_backward grows a per-stream workspace with
 * cudaMalloc on first use; this variant keeps its scratch (per-block partial
 * sums, one lambda and one counter per row) in a single array compiled into
 * the library, LAPSUM_NOALLOC_SCRATCH_BYTES per GPU, which every GPU that
 * loads the library holds until the process exits.
 *
 * Result: the same VJP as lapsum_backward, grad_out[i] = (f_i/t)(g_i -
 * <g,f>/sum f) per row, to within fp32 rounding (not bit-identical: the partial
 * sums are grouped differently).  Arguments as lapsum_backward; every pointer is
 * caller-owned device memory; nothing is allocated or freed.
 *
 * Limit: rows <= 7281 per call (any n < 2^31).  A call needs about
 * rows * (24 B + 12 B) of scratch with one block per row, more blocks per row
 * (and the same total) for fewer rows; a call that would not fit returns
 * LAPSUM_ERR_ARG before anything is enqueued.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) and keeps it for later calls.
 * All calls on a device share the one array: each call clears the counters it
 * needs, but two calls that overlap on the GPU (different streams, or host
 * threads) race on it -- order them on one stream.
 */
#define LAPSUM_NOALLOC_SCRATCH_BYTES 262144
LAPSUM_API int lapsum_backward_noalloc(const float *scores_dev, const double *b_dev,
                                       const float *g_dev, int64_t rows, int64_t n, double t,
                                       float *grad_out_dev, struct CUstream_st *stream);

/*
 * One row split across GPUs ("Fast LapSum", technical summary section 4.1:
 * rows of 1e8 scores and beyond, past one GPU's memory).  The row of n_total
 * scores is cut into contiguous slices, one per rank (one process per GPU);
 * rank q holds scores [offset_q, offset_q + n_local_q).  Every rank calls the
 * entry points below on its slice, in this order, on one stream, and exchanges
 * the small device buffers they produce with its collective library between the
 * calls (exact_budget_soft_b200.sharded does it with torch.distributed/NCCL):
 *
 *   lapsum_shard_plan        sizes of the exchange buffers (host only)
 *   lapsum_shard_sample      this rank's share of the bracketing sample
 *       -> all-reduce (sum) of the xbuf words over the ranks (as int32 or uint32)
 *   lapsum_shard_stream      bracket (identical on every rank) and the streaming
 *                            pass over the slice, certification terms folded in
 *       -> all-gather of the LAPSUM_SHARD_PART-double records, rank order;
 *          all-gather of each slice's band scores (record[2] of them), rank order
 *   lapsum_shard_solve       the row's counts and sums, the verdict, b
 *       (verdict 0: the bracket failed certification; the caller gathers the
 *        whole row and solves it with lapsum_forward_ex, force_path FULLSORT)
 *   lapsum_shard_p           p of the slice at b
 * and for the VJP:
 *   lapsum_shard_vjp_partial {sum e, sum g e, min |x|} of the slice, e = e^{shift-|x|}
 *       -> all-gather of the 3-double records, rank order; if the summed e is
 *          below 2^-96 (every score far from b), call it again with shift =
 *          the smallest min |x| over the ranks and all-gather again
 *   lapsum_shard_vjp_apply   grad of the slice
 *
 * The sample is the one-GPU sample of the whole row (same Philox counters, the
 * index drawn over n_total; each rank fills the draws that land in its slice),
 * so the bracket, the counts and the verdict equal those of lapsum_forward_ex on
 * the whole row (certify = LAPSUM_CERTIFY_FUSED).  Sums are combined in rank
 * order on every rank, so every rank gets the same b.  Options as for
 * lapsum_forward_ex, except widen and force_path (LAPSUM_ERR_ARG).  Pointers
 * are device memory on the rank's GPU; the library's per-stream workspace
 * carries state from one call to the next (lapsum_get_stats after
 * lapsum_shard_solve reports the whole row's bracket, counts and verdict).
 */
#define LAPSUM_SHARD_PART 10   /* c_L c_R c_band S_L S_R hL lR kmax kinv status (doubles) */

/* xbuf_words: uint32 words of the sample exchange buffer; band_cap: capacity of
 * every band buffer (a slice's, and the gathered band's: more fails certification). */
LAPSUM_API int lapsum_shard_plan(int64_t n_total, double k, const lapsum_options *opt,
                                 int64_t *xbuf_words, int64_t *band_cap);

/* Fills xbuf_dev[xbuf_words] with this slice's share of the sample (zero where
 * another rank owns the draw) and its select histograms; clears the workspace. */
LAPSUM_API int lapsum_shard_sample(const float *scores_dev, int64_t n_local, int64_t offset, int64_t n_total,
                                   double k, double t, const lapsum_options *opt, uint32_t *xbuf_dev,
                                   struct CUstream_st *stream);

/* From the summed xbuf: the bracket; then the slice's streaming pass.  Writes its
 * record part_dev[LAPSUM_SHARD_PART] and its band scores to band_dev[band_cap]
 * (record[2] of them; a count above band_cap keeps counting, and fails the row). */
LAPSUM_API int lapsum_shard_stream(const float *scores_dev, int64_t n_local, int64_t offset, int64_t n_total,
                                   double k, double t, const lapsum_options *opt, const uint32_t *xbuf_dev,
                                   double *part_dev, float *band_dev, struct CUstream_st *stream);

/* parts_dev[ranks][LAPSUM_SHARD_PART] in rank order; band_all_dev: the ranks'
 * band scores concatenated (band_total of them).  Writes b_out_dev[0] (fp64) and
 * verdict_out_dev[0] (1 certified; 0: use the full-sort fallback). */
LAPSUM_API int lapsum_shard_solve(const double *parts_dev, int64_t ranks, const float *band_all_dev,
                                  int64_t band_total, int64_t n_total, double k, double t,
                                  const lapsum_options *opt, double *b_out_dev, int32_t *verdict_out_dev,
                                  struct CUstream_st *stream);

/* p_out_dev[n_local] = F((scores - b)/t) for the slice, b = b_dev[0]. */
LAPSUM_API int lapsum_shard_p(const float *scores_dev, int64_t n_local, double t, const double *b_dev,
                              float *p_out_dev, struct CUstream_st *stream);

/* part_dev[3] = {sum_i e_i, sum_i g_i e_i, min_i |x_i|} over the slice,
 * e_i = e^{shift - |x_i|}, x_i = (scores_i - b)/t; shift >= 0. */
LAPSUM_API int lapsum_shard_vjp_partial(const float *scores_dev, const double *b_dev, const float *g_dev,
                                        int64_t n_local, double t, double shift, double *part_dev,
                                        struct CUstream_st *stream);

/* lambda = sum(sum g e)/sum(sum e) over parts_dev[ranks][3] (one shift for all,
 * rank order); grad_out_dev[n_local] = (f_i/t)(g_i - lambda) for the slice. */
LAPSUM_API int lapsum_shard_vjp_apply(const float *scores_dev, const double *b_dev, const float *g_dev,
                                      int64_t n_local, double t, const double *parts_dev, int64_t ranks,
                                      float *grad_out_dev, struct CUstream_st *stream);

/* Number of kernel launches enqueued by this library since load (a counter). */
LAPSUM_API int64_t lapsum_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* LAPSUM_H */
