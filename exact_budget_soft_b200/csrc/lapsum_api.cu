// lapsum_api.cu -- the C ABI (include/lapsum.h): argument checks, per-stream
// workspace, the launch sequence of each solver path, diagnostics, timing.
//
// Paths ("Fast LapSum: Exact Differentiable Top-k at Million Scale",
// technical summary section 2.2, and the abstract):
//   full sort, n <= 32768      one launch: one CTA per row sorts, scans, solves
//                              and writes p
//   full sort, longer rows     device radix sort -> locate-scan -> p pass
//   bracketing (n >= 2^20 by   sample -> select -> streaming pass -> band select
//   default; rows of a batch   (one CTA per row) -> certification (or folded into
//   each bracketed)            the streaming pass) -> optional widening round ->
//                              gated full-sort fallback -> p pass
//   VJP                        one CTA per short row, else reduce -> apply
//   host buffers               lapsum_step_host: the copies on two side streams
// No step synchronises the host: the band size and the verdict live in device
// memory and every gated kernel returns at once when it has nothing to do.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <utility>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/lapsum.h"
#include "lapsum_internal.h"
#include "lapsum_kernels.h"

namespace lapsum {

namespace {
std::mutex g_dev_mu;
std::map<int, int> g_dev_sms;
std::map<std::tuple<int, const void *, size_t>, cudaError_t> g_dev_smem;
std::map<std::tuple<int, const void *, int, size_t>, int> g_dev_resident;
int current_device() {
    int dev = 0;
    cudaGetDevice(&dev);
    return dev;
}
}  // namespace

int device_sm_count() {
    const int dev = current_device();
    std::lock_guard<std::mutex> lk(g_dev_mu);
    auto it = g_dev_sms.find(dev);
    if (it != g_dev_sms.end()) return it->second;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
    g_dev_sms[dev] = sms;
    return sms;
}

cudaError_t set_max_dynamic_smem(const void *kern, size_t bytes) {
    const auto key = std::make_tuple(current_device(), kern, bytes);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    auto it = g_dev_smem.find(key);
    if (it != g_dev_smem.end()) return it->second;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    g_dev_smem[key] = e;
    return e;
}

std::map<int, bool> g_coop_pdl_refused;
bool coop_pdl_refused() {
    const int dev = current_device();
    std::lock_guard<std::mutex> lk(g_dev_mu);
    return g_coop_pdl_refused.count(dev) != 0;
}
void coop_pdl_refuse() {
    const int dev = current_device();
    std::lock_guard<std::mutex> lk(g_dev_mu);
    g_coop_pdl_refused[dev] = true;
}

cudaError_t resident_ctas(const void *kern, int threads, size_t smem, int *out) {
    const int sms = device_sm_count();
    const auto key = std::make_tuple(current_device(), kern, threads, smem);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    auto it = g_dev_resident.find(key);
    if (it != g_dev_resident.end()) {
        *out = it->second;
        return cudaSuccess;
    }
    int per_sm = 0;
    const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    *out = g_dev_resident[key] = per_sm * sms;
    return cudaSuccess;
}

}  // namespace lapsum

using namespace lapsum;

namespace {

// ------------------------------------------------------------ profiling --
struct ProfRec {
    const char *name;
    cudaEvent_t e0, e1;
};
struct ProfAcc {
    int64_t launches = 0;
    double ms = 0.0;
};
std::mutex g_prof_mu;
int g_prof_mode = 0;
std::string g_prof_filter;
std::vector<ProfRec> g_prof_pending;
std::vector<std::pair<std::string, ProfAcc>> g_prof_acc;
std::vector<cudaEvent_t> g_event_pool;
int64_t g_launches = 0;

cudaEvent_t take_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e;
    cudaEventCreate(&e);
    return e;
}

// RAII: counts one kernel launch, names it for tracing tools (an NVTX range
// around the host-side launch, named after the solver step: free when no tool
// is attached) and, when profiling, brackets it with events.
struct Launch {
    const char *name;
    cudaStream_t st;
    cudaEvent_t e0 = nullptr;
    Launch(const char *nm, cudaStream_t s) : name(nm), st(s) {
        nvtxRangePushA(nm);
        std::lock_guard<std::mutex> lk(g_prof_mu);
        ++g_launches;
        if (g_prof_mode && (g_prof_filter.empty() || std::strstr(nm, g_prof_filter.c_str()))) {
            e0 = take_event();
            cudaEventRecord(e0, st);
        }
    }
    ~Launch() {
        nvtxRangePop();
        if (!e0) return;
        std::lock_guard<std::mutex> lk(g_prof_mu);
        cudaEvent_t e1 = take_event();
        cudaEventRecord(e1, st);
        g_prof_pending.push_back({name, e0, e1});
    }
};

// ------------------------------------------------------------ workspace --
// The checked build (-DLAPSUM_CHECKED) puts GUARD_BYTES of a fixed pattern after
// every workspace buffer and verifies them at the end of every call.
#ifdef LAPSUM_CHECKED
constexpr size_t GUARD_BYTES = 256;
#else
constexpr size_t GUARD_BYTES = 0;
#endif
constexpr unsigned char GUARD_FILL = 0xA5;

// A new buffer is zeroed (and its guard filled) on the caller's stream st, so the
// call's kernels, queued after it on st, see the zeros whatever kind of stream st
// is (a plain cudaMemset runs on the legacy default stream, which a non-blocking
// stream is not ordered after).  cudaFree of an outgrown buffer waits for the
// device, so no queued kernel still reads it.
template <typename T>
cudaError_t grow(T *&p, size_t &have, size_t need, cudaStream_t st) {
    if (need <= have && p) return cudaSuccess;
    if (p) {
        cudaFree(p);
        p = nullptr;
        have = 0;
    }
    size_t n = need < 64 ? 64 : need;
    cudaError_t e = cudaMalloc(reinterpret_cast<void **>(&p), n * sizeof(T) + GUARD_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(p, 0, n * sizeof(T), st);
    if (e == cudaSuccess && GUARD_BYTES)
        e = cudaMemsetAsync(reinterpret_cast<char *>(p) + n * sizeof(T), GUARD_FILL, GUARD_BYTES, st);
    have = n;
    return e;
}

struct Workspace {
    Ctl *ctl = nullptr;               size_t ctl_n = 0;
    double *partials = nullptr;       size_t partials_n = 0;
    uint32_t *skeys = nullptr;        size_t skeys_n = 0;
    uint32_t *hist1 = nullptr;        size_t hist1_n = 0;
    uint32_t *selcand = nullptr;      size_t selcand_n = 0;
    float *band = nullptr;            size_t band_n = 0;
    uint32_t *keys0 = nullptr;        size_t keys0_n = 0;
    unsigned long long *hist = nullptr; size_t hist_n = 0;
    uint32_t *chunkcnt = nullptr; size_t chunkcnt_n = 0;
    double *tilebuf = nullptr;        size_t tilebuf_n = 0;
    int64_t rows = 1;                 // rows of the last solve (their control blocks hold its stats)

    void release() {
        cudaFree(ctl); cudaFree(partials); cudaFree(skeys); cudaFree(hist1); cudaFree(selcand); cudaFree(band);
        cudaFree(keys0); cudaFree(hist);
        cudaFree(chunkcnt); cudaFree(tilebuf);
        *this = Workspace();
    }

    // checked build: every buffer's guard bytes still hold the fill pattern
    // (synchronises the stream); LAPSUM_ERR_BOUNDS otherwise
    int verify_guards(cudaStream_t st) const {
        if (!GUARD_BYTES) return LAPSUM_OK;
        const std::pair<const void *, size_t> bufs[] = {
            {ctl, ctl_n * sizeof(Ctl)}, {partials, partials_n * sizeof(double)},
            {skeys, skeys_n * 4}, {hist1, hist1_n * 4}, {selcand, selcand_n * 4}, {band, band_n * 4},
            {keys0, keys0_n * 4}, {hist, hist_n * 8}, {chunkcnt, chunkcnt_n * 4},
            {tilebuf, tilebuf_n * 8}};
        if (cudaStreamSynchronize(st) != cudaSuccess) return LAPSUM_ERR_CUDA;
        constexpr size_t NG = GUARD_BYTES ? GUARD_BYTES : 1;
        unsigned char g[NG];
        for (const auto &b : bufs) {
            if (!b.first) continue;
            if (cudaMemcpy(g, static_cast<const char *>(b.first) + b.second, NG, cudaMemcpyDeviceToHost) != cudaSuccess)
                return LAPSUM_ERR_CUDA;
            for (size_t i = 0; i < NG; ++i)
                if (g[i] != GUARD_FILL) return LAPSUM_ERR_BOUNDS;
        }
        return LAPSUM_OK;
    }
};

std::mutex g_ws_mu;
std::map<std::pair<int, cudaStream_t>, Workspace *> g_ws;

Workspace *get_ws(cudaStream_t st) {
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(g_ws_mu);
    auto key = std::make_pair(dev, st);
    auto it = g_ws.find(key);
    if (it != g_ws.end()) return it->second;
    Workspace *w = new Workspace();
    g_ws[key] = w;
    return w;
}

// Control blocks and per-block partials for a batch of rows.
cudaError_t ws_base(Workspace *w, int64_t rows, cudaStream_t st) {
    cudaError_t e = grow(w->ctl, w->ctl_n, (size_t)rows, st);
    if (e == cudaSuccess) e = grow(w->partials, w->partials_n, (size_t)(rows * partial_stride(rows)), st);
    return e;
}

// The device sort's buffers.  Its second key buffer is the caller's p output
// (n floats per row, written only by the p pass after the sort), so the
// workspace holds one key buffer of the row, not two.
cudaError_t ws_sort(Workspace *w, int64_t cap, cudaStream_t st) {
    cudaError_t e = grow(w->keys0, w->keys0_n, (size_t)cap, st);
    if (e == cudaSuccess) e = grow(w->hist, w->hist_n, 4 * 256 + 6, st);   // + give-up/clean-up counts, per-sign varying bits
    if (e == cudaSuccess) e = grow(w->chunkcnt, w->chunkcnt_n, (size_t)4 * 256 * sort_grid_max(), st);
    if (e == cudaSuccess) e = grow(w->tilebuf, w->tilebuf_n, (size_t)sort_record_doubles(cap), st);
    return e;
}

SortArgs sort_args(Workspace *w, const float *src, float *p_out, int64_t n, int64_t cap, int32_t gate,
                   int32_t spin_cap, double k, double t) {
    SortArgs A{};
    A.k = k;
    A.t = t;
    A.src = src;
    A.n_host = n;
    A.cap = cap;
    A.keys[0] = w->keys0;
    A.keys[1] = reinterpret_cast<uint32_t *>(p_out);
    A.hist = w->hist;
    A.chunkcnt = w->chunkcnt;
    A.tilebuf = w->tilebuf;
    A.ctl = w->ctl;
    A.gate = gate;
    A.spin_cap = spin_cap;
    A.rows = 1;
    A.src_stride = 0;
    return A;
}

int map_err(cudaError_t e) {
    if (e == cudaSuccess) return LAPSUM_OK;
    if (e == cudaErrorMemoryAllocation) return LAPSUM_ERR_ALLOC;
    return LAPSUM_ERR_CUDA;
}

#define LAPSUM_TRY(expr)                            \
    do {                                            \
        cudaError_t _e = (expr);                    \
        if (_e != cudaSuccess) return map_err(_e);  \
    } while (0)

// ---------------------------------------------------- binomial ranks --
// Ranks of the binomial order-statistic bracket ("Fast LapSum" abstract and
// technical summary section 2.2 step 1): X = #{y_j > b} ~ Binomial(s, pi = k/n).
//   jR = largest j with P(X < j) <= delta/2 (0 -> a_R = +inf),
//   jL = smallest j with P(X >= j) <= delta/2 (s+1 -> a_L = -inf).
// The pmf is built outward from the mode by the ratio recurrence
// pmf(j+1)/pmf(j) = (s-j)/(j+1) * pi/(1-pi), relative to the mode (no logs per
// term), until terms fall below 1e-300 of the mode; the mode's own value comes
// from lgamma.  Results are memoised per (s, pi, delta).
void binomial_ranks_compute(int64_t s, double pi, double delta, int64_t &jR, int64_t &jL) {
    int64_t mode = (int64_t)std::floor((double)(s + 1) * pi);
    if (mode > s) mode = s;
    const double lmode = std::lgamma((double)s + 1.0) - std::lgamma((double)mode + 1.0) -
                         std::lgamma((double)(s - mode) + 1.0) + (double)mode * std::log(pi) +
                         (double)(s - mode) * std::log1p(-pi);
    const double pmode = std::exp(lmode);
    const double odds = pi / (1.0 - pi);
    std::vector<double> up, down;   // relative pmf above / below the mode
    double w = 1.0;
    for (int64_t j = mode; j < s && w > 1e-300; ++j) {
        w *= ((double)(s - j) / (double)(j + 1)) * odds;
        up.push_back(w);            // pmf(j+1)/pmf(mode)
    }
    w = 1.0;
    for (int64_t j = mode; j > 0 && w > 1e-300; --j) {
        w *= ((double)j / (double)(s - j + 1)) / odds;
        down.push_back(w);          // pmf(j-1)/pmf(mode)
    }
    const int64_t lo = mode - (int64_t)down.size();   // smallest j with a stored term
    const int64_t hi = mode + (int64_t)up.size();
    auto rel = [&](int64_t j) -> double {
        if (j == mode) return 1.0;
        if (j > mode) return up[(size_t)(j - mode - 1)];
        return down[(size_t)(mode - j - 1)];
    };
    const double half = 0.5 * delta / pmode;   // thresholds in units of pmf(mode)
    // lower tail P(X < j), smallest terms first (Kahan)
    double acc = 0.0, comp = 0.0;
    jR = lo;                                       // P(X < lo) is negligible
    for (int64_t j = lo + 1; j <= s + 1 && j - 1 <= hi; ++j) {
        const double y = rel(j - 1) - comp, tt = acc + y;
        comp = (tt - acc) - y;
        acc = tt;                                  // acc = P(X < j) / pmf(mode)
        if (acc <= half) jR = j; else break;
    }
    if (jR > s) jR = s;
    acc = 0.0; comp = 0.0;
    jL = hi + 1;                                   // P(X >= hi+1) is negligible
    for (int64_t j = hi; j >= lo; --j) {
        const double y = rel(j) - comp, tt = acc + y;
        comp = (tt - acc) - y;
        acc = tt;                                  // acc = P(X >= j) / pmf(mode)
        if (acc <= half) jL = j; else break;
    }
    if (jL > s + 1) jL = s + 1;
}

struct RankKey {
    int64_t s;
    uint64_t pi_bits, delta_bits;
    bool operator<(const RankKey &o) const {
        if (s != o.s) return s < o.s;
        if (pi_bits != o.pi_bits) return pi_bits < o.pi_bits;
        return delta_bits < o.delta_bits;
    }
};
std::mutex g_rank_mu;
std::map<RankKey, std::pair<int64_t, int64_t>> g_rank_cache;

void binomial_ranks(int64_t s, double pi, double delta, int64_t &jR, int64_t &jL) {
    RankKey key{s, 0, 0};
    std::memcpy(&key.pi_bits, &pi, 8);
    std::memcpy(&key.delta_bits, &delta, 8);
    {
        std::lock_guard<std::mutex> lk(g_rank_mu);
        auto it = g_rank_cache.find(key);
        if (it != g_rank_cache.end()) {
            jR = it->second.first;
            jL = it->second.second;
            return;
        }
    }
    binomial_ranks_compute(s, pi, delta, jR, jL);
    std::lock_guard<std::mutex> lk(g_rank_mu);
    if (g_rank_cache.size() > 4096) g_rank_cache.clear();
    g_rank_cache[key] = {jR, jL};
}

int check_args(const float *scores, int64_t rows, int64_t n, double k, double t) {
    if (!scores || rows < 1 || n < 1 || n >= (int64_t(1) << 31)) return LAPSUM_ERR_ARG;
    if (!(k > 0.0) || !(k < (double)n) || !std::isfinite(k)) return LAPSUM_ERR_ARG;
    if (!(t >= LAPSUM_T_MIN && t <= LAPSUM_T_MAX)) return LAPSUM_ERR_ARG;
    return LAPSUM_OK;
}

// The options a forward accepts for `rows` rows of n scores (opt null: the
// defaults), and the solver path they select.
int check_options(const lapsum_options &opt, int64_t rows, int64_t n, int *path_out) {
    if (opt.delta != 0.0 && !(opt.delta > 0.0 && opt.delta < 1.0)) return LAPSUM_ERR_ARG;
    if (opt.sample_size < 0 || opt.band_cap < 0 || opt.spin_cap < -1) return LAPSUM_ERR_ARG;
    if (opt.force_path < 0 || opt.force_path > 2) return LAPSUM_ERR_ARG;
    if (opt.certify != LAPSUM_CERTIFY_PASS && opt.certify != LAPSUM_CERTIFY_FUSED) return LAPSUM_ERR_ARG;
    if (opt.widen != 0 && opt.widen != 1) return LAPSUM_ERR_ARG;
    int path = opt.force_path;
    if (path == LAPSUM_PATH_AUTO)   // long rows bracket, one or many (a batch shares the kernels)
        path = n >= (int64_t(1) << 20) ? LAPSUM_PATH_BRACKET : LAPSUM_PATH_FULLSORT;
    if (path == LAPSUM_PATH_BRACKET && rows > 65535) return LAPSUM_ERR_ARG;   // grid.y holds the row
    if (path_out) *path_out = path;
    return LAPSUM_OK;
}

// Full sort of long rows on the device (also the certification fallback): one
// cooperative kernel walks the rows, each gated by its own control block.
int full_sort_rows(Workspace *w, const float *r, float *p_out, int64_t rows, int64_t n, double k, double t,
                   int32_t gate, int32_t spin_cap, cudaStream_t st) {
    LAPSUM_TRY(ws_sort(w, n, st));
    SortArgs A = sort_args(w, r, p_out, n, n, gate, spin_cap, k, t);
    A.rows = rows;
    A.src_stride = n;
    {
        Launch L("radix_sort", st);   // sort and locate, one cooperative kernel
        LAPSUM_TRY(launch_radix_sort(A, k, t, st));
    }
    return LAPSUM_OK;
}

}  // namespace

namespace lapsum {
struct ShardWs {
    Ctl *ctl;
    double *partials;
    uint32_t *skeys, *hist1, *cand;
    float *band;
    int64_t band_cap;
};
// The stream's workspace for one slice of a split row (k_shard.cu): a control
// block and partials for one row, sample keys (s), select histograms and
// candidates, a band buffer of band_cap scores.  Zero sizes keep what is there.
int shard_workspace(struct CUstream_st *stream, int64_t s, int64_t band_cap, ShardWs *out) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    Workspace *w = get_ws(st);
    w->rows = 1;
    LAPSUM_TRY(ws_base(w, 1, st));
    LAPSUM_TRY(grow(w->skeys, w->skeys_n, (size_t)std::max<int64_t>(s, 1), st));
    LAPSUM_TRY(grow(w->hist1, w->hist1_n, (size_t)HIST_WORDS, st));
    LAPSUM_TRY(grow(w->selcand, w->selcand_n, (size_t)SEL_CAND_WORDS, st));
    LAPSUM_TRY(grow(w->band, w->band_n, (size_t)std::max<int64_t>(band_cap, 1), st));
    *out = ShardWs{w->ctl, w->partials, w->skeys, w->hist1, w->selcand, w->band, (int64_t)w->band_n};
    return LAPSUM_OK;
}
}  // namespace lapsum

// ===================================================================== ABI --
extern "C" {

const char *lapsum_strerror(int code) {
    switch (code) {
        case LAPSUM_OK: return "ok";
        case LAPSUM_ERR_ARG: return "invalid argument";
        case LAPSUM_ERR_NONFINITE: return "non-finite score";
        case LAPSUM_ERR_ALLOC: return "workspace allocation failed";
        case LAPSUM_ERR_DEVICE_TIMEOUT: return "an inter-block wait gave up (spin cap)";
        case LAPSUM_ERR_CUDA: return "CUDA runtime error";
        case LAPSUM_ERR_NO_ROOT: return "no crossing found";
        case LAPSUM_ERR_BOUNDS: return "checked build: an index or a guard word was out of bounds";
        default: return "unknown error";
    }
}

static int forward_impl(const float *scores, int64_t rows, int64_t n, double k, double t,
                        float *p_out, double *b_out, const lapsum_options *opt_in,
                        struct CUstream_st *stream_in);

int lapsum_forward_ex(const float *scores, int64_t rows, int64_t n, double k, double t,
                      float *p_out, double *b_out, const lapsum_options *opt_in,
                      struct CUstream_st *stream_in) {
    const int rc = forward_impl(scores, rows, n, k, t, p_out, b_out, opt_in, stream_in);
    if (rc || !GUARD_BYTES) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_in);
    return get_ws(st)->verify_guards(st);
}

static int forward_impl(const float *scores, int64_t rows, int64_t n, double k, double t,
                        float *p_out, double *b_out, const lapsum_options *opt_in,
                        struct CUstream_st *stream_in) {
    int rc = check_args(scores, rows, n, k, t);
    if (rc) return rc;
    if (!p_out || !b_out) return LAPSUM_ERR_ARG;
    lapsum_options opt{};
    if (opt_in) opt = *opt_in;
    int path = LAPSUM_PATH_AUTO;
    rc = check_options(opt, rows, n, &path);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_in);
    // spin_cap -1: grid-barrier waits give up at their first poll (exercises the timeout path)
    const int32_t spin_cap = opt.spin_cap > 0 ? opt.spin_cap : (opt.spin_cap == 0 ? (1 << 20) : 0);
    Workspace *w = get_ws(st);
    w->rows = path == LAPSUM_PATH_FULLSORT && n <= rowsolve_capacity() ? 1 : rows;
    LAPSUM_TRY(ws_base(w, w->rows, st));

    if (path == LAPSUM_PATH_FULLSORT) {
        if (n <= rowsolve_capacity()) {
            LAPSUM_TRY(cudaMemsetAsync(w->ctl, 0, sizeof(Ctl), st));
            Launch L("rowsolve", st);
            LAPSUM_TRY(launch_rowsolve_rows(scores, rows, n, k, t, p_out, b_out, w->ctl, st));
            return LAPSUM_OK;
        }
        LAPSUM_TRY(cudaMemsetAsync(w->ctl, 0, sizeof(Ctl) * (size_t)rows, st));
        rc = full_sort_rows(w, scores, p_out, rows, n, k, t, GATE_ALWAYS, spin_cap, st);
        if (rc) return rc;
        Launch L("p_pass", st);
        LAPSUM_TRY(launch_p_pass(scores, rows, n, t, p_out, b_out, w->ctl, w->partials, st));
        return LAPSUM_OK;
    }

    // ---------------------------------------------------- bracketing --
    BracketParams P{};
    P.r = scores;
    P.n = n;
    P.rows = rows;
    P.k = k;
    P.t = t;
    P.inv_t = 1.0 / t;
    P.seed = opt.seed;
    P.row = 0;
    P.shard_off = 0;
    P.n_total = n;
    int64_t s = 0, band_cap = 0;
    rc = lapsum_bracket_plan(n, k, &opt, &s, &P.jR, &P.jL, &band_cap);
    if (rc) return rc;
    P.s = s;
    P.band_cap = band_cap;
    P.spin_cap = spin_cap;
    P.fused_cert = opt.certify == LAPSUM_CERTIFY_FUSED;
    P.widen = opt.widen;
    // the widening round, on the same sample: the ranks of confidence delta^2,
    // moved at least one first-round spread (jL - jR, at least 1) beyond the first
    // round's ranks and clipped to [0, s + 1]; its band lies between a first-round
    // end and the new end on the side that was missed
    BracketParams P2{};
    if (opt.widen) {
        P2 = P;
        P2.round2 = 1;
        const double delta = opt.delta != 0.0 ? opt.delta : 1e-6;
        binomial_ranks(s, k / (double)n, std::max(delta * delta, 1e-300), P2.jR, P2.jL);
        const int64_t spread = std::max<int64_t>(1, P.jL - P.jR);
        P2.jR = std::max<int64_t>(0, std::min(P2.jR, P.jR - spread));
        P2.jL = std::min<int64_t>(s + 1, std::max(P2.jL, P.jL + spread));
        int64_t cap2 = opt.band_cap;
        if (cap2 == 0) {
            const int64_t gap = std::max(P.jR - P2.jR, P2.jL - P.jL);
            const double want = 4.0 * (double)n * (double)(gap + 2) / (double)s;
            cap2 = std::max<int64_t>(65536, (int64_t)std::ceil(want));
        }
        P2.band_cap = std::min<int64_t>(cap2, n);
    }
    const int64_t band_buf = std::max(band_cap, opt.widen ? P2.band_cap : int64_t(0));
    const size_t R = (size_t)rows;
    LAPSUM_TRY(grow(w->skeys, w->skeys_n, R * (size_t)s, st));
    LAPSUM_TRY(grow(w->hist1, w->hist1_n, R * (size_t)HIST_WORDS, st));
    LAPSUM_TRY(grow(w->selcand, w->selcand_n, R * (size_t)SEL_CAND_WORDS, st));
    LAPSUM_TRY(grow(w->band, w->band_n, R * (size_t)band_buf, st));
    LAPSUM_TRY(ws_sort(w, n, st));   // the fallback may sort a whole row (rows one after another)

    P2.band = P.band = w->band;
    P2.keys = P.keys = w->skeys;
    P2.hist1 = P.hist1 = w->hist1;
    P2.cand = P.cand = w->selcand;
    P2.partials = P.partials = w->partials;
    P2.part_stride = P.part_stride = partial_stride(rows);
    P2.ctl = P.ctl = w->ctl;

    LAPSUM_TRY(cudaMemsetAsync(w->ctl, 0, sizeof(Ctl) * R, st));
    // one bracketing round: sample, select, stream, band solve, certification
    auto bracket_round = [&](const BracketParams &Q) -> int {
        const bool r2 = Q.round2 != 0;   // profiling names are literals (the profiler keeps the pointer)
        { Launch L(r2 ? "widen_sample" : "sample", st); LAPSUM_TRY(launch_sample(Q, st)); }
        { Launch L(r2 ? "widen_select" : "select", st); LAPSUM_TRY(launch_select(Q, st)); }
        { Launch L(r2 ? "widen_stream_pass" : "stream_pass", st); LAPSUM_TRY(launch_stream_pass(Q, st)); }
        { Launch L(r2 ? "widen_band_select" : "band_select", st); LAPSUM_TRY(launch_band_select(w->band, rows, k, t, w->ctl, Q.band_cap, Q.round2, st)); }
        if (!Q.fused_cert) { Launch L(r2 ? "widen_certify" : "certify", st); LAPSUM_TRY(launch_certify(Q, st)); }
        return LAPSUM_OK;
    };
    rc = bracket_round(P);
    if (rc) return rc;
    if (opt.widen) {
        rc = bracket_round(P2);
        if (rc) return rc;
    }
    rc = full_sort_rows(w, scores, p_out, rows, n, k, t, GATE_FALLBACK, spin_cap, st);
    if (rc) return rc;
    { Launch L("p_pass", st); LAPSUM_TRY(launch_p_pass(scores, rows, n, t, p_out, b_out, w->ctl, w->partials, st)); }
    return LAPSUM_OK;
}

int lapsum_bracket_plan(int64_t n, double k, const lapsum_options *opt_in, int64_t *s_out,
                        int64_t *jR, int64_t *jL, int64_t *band_cap_out) {
    if (n < 1 || !(k > 0.0) || !(k < (double)n) || !s_out || !jR || !jL || !band_cap_out)
        return LAPSUM_ERR_ARG;
    lapsum_options opt{};
    if (opt_in) opt = *opt_in;
    if (opt.delta != 0.0 && !(opt.delta > 0.0 && opt.delta < 1.0)) return LAPSUM_ERR_ARG;
    if (opt.sample_size < 0 || opt.band_cap < 0) return LAPSUM_ERR_ARG;
    int64_t s = opt.sample_size;
    if (s == 0) {
        int64_t pw = 1;
        while (pw * 2 <= n / 64) pw *= 2;
        s = std::min<int64_t>(65536, std::max<int64_t>(4096, pw));
    }
    if (s > (int64_t(1) << 24)) return LAPSUM_ERR_ARG;
    const double delta = opt.delta != 0.0 ? opt.delta : 1e-6;
    binomial_ranks(s, k / (double)n, delta, *jR, *jL);
    int64_t band_cap = opt.band_cap;
    if (band_cap == 0) {
        const double want = 4.0 * (double)n * (double)(*jL - *jR + 2) / (double)s;
        band_cap = std::max<int64_t>(65536, (int64_t)std::ceil(want));
    }
    *band_cap_out = std::min<int64_t>(band_cap, n);
    *s_out = s;
    return LAPSUM_OK;
}

int lapsum_forward(const float *scores, int64_t rows, int64_t n, double k, double t, float *p_out,
                   double *b_out, struct CUstream_st *stream) {
    return lapsum_forward_ex(scores, rows, n, k, t, p_out, b_out, nullptr, stream);
}

int lapsum_backward(const float *scores, const double *b, const float *g, int64_t rows, int64_t n,
                    double t, float *grad_out, struct CUstream_st *stream_in) {
    if (!scores || !b || !g || !grad_out || rows < 1 || n < 1 || n >= (int64_t(1) << 31))
        return LAPSUM_ERR_ARG;
    if (!(t >= LAPSUM_T_MIN && t <= LAPSUM_T_MAX)) return LAPSUM_ERR_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_in);
    if (n <= 65536 || rows > 65535) {   // short rows: one CTA per row
        Launch L("rowvjp", st);
        LAPSUM_TRY(launch_rowvjp(scores, b, g, rows, n, t, grad_out, st));
        return LAPSUM_OK;
    }
    // long rows: the streaming passes, the rows of a batch sharing the grid
    Workspace *w = get_ws(st);
    LAPSUM_TRY(ws_base(w, rows, st));
    { Launch L("vjp_reduce", st); LAPSUM_TRY(launch_vjp_reduce(scores, b, g, rows, n, t, w->ctl, w->partials, st)); }
    { Launch L("vjp_apply", st); LAPSUM_TRY(launch_vjp_apply(scores, b, g, rows, n, t, w->ctl, grad_out, st)); }
    return w->verify_guards(st);
}

// ---- one step on host buffers: copies on two side streams per device ----
namespace {
struct SideStreams {
    cudaStream_t h2d = nullptr, d2h = nullptr;
};
std::mutex g_side_mu;
std::map<int, SideStreams> g_side;

cudaError_t side_streams(SideStreams *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(g_side_mu);
    SideStreams &s = g_side[dev];
    if (!s.h2d && (e = cudaStreamCreateWithFlags(&s.h2d, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if (!s.d2h && (e = cudaStreamCreateWithFlags(&s.d2h, cudaStreamNonBlocking)) != cudaSuccess) return e;
    *out = s;
    return cudaSuccess;
}

// Events of one call: released when the call returns (the device keeps an
// event it still has to complete).
struct StepEvents {
    cudaEvent_t e[6] = {};
    cudaError_t create() {
        for (auto &x : e) {
            const cudaError_t r = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
            if (r != cudaSuccess) return r;
        }
        return cudaSuccess;
    }
    ~StepEvents() {
        for (auto &x : e)
            if (x) cudaEventDestroy(x);
    }
};
}  // namespace

int lapsum_step_host(const float *scores_h, const float *g_h, int64_t rows, int64_t n, double k, double t,
                     float *p_h, double *b_h, float *grad_h, const lapsum_options *opt, float *scores_dev,
                     float *g_dev, float *p_dev, double *b_dev, float *grad_dev, struct CUstream_st *stream_in) {
    if (!scores_h || !g_h || !p_h || !b_h || !grad_h || !g_dev || !p_dev || !b_dev || !grad_dev) return LAPSUM_ERR_ARG;
    int rc = check_args(scores_dev, rows, n, k, t);
    if (rc != LAPSUM_OK) return rc;
    {
        lapsum_options o{};
        if (opt) o = *opt;
        rc = check_options(o, rows, n, nullptr);
        if (rc != LAPSUM_OK) return rc;
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_in);
    const size_t bytes = (size_t)rows * (size_t)n * sizeof(float);
    SideStreams ss;
    LAPSUM_TRY(side_streams(&ss));
    StepEvents ev;   // 0 start, 1 scores in, 2 g in, 3 forward done, 4 backward done, 5 copies out
    LAPSUM_TRY(ev.create());
    LAPSUM_TRY(cudaEventRecord(ev.e[0], st));   // after the caller's earlier work on `stream`
    LAPSUM_TRY(cudaStreamWaitEvent(ss.h2d, ev.e[0], 0));
    LAPSUM_TRY(cudaMemcpyAsync(scores_dev, scores_h, bytes, cudaMemcpyHostToDevice, ss.h2d));
    LAPSUM_TRY(cudaEventRecord(ev.e[1], ss.h2d));
    LAPSUM_TRY(cudaMemcpyAsync(g_dev, g_h, bytes, cudaMemcpyHostToDevice, ss.h2d));
    LAPSUM_TRY(cudaEventRecord(ev.e[2], ss.h2d));
    LAPSUM_TRY(cudaStreamWaitEvent(st, ev.e[1], 0));
    // a call that fails past this point still leaves `stream` waiting for every
    // copy it queued, so the caller may reuse the buffers once the stream is done
    auto fail = [&](int code) {
        cudaStreamWaitEvent(st, ev.e[2], 0);
        if (cudaEventRecord(ev.e[5], ss.d2h) == cudaSuccess) cudaStreamWaitEvent(st, ev.e[5], 0);
        return code;
    };
    rc = lapsum_forward_ex(scores_dev, rows, n, k, t, p_dev, b_dev, opt, stream_in);
    if (rc != LAPSUM_OK) return fail(rc);
    LAPSUM_TRY(cudaEventRecord(ev.e[3], st));
    LAPSUM_TRY(cudaStreamWaitEvent(ss.d2h, ev.e[3], 0));   // p and b leave while g arrives
    LAPSUM_TRY(cudaMemcpyAsync(p_h, p_dev, bytes, cudaMemcpyDeviceToHost, ss.d2h));
    LAPSUM_TRY(cudaMemcpyAsync(b_h, b_dev, (size_t)rows * sizeof(double), cudaMemcpyDeviceToHost, ss.d2h));
    LAPSUM_TRY(cudaStreamWaitEvent(st, ev.e[2], 0));
    rc = lapsum_backward(scores_dev, b_dev, g_dev, rows, n, t, grad_dev, stream_in);
    if (rc != LAPSUM_OK) return fail(rc);
    LAPSUM_TRY(cudaEventRecord(ev.e[4], st));
    LAPSUM_TRY(cudaStreamWaitEvent(ss.d2h, ev.e[4], 0));
    LAPSUM_TRY(cudaMemcpyAsync(grad_h, grad_dev, bytes, cudaMemcpyDeviceToHost, ss.d2h));
    LAPSUM_TRY(cudaEventRecord(ev.e[5], ss.d2h));
    LAPSUM_TRY(cudaStreamWaitEvent(st, ev.e[5], 0));   // `stream` completes once every copy has
    return LAPSUM_OK;
}

static void fill_stats(const Ctl &c, lapsum_stats *out) {
    std::memset(out, 0, sizeof(*out));
    out->path = c.path == 2 ? LAPSUM_PATH_BRACKET : LAPSUM_PATH_FULLSORT;
    out->verdict = c.path == 2 ? c.verdict : -1;
    out->status = c.status;
    out->fallback = c.fallback_ran;
    out->s = c.s;
    out->jR = c.jR;
    out->jL = c.jL;
    out->c_L = (int64_t)c.c_L;
    out->c_band = (int64_t)c.c_band;
    out->c_R = (int64_t)c.c_R;
    out->a_L = c.a_L;
    out->a_R = c.a_R;
    out->S_L = c.S_L;
    out->S_R = c.S_R;
    out->G_aL = c.G_aL;
    out->G_aR = c.G_aR;
    out->b = c.b;
    out->sum_p = c.sum_p;
    out->j_star = c.j_star;
    out->widened = c.widened;
    out->flags = c.flags;
}

static int stats_rc(const Ctl &c) {
    if (c.status & ST_BOUNDS) return LAPSUM_ERR_BOUNDS;
    if (c.status & ST_NONFINITE) return LAPSUM_ERR_NONFINITE;
    if (c.status & ST_TIMEOUT) return LAPSUM_ERR_DEVICE_TIMEOUT;
    if ((c.status & ST_NO_ROOT) && !(c.path == 2 && c.fallback_ran)) return LAPSUM_ERR_NO_ROOT;
    return LAPSUM_OK;
}

int lapsum_get_stats(lapsum_stats *out, struct CUstream_st *stream_in) {
    if (!out) return LAPSUM_ERR_ARG;
    int64_t got = 0;
    return lapsum_get_stats_rows(out, 1, &got, stream_in);
}

int lapsum_get_stats_rows(lapsum_stats *out, int64_t max_rows, int64_t *rows_out,
                          struct CUstream_st *stream_in) {
    if (!out || !rows_out || max_rows < 1) return LAPSUM_ERR_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_in);
    Workspace *w = get_ws(st);
    *rows_out = 0;
    std::memset(out, 0, sizeof(*out) * (size_t)max_rows);
    if (!w->ctl) return LAPSUM_OK;
    LAPSUM_TRY(cudaStreamSynchronize(st));
    const int64_t rows = std::min<int64_t>(w->rows, (int64_t)w->ctl_n);
    std::vector<Ctl> c((size_t)rows);
    LAPSUM_TRY(cudaMemcpy(c.data(), w->ctl, sizeof(Ctl) * (size_t)rows, cudaMemcpyDeviceToHost));
    int rc = LAPSUM_OK;
    for (int64_t i = 0; i < rows; ++i) {   // the first error over all rows of the last solve
        const int ri = stats_rc(c[(size_t)i]);
        if (rc == LAPSUM_OK) rc = ri;
        if (i < max_rows) fill_stats(c[(size_t)i], out + i);
    }
    *rows_out = std::min(rows, max_rows);
    return rc;
}

int lapsum_release(void) {
    cudaDeviceSynchronize();
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(g_ws_mu);
    for (auto it = g_ws.begin(); it != g_ws.end();) {
        if (it->first.first == dev) {
            it->second->release();
            delete it->second;
            it = g_ws.erase(it);
        } else {
            ++it;
        }
    }
    return LAPSUM_OK;
}

int lapsum_profile_enable(int mode) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (mode == 2) {
        for (auto &r : g_prof_pending) {
            g_event_pool.push_back(r.e0);
            g_event_pool.push_back(r.e1);
        }
        g_prof_pending.clear();
        g_prof_acc.clear();
        mode = g_prof_mode;
    }
    g_prof_mode = mode ? 1 : 0;
    return LAPSUM_OK;
}

int lapsum_profile_filter(const char *substring) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_filter = substring ? substring : "";
    return LAPSUM_OK;
}

int lapsum_selftest_math(int which, const double *in, double *out, double *ref, int64_t n,
                         struct CUstream_st *stream_in) {
    if (!in || !out || !ref || n < 1 || (which != 0 && which != 1)) return LAPSUM_ERR_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_in);
    LAPSUM_TRY(launch_selftest_math(which, in, out, ref, n, st));
    LAPSUM_TRY(cudaStreamSynchronize(st));
    return LAPSUM_OK;
}

int lapsum_profile_read(const char **names, int64_t *launches, double *total_ms, int max) {
    cudaDeviceSynchronize();
    std::lock_guard<std::mutex> lk(g_prof_mu);
    for (auto &r : g_prof_pending) {
        float ms = 0.f;
        cudaEventElapsedTime(&ms, r.e0, r.e1);
        bool found = false;
        for (auto &a : g_prof_acc) {
            if (a.first == r.name) {
                a.second.launches += 1;
                a.second.ms += ms;
                found = true;
                break;
            }
        }
        if (!found) g_prof_acc.push_back({std::string(r.name), ProfAcc{1, (double)ms}});
        g_event_pool.push_back(r.e0);
        g_event_pool.push_back(r.e1);
    }
    g_prof_pending.clear();
    int i = 0;
    for (auto &a : g_prof_acc) {
        if (i >= max) break;
        if (names) names[i] = a.first.c_str();
        if (launches) launches[i] = a.second.launches;
        if (total_ms) total_ms[i] = a.second.ms;
        ++i;
    }
    return (int)g_prof_acc.size();
}

int64_t lapsum_launch_count(void) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    return g_launches;
}

}  // extern "C"
