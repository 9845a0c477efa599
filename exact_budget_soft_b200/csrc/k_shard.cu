// k_shard.cu -- one row split across GPUs ("Fast LapSum: Exact Differentiable
// Top-k at Million Scale", technical summary section 4.1: rows of 1e8 scores
// and beyond).  Each rank holds a contiguous slice of the row; the steps of the
// bracketing path run on the slices and the ranks exchange a few small buffers
// between them (the caller's collectives: an all-reduce of the sample, an
// all-gather of the partial sums and of the band scores, an all-gather of the
// VJP sums).  The bracket, the band solve and the certification verdict are the
// same computation on every rank, from the same exchanged data.
//
//   sample   the kernel-noised sample of the WHOLE row (same Philox counters as
//            one GPU): each rank fills the draws whose index lands in its slice;
//            summing the ranks' buffers gives every rank the full sample, so the
//            bracket equals the one-GPU bracket bit for bit.
//   stream   the order statistics (select, replicated), then the streaming pass
//            with the certification terms folded in, over the slice: counts,
//            tail sums, band-term sums, band key range, the slice's band scores.
//   solve    partial sums combined in rank order (so every rank gets the same
//            bits), the verdict, the band select on the gathered band -> b.
//   p        p of the slice at the shared b.
//   VJP      {sum e, sum g e, min |x|} per slice, combined in rank order.
#include <algorithm>
#include <cmath>
#include <cstring>

#include "../../include/lapsum.h"
#include "lapsum_device.cuh"
#include "lapsum_kernels.h"

namespace lapsum {

// Partial record of one slice's streaming pass (doubles; counts and keys are
// exact in fp64): the layout of LAPSUM_SHARD_PART.
enum : int {
    SP_CL = 0, SP_CR, SP_CBAND, SP_SL, SP_SR, SP_HL, SP_LR, SP_KMAX, SP_KINV, SP_STATUS,
    SP_WORDS
};
static_assert(SP_WORDS == LAPSUM_SHARD_PART, "partial record layout");

__global__ void shard_export_kernel(const Ctl *ctl, double *part) {
    pdl_enter();
    if (threadIdx.x != 0) return;
    part[SP_CL] = (double)ctl->c_L;
    part[SP_CR] = (double)ctl->c_R;
    part[SP_CBAND] = (double)ctl->c_band;
    part[SP_SL] = ctl->S_L;
    part[SP_SR] = ctl->S_R;
    part[SP_HL] = ctl->hL;
    part[SP_LR] = ctl->lR;
    part[SP_KMAX] = (double)ctl->band_kmax;
    part[SP_KINV] = (double)ctl->band_kinv;
    part[SP_STATUS] = (double)ctl->status;
}

// The whole row's counts and sums from the ranks' records (summed in rank
// order), and the certification verdict as the one-GPU fused pass decides it:
// G(a_L) >= k > G(a_R), the band fits, the counts cover the row, every score
// finite.
__global__ void shard_combine_kernel(Ctl *ctl, const double *parts, int64_t ranks, int64_t n_total, double k,
                                     double inv_t, int64_t band_cap) {
    pdl_enter();
    if (threadIdx.x != 0) return;
    double cL = 0, cR = 0, cb = 0, SL = 0, SR = 0, hL = 0, lR = 0;
    uint32_t kmax = 0, kinv = 0;
    int32_t status = 0;
    for (int64_t q = 0; q < ranks; ++q) {
        const double *p = parts + q * SP_WORDS;
        cL += p[SP_CL];
        cR += p[SP_CR];
        cb += p[SP_CBAND];
        SL += p[SP_SL];
        SR += p[SP_SR];
        hL += p[SP_HL];
        lR += p[SP_LR];
        kmax = max(kmax, (uint32_t)p[SP_KMAX]);
        kinv = max(kinv, (uint32_t)p[SP_KINV]);
        status |= (int32_t)p[SP_STATUS];
    }
    const unsigned long long icL = (unsigned long long)cL, icR = (unsigned long long)cR,
                             icb = (unsigned long long)cb;
    ctl->c_L = icL;
    ctl->c_R = icR;
    ctl->c_band = icb;
    ctl->S_L = SL;
    ctl->S_R = SR;
    ctl->hL = hL;
    ctl->lR = lR;
    ctl->band_kmax = kmax;
    ctl->band_kinv = kinv;
    ctl->status |= status & ST_NONFINITE;
    const double daL = ctl->a_L, daR = ctl->a_R;
    const double rho = (isinf(daR) || isinf(daL)) ? 0.0 : exp(-(daR - daL) * inv_t);
    const double GaL = (double)(icb + icR) - 0.5 * fma(rho, SR, hL) + 0.5 * SL;
    const double GaR = (double)icR - 0.5 * SR + 0.5 * fma(rho, SL, lR);
    ctl->G_aL = GaL;
    ctl->G_aR = GaR;
    const bool sound = icb <= (unsigned long long)band_cap && icL + icb + icR == (unsigned long long)n_total &&
                       (ctl->status & ST_NONFINITE) == 0;
    ctl->verdict = (sound && GaL >= k && GaR < k) ? 1 : 0;
    ctl->widen_dir = 0;
    if (icb > (unsigned long long)band_cap) atomicOr(&ctl->status, ST_BAND_OVERFLOW);
}

__global__ void shard_result_kernel(const Ctl *ctl, double *b_out, int32_t *verdict_out) {
    pdl_enter();
    if (threadIdx.x != 0) return;
    if (b_out) *b_out = ctl->b;
    if (verdict_out) *verdict_out = ctl->verdict;
}

__global__ void shard_set_b_kernel(Ctl *ctl, const double *b) {
    pdl_enter();
    if (threadIdx.x == 0) ctl->b = *b;
}

// lambda = sum g e / sum e over every slice's record {sum e, sum g e, min |x2|},
// in rank order.
__global__ void shard_vjp_combine_kernel(Ctl *ctl, const double *parts, int64_t ranks) {
    pdl_enter();
    if (threadIdx.x != 0) return;
    double sf = 0.0, sgf = 0.0;
    for (int64_t q = 0; q < ranks; ++q) {
        sf += parts[3 * q];
        sgf += parts[3 * q + 1];
    }
    ctl->vjp_lambda = sgf / sf;
}

}  // namespace lapsum

// =================================================================== ABI --
using namespace lapsum;

namespace lapsum {
// the per-stream workspace of lapsum_api.cu
struct ShardWs {
    Ctl *ctl;
    double *partials;
    uint32_t *skeys, *hist1, *cand;
    float *band;
    int64_t band_cap;
};
int shard_workspace(struct CUstream_st *stream, int64_t s, int64_t band_cap, ShardWs *out);
}  // namespace lapsum

namespace {

int map_cuda(cudaError_t e) { return e == cudaSuccess ? LAPSUM_OK : (e == cudaErrorMemoryAllocation ? LAPSUM_ERR_ALLOC : LAPSUM_ERR_CUDA); }

#define SHARD_TRY(expr)                                 \
    do {                                                \
        const cudaError_t _e = (expr);                  \
        if (_e != cudaSuccess) return map_cuda(_e);     \
    } while (0)

int check_slice(const float *scores, int64_t n_local, int64_t offset, int64_t n_total, double k, double t) {
    if (!scores || n_local < 1 || offset < 0 || n_total < 2 || n_total >= (int64_t(1) << 40)) return LAPSUM_ERR_ARG;
    if (offset + n_local > n_total || n_local >= (int64_t(1) << 31)) return LAPSUM_ERR_ARG;
    if (!(k > 0.0) || !(k < (double)n_total) || !std::isfinite(k)) return LAPSUM_ERR_ARG;
    if (!(t >= LAPSUM_T_MIN && t <= LAPSUM_T_MAX)) return LAPSUM_ERR_ARG;
    return LAPSUM_OK;
}

int slice_params(const float *scores, int64_t n_local, int64_t offset, int64_t n_total, double k, double t,
                 const lapsum_options *opt, BracketParams &P, int64_t &band_cap) {
    lapsum_options o{};
    if (opt) o = *opt;
    if (o.widen != 0 || o.force_path == LAPSUM_PATH_FULLSORT) return LAPSUM_ERR_ARG;   // not on split rows
    int64_t s = 0;
    int rc = lapsum_bracket_plan(n_total, k, &o, &s, &P.jR, &P.jL, &band_cap);
    if (rc) return rc;
    P.r = scores;
    P.n = n_local;
    P.rows = 1;
    P.k = k;
    P.t = t;
    P.inv_t = 1.0 / t;
    P.seed = o.seed;
    P.row = 0;
    P.s = s;
    P.band_cap = band_cap;
    P.spin_cap = 1 << 20;
    P.fused_cert = 1;
    P.widen = 0;
    P.round2 = 0;
    P.shard_off = offset;
    P.n_total = n_total;
    return LAPSUM_OK;
}

}  // namespace

extern "C" {

int lapsum_shard_plan(int64_t n_total, double k, const lapsum_options *opt, int64_t *xbuf_words,
                      int64_t *band_cap) {
    if (!xbuf_words || !band_cap) return LAPSUM_ERR_ARG;
    int64_t s = 0, jR = 0, jL = 0;
    const int rc = lapsum_bracket_plan(n_total, k, opt, &s, &jR, &jL, band_cap);
    if (rc) return rc;
    *xbuf_words = s + HIST_WORDS;
    return LAPSUM_OK;
}

int lapsum_shard_sample(const float *scores, int64_t n_local, int64_t offset, int64_t n_total, double k, double t,
                        const lapsum_options *opt, uint32_t *xbuf, struct CUstream_st *stream_in) {
    int rc = check_slice(scores, n_local, offset, n_total, k, t);
    if (rc) return rc;
    if (!xbuf) return LAPSUM_ERR_ARG;
    BracketParams P{};
    int64_t band_cap = 0;
    rc = slice_params(scores, n_local, offset, n_total, k, t, opt, P, band_cap);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_in);
    ShardWs w{};
    rc = shard_workspace(stream_in, P.s, band_cap, &w);
    if (rc) return rc;
    SHARD_TRY(cudaMemsetAsync(w.ctl, 0, sizeof(Ctl), st));
    SHARD_TRY(cudaMemsetAsync(xbuf, 0, (size_t)(P.s + HIST_WORDS) * sizeof(uint32_t), st));
    P.keys = xbuf;
    P.hist1 = xbuf + P.s;
    P.ctl = w.ctl;
    P.partials = w.partials;
    P.part_stride = partial_stride(1);
    P.band = w.band;
    P.cand = w.cand;
    SHARD_TRY(launch_sample(P, st));
    return LAPSUM_OK;
}

int lapsum_shard_stream(const float *scores, int64_t n_local, int64_t offset, int64_t n_total, double k, double t,
                        const lapsum_options *opt, const uint32_t *xbuf, double *part, float *band_out,
                        struct CUstream_st *stream_in) {
    int rc = check_slice(scores, n_local, offset, n_total, k, t);
    if (rc) return rc;
    if (!xbuf || !part || !band_out) return LAPSUM_ERR_ARG;
    BracketParams P{};
    int64_t band_cap = 0;
    rc = slice_params(scores, n_local, offset, n_total, k, t, opt, P, band_cap);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_in);
    ShardWs w{};
    rc = shard_workspace(stream_in, P.s, band_cap, &w);
    if (rc) return rc;
    // the summed sample and histograms into the workspace; the select reads them there
    SHARD_TRY(cudaMemcpyAsync(w.skeys, xbuf, (size_t)P.s * sizeof(uint32_t), cudaMemcpyDeviceToDevice, st));
    SHARD_TRY(cudaMemcpyAsync(w.hist1, xbuf + P.s, (size_t)HIST_WORDS * sizeof(uint32_t), cudaMemcpyDeviceToDevice, st));
    P.keys = w.skeys;
    P.hist1 = w.hist1;
    P.cand = w.cand;
    P.ctl = w.ctl;
    P.partials = w.partials;
    P.part_stride = partial_stride(1);
    P.band = band_out;   // the slice's band scores go straight to the caller's exchange buffer
    SHARD_TRY(launch_select(P, st));
    SHARD_TRY(launch_stream_pass(P, st));
    SHARD_TRY(launch_k(shard_export_kernel, 1, 32, 0, st, (const Ctl *)w.ctl, part));
    return LAPSUM_OK;
}

int lapsum_shard_solve(const double *parts, int64_t ranks, const float *band_all, int64_t band_total,
                       int64_t n_total, double k, double t, const lapsum_options *opt, double *b_out,
                       int32_t *verdict_out, struct CUstream_st *stream_in) {
    if (!parts || ranks < 1 || band_total < 0 || (band_total > 0 && !band_all) || !b_out || !verdict_out)
        return LAPSUM_ERR_ARG;
    if (n_total < 2 || !(k > 0.0) || !(k < (double)n_total) || !(t >= LAPSUM_T_MIN && t <= LAPSUM_T_MAX))
        return LAPSUM_ERR_ARG;
    lapsum_options o{};
    if (opt) o = *opt;
    int64_t s = 0, jR = 0, jL = 0, band_cap = 0;
    int rc = lapsum_bracket_plan(n_total, k, &o, &s, &jR, &jL, &band_cap);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_in);
    ShardWs w{};
    rc = shard_workspace(stream_in, s, band_cap, &w);
    if (rc) return rc;
    SHARD_TRY(launch_k(shard_combine_kernel, 1, 32, 0, st, w.ctl, parts, ranks, n_total, k, 1.0 / t, band_cap));
    const int64_t nb = std::min(band_total, band_cap);
    if (nb > 0)
        SHARD_TRY(cudaMemcpyAsync(w.band, band_all, (size_t)nb * sizeof(float), cudaMemcpyDeviceToDevice, st));
    SHARD_TRY(launch_band_select(w.band, 1, k, t, w.ctl, band_cap, 0, st));
    SHARD_TRY(launch_k(shard_result_kernel, 1, 32, 0, st, (const Ctl *)w.ctl, b_out, verdict_out));
    return LAPSUM_OK;
}

int lapsum_shard_p(const float *scores, int64_t n_local, double t, const double *b, float *p_out,
                   struct CUstream_st *stream_in) {
    if (!scores || !b || !p_out || n_local < 1 || n_local >= (int64_t(1) << 31)) return LAPSUM_ERR_ARG;
    if (!(t >= LAPSUM_T_MIN && t <= LAPSUM_T_MAX)) return LAPSUM_ERR_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_in);
    ShardWs w{};
    const int rc = shard_workspace(stream_in, 0, 0, &w);
    if (rc) return rc;
    SHARD_TRY(launch_k(shard_set_b_kernel, 1, 32, 0, st, w.ctl, b));
    SHARD_TRY(launch_p_pass(scores, 1, n_local, t, p_out, nullptr, w.ctl, w.partials, st));
    return LAPSUM_OK;
}

int lapsum_shard_vjp_partial(const float *scores, const double *b, const float *g, int64_t n_local, double t,
                             double shift, double *part, struct CUstream_st *stream_in) {
    if (!scores || !b || !g || !part || n_local < 1 || n_local >= (int64_t(1) << 31)) return LAPSUM_ERR_ARG;
    if (!(t >= LAPSUM_T_MIN && t <= LAPSUM_T_MAX) || !(shift >= 0.0) || !std::isfinite(shift)) return LAPSUM_ERR_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_in);
    ShardWs w{};
    const int rc = shard_workspace(stream_in, 0, 0, &w);
    if (rc) return rc;
    // the slice minimum starts at the largest float the byte pattern 0x7f gives (3.4e38)
    SHARD_TRY(cudaMemsetAsync(&w.ctl->vjp_min, 0x7f, sizeof(float), st));
    SHARD_TRY(cudaMemsetAsync(&w.ctl->ticket[3], 0, sizeof(unsigned), st));
    SHARD_TRY(launch_vjp_slice_partial(scores, b, g, n_local, t, (float)(shift * LOG2E), w.ctl,
                                       w.partials, part, st));
    return LAPSUM_OK;
}

int lapsum_shard_vjp_apply(const float *scores, const double *b, const float *g, int64_t n_local, double t,
                           const double *parts, int64_t ranks, float *grad_out, struct CUstream_st *stream_in) {
    if (!scores || !b || !g || !parts || !grad_out || ranks < 1 || n_local < 1 || n_local >= (int64_t(1) << 31))
        return LAPSUM_ERR_ARG;
    if (!(t >= LAPSUM_T_MIN && t <= LAPSUM_T_MAX)) return LAPSUM_ERR_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_in);
    ShardWs w{};
    const int rc = shard_workspace(stream_in, 0, 0, &w);
    if (rc) return rc;
    SHARD_TRY(launch_k(shard_vjp_combine_kernel, 1, 32, 0, st, w.ctl, parts, ranks));
    SHARD_TRY(launch_vjp_apply(scores, b, g, 1, n_local, t, w.ctl, grad_out, st));
    return LAPSUM_OK;
}

}  // extern "C"
