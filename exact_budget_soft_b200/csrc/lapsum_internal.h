// lapsum_internal.h -- state shared by the host orchestration and the kernels.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace lapsum {

// Device error bits (lapsum_stats.status).
enum : int32_t {
    ST_NONFINITE = 1,
    ST_TIMEOUT = 2,
    ST_BAND_OVERFLOW = 4,
    ST_NO_ROOT = 8,
    ST_BOUNDS = 16,   // checked build: a computed index fell outside its buffer (the access was skipped)
};

// Device-resident control block of one single-row solve.  Every field is
// written by a kernel and read by a later kernel on the same stream; the host
// only clears it (one memset per call) and copies it back for diagnostics.
struct Ctl {
    // bracket (sample + select)
    float a_L, a_R;
    int64_t jR, jL, s;
    // streaming pass
    unsigned long long c_L, c_R, c_band;
    double S_L, S_R;
    unsigned int band_kmax;   // largest descending-order key in the band (every band score,
    unsigned int band_kinv;   //   past the capacity too) and the largest complemented key
    // certification pass
    double G_aL, G_aR;
    int32_t verdict;          // 1 certified, 0 not (fallback must run), -1 n/a
    int32_t widen_dir;        // failed certification: +1 b at or above a_R, -1 below a_L, 0 other
    int32_t widened;          // the widening round is running (or ran)
    int32_t status;           // ST_* bits
    int32_t path;
    int32_t fallback_ran;
    // solution
    double b;
    int64_t j_star;
    double sum_p;
    // single-pass "last block" tickets (zeroed with the block)
    unsigned int ticket[8];
    unsigned int sel_cnt[2];  // select: keys under each target's 16-bit prefix
    // device-wide sort
    unsigned int gbar_count;  // grid barrier of the cooperative sort: arrivals
    unsigned int gbar_gen;    //   and generation
    // backward
    double hL, lR;            // fused certification: band terms vs a_L and vs a_R
    double vjp_lambda;
    float vjp_min;            // split rows: the slice's smallest |x| (base 2; cleared to +inf)
    int32_t vjp_shift;        // sum f too small for fp32 terms: recompute lambda shifted
    int32_t flags;            // FLAG_* bits: which rare routes ran
};

// Rare routes a solve took (lapsum_stats.flags).
enum : int32_t {
    FLAG_SELECT_ALL_KEYS = 1,   // the select's candidate buffer overflowed: it walked every sample key
};

// Kernel-facing parameters of a bracketing solve.
// Kernel-facing parameters of a bracketing solve of `rows` rows (grid.y = row).
// Pointers are the bases of row 0; every per-row array has a fixed row stride
// (see at_row), so a kernel first takes its row's view.
struct BracketParams {
    const float *r;           // scores [rows][n]
    int64_t n;
    int64_t rows;
    double k, t, inv_t;
    uint64_t seed;
    int64_t row;              // the row of this view (the sample's Philox counter word)
    int64_t s;
    int64_t jR, jL;
    int64_t band_cap;
    float *band;              // band buffers [rows][band_cap]
    uint32_t *keys;           // sample keys [rows][s]
    uint32_t *hist1;          // [rows][HIST_WORDS] select histograms of the top 16 and top 8
                              //   key bits (zero between solves: the streaming pass clears them)
    uint32_t *cand;           // [rows][2][SEL_CAND] keys under each target's 16-bit prefix
    double *partials;         // per-block partials [rows][part_stride]
    int64_t part_stride;
    Ctl *ctl;                 // control blocks [rows]
    int32_t spin_cap;
    int32_t fused_cert;       // certification folded into the streaming pass
    int32_t widen;            // a widening round follows a missed bracket
    int32_t round2;           // this launch belongs to the widening round
    // a row split across ranks: this rank holds scores [shard_off, shard_off + n) of
    // a row of n_total (the sample draws global indices; 0 and n for a whole row)
    int64_t shard_off;
    int64_t n_total;
};

constexpr int64_t HIST_WORDS = 65536 + 256;
constexpr int64_t SEL_CAND_WORDS = 2 * 8192;

// The view of one row: every per-row pointer moved to that row.
__host__ __device__ inline BracketParams at_row(const BracketParams &P, int64_t row) {
    BracketParams Q = P;
    Q.row = row;
    Q.r = P.r + row * P.n;
    Q.band = P.band + row * P.band_cap;
    Q.keys = P.keys + row * P.s;
    Q.hist1 = P.hist1 + row * HIST_WORDS;
    Q.cand = P.cand + row * SEL_CAND_WORDS;
    Q.partials = P.partials + row * P.part_stride;
    Q.ctl = P.ctl + row;
    return Q;
}

}  // namespace lapsum
