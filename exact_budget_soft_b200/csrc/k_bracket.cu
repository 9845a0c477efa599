// k_bracket.cu -- probabilistic bracketing and the streaming passes
// ("Fast LapSum: Exact Differentiable Top-k at Million Scale": technical
// summary section 2.2 steps 1-4, and the abstract).
//
//   sample_kernel   kernel-noised sample y_j = r_{I_j} + t L_j (Philox4x64-10)
//   select_kernel   exact order statistics y_(jR), y_(jL) by 3-round radix select
//                   over a grid (last CTA finishes)
//   oob_kernel<OOB_STREAM>  streaming pass: counts and stable tail sums of the
//                      scores outside [a_L, a_R), band compaction
//   oob_kernel<OOB_CERT>  certification pass: G(a_L), G(a_R) and the verdict
//   p_kernel        p = F((r - b)/t)
//   vjp_*_kernel    <g,f>/sum f, then grad = (f/t)(g - <g,f>/sum f)
//
// The long passes are persistent grids that walk the row in 8 KB chunks staged
// in shared memory by bulk copies (bulk_stream), chunk c to block c mod grid, so
// every per-block partial covers a fixed set of elements and the "last block"
// combine (one atomic ticket, fixed summation order) makes every reduction
// bitwise reproducible.
#include <cstdint>

#include "lapsum_device.cuh"
#include "lapsum_kernels.h"

namespace lapsum {

constexpr int SBLOCK = 256;     // threads per block of the streaming passes
constexpr int SBLOCKS_PER_SM = 4;

int stream_grid(int per_sm) { return device_sm_count() * per_sm; }
int stream_grid() { return stream_grid(SBLOCKS_PER_SM); }

// ------------------------------------------------------ last-block combine --
// Every block contributes NV doubles (valid in thread 0).  The block that
// arrives last sums the partials in a fixed order; returns true there, with the
// totals in thread 0's v[].
template <int BLOCK, int NV>
__device__ bool last_block_sum(double (&v)[NV], double *partials, unsigned *ticket,
                               double *scratch) {
    __shared__ bool s_last;
    const int tid = threadIdx.x;
    const int G = gridDim.x;
    if (tid == 0) {
#pragma unroll
        for (int i = 0; i < NV; ++i) partials[(size_t)i * G + blockIdx.x] = v[i];
        __threadfence();
        unsigned tk = atomicAdd(ticket, 1u);
        s_last = (tk == (unsigned)G - 1);
    }
    __syncthreads();
    if (!s_last) return false;
    __threadfence();
    // each thread sums its blocks j = tid, tid + BLOCK, ... in that order; the NV
    // values of JW of them are loaded together, so the combine waits for one L2
    // round trip per JW blocks instead of one per block and value
    constexpr int JW = NV >= 8 ? 1 : 8 / NV;
    double w[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) w[i] = 0.0;
    for (int j0 = tid; j0 < G; j0 += JW * BLOCK) {
        double x[NV][JW];
#pragma unroll
        for (int i = 0; i < NV; ++i)
#pragma unroll
            for (int u = 0; u < JW; ++u) {
                const int j = j0 + u * BLOCK;
                x[i][u] = j < G ? __ldcg(partials + (size_t)i * G + j) : 0.0;
            }
#pragma unroll
        for (int i = 0; i < NV; ++i)
#pragma unroll
            for (int u = 0; u < JW; ++u)
                if (j0 + u * BLOCK < G) w[i] += x[i][u];
    }
    block_sum<BLOCK, NV>(w, scratch);
    if (tid == 0) {
#pragma unroll
        for (int i = 0; i < NV; ++i) v[i] = w[i];
        *ticket = 0u;
    }
    return true;
}

// ================================================================ sample --
// Philox4x64-10 (Salmon et al., SC'11): per round, multiply words 0 and 2 by the
// round multipliers, cross the high halves over and xor in the key; the key is
// bumped by two Weyl constants between rounds.
__device__ __forceinline__ void philox4x64_10(uint64_t &x0, uint64_t &x1, uint64_t &x2,
                                              uint64_t &x3, uint64_t k0, uint64_t k1) {
    const uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
    const uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        uint64_t h0 = __umul64hi(M0, x0), l0 = M0 * x0;
        uint64_t h1 = __umul64hi(M1, x2), l1 = M1 * x2;
        uint64_t y0 = h1 ^ x1 ^ k0, y2 = h0 ^ x3 ^ k1;
        x0 = y0;
        x1 = l1;
        x2 = y2;
        x3 = l0;
        k0 += W0;
        k1 += W1;
    }
}

// ln x for the sampler, from ln m = 2 atanh((m-1)/(m+1)), x = m 2^e with m in
// [sqrt(1/2), sqrt(2)): atanh(s)/s = sum_j s^{2j}/(2j+1), 11 terms (|s| <= 0.1716),
// ln x = e ln2 + ln m.  Written with explicitly rounded IEEE operations only, so
// a CPU evaluating the same formula in the same order gets the same bits.
__device__ __forceinline__ double sample_ln(double x) {
    uint64_t bits = (uint64_t)__double_as_longlong(x);
    int64_t e = (int64_t)((bits >> 52) & 0x7ff) - 1022;
    double m = __longlong_as_double((long long)((bits & 0x800FFFFFFFFFFFFFull) | (0x3FEull << 52)));
    if (m < 0x1.6a09e667f3bcdp-1) {
        m = __dadd_rn(m, m);
        e -= 1;
    }
    double s = __ddiv_rn(__dsub_rn(m, 1.0), __dadd_rn(m, 1.0));
    double z = __dmul_rn(s, s);
    double p = 1.0 / 21.0;                 // correctly rounded constants, folded by the compiler
    p = __fma_rn(p, z, 1.0 / 19.0);
    p = __fma_rn(p, z, 1.0 / 17.0);
    p = __fma_rn(p, z, 1.0 / 15.0);
    p = __fma_rn(p, z, 1.0 / 13.0);
    p = __fma_rn(p, z, 1.0 / 11.0);
    p = __fma_rn(p, z, 1.0 / 9.0);
    p = __fma_rn(p, z, 1.0 / 7.0);
    p = __fma_rn(p, z, 1.0 / 5.0);
    p = __fma_rn(p, z, 1.0 / 3.0);
    p = __fma_rn(p, z, 1.0);
    double lnm = __dmul_rn(__dadd_rn(s, s), p);
    return __fma_rn((double)e, 0x1.62e42fefa39efp-1, lnm);
}

constexpr uint64_t SAMPLE_TAG = 0x4C41505355534D50ull;   // Philox key word 1

// The widening round's first two kernels run only after a missed bracket (the
// certification left a direction); the rest run once the select has started it.
__device__ __forceinline__ bool widen_starts(const BracketParams &P) {
    return P.ctl->verdict == 0 && P.ctl->widen_dir != 0;
}
__device__ __forceinline__ bool round_skipped(const BracketParams &P) {
    return P.round2 && !P.ctl->widened;
}
constexpr int SEL_BINS = 65536;   // select histogram of the top 16 key bits (then 256 of the top 8)

// y_j = r_{I_j} + t L_j: I_j uniform on [0, n) (high word of u0 * n), L_j ~
// Laplace(0,1) = a random sign times -ln U, U = ((u1 >> 11) + 1) 2^-53 in (0, 1].
// This is the operator's own noise kernel, so P(y_j > b) = k/n.  The key kept
// is the fp32 value rounded toward -inf (monotone, so order statistics commute
// with it), in the descending-order key space.
__global__ void __launch_bounds__(256) sample_kernel(BracketParams Pg) {
    const BracketParams P = at_row(Pg, blockIdx.y);
    __shared__ uint32_t s_h0[256];
    s_h0[threadIdx.x] = 0u;
    pdl_enter();
    if (P.round2) {   // the same sample again, for the widened ranks
        if (!widen_starts(P)) return;
        if (blockIdx.x == 0 && threadIdx.x < 2) P.ctl->sel_cnt[threadIdx.x] = 0u;
    }
    __syncthreads();
    const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    // the index is drawn over the whole row; a rank holding one slice of a split
    // row keeps the draws that land in its slice (the others hold the rest)
    bool mine = false;
    int64_t I = 0;
    uint64_t x1 = 0;
    if (j < P.s) {
        uint64_t x0 = (uint64_t)j, x2 = 0, x3 = 0;
        x1 = (uint64_t)P.row;
        philox4x64_10(x0, x1, x2, x3, P.seed, SAMPLE_TAG);
        I = (int64_t)__umul64hi(x0, (uint64_t)P.n_total) - P.shard_off;
        mine = I >= 0 && I < P.n;
        if (mine && !in_bounds(I < P.n && P.s <= (int64_t)gridDim.x * blockDim.x, &P.ctl->status)) mine = false;
        if (!mine) P.keys[j] = 0u;   // a split row's exchange sums the ranks' shares
    }
    if (mine) {
        const double U = (double)((x1 >> 11) + 1ull) * 0x1p-53;
        const double E = -sample_ln(U);
        const double L = (x1 & 1ull) ? E : -E;
        const double y = __dadd_rn((double)__ldg(P.r + I), __dmul_rn(P.t, L));
        const uint32_t key = desc_key(__double2float_rd(y));
        P.keys[j] = key;
        // histograms of the top 16 bits (global, warp-aggregated) and top 8 bits
        const uint32_t bin = key >> 16;
        const unsigned peers = __match_any_sync(__activemask(), bin);
        if ((threadIdx.x & 31) == __ffs(peers) - 1) {
            atomicAdd(P.hist1 + bin, (uint32_t)__popc(peers));
            atomicAdd(&s_h0[bin >> 8], (uint32_t)__popc(peers));
        }
    }
    __syncthreads();
    const uint32_t c = s_h0[threadIdx.x];
    if (c) atomicAdd(P.hist1 + SEL_BINS + threadIdx.x, c);
}

// ================================================================ select --
// The jR-th and jL-th smallest sample keys (= the jR-th and jL-th largest
// values) by a radix select over bits [31:16] (histogram built by the sampler,
// shared by both targets), then [15:8] and [7:0] over the keys under each
// target's 16-bit prefix, gathered in shared memory.  Bracket ends rounded outward:
//   a_R = nextup(y_(jR) rounded down) (> y_(jR)),  a_L = y_(jL) rounded down;
//   jR = 0 -> a_R = +inf,  jL = s + 1 -> a_L = -inf.
__device__ __forceinline__ uint32_t block_incl_scan_u32(uint32_t v, uint32_t *s_w) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t p = __shfl_up_sync(FULL, x, o);
        if (lane >= o) x += p;
    }
    if (lane == 31) s_w[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = lane < (int)(blockDim.x >> 5) ? s_w[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t p = __shfl_up_sync(FULL, w, o);
            if (lane >= o) w += p;
        }
        s_w[lane] = w;
    }
    __syncthreads();
    uint32_t r = x + (warp > 0 ? s_w[warp - 1] : 0u);
    __syncthreads();
    return r;
}


constexpr int SEL_CAND = 8192;   // candidate keys per target kept (global buffer)
constexpr int SEL_GRID = 64;     // select CTAs
constexpr int SEL_BLOCK = 256;

// Radix select over a grid: every CTA finds the two targets' 16-bit prefixes
// from the sampler's histograms (top 8 bits, then the 256 bins of the top-16
// histogram under the chosen byte), gathers the keys of its share of the sample
// that carry one of the prefixes into a global candidate buffer, and the last
// CTA to finish runs rounds 2 and 3 (bits 15..8, 7..0) over the candidates (or
// over every key when a prefix holds more than the buffer).
__global__ void __launch_bounds__(SEL_BLOCK) select_kernel(BracketParams Pg) {
    static_assert(2 * SEL_CAND == SEL_CAND_WORDS, "candidate buffer stride");
    const BracketParams P = at_row(Pg, blockIdx.y);
    __shared__ uint32_t s_w[SEL_BLOCK / 32];
    __shared__ uint32_t h8[2][256];
    __shared__ uint32_t s_pref[2], s_rank[2], s_bin0[2];
    __shared__ bool s_last;
    pdl_enter();
    if (P.round2 && !widen_starts(P)) return;
    const int tid = threadIdx.x, lane = tid & 31;
    const int64_t s = P.s;
    Ctl *ctl = P.ctl;
    const bool valid[2] = {P.jR >= 1, P.jL <= P.s};
    const uint32_t want0[2] = {(uint32_t)(valid[0] ? P.jR : 1), (uint32_t)(valid[1] ? P.jL : 1)};
    if (tid < 2) { s_bin0[tid] = 0u; s_rank[tid] = 1u; s_pref[tid] = 0u; }
    // ---- round 1a: the top byte of each target (thread t owns bin t)
    {
        const uint32_t c = __ldcg(P.hist1 + SEL_BINS + tid);
        const uint32_t incl = block_incl_scan_u32(c, s_w);
#pragma unroll
        for (int q = 0; q < 2; ++q)
            if (incl - c < want0[q] && want0[q] <= incl) {
                s_bin0[q] = (uint32_t)tid;
                s_rank[q] = want0[q] - (incl - c);
            }
        __syncthreads();
    }
    // ---- round 1b: the second byte, from the 256 top-16 bins under the first
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const uint32_t b0 = s_bin0[q], want = s_rank[q];
        const uint32_t c = __ldcg(P.hist1 + b0 * 256 + tid);
        const uint32_t incl = block_incl_scan_u32(c, s_w);
        if (incl - c < want && want <= incl) {
            s_pref[q] = ((b0 << 8) | (uint32_t)tid) << 16;
            s_rank[q] = want - (incl - c);
        }
        __syncthreads();
    }
    // ---- gather this CTA's keys under either prefix
    const uint32_t pf[2] = {s_pref[0], s_pref[1]};
    {
        auto take = [&](uint32_t key, bool in) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const bool m = in && valid[q] && (key & 0xffff0000u) == pf[q];
                const unsigned bal = __ballot_sync(FULL, m);
                if (!bal) continue;
                uint32_t base = 0;
                if (lane == __ffs(bal) - 1) base = atomicAdd(&ctl->sel_cnt[q], (uint32_t)__popc(bal));
                base = __shfl_sync(FULL, base, __ffs(bal) - 1) + __popc(bal & ((1u << lane) - 1u));
                if (m && base < SEL_CAND) P.cand[q * SEL_CAND + base] = key;
            }
        };
        const uint4 *k4 = reinterpret_cast<const uint4 *>(P.keys);
        const int64_t s4 = s / 4;
        const int64_t stride = (int64_t)gridDim.x * SEL_BLOCK;
        for (int64_t i0 = (int64_t)blockIdx.x * SEL_BLOCK; i0 < s4; i0 += stride) {
            const int64_t i = i0 + tid;
            const bool in = i < s4;
            const uint4 kv = in ? k4[i] : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t kk[4] = {kv.x, kv.y, kv.z, kv.w};
            bool hit = false;   // candidates are rare: one vote for four keys
#pragma unroll
            for (int e = 0; e < 4; ++e)
                hit |= in && (((kk[e] & 0xffff0000u) == pf[0] && valid[0]) || ((kk[e] & 0xffff0000u) == pf[1] && valid[1]));
            if (!__any_sync(FULL, hit)) continue;
#pragma unroll
            for (int e = 0; e < 4; ++e) take(kk[e], in);
        }
        if (blockIdx.x == 0)
            for (int64_t i0 = 4 * s4; i0 < s; i0 += SEL_BLOCK) {
                const int64_t i = i0 + tid;
                take(i < s ? P.keys[i] : 0u, i < s);
            }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&ctl->ticket[5], 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // ---- last CTA: rounds 2, 3 over the candidates
    const uint32_t cnt[2] = {__ldcg(&ctl->sel_cnt[0]), __ldcg(&ctl->sel_cnt[1])};
    const bool fast[2] = {cnt[0] <= SEL_CAND, cnt[1] <= SEL_CAND};
    uint32_t mask = 0xffff0000u;
#pragma unroll 1
    for (int sh = 8; sh >= 0; sh -= 8) {
        for (int i = tid; i < 2 * 256; i += SEL_BLOCK) (&h8[0][0])[i] = 0u;
        __syncthreads();
        const uint32_t pq[2] = {s_pref[0], s_pref[1]};
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            if (!valid[q]) continue;
            const int64_t c = fast[q] ? (int64_t)cnt[q] : s;
            for (int64_t i = tid; i < c; i += SEL_BLOCK) {
                const uint32_t key = fast[q] ? __ldcg(P.cand + q * SEL_CAND + i) : P.keys[i];
                if ((key & mask) == pq[q]) atomicAdd(&h8[q][(key >> sh) & 0xffu], 1u);
            }
        }
        __syncthreads();
        if (tid < 64) {   // warp q scans target q's 256 bins (8 per lane)
            const int q = tid >> 5;
            if (valid[q]) {
                uint32_t v[8], run = 0;
#pragma unroll
                for (int u = 0; u < 8; ++u) { v[u] = h8[q][lane * 8 + u]; run += v[u]; }
                uint32_t incl = run;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t p = __shfl_up_sync(FULL, incl, o);
                    if (lane >= o) incl += p;
                }
                const uint32_t want = s_rank[q];
                uint32_t cum = incl - run;
                if (cum < want && want <= incl) {
                    for (int u = 0; u < 8; ++u) {
                        if (cum + v[u] >= want) {
                            s_pref[q] |= (uint32_t)(lane * 8 + u) << sh;
                            s_rank[q] = want - cum;
                            break;
                        }
                        cum += v[u];
                    }
                }
            }
        }
        mask |= 0xffu << sh;
        __syncthreads();
    }
    P.hist1[SEL_BINS + tid] = 0u;   // the top-byte histogram; the streaming pass clears the rest
    if (tid == 0) {
        if ((valid[0] && !fast[0]) || (valid[1] && !fast[1])) ctl->flags |= FLAG_SELECT_ALL_KEYS;
        const float yR = desc_key_to_float(s_pref[0]);
        const float yL = desc_key_to_float(s_pref[1]);
        const float aR = valid[0] ? nextafterf(yR, CUDART_INF_F) : CUDART_INF_F;
        const float aL = valid[1] ? yL : -CUDART_INF_F;
        if (P.round2) {   // the missed side becomes the bracket; the stream starts afresh
            if (ctl->widen_dir > 0) {   // b >= old a_R
                ctl->a_L = ctl->a_R;
                ctl->jL = ctl->jR;
                ctl->a_R = aR;
                ctl->jR = P.jR;
            } else {                    // b < old a_L
                ctl->a_R = ctl->a_L;
                ctl->jR = ctl->jL;
                ctl->a_L = aL;
                ctl->jL = P.jL;
            }
            ctl->c_band = 0ull;
            ctl->band_kmax = 0u;
            ctl->band_kinv = 0u;
            atomicAnd(&ctl->status, ~(ST_NO_ROOT | ST_BAND_OVERFLOW));   // the first band solve's misses
            ctl->widened = 1;
        } else {
            ctl->a_R = aR;
            ctl->a_L = aL;
            ctl->jR = P.jR;
            ctl->jL = P.jL;
        }
        ctl->s = P.s;
        ctl->path = 2;
        ctl->verdict = -1;
        ctl->ticket[5] = 0u;
    }
}

// ===================================================== out-of-band passes --
// The streaming pass (technical summary section 2.2, step 2) and the
// certification pass (step 4, abstract) walk every score once and, for each
// score outside [a_L, a_R), add its tail term
//   below a_L:  e^{(r - a_L)/t},    at or above a_R:  e^{-(r - a_R)/t}.
// Terms come in three tiers by z = |r - a|/t: z <= 16 (can move the budget by
// more than ~1e-7): fp64 from an fp64 z; 16 < z <= 40: fp32 ex2; z > 40
// (< 4.3e-18 each): dropped.  A warp whose 128 scores all lie at z > 16 below
// a_L takes a fast path (count, or count + fp32 terms) -- the bulk of a long
// row -- so the pass stays memory-bound.  Non-finite scores never take it
// (the float4 bounds use NaN-propagating max and a finite-min check).
constexpr float NEAR2 = 23.083120654223414f;   // 16 log2(e)

struct Ends {
    float aL, aR, s2;          // s2 = log2(e)/t
    float midL, farL;          // x < midL: z > 16 below a_L; x < farL: z > 40
    double daL, daR, inv_t, s2d;
    const double *tab;         // 2^{-j/32}, shared memory
};
__device__ __forceinline__ Ends make_ends(const Ctl *ctl, double inv_t) {
    Ends E;
    E.aL = ctl->a_L;
    E.aR = ctl->a_R;
    E.daL = E.aL;
    E.daR = E.aR;
    E.inv_t = inv_t;
    E.s2d = inv_t * LOG2E;
    E.s2 = (float)E.s2d;
    // thresholds in score space, rounded toward a_L (the fast paths then only
    // ever take scores at or beyond their tier bound, up to fp32 rounding)
    E.midL = (float)(E.daL - 16.0 / inv_t);
    E.farL = (float)(E.daL - 40.0 / inv_t);
    return E;
}
__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float max_nan(float a, float b) {
    float y;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(y) : "f"(a), "f"(b));
    return y;
}
// tiered e^{-z} with z = (hi - lo)/t
__device__ __forceinline__ void tier2(float hi, float lo, double dhi, double dlo, const Ends &E,
                                      double &acc64, float &acc32) {
    const float z2 = (hi - lo) * E.s2;
    if (z2 <= NEAR2) acc64 += exp2_neg((dhi - dlo) * E.s2d, E.tab);
    else acc32 += ex2_ftz(-z2);
}

struct OobAcc {
    uint32_t cL, cR, cB;        // stream: below, above; certify: (unused), >= a_R, < a_L
    uint32_t np;                // certify: scores seen (>= a_L is np - cB for a finite row)
    uint32_t kmax, kinv;        // stream: largest band key and largest complemented band key
    double SL, SR, hL, lR;      // near terms: below, above, band vs a_L, band vs a_R
    float SL2, SR2, hL2, lR2;   // far terms
    float mx;                   // max |score|, NaN-propagating: not finite -> a non-finite score
};

// Append a band score at a warp-aggregated slot of the band buffer (the count
// keeps going past the capacity so the overflow is visible).
__device__ __forceinline__ void band_push(float x, bool inb, float *band, unsigned long long cap,
                                          unsigned long long *ctr, int lane, OobAcc &a) {
    const unsigned m = __ballot_sync(FULL, inb);
    if (!m) return;
    if (inb) {
        a.kmax = max(a.kmax, desc_key(x));
        a.kinv = max(a.kinv, ~desc_key(x));
    }
    const int leader = __ffs(m) - 1;
    unsigned long long base = 0;
    if (lane == leader) base = atomicAdd(ctr, (unsigned long long)__popc(m));
    base = __shfl_sync(FULL, base, leader) + __popc(m & ((1u << lane) - 1u));
    if (inb && base < cap) band[base] = x;
}

// Pass modes: the streaming pass, the certification pass, and the streaming
// pass with the certification folded in (band scores also add their two
// certification terms; the verdict comes out of the same pass).
enum : int { OOB_STREAM = 0, OOB_CERT = 1, OOB_STREAM_CERT = 2 };

// General path, one score.  Returns "in the band" (streaming modes).  Written
// to keep a warp of mixed scores together: every out-of-band score forms its
// fp32 tail term, and the masks pick where it goes; only the rare scores near
// an end (fp64 term) and band scores (certification terms) branch.
template <int MODE>
__device__ __forceinline__ bool oob_one(float x, bool valid, const Ends &E, OobAcc &a) {
    constexpr bool CERT = MODE == OOB_CERT;
    if (!valid) return false;
    a.mx = max_nan(a.mx, fabsf(x));
    const bool above = x >= E.aR, below = x < E.aL;
    const bool inb = !above && !below && x == x;
    if (CERT) {
        a.cR += above;
        a.cB += below;
        a.np += 1;
    } else {
        a.cR += above;
        a.cL += below;
    }
    const float z2 = (above ? x - E.aR : E.aL - x) * E.s2;   // tail exponent in base-2 units
    const bool near = (above || below) && z2 <= NEAR2;
    const float f = ex2_ftz(-z2);
    a.SR2 += (above && !near) ? f : 0.f;
    a.SL2 += (below && !near) ? f : 0.f;
    if (near) {
        if (above) a.SR += exp2_neg(((double)x - E.daR) * E.s2d, E.tab);
        else       a.SL += exp2_neg((E.daL - (double)x) * E.s2d, E.tab);
    }
    if (MODE != OOB_STREAM && inb) {
        tier2(x, E.aL, (double)x, E.daL, E, a.hL, a.hL2);
        tier2(E.aR, x, E.daR, (double)x, E, a.lR, a.lR2);
    }
    return inb;
}

// One float4 of the pass; `ok` false for padding lanes (whole warps iterate).
// Tail terms of a float4 against one end a: e^{-(x-a)/t} (UP) or e^{-(a-x)/t};
// four equal scores take one term.
template <bool UP>
__device__ __forceinline__ void tier4(const float4 v, bool equal, float af, double ad, const Ends &E,
                                      double &acc64, float &acc32) {
    double s01 = 0.0, s23 = 0.0;
    float f01 = 0.f, f23 = 0.f;
    auto one = [&](float x, double &s, float &f) {
        if (UP) tier2(x, af, (double)x, ad, E, s, f);
        else    tier2(af, x, ad, (double)x, E, s, f);
    };
    if (equal) {
        one(v.x, s01, f01);
        s01 *= 4.0;
        f01 *= 4.0f;
    } else {
        one(v.x, s01, f01);
        one(v.y, s01, f01);
        one(v.z, s23, f23);
        one(v.w, s23, f23);
    }
    acc64 += s01 + s23;
    acc32 += f01 + f23;
}

// Append the band scores of a float4 (bit i of m: component i) at consecutive
// slots: one warp scan and one atomic per warp (the count keeps going past the
// capacity so the overflow is visible).
__device__ __forceinline__ void band_push4(const float4 v, int m, float *band, unsigned long long cap,
                                           unsigned long long *ctr, int lane, OobAcc &a) {
    const int cnt = __popc(m);
    int inc = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int p = __shfl_up_sync(FULL, inc, o);
        if (lane >= o) inc += p;
    }
    const int total = __shfl_sync(FULL, inc, 31);
    if (total == 0) return;
    {
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (m & (1 << i)) {
                const uint32_t kk = desc_key(vv[i]);
                a.kmax = max(a.kmax, kk);
                a.kinv = max(a.kinv, ~kk);
            }
    }
    unsigned long long base = 0;
    if (lane == 31) base = atomicAdd(ctr, (unsigned long long)total);
    base = __shfl_sync(FULL, base, 31) + (unsigned long long)(inc - cnt);
    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (m & (1 << i)) {
            if (base < cap) band[base] = vv[i];
            ++base;
        }
    }
}

// One float4 of the pass; `ok` false for padding lanes (whole warps iterate).
// Warp-uniform fast paths for float4s wholly far below a_L, wholly below it,
// wholly at or above a_R, or wholly inside the band; the general path otherwise.
template <int MODE>
__device__ __forceinline__ void oob_vec(const float4 v, bool ok, const Ends &E, OobAcc &a,
                                        const BracketParams &P, unsigned long long cap, int lane) {
    constexpr bool CERT = MODE == OOB_CERT;
    constexpr bool BANDTERMS = MODE != OOB_STREAM;
    const float mx = max_nan(max_nan(v.x, v.y), max_nan(v.z, v.w));
    const float mn = fminf(fminf(v.x, v.y), fminf(v.z, v.w));
    const bool fin = mn > -CUDART_INF_F && mx < CUDART_INF_F;    // false for NaN too
    const bool equal = mx == mn;
    if (__all_sync(FULL, !ok || (mx < E.farL && fin))) {
        if (ok) { if (CERT) { a.cB += 4; a.np += 4; } else a.cL += 4; }
        return;
    }
    if (__all_sync(FULL, !ok || (mx < E.midL && fin))) {
        if (ok) {
            if (CERT) { a.cB += 4; a.np += 4; } else a.cL += 4;
            a.SL2 += (ex2_ftz((v.x - E.aL) * E.s2) + ex2_ftz((v.y - E.aL) * E.s2)) +
                     (ex2_ftz((v.z - E.aL) * E.s2) + ex2_ftz((v.w - E.aL) * E.s2));
        }
        return;
    }
    if (__all_sync(FULL, !ok || (mx < E.aL && fin))) {            // below a_L, some near it
        if (ok) {
            if (CERT) { a.cB += 4; a.np += 4; } else a.cL += 4;
            tier4<false>(v, equal, E.aL, E.daL, E, a.SL, a.SL2);
        }
        return;
    }
    if (__all_sync(FULL, !ok || (mn >= E.aR && fin))) {           // at or above a_R
        if (ok) {
            if (CERT) { a.cR += 4; a.np += 4; } else a.cR += 4;
            tier4<true>(v, equal, E.aR, E.daR, E, a.SR, a.SR2);
        }
        return;
    }
    if (__all_sync(FULL, !ok || (mn >= E.aL && mx < E.aR && fin))) {   // inside the band
        if (ok && BANDTERMS) {
            if (CERT) a.np += 4;
            tier4<true>(v, equal, E.aL, E.daL, E, a.hL, a.hL2);
            tier4<false>(v, equal, E.aR, E.daR, E, a.lR, a.lR2);
        }
        if (!CERT) band_push4(v, ok ? 0xF : 0, P.band, cap, &P.ctl->c_band, lane, a);
        return;
    }
    const bool b0 = oob_one<MODE>(v.x, ok, E, a);
    const bool b1 = oob_one<MODE>(v.y, ok, E, a);
    const bool b2 = oob_one<MODE>(v.z, ok, E, a);
    const bool b3 = oob_one<MODE>(v.w, ok, E, a);
    if (!CERT) {
        const int m = (b0 ? 1 : 0) | (b1 ? 2 : 0) | (b2 ? 4 : 0) | (b3 ? 8 : 0);
        if (__any_sync(FULL, m != 0)) band_push4(v, m, P.band, cap, &P.ctl->c_band, lane, a);
    }
}

// ---- one chunk per thread (two float4s) at a time --------------------------
// Sparse band scores of a streaming pass go to a queue in shared memory, written
// out with one global atomic per CTA at the end (a warp-aggregated global push
// only if the queue fills).
constexpr int BQ = 2048;

__device__ __forceinline__ float pick8(const float4 &u, const float4 &w, int i) {
    const float lo = (i & 2) ? ((i & 1) ? u.w : u.z) : ((i & 1) ? u.y : u.x);
    const float hi = (i & 2) ? ((i & 1) ? w.w : w.z) : ((i & 1) ? w.y : w.x);
    return (i & 4) ? hi : lo;
}

// The common part of the general path for one score: the counts, and the fp32
// tail term of a score more than 16 t beyond its end (the bulk of a long row);
// every other score -- near an end (fp64 term), in the band, or not a number --
// only sets its bit in sp_m, to be staged (special_tail, special_band).  About
// sixteen instructions, with the two ends' sums kept apart by predicated adds.
template <int MODE>
__device__ __forceinline__ void oob_cheap(float x, int bit, const Ends &E, OobAcc &a, uint32_t &sp_m) {
    constexpr bool CERT = MODE == OOB_CERT;
    a.mx = max_nan(a.mx, fabsf(x));
    const bool above = x >= E.aR, below = x < E.aL;
    if (CERT) {
        a.cR += above;
        a.cB += below;
    } else {
        a.cR += above;
        a.cL += below;
    }
    const float z2 = (above ? x - E.aR : E.aL - x) * E.s2;   // base-2 distance beyond the end (band: <= 0)
    const float f = ex2_ftz(-z2);
    const bool far = z2 > NEAR2;                             // false for NaN
    if (far && above) a.SR2 += f;
    if (far && below) a.SL2 += f;
    if (!(far && (above || below))) sp_m |= 1u << bit;
}

// The rare scores of a general chunk -- near an end (fp64 tail term) or in the
// band (queue slot, or the two certification terms) -- are staged in a per-warp
// queue in shared memory and handled 32 at a time, one per lane, so a warp never
// loops as often as its busiest lane has such scores, and every batch but the
// last is full however many a chunk has (on tied levels in random order, a
// large t puts ~40% of the scores within 16 t of an end).
constexpr int SQ = 32 + 8 * 32;   // staged scores per warp: below 32 between chunks, at most 256 added

// The fp64 tail term of a staged score out of the band (act false, or a band
// score: nothing).  Branch-free, so that two calls interleave their chains; the
// term of a score it does not add is formed and dropped.
__device__ __forceinline__ void special_tail(float x, bool act, const Ends &E, OobAcc &a) {
    const bool above = act && x >= E.aR, below = act && x < E.aL;
    const double w = above ? ((double)x - E.daR) * E.s2d : (E.daL - (double)x) * E.s2d;
    const double e = exp2_neg(fmax(w, 0.0), E.tab);
    a.SR += above ? e : 0.0;
    a.SL += below ? e : 0.0;
}

// One rare score per lane (act false: nothing), by the whole warp, once its tail
// term is in: for a band score its queue slot and/or its two certification
// terms.  Not-a-number scores take neither (the status reports them).
template <int MODE>
__device__ __forceinline__ void special_band(float x, bool act, const Ends &E, OobAcc &a, const BracketParams &P,
                                             unsigned long long cap, int lane, float *s_bq, unsigned *s_bn) {
    constexpr bool CERT = MODE == OOB_CERT;
    constexpr bool BANDTERMS = MODE != OOB_STREAM;
    const bool inb = act && x >= E.aL && x < E.aR;   // false for NaN
    if (BANDTERMS && inb) {   // the band score's two certification terms
        tier2(x, E.aL, (double)x, E.daL, E, a.hL, a.hL2);
        tier2(E.aR, x, E.daR, (double)x, E, a.lR, a.lR2);
    }
    if (!CERT) {   // the band scores into the CTA's queue
        const unsigned m = __ballot_sync(FULL, inb);
        if (m) {
            const int leader = __ffs(m) - 1;
            unsigned base = 0;
            if (lane == leader) base = atomicAdd(s_bn, (unsigned)__popc(m));
            const unsigned slot = __shfl_sync(FULL, base, leader) + __popc(m & ((1u << lane) - 1u));
            if (inb) {
                a.kmax = max(a.kmax, desc_key(x));
                a.kinv = max(a.kinv, ~desc_key(x));
                if (slot < (unsigned)BQ) s_bq[slot] = x;
            }
            band_push(x, inb && slot >= (unsigned)BQ, P.band, cap, &P.ctl->c_band, lane, a);   // queue full
        }
    }
}

// Up to 32 staged scores, one per lane (lanes >= cnt idle).
template <int MODE>
__device__ __forceinline__ void special_batch(const float *q, int cnt, const Ends &E, OobAcc &a,
                                              const BracketParams &P, unsigned long long cap, int lane,
                                              float *s_bq, unsigned *s_bn) {
    const bool act = lane < cnt;
    const float x = act ? q[lane] : 0.f;
    special_tail(x, act, E, a);
    special_band<MODE>(x, act, E, a, P, cap, lane, s_bq, s_bn);
}
// 64 staged scores, two per lane: both tail terms first (independent chains).
template <int MODE>
__device__ __forceinline__ void special_batch2(const float *q, const Ends &E, OobAcc &a, const BracketParams &P,
                                               unsigned long long cap, int lane, float *s_bq, unsigned *s_bn) {
    const float x0 = q[lane], x1 = q[32 + lane];
    special_tail(x0, true, E, a);
    special_tail(x1, true, E, a);
    special_band<MODE>(x0, true, E, a, P, cap, lane, s_bq, s_bn);
    special_band<MODE>(x1, true, E, a, P, cap, lane, s_bq, s_bn);
}

template <int MODE, bool ADAPT>
__device__ __forceinline__ void oob_chunk(const float4 v0, const float4 v1, const Ends &E, OobAcc &a,
                                          const BracketParams &P, unsigned long long cap, int lane,
                                          float *s_bq, unsigned *s_bn, float *sq, unsigned &sq_n,
                                          unsigned &hist, unsigned &tick) {
    constexpr bool CERT = MODE == OOB_CERT;
    constexpr bool BANDTERMS = MODE != OOB_STREAM;
    // ADAPT: hist records which of the warp's last 16 chunks took the general
    // path.  When 12 or more did (random score order), the fast-path tests are
    // skipped, except on every 16th chunk, which keeps the history fresh; every
    // chunk is correct on the general path.
    bool try_fast = true;
    if (ADAPT) {
        try_fast = __popc(hist & 0xffffu) < 12 || (tick & 15u) == 0u;
        hist <<= 1;
        ++tick;
    }
    if (try_fast) {
        const float mx = max_nan(max_nan(max_nan(v0.x, v0.y), max_nan(v0.z, v0.w)),
                                 max_nan(max_nan(v1.x, v1.y), max_nan(v1.z, v1.w)));
        const float mn = fminf(fminf(fminf(v0.x, v0.y), fminf(v0.z, v0.w)),
                               fminf(fminf(v1.x, v1.y), fminf(v1.z, v1.w)));
        const bool fin = mn > -CUDART_INF_F && mx < CUDART_INF_F;
        // a whole warp on one side (sorted or clustered scores): eight scores at once
        const bool eq0 = v0.x == v0.y && v0.y == v0.z && v0.z == v0.w;
        const bool eq1 = v1.x == v1.y && v1.y == v1.z && v1.z == v1.w;
        if (__all_sync(FULL, mx < E.farL && fin)) {            // far below a_L: counts only
            if (CERT) { a.cB += 8; a.np += 8; } else a.cL += 8;
            return;
        }
        if (__all_sync(FULL, mx < E.midL && fin)) {            // below a_L, fp32 terms
            if (CERT) { a.cB += 8; a.np += 8; } else a.cL += 8;
            if (__all_sync(FULL, eq0 && eq1)) {   // tied scores: one term per float4 (4a = (a + a) + (a + a))
                a.SL2 += 4.f * ex2_ftz((v0.x - E.aL) * E.s2) + 4.f * ex2_ftz((v1.x - E.aL) * E.s2);
                return;
            }
            a.SL2 += ((ex2_ftz((v0.x - E.aL) * E.s2) + ex2_ftz((v0.y - E.aL) * E.s2)) +
                      (ex2_ftz((v0.z - E.aL) * E.s2) + ex2_ftz((v0.w - E.aL) * E.s2))) +
                     ((ex2_ftz((v1.x - E.aL) * E.s2) + ex2_ftz((v1.y - E.aL) * E.s2)) +
                      (ex2_ftz((v1.z - E.aL) * E.s2) + ex2_ftz((v1.w - E.aL) * E.s2)));
            return;
        }
        if (__all_sync(FULL, mx < E.aL && fin)) {              // below a_L, some near it
            if (CERT) { a.cB += 8; a.np += 8; } else a.cL += 8;
            tier4<false>(v0, eq0, E.aL, E.daL, E, a.SL, a.SL2);
            tier4<false>(v1, eq1, E.aL, E.daL, E, a.SL, a.SL2);
            return;
        }
        if (__all_sync(FULL, mn >= E.aR && fin)) {             // at or above a_R
            if (CERT) { a.cR += 8; a.np += 8; } else a.cR += 8;
            tier4<true>(v0, eq0, E.aR, E.daR, E, a.SR, a.SR2);
            tier4<true>(v1, eq1, E.aR, E.daR, E, a.SR, a.SR2);
            return;
        }
        if (__all_sync(FULL, mn >= E.aL && mx < E.aR && fin)) {   // inside the band
            if (BANDTERMS) {
                if (CERT) a.np += 8;
                tier4<true>(v0, eq0, E.aL, E.daL, E, a.hL, a.hL2);
                tier4<false>(v0, eq0, E.aR, E.daR, E, a.lR, a.lR2);
                tier4<true>(v1, eq1, E.aL, E.daL, E, a.hL, a.hL2);
                tier4<false>(v1, eq1, E.aR, E.daR, E, a.lR, a.lR2);
            }
            if (!CERT) {
                band_push4(v0, 0xF, P.band, cap, &P.ctl->c_band, lane, a);
                band_push4(v1, 0xF, P.band, cap, &P.ctl->c_band, lane, a);
            }
            return;
        }
    }
    if (ADAPT) hist |= 1u;
    // general path: the cheap part for all eight, then the marked ones
    uint32_t sp = 0;
    oob_cheap<MODE>(v0.x, 0, E, a, sp);
    oob_cheap<MODE>(v0.y, 1, E, a, sp);
    oob_cheap<MODE>(v0.z, 2, E, a, sp);
    oob_cheap<MODE>(v0.w, 3, E, a, sp);
    oob_cheap<MODE>(v1.x, 4, E, a, sp);
    oob_cheap<MODE>(v1.y, 5, E, a, sp);
    oob_cheap<MODE>(v1.z, 6, E, a, sp);
    oob_cheap<MODE>(v1.w, 7, E, a, sp);
    if (CERT) a.np += 8;
    const unsigned cnt = __popc(sp);
    // stage them at the warp's fill level, each lane after the lanes below it
    // (an inclusive scan of the counts: no atomics), then handle them 64 or 32
    // at a time
    unsigned incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(FULL, incl, o);
        if (lane >= o) incl += y;
    }
    const unsigned total = __shfl_sync(FULL, incl, 31);
    if (total == 0) return;
    unsigned pos = sq_n + incl - cnt;
    while (sp) {
        if (in_bounds(pos < (unsigned)SQ, &P.ctl->status)) sq[pos] = pick8(v0, v1, __ffs(sp) - 1);
        ++pos;
        sp &= sp - 1;
    }
    __syncwarp();
    sq_n += total;
    while (sq_n >= 64) {
        sq_n -= 64;
        special_batch2<MODE>(sq + sq_n, E, a, P, cap, lane, s_bq, s_bn);
    }
    if (sq_n >= 32) {
        sq_n -= 32;
        special_batch<MODE>(sq + sq_n, 32, E, a, P, cap, lane, s_bq, s_bn);
    }
    __syncwarp();   // the batch's reads are done before the next chunk stages over them
}

// The verdict, and for a failed first round with widening enabled the side the
// threshold lies on: a bracket whose counts agree and whose band fits, but with
// G(a_R) >= k (b at or above a_R) or G(a_L) < k (b below a_L), was missed.
__device__ __forceinline__ void set_verdict(const BracketParams &P, bool ok, bool sound, double GaL,
                                            double GaR) {
    Ctl *ctl = P.ctl;
    ctl->verdict = ok ? 1 : 0;
    int dir = 0;
    if (!ok && sound && P.widen && !P.round2) dir = GaR >= P.k ? 1 : (GaL < P.k ? -1 : 0);
    ctl->widen_dir = dir;
}

// CERT = false: streaming pass (forward over the row): c_L, c_R, S_L, S_R and
//               the band.
// CERT = true:  certification pass (backward over the row, starting on what
//               the streaming pass left in L2):
//   G(a) = #{r >= a} - 1/2 sum_{r>=a} e^{-(r-a)/t} + 1/2 sum_{r<a} e^{(r-a)/t}
// at a = a_L and a = a_R.  Scores outside the band share one exponential
// between the two ends (e^{-(r-a_L)/t} = e^{-(r-a_R)/t} e^{-(a_R-a_L)/t} and its
// mirror image below); band scores take two.  Verdict: G(a_L) >= k > G(a_R),
// the band fits its buffer, both passes agree on every membership count, and
// every score is finite.
// MINB: CTAs per SM the registers are sized for.  The streaming pass fits four
// at 64 registers; the certification passes keep more accumulators and were
// measured faster at three (80 registers) on one row and at four on a batch of
// random-order rows (195 -> 170 us per 256 MB), so the certification pass is
// built both ways.  ADAPT: skip the chunk fast-path tests on random-order runs
// of chunks (oob_chunk); measured faster on the streaming pass and on the
// batched certification pass, slower (+3%) on the one-row certification pass
// of sorted scores.
template <int MODE, int MINB = (MODE == OOB_STREAM ? SBLOCKS_PER_SM : 3), bool ADAPT = (MODE == OOB_STREAM)>
__global__ void __launch_bounds__(SBLOCK, MINB) oob_kernel(BracketParams Pg) {
    const BracketParams P = at_row(Pg, blockIdx.y);
    constexpr bool CERT = MODE == OOB_CERT;
    static_assert(2 * SBLOCK == BULK_F4, "two vectors per thread per chunk");
    extern __shared__ __align__(128) unsigned char dsm[];
    __shared__ double s_red[7 * (SBLOCK / 32)];
    __shared__ double s_tab[32];
    __shared__ float s_bq[CERT ? 1 : BQ];   // sparse band scores of this CTA
    __shared__ float s_sq[SBLOCK / 32][SQ];   // staged rare scores, per warp
    __shared__ unsigned s_bn;
    __shared__ unsigned long long s_bbase;
    exp2_table_init(s_tab);
    if (threadIdx.x == 0) s_bn = 0u;
    pdl_enter();
    if (round_skipped(P)) return;
    if (!CERT) {   // the select histogram is spent: clear it for the next solve
        uint4 *h = reinterpret_cast<uint4 *>(P.hist1);
        for (int64_t i = (int64_t)blockIdx.x * SBLOCK + threadIdx.x; i < SEL_BINS / 4; i += (int64_t)gridDim.x * SBLOCK)
            h[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    Ctl *ctl = P.ctl;
    Ends E = make_ends(ctl, P.inv_t);
    E.tab = s_tab;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const unsigned long long cap = (unsigned long long)P.band_cap;
    OobAcc acc{0, 0, 0, 0, 0u, 0u, 0.0, 0.0, 0.0, 0.0, 0.f, 0.f, 0.f, 0.f, 0.f};
    const int64_t n = P.n;
    const int64_t gtid = (int64_t)blockIdx.x * SBLOCK + threadIdx.x;
    const int64_t gstride = (int64_t)gridDim.x * SBLOCK;
    const bool aligned = (reinterpret_cast<uintptr_t>(P.r) & 15) == 0;
    const int64_t n4 = aligned ? n / 4 : 0;
    const float4 *r4 = reinterpret_cast<const float4 *>(P.r);
    int64_t done4 = 0;
    if (aligned) {
        const float4 *src[1] = {r4};
        float *sq = s_sq[threadIdx.x >> 5];
        unsigned sq_n = 0, hist = 0, tick = 0;   // the same in every lane of a warp
        done4 = bulk_stream<1>(src, n4, CERT, dsm, &ctl->status, [&](const float4 *const *ch, int64_t) {
            oob_chunk<MODE, ADAPT>(lds128(ch[0] + threadIdx.x), lds128(ch[0] + threadIdx.x + SBLOCK), E, acc, P, cap,
                                   lane, s_bq, &s_bn, sq, sq_n, hist, tick);
        });
        __syncwarp();
        if (sq_n) special_batch<MODE>(sq, (int)sq_n, E, acc, P, cap, lane, s_bq, &s_bn);
    }
    // vectors after the last full chunk (whole warps iterate together)
    const int64_t tv = n4 - done4;
    const int64_t tvw = (tv + gstride - 1) / gstride * gstride;
    for (int64_t i = gtid; i < tvw; i += gstride) {
        const bool ok = i < tv;
        const float4 v = ok ? r4[done4 + i] : make_float4(0.f, 0.f, 0.f, 0.f);
        oob_vec<MODE>(v, ok, E, acc, P, cap, lane);
    }
    const int64_t rem0 = n4 * 4;
    const int64_t remw = rem0 + ((n - rem0 + gstride - 1) / gstride) * gstride;
    for (int64_t j = rem0 + gtid; j < remw; j += gstride) {
        const bool ok = j < n;
        const float x = ok ? P.r[j] : 0.f;
        const bool bb = oob_one<MODE>(x, ok, E, acc);
        if (!CERT) band_push(x, bb, P.band, cap, &ctl->c_band, lane, acc);
    }
    if (__syncthreads_or(!(acc.mx < CUDART_INF_F)) && threadIdx.x == 0) atomicOr(&ctl->status, ST_NONFINITE);
    if (!CERT) {
        __shared__ uint32_t s_two[2];
        band_range_flush(ctl, acc.kmax, acc.kinv, s_two);
        // the queued band scores: one slot range per CTA
        const unsigned nq = min(s_bn, (unsigned)BQ);
        if (nq) {
            if (threadIdx.x == 0) s_bbase = atomicAdd(&ctl->c_band, (unsigned long long)nq);
            __syncthreads();
            for (unsigned i = threadIdx.x; i < nq; i += SBLOCK) {
                const unsigned long long slot = s_bbase + i;
                if (slot < cap) P.band[slot] = s_bq[i];
            }
        }
    }
    if constexpr (MODE == OOB_STREAM) {
        double v[4] = {(double)acc.cL, (double)acc.cR, acc.SL + (double)acc.SL2, acc.SR + (double)acc.SR2};
        block_sum<SBLOCK, 4>(v, s_red);
        if (last_block_sum<SBLOCK, 4>(v, P.partials, &ctl->ticket[0], s_red) && threadIdx.x == 0) {
            ctl->c_L = (unsigned long long)v[0];
            ctl->c_R = (unsigned long long)v[1];
            ctl->S_L = v[2];
            ctl->S_R = v[3];
        }
        return;
    }
    if constexpr (MODE == OOB_STREAM_CERT) {
        double v[6] = {(double)acc.cL, (double)acc.cR, acc.SL + (double)acc.SL2, acc.SR + (double)acc.SR2,
                       acc.hL + (double)acc.hL2, acc.lR + (double)acc.lR2};
        block_sum<SBLOCK, 6>(v, s_red);
        if (last_block_sum<SBLOCK, 6>(v, P.partials, &ctl->ticket[0], s_red) && threadIdx.x == 0) {
            const unsigned long long cL = (unsigned long long)v[0], cR = (unsigned long long)v[1];
            const unsigned long long cb = ctl->c_band;
            ctl->c_L = cL;
            ctl->c_R = cR;
            ctl->S_L = v[2];
            ctl->S_R = v[3];
            // G(a_L), G(a_R) from the same terms: band scores are at or above a_L
            // and below a_R; out-of-band scores share one term between the ends
            const double rho = (E.aR == CUDART_INF_F || E.aL == -CUDART_INF_F) ? 0.0
                                                                               : exp(-(E.daR - E.daL) * E.inv_t);
            const double GaL = (double)(cb + cR) - 0.5 * fma(rho, v[3], v[4]) + 0.5 * v[2];
            const double GaR = (double)cR - 0.5 * v[3] + 0.5 * fma(rho, v[2], v[5]);
            ctl->G_aL = GaL;
            ctl->G_aR = GaR;
            ctl->hL = v[4];
            ctl->lR = v[5];
            const bool sound = (cb <= (unsigned long long)P.band_cap) &&
                               (cL + cb + cR == (unsigned long long)n) && ((ctl->status & ST_NONFINITE) == 0);
            const bool ok = sound && (GaL >= P.k) && (GaR < P.k);
            set_verdict(P, ok, sound, GaL, GaR);
            if (cb > (unsigned long long)P.band_cap) atomicOr(&ctl->status, ST_BAND_OVERFLOW);
        }
        return;
    }
    double v[7] = {(double)(acc.np - acc.cB), (double)acc.cR, (double)acc.cB, acc.SR + (double)acc.SR2,
                   acc.SL + (double)acc.SL2, acc.hL + (double)acc.hL2, acc.lR + (double)acc.lR2};
    block_sum<SBLOCK, 7>(v, s_red);
    if (last_block_sum<SBLOCK, 7>(v, P.partials + 8 * (size_t)gridDim.x, &ctl->ticket[1], s_red) &&
        threadIdx.x == 0) {
        const double cntL = v[0], cntR = v[1], cntB = v[2];
        const double rho = (E.aR == CUDART_INF_F || E.aL == -CUDART_INF_F) ? 0.0 : exp(-(E.daR - E.daL) * E.inv_t);
        const double GaL = cntL - 0.5 * fma(rho, v[3], v[5]) + 0.5 * v[4];
        const double GaR = cntR - 0.5 * v[3] + 0.5 * fma(rho, v[4], v[6]);
        ctl->G_aL = GaL;
        ctl->G_aR = GaR;
        const unsigned long long cL = ctl->c_L, cR = ctl->c_R, cb = ctl->c_band;
        const bool sound = (cb <= (unsigned long long)P.band_cap) && (cL + cb + cR == (unsigned long long)n) &&
                           ((unsigned long long)cntR == cR) && ((unsigned long long)(cntL - cntR) == cb) &&
                           ((unsigned long long)cntB == cL) && ((ctl->status & ST_NONFINITE) == 0);
        const bool ok = sound && (GaL >= P.k) && (GaR < P.k);
        set_verdict(P, ok, sound, GaL, GaR);
        if (cb > (unsigned long long)P.band_cap) atomicOr(&ctl->status, ST_BAND_OVERFLOW);
    }
}

// ================================================================= p pass --
// p = F((r - b)/t), walking forward (the certification pass left the head of
// the row in L2).  Also sum p (fp64 over fp32 float4 partials) for diagnostics.
// Four p at once, one lane at a time (any subset of a warp may call it).
__device__ __forceinline__ float4 p_vec_lane(const float4 v, const PForm &pf) {
    return make_float4(pf(v.x), pf(v.y), pf(v.z), pf(v.w));
}

// Eight p (one chunk slot pair) at once: the fp32 value for all, then the fp64
// value of the mid-range ones, one per lane per round (the lane's first pending
// one), so a warp evaluates the fp64 form as often as its busiest lane has a
// mid-range score -- usually once -- not once per slot that any lane needs.
// Every lane of the warp must call it together.
__device__ __forceinline__ void p_vec8(const float4 v0, const float4 v1, const PForm &pf, float4 &o0, float4 &o1) {
    unsigned mm = 0;
    mm |= pf.fast(v0.x, o0.x) ? 1u : 0u;
    mm |= pf.fast(v0.y, o0.y) ? 2u : 0u;
    mm |= pf.fast(v0.z, o0.z) ? 4u : 0u;
    mm |= pf.fast(v0.w, o0.w) ? 8u : 0u;
    mm |= pf.fast(v1.x, o1.x) ? 16u : 0u;
    mm |= pf.fast(v1.y, o1.y) ? 32u : 0u;
    mm |= pf.fast(v1.z, o1.z) ? 64u : 0u;
    mm |= pf.fast(v1.w, o1.w) ? 128u : 0u;
    while (__any_sync(FULL, mm != 0u)) {
        const int i = mm ? __ffs(mm) - 1 : 0;
        const float q = pf.mid(pick8(v0, v1, i));
        const unsigned hit = mm & (0u - mm);   // the slot this lane fills (0: none)
        o0.x = (hit & 1u) ? q : o0.x;
        o0.y = (hit & 2u) ? q : o0.y;
        o0.z = (hit & 4u) ? q : o0.z;
        o0.w = (hit & 8u) ? q : o0.w;
        o1.x = (hit & 16u) ? q : o1.x;
        o1.y = (hit & 32u) ? q : o1.y;
        o1.z = (hit & 64u) ? q : o1.z;
        o1.w = (hit & 128u) ? q : o1.w;
        mm &= mm - 1u;
    }
}

__global__ void __launch_bounds__(SBLOCK, SBLOCKS_PER_SM)
p_kernel(const float *__restrict__ r_, int64_t n, double inv_t, float *__restrict__ p_,
         double *__restrict__ b_out_, Ctl *ctl_, double *partials_, int64_t pstride) {
    const int64_t row = blockIdx.y;   // rows of a batch: one grid.y slice each
    const float *__restrict__ r = r_ + row * n;
    float *__restrict__ p = p_ + row * n;
    double *b_out = b_out_ ? b_out_ + row : nullptr;
    Ctl *ctl = ctl_ + row;
    double *partials = partials_ + row * pstride;
    extern __shared__ __align__(128) unsigned char dsm[];
    __shared__ double s_red[SBLOCK / 32];
    pdl_enter();
    const double b = ctl->b;
    const PForm xf = make_pform(b, inv_t * LOG2E);
    const int64_t gtid = (int64_t)blockIdx.x * SBLOCK + threadIdx.x;
    const int64_t gstride = (int64_t)gridDim.x * SBLOCK;
    const bool aligned = ((reinterpret_cast<uintptr_t>(r) | reinterpret_cast<uintptr_t>(p)) & 15) == 0;
    const int64_t n4 = aligned ? n / 4 : 0;
    const float4 *r4 = reinterpret_cast<const float4 *>(r);
    float4 *p4 = reinterpret_cast<float4 *>(p);
    double ps = 0.0;
    int64_t done4 = 0;
    if (aligned) {
        const float4 *src[1] = {r4};
        done4 = bulk_stream<1>(src, n4, false, dsm, &ctl->status, [&](const float4 *const *ch, int64_t base4) {
            const float4 v0 = lds128(ch[0] + threadIdx.x), v1 = lds128(ch[0] + threadIdx.x + SBLOCK);
            float4 o0, o1;
            if (__all_sync(FULL, v0.x == v0.y && v0.y == v0.z && v0.z == v0.w && v1.x == v1.y && v1.y == v1.z &&
                                     v1.z == v1.w)) {   // tied scores (one vote a chunk): one p per float4
                float q0, q1;
                const bool m0 = xf.fast(v0.x, q0), m1 = xf.fast(v1.x, q1);
                if (__any_sync(FULL, m0 || m1)) {
                    if (m0) q0 = xf.mid(v0.x);
                    if (m1) q1 = xf.mid(v1.x);
                }
                o0 = make_float4(q0, q0, q0, q0);
                o1 = make_float4(q1, q1, q1, q1);
            } else {
                p_vec8(v0, v1, xf, o0, o1);
            }
            __stcs(p4 + base4 + threadIdx.x, o0);
            __stcs(p4 + base4 + threadIdx.x + SBLOCK, o1);
            ps += (double)(((o0.x + o0.y) + (o0.z + o0.w)) + ((o1.x + o1.y) + (o1.z + o1.w)));
        });
    }
    for (int64_t i = done4 + gtid; i < n4; i += gstride) {
        const float4 o = p_vec_lane(r4[i], xf);   // the tail: not every lane of a warp is here
        __stcs(p4 + i, o);
        ps += (double)((o.x + o.y) + (o.z + o.w));
    }
    for (int64_t j = n4 * 4 + gtid; j < n; j += gstride) {
        const float o = xf(r[j]);
        ps += (double)o;
        p[j] = o;
    }
    double v[1] = {ps};
    block_sum<SBLOCK, 1>(v, s_red);
    if (last_block_sum<SBLOCK, 1>(v, partials + 16 * (size_t)gridDim.x, &ctl->ticket[2], s_red) &&
        threadIdx.x == 0) {
        ctl->sum_p = v[0];
        if (b_out) *b_out = b;
    }
}

// =================================================================== VJP --
// <g,f> and sum f of one long row (walking backward: the p pass left the tail
// in L2).  Terms are e^{-|x|} in fp32; each thread sums the
// terms of one chunk (eight scores: positive terms, and g e products whose
// fp32 rounding is ~1e-7 of their magnitudes) in fp32 and adds that partial to
// fp64 accumulators, so the fp64 pipe sees two adds per eight scores.  If
// sum e is below 2^-96 (every score farther than ~66 t from b: some terms may
// have lost significant bits as fp32 denormals, or underflowed), the last block
// raises a flag and vjp_shifted_kernel recomputes the ratio from terms shifted
// by the running minimum of |x| (the shift cancels in <g,f>/sum f).
// SLICE: one slice of a row split across ranks -- the terms are shifted by
// 2^{sh2} (sh2 = 0, or the smallest |x2| over every rank when the plain sums
// are too small), and the last block writes {sum e, sum g e, min |x2|} to
// part_out for the ranks' exchange instead of lambda.
template <bool SLICE>
__global__ void __launch_bounds__(SBLOCK, SBLOCKS_PER_SM)
vjp_reduce_kernel(const float *__restrict__ r_, const double *__restrict__ b_in_,
                  const float *__restrict__ g_, int64_t n, double inv_t, Ctl *ctl_, double *partials_,
                  int64_t pstride, float sh2, double *part_out) {
    const int64_t row = blockIdx.y;
    const float *__restrict__ r = r_ + row * n;
    const float *__restrict__ g = g_ + row * n;
    const double *b_in = b_in_ + row;
    Ctl *ctl = ctl_ + row;
    double *partials = partials_ + row * pstride;
    extern __shared__ __align__(128) unsigned char dsm[];
    __shared__ double s_red[2 * (SBLOCK / 32)];
    pdl_enter();
    const double b = *b_in;
    const XForm xf = make_xform(b, inv_t * LOG2E);
    const int64_t gtid = (int64_t)blockIdx.x * SBLOCK + threadIdx.x;
    const int64_t gstride = (int64_t)gridDim.x * SBLOCK;
    const bool aligned = ((reinterpret_cast<uintptr_t>(r) | reinterpret_cast<uintptr_t>(g)) & 15) == 0;
    const int64_t n4 = aligned ? n / 4 : 0;
    const float4 *r4 = reinterpret_cast<const float4 *>(r);
    const float4 *g4 = reinterpret_cast<const float4 *>(g);
    double sf = 0.0, sgf = 0.0;
    float amin = CUDART_INF_F;   // SLICE: smallest |x2| of the thread's scores
    auto term = [&](float r1) {
        const float a = fabsf(xf(r1));
        if (SLICE) amin = fminf(amin, a);
        return SLICE ? exp2f(sh2 - a) : exp2f(-a);
    };
    auto part4 = [&](const float4 v, const float4 w, float &f32, float &gf32) {
        const float e0 = term(v.x), e1 = term(v.y);
        const float e2 = term(v.z), e3 = term(v.w);
        f32 += (e0 + e1) + (e2 + e3);
        gf32 = fmaf(w.x, e0, gf32);
        gf32 = fmaf(w.y, e1, gf32);
        gf32 = fmaf(w.z, e2, gf32);
        gf32 = fmaf(w.w, e3, gf32);
    };
    int64_t done4 = 0;
    if (aligned) {
        const float4 *src[2] = {r4, g4};
        done4 = bulk_stream<2>(src, n4, true, dsm, &ctl->status, [&](const float4 *const *ch, int64_t) {
            float f32 = 0.f, gf32 = 0.f;
            part4(lds128(ch[0] + threadIdx.x), lds128(ch[1] + threadIdx.x), f32, gf32);
            part4(lds128(ch[0] + threadIdx.x + SBLOCK), lds128(ch[1] + threadIdx.x + SBLOCK), f32, gf32);
            sf += (double)f32;
            sgf += (double)gf32;
        });
    }
    for (int64_t i = done4 + gtid; i < n4; i += gstride) {
        float f32 = 0.f, gf32 = 0.f;
        part4(r4[i], g4[i], f32, gf32);
        sf += (double)f32;
        sgf += (double)gf32;
    }
    for (int64_t i = n4 * 4 + gtid; i < n; i += gstride) {
        const float e = term(r[i]);
        sf += (double)e;
        sgf = fma((double)g[i], (double)e, sgf);
    }
    if (SLICE) {   // the slice's smallest |x2|: block minimum, then one atomic per block
        __shared__ unsigned s_min;
        if (threadIdx.x == 0) s_min = 0x7f800000u;
        __syncthreads();
        amin = fminf(amin, __shfl_xor_sync(FULL, amin, 16));
        amin = fminf(amin, __shfl_xor_sync(FULL, amin, 8));
        amin = fminf(amin, __shfl_xor_sync(FULL, amin, 4));
        amin = fminf(amin, __shfl_xor_sync(FULL, amin, 2));
        amin = fminf(amin, __shfl_xor_sync(FULL, amin, 1));
        if ((threadIdx.x & 31) == 0) atomicMin(&s_min, __float_as_uint(amin));   // amin >= 0: bits order as values
        __syncthreads();
        if (threadIdx.x == 0) atomicMin(reinterpret_cast<unsigned *>(&ctl->vjp_min), s_min);
    }
    double v[2] = {sf, sgf};
    block_sum<SBLOCK, 2>(v, s_red);
    if (last_block_sum<SBLOCK, 2>(v, partials, &ctl->ticket[3], s_red) && threadIdx.x == 0) {
        if (SLICE) {
            __threadfence();
            part_out[0] = v[0];
            part_out[1] = v[1];
            // the slice's smallest |x| in natural units (|x2| = |x| log2 e)
            part_out[2] = (double)__uint_as_float(atomicAdd(reinterpret_cast<unsigned *>(&ctl->vjp_min), 0u)) / LOG2E;
            return;
        }
        ctl->vjp_lambda = v[1] / v[0];
        // below 2^-96 some terms may be denormal in fp32 (fewer significant
        // bits) or lost; the shifted recomputation keeps every term's precision
        ctl->vjp_shift = !(v[0] >= 0x1p-96);
    }
}

struct ShiftSumG {
    float m;
    double sf, sgf;
};
__device__ __forceinline__ void ss_add(ShiftSumG &s, float ax, float g) {
    ax = fminf(ax, 3.0e38f);   // |x| may overflow fp32 (t tiny): keep the shift finite
    if (ax < s.m) {
        const double sc = (double)exp2f(ax - s.m);
        s.sf *= sc;
        s.sgf *= sc;
        s.m = ax;
    }
    const double e = (double)exp2f(s.m - ax);
    s.sf += e;
    s.sgf = fma((double)g, e, s.sgf);
}
__device__ __forceinline__ ShiftSumG ss_merge(ShiftSumG a, ShiftSumG b) {
    if (b.sf == 0.0) return a;
    if (a.sf == 0.0) return b;
    ShiftSumG r;
    r.m = fminf(a.m, b.m);
    const double fa = (double)exp2f(r.m - a.m), fb = (double)exp2f(r.m - b.m);
    r.sf = a.sf * fa + b.sf * fb;
    r.sgf = a.sgf * fa + b.sgf * fb;
    return r;
}

// Rare path: sum f was below 2^-96 in vjp_reduce_kernel (b far from every score).
__global__ void __launch_bounds__(SBLOCK)
vjp_shifted_kernel(const float *__restrict__ r_, const double *__restrict__ b_in_,
                   const float *__restrict__ g_, int64_t n, double inv_t, Ctl *ctl_, double *partials_,
                   int64_t pstride) {
    const int64_t row = blockIdx.y;
    const float *__restrict__ r = r_ + row * n;
    const float *__restrict__ g = g_ + row * n;
    const double *b_in = b_in_ + row;
    Ctl *ctl = ctl_ + row;
    double *partials = partials_ + row * pstride;
    __shared__ ShiftSumG s_w[SBLOCK / 32];
    __shared__ bool s_last;
    pdl_enter();
    if (!ctl->vjp_shift) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const XForm xf = make_xform(*b_in, inv_t * LOG2E);
    ShiftSumG ss{CUDART_INF_F, 0.0, 0.0};
    for (int64_t i = (int64_t)blockIdx.x * SBLOCK + tid; i < n; i += (int64_t)gridDim.x * SBLOCK)
        ss_add(ss, fabsf(xf(r[i])), g[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ShiftSumG q{__shfl_xor_sync(FULL, ss.m, o), __shfl_xor_sync(FULL, ss.sf, o),
                    __shfl_xor_sync(FULL, ss.sgf, o)};
        ss = ss_merge(ss, q);
    }
    if (lane == 0) s_w[warp] = ss;
    __syncthreads();
    const int G = gridDim.x;
    if (tid == 0) {
        ShiftSumG a = s_w[0];
        for (int w = 1; w < SBLOCK / 32; ++w) a = ss_merge(a, s_w[w]);
        partials[blockIdx.x] = (double)a.m;
        partials[G + blockIdx.x] = a.sf;
        partials[2 * G + blockIdx.x] = a.sgf;
        __threadfence();
        s_last = atomicAdd(&ctl->ticket[7], 1u) == (unsigned)G - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (tid == 0) {
        ShiftSumG a{CUDART_INF_F, 0.0, 0.0};
        for (int j = 0; j < G; ++j) {
            ShiftSumG q{(float)__ldcg(partials + j), __ldcg(partials + G + j), __ldcg(partials + 2 * G + j)};
            a = ss_merge(a, q);
        }
        ctl->vjp_lambda = a.sgf / a.sf;
        ctl->ticket[7] = 0u;
    }
}

__global__ void __launch_bounds__(SBLOCK, SBLOCKS_PER_SM)
vjp_apply_kernel(const float *__restrict__ r_, const double *__restrict__ b_in_,
                 const float *__restrict__ g_, int64_t n, double inv_t, const Ctl *ctl_,
                 float *__restrict__ grad_) {
    const int64_t row = blockIdx.y;
    const float *__restrict__ r = r_ + row * n;
    const float *__restrict__ g = g_ + row * n;
    const double *b_in = b_in_ + row;
    const Ctl *ctl = ctl_ + row;
    float *__restrict__ grad = grad_ + row * n;
    extern __shared__ __align__(128) unsigned char dsm[];
    pdl_enter();
    const XForm xf = make_xform(*b_in, inv_t * LOG2E);
    const double lam = ctl->vjp_lambda;
    const float lam_hi = (float)lam, lam_lo = (float)(lam - (double)lam_hi);
    const float hit = vjp_scale2(inv_t);   // log2(1/(2t))
    const int64_t gtid = (int64_t)blockIdx.x * SBLOCK + threadIdx.x;
    const int64_t gstride = (int64_t)gridDim.x * SBLOCK;
    const bool aligned = ((reinterpret_cast<uintptr_t>(r) | reinterpret_cast<uintptr_t>(g) |
                           reinterpret_cast<uintptr_t>(grad)) & 15) == 0;
    const int64_t n4 = aligned ? n / 4 : 0;
    const float4 *r4 = reinterpret_cast<const float4 *>(r);
    const float4 *g4 = reinterpret_cast<const float4 *>(g);
    float4 *o4 = reinterpret_cast<float4 *>(grad);
    auto apply4 = [&](const float4 v, const float4 w) {
        float4 o;
        o.x = vjp_term2(xf(v.x), w.x, hit, lam_hi, lam_lo);
        o.y = vjp_term2(xf(v.y), w.y, hit, lam_hi, lam_lo);
        o.z = vjp_term2(xf(v.z), w.z, hit, lam_hi, lam_lo);
        o.w = vjp_term2(xf(v.w), w.w, hit, lam_hi, lam_lo);
        return o;
    };
    int64_t done4 = 0;
    if (aligned) {
        const float4 *src[2] = {r4, g4};
        done4 = bulk_stream<2>(src, n4, false, dsm, const_cast<int32_t *>(&ctl->status),
                               [&](const float4 *const *ch, int64_t base4) {
            __stcs(o4 + base4 + threadIdx.x, apply4(lds128(ch[0] + threadIdx.x), lds128(ch[1] + threadIdx.x)));
            __stcs(o4 + base4 + threadIdx.x + SBLOCK,
                   apply4(lds128(ch[0] + threadIdx.x + SBLOCK), lds128(ch[1] + threadIdx.x + SBLOCK)));
        });
    }
    for (int64_t i = done4 + gtid; i < n4; i += gstride) __stcs(o4 + i, apply4(r4[i], g4[i]));
    for (int64_t i = n4 * 4 + gtid; i < n; i += gstride)
        grad[i] = vjp_term2(xf(r[i]), g[i], hit, lam_hi, lam_lo);
}

// ============================================================= self-test --
__global__ void selftest_math_kernel(int which, const double *in, double *out, double *ref, int64_t n) {
    __shared__ double s_tab[32];
    exp2_table_init(s_tab);
    __syncthreads();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const double x = in[i];
        if (which == 0) {
            out[i] = exp2_neg(x, s_tab);
            ref[i] = exp2(-x);
        } else {
            out[i] = sample_ln(x);
            ref[i] = log(x);
        }
    }
}

// ============================================================= launchers --
cudaError_t launch_selftest_math(int which, const double *in, double *out, double *ref, int64_t n,
                                 cudaStream_t st) {
    selftest_math_kernel<<<148, 256, 0, st>>>(which, in, out, ref, n);
    return cudaGetLastError();
}
// Streaming grids for a batch: the CTAs of one full-device grid shared out
// among the rows (grid.y = row), at least one each.
static dim3 row_grid(int per_sm, int64_t rows) {
    const int64_t g = stream_grid(per_sm) / rows;
    return dim3((unsigned)(g < 1 ? 1 : g), (unsigned)rows);
}
int64_t partial_stride(int64_t rows) {
    return 24 * (int64_t)row_grid(SBLOCKS_PER_SM, rows).x + 64;
}

cudaError_t launch_sample(const BracketParams &P, cudaStream_t st) {
    return launch_k(sample_kernel, dim3((unsigned)((P.s + 255) / 256), (unsigned)P.rows), 256, 0, st, P);
}
// 64 CTAs for one row; a batch shares about four CTAs per SM among its rows
cudaError_t launch_select(const BracketParams &P, cudaStream_t st) {
    int64_t per_row = (int64_t)stream_grid() / P.rows;
    per_row = per_row < 1 ? 1 : (per_row > SEL_GRID ? SEL_GRID : per_row);
    return launch_k(select_kernel, dim3((unsigned)per_row, (unsigned)P.rows), SEL_BLOCK, 0, st, P);
}
int select_cand_capacity() { return SEL_CAND; }
template <typename K>
static cudaError_t set_smem(K kern, size_t bytes) {
    return set_max_dynamic_smem(reinterpret_cast<const void *>(kern), bytes);
}

cudaError_t launch_stream_pass(const BracketParams &P, cudaStream_t st) {
    const cudaError_t once = set_smem(oob_kernel<OOB_STREAM>, bulk_smem_bytes<1>());
    const cudaError_t once2 = set_smem(oob_kernel<OOB_STREAM_CERT>, bulk_smem_bytes<1>());
    if (once != cudaSuccess) return once;
    if (once2 != cudaSuccess) return once2;
    if (P.fused_cert)
        return launch_k(oob_kernel<OOB_STREAM_CERT>, row_grid(3, P.rows), SBLOCK, bulk_smem_bytes<1>(), st, P);
    return launch_k(oob_kernel<OOB_STREAM>, row_grid(SBLOCKS_PER_SM, P.rows), SBLOCK, bulk_smem_bytes<1>(), st, P);
}
cudaError_t launch_certify(const BracketParams &P, cudaStream_t st) {
    const cudaError_t once = set_smem(oob_kernel<OOB_CERT, 3>, bulk_smem_bytes<1>());
    const cudaError_t once4 = set_smem(oob_kernel<OOB_CERT, 4, true>, bulk_smem_bytes<1>());
    if (once != cudaSuccess || once4 != cudaSuccess) return once != cudaSuccess ? once : once4;
    if (P.rows > 1)
        return launch_k(oob_kernel<OOB_CERT, 4, true>, row_grid(4, P.rows), SBLOCK, bulk_smem_bytes<1>(), st, P);
    return launch_k(oob_kernel<OOB_CERT, 3>, row_grid(3, P.rows), SBLOCK, bulk_smem_bytes<1>(), st, P);
}
cudaError_t launch_p_pass(const float *r, int64_t rows, int64_t n, double t, float *p, double *b_out, Ctl *ctl,
                          double *partials, cudaStream_t st) {
    const cudaError_t once = set_smem(p_kernel, bulk_smem_bytes<1>());
    if (once != cudaSuccess) return once;
    return launch_k(p_kernel, row_grid(SBLOCKS_PER_SM, rows), SBLOCK, bulk_smem_bytes<1>(), st, r, n, 1.0 / t, p,
                    b_out, ctl, partials, partial_stride(rows));
}
cudaError_t launch_vjp_reduce(const float *r, const double *b, const float *g, int64_t rows, int64_t n, double t,
                              Ctl *ctl, double *partials, cudaStream_t st) {
    const cudaError_t once = set_smem(vjp_reduce_kernel<false>, bulk_smem_bytes<2>());
    if (once != cudaSuccess) return once;
    const int64_t ps = partial_stride(rows);
    cudaError_t e = launch_k(vjp_reduce_kernel<false>, row_grid(SBLOCKS_PER_SM, rows), SBLOCK, bulk_smem_bytes<2>(),
                             st, r, b, g, n, 1.0 / t, ctl, partials, ps, 0.0f, (double *)nullptr);
    if (e != cudaSuccess) return e;
    dim3 gs = row_grid(SBLOCKS_PER_SM, rows);
    gs.x = gs.x / SBLOCKS_PER_SM < 1 ? 1 : gs.x / SBLOCKS_PER_SM;
    return launch_k(vjp_shifted_kernel, gs, SBLOCK, 0, st, r, b, g, n, 1.0 / t, ctl, partials, ps);
}
cudaError_t launch_vjp_slice_partial(const float *r, const double *b, const float *g, int64_t n, double t,
                                     float sh2, Ctl *ctl, double *partials, double *part_out, cudaStream_t st) {
    const cudaError_t once = set_smem(vjp_reduce_kernel<true>, bulk_smem_bytes<2>());
    if (once != cudaSuccess) return once;
    return launch_k(vjp_reduce_kernel<true>, row_grid(SBLOCKS_PER_SM, 1), SBLOCK, bulk_smem_bytes<2>(), st, r, b, g,
                    n, 1.0 / t, ctl, partials, partial_stride(1), sh2, part_out);
}
cudaError_t launch_vjp_apply(const float *r, const double *b, const float *g, int64_t rows, int64_t n, double t,
                             const Ctl *ctl, float *grad, cudaStream_t st) {
    const cudaError_t once = set_smem(vjp_apply_kernel, bulk_smem_bytes<2>());
    if (once != cudaSuccess) return once;
    return launch_k(vjp_apply_kernel, row_grid(SBLOCKS_PER_SM, rows), SBLOCK, bulk_smem_bytes<2>(), st, r, b, g, n,
                    1.0 / t, ctl, grad);
}

}  // namespace lapsum
