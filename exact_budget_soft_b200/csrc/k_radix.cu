// k_radix.cu -- device-wide sort and locate-scan for rows too long for one
// CTA: the full-sort solver of "Fast LapSum: Exact Differentiable Top-k at
// Million Scale" (technical summary section 2.2) on a whole row (the fallback
// of the abstract, when certification fails) or on a band of the bracketing
// path (step 3) that exceeds the one-CTA capacity.
//
// Sort: keys-only LSD radix sort of the descending-order uint32 keys, 8-bit
// digits, "onesweep" style:
//   radix_hist_kernel   one read: all four digit histograms (per-thread run
//                       length combining, so long runs of tied scores cost one
//                       shared atomic per run), exclusive digit bases, and the
//                       set of digits on which every key agrees (those passes
//                       are skipped);
//   radix_pass_kernel   per digit: tiles taken in launch order from an atomic
//                       counter, in-tile stable ranking (per-warp histograms,
//                       __match_any_sync), decoupled look-back over earlier
//                       tiles for the global digit offsets (every wait bounded
//                       by a spin cap), a shared-memory scatter and coalesced
//                       runs of writes.
// Locate: one kernel; every CTA reduces one tile of sorted values to its two
// affine maps (prefix P, suffix Q); the last CTA scans the tile maps, finds the
// tile whose end brackets G = k, re-scans that tile in shared memory and takes
// the closed-form root.
//
// The host never learns the band size or the certification verdict: every
// kernel reads its element count and its gate from the control block and
// returns at once when it has nothing to do.
#include <cstdint>

#include "lapsum_device.cuh"
#include "lapsum_kernels.h"
#include "scan_solve.cuh"

namespace lapsum {

constexpr int RB = 512;             // radix pass: threads
constexpr int RK = 16;              // keys per thread
constexpr int RTILE = RB * RK;      // 8192 keys per tile
constexpr int RNW = RB / 32;
constexpr int HB = 256;             // histogram kernel threads

constexpr int LB = 1024;            // locate: threads
constexpr int LK = 16;              // values per thread
constexpr int LTILE = LB * LK;      // 16384 values per tile

int radix_tile() { return RTILE; }
int locate_tile() { return LTILE; }

// Element count behind a gate; < 0 means "nothing to do".
__device__ __forceinline__ int64_t gated_n(const SortArgs &A) {
    const Ctl *c = A.ctl;
    if (A.gate == GATE_BAND) {
        if (c->path != 2) return -1;
        const unsigned long long cb = c->c_band;
        if (cb <= (unsigned long long)A.small_cap || cb > (unsigned long long)A.cap) return -1;
        return (int64_t)cb;
    }
    if (A.gate == GATE_FALLBACK) {
        if (c->verdict != 0) return -1;
    }
    return A.n_host;
}

// n copies of one value c, between the seeds of the locate step (the band of a
// tied level, or a row whose scores are all equal): the threshold curve is
// constant across the run, G(c) = m0 + n/2 - d_top P_top/2 + d_bot Q_bot/2, and
// (G decreasing) the root lies in [bot, c] when G(c) <= k, else in [c, top).
__device__ void solve_equal_run(const SortArgs &A, int64_t n) {
    Ctl *ctl = A.ctl;
    double m0 = 0.0, top = CUDART_INF, P_top = 0.0, bot = -CUDART_INF, Q_bot = 0.0;
    if (A.gate == GATE_BAND) {
        m0 = (double)ctl->c_R;
        top = (double)ctl->a_R;
        P_top = ctl->S_R;
        bot = (double)ctl->a_L;
        Q_bot = ctl->S_L;
    }
    const double c = (double)A.src[0];
    const double d_top = top == CUDART_INF ? 0.0 : exp((c - top) / A.t);
    const double d_bot = bot == -CUDART_INF ? 0.0 : exp((bot - c) / A.t);
    const double nn = (double)n;
    const double Gc = m0 + 0.5 * nn - 0.5 * d_top * P_top + 0.5 * d_bot * Q_bot;
    double b;
    if (Gc <= A.k) {   // G decreasing: the root is at or below c
        b = solve_interval(c, bot, m0 + nn, nn + d_top * P_top, Q_bot, d_bot, A.k, A.t);
        ctl->j_star = n - 1;
    } else {
        b = solve_interval(top, c, m0, P_top, nn + d_bot * Q_bot, d_top, A.k, A.t);
        ctl->j_star = -1;
    }
    ctl->b = b;
    if (A.gate == GATE_FALLBACK) ctl->fallback_ran = 1;
}

// ------------------------------------------------------------ histogram --
__global__ void __launch_bounds__(HB) radix_hist_kernel(SortArgs A) {
    __shared__ uint32_t h[4][256];
    __shared__ bool s_last;
    __shared__ int s_trivial[4];
    pdl_enter();
    const int64_t n = gated_n(A);
    if (n < 0) return;
    const int tid = threadIdx.x;
    for (int i = tid; i < 4 * 256; i += HB) (&h[0][0])[i] = 0;
    __syncthreads();
    uint32_t cur[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
    uint32_t cnt[4] = {0, 0, 0, 0};
    const int64_t gstride = (int64_t)gridDim.x * HB;
    for (int64_t i = (int64_t)blockIdx.x * HB + tid; i < n; i += gstride) {
        const uint32_t key = desc_key(A.src[i]);
#pragma unroll
        for (int d = 0; d < 4; ++d) {
            const uint32_t bin = (key >> (8 * d)) & 0xffu;
            if (bin == cur[d]) {
                ++cnt[d];
            } else {
                if (cnt[d]) atomicAdd(&h[d][cur[d]], cnt[d]);
                cur[d] = bin;
                cnt[d] = 1;
            }
        }
    }
#pragma unroll
    for (int d = 0; d < 4; ++d)
        if (cnt[d]) atomicAdd(&h[d][cur[d]], cnt[d]);
    __syncthreads();
    for (int i = tid; i < 4 * 256; i += HB) {
        const uint32_t c = (&h[0][0])[i];
        if (c) atomicAdd(A.hist + i, (unsigned long long)c);
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&A.ctl->ticket[4], 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // exclusive digit bases (thread tid owns bin tid of every digit); a digit
    // whose histogram has one bin holding every key is skipped
    static_assert(HB == 256, "one thread per bin");
    __shared__ uint32_t s_wsum[HB / 32];
    for (int d = 0; d < 4; ++d) {
        const uint32_t c = (uint32_t)__ldcg(A.hist + d * 256 + tid);
        const int lane = tid & 31, warp = tid >> 5;
        uint32_t inc = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t p = __shfl_up_sync(FULL, inc, o);
            if (lane >= o) inc += p;
        }
        if (lane == 31) s_wsum[warp] = inc;
        __syncthreads();
        uint32_t off = 0;
        for (int w = 0; w < warp; ++w) off += s_wsum[w];
        A.dbase[d * 256 + tid] = off + inc - c;
        const int triv = __syncthreads_or(c == (uint32_t)n);
        if (tid == 0) s_trivial[d] = triv;
        __syncthreads();
    }
    for (int i = tid; i < 4 * 256; i += HB) A.hist[i] = 0ull;   // ready for the next sort
    if (tid == 0) {
        A.ctl->sort_skip = s_trivial[0] | (s_trivial[1] << 1) | (s_trivial[2] << 2) | (s_trivial[3] << 3);
        const bool all_equal = s_trivial[0] && s_trivial[1] && s_trivial[2] && s_trivial[3];
        A.ctl->sort_solved = all_equal ? 1 : 0;
        if (all_equal) solve_equal_run(A, n);
        A.ctl->sort_cur = -1;
        A.ctl->ticket[4] = 0u;
    }
}

// ----------------------------------------------------------- one digit --
constexpr unsigned long long LB_AGG = 1ull << 62;
constexpr unsigned long long LB_PREFIX = 2ull << 62;

__device__ __forceinline__ unsigned long long lb_pack(unsigned long long flag, uint32_t epoch,
                                                      uint32_t v) {
    return flag | ((unsigned long long)(epoch & 0x3fffffffu) << 32) | v;
}

__global__ void __launch_bounds__(RB, 1) radix_pass_kernel(SortArgs A, int pass, uint32_t epoch) {
    extern __shared__ __align__(16) unsigned char smem[];
    uint32_t *s_keys = reinterpret_cast<uint32_t *>(smem);            // RTILE
    uint32_t *s_hist = s_keys + RTILE;                                 // RNW * 256
    uint32_t *s_dstart = s_hist + RNW * 256;                           // 256: in-tile digit start
    uint32_t *s_gofs = s_dstart + 256;                                 // 256: global base - dstart
    __shared__ int s_tile, s_cur;
    __shared__ bool s_last;

    pdl_enter();
    const int64_t n = gated_n(A);
    if (n < 0) return;
    Ctl *ctl = A.ctl;
    if (ctl->sort_skip & (1 << pass)) return;   // every key agrees on this digit
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int sh = 8 * pass;
    const int64_t ntiles = (n + RTILE - 1) / RTILE;
    if (tid == 0) s_cur = ctl->sort_cur;
    __syncthreads();
    const int cur = s_cur;
    // persistent: tiles are claimed in order from one counter, so a tile only
    // ever waits on tiles already claimed by running CTAs
    for (;;) {
        if (tid == 0) s_tile = (int)atomicAdd(&ctl->tile_ctr[pass], 1u);
        __syncthreads();
        const int tile = s_tile;
        if (tile >= ntiles) break;
        const uint32_t *src = cur < 0 ? nullptr : (cur == 0 ? A.keys[0] : A.keys[1]);
        uint32_t *dst = cur == 0 ? A.keys[1] : A.keys[0];
        const int64_t base = (int64_t)tile * RTILE;
        const int cnt_tile = (int)min((int64_t)RTILE, n - base);
        for (int i = tid; i < RNW * 256; i += RB) s_hist[i] = 0;
        __syncthreads();
        // load (warp-striped) and count digits per warp
        uint32_t key[RK];
        uint32_t *my_hist = s_hist + warp * 256;
        const unsigned lt_mask = (1u << lane) - 1u;
#pragma unroll
        for (int i = 0; i < RK; ++i) {
            const int li = warp * 32 * RK + i * 32 + lane;
            const bool v = li < cnt_tile;
            uint32_t kk = 0xffffffffu;
            if (v) kk = src ? src[base + li] : desc_key(A.src[base + li]);
            key[i] = kk;
            const uint32_t d = v ? ((kk >> sh) & 0xffu) : 0x100u;
            const unsigned peers = __match_any_sync(FULL, d);
            if (v && lane == __ffs(peers) - 1) my_hist[d] += __popc(peers);
            __syncwarp();
        }
        __syncthreads();
        uint32_t tot = 0;
        if (tid < 256) {
            for (int w = 0; w < RNW; ++w) {
                const uint32_t c = s_hist[w * 256 + tid];
                s_hist[w * 256 + tid] = tot;
                tot += c;
            }
            // publish this tile's digit count, then look back for the exclusive prefix
            unsigned long long *lb = A.lookback + (size_t)tile * 256 + tid;
            uint32_t excl = 0;
            if (tile == 0) {
                st_release_u64(lb, lb_pack(LB_PREFIX, epoch, tot));
            } else {
                st_release_u64(lb, lb_pack(LB_AGG, epoch, tot));
                for (int p = tile - 1; p >= 0;) {
                    const unsigned long long *q = A.lookback + (size_t)p * 256 + tid;
                    unsigned long long v;
                    int it = 0;
                    for (;;) {
                        v = ld_acquire_u64(q);
                        if (((v >> 32) & 0x3fffffffu) == (epoch & 0x3fffffffu) && (v >> 62) != 0) break;
                        if (++it > A.spin_cap) {
                            atomicOr(&ctl->status, ST_TIMEOUT);
                            v = LB_PREFIX;   // give up: treat as a zero prefix
                            break;
                        }
                        __nanosleep(32);
                    }
                    excl += (uint32_t)(v & 0xffffffffu);
                    if ((v >> 62) == 2) break;
                    --p;
                }
                st_release_u64(lb, lb_pack(LB_PREFIX, epoch, excl + tot));
            }
            s_gofs[tid] = A.dbase[pass * 256 + tid] + excl;
            s_dstart[tid] = tot;   // temporarily the tile total of digit tid
        }
        __syncthreads();
        if (warp == 0) {   // exclusive scan of the 256 in-tile digit totals
            uint32_t v[8], run = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) { v[j] = s_dstart[lane * 8 + j]; run += v[j]; }
            uint32_t inc = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t p = __shfl_up_sync(FULL, inc, o);
                if (lane >= o) inc += p;
            }
            uint32_t ex = inc - run;
#pragma unroll
            for (int j = 0; j < 8; ++j) { const uint32_t c = v[j]; s_dstart[lane * 8 + j] = ex; ex += c; }
        }
        __syncthreads();
        if (tid < 256) s_gofs[tid] -= s_dstart[tid];
        for (int i = tid; i < RNW * 256; i += RB) s_hist[i] += s_dstart[i & 255];
        __syncthreads();
        // scatter into shared memory by (digit, warp, traversal order): stable
#pragma unroll
        for (int i = 0; i < RK; ++i) {
            const int li = warp * 32 * RK + i * 32 + lane;
            const bool v = li < cnt_tile;
            const uint32_t d = v ? ((key[i] >> sh) & 0xffu) : 0x100u;
            const unsigned peers = __match_any_sync(FULL, d);
            const int leader = __ffs(peers) - 1;
            uint32_t bs = 0;
            if (v && lane == leader) {
                bs = my_hist[d];
                my_hist[d] = bs + __popc(peers);
            }
            bs = __shfl_sync(FULL, bs, leader) + __popc(peers & lt_mask);
            if (v) s_keys[bs] = key[i];
            __syncwarp();
        }
        __syncthreads();
        for (int i = tid; i < cnt_tile; i += RB) {
            const uint32_t kk = s_keys[i];
            dst[(uint32_t)(s_gofs[(kk >> sh) & 0xffu] + (uint32_t)i)] = kk;
        }
        __syncthreads();
    }
    // the last CTA to finish publishes the new key buffer and rearms the counters
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&ctl->ticket[5], 1u) == gridDim.x - 1;
    __syncthreads();
    if (s_last && tid == 0) {
        ctl->sort_cur = cur >= 0 ? (cur ^ 1) : 0;
        ctl->tile_ctr[pass] = 0u;
        ctl->ticket[5] = 0u;
    }
}

// --------------------------------------------------------------- locate --
struct TileRec {
    double pa, ps;     // tile prefix map  P_end = pa * P_before + ps
    double qa, qs;     // tile suffix map  Q_first = qa * Q_after + qs
    double d_out;      // link from the tile's last value to the next value
    double p_end;      // filled by the last CTA
    double q_after;    // filled by the last CTA
    double pad;
};

__device__ __forceinline__ double sorted_val(const uint32_t *keys, const float *src, int64_t j) {
    return keys ? (double)desc_key_to_float(keys[j]) : (double)src[j];
}

__global__ void __launch_bounds__(LB, 1) locate_kernel(SortArgs A, double k, double t, double inv_t) {
    extern __shared__ __align__(16) unsigned char smem[];
    uint32_t *s_keys = reinterpret_cast<uint32_t *>(smem);                 // LTILE
    void *scratch = smem + (LTILE + LTILE / 32) * 4;                         // >= 6 KB
    __shared__ bool s_last;
    __shared__ int s_tstar;
    __shared__ double s_tab[32];
    exp2_table_init(s_tab);

    pdl_enter();
    const int64_t n = gated_n(A);
    if (n < 0) return;
    Ctl *ctl = A.ctl;
    if (ctl->sort_solved) return;   // every key equal: solved by the histogram kernel
    const int tid = threadIdx.x, lane = tid & 31;
    const int cur = ctl->sort_cur;
    const uint32_t *keys_cur = cur < 0 ? nullptr : (cur == 0 ? A.keys[0] : A.keys[1]);
    const double s2d = inv_t * LOG2E;
    __syncthreads();   // s_tab
    double m0 = 0.0, top = CUDART_INF, P_top = 0.0, bot = -CUDART_INF, Q_bot = 0.0;
    if (A.gate == GATE_BAND) {
        m0 = (double)ctl->c_R;
        top = (double)ctl->a_R;
        P_top = ctl->S_R;
        bot = (double)ctl->a_L;
        Q_bot = ctl->S_L;
    }
    TileRec *rec = reinterpret_cast<TileRec *>(A.tilebuf);
    const int64_t ntiles = (n + LTILE - 1) / LTILE;
    auto val = [&](int64_t j) -> double {
        if (j < 0) return top;
        if (j >= n) return bot;
        return sorted_val(keys_cur, A.src, j);
    };
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t j0 = tile * LTILE + (int64_t)tid * LK;
        const int64_t j1 = min(j0 + LK, n) - 1;
        Aff mp = aff_id(), mq = aff_id();
        double d_last = 0.0;
        if (j0 < n) {
            double cprev = val(j0 - 1);
            double c = val(j0);
            double dprev = (cprev == CUDART_INF || c == -CUDART_INF) ? 0.0 : link_exp((cprev - c) * s2d, s_tab);
            for (int64_t j = j0; j <= j1; ++j) {
                mp = {mp.a * dprev, fma(mp.s, dprev, 1.0)};
                const double cn = val(j + 1);
                const double d = (c == CUDART_INF || cn == -CUDART_INF) ? 0.0 : link_exp((c - cn) * s2d, s_tab);
                mq = {mq.a * d, mq.s + mq.a};
                dprev = d;
                c = cn;
            }
            d_last = dprev;
        }
        Aff pe, qe;
        block_scan_excl_both<LB>(mp, mq, pe, qe, reinterpret_cast<Aff *>(scratch));
        const int64_t tile_end = min((tile + 1) * LTILE, n) - 1;
        const int owner = (int)((tile_end - tile * LTILE) / LK);
        if (tid == owner) {
            const Aff P = aff_then(pe, mp);
            rec[tile].pa = P.a;
            rec[tile].ps = P.s;
            rec[tile].d_out = d_last;
        }
        if (tid == 0) {
            const Aff Q = aff_then(qe, mq);
            rec[tile].qa = Q.a;
            rec[tile].qs = Q.s;
        }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&ctl->ticket[6], 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // ---- last CTA: scan the tile maps, find the crossing tile, re-scan it
    Aff *sc = reinterpret_cast<Aff *>(scratch);
    double carry_p = P_top;
    for (int64_t c0 = 0; c0 < ntiles; c0 += LB) {
        const int64_t T = c0 + tid;
        Aff m = aff_id();
        if (T < ntiles) m = {__ldcg(&rec[T].pa), __ldcg(&rec[T].ps)};
        Aff pe, qe;
        block_scan_excl_both<LB>(m, aff_id(), pe, qe, sc);
        const Aff inc = aff_then(pe, m);
        if (T < ntiles) rec[T].p_end = fma(inc.a, carry_p, inc.s);
        // carry = inclusive of the chunk's last tile
        __shared__ double s_carry;
        const int64_t lastT = min(c0 + LB, ntiles) - 1;
        if (T == lastT) s_carry = fma(inc.a, carry_p, inc.s);
        __syncthreads();
        carry_p = s_carry;
        __syncthreads();
    }
    __threadfence_block();
    double carry_q = Q_bot;
    int best = -1;
    const int64_t nchunks = (ntiles + LB - 1) / LB;
    for (int64_t ci = nchunks - 1; ci >= 0; --ci) {
        const int64_t c0 = ci * LB;
        const int64_t T = c0 + tid;
        Aff m = aff_id();
        if (T < ntiles) m = {__ldcg(&rec[T].qa), __ldcg(&rec[T].qs)};
        Aff pe, qe;
        block_scan_excl_both<LB>(aff_id(), m, pe, qe, sc);
        // qe: maps of tiles T+1 .. chunk end applied (chunk-relative), then carry
        const double Qa = fma(qe.a, carry_q, qe.s);     // Q at the value after tile T
        if (T < ntiles) {
            rec[T].q_after = Qa;
            const int64_t tend = min((T + 1) * LTILE, n) - 1;
            const double G = (m0 + (double)(tend + 1)) - 0.5 * __ldcg(&rec[T].p_end) +
                             0.5 * __ldcg(&rec[T].d_out) * Qa;
            if (G <= k) best = max(best, (int)T);
        }
        __shared__ double s_cq;
        if (tid == 0) s_cq = fma(aff_then(qe, m).a, carry_q, aff_then(qe, m).s);
        __syncthreads();
        carry_q = s_cq;
        __syncthreads();
    }
    best = warp_max_int(best);
    if (tid == 0) s_tstar = -1;
    __syncthreads();
    if (lane == 0) atomicMax(&s_tstar, best);
    __syncthreads();
    const int64_t TT = min((int64_t)s_tstar + 1, ntiles - 1);
    const int64_t t0 = TT * LTILE;
    const int cnt = (int)min((int64_t)LTILE, n - t0);
    for (int i = tid; i < cnt; i += LB) {
        s_keys[spad(i)] = keys_cur ? keys_cur[t0 + i] : desc_key(A.src[t0 + i]);
    }
    __syncthreads();
    const double ptop = TT == 0 ? P_top : __ldcg(&rec[TT - 1].p_end);
    const double vtop = val(t0 - 1);
    const double qbot = __ldcg(&rec[TT].q_after);
    const double vbot = val(t0 + cnt);
    int64_t js = 0;
    const double b = block_scan_solve<LB, LK>(s_keys, cnt, k, t, inv_t, m0 + (double)t0, vtop, ptop,
                                              vbot, qbot, scratch, &js, &ctl->status, s_tab);
    if (tid == 0) {
        ctl->b = b;
        ctl->j_star = t0 + js;
        if (A.gate == GATE_FALLBACK) ctl->fallback_ran = 1;
        ctl->ticket[6] = 0u;
    }
}

// ------------------------------------------------------------ launchers --
static int num_sms() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
}

cudaError_t launch_radix_sort(SortArgs &A, double k, double t, cudaStream_t st) {
    (void)k;
    (void)t;
    const int64_t cap = A.cap;
    static bool attr = false;
    const size_t smem = (size_t)RTILE * 4 + (size_t)RNW * 256 * 4 + 2 * 256 * 4;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(radix_pass_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    int64_t hg = (cap + HB * 16 - 1) / (HB * 16);
    if (hg > (int64_t)num_sms() * 2) hg = (int64_t)num_sms() * 2;
    int hgrid = (int)hg;
    if (hgrid < 1) hgrid = 1;
    cudaError_t e = launch_k(radix_hist_kernel, hgrid, HB, 0, st, A);
    if (e != cudaSuccess) return e;
    int64_t pt = (cap + RTILE - 1) / RTILE;
    if (pt > num_sms()) pt = num_sms();   // persistent: one CTA per SM claims tiles in order
    const unsigned ptiles = (unsigned)pt;
    for (int pass = 0; pass < 4; ++pass) {
        e = launch_k(radix_pass_kernel, ptiles, RB, smem, st, A, pass, A.epoch * 4u + (uint32_t)pass);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_locate(const SortArgs &A, double k, double t, cudaStream_t st) {
    static bool attr = false;
    const size_t smem = (size_t)(LTILE + LTILE / 32) * 4 + 16384;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(locate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    int64_t lg = (A.cap + LTILE - 1) / LTILE;
    if (lg > num_sms()) lg = num_sms();
    const unsigned grid = (unsigned)lg;
    return launch_k(locate_kernel, grid, LB, smem, st, A, k, t, 1.0 / t);
}

}  // namespace lapsum
