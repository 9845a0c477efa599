// k_radix.cu -- device-wide sort and locate-scan for rows too long for one
// CTA: the full-sort solver of "Fast LapSum: Exact Differentiable Top-k at
// Million Scale" (technical summary section 2.2) on a whole row (the fallback
// of the abstract, when certification fails) or on a band of the bracketing
// path (step 3) that exceeds the one-CTA capacity.
//
// Sort: keys-only LSD radix sort of the descending-order uint32 keys, 8-bit
// digits, in one cooperative kernel (radix_sort_kernel, described below).
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
// keys per thread K: 16 (8192-key tiles) for long rows, 4 (2048-key tiles, more
// CTAs in parallel) when the sort holds at most SMALL_SORT keys
#define TILE_K(K) (RB * (K))
constexpr int RK_BIG = 16, RK_SMALL = 4;
constexpr int64_t SMALL_SORT = int64_t(1) << 20;
constexpr int RNW = RB / 32;
constexpr int HB = 256;             // histogram kernel threads

constexpr int LB = 1024;            // locate: threads
constexpr int LK = 16;              // values per thread
constexpr int LTILE = LB * LK;      // 16384 values per tile
constexpr int LOC_KEY_WORDS = LTILE + LTILE / 32 + 8;   // padded tile + two halo entries

int radix_tile() { return TILE_K(RK_BIG); }
int locate_tile() { return LTILE; }

// Element count behind a gate; < 0 means "nothing to do".
__device__ __forceinline__ int64_t gated_n(const SortArgs &A) {
    const Ctl *c = A.ctl;
    if (A.gate == GATE_BAND) {
        if (c->path != 2) return -1;
        if (A.round2 && !c->widened) return -1;
        const unsigned long long cb = c->c_band;
        if (cb <= (unsigned long long)A.small_cap || cb > (unsigned long long)A.cap) return -1;
        if (band_tied(c)) return -1;   // one tied value: the band solver takes it in closed form
        return (int64_t)cb;
    }
    if (A.gate == GATE_FALLBACK) {
        if (c->verdict != 0) return -1;
    }
    return A.n_host;
}

// n copies of one value c, between the seeds of the locate step (a row whose
// scores are all equal, or the band of one tied level): closed form.
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
    bool above = false;
    ctl->b = solve_equal_run_values((double)A.src[0], (double)n, m0, top, P_top, bot, Q_bot, A.k, A.t, &above);
    ctl->j_star = above ? n - 1 : -1;
    if (A.gate == GATE_FALLBACK) ctl->fallback_ran = 1;
}

// ------------------------------------------------------------ sort --
// One cooperative kernel (every CTA resident, bounded grid barriers between
// phases).  CTA c owns a contiguous chunk of tiles [t0, t1) in every pass.
//
//   phase H   each CTA: the four digit histograms of its chunk (per-thread run
//             length combining, so long runs of tied scores cost one shared
//             atomic per run) -> chunk counts of all four digits, and the
//             global histograms.  Barrier.  Every CTA then derives the digit
//             bases and the digits on which every key agrees (those passes
//             are skipped; all four: one value, solved in closed form).
//   pass p    count (not for the first pass run: phase H counted the input
//             order): the chunk's digit-p counts.  Barrier.  Each CTA sums the
//             counts of the chunks before its own (its global start of every
//             digit), then walks its tiles in order: a stable in-tile ranking
//             (per-warp digit histograms, __match_any_sync), a shared-memory
//             scatter and coalesced runs of writes, each digit's running
//             offset advanced by the tile's count.  Barrier.
//
// Each CTA stages its next tile in shared memory by one bulk copy while it
// works on the current one.  Data written inside the kernel by other CTAs is
// read through L2 (ld.global.cg or bulk copies), never through L1.

// The tile's keys, warp-striped (key i of lane l of warp w is tile element
// w*32*K + i*32 + l), all K loads in flight at once; keys past the end of the
// row read as 0xffffffff.  src == nullptr: the first pass, keys from the scores.
template <int K>
__device__ __forceinline__ void load_tile(const SortArgs &A, const uint32_t *src, int64_t base, int cnt_tile,
                                          uint32_t (&key)[K]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int l0 = warp * 32 * K + lane;
    if (src) {
#pragma unroll
        for (int i = 0; i < K; ++i)
            key[i] = l0 + i * 32 < cnt_tile ? __ldcg(src + base + l0 + i * 32) : 0xffffffffu;
    } else {
        float x[K];
#pragma unroll
        for (int i = 0; i < K; ++i) x[i] = l0 + i * 32 < cnt_tile ? __ldg(A.src + base + l0 + i * 32) : 0.0f;
#pragma unroll
        for (int i = 0; i < K; ++i) key[i] = l0 + i * 32 < cnt_tile ? desc_key(x[i]) : 0xffffffffu;
    }
}

// Double-buffered tile staging: only full tiles of a 16-byte-aligned source
// are copied (one bulk copy each, completion counted on an mbarrier); the
// ragged last tile takes plain loads.
template <int K>
struct TileStage {
    uint32_t *buf;      // 2 * TILE_K(K) words
    uint64_t *bar;      // 2 mbarriers
    const char *gsrc;   // 4-byte elements: the keys, or the scores
    bool bulk_ok;
    int64_t n;
};

template <int K>
__device__ __forceinline__ bool stage_full(const TileStage<K> &S, int64_t tile) {
    return S.bulk_ok && (tile + 1) * TILE_K(K) <= S.n;
}

// thread 0; the buffer must be free (its last readers are past a barrier)
template <int K>
__device__ __forceinline__ void stage_issue(const TileStage<K> &S, int slot, int64_t tile) {
    if (!stage_full(S, tile)) return;
    fence_proxy_async_smem();
    mbar_expect_tx(&S.bar[slot], TILE_K(K) * 4);
    bulk_load(S.buf + slot * TILE_K(K), S.gsrc + (size_t)tile * TILE_K(K) * 4, TILE_K(K) * 4, &S.bar[slot]);
}

template <int K>
__device__ __forceinline__ void stage_source(TileStage<K> &S, const SortArgs &A, const uint32_t *src) {
    S.gsrc = src ? reinterpret_cast<const char *>(src) : reinterpret_cast<const char *>(A.src);
    S.bulk_ok = (reinterpret_cast<uintptr_t>(S.gsrc) & 15u) == 0;
}

// The tile's keys into registers: from its staged copy (waiting, bounded, for
// the copy) or by plain loads.  Returns false when the wait gave up.
template <int K>
__device__ __forceinline__ bool stage_keys(const TileStage<K> &S, const SortArgs &A, const uint32_t *src, int slot,
                                           uint32_t &ph, int64_t tile, int cnt_tile, uint32_t (&key)[K]) {
    if (!stage_full(S, tile)) {
        load_tile(A, src, tile * TILE_K(K), cnt_tile, key);
        return true;
    }
    const bool ok = mbar_wait(&S.bar[slot], (ph >> slot) & 1u, BULK_WAIT_CAP);
    ph ^= 1u << slot;
    const uint32_t *sb = S.buf + slot * TILE_K(K);
    const int l0 = (threadIdx.x >> 5) * 32 * K + (threadIdx.x & 31);
    if (src) {
#pragma unroll
        for (int i = 0; i < K; ++i) key[i] = sb[l0 + i * 32];
    } else {
#pragma unroll
        for (int i = 0; i < K; ++i) key[i] = desc_key(__uint_as_float(sb[l0 + i * 32]));
    }
    return ok;
}

template <int K>
constexpr size_t stage_bytes() { return 2 * TILE_K(K) * 4 + 2 * sizeof(uint64_t); }

// Adds this warp's digit counts of the tile to my_hist (the warp's 256 counters).
template <int K>
__device__ __forceinline__ void warp_count(const uint32_t (&key)[K], int cnt_tile, int sh, uint32_t *my_hist) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int i = 0; i < K; ++i) {
        const int li = warp * 32 * K + i * 32 + lane;
        const bool v = li < cnt_tile;
        const uint32_t d = v ? ((key[i] >> sh) & 0xffu) : 0x100u;
        const unsigned peers = __match_any_sync(FULL, d);
        if (v && lane == __ffs(peers) - 1) my_hist[d] += __popc(peers);
        __syncwarp();
    }
}

// Walks the CTA's chunk of tiles in order with one tile staged ahead, calling
// body(tile, cnt_tile, key) with every thread's keys; a barrier follows each
// body, so the staging buffers are free again.  Returns false if a wait gave up.
template <int K, typename Body>
__device__ __forceinline__ bool walk_chunk(TileStage<K> &S, const SortArgs &A, const uint32_t *src, int64_t t0,
                                           int64_t t1, uint32_t &ph, Body &&body) {
    bool ok = true;
    stage_source(S, A, src);
    if (threadIdx.x == 0 && t0 < t1) stage_issue(S, 0, t0);
    int slot = 0;
    for (int64_t tile = t0; tile < t1; ++tile, slot ^= 1) {
        if (threadIdx.x == 0 && tile + 1 < t1) stage_issue(S, slot ^ 1, tile + 1);
        const int cnt_tile = (int)min((int64_t)TILE_K(K), S.n - tile * TILE_K(K));
        uint32_t key[K];
        ok &= stage_keys(S, A, src, slot, ph, tile, cnt_tile, key);
        body(tile, cnt_tile, key, S.buf + slot * TILE_K(K));
        __syncthreads();
    }
    return ok;
}

template <int K>
constexpr size_t sort_smem() { return stage_bytes<K>() + (size_t)(RNW * 256 + 4 * 256 + 4 * 256) * 4; }
constexpr int SORT_GMAX = 320;   // CTAs of the sort grid at most (chunk counts per digit)

template <int K>
__global__ void __launch_bounds__(RB, 2) radix_sort_kernel(SortArgs A) {
    extern __shared__ __align__(16) unsigned char smem[];
    uint32_t *s_hist = reinterpret_cast<uint32_t *>(smem + stage_bytes<K>());   // RNW * 256: per-warp digit counts
    uint32_t *s_dstart = s_hist + RNW * 256;   // 256: in-tile digit start
    uint32_t *s_gofs = s_dstart + 256;         // 256: global offset - in-tile start
    uint32_t *s_run = s_gofs + 256;            // 256: running global offset of each digit
    uint32_t *s_tot = s_run + 256;             // 256: scratch (tile totals)
    uint32_t *s_h4 = s_tot + 256;              // 4 * 256: phase-H histograms, then digit bases
    __shared__ int s_skip, s_solved;
    pdl_wait();
    const int64_t n = gated_n(A);
    if (n < 0) return;   // the gate reads the same control words in every CTA
    Ctl *ctl = A.ctl;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = gridDim.x, c = blockIdx.x;
    const int64_t ntiles = (n + TILE_K(K) - 1) / TILE_K(K);
    const int64_t t0 = (int64_t)c * ntiles / G, t1 = (int64_t)(c + 1) * ntiles / G;
    uint32_t *csum = A.chunkcnt;   // [4][256][G]
    auto bar = [&]() { grid_sync(&ctl->gbar_count, &ctl->gbar_gen, A.spin_cap, &ctl->status); };
    TileStage<K> S;
    S.buf = reinterpret_cast<uint32_t *>(smem);
    S.bar = reinterpret_cast<uint64_t *>(smem + 2 * TILE_K(K) * 4);
    S.n = n;
    if (tid == 0) {
        mbar_init(&S.bar[0], 1);
        mbar_init(&S.bar[1], 1);
        mbar_init_fence();
    }
    for (int i = tid; i < 4 * 256; i += RB) s_h4[i] = 0;
    __syncthreads();
    uint32_t ph = 0;
    bool ok = true;

    // ---- phase H: the chunk's four digit histograms
    {
        uint32_t cur[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
        uint32_t cnt[4] = {0, 0, 0, 0};
        ok &= walk_chunk(S, A, nullptr, t0, t1, ph, [&](int64_t, int cnt_tile, const uint32_t (&key)[K], uint32_t *) {
            const int l0 = warp * 32 * K + lane;
#pragma unroll
            for (int i = 0; i < K; ++i) {
                if (l0 + i * 32 >= cnt_tile) break;
#pragma unroll
                for (int d = 0; d < 4; ++d) {
                    const uint32_t bin = (key[i] >> (8 * d)) & 0xffu;
                    if (bin == cur[d]) {
                        ++cnt[d];
                    } else {
                        if (cnt[d]) atomicAdd(&s_h4[d * 256 + cur[d]], cnt[d]);
                        cur[d] = bin;
                        cnt[d] = 1;
                    }
                }
            }
        });
#pragma unroll
        for (int d = 0; d < 4; ++d)
            if (cnt[d]) atomicAdd(&s_h4[d * 256 + cur[d]], cnt[d]);
        __syncthreads();
        for (int i = tid; i < 4 * 256; i += RB) {
            const uint32_t v = s_h4[i];
            csum[(size_t)i * G + c] = v;
            if (v) atomicAdd(A.hist + i, (unsigned long long)v);
        }
    }
    bar();
    // digit bases and skip flags, the same in every CTA (thread d owns bin d)
    if (tid == 0) { s_skip = 0; s_solved = 0; }
    __syncthreads();
    for (int d4 = 0; d4 < 4; ++d4) {
        uint32_t v = 0;
        if (tid < 256) v = (uint32_t)__ldcg(A.hist + d4 * 256 + tid);
        uint32_t inc = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(FULL, inc, o);
            if (lane >= o) inc += y;
        }
        if (lane == 31 && tid < 256) s_tot[warp] = inc;
        __syncthreads();
        if (tid < 256) {
            uint32_t off = 0;
            for (int w = 0; w < warp; ++w) off += s_tot[w];
            s_h4[d4 * 256 + tid] = off + inc - v;   // exclusive base of bin tid
            if (v == (uint32_t)n) atomicOr(&s_skip, 1 << d4);
        }
        __syncthreads();
    }
    const int skip = s_skip;
    int cur = -1;   // key buffer of the current order (-1: the scores)
    if (skip == 15) {   // every key equal
        if (c == 0 && tid == 0) solve_equal_run(A, n);
    } else {
        bool first = true;
        for (int pass = 0; pass < 4; ++pass) {
            if (skip & (1 << pass)) continue;
            const int sh = 8 * pass;
            const uint32_t *src = cur < 0 ? nullptr : (cur == 0 ? A.keys[0] : A.keys[1]);
            uint32_t *dst = cur == 0 ? A.keys[1] : A.keys[0];
            uint32_t *crow = csum + (size_t)pass * 256 * G;   // [256][G] of this digit
            if (!first) {   // the chunk's digit counts in the current order
                for (int i = tid; i < RNW * 256; i += RB) s_hist[i] = 0;
                __syncthreads();
                ok &= walk_chunk(S, A, src, t0, t1, ph, [&](int64_t, int cnt_tile, const uint32_t (&key)[K], uint32_t *) {
                    warp_count(key, cnt_tile, sh, s_hist + warp * 256);
                });
                if (tid < 256) {
                    uint32_t tot = 0;
#pragma unroll
                    for (int w = 0; w < RNW; ++w) tot += s_hist[w * 256 + tid];
                    crow[(size_t)tid * G + c] = tot;
                }
                bar();
            }
            // global start of every digit in this chunk: base + counts of earlier
            // chunks (a warp per digit, four digits' loads in flight at once)
            for (int j = 0; j < 256 / RNW; j += 4) {
                uint32_t acc[4] = {0, 0, 0, 0};
#pragma unroll
                for (int u = 0; u < SORT_GMAX / 32; ++u) {
                    const int q = lane + 32 * u;
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj)
                        if (q < c) acc[jj] += __ldcg(crow + (size_t)(warp * (256 / RNW) + j + jj) * G + q);
                }
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    uint32_t a = acc[jj];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(FULL, a, o);
                    const int d = warp * (256 / RNW) + j + jj;
                    if (lane == 0) s_run[d] = s_h4[pass * 256 + d] + a;
                }
            }
            __syncthreads();
            ok &= walk_chunk(S, A, src, t0, t1, ph, [&](int64_t, int cnt_tile, const uint32_t (&key)[K], uint32_t *s_keys) {
                for (int i = tid; i < RNW * 256; i += RB) s_hist[i] = 0;
                __syncthreads();   // every key is in registers: s_keys is free too
                uint32_t *my_hist = s_hist + warp * 256;
                warp_count(key, cnt_tile, sh, my_hist);
                __syncthreads();
                if (tid < 256) {   // per digit: exclusive offsets of the warps, tile total
                    uint32_t tot = 0;
#pragma unroll
                    for (int w = 0; w < RNW; ++w) {
                        const uint32_t cw = s_hist[w * 256 + tid];
                        s_hist[w * 256 + tid] = tot;
                        tot += cw;
                    }
                    s_tot[tid] = tot;
                    s_gofs[tid] = s_run[tid];
                    s_run[tid] += tot;
                }
                __syncthreads();
                if (warp == 0) {   // exclusive scan of the 256 tile totals
                    uint32_t v[8], run = 0;
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) { v[jj] = s_tot[lane * 8 + jj]; run += v[jj]; }
                    uint32_t inc = run;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const uint32_t y = __shfl_up_sync(FULL, inc, o);
                        if (lane >= o) inc += y;
                    }
                    uint32_t ex = inc - run;
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) { const uint32_t cc = v[jj]; s_dstart[lane * 8 + jj] = ex; ex += cc; }
                }
                __syncthreads();
                if (tid < 256) s_gofs[tid] -= s_dstart[tid];
                for (int i = tid; i < RNW * 256; i += RB) s_hist[i] += s_dstart[i & 255];
                __syncthreads();
                // scatter into shared memory by (digit, warp, traversal order): stable
                const unsigned lt_mask = (1u << lane) - 1u;
#pragma unroll
                for (int i = 0; i < K; ++i) {
                    const int li = warp * 32 * K + i * 32 + lane;
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
                // runs of one digit are consecutive in s_keys and in dst: coalesced writes
                for (int i = tid; i < cnt_tile; i += RB) {
                    const uint32_t kk = s_keys[i];
                    dst[(uint32_t)(s_gofs[(kk >> sh) & 0xffu] + (uint32_t)i)] = kk;
                }
            });
            bar();   // the pass's keys are all written before the next pass reads them
            cur = cur == 0 ? 1 : 0;
            first = false;
        }
    }
    if (!ok) atomicOr(&ctl->status, ST_TIMEOUT);
    bar();   // every CTA has read the global histograms
    if (c == 0) {
        for (int i = tid; i < 4 * 256; i += RB) A.hist[i] = 0ull;   // ready for the next sort
        if (tid == 0) {
            ctl->sort_cur = cur;
            ctl->sort_solved = skip == 15 ? 1 : 0;
        }
    }
    pdl_trigger();
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
    void *scratch = smem + LOC_KEY_WORDS * 4;                                // >= 6 KB
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
    // staged tile: s_keys[spad(i + 1)] holds sorted position tile*LTILE + i for
    // i = -1 .. cnt (the two halo entries are the neighbours or the seeds)
    const uint32_t key_top = desc_key((float)top), key_bot = desc_key((float)bot);
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t t0 = tile * LTILE;
        const int cnt = (int)min((int64_t)LTILE, n - t0);
        uint32_t kv[LK];
#pragma unroll
        for (int u = 0; u < LK; ++u) {   // coalesced, all loads in flight at once
            const int i = u * LB + tid;
            kv[u] = 0u;
            if (i < cnt) kv[u] = keys_cur ? __ldcs(keys_cur + t0 + i) : desc_key(__ldg(A.src + t0 + i));
        }
#pragma unroll
        for (int u = 0; u < LK; ++u) {
            const int i = u * LB + tid;
            if (i < cnt) s_keys[spad(i + 1)] = kv[u];
        }
        if (tid == 0) {
            s_keys[spad(0)] = t0 == 0 ? key_top
                                      : (keys_cur ? keys_cur[t0 - 1] : desc_key(A.src[t0 - 1]));
            s_keys[spad(cnt + 1)] = t0 + cnt >= n ? key_bot
                                      : (keys_cur ? keys_cur[t0 + cnt] : desc_key(A.src[t0 + cnt]));
        }
        __syncthreads();
        auto sval = [&](int i) -> double { return (double)desc_key_to_float(s_keys[spad(i + 1)]); };
        const int l0 = tid * LK;
        const int l1 = min(l0 + LK, cnt) - 1;
        Aff mp = aff_id(), mq = aff_id();
        double d_last = 0.0;
        if (l0 < cnt) {
            double cprev = sval(l0 - 1);
            double c = sval(l0);
            double dprev = (cprev == CUDART_INF || c == -CUDART_INF) ? 0.0 : link_exp((cprev - c) * s2d, s_tab);
            for (int j = l0; j <= l1; ++j) {
                mp = {mp.a * dprev, fma(mp.s, dprev, 1.0)};
                const double cn = sval(j + 1);
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

int sort_grid_max() { return SORT_GMAX; }

template <int K>
static cudaError_t launch_sort_k(SortArgs &A, cudaStream_t st) {
    static int resident = 0;   // CTAs of this sort kernel that fit the device at once
    if (!resident) {
        cudaError_t e = cudaFuncSetAttribute(radix_sort_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)sort_smem<K>());
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, radix_sort_kernel<K>, RB, sort_smem<K>());
        if (e != cudaSuccess) return e;
        if (per_sm < 1) return cudaErrorInvalidConfiguration;
        resident = per_sm * num_sms();
    }
    int64_t g = (A.cap + TILE_K(K) - 1) / TILE_K(K);
    if (g > resident) g = resident;
    if (g > SORT_GMAX) g = SORT_GMAX;
    if (g < 1) g = 1;
    return launch_coop(radix_sort_kernel<K>, (unsigned)g, RB, sort_smem<K>(), st, A);
}

// The tile size follows the capacity of the sort (the host does not know the
// band's size): small sorts take small tiles, so more CTAs share the work.
cudaError_t launch_radix_sort(SortArgs &A, double k, double t, cudaStream_t st) {
    (void)k;
    (void)t;
    if (A.cap <= SMALL_SORT) return launch_sort_k<RK_SMALL>(A, st);
    return launch_sort_k<RK_BIG>(A, st);
}

cudaError_t launch_locate(const SortArgs &A, double k, double t, cudaStream_t st) {
    static bool attr = false;
    const size_t smem = (size_t)LOC_KEY_WORDS * 4 + 16384;
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
