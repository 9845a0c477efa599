// k_radix.cu -- device-wide sort and locate-scan for rows too long for one
// CTA: the full-sort solver of "Fast LapSum: Exact Differentiable Top-k at
// Million Scale" (technical summary section 2.2) on a whole row (the fallback
// of the abstract, when certification fails) or on a band of the bracketing
// path (step 3) that exceeds the one-CTA capacity.
//
// Sort: keys-only LSD radix sort of the descending-order uint32 keys, 8-bit
// digits, reduce-then-scan per digit:
//   radix_hist_kernel     one read: all four digit histograms (per-thread run
//                         length combining, so long runs of tied scores cost
//                         one shared atomic per run), exclusive digit bases,
//                         and the digits on which every key agrees (those
//                         passes are skipped; all four: solved in closed form);
//   radix_count_kernel    per 8192-key tile, its 256 digit counts;
//   radix_scan_kernel     per digit, the counts of earlier tiles -> offsets;
//   radix_scatter_kernel  per tile, a stable in-tile ranking (per-warp digit
//                         histograms, __match_any_sync), a shared-memory
//                         scatter and coalesced runs of writes at the offsets.
// The count and scatter kernels stage each CTA's next tile in shared memory by
// one bulk copy while they work on the current one.  No CTA waits on another.
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
constexpr int LOC_KEY_WORDS = LTILE + LTILE / 32 + 8;   // padded tile + two halo entries

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
    auto count = [&](float x) {   // run-length combining per digit
        const uint32_t key = desc_key(x);
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
    };
    // each thread takes chunks of 16 consecutive scores (four 16-byte loads, so
    // runs of tied scores combine); the next chunk is loaded while this one is
    // counted (one copy of the counting code: a rotation, not an unrolled batch)
    const int64_t gstride = (int64_t)gridDim.x * HB;
    const int64_t nch = (reinterpret_cast<uintptr_t>(A.src) & 15u) == 0 ? n / 16 : 0;
    const float4 *src4 = reinterpret_cast<const float4 *>(A.src);
    auto load_chunk = [&](int64_t c, float4 (&v)[4]) {
#pragma unroll
        for (int q = 0; q < 4; ++q) v[q] = c < nch ? __ldg(src4 + c * 4 + q) : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    float4 cur4[4];
    int64_t c = (int64_t)blockIdx.x * HB + tid;
    load_chunk(c, cur4);
#pragma unroll 1
    for (; c < nch; c += gstride) {
        float4 nxt4[4];
        load_chunk(c + gstride, nxt4);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            count(cur4[q].x);
            count(cur4[q].y);
            count(cur4[q].z);
            count(cur4[q].w);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) cur4[q] = nxt4[q];
    }
    for (int64_t i = nch * 16 + (int64_t)blockIdx.x * HB + tid; i < n; i += gstride) count(__ldg(A.src + i));
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
// A pass (skipped when every key agrees on its digit) is reduce-then-scan:
//   radix_count_kernel    each tile's 256 digit counts -> cnt[d][tile]
//   radix_scan_kernel     per digit d, cnt[d][.] -> global offsets in place:
//                         dbase[d] + the count of d in all earlier tiles
//   radix_scatter_kernel  each tile ranks its keys stably in shared memory and
//                         writes every digit's run at the run's offset
// No CTA ever waits on another, so the pass has no spin waits at all; the
// price is one more read of the keys than a single-sweep sort.

// Row stride of the count table (a multiple of 4 entries, for 16-byte loads).
__host__ __device__ __forceinline__ int64_t cnt_stride(int64_t ntiles) { return (ntiles + 3) & ~int64_t(3); }

__device__ __forceinline__ const uint32_t *pass_keys_in(const SortArgs &A, int cur) {
    return cur < 0 ? nullptr : (cur == 0 ? A.keys[0] : A.keys[1]);
}

// The tile's keys, warp-striped (key i of lane l of warp w is tile element
// w*32*RK + i*32 + l), all RK loads in flight at once; keys past the end of the
// row read as 0xffffffff.  src == nullptr: the first pass, keys from the scores.
__device__ __forceinline__ void load_tile(const SortArgs &A, const uint32_t *src, int64_t base, int cnt_tile,
                                          uint32_t (&key)[RK]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int l0 = warp * 32 * RK + lane;
    if (src) {
#pragma unroll
        for (int i = 0; i < RK; ++i)
            key[i] = l0 + i * 32 < cnt_tile ? __ldcs(src + base + l0 + i * 32) : 0xffffffffu;
    } else {
        float x[RK];
#pragma unroll
        for (int i = 0; i < RK; ++i) x[i] = l0 + i * 32 < cnt_tile ? __ldg(A.src + base + l0 + i * 32) : 0.0f;
#pragma unroll
        for (int i = 0; i < RK; ++i) key[i] = l0 + i * 32 < cnt_tile ? desc_key(x[i]) : 0xffffffffu;
    }
}

// Double-buffered tile staging for the pass kernels: tiles are grid-strided, so
// each CTA knows its next tile and copies it (one bulk copy, completion counted
// on an mbarrier) while it works on the current one.  Only full tiles of a
// 16-byte-aligned source are staged; the rest take plain loads.
struct TileStage {
    uint32_t *buf;      // 2 * RTILE words
    uint64_t *bar;      // 2 mbarriers
    const char *gsrc;   // 4-byte elements: the keys, or the scores on the first pass
    bool bulk_ok;
    int64_t n;
};

__device__ __forceinline__ bool stage_full(const TileStage &S, int64_t tile) {
    return S.bulk_ok && (tile + 1) * RTILE <= S.n;
}

// thread 0; the buffer must be free (its last readers are past a barrier)
__device__ __forceinline__ void stage_issue(const TileStage &S, int slot, int64_t tile) {
    if (!stage_full(S, tile)) return;
    fence_proxy_async_smem();
    mbar_expect_tx(&S.bar[slot], RTILE * 4);
    bulk_load(S.buf + slot * RTILE, S.gsrc + (size_t)tile * RTILE * 4, RTILE * 4, &S.bar[slot]);
}

__device__ __forceinline__ void stage_init(TileStage &S, const SortArgs &A, const uint32_t *src, int64_t n,
                                           unsigned char *smem) {
    S.buf = reinterpret_cast<uint32_t *>(smem);
    S.bar = reinterpret_cast<uint64_t *>(smem + 2 * RTILE * 4);
    S.gsrc = src ? reinterpret_cast<const char *>(src) : reinterpret_cast<const char *>(A.src);
    S.bulk_ok = (reinterpret_cast<uintptr_t>(S.gsrc) & 15u) == 0;
    S.n = n;
    if (threadIdx.x == 0) {
        mbar_init(&S.bar[0], 1);
        mbar_init(&S.bar[1], 1);
        mbar_init_fence();
    }
    __syncthreads();
    if (threadIdx.x == 0 && (int64_t)blockIdx.x * RTILE < n) stage_issue(S, 0, blockIdx.x);
}

// The tile's keys into registers: from its staged copy (waiting, bounded, for
// the copy) or by plain loads.  Returns false when the wait gave up.
__device__ __forceinline__ bool stage_keys(const TileStage &S, const SortArgs &A, const uint32_t *src, int slot,
                                           uint32_t &ph, int64_t tile, int cnt_tile, uint32_t (&key)[RK]) {
    if (!stage_full(S, tile)) {
        load_tile(A, src, tile * RTILE, cnt_tile, key);
        return true;
    }
    const bool ok = mbar_wait(&S.bar[slot], (ph >> slot) & 1u, BULK_WAIT_CAP);
    ph ^= 1u << slot;
    const uint32_t *sb = S.buf + slot * RTILE;
    const int l0 = (threadIdx.x >> 5) * 32 * RK + (threadIdx.x & 31);
    if (src) {
#pragma unroll
        for (int i = 0; i < RK; ++i) key[i] = sb[l0 + i * 32];
    } else {
#pragma unroll
        for (int i = 0; i < RK; ++i) key[i] = desc_key(__uint_as_float(sb[l0 + i * 32]));
    }
    return ok;
}

constexpr size_t STAGE_BYTES = 2 * RTILE * 4 + 2 * sizeof(uint64_t);

// Adds this warp's digit counts of the tile to my_hist (the warp's 256 counters).
__device__ __forceinline__ void warp_count(const uint32_t (&key)[RK], int cnt_tile, int sh, uint32_t *my_hist) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int i = 0; i < RK; ++i) {
        const int li = warp * 32 * RK + i * 32 + lane;
        const bool v = li < cnt_tile;
        const uint32_t d = v ? ((key[i] >> sh) & 0xffu) : 0x100u;
        const unsigned peers = __match_any_sync(FULL, d);
        if (v && lane == __ffs(peers) - 1) my_hist[d] += __popc(peers);
        __syncwarp();
    }
}

// Common gate of the three pass kernels: the element count, or < 0 to return.
__device__ __forceinline__ int64_t pass_n(const SortArgs &A, int pass) {
    const int64_t n = gated_n(A);
    if (n < 0) return -1;
    if (A.ctl->sort_skip & (1 << pass)) return -1;   // every key agrees on this digit
    return n;
}

__global__ void __launch_bounds__(RB, 2) radix_count_kernel(SortArgs A, int pass) {
    extern __shared__ __align__(16) unsigned char smem[];
    uint32_t *s_hist = reinterpret_cast<uint32_t *>(smem + STAGE_BYTES);   // RNW * 256
    pdl_enter();
    const int64_t n = pass_n(A, pass);
    if (n < 0) return;
    const uint32_t *src = pass_keys_in(A, A.ctl->sort_cur);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int64_t ntiles = (n + RTILE - 1) / RTILE, nts = cnt_stride(ntiles);
    uint32_t *cnt = A.tilecnt;
    TileStage S;
    stage_init(S, A, src, n, smem);
    uint32_t ph = 0;
    bool ok = true;
    int slot = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, slot ^= 1) {
        if (tid == 0 && tile + gridDim.x < ntiles) stage_issue(S, slot ^ 1, tile + gridDim.x);
        const int cnt_tile = (int)min((int64_t)RTILE, n - tile * RTILE);
        uint32_t key[RK];
        ok &= stage_keys(S, A, src, slot, ph, tile, cnt_tile, key);
        for (int i = tid; i < RNW * 256; i += RB) s_hist[i] = 0;
        __syncthreads();
        warp_count(key, cnt_tile, 8 * pass, s_hist + warp * 256);
        __syncthreads();
        if (tid < 256) {
            uint32_t tot = 0;
#pragma unroll
            for (int w = 0; w < RNW; ++w) tot += s_hist[w * 256 + tid];
            cnt[(size_t)tid * nts + tile] = tot;
        }
        __syncthreads();   // sums read, staged keys read: both buffers may be reused
    }
    if (!ok) atomicOr(&A.ctl->status, ST_TIMEOUT);
}

constexpr int SB = 1024;   // scan: threads, one CTA per digit

__global__ void __launch_bounds__(SB) radix_scan_kernel(SortArgs A, int pass) {
    __shared__ uint32_t s_w[SB / 32];
    pdl_enter();
    const int64_t n = pass_n(A, pass);
    if (n < 0) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t ntiles = (n + RTILE - 1) / RTILE, nts = cnt_stride(ntiles);
    uint4 *row = reinterpret_cast<uint4 *>(A.tilecnt + (size_t)blockIdx.x * nts);
    uint32_t carry = A.dbase[pass * 256 + blockIdx.x];
    const int64_t nv = nts / 4;   // 16-byte vectors of the row (entries past ntiles are never read)
    for (int64_t v0 = 0; v0 < nv; v0 += SB) {
        const int64_t vi = v0 + tid;
        uint4 x = make_uint4(0u, 0u, 0u, 0u);
        if (vi < nv) x = row[vi];
        const uint32_t t4 = x.x + x.y + x.z + x.w;
        uint32_t inc = t4;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(FULL, inc, o);
            if (lane >= o) inc += y;
        }
        if (lane == 31) s_w[warp] = inc;
        __syncthreads();
        uint32_t wofs = 0, total = 0;
#pragma unroll
        for (int w = 0; w < SB / 32; ++w) {
            const uint32_t c = s_w[w];
            wofs += w < warp ? c : 0u;
            total += c;
        }
        __syncthreads();   // s_w is rewritten by the next chunk
        if (vi < nv) {
            uint32_t e = carry + wofs + inc - t4;
            uint4 o;
            o.x = e; e += x.x;
            o.y = e; e += x.y;
            o.z = e; e += x.z;
            o.w = e;
            row[vi] = o;
        }
        carry += total;
    }
}

__global__ void __launch_bounds__(RB, 2) radix_scatter_kernel(SortArgs A, int pass) {
    extern __shared__ __align__(16) unsigned char smem[];
    uint32_t *s_hist = reinterpret_cast<uint32_t *>(smem + STAGE_BYTES);   // RNW * 256
    uint32_t *s_dstart = s_hist + RNW * 256;                           // 256: in-tile digit start
    uint32_t *s_gofs = s_dstart + 256;                                 // 256: global offset - dstart
    __shared__ bool s_last;
    pdl_enter();
    const int64_t n = pass_n(A, pass);
    if (n < 0) return;
    Ctl *ctl = A.ctl;
    const int cur = ctl->sort_cur;
    const uint32_t *src = pass_keys_in(A, cur);
    uint32_t *dst = cur == 0 ? A.keys[1] : A.keys[0];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int sh = 8 * pass;
    const int64_t ntiles = (n + RTILE - 1) / RTILE, nts = cnt_stride(ntiles);
    const uint32_t *ofs = A.tilecnt;
    const unsigned lt_mask = (1u << lane) - 1u;
    TileStage S;
    stage_init(S, A, src, n, smem);
    uint32_t ph = 0;
    bool ok = true;
    int slot = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, slot ^= 1) {
        if (tid == 0 && tile + gridDim.x < ntiles) stage_issue(S, slot ^ 1, tile + gridDim.x);
        const int cnt_tile = (int)min((int64_t)RTILE, n - tile * RTILE);
        uint32_t key[RK];
        ok &= stage_keys(S, A, src, slot, ph, tile, cnt_tile, key);
        // this tile's buffer becomes its scatter buffer once every key is in registers
        uint32_t *s_keys = S.buf + slot * RTILE;
        for (int i = tid; i < RNW * 256; i += RB) s_hist[i] = 0;
        __syncthreads();
        uint32_t *my_hist = s_hist + warp * 256;
        warp_count(key, cnt_tile, sh, my_hist);
        __syncthreads();
        if (tid < 256) {   // per digit: exclusive offsets of the warps, tile total
            uint32_t tot = 0;
#pragma unroll
            for (int w = 0; w < RNW; ++w) {
                const uint32_t c = s_hist[w * 256 + tid];
                s_hist[w * 256 + tid] = tot;
                tot += c;
            }
            s_dstart[tid] = tot;
            s_gofs[tid] = __ldg(ofs + (size_t)tid * nts + tile);
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
        // runs of one digit are consecutive in s_keys and in dst: coalesced writes
        for (int i = tid; i < cnt_tile; i += RB) {
            const uint32_t kk = s_keys[i];
            dst[(uint32_t)(s_gofs[(kk >> sh) & 0xffu] + (uint32_t)i)] = kk;
        }
        __syncthreads();
    }
    if (!ok) atomicOr(&ctl->status, ST_TIMEOUT);
    // the last CTA to finish publishes the new key buffer
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&ctl->ticket[5], 1u) == gridDim.x - 1;
    __syncthreads();
    if (s_last && tid == 0) {
        ctl->sort_cur = cur >= 0 ? (cur ^ 1) : 0;
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

cudaError_t launch_radix_sort(SortArgs &A, double k, double t, cudaStream_t st) {
    (void)k;
    (void)t;
    const int64_t cap = A.cap;
    static bool attr = false;
    const size_t smem_c = STAGE_BYTES + (size_t)RNW * 256 * 4;
    const size_t smem = STAGE_BYTES + (size_t)RNW * 256 * 4 + 2 * 256 * 4;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(radix_count_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_c);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(radix_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    int64_t hg = (cap + HB * 32 - 1) / (HB * 32);
    if (hg > (int64_t)num_sms() * 4) hg = (int64_t)num_sms() * 4;
    int hgrid = (int)hg;
    if (hgrid < 1) hgrid = 1;
    cudaError_t e = launch_k(radix_hist_kernel, hgrid, HB, 0, st, A);
    if (e != cudaSuccess) return e;
    int64_t pt = (cap + RTILE - 1) / RTILE;
    if (pt > 2 * num_sms()) pt = 2 * num_sms();   // two CTAs per SM, tiles grid-strided
    const unsigned ptiles = (unsigned)pt;
    for (int pass = 0; pass < 4; ++pass) {
        e = launch_k(radix_count_kernel, ptiles, RB, smem_c, st, A, pass);
        if (e == cudaSuccess) e = launch_k(radix_scan_kernel, 256u, SB, 0, st, A, pass);
        if (e == cudaSuccess) e = launch_k(radix_scatter_kernel, ptiles, RB, smem, st, A, pass);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
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
