// k_radix.cu -- device-wide sort and locate-scan for rows too long for one
// CTA: the full-sort solver of "Fast LapSum: Exact Differentiable Top-k at
// Million Scale" (technical summary section 2.2) on a whole row: the full-sort
// path for long rows, and the fallback of the abstract when certification fails.
//
// Sort: keys-only LSD radix sort of the descending-order uint32 keys, 8-bit
// digits, in one cooperative kernel (radix_sort_kernel, described below).
// Locate (the same kernel, after the last pass): tile and chunk maps of the
// prefix/suffix scans, then one CTA narrows the crossing down chunk -> tile ->
// value and takes the closed-form root.
//
// The host never learns the certification verdict: the fallback sort reads its
// gate from each row's control block and skips the rows with nothing to do.
#include <climits>
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



// The two words after the four global digit histograms: a count of sorts that
// gave up (possibly leaving partial counts in the histograms), and the count at
// the last clean-up.  They differ while the histograms need clearing.
__device__ __forceinline__ unsigned long long *A_hist_dirty(const SortArgs &A) { return A.hist + 4 * 256; }
__device__ __forceinline__ unsigned long long *A_hist_cleaned(const SortArgs &A) { return A.hist + 4 * 256 + 1; }
// Four more words: for each sign class of the keys (negative scores, then the
// rest), the OR of the keys and the OR of their complements -- the bits that
// vary within the class are the AND of the two.  A digit whose bits vary within
// neither class is decided by the sign, so its pass changes no order among keys
// that tie on the higher digits: it is skipped like a constant digit.  (Scores
// quantised to a few mantissa bits -- tied levels -- skip two of four passes.)
__device__ __forceinline__ unsigned long long *A_sign_bits(const SortArgs &A) { return A.hist + 4 * 256 + 2; }
__device__ __forceinline__ unsigned long long ld_volatile_u64(const unsigned long long *p) {
    return *reinterpret_cast<const volatile unsigned long long *>(p);
}

// Element count behind a gate; < 0 means "nothing to do".
__device__ __forceinline__ int64_t gated_n(const SortArgs &A) {
    if (A.gate == GATE_FALLBACK && A.ctl->verdict != 0) return -1;
    return A.n_host;
}

// n copies of one value c (a row whose scores are all equal): closed form.
__device__ void solve_equal_run(const SortArgs &A, int64_t n) {
    Ctl *ctl = A.ctl;
    bool above = false;
    ctl->b = solve_equal_run_values((double)A.src[0], (double)n, 0.0, CUDART_INF, 0.0, -CUDART_INF, 0.0, A.k,
                                    A.t, &above);
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
// Counts need no order: a warp whose keys all share the digit (sorted or tied
// scores) adds them at once, any other warp takes one shared atomic per key.
// WHOLE: first test the warp's keys together (one vote for all K of them; the
// count walks, where no ranking state competes for registers).
template <int K, bool WHOLE>
__device__ __forceinline__ void warp_count(const uint32_t (&key)[K], int cnt_tile, int sh, uint32_t *my_hist) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (WHOLE) {   // every key of the warp on the digit of its first key (lane 0's key 0): one add
        const uint32_t d0 = __shfl_sync(FULL, (key[0] >> sh) & 0xffu, 0);
        bool same = true;
        uint32_t nv = 0;
#pragma unroll
        for (int i = 0; i < K; ++i) {
            const bool v = warp * 32 * K + i * 32 + lane < cnt_tile;
            same &= !v || ((key[i] >> sh) & 0xffu) == d0;
            nv += v;
        }
        if (__all_sync(FULL, same)) {
            nv = __reduce_add_sync(FULL, nv);   // 0: the warp lies past the end of the tile
            if (lane == 0 && nv) my_hist[d0] += nv;
            __syncwarp();
            return;
        }
    }
#pragma unroll
    for (int i = 0; i < K; ++i) {
        const int li = warp * 32 * K + i * 32 + lane;
        const bool v = li < cnt_tile;
        const uint32_t d = v ? ((key[i] >> sh) & 0xffu) : 0x100u;
        if (__all_sync(FULL, d == __shfl_sync(FULL, d, 0))) {
            if (lane == 0 && d < 0x100u) my_hist[d] += 32u;
        } else if (v) {
            atomicAdd(&my_hist[d], 1u);
        }
    }
    __syncwarp();
}

// Walks the CTA's chunk of tiles in order with one tile staged ahead, calling
// body(tile, cnt_tile, key) with every thread's keys; a barrier follows each
// body, so the staging buffers are free again.  Returns false if a wait gave up
// (in any thread): ST_TIMEOUT is set, no further copy is issued, the copies in
// flight are waited for (bounded), and the caller must return.
template <int K, typename Body>
__device__ __forceinline__ bool walk_chunk(TileStage<K> &S, const SortArgs &A, const uint32_t *src, int64_t t0,
                                           int64_t t1, uint32_t &ph, Body &&body) {
    stage_source(S, A, src);
    if (threadIdx.x == 0 && t0 < t1) stage_issue(S, 0, t0);
    int slot = 0;
    for (int64_t tile = t0; tile < t1; ++tile, slot ^= 1) {
        if (threadIdx.x == 0 && tile + 1 < t1) stage_issue(S, slot ^ 1, tile + 1);
        const int cnt_tile = (int)min((int64_t)TILE_K(K), S.n - tile * TILE_K(K));
        uint32_t key[K];
        const bool ok = stage_keys(S, A, src, slot, ph, tile, cnt_tile, key);
        body(tile, cnt_tile, key, S.buf + slot * TILE_K(K));
        if (!__syncthreads_and(ok)) {
            if (threadIdx.x == 0) {
                atomicOr(&A.ctl->status, ST_TIMEOUT);
                // this tile's copy (its phase bit already flipped) and the next one's
                if (stage_full(S, tile)) mbar_wait(&S.bar[slot], ((ph >> slot) & 1u) ^ 1u, BULK_WAIT_CAP);
                if (tile + 1 < t1 && stage_full(S, tile + 1))
                    mbar_wait(&S.bar[slot ^ 1], (ph >> (slot ^ 1)) & 1u, BULK_WAIT_CAP);
            }
            __syncthreads();
            return false;
        }
    }
    return true;
}

// ------------------------------------------------------------ locate --
// After the last pass the sorted values c_0 >= c_1 >= ... sit in one key buffer.
// The threshold curve is evaluated by affine scans (prefix P_j = 1 + d_{j-1}
// P_{j-1}, suffix Q_j = 1 + d_j Q_{j+1}, links d_j = e^{(c_{j+1} - c_j)/t}):
//   1. every CTA reduces each tile of its chunk to its two maps (a tile record)
//      and composes them into its chunk's maps (a chunk record);   barrier;
//   2. CTA 0 scans the chunk maps and finds the chunk whose end first has
//      G > k -- the crossing is in it (or below the last value);
//   3. CTA 0 scans that chunk's tile maps and finds the crossing tile;
//   4. CTA 0 re-scans that tile element by element and takes the closed-form
//      root (block_scan_solve).
struct TileRec {
    double pa, ps;     // tile prefix map  P_end = pa * P_before + ps
    double qa, qs;     // tile suffix map  Q_first = qa * Q_after + qs
    double d_out;      // link from the tile's last value to the next value
    double p_end;      // filled by CTA 0 for the tiles of the crossing chunk
    double q_after;
    double pad;
};
struct ChunkRec {
    double pa, ps, qa, qs;   // the chunk's composed maps (identity when it has no tile)
    double d_out;            // link out of the chunk's last value
    double last;             // index of the chunk's last value, -1 when it has no tile
    double pad[2];
};

struct Seeds {   // what lies above and below the sorted values
    double m0, top, P_top, bot, Q_bot;
};
__device__ __forceinline__ Seeds locate_seeds(const SortArgs &) {
    return Seeds{0.0, CUDART_INF, 0.0, -CUDART_INF, 0.0};   // a whole row: nothing above or below
}

// Step 1 for one CTA: its tiles' records and its chunk record.  The tiles are
// staged in shared memory one ahead (bulk copies into the sort's two tile
// buffers; plain loads for a ragged or unaligned tile), and each thread maps
// its K consecutive values.  A tile's suffix map needs the link out of its last
// value, which the next tile supplies (its first value's link in): the map is
// kept up to that link and completed one tile later (the chunk's last tile
// from one load after the walk), so no tile waits on a value beyond it.
// Returns false when a copy wait gave up (ST_TIMEOUT set, copies in flight
// awaited); the caller must return.
template <int K>
__device__ bool locate_tiles(const SortArgs &A, TileStage<K> &S, uint32_t &ph, const uint32_t *sorted, int64_t n,
                             int64_t t0, int64_t t1, const Seeds &z, TileRec *rec, ChunkRec *crec, Aff *sc,
                             const double *tab) {
    constexpr int TILE = TILE_K(K);
    constexpr int NW = RB / 32;
    static_assert(K % 4 == 0, "a thread reads its values as uint4");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const double s2d = (1.0 / A.t) * LOG2E;
    __shared__ float s_last;              // the last value of the tile just mapped
    __shared__ float s_wend[2][NW];       // each warp's first and last value
    // link between neighbours hi >= lo: e^{-(hi - lo)/t}; 0 against an infinite end
    auto link = [&](double hi, double lo) -> double {
        return (hi == CUDART_INF || lo == -CUDART_INF) ? 0.0 : link_exp((hi - lo) * s2d, tab);
    };
    Aff Pc = aff_id(), Qc = aff_id(), Qprev = aff_id();   // thread 0: chunk maps, last tile's partial Q map
    double vprev = 0.0;                                    // thread 0: the value before the tile
    if (tid == 0) vprev = t0 == 0 ? z.top : (double)desc_key_to_float(__ldcg(sorted + t0 * TILE - 1));
    stage_source(S, A, sorted);
    if (tid == 0 && t0 < t1) stage_issue(S, 0, t0);
    int slot = 0;
    for (int64_t tile = t0; tile < t1; ++tile, slot ^= 1) {
        if (tid == 0 && tile + 1 < t1) stage_issue(S, slot ^ 1, tile + 1);
        const int64_t base = tile * TILE;
        const int cnt = (int)min((int64_t)TILE, n - base);
        const int l0 = tid * K;
        const int nk = max(0, min(K, cnt - l0));   // this thread's values
        float c[K];   // this thread's values (fp32 scores; links are formed in fp64)
        bool ok = true;
        if (stage_full(S, tile)) {
            ok = mbar_wait(&S.bar[slot], (ph >> slot) & 1u, BULK_WAIT_CAP);
            ph ^= 1u << slot;
            const uint4 *q = reinterpret_cast<const uint4 *>(S.buf + slot * TILE + l0);
#pragma unroll
            for (int v = 0; v < K / 4; ++v) {
                const uint4 w = q[v];
                c[4 * v + 0] = desc_key_to_float(w.x);
                c[4 * v + 1] = desc_key_to_float(w.y);
                c[4 * v + 2] = desc_key_to_float(w.z);
                c[4 * v + 3] = desc_key_to_float(w.w);
            }
        } else {
#pragma unroll
            for (int u = 0; u < K; ++u) c[u] = u < nk ? desc_key_to_float(__ldcg(sorted + base + l0 + u)) : 0.0f;
        }
        float clast = c[0];
#pragma unroll
        for (int u = 1; u < K; ++u) clast = u < nk ? c[u] : clast;
        if (lane == 0) s_wend[0][warp] = c[0];
        if (lane == 31) s_wend[1][warp] = clast;
        if (!__syncthreads_and(ok)) {
            if (tid == 0) {
                atomicOr(&A.ctl->status, ST_TIMEOUT);
                if (stage_full(S, tile)) mbar_wait(&S.bar[slot], ((ph >> slot) & 1u) ^ 1u, BULK_WAIT_CAP);
                if (tile + 1 < t1 && stage_full(S, tile + 1))
                    mbar_wait(&S.bar[slot ^ 1], (ph >> (slot ^ 1)) & 1u, BULK_WAIT_CAP);
            }
            __syncthreads();
            return false;
        }
        // the values either side of this thread's run
        const float up = __shfl_up_sync(FULL, clast, 1), dn = __shfl_down_sync(FULL, c[0], 1);
        const double before = tid == 0 ? vprev : (double)(lane > 0 ? up : s_wend[1][warp - 1]);
        const float after = lane < 31 ? dn : (warp < NW - 1 ? s_wend[0][warp + 1] : 0.0f);
        // P: x -> 1 + d x over the run in order, d the link into each value; Q:
        // x -> 1 + d x right to left, d the link out of each value, the tile's last
        // value taking d = 1 (its link out is applied later)
        const double din = link(before, (double)c[0]);   // into the run's first value
        Aff mp = aff_id(), mq = aff_id();
        bool flat = nk > 0;   // every value of the run equal (tied scores): every inner link is 1
                              // (a non-finite row is reported, not solved)
#pragma unroll
        for (int u = 1; u < K; ++u) flat &= u >= nk || c[u] == c[0];
        if (flat) {   // P_end = nk + din P_before, Q_first = nk + dout Q_after
            const double dout = l0 + nk < cnt ? link((double)clast, (double)after) : 1.0;
            mp = {din, (double)nk};
            mq = {dout, (double)nk};
        } else {
            double dcur = din;
#pragma unroll
            for (int u = 0; u < K; ++u) {
                if (u < nk) {
                    mp = {mp.a * dcur, fma(mp.s, dcur, 1.0)};
                    const double dnext = u + 1 < nk ? link((double)c[u], (double)c[(u + 1) % K])
                                                    : (l0 + nk < cnt ? link((double)c[u], (double)after) : 1.0);
                    mq = {mq.a * dnext, mq.s + mq.a};
                    dcur = dnext;
                }
            }
        }
        // the tile's two maps: a tree over the warp's lanes (P in thread order, Q the
        // other way round), then thread 0 over the warps
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const Aff pp = shfl_down_aff(mp, o), pq = shfl_down_aff(mq, o);
            if (lane + o < 32) {   // lane l (a multiple of 2o) takes lanes l + o .. l + 2o - 1
                mp = aff_then(mp, pp);
                mq = aff_then(pq, mq);
            }
        }
        if (lane == 0) {
            sc[warp] = mp;
            sc[NW + warp] = mq;
        }
        if (tid == (cnt - 1) / K) s_last = clast;   // the tile's last value is this thread's
        __syncthreads();
        if (tid == 0) {
            Aff P = sc[0], Q = sc[NW];
            for (int w = 1; w < NW; ++w) {
                P = aff_then(P, sc[w]);
                Q = aff_then(sc[NW + w], Q);
            }
            rec[tile].pa = P.a;
            rec[tile].ps = P.s;
            if (tile > t0) {   // the link into this tile completes the previous tile's Q map
                const Aff Qf = {Qprev.a * din, Qprev.s};
                rec[tile - 1].qa = Qf.a;
                rec[tile - 1].qs = Qf.s;
                rec[tile - 1].d_out = din;
                Qc = aff_then(Qf, Qc);
            }
            Pc = aff_then(Pc, P);
            Qprev = Q;
            vprev = s_last;
        }
        __syncthreads();   // the stage buffer and the scratch are reused by the next tile
    }
    if (tid == 0) {
        double dc = 0.0;
        if (t1 > t0) {   // the chunk's last tile: its link out, to the value after the chunk
            const int64_t e = min(t1 * TILE, n);
            const double vnext = e >= n ? z.bot : (double)desc_key_to_float(__ldcg(sorted + e));
            dc = link(vprev, vnext);
            const Aff Qf = {Qprev.a * dc, Qprev.s};
            rec[t1 - 1].qa = Qf.a;
            rec[t1 - 1].qs = Qf.s;
            rec[t1 - 1].d_out = dc;
            Qc = aff_then(Qf, Qc);
        }
        ChunkRec r;
        r.pa = Pc.a;
        r.ps = Pc.s;
        r.qa = Qc.a;
        r.qs = Qc.s;
        r.d_out = dc;
        r.last = t1 > t0 ? (double)(min(t1 * TILE, n) - 1) : -1.0;
        r.pad[0] = r.pad[1] = 0.0;
        crec[blockIdx.x] = r;
    }
    return true;
}

// max (or min, with neg = true) of one int over the CTA
__device__ __forceinline__ int block_max_int(int v, int *s_w) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(FULL, v, o));
    if (lane == 0) s_w[warp] = v;
    __syncthreads();
    int m = s_w[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = max(m, s_w[w]);
    __syncthreads();
    return m;
}

// Steps 2-4, CTA 0 alone, after the barrier that follows step 1.
template <int K>
__device__ void locate_finish(const SortArgs &A, const uint32_t *sorted, int64_t n, const Seeds &z, TileRec *rec,
                              const ChunkRec *crec, uint32_t *s_t, void *scratch, const double *tab) {
    constexpr int TILE = TILE_K(K);
    const int tid = threadIdx.x;
    const int G = gridDim.x;
    const int64_t ntiles = (n + TILE - 1) / TILE;
    Ctl *ctl = A.ctl;
    Aff *sc = reinterpret_cast<Aff *>(scratch);
    __shared__ int s_w[RB / 32];
    __shared__ double s_d[2];
    // ---- step 2: the chunk maps (G <= RB chunks: one scan)
    Aff mP = aff_id(), mQ = aff_id();
    double dO = 0.0, last = -1.0;
    if (tid < G) {
        const ChunkRec *r = crec + tid;
        mP = {__ldcg(&r->pa), __ldcg(&r->ps)};
        mQ = {__ldcg(&r->qa), __ldcg(&r->qs)};
        dO = __ldcg(&r->d_out);
        last = __ldcg(&r->last);
    }
    Aff pe, qe;
    block_scan_excl_both<RB>(mP, mQ, pe, qe, sc);
    const double Pb = fma(pe.a, z.P_top, pe.s);   // P before the chunk's first value
    const double Qa = fma(qe.a, z.Q_bot, qe.s);   // Q after the chunk's last value
    const bool full = tid < G && last >= 0.0;
    int cand = -1;
    if (full) {
        const double Pend = fma(mP.a, Pb, mP.s);
        const double Gend = (z.m0 + last + 1.0) - 0.5 * Pend + 0.5 * dO * Qa;
        if (Gend <= A.k) cand = tid;
    }
    const int cstar = block_max_int(cand, s_w);
    // the crossing chunk: the first chunk with tiles after cstar, else the last one with tiles
    const int nxt = -block_max_int(full && tid > cstar ? -tid : INT_MIN + 1, s_w);
    const int lastfull = block_max_int(full ? tid : -1, s_w);
    const int tgt = (nxt != INT_MAX) ? nxt : lastfull;
    if (tid == tgt) {
        s_d[0] = Pb;
        s_d[1] = Qa;
    }
    __syncthreads();
    const double Pin = s_d[0], Qout = s_d[1];
    const int64_t T0 = (int64_t)tgt * ntiles / G, T1 = (int64_t)(tgt + 1) * ntiles / G;
    // ---- step 3: the tiles of that chunk (forward P, backward Q, RB tiles at a time)
    __shared__ double s_carry;
    double carry_p = Pin;
    for (int64_t c0 = T0; c0 < T1; c0 += RB) {
        const int64_t T = c0 + tid;
        Aff m = aff_id();
        if (T < T1) m = {__ldcg(&rec[T].pa), __ldcg(&rec[T].ps)};
        Aff p2, q2;
        block_scan_excl_both<RB>(m, aff_id(), p2, q2, sc);
        const Aff inc = aff_then(p2, m);
        if (T < T1) rec[T].p_end = fma(inc.a, carry_p, inc.s);
        const int64_t lastT = min(c0 + RB, T1) - 1;
        if (T == lastT) s_carry = fma(inc.a, carry_p, inc.s);
        __syncthreads();
        carry_p = s_carry;
        __syncthreads();
    }
    double carry_q = Qout;
    int best = -1;   // last tile (offset from T0) with G <= k at its end
    const int64_t nck = (T1 - T0 + RB - 1) / RB;
    for (int64_t ci = nck - 1; ci >= 0; --ci) {
        const int64_t c0 = T0 + ci * RB;
        const int64_t T = c0 + tid;
        Aff m = aff_id();
        if (T < T1) m = {__ldcg(&rec[T].qa), __ldcg(&rec[T].qs)};
        Aff p2, q2;
        block_scan_excl_both<RB>(aff_id(), m, p2, q2, sc);
        const double Qa_t = fma(q2.a, carry_q, q2.s);   // Q after tile T
        if (T < T1) {
            rec[T].q_after = Qa_t;
            const int64_t tend = min((T + 1) * TILE, n) - 1;
            const double Gt = (z.m0 + (double)(tend + 1)) - 0.5 * rec[T].p_end + 0.5 * __ldcg(&rec[T].d_out) * Qa_t;
            if (Gt <= A.k) best = max(best, (int)(T - T0));
        }
        if (tid == 0) {
            const Aff all = aff_then(q2, m);
            s_carry = fma(all.a, carry_q, all.s);
        }
        __syncthreads();
        carry_q = s_carry;
        __syncthreads();
    }
    best = block_max_int(best, s_w);
    const int64_t TT = min(T0 + best + 1, T1 - 1);
    // ---- step 4: the crossing tile, element by element
    const int64_t t0v = TT * TILE;
    const int cnt = (int)min((int64_t)TILE, n - t0v);
    for (int i = tid; i < cnt; i += RB) s_t[spad(i)] = __ldcg(sorted + t0v + i);
    __syncthreads();
    const double ptop = TT == T0 ? Pin : rec[TT - 1].p_end;
    const double qbot = rec[TT].q_after;
    const double vtop = t0v == 0 ? z.top : (double)desc_key_to_float(__ldcg(sorted + t0v - 1));
    const double vbot = t0v + cnt >= n ? z.bot : (double)desc_key_to_float(__ldcg(sorted + t0v + cnt));
    int64_t js = 0;
    const double b = block_scan_solve<RB, K>(s_t, cnt, A.k, A.t, 1.0 / A.t, z.m0 + (double)t0v, vtop, ptop, vbot,
                                             qbot, scratch, &js, &ctl->status, tab);
    if (tid == 0) {
        ctl->b = b;
        ctl->j_star = t0v + js;
        if (A.gate == GATE_FALLBACK) ctl->fallback_ran = 1;
    }
}

template <int K>
constexpr size_t sort_smem() { return stage_bytes<K>() + (size_t)(RNW * 256 + 4 * 256 + 4 * 256) * 4; }
constexpr int SORT_GMAX = 320;   // CTAs of the sort grid at most (chunk counts per digit)

template <int K>
__global__ void __launch_bounds__(RB, 2) radix_sort_kernel(SortArgs Ag) {
    extern __shared__ __align__(16) unsigned char smem[];
    uint32_t *s_hist = reinterpret_cast<uint32_t *>(smem + stage_bytes<K>());   // RNW * 256: per-warp digit counts
    uint32_t *s_dstart = s_hist + RNW * 256;   // 256: in-tile digit start
    uint32_t *s_gofs = s_dstart + 256;         // 256: global offset - in-tile start
    uint32_t *s_run = s_gofs + 256;            // 256: running global offset of each digit
    uint32_t *s_tot = s_run + 256;             // 256: scratch (tile totals)
    uint32_t *s_h4 = s_tot + 256;              // 4 * 256: phase-H histograms, then digit bases
    __shared__ int s_skip;
    __shared__ uint32_t s_d0;   // a scatter tile's first digit
    __shared__ double s_tab[32];
    pdl_wait();
    {   // every row's gate closed (the certification passed everywhere): nothing to do,
        // and nothing else is touched (a clean-up owed by an earlier give-up waits for
        // the next launch that sorts)
        bool open = false;
        for (int64_t r = threadIdx.x; r < Ag.rows; r += RB) {
            SortArgs A = Ag;
            A.ctl = Ag.ctl + r;
            open |= gated_n(A) >= 0;
        }
        if (!__syncthreads_or(open)) {
            pdl_trigger();
            return;
        }
    }
    exp2_table_init(s_tab);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = gridDim.x, c = blockIdx.x;
    TileStage<K> S;
    S.buf = reinterpret_cast<uint32_t *>(smem);
    S.bar = reinterpret_cast<uint64_t *>(smem + 2 * TILE_K(K) * 4);
    if (tid == 0) {
        mbar_init(&S.bar[0], 1);
        mbar_init(&S.bar[1], 1);
        mbar_init_fence();
    }
    __syncthreads();
    // A sort that gave up on an earlier launch may have left partial counts in the
    // global digit histograms (the word after them says so; every CTA reads it
    // before any count is added, so all take the same branch): clear them first.
    const unsigned long long gave_up = ld_volatile_u64(A_hist_dirty(Ag));
    if (gave_up != ld_volatile_u64(A_hist_cleaned(Ag))) {
        if (c == 0) {
            for (int i = tid; i < 4 * 256; i += RB) Ag.hist[i] = 0ull;
            if (tid < 4) A_sign_bits(Ag)[tid] = 0ull;
        }
        if (!grid_sync(&Ag.ctl->gbar_count, &Ag.ctl->gbar_gen, Ag.spin_cap, &Ag.ctl->status)) {
            if (tid == 0) atomicAdd(A_hist_dirty(Ag), 1ull);
            return;
        }
        if (c == 0 && tid == 0) *A_hist_cleaned(Ag) = gave_up;   // a give-up later in this launch counts again
    }
    uint32_t ph = 0;   // mbarrier phases, carried from row to row
    // the rows of a batch, one after another (each gated by its own control block)
    // The gates of a block of RB rows are read together (one thread per row) and
    // the open rows listed in row order -- the same list in every CTA.
    __shared__ int s_open[RB];
    __shared__ int s_wopen[RNW];
    for (int64_t r0 = 0; r0 < Ag.rows; r0 += RB) {
        int nopen = 0;
        {
            bool open = false;
            if (r0 + tid < Ag.rows) {
                SortArgs A = Ag;
                A.ctl = Ag.ctl + r0 + tid;
                open = gated_n(A) >= 0;
            }
            const unsigned m = __ballot_sync(FULL, open);
            if (lane == 0) s_wopen[warp] = __popc(m);
            __syncthreads();
            int before = 0;
            for (int w = 0; w < RNW; ++w) {
                before += w < warp ? s_wopen[w] : 0;
                nopen += s_wopen[w];
            }
            if (open) s_open[before + __popc(m & ((1u << lane) - 1u))] = tid;
            __syncthreads();
        }
        for (int oi = 0; oi < nopen; ++oi) {
            const int64_t row = r0 + s_open[oi];
            SortArgs A = Ag;
            A.src = Ag.src + row * Ag.src_stride;
            A.ctl = Ag.ctl + row;
            const int64_t n = gated_n(A);
            Ctl *ctl = A.ctl;
            const int64_t ntiles = (n + TILE_K(K) - 1) / TILE_K(K);
            const int64_t t0 = (int64_t)c * ntiles / G, t1 = (int64_t)(c + 1) * ntiles / G;
            uint32_t *csum = A.chunkcnt;   // [4][256][G]
            // a barrier or copy wait that gives up ends the kernel for this CTA (every
            // CTA then leaves at its next barrier, each wait bounded)
            auto bar = [&]() -> bool {
                const bool ok = grid_sync(&ctl->gbar_count, &ctl->gbar_gen, A.spin_cap, &ctl->status);
                if (!ok && tid == 0) atomicAdd(A_hist_dirty(A), 1ull);
                return ok;
            };
            S.n = n;
            for (int i = tid; i < 4 * 256; i += RB) s_h4[i] = 0;
            __syncthreads();

            // ---- phase H: the chunk's four digit histograms
            {
                uint32_t cur[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
                uint32_t cnt[4] = {0, 0, 0, 0};
                uint32_t sor[2] = {0u, 0u}, snot[2] = {0u, 0u};   // per sign class: OR of keys, of ~keys
                const bool walked = walk_chunk(S, A, nullptr, t0, t1, ph, [&](int64_t, int cnt_tile, const uint32_t (&key)[K], uint32_t *) {
                    const int l0 = warp * 32 * K + lane;
                    {   // the warp's keys all equal to its first (tied scores in order): one add per digit
                        const uint32_t k0 = __shfl_sync(FULL, key[0], 0);
                        bool same = true;
                        uint32_t nv = 0;
#pragma unroll
                        for (int i = 0; i < K; ++i) {
                            const bool v = l0 + i * 32 < cnt_tile;
                            same &= !v || key[i] == k0;
                            nv += v;
                        }
                        if (__all_sync(FULL, same)) {
                            nv = __reduce_add_sync(FULL, nv);   // 0: the warp lies past the end of the tile
                            if (lane == 0 && nv) {
#pragma unroll
                                for (int d = 0; d < 4; ++d) atomicAdd(&s_h4[d * 256 + ((k0 >> (8 * d)) & 0xffu)], nv);
                                const bool ng = k0 >> 31;
                                sor[0] |= ng ? 0u : k0;
                                snot[0] |= ng ? 0u : ~k0;
                                sor[1] |= ng ? k0 : 0u;
                                snot[1] |= ng ? ~k0 : 0u;
                            }
                            return;
                        }
                    }
#pragma unroll
                    for (int i = 0; i < K; ++i) {
                        if (l0 + i * 32 >= cnt_tile) break;
                        const bool ng = key[i] >> 31;
                        sor[0] |= ng ? 0u : key[i];
                        snot[0] |= ng ? 0u : ~key[i];
                        sor[1] |= ng ? key[i] : 0u;
                        snot[1] |= ng ? ~key[i] : 0u;
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
                if (!walked) {
                    if (tid == 0) atomicAdd(A_hist_dirty(A), 1ull);
                    return;
                }
#pragma unroll
                for (int d = 0; d < 4; ++d)
                    if (cnt[d]) atomicAdd(&s_h4[d * 256 + cur[d]], cnt[d]);
#pragma unroll
                for (int q = 0; q < 2; ++q) {   // the CTA's varying bits per sign class, then the grid's
                    sor[q] = __reduce_or_sync(FULL, sor[q]);
                    snot[q] = __reduce_or_sync(FULL, snot[q]);
                    if (lane == 0 && (sor[q] | snot[q])) {
                        atomicOr(reinterpret_cast<unsigned long long *>(A_sign_bits(A) + 2 * q), (unsigned long long)sor[q]);
                        atomicOr(reinterpret_cast<unsigned long long *>(A_sign_bits(A) + 2 * q + 1),
                                 (unsigned long long)snot[q]);
                    }
                }
                __syncthreads();
                for (int i = tid; i < 4 * 256; i += RB) {
                    const uint32_t v = s_h4[i];
                    csum[(size_t)i * G + c] = v;
                    if (v) atomicAdd(A.hist + i, (unsigned long long)v);
                }
            }
            if (!bar()) return;
            // digit bases and skip flags, the same in every CTA (thread d owns bin d)
            if (tid == 0) {
                const unsigned long long *sb = A_sign_bits(A);
                const uint32_t vary = (uint32_t)(__ldcg(sb) & __ldcg(sb + 1)) | (uint32_t)(__ldcg(sb + 2) & __ldcg(sb + 3));
                int sk = 0;
                for (int d4 = 0; d4 < 3; ++d4)   // the top digit holds the sign: skipped only when constant (below)
                    if (((vary >> (8 * d4)) & 0xffu) == 0u) sk |= 1 << d4;
                s_skip = sk;
            }
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
                int uni_tiles = 0;   // this CTA's tiles on one digit in the last pass (the same in every thread)
                for (int pass = 0; pass < 4; ++pass) {
                    if (skip & (1 << pass)) continue;
                    // count with whole-warp votes where the last pass mostly met uniform tiles
                    // (sorted or tied scores); per-key votes otherwise
                    const bool whole = 2 * uni_tiles >= (int)(t1 - t0);
                    uni_tiles = 0;
                    const int sh = 8 * pass;
                    const uint32_t *src = cur < 0 ? nullptr : (cur == 0 ? A.keys[0] : A.keys[1]);
                    uint32_t *dst = cur == 0 ? A.keys[1] : A.keys[0];
                    uint32_t *crow = csum + (size_t)pass * 256 * G;   // [256][G] of this digit
                    if (!first) {   // the chunk's digit counts in the current order
                        for (int i = tid; i < RNW * 256; i += RB) s_hist[i] = 0;
                        __syncthreads();
                        if (!walk_chunk(S, A, src, t0, t1, ph, [&](int64_t, int cnt_tile, const uint32_t (&key)[K], uint32_t *) {
                                if (whole) warp_count<K, true>(key, cnt_tile, sh, s_hist + warp * 256);
                                else warp_count<K, false>(key, cnt_tile, sh, s_hist + warp * 256);
                            })) {
                            if (tid == 0) atomicAdd(A_hist_dirty(A), 1ull);
                            return;
                        }
                        if (tid < 256) {
                            uint32_t tot = 0;
#pragma unroll
                            for (int w = 0; w < RNW; ++w) tot += s_hist[w * 256 + tid];
                            crow[(size_t)tid * G + c] = tot;
                        }
                        if (!bar()) return;
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
                    const bool walked = walk_chunk(S, A, src, t0, t1, ph, [&](int64_t, int cnt_tile, const uint32_t (&key)[K], uint32_t *s_keys) {
                        if (tid == 0) s_d0 = (key[0] >> sh) & 0xffu;   // thread 0 holds the tile's first key
                        for (int i = tid; i < RNW * 256; i += RB) s_hist[i] = 0;
                        __syncthreads();   // every key is in registers: s_keys is free too
                        uint32_t *my_hist = s_hist + warp * 256;
                        warp_count<K, false>(key, cnt_tile, sh, my_hist);
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
                        if (s_tot[s_d0] == (uint32_t)cnt_tile) {   // one digit across the tile (sorted or tied
                            // scores): it keeps its order, so it is written out as it stands
                            const uint32_t base0 = s_gofs[s_d0];
#pragma unroll
                            for (int i = 0; i < K; ++i) {
                                const int li = warp * 32 * K + i * 32 + lane;
                                const uint32_t at = base0 + (uint32_t)li;
                                if (li < cnt_tile && in_bounds(at < (uint32_t)n, &ctl->status)) dst[at] = key[i];
                            }
                            ++uni_tiles;
                            return;   // walk_chunk's barrier follows
                        }
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
                            // lanes holding the same digit: all of them when the warp's keys
                            // agree on it (sorted or tied scores: one vote), else a match
                            // (eight ballots measured slower here: this kernel is bound by
                            // the ALU pipe they use)
                            const bool uni = __all_sync(FULL, d == __shfl_sync(FULL, d, 0));
                            const unsigned peers = uni ? FULL : __match_any_sync(FULL, d);
                            const int leader = __ffs(peers) - 1;
                            uint32_t bs = 0;
                            if (v && lane == leader) {
                                bs = my_hist[d];
                                my_hist[d] = bs + __popc(peers);
                            }
                            bs = __shfl_sync(FULL, bs, leader) + __popc(peers & lt_mask);
                            if (v && in_bounds(bs < (uint32_t)TILE_K(K), &ctl->status)) s_keys[bs] = key[i];
                            __syncwarp();
                        }
                        __syncthreads();
                        // runs of one digit are consecutive in s_keys and in dst: coalesced writes
                        for (int i = tid; i < cnt_tile; i += RB) {
                            const uint32_t kk = s_keys[i];
                            const uint32_t at = s_gofs[(kk >> sh) & 0xffu] + (uint32_t)i;
                            if (in_bounds(at < (uint32_t)n, &ctl->status)) dst[at] = kk;
                        }
                    });
                    if (!walked) {
                        if (tid == 0) atomicAdd(A_hist_dirty(A), 1ull);
                        return;
                    }
                    if (!bar()) return;   // the pass's keys are all written before the next pass reads them
                    cur = cur == 0 ? 1 : 0;
                    first = false;
                }
            }
            // locate: tile and chunk maps of the sorted values (every CTA, its chunk)
            const uint32_t *sorted = cur == 0 ? A.keys[0] : A.keys[1];
            const Seeds z = locate_seeds(A);
            ChunkRec *crec = reinterpret_cast<ChunkRec *>(A.tilebuf);
            TileRec *rec = reinterpret_cast<TileRec *>(A.tilebuf + 8 * SORT_GMAX);
            if (skip != 15 &&
                !locate_tiles<K>(A, S, ph, sorted, n, t0, t1, z, rec, crec, reinterpret_cast<Aff *>(s_hist), s_tab)) {
                if (tid == 0) atomicAdd(A_hist_dirty(A), 1ull);
                return;
            }
            if (!bar()) return;   // the maps are complete, and every CTA has read the global histograms
            if (c == 0) {
                for (int i = tid; i < 4 * 256; i += RB) A.hist[i] = 0ull;   // ready for the next sort
                if (tid < 4) A_sign_bits(A)[tid] = 0ull;
                if (skip != 15) locate_finish<K>(A, sorted, n, z, rec, crec, S.buf, s_hist, s_tab);
            }
            if (!bar()) return;   // the next row reuses the global scratch
            __syncthreads();   // s_open is rewritten by the next block of rows
        }
    }
    pdl_trigger();
}

// ------------------------------------------------------------ launchers --
int sort_grid_max() { return SORT_GMAX; }

// Doubles of locate records a sort of up to cap keys needs: chunk records, then
// one record per tile (8192-key tiles, or 2048 when cap <= SMALL_SORT).
int64_t sort_record_doubles(int64_t cap) {
    const int64_t tiles = cap <= SMALL_SORT ? (cap + TILE_K(RK_SMALL) - 1) / TILE_K(RK_SMALL)
                                            : (cap + TILE_K(RK_BIG) - 1) / TILE_K(RK_BIG);
    return 8 * ((int64_t)SORT_GMAX + tiles + 1);
}

template <int K>
static cudaError_t launch_sort_k(SortArgs &A, cudaStream_t st) {
    const void *kern = reinterpret_cast<const void *>(radix_sort_kernel<K>);
    cudaError_t e = set_max_dynamic_smem(kern, sort_smem<K>());
    if (e != cudaSuccess) return e;
    int resident = 0;   // CTAs of this sort kernel that fit the current device at once
    e = resident_ctas(kern, RB, sort_smem<K>(), &resident);
    if (e != cudaSuccess) return e;
    int64_t g = (A.cap + TILE_K(K) - 1) / TILE_K(K);
    if (g > resident) g = resident;
    if (g > SORT_GMAX) g = SORT_GMAX;
    if (g < 1) g = 1;
    return launch_coop(radix_sort_kernel<K>, (unsigned)g, RB, sort_smem<K>(), st, A);
}

// The tile size follows the capacity of the sort: small sorts take small
// tiles, so more CTAs share the work.
cudaError_t launch_radix_sort(SortArgs &A, double k, double t, cudaStream_t st) {
    (void)k;
    (void)t;
    if (A.cap <= SMALL_SORT) return launch_sort_k<RK_SMALL>(A, st);
    return launch_sort_k<RK_BIG>(A, st);
}


}  // namespace lapsum
