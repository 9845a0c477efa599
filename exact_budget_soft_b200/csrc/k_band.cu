// k_band.cu -- the band solve of the bracketing path: the threshold b inside
// [a_L, a_R) from the band scores and the streaming pass's counts and tail sums
// ("Fast LapSum: Exact Differentiable Top-k at Million Scale", technical summary
// section 2.2 step 3; the root of one interval in closed form, section 2.1).
//
// One CTA per row.  Instead of sorting the band, the CTA narrows it with a radix
// select steered by G itself:
//   * the band's key range is cut into at most 1024 bins of 2^s consecutive keys;
//     one sweep over the band gives every bin its count, its smallest and largest
//     key, and two tail sums referenced to the bin's own edges,
//         A_j = sum_{r in bin j} e^{(r - e_j)/t},  B_j = sum_{r in bin j} e^{(e_{j+1} - r)/t}
//     (e_j > r >= e_{j+1}, so every term is at most 1);
//   * affine recurrences over the bins -- the maps of the sorted scan, one per
//     bin instead of one per score --
//         U_{j+1} = B_j + d_j U_j,   V_j = A_j + d_j V_{j+1},   d_j = e^{(e_{j+1} - e_j)/t}
//     give G at every edge, G(e_j) = C_j - U_j/2 + V_j/2 (C_j: scores >= e_j);
//   * G falls as b rises, so the bin whose top edge has G < k and whose bottom
//     edge has G >= k holds b; it becomes the new band, the scores above and
//     below it folded into (C, U) and V.
// Each step leaves a key range shorter by ten bits, so at most four steps end
// on a band of one value (any count) or an empty one, where the root has a
// closed form -- no sort at all.  A band of more than WINDOW_MIN scores first
// takes a cheaper step (band_window): bin counts alone bound G at every edge,
// which leaves a window of a few bins; one more sweep sums the tail terms
// outside the window and copies its scores to shared memory, where the later
// steps run.  The sums are fixed point (2^-62 units, exact integers), so b does
// not depend on the order in which threads add.
#include <cstdint>

#include "lapsum_device.cuh"
#include "lapsum_kernels.h"

namespace lapsum {

constexpr int BS_BLOCK = 1024;
constexpr int BS_BITS = 10;
constexpr int BS_BINS = 1 << BS_BITS;   // one bin per thread in the scan
constexpr int BS_NW = BS_BLOCK / 32;
constexpr int GATHER_CAP = 4096;        // bands this small are swept from shared memory
constexpr int WINDOW_MIN = 16384;       // bands longer than this take the window step first

// A band (or sub-band) and what lies outside it.
struct SubBand {
    unsigned long long m0;     // scores at or above top
    unsigned long long n;      // scores inside [bot, top)
    double top, P_top;         // P_top = sum_{r >= top} e^{(top - r)/t}
    double bot, Q_bot;         // Q_bot = sum_{r < bot} e^{(r - bot)/t}
    uint32_t klo, khi;         // smallest and largest descending-order key inside
};

// Fixed-point sum of terms in [0, 1]: q = round(v 2^62) added to a 96-bit
// integer held in three 32-bit words (w[0] lowest), each add carrying into the
// next word itself.  Every word sees the same additions in any order, and each
// add wraps its word at most once, so the carries -- and the total -- do not
// depend on the order of the adds.  (Shared-memory atomics are native only at
// 32 bits.)
__device__ __forceinline__ void fix_add(unsigned *w, double v) {
    const unsigned long long q = __double2ull_rn(v * 0x1p62);
    const unsigned lo = (unsigned)q;
    const unsigned o0 = atomicAdd(&w[0], lo);
    const unsigned mid = (unsigned)(q >> 32) + (o0 + lo < o0 ? 1u : 0u);   // <= 2^30 + 1
    if (mid) {
        const unsigned o1 = atomicAdd(&w[1], mid);
        if (o1 + mid < o1) atomicAdd(&w[2], 1u);
    }
}
__device__ __forceinline__ double fix_value(const unsigned *w) {
    return fma((double)w[2], 4.0, fma((double)w[1], 0x1p-30, (double)w[0] * 0x1p-62));
}

// Per-bin sums of one step (dynamic shared memory).
struct BinSums {
    unsigned cnt[BS_BINS];
    unsigned kmin[BS_BINS];
    unsigned kmax[BS_BINS];
    unsigned fa[BS_BINS][3], fb[BS_BINS][3];   // fixed-point A_j and B_j
};

// Exclusive block scans of three maps per thread: U-maps forward (thread
// order), V-maps backward, counts forward.  scratch: 3 * BS_NW Aff.
__device__ __forceinline__ void block_scan3(Aff mu, Aff mv, unsigned c, Aff &mu_ex, Aff &mv_ex, unsigned &c_ex,
                                            Aff *scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const Aff fi = warp_scan_fwd(mu, lane);
    const Aff bi = warp_scan_bwd(mv, lane);
    unsigned ci = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned p = __shfl_up_sync(FULL, ci, o);
        if (lane >= o) ci += p;
    }
    if (lane == 31) {
        scratch[warp] = fi;
        scratch[2 * BS_NW + warp] = Aff{0.0, (double)ci};
    }
    if (lane == 0) scratch[BS_NW + warp] = bi;
    __syncthreads();
    if (warp == 0) {   // BS_NW == 32: one lane per warp
        Aff wf = warp_scan_fwd(scratch[lane], lane);
        Aff wb = warp_scan_bwd(scratch[BS_NW + lane], lane);
        double wc = scratch[2 * BS_NW + lane].s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double p = __shfl_up_sync(FULL, wc, o);
            if (lane >= o) wc += p;
        }
        __syncwarp();
        scratch[lane] = wf;                        // warps 0..lane
        scratch[BS_NW + lane] = wb;                // warps lane..31
        scratch[2 * BS_NW + lane] = Aff{0.0, wc};  // counts of warps 0..lane
    }
    __syncthreads();
    Aff fe = shfl_up_aff(fi, 1);
    if (lane == 0) fe = aff_id();
    if (warp > 0) fe = aff_then(scratch[warp - 1], fe);
    Aff be = shfl_down_aff(bi, 1);
    if (lane == 31) be = aff_id();
    if (warp < BS_NW - 1) be = aff_then(scratch[BS_NW + warp + 1], be);
    mu_ex = fe;
    mv_ex = be;
    c_ex = (ci - c) + (warp > 0 ? (unsigned)scratch[2 * BS_NW + warp - 1].s : 0u);
}

// Two affine maps with one multiplier, x -> a x + s1 and y -> a y + s2 (the
// upper and lower bounds of the window step share d_j).
struct Aff2 {
    double a, s1, s2;
};
__device__ __forceinline__ Aff2 aff2_then(Aff2 f, Aff2 g) {   // first f, then g
    return {g.a * f.a, fma(g.a, f.s1, g.s1), fma(g.a, f.s2, g.s2)};
}
__device__ __forceinline__ Aff2 shfl_aff2(Aff2 v, int o, bool up) {
    return up ? Aff2{__shfl_up_sync(FULL, v.a, o), __shfl_up_sync(FULL, v.s1, o), __shfl_up_sync(FULL, v.s2, o)}
              : Aff2{__shfl_down_sync(FULL, v.a, o), __shfl_down_sync(FULL, v.s1, o), __shfl_down_sync(FULL, v.s2, o)};
}
// Exclusive block scans of a paired map per thread: forward (thread order) and
// backward.  scratch: 2 * BS_NW Aff2.
__device__ __forceinline__ void block_scan_pair(Aff2 f, Aff2 b, Aff2 &f_ex, Aff2 &b_ex, Aff2 *scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    Aff2 fi = f, bi = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const Aff2 p = shfl_aff2(fi, o, true), q = shfl_aff2(bi, o, false);
        if (lane >= o) fi = aff2_then(p, fi);
        if (lane + o < 32) bi = aff2_then(q, bi);
    }
    if (lane == 31) scratch[warp] = fi;
    if (lane == 0) scratch[BS_NW + warp] = bi;
    __syncthreads();
    if (warp == 0) {   // BS_NW == 32
        Aff2 wf = scratch[lane], wb = scratch[BS_NW + lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const Aff2 p = shfl_aff2(wf, o, true), q = shfl_aff2(wb, o, false);
            if (lane >= o) wf = aff2_then(p, wf);
            if (lane + o < 32) wb = aff2_then(q, wb);
        }
        __syncwarp();
        scratch[lane] = wf;
        scratch[BS_NW + lane] = wb;
    }
    __syncthreads();
    const Aff2 id{1.0, 0.0, 0.0};
    Aff2 fe = shfl_aff2(fi, 1, true), be = shfl_aff2(bi, 1, false);
    if (lane == 0) fe = id;
    if (lane == 31) be = id;
    if (warp > 0) fe = aff2_then(scratch[warp - 1], fe);
    if (warp < BS_NW - 1) be = aff2_then(scratch[BS_NW + warp + 1], be);
    f_ex = fe;
    b_ex = be;
}

// Bin width 2^s for a key range of width w: at most BS_BINS bins.
__device__ __forceinline__ int bin_shift(uint32_t w) {
    const int bits = 32 - __clz(w);
    return bits > BS_BITS ? bits - BS_BITS : 0;
}
// Edge e_j of the J bins of 2^s keys over [klo, khi]: e_0 = top, e_J = bot, and
// between them the value of the largest key of bin j - 1 (so bin j holds the
// scores r with e_{j+1} <= r < e_j).
__device__ __forceinline__ double bin_edge(uint32_t klo, int s, unsigned J, unsigned j, double top, double bot) {
    if (j == 0) return top;
    if (j >= J) return bot;
    return (double)desc_key_to_float(klo + (j << s) - 1u);
}

// One narrowing step, by the whole CTA: bins over the current sub-band S (in
// shared memory), a block scan over the bins (thread j owns bin j), and S left
// holding the bin that contains b.  The first step over the whole band also
// flags a root outside [a_L, a_R) (status non-null); later steps take the bin
// whose edges straddle k as computed, with no flag, as an edge's G can differ
// from the step before it by rounding.
__device__ __noinline__ void band_level(const float *src, int64_t nsrc, SubBand &S, BinSums &B, Aff *scratch,
                                       unsigned *hit, double s2d, double k, const double *tab, int32_t *status,
                                       int32_t *bstatus) {
    const int tid = threadIdx.x;
    const uint32_t klo = S.klo, khi = S.khi;
    const double top = S.top, bot = S.bot;
    const int s = bin_shift(khi - klo);
    const unsigned J = ((khi - klo) >> s) + 1u;   // <= BS_BINS
    if (tid < (int)J) {
        B.cnt[tid] = 0u;
        B.kmin[tid] = 0xffffffffu;
        B.kmax[tid] = 0u;
#pragma unroll
        for (int q = 0; q < 3; ++q) B.fa[tid][q] = B.fb[tid][q] = 0u;
    }
    if (tid == 0) *hit = 0xffffffffu;
    __syncthreads();
    auto add = [&](float x) {
        const uint32_t kk = desc_key(x);
        if (kk < klo || kk > khi) return;
        const unsigned j = (kk - klo) >> s;
        if (!in_bounds(j < J && J <= (unsigned)BS_BINS, bstatus)) return;
        const double xd = (double)x;
        const double eh = bin_edge(klo, s, J, j, top, bot);
        const double el = bin_edge(klo, s, J, j + 1, top, bot);
        atomicAdd(&B.cnt[j], 1u);
        atomicMin(&B.kmin[j], kk);
        atomicMax(&B.kmax[j], kk);
        fix_add(B.fa[j], link_exp((eh - xd) * s2d, tab));   // e^{(r - e_j)/t}
        fix_add(B.fb[j], link_exp((xd - el) * s2d, tab));   // e^{(e_{j+1} - r)/t}
    };
    int64_t i = tid;
    for (; i + 3 * BS_BLOCK < nsrc; i += 4 * BS_BLOCK) {   // four loads in flight
        const float x0 = src[i], x1 = src[i + BS_BLOCK], x2 = src[i + 2 * BS_BLOCK], x3 = src[i + 3 * BS_BLOCK];
        add(x0);
        add(x1);
        add(x2);
        add(x3);
    }
    for (; i < nsrc; i += BS_BLOCK) add(src[i]);
    __syncthreads();

    // thread j: bin j (bins past J carry identity maps)
    const unsigned j = (unsigned)tid;
    const double e_hi = bin_edge(klo, s, J, j, top, bot), e_lo = bin_edge(klo, s, J, j + 1, top, bot);
    unsigned c = 0u;
    double A = 0.0, Bj = 0.0, d = 1.0;
    if (j < J) {
        c = B.cnt[j];
        A = fix_value(B.fa[j]);
        Bj = fix_value(B.fb[j]);
        d = link_exp((e_hi - e_lo) * s2d, tab);   // 0 across an infinite edge
    }
    Aff mu_ex, mv_ex;
    unsigned c_ex;
    block_scan3(Aff{d, Bj}, Aff{d, A}, c, mu_ex, mv_ex, c_ex, scratch);   // U_{j+1} = d U_j + B, V_j = d V_{j+1} + A
    const double U = fma(mu_ex.a, S.P_top, mu_ex.s);           // U_j
    const double Vn = fma(mv_ex.a, S.Q_bot, mv_ex.s);          // V_{j+1}
    const unsigned long long C = S.m0 + c_ex;                  // C_j
    const double Gn = (double)(C + c) - 0.5 * fma(d, U, Bj) + 0.5 * Vn;   // G(e_{j+1})
    if (status && j == 0) {
        const double G0 = (double)C - 0.5 * U + 0.5 * fma(d, Vn, A);
        if (!(G0 < k)) atomicOr(status, ST_NO_ROOT);   // G(a_R) >= k: b at or above a_R
    }
    if (j < J && (Gn >= k || j + 1 == J)) atomicMin(hit, j);   // the first bin whose bottom edge has G >= k
    __syncthreads();
    if (j == *hit) {
        if (status && !(Gn >= k)) atomicOr(status, ST_NO_ROOT);   // G(a_L) < k: b below a_L
        S = SubBand{C, c, e_hi, U, e_lo, Vn, B.kmin[j], B.kmax[j]};
    }
    __syncthreads();
}

// Exclusive block scan of one count per thread.  scratch: BS_NW words.
__device__ __forceinline__ unsigned block_excl_count(unsigned c, unsigned *scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned ci = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned p = __shfl_up_sync(FULL, ci, o);
        if (lane >= o) ci += p;
    }
    __syncthreads();   // scratch free
    if (lane == 31) scratch[warp] = ci;
    __syncthreads();
    if (warp == 0) {
        unsigned w = scratch[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned p = __shfl_up_sync(FULL, w, o);
            if (lane >= o) w += p;
        }
        __syncwarp();
        scratch[lane] = w;
    }
    __syncthreads();
    return (ci - c) + (warp > 0 ? scratch[warp - 1] : 0u);
}

// Scratch of the window step.
struct WinScratch {
    unsigned jlo, jhi;                        // window of bins [jlo, jhi)
    unsigned long long c_lo, c_hi;            // scores at or above its top and bottom edges
    unsigned kmn, kmx;                        // key range of the scores inside
    unsigned long long red[4][BS_NW];         // per-warp fixed-point sums
};

// The first step on a long band, with one atomic per score.  A sweep counts the
// scores per bin; the scans of the per-bin maps with every term at its largest
// (1) and at its smallest (d_j) bound U and V, hence G, at every edge.  An edge
// whose upper bound is below k lies above b; one whose lower bound reaches k lies
// at or below b; the bins between the last edge of the first kind and the first
// of the second hold b (a few bins: the bounds differ by a factor e^{width/t}).
// A second sweep sums the tail terms of the scores above and below that window
// (per-thread fixed point, no atomics) and copies the window's own scores to
// shared memory.  S becomes the window; returns true when the copy holds it.
__device__ __noinline__ bool band_window(const float *src, int64_t nsrc, SubBand &S, BinSums &B, Aff *scratch,
                                        WinScratch &W, float *buf, unsigned *got, double s2d, double k,
                                        const double *tab, int32_t *status) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t klo = S.klo, khi = S.khi;
    const double top = S.top, bot = S.bot;
    const int s = bin_shift(khi - klo);
    const unsigned J = ((khi - klo) >> s) + 1u;
    if (tid < (int)J) B.cnt[tid] = 0u;
    if (tid == 0) {
        W.jlo = 0u;
        W.jhi = J;
        W.kmn = 0xffffffffu;
        W.kmx = 0u;
        *got = 0u;
    }
    __syncthreads();
    auto count = [&](float x) {
        const uint32_t kk = desc_key(x);
        if (kk >= klo && kk <= khi) atomicAdd(&B.cnt[(kk - klo) >> s], 1u);
    };
    int64_t i = tid;
    for (; i + 3 * BS_BLOCK < nsrc; i += 4 * BS_BLOCK) {
        const float x0 = src[i], x1 = src[i + BS_BLOCK], x2 = src[i + 2 * BS_BLOCK], x3 = src[i + 3 * BS_BLOCK];
        count(x0);
        count(x1);
        count(x2);
        count(x3);
    }
    for (; i < nsrc; i += BS_BLOCK) count(src[i]);
    __syncthreads();

    // bounds of G at the edges (thread j: edge j, and the bottom edge J by thread J - 1)
    const unsigned j = (unsigned)tid;
    const double e_hi = bin_edge(klo, s, J, j, top, bot), e_lo = bin_edge(klo, s, J, j + 1, top, bot);
    const unsigned c = j < J ? B.cnt[j] : 0u;
    const double d = j < J ? link_exp((e_hi - e_lo) * s2d, tab) : 1.0;
    const double cmax = (double)c, cmin = (double)c * d;   // a bin's term sum lies in [c d, c]
    Aff2 fu, bv;   // U maps forward, V maps backward; the third word of fu carries the counts
    block_scan_pair(Aff2{d, cmax, cmin}, Aff2{d, cmax, cmin}, fu, bv, reinterpret_cast<Aff2 *>(scratch));
    const double Pmax = fma(fu.a, S.P_top, fu.s1), Pmin = fma(fu.a, S.P_top, fu.s2);    // U at edge j
    const double Vmax1 = fma(bv.a, S.Q_bot, bv.s1), Vmin1 = fma(bv.a, S.Q_bot, bv.s2);  // V at edge j + 1
    const unsigned c_ex = block_excl_count(c, reinterpret_cast<unsigned *>(W.red));
    const unsigned long long C = S.m0 + c_ex;
    auto judge = [&](unsigned e, unsigned long long Ce, double Pmx, double Pmn, double Vmx, double Vmn) {
        const double slack = 1e-12 * ((double)Ce + Pmx + Vmx + 1.0);   // rounding of the scans
        const double Ghi = (double)Ce - 0.5 * Pmn + 0.5 * Vmx + slack;
        const double Glo = (double)Ce - 0.5 * Pmx + 0.5 * Vmn - slack;
        if (Ghi < k) atomicMax(&W.jlo, e);   // edge e lies above b
        if (Glo >= k) atomicMin(&W.jhi, e);  // edge e lies at or below b
        if (status && e == 0 && Glo >= k) atomicOr(status, ST_NO_ROOT);   // G(a_R) >= k
        if (status && e == J && Ghi < k) atomicOr(status, ST_NO_ROOT);    // G(a_L) < k
    };
    if (j < J) judge(j, C, Pmax, Pmin, fma(d, Vmax1, cmax), fma(d, Vmin1, cmin));
    if (j + 1 == J) judge(J, C + c, fma(d, Pmax, cmax), fma(d, Pmin, cmin), Vmax1, Vmin1);
    __syncthreads();
    const unsigned jw0 = min(W.jlo, J - 1u);
    const unsigned jw1 = min(max(W.jhi, jw0 + 1u), J);
    if (j == jw0) W.c_lo = C;
    if (j == jw1) W.c_hi = C;
    if (j + 1 == J && jw1 == J) W.c_hi = C + c;
    const uint32_t kw_lo = klo + (jw0 << s);
    const uint32_t kw_hi = jw1 == J ? khi : klo + (jw1 << s) - 1u;
    const double E_top = bin_edge(klo, s, J, jw0, top, bot), E_bot = bin_edge(klo, s, J, jw1, top, bot);

    // second sweep: exact tail sums outside the window, the window's scores copied
    unsigned long long ah = 0, al = 0, bh = 0, bl = 0;
    unsigned kmn = 0xffffffffu, kmx = 0u;
    auto visit = [&](float x) {
        const uint32_t kk = desc_key(x);
        const bool up = kk < kw_lo, down = kk > kw_hi;   // above the window (r >= E_top), below (r < E_bot)
        const double xd = (double)x;
        const double w = up ? (xd - E_top) * s2d : (down ? (E_bot - xd) * s2d : 0.0);
        const unsigned long long q = __double2ull_rn(link_exp(w, tab) * 0x1p62);   // one term for either side
        const unsigned long long qh = q >> 30, ql = q & 0x3fffffffull;
        ah += up ? qh : 0ull;
        al += up ? ql : 0ull;
        bh += down ? qh : 0ull;
        bl += down ? ql : 0ull;
        if (!up && !down) {
            kmn = min(kmn, kk);
            kmx = max(kmx, kk);
            const unsigned slot = atomicAdd(got, 1u);
            if (slot < (unsigned)GATHER_CAP) buf[slot] = x;
        }
    };
    i = tid;
    for (; i + 3 * BS_BLOCK < nsrc; i += 4 * BS_BLOCK) {
        const float x0 = src[i], x1 = src[i + BS_BLOCK], x2 = src[i + 2 * BS_BLOCK], x3 = src[i + 3 * BS_BLOCK];
        visit(x0);
        visit(x1);
        visit(x2);
        visit(x3);
    }
    for (; i < nsrc; i += BS_BLOCK) visit(src[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ah += __shfl_xor_sync(FULL, ah, o);
        al += __shfl_xor_sync(FULL, al, o);
        bh += __shfl_xor_sync(FULL, bh, o);
        bl += __shfl_xor_sync(FULL, bl, o);
        kmn = min(kmn, __shfl_xor_sync(FULL, kmn, o));
        kmx = max(kmx, __shfl_xor_sync(FULL, kmx, o));
    }
    if (lane == 0) {
        W.red[0][warp] = ah;
        W.red[1][warp] = al;
        W.red[2][warp] = bh;
        W.red[3][warp] = bl;
        atomicMin(&W.kmn, kmn);
        atomicMax(&W.kmx, kmx);
    }
    __syncthreads();
    if (tid == 0) {
        unsigned long long t4[4] = {0, 0, 0, 0};
        for (int w = 0; w < BS_NW; ++w)
            for (int q = 0; q < 4; ++q) t4[q] += W.red[q][w];
        const double sa = fma((double)t4[0], 0x1p-32, (double)t4[1] * 0x1p-62);
        const double sb = fma((double)t4[2], 0x1p-32, (double)t4[3] * 0x1p-62);
        const double U = jw0 == 0 ? S.P_top : fma(S.P_top, link_exp((top - E_top) * s2d, tab), sa);
        const double V = jw1 == J ? S.Q_bot : fma(S.Q_bot, link_exp((E_bot - bot) * s2d, tab), sb);
        S = SubBand{W.c_lo, W.c_hi - W.c_lo, E_top, U, E_bot, V, W.kmn, W.kmx};
    }
    __syncthreads();
    return S.n <= (unsigned long long)GATHER_CAP;
}

// The steps are out of line: a band of one value (quantised scores) or an
// empty band only runs the short path below, and keeping the steps' code apart
// measured 4 us faster per launch on such a band.
__global__ void __launch_bounds__(BS_BLOCK, 1)
band_select_kernel(const float *__restrict__ band_all, int64_t band_cap, double k, double t, double inv_t,
                   Ctl *ctl_all, int32_t round2) {
    extern __shared__ __align__(16) unsigned char dsm[];
    BinSums &s_bins = *reinterpret_cast<BinSums *>(dsm);
    __shared__ Aff s_scan[3 * BS_NW];
    __shared__ WinScratch s_win;
    __shared__ unsigned s_hit;
    __shared__ SubBand s_sb;
    __shared__ double s_tab[32];
    __shared__ float s_buf[GATHER_CAP];
    __shared__ unsigned s_got;
    exp2_table_init(s_tab);
    pdl_enter();

    const int tid = threadIdx.x;
    Ctl *ctl = ctl_all + blockIdx.x;
    if (round2 && !ctl->widened) return;   // the widening round did not start
    const unsigned long long cb = ctl->c_band;
    if (cb > (unsigned long long)band_cap) {
        if (tid == 0) atomicOr(&ctl->status, ST_BAND_OVERFLOW);
        return;
    }
    const double s2d = inv_t * LOG2E;
    const unsigned long long c_R = ctl->c_R;
    if (tid == 0) {
        s_sb.m0 = c_R;
        s_sb.n = cb;
        s_sb.top = (double)ctl->a_R;
        s_sb.P_top = ctl->S_R;
        s_sb.bot = (double)ctl->a_L;
        s_sb.Q_bot = ctl->S_L;
        s_sb.klo = ~ctl->band_kinv;   // largest band score
        s_sb.khi = ctl->band_kmax;    // smallest band score
    }
    __syncthreads();   // s_tab, s_sb
    const float *src = band_all + (int64_t)blockIdx.x * band_cap;
    int64_t nsrc = (int64_t)cb;
    bool first = true, gathered = false;
    if (s_sb.n > (unsigned long long)WINDOW_MIN && s_sb.klo < s_sb.khi) {   // a long band: counts, bounds, window
        gathered = band_window(src, nsrc, s_sb, s_bins, s_scan, s_win, s_buf, &s_got, s2d, k, s_tab, &ctl->status);
        if (gathered) {
            src = s_buf;
            nsrc = min(s_got, (unsigned)GATHER_CAP);   // the window's count by construction
        }
        first = false;
    }
    for (int it = 0; it < 4; ++it) {   // four steps reach a single key
        if (s_sb.n == 0 || s_sb.klo >= s_sb.khi) break;
        if (!gathered && s_sb.n <= (unsigned long long)GATHER_CAP) {   // later steps sweep a copy
            if (tid == 0) s_got = 0u;
            __syncthreads();
            const uint32_t klo = s_sb.klo, khi = s_sb.khi;
            for (int64_t i = tid; i < nsrc; i += BS_BLOCK) {
                const float x = src[i];
                const uint32_t kk = desc_key(x);
                if (kk >= klo && kk <= khi) {
                    const unsigned slot = atomicAdd(&s_got, 1u);
                    if (slot < (unsigned)GATHER_CAP) s_buf[slot] = x;
                }
            }
            __syncthreads();
            src = s_buf;
            nsrc = min(s_got, (unsigned)GATHER_CAP);   // the band's count by construction
            gathered = true;
        }
        band_level(src, nsrc, s_sb, s_bins, s_scan, &s_hit, s2d, k, s_tab, first ? &ctl->status : nullptr,
                   &ctl->status);
        first = false;
    }
    if (tid != 0) return;
    const SubBand S = s_sb;
    const int64_t above = (int64_t)(S.m0 - c_R);   // band scores above the final band
    if (S.n == 0) {   // no score in [bot, top): one interval
        const double ed = link_exp((S.top - S.bot) * s2d, s_tab);
        const double m0 = (double)S.m0;
        const double Gt = m0 - 0.5 * S.P_top + 0.5 * ed * S.Q_bot;
        const double Gb = m0 - 0.5 * ed * S.P_top + 0.5 * S.Q_bot;
        if (first && (!(Gt < k) || !(Gb >= k))) atomicOr(&ctl->status, ST_NO_ROOT);
        ctl->b = solve_interval(S.top, S.bot, m0, S.P_top, S.Q_bot, ed, k, t);
        ctl->j_star = above - 1;
        return;
    }
    // one value, of any count (klo == khi once the loop ends)
    bool at_or_above = false;
    ctl->b = solve_equal_run_values((double)desc_key_to_float(S.klo), (double)S.n, (double)S.m0, S.top, S.P_top,
                                    S.bot, S.Q_bot, k, t, &at_or_above);
    ctl->j_star = at_or_above ? above + (int64_t)S.n - 1 : above - 1;
}

cudaError_t launch_band_select(const float *band, int64_t rows, double k, double t, Ctl *ctl, int64_t band_cap,
                               int32_t round2, cudaStream_t st) {
    const cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void *>(band_select_kernel), sizeof(BinSums));
    if (e != cudaSuccess) return e;
    return launch_k(band_select_kernel, (unsigned)rows, BS_BLOCK, sizeof(BinSums), st, band, band_cap, k, t,
                    1.0 / t, ctl, round2);
}

}  // namespace lapsum
