// lapsum_device.cuh -- device building blocks shared by the kernels.
//
// Notation ("Fast LapSum: Exact Differentiable Top-k at Million Scale",
// technical summary sections 2.1-2.2): scores sorted descending
// c_0 >= c_1 >= ... >= c_{n-1}, temperature t, budget k, Laplace CDF F,
// G(b) = sum_i F((c_i - b)/t) (continuous, strictly decreasing).
//
// Stable threshold curve (the "single stable prefix/suffix scan" of the
// full-sort solver): with links d_j = e^{(c_{j+1} - c_j)/t} <= 1,
//   P_j = sum_{i<=j} e^{(c_j - c_i)/t} = 1 + d_{j-1} P_{j-1}      (prefix)
//   Q_j = sum_{i>=j} e^{(c_i - c_j)/t} = 1 + d_j Q_{j+1}          (suffix)
//   G(c_j) = m0 + (j+1) - P_j/2 + d_j Q_{j+1}/2
// where m0 scores lie above c_0 (0 for a full row; the count above a_R for a
// band).  Every factor is <= 1, so nothing overflows ("max-shifted"), and each
// recurrence is an affine map x -> a x + s, composed associatively in scans.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "lapsum_internal.h"

namespace lapsum {

constexpr unsigned FULL = 0xffffffffu;

// ------------------------------------------------------- checked build --
// Built with -DLAPSUM_CHECKED (liblapsum_checked.so), every computed index of a
// store or gather below is tested against its buffer before the access: an
// index outside sets ST_BOUNDS in the row's status word (reported as
// LAPSUM_ERR_BOUNDS) and the access is skipped -- never a trap.  In the normal
// build the test compiles away.
#ifdef LAPSUM_CHECKED
__device__ __forceinline__ bool in_bounds(bool ok, int32_t *status) {
    if (!ok && status) atomicOr(status, ST_BOUNDS);
    return ok;
}
#else
__device__ __forceinline__ bool in_bounds(bool, int32_t *) { return true; }
#endif

// ---------------------------------------------------------------- keys --
// Order-preserving map float -> uint32 whose ASCENDING order is the DESCENDING
// order of the floats (largest score first).
__device__ __forceinline__ uint32_t desc_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? u : (u ^ 0x7fffffffu);
}
__device__ __forceinline__ float desc_key_to_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? k : (k ^ 0x7fffffffu));
}

// Folds a CTA's band-key maxima (per thread; 0 for none) into those two words:
// one shared and one global atomic per CTA.  Every thread of the CTA calls it.
__device__ __forceinline__ void band_range_flush(Ctl *c, uint32_t kmax, uint32_t kinv, uint32_t *s_two) {
    if (threadIdx.x == 0) { s_two[0] = 0u; s_two[1] = 0u; }
    __syncthreads();
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    kinv = __reduce_max_sync(0xffffffffu, kinv);
    if ((threadIdx.x & 31) == 0 && (kmax | kinv)) {
        atomicMax(&s_two[0], kmax);
        atomicMax(&s_two[1], kinv);
    }
    __syncthreads();
    if (threadIdx.x == 0 && (s_two[0] | s_two[1])) {
        atomicMax(&c->band_kmax, s_two[0]);
        atomicMax(&c->band_kinv, s_two[1]);
    }
}

// ------------------------------------------------------- affine maps --
struct Aff {
    double a, s;   // x -> a x + s
};
__device__ __forceinline__ Aff aff_id() { return {1.0, 0.0}; }
// first f, then g
__device__ __forceinline__ Aff aff_then(Aff f, Aff g) { return {g.a * f.a, fma(g.a, f.s, g.s)}; }
__device__ __forceinline__ Aff shfl_up_aff(Aff v, int o) {
    return {__shfl_up_sync(FULL, v.a, o), __shfl_up_sync(FULL, v.s, o)};
}
__device__ __forceinline__ Aff shfl_down_aff(Aff v, int o) {
    return {__shfl_down_sync(FULL, v.a, o), __shfl_down_sync(FULL, v.s, o)};
}
// Inclusive warp scan in lane order: lane l gets map_0 then ... then map_l.
__device__ __forceinline__ Aff warp_scan_fwd(Aff v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        Aff p = shfl_up_aff(v, o);
        if (lane >= o) v = aff_then(p, v);
    }
    return v;
}
// Inclusive warp scan in reverse lane order: lane l gets map_31 then ... then map_l.
__device__ __forceinline__ Aff warp_scan_bwd(Aff v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        Aff p = shfl_down_aff(v, o);
        if (lane + o < 32) v = aff_then(p, v);
    }
    return v;
}

// Block-wide EXCLUSIVE scans of one affine map per thread (thread order).
// fwd: thread i gets map_0 then ... then map_{i-1};
// bwd: thread i gets map_{NT-1} then ... then map_{i+1}.
// scratch: 2*NW Aff in shared memory.  Contains __syncthreads.
template <int BLOCK>
__device__ __forceinline__ void block_scan_excl_both(Aff fwd, Aff bwd, Aff &fwd_ex, Aff &bwd_ex,
                                                     Aff *scratch) {
    constexpr int NW = BLOCK / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    Aff fi = warp_scan_fwd(fwd, lane);
    Aff bi = warp_scan_bwd(bwd, lane);
    if (lane == 31) scratch[warp] = fi;
    if (lane == 0) scratch[NW + warp] = bi;
    __syncthreads();
    if (warp == 0) {
        Aff wf = lane < NW ? scratch[lane] : aff_id();
        Aff wb = lane < NW ? scratch[NW + lane] : aff_id();
        wf = warp_scan_fwd(wf, lane);
        // reverse order over the NW warps: lanes >= NW carry the identity
        wb = warp_scan_bwd(wb, lane);
        __syncwarp();
        if (lane < NW) {
            scratch[lane] = wf;        // inclusive over warps 0..lane
            scratch[NW + lane] = wb;   // inclusive over warps lane..NW-1
        }
    }
    __syncthreads();
    Aff fe = shfl_up_aff(fi, 1);
    if (lane == 0) fe = aff_id();
    if (warp > 0) fe = aff_then(scratch[warp - 1], fe);
    Aff be = shfl_down_aff(bi, 1);
    if (lane == 31) be = aff_id();
    if (warp < NW - 1) be = aff_then(scratch[NW + warp + 1], be);
    fwd_ex = fe;
    bwd_ex = be;
    __syncthreads();
}

// ------------------------------------------------------- reductions --
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    return v;
}
__device__ __forceinline__ int warp_max_int(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(FULL, v, o));
    return v;
}

// Fixed-order block sum of up to 4 doubles (result valid in thread 0).
template <int BLOCK, int N>
__device__ __forceinline__ void block_sum(double (&v)[N], double *scratch /* N*NW */) {
    constexpr int NW = BLOCK / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = warp_sum(v[i]);
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < N; ++i) scratch[i * NW + warp] = v[i];
    }
    __syncthreads();
    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < N; ++i) {
            double s = 0.0;
            for (int w = 0; w < NW; ++w) s += scratch[i * NW + w];
            v[i] = s;
        }
    }
    __syncthreads();
}

// ---------------------------------------------------- closed-form root --
// Root of G(b) = k inside one interval [L, U] between consecutive sorted
// values ("closed-form root within the interval where the budget equation
// balances", technical summary section 2.2).  In the interval
//   G(b) = A - (P_U/2) e^{(b-U)/t} + (Q_L/2) e^{(L-b)/t},
// A = #scores >= U, P_U = sum_{r>=U} e^{(U-r)/t}, Q_L = sum_{r<=L} e^{(r-L)/t},
// e_d = e^{(L-U)/t}.  With v = e^{(b-L)/t} in [1, 1/e_d] this is the quadratic
//   (P_U e_d / 2) v^2 + (k - A) v - Q_L/2 = 0,
// (the unshifted form is 1/2 S- u^2 + (k-m) u - 1/2 S+ = 0, u = e^{b/t}),
// whose positive root is taken in the cancellation-free form for the sign of
// k - A.  L = -inf (nothing below) uses w = e^{(b-U)/t}: A - P_U w/2 = k.
__device__ __forceinline__ double solve_interval(double U, double L, double A, double P_U,
                                                 double Q_L, double e_d, double k, double t) {
    if (L == -CUDART_INF) {
        double w = 2.0 * (A - k) / P_U;
        return U + t * log(w);
    }
    double a2 = P_U * e_d;
    double bq = k - A;
    double sq = sqrt(fma(bq, bq, a2 * Q_L));
    double v;
    if (bq >= 0.0) v = (bq + sq) > 0.0 ? Q_L / (bq + sq) : 1.0;
    else           v = (sq - bq) / a2;
    if (!(v >= 1.0)) v = 1.0;
    double b = L + t * log(v);
    if (b > U) b = U;
    return b;
}

// nn copies of one value c between the seeds of a solve (m0 scores above, the
// sum P_top of e^{(top-r)/t} over them ending at value top, Q_bot likewise below
// from bot): the threshold curve is flat across the run,
//   G(c) = m0 + nn/2 - d_top P_top/2 + d_bot Q_bot/2,
// and (G decreasing) the root lies in [bot, c] when G(c) <= k, else in [c, top).
// *above_run: whether the run is above the root (j* = last of the run) or not.
__device__ __forceinline__ double solve_equal_run_values(double c, double nn, double m0, double top,
                                                         double P_top, double bot, double Q_bot, double k,
                                                         double t, bool *above_run) {
    const double d_top = top == CUDART_INF ? 0.0 : exp((c - top) / t);
    const double d_bot = bot == -CUDART_INF ? 0.0 : exp((bot - c) / t);
    const double Gc = m0 + 0.5 * nn - 0.5 * d_top * P_top + 0.5 * d_bot * Q_bot;
    if (Gc <= k) {
        *above_run = true;
        return solve_interval(c, bot, m0 + nn, nn + d_top * P_top, Q_bot, d_bot, k, t);
    }
    *above_run = false;
    return solve_interval(top, c, m0, P_top, nn + d_bot * Q_bot, d_top, k, t);
}

// ----------------------------------------------- fp32 elementwise math --
constexpr float LOG2E_F = 1.4426950408889634f;
constexpr double LOG2E = 1.4426950408889634;

// x = (r - b)/t in fp32 from a hi/lo split of the fp64 threshold b:
//   x = ((r - b_hi) - b_lo) * s.
// Near the threshold r - b_hi is exact (Sterbenz), so x keeps fp32 relative
// accuracy however close r is to b; s = log2(e)/t gives x in base-2 units.
struct XForm {
    float b_hi, b_lo, s;
    __device__ __forceinline__ float operator()(float r) const { return ((r - b_hi) - b_lo) * s; }
};
__device__ __forceinline__ XForm make_xform(double b, double scale) {
    XForm f;
    f.b_hi = (float)b;
    f.b_lo = (float)(b - (double)f.b_hi);
    f.s = (float)scale;
    return f;
}

// Laplace CDF from the base-2 argument x2 = x log2(e):
// F = 2^{x2}/2 (x2 < 0), 1 - 2^{-x2}/2 (x2 >= 0).
__device__ __forceinline__ float laplace_cdf2(float x2) {
    const float e = 0.5f * exp2f(-fabsf(x2));
    return x2 < 0.0f ? e : 1.0f - e;
}

// The returned p = F((r - b)/t), written so that sum p keeps the budget k over
// millions of scores (the method's exact-budget property, technical summary
// section 2.1).  Two systematic errors of a plain fp32 evaluation would add up
// over the row instead of cancelling:
//  * the fp32 scale s = log2(e)/t carries one relative rounding error shared by
//    every score; s is split into s_hi + s_lo and x2 = d s_hi + d s_lo by an fma,
//    so what is left is each score's own rounding;
//  * where p is mid-range (|x2| < 1, p in (1/4, 3/4)) every score's p is of the
//    same size and any bias of the fp32 exponential would add up linearly, so
//    there p is formed in fp64 from the fp64 threshold and rounded once.
// Elsewhere p < 1/4 or 1 - p < 1/4 and the fp32 value is used.
struct PForm {
    float b_hi, b_lo, s_hi, s_lo;
    double b, s2d;
    // fp32 p into out; true if p is mid-range (then mid() gives the value to keep)
    __device__ __forceinline__ bool fast(float r, float &out) const {
        const float d = (r - b_hi) - b_lo;
        const float x2 = fmaf(d, s_lo, d * s_hi);
        out = laplace_cdf2(x2);
        return fabsf(x2) < 1.0f;
    }
    __device__ __forceinline__ float mid(float r) const {
        const double xd = ((double)r - b) * s2d;
        const double e = 0.5 * exp2(-fabs(xd));
        return (float)(xd < 0.0 ? e : 1.0 - e);
    }
    __device__ __forceinline__ float operator()(float r) const {
        float o;
        return fast(r, o) ? mid(r) : o;
    }
};
__device__ __forceinline__ PForm make_pform(double b, double scale) {
    PForm f;
    f.b = b;
    f.s2d = scale;
    f.b_hi = (float)b;
    f.b_lo = (float)(b - (double)f.b_hi);
    f.s_hi = (float)scale;
    f.s_lo = (float)(scale - (double)f.s_hi);
    return f;
}

// One VJP output, (f/t)(g - lambda), f = e^{-|x|}/2, from the base-2 argument.
// The factor 1/(2t) enters the exponent, f/t = 2^{l2h - |x2|} with
// l2h = log2(1/(2t)) (vjp_scale2), so an output that fp32 can hold comes out
// even where f alone would underflow (t tiny, b far from every score).
// g - lambda uses a hi/lo split of the fp64 lambda: when a few scores carry
// almost all of sum f, lambda sits within an fp32 ulp of their g, and the split
// keeps the difference exact.
__device__ __forceinline__ float vjp_term2(float x2, float g, float l2h, float lam_hi, float lam_lo) {
    return exp2f(l2h - fabsf(x2)) * ((g - lam_hi) - lam_lo);
}
__device__ __forceinline__ float vjp_scale2(double inv_t) { return (float)log2(0.5 * inv_t); }

// ----------------------------------------------------- near-tier exp --
// 2^{-w} for 0 <= w <= 1000, the fp64 terms of the tail sums.  Table-driven
// reduction after P. T. P. Tang, "Table-driven implementation of the
// exponential function in IEEE floating-point arithmetic", ACM TOMS 15 (1989):
//   N = rint(32 w) = 32 m + j,  r = w - N/32 in [-1/64, 1/64],
//   2^{-w} = 2^{-m} * 2^{-j/32} * 2^{-r},
// 2^{-r} = e^{-r ln 2} by its Taylor polynomial to degree 6 (remainder
// < 4e-18), the 32 table values 2^{-j/32} from the library exp2 (computed once
// per block into shared memory), 2^{-m} applied to the exponent field.  About
// 11 fp64 operations; relative error a few ulp (tested against exp).
constexpr double EXP_LN2 = 0x1.62e42fefa39efp-1;
constexpr double EXP_C1 = -EXP_LN2;
constexpr double EXP_C2 = EXP_LN2 * EXP_LN2 / 2.0;
constexpr double EXP_C3 = -EXP_LN2 * EXP_LN2 * EXP_LN2 / 6.0;
constexpr double EXP_C4 = EXP_LN2 * EXP_LN2 * EXP_LN2 * EXP_LN2 / 24.0;
constexpr double EXP_C5 = -EXP_LN2 * EXP_LN2 * EXP_LN2 * EXP_LN2 * EXP_LN2 / 120.0;
constexpr double EXP_C6 = EXP_LN2 * EXP_LN2 * EXP_LN2 * EXP_LN2 * EXP_LN2 * EXP_LN2 / 720.0;

// Fill a 32-entry shared table with 2^{-j/32} (call before use, then sync).
__device__ __forceinline__ void exp2_table_init(double *tab) {
    if (threadIdx.x < 32) tab[threadIdx.x] = exp2(-(double)threadIdx.x / 32.0);
}
__device__ __forceinline__ double exp2_neg(double w, const double *tab) {
    const double big = 0x1.8p52;
    const double tt = fma(w, 32.0, big);                   // N in the low mantissa bits
    const int N = (int)(uint32_t)__double_as_longlong(tt);
    const double r = fma(tt - big, -0.03125, w);           // w - N/32, exact
    double p = EXP_C6;
    p = fma(p, r, EXP_C5);
    p = fma(p, r, EXP_C4);
    p = fma(p, r, EXP_C3);
    p = fma(p, r, EXP_C2);
    p = fma(p, r, EXP_C1);
    p = fma(p, r, 1.0);
    const double v = tab[N & 31] * p;
    return __longlong_as_double(__double_as_longlong(v) - ((long long)(N >> 5) << 52));
}

// A link of the threshold curve, e^{-(hi - lo)/t} = 2^{-w}, w = (hi - lo) log2(e)/t >= 0
// (w > 1000 is below 2^{-1000}: zero for every sum it enters; w = 0, a tie, is
// exactly 1, which exp2_neg also returns -- the branch only skips the work).
__device__ __forceinline__ double link_exp(double w, const double *tab) {
    if (w == 0.0) return 1.0;
    return w <= 1000.0 ? exp2_neg(w, tab) : 0.0;
}

// ------------------------------------------------ bulk-copy pipeline --
// Streaming passes move the row through shared memory with 1D bulk copies
// (cp.async.bulk, completion counted in bytes on an mbarrier): each CTA keeps
// STAGES chunks in flight however many registers its threads need, so the
// read rate does not hinge on occupancy.  Chunks go to CTAs round-robin (or in
// reverse, to start on the part of the row a previous pass left in L2); the
// ragged tail is left to plain loads.  Every wait is bounded.
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait; returns false (and leaves the error to the caller) on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int cap) {
    for (int it = 0; it < cap; ++it)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// 16-byte shared-memory load through an explicit shared address (chunk pointers
// handed to a body lambda would otherwise be read with generic loads)
__device__ __forceinline__ float4 lds128(const float4 *p) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(smem_addr(p)));
    return v;
}

constexpr int BULK_F4 = 512;                    // float4 per source per chunk (8 KB)
constexpr int BULK_WAIT_CAP = 1 << 22;
// stages in flight: 4 chunks of one source, 3 of two (48 KB per CTA, so four
// CTAs of either kind fit one SM's shared memory)
template <int NSRC>
constexpr int bulk_stages() { return NSRC == 1 ? 4 : 3; }

// Shared memory of a pipeline with NSRC sources (dynamic, 16-byte aligned): the
// stages, then one mbarrier per stage.
template <int NSRC>
constexpr size_t bulk_smem_bytes() {
    return (size_t)bulk_stages<NSRC>() * NSRC * BULK_F4 * 16 + 8 * bulk_stages<NSRC>();
}

// Streams the full chunks of NSRC float4 arrays of n4 vectors through shared
// memory and calls body(const float4 *chunk[NSRC], int64_t first_vector) once
// per chunk, by every thread of the CTA (each thread reads its own vectors of
// the chunk).  Returns the number of vectors covered by full chunks (the rest
// is the caller's tail).  One mbarrier per stage counts the bytes of its copy;
// a CTA barrier after each chunk frees its stage, and thread 0 refills it with
// the chunk STAGES ahead.  (Measured against a split full/empty mbarrier ring
// with one arrival per warp: as fast on random score order, 3.5% faster on the
// sorted 1e8 row.)  If a wait gives up (in any thread), the CTA sets
// ST_TIMEOUT, issues no further copy, waits (bounded again) for the copies it
// has in flight and stops streaming; the caller's result is then invalid and
// the error reaches the host through the status word.
template <int NSRC, typename Body>
__device__ __forceinline__ int64_t bulk_stream(const float4 *const (&src)[NSRC], int64_t n4, bool reverse,
                                               unsigned char *smem, int32_t *status, Body &&body) {
    constexpr int BULK_STAGES = bulk_stages<NSRC>();
    float4 *buf = reinterpret_cast<float4 *>(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)BULK_STAGES * NSRC * BULK_F4 * 16);
    const int64_t nch = n4 / BULK_F4;
    const int64_t G = gridDim.x;
    const int64_t mine = nch > blockIdx.x ? (nch - 1 - blockIdx.x) / G + 1 : 0;
    auto chunk_of = [&](int64_t i) -> int64_t {
        const int64_t c = blockIdx.x + i * G;
        return reverse ? nch - 1 - c : c;
    };
    constexpr uint32_t BYTES = BULK_F4 * 16;
    if (threadIdx.x == 0) {
        for (int s = 0; s < BULK_STAGES; ++s) mbar_init(&bars[s], 1);
        mbar_init_fence();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int s = 0; s < BULK_STAGES && s < mine; ++s) {
            mbar_expect_tx(&bars[s], BYTES * NSRC);
            const int64_t c = chunk_of(s);
#pragma unroll
            for (int q = 0; q < NSRC; ++q)
                bulk_load(buf + ((size_t)s * NSRC + q) * BULK_F4, src[q] + c * BULK_F4, BYTES, &bars[s]);
        }
    }
    for (int64_t i = 0; i < mine; ++i) {
        const int s = (int)(i % BULK_STAGES);
        const uint32_t parity = (uint32_t)((i / BULK_STAGES) & 1);
        const bool ok = mbar_wait(&bars[s], parity, BULK_WAIT_CAP);
        const float4 *chunk[NSRC];
#pragma unroll
        for (int q = 0; q < NSRC; ++q) chunk[q] = buf + ((size_t)s * NSRC + q) * BULK_F4;
        body(chunk, chunk_of(i) * BULK_F4);
        if (!__syncthreads_and(ok)) {   // every thread is done with stage s; a wait gave up
            if (threadIdx.x == 0) {
                if (status) atomicOr(status, ST_TIMEOUT);
                // the copies issued and not yet consumed: chunks i .. i + STAGES - 1
                for (int64_t j = i; j < i + BULK_STAGES && j < mine; ++j)
                    mbar_wait(&bars[j % BULK_STAGES], (uint32_t)((j / BULK_STAGES) & 1), BULK_WAIT_CAP);
            }
            __syncthreads();
            return nch * BULK_F4;
        }
        if (threadIdx.x == 0 && i + BULK_STAGES < mine) {
            fence_proxy_async_smem();
            mbar_expect_tx(&bars[s], BYTES * NSRC);
            const int64_t c = chunk_of(i + BULK_STAGES);
#pragma unroll
            for (int q = 0; q < NSRC; ++q)
                bulk_load(buf + ((size_t)s * NSRC + q) * BULK_F4, src[q] + c * BULK_F4, BYTES, &bars[s]);
        }
    }
    return nch * BULK_F4;
}

// ------------------------------------------- programmatic dependent launch --
// Every kernel of a solve is launched with programmatic stream serialization:
// it may be scheduled while its predecessor drains, so it first waits for the
// predecessor's results (griddepcontrol.wait; a no-op when launched plainly)
// and then lets its own successor start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_enter() {
    pdl_wait();
    pdl_trigger();
}

// ------------------------------------------------ bounded device waits --
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u32(unsigned *p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Grid-wide barrier of a cooperative launch (every CTA is resident): an
// arrival counter and a generation word in device memory; the last CTA to
// arrive resets the counter and advances the generation.  The wait is bounded:
// after cap polls (or as soon as another CTA has given up: ST_TIMEOUT in
// *status) the CTA sets ST_TIMEOUT and the barrier returns false.  The caller
// then returns at once, so no CTA runs a phase after a barrier that did not
// complete; the CTAs still waiting give up in turn (the one that left never
// arrives again), each after a bounded wait.  A CTA also skips arriving when
// the status already carries ST_TIMEOUT.
__device__ __forceinline__ int32_t ld_volatile_s32(const int32_t *p) {
    return *reinterpret_cast<const volatile int32_t *>(p);
}
__device__ __forceinline__ bool grid_sync(unsigned *count, unsigned *gen, int cap, int32_t *status) {
    __shared__ int s_gave_up;
    __syncthreads();
    if (threadIdx.x == 0) {
        int gave_up = (ld_volatile_s32(status) & ST_TIMEOUT) != 0;
        if (!gave_up) {
            const unsigned g = ld_acquire_u32(gen);   // read before arriving: it cannot advance yet
            __threadfence();
            if (atomicAdd(count, 1u) == gridDim.x - 1) {
                atomicExch(count, 0u);
                __threadfence();
                st_release_u32(gen, g + 1u);
            } else {
                int it = 0;
                while (ld_acquire_u32(gen) == g) {
                    if (++it > cap || (ld_volatile_s32(status) & ST_TIMEOUT)) {
                        atomicOr(status, ST_TIMEOUT);
                        gave_up = 1;
                        break;
                    }
                    __nanosleep(64);
                }
            }
            __threadfence();
        }
        s_gave_up = gave_up;
    }
    __syncthreads();
    return s_gave_up == 0;
}

}  // namespace lapsum
