// k_rows.cu -- full-sort solver inside one CTA ("Fast LapSum: Exact
// Differentiable Top-k at Million Scale", technical summary section 2.2,
// full-sort solver): sort the row, one stable prefix/suffix scan of the
// threshold curve, interval search, closed-form root; then p = F((r-b)/t).
//
// One CTA owns one row of up to BLOCK*KPT scores (32768 at 1024 x 32):
//  * sort of the order-preserving uint32 keys: a bitonic network on each thread's
//    keys in registers, then merge-path levels in shared memory (block_merge_sort);
//  * each thread then owns a run of KPT consecutive sorted scores: it forms the
//    links d_j and the run's two affine maps (prefix P and suffix Q), a block
//    scan composes them, G is evaluated at every run end, the crossing run is
//    found by a max-reduction and re-scanned lane-per-element by one warp, and
//    the closed-form root gives b;
//  * the same CTA streams its row again to write p (the row is L2-resident).
// The band of the bracketing path goes to k_band.cu, which narrows it first
// and hands only the part holding b to the same block sort and scan.
#include <cstdint>

#include "lapsum_device.cuh"
#include "lapsum_kernels.h"
#include "scan_solve.cuh"

namespace lapsum {

template <int BLOCK, int KPT>
__global__ void __launch_bounds__(BLOCK, 1)
rowsolve_kernel(const float *__restrict__ scores, int64_t n_arg, double k, double t, double inv_t,
                float *__restrict__ p_out, double *__restrict__ b_out, Ctl *ctl) {
    using C = RowCfg<BLOCK, KPT>;
    extern __shared__ __align__(16) unsigned char smem[];
    uint32_t *s_keys = reinterpret_cast<uint32_t *>(smem);
    uint32_t *s_hist = reinterpret_cast<uint32_t *>(smem + C::SMEM_KEYS);
    __shared__ double s_b;
    __shared__ double s_tab[32];
    exp2_table_init(s_tab);
    pdl_enter();

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = (int)n_arg;
    const float *row = scores + (int64_t)blockIdx.x * n_arg;
    const double m0 = 0.0, top = CUDART_INF, P_top = 0.0, bot = -CUDART_INF, Q_bot = 0.0;
    __syncthreads();   // s_tab

    // ---- load keys (warp-striped; any order is a valid input order), pad with the
    // largest key (sorts last), then sort (a bitonic network per thread, merge
    // levels in shared memory: measured faster than an 8-bit radix sort here)
    uint32_t key[KPT];
    bool bad = false;
#pragma unroll
    for (int i = 0; i < KPT; ++i) {
        const int idx = warp * C::SEG + i * 32 + lane;
        uint32_t kk = 0xffffffffu;
        if (idx < n) {
            const float v = row[idx];
            bad |= !isfinite(v);
            kk = desc_key(v);
        }
        key[i] = kk;
    }
    if (__syncthreads_or(bad) && tid == 0 && ctl) atomicOr(&ctl->status, ST_NONFINITE);

    block_merge_sort<BLOCK, KPT>(key, s_keys);
    __syncthreads();

    int64_t jstar = 0;
    int32_t *st = ctl ? &ctl->status : nullptr;
    double b = block_scan_solve<BLOCK, KPT>(s_keys, n, k, t, inv_t, m0, top, P_top, bot, Q_bot,
                                            s_hist, blockIdx.x == 0 ? &jstar : nullptr, st, s_tab);
    if (tid == 0) {
        s_b = b;
        b_out[blockIdx.x] = b;
        if (blockIdx.x == 0 && ctl) { ctl->b = b; ctl->j_star = jstar; }
    }
    __syncthreads();

    // ---- p = F((r - b)/t) for the row
    b = s_b;
    const PForm pf = make_pform(b, inv_t * LOG2E);
    float *prow = p_out + (int64_t)blockIdx.x * n_arg;
    const bool vec = ((n & 3) == 0) && ((reinterpret_cast<uintptr_t>(row) & 15) == 0) &&
                     ((reinterpret_cast<uintptr_t>(prow) & 15) == 0);
    double psum = 0.0;
    if (vec) {
        const float4 *r4 = reinterpret_cast<const float4 *>(row);
        float4 *p4 = reinterpret_cast<float4 *>(prow);
        for (int i = tid; i < n / 4; i += BLOCK) {
            float4 v = r4[i], o;
            o.x = pf(v.x);
            o.y = pf(v.y);
            o.z = pf(v.z);
            o.w = pf(v.w);
            psum += ((double)o.x + (double)o.y) + ((double)o.z + (double)o.w);
            p4[i] = o;
        }
    } else {
        for (int i = tid; i < n; i += BLOCK) {
            float o = pf(row[i]);
            psum += (double)o;
            prow[i] = o;
        }
    }
    if (blockIdx.x == 0 && ctl) {
        double v[1] = {psum};
        block_sum<BLOCK, 1>(v, reinterpret_cast<double *>(s_hist));
        if (tid == 0) ctl->sum_p = v[0];
    }
}

// ------------------------------------------------------------------ VJP --
// Per-row analytic VJP (technical summary section 2.1):
//   grad_i = (f_i/t)(g_i - lambda),  lambda = <g,f>/sum f,  f_i = e^{-|x_i|}/2.
// lambda is accumulated from terms shifted by the running minimum of |x|
// (in base-2 units, x log2 e)
// (the shift cancels in the ratio), so it stays defined when every f_i
// underflows.  Sums in fp64 with a fixed-order block combine.  The second
// sweep re-reads the row from L2.
struct ShiftSum {
    float m;       // running min |x| (terms are e^{m - |x|} <= 1)
    double sf, sgf;
};
__device__ __forceinline__ void shift_add(ShiftSum &s, float ax, float g) {
    ax = fminf(ax, 3.0e38f);   // |x| may overflow fp32 (t tiny): keep the shift finite
    if (ax < s.m) {
        double sc = (double)exp2f(ax - s.m);   // 0 when s.m = +inf
        s.sf *= sc;
        s.sgf *= sc;
        s.m = ax;
    }
    double e = (double)exp2f(s.m - ax);
    s.sf += e;
    s.sgf = fma((double)g, e, s.sgf);
}
__device__ __forceinline__ ShiftSum shift_merge(ShiftSum a, ShiftSum b) {
    if (b.sf == 0.0) return a;
    if (a.sf == 0.0) return b;
    ShiftSum r;
    r.m = fminf(a.m, b.m);
    double fa = (double)exp2f(r.m - a.m), fb = (double)exp2f(r.m - b.m);
    r.sf = a.sf * fa + b.sf * fb;
    r.sgf = a.sgf * fa + b.sgf * fb;
    return r;
}
__device__ __forceinline__ ShiftSum shfl_xor_ss(ShiftSum s, int o) {
    return {__shfl_xor_sync(FULL, s.m, o), __shfl_xor_sync(FULL, s.sf, o),
            __shfl_xor_sync(FULL, s.sgf, o)};
}

template <int BLOCK>
__global__ void __launch_bounds__(BLOCK)
rowvjp_kernel(const float *__restrict__ scores, const double *__restrict__ b_in,
              const float *__restrict__ g, int64_t n, double inv_t, float *__restrict__ grad) {
    __shared__ ShiftSum s_ss[BLOCK / 32];
    __shared__ double s_lam;
    pdl_enter();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t off = (int64_t)blockIdx.x * n;
    const float *r = scores + off;
    const float *gg = g + off;
    float *out = grad + off;
    const XForm xf = make_xform(b_in[blockIdx.x], inv_t * LOG2E);
    const bool vec = ((n & 3) == 0) && ((reinterpret_cast<uintptr_t>(r) & 15) == 0) &&
                     ((reinterpret_cast<uintptr_t>(gg) & 15) == 0) &&
                     ((reinterpret_cast<uintptr_t>(out) & 15) == 0);
    ShiftSum ss{CUDART_INF_F, 0.0, 0.0};
    if (vec) {
        const float4 *r4 = reinterpret_cast<const float4 *>(r);
        const float4 *g4 = reinterpret_cast<const float4 *>(gg);
        for (int64_t i = tid; i < n / 4; i += BLOCK) {
            float4 v = r4[i], w = g4[i];
            shift_add(ss, fabsf(xf(v.x)), w.x);
            shift_add(ss, fabsf(xf(v.y)), w.y);
            shift_add(ss, fabsf(xf(v.z)), w.z);
            shift_add(ss, fabsf(xf(v.w)), w.w);
        }
    } else {
        for (int64_t i = tid; i < n; i += BLOCK) shift_add(ss, fabsf(xf(r[i])), gg[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss = shift_merge(ss, shfl_xor_ss(ss, o));
    if (lane == 0) s_ss[warp] = ss;
    __syncthreads();
    if (tid == 0) {
        ShiftSum a = s_ss[0];
        for (int w = 1; w < BLOCK / 32; ++w) a = shift_merge(a, s_ss[w]);
        s_lam = a.sgf / a.sf;
    }
    __syncthreads();
    const double lam = s_lam;
    const float lam_hi = (float)lam, lam_lo = (float)(lam - (double)lam_hi);
    const float hit = vjp_scale2(inv_t);   // log2(1/(2t))
    if (vec) {
        const float4 *r4 = reinterpret_cast<const float4 *>(r);
        const float4 *g4 = reinterpret_cast<const float4 *>(gg);
        float4 *o4 = reinterpret_cast<float4 *>(out);
        for (int64_t i = tid; i < n / 4; i += BLOCK) {
            float4 v = r4[i], w = g4[i], o;
            o.x = vjp_term2(xf(v.x), w.x, hit, lam_hi, lam_lo);
            o.y = vjp_term2(xf(v.y), w.y, hit, lam_hi, lam_lo);
            o.z = vjp_term2(xf(v.z), w.z, hit, lam_hi, lam_lo);
            o.w = vjp_term2(xf(v.w), w.w, hit, lam_hi, lam_lo);
            o4[i] = o;
        }
    } else {
        for (int64_t i = tid; i < n; i += BLOCK) out[i] = vjp_term2(xf(r[i]), gg[i], hit, lam_hi, lam_lo);
    }
}

// One row of up to BLOCK * EPT scores per CTA, read from HBM once: each thread
// keeps |x2| of its EPT scores in registers and the row's g in shared memory.
//   1. m = min |x2| over the row (block minimum);
//   2. e_i = 2^{m - |x2_i|} (the largest is 1: no underflow however far b is),
//      lambda = sum g e / sum e (fp32 per thread, fp64 across the block);
//   3. grad_i = e_i 2^{l2h - m} (g_i - lambda), l2h = log2(1/(2t)) -- or, when
//      2^{l2h - m} is not a normal fp32 number (b farther than ~87 t from every
//      score and t not small), from 2^{l2h - |x2_i|} directly, re-reading r.
template <int BLOCK, int EPT>
__global__ void __launch_bounds__(BLOCK, 1)
rowvjp_reg_kernel(const float *__restrict__ scores, const double *__restrict__ b_in,
                  const float *__restrict__ g, int64_t n_arg, double inv_t, float *__restrict__ grad) {
    static_assert(EPT % 4 == 0, "float4 slots");
    extern __shared__ __align__(16) float s_g[];
    __shared__ float s_min[BLOCK / 32];
    __shared__ double s_red[2 * (BLOCK / 32)];
    pdl_enter();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = (int)n_arg;
    const int64_t off = (int64_t)blockIdx.x * n_arg;
    const float *r = scores + off;
    const float *gg = g + off;
    float *out = grad + off;
    const XForm xf = make_xform(b_in[blockIdx.x], inv_t * LOG2E);
    const bool vec = ((n & 3) == 0) && ((reinterpret_cast<uintptr_t>(r) | reinterpret_cast<uintptr_t>(gg) |
                                         reinterpret_cast<uintptr_t>(out)) & 15) == 0;
    // slot i of thread t: element 4 (t + (i/4) BLOCK) + i%4 (vector rows), else t + i BLOCK
    auto elem = [&](int i) -> int { return vec ? 4 * (tid + (i >> 2) * BLOCK) + (i & 3) : tid + i * BLOCK; };
    float ax[EPT];
    float amin = CUDART_INF_F;
    if (vec) {
        const float4 *r4 = reinterpret_cast<const float4 *>(r);
        const float4 *g4 = reinterpret_cast<const float4 *>(gg);
        float4 *sg4 = reinterpret_cast<float4 *>(s_g);
#pragma unroll
        for (int q = 0; q < EPT / 4; ++q) {
            const int i4 = tid + q * BLOCK;
            if (4 * i4 < n) {
                const float4 v = r4[i4];
                sg4[i4] = g4[i4];
                ax[4 * q + 0] = fabsf(xf(v.x));
                ax[4 * q + 1] = fabsf(xf(v.y));
                ax[4 * q + 2] = fabsf(xf(v.z));
                ax[4 * q + 3] = fabsf(xf(v.w));
            } else {
                ax[4 * q + 0] = ax[4 * q + 1] = ax[4 * q + 2] = ax[4 * q + 3] = CUDART_INF_F;
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < EPT; ++i) {
            const int j = tid + i * BLOCK;
            if (j < n) {
                s_g[j] = gg[j];
                ax[i] = fabsf(xf(r[j]));
            } else {
                ax[i] = CUDART_INF_F;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < EPT; ++i) amin = fminf(amin, fminf(ax[i], 3.0e38f));   // finite: |x| may overflow fp32
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amin = fminf(amin, __shfl_xor_sync(FULL, amin, o));
    if (lane == 0) s_min[warp] = amin;
    __syncthreads();   // also: s_g complete
    float m = s_min[0];
#pragma unroll
    for (int w = 1; w < BLOCK / 32; ++w) m = fminf(m, s_min[w]);
    float sf = 0.f, sgf = 0.f;
#pragma unroll
    for (int i = 0; i < EPT; ++i) {
        const float e = exp2f(m - ax[i]);   // padding slots: 2^-inf = 0
        const int j = elem(i);
        const float gj = j < n ? s_g[j] : 0.f;
        sf += e;
        sgf = fmaf(gj, e, sgf);
        ax[i] = e;
    }
    double v[2] = {(double)sf, (double)sgf};
    block_sum<BLOCK, 2>(v, s_red);
    if (tid == 0) s_red[0] = v[1] / v[0];
    __syncthreads();
    const double lam = s_red[0];
    const float lam_hi = (float)lam, lam_lo = (float)(lam - (double)lam_hi);
    const float l2h = vjp_scale2(inv_t);
    const float cexp = l2h - m;
    if (cexp >= -125.0f) {   // 2^{l2h - m} is a normal fp32 number: scale the kept e_i
        const float C = exp2f(cexp);
        if (vec) {
            float4 *o4 = reinterpret_cast<float4 *>(out);
            const float4 *sg4 = reinterpret_cast<const float4 *>(s_g);
#pragma unroll
            for (int q = 0; q < EPT / 4; ++q) {
                const int i4 = tid + q * BLOCK;
                if (4 * i4 < n) {
                    const float4 w = sg4[i4];
                    float4 o;
                    o.x = (ax[4 * q + 0] * C) * ((w.x - lam_hi) - lam_lo);
                    o.y = (ax[4 * q + 1] * C) * ((w.y - lam_hi) - lam_lo);
                    o.z = (ax[4 * q + 2] * C) * ((w.z - lam_hi) - lam_lo);
                    o.w = (ax[4 * q + 3] * C) * ((w.w - lam_hi) - lam_lo);
                    o4[i4] = o;
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < EPT; ++i) {
                const int j = tid + i * BLOCK;
                if (j < n) out[j] = (ax[i] * C) * ((s_g[j] - lam_hi) - lam_lo);
            }
        }
    } else {   // every output is below 2^-125 |g - lambda|: each from its own exponent
#pragma unroll
        for (int i = 0; i < EPT; ++i) {
            const int j = elem(i);
            if (j < n) out[j] = vjp_term2(xf(r[j]), s_g[j], l2h, lam_hi, lam_lo);
        }
    }
}

// ------------------------------------------------------------ launchers --
template <int BLOCK, int KPT>
static cudaError_t launch_rowsolve(const float *scores, int64_t rows, int64_t n, double k, double t,
                                   float *p, double *b, Ctl *ctl, cudaStream_t st) {
    using C = RowCfg<BLOCK, KPT>;
    auto kern = rowsolve_kernel<BLOCK, KPT>;
    const cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void *>(kern), C::SMEM);
    if (e != cudaSuccess) return e;
    return launch_k(kern, (unsigned)rows, BLOCK, C::SMEM, st, scores, n, k, t, 1.0 / t, p, b, ctl);
}

int rowsolve_capacity() { return RowCfg<1024, 32>::CAP; }

cudaError_t launch_rowsolve_rows(const float *scores, int64_t rows, int64_t n, double k, double t,
                                 float *p, double *b, Ctl *ctl, cudaStream_t st) {
    // Few rows (at most two per SM): each row's latency is the time, so a row takes
    // a full 1024-thread CTA with as few keys per thread as it needs (shorter
    // sequential runs in the sort and the scan).  Many short rows: 256-thread CTAs,
    // eight per SM.
    const bool few = rows <= 2 * (int64_t)device_sm_count();
    if (n <= RowCfg<1024, 4>::CAP && few) return launch_rowsolve<1024, 4>(scores, rows, n, k, t, p, b, ctl, st);
    if (n <= RowCfg<256, 16>::CAP) return launch_rowsolve<256, 16>(scores, rows, n, k, t, p, b, ctl, st);
    if (n <= RowCfg<1024, 8>::CAP && few) return launch_rowsolve<1024, 8>(scores, rows, n, k, t, p, b, ctl, st);
    if (n <= RowCfg<1024, 16>::CAP && few) return launch_rowsolve<1024, 16>(scores, rows, n, k, t, p, b, ctl, st);
    return launch_rowsolve<1024, 32>(scores, rows, n, k, t, p, b, ctl, st);
}

cudaError_t launch_rowvjp(const float *scores, const double *b, const float *g, int64_t rows,
                          int64_t n, double t, float *grad, cudaStream_t st) {
    if (n <= 1024 * 32) {   // the row's |x| in registers and its g in shared memory: one read
        auto kern = rowvjp_reg_kernel<1024, 32>;
        const size_t smem = (size_t)((n + 3) & ~int64_t(3)) * sizeof(float);
        const cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void *>(kern), 1024 * 32 * sizeof(float));
        if (e != cudaSuccess) return e;
        return launch_k(kern, (unsigned)rows, 1024, smem, st, scores, b, g, n, 1.0 / t, grad);
    }
    return launch_k(rowvjp_kernel<1024>, (unsigned)rows, 1024, 0, st, scores, b, g, n, 1.0 / t, grad);
}

}  // namespace lapsum
