// k_noalloc.cu -- a backward (VJP) entry point that allocates no device memory.
//
// Who needs it: code that must not call cudaMalloc on the hot path -- e.g. an
// inference plugin whose host framework owns all device memory, or a process
// running under a fixed memory budget.  lapsum_backward keeps per-stream scratch that it grows with
// cudaMalloc on first use; this variant instead uses one fixed array compiled
// into the library (LAPSUM_NOALLOC_SCRATCH_BYTES per GPU, held for the life of
// the process by every GPU that loads the library).
//
// Computation: identical in meaning to lapsum_backward -- per row,
//   grad_i = (f_i/t)(g_i - <g,f>/sum f),  f_i = exp(-|r_i - b|/t)/2.
// One launch reduces every row at once (each row gets B blocks; per-block
// partials are terms shifted by the block's smallest |x|, so the ratio stays
// defined when every f underflows), the last block of a row combines that
// row's partials in block order and stores lambda; a second launch applies.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/lapsum.h"
#include "lapsum_device.cuh"
#include "lapsum_kernels.h"

namespace lapsum {

// The scratch array.  Layout for a call with R rows and B blocks per row:
//   double part[R][B][3]   (shift m, sum f, sum g f of each block)
//   double lambda[R]
//   unsigned ticket[R]     (cleared at the start of every call)
static __device__ __align__(256) unsigned char g_noalloc_scratch[LAPSUM_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int NB = 256;   // threads per block

struct ShiftAcc {
    float m;
    double sf, sgf;
};
__device__ __forceinline__ void sa_add(ShiftAcc &s, float ax, float g) {
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
__device__ __forceinline__ ShiftAcc sa_merge(ShiftAcc a, ShiftAcc b) {
    if (b.sf == 0.0) return a;
    if (a.sf == 0.0) return b;
    ShiftAcc r;
    r.m = fminf(a.m, b.m);
    const double fa = (double)exp2f(r.m - a.m), fb = (double)exp2f(r.m - b.m);
    r.sf = a.sf * fa + b.sf * fb;
    r.sgf = a.sgf * fa + b.sgf * fb;
    return r;
}

size_t scratch_need(int64_t rows, int64_t B) {
    return (size_t)rows * (size_t)B * 3 * sizeof(double) + (size_t)rows * sizeof(double) +
           (size_t)rows * sizeof(unsigned);
}

// grid = rows * B; block (row, j) covers the j-th slice of the row, grid-stride
__global__ void __launch_bounds__(NB)
noalloc_reduce_kernel(const float *__restrict__ r, const double *__restrict__ b_in,
                      const float *__restrict__ g, int64_t n, int64_t B, double inv_t,
                      unsigned char *scratch, int64_t rows) {
    __shared__ ShiftAcc s_w[NB / 32];
    __shared__ bool s_last;
    double *part = reinterpret_cast<double *>(scratch);
    double *lam = part + rows * B * 3;
    unsigned *ticket = reinterpret_cast<unsigned *>(lam + rows);
    const int64_t row = blockIdx.x / B, j = blockIdx.x % B;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float *rr = r + row * n;
    const float *gg = g + row * n;
    const XForm xf = make_xform(b_in[row], inv_t * LOG2E);
    ShiftAcc s{CUDART_INF_F, 0.0, 0.0};
    for (int64_t i = j * NB + tid; i < n; i += B * NB) sa_add(s, fabsf(xf(rr[i])), gg[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ShiftAcc q{__shfl_xor_sync(FULL, s.m, o), __shfl_xor_sync(FULL, s.sf, o),
                   __shfl_xor_sync(FULL, s.sgf, o)};
        s = sa_merge(s, q);
    }
    if (lane == 0) s_w[warp] = s;
    __syncthreads();
    if (tid == 0) {
        ShiftAcc a = s_w[0];
        for (int w = 1; w < NB / 32; ++w) a = sa_merge(a, s_w[w]);
        double *pp = part + (row * B + j) * 3;
        pp[0] = (double)a.m;
        pp[1] = a.sf;
        pp[2] = a.sgf;
        __threadfence();
        s_last = atomicAdd(&ticket[row], 1u) == (unsigned)B - 1;
    }
    __syncthreads();
    if (!s_last || tid != 0) return;
    __threadfence();
    ShiftAcc a{CUDART_INF_F, 0.0, 0.0};
    for (int64_t q = 0; q < B; ++q) {
        const double *pp = part + (row * B + q) * 3;
        ShiftAcc c{(float)__ldcg(pp), __ldcg(pp + 1), __ldcg(pp + 2)};
        a = sa_merge(a, c);
    }
    lam[row] = a.sgf / a.sf;
}

__global__ void __launch_bounds__(NB)
noalloc_apply_kernel(const float *__restrict__ r, const double *__restrict__ b_in,
                     const float *__restrict__ g, int64_t n, int64_t B, double inv_t,
                     const unsigned char *scratch, int64_t rows, float *__restrict__ grad) {
    const double *lam_all = reinterpret_cast<const double *>(scratch) + rows * B * 3;
    const int64_t row = blockIdx.x / B, j = blockIdx.x % B;
    const float *rr = r + row * n;
    const float *gg = g + row * n;
    float *out = grad + row * n;
    const XForm xf = make_xform(b_in[row], inv_t * LOG2E);
    const double lam = lam_all[row];
    const float lam_hi = (float)lam, lam_lo = (float)(lam - (double)lam_hi);
    const float hit = vjp_scale2(inv_t);   // log2(1/(2t))
    for (int64_t i = j * NB + threadIdx.x; i < n; i += B * NB)
        out[i] = vjp_term2(xf(rr[i]), gg[i], hit, lam_hi, lam_lo);
}

// Per-device address of the scratch array, resolved once.
std::mutex g_mu;
void *g_addr[64];
bool g_ready[64];

int scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LAPSUM_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_ready[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LAPSUM_ERR_CUDA;
        g_addr[dev] = p;
        g_ready[dev] = true;
    }
    *out = g_addr[dev];
    return LAPSUM_OK;
}

}  // namespace
}  // namespace lapsum

using namespace lapsum;

extern "C" int lapsum_backward_noalloc(const float *scores, const double *b, const float *g,
                                       int64_t rows, int64_t n, double t, float *grad_out,
                                       struct CUstream_st *stream_in) {
    if (!scores || !b || !g || !grad_out || rows < 1 || n < 1 || n >= (int64_t(1) << 31))
        return LAPSUM_ERR_ARG;
    if (!(t >= LAPSUM_T_MIN && t <= LAPSUM_T_MAX)) return LAPSUM_ERR_ARG;
    // blocks per row: about four per SM in total, at least one per row
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t B = (4 * (int64_t)sms + rows - 1) / rows;
    const int64_t per_row_max = (n + NB - 1) / NB;
    if (B > per_row_max) B = per_row_max;
    if (B < 1) B = 1;
    if (scratch_need(rows, B) > (size_t)LAPSUM_NOALLOC_SCRATCH_BYTES) return LAPSUM_ERR_ARG;
    if ((int64_t)rows * B > (int64_t)0x7fffffff) return LAPSUM_ERR_ARG;
    void *addr = nullptr;
    int rc = scratch_address(&addr);
    if (rc) return rc;
    unsigned char *scratch = static_cast<unsigned char *>(addr);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_in);
    unsigned *ticket = reinterpret_cast<unsigned *>(scratch + (size_t)rows * B * 3 * sizeof(double) +
                                                   (size_t)rows * sizeof(double));
    if (cudaMemsetAsync(ticket, 0, (size_t)rows * sizeof(unsigned), st) != cudaSuccess) return LAPSUM_ERR_CUDA;
    const unsigned grid = (unsigned)(rows * B);
    noalloc_reduce_kernel<<<grid, NB, 0, st>>>(scores, b, g, n, B, 1.0 / t, scratch, rows);
    if (cudaGetLastError() != cudaSuccess) return LAPSUM_ERR_CUDA;
    noalloc_apply_kernel<<<grid, NB, 0, st>>>(scores, b, g, n, B, 1.0 / t, scratch, rows, grad_out);
    if (cudaGetLastError() != cudaSuccess) return LAPSUM_ERR_CUDA;
    return LAPSUM_OK;
}
