// lapsum_kernels.h -- host-side launchers of the kernels (internal).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "lapsum_internal.h"

namespace lapsum {

// Launch with programmatic stream serialization (the kernel calls pdl_enter()
// before touching its predecessor's results).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                            Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// A cooperative launch (every CTA resident at once, so CTAs may wait on one
// another at grid barriers).  With programmatic stream serialization as well
// when the runtime takes the pair (the kernel's CTAs are then scheduled while
// its predecessor drains, and wait for it with griddepcontrol.wait before any
// grid barrier); if it refuses the pair, a plain cooperative launch in stream
// order (the refusal is remembered per device).
bool coop_pdl_refused();
void coop_pdl_refuse();
template <typename... KArgs, typename... Args>
inline cudaError_t launch_coop(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                               Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = coop_pdl_refused() ? 1 : 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
    if (e != cudaSuccess && cfg.numAttrs == 2 &&
        (e == cudaErrorInvalidValue || e == cudaErrorNotSupported || e == cudaErrorInvalidConfiguration)) {
        (void)cudaGetLastError();   // the launch did not happen: try without the pair
        coop_pdl_refuse();
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
    }
    return e;
}

// Per-device launch set-up (lapsum_api.cu), cached per (device, kernel) under a
// lock, so a process that drives several GPUs configures each one:
int device_sm_count();   // SMs of the current device
cudaError_t set_max_dynamic_smem(const void *kern, size_t bytes);   // once per (device, kernel, size)
// CTAs of `kern` (block threads, dynamic smem bytes) resident on the current device at once
cudaError_t resident_ctas(const void *kern, int threads, size_t smem, int *out);

// in-CTA full-sort solver (k_rows.cu)
int rowsolve_capacity();
cudaError_t launch_rowsolve_rows(const float *scores, int64_t rows, int64_t n, double k, double t,
                                 float *p, double *b, Ctl *ctl, cudaStream_t st);
// band solve of the bracketing path, one CTA per row (k_band.cu)
cudaError_t launch_band_select(const float *band, int64_t rows, double k, double t, Ctl *ctl, int64_t band_cap,
                               int32_t round2, cudaStream_t st);
cudaError_t launch_rowvjp(const float *scores, const double *b, const float *g, int64_t rows,
                          int64_t n, double t, float *grad, cudaStream_t st);

// bracketing pipeline and streaming passes (k_bracket.cu)
int stream_grid();
int64_t partial_stride(int64_t rows);   // doubles of per-block partials per row
cudaError_t launch_sample(const BracketParams &P, cudaStream_t st);
cudaError_t launch_select(const BracketParams &P, cudaStream_t st);
int select_cand_capacity();
cudaError_t launch_stream_pass(const BracketParams &P, cudaStream_t st);
cudaError_t launch_certify(const BracketParams &P, cudaStream_t st);
cudaError_t launch_p_pass(const float *r, int64_t rows, int64_t n, double t, float *p, double *b_out, Ctl *ctl,
                          double *partials, cudaStream_t st);
cudaError_t launch_vjp_reduce(const float *r, const double *b, const float *g, int64_t rows, int64_t n, double t,
                              Ctl *ctl, double *partials, cudaStream_t st);
cudaError_t launch_selftest_math(int which, const double *in, double *out, double *ref, int64_t n,
                                cudaStream_t st);
// one slice of a split row: {sum e, sum g e, min |x2|} with terms 2^{sh2 - |x2|}
// (ctl->vjp_min and ticket[3] of the row's control block must start at +inf / 0)
cudaError_t launch_vjp_slice_partial(const float *r, const double *b, const float *g, int64_t n, double t,
                                     float sh2, Ctl *ctl, double *partials, double *part_out, cudaStream_t st);
cudaError_t launch_vjp_apply(const float *r, const double *b, const float *g, int64_t rows, int64_t n, double t,
                             const Ctl *ctl, float *grad, cudaStream_t st);

// device-wide radix sort + locate-scan (k_radix.cu)
enum Gate : int32_t { GATE_ALWAYS = 0, GATE_FALLBACK = 2 };
struct SortArgs {
    const float *src;          // fp32 scores (keys made on the fly) of row 0
    int64_t src_stride;        // floats from one row's source to the next
    int64_t rows;              // rows the kernel walks, one after another (each gated)
    int64_t n_host;            // element count
    int64_t cap;               // upper bound of the element count (grid sizing)
    uint32_t *keys[2];         // ping-pong key buffers [cap]: the workspace's, and the caller's p output
    unsigned long long *hist;  // [4][256], then two words: sorts that gave up, and that count at the last clean-up,
                               // then four: per sign class, the OR of the keys and of their complements
    uint32_t *chunkcnt;        // [4][256][grid]: digit counts of each CTA's chunk of tiles
    double *tilebuf;           // locate per-tile data
    Ctl *ctl;
    int32_t gate;
    int32_t spin_cap;          // grid-barrier polls before a wait gives up
    double k, t;               // budget and temperature (all-equal shortcut)
};
int sort_grid_max();
int64_t sort_record_doubles(int64_t cap);
cudaError_t launch_radix_sort(SortArgs &A, double k, double t, cudaStream_t st);

}  // namespace lapsum
