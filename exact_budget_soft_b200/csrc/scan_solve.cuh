// scan_solve.cuh -- in-CTA merge sort and the threshold-curve scan/solve
// (full-sort solver of "Fast LapSum: Exact Differentiable Top-k at Million
// Scale", technical summary section 2.2), shared by the one-CTA row solver and
// the last CTA of the device-wide locate kernel.
#pragma once
#include <cstdint>

#include "lapsum_device.cuh"

namespace lapsum {

// Shared-memory slot of sorted position j: one pad word per 32 keys, so a thread
// walking its own run of consecutive positions hits a different bank from its
// neighbours (the scan reads runs; unpadded, all 32 lanes would share a bank).
__device__ __forceinline__ int spad(int j) { return j + (j >> 5); }

template <int BLOCK, int KPT>
struct RowCfg {
    static constexpr int NW = BLOCK / 32;
    static constexpr int CAP = BLOCK * KPT;
    static constexpr int SEG = 32 * KPT;   // keys per warp segment
    static constexpr size_t SMEM_KEYS = size_t(CAP + CAP / 32) * 4;
    static constexpr size_t SMEM_HIST = size_t(NW) * 256 * 4;
    static constexpr size_t SMEM = SMEM_KEYS + SMEM_HIST + 256 * 4 + 2048;
};

// Ascending sorting network on N keys in registers (bitonic: log2 N (log2 N + 1)/2
// stages of N/2 compare-exchanges; every index is a compile-time constant).
template <int N>
__device__ __forceinline__ void bitonic_regs(uint32_t (&k)[N]) {
#pragma unroll
    for (int kk = 2; kk <= N; kk <<= 1) {
#pragma unroll
        for (int j = kk >> 1; j > 0; j >>= 1) {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const uint32_t a = k[i], b = k[l];
                    const uint32_t lo = min(a, b), hi = max(a, b);
                    if ((i & kk) == 0) { k[i] = lo; k[l] = hi; } else { k[i] = hi; k[l] = lo; }
                }
            }
        }
    }
}

// Merges the 32 lanes' ascending runs of KPT keys (KPT a power of two) into one
// ascending run of 32 KPT keys, lane l holding positions l KPT .. l KPT + KPT - 1:
// the phases of a bitonic sorting network, each opening with a stage that
// compares a key with its mirror image in the phase's block (so that both halves
// may come in ascending), then half-cleaners -- across lanes by shuffles, then
// within each lane's registers.  No branch depends on the data.
template <int KPT>
__device__ __forceinline__ void warp_bitonic_merge(uint32_t (&k)[KPT]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {   // blocks of 2m lanes
        const bool lower = (lane & m) == 0;
#pragma unroll
        for (int i = 0; i < KPT / 2; ++i) {   // key i against the partner's key KPT - 1 - i, and back
            const uint32_t a = k[i], b = k[KPT - 1 - i];
            const uint32_t pa = __shfl_xor_sync(FULL, b, 2 * m - 1), pb = __shfl_xor_sync(FULL, a, 2 * m - 1);
            k[i] = lower ? min(a, pa) : max(a, pa);
            k[KPT - 1 - i] = lower ? min(b, pb) : max(b, pb);
        }
#pragma unroll
        for (int h = m >> 1; h > 0; h >>= 1) {   // lanes h apart
            const bool lo = (lane & h) == 0;
#pragma unroll
            for (int i = 0; i < KPT; ++i) {
                const uint32_t v = __shfl_xor_sync(FULL, k[i], h);
                k[i] = lo ? min(k[i], v) : max(k[i], v);
            }
        }
#pragma unroll
        for (int j = KPT >> 1; j > 0; j >>= 1) {   // registers j apart
#pragma unroll
            for (int i = 0; i < KPT; ++i) {
                if ((i & j) == 0) {
                    const uint32_t a = k[i], b = k[i | j];
                    k[i] = min(a, b);
                    k[i | j] = max(a, b);
                }
            }
        }
    }
}

// Block-wide merge sort of KPT keys per thread (ascending), the alternative to
// the radix sort for one CTA's row: each thread sorts its keys in registers
// (bitonic network), each warp merges its lanes' runs in registers
// (warp_bitonic_merge), then log2(BLOCK / 32) merge levels double the sorted runs
// in shared memory.  At a level of runs of L, thread t produces outputs
// [KPT t, KPT t + KPT) of the merge of its pair of runs: it finds where its
// outputs start by a binary search on the merge path (the first i with
// A[i] > B[o - i - 1]) and then merges KPT elements sequentially: a compare, a
// select and a shared-memory load per output.  On return the sorted keys are in
// s_keys (position j at spad(j)).
template <int BLOCK, int KPT>
__device__ __forceinline__ void block_merge_sort(uint32_t (&key)[KPT], uint32_t *s_keys) {
    constexpr int CAP = BLOCK * KPT;
    const int tid = threadIdx.x;
    bitonic_regs<KPT>(key);
    warp_bitonic_merge<KPT>(key);
#pragma unroll
    for (int q = 0; q < KPT; ++q) s_keys[spad(KPT * tid + q)] = key[q];
    __syncthreads();
#pragma unroll 1
    for (int L = 32 * KPT; L < CAP; L <<= 1) {
        const int out0 = KPT * tid;
        const int base = out0 & ~(2 * L - 1);
        const int o = out0 - base;                 // output offset within the pair's merge
        const int A0 = base, B0 = base + L;        // the pair's two sorted runs of L keys
        int lo = o > L ? o - L : 0, hi = o < L ? o : L;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (s_keys[spad(A0 + mid)] <= s_keys[spad(B0 + o - mid - 1)]) lo = mid + 1;
            else hi = mid;
        }
        int i = lo, j = o - lo;
        uint32_t a = i < L ? s_keys[spad(A0 + i)] : 0u, b = j < L ? s_keys[spad(B0 + j)] : 0u;
#pragma unroll
        for (int q = 0; q < KPT; ++q) {
            const bool ta = i < L && (j >= L || a <= b);
            key[q] = ta ? a : b;
            if (ta) {
                ++i;
                a = i < L ? s_keys[spad(A0 + i)] : 0u;
            } else {
                ++j;
                b = j < L ? s_keys[spad(B0 + j)] : 0u;
            }
        }
        __syncthreads();   // every thread has read its inputs
#pragma unroll
        for (int q = 0; q < KPT; ++q) s_keys[spad(out0 + q)] = key[q];
        __syncthreads();
    }
}

// Solve the sorted values held in s_keys (position j at spad(j); descending scores).
//   m0      scores above the first value (band: the count at or above a_R)
//   top     value above c_0 that P_top refers to (a_R, or +inf)
//   P_top   sum_{scores above} e^{(top - r)/t}
//   bot     value below c_{n-1} that Q_bot refers to (a_L, or -inf)
//   Q_bot   sum_{scores below} e^{(r - bot)/t}
// Returns b in thread 0 (and j_star = index of the last value >= b, -1 if none).
// Requires n >= 1.
template <int BLOCK, int KPT>
__device__ double block_scan_solve(const uint32_t *s_keys, int n, double k, double t, double inv_t,
                                   double m0, double top, double P_top, double bot, double Q_bot,
                                   void *scratch_v, int64_t *j_star_out, int32_t *status,
                                   const double *tab) {
    const double s2d = inv_t * LOG2E;
    constexpr int R = KPT;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    Aff *sc = reinterpret_cast<Aff *>(scratch_v);               // 2*NW Aff
    int *s_int = reinterpret_cast<int *>(sc + 2 * (BLOCK / 32)); // [0]: r*, [1..NW]: per warp
    double *s_dbl = reinterpret_cast<double *>(s_int + 40);      // handoff

    auto val = [&](int j) -> double {
        if (j < 0) return top;
        if (j >= n) return bot;
        return (double)desc_key_to_float(s_keys[spad(j)]);
    };
    // link d_j = e^{(c_{j+1} - c_j)/t}, j in [-1, n-1] (virtual top/bottom at the ends)
    auto link = [&](int j) -> double {
        double hi = val(j), lo = val(j + 1);
        if (hi == CUDART_INF || lo == -CUDART_INF) return 0.0;
        return link_exp((hi - lo) * s2d, tab);
    };

    const int j0 = tid * R;
    const int j1 = min(j0 + R, n) - 1;   // run [j0, j1], empty if j1 < j0
    Aff mp = aff_id(), mq = aff_id();
    double d_out = 0.0;
    if (j0 < n) {
        // P: x -> 1 + d_{j-1} x for j = j0..j1; Q: x -> 1 + d_j x, composed right-to-left
        double dprev = link(j0 - 1);
        double cprev = val(j0);
        for (int j = j0; j <= j1; ++j) {
            mp = {mp.a * dprev, fma(mp.s, dprev, 1.0)};
            double cn = val(j + 1);
            double d = (cprev == CUDART_INF || cn == -CUDART_INF) ? 0.0 : link_exp((cprev - cn) * s2d, tab);
            // append Q-map of j on the right: T(x) = A(1 + d x) + S
            mq = {mq.a * d, mq.s + mq.a};
            dprev = d;
            cprev = cn;
        }
        d_out = dprev;   // d_{j1}
    }
    Aff pe, qe;
    block_scan_excl_both<BLOCK>(mp, mq, pe, qe, sc);
    const double P_in = fma(pe.a, P_top, pe.s);        // P_{j0-1}
    const double Q_after = fma(qe.a, Q_bot, qe.s);     // Q_{j1+1}
    const double P_end = fma(mp.a, P_in, mp.s);        // P_{j1}
    // G at the run end
    int cand = -1;
    if (j0 < n) {
        double G = (m0 + (double)(j1 + 1)) - 0.5 * P_end + 0.5 * d_out * Q_after;
        if (G <= k) cand = tid;
    }
    // r* = max candidate run
    cand = warp_max_int(cand);
    if (lane == 0) s_int[1 + warp] = cand;
    __syncthreads();
    if (tid == 0) {
        int m = -1;
        for (int w = 0; w < BLOCK / 32; ++w) m = max(m, s_int[1 + w]);
        s_int[0] = m;
    }
    __syncthreads();
    const int rstar = s_int[0];
    const int nruns = (n + R - 1) / R;
    const int rr = rstar + 1;   // run holding the crossing (== nruns: below the last value)
    if (tid == rr) {
        s_dbl[0] = P_in;
        s_dbl[1] = Q_after;
    }
    if (rr == nruns && tid == nruns - 1) {   // crossing between c_{n-1} and the bottom
        s_dbl[0] = P_end;
    }
    __syncthreads();
    double b = 0.0;
    if (warp == 0) {
        double U, L, A, PU, QL, ed;
        int jstar;
        if (rr >= nruns) {
            jstar = n - 1;
            U = val(n - 1);
            L = bot;
            A = m0 + n;
            PU = s_dbl[0];
            QL = Q_bot;
            ed = link(n - 1);
        } else {
            const int r0 = rr * R;
            const int cnt = min(R, n - r0);
            const double Pin = s_dbl[0], Qaft = s_dbl[1];
            const int j = r0 + lane;
            const bool act = lane < cnt;
            double din = act ? link(j - 1) : 1.0;       // d_{j-1}
            double dj = act ? link(j) : 1.0;            // d_j
            Aff pm = act ? Aff{din, 1.0} : aff_id();
            Aff qm = act ? Aff{dj, 1.0} : aff_id();
            pm = warp_scan_fwd(pm, lane);
            qm = warp_scan_bwd(qm, lane);
            double Pj = fma(pm.a, Pin, pm.s);           // P_j
            double Qj = fma(qm.a, Qaft, qm.s);          // Q_j
            double Qn = __shfl_down_sync(FULL, Qj, 1);  // Q_{j+1}
            if (lane == cnt - 1) Qn = Qaft;
            double G = (m0 + (double)(j + 1)) - 0.5 * Pj + 0.5 * dj * Qn;
            unsigned bal = __ballot_sync(FULL, act && G <= k);
            int hl = bal ? 31 - __clz(bal) : -1;         // last lane with G_j <= k
            double Q0 = __shfl_sync(FULL, Qj, 0);
            double d0 = __shfl_sync(FULL, din, 0);
            double Ph = __shfl_sync(FULL, Pj, hl < 0 ? 0 : hl);
            double Qh = __shfl_sync(FULL, Qn, hl < 0 ? 0 : hl);
            double dh = __shfl_sync(FULL, dj, hl < 0 ? 0 : hl);
            if (hl < 0) {   // crossing between c_{r0-1} (or the top) and c_{r0}
                jstar = r0 - 1;
                U = val(r0 - 1);
                L = val(r0);
                A = m0 + r0;
                PU = Pin;
                QL = Q0;
                ed = d0;
            } else {
                jstar = r0 + hl;
                U = val(jstar);
                L = val(jstar + 1);
                A = m0 + jstar + 1;
                PU = Ph;
                QL = Qh;
                ed = dh;
            }
        }
        if (lane == 0) {
            if (jstar == -1 && U != CUDART_INF) {   // b between c_0 and top: needs G(top) <= k
                const double Gt = A - 0.5 * PU + 0.5 * ed * QL;
                if (Gt > k && status) atomicOr(status, ST_NO_ROOT);
            }
            if (jstar == n - 1 && L != -CUDART_INF) {
                double Gb = (m0 + n) - 0.5 * ed * PU + 0.5 * Q_bot;
                if (Gb < k && status) atomicOr(status, ST_NO_ROOT);
            }
            b = solve_interval(U, L, A, PU, QL, ed, k, t);
            if (j_star_out) *j_star_out = jstar;
        }
    }
    return b;
}

}  // namespace lapsum
