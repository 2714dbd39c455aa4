// Work planning for the segment split, and the scan that chains segment states.
//
// A sequence is cut into coarse segments (one CTA of the main chunk kernel per
// segment and head) and each coarse segment into R fine units of sub_len tokens
// (a multiple of the 128-token chunk). This is the single-GPU form of the
// report's "local recursion + global correction" (Ling & Ring 2.6 Technical
// Report, blog post news.neo-ai.one/en/article/3021, section "Long-Context
// Training: Context Parallel for Lightning Attention"):
//   1. every fine unit f that lies before its sequence's last coarse segment gets
//      its state dS_f from a zero start (state kernel); the first unit of a
//      sequence also folds in the decayed initial state and keeps a copy of it;
//   2. the main kernel's CTA for coarse segment j forms the state entering it,
//      sum over earlier units f of lambda^(tokens from the end of f to the
//      segment start) dS_f (the "global correction"), and runs the segment.
// Uniform batches (nseq sequences of N tokens) map unit indices arithmetically;
// packed varlen batches use the lists built by la_plan_kernel.
#pragma once

#include "la_ptx.cuh"

namespace la {

enum UnitFlags { kUnitFirst = 1, kUnitLast = 2 };  // coarse: first / last segment of its sequence
// fine: first / last unit of its sequence, inside its sequence's last / first segment
enum FineFlags { kFineFirst = 1, kFineInLast = 2, kFineInFirst = 4, kFineLast = 8 };

struct WorkMap {
    // packed batches: lists written by la_plan_kernel (null for uniform batches)
    const int4 *fine;        // {tok0, len, seq, flags}
    const int4 *coarse;      // {tok0, len, seq, flags | first_fine << 2}
    const int *seq_fine;     // [nseq + 1] first fine unit of each sequence
    const int *seq_coarse;   // [nseq + 1] first coarse unit of each sequence
    const int *counts;       // [2] fine and coarse units planned
    // uniform batches
    int N;                   // tokens per sequence (0 for packed batches)
    int nf, nc;              // fine / coarse units per sequence (uniform batches)
    // both
    int nseq;
    int sub_len;             // fine unit length
    int R;                   // fine units per coarse segment
    int all_units;           // state pass: compute every fine unit's state (a shard's units)
};

__device__ __forceinline__ bool fine_unit(const WorkMap &m, int u, int4 &out) {
    if (m.fine) {
        if (u >= m.counts[0]) return false;
        out = m.fine[u];
        return true;
    }
    const int seq = u / m.nf, f = u - seq * m.nf;
    if (seq >= m.nseq) return false;
    const int len = max(0, min(m.sub_len, m.N - f * m.sub_len));
    const int flags = (f == 0 ? kFineFirst : 0) | (f / m.R == m.nc - 1 ? kFineInLast : 0) |
                      (f / m.R == 0 ? kFineInFirst : 0) | (f == m.nf - 1 ? kFineLast : 0);
    out = make_int4(seq * m.N + f * m.sub_len, len, seq, flags);
    return true;
}

// Coarse unit w: {tok0, len, seq, flags}; first_fine = index of its first fine unit.
__device__ __forceinline__ bool coarse_unit(const WorkMap &m, int w, int4 &out, int &first_fine) {
    if (m.coarse) {
        if (w >= m.counts[1]) return false;
        const int4 c = m.coarse[w];
        out = make_int4(c.x, c.y, c.z, c.w & 3);
        first_fine = c.w >> 2;
        return true;
    }
    const int seq = w / m.nc, j = w - seq * m.nc;
    if (seq >= m.nseq) return false;
    const int seg = m.R * m.sub_len;
    const int len = max(0, min(seg, m.N - j * seg));
    const int flags = (j == 0 ? kUnitFirst : 0) | (j == m.nc - 1 ? kUnitLast : 0);
    out = make_int4(seq * m.N + j * seg, len, seq, flags);
    first_fine = seq * m.nf + j * m.R;
    return true;
}

// First fine unit of sequence `seq`.
__device__ __forceinline__ int seq_first_fine(const WorkMap &m, int seq) {
    return m.fine ? m.seq_fine[seq] : seq * m.nf;
}

// One past the last fine unit of sequence `seq`.
__device__ __forceinline__ int seq_end_fine(const WorkMap &m, int seq) {
    return m.fine ? m.seq_fine[seq + 1] : (seq + 1) * m.nf;
}

constexpr int kPlanThreads = 1024;

// Inclusive block-wide sum scan of one int per thread (kPlanThreads threads).
__device__ __forceinline__ int block_inclusive_scan(int x, int *warp_sums) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[w] = x;
    __syncthreads();
    if (w == 0) {
        int s = warp_sums[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        warp_sums[lane] = s;
    }
    __syncthreads();
    const int r = x + (w > 0 ? warp_sums[w - 1] : 0);
    __syncthreads();
    return r;
}

// One CTA, packed batches. Sequence i spans tokens [cu[i], cu[i+1]); it gets
// nf_i = max(1, ceil(len_i / sub_len)) fine units and ceil(nf_i / R) coarse
// segments (a zero-length sequence still gets one of each, so that its state is
// passed through). A malformed cu is clamped into [0, T] and recorded.
__global__ void __launch_bounds__(kPlanThreads) la_plan_kernel(const int32_t *cu, int nseq, int T, int sub_len, int R,
                                                              int cap_fine, int cap_coarse, int4 *fine, int4 *coarse,
                                                              int *seq_fine, int *seq_coarse, int *counts) {
    __shared__ int warp_sums[32];
    __shared__ int run_f, run_c;
    if (threadIdx.x == 0) run_f = run_c = 0;
    __syncthreads();
    bool bad = false;
    for (int base = 0; base < nseq; base += kPlanThreads) {
        const int i = base + threadIdx.x;
        int a = 0, b = 0;
        if (i < nseq) {
            const int ra = cu[i], rb = cu[i + 1];
            if ((i == 0 && ra != 0) || rb < ra || (i == nseq - 1 && rb != T)) bad = true;
            a = min(max(ra, 0), T);
            b = min(max(rb, a), T);
        }
        const int len = b - a;
        const int nf = i < nseq ? max(1, (len + sub_len - 1) / sub_len) : 0;
        const int nc = (nf + R - 1) / R;
        const int incl_f = block_inclusive_scan(nf, warp_sums);
        const int incl_c = block_inclusive_scan(nc, warp_sums);
        const int ff = run_f + incl_f - nf, fc = run_c + incl_c - nc;
        if (i < nseq) {
            seq_fine[i] = ff;
            seq_coarse[i] = fc;
            for (int f = 0; f < nf; ++f) {
                if (ff + f >= cap_fine) {
                    bad = true;
                    break;
                }
                const int flags = (f == 0 ? kFineFirst : 0) | (f / R == nc - 1 ? kFineInLast : 0) |
                                  (f / R == 0 ? kFineInFirst : 0) | (f == nf - 1 ? kFineLast : 0);
                fine[ff + f] = make_int4(a + f * sub_len, max(0, min(sub_len, len - f * sub_len)), i, flags);
            }
            const int seg = R * sub_len;
            for (int j = 0; j < nc; ++j) {
                if (fc + j >= cap_coarse || ff + j * R >= cap_fine) {
                    bad = true;
                    break;
                }
                const int flags = (j == 0 ? kUnitFirst : 0) | (j == nc - 1 ? kUnitLast : 0);
                coarse[fc + j] = make_int4(a + j * seg, max(0, min(seg, len - j * seg)), i, flags | ((ff + j * R) << 2));
            }
        }
        __syncthreads();
        if (threadIdx.x == kPlanThreads - 1) {
            run_f += incl_f;
            run_c += incl_c;
        }
        __syncthreads();
    }
    if (bad) record_status(1 /* LA_ERR_INVALID_ARGUMENT */);
    if (threadIdx.x == 0) {
        seq_fine[nseq] = run_f;
        seq_coarse[nseq] = run_c;
        counts[0] = min(run_f, cap_fine);
        counts[1] = min(run_c, cap_coarse);
    }
}

}  // namespace la
