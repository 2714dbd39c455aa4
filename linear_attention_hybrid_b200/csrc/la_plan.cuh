// Work planning for the segment split, and the scan that chains segment states.
//
// A sequence is cut into coarse segments (one CTA of the main chunk kernel per
// segment and head) and each coarse segment into R fine units of sub_len tokens
// (a multiple of the 128-token chunk). This is the single-GPU form of the
// report's "local recursion + global correction" (Ling & Ring 2.6 Technical
// Report, blog post news.neo-ai.one/en/article/3021, section "Long-Context
// Training: Context Parallel for Lightning Attention"):
//   1. every fine unit that lies before its sequence's last coarse segment gets
//      its state dS_f from a zero start (state kernel);
//   2. la_seg_scan_kernel chains them, S_{f+1} = lambda^(L_f) S_f + dS_f from the
//      initial state, and stores the state entering each coarse segment in the
//      slot of that segment's first fine unit;
//   3. the main kernel runs each coarse segment from that state.
// Uniform batches (nseq sequences of N tokens) map unit indices arithmetically;
// packed varlen batches use the lists built by la_plan_kernel.
#pragma once

#include "la_ptx.cuh"

namespace la {

enum UnitFlags { kUnitFirst = 1, kUnitLast = 2 };  // coarse: first / last segment of its sequence
enum FineFlags { kFineFirst = 1, kFineInLast = 2 };  // fine: first of its sequence / inside the last segment

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
    const int flags = (f == 0 ? kFineFirst : 0) | (f / m.R == m.nc - 1 ? kFineInLast : 0);
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
                const int flags = (f == 0 ? kFineFirst : 0) | (f / R == nc - 1 ? kFineInLast : 0);
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

// grid (H, min(nseq, 65535)), kScanThreads threads: one CTA walks one (sequence,
// head) through its fine units, each thread owning D*D / kScanThreads state
// entries. At the start of coarse segment j (fine unit jR) the state entering
// it replaces dS in that unit's workspace slot; the walk stops at the last
// segment. Sequences with a single segment are left to the main kernel. Unit
// indices are clamped to the plan, so no slot past the workspace is touched
// even when a malformed cu_seqlens over-counts units.
constexpr int kScanThreads = 1024;

template <int D>
__global__ void __launch_bounds__(kScanThreads) la_seg_scan_kernel(const WorkMap m, int H, const float *s_init,
                                                                   const float *slopes, float *seg_state) {
    constexpr int kVec = D * D / 4 / kScanThreads;  // float4 per thread
    const int h = blockIdx.x;
    const float g = decay_log2(slopes, h, H);
    for (int seq = blockIdx.y; seq < m.nseq; seq += gridDim.y) {
        int ff, nf, nc;
        if (m.fine) {
            const int cf = m.counts[0];
            const int lo = min(m.seq_fine[seq], cf), hi = min(m.seq_fine[seq + 1], cf);
            ff = lo;
            nf = hi - lo;
            nc = m.seq_coarse[seq + 1] - m.seq_coarse[seq];
        } else {
            ff = seq * m.nf;
            nf = m.nf;
            nc = m.nc;
        }
        if (nc <= 1) continue;
        float4 S[kVec];
#pragma unroll
        for (int v = 0; v < kVec; ++v) {
            const int e = threadIdx.x + v * kScanThreads;
            S[v] = s_init ? reinterpret_cast<const float4 *>(s_init + (static_cast<size_t>(seq) * H + h) * D * D)[e]
                          : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int f = 0; f < nf; ++f) {
            const int u = ff + f;
            const int j = f / m.R;
            float4 *slot = reinterpret_cast<float4 *>(seg_state + (static_cast<size_t>(u) * H + h) * D * D);
            const bool in_last = (j >= nc - 1);
            float4 d[kVec];
#pragma unroll
            for (int v = 0; v < kVec; ++v)
                d[v] = in_last ? make_float4(0.f, 0.f, 0.f, 0.f) : slot[threadIdx.x + v * kScanThreads];
            if (f % m.R == 0) {
#pragma unroll
                for (int v = 0; v < kVec; ++v) slot[threadIdx.x + v * kScanThreads] = S[v];
            }
            if (in_last) break;
            int4 fu;
            if (!fine_unit(m, u, fu)) break;
            const float lamL = exp2f(g * static_cast<float>(fu.y));
#pragma unroll
            for (int v = 0; v < kVec; ++v) {
                S[v].x = fmaf(lamL, S[v].x, d[v].x);
                S[v].y = fmaf(lamL, S[v].y, d[v].y);
                S[v].z = fmaf(lamL, S[v].z, d[v].z);
                S[v].w = fmaf(lamL, S[v].w, d[v].w);
            }
        }
    }
}

}  // namespace la
