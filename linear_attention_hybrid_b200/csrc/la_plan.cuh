// Work planning for the segment split, and the scan that chains segment states.
//
// A sequence is cut into segments of `seg_len` tokens (a multiple of the
// 128-token chunk). Each (segment, head) is one CTA of the chunk kernel. The
// single-GPU form of the report's "local recursion + global correction"
// (Ling & Ring 2.6 Technical Report, blog post news.neo-ai.one/en/article/3021,
// section "Long-Context Training: Context Parallel for Lightning Attention"):
//   1. every segment but the last of each sequence computes its state dS from
//      a zero start (chunk kernel, state-only pass);
//   2. la_seg_scan_kernel turns those into the state entering each segment,
//      S_in[0] = S0, S_in[j+1] = lambda^(L_j) S_in[j] + dS_j;
//   3. the chunk kernel runs every segment from its S_in.
#pragma once

#include "la_ptx.cuh"

namespace la {

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

// One CTA. Sequence i spans tokens [cu[i], cu[i+1]) (or [i*N, (i+1)*N) when cu
// is null). Writes units[] = {tok0, len, seq, flags} for every segment of
// every sequence (a zero-length sequence still gets one unit so that its state
// is passed through), seq_first[i] = index of its first unit, seq_first[nseq]
// = total, and *n_units. A malformed cu is clamped into [0, T] and recorded.
__global__ void __launch_bounds__(kPlanThreads) la_plan_kernel(const int32_t *cu, int nseq, int N_uniform, int T,
                                                              int seg_len, int cap, int4 *units, int *seq_first,
                                                              int *n_units) {
    __shared__ int warp_sums[32];
    __shared__ int running;
    if (threadIdx.x == 0) running = 0;
    __syncthreads();
    bool bad = false;
    for (int base = 0; base < nseq; base += kPlanThreads) {
        const int i = base + threadIdx.x;
        int a = 0, b = 0;
        if (i < nseq) {
            if (cu) {
                const int ra = cu[i], rb = cu[i + 1];
                if ((i == 0 && ra != 0) || rb < ra || (i == nseq - 1 && rb != T)) bad = true;
                a = min(max(ra, 0), T);
                b = min(max(rb, a), T);
            } else {
                a = i * N_uniform;
                b = a + N_uniform;
            }
        }
        const int len = b - a;
        const int nseg = i < nseq ? max(1, (len + seg_len - 1) / seg_len) : 0;
        const int incl = block_inclusive_scan(nseg, warp_sums);
        const int first = running + incl - nseg;
        if (i < nseq) {
            seq_first[i] = first;
            for (int j = 0; j < nseg; ++j) {
                const int uidx = first + j;
                if (uidx >= cap) {
                    bad = true;
                    break;
                }
                const int flags = (j == 0 ? kUnitFirst : 0) | (j == nseg - 1 ? kUnitLast : 0);
                units[uidx] = make_int4(a + j * seg_len, min(seg_len, len - j * seg_len), i, flags);
            }
        }
        __syncthreads();
        if (threadIdx.x == kPlanThreads - 1) running += incl;
        __syncthreads();
    }
    if (bad) record_status(1 /* LA_ERR_INVALID_ARGUMENT */);
    if (threadIdx.x == 0) {
        seq_first[nseq] = running;
        *n_units = min(running, cap);
    }
}

// grid (D*D/4/256, H, min(nseq, 65535)), 256 threads: each thread walks one
// float4 of the state of one (sequence, head) through that sequence's
// segments, replacing dS_j in the workspace by the state S_in[j] entering
// segment j. Sequences with a single segment are left to the chunk kernel.
// Unit indices are clamped to the plan size, so no slot past the workspace is
// touched even when a malformed cu_seqlens over-counts segments.
template <int D>
__global__ void __launch_bounds__(256) la_seg_scan_kernel(const int4 *units, const int *seq_first,
                                                          const int *n_units, int nseq, int H, const float *s_init,
                                                          const float *slopes, float *seg_state) {
    constexpr int kVec = D * D / 4;
    const int e = blockIdx.x * 256 + threadIdx.x;
    const int h = blockIdx.y;
    if (e >= kVec) return;
    const float g = decay_log2(slopes, h, H);
    const int nu = *n_units;
    for (int seq = blockIdx.z; seq < nseq; seq += gridDim.z) {
        // units beyond the plan's capacity exist only for a malformed cu_seqlens: never index past it
        const int l = min(seq_first[seq + 1], nu);
        const int f = min(seq_first[seq], l);
        if (l - f <= 1) continue;
        float4 S = make_float4(0.f, 0.f, 0.f, 0.f);
        if (s_init) S = reinterpret_cast<const float4 *>(s_init + (static_cast<size_t>(seq) * H + h) * D * D)[e];
        for (int uix = f; uix < l; ++uix) {
            float4 *slot = reinterpret_cast<float4 *>(seg_state + (static_cast<size_t>(uix) * H + h) * D * D) + e;
            const bool last = (uix == l - 1);
            const float4 d = last ? make_float4(0.f, 0.f, 0.f, 0.f) : *slot;
            *slot = S;
            if (!last) {
                const float lamL = exp2f(g * static_cast<float>(units[uix].y));
                S.x = fmaf(lamL, S.x, d.x);
                S.y = fmaf(lamL, S.y, d.y);
                S.z = fmaf(lamL, S.z, d.z);
                S.w = fmaf(lamL, S.w, d.w);
            }
        }
    }
}

}  // namespace la
