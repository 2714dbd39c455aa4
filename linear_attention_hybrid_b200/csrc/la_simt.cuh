// Chunked Lightning Attention prefill on the CUDA cores in fp32 (FFMA).
//
// Used for fp32 inputs (a 1e-4 bound is out of reach of bf16 / tf32 tensor-core
// products) and for calls with no tokens at all; bf16 inputs, D = 64 included,
// run on the tensor cores.
// Tin is the type of q, k, v (bf16 or fp32) and Tout the type of o (bf16, fp16 or fp32).
// Same chunk algebra as the tensor-core kernel, with C = 64, all in fp32:
//   A[i,s] = lambda^(i-s) (q_i . k_s) for s <= i,
//   o_i    = sum_s A[i,s] v_s + lambda^(i+1) q_i S,
//   S     <- lambda^Lc S + sum_s lambda^(Lc-1-s) k_s^T v_s.
// One CTA per (sequence, head) and slice of Dc value columns, 256 threads: the
// columns of S and o evolve independently, so when few (sequence, head) pairs
// would leave SMs idle each is split over D / Dc CTAs, every one making the
// whole score tile A but only its Dc columns of o and S. The state slice S
// (D x Dc fp32) and the chunk's q, k (whole rows) and v (the slice) stay in
// shared memory.
//
// kRev runs the same recurrence backwards in time (the reverse sweep of the
// backward pass): chunks from the sequence end to its start, and inside a chunk
//   A[i,s] = lambda^(s-i) (q_i . k_s) for s >= i,
//   o_i    = sum_s A[i,s] v_s + lambda^(Lc-1-i) q_i S,
//   S     <- lambda^Lc S + sum_s lambda^(s+1) k_s^T v_s,
// so that S entering a chunk is lambda times the state at the token after it,
// s_init is the state after the sequence's last token and s_final the state
// (times lambda) at its first token.
#pragma once

#include <cuda_fp16.h>

#include "la_ptx.cuh"

namespace la {

constexpr int kSimtC = 64;
constexpr int kSimtThreads = 256;

template <int D, int Dc = D>
struct SimtCfg {
    static constexpr int kRow = D + 1;  // padded row (floats) of the q / k chunk tiles
    static constexpr size_t kSmemBytes =
        sizeof(float) * (static_cast<size_t>(D) * Dc + 2 * kSimtC * kRow + kSimtC * Dc + kSimtC * (kSimtC + 1) + kSimtC);
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f32(float &d, float x) { d = x; }
__device__ __forceinline__ void from_f32(__nv_bfloat16 &d, float x) { d = __float2bfloat16_rn(x); }
__device__ __forceinline__ void from_f32(__half &d, float x) { d = __float2half_rn(x); }

template <typename Tin, typename Tout, int D, bool kRev = false, int Dc = D>
__global__ void __launch_bounds__(kSimtThreads) la_simt_prefill_kernel(const Tin *q, const Tin *k, const Tin *v,
                                                                       Tout *o, const int32_t *cu, int N_uniform,
                                                                       int T, int H, const float *s_init,
                                                                       float *s_final, const float *slopes) {
    using Cfg = SimtCfg<D, Dc>;
    static_assert(D % Dc == 0, "column slices divide the head dim");
    constexpr int C = kSimtC;
    extern __shared__ float fsm[];
    float *S = fsm;                          // [D][Dc] columns c0 .. c0+Dc-1 of the state
    float *Qs = S + D * Dc;                  // [C][D+1]
    float *Ks = Qs + C * Cfg::kRow;          // [C][D+1]
    float *Vs = Ks + C * Cfg::kRow;          // [C][Dc]
    float *As = Vs + C * Dc;                 // [C][C+1]
    float *w = As + C * (C + 1);             // [C] lambda^(Lc-1-s) (kRev: lambda^(s+1))

    const int seq = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int c0 = static_cast<int>(blockIdx.z) * Dc;   // first value column of this CTA
    int a, b;
    if (cu) {
        a = min(max(cu[seq], 0), T);
        b = min(max(cu[seq + 1], a), T);
    } else {
        a = seq * N_uniform;
        b = a + N_uniform;
    }
    const float g = decay_log2(slopes, h, H);
    const size_t sbase = (static_cast<size_t>(seq) * H + h) * D * D;

    for (int idx = tid; idx < D * Dc; idx += kSimtThreads) {
        const int d = idx / Dc, j = idx % Dc;
        S[idx] = s_init ? s_init[sbase + static_cast<size_t>(d) * D + c0 + j] : 0.f;
    }

    const int nch = (b - a + C - 1) / C;
    for (int n = 0; n < nch; ++n) {
        const int t0 = a + C * (kRev ? nch - 1 - n : n);
        const int Lc = min(C, b - t0);
        __syncthreads();  // previous chunk fully consumed
        for (int idx = tid; idx < C * D; idx += kSimtThreads) {
            const int r = idx / D, c = idx % D;
            float qv = 0.f, kv = 0.f, vv = 0.f;
            if (r < Lc) {
                const size_t gi = (static_cast<size_t>(t0 + r) * H + h) * D + c;
                qv = to_f32(q[gi]);
                kv = to_f32(k[gi]);
                if (c >= c0 && c < c0 + Dc) vv = to_f32(v[gi]);
            }
            Qs[r * Cfg::kRow + c] = qv;
            Ks[r * Cfg::kRow + c] = kv;
            if (c >= c0 && c < c0 + Dc) Vs[r * Dc + (c - c0)] = vv;
        }
        for (int s = tid; s < C; s += kSimtThreads)
            w[s] = s < Lc ? exp2f(g * static_cast<float>(kRev ? s + 1 : Lc - 1 - s)) : 0.f;
        __syncthreads();
        // A[i,s] = lambda^(i-s) q_i . k_s for s <= i (kRev: lambda^(s-i) for s >= i; rows past Lc are zero)
        for (int idx = tid; idx < C * C; idx += kSimtThreads) {
            const int i = idx / C, s = idx % C;
            float acc = 0.f;
            if (kRev ? s >= i : s <= i) {
#pragma unroll 8
                for (int d = 0; d < D; ++d) acc = fmaf(Qs[i * Cfg::kRow + d], Ks[s * Cfg::kRow + d], acc);
                acc *= exp2f(g * static_cast<float>(kRev ? s - i : i - s));
            }
            As[i * (C + 1) + s] = acc;
        }
        __syncthreads();
        // o_i = sum_s A[i,s] v_s + lambda^(i+1) q_i S (kRev: lambda^(Lc-1-i))
        for (int idx = tid; idx < C * Dc; idx += kSimtThreads) {
            const int i = idx / Dc, j = idx % Dc;
            if (i >= Lc) continue;
            float intra = 0.f, inter = 0.f;
            for (int s = kRev ? i : 0; s <= (kRev ? Lc - 1 : i); ++s) intra = fmaf(As[i * (C + 1) + s], Vs[s * Dc + j], intra);
#pragma unroll 8
            for (int d = 0; d < D; ++d) inter = fmaf(Qs[i * Cfg::kRow + d], S[d * Dc + j], inter);
            const float val = fmaf(exp2f(g * static_cast<float>(kRev ? Lc - 1 - i : i + 1)), inter, intra);
            from_f32(o[(static_cast<size_t>(t0 + i) * H + h) * D + c0 + j], val);
        }
        __syncthreads();
        // S <- lambda^Lc S + sum_s w_s k_s^T v_s
        const float lamL = exp2f(g * static_cast<float>(Lc));
        for (int idx = tid; idx < D * Dc; idx += kSimtThreads) {
            const int d = idx / Dc, j = idx % Dc;
            float acc = 0.f;
            for (int s = 0; s < Lc; ++s) acc = fmaf(w[s] * Ks[s * Cfg::kRow + d], Vs[s * Dc + j], acc);
            S[idx] = fmaf(lamL, S[idx], acc);
        }
    }
    __syncthreads();
    if (s_final)
        for (int idx = tid; idx < D * Dc; idx += kSimtThreads) {
            const int d = idx / Dc, j = idx % Dc;
            s_final[sbase + static_cast<size_t>(d) * D + c0 + j] = S[idx];
        }
}

}  // namespace la
