// One Lightning Attention decode step, state updated in place:
//   S <- lambda S + k^T v,   o = q S   (the output includes the current token).
// This is the recurrent form the report's context-parallel section refers to
// (Ling & Ring 2.6 Technical Report, blog post
// news.neo-ai.one/en/article/3021, section "Long-Context Training: Context
// Parallel for Lightning Attention"). At 0.5 FLOP per state byte it is bound
// by HBM: every fp32 state entry is read once and written once per step.
//
// Several consecutive decode steps of a sequence can run in one launch (for
// multi-token or speculative decoding): the state stays in registers across
// them, so K tokens cost one read and one write of the state instead of K.
//
// One CTA per (sequence, head), 256 threads. Thread (ty, tx) owns columns
// 4tx..4tx+3 of rows [ty*RPT, ty*RPT + RPT): a warp streams whole 512-byte
// (D = 128) state rows with 16-byte loads and stores that bypass L1, all loads
// of a thread issued before any arithmetic. Per token, the D partial sums of o
// are reduced across the TY row groups in shared memory.
//
// kGate fuses the output group RMSNorm + sigmoid gate (one group per token and
// head): y = w_h * o / sqrt(mean(o^2) + eps) * sigmoid(z), z read beside o.
#pragma once

#include "la_ptx.cuh"
#include "la_simt.cuh"

namespace la {

constexpr int kDecodeThreads = 256;

constexpr int kDecodeTokenBlock = 16;  // tokens whose q, k, v are staged in shared memory at once

// Output norm + gate of the decode kernel (kGate): gate [B, steps, H, D] in the input type, weight [H, D].
template <typename Tin>
struct DecodeGate {
    const Tin *gate;
    const float *weight;
    float eps;
};

// q, k, v, o: [B, steps, H, D]; state: [B, H, D, D], read once and written once. Grid: B * H.
template <typename Tin, typename Tout, int D, bool kGate = false>
__global__ void __launch_bounds__(kDecodeThreads) la_decode_kernel(const Tin *__restrict__ q,
                                                                   const Tin *__restrict__ k,
                                                                   const Tin *__restrict__ v, Tout *__restrict__ o,
                                                                   float *__restrict__ state, int H, int steps,
                                                                   const float *__restrict__ slopes,
                                                                   const DecodeGate<Tin> ng = {}) {
    constexpr int TX = D / 4;
    constexpr int TY = kDecodeThreads / TX;
    constexpr int RPT = D / TY;
    __shared__ float red[TY][D];
    __shared__ float wss[D / 32];   // kGate: per-warp partial sums of o^2
    __shared__ float sq[kDecodeTokenBlock][D], sk[kDecodeTokenBlock][D], sv[kDecodeTokenBlock][D];

    const int bh = blockIdx.x;
    const int b = bh / H, h = bh - b * H;
    const int tx = threadIdx.x % TX, ty = threadIdx.x / TX;
    float *Sb = state + static_cast<size_t>(bh) * D * D + static_cast<size_t>(ty) * RPT * D + 4 * tx;

    float4 Sv[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) Sv[m] = ld_stream_f4(Sb + static_cast<size_t>(m) * D);

    const float lam = exp2f(decay_log2(slopes, h, H));
    for (int t0 = 0; t0 < steps; t0 += kDecodeTokenBlock) {
        const int nt = min(kDecodeTokenBlock, steps - t0);
        // q, k, v of the next tokens into shared memory (coalesced; the previous block has been consumed)
        __syncthreads();
        for (int e = threadIdx.x; e < nt * D; e += kDecodeThreads) {
            const int tt = e / D, d = e - tt * D;
            const size_t g = (static_cast<size_t>(b * steps + t0 + tt) * H + h) * D + d;
            sq[tt][d] = to_f32(q[g]);
            sk[tt][d] = to_f32(k[g]);
            sv[tt][d] = to_f32(v[g]);
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            const float v0 = sv[tt][4 * tx + 0], v1 = sv[tt][4 * tx + 1];
            const float v2 = sv[tt][4 * tx + 2], v3 = sv[tt][4 * tx + 3];
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int m = 0; m < RPT; ++m) {
                const int r = ty * RPT + m;
                const float kr = sk[tt][r];
                const float qr = sq[tt][r];
                float4 s = Sv[m];
                s.x = fmaf(lam, s.x, kr * v0);
                s.y = fmaf(lam, s.y, kr * v1);
                s.z = fmaf(lam, s.z, kr * v2);
                s.w = fmaf(lam, s.w, kr * v3);
                Sv[m] = s;
                acc.x = fmaf(qr, s.x, acc.x);
                acc.y = fmaf(qr, s.y, acc.y);
                acc.z = fmaf(qr, s.z, acc.z);
                acc.w = fmaf(qr, s.w, acc.w);
            }
            if (t0 + tt + 1 == steps) {
#pragma unroll
                for (int m = 0; m < RPT; ++m) st_stream_f4(Sb + static_cast<size_t>(m) * D, Sv[m]);
            }
            if (tt > 0) __syncthreads();  // the previous token's reduction has read red[][]
            red[ty][4 * tx + 0] = acc.x;
            red[ty][4 * tx + 1] = acc.y;
            red[ty][4 * tx + 2] = acc.z;
            red[ty][4 * tx + 3] = acc.w;
            __syncthreads();
            const size_t orow = (static_cast<size_t>(b * steps + t0 + tt) * H + h) * D;
            float sum = 0.f;
            if (threadIdx.x < D) {
#pragma unroll
                for (int y = 0; y < TY; ++y) sum += red[y][threadIdx.x];
                if constexpr (!kGate) from_f32(o[orow + threadIdx.x], sum);
            }
            if constexpr (kGate) {
                if (threadIdx.x < D) {
                    float x = sum * sum;
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
                    if ((threadIdx.x & 31) == 0) wss[threadIdx.x >> 5] = x;
                }
                __syncthreads();
                if (threadIdx.x < D) {
                    float tot = 0.f;
#pragma unroll
                    for (int w = 0; w < D / 32; ++w) tot += wss[w];
                    const float r = rsqrtf(tot * (1.f / D) + ng.eps);
                    const float z = to_f32(ng.gate[orow + threadIdx.x]);
                    const float g = 1.f / (1.f + __expf(-z));
                    from_f32(o[orow + threadIdx.x], sum * r * ng.weight[static_cast<size_t>(h) * D + threadIdx.x] * g);
                }
            }
        }
    }
}

}  // namespace la
