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
// One CTA per (sequence, head) and slice of kCols state columns, 256 threads.
// The columns of S evolve independently and o_j needs column j only, so the
// plain decode splits each 128-column state over two CTAs (half the registers
// per thread: four CTAs per SM instead of two, so state loads stay in flight
// while other CTAs run their token loops). Thread (ty, tx) owns columns
// 4tx..4tx+3 of its slice in rows [ty*RPT, ty*RPT + RPT): a warp streams
// 256-byte row slices with 16-byte loads and stores that bypass L1, all loads
// of a thread issued before any arithmetic. The kCols partial sums of each
// token's output are reduced across the TY row groups in shared memory, for a
// block of tokens at a time.
//
// kGate fuses the output group RMSNorm + sigmoid gate (one group per token and
// head): y = w_h * o / sqrt(mean(o^2) + eps) * sigmoid(z), z read beside o. It
// keeps whole rows per CTA (the norm needs the row's sum of squares), bounded to
// 80 registers so that three CTAs share an SM.
#pragma once

#include "la_ptx.cuh"
#include "la_simt.cuh"

namespace la {

constexpr int kDecodeThreads = 256;

// tokens whose q, k, v (and partial outputs) are staged in shared memory at once: 8 tokens x 8 row groups
// (256 threads) of 128 partial sums, or x 16 row groups of 64, fit the 48 KB of static shared memory
template <int kThreads>
__host__ __device__ constexpr int decode_token_block() { return kThreads == 256 ? 8 : 4; }

// Output norm + gate of the decode kernel (kGate): gate [B, steps, H, D] in the input type, weight [H, D].
template <typename Tin>
struct DecodeGate {
    const Tin *gate;
    const float *weight;
    float eps;
};

// q, k, v, o: [B, steps, H, D]; state: [B, H, D, D], read once and written once. Grid: B * H * (D / kCols).
// Per block of up to decode_token_block() tokens: the tokens' q, k, v are staged, every thread runs the token
// loop on its state rows (no barrier inside it), writing its partial sums of each token's output to
// shared memory; one barrier, then the partial sums of all the block's outputs are reduced at once.
template <typename Tin, typename Tout, int D, bool kGate = false, int kThreads = kDecodeThreads, int kCols = D>
__global__ void __launch_bounds__(kThreads, kCols == D ? (kGate ? 3 : 2) : 4) la_decode_kernel(const Tin *__restrict__ q,
                                                                   const Tin *__restrict__ k,
                                                                   const Tin *__restrict__ v, Tout *__restrict__ o,
                                                                   float *__restrict__ state, int H, int steps,
                                                                   const float *__restrict__ slopes,
                                                                   const DecodeGate<Tin> ng = {}) {
    static_assert(!kGate || kCols == D, "the norm + gate needs whole output rows");
    static_assert(D % kCols == 0 && kCols % 4 == 0, "column slices of 16-byte groups");
    constexpr int kSplit = D / kCols;
    constexpr int TX = kCols / 4;
    constexpr int TY = kThreads / TX;
    constexpr int RPT = D / TY;
    constexpr int TB = decode_token_block<kThreads>();
    __shared__ float red[TB][TY][kCols];              // partial sums of each token's output, per row group
    __shared__ float sq[TB][D], sk[TB][D], sv[TB][D];
    __shared__ float wss[kThreads / D][D / 32];  // kGate: per-warp partial squares of a token's outputs

    const int bh = blockIdx.x / kSplit;
    const int c0 = (blockIdx.x - bh * kSplit) * kCols;   // first state column (and output) of this CTA
    const int b = bh / H, h = bh - b * H;
    const int tx = threadIdx.x % TX, ty = threadIdx.x / TX;
    float *Sb = state + static_cast<size_t>(bh) * D * D + static_cast<size_t>(ty) * RPT * D + c0 + 4 * tx;

    float4 Sv[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) Sv[m] = ld_stream_f4(Sb + static_cast<size_t>(m) * D);

    const float lam = exp2f(decay_log2(slopes, h, H));
    for (int t0 = 0; t0 < steps; t0 += TB) {
        const int nt = min(TB, steps - t0);
        // q, k, v of the next tokens into shared memory (coalesced; the previous block has been consumed)
        __syncthreads();
        for (int e = threadIdx.x; e < nt * D; e += kThreads) {
            const int tt = e / D, d = e - tt * D;
            const size_t g = (static_cast<size_t>(b * steps + t0 + tt) * H + h) * D + d;
            sq[tt][d] = to_f32(q[g]);
            sk[tt][d] = to_f32(k[g]);
            sv[tt][d] = to_f32(v[g]);
        }
        __syncthreads();
        // per state entry: s = lambda s + k_r v_j (the product rounded, then one fused multiply-add) and
        // acc_j += q_r s, in paired fp32 operations (two lanes of the same operations per instruction)
        const float2 lam2 = make_float2(lam, lam);
        for (int tt = 0; tt < nt; ++tt) {
            const float2 v01 = make_float2(sv[tt][c0 + 4 * tx + 0], sv[tt][c0 + 4 * tx + 1]);
            const float2 v23 = make_float2(sv[tt][c0 + 4 * tx + 2], sv[tt][c0 + 4 * tx + 3]);
            float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
#pragma unroll
            for (int m = 0; m < RPT; ++m) {
                const int r = ty * RPT + m;
                const float2 kr = make_float2(sk[tt][r], sk[tt][r]);
                const float2 qr = make_float2(sq[tt][r], sq[tt][r]);
                float4 s = Sv[m];
                const float2 s01 = __ffma2_rn(lam2, make_float2(s.x, s.y), __fmul2_rn(kr, v01));
                const float2 s23 = __ffma2_rn(lam2, make_float2(s.z, s.w), __fmul2_rn(kr, v23));
                Sv[m] = make_float4(s01.x, s01.y, s23.x, s23.y);
                a01 = __ffma2_rn(qr, s01, a01);
                a23 = __ffma2_rn(qr, s23, a23);
            }
            *reinterpret_cast<float4 *>(&red[tt][ty][4 * tx]) = make_float4(a01.x, a01.y, a23.x, a23.y);
        }
        if (t0 + nt == steps) {
#pragma unroll
            for (int m = 0; m < RPT; ++m) st_stream_f4(Sb + static_cast<size_t>(m) * D, Sv[m]);
        }
        __syncthreads();
        if constexpr (!kGate) {
            // the block's outputs: nt x kCols sums over the TY row groups
            for (int e = threadIdx.x; e < nt * kCols; e += kThreads) {
                const int tt = e / kCols, j = e - tt * kCols;
                float sum = 0.f;
#pragma unroll
                for (int y = 0; y < TY; ++y) sum += red[tt][y][j];
                from_f32(o[(static_cast<size_t>(b * steps + t0 + tt) * H + h) * D + c0 + j], sum);
            }
        } else {
            // D threads per token (kThreads / D tokens at a time): each sums one output over the row
            // groups, the token's mean square comes from warp shuffles and one value per warp, then the norm
            // and gate
            constexpr int TPI = kThreads / D;
            const int grp = threadIdx.x / D, j = threadIdx.x - grp * D, lane = threadIdx.x & 31;
            for (int tb = 0; tb < nt; tb += TPI) {
                const int tt = tb + grp;
                float sum = 0.f;
                if (tt < nt) {
#pragma unroll
                    for (int y = 0; y < TY; ++y) sum += red[tt][y][j];
                }
                float x = sum * sum;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
                if (lane == 0) wss[grp][j >> 5] = x;
                __syncthreads();
                if (tt < nt) {
                    float tot = 0.f;
#pragma unroll
                    for (int w = 0; w < D / 32; ++w) tot += wss[grp][w];
                    const float rn = rsqrtf(tot * (1.f / D) + ng.eps);
                    const size_t orow = (static_cast<size_t>(b * steps + t0 + tt) * H + h) * D;
                    const float z = to_f32(ng.gate[orow + j]);
                    const float g = 1.f / (1.f + __expf(-z));
                    from_f32(o[orow + j], sum * rn * ng.weight[static_cast<size_t>(h) * D + j] * g);
                }
                if (tb + TPI < nt) __syncthreads();   // the next tokens' partial squares reuse wss
            }
        }
    }
}

}  // namespace la
