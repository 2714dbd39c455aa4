// Combining the states of consecutive shards of a sequence.
//
// A sequence cut into shards of L tokens each (fine units on one GPU, or the
// ranks of a context-parallel group, one shard per GPU) is computed shard by
// shard from a zero state, and the state entering shard u is recovered from the
// states dS_u' the earlier shards produced: the "local recursion + global
// correction" of the Ling & Ring 2.6 Technical Report (blog post
// news.neo-ai.one/en/article/3021, section "Long-Context Training: Context
// Parallel for Lightning Attention"). With S_t = lambda S_{t-1} + k_t^T v_t,
//
//   S_in(u) = lambda^(u L) S_0 + sum_{u' < u} lambda^((u-1-u') L) dS_u'.
//
// Elementwise over [heads, D, D]: the kernel is bound by reading u + 1 states.
#pragma once

#include "la_ptx.cuh"

namespace la {

constexpr int kCombineThreads = 256;

// The state after u consecutive units, the first u - 1 of L tokens and the last of
// last_len tokens (last_len <= L; equal to L for equal units):
//   out[b, h] = lambda_h^(E_s0) s0[b, h] + sum_{u' < u} lambda_h^(E_u') src(u', b, h),
// with E_u' the tokens after unit u' ends ((u - 2 - u') L + last_len, and 0 for u' = u - 1),
// E_s0 = (u - 1) L + last_len, and src(u', b, h) starting at (u' * stride_u + b * stride_b + h) * DD
// floats. u = 0 gives s0 (or zero). DD is a multiple of 4. Grid: (blocks over DD / 4, B * H).
__global__ void __launch_bounds__(kCombineThreads) la_combine_states_kernel(const float *src, int u, long long stride_u,
                                                                           long long stride_b, int H, int DD, int L,
                                                                           int last_len, const float *slopes,
                                                                           const float *s0, float *out) {
    const int bh = blockIdx.y;
    const int b = bh / H, h = bh - b * H;
    const float g = decay_log2(slopes, h, H);
    const size_t base_out = static_cast<size_t>(bh) * DD;
    for (int e = (blockIdx.x * blockDim.x + threadIdx.x) * 4; e < DD; e += gridDim.x * blockDim.x * 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (s0) {
            const float ex = u > 0 ? static_cast<float>(u - 1) * static_cast<float>(L) + static_cast<float>(last_len) : 0.f;
            const float w = exp2f(g * ex);
            const float4 z = *reinterpret_cast<const float4 *>(s0 + base_out + e);
            acc = make_float4(w * z.x, w * z.y, w * z.z, w * z.w);
        }
        for (int up = 0; up < u; ++up) {
            const float ex = up + 1 < u ? static_cast<float>(u - 2 - up) * static_cast<float>(L) + static_cast<float>(last_len)
                                        : 0.f;
            const float w = exp2f(g * ex);
            const float4 x = *reinterpret_cast<const float4 *>(src + (up * stride_u + b * stride_b + h) * DD + e);
            acc.x = fmaf(w, x.x, acc.x);
            acc.y = fmaf(w, x.y, acc.y);
            acc.z = fmaf(w, x.z, acc.z);
            acc.w = fmaf(w, x.w, acc.w);
        }
        *reinterpret_cast<float4 *>(out + base_out + e) = acc;
    }
}

// The reversed direction (the backward pass's sweep from the right): the state
// entering a stretch of the sequence from its right end, from the reversed
// states dH_j of the units after it (each from a zero start, weights
// lambda^(s+1) from its own start; unit j begins j L tokens after the stretch
// ends) and the state s_end given past the sequence end:
//   out[b, h] = sum_{j < n} lambda_h^(j L) src(j, b, h) + lambda_h^(end_exp) s_end[b, h],
// src(j, b, h) starting at (j * stride_u + b * stride_b + h) * DD floats. Grid as above.
__global__ void __launch_bounds__(kCombineThreads) la_combine_states_rev_kernel(const float *src, int n, long long stride_u,
                                                                               long long stride_b, int H, int DD, int L,
                                                                               const float *slopes, const float *s_end,
                                                                               float end_exp, float *out) {
    const int bh = blockIdx.y;
    const int b = bh / H, h = bh - b * H;
    const float g = decay_log2(slopes, h, H);
    const size_t base_out = static_cast<size_t>(bh) * DD;
    for (int e = (blockIdx.x * blockDim.x + threadIdx.x) * 4; e < DD; e += gridDim.x * blockDim.x * 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (s_end) {
            const float w = exp2f(g * end_exp);
            const float4 z = *reinterpret_cast<const float4 *>(s_end + base_out + e);
            acc = make_float4(w * z.x, w * z.y, w * z.z, w * z.w);
        }
        for (int j = 0; j < n; ++j) {
            const float w = exp2f(g * static_cast<float>(j) * static_cast<float>(L));
            const float4 x = *reinterpret_cast<const float4 *>(src + (j * stride_u + b * stride_b + h) * DD + e);
            acc.x = fmaf(w, x.x, acc.x);
            acc.y = fmaf(w, x.y, acc.y);
            acc.z = fmaf(w, x.z, acc.z);
            acc.w = fmaf(w, x.w, acc.w);
        }
        *reinterpret_cast<float4 *>(out + base_out + e) = acc;
    }
}

// Packed varlen batches sharded along the token axis (context parallelism over varlen sequences: rank r
// holds tokens [r L, (r+1) L) of the packed batch, so a sequence may start on one rank and end on any later
// one). The state entering the part of a sequence on some rank combines, for that one sequence, the states
// its parts on other ranks produced from a zero start, each with its own decay exponent (the tokens between
// that part's end and the point the state enters), and optionally a given state (the sequence's initial
// state, or the gradient of its final state in the reversed direction) with its own exponent:
//   out[h] = lambda_h^(s0_exp) s0[h] + sum_j lambda_h^(exps[j]) src(idx[j], h),
// src(i, h) starting at (i * stride + h) * DD floats. The host works out the terms from the sequence
// boundaries. Grid: (blocks over DD / 4, H).
constexpr int kMaxCombineTerms = 64;
struct CombineTerms {
    int n;                          // terms from src
    int idx[kMaxCombineTerms];      // which state of src (a rank)
    float exps[kMaxCombineTerms];   // decay exponent (tokens) of each
    float s0_exp;                   // exponent of s0 (ignored when s0 is null)
};

__global__ void __launch_bounds__(kCombineThreads) la_combine_terms_kernel(const float *src, long long stride,
                                                                          const CombineTerms t, const float *s0,
                                                                          int H, int DD, const float *slopes,
                                                                          float *out) {
    const int h = blockIdx.y;
    const float g = decay_log2(slopes, h, H);
    const size_t base_out = static_cast<size_t>(h) * DD;
    for (int e = (blockIdx.x * blockDim.x + threadIdx.x) * 4; e < DD; e += gridDim.x * blockDim.x * 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (s0) {
            const float w = exp2f(g * t.s0_exp);
            const float4 z = *reinterpret_cast<const float4 *>(s0 + base_out + e);
            acc = make_float4(w * z.x, w * z.y, w * z.z, w * z.w);
        }
        for (int j = 0; j < t.n; ++j) {
            const float w = exp2f(g * t.exps[j]);
            const float4 x = *reinterpret_cast<const float4 *>(src + (t.idx[j] * stride + h) * DD + e);
            acc.x = fmaf(w, x.x, acc.x);
            acc.y = fmaf(w, x.y, acc.y);
            acc.z = fmaf(w, x.z, acc.z);
            acc.w = fmaf(w, x.w, acc.w);
        }
        *reinterpret_cast<float4 *>(out + base_out + e) = acc;
    }
}

}  // namespace la
