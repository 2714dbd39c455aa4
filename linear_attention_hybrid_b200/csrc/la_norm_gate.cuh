// Output group RMSNorm + sigmoid gate, one fused streaming pass.
//
// The report's "linghe" section (Ling & Ring 2.6 Technical Report, blog post
// news.neo-ai.one/en/article/3021) lists "Group RMSNorm + Sigmoid Gate" among
// the fused kernels of the attention module's BF16 inference, with no formula.
// Here every (token, head) row of D attention outputs is one group:
//
//     y = w_h * o / sqrt(mean_d(o^2) + eps) * sigmoid(z),
//
// z being the gate pre-activation (a projection of the layer input made by the
// caller) and w the learned per-channel scale [H, D]. The pass reads o and z
// and writes y once (y may be o itself): HBM-bound, D / 8 lanes per row with
// 8 consecutive values each (16-byte accesses), the row's sum of squares
// reduced by warp shuffles. (Folding it into the prefill kernel's own output store was
// measured slower: no shared memory is left there for the gate tile, and the
// only slot free before the store frees up too late for its load to arrive.)
#pragma once

#include <type_traits>

#include "la_ptx.cuh"
#include "la_simt.cuh"

namespace la {

constexpr int kNormGateThreads = 256;

template <typename T, int N>
struct Vec {
    T v[N];
};

// N values of T (N * sizeof(T) a multiple of 16 bytes) in 16-byte accesses.
template <typename T, int N>
__device__ __forceinline__ Vec<T, N> load_vec(const T *p) {
    static_assert((sizeof(T) * N) % 16 == 0, "16-byte accesses");
    Vec<T, N> r;
#pragma unroll
    for (int k = 0; k < static_cast<int>(sizeof(T) * N / 16); ++k)
        reinterpret_cast<uint4 *>(r.v)[k] = reinterpret_cast<const uint4 *>(p)[k];
    return r;
}

template <typename T, int N>
__device__ __forceinline__ void store_vec(T *p, const Vec<T, N> &r) {
#pragma unroll
    for (int k = 0; k < static_cast<int>(sizeof(T) * N / 16); ++k)
        reinterpret_cast<uint4 *>(p)[k] = reinterpret_cast<const uint4 *>(r.v)[k];
}

// 8 consecutive values (16 or 32 bytes) to fp32, pairwise.
__device__ __forceinline__ void to_f32x8(const Vec<__half, 8> &v, float (&x)[8]) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(reinterpret_cast<const __half2 *>(v.v)[e]);
        x[2 * e] = f.x;
        x[2 * e + 1] = f.y;
    }
}
__device__ __forceinline__ void to_f32x8(const Vec<__nv_bfloat16, 8> &v, float (&x)[8]) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const uint32_t u = reinterpret_cast<const uint32_t *>(v.v)[e];
        x[2 * e] = bf16lo_to_f32(u);
        x[2 * e + 1] = bf16hi_to_f32(u);
    }
}
__device__ __forceinline__ void to_f32x8(const Vec<float, 8> &v, float (&x)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = v.v[e];
}
__device__ __forceinline__ void from_f32x8(Vec<__half, 8> &v, const float (&x)[8]) {
#pragma unroll
    for (int e = 0; e < 4; ++e) reinterpret_cast<__half2 *>(v.v)[e] = __floats2half2_rn(x[2 * e], x[2 * e + 1]);
}
__device__ __forceinline__ void from_f32x8(Vec<__nv_bfloat16, 8> &v, const float (&x)[8]) {
#pragma unroll
    for (int e = 0; e < 4; ++e) reinterpret_cast<uint32_t *>(v.v)[e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
}
__device__ __forceinline__ void from_f32x8(Vec<float, 8> &v, const float (&x)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) v.v[e] = x[e];
}

// The gate's sigmoid. For a bf16 gate (16-bit or bf16-derived outputs): sigmoid(z) = (1 + tanh(z / 2)) / 2
// on the hardware tanh, one special-function operation per value instead of an exponential and a
// reciprocal (which made this pass 6% slower on B200); tanh.approx.f32 has a relative error of about
// 2^-11, so the sigmoid's absolute error stays near 2^-12, the size of an fp16 output's own rounding at 1
// and far inside the 2e-2 x RMS bound of these paths. An fp32 gate (the all-fp32 path, bound 1e-4) takes
// the hardware exponential and a fast reciprocal (a few ulp).
template <typename Tg>
__device__ __forceinline__ float gate_sigmoid(float z) {
    if constexpr (std::is_same<Tg, float>::value) {
        return __fdividef(1.f, 1.f + __expf(-z));
    } else {
        float t;
        asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
        return fmaf(0.5f, t, 0.5f);
    }
}

// o, y: [rows, D] in Tout (rows = T * H < 2^31, head h = row % H); z: [rows, D] in Tg; w: [H, D] fp32; y may
// be o. A row is held by D / 8 lanes, 8 consecutive values each; a warp takes 32 / (D / 8) rows per step
// and kNormGateSteps steps at once (all loads issued before any arithmetic).
constexpr int kNormGateSteps = 2;
template <typename Tout, typename Tg, int D>
__global__ void __launch_bounds__(kNormGateThreads, 4) la_norm_gate_kernel(const Tout *o, const Tg *__restrict__ z,
                                                                           const float *__restrict__ w, float eps,
                                                                           Tout *y, int rows, int H) {
    constexpr int E = 8;                 // values per lane
    constexpr int LPR = D / E;           // lanes per row
    constexpr int RPW = 32 / LPR;        // rows per warp step
    constexpr int RPI = RPW * kNormGateSteps;
    const int lane = threadIdx.x & 31;
    const int sub = lane / LPR, col = (lane % LPR) * E;
    const int warp = blockIdx.x * (kNormGateThreads / 32) + (threadIdx.x >> 5);
    const int nwarps = gridDim.x * (kNormGateThreads / 32);
    for (int r0 = warp * RPI; r0 < rows; r0 += nwarps * RPI) {
        Vec<Tout, E> ov[kNormGateSteps];
        Vec<Tg, E> zv[kNormGateSteps];
#pragma unroll
        for (int st = 0; st < kNormGateSteps; ++st) {
            const int r = r0 + st * RPW + sub;
            if (r < rows) {
                const size_t base = static_cast<size_t>(r) * D + col;
                ov[st] = load_vec<Tout, E>(o + base);
                zv[st] = load_vec<Tg, E>(z + base);
            }
        }
#pragma unroll
        for (int st = 0; st < kNormGateSteps; ++st) {
            const int r = r0 + st * RPW + sub;
            float x[E], zz[E], ss = 0.f;
            to_f32x8(ov[st], x);
#pragma unroll
            for (int e = 0; e < E; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
            for (int off = LPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            if (r >= rows) continue;
            const float rn = rsqrtf(ss * (1.f / D) + eps);
            const float4 *wr = reinterpret_cast<const float4 *>(w + (r % H) * D + col);
            const float4 w0 = __ldg(wr), w1 = __ldg(wr + 1);
            const float wv[E] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            to_f32x8(zv[st], zz);
#pragma unroll
            for (int e = 0; e < E; ++e) x[e] = x[e] * rn * wv[e] * gate_sigmoid<Tg>(zz[e]);
            Vec<Tout, E> yv;
            from_f32x8(yv, x);
            store_vec<Tout, E>(y + static_cast<size_t>(r) * D + col, yv);
        }
    }
}

}  // namespace la
