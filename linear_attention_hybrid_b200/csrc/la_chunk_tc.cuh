// Chunked Lightning Attention prefill on the sm_100a tensor cores (tcgen05 +
// TMEM), fed by TMA.
//
// The recurrence S_t = lambda S_{t-1} + k_t^T v_t, o_t = q_t S_t has a serial
// dependency along the sequence (Ling & Ring 2.6 Technical Report, blog post
// news.neo-ai.one/en/article/3021, section "Long-Context Training: Context
// Parallel for Lightning Attention"). Blocking it into chunks of C = 128
// tokens turns each chunk into four dense contractions (the O(n) form of
// section "Hybrid Linear Attention"); with rows i and columns s 0-based inside
// the chunk, Lc valid rows, and S the state entering the chunk:
//
//   A      = Q K^T                                  (C x C,  tensor core)
//   P[i,s] = A[i,s] lambda^(i-s)  for s <= i, else 0 (registers, CUDA cores)
//   O      = P V + diag(lambda^(i+1)) (Q S)         (two accumulators, tensor core)
//   S     <- lambda^Lc S + (diag(lambda^(Lc-1-s)) K)^T V   (tensor core + registers)
//
// One CTA owns one work unit: a segment of one sequence for one head. Warp
// roles (320 threads):
//   warp 0     TMA producer: Q, K, V tiles of each chunk into a 2-stage ring;
//   warp 1     tcgen05.mma issuer (one thread) and TMEM owner;
//   warps 2-9  epilogue: two warpgroups, each owning 64 of the 128 columns of
//              every 128-row TMEM tile; warp w reads TMEM lanes 32*(w%4)...
// TMEM (512 columns): [0,128) scores A, overwritten in place by P as packed
// bf16; [128,256) O_intra = P V; [256,384) O_inter = Q S; [384,512) dS.
// The fp32 state S never leaves the chip: each epilogue thread keeps 64
// entries of its row of S in registers, and a bf16 copy in shared memory
// (128-byte-swizzled, MN-major) is the B operand of the next Q S product.
//
// kStateOnly = true is the first pass of the segment split: only K and V are
// loaded, only dS is formed, and the unit's segment state from a zero start
// is written to the workspace.
#pragma once

#include "la_ptx.cuh"

namespace la {

constexpr int kC = 128;                  // chunk length = MMA M
constexpr int kD = 128;                  // head dim handled by this kernel
constexpr int kSlabBytes = 128 * 128;    // [128 rows x 64 bf16] slab, 128-byte rows
constexpr int kTileBytes = 2 * kSlabBytes;  // [128 x 128] bf16 tile = two slabs
constexpr int kTcThreads = 320;

enum UnitFlags { kUnitFirst = 1, kUnitLast = 2 };

struct ChunkArgs {
    __nv_bfloat16 *o;           // [T, H, D]
    const float *s_init;        // [nseq, H, D, D] or null
    float *s_final;             // [nseq, H, D, D] or null
    const float *slopes;        // [H] or null
    const int4 *units;          // plan: {tok0, len, seq, flags}
    const int *n_units;         // plan size (device)
    float *seg_state;           // [cap, H, D, D] workspace
    int H;
};

template <bool kStateOnly>
struct ChunkCfg {
    static constexpr int kStages = kStateOnly ? 3 : 2;
    static constexpr int kStageBytes = (kStateOnly ? 2 : 3) * kTileBytes;
    static constexpr int kSbfBytes = kStateOnly ? 0 : kTileBytes;
    static constexpr int kBarOffset = kStages * kStageBytes + kSbfBytes;
    static constexpr int kSmemBytes = kBarOffset + 256 + 1024;  // barriers + alignment slack
    static constexpr uint32_t kTmemCols = kStateOnly ? 128 : 512;
    static constexpr uint32_t kColA = 0, kColOn = 128, kColOi = 256;
    static constexpr uint32_t kColDs = kStateOnly ? 0 : 384;
};

// K-major operand (rows = M or N, 128 bf16 along K split in two 64-wide slabs),
// 16-element K step kk.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int kk) {
    return smem_desc_sw128(tile + (kk >> 2) * kSlabBytes + (kk & 3) * 32, 16, 1024);
}
// MN-major operand (rows = K, 128-byte rows holding 64 MN elements, two MN slabs
// 16 KB apart), 16-row K step kk.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile, int kk) {
    return smem_desc_sw128(tile + kk * 2048, kSlabBytes, 1024);
}
// TMEM column of the packed P block b (32 P columns -> 16 TMEM columns).
__device__ __forceinline__ uint32_t p_block_col(int b) { return 64u * (b >> 1) + 16u * (b & 1); }
// TMEM column of the 16-wide K step kk of P.
__device__ __forceinline__ uint32_t p_kstep_col(int kk) { return 64u * (kk >> 2) + 8u * (kk & 3); }

// Warp-uniform bounded wait: lane 0 waits, the result is broadcast.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, int lane) {
    int ok = 1;
    if (lane == 0) ok = mbar_wait(bar, parity) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ bool warp_aborted(const int *flag, int lane) {
    int a = 0;
    if (lane == 0) a = *reinterpret_cast<const volatile int *>(flag);
    return __shfl_sync(0xffffffffu, a, 0) != 0;
}

// Scale one 128-byte row of bf16 (8 x 16-byte chunks) in shared memory by `f`.
// Chunks are visited starting at (row & 7) so that a warp's 32 rows hit all banks.
__device__ __forceinline__ void scale_row_bf16(uint8_t *row_ptr, int row, float f) {
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
        const int j = (jj + row) & 7;
        uint4 x = *reinterpret_cast<uint4 *>(row_ptr + 16 * j);
        uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int m = 0; m < 4; ++m) w[m] = pack_bf16x2(bf16lo_to_f32(w[m]) * f, bf16hi_to_f32(w[m]) * f);
        *reinterpret_cast<uint4 *>(row_ptr + 16 * j) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Store 64 fp32 state entries of row `row` (columns [64*half, 64*half+64)) as
// bf16 into the MN-major swizzled state tile: slab `half`, 128-byte row `row`,
// 16-byte chunk j lands at j ^ (row & 7).
__device__ __forceinline__ void store_state_bf16(uint8_t *sbf, int half, int row, const float (&S)[64]) {
    uint8_t *base = sbf + half * kSlabBytes + row * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint4 w = make_uint4(pack_bf16x2(S[8 * j + 0], S[8 * j + 1]), pack_bf16x2(S[8 * j + 2], S[8 * j + 3]),
                             pack_bf16x2(S[8 * j + 4], S[8 * j + 5]), pack_bf16x2(S[8 * j + 6], S[8 * j + 7]));
        *reinterpret_cast<uint4 *>(base + 16 * (j ^ (row & 7))) = w;
    }
}

template <bool kStateOnly>
__global__ void __launch_bounds__(kTcThreads, 1)
    la_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const ChunkArgs args) {
    using Cfg = ChunkCfg<kStateOnly>;
    constexpr int NST = Cfg::kStages;

    const int unit = blockIdx.x;
    const int h = blockIdx.y;
    if (unit >= *args.n_units) return;
    const int4 u = args.units[unit];
    if (kStateOnly && (u.w & kUnitLast)) return;  // the last segment's own state is never needed
    const int tok0 = u.x, len = u.y, seq = u.z, flags = u.w;
    const int nchunks = (len + kC - 1) / kC;
    const int H = args.H;
    const float g = decay_log2(args.slopes, h, H);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sbf = smem + NST * Cfg::kStageBytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOffset);
    uint64_t *full = bars;              // [NST] TMA landed
    uint64_t *empty = bars + NST;       // [NST] stage free again
    uint64_t *bar_S = bars + 2 * NST;   // scores A ready in TMEM
    uint64_t *bar_P = bar_S + 1;        // P in TMEM and K' in smem ready (8 epilogue warps)
    uint64_t *bar_O = bar_S + 2;        // O_intra, O_inter, dS ready
    uint64_t *bar_Sd = bar_S + 3;       // state consumed dS and (full) wrote its bf16 copy (8 warps)
    uint64_t *bar_Of = bar_S + 4;       // O accumulators drained (8 warps)
    uint64_t *bar_done = bar_S + 5;     // every MMA retired
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_S + 6);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(bar_S, 1);
        mbar_init(bar_P, 8);
        mbar_init(bar_O, 1);
        mbar_init(bar_Sd, 8);
        mbar_init(bar_Of, 8);
        mbar_init(bar_done, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            if (!kStateOnly) tma_prefetch_desc(&tm_q);
            int issued = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % NST;
                const uint32_t r = static_cast<uint32_t>(c / NST);
                if (r > 0 && !mbar_wait(&empty[s], (r - 1) & 1)) {
                    *reinterpret_cast<volatile int *>(abort_flag) = 1;
                    break;
                }
                if (*reinterpret_cast<volatile int *>(abort_flag)) break;
                uint8_t *st = smem + s * Cfg::kStageBytes;
                const int t = tok0 + c * kC;
                mbar_arrive_expect_tx(&full[s], Cfg::kStageBytes);
                uint8_t *kt = st + (kStateOnly ? 0 : kTileBytes);
                uint8_t *vt = kt + kTileBytes;
                if (!kStateOnly) {
                    tma_load_3d(st, &tm_q, 0, h, t, &full[s]);
                    tma_load_3d(st + kSlabBytes, &tm_q, 64, h, t, &full[s]);
                }
                tma_load_3d(kt, &tm_k, 0, h, t, &full[s]);
                tma_load_3d(kt + kSlabBytes, &tm_k, 64, h, t, &full[s]);
                tma_load_3d(vt, &tm_v, 0, h, t, &full[s]);
                tma_load_3d(vt + kSlabBytes, &tm_v, 64, h, t, &full[s]);
                issued = c + 1;
            }
            // Never leave with a copy in flight: wait (bounded) for the last load of each stage.
            for (int c = (issued > NST ? issued - NST : 0); c < issued; ++c)
                mbar_wait(&full[c % NST], static_cast<uint32_t>(c / NST) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_qk = idesc_bf16_f32(kC, kC, false, false);
            constexpr uint32_t id_pv = idesc_bf16_f32(kC, kD, false, true);
            constexpr uint32_t id_qs = idesc_bf16_f32(kC, kD, false, true);
            constexpr uint32_t id_ds = idesc_bf16_f32(kD, kD, true, true);
            const uint32_t sbf_addr = smem_u32(sbf);
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % NST;
                const uint32_t r = static_cast<uint32_t>(c / NST);
                if (!mbar_wait(&full[s], r & 1)) break;
                tc_fence_after();
                const uint32_t st = smem_u32(smem + s * Cfg::kStageBytes);
                const uint32_t qa = st;
                const uint32_t ka = st + (kStateOnly ? 0 : kTileBytes);
                const uint32_t va = ka + kTileBytes;
                if (!kStateOnly) {
                    // A = Q K^T
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk)
                        mma_ss(tmem + Cfg::kColA, desc_kmajor(qa, kk), desc_kmajor(ka, kk), id_qk, kk > 0);
                    mma_commit(bar_S);
                    // O_inter = Q S (needs the bf16 state of the previous chunk and drained O)
                    if (!mbar_wait(bar_Sd, static_cast<uint32_t>(c) & 1)) break;
                    if (c > 0 && !mbar_wait(bar_Of, static_cast<uint32_t>(c - 1) & 1)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk)
                        mma_ss(tmem + Cfg::kColOi, desc_kmajor(qa, kk), desc_mnmajor(sbf_addr, kk), id_qs, kk > 0);
                    // O_intra = P V (P from TMEM)
                    if (!mbar_wait(bar_P, static_cast<uint32_t>(c) & 1)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kC / 16; ++kk)
                        mma_ts(tmem + Cfg::kColOn, tmem + Cfg::kColA + p_kstep_col(kk), desc_mnmajor(va, kk), id_pv,
                               kk > 0);
                } else {
                    if (c > 0 && !mbar_wait(bar_Sd, static_cast<uint32_t>(c - 1) & 1)) break;
                    if (!mbar_wait(bar_P, static_cast<uint32_t>(c) & 1)) break;
                    tc_fence_after();
                }
                // dS = K'^T V
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ss(tmem + Cfg::kColDs, desc_mnmajor(ka, kk), desc_mnmajor(va, kk), id_ds, kk > 0);
                mma_commit(bar_O);
                mma_commit(&empty[s]);
            }
            mma_commit(bar_done);
            mbar_wait(bar_done, 0);
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 2..9)
        const int e = warp - 2;          // 0..7
        const int q4 = warp & 3;         // TMEM lane quarter this warp may access
        const int hf = e >> 2;           // column half
        const int i = 32 * q4 + lane;    // TMEM lane = chunk row i (A, O) or state row dk (dS)
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * q4) << 16);
        const float lam = exp2f(g);
        const size_t DD = static_cast<size_t>(kD) * kD;

        float S[64];
        {
            const float *src = nullptr;
            if (!kStateOnly) {
                if ((flags & kUnitFirst) && (flags & kUnitLast)) {
                    if (args.s_init) src = args.s_init + (static_cast<size_t>(seq) * H + h) * DD;
                } else {
                    src = args.seg_state + (static_cast<size_t>(unit) * H + h) * DD;
                }
            }
            if (src) {
                const float4 *p = reinterpret_cast<const float4 *>(src + static_cast<size_t>(i) * kD + 64 * hf);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float4 x = p[j];
                    S[4 * j] = x.x;
                    S[4 * j + 1] = x.y;
                    S[4 * j + 2] = x.z;
                    S[4 * j + 3] = x.w;
                }
            } else {
#pragma unroll
                for (int j = 0; j < 64; ++j) S[j] = 0.f;
            }
        }
        if (!kStateOnly) {
            store_state_bf16(sbf, hf, i, S);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_Sd);
        }

        const int et = e * 32 + lane;     // 0..255, for the K' rescale
        const int krow = et & 127;
        const int kslab = et >> 7;

        for (int c = 0; c < nchunks; ++c) {
            if (warp_aborted(abort_flag, lane)) break;
            const int s = c % NST;
            const uint32_t r = static_cast<uint32_t>(c / NST);
            const int Lc = min(kC, len - c * kC);
            uint8_t *st = smem + s * Cfg::kStageBytes;

            if (!kStateOnly) {
                // ---- P = decay-masked A, packed to bf16 in place in TMEM
                if (!warp_wait(bar_S, static_cast<uint32_t>(c) & 1, lane)) {
                    if (lane == 0) *reinterpret_cast<volatile int *>(abort_flag) = 1;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int bb = 0; bb < 2; ++bb) {
                    const int b = 2 * hf + bb;  // 32-column block of A
                    uint32_t pk[16];
                    if (b > q4) {
#pragma unroll
                        for (int m = 0; m < 16; ++m) pk[m] = 0u;
                    } else {
                        float a[32];
                        tmem_ld32(lane_addr + Cfg::kColA + 32 * b, a);
                        tmem_ld_wait();
                        const bool diag = (b == q4);
                        // walk s from the block's last column down: the factor grows by lambda per step
                        float f = diag ? 1.f : exp2f(g * static_cast<float>(i - (32 * b + 31)));
#pragma unroll
                        for (int j = 31; j >= 0; --j) {
                            const bool ok = !diag || (32 * b + j <= i);
                            a[j] = ok ? a[j] * f : 0.f;
                            f = ok ? f * lam : f;
                        }
#pragma unroll
                        for (int m = 0; m < 16; ++m) pk[m] = pack_bf16x2(a[2 * m], a[2 * m + 1]);
                    }
                    tmem_st16(lane_addr + Cfg::kColA + p_block_col(b), pk);
                }
                tmem_st_wait();
                tc_fence_before();
            }

            // ---- K' = diag(lambda^(Lc-1-s)) K in place (rows past the segment end -> 0)
            if (!warp_wait(&full[s], r & 1, lane)) {
                if (lane == 0) *reinterpret_cast<volatile int *>(abort_flag) = 1;
                break;
            }
            {
                const float f = krow < Lc ? exp2f(g * static_cast<float>(Lc - 1 - krow)) : 0.f;
                uint8_t *kt = st + (kStateOnly ? 0 : kTileBytes);
                scale_row_bf16(kt + kslab * kSlabBytes + krow * 128, krow, f);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_P);

            // ---- state update S = lambda^Lc S + dS
            if (!warp_wait(bar_O, static_cast<uint32_t>(c) & 1, lane)) {
                if (lane == 0) *reinterpret_cast<volatile int *>(abort_flag) = 1;
                break;
            }
            tc_fence_after();
            {
                const float lamL = exp2f(g * static_cast<float>(Lc));
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float d[32];
                    tmem_ld32(lane_addr + Cfg::kColDs + 64 * hf + 32 * half, d);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) S[32 * half + j] = fmaf(lamL, S[32 * half + j], d[j]);
                }
            }
            if (!kStateOnly) {
                store_state_bf16(sbf, hf, i, S);
                fence_proxy_async_smem();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_Sd);

            if (!kStateOnly) {
                // ---- O = O_intra + lambda^(i+1) O_inter -> bf16 -> global (valid rows only)
                const float rs = exp2f(g * static_cast<float>(i + 1));
                __nv_bfloat16 *orow =
                    args.o + (static_cast<size_t>(tok0 + c * kC + i) * H + h) * kD + 64 * hf;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float on[32], oi[32];
                    tmem_ld32(lane_addr + Cfg::kColOn + 64 * hf + 32 * half, on);
                    tmem_ld32(lane_addr + Cfg::kColOi + 64 * hf + 32 * half, oi);
                    tmem_ld_wait();
                    if (i < Lc) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint4 w;
                            w.x = pack_bf16x2(fmaf(rs, oi[8 * j + 0], on[8 * j + 0]), fmaf(rs, oi[8 * j + 1], on[8 * j + 1]));
                            w.y = pack_bf16x2(fmaf(rs, oi[8 * j + 2], on[8 * j + 2]), fmaf(rs, oi[8 * j + 3], on[8 * j + 3]));
                            w.z = pack_bf16x2(fmaf(rs, oi[8 * j + 4], on[8 * j + 4]), fmaf(rs, oi[8 * j + 5], on[8 * j + 5]));
                            w.w = pack_bf16x2(fmaf(rs, oi[8 * j + 6], on[8 * j + 6]), fmaf(rs, oi[8 * j + 7], on[8 * j + 7]));
                            st_global_v4(orow + 32 * half + 8 * j, w);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_Of);
            }
        }

        // ---- write the state this unit produces
        float *dst = nullptr;
        if (kStateOnly) {
            dst = args.seg_state + (static_cast<size_t>(unit) * H + h) * DD;
        } else if ((flags & kUnitLast) && args.s_final) {
            dst = args.s_final + (static_cast<size_t>(seq) * H + h) * DD;
        }
        if (dst) {
            float4 *p = reinterpret_cast<float4 *>(dst + static_cast<size_t>(i) * kD + 64 * hf);
#pragma unroll
            for (int j = 0; j < 16; ++j) p[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

}  // namespace la
