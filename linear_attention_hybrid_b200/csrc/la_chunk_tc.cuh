// Chunked Lightning Attention prefill on the sm_100a tensor cores (tcgen05 +
// TMEM), fed by TMA.
//
// The recurrence S_t = lambda S_{t-1} + k_t^T v_t, o_t = q_t S_t has a serial
// dependency along the sequence (Ling & Ring 2.6 Technical Report, blog post
// news.neo-ai.one/en/article/3021, section "Long-Context Training: Context
// Parallel for Lightning Attention"). Blocking it into chunks of C = 128
// tokens turns each chunk into dense contractions (the O(n) form of section
// "Hybrid Linear Attention"); with rows i and columns s 0-based inside the
// chunk, Lc valid rows, and S the state entering the chunk:
//
//   A      = Q K^T                                     (C x C,  tensor core)
//   P[i,s] = A[i,s] lambda^(i-s)  for s <= i, else 0   (registers)
//   O      = P V + diag(lambda^(i+1)) (Q S)            (tensor core, two accumulators)
//   S     <- lambda^Lc S + (diag(lambda^(Lc-1-s)) K)^T V  (tensor core + registers)
//
// Precision. Q, K, V are bf16 inputs, so their products are exact in the fp32
// accumulators. P, S and K' = diag(lambda^(Lc-1-s)) K are made here in fp32;
// rounding them to bf16 once costs up to 2^-9 relative per entry, which for
// long-memory heads adds up to about the whole 2e-2 max-error budget. Each is
// therefore split as x = hi + lo with hi = bf16(x), lo = bf16(x - hi), and both
// halves are multiplied (relative error ~2^-17): 7 products of 128^3 per chunk.
//
// Roles (352 threads): warp 0 issues TMA loads, warp 1 (one thread) issues
// tcgen05.mma and owns TMEM, warps 2-9 are the epilogue: two warpgroups, each
// owning 64 of the 128 columns of every 128-lane TMEM tile (warp w may touch
// lanes 32*(w%4)..+31 only); warp 10 issues the TMA stores of O and waits for
// them, so no other warp blocks on an output transfer.
//
// TMEM, 512 columns: [0,128) scores A; each 32-column block b is overwritten in
// place by P_hi (16 columns of packed bf16 pairs) then P_lo (16 columns);
// [128,256) O_intra = P V; [256,384) O_inter = Q S; [384,512) dS = K'^T V.
// The fp32 state S never leaves the chip: each epilogue thread keeps 64 entries
// of one row in registers.
//
// Shared memory: two (Q, K) slot pairs and one V slot (each slot a [128 x 128]
// bf16 tile as two 64-column slabs with 128-byte rows and the 128-byte
// swizzle), plus a 64 KB output staging area. Pair c%2 is reused within chunk
// c's life:
//   Q slot: Q_c -> K'_lo(c) once Q S is done -> S_lo(c) once dS is done
//   K slot: K_c -> K'_hi(c) in place           -> S_hi(c) once dS is done
// and S(c) is read by the next chunk's Q S, after which Q and K of chunk c+2
// load into the pair. V of chunk c+1 loads once dS of chunk c is done. O is
// staged as soon as P V is done (before dS) and leaves by TMA while the next
// chunk computes.
#pragma once

#include "la_ptx.cuh"

namespace la {

constexpr int kC = 128;                     // chunk length = MMA M
constexpr int kD = 128;                     // head dim handled by this kernel
constexpr int kSlabBytes = 128 * 128;       // [128 rows x 64 bf16] slab, 128-byte rows
constexpr int kTileBytes = 2 * kSlabBytes;  // [128 x 128] bf16 tile = two slabs
constexpr int kTcThreads = 352;    // main kernel: producer, MMA, 8 epilogue warps, store warp
constexpr int kStoreWarp = 10;
constexpr int kStateThreads = 320; // state-only kernel: producer, MMA, 8 epilogue warps

enum UnitFlags { kUnitFirst = 1, kUnitLast = 2 };

// Phase timestamps of one CTA (unit 0, head 0), for profiling builds only
// (compiled with LA_TRACE_PHASES); read with la_debug_phase_dump.
#ifdef LA_TRACE_PHASES
constexpr int kPhaseChunks = 64, kPhaseEvents = 24;
__device__ long long g_la_phase[kPhaseChunks][kPhaseEvents];
#define LA_PHASE(c, ev)                                                                        \
    do {                                                                                       \
        if (blockIdx.x == 0 && blockIdx.y == 0 && (c) < kPhaseChunks) g_la_phase[(c)][(ev)] = clock64(); \
    } while (0)
#else
#define LA_PHASE(c, ev) \
    do {                \
    } while (0)
#endif

struct ChunkArgs {
    void *o;                    // [T, H, D], bf16 or fp32 (the kernel's OutT)
    const float *s_init;        // [nseq, H, D, D] or null
    float *s_final;             // [nseq, H, D, D] or null
    const float *slopes;        // [H] or null
    const int4 *units;          // plan: {tok0, len, seq, flags}
    const int *n_units;         // plan size (device)
    float *seg_state;           // [cap, H, D, D] workspace
    int H;
};

// Shared memory of the main kernel: two (Q, K) slot pairs, one V slot and a
// 64 KB output staging area (fp32 [128 x 128]).
struct ChunkCfg {
    static constexpr int kOffQ = 0;                       // 2 x 32 KB
    static constexpr int kOffK = 2 * kTileBytes;          // 2 x 32 KB
    static constexpr int kOffV = 4 * kTileBytes;          // 32 KB
    static constexpr int kOffO = 5 * kTileBytes;          // 64 KB
    static constexpr int kBarOffset = 7 * kTileBytes;
    static constexpr int kSmemBytes = kBarOffset + 256 + 1024;  // barriers + alignment slack
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColA = 0, kColOn = 128, kColOi = 256, kColDs = 384;
};

struct StateCfg {
    static constexpr int kStages = 2;
    static constexpr int kStageBytes = 3 * kTileBytes;  // K, V, K'_lo
    static constexpr int kBarOffset = kStages * kStageBytes;
    static constexpr int kSmemBytes = kBarOffset + 256 + 1024;
    static constexpr uint32_t kTmemCols = 128;
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
// TMEM column (within the score tile) of the 16-wide K step kk of P_hi; P_lo is 16 further.
__device__ __forceinline__ uint32_t p_hi_col(int kk) { return 32u * (kk >> 1) + 8u * (kk & 1); }

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

__device__ __forceinline__ void set_abort(int *flag) { *reinterpret_cast<volatile int *>(flag) = 1; }

// Split x = hi + lo into two bf16 pairs (lo carries the bits hi drops).
__device__ __forceinline__ void split_pack(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    hi = pack_bf16x2(x0, x1);
    lo = pack_bf16x2(x0 - bf16lo_to_f32(hi), x1 - bf16hi_to_f32(hi));
}

// K' = f * K for one 128-byte row of a K tile: hi written back in place, lo to
// the same position of another tile. Chunks are visited starting at (row & 7)
// so that a warp's 32 rows hit every bank.
__device__ __forceinline__ void scale_row_split(uint8_t *row_hi, uint8_t *row_lo, int row, float f) {
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
        const int j = (jj + row) & 7;
        const uint4 x = *reinterpret_cast<const uint4 *>(row_hi + 16 * j);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) split_pack(bf16lo_to_f32(w[m]) * f, bf16hi_to_f32(w[m]) * f, hi[m], lo[m]);
        *reinterpret_cast<uint4 *>(row_hi + 16 * j) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4 *>(row_lo + 16 * j) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
}

// Store 64 fp32 state entries of row `row` (columns [64*half, 64*half+64)) split
// into bf16 hi / lo, into two MN-major swizzled state tiles: slab `half`,
// 128-byte row `row`, 16-byte chunk j at j ^ (row & 7).
__device__ __forceinline__ void store_state_split(uint8_t *t_hi, uint8_t *t_lo, int half, int row,
                                                  const float (&S)[64]) {
    const int off = half * kSlabBytes + row * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) split_pack(S[8 * j + 2 * m], S[8 * j + 2 * m + 1], hi[m], lo[m]);
        const int c = 16 * (j ^ (row & 7));
        *reinterpret_cast<uint4 *>(t_hi + off + c) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        if (t_lo) *reinterpret_cast<uint4 *>(t_lo + off + c) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
}

// Store 32 consecutive fp32 values of one output row to global memory as bf16 (4 x 16 B) or fp32 (8 x 16 B).
__device__ __forceinline__ void store_row32(__nv_bfloat16 *dst, const float (&x)[32]) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
        st_global_v4(dst + 8 * j, make_uint4(pack_bf16x2(x[8 * j + 0], x[8 * j + 1]), pack_bf16x2(x[8 * j + 2], x[8 * j + 3]),
                                             pack_bf16x2(x[8 * j + 4], x[8 * j + 5]), pack_bf16x2(x[8 * j + 6], x[8 * j + 7])));
}
__device__ __forceinline__ void store_row32(float *dst, const float (&x)[32]) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
        st_global_v4(dst + 4 * j, make_uint4(__float_as_uint(x[4 * j]), __float_as_uint(x[4 * j + 1]),
                                             __float_as_uint(x[4 * j + 2]), __float_as_uint(x[4 * j + 3])));
}

// Stage 32 consecutive output values of row `row` (columns [32*q32, 32*q32+32)) in
// shared memory for a TMA store with the 128-byte swizzle.
// fp32: box q32 is a [128 rows x 32 fp32] tile of 16 KB.
__device__ __forceinline__ void stage_row32(uint8_t *stg, int q32, int row, const float (&x)[32], float *) {
    uint8_t *base = stg + q32 * kSlabBytes + row * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint4 *>(base + 16 * (j ^ (row & 7))) =
            make_uint4(__float_as_uint(x[4 * j]), __float_as_uint(x[4 * j + 1]), __float_as_uint(x[4 * j + 2]),
                       __float_as_uint(x[4 * j + 3]));
}
// bf16: box q32/2 is a [128 rows x 64 bf16] tile of 16 KB; 32 values fill half a row.
__device__ __forceinline__ void stage_row32(uint8_t *stg, int q32, int row, const float (&x)[32], __nv_bfloat16 *) {
    uint8_t *base = stg + (q32 >> 1) * kSlabBytes + row * 128;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int c = 4 * (q32 & 1) + j;
        *reinterpret_cast<uint4 *>(base + 16 * (c ^ (row & 7))) =
            make_uint4(pack_bf16x2(x[8 * j + 0], x[8 * j + 1]), pack_bf16x2(x[8 * j + 2], x[8 * j + 3]),
                       pack_bf16x2(x[8 * j + 4], x[8 * j + 5]), pack_bf16x2(x[8 * j + 6], x[8 * j + 7]));
    }
}

// Output tile boxes: fp32 -> 4 boxes of 32 columns, bf16 -> 2 boxes of 64 columns.
template <typename OutT>
struct OutBoxes {
    static constexpr int kCount = sizeof(OutT) == 4 ? 4 : 2;
    static constexpr int kCols = kD / kCount;
};

// ============================================================================ main chunk kernel
template <typename OutT>
__global__ void __launch_bounds__(kTcThreads, 1)
    la_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                       const ChunkArgs args) {
    using Cfg = ChunkCfg;
    const int unit = blockIdx.x;
    const int h = blockIdx.y;
    if (unit >= *args.n_units) return;
    const int4 u = args.units[unit];
    const int tok0 = u.x, len = u.y, seq = u.z, flags = u.w;
    const int nchunks = (len + kC - 1) / kC;
    const int H = args.H;
    const float g = decay_log2(args.slopes, h, H);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *v_slot = smem + Cfg::kOffV;
    uint8_t *stg = smem + Cfg::kOffO;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOffset);
    uint64_t *full_qk = bars;            // [2] Q and K of a chunk landed
    uint64_t *empty_qk = bars + 2;       // [2] slot pair free again (the state it held was read)
    uint64_t *full_v = bars + 4;         // V landed
    uint64_t *empty_v = bars + 5;        // V slot free (dS of the previous chunk done)
    uint64_t *bar_S = bars + 6;          // A = Q K^T in TMEM
    uint64_t *bar_QS = bars + 7;         // O_inter = Q S done (Q slot readable as scratch)
    uint64_t *bar_PV = bars + 8;         // O_intra = P V done
    uint64_t *bar_O = bars + 9;          // dS done
    uint64_t *bar_P = bars + 10;         // P hi/lo in TMEM (8 epilogue warps)
    uint64_t *bar_K = bars + 11;         // K' hi/lo in shared memory (8 warps)
    uint64_t *bar_Of = bars + 12;        // O accumulators read (8 warps)
    uint64_t *bar_E = bars + 13;         // O staged (8 warps)
    uint64_t *bar_F = bars + 14;         // O staging free again (store warp)
    uint64_t *bar_Sd = bars + 15;        // dS read and S hi/lo written (8 warps)
    uint64_t *bar_done = bars + 16;      // every MMA retired
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 17);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    auto q_slot = [&](int s) { return smem + Cfg::kOffQ + s * kTileBytes; };
    auto k_slot = [&](int s) { return smem + Cfg::kOffK + s * kTileBytes; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&full_qk[s], 1);
            mbar_init(&empty_qk[s], 1);
        }
        mbar_init(full_v, 1);
        mbar_init(empty_v, 1);
        mbar_init(bar_S, 1);
        mbar_init(bar_QS, 1);
        mbar_init(bar_PV, 1);
        mbar_init(bar_O, 1);
        mbar_init(bar_P, 8);
        mbar_init(bar_K, 8);
        mbar_init(bar_Of, 8);
        mbar_init(bar_E, 8);
        mbar_init(bar_F, 1);
        mbar_init(bar_Sd, 8);
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
        // Q, K of chunk c go to slot pair c%2 once the state that pair held has been read
        // (Q S of chunk c-1); V of chunk c once dS of chunk c-1 is done.
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int issued_qk = 0, issued_v = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c & 1;
                const int t = tok0 + c * kC;
                if (c >= 1 && !mbar_wait(&empty_qk[s], static_cast<uint32_t>((c - 1) >> 1) & 1)) break;
                if (*reinterpret_cast<volatile int *>(abort_flag)) break;
                LA_PHASE(c, 16);
                mbar_arrive_expect_tx(&full_qk[s], 2 * kTileBytes);
                tma_load_3d(q_slot(s), &tm_q, 0, h, t, &full_qk[s]);
                tma_load_3d(q_slot(s) + kSlabBytes, &tm_q, 64, h, t, &full_qk[s]);
                tma_load_3d(k_slot(s), &tm_k, 0, h, t, &full_qk[s]);
                tma_load_3d(k_slot(s) + kSlabBytes, &tm_k, 64, h, t, &full_qk[s]);
                issued_qk = c + 1;
                if (c >= 1 && !mbar_wait(empty_v, static_cast<uint32_t>(c - 1) & 1)) break;
                if (*reinterpret_cast<volatile int *>(abort_flag)) break;
                LA_PHASE(c, 17);
                mbar_arrive_expect_tx(full_v, kTileBytes);
                tma_load_3d(v_slot, &tm_v, 0, h, t, full_v);
                tma_load_3d(v_slot + kSlabBytes, &tm_v, 64, h, t, full_v);
                issued_v = c + 1;
            }
            if (issued_qk < nchunks) set_abort(abort_flag);
            // Never leave with a copy in flight: wait (bounded) for the last loads.
            for (int c = (issued_qk > 2 ? issued_qk - 2 : 0); c < issued_qk; ++c)
                mbar_wait(&full_qk[c & 1], static_cast<uint32_t>(c >> 1) & 1);
            if (issued_v > 0) mbar_wait(full_v, static_cast<uint32_t>(issued_v - 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_qk = idesc_bf16_f32(kC, kC, false, false);
            constexpr uint32_t id_pv = idesc_bf16_f32(kC, kD, false, true);
            constexpr uint32_t id_qs = idesc_bf16_f32(kC, kD, false, true);
            constexpr uint32_t id_ds = idesc_bf16_f32(kD, kD, true, true);
            const uint32_t va = smem_u32(v_slot);
            for (int c = 0; c < nchunks; ++c) {
                const int s = c & 1;
                const uint32_t qa = smem_u32(q_slot(s)), ka = smem_u32(k_slot(s));
                // the state entering chunk c: S_hi in the K slot, S_lo in the Q slot of pair c-1
                const uint32_t shi = smem_u32(k_slot(s ^ 1)), slo = smem_u32(q_slot(s ^ 1));
                if (!mbar_wait(&full_qk[s], static_cast<uint32_t>(c >> 1) & 1)) break;
                LA_PHASE(c, 0);
                tc_fence_after();
                // A = Q K^T
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    mma_ss(tmem + Cfg::kColA, desc_kmajor(qa, kk), desc_kmajor(ka, kk), id_qk, kk > 0);
                mma_commit(bar_S);
                LA_PHASE(c, 1);
                // O_inter = Q (S_hi + S_lo)
                if (!mbar_wait(bar_Sd, static_cast<uint32_t>(c) & 1)) break;
                if (c > 0 && !mbar_wait(bar_Of, static_cast<uint32_t>(c - 1) & 1)) break;
                LA_PHASE(c, 2);
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    mma_ss(tmem + Cfg::kColOi, desc_kmajor(qa, kk), desc_mnmajor(shi, kk), id_qs, kk > 0);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    mma_ss(tmem + Cfg::kColOi, desc_kmajor(qa, kk), desc_mnmajor(slo, kk), id_qs, 1);
                mma_commit(bar_QS);
                mma_commit(&empty_qk[s ^ 1]);
                LA_PHASE(c, 3);
                // O_intra = (P_hi + P_lo) V, P from TMEM
                if (!mbar_wait(full_v, static_cast<uint32_t>(c) & 1)) break;
                if (!mbar_wait(bar_P, static_cast<uint32_t>(c) & 1)) break;
                LA_PHASE(c, 4);
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ts(tmem + Cfg::kColOn, tmem + Cfg::kColA + p_hi_col(kk), desc_mnmajor(va, kk), id_pv, kk > 0);
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ts(tmem + Cfg::kColOn, tmem + Cfg::kColA + p_hi_col(kk) + 16, desc_mnmajor(va, kk), id_pv, 1);
                mma_commit(bar_PV);
                LA_PHASE(c, 5);
                // dS = (K'_hi + K'_lo)^T V
                if (!mbar_wait(bar_K, static_cast<uint32_t>(c) & 1)) break;
                LA_PHASE(c, 6);
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ss(tmem + Cfg::kColDs, desc_mnmajor(ka, kk), desc_mnmajor(va, kk), id_ds, kk > 0);
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ss(tmem + Cfg::kColDs, desc_mnmajor(qa, kk), desc_mnmajor(va, kk), id_ds, 1);
                mma_commit(bar_O);
                mma_commit(empty_v);
                LA_PHASE(c, 7);
            }
            mma_commit(bar_done);
            mbar_wait(bar_done, 0);
        }
    } else if (warp == kStoreWarp) {
        // ------------------------------------------------------------ output store warp
        if (lane == 0) {
            for (int c = 0; c < nchunks; ++c) {
                if (!mbar_wait(bar_E, static_cast<uint32_t>(c) & 1)) {
                    set_abort(abort_flag);
                    break;
                }
                const int Lc = min(kC, len - c * kC);
                if (Lc == kC) {
                    using Box = OutBoxes<OutT>;
#pragma unroll
                    for (int bx = 0; bx < Box::kCount; ++bx)
                        tma_store_3d(&tm_o, stg + bx * kSlabBytes, bx * Box::kCols, h, tok0 + c * kC);
                    tma_store_commit();
                    LA_PHASE(c, 20);
                    tma_store_wait_read();
                }
                mbar_arrive(bar_F);
                LA_PHASE(c, 15);
            }
            tma_store_wait_all();
        }
    } else if (warp >= 2 && warp < 10) {
        // ------------------------------------------------------------ epilogue (warps 2..9)
        const int e = warp - 2;          // 0..7
        const int q4 = warp & 3;         // TMEM lane quarter this warp may access
        const int hf = e >> 2;           // column half
        const int i = 32 * q4 + lane;    // TMEM lane = chunk row i (A, O) or state row dk (dS)
        const int et = e * 32 + lane;    // 0..255
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * q4) << 16);
        const float lam = exp2f(g);
        const size_t DD = static_cast<size_t>(kD) * kD;

        float S[64];
        {
            const float *src = nullptr;
            if ((flags & kUnitFirst) && (flags & kUnitLast)) {
                if (args.s_init) src = args.s_init + (static_cast<size_t>(seq) * H + h) * DD;
            } else {
                src = args.seg_state + (static_cast<size_t>(unit) * H + h) * DD;
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
        // the state entering chunk 0 sits in slot pair 1 (free until Q S of chunk 0 has read it)
        store_state_split(k_slot(1), q_slot(1), hf, i, S);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_Sd);

        bool ok = true;
        for (int c = 0; c < nchunks && ok; ++c) {
            if (warp_aborted(abort_flag, lane)) break;
            const int s = c & 1;
            const int Lc = min(kC, len - c * kC);

            // ---- P = decay-masked A, split into bf16 hi / lo, in place in TMEM
            if (!(ok = warp_wait(bar_S, static_cast<uint32_t>(c) & 1, lane))) break;
            if (et == 0) LA_PHASE(c, 8);
            tc_fence_after();
#pragma unroll
            for (int bb = 0; bb < 2; ++bb) {
                const int b = 2 * hf + bb;  // 32-column block of A
                uint32_t hi[16], lo[16];
                if (b > q4) {
#pragma unroll
                    for (int m = 0; m < 16; ++m) hi[m] = lo[m] = 0u;
                } else {
                    float a[32];
                    tmem_ld32(lane_addr + Cfg::kColA + 32 * b, a);
                    tmem_ld_wait();
                    const bool diag = (b == q4);
                    // walk s down from the block's last column: the factor grows by lambda per step
                    float f = diag ? 1.f : exp2f(g * static_cast<float>(i - (32 * b + 31)));
#pragma unroll
                    for (int j = 31; j >= 0; --j) {
                        const bool in = !diag || (32 * b + j <= i);
                        a[j] = in ? a[j] * f : 0.f;
                        f = in ? f * lam : f;
                    }
#pragma unroll
                    for (int m = 0; m < 16; ++m) split_pack(a[2 * m], a[2 * m + 1], hi[m], lo[m]);
                }
                tmem_st16(lane_addr + Cfg::kColA + 32 * b, hi);
                tmem_st16(lane_addr + Cfg::kColA + 32 * b + 16, lo);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_P);
            if (et == 0) LA_PHASE(c, 9);
            if (et == 255) LA_PHASE(c, 18);

            // ---- K' = diag(lambda^(Lc-1-s)) K: hi in place, lo in the (already read) Q slot
            if (!(ok = warp_wait(&full_qk[s], static_cast<uint32_t>(c >> 1) & 1, lane))) break;
            if (!(ok = warp_wait(bar_QS, static_cast<uint32_t>(c) & 1, lane))) break;
            if (et == 0) LA_PHASE(c, 10);
            {
                const int krow = et & 127, kslab = et >> 7;
                const float f = krow < Lc ? exp2f(g * static_cast<float>(Lc - 1 - krow)) : 0.f;
                const int off = kslab * kSlabBytes + krow * 128;
                scale_row_split(k_slot(s) + off, q_slot(s) + off, krow, f);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_K);
            if (et == 0) LA_PHASE(c, 11);

            // ---- O = O_intra + lambda^(i+1) O_inter: staged for the store warp, or stored row by row
            //      (a chunk cut short by its sequence end must not write past it)
            if (!(ok = warp_wait(bar_PV, static_cast<uint32_t>(c) & 1, lane))) break;
            if (c > 0 && !(ok = warp_wait(bar_F, static_cast<uint32_t>(c - 1) & 1, lane))) break;
            if (et == 0) LA_PHASE(c, 12);
            tc_fence_after();
            {
                const bool whole = (Lc == kC);
                const float rs = exp2f(g * static_cast<float>(i + 1));
                OutT *orow = static_cast<OutT *>(args.o) + (static_cast<size_t>(tok0 + c * kC + i) * H + h) * kD + 64 * hf;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float on[32], oi[32];
                    tmem_ld32(lane_addr + Cfg::kColOn + 64 * hf + 32 * half, on);
                    tmem_ld32(lane_addr + Cfg::kColOi + 64 * hf + 32 * half, oi);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) on[j] = fmaf(rs, oi[j], on[j]);
                    if (whole) stage_row32(stg, 2 * hf + half, i, on, static_cast<OutT *>(nullptr));
                    else if (i < Lc) store_row32(orow + 32 * half, on);
                }
                tc_fence_before();
                if (whole) fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar_Of);
                mbar_arrive(bar_E);
            }
            if (et == 0) LA_PHASE(c, 14);
            if (et == 255) LA_PHASE(c, 19);

            // ---- S = lambda^Lc S + dS; S_hi -> this pair's K slot, S_lo -> its Q slot (both read by dS)
            if (!(ok = warp_wait(bar_O, static_cast<uint32_t>(c) & 1, lane))) break;
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
            store_state_split(k_slot(s), q_slot(s), hf, i, S);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_Sd);
            if (et == 0) LA_PHASE(c, 13);
        }

        // ---- the state after this unit
        if (ok && (flags & kUnitLast) && args.s_final) {
            float4 *p = reinterpret_cast<float4 *>(args.s_final + (static_cast<size_t>(seq) * H + h) * DD +
                                                   static_cast<size_t>(i) * kD + 64 * hf);
#pragma unroll
            for (int j = 0; j < 16; ++j) p[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
        }
        if (!ok && lane == 0) set_abort(abort_flag);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

// ============================================================================ segment-state kernel
// First pass of the segment split: the state dS a segment produces from a zero
// start, S <- lambda^Lc S + (K'_hi + K'_lo)^T V per chunk, written to the
// workspace. Only K and V are read.
__global__ void __launch_bounds__(kStateThreads, 1)
    la_state_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const ChunkArgs args) {
    using Cfg = StateCfg;
    const int unit = blockIdx.x;
    const int h = blockIdx.y;
    if (unit >= *args.n_units) return;
    const int4 u = args.units[unit];
    if (u.w & kUnitLast) return;  // the last segment's own state is never needed
    const int tok0 = u.x, len = u.y;
    const int nchunks = (len + kC - 1) / kC;
    const int H = args.H;
    const float g = decay_log2(args.slopes, h, H);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOffset);
    uint64_t *full = bars;           // [2]
    uint64_t *empty = bars + 2;      // [2]
    uint64_t *bar_K = bars + 4;      // K' hi/lo ready (8 warps)
    uint64_t *bar_O = bars + 5;      // dS ready
    uint64_t *bar_Sd = bars + 6;     // dS consumed (8 warps)
    uint64_t *bar_done = bars + 7;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 8);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
    auto k_slot = [&](int s) { return smem + s * Cfg::kStageBytes; };
    auto v_slot = [&](int s) { return smem + s * Cfg::kStageBytes + kTileBytes; };
    auto x_slot = [&](int s) { return smem + s * Cfg::kStageBytes + 2 * kTileBytes; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(bar_K, 8);
        mbar_init(bar_O, 1);
        mbar_init(bar_Sd, 8);
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
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int issued = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c & 1;
                if (c >= 2 && !mbar_wait(&empty[s], static_cast<uint32_t>((c - 2) >> 1) & 1)) {
                    set_abort(abort_flag);
                    break;
                }
                if (*reinterpret_cast<volatile int *>(abort_flag)) break;
                const int t = tok0 + c * kC;
                mbar_arrive_expect_tx(&full[s], 2 * kTileBytes);
                tma_load_3d(k_slot(s), &tm_k, 0, h, t, &full[s]);
                tma_load_3d(k_slot(s) + kSlabBytes, &tm_k, 64, h, t, &full[s]);
                tma_load_3d(v_slot(s), &tm_v, 0, h, t, &full[s]);
                tma_load_3d(v_slot(s) + kSlabBytes, &tm_v, 64, h, t, &full[s]);
                issued = c + 1;
            }
            for (int c = (issued > 2 ? issued - 2 : 0); c < issued; ++c)
                mbar_wait(&full[c & 1], static_cast<uint32_t>(c >> 1) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t id_ds = idesc_bf16_f32(kD, kD, true, true);
            for (int c = 0; c < nchunks; ++c) {
                const int s = c & 1;
                const uint32_t ka = smem_u32(k_slot(s)), va = smem_u32(v_slot(s)), xa = smem_u32(x_slot(s));
                if (c > 0 && !mbar_wait(bar_Sd, static_cast<uint32_t>(c - 1) & 1)) break;
                if (!mbar_wait(bar_K, static_cast<uint32_t>(c) & 1)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ss(tmem, desc_mnmajor(ka, kk), desc_mnmajor(va, kk), id_ds, kk > 0);
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ss(tmem, desc_mnmajor(xa, kk), desc_mnmajor(va, kk), id_ds, 1);
                mma_commit(bar_O);
                mma_commit(&empty[s]);
            }
            mma_commit(bar_done);
            mbar_wait(bar_done, 0);
        }
    } else if (warp >= 2 && warp < 10) {
        const int e = warp - 2;
        const int q4 = warp & 3;
        const int hf = e >> 2;
        const int i = 32 * q4 + lane;
        const int et = e * 32 + lane;
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * q4) << 16);
        float S[64];
#pragma unroll
        for (int j = 0; j < 64; ++j) S[j] = 0.f;
        bool ok = true;
        for (int c = 0; c < nchunks && ok; ++c) {
            if (warp_aborted(abort_flag, lane)) break;
            const int s = c & 1;
            const uint32_t r = static_cast<uint32_t>(c >> 1);
            const int Lc = min(kC, len - c * kC);
            if (!(ok = warp_wait(&full[s], r & 1, lane))) break;
            {
                const int krow = et & 127, kslab = et >> 7;
                const float f = krow < Lc ? exp2f(g * static_cast<float>(Lc - 1 - krow)) : 0.f;
                const int off = kslab * kSlabBytes + krow * 128;
                scale_row_split(k_slot(s) + off, x_slot(s) + off, krow, f);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_K);
            if (!(ok = warp_wait(bar_O, static_cast<uint32_t>(c) & 1, lane))) break;
            tc_fence_after();
            const float lamL = exp2f(g * static_cast<float>(Lc));
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float d[32];
                tmem_ld32(lane_addr + 64 * hf + 32 * half, d);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) S[32 * half + j] = fmaf(lamL, S[32 * half + j], d[j]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_Sd);
        }
        if (ok) {
            float4 *p = reinterpret_cast<float4 *>(args.seg_state + (static_cast<size_t>(unit) * H + h) * kD * kD +
                                                   static_cast<size_t>(i) * kD + 64 * hf);
#pragma unroll
            for (int j = 0; j < 16; ++j) p[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
        } else if (lane == 0) {
            set_abort(abort_flag);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

}  // namespace la
