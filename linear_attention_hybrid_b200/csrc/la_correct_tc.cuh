// Entry states and output correction of the corrected segment split (forward
// prefill), on the sm_100a tensor cores.
//
// The report's single-GPU "local recursion + global correction" (Ling & Ring
// 2.6 Technical Report, blog post news.neo-ai.one/en/article/3021, section
// "Long-Context Training: Context Parallel for Lightning Attention": each
// sub-sequence runs its own recursion, then its outputs are corrected for the
// state entering it). In the corrected split every coarse segment of a
// sequence starts at once: the entry segment from the given initial state,
// every other one from zero. Each writes its outputs and its exit state X_f
// (la_chunk_tc_kernel with `corrected` set). A token's output depends on the
// state entering its segment only through lambda^(t - t_w + 1) q_t E_w, t_w the
// segment's first token, so with
//   E_w = sum over the sequence's earlier segments f of lambda^(t_w - end_f) X_f
// (the state that truly enters segment w), the output of chunk c (0-based in
// the segment, rows i) is completed by
//   O_c += diag(lambda^(cC + i + 1)) Q_c E_w
// and the sequence's final state is the sum over all its segments f of
// lambda^(end - end_f) X_f.
//
// la_entry_state_kernel forms every E_w once, split into bf16 hi + lo exactly
// as the chunk kernel stores S for its Q S product (the two swizzled 32 KB
// shared-memory tiles, written to the workspace as one 64 KB image), and the
// final states. la_correct_tc_kernel then runs one CTA per (segment, piece of
// a few chunks, head), slow-decay heads first: the E image arrives by one bulk
// copy (with two segments per sequence E_w is the exit state of segment w-1 and
// the CTA splits it itself; the first piece then also forms the final state),
// and per chunk the tensor core forms Q_c (E_hi + E_lo) into a
// double-buffered TMEM accumulator while TMA brings the next Q tiles (three
// stages); 16 epilogue
// warps stage the scaled product in the output type and a reduce warp adds it to
// the outputs in global memory with a TMA reduce-add (atomic, in L2), so the
// outputs are never read here. Chunks whose largest factor lambda^(cC + 1) is
// below 2^-150 (0 in fp32 on every row) are skipped.
#pragma once

#include "la_chunk_tc.cuh"

namespace la {

constexpr int kEntryThreads = 512;
constexpr int kCorrThreads = 608;   // producer, MMA, reduce warp, 16 epilogue warps
constexpr int kCorrStoreWarp = 2;
constexpr int kCorrEpi0 = 3;
constexpr int kCorrWarps = 16;
constexpr uint32_t kEntryImageBytes = 2 * kTileBytes;   // E_hi tile, then E_lo tile

template <typename OutT>
struct CorrCfg {
    using St = OutStaging<OutT>;
    static constexpr int kOffE = 0;                                       // E image (64 KB)
    static constexpr int kQStages = 3;
    static constexpr int kOffQ = 2 * kTileBytes;                          // Q stages
    static constexpr int kOBytes = kC * kD * static_cast<int>(sizeof(OutT));   // a correction tile as TMA boxes
    static constexpr int kOStages = sizeof(OutT) == 4 ? 1 : 2;
    static constexpr int kOffO = kOffQ + kQStages * kTileBytes;
    static constexpr int kBarOffset = kOffO + kOStages * kOBytes;
    static constexpr int kSmemBytes = kBarOffset + 256 + 1024;
    static constexpr uint32_t kTmemCols = 256;                            // two accumulators
    static_assert(kSmemBytes <= 232448, "the correction kernel's shared memory exceeds 227 KB");
};

struct CorrArgs {
    void *o;                    // [T, H, D] outputs of the segments, corrected in place
    float *s_final;             // [nseq, H, D, D] or null
    const float *slopes;        // [H] or null
    WorkMap map;                // R = 1: one fine unit per coarse segment
    const float *seg_state;     // [fine units, H, 128, 128]: exit state X of each segment
    uint8_t *e_img;             // [coarse units, H] 64 KB images of E_hi / E_lo, or null: two segments per
                                // sequence, E_w is the exit state of segment w-1, formed by the correction CTA
    int H;
    int D;
    int units;                  // coarse units planned (the entry kernel's grid)
    int chunks;                 // chunks per correction piece
    int pieces;                 // pieces per segment
    int items;                  // correction CTAs per head
};

// The final state of multi-segment sequence `seq`, sum over its segments f of lambda^(end - end_f) X_f: thread
// t of `nthreads` takes rows t / 4, t / 4 + nthreads / 4, .. and columns 32 (t % 4)..+31 (nthreads a multiple of 4).
__device__ __forceinline__ void final_state(const CorrArgs &args, int seq, int h, float g, int t, int nthreads) {
    const int H = args.H, Dm = args.D;
    const size_t kDD = static_cast<size_t>(kD) * kD;
    const int f0 = seq_first_fine(args.map, seq), f1 = seq_end_fine(args.map, seq);
    if (f1 - f0 < 2 || !args.s_final) return;   // one segment: the chunk kernel wrote its final state
    int4 last;
    if (!fine_unit(args.map, f1 - 1, last)) return;
    const int end = last.x + last.y;
    const int cq = t & 3;
    for (int i = t >> 2; i < kD; i += nthreads >> 2) {
        float S[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) S[j] = 0.f;
#pragma unroll 4
        for (int f = f0; f < f1; ++f) {
            int4 fu;
            if (!fine_unit(args.map, f, fu)) break;
            acc_row32(S, args.seg_state + (static_cast<size_t>(f) * H + h) * kDD + static_cast<size_t>(i) * kD + 32 * cq,
                      exp2f(g * static_cast<float>(end - (fu.x + fu.y))));
        }
        if (i < Dm && 32 * cq < Dm) {
            float4 *dst = reinterpret_cast<float4 *>(args.s_final + (static_cast<size_t>(seq) * H + h) * Dm * Dm +
                                                     static_cast<size_t>(i) * Dm + 32 * cq);
#pragma unroll
            for (int j = 0; j < 8; ++j) dst[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
        }
    }
}

// ---------------------------------------------------------------------------- entry states
// Blocks [0, units): E_w of coarse unit w (not a sequence's first) as a split image; blocks [units,
// units + nseq): the final state of a multi-segment sequence. Thread t: row t / 4, columns 32 (t % 4)..+31.
__global__ void __launch_bounds__(kEntryThreads) la_entry_state_kernel(const CorrArgs args) {
    griddep_launch_dependents();   // the correction grid may be scheduled; it waits for this one
    griddep_wait();                // the segments' exit states
    const int H = args.H, h = blockIdx.y;
    const float g = decay_log2(args.slopes, h, H);
    const size_t kDD = static_cast<size_t>(kD) * kD;
    const int i = threadIdx.x >> 2, cq = threadIdx.x & 3;
    const size_t colw = static_cast<size_t>(i) * kD + 32 * cq;
    float S[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) S[j] = 0.f;
    if (static_cast<int>(blockIdx.x) < args.units) {
        const int w = blockIdx.x;
        int4 u;
        int first_fine;
        if (!coarse_unit(args.map, w, u, first_fine) || (u.w & kUnitFirst)) return;
#pragma unroll 4
        for (int f = seq_first_fine(args.map, u.z); f < first_fine; ++f) {
            int4 fu;
            if (!fine_unit(args.map, f, fu)) break;
            acc_row32(S, args.seg_state + (static_cast<size_t>(f) * H + h) * kDD + colw,
                      exp2f(g * static_cast<float>(u.x - (fu.x + fu.y))));
        }
        uint8_t *img = args.e_img + (static_cast<size_t>(w) * H + h) * kEntryImageBytes;
        store_state_split32(img, img + kTileBytes, cq >> 1, cq & 1, i, S);
        return;
    }
    const int seq = blockIdx.x - args.units;
    if (seq < args.map.nseq) final_state(args, seq, h, g, threadIdx.x, kEntryThreads);
}

// ---------------------------------------------------------------------------- output correction
// Segment and piece of correction item x: uniform batches enumerate the segments after the first of every
// sequence, packed batches every coarse unit (the first segments and those past the list exit).
__device__ __forceinline__ int corr_unit(const WorkMap &m, int pieces, int x, int &piece) {
    const int seg = x / pieces;
    piece = x - seg * pieces;
    if (m.coarse) return seg;
    const int per = m.nc - 1;
    const int seq = seg / per;
    return seq * m.nc + 1 + (seg - seq * per);
}

// Row `row`, columns [32 cq, +32) of an O tile held as the TMA boxes of OutStaging (128-byte swizzle).
__device__ __forceinline__ uint8_t *o_chunk_addr(uint8_t *tile, int row, int cq, int j, float *) {
    using St = OutStaging<float>;   // boxes of 32 columns, two rounds of 64 rows; chunk j of 4 values
    const int rd = row / St::kRows, r = row % St::kRows;
    return tile + (rd * St::kBoxes + cq) * St::kBoxBytes + r * 128 + 16 * (j ^ (r & 7));
}
template <typename T16>
__device__ __forceinline__ uint8_t *o_chunk_addr(uint8_t *tile, int row, int cq, int j, T16 *) {
    using St = OutStaging<T16>;     // boxes of 64 columns, one round; chunk j of 8 values
    return tile + (cq >> 1) * St::kBoxBytes + row * 128 + 16 * ((4 * (cq & 1) + j) ^ (row & 7));
}
__device__ __forceinline__ void o_tile_write32(uint8_t *tile, int row, int cq, const float (&x)[32], float *) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
        *reinterpret_cast<float4 *>(o_chunk_addr(tile, row, cq, j, (float *)nullptr)) =
            make_float4(x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3]);
}
template <typename T16>
__device__ __forceinline__ void o_tile_write32(uint8_t *tile, int row, int cq, const float (&x)[32], T16 *) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4 *>(o_chunk_addr(tile, row, cq, j, (T16 *)nullptr)) =
            make_uint4(pack2(x[8 * j], x[8 * j + 1], (T16 *)nullptr), pack2(x[8 * j + 2], x[8 * j + 3], (T16 *)nullptr),
                       pack2(x[8 * j + 4], x[8 * j + 5], (T16 *)nullptr), pack2(x[8 * j + 6], x[8 * j + 7], (T16 *)nullptr));
}
// The first 16 values of a 32-value register array, as an array reference.
__device__ __forceinline__ float (&x16(float (&x)[32]))[16] { return *reinterpret_cast<float (*)[16]>(&x[0]); }

// Row `row`, columns [16 q, +16) of an O tile held as the TMA boxes of OutStaging.
__device__ __forceinline__ void o_tile_write16(uint8_t *tile, int row, int q, const float (&x)[16], float *) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
        *reinterpret_cast<float4 *>(o_chunk_addr(tile, row, q >> 1, 4 * (q & 1) + j, (float *)nullptr)) =
            make_float4(x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3]);
}
template <typename T16>
__device__ __forceinline__ void o_tile_write16(uint8_t *tile, int row, int q, const float (&x)[16], T16 *) {
#pragma unroll
    for (int j = 0; j < 2; ++j)
        *reinterpret_cast<uint4 *>(o_chunk_addr(tile, row, q >> 1, 2 * (q & 1) + j, (T16 *)nullptr)) =
            make_uint4(pack2(x[8 * j], x[8 * j + 1], (T16 *)nullptr), pack2(x[8 * j + 2], x[8 * j + 3], (T16 *)nullptr),
                       pack2(x[8 * j + 4], x[8 * j + 5], (T16 *)nullptr), pack2(x[8 * j + 6], x[8 * j + 7], (T16 *)nullptr));
}

// kD64: the head dimension is 64. Q is one 64-column slab per chunk, and the correction is one N = 128 product
// of 4 K-steps on [E_hi | E_lo] (the first slabs of the E_hi and E_lo tiles, one tile apart: the B operand's
// slab stride is a tile), whose two 64-column halves the epilogue adds.
template <typename OutT, bool kD64 = false>
__global__ void __launch_bounds__(kCorrThreads, 1)
    la_correct_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
                         const CorrArgs args) {
    using Cfg = CorrCfg<OutT>;
    using St = OutStaging<OutT>;
    constexpr uint32_t kQBytes = kD64 ? kSlabBytes : kTileBytes;   // bytes of one Q load
    const int H = args.H;
    const int h = H - 1 - static_cast<int>(blockIdx.y);   // slow-decay heads (most chunks) first
    const float g = decay_log2(args.slopes, h, H);
    const int Dm = args.D;
    const bool direct = args.e_img == nullptr;

    int piece;
    const int w = corr_unit(args.map, args.pieces, blockIdx.x, piece);
    int4 u;
    int first_fine;
    if (!coarse_unit(args.map, w, u, first_fine) || (u.w & kUnitFirst)) return;
    const int tok0 = u.x, len = u.y;
    const int nchunks = (len + kC - 1) / kC;
    // chunks c with g (cC + 1) >= -150: the others' factors are below 2^-150 on every row
    int n_act = nchunks;
    if (g < 0.f) {
        const float lim = (-150.f / g - 1.f) / static_cast<float>(kC);
        if (lim < static_cast<float>(nchunks)) n_act = max(0, static_cast<int>(floorf(lim)) + 1);
    }
    const int c0 = piece * args.chunks;
    // without an entry-state grid, the first piece of a sequence's last segment also forms its final state
    const bool do_final = direct && piece == 0 && (u.w & kUnitLast) && args.s_final;
    if (c0 >= n_act) {
        if (do_final) {
            griddep_wait();   // the segments' exit states
            final_state(args, u.z, h, g, threadIdx.x, kCorrThreads);
        }
        return;
    }
    const int n = min(args.chunks, n_act - c0);
    if (threadIdx.x == 0) LA_CTA_TIME(1, 0);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOffset);
    uint64_t *e_full = bars;          // E image landed (or split by the epilogue)
    uint64_t *q_full = bars + 1;      // [kQStages] Q of a stage landed
    uint64_t *q_empty = bars + 4;     // [kQStages] Q stage read by the tensor core
    uint64_t *o_done = bars + 7;      // [kOStages] correction staged (16 warps)
    uint64_t *o_free = bars + 9;      // [kOStages] staging read by the reduce
    uint64_t *acc_full = bars + 11;   // [2] accumulator written
    uint64_t *acc_free = bars + 13;   // [2] accumulator read (16 warps)
    uint64_t *bar_done = bars + 15;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 16);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
    uint8_t *e_hi = smem + Cfg::kOffE, *e_lo = smem + Cfg::kOffE + kTileBytes;
    auto q_slot = [&](int s) { return smem + Cfg::kOffQ + s * kTileBytes; };
    auto o_slot = [&](int s) { return smem + Cfg::kOffO + s * Cfg::kOBytes; };
    // boxes of an O tile that hold real columns (D = 64 leaves the upper ones out)
    const int boxes = min(St::kBoxes, (Dm + St::kBoxCols - 1) / St::kBoxCols);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(e_full, direct ? kCorrWarps : 1);
        for (int s = 0; s < Cfg::kQStages; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&acc_full[s], 1);
            mbar_init(&acc_free[s], kCorrWarps);
        }
        for (int s = 0; s < Cfg::kOStages; ++s) {
            mbar_init(&o_done[s], kCorrWarps);
            mbar_init(&o_free[s], 1);
        }
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
        // ------------------------------------------------------------ TMA producer (Q and the E image)
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            auto load_q = [&](int k) {
                const int s = k % Cfg::kQStages, t = tok0 + (c0 + k) * kC;
                mbar_arrive_expect_tx(&q_full[s], kQBytes);
                tma_load_3d(q_slot(s), &tm_q, 0, h, t, &q_full[s]);
                if (!kD64) tma_load_3d(q_slot(s) + kSlabBytes, &tm_q, 64, h, t, &q_full[s]);
            };
            // Q is an input: its first tiles load (and the rest go to L2) before the grids this one depends on
            // have ended
            int qi = 0;
            for (; qi < min(n, Cfg::kQStages); ++qi) load_q(qi);
            for (int k = Cfg::kQStages; k < n; ++k) {
                const int t = tok0 + (c0 + k) * kC;
                tma_prefetch_l2_3d(&tm_q, 0, h, t);
                if (!kD64) tma_prefetch_l2_3d(&tm_q, 64, h, t);
            }
            griddep_wait();   // the segments' outputs and the entry-state grid's images
            if (!direct) {
                mbar_arrive_expect_tx(e_full, kEntryImageBytes);
                const uint8_t *img = args.e_img + (static_cast<size_t>(w) * H + h) * kEntryImageBytes;
                bulk_load(e_hi, img, kTileBytes, e_full);
                bulk_load(e_lo, img + kTileBytes, kTileBytes, e_full);
            }
            bool fine = true;
            // Q of chunk k + stages once the products of chunk k have read its stage
            for (int k = 0; qi < n; ++k) {
                if (*reinterpret_cast<volatile int *>(abort_flag)) break;
                if (!(fine = mbar_wait(&q_empty[k % Cfg::kQStages], static_cast<uint32_t>(k / Cfg::kQStages) & 1))) break;
                LA_SPHASE(qi, 6);
                load_q(qi++);
            }
            if (!fine || qi < n) set_abort(abort_flag);
            // never leave with a copy in flight
            if (!direct) mbar_wait(e_full, 0);
            for (int k = (qi > Cfg::kQStages ? qi - Cfg::kQStages : 0); k < qi; ++k)
                mbar_wait(&q_full[k % Cfg::kQStages], static_cast<uint32_t>(k / Cfg::kQStages) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_qe = idesc_bf16_f32(kC, kD, false, true);   // A = Q (K-major), B = E (MN-major)
            const uint32_t ehd = dlo_mnmajor(smem_u32(e_hi)), eld = dlo_mnmajor(smem_u32(e_lo));
            const uint32_t e2d = desc_lo_sw128(smem_u32(e_hi), kTileBytes);   // D = 64: [E_hi | E_lo]
            bool fine = mbar_wait(e_full, 0);
            for (int k = 0; k < n && fine; ++k) {
                const int s = k & 1, sq = k % Cfg::kQStages;
                if (!(fine = mbar_wait(&q_full[sq], static_cast<uint32_t>(k / Cfg::kQStages) & 1))) break;
                if (k >= 2 && !(fine = mbar_wait(&acc_free[s], static_cast<uint32_t>((k - 2) >> 1) & 1))) break;
                LA_SPHASE(k, 7);
                tc_fence_after();
                const uint32_t qd = dlo_kmajor(smem_u32(q_slot(sq)));
                const uint32_t acc = tmem + 128u * static_cast<uint32_t>(s);
                if (kD64) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss_w(acc, qd + dstep_kmajor(kk), kDescHi, e2d + dstep_mnmajor(kk), kDescHi, id_qe, kk > 0);
                } else {
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk)
                        mma_ss_w(acc, qd + dstep_kmajor(kk), kDescHi, ehd + dstep_mnmajor(kk), kDescHi, id_qe, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk)
                        mma_ss_w(acc, qd + dstep_kmajor(kk), kDescHi, eld + dstep_mnmajor(kk), kDescHi, id_qe, 1);
                }
                mma_commit(&q_empty[sq]);
                mma_commit(&acc_full[s]);
                LA_SPHASE(k, 1);
            }
            if (!fine) set_abort(abort_flag);
            mma_commit(bar_done);
            mbar_wait(bar_done, 0);
        }
    } else if (warp == kCorrStoreWarp) {
        // ------------------------------------------------------------ reduce warp
        // each staged correction is added to the outputs in global memory by TMA (atomically, in L2); a chunk
        // cut short by its sequence end carries zeros in the rows past it, which leaves those rows as they are
        if (lane == 0) {
            tma_prefetch_desc(&tm_o);
            for (int k = 0; k < n; ++k) {
                const int so = k % Cfg::kOStages;
                if (!mbar_wait(&o_done[so], static_cast<uint32_t>(k / Cfg::kOStages) & 1)) {
                    set_abort(abort_flag);
                    break;
                }
                const int t = tok0 + (c0 + k) * kC;
                for (int rd = 0; rd < St::kRounds; ++rd)
                    for (int bx = 0; bx < boxes; ++bx)
                        tma_reduce_add_3d(&tm_o, o_slot(so) + (rd * St::kBoxes + bx) * St::kBoxBytes, bx * St::kBoxCols,
                                          h, t + rd * St::kRows);
                tma_store_commit();
                tma_store_wait_read();
                LA_SPHASE(k, 5);
                mbar_arrive(&o_free[so]);
            }
            tma_store_wait_all();
        }
    } else if (warp >= kCorrEpi0 && warp < kCorrEpi0 + kCorrWarps) {
        // ------------------------------------------------------------ epilogue (16 warps)
        const int e = warp - kCorrEpi0;
        const int q4 = warp & 3;                 // TMEM lane quarter this warp may access
        const int cq = e >> 2;                   // 32-column quarter
        const int i = 32 * q4 + lane;            // chunk row
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * q4) << 16);
        const bool cols = 32 * cq < Dm;
        if (direct) {
            // E_w = the exit state of segment w - 1 (the sequence's first), split into the E tiles
            griddep_wait();
            float S[32];
            acc_row32_set(S, args.seg_state + (static_cast<size_t>(first_fine - 1) * H + h) * kD * kD +
                                 static_cast<size_t>(i) * kD + 32 * cq);
            store_state_split32(e_hi, e_lo, cq >> 1, cq & 1, i, S);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(e_full);
        }
        bool ok = true;
        for (int k = 0; k < n && ok; ++k) {
            if (warp_aborted(abort_flag, lane)) break;
            const int s = k & 1, so = k % Cfg::kOStages;
            const int c = c0 + k;
            const int Lc = min(kC, len - c * kC);
            if (!(ok = warp_wait(&acc_full[s], static_cast<uint32_t>(k >> 1) & 1, lane))) break;
            if (k == 0 && e == 0 && lane == 0) LA_CTA_TIME(1, 2);
            if (e == 0 && lane == 0) LA_SPHASE(k, 2);
            tc_fence_after();
            // D = 64: columns 16 cq..+15, the sum of the product's two halves; else columns 32 cq..+31
            float x[32];
            if (kD64) {
                float y[16];
                tmem_ld16(lane_addr + 128u * static_cast<uint32_t>(s) + 16 * cq, x16(x));
                tmem_ld16(lane_addr + 128u * static_cast<uint32_t>(s) + 64 + 16 * cq, y);
                tmem_ld_wait();
#pragma unroll
                for (int m = 0; m < 16; ++m) x[m] += y[m];
            } else {
                tmem_ld32(lane_addr + 128u * static_cast<uint32_t>(s) + 32 * cq, x);
                tmem_ld_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_free[s]);
            // the staging tile is free once the reduce of chunk k - stages has read it
            if (k >= Cfg::kOStages &&
                !(ok = warp_wait(&o_free[so], static_cast<uint32_t>(k / Cfg::kOStages - 1) & 1, lane)))
                break;
            if (e == 0 && lane == 0) LA_SPHASE(k, 3);
            if (kD64 || cols) {
                if (i < Lc) {
                    const float rs = exp2f(g * static_cast<float>(c * kC + i + 1));
                    const float2 rs2 = make_float2(rs, rs);
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const float2 r = __fmul2_rn(make_float2(x[2 * m], x[2 * m + 1]), rs2);
                        x[2 * m] = r.x;
                        x[2 * m + 1] = r.y;
                    }
                } else {
#pragma unroll
                    for (int m = 0; m < 32; ++m) x[m] = 0.f;   // rows past the sequence end: add nothing
                }
                if (kD64) o_tile_write16(o_slot(so), i, cq, x16(x), static_cast<OutT *>(nullptr));
                else o_tile_write32(o_slot(so), i, cq, x, static_cast<OutT *>(nullptr));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&o_done[so]);
            if (e == 0 && lane == 0) LA_SPHASE(k, 4);
        }
        if (!ok && lane == 0) set_abort(abort_flag);
        if (do_final) final_state(args, u.z, h, g, e * 32 + lane, 32 * kCorrWarps);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
    if (threadIdx.x == 0) LA_CTA_TIME(1, 1);
}

}  // namespace la
