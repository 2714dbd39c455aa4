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
//   S     <- lambda^Lc S + (diag(lambda^(Lc-1-s)) K)^T V  (tensor core, accumulating into S)
//
// Precision. Q, K, V are bf16 inputs, so their products are exact in the fp32
// accumulators. P, S and K' = diag(lambda^(Lc-1-s)) K are made here in fp32;
// rounding them to bf16 once costs up to 2^-9 relative per entry, which for
// long-memory heads adds up to about the whole 2e-2 max-error budget. Each is
// therefore split as x = hi + lo with hi = bf16(x), lo = bf16(x - hi), and both
// halves are multiplied (relative error ~2^-17): 7 products of 128^3 per chunk.
//
// Roles (608 threads): warp 0 issues TMA loads, warp 1 (one thread) issues
// tcgen05.mma and owns TMEM, warp 2 issues the TMA stores of O, and warps 3-18
// run the epilogue: 16 warps, warp w on TMEM lanes 32*(w%4)..+31 (the only
// lanes it may touch) and on one 32-column quarter of every 128-column tile.
// Per chunk the tensor core runs QK(c) | QS(c) | PV(c) | dS(c) and the
// epilogue runs each phase with all 16 warps, inside the product it feeds on:
//   P(c)    after QK(c), while QS(c) runs     -> PV(c)
//   K'(c)   after QS(c), while PV(c) runs     -> dS(c)
//   O(c)    after PV(c), while dS(c) runs     -> TMA store
//   S(c)    after dS(c), while QK(c+1) runs   -> QS(c+1), dS(c+1)
// Only the state chain dS(c) -> S(c) -> QS(c+1) is serial.
//
// TMEM, 512 columns: [0,128) scores A; each 32-column block b is overwritten in
// place by P_hi (16 columns of packed bf16 pairs) then P_lo (16 columns);
// [128,256) O_intra = P V; [256,384) O_inter = Q S; [384,512) the fp32 state S,
// which dS accumulates into.
//
// Shared memory (224 KB): two slots each of Q, K and V and one slot X (each a
// [128 x 128] bf16 tile as two 64-column slabs with 128-byte rows and the
// 128-byte swizzle). With p = c%2, the slots live through:
//   Q[p]: Q_c (read by QK, QS) -> O_c staging for the TMA store -> Q_{c+2}
//   K[p]: K_c (read by QK) -> K'_hi(c) in place (read by dS) -> K_{c+2}
//   V[p]: V_c (read by PV, dS) -> S_hi(c) (read by QS(c+1)) -> V_{c+2}
//   X   : S_lo(c-1) (read by QS(c)) -> K'_lo(c) (read by dS(c)) -> S_lo(c)
// so K_{c+2} loads as soon as dS(c) is done, Q_{c+2} once O_c has left, and
// V_{c+2} once QS(c+1) is done: every load has about a chunk of products to
// arrive in.
#pragma once

#include <cuda_fp16.h>

#include "la_plan.cuh"
#include "la_ptx.cuh"

namespace la {

constexpr int kC = 128;                     // chunk length = MMA M
constexpr int kD = 128;                     // head dim handled by this kernel
constexpr int kSlabBytes = 128 * 128;       // [128 rows x 64 bf16] slab, 128-byte rows
constexpr int kTileBytes = 2 * kSlabBytes;  // [128 x 128] bf16 tile = two slabs
constexpr int kTcThreads = 608;    // main kernel: producer, MMA, store warp, 16 epilogue warps
constexpr int kStoreWarp = 2;
constexpr int kEpi0 = 3;           // epilogue: warps 3..18
constexpr int kEpiWarps = 16;
constexpr int kStateThreads = 576; // state-only kernel: producer, MMA, 16 K' warps


// Profiling builds only: per-chunk phase timestamps of a few CTAs (LA_TRACE_PHASES) and
// start / end times of every CTA (LA_TRACE_CTA or LA_TRACE_PHASES), all from the global timer (ns);
// read with la_debug_phase_dump, la_debug_sphase_dump and la_debug_cta_dump.
#if defined(LA_TRACE_PHASES) || defined(LA_TRACE_CTA)
#define LA_TRACE_ANY 1
constexpr int kPhaseSlots = 8, kPhaseChunks = 64, kPhaseEvents = 24;
constexpr int kTraceCtas = 8192;
// Start / end (global timer, ns) of every CTA of the chunk kernel (0) and the state kernel (1).
__device__ long long g_la_cta[2][kTraceCtas][4];
#define LA_CTA_TIME(kid, slot)                                                                \
    do {                                                                                      \
        const int cta_ = blockIdx.y * gridDim.x + blockIdx.x;                                 \
        if (cta_ < kTraceCtas) g_la_cta[(kid)][cta_][(slot)] = (long long)globaltimer_ns();   \
    } while (0)
#else
#define LA_CTA_TIME(kid, slot) \
    do {                       \
    } while (0)
#endif
#ifdef LA_TRACE_PHASES
// Traced CTAs: units 0 and 1 of heads 0, 5, 10 and 15 (slot = 2 * (head / 5) + unit).
__device__ long long g_la_phase[kPhaseSlots][kPhaseChunks][kPhaseEvents];
#define LA_PHASE(c, ev)                                                                                   \
    do {                                                                                                  \
        if (blockIdx.x < 2 && blockIdx.y % 5 == 0 && blockIdx.y < 20 && (c) < kPhaseChunks)               \
            g_la_phase[2 * (blockIdx.y / 5) + blockIdx.x][(c)][(ev)] = (long long)globaltimer_ns();      \
    } while (0)
__device__ long long g_la_sphase[kPhaseSlots][kPhaseChunks][8];
#define LA_SPHASE(c, ev)                                                                                  \
    do {                                                                                                  \
        if (blockIdx.x < 2 && blockIdx.y % 5 == 0 && blockIdx.y < 20 && (c) < kPhaseChunks)               \
            g_la_sphase[2 * (blockIdx.y / 5) + blockIdx.x][(c)][(ev)] = (long long)globaltimer_ns();     \
    } while (0)
#else
#define LA_PHASE(c, ev) \
    do {                \
    } while (0)
#define LA_SPHASE(c, ev) \
    do {                 \
    } while (0)
#endif

// D is the head dimension of the tensors: 128, or 64, in which case every 128-wide tile's second
// 64-column slab is read past the rows' end (zero fill by TMA) and the padded rows and columns of Q, K,
// V, S and O stay zero: q . k, the state and the outputs are those of D = 64, and only the first D
// columns of O (and D x D of the states) are stored.
struct ChunkArgs {
    void *o;                    // [T, H, D] in the kernel's OutT
    const float *s_init;        // [nseq, H, D, D] or null
    float *s_final;             // [nseq, H, D, D] or null
    const float *slopes;        // [H] or null
    WorkMap map;                // fine / coarse units
    float *seg_state;           // [fine units, H, seg_ld, seg_ld]: dS of each fine unit
    float *s0_copy;             // [nseq, H, D, D] workspace: initial states of multi-segment sequences
    int H;
    int D;                      // 128 or 64
    int seg_ld;                 // 128 (the prefill's workspace), or D (a shard's states, in the caller's layout)
};

// Shared memory of the main kernel: two slots each of Q, K and V and the X slot (32 KB each).
struct ChunkCfg {
    static constexpr int kOffQ = 0;                // 2 x 32 KB
    static constexpr int kOffK = 2 * kTileBytes;   // 2 x 32 KB
    static constexpr int kOffV = 4 * kTileBytes;   // 2 x 32 KB
    static constexpr int kOffX = 6 * kTileBytes;   // 32 KB
    static constexpr int kBarOffset = 7 * kTileBytes;
    static constexpr int kSmemBytes = kBarOffset + 256 + 1024;  // barriers + alignment slack
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColA = 0, kColOn = 128, kColOi = 256, kColS = 384;
};

struct StateCfg {
    static constexpr int kStages = 3;
    static constexpr int kStageBytes = 2 * kTileBytes;   // K, V
    // a 16 x 16 identity as the B operand of the products that copy K^T into TMEM: 16 rows of 64 bf16 (K-major,
    // 128-byte rows with the 128-byte swizzle, like every other operand tile), only the first 16 columns used
    static constexpr int kOffI = kStages * kStageBytes;
    static constexpr int kIdentityBytes = 16 * 128;
    static constexpr int kBarOffset = kOffI + kIdentityBytes;
    static constexpr int kSmemBytes = kBarOffset + 256 + 1024;
    // TMEM: dS [0,128); K^T then K' hi/lo of chunks 0, 2, .. at [128,256) and of chunks 1, 3, .. at [256,384)
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColD = 0, kColKT = 128;
    static constexpr int kScaleWarps = 16;
};

// MN-major operand (rows = K, 128-byte rows holding 64 MN elements, two MN slabs
// 16 KB apart), 16-row K step kk.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile, int kk) {
    return smem_desc_sw128(tile + kk * 2048, kSlabBytes, 1024);
}
// The same as descriptor words: the low word of a tile's K-major (LBO 16 B) or MN-major (LBO =
// the 16 KB slab stride) descriptor, the K step's offset in 16-byte units, and the common high
// word (SBO 1024 B: eight 128-byte rows).
__device__ __forceinline__ uint32_t dlo_kmajor(uint32_t tile) { return desc_lo_sw128(tile, 16); }
__device__ __forceinline__ uint32_t dlo_mnmajor(uint32_t tile) { return desc_lo_sw128(tile, kSlabBytes); }
__host__ __device__ constexpr uint32_t dstep_kmajor(int kk) { return ((kk >> 2) * kSlabBytes + (kk & 3) * 32) >> 4; }
__host__ __device__ constexpr uint32_t dstep_mnmajor(int kk) { return (kk * 2048) >> 4; }
constexpr uint32_t kDescHi = desc_hi_sw128(1024);

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

// Split the pair x = hi + lo into two bf16 pairs (lo carries the bits hi drops;
// x - hi is exact in fp32). Paired fp32 arithmetic (sm_100) halves the
// instruction count of the subtraction.
__device__ __forceinline__ void split2(float2 x, uint32_t &hi, uint32_t &lo) {
    hi = pack_bf16x2(x.x, x.y);
    const float2 h = make_float2(bf16lo_to_f32(hi), bf16hi_to_f32(hi));
    const float2 d = __ffma2_rn(h, make_float2(-1.f, -1.f), x);
    lo = pack_bf16x2(d.x, d.y);
}

// K' for half of a 128-byte row: part 0 takes the 16-byte chunks (row + 0..3) & 7,
// part 1 the chunks (row + 4..7) & 7 (hi in place, lo to the same position of
// another tile).
__device__ __forceinline__ void scale_row_split_half(uint8_t *row_hi, uint8_t *row_lo, int row, int part, float f) {
    const float2 ff = make_float2(f, f);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        const int j = (4 * part + jj + row) & 7;
        const uint4 x = *reinterpret_cast<const uint4 *>(row_hi + 16 * j);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int m = 0; m < 4; ++m)
            split2(__fmul2_rn(make_float2(bf16lo_to_f32(w[m]), bf16hi_to_f32(w[m])), ff), hi[m], lo[m]);
        *reinterpret_cast<uint4 *>(row_hi + 16 * j) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4 *>(row_lo + 16 * j) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
}

// Store 32 fp32 state entries of row `row`, columns [64*slab + 32*h2, +32),
// split into bf16 hi / lo, into two MN-major swizzled state tiles: slab `slab`,
// 128-byte row `row`, 16-byte chunk j at j ^ (row & 7).
__device__ __forceinline__ void store_state_split32(uint8_t *t_hi, uint8_t *t_lo, int slab, int h2, int row,
                                                    const float (&S)[32]) {
    const int off = slab * kSlabBytes + row * 128;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) split2(make_float2(S[8 * j + 2 * m], S[8 * j + 2 * m + 1]), hi[m], lo[m]);
        const int c = 16 * ((4 * h2 + j) ^ (row & 7));
        *reinterpret_cast<uint4 *>(t_hi + off + c) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4 *>(t_lo + off + c) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
}

// S[0..31] += w * src[0..31] (src 16-byte aligned fp32).
__device__ __forceinline__ void acc_row32(float (&S)[32], const float *src, float w) {
    const float4 *p = reinterpret_cast<const float4 *>(src);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float4 x = p[j];
        S[4 * j] = fmaf(w, x.x, S[4 * j]);
        S[4 * j + 1] = fmaf(w, x.y, S[4 * j + 1]);
        S[4 * j + 2] = fmaf(w, x.z, S[4 * j + 2]);
        S[4 * j + 3] = fmaf(w, x.w, S[4 * j + 3]);
    }
}

// fp16 pairs: cvt.rn.f16x2.f32 d, a, b puts a in the upper half and b in the lower half.
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi, __nv_bfloat16 *) { return pack_bf16x2(lo, hi); }
__device__ __forceinline__ uint32_t pack2(float lo, float hi, __half *) { return pack_half2(lo, hi); }

// Output staging geometry for a TMA store with the 128-byte swizzle. A box is
// 128 bytes of columns wide (32 fp32 or 64 16-bit values) and kRows rows high;
// the 32 KB staging area holds one round of kBoxes boxes. fp32 needs two rounds
// (rows 0-63, then 64-127) per chunk, 16-bit outputs one.
template <typename OutT>
struct OutStaging {
    static constexpr int kRounds = sizeof(OutT) == 4 ? 2 : 1;
    static constexpr int kRows = kC / kRounds;
    static constexpr int kBoxCols = 128 / static_cast<int>(sizeof(OutT));
    static constexpr int kBoxes = kD / kBoxCols;
    static constexpr int kBoxBytes = kRows * 128;
};

// Stage 16 output values of row `row` (of the current round), columns
// [64*hf + 16*qq, +16), at their swizzled box positions: 16-byte chunk j of a
// 128-byte box row lands at j ^ (row & 7).
__device__ __forceinline__ void stage16(uint8_t *stg, int hf, int qq, int row, const float (&x)[16], float *) {
    using St = OutStaging<float>;
    uint8_t *base = stg + (2 * hf + (qq >> 1)) * St::kBoxBytes + row * 128;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4 *>(base + 16 * ((4 * (qq & 1) + j) ^ (row & 7))) =
            make_uint4(__float_as_uint(x[4 * j]), __float_as_uint(x[4 * j + 1]), __float_as_uint(x[4 * j + 2]),
                       __float_as_uint(x[4 * j + 3]));
}
template <typename T16>
__device__ __forceinline__ void stage16(uint8_t *stg, int hf, int qq, int row, const float (&x)[16], T16 *) {
    using St = OutStaging<T16>;
    uint8_t *base = stg + hf * St::kBoxBytes + row * 128;
#pragma unroll
    for (int j = 0; j < 2; ++j)
        *reinterpret_cast<uint4 *>(base + 16 * ((2 * qq + j) ^ (row & 7))) =
            make_uint4(pack2(x[8 * j], x[8 * j + 1], (T16 *)nullptr), pack2(x[8 * j + 2], x[8 * j + 3], (T16 *)nullptr),
                       pack2(x[8 * j + 4], x[8 * j + 5], (T16 *)nullptr), pack2(x[8 * j + 6], x[8 * j + 7], (T16 *)nullptr));
}

// Store 16 consecutive output values of one row directly (chunks cut short by their sequence end).
__device__ __forceinline__ void store16(float *dst, const float (&x)[16]) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
        st_global_v4(dst + 4 * j, make_uint4(__float_as_uint(x[4 * j]), __float_as_uint(x[4 * j + 1]),
                                             __float_as_uint(x[4 * j + 2]), __float_as_uint(x[4 * j + 3])));
}
template <typename T16>
__device__ __forceinline__ void store16(T16 *dst, const float (&x)[16]) {
#pragma unroll
    for (int j = 0; j < 2; ++j)
        st_global_v4(dst + 8 * j, make_uint4(pack2(x[8 * j], x[8 * j + 1], (T16 *)nullptr),
                                             pack2(x[8 * j + 2], x[8 * j + 3], (T16 *)nullptr),
                                             pack2(x[8 * j + 4], x[8 * j + 5], (T16 *)nullptr),
                                             pack2(x[8 * j + 6], x[8 * j + 7], (T16 *)nullptr)));
}

// ============================================================================ main chunk kernel
// kRev runs the recurrence backwards in time (the reverse sweep of the backward
// pass) over the same 128-token tiles: chunks are taken from the segment's end
// to its start, and every decay exponent is mirrored inside the chunk,
//   P[i,s] = A[i,s] lambda^(s-i)  for s >= i (and s < Lc), else 0,
//   O      = P V + diag(lambda^(Lc-1-i)) (Q S),
//   S     <- lambda^Lc S + (diag(lambda^(s+1)) K)^T V,
// so S entering a chunk is lambda times the state at the token after it. The
// state given to a sequence is the one after its last token, the state returned
// is lambda times the one at its first token, and the segment split runs the
// other way round (a segment starts from the states of the units after it).
template <typename OutT, bool kRev = false>
__global__ void __launch_bounds__(kTcThreads, 1)
    la_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                       const ChunkArgs args) {
    using Cfg = ChunkCfg;
    using Stg = OutStaging<OutT>;
    // Uniform batches are dispatched segment-major: every sequence's entry segment (the first one,
    // the last with kRev; it does not wait for the segment-state pass) is scheduled before the others.
    int unit = blockIdx.x, h = blockIdx.y;
    if (!args.map.fine) {
        const int per_seg = args.map.nseq * args.H;
        const int L = blockIdx.y * gridDim.x + blockIdx.x;
        const int j = L / per_seg, rem = L - j * per_seg;
        unit = (rem / args.H) * args.map.nc + (kRev ? args.map.nc - 1 - j : j);
        h = rem % args.H;
    }
    int4 u;
    int first_fine;
    if (!coarse_unit(args.map, unit, u, first_fine)) return;
    if (threadIdx.x == 0) LA_CTA_TIME(0, 0);
    const int tok0 = u.x, len = u.y, seq = u.z, flags = u.w;
    const int nchunks = (len + kC - 1) / kC;
    const int H = args.H;
    const float g = decay_log2(args.slopes, h, H);
    // the segment the sequence is entered by (it reads the given state) and the one it leaves by
    constexpr int kEntry = kRev ? kUnitLast : kUnitFirst, kExit = kRev ? kUnitFirst : kUnitLast;
    // position (in chunks from the segment start) of the c-th chunk processed
    auto chunk_at = [&](int c) { return kRev ? nchunks - 1 - c : c; };

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *x_slot = smem + Cfg::kOffX;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOffset);
    uint64_t *full_q = bars;             // [2] Q of a chunk landed
    uint64_t *full_k = bars + 2;         // [2] K of a chunk landed
    uint64_t *full_v = bars + 4;         // [2] V of a chunk landed
    uint64_t *empty_k = bars + 6;        // [2] K slot free (dS of the chunk in it done)
    uint64_t *empty_v = bars + 8;        // [2] V slot free (Q S has read the S_hi it held)
    uint64_t *q_free = bars + 10;        // [2] Q slot free (its O staging has been read by the store)
    uint64_t *bar_QK = bars + 12;        // A = Q K^T done
    uint64_t *bar_QS = bars + 13;        // O_inter = Q S done (X and the previous V slot read)
    uint64_t *bar_PV = bars + 14;        // O_intra = P V done
    uint64_t *bar_dS = bars + 15;        // dS accumulated into S
    uint64_t *bar_P = bars + 16;         // P hi/lo in TMEM (16 warps)
    uint64_t *bar_K = bars + 17;         // K' hi/lo in shared memory (16 warps)
    uint64_t *bar_Of = bars + 18;        // O accumulators read (16 warps)
    uint64_t *bar_S = bars + 19;         // S hi/lo written, S rescaled in TMEM (16 warps)
    uint64_t *bar_E = bars + 20;         // [round][pair] O staging round written (16 / rounds warps)
    uint64_t *bar_F = bars + 24;         // O staging round 0 read by the store (two-round outputs)
    uint64_t *bar_done = bars + 25;      // every MMA retired
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 26);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    auto q_slot = [&](int s) { return smem + Cfg::kOffQ + s * kTileBytes; };
    auto k_slot = [&](int s) { return smem + Cfg::kOffK + s * kTileBytes; };
    auto v_slot = [&](int s) { return smem + Cfg::kOffV + s * kTileBytes; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&full_q[s], 1);
            mbar_init(&full_k[s], 1);
            mbar_init(&full_v[s], 1);
            mbar_init(&empty_k[s], 1);
            mbar_init(&empty_v[s], 1);
            mbar_init(&q_free[s], 1);
            mbar_init(&bar_E[s], kEpiWarps / Stg::kRounds);
            mbar_init(&bar_E[2 + s], kEpiWarps / Stg::kRounds);
        }
        mbar_init(bar_QK, 1);
        mbar_init(bar_QS, 1);
        mbar_init(bar_PV, 1);
        mbar_init(bar_dS, 1);
        mbar_init(bar_P, kEpiWarps);
        mbar_init(bar_K, kEpiWarps);
        mbar_init(bar_Of, kEpiWarps);
        mbar_init(bar_S, kEpiWarps);
        mbar_init(bar_F, 1);
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
        // Chunk c goes to pair c%2: K once dS of chunk c-2 is done, Q once the O of chunk c-2
        // staged in that Q slot has been read by the store, V once Q S of chunk c-1 has read the
        // S_hi of chunk c-2 held in that V slot.
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int issued_q = 0, issued_k = 0, issued_v = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c & 1;
                const int t = tok0 + chunk_at(c) * kC;
                if (c >= 2 && !mbar_wait(&empty_k[s], static_cast<uint32_t>((c - 2) >> 1) & 1)) break;
                if (*reinterpret_cast<volatile int *>(abort_flag)) break;
                LA_PHASE(c, 15);
                mbar_arrive_expect_tx(&full_k[s], kTileBytes);
                tma_load_3d(k_slot(s), &tm_k, 0, h, t, &full_k[s]);
                tma_load_3d(k_slot(s) + kSlabBytes, &tm_k, 64, h, t, &full_k[s]);
                issued_k = c + 1;
                if (c >= 2 && !mbar_wait(&q_free[s], static_cast<uint32_t>((c - 2) >> 1) & 1)) break;
                if (*reinterpret_cast<volatile int *>(abort_flag)) break;
                LA_PHASE(c, 16);
                mbar_arrive_expect_tx(&full_q[s], kTileBytes);
                tma_load_3d(q_slot(s), &tm_q, 0, h, t, &full_q[s]);
                tma_load_3d(q_slot(s) + kSlabBytes, &tm_q, 64, h, t, &full_q[s]);
                issued_q = c + 1;
                if (c >= 1 && !mbar_wait(&empty_v[s], static_cast<uint32_t>((c - 1) >> 1) & 1)) break;
                if (*reinterpret_cast<volatile int *>(abort_flag)) break;
                LA_PHASE(c, 17);
                mbar_arrive_expect_tx(&full_v[s], kTileBytes);
                tma_load_3d(v_slot(s), &tm_v, 0, h, t, &full_v[s]);
                tma_load_3d(v_slot(s) + kSlabBytes, &tm_v, 64, h, t, &full_v[s]);
                issued_v = c + 1;
            }
            if (issued_v < nchunks) set_abort(abort_flag);
            // Never leave with a copy in flight: wait (bounded) for the last loads of each slot.
            for (int c = (issued_k > 2 ? issued_k - 2 : 0); c < issued_k; ++c)
                mbar_wait(&full_k[c & 1], static_cast<uint32_t>(c >> 1) & 1);
            for (int c = (issued_q > 2 ? issued_q - 2 : 0); c < issued_q; ++c)
                mbar_wait(&full_q[c & 1], static_cast<uint32_t>(c >> 1) & 1);
            for (int c = (issued_v > 2 ? issued_v - 2 : 0); c < issued_v; ++c)
                mbar_wait(&full_v[c & 1], static_cast<uint32_t>(c >> 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_qk = idesc_bf16_f32(kC, kC, false, false);
            constexpr uint32_t id_pv = idesc_bf16_f32(kC, kD, false, true);
            constexpr uint32_t id_qs = idesc_bf16_f32(kC, kD, false, true);
            constexpr uint32_t id_ds = idesc_bf16_f32(kD, kD, true, true);
            const uint32_t xd = dlo_mnmajor(smem_u32(x_slot));
            for (int c = 0; c < nchunks; ++c) {
                const int s = c & 1;
                const uint32_t r = static_cast<uint32_t>(c >> 1) & 1;
                const uint32_t qd = dlo_kmajor(smem_u32(q_slot(s))), kdk = dlo_kmajor(smem_u32(k_slot(s)));
                const uint32_t kdm = dlo_mnmajor(smem_u32(k_slot(s))), vd = dlo_mnmajor(smem_u32(v_slot(s)));
                // the state entering chunk c: S_hi in the V slot of pair c-1, S_lo in X
                const uint32_t shd = dlo_mnmajor(smem_u32(v_slot(s ^ 1)));
                // A = Q K^T (the score tile is free: P V of chunk c-1 was issued before)
                if (!mbar_wait(&full_k[s], r)) break;
                LA_PHASE(c, 19);
                if (!mbar_wait(&full_q[s], r)) break;
                LA_PHASE(c, 20);
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    mma_ss_w(tmem + Cfg::kColA, qd + dstep_kmajor(kk), kDescHi, kdk + dstep_kmajor(kk), kDescHi, id_qk, kk > 0);
                mma_commit(bar_QK);
                LA_PHASE(c, 0);
                if (c == 0) LA_CTA_TIME(0, 2);
                // O_inter = Q (S_hi + S_lo): needs the state pass of chunk c-1 and O of chunk c-1 read
                if (!mbar_wait(bar_S, static_cast<uint32_t>(c) & 1)) break;
                if (c > 0 && !mbar_wait(bar_Of, static_cast<uint32_t>(c - 1) & 1)) break;
                LA_PHASE(c, 1);
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    mma_ss_w(tmem + Cfg::kColOi, qd + dstep_kmajor(kk), kDescHi, shd + dstep_mnmajor(kk), kDescHi, id_qs, kk > 0);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    mma_ss_w(tmem + Cfg::kColOi, qd + dstep_kmajor(kk), kDescHi, xd + dstep_mnmajor(kk), kDescHi, id_qs, 1);
                mma_commit(bar_QS);
                mma_commit(&empty_v[s ^ 1]);
                LA_PHASE(c, 2);
                // O_intra = (P_hi + P_lo) V, P from TMEM
                if (!mbar_wait(&full_v[s], r)) break;
                LA_PHASE(c, 21);
                if (!mbar_wait(bar_P, static_cast<uint32_t>(c) & 1)) break;
                LA_PHASE(c, 3);
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ts_w(tmem + Cfg::kColOn, tmem + Cfg::kColA + p_hi_col(kk), vd + dstep_mnmajor(kk), kDescHi, id_pv, kk > 0);
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ts_w(tmem + Cfg::kColOn, tmem + Cfg::kColA + p_hi_col(kk) + 16, vd + dstep_mnmajor(kk), kDescHi, id_pv, 1);
                mma_commit(bar_PV);
                LA_PHASE(c, 4);
                // S += (K'_hi + K'_lo)^T V (S was rescaled by lambda^Lc in the state pass of chunk c-1)
                if (!mbar_wait(bar_K, static_cast<uint32_t>(c) & 1)) break;
                LA_PHASE(c, 5);
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ss_w(tmem + Cfg::kColS, kdm + dstep_mnmajor(kk), kDescHi, vd + dstep_mnmajor(kk), kDescHi, id_ds, 1);
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ss_w(tmem + Cfg::kColS, xd + dstep_mnmajor(kk), kDescHi, vd + dstep_mnmajor(kk), kDescHi, id_ds, 1);
                mma_commit(bar_dS);
                mma_commit(&empty_k[s]);
                LA_PHASE(c, 6);
                if (c == nchunks - 1) LA_CTA_TIME(0, 3);
            }
            mma_commit(bar_done);
            mbar_wait(bar_done, 0);
        }
    } else if (warp == kStoreWarp) {
        // ------------------------------------------------------------ output store warp
        // O of chunk c is staged in the Q slot of its pair (one round for 16-bit outputs, two of 64
        // rows for fp32); once the store has read it, that Q slot takes Q of chunk c+2.
        if (lane == 0) {
            for (int c = 0; c < nchunks; ++c) {
                const int s = c & 1;
                const int ci = chunk_at(c);
                const bool whole = (min(kC, len - ci * kC) == kC);
                bool fine = true;
                for (int rd = 0; rd < Stg::kRounds; ++rd) {
                    if (!mbar_wait(&bar_E[2 * rd + s], static_cast<uint32_t>(c >> 1) & 1)) {
                        fine = false;
                        break;
                    }
                    if (whole) {
#pragma unroll
                        for (int bx = 0; bx < Stg::kBoxes; ++bx)
                            if (bx * Stg::kBoxCols < args.D)   // the columns past D are padding
                                tma_store_3d(&tm_o, q_slot(s) + bx * Stg::kBoxBytes, bx * Stg::kBoxCols, h,
                                             tok0 + ci * kC + rd * Stg::kRows);
                        tma_store_commit();
                        tma_store_wait_read();
                    }
                    if (rd + 1 < Stg::kRounds) mbar_arrive(bar_F);
                }
                if (!fine) {
                    set_abort(abort_flag);
                    break;
                }
                mbar_arrive(&q_free[s]);
                LA_PHASE(c, 18);
            }
            tma_store_wait_all();
        }
    } else if (warp >= kEpi0 && warp < kEpi0 + kEpiWarps) {
        // ------------------------------------------------------------ epilogue (warps 3..18)
        const int e = warp - kEpi0;        // 0..15
        const int q4 = warp & 3;           // TMEM lane quarter this warp may access
        const int cq = e >> 2;             // 32-column quarter of every 128-column tile
        const int i = 32 * q4 + lane;      // TMEM lane: chunk row i (A, O) or state row dk (S)
        const int et = e * 32 + lane;      // 0..511: K row (et & 127), slab ((et >> 7) & 1), half row (et >> 8)
        const int rd = Stg::kRounds == 2 ? (q4 >> 1) : 0;   // output staging round of this warp's rows
        const bool tracer = (e == 0 && lane == 0);           // rows 96..127, columns 0..31
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * q4) << 16);
        const uint32_t s_col = lane_addr + Cfg::kColS + 32 * cq;
        const float lam = exp2f(g);
        const float2 lam2 = make_float2(lam * lam, lam * lam);
        const int Dm = args.D;
        const size_t DD = static_cast<size_t>(Dm) * Dm;         // caller's states: [., H, D, D]
        const size_t kDD = static_cast<size_t>(kD) * kD;        // workspace segment states: [., H, 128, 128]
        const bool in_state = i < Dm && 32 * cq < Dm;          // this thread's 32 state entries are not padding
        float *fin = ((flags & kExit) && args.s_final && in_state)
                         ? args.s_final + (static_cast<size_t>(seq) * H + h) * DD + static_cast<size_t>(i) * Dm + 32 * cq
                         : nullptr;

        // The state entering this segment (row i, columns 32*cq..+31). A single-segment sequence
        // reads its initial state; otherwise only the workspace is read (final_state may alias
        // initial_state, and another CTA of this sequence writes it): the entry segment takes the
        // copy of the initial state, another segment sums the decayed states of every fine unit
        // before it (after it with kRev; the unit the sequence is entered by already carries the
        // decayed initial state). Its hi / lo go to V slot 1 and X (read by Q S of the first chunk
        // processed), lambda^L0 S to TMEM.
        {
            // the workspace is written by the segment-state pass, which may still be running
            if (!((flags & kUnitFirst) && (flags & kUnitLast)) && (!(flags & kEntry) || args.s_init)) griddep_wait();
            float S[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) S[j] = 0.f;
            const size_t col = static_cast<size_t>(i) * Dm + 32 * cq;    // in the caller's states
            const size_t colw = static_cast<size_t>(i) * kD + 32 * cq;   // in the workspace states
            if ((flags & kUnitFirst) && (flags & kUnitLast)) {
                if (args.s_init && in_state) acc_row32(S, args.s_init + (static_cast<size_t>(seq) * H + h) * DD + col, 1.f);
            } else if (flags & kEntry) {
                if (args.s_init && in_state) acc_row32(S, args.s0_copy + (static_cast<size_t>(seq) * H + h) * DD + col, 1.f);
            } else if (!kRev) {
                for (int f = seq_first_fine(args.map, seq); f < first_fine; ++f) {
                    int4 fu;
                    if (!fine_unit(args.map, f, fu)) break;
                    const float w = exp2f(g * static_cast<float>(tok0 - (fu.x + fu.y)));
                    acc_row32(S, args.seg_state + (static_cast<size_t>(f) * H + h) * kDD + colw, w);
                }
            } else {
                // the units after this segment (which is not the last, so it holds R of them)
                const int end = seq_end_fine(args.map, seq);
                for (int f = first_fine + args.map.R; f < end; ++f) {
                    int4 fu;
                    if (!fine_unit(args.map, f, fu)) break;
                    const float w = exp2f(g * static_cast<float>(fu.x - (tok0 + len)));
                    acc_row32(S, args.seg_state + (static_cast<size_t>(f) * H + h) * kDD + colw, w);
                }
            }
            if (nchunks == 0) {
                if (fin) {
                    float4 *p = reinterpret_cast<float4 *>(fin);
#pragma unroll
                    for (int j = 0; j < 8; ++j) p[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
                }
            } else {
                store_state_split32(v_slot(1), x_slot, cq >> 1, cq & 1, i, S);
                const float l0 = exp2f(g * static_cast<float>(min(kC, len - chunk_at(0) * kC)));
#pragma unroll
                for (int j = 0; j < 32; ++j) S[j] *= l0;
                tmem_st32(s_col, S);
                tmem_st_wait();
                fence_proxy_async_smem();
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_S);

        bool ok = true;
        for (int c = 0; c < nchunks && ok; ++c) {
            if (warp_aborted(abort_flag, lane)) break;
            const int s = c & 1;
            const int ci = chunk_at(c);
            const int Lc = min(kC, len - ci * kC);

            // ---- P = decay-masked A for this warp's 32-column block, split into bf16 hi / lo in place
            if (!(ok = warp_wait(bar_QK, static_cast<uint32_t>(c) & 1, lane))) break;
            if (tracer) LA_PHASE(c, 7);
            tc_fence_after();
            {
                const uint32_t col = lane_addr + Cfg::kColA + 32 * cq;  // P_hi at +0..15, P_lo at +16..31
                if (kRev ? cq < q4 : cq > q4) {
                    const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
                    for (int q = 0; q < 4; ++q) tmem_st8(col + 8 * q, z);
                } else {
                    // both 16-column halves are read before either is overwritten (P_hi of columns
                    // 16..31 lands on A columns 8..15)
                    float a[2][16];
                    tmem_ld16(col, a[0]);
                    tmem_ld16(col + 16, a[1]);
                    tmem_ld_wait();
                    if (kRev && 32 * cq + 32 > Lc) {
                        // a chunk cut short by its sequence end: columns past it hold other tokens
#pragma unroll
                        for (int sb = 0; sb < 2; ++sb)
#pragma unroll
                            for (int j = 0; j < 16; ++j) a[sb][j] = 32 * cq + 16 * sb + j < Lc ? a[sb][j] : 0.f;
                    }
                    if (kRev && cq == q4) {
                        // diagonal block: s >= i is j >= lane; walking j up from the diagonal the
                        // factor lambda^(j - lane) grows by lambda per step
                        float f = 1.f;
#pragma unroll
                        for (int sb = 0; sb < 2; ++sb) {
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const bool in = 16 * sb + j >= lane;
                                a[sb][j] = in ? a[sb][j] * f : 0.f;
                                f = in ? f * lam : f;
                            }
                            uint32_t hi[8], lo[8];
#pragma unroll
                            for (int m = 0; m < 8; ++m) split2(make_float2(a[sb][2 * m], a[sb][2 * m + 1]), hi[m], lo[m]);
                            tmem_st8(col + 8 * sb, hi);
                            tmem_st8(col + 16 + 8 * sb, lo);
                        }
                    } else if (kRev) {
                        // above the diagonal: factors lambda^(s-i) of the column pair (2m, 2m+1), walking m up
                        const float f0 = exp2f(g * static_cast<float>(32 * cq - i));
                        float2 fp = make_float2(f0, f0 * lam);
#pragma unroll
                        for (int sb = 0; sb < 2; ++sb) {
                            uint32_t hi[8], lo[8];
#pragma unroll
                            for (int m = 0; m < 8; ++m) {
                                split2(__fmul2_rn(make_float2(a[sb][2 * m], a[sb][2 * m + 1]), fp), hi[m], lo[m]);
                                fp = __fmul2_rn(fp, lam2);
                            }
                            tmem_st8(col + 8 * sb, hi);
                            tmem_st8(col + 16 + 8 * sb, lo);
                        }
                    } else if (cq == q4) {
                        // diagonal block: s <= i is j <= lane; walking j down from the diagonal the
                        // factor lambda^(lane - j) grows by lambda per step
                        float f = 1.f;
#pragma unroll
                        for (int sb = 1; sb >= 0; --sb) {
#pragma unroll
                            for (int j = 15; j >= 0; --j) {
                                const bool in = 16 * sb + j <= lane;
                                a[sb][j] = in ? a[sb][j] * f : 0.f;
                                f = in ? f * lam : f;
                            }
                            uint32_t hi[8], lo[8];
#pragma unroll
                            for (int m = 0; m < 8; ++m) split2(make_float2(a[sb][2 * m], a[sb][2 * m + 1]), hi[m], lo[m]);
                            tmem_st8(col + 8 * sb, hi);
                            tmem_st8(col + 16 + 8 * sb, lo);
                        }
                    } else {
                        // below the diagonal: factors lambda^(i-s) of the column pair (2m, 2m+1), walking m down
                        const float f31 = exp2f(g * static_cast<float>(i - 32 * cq - 31));
                        float2 fp = make_float2(f31 * lam, f31);
#pragma unroll
                        for (int sb = 1; sb >= 0; --sb) {
                            uint32_t hi[8], lo[8];
#pragma unroll
                            for (int m = 7; m >= 0; --m) {
                                split2(__fmul2_rn(make_float2(a[sb][2 * m], a[sb][2 * m + 1]), fp), hi[m], lo[m]);
                                fp = __fmul2_rn(fp, lam2);
                            }
                            tmem_st8(col + 8 * sb, hi);
                            tmem_st8(col + 16 + 8 * sb, lo);
                        }
                    }
                }
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_P);
            if (tracer) LA_PHASE(c, 8);

            // ---- K' = diag(lambda^(Lc-1-s)) K (kRev: lambda^(s+1)): hi in place (Q K^T has read K), lo into
            //      X (Q S has read S_lo)
            if (!(ok = warp_wait(bar_QS, static_cast<uint32_t>(c) & 1, lane))) break;
            if (tracer) LA_PHASE(c, 9);
            {
                const int krow = et & 127, kslab = (et >> 7) & 1, part = et >> 8;
                const float f = krow < Lc ? exp2f(g * static_cast<float>(kRev ? krow + 1 : Lc - 1 - krow)) : 0.f;
                const int off = kslab * kSlabBytes + krow * 128;
                scale_row_split_half(k_slot(s) + off, x_slot + off, krow, part, f);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_K);
            if (tracer) LA_PHASE(c, 10);

            // ---- O = O_intra + lambda^(i+1) O_inter (kRev: lambda^(Lc-1-i)): accumulators read first (Q S and P V of the next
            //      chunk may then run), then staged in this pair's Q slot for the store warp, or stored
            //      row by row (a chunk cut short by its sequence end must not write past it)
            if (!(ok = warp_wait(bar_PV, static_cast<uint32_t>(c) & 1, lane))) break;
            if (tracer) LA_PHASE(c, 11);
            tc_fence_after();
            float o[2][16];
            {
                const float rs = exp2f(g * static_cast<float>(kRev ? max(Lc - 1 - i, 0) : i + 1));
                const float2 rs2 = make_float2(rs, rs);
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    float oi[16];
                    tmem_ld16(lane_addr + Cfg::kColOn + 32 * cq + 16 * k, o[k]);
                    tmem_ld16(lane_addr + Cfg::kColOi + 32 * cq + 16 * k, oi);
                    tmem_ld_wait();
#pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        const float2 r = __ffma2_rn(make_float2(oi[2 * m], oi[2 * m + 1]), rs2,
                                                    make_float2(o[k][2 * m], o[k][2 * m + 1]));
                        o[k][2 * m] = r.x;
                        o[k][2 * m + 1] = r.y;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_Of);
            if (Lc == kC) {
                // two-round outputs: rows 64..127 wait until the store has read rows 0..63
                if (rd == 1 && !(ok = warp_wait(bar_F, static_cast<uint32_t>(c) & 1, lane))) break;
#pragma unroll
                for (int k = 0; k < 2; ++k)
                    stage16(q_slot(s), cq >> 1, 2 * (cq & 1) + k, i - rd * Stg::kRows, o[k], static_cast<OutT *>(nullptr));
                fence_proxy_async_smem();
            } else if (i < Lc && 32 * cq < Dm) {
                OutT *orow = static_cast<OutT *>(args.o) + (static_cast<size_t>(tok0 + ci * kC + i) * H + h) * Dm + 32 * cq;
#pragma unroll
                for (int k = 0; k < 2; ++k) store16(orow + 16 * k, o[k]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_E[2 * rd + s]);
            if (tracer) LA_PHASE(c, 12);

            // ---- state pass: S(c) hi -> this pair's V slot, lo -> X (dS has read V and K'_lo), then
            //      S *= lambda^L of the next chunk in TMEM; after the last chunk, S is the final state
            if (!(ok = warp_wait(bar_dS, static_cast<uint32_t>(c) & 1, lane))) break;
            if (tracer) LA_PHASE(c, 13);
            tc_fence_after();
            {
                float sv[32];
                tmem_ld32(s_col, sv);
                tmem_ld_wait();
                if (c + 1 < nchunks) {
                    store_state_split32(v_slot(s), x_slot, cq >> 1, cq & 1, i, sv);
                    const float ln = exp2f(g * static_cast<float>(min(kC, len - chunk_at(c + 1) * kC)));
                    const float2 ln2 = make_float2(ln, ln);
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const float2 r = __fmul2_rn(make_float2(sv[2 * m], sv[2 * m + 1]), ln2);
                        sv[2 * m] = r.x;
                        sv[2 * m + 1] = r.y;
                    }
                    tmem_st32(s_col, sv);
                    tmem_st_wait();
                    fence_proxy_async_smem();
                } else if (fin) {
                    float4 *p = reinterpret_cast<float4 *>(fin);
#pragma unroll
                    for (int j = 0; j < 8; ++j) p[j] = make_float4(sv[4 * j], sv[4 * j + 1], sv[4 * j + 2], sv[4 * j + 3]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_S);
            if (tracer) LA_PHASE(c, 14);
        }
        if (!ok && lane == 0) set_abort(abort_flag);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
    if (threadIdx.x == 0) LA_CTA_TIME(0, 1);
}

// ============================================================================ segment-state kernel
// First pass of the segment split: the state a fine unit of Lu tokens produces
// from a zero start, dS = sum_p lambda^(Lu-1-p) k_p^T v_p over its positions p,
// written to the workspace slot of the unit. The decay of every token to the
// unit's end is folded into K' = diag(lambda^(Lu-1-p)) K (split bf16 hi + lo),
// so the products of all chunks accumulate into one TMEM tile and no state is
// carried through registers. (A weight that underflows is below 2^-126 of the
// largest one, where the true contribution is negligible.) Only K and V are
// read, through three stages.
//
// K' never passes through shared memory. Per chunk the tensor core first copies
// K^T into TMEM: eight products of M = 128 features by N = 16 tokens by K = 16
// tokens, A = the chunk's K tile read feature-major (as an A operand) and B = a
// 16 x 16 identity, each writing the 16 columns of its tokens (exact: every
// product is one bf16 value times 1). The 16 scale warps then read those columns
// (lane = feature, column = token), multiply each column by its token's weight,
// split the result into bf16 hi and lo and write them back in place, laid out as
// the A operand of a TMEM-A product (the layout P takes in the chunk kernel); dS
// then accumulates from it with only V read from shared memory. K^T / K' is
// double buffered, so the scale pass of chunk c runs while the products of chunk
// c-1 do. Roles: warp 0 TMA, warp 1 MMA, warps 2-17 the scale pass and finally
// the drain of the accumulator.
// kRev (the reverse sweep of the backward pass): the weights are lambda^(p+1),
// the decay from the unit's start, units of the sequence's first segment are
// skipped, and the last unit of a sequence carries the given state.
template <bool kRev = false>
__global__ void __launch_bounds__(kStateThreads, 1)
    la_state_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const ChunkArgs args) {
    using Cfg = StateCfg;
    griddep_launch_dependents();  // the chunk kernel may be scheduled now; what needs this pass waits for it
    const int unit = blockIdx.x;
    const int h = blockIdx.y;
    int4 u;
    if (!fine_unit(args.map, unit, u)) return;
    // units inside the segment a sequence is left by: their state is never needed
    if (!args.map.all_units && (u.w & (kRev ? kFineInFirst : kFineInLast))) return;
    if (threadIdx.x == 0) LA_CTA_TIME(1, 0);
    const int tok0 = u.x, len = u.y;
    const int nchunks = (len + kC - 1) / kC;
    const int H = args.H;
    const float g = decay_log2(args.slopes, h, H);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOffset);
    uint64_t *full = bars;                   // [3] K, V of a stage landed
    uint64_t *empty = bars + 3;              // [3] stage consumed by the tensor core
    // [2] K^T of chunk c copied into its TMEM buffer (c % 2) / scaled and split there (16 warps). A warp cannot
    // arrive for chunk c+2 before every warp has for chunk c: its K^T is only copied after the products of
    // chunk c, which wait for all sixteen.
    uint64_t *kx = bars + 6;
    uint64_t *kp = bars + 8;
    uint64_t *bar_O = bars + 10;             // every product accumulated
    uint64_t *bar_done = bars + 11;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 12);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
    auto k_slot = [&](int s) { return smem + s * Cfg::kStageBytes; };
    auto v_slot = [&](int s) { return smem + s * Cfg::kStageBytes + kTileBytes; };
    uint8_t *i_tile = smem + Cfg::kOffI;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&kx[b], 1);
            mbar_init(&kp[b], Cfg::kScaleWarps);
        }
        mbar_init(bar_O, 1);
        mbar_init(bar_done, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (threadIdx.x >= 64 && threadIdx.x < 64 + 16 * 8) {
        // the identity: row n holds a 1 at column n (16-byte chunk n / 8, swizzled to (n / 8) ^ (n % 8))
        const int t = threadIdx.x - 64, n = t >> 3, j = t & 7;
        uint4 x = make_uint4(0u, 0u, 0u, 0u);
        if (j == ((n >> 3) ^ (n & 7))) {
            const uint32_t one = 0x3f80u << (16 * (n & 1));   // bf16 1.0 in the low or high half of a word
            const int w = (n & 7) >> 1;
            if (w == 0) x.x = one;
            if (w == 1) x.y = one;
            if (w == 2) x.z = one;
            if (w == 3) x.w = one;
        }
        *reinterpret_cast<uint4 *>(i_tile + n * 128 + j * 16) = x;
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto kt_col = [&](int c) { return Cfg::kColKT + 128u * static_cast<uint32_t>(c & 1); };

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int issued = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % Cfg::kStages;
                if (c >= Cfg::kStages &&
                    !mbar_wait(&empty[s], static_cast<uint32_t>((c - Cfg::kStages) / Cfg::kStages) & 1)) {
                    set_abort(abort_flag);
                    break;
                }
                if (*reinterpret_cast<volatile int *>(abort_flag)) break;
                const int t = tok0 + c * kC;
                LA_SPHASE(c, 0);
                mbar_arrive_expect_tx(&full[s], 2 * kTileBytes);
                tma_load_3d(k_slot(s), &tm_k, 0, h, t, &full[s]);
                tma_load_3d(k_slot(s) + kSlabBytes, &tm_k, 64, h, t, &full[s]);
                tma_load_3d(v_slot(s), &tm_v, 0, h, t, &full[s]);
                tma_load_3d(v_slot(s) + kSlabBytes, &tm_v, 64, h, t, &full[s]);
                issued = c + 1;
            }
            // never leave with a copy in flight: wait (bounded) for the last loads of each stage
            for (int c = (issued > Cfg::kStages ? issued - Cfg::kStages : 0); c < issued; ++c)
                mbar_wait(&full[c % Cfg::kStages], static_cast<uint32_t>(c / Cfg::kStages) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t id_kx = idesc_bf16_f32(kD, 16, true, false);   // M = features, N = 16 tokens
            constexpr uint32_t id_ds = idesc_bf16_f32(kD, kD, false, true);   // A = K'^T from TMEM, B = V
            const uint32_t idl = dlo_kmajor(smem_u32(i_tile));
            bool fine = true;
            // K^T of chunk c into TMEM (the stage holding it has landed; its buffer was last read by the products
            // of chunk c-2, issued before)
            auto copy_kt = [&](int c) -> bool {
                const int s = c % Cfg::kStages;
                if (!mbar_wait(&full[s], static_cast<uint32_t>(c / Cfg::kStages) & 1)) return false;
                LA_SPHASE(c, 4);
                tc_fence_after();
                const uint32_t kdl = dlo_mnmajor(smem_u32(k_slot(s)));
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ss_w(tmem + kt_col(c) + 16u * kk, kdl + dstep_mnmajor(kk), kDescHi, idl, kDescHi, id_kx, 0);
                mma_commit(&kx[c & 1]);
                return true;
            };
            // dS += (K'_hi + K'_lo)^T V of chunk c, once the scale pass has written K' hi / lo
            auto products = [&](int c) -> bool {
                const int s = c % Cfg::kStages;
                if (!mbar_wait(&kp[c & 1], static_cast<uint32_t>(c >> 1) & 1)) return false;
                LA_SPHASE(c, 5);
                tc_fence_after();
                const uint32_t vd = dlo_mnmajor(smem_u32(v_slot(s)));
                const uint32_t a = tmem + kt_col(c);
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ts_w(tmem + Cfg::kColD, a + p_hi_col(kk), vd + dstep_mnmajor(kk), kDescHi, id_ds,
                             (c > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ts_w(tmem + Cfg::kColD, a + p_hi_col(kk) + 16, vd + dstep_mnmajor(kk), kDescHi, id_ds, 1u);
                mma_commit(&empty[s]);
                return true;
            };
            for (int c = 0; c < nchunks && fine; ++c) {
                if (!(fine = copy_kt(c))) break;
                if (c > 0 && !(fine = products(c - 1))) break;
            }
            if (fine && nchunks > 0) fine = products(nchunks - 1);
            if (!fine) set_abort(abort_flag);
            mma_commit(bar_O);
            mma_commit(bar_done);
            mbar_wait(bar_done, 0);
        }
    } else if (warp >= 2 && warp < 2 + Cfg::kScaleWarps) {
        const int e = warp - 2;                 // 0..15
        const int q4 = warp & 3;                // TMEM lane quarter this warp may access
        const int cq = e >> 2;                  // 32-token quarter of the chunk (K' pass) / 32-column quarter (drain)
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * q4) << 16);
        const float lam = exp2f(g);
        const float2 lam2 = make_float2(lam * lam, lam * lam);
        bool ok = true;
        for (int c = 0; c < nchunks && ok; ++c) {
            if (warp_aborted(abort_flag, lane)) {
                ok = false;
                break;
            }
            if (!(ok = warp_wait(&kx[c & 1], static_cast<uint32_t>(c >> 1) & 1, lane))) break;
            if (e == 0 && lane == 0) LA_SPHASE(c, 1);
            tc_fence_after();
            // this thread: feature 32*q4 + lane, tokens p0 .. p0+31 of the unit (columns 32*cq.. of the chunk)
            const uint32_t col = lane_addr + kt_col(c) + 32u * cq;   // K'_hi at +0..15, K'_lo at +16..31
            float a[2][16];
            tmem_ld16(col, a[0]);
            tmem_ld16(col + 16, a[1]);
            tmem_ld_wait();
            const int p0 = c * kC + 32 * cq;
            if (p0 + 31 < len) {
                // whole block: weights walk by lambda from the end nearest the decay origin
                if (!kRev) {
                    const float w31 = exp2f(g * static_cast<float>(len - 1 - (p0 + 31)));
                    float2 fp = make_float2(w31 * lam, w31);
#pragma unroll
                    for (int sb = 1; sb >= 0; --sb) {
                        uint32_t hi[8], lo[8];
#pragma unroll
                        for (int m = 7; m >= 0; --m) {
                            split2(__fmul2_rn(make_float2(a[sb][2 * m], a[sb][2 * m + 1]), fp), hi[m], lo[m]);
                            fp = __fmul2_rn(fp, lam2);
                        }
                        tmem_st8(col + 8 * sb, hi);
                        tmem_st8(col + 16 + 8 * sb, lo);
                    }
                } else {
                    const float w0 = exp2f(g * static_cast<float>(p0 + 1));
                    float2 fp = make_float2(w0, w0 * lam);
#pragma unroll
                    for (int sb = 0; sb < 2; ++sb) {
                        uint32_t hi[8], lo[8];
#pragma unroll
                        for (int m = 0; m < 8; ++m) {
                            split2(__fmul2_rn(make_float2(a[sb][2 * m], a[sb][2 * m + 1]), fp), hi[m], lo[m]);
                            fp = __fmul2_rn(fp, lam2);
                        }
                        tmem_st8(col + 8 * sb, hi);
                        tmem_st8(col + 16 + 8 * sb, lo);
                    }
                }
            } else {
                // the unit's last chunk, cut short: each weight on its own, zero past the unit's end (whatever
                // the columns there hold)
#pragma unroll
                for (int sb = 0; sb < 2; ++sb) {
                    uint32_t hi[8], lo[8];
#pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        float w[2];
#pragma unroll
                        for (int t = 0; t < 2; ++t) {
                            const int p = p0 + 16 * sb + 2 * m + t;
                            w[t] = p < len ? exp2f(g * static_cast<float>(kRev ? p + 1 : len - 1 - p)) : 0.f;
                        }
                        const float x0 = w[0] != 0.f ? a[sb][2 * m] * w[0] : 0.f;
                        const float x1 = w[1] != 0.f ? a[sb][2 * m + 1] * w[1] : 0.f;
                        split2(make_float2(x0, x1), hi[m], lo[m]);
                    }
                    tmem_st8(col + 8 * sb, hi);
                    tmem_st8(col + 16 + 8 * sb, lo);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&kp[c & 1]);
            if (e == 0 && lane == 0) LA_SPHASE(c, 2);
        }
        if (ok) ok = warp_wait(bar_O, 0, lane);
        if (ok) {
            tc_fence_after();
            const int i = 32 * q4 + lane;
            const int Dm = args.D, ld = args.seg_ld;
            const size_t DD = static_cast<size_t>(Dm) * Dm, LL = static_cast<size_t>(ld) * ld;
            const size_t row = static_cast<size_t>(i) * ld + 32 * cq;     // in the unit states
            const size_t urow = static_cast<size_t>(i) * Dm + 32 * cq;    // in the caller's states
            const bool in_state = i < Dm && 32 * cq < Dm;
            // the unit a sequence is entered by (its first, its last with kRev) also carries the initial
            // state, decayed over the unit, and keeps a copy of it for the entry segment
            const float *s0 = (u.w & (kRev ? kFineLast : kFineFirst)) && args.s_init && in_state
                                  ? args.s_init + (static_cast<size_t>(u.z) * H + h) * DD + urow
                                  : nullptr;
            const float lamL = exp2f(g * static_cast<float>(len));
            // unit states in 128 x 128 tiles keep the padding (zeros); in D x D only the entries that exist
            float4 *dst = (ld == kD || in_state)
                              ? reinterpret_cast<float4 *>(args.seg_state + (static_cast<size_t>(unit) * H + h) * LL + row)
                              : nullptr;
            float4 *cpy = s0 ? reinterpret_cast<float4 *>(args.s0_copy + (static_cast<size_t>(u.z) * H + h) * DD + urow)
                             : nullptr;
            float d[32];
            if (nchunks > 0) {
                tmem_ld32(lane_addr + Cfg::kColD + 32 * cq, d);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) d[j] = 0.f;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float4 x = make_float4(d[4 * j], d[4 * j + 1], d[4 * j + 2], d[4 * j + 3]);
                if (s0) {
                    const float4 z = reinterpret_cast<const float4 *>(s0)[j];
                    cpy[j] = z;
                    x.x = fmaf(lamL, z.x, x.x);
                    x.y = fmaf(lamL, z.y, x.y);
                    x.z = fmaf(lamL, z.z, x.z);
                    x.w = fmaf(lamL, z.w, x.w);
                }
                if (dst) dst[j] = x;
            }
        } else if (lane == 0) {
            set_abort(abort_flag);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
    if (threadIdx.x == 0) LA_CTA_TIME(1, 1);
}

}  // namespace la
