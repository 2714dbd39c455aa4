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
//   O      = P V + diag(lambda^(i+1)) (Q S)            (tensor core, one accumulator)
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
// Per chunk c the tensor core runs
//   Q S(c) | dS(c) | P V(c) | Q K^T(c+1) | K^T copy(c+1)
// and the epilogue, with all 16 warps, K'(c) | P(c) | Oi(c) | S(c) | O(c):
//   K'(c)  after the K^T copy: K^T (an identity product put it in TMEM, lane =
//          feature) weighted by lambda^(Lc-1-s), split into hi / lo in place
//   P(c)   after Q K^T(c): A masked and weighted, split into hi / lo in place
//   Oi(c)  after Q S(c): the O accumulator scaled by lambda^(i+1) in place
//   S(c)   after dS(c): S hi / lo to their tiles for Q S(c+1), S rescaled
//   O(c)   after P V(c) (accumulated onto the scaled Q S): staged for the store
// The state chain S(c-1) -> Q S(c) -> dS(c) -> S(c) holds only those two
// products: K'(c) is made while Q S(c) runs, and the S hi / lo have tiles of
// their own, so the state pass does not wait for P V.
//
// TMEM, 512 columns: [0,128) scores A, each 32-column block b overwritten in
// place by P_hi (16 columns of packed bf16 pairs) then P_lo (16 columns);
// [128,256) O; [256,384) the fp32 state S, which dS accumulates into;
// [384,512) K^T, then K'_hi / K'_lo in the layout of P (the A operand of dS).
//
// Shared memory (226 KB): 32 KB tiles ([128 x 128] bf16 as two 64-column slabs
// with 128-byte rows and the 128-byte swizzle) and the 16 x 16 identity:
//   Q[p] (p = c%2): Q_c (read by Q K^T, Q S) -> O_c staging -> Q_{c+2}
//   K (one slot):   K_c (read by Q K^T and the K^T copy, at the end of chunk
//                   c-1's products) -> K_{c+1}, which has a chunk to arrive in
//   V[p]:           V_c (read by dS, P V) -> V_{c+2}
//   S_hi, S_lo:     the state entering the next chunk (read by its Q S)
//
// D = 64 has an instance of its own: Q, K and V are one 64-column slab each, Q K^T
// and Q S take 4 K steps, P V and dS are N = 64 products, and the room this frees
// is spent on shorter chains: K gets a second slot (in the S_lo tile), O is staged
// in the second half of its Q slot (so Q S frees a Q slot), Q S is one N = 128
// product on [S_hi | S_lo] (the two slabs of the S_hi tile), and dS is one stacked
// product: K is loaded into both slabs of its slot, so the K^T copy puts the 64
// features in TMEM lanes 0..63 and again in lanes 64..127, which take K'_hi and
// K'_lo, and S accumulates as [S_top; S_bot] with S = S_top + S_bot. S_bot is
// about 2^-8 of S, so its bf16 image (rows 64..127 of the S_hi tile's first slab)
// adds one N = 64 product to Q S and no lo half; the exit state adds the two.
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
constexpr int kPhaseSlots = 8, kPhaseChunks = 64, kPhaseEvents = 64;
constexpr int kTraceCtas = 8192;
// Start / end (global timer, ns) of every CTA of the chunk kernel (0) and the state or correction kernel (1);
// slots 4 + slot hold the SM clock counter at the same points (their ratio is the SM clock).
__device__ long long g_la_cta[2][kTraceCtas][8];
#define LA_CTA_TIME(kid, slot)                                                                \
    do {                                                                                      \
        const int cta_ = blockIdx.y * gridDim.x + blockIdx.x;                                 \
        if (cta_ < kTraceCtas) {                                                              \
            g_la_cta[(kid)][cta_][(slot)] = (long long)globaltimer_ns();                      \
            g_la_cta[(kid)][cta_][4 + (slot)] = (long long)clock64();                         \
        }                                                                                     \
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
    // Corrected split (forward only): no state pass runs first. A sequence's entry segment starts from its
    // initial state, every other segment from zero, and each segment of a multi-segment sequence leaves its
    // exit state in the workspace slot of its (only) fine unit; la_correct_tc_kernel then adds the entry-state
    // terms to the outputs and forms the final states.
    int corrected;
};

constexpr int kIdentityBytes = 16 * 128;   // the 16 x 16 identity operand of the K^T copies

// Shared memory of the main kernel (32 KB tiles): two Q slots, one K slot, two V slots, the S_hi and S_lo
// tiles, the identity; the barriers in the alignment gap before the tiles when it has room, else after them.
// TMEM: scores / P [0,128), the O accumulator [128,256), the state S [256,384), K^T / K' [384,512).
struct ChunkCfg {
    static constexpr int kOffQ = 0;                // 2 x 32 KB
    static constexpr int kOffK = 2 * kTileBytes;   // 32 KB
    static constexpr int kOffV = 3 * kTileBytes;   // 2 x 32 KB
    static constexpr int kOffSH = 5 * kTileBytes;
    static constexpr int kOffSL = 6 * kTileBytes;
    static constexpr int kOffI = 7 * kTileBytes;
    static constexpr int kTileEnd = kOffI + kIdentityBytes;
    static constexpr int kBarBytes = 256;
    // 1024 bytes of alignment slack: a gap of at least kBarBytes holds the barriers, a smaller one leaves
    // room for them after the tiles
    static constexpr int kSmemBytes = kTileEnd + 1024;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColA = 0, kColO = 128, kColS = 256, kColKT = 384;
};
static_assert(ChunkCfg::kSmemBytes <= 232448, "the chunk kernel's shared memory exceeds 227 KB");

struct StateCfg {
    static constexpr int kStages = 3;
    static constexpr int kStageBytes = 2 * kTileBytes;   // K, V
    // a 16 x 16 identity as the B operand of the products that copy K^T into TMEM: 16 rows of 64 bf16 (K-major,
    // 128-byte rows with the 128-byte swizzle, like every other operand tile), only the first 16 columns used
    static constexpr int kOffI = kStages * kStageBytes;
    static constexpr int kBarOffset = kOffI + kIdentityBytes;
    static constexpr int kSmemBytes = kBarOffset + 256 + 1024;
    // TMEM: dS [0,128); K^T then K' hi/lo of chunks 0, 2, .. at [128,256) and of chunks 1, 3, .. at [256,384)
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColD = 0, kColKT = 128;
    static constexpr int kScaleWarps = 16;
};

// O tiles as TMA boxes with the 128-byte swizzle: a box is 128 bytes of columns wide (32 fp32 or 64 16-bit
// values) and kRows rows high; a 16-bit tile is one round of kBoxes boxes (32 KB), an fp32 tile two rounds
// (rows 0-63, then 64-127) of 32 KB.
template <typename OutT>
struct OutStaging {
    static constexpr int kRounds = sizeof(OutT) == 4 ? 2 : 1;
    static constexpr int kRows = kC / kRounds;
    static constexpr int kBoxCols = 128 / static_cast<int>(sizeof(OutT));
    static constexpr int kBoxes = kD / kBoxCols;
    static constexpr int kBoxBytes = kRows * 128;
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

// S[0..31] = src[0..31] (src 16-byte aligned fp32).
__device__ __forceinline__ void acc_row32_set(float (&S)[32], const float *src) {
    const float4 *p = reinterpret_cast<const float4 *>(src);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float4 x = p[j];
        S[4 * j] = x.x;
        S[4 * j + 1] = x.y;
        S[4 * j + 2] = x.z;
        S[4 * j + 3] = x.w;
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

// Stage 16 output values of row `row` (of the current round), columns [64*hf + 16*qq, +16), at their
// swizzled box positions: 16-byte chunk j of a 128-byte box row lands at j ^ (row & 7).
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

// A 16 x 16 bf16 identity as a K-major operand tile with the 128-byte swizzle (16 rows of 128 bytes, only
// the first 16 columns used); thread t (0..127) writes the 16-byte chunk t % 8 of row t / 8: row n holds its
// 1 in chunk n / 8, swizzled to (n / 8) ^ (n % 8).
__device__ __forceinline__ void write_identity16(uint8_t *tile, int t) {
    const int n = t >> 3, j = t & 7;
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (j == ((n >> 3) ^ (n & 7))) {
        const uint32_t one = 0x3f80u << (16 * (n & 1));   // bf16 1.0 in the low or high half of a word
        const int w = (n & 7) >> 1;
        if (w == 0) x.x = one;
        if (w == 1) x.y = one;
        if (w == 2) x.z = one;
        if (w == 3) x.w = one;
    }
    *reinterpret_cast<uint4 *>(tile + n * 128 + j * 16) = x;
    fence_proxy_async_smem();
}

// Which halves of a split K' block go to TMEM: hi at col+0..15 and lo at col+16..31, or only one of them at
// col+0..15 (the D = 64 kernel stacks K'_hi of features 0..63 and K'_lo of the same features in lanes 64..127).
enum KPart { kHiLo = 0, kHiOnly = 1, kLoOnly = 2 };

// K' of one feature: the K^T values a (tokens p0..p0+31 of a run of `len` tokens) weighted by
// lambda^(len-1-p) (kRev: lambda^(p+1)), zero past len, split into bf16 hi / lo and stored to TMEM at `col`
// (this thread's lane) as the A operand of a TMEM-A product. The caller waits for the stores.
template <bool kRev, int kPart = kHiLo>
__device__ __forceinline__ void scale_split_store(uint32_t col, float (&a)[2][16], float g, float lam, int p0, int len) {
    const float2 lam2 = make_float2(lam * lam, lam * lam);
    auto put = [&](int sb, const uint32_t (&hi)[8], const uint32_t (&lo)[8]) {
        if (kPart == kHiLo) {
            tmem_st8(col + 8 * sb, hi);
            tmem_st8(col + 16 + 8 * sb, lo);
        } else {
            tmem_st8(col + 8 * sb, kPart == kHiOnly ? hi : lo);
        }
    };
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
                put(sb, hi, lo);
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
                put(sb, hi, lo);
            }
        }
    } else {
        // a block cut short: each weight on its own, zero past the run's end (whatever the columns there hold)
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
            put(sb, hi, lo);
        }
    }
}

// K' from the K^T a tensor-core copy put into TMEM (lane = feature, column = token; exact bf16 values),
// written back in place.
template <bool kRev, int kPart = kHiLo>
__device__ __forceinline__ void scale_split_kt(uint32_t col, float g, float lam, int p0, int len) {
    float a[2][16];
    tmem_ld16(col, a[0]);
    tmem_ld16(col + 16, a[1]);
    tmem_ld_wait();
    scale_split_store<kRev, kPart>(col, a, g, lam, p0, len);
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
template <typename OutT, bool kRev = false, bool kD64 = false>
__global__ void __launch_bounds__(kTcThreads, 1)
    la_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                       const ChunkArgs args) {
    using Cfg = ChunkCfg;
    using Stg = OutStaging<OutT>;
    // head dimension the products run over: 64 for the D = 64 instance, which loads one 64-column slab of
    // Q and V per chunk (K: the same slab into both halves of its slot) and multiplies only the real columns
    constexpr int kDv = kD64 ? 64 : kD;
    constexpr uint32_t kOpBytes = kD64 ? kSlabBytes : kTileBytes;   // bytes of one Q, K or V tile load
    // the output correction that may follow (programmatic dependent launch) waits for this grid on the device
    griddep_launch_dependents();
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

    // The tiles start at the first 1024-byte boundary of the dynamic shared memory; the barriers sit in the
    // gap before it when it has room, else after the tiles (both fit in kSmemBytes).
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem - smem_raw >= Cfg::kBarBytes ? smem - Cfg::kBarBytes
                                                                                   : smem + Cfg::kTileEnd);
    uint64_t *full_q = bars;             // [2] Q of a chunk landed
    uint64_t *full_k = bars + 2;         // K of a chunk landed
    uint64_t *full_v = bars + 3;         // [2] V of a chunk landed
    uint64_t *q_free = bars + 5;         // [2] Q slot free (the O staged in it has been read by the store)
    uint64_t *k_free = bars + 7;         // K slot free (Q K^T and the K^T copy of its chunk done)
    uint64_t *empty_v = bars + 8;        // [2] V slot free (dS and P V of its chunk done)
    uint64_t *bar_QK = bars + 10;        // A = Q K^T done
    uint64_t *bar_QS = bars + 11;        // O = Q S done
    uint64_t *bar_PV = bars + 12;        // O += P V done
    uint64_t *bar_dS = bars + 13;        // dS accumulated into S
    uint64_t *bar_KT = bars + 14;        // K^T copied into TMEM
    uint64_t *bar_P = bars + 15;         // P hi/lo in TMEM (16 warps)
    uint64_t *bar_K = bars + 16;         // K' hi/lo in TMEM (16 warps)
    uint64_t *bar_Oi = bars + 17;        // Q S scaled in the O accumulator (16 warps)
    uint64_t *bar_Of = bars + 18;        // O read out of the accumulator (16 warps)
    uint64_t *bar_S = bars + 19;         // S hi/lo written, S rescaled in TMEM (16 warps)
    uint64_t *bar_E = bars + 20;         // [round][pair] O staging round written (16 / rounds warps)
    uint64_t *bar_F = bars + 24;         // O staging round 0 read by the store (two-round outputs)
    uint64_t *bar_done = bars + 25;      // every MMA retired
    uint64_t *full_k1 = bars + 26;       // D = 64: K of a chunk landed in the second K slot
    uint64_t *k_free1 = bars + 27;       // D = 64: second K slot free
    uint64_t *stg_free = bars + 28;      // [2] D = 64: O staging half of a Q slot read by the store
    uint64_t *bar_Sx = bars + 30;        // D = 64: the stacked state's lower half parked for the exit state (4 warps)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 31);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    auto q_slot = [&](int s) { return smem + Cfg::kOffQ + s * kTileBytes; };
    uint8_t *k_tile = smem + Cfg::kOffK;
    auto v_slot = [&](int s) { return smem + Cfg::kOffV + s * kTileBytes; };
    uint8_t *sh_tile = smem + Cfg::kOffSH, *sl_tile = smem + Cfg::kOffSL;
    uint8_t *i_tile = smem + Cfg::kOffI;
    // D = 64 has room to spare: K takes two slots (the second in the S_lo tile, which S_lo then leaves free;
    // K fills both slabs of a slot), and O is staged in the second half of its Q slot, so a Q slot is free
    // once Q S has read it
    constexpr int kKSlots = kD64 ? 2 : 1;
    auto k_slot = [&](int s) { return s == 0 ? k_tile : sl_tile; };
    auto kfull = [&](int s) { return s == 0 ? full_k : full_k1; };
    auto kfree = [&](int s) { return s == 0 ? k_free : k_free1; };
    auto stg_slot = [&](int s) { return kD64 ? q_slot(s) + kSlabBytes : q_slot(s); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&full_q[s], 1);
            mbar_init(&full_v[s], 1);
            mbar_init(&q_free[s], 1);
            mbar_init(&empty_v[s], 1);
            mbar_init(&bar_E[s], kEpiWarps / Stg::kRounds);
            mbar_init(&bar_E[2 + s], kEpiWarps / Stg::kRounds);
        }
        mbar_init(full_k, 1);
        mbar_init(k_free, 1);
        mbar_init(full_k1, 1);
        mbar_init(k_free1, 1);
        mbar_init(&stg_free[0], 1);
        mbar_init(&stg_free[1], 1);
        mbar_init(bar_Sx, 4);
        mbar_init(bar_F, 1);
        mbar_init(bar_QK, 1);
        mbar_init(bar_QS, 1);
        mbar_init(bar_PV, 1);
        mbar_init(bar_dS, 1);
        mbar_init(bar_KT, 1);
        mbar_init(bar_P, kEpiWarps);
        mbar_init(bar_K, kEpiWarps);
        mbar_init(bar_Oi, kEpiWarps);
        mbar_init(bar_Of, kEpiWarps);
        mbar_init(bar_S, kEpiWarps);
        mbar_init(bar_done, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (threadIdx.x >= 64 && threadIdx.x < 64 + 16 * 8) write_identity16(i_tile, threadIdx.x - 64);
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
        // Chunk c: V into pair c%2 once dS and P V of chunk c-2 are done; K into its slot once Q K^T and the
        // K^T copy of the chunk before in that slot are done; Q into pair c%2 once the O of chunk c-2 staged
        // there has been read by the store (D = 64: once Q S of chunk c-2 is done).
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int issued_q = 0, issued_k = 0, issued_v = 0;
            // K and Q of chunk c: K into its slot once Q K^T and the K^T copy of the chunk before in that slot
            // are done (D = 64: into both slabs, the second load served by L2), Q into pair c%2 once the slot is
            // free
            auto load_kq = [&](int c) -> bool {
                const int s = c & 1, ks = c % kKSlots;
                const int t = tok0 + chunk_at(c) * kC;
                if (c >= kKSlots && !mbar_wait(kfree(ks), static_cast<uint32_t>((c - kKSlots) / kKSlots) & 1)) return false;
                if (*reinterpret_cast<volatile int *>(abort_flag)) return false;
                LA_PHASE(c, 15);
                mbar_arrive_expect_tx(kfull(ks), kTileBytes);
                tma_load_3d(k_slot(ks), &tm_k, 0, h, t, kfull(ks));
                tma_load_3d(k_slot(ks) + kSlabBytes, &tm_k, kD64 ? 0 : 64, h, t, kfull(ks));
                issued_k = c + 1;
                if (c >= 2 && !mbar_wait(&q_free[s], static_cast<uint32_t>((c - 2) >> 1) & 1)) return false;
                if (*reinterpret_cast<volatile int *>(abort_flag)) return false;
                LA_PHASE(c, 16);
                mbar_arrive_expect_tx(&full_q[s], kOpBytes);
                tma_load_3d(q_slot(s), &tm_q, 0, h, t, &full_q[s]);
                if (!kD64) tma_load_3d(q_slot(s) + kSlabBytes, &tm_q, 64, h, t, &full_q[s]);
                issued_q = c + 1;
                return true;
            };
            // The loads are issued in the order their slots come free: V(c), then K and Q of chunk c + kAhead
            // (D = 64, whose K and Q slots free a chunk earlier than V's, runs them one chunk ahead).
            constexpr int kAhead = kD64 ? 1 : 0;
            bool fine = true;
            for (int c = 0; c < kAhead && c < nchunks && fine; ++c) fine = load_kq(c);
            for (int c = 0; c < nchunks && fine; ++c) {
                const int s = c & 1;
                const int t = tok0 + chunk_at(c) * kC;
                if (c >= 2 && !mbar_wait(&empty_v[s], static_cast<uint32_t>((c - 2) >> 1) & 1)) break;
                if (*reinterpret_cast<volatile int *>(abort_flag)) break;
                LA_PHASE(c, 17);
                mbar_arrive_expect_tx(&full_v[s], kOpBytes);
                tma_load_3d(v_slot(s), &tm_v, 0, h, t, &full_v[s]);
                if (!kD64) tma_load_3d(v_slot(s) + kSlabBytes, &tm_v, 64, h, t, &full_v[s]);
                issued_v = c + 1;
                if (c + kAhead < nchunks) fine = load_kq(c + kAhead);
            }
            if (issued_q < nchunks || issued_k < nchunks || issued_v < nchunks) set_abort(abort_flag);
            // Never leave with a copy in flight: wait (bounded) for the last loads of each slot.
            for (int c = (issued_k > kKSlots ? issued_k - kKSlots : 0); c < issued_k; ++c)
                mbar_wait(kfull(c % kKSlots), static_cast<uint32_t>(c / kKSlots) & 1);
            for (int c = (issued_q > 2 ? issued_q - 2 : 0); c < issued_q; ++c)
                mbar_wait(&full_q[c & 1], static_cast<uint32_t>(c >> 1) & 1);
            for (int c = (issued_v > 2 ? issued_v - 2 : 0); c < issued_v; ++c)
                mbar_wait(&full_v[c & 1], static_cast<uint32_t>(c >> 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Per chunk: Q S(c), dS(c), P V(c), Q K^T(c+1), K^T copy(c+1). The state chain S(c-1) -> Q S(c)
        // -> dS(c) -> S(c) holds no product beyond those two: K'(c) is made while Q S(c) runs and the S
        // hi / lo have slots of their own, so the state pass need not wait for P V.
        if (lane == 0) {
            constexpr uint32_t id_qk = idesc_bf16_f32(kC, kC, false, false);
            constexpr uint32_t id_pv = idesc_bf16_f32(kC, kDv, false, true);
            // D = 64: Q S is one N = 128 product on [S_hi | S_lo], the two 64-column slabs of the S_hi tile
            constexpr uint32_t id_qs = idesc_bf16_f32(kC, kD, false, true);
            constexpr uint32_t id_ds = idesc_bf16_f32(kD, kDv, false, true);  // A = K'^T from TMEM, B = V
            constexpr uint32_t id_sb = idesc_bf16_f32(kC, 64, false, true);   // D = 64: Q times the stacked lower state
            constexpr uint32_t id_kx = idesc_bf16_f32(kD, 16, true, false);   // M = features, N = 16 tokens
            const uint32_t idl = dlo_kmajor(smem_u32(i_tile));
            const uint32_t shd = dlo_mnmajor(smem_u32(sh_tile)), sld = dlo_mnmajor(smem_u32(sl_tile));
            bool fine = true;
            // A = Q K^T of chunk c (the score tile is free: P V of chunk c-1 was issued before), then K^T of
            // chunk c into TMEM (exact: each product is one bf16 value times 1; the tile was last read by dS
            // of chunk c-1, issued before); the K slot is then free
            auto qk_copy = [&](int c) -> bool {
                const int s = c & 1;
                const int ks = c % kKSlots;
                const uint32_t kdk = dlo_kmajor(smem_u32(k_slot(ks))), kdm = dlo_mnmajor(smem_u32(k_slot(ks)));
                if (!mbar_wait(kfull(ks), static_cast<uint32_t>(c / kKSlots) & 1)) return false;
                LA_PHASE(c, 19);
                if (!mbar_wait(&full_q[s], static_cast<uint32_t>(c >> 1) & 1)) return false;
                LA_PHASE(c, 20);
                tc_fence_after();
                const uint32_t qd = dlo_kmajor(smem_u32(q_slot(s)));
#pragma unroll
                for (int kk = 0; kk < kDv / 16; ++kk)
                    mma_ss_w(tmem + Cfg::kColA, qd + dstep_kmajor(kk), kDescHi, kdk + dstep_kmajor(kk), kDescHi, id_qk, kk > 0);
                mma_commit(bar_QK);
                LA_PHASE(c, 0);
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ss_w(tmem + Cfg::kColKT + 16u * kk, kdm + dstep_mnmajor(kk), kDescHi, idl, kDescHi, id_kx, 0);
                mma_commit(bar_KT);
                mma_commit(kfree(ks));
                return true;
            };
            if (nchunks > 0) fine = qk_copy(0);
            if (fine) LA_CTA_TIME(0, 2);
            for (int c = 0; c < nchunks && fine; ++c) {
                const int s = c & 1;
                const uint32_t r = static_cast<uint32_t>(c >> 1) & 1;
                // O = Q (S_hi + S_lo), the state entering chunk c, once the state pass of chunk c-1 is done and
                // O of chunk c-1 has been read out of the accumulator
                if (!(fine = mbar_wait(bar_S, static_cast<uint32_t>(c) & 1))) break;
                if (c > 0 && !(fine = mbar_wait(bar_Of, static_cast<uint32_t>(c - 1) & 1))) break;
                LA_PHASE(c, 1);
                tc_fence_after();
                {
                    const uint32_t qd = dlo_kmajor(smem_u32(q_slot(s)));
#pragma unroll
                    for (int kk = 0; kk < kDv / 16; ++kk)
                        mma_ss_w(tmem + Cfg::kColO, qd + dstep_kmajor(kk), kDescHi, shd + dstep_mnmajor(kk), kDescHi, id_qs, kk > 0);
                    if (!kD64) {
#pragma unroll
                        for (int kk = 0; kk < kD / 16; ++kk)
                            mma_ss_w(tmem + Cfg::kColO, qd + dstep_kmajor(kk), kDescHi, sld + dstep_mnmajor(kk), kDescHi, id_qs, 1);
                    } else {
                        // + Q S_bot (rows 64..127 of the S_hi tile's first slab) onto Q S_hi
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_ss_w(tmem + Cfg::kColO, qd + dstep_kmajor(kk), kDescHi, shd + dstep_mnmajor(kk + 4), kDescHi, id_sb, 1);
                    }
                }
                mma_commit(bar_QS);
                if (kD64) mma_commit(&q_free[s]);   // the last product that reads Q of chunk c
                LA_PHASE(c, 2);
                // S += (K'_hi + K'_lo)^T V, K' from TMEM (S was rescaled by lambda^Lc in the state pass of chunk c-1)
                if (!(fine = mbar_wait(bar_K, static_cast<uint32_t>(c) & 1))) break;
                if (!(fine = mbar_wait(&full_v[s], r))) break;
                LA_PHASE(c, 5);
                tc_fence_after();
                const uint32_t vd = dlo_mnmajor(smem_u32(v_slot(s)));
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ts_w(tmem + Cfg::kColS, tmem + Cfg::kColKT + p_hi_col(kk), vd + dstep_mnmajor(kk), kDescHi, id_ds, 1);
                if (!kD64) {   // D = 64 stacks K'_lo under K'_hi: one product makes [S_top; S_bot]
#pragma unroll
                    for (int kk = 0; kk < kC / 16; ++kk)
                        mma_ts_w(tmem + Cfg::kColS, tmem + Cfg::kColKT + p_hi_col(kk) + 16, vd + dstep_mnmajor(kk), kDescHi, id_ds, 1);
                }
                mma_commit(bar_dS);
                LA_PHASE(c, 6);
                // O += (P_hi + P_lo) V, P from TMEM, onto the scaled Q S
                if (!(fine = mbar_wait(bar_P, static_cast<uint32_t>(c) & 1))) break;
                if (!(fine = mbar_wait(bar_Oi, static_cast<uint32_t>(c) & 1))) break;
                LA_PHASE(c, 3);
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ts_w(tmem + Cfg::kColO, tmem + Cfg::kColA + p_hi_col(kk), vd + dstep_mnmajor(kk), kDescHi, id_pv, 1);
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    mma_ts_w(tmem + Cfg::kColO, tmem + Cfg::kColA + p_hi_col(kk) + 16, vd + dstep_mnmajor(kk), kDescHi, id_pv, 1);
                mma_commit(bar_PV);
                mma_commit(&empty_v[s]);
                LA_PHASE(c, 4);
                if (c == nchunks - 1) LA_CTA_TIME(0, 3);
                if (c + 1 < nchunks && !(fine = qk_copy(c + 1))) break;
            }
            if (!fine) set_abort(abort_flag);
            mma_commit(bar_done);
            mbar_wait(bar_done, 0);
        }
    } else if (warp == kStoreWarp) {
        // ------------------------------------------------------------ output store warp
        // O of chunk c is staged in the Q slot of its pair (one round for 16-bit outputs, two of 64
        // rows for fp32); once the store has read it, that Q slot takes Q of chunk c+2 (D = 64: O is
        // staged in the slot's second half, which then takes O of chunk c+2).
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
                                tma_store_3d(&tm_o, stg_slot(s) + bx * Stg::kBoxBytes, bx * Stg::kBoxCols, h,
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
                mbar_arrive(kD64 ? &stg_free[s] : &q_free[s]);
                LA_PHASE(c, 18);
            }
            tma_store_wait_all();
        }
    } else if (warp >= kEpi0 && warp < kEpi0 + kEpiWarps) {
        // ------------------------------------------------------------ epilogue (warps 3..18)
        const int e = warp - kEpi0;        // 0..15
        const int q4 = warp & 3;           // TMEM lane quarter this warp may access
        const int cq = e >> 2;             // 32-column quarter of every 128-column tile
        const int i = 32 * q4 + lane;      // TMEM lane: chunk row i (A, O), state row dk (S) or feature (K')
        const int rd = Stg::kRounds == 2 ? (q4 >> 1) : 0;   // output staging round of this warp's rows
        const bool tracer = (e == 1 && lane == 0);           // rows 0..31 of column quarter 0
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * q4) << 16);
        const uint32_t s_col = lane_addr + Cfg::kColS + 32 * cq;
        const float lam = exp2f(g);
        const float2 lam2 = make_float2(lam * lam, lam * lam);
        const int Dm = args.D;
        const size_t DD = static_cast<size_t>(Dm) * Dm;         // caller's states: [., H, D, D]
        const size_t kDD = static_cast<size_t>(kD) * kD;        // workspace segment states: [., H, 128, 128]
        const bool in_state = i < Dm && 32 * cq < Dm;          // this thread's 32 state entries are not padding
        // D = 64: the state's 64 columns are held by the column quarters 0 and 1 (rows 64..127 stay zero)
        const bool s_owner = !kD64 || cq < 2;
        // S(row i, 32 columns) hi / lo into the S tiles: D = 64 puts S_hi in slab 0 and S_lo in slab 1 of the
        // S_hi tile (the B operand [S_hi | S_lo] of one N = 128 product)
        auto put_state = [&](const float (&S)[32]) {
            if (kD64) store_state_split32(sh_tile, sh_tile + kSlabBytes, 0, cq & 1, i, S);
            else store_state_split32(sh_tile, sl_tile, cq >> 1, cq & 1, i, S);
        };
        const bool multi = !((flags & kUnitFirst) && (flags & kUnitLast));   // the sequence has several segments
        const bool corrected = !kRev && args.corrected;
        float *fin = (corrected && multi)
                         ? args.seg_state + (static_cast<size_t>(first_fine) * H + h) * kDD + static_cast<size_t>(i) * kD + 32 * cq
                     : ((flags & kExit) && args.s_final && in_state)
                         ? args.s_final + (static_cast<size_t>(seq) * H + h) * DD + static_cast<size_t>(i) * Dm + 32 * cq
                         : nullptr;

        // The state entering this segment (row i, columns 32*cq..+31). A single-segment sequence
        // reads its initial state; otherwise only the workspace is read (final_state may alias
        // initial_state, and another CTA of this sequence writes it): the entry segment takes the
        // copy of the initial state, another segment sums the decayed states of every fine unit
        // before it (after it with kRev; the unit the sequence is entered by already carries the
        // decayed initial state). Its hi / lo go to the S tiles (read by Q S of the first chunk
        // processed), lambda^L0 S to TMEM. In a corrected split the entry segment reads
        // the initial state itself (the final state is written after this grid) and the others start
        // from zero.
        {
            // the workspace is written by the segment-state pass, which may still be running
            if (!corrected && multi && (!(flags & kEntry) || args.s_init)) griddep_wait();
            float S[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) S[j] = 0.f;
            const size_t col = static_cast<size_t>(i) * Dm + 32 * cq;    // in the caller's states
            const size_t colw = static_cast<size_t>(i) * kD + 32 * cq;   // in the workspace states
            if (!multi || (corrected && (flags & kUnitFirst))) {
                if (args.s_init && in_state) acc_row32(S, args.s_init + (static_cast<size_t>(seq) * H + h) * DD + col, 1.f);
            } else if (corrected) {
                // zero
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
            } else if (s_owner) {
                put_state(S);
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

            // ---- K' = K^T weighted by lambda^(Lc-1-s) (kRev: lambda^(s+1)), zero past Lc, split into bf16
            //      hi / lo in place in TMEM (this warp: features i, tokens 32*cq..+31). D = 64 stacks the
            //      halves: lanes 0..63 keep K'_hi of features 0..63, lanes 64..127 (the same features) K'_lo.
            if (!(ok = warp_wait(bar_KT, static_cast<uint32_t>(c) & 1, lane))) break;
            if (tracer) LA_PHASE(c, 9);
            tc_fence_after();
            {
                const uint32_t col = lane_addr + Cfg::kColKT + 32 * cq;
                if (!kD64) scale_split_kt<kRev, kHiLo>(col, g, lam, 32 * cq, Lc);
                else if (q4 < 2) scale_split_kt<kRev, kHiOnly>(col, g, lam, 32 * cq, Lc);
                else scale_split_kt<kRev, kLoOnly>(col, g, lam, 32 * cq, Lc);
                tmem_st_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_K);
            if (tracer) LA_PHASE(c, 10);

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

            // ---- Q S in the O accumulator scaled in place by lambda^(i+1) (kRev: lambda^(Lc-1-i)); P V then
            //      accumulates onto it
            if (!(ok = warp_wait(bar_QS, static_cast<uint32_t>(c) & 1, lane))) break;
            if (tracer) LA_PHASE(c, 11);
            tc_fence_after();
            if (kD64) {
                // columns 16*cq..+15: Q S_hi (columns 0..63) plus Q S_lo (64..127), scaled, into columns 0..63
                float a[16], b[16];
                tmem_ld16(lane_addr + Cfg::kColO + 16 * cq, a);
                tmem_ld16(lane_addr + Cfg::kColO + 64 + 16 * cq, b);
                tmem_ld_wait();
                const float rs = exp2f(g * static_cast<float>(kRev ? max(Lc - 1 - i, 0) : i + 1));
                uint32_t r[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) r[j] = __float_as_uint((a[j] + b[j]) * rs);
                tmem_st16(lane_addr + Cfg::kColO + 16 * cq, r);
                tmem_st_wait();
            } else {
                float oi[32];
                tmem_ld32(lane_addr + Cfg::kColO + 32 * cq, oi);
                tmem_ld_wait();
                const float rs = exp2f(g * static_cast<float>(kRev ? max(Lc - 1 - i, 0) : i + 1));
                const float2 rs2 = make_float2(rs, rs);
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float2 x = __fmul2_rn(make_float2(oi[2 * m], oi[2 * m + 1]), rs2);
                    oi[2 * m] = x.x;
                    oi[2 * m + 1] = x.y;
                }
                tmem_st32(lane_addr + Cfg::kColO + 32 * cq, oi);
                tmem_st_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_Oi);
            if (lane == 0) LA_PHASE(c, 40 + e);

            // ---- state pass: S(c) hi / lo -> the S tiles (Q S of chunk c has read them: it ran before dS),
            //      then S *= lambda^L of the next chunk in TMEM; after the last chunk, S is the segment's exit
            //      state
            if (!(ok = warp_wait(bar_dS, static_cast<uint32_t>(c) & 1, lane))) break;
            if (tracer) LA_PHASE(c, 13);
            tc_fence_after();
            if (!s_owner) {
                // D = 64, columns 64..127: no state; a workspace exit state keeps its padding at zero
                if (c + 1 == nchunks && fin) {
                    float4 *p = reinterpret_cast<float4 *>(fin);
#pragma unroll
                    for (int j = 0; j < 8; ++j) p[j] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            } else {
                float sv[32];
                tmem_ld32(s_col, sv);
                tmem_ld_wait();
                if (c + 1 < nchunks) {
                    put_state(sv);
                    const float ln = exp2f(g * static_cast<float>(min(kC, len - chunk_at(c + 1) * kC)));
                    const float2 ln2 = make_float2(ln, ln);
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const float2 x = __fmul2_rn(make_float2(sv[2 * m], sv[2 * m + 1]), ln2);
                        sv[2 * m] = x.x;
                        sv[2 * m + 1] = x.y;
                    }
                    tmem_st32(s_col, sv);
                    tmem_st_wait();
                    fence_proxy_async_smem();
                } else {
                    if (kD64) {
                        // the exit state is S_top + S_bot: rows 64..127 park their S_bot in the free second half
                        // of V slot 0 ([64 x 64] fp32), rows 0..63 add it; the workspace's rows 64..127 are padding
                        float *park = reinterpret_cast<float *>(v_slot(0) + kSlabBytes);
                        if (q4 >= 2) {
                            float4 *pp = reinterpret_cast<float4 *>(park + (i - 64) * 64 + 32 * cq);
#pragma unroll
                            for (int j = 0; j < 8; ++j) pp[j] = make_float4(sv[4 * j], sv[4 * j + 1], sv[4 * j + 2], sv[4 * j + 3]);
                            __syncwarp();
                            if (lane == 0) mbar_arrive(bar_Sx);
#pragma unroll
                            for (int j = 0; j < 32; ++j) sv[j] = 0.f;
                        } else {
                            if (!(ok = warp_wait(bar_Sx, 0, lane))) break;
                            const float4 *pp = reinterpret_cast<const float4 *>(park + i * 64 + 32 * cq);
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const float4 x = pp[j];
                                sv[4 * j] += x.x;
                                sv[4 * j + 1] += x.y;
                                sv[4 * j + 2] += x.z;
                                sv[4 * j + 3] += x.w;
                            }
                        }
                    }
                    if (fin) {
                        float4 *p = reinterpret_cast<float4 *>(fin);
#pragma unroll
                        for (int j = 0; j < 8; ++j) p[j] = make_float4(sv[4 * j], sv[4 * j + 1], sv[4 * j + 2], sv[4 * j + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_S);
            if (tracer) LA_PHASE(c, 14);

            // ---- O = P V + the scaled Q S: read out of the accumulator (Q S of the next chunk may then run),
            //      then staged in this pair's Q slot for the store warp, or stored row by row (a chunk cut
            //      short by its sequence end must not write past it)
            if (!(ok = warp_wait(bar_PV, static_cast<uint32_t>(c) & 1, lane))) break;
            if (tracer) LA_PHASE(c, 12);
            tc_fence_after();
            {
                // D = 64: columns 16*cq..+15 of the 64; else 32*cq..+31
                constexpr int kParts = kD64 ? 1 : 2;
                const int c0 = kD64 ? 16 * cq : 32 * cq;
                float o[2][16];
#pragma unroll
                for (int k = 0; k < kParts; ++k) tmem_ld16(lane_addr + Cfg::kColO + c0 + 16 * k, o[k]);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_Of);
                if (lane == 0) LA_PHASE(c, 24 + e);
                if (Lc == kC) {
                    // D = 64: the store has read O of chunk c-2 from this staging half
                    if (kD64 && c >= 2 && !(ok = warp_wait(&stg_free[s], static_cast<uint32_t>((c - 2) >> 1) & 1, lane)))
                        break;
                    // two-round outputs: rows 64..127 wait until the store has read rows 0..63
                    if (rd == 1 && !(ok = warp_wait(bar_F, static_cast<uint32_t>(c) & 1, lane))) break;
#pragma unroll
                    for (int k = 0; k < kParts; ++k)
                        stage16(stg_slot(s), kD64 ? 0 : cq >> 1, kD64 ? cq : 2 * (cq & 1) + k, i - rd * Stg::kRows, o[k],
                                static_cast<OutT *>(nullptr));
                    fence_proxy_async_smem();
                } else if (i < Lc && c0 < Dm) {
                    OutT *orow = static_cast<OutT *>(args.o) + (static_cast<size_t>(tok0 + ci * kC + i) * H + h) * Dm + c0;
#pragma unroll
                    for (int k = 0; k < kParts; ++k) store16(orow + 16 * k, o[k]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_E[2 * rd + s]);
            }
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
    if (threadIdx.x >= 64 && threadIdx.x < 64 + 16 * 8) write_identity16(i_tile, threadIdx.x - 64);
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
            // this thread: feature 32*q4 + lane, tokens c*C + 32*cq .. +31 of the unit (columns 32*cq.. of the chunk)
            scale_split_kt<kRev>(lane_addr + kt_col(c) + 32u * cq, g, lam, c * kC + 32 * cq, len);
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
