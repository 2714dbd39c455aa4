// C ABI of the Lightning Attention library (declarations and contracts in
// include/la.h): argument checks, work planning, tensor-map encoding and
// kernel launches. Everything runs on the caller's stream; nothing here
// allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "la.h"
#include "la_bwd.cuh"
#include "la_chunk_tc.cuh"
#include "la_correct_tc.cuh"
#include "la_cp.cuh"
#include "la_decode.cuh"
#include "la_norm_gate.cuh"
#include "la_plan.cuh"
#include "la_simt.cuh"

namespace {

thread_local std::string t_last_error;
thread_local int t_last_launches = 0;

la_status fail(la_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return s;
}

// ---------------------------------------------------------------- tracing
struct TraceRec {
    const char *name;
    cudaEvent_t a, b;
};
thread_local bool t_trace = false;
thread_local std::vector<TraceRec> t_recs;
thread_local std::vector<cudaEvent_t> t_pool;

cudaEvent_t pooled_event() {
    if (!t_pool.empty()) {
        cudaEvent_t e = t_pool.back();
        t_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

void trace_pre(const char *name, cudaStream_t st) {
    if (!t_trace) return;
    TraceRec r{name, pooled_event(), pooled_event()};
    if (!r.a || !r.b) return;
    cudaEventRecord(r.a, st);
    t_recs.push_back(r);
}

void trace_post(cudaStream_t st) {
    if (!t_trace || t_recs.empty()) return;
    cudaEventRecord(t_recs.back().b, st);
}

la_status cuda_fail(cudaError_t e, const char *what) {
    return fail(LA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlap(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool valid_dtype(la_dtype dt) {
    return dt == LA_BF16 || dt == LA_FP32 || dt == LA_BF16_F32OUT || dt == LA_BF16_F16OUT;
}
size_t in_bytes(la_dtype dt) { return dt == LA_FP32 ? 4 : 2; }
size_t out_bytes(la_dtype dt) { return (dt == LA_BF16 || dt == LA_BF16_F16OUT) ? 2 : 4; }

// ---------------------------------------------------------------- driver entry point for TMA maps
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [T, H, D] viewed as a 3-D tensor (D, H, T) with boxes of (128 bytes of
// features) x 1 x box_rows tokens and the 128-byte swizzle: a box is a
// [box_rows x 64 16-bit] or [box_rows x 32 fp32] slab.
la_status make_map(CUtensorMap *m, const void *base, int64_t T, int H, int D, CUtensorMapDataType type,
                   int box_rows = la::kC) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return fail(LA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint64_t es = type == CU_TENSOR_MAP_DATA_TYPE_FLOAT32 ? 4 : 2;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                          static_cast<cuuint64_t>(std::max<int64_t>(T, 1))};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * es, static_cast<cuuint64_t>(H) * D * es};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / es), 1, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, type, 3,
                    const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(LA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
    return LA_OK;
}

// ---------------------------------------------------------------- planning
// CTAs the segment split aims for: about one main-kernel unit per SM of a
// 148-SM B200 for uniform batches, two for packed batches (uneven tails balance
// over two waves); the state pass splits its share of the work finer. Fixed
// numbers keep workspace sizes device-independent.
constexpr int kSmCount = 148;

// Plan overrides for tuning sweeps exist only in profiling builds (compiled with -DLA_PLAN_OVERRIDES):
// the shipped library's plan is a fixed function of the call's arguments, so a workspace size
// queried earlier always matches the call, and no call reads the process environment.
#ifdef LA_PLAN_OVERRIDES
int plan_override(const char *name) {
    const char *s = std::getenv(name);
    return s ? std::atoi(s) : 0;
}
#else
constexpr int plan_override(const char *) { return 0; }
#endif

struct Plan {
    bool tensor_core = false;  // bf16 inputs, T > 0 (D = 64 has chunk and correction instances of its own)
    bool segmented = false;    // some sequence spans more than one coarse segment
    bool corrected = false;    // segmented, forward, whole GPU: segments start at once, outputs corrected after
    int corr_chunks = 0, corr_pieces = 0, corr_items = 0;   // output correction: chunks per CTA, CTAs per segment / head
    bool corr_direct = false;  // two segments per sequence: the correction forms each entry state itself
    bool planned = false;      // packed batch: unit lists built on the device
    int sub_len = 0;           // fine unit length (multiple of 128)
    int R = 1;                 // fine units per coarse segment
    int nf = 0, nc = 0;        // per sequence (uniform batches)
    int cap_fine = 0, cap_coarse = 0;
    size_t off_fine = 0, off_coarse = 0, off_seq_fine = 0, off_seq_coarse = 0, off_counts = 0, off_state = 0,
           off_s0 = 0, off_eimg = 0;
    size_t bytes = 0;
};

int round_chunks(int64_t tokens) { return static_cast<int>((tokens + la::kC - 1) / la::kC); }

// `concurrency`: how many such calls run at once (the backward pass's three sweeps), so that the segment
// split only fills the share of the GPU a call gets.
Plan make_plan(int64_t T, int nseq, int N_uniform, int H, int D, la_dtype dt, bool reverse = false,
               int concurrency = 1) {
    Plan p;
    p.tensor_core = (dt != LA_FP32 && (D == 128 || D == 64) && T > 0);
    if (!p.tensor_core) return p;
    p.planned = (N_uniform == 0);
    const int64_t max_len = p.planned ? T : N_uniform;
    const int max_chunks = std::max(1, round_chunks(max_len));
    // The forward pass on the whole GPU uses the corrected split: its segments need no state pass before
    // them, so they all start at once, about one per SM; the state they miss is added to their outputs
    // afterwards, which reads and rewrites the stored outputs. That second rounding fits the error budget
    // of fp16 (2^-11) and fp32 outputs, not of bf16 (2^-8), whose storage alone can take most of it: bf16
    // outputs keep the state pass, and so do the backward sweeps (and any call sharing the GPU).
    const bool correctable = !reverse && concurrency == 1 && dt != LA_BF16 && plan_override("LA_NO_CORRECT") <= 0;
    // coarse segment length (chunks)
    int seg_chunks;
    bool two_seg = false;
    if (plan_override("LA_SEG_LEN") > 0) {
        seg_chunks = std::max(1, round_chunks(plan_override("LA_SEG_LEN")));
    } else if (correctable && !p.planned) {
        const int per_seq = std::max(1, kSmCount / std::max(1, nseq * H));
        seg_chunks = (max_chunks + per_seq - 1) / per_seq;
    } else if (!p.planned) {
        const int per_seq = std::max(1, kSmCount / std::max(1, nseq * H * concurrency));
        if (per_seq == 2 && max_chunks >= 4 && concurrency == 1) {
            // Two segments per sequence. The first needs no state pass and runs from the start, beside
            // the pass over it (one unit per sequence and head, so both fit on the GPU at once); the
            // second starts when that pass ends. Balanced when L0 * t_main = L0 * t_state + L1 * t_main
            // (t_state / t_main = 1.7 / 3.7 measured alone); timing the step over first-segment lengths
            // on B200 puts its optimum at about 0.69 of the sequence (22 of 32 chunks).
            seg_chunks = std::min(max_chunks - 1, std::max(1, (max_chunks * 11 + 8) / 16));
            // reversed in time, the sequence is entered by its last segment, which takes no state pass;
            // timing the backward pass on B200 puts its optimum at about 0.56 of the sequence (18 of 32
            // chunks: the reversed chunk kernel is slower per chunk, its state pass faster)
            if (reverse) seg_chunks = std::min(max_chunks - 1, std::max(1, max_chunks - (max_chunks * 9 + 8) / 16));
            two_seg = true;
        } else {
            seg_chunks = (max_chunks + per_seq - 1) / per_seq;
        }
    } else {
        const int64_t target = std::max<int64_t>(1, 2 * kSmCount / concurrency);
        seg_chunks = std::max<int>(1, round_chunks((T * H + target - 1) / target));
    }
    // segments of at least two chunks: a one-chunk segment's prologue and state unit cost more than its
    // parallelism saves (B=1, N=1024, H=16 on B200: 41.6 us with one-chunk segments, 35.3 us with two)
    if (plan_override("LA_SEG_LEN") <= 0) seg_chunks = std::max(seg_chunks, 2);
    seg_chunks = std::min(seg_chunks, max_chunks);
    const int nc_max = (max_chunks + seg_chunks - 1) / seg_chunks;
    // fine units: enough that the state pass over all but the last segments fills the GPU
    int R = 1;
    if (plan_override("LA_SUB_R") > 0) {
        R = plan_override("LA_SUB_R");
    } else if (nc_max > 1 && !two_seg) {
        const int64_t state_units = (p.planned ? (T / (static_cast<int64_t>(seg_chunks) * la::kC)) * H
                                               : static_cast<int64_t>(nseq) * H * (nc_max - 1)) * concurrency;
        // finer state units while the pass has SMs to spare, each of at least two chunks (one-chunk units
        // measured slower: B=1, N=1024 / 2048 / 4096, H=16 on B200, 41.8 / 50.7 / 81.1 us against 35.3 / 44.0 /
        // 56.2 us with two-chunk or longer ones)
        while (R < seg_chunks && state_units * R * 2 <= kSmCount && (seg_chunks + 2 * R - 1) / (2 * R) >= 2) R *= 2;
    }
    R = std::max(1, std::min(R, seg_chunks));
    if (correctable) R = 1;   // the corrected split keeps one exit state per segment
    const int sub_chunks = (seg_chunks + R - 1) / R;
    p.R = R;
    p.sub_len = sub_chunks * la::kC;
    const int64_t seg_len = static_cast<int64_t>(p.sub_len) * R;
    p.segmented = max_len > seg_len;
    p.corrected = correctable && p.segmented;
    if (!p.planned) {
        p.nf = std::max(1, static_cast<int>((N_uniform + p.sub_len - 1) / p.sub_len));
        p.nc = (p.nf + R - 1) / R;
        p.cap_fine = nseq * p.nf;
        p.cap_coarse = nseq * p.nc;
    } else {
        p.cap_fine = static_cast<int>(T / p.sub_len + nseq + 1);
        p.cap_coarse = static_cast<int>(T / seg_len + nseq + 1);
    }
    if (p.corrected) {
        // pieces of half a segment up to 16 chunks, else of 8 chunks: with the chunks of fast-decaying heads
        // skipped this keeps the correction grid within one wave (B=4, N=4096, H=16 on B200, steps back to back:
        // 104 CTAs of up to 8 chunks, 91.2 us per step against 91.9-92.4 with 6-chunk and more with 3-, 4- or
        // 5-chunk pieces; B=1, N=65536, H=16: 8-chunk pieces 310 us, 16-chunk ones within 1 %)
        p.corr_chunks = plan_override("LA_CORR_CHUNKS") > 0 ? plan_override("LA_CORR_CHUNKS")
                        : std::min(8, std::max(1, (seg_chunks + 1) / 2));
        p.corr_pieces = (seg_chunks + p.corr_chunks - 1) / p.corr_chunks;
        p.corr_items = (p.planned ? p.cap_coarse : nseq * (p.nc - 1)) * p.corr_pieces;
        p.corr_direct = !p.planned && p.nc == 2;
    }
    size_t off = 0;
    if (p.planned) {
        p.off_fine = off;
        off = align_up(off + sizeof(int4) * p.cap_fine, 256);
        p.off_coarse = off;
        off = align_up(off + sizeof(int4) * p.cap_coarse, 256);
        p.off_seq_fine = off;
        off = align_up(off + sizeof(int) * (nseq + 1), 256);
        p.off_seq_coarse = off;
        off = align_up(off + sizeof(int) * (nseq + 1), 256);
        p.off_counts = off;
        off = align_up(off + sizeof(int) * 2, 256);
    }
    // segment states in the kernels' 128 x 128 tiles; the initial-state copies in the caller's D x D
    p.off_state = off;
    if (p.segmented) off += sizeof(float) * static_cast<size_t>(p.cap_fine) * H * la::kD * la::kD;
    p.off_s0 = off;
    if (p.segmented && !p.corrected) off += sizeof(float) * static_cast<size_t>(nseq) * H * D * D;
    // corrected split: the entry state of every segment as its split 64 KB image
    p.off_eimg = off;
    if (p.corrected && !p.corr_direct) off += static_cast<size_t>(la::kEntryImageBytes) * p.cap_coarse * H;
    p.bytes = off;
    return p;
}

template <typename K>
la_status set_smem(K kernel, size_t bytes) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    return LA_OK;
}

la_status check_launch(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, what);
    return LA_OK;
}

la_status check_common(const void *q, const void *k, const void *v, const void *o, int64_t T, int H, int D,
                       la_dtype dt, const float *s0, const float *sN) {
    if (!valid_dtype(dt)) return fail(LA_ERR_INVALID_ARGUMENT, "dtype %d is not a la_dtype", dt);
    if (D != 64 && D != 128) return fail(LA_ERR_UNSUPPORTED, "head dim D=%d: only 64 and 128 are supported", D);
    if (H < 1 || H > 65535) return fail(LA_ERR_INVALID_ARGUMENT, "H=%d must be in [1, 65535]", H);
    if (T < 0) return fail(LA_ERR_INVALID_ARGUMENT, "token count %lld < 0", static_cast<long long>(T));
    if (T * H * D >= (int64_t(1) << 31))
        return fail(LA_ERR_UNSUPPORTED, "T*H*D = %lld elements must be < 2^31", static_cast<long long>(T * H * D));
    if (T > 0 && (!q || !k || !v || !o)) return fail(LA_ERR_INVALID_ARGUMENT, "q, k, v and o must be non-null");
    const void *ptrs[6] = {q, k, v, o, s0, sN};
    const char *names[6] = {"q", "k", "v", "o", "initial_state", "final_state"};
    for (int i = 0; i < 6; ++i)
        if (ptrs[i] && !aligned(ptrs[i], 16)) return fail(LA_ERR_INVALID_ARGUMENT, "%s is not 16-byte aligned", names[i]);
    const size_t ib = static_cast<size_t>(T) * H * D * in_bytes(dt), ob = static_cast<size_t>(T) * H * D * out_bytes(dt);
    if (ib && (overlap(o, ob, q, ib) || overlap(o, ob, k, ib) || overlap(o, ob, v, ib)))
        return fail(LA_ERR_INVALID_ARGUMENT, "o must not overlap q, k or v");
    return LA_OK;
}

template <typename Tin, typename Tout, bool kRev, int D, int Dc>
la_status launch_simt_cols(const void *q, const void *k, const void *v, void *o, const int32_t *cu, int nseq, int N,
                           int64_t T, int H, const float *s0, float *sN, const float *slopes, cudaStream_t st) {
    auto kern = la::la_simt_prefill_kernel<Tin, Tout, D, kRev, Dc>;
    la_status r;
    if ((r = set_smem(kern, la::SimtCfg<D, Dc>::kSmemBytes)) != LA_OK) return r;
    trace_pre("la_simt_prefill_kernel", st);
    kern<<<dim3(nseq, H, D / Dc), la::kSimtThreads, la::SimtCfg<D, Dc>::kSmemBytes, st>>>(
        static_cast<const Tin *>(q), static_cast<const Tin *>(k), static_cast<const Tin *>(v), static_cast<Tout *>(o),
        cu, N, static_cast<int>(T), H, s0, sN, slopes);
    trace_post(st);
    return LA_OK;
}

// The CUDA-core prefill: each (sequence, head) split over D / Dc CTAs by value columns (Dc >= 32) while the
// CTAs would otherwise leave SMs idle (each split repeats the chunk's score tile, so large batches keep one
// CTA per pair).
template <typename Tin, typename Tout, bool kRev>
la_status launch_simt(const void *q, const void *k, const void *v, void *o, const int32_t *cu, int nseq, int N,
                      int64_t T, int H, int D, const float *s0, float *sN, const float *slopes, cudaStream_t st) {
    const long long pairs = static_cast<long long>(nseq) * H;
    int split = 1;
    while (split < D / 32 && pairs * split * 2 <= 2 * kSmCount) split *= 2;
    la_status r;
    if (D == 64) {
        r = split == 1 ? launch_simt_cols<Tin, Tout, kRev, 64, 64>(q, k, v, o, cu, nseq, N, T, H, s0, sN, slopes, st)
                       : launch_simt_cols<Tin, Tout, kRev, 64, 32>(q, k, v, o, cu, nseq, N, T, H, s0, sN, slopes, st);
    } else {
        r = split == 1   ? launch_simt_cols<Tin, Tout, kRev, 128, 128>(q, k, v, o, cu, nseq, N, T, H, s0, sN, slopes, st)
            : split == 2 ? launch_simt_cols<Tin, Tout, kRev, 128, 64>(q, k, v, o, cu, nseq, N, T, H, s0, sN, slopes, st)
                         : launch_simt_cols<Tin, Tout, kRev, 128, 32>(q, k, v, o, cu, nseq, N, T, H, s0, sN, slopes, st);
    }
    if (r != LA_OK) return r;
    t_last_launches = 1;
    return check_launch("la_simt_prefill_kernel launch");
}

// Output group RMSNorm + sigmoid gate: its operands (fused into the decode kernel's store; a streaming
// pass after the prefill).
struct NormGate {
    const void *gate;     // like q, in the input type
    const float *weight;  // [H, D] fp32
    float eps;
};

la_status check_norm_gate(const NormGate *ng, const void *o, size_t o_bytes, size_t in_bytes_total) {
    if (!ng) return LA_OK;
    if (!ng->gate || !ng->weight) return fail(LA_ERR_INVALID_ARGUMENT, "gate and norm_weight must be non-null");
    if (!aligned(ng->gate, 16) || !aligned(ng->weight, 16))
        return fail(LA_ERR_INVALID_ARGUMENT, "gate and norm_weight must be 16-byte aligned");
    if (!(ng->eps >= 0.f) || !std::isfinite(ng->eps)) return fail(LA_ERR_INVALID_ARGUMENT, "eps must be finite and >= 0");
    if (o_bytes && overlap(o, o_bytes, ng->gate, in_bytes_total))
        return fail(LA_ERR_INVALID_ARGUMENT, "o must not overlap the gate");
    return LA_OK;
}

template <typename Tin, typename Tout, int D, int kThreads>
void launch_decode_t(const void *q, const void *k, const void *v, void *o, float *state, unsigned blocks, int H,
                     int steps, const float *slopes, const NormGate *ng, cudaStream_t st) {
    if (ng) {
        const la::DecodeGate<Tin> g{static_cast<const Tin *>(ng->gate), ng->weight, ng->eps};
        la::la_decode_kernel<Tin, Tout, D, true, kThreads><<<blocks, kThreads, 0, st>>>(
            static_cast<const Tin *>(q), static_cast<const Tin *>(k), static_cast<const Tin *>(v),
            static_cast<Tout *>(o), state, H, steps, slopes, g);
    } else {
        // the plain decode splits each state's columns over two CTAs (D = 128)
        constexpr int kCols = D == 128 ? 64 : D;
        la::la_decode_kernel<Tin, Tout, D, false, kThreads, kCols><<<blocks * (D / kCols), kThreads, 0, st>>>(
            static_cast<const Tin *>(q), static_cast<const Tin *>(k), static_cast<const Tin *>(v),
            static_cast<Tout *>(o), state, H, steps, slopes, la::DecodeGate<Tin>{});
    }
}

// One shape for single steps and several tokens per launch, so that K tokens in one launch do exactly the
// arithmetic of K single steps (512 threads with half the rows each were measured no faster for K = 8).
template <typename Tin, typename Tout, int D>
void launch_decode(const void *q, const void *k, const void *v, void *o, float *state, unsigned blocks, int H,
                   int steps, const float *slopes, const NormGate *ng, cudaStream_t st) {
    launch_decode_t<Tin, Tout, D, la::kDecodeThreads>(q, k, v, o, state, blocks, H, steps, slopes, ng, st);
}

// Shared body of la_decode_step and la_decode_steps: `steps` consecutive tokens per sequence.
la_status decode_impl(const void *q, const void *k, const void *v, void *o, float *state, int B, int steps, int H,
                      int D, la_dtype dtype, const float *slopes, la_stream_t stream, const NormGate *ng = nullptr) {
    t_last_launches = 0;
    if (B < 1) return fail(LA_ERR_INVALID_ARGUMENT, "B=%d must be >= 1", B);
    if (steps < 0) return fail(LA_ERR_INVALID_ARGUMENT, "steps=%d must be >= 0", steps);
    if (!state) return fail(LA_ERR_INVALID_ARGUMENT, "state must be non-null");
    if (steps == 0) return LA_OK;
    la_status r = check_common(q, k, v, o, static_cast<int64_t>(B) * steps, H, D, dtype, state, nullptr);
    if (r != LA_OK) return r;
    {
        const size_t n = static_cast<size_t>(B) * steps * H * D;
        if ((r = check_norm_gate(ng, o, n * out_bytes(dtype), n * in_bytes(dtype))) != LA_OK) return r;
    }
    const size_t sbytes = static_cast<size_t>(B) * H * D * D * 4;
    const size_t n = static_cast<size_t>(B) * steps * H * D;
    const size_t ib = n * in_bytes(dtype), ob = n * out_bytes(dtype);
    if (overlap(state, sbytes, o, ob) || overlap(state, sbytes, q, ib) || overlap(state, sbytes, k, ib) ||
        overlap(state, sbytes, v, ib))
        return fail(LA_ERR_INVALID_ARGUMENT, "state must not overlap q, k, v or o");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const unsigned blocks = static_cast<unsigned>(B) * static_cast<unsigned>(H);
    trace_pre("la_decode_kernel", st);
    if (dtype == LA_BF16) {
        if (D == 128) launch_decode<__nv_bfloat16, __nv_bfloat16, 128>(q, k, v, o, state, blocks, H, steps, slopes, ng, st);
        else launch_decode<__nv_bfloat16, __nv_bfloat16, 64>(q, k, v, o, state, blocks, H, steps, slopes, ng, st);
    } else if (dtype == LA_BF16_F32OUT) {
        if (D == 128) launch_decode<__nv_bfloat16, float, 128>(q, k, v, o, state, blocks, H, steps, slopes, ng, st);
        else launch_decode<__nv_bfloat16, float, 64>(q, k, v, o, state, blocks, H, steps, slopes, ng, st);
    } else if (dtype == LA_BF16_F16OUT) {
        if (D == 128) launch_decode<__nv_bfloat16, __half, 128>(q, k, v, o, state, blocks, H, steps, slopes, ng, st);
        else launch_decode<__nv_bfloat16, __half, 64>(q, k, v, o, state, blocks, H, steps, slopes, ng, st);
    } else {
        if (D == 128) launch_decode<float, float, 128>(q, k, v, o, state, blocks, H, steps, slopes, ng, st);
        else launch_decode<float, float, 64>(q, k, v, o, state, blocks, H, steps, slopes, ng, st);
    }
    trace_post(st);
    r = check_launch("la_decode_kernel launch");
    if (r == LA_OK) t_last_launches = 1;
    return r;
}

// The chunk kernel instance for an output type, direction and head dimension.
template <typename OutT>
auto chunk_kernel(bool reverse, int D) {
    if (D == 64) return reverse ? la::la_chunk_tc_kernel<OutT, true, true> : la::la_chunk_tc_kernel<OutT, false, true>;
    return reverse ? la::la_chunk_tc_kernel<OutT, true, false> : la::la_chunk_tc_kernel<OutT, false, false>;
}

template <bool kRev>
la_status launch_simt_dt(const void *q, const void *k, const void *v, void *o, const int32_t *cu, int nseq, int N,
                         int64_t T, int H, int D, la_dtype dt, const float *s0, float *sN, const float *slopes,
                         cudaStream_t st) {
    if (dt == LA_FP32) return launch_simt<float, float, kRev>(q, k, v, o, cu, nseq, N, T, H, D, s0, sN, slopes, st);
    if (dt == LA_BF16_F32OUT)
        return launch_simt<__nv_bfloat16, float, kRev>(q, k, v, o, cu, nseq, N, T, H, D, s0, sN, slopes, st);
    if (dt == LA_BF16_F16OUT)
        return launch_simt<__nv_bfloat16, __half, kRev>(q, k, v, o, cu, nseq, N, T, H, D, s0, sN, slopes, st);
    return launch_simt<__nv_bfloat16, __nv_bfloat16, kRev>(q, k, v, o, cu, nseq, N, T, H, D, s0, sN, slopes, st);
}

// The output correction of a corrected split, launched with the entry-state grid's configuration.
template <typename OutT>
la_status launch_correct(cudaLaunchConfig_t cfg, const CUtensorMap &tq, const CUtensorMap &to, const la::CorrArgs &ca) {
    auto kc = ca.D == 64 ? la::la_correct_tc_kernel<OutT, true> : la::la_correct_tc_kernel<OutT, false>;
    la_status r;
    if ((r = set_smem(kc, la::CorrCfg<OutT>::kSmemBytes)) != LA_OK) return r;
    trace_pre("la_correct_tc_kernel", cfg.stream);
    cfg.gridDim = dim3(static_cast<unsigned>(ca.items), ca.H);
    cfg.blockDim = dim3(la::kCorrThreads);
    cfg.dynamicSmemBytes = la::CorrCfg<OutT>::kSmemBytes;
    cudaLaunchKernelEx(&cfg, kc, tq, to, ca);
    trace_post(cfg.stream);
    return check_launch("la_correct_tc_kernel launch");
}

// Shared body of la_prefill and la_prefill_varlen (and of the three sweeps of the backward
// pass): sequences are either given by a device cu_seqlens or are nseq runs of N_uniform
// tokens; `reverse` runs the recurrence backwards in time (the kernels' kRev form).
la_status prefill_impl(const void *q, const void *k, const void *v, void *o, const int32_t *cu, int nseq, int N_uniform,
                       int64_t T, int H, int D, la_dtype dt, const float *s0, float *sN, const float *slopes,
                       void *ws, size_t ws_bytes, cudaStream_t st, bool reverse = false, int concurrency = 1) {
    t_last_launches = 0;
    la_status r = check_common(q, k, v, o, T, H, D, dt, s0, sN);
    if (r != LA_OK) return r;
    if (nseq < 1) return fail(LA_ERR_INVALID_ARGUMENT, "need at least one sequence (got %d)", nseq);
    if (nseq > 65535 * 64) return fail(LA_ERR_UNSUPPORTED, "nseq=%d too large", nseq);
    const Plan p = make_plan(T, nseq, N_uniform, H, D, dt, reverse, concurrency);
    if (p.bytes > 0) {
        if (!ws) return fail(LA_ERR_WORKSPACE, "workspace of %zu bytes required, got NULL", p.bytes);
        if (ws_bytes < p.bytes) return fail(LA_ERR_WORKSPACE, "workspace of %zu bytes required, got %zu", p.bytes, ws_bytes);
        if (!aligned(ws, 256)) return fail(LA_ERR_INVALID_ARGUMENT, "workspace is not 256-byte aligned");
    }
    if (!p.tensor_core) {
        if (nseq > 65535) return fail(LA_ERR_UNSUPPORTED, "nseq=%d > 65535 on the CUDA-core path", nseq);
        return reverse ? launch_simt_dt<true>(q, k, v, o, cu, nseq, N_uniform, T, H, D, dt, s0, sN, slopes, st)
                       : launch_simt_dt<false>(q, k, v, o, cu, nseq, N_uniform, T, H, D, dt, s0, sN, slopes, st);
    }

    CUtensorMap tq, tk, tv, to;
    if ((r = make_map(&tq, q, T, H, D, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)) != LA_OK) return r;
    if ((r = make_map(&tk, k, T, H, D, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)) != LA_OK) return r;
    if ((r = make_map(&tv, v, T, H, D, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)) != LA_OK) return r;
    if (dt == LA_BF16_F32OUT)
        r = make_map(&to, o, T, H, D, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, la::OutStaging<float>::kRows);
    else if (dt == LA_BF16_F16OUT)
        r = make_map(&to, o, T, H, D, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, la::OutStaging<__half>::kRows);
    else
        r = make_map(&to, o, T, H, D, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, la::OutStaging<__nv_bfloat16>::kRows);
    if (r != LA_OK) return r;

    uint8_t *w = static_cast<uint8_t *>(ws);
    la::WorkMap map{};
    map.nseq = nseq;
    map.sub_len = p.sub_len;
    map.R = p.R;
    int launches = 0;
    if (p.planned) {
        int4 *fine = reinterpret_cast<int4 *>(w + p.off_fine);
        int4 *coarse = reinterpret_cast<int4 *>(w + p.off_coarse);
        int *seq_fine = reinterpret_cast<int *>(w + p.off_seq_fine);
        int *seq_coarse = reinterpret_cast<int *>(w + p.off_seq_coarse);
        int *counts = reinterpret_cast<int *>(w + p.off_counts);
        trace_pre("la_plan_kernel", st);
        la::la_plan_kernel<<<1, la::kPlanThreads, 0, st>>>(cu, nseq, static_cast<int>(T), p.sub_len, p.R, p.cap_fine,
                                                            p.cap_coarse, fine, coarse, seq_fine, seq_coarse, counts);
        trace_post(st);
        ++launches;
        if ((r = check_launch("la_plan_kernel launch")) != LA_OK) return r;
        map.fine = fine;
        map.coarse = coarse;
        map.seq_fine = seq_fine;
        map.seq_coarse = seq_coarse;
        map.counts = counts;
    } else {
        map.N = N_uniform;
        map.nf = p.nf;
        map.nc = p.nc;
    }

    la::ChunkArgs a;
    a.o = o;
    a.s_init = s0;
    a.s_final = sN;
    a.slopes = slopes;
    a.map = map;
    a.seg_state = p.segmented ? reinterpret_cast<float *>(w + p.off_state) : nullptr;
    a.s0_copy = p.segmented && !p.corrected ? reinterpret_cast<float *>(w + p.off_s0) : nullptr;
    a.H = H;
    a.D = D;
    a.seg_ld = la::kD;
    a.corrected = p.corrected ? 1 : 0;

    if (p.segmented && !p.corrected) {
        auto ks = reverse ? la::la_state_tc_kernel<true> : la::la_state_tc_kernel<false>;
        if ((r = set_smem(ks, la::StateCfg::kSmemBytes)) != LA_OK) return r;
        trace_pre("la_state_tc_kernel", st);
        ks<<<dim3(p.cap_fine, H), la::kStateThreads, la::StateCfg::kSmemBytes, st>>>(tk, tv, a);
        trace_post(st);
        ++launches;
        if ((r = check_launch("la_state_tc_kernel launch")) != LA_OK) return r;
    }
    auto km = dt == LA_BF16          ? chunk_kernel<__nv_bfloat16>(reverse, D)
              : dt == LA_BF16_F16OUT ? chunk_kernel<__half>(reverse, D)
                                     : chunk_kernel<float>(reverse, D);
    if ((r = set_smem(km, la::ChunkCfg::kSmemBytes)) != LA_OK) return r;
    trace_pre("la_chunk_tc_kernel", st);
    {
        // after a segment-state pass: programmatic dependent launch, so the first segments start on
        // the SMs that pass leaves free (the CTAs that read its output wait for it on the device)
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(p.cap_coarse, H);
        cfg.blockDim = dim3(la::kTcThreads);
        cfg.dynamicSmemBytes = la::ChunkCfg::kSmemBytes;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = p.segmented && !p.corrected && plan_override("LA_NO_PDL") <= 0 ? 1 : 0;
        cudaLaunchKernelEx(&cfg, km, tq, tk, tv, to, a);
    }
    trace_post(st);
    ++launches;
    if ((r = check_launch("la_chunk_tc_kernel launch")) != LA_OK) return r;
    if (p.corrected) {
        la::CorrArgs ca;
        ca.o = o;
        ca.s_final = sN;
        ca.slopes = slopes;
        ca.map = map;
        ca.seg_state = a.seg_state;
        ca.e_img = p.corr_direct ? nullptr : w + p.off_eimg;
        ca.H = H;
        ca.D = D;
        ca.units = p.cap_coarse;
        ca.chunks = p.corr_chunks;
        ca.pieces = p.corr_pieces;
        ca.items = p.corr_items;
        // programmatic dependent launches: each grid is scheduled onto the SMs the previous one leaves (or
        // never used) and waits on the device for what it reads
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.stream = st;
        cfg.attrs = attr;
        cfg.numAttrs = plan_override("LA_NO_PDL") <= 0 ? 1 : 0;
        if (!p.corr_direct) {
            trace_pre("la_entry_state_kernel", st);
            cfg.gridDim = dim3(static_cast<unsigned>(p.cap_coarse + nseq), H);
            cfg.blockDim = dim3(la::kEntryThreads);
            cfg.dynamicSmemBytes = 0;
            cudaLaunchKernelEx(&cfg, la::la_entry_state_kernel, ca);
            trace_post(st);
            ++launches;
            if ((r = check_launch("la_entry_state_kernel launch")) != LA_OK) return r;
        }
        if (p.corr_items > 0) {
            la_status rc;
            if (dt == LA_BF16_F16OUT) rc = launch_correct<__half>(cfg, tq, to, ca);
            else rc = launch_correct<float>(cfg, tq, to, ca);
            if (rc != LA_OK) return rc;
            ++launches;
        }
    }
    t_last_launches = launches;
    return LA_OK;
}

// ---------------------------------------------------------------- output norm + gate
// One wave of resident blocks (grid-stride loop inside), never more blocks than there are rows for.
template <typename K>
unsigned resident_grid(K kernel, int threads, long long blocks_needed) {
    int dev = 0, sms = kSmCount, per_sm = 1;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0);
    const long long cap = static_cast<long long>(std::max(1, sms)) * std::max(1, per_sm);
    return static_cast<unsigned>(std::max<long long>(1, std::min(blocks_needed, cap)));
}

template <typename Tout, typename Tg, int D>
void launch_norm_gate_d(const void *o, const void *gate, const float *w, float eps, void *y, long long rows, int H,
                        cudaStream_t st) {
    auto kern = la::la_norm_gate_kernel<Tout, Tg, D>;
    // rows per block and grid-stride iteration: 8 warps x (32 / (D / 8)) rows x kNormGateSteps
    const long long rows_per_block = (la::kNormGateThreads / 32) * (32 / (D / 8)) * la::kNormGateSteps;
    const unsigned grid = resident_grid(kern, la::kNormGateThreads, (rows + rows_per_block - 1) / rows_per_block);
    kern<<<grid, la::kNormGateThreads, 0, st>>>(static_cast<const Tout *>(o), static_cast<const Tg *>(gate), w, eps,
                                               static_cast<Tout *>(y), static_cast<int>(rows), H);
}

template <typename Tout, typename Tg>
void launch_norm_gate_t(const void *o, const void *gate, const float *w, float eps, void *y, long long rows, int H, int D,
                        cudaStream_t st) {
    if (D == 128) launch_norm_gate_d<Tout, Tg, 128>(o, gate, w, eps, y, rows, H, st);
    else launch_norm_gate_d<Tout, Tg, 64>(o, gate, w, eps, y, rows, H, st);
}

// y = w * o / sqrt(mean(o^2) + eps) * sigmoid(gate) over T * H rows of D (y may be o); o and y in the output
// type of dt, the gate in its input type. Arguments are checked by the caller.
la_status launch_norm_gate(const void *o, const NormGate &ng, void *y, int64_t T, int H, int D, la_dtype dt,
                           cudaStream_t st) {
    const long long rows = static_cast<long long>(T) * H;
    if (rows == 0) return LA_OK;
    trace_pre("la_norm_gate_kernel", st);
    if (dt == LA_BF16) launch_norm_gate_t<__nv_bfloat16, __nv_bfloat16>(o, ng.gate, ng.weight, ng.eps, y, rows, H, D, st);
    else if (dt == LA_BF16_F16OUT) launch_norm_gate_t<__half, __nv_bfloat16>(o, ng.gate, ng.weight, ng.eps, y, rows, H, D, st);
    else if (dt == LA_BF16_F32OUT) launch_norm_gate_t<float, __nv_bfloat16>(o, ng.gate, ng.weight, ng.eps, y, rows, H, D, st);
    else launch_norm_gate_t<float, float>(o, ng.gate, ng.weight, ng.eps, y, rows, H, D, st);
    trace_post(st);
    return check_launch("la_norm_gate_kernel launch");
}

// la_prefill / la_prefill_varlen, then the output norm + gate in place on o.
la_status prefill_norm_gate_impl(const void *q, const void *k, const void *v, const NormGate &ng, void *o,
                                 const int32_t *cu, int nseq, int N_uniform, int64_t T, int H, int D, la_dtype dt,
                                 const float *s0, float *sN, const float *slopes, void *ws, size_t ws_bytes,
                                 cudaStream_t st) {
    t_last_launches = 0;
    la_status r = check_common(q, k, v, o, T, H, D, dt, s0, sN);
    if (r != LA_OK) return r;
    const size_t n = static_cast<size_t>(T) * H * D;
    if ((r = check_norm_gate(&ng, o, n * out_bytes(dt), n * in_bytes(dt))) != LA_OK) return r;
    if ((r = prefill_impl(q, k, v, o, cu, nseq, N_uniform, T, H, D, dt, s0, sN, slopes, ws, ws_bytes, st)) != LA_OK)
        return r;
    const int launches = t_last_launches;
    if ((r = launch_norm_gate(o, ng, o, T, H, D, dt, st)) != LA_OK) return r;
    t_last_launches = launches + (T > 0 ? 1 : 0);
    return LA_OK;
}

// ---------------------------------------------------------------- backward pass
// Workspace: the transposed initial state and d_final_state (one [nseq, H, D, D] fp32 slot each),
// then the workspace the sweeps share (they run one after another on the stream).
// The sweeps share the GPU (the caller's stream and two side streams), each with its own workspace slot.
// Usually all three run at once, each planned for a third of the GPU. A uniform batch whose (sequence,
// head) pairs P fill the GPU with two unsegmented sweeps but not with three (2P <= SMs < 3P) would run
// its third sweep as a second, mostly empty wave; there the dv sweep runs first on its own, with the
// whole GPU's plan, and the dq and dk sweeps then share the GPU unsegmented (B=4, N=4096, H=16 on B200:
// 240 -> 223 us). Other orders measured no better on other shapes (varlen, fewer or more pairs).
constexpr int kBwdSweeps = 3;
bool bwd_dv_first(int nseq, int N_uniform, int H) {
    const long long pairs = static_cast<long long>(nseq) * H;
    return N_uniform > 0 && 2 * pairs <= kSmCount && 3 * pairs > kSmCount;
}
struct BwdPlan {
    size_t off_s0t = 0, off_dsnt = 0, off_sweep[3] = {0, 0, 0}, bytes = 0, sweep_bytes = 0;
};

BwdPlan make_bwd_plan(int64_t T, int nseq, int N_uniform, int H, int D, la_dtype dt) {
    BwdPlan b;
    const size_t sb = align_up(sizeof(float) * static_cast<size_t>(nseq) * H * D * D, 256);
    b.off_s0t = 0;
    b.off_dsnt = sb;
    size_t sweep = 0;
    if (bwd_dv_first(nseq, N_uniform, H)) {
        sweep = std::max({make_plan(T, nseq, N_uniform, H, D, dt, true, 1).bytes,
                          make_plan(T, nseq, N_uniform, H, D, dt, false, 2).bytes,
                          make_plan(T, nseq, N_uniform, H, D, dt, true, 2).bytes});
    } else {
        sweep = std::max(make_plan(T, nseq, N_uniform, H, D, dt, false, kBwdSweeps).bytes,
                         make_plan(T, nseq, N_uniform, H, D, dt, true, kBwdSweeps).bytes);
    }
    b.sweep_bytes = align_up(sweep, 256);
    for (int i = 0; i < 3; ++i) b.off_sweep[i] = 2 * sb + i * b.sweep_bytes;
    b.bytes = 2 * sb + 3 * b.sweep_bytes;
    return b;
}

// Two side streams and the events that fork them from and join them back into a caller's stream, per
// thread and device (so that concurrent calls never share them). A fork-join through events also works
// while the caller's stream is being captured into a CUDA graph.
struct SideStreams {
    cudaStream_t s[2] = {nullptr, nullptr};
    cudaEvent_t fork = nullptr, join[2] = {nullptr, nullptr};
    bool ok = false;
};

SideStreams &side_streams() {
    thread_local std::map<int, SideStreams> cache;
    int dev = 0;
    cudaGetDevice(&dev);
    SideStreams &ss = cache[dev];
    if (!ss.ok) {
        bool good = true;
        for (int i = 0; i < 2; ++i) {
            good = good && cudaStreamCreateWithFlags(&ss.s[i], cudaStreamNonBlocking) == cudaSuccess;
            good = good && cudaEventCreateWithFlags(&ss.join[i], cudaEventDisableTiming) == cudaSuccess;
        }
        good = good && cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) == cudaSuccess;
        ss.ok = good;
    }
    return ss;
}

la_status launch_transpose(const float *src, float *dst, int count, int D, cudaStream_t st) {
    trace_pre("la_transpose_states_kernel", st);
    la::la_transpose_states_kernel<<<dim3(D / la::kTransposeTile, D / la::kTransposeTile, count), dim3(32, 8), 0, st>>>(
        src, dst, D);
    trace_post(st);
    return check_launch("la_transpose_states_kernel launch");
}

// Shared body of la_prefill_backward and la_prefill_varlen_backward: the state transposes, then
// the dq sweep (forward in time) and the dk and dv sweeps (backward in time) as prefill runs.
la_status backward_impl(const void *q, const void *k, const void *v, const void *dout, void *dq, void *dk, void *dv,
                        const int32_t *cu, int nseq, int N_uniform, int64_t T, int H, int D, la_dtype dt,
                        const float *s0, const float *dsN, float *ds0, const float *slopes, void *ws, size_t ws_bytes,
                        cudaStream_t st) {
    t_last_launches = 0;
    la_status r = check_common(q, k, v, dq, T, H, D, dt, s0, dsN);
    if (r != LA_OK) return r;
    if (nseq < 1) return fail(LA_ERR_INVALID_ARGUMENT, "need at least one sequence (got %d)", nseq);
    if (T > 0 && (!dout || !dk || !dv)) return fail(LA_ERR_INVALID_ARGUMENT, "dout, dk and dv must be non-null");
    const void *ptrs[4] = {dout, dk, dv, ds0};
    const char *names[4] = {"dout", "dk", "dv", "d_initial_state"};
    for (int i = 0; i < 4; ++i)
        if (ptrs[i] && !aligned(ptrs[i], 16)) return fail(LA_ERR_INVALID_ARGUMENT, "%s is not 16-byte aligned", names[i]);
    const size_t ib = static_cast<size_t>(T) * H * D * in_bytes(dt), ob = static_cast<size_t>(T) * H * D * out_bytes(dt);
    if (ob) {
        const void *ins[4] = {q, k, v, dout};
        void *outs[3] = {dq, dk, dv};
        for (int a = 0; a < 3; ++a) {
            for (int b = 0; b < 4; ++b)
                if (overlap(outs[a], ob, ins[b], ib))
                    return fail(LA_ERR_INVALID_ARGUMENT, "dq, dk and dv must not overlap q, k, v or dout");
            for (int b = a + 1; b < 3; ++b)
                if (overlap(outs[a], ob, outs[b], ob)) return fail(LA_ERR_INVALID_ARGUMENT, "dq, dk and dv must not overlap");
        }
    }
    const BwdPlan bp = make_bwd_plan(T, nseq, N_uniform, H, D, dt);
    if (!ws) return fail(LA_ERR_WORKSPACE, "workspace of %zu bytes required, got NULL", bp.bytes);
    if (ws_bytes < bp.bytes) return fail(LA_ERR_WORKSPACE, "workspace of %zu bytes required, got %zu", bp.bytes, ws_bytes);
    if (!aligned(ws, 256)) return fail(LA_ERR_INVALID_ARGUMENT, "workspace is not 256-byte aligned");
    uint8_t *w = static_cast<uint8_t *>(ws);
    float *s0t = s0 ? reinterpret_cast<float *>(w + bp.off_s0t) : nullptr;
    float *dsnt = dsN ? reinterpret_cast<float *>(w + bp.off_dsnt) : nullptr;
    void *sweep_ws[3];
    for (int i = 0; i < 3; ++i) sweep_ws[i] = bp.sweep_bytes ? w + bp.off_sweep[i] : nullptr;
    SideStreams &side = side_streams();
    if (!side.ok) return fail(LA_ERR_CUDA, "could not create the backward pass's side streams");
    int launches = 0;
    // both transposes read their inputs before any sweep writes d_initial_state (which may alias either)
    if (s0) {
        if ((r = launch_transpose(s0, s0t, nseq * H, D, st)) != LA_OK) return r;
        ++launches;
    }
    if (dsN) {
        if ((r = launch_transpose(dsN, dsnt, nseq * H, D, st)) != LA_OK) return r;
        ++launches;
    }
    // The three sweeps are independent: dq on side stream 0, dk on side stream 1, dv on the caller's stream.
    // The side streams start after whatever precedes them on the caller's stream (the transposes, and the dv
    // sweep when it runs first), and the caller's stream waits for both before anything it enqueues next.
    la_status rs[3] = {LA_OK, LA_OK, LA_OK};
    int sweep_launches = 0;
    const bool dv_first = bwd_dv_first(nseq, N_uniform, H);
    // dv = backward(q <- k, k <- q, v <- dO, dS_N), whose final state is dS_0
    auto sweep_dv = [&](int concurrency) {
        rs[2] = prefill_impl(k, q, dout, dv, cu, nseq, N_uniform, T, H, D, dt, dsN, ds0, slopes, sweep_ws[2],
                             bp.sweep_bytes, st, true, concurrency);
        sweep_launches += rs[2] == LA_OK ? t_last_launches : 0;
    };
    if (dv_first) sweep_dv(1);
    cudaError_t ce = cudaEventRecord(side.fork, st);
    for (int i = 0; i < 2 && ce == cudaSuccess; ++i) ce = cudaStreamWaitEvent(side.s[i], side.fork, 0);
    if (ce != cudaSuccess) return cuda_fail(ce, "forking the backward pass's sweeps");
    const int conc = dv_first ? 2 : kBwdSweeps;
    // dq = forward(q <- dO, k <- v, v <- k, S0^T)
    rs[0] = prefill_impl(dout, v, k, dq, cu, nseq, N_uniform, T, H, D, dt, s0t, nullptr, slopes, sweep_ws[0],
                         bp.sweep_bytes, side.s[0], false, conc);
    sweep_launches += rs[0] == LA_OK ? t_last_launches : 0;
    // dk = backward(q <- v, k <- dO, v <- q, dS_N^T)
    rs[1] = prefill_impl(v, dout, q, dk, cu, nseq, N_uniform, T, H, D, dt, dsnt, nullptr, slopes, sweep_ws[1],
                         bp.sweep_bytes, side.s[1], true, conc);
    sweep_launches += rs[1] == LA_OK ? t_last_launches : 0;
    if (!dv_first) sweep_dv(kBwdSweeps);
    // join whatever was enqueued, also after a failure, so that the caller's stream orders after it
    for (int i = 0; i < 2; ++i) {
        cudaError_t je = cudaEventRecord(side.join[i], side.s[i]);
        if (je == cudaSuccess) je = cudaStreamWaitEvent(st, side.join[i], 0);
        if (je != cudaSuccess && ce == cudaSuccess) ce = je;
    }
    for (int i = 0; i < 3; ++i)
        if (rs[i] != LA_OK) return rs[i];
    if (ce != cudaSuccess) return cuda_fail(ce, "joining the backward pass's sweeps");
    t_last_launches = launches + sweep_launches;
    return LA_OK;
}

// Fine units of a shard for its state pass: enough (sequence, head, unit) CTAs to fill the GPU.
struct ShardPlan {
    int units = 1;   // U
    int len = 0;     // tokens per unit (a multiple of the chunk), the last one may be shorter
};

ShardPlan make_shard_plan(int B, int N, int H) {
    ShardPlan sp;
    const int chunks = std::max(1, round_chunks(N));
    const int want = std::max(1, std::min(chunks, kSmCount / std::max(1, B * H)));
    const int unit_chunks = (chunks + want - 1) / want;
    sp.len = unit_chunks * la::kC;
    sp.units = std::max(1, (N + sp.len - 1) / sp.len);
    return sp;
}

la_status launch_combine(const float *src, int u, long long stride_u, long long stride_b, int B, int H, int D, int L,
                         int last_len, const float *slopes, const float *s0, float *out, cudaStream_t st) {
    const int DD = D * D;
    dim3 grid(std::max(1, DD / 4 / la::kCombineThreads), B * H);
    trace_pre("la_combine_states_kernel", st);
    la::la_combine_states_kernel<<<grid, la::kCombineThreads, 0, st>>>(src, u, stride_u, stride_b, H, DD, L, last_len,
                                                                      slopes, s0, out);
    trace_post(st);
    return check_launch("la_combine_states_kernel launch");
}

la_status launch_combine_rev(const float *src, int n, long long stride_u, long long stride_b, int B, int H, int D, int L,
                             const float *slopes, const float *s_end, float end_exp, float *out, cudaStream_t st) {
    const int DD = D * D;
    dim3 grid(std::max(1, DD / 4 / la::kCombineThreads), B * H);
    trace_pre("la_combine_states_rev_kernel", st);
    la::la_combine_states_rev_kernel<<<grid, la::kCombineThreads, 0, st>>>(src, n, stride_u, stride_b, H, DD, L, slopes,
                                                                          s_end, end_exp, out);
    trace_post(st);
    return check_launch("la_combine_states_rev_kernel launch");
}

// Shared body of la_shard_state and la_shard_state_reverse: the state pass over a shard's fine units (k, v
// in the kernel's roles), then their combination: from the shard's end (forward: weights
// lambda^(L-1-s) of the shard's length) or from its start (reverse: weights lambda^(s+1)).
la_status shard_state_impl(const void *k, const void *v, int B, int N, int H, int D, la_dtype dtype, const float *slopes,
                           float *delta_state, void *workspace, size_t workspace_bytes, la_stream_t stream, bool reverse) {
    t_last_launches = 0;
    if (!valid_dtype(dtype)) return fail(LA_ERR_INVALID_ARGUMENT, "dtype %d is not a la_dtype", dtype);
    if (dtype == LA_FP32) return fail(LA_ERR_UNSUPPORTED, "shard states run on the tensor cores: bf16 inputs only");
    if (D != 64 && D != 128) return fail(LA_ERR_UNSUPPORTED, "head dim D=%d: only 64 and 128 are supported", D);
    if (B < 1 || N < 0 || H < 1 || H > 65535)
        return fail(LA_ERR_INVALID_ARGUMENT, "B=%d >= 1, N=%d >= 0 and H=%d in [1, 65535] required", B, N, H);
    const int64_t T = static_cast<int64_t>(B) * N;
    if (T * H * D >= (int64_t(1) << 31))
        return fail(LA_ERR_UNSUPPORTED, "B*N*H*D = %lld elements must be < 2^31", static_cast<long long>(T * H * D));
    if (!delta_state || !aligned(delta_state, 16))
        return fail(LA_ERR_INVALID_ARGUMENT, "delta_state must be a non-null 16-byte aligned pointer");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t state_bytes = sizeof(float) * static_cast<size_t>(B) * H * D * D;
    if (N == 0) {
        cudaError_t e = cudaMemsetAsync(delta_state, 0, state_bytes, st);
        return e == cudaSuccess ? LA_OK : cuda_fail(e, "cudaMemsetAsync");
    }
    if (!k || !v || !aligned(k, 16) || !aligned(v, 16))
        return fail(LA_ERR_INVALID_ARGUMENT, "the two inputs must be non-null 16-byte aligned pointers");
    const ShardPlan sp = make_shard_plan(B, N, H);
    const size_t need = sp.units > 1 ? sizeof(float) * static_cast<size_t>(sp.units) * B * H * D * D : 0;
    if (need > 0) {
        if (!workspace || workspace_bytes < need)
            return fail(LA_ERR_WORKSPACE, "workspace of %zu bytes needed (la_shard_state_workspace_size)", need);
        if (!aligned(workspace, 256)) return fail(LA_ERR_INVALID_ARGUMENT, "workspace must be 256-byte aligned");
    }
    la_status r;
    CUtensorMap tk, tv;
    if ((r = make_map(&tk, k, T, H, D, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)) != LA_OK) return r;
    if ((r = make_map(&tv, v, T, H, D, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)) != LA_OK) return r;
    // One sequence per batch row, cut into sp.units fine units, every one of which gets its state.
    la::WorkMap map{};
    map.N = N;
    map.nf = sp.units;
    map.nc = 2;
    map.nseq = B;
    map.sub_len = sp.len;
    map.R = sp.units;
    map.all_units = 1;
    la::ChunkArgs a{};
    a.map = map;
    a.slopes = slopes;
    a.H = H;
    a.seg_state = need > 0 ? static_cast<float *>(workspace) : delta_state;
    a.D = D;
    a.seg_ld = D;   // the unit states are the caller's (or combined into them): [., H, D, D]
    auto ks = reverse ? la::la_state_tc_kernel<true> : la::la_state_tc_kernel<false>;
    if ((r = set_smem(ks, la::StateCfg::kSmemBytes)) != LA_OK) return r;
    trace_pre("la_state_tc_kernel", st);
    ks<<<dim3(B * sp.units, H), la::kStateThreads, la::StateCfg::kSmemBytes, st>>>(tk, tv, a);
    trace_post(st);
    int launches = 1;
    if ((r = check_launch("la_state_tc_kernel launch")) != LA_OK) return r;
    if (need > 0) {
        // units of sequence b are slots b * U + f of the workspace: [B, U, H, D, D]
        const float *ws = static_cast<const float *>(workspace);
        r = reverse ? launch_combine_rev(ws, sp.units, H, static_cast<long long>(sp.units) * H, B, H, D, sp.len, slopes,
                                         nullptr, 0.f, delta_state, st)
                    : launch_combine(ws, sp.units, H, static_cast<long long>(sp.units) * H, B, H, D, sp.len,
                                     N - (sp.units - 1) * sp.len, slopes, nullptr, delta_state, st);
        if (r != LA_OK) return r;
        ++launches;
    }
    t_last_launches = launches;
    return LA_OK;
}

// Shard `rank` of R equal shards [rank L, (rank+1) L) of a packed batch, from the host copy of its
// cu_seqlens (checked here: cu[0] = 0, non-decreasing, T = cu[nseq] > 0 divisible by R).
struct VarlenShard {
    int64_t T = 0, L = 0, s = 0, e = 0;
};

la_status varlen_shard(const int32_t *cu, int nseq, int R, int rank, VarlenShard &sh) {
    if (!cu) return fail(LA_ERR_INVALID_ARGUMENT, "cu_seqlens (a host array) must be non-null");
    if (nseq < 1) return fail(LA_ERR_INVALID_ARGUMENT, "need at least one sequence (got %d)", nseq);
    if (R < 1 || rank < 0 || rank >= R) return fail(LA_ERR_INVALID_ARGUMENT, "rank=%d must be in [0, R=%d)", rank, R);
    if (R > la::kMaxCombineTerms)
        return fail(LA_ERR_UNSUPPORTED, "R=%d ranks: at most %d are supported", R, la::kMaxCombineTerms);
    if (cu[0] != 0) return fail(LA_ERR_INVALID_ARGUMENT, "cu_seqlens[0]=%d must be 0", cu[0]);
    for (int i = 0; i < nseq; ++i)
        if (cu[i + 1] < cu[i]) return fail(LA_ERR_INVALID_ARGUMENT, "cu_seqlens decreases at %d", i + 1);
    sh.T = cu[nseq];
    if (sh.T <= 0 || sh.T % R != 0)
        return fail(LA_ERR_INVALID_ARGUMENT, "T=%lld tokens must be > 0 and divisible by R=%d", static_cast<long long>(sh.T),
                    R);
    sh.L = sh.T / R;
    sh.s = rank * sh.L;
    sh.e = sh.s + sh.L;
    return LA_OK;
}

// Index of the (non-empty) sequence that holds token t < T: cu[i] <= t < cu[i+1].
int seq_holding(const int32_t *cu, int nseq, int64_t t) {
    return static_cast<int>(std::upper_bound(cu, cu + nseq + 1, static_cast<int32_t>(t)) - cu) - 1;
}

la_status launch_combine_terms(const float *src, long long stride, const la::CombineTerms &t, const float *s0, int H,
                               int D, const float *slopes, float *out, cudaStream_t st) {
    const int DD = D * D;
    dim3 grid(std::max(1, DD / 4 / la::kCombineThreads), H);
    trace_pre("la_combine_terms_kernel", st);
    la::la_combine_terms_kernel<<<grid, la::kCombineThreads, 0, st>>>(src, stride, t, s0, H, DD, slopes, out);
    trace_post(st);
    return check_launch("la_combine_terms_kernel launch");
}

la_status check_varlen_cp(const float *gathered, int R, const float *given, const float *out, int H, int D,
                          bool needs_gathered, int nseq, const char *given_name, const char *out_name) {
    if (H < 1 || H > 65535) return fail(LA_ERR_INVALID_ARGUMENT, "H=%d must be in [1, 65535]", H);
    if (D != 64 && D != 128) return fail(LA_ERR_UNSUPPORTED, "head dim D=%d: only 64 and 128 are supported", D);
    if (!out || !aligned(out, 16)) return fail(LA_ERR_INVALID_ARGUMENT, "%s must be non-null and 16-byte aligned", out_name);
    if (needs_gathered && (!gathered || !aligned(gathered, 16)))
        return fail(LA_ERR_INVALID_ARGUMENT, "gathered must be non-null and 16-byte aligned");
    if (given && !aligned(given, 16)) return fail(LA_ERR_INVALID_ARGUMENT, "%s must be 16-byte aligned", given_name);
    const size_t sz = sizeof(float) * static_cast<size_t>(H) * D * D;
    if (gathered && overlap(out, sz, gathered, sz * R))
        return fail(LA_ERR_INVALID_ARGUMENT, "%s must not overlap gathered", out_name);
    if (given && overlap(out, sz, given, sz * nseq))
        return fail(LA_ERR_INVALID_ARGUMENT, "%s must not overlap %s", out_name, given_name);
    return LA_OK;
}

}  // namespace

extern "C" {

size_t la_shard_state_workspace_size(int B, int N, int H, int D, la_dtype dtype) {
    if (B < 1 || N < 1 || H < 1 || (D != 64 && D != 128) || dtype == LA_FP32 || !valid_dtype(dtype)) return 0;
    const ShardPlan sp = make_shard_plan(B, N, H);
    return sp.units > 1 ? sizeof(float) * static_cast<size_t>(sp.units) * B * H * D * D : 0;
}

la_status la_shard_state(const void *k, const void *v, int B, int N, int H, int D, la_dtype dtype,
                         const float *slopes, float *delta_state, void *workspace, size_t workspace_bytes,
                         la_stream_t stream) {
    return shard_state_impl(k, v, B, N, H, D, dtype, slopes, delta_state, workspace, workspace_bytes, stream, false);
}

la_status la_shard_state_reverse(const void *q, const void *dout, int B, int N, int H, int D, la_dtype dtype,
                                 const float *slopes, float *delta_state, void *workspace, size_t workspace_bytes,
                                 la_stream_t stream) {
    return shard_state_impl(q, dout, B, N, H, D, dtype, slopes, delta_state, workspace, workspace_bytes, stream, true);
}

la_status la_cp_entry_state(const float *gathered, int R, int rank, int B, int H, int D, int L,
                            const float *initial_state, const float *slopes, float *s_in, la_stream_t stream) {
    t_last_launches = 0;
    if (R < 1 || rank < 0 || rank >= R) return fail(LA_ERR_INVALID_ARGUMENT, "rank=%d must be in [0, R=%d)", rank, R);
    if (B < 1 || H < 1 || H > 65535 || L < 0)
        return fail(LA_ERR_INVALID_ARGUMENT, "B=%d >= 1, H=%d in [1, 65535] and L=%d >= 0 required", B, H, L);
    if (D != 64 && D != 128) return fail(LA_ERR_UNSUPPORTED, "head dim D=%d: only 64 and 128 are supported", D);
    if (!s_in || !aligned(s_in, 16)) return fail(LA_ERR_INVALID_ARGUMENT, "s_in must be non-null and 16-byte aligned");
    if (rank > 0 && (!gathered || !aligned(gathered, 16)))
        return fail(LA_ERR_INVALID_ARGUMENT, "gathered must be non-null and 16-byte aligned");
    if (initial_state && !aligned(initial_state, 16))
        return fail(LA_ERR_INVALID_ARGUMENT, "initial_state must be 16-byte aligned");
    const size_t sz = sizeof(float) * static_cast<size_t>(B) * H * D * D;
    if (gathered && overlap(s_in, sz, gathered, sz * R)) return fail(LA_ERR_INVALID_ARGUMENT, "s_in must not overlap gathered");
    la_status r = launch_combine(gathered, rank, static_cast<long long>(B) * H, H, B, H, D, L, L, slopes, initial_state,
                                 s_in, reinterpret_cast<cudaStream_t>(stream));
    if (r == LA_OK) t_last_launches = 1;
    return r;
}

la_status la_cp_reverse_entry_state(const float *gathered, int R, int rank, int B, int H, int D, int L,
                                    const float *d_final_state, const float *slopes, float *h_in, la_stream_t stream) {
    t_last_launches = 0;
    if (R < 1 || rank < 0 || rank >= R) return fail(LA_ERR_INVALID_ARGUMENT, "rank=%d must be in [0, R=%d)", rank, R);
    if (B < 1 || H < 1 || H > 65535 || L < 0)
        return fail(LA_ERR_INVALID_ARGUMENT, "B=%d >= 1, H=%d in [1, 65535] and L=%d >= 0 required", B, H, L);
    if (D != 64 && D != 128) return fail(LA_ERR_UNSUPPORTED, "head dim D=%d: only 64 and 128 are supported", D);
    if (!h_in || !aligned(h_in, 16)) return fail(LA_ERR_INVALID_ARGUMENT, "h_in must be non-null and 16-byte aligned");
    if (rank < R - 1 && (!gathered || !aligned(gathered, 16)))
        return fail(LA_ERR_INVALID_ARGUMENT, "gathered must be non-null and 16-byte aligned");
    if (d_final_state && !aligned(d_final_state, 16))
        return fail(LA_ERR_INVALID_ARGUMENT, "d_final_state must be 16-byte aligned");
    const size_t sz = sizeof(float) * static_cast<size_t>(B) * H * D * D;
    if (gathered && overlap(h_in, sz, gathered, sz * R)) return fail(LA_ERR_INVALID_ARGUMENT, "h_in must not overlap gathered");
    const long long stride_u = static_cast<long long>(B) * H;
    // the shards after this one, nearest first: shard rank + 1 + j begins j L tokens after this one ends
    const float *src = rank < R - 1 ? gathered + (rank + 1) * stride_u * D * D : nullptr;
    la_status r = launch_combine_rev(src, R - 1 - rank, stride_u, H, B, H, D, L, slopes, d_final_state,
                                     static_cast<float>(R - 1 - rank) * static_cast<float>(L), h_in,
                                     reinterpret_cast<cudaStream_t>(stream));
    if (r == LA_OK) t_last_launches = 1;
    return r;
}

la_status la_cp_varlen_entry_state(const float *gathered, int R, int rank, const int32_t *cu_seqlens, int nseq, int H,
                                   int D, const float *initial_state, const float *slopes, float *s_in,
                                   la_stream_t stream) {
    t_last_launches = 0;
    VarlenShard sh;
    la_status r = varlen_shard(cu_seqlens, nseq, R, rank, sh);
    if (r != LA_OK) return r;
    const int32_t *cu = cu_seqlens;
    const int i0 = seq_holding(cu, nseq, sh.s);   // the sequence holding the shard's first token
    const bool continues = cu[i0] < sh.s;        // it started on an earlier rank
    if ((r = check_varlen_cp(gathered, R, initial_state, s_in, H, D, continues, nseq, "initial_state", "s_in")) != LA_OK)
        return r;
    const size_t hdd = static_cast<size_t>(H) * D * D;
    la::CombineTerms t{};
    const float *s0 = nullptr;
    if (continues) {
        // its parts on ranks r0 .. rank-1 each end where the next rank starts: (rank-1-r') L tokens before s
        const int r0 = static_cast<int>(cu[i0] / sh.L);
        for (int rp = r0; rp < rank; ++rp) {
            t.idx[t.n] = rp;
            t.exps[t.n] = static_cast<float>(rank - 1 - rp) * static_cast<float>(sh.L);
            ++t.n;
        }
        if (initial_state) s0 = initial_state + static_cast<size_t>(i0) * hdd;
        t.s0_exp = static_cast<float>(sh.s - cu[i0]);
    } else if (initial_state) {
        // the first part here starts its sequence (the first sequence at token s, possibly an empty one)
        const int first = static_cast<int>(std::lower_bound(cu, cu + nseq + 1, static_cast<int32_t>(sh.s)) - cu);
        s0 = initial_state + static_cast<size_t>(first) * hdd;
        t.s0_exp = 0.f;
    }
    r = launch_combine_terms(gathered, static_cast<long long>(H), t, s0, H, D, slopes, s_in,
                             reinterpret_cast<cudaStream_t>(stream));
    if (r == LA_OK) t_last_launches = 1;
    return r;
}

la_status la_cp_varlen_reverse_entry_state(const float *gathered, int R, int rank, const int32_t *cu_seqlens, int nseq,
                                           int H, int D, const float *d_final_state, const float *slopes, float *h_in,
                                           la_stream_t stream) {
    t_last_launches = 0;
    VarlenShard sh;
    la_status r = varlen_shard(cu_seqlens, nseq, R, rank, sh);
    if (r != LA_OK) return r;
    const int32_t *cu = cu_seqlens;
    const int i1 = seq_holding(cu, nseq, sh.e - 1);   // the sequence holding the shard's last token
    const bool continues = cu[i1 + 1] > sh.e;        // it ends on a later rank
    if ((r = check_varlen_cp(gathered, R, d_final_state, h_in, H, D, continues, nseq, "d_final_state", "h_in")) != LA_OK)
        return r;
    const size_t hdd = static_cast<size_t>(H) * D * D;
    la::CombineTerms t{};
    const float *s_end = nullptr;
    if (continues) {
        // its parts on ranks rank+1 .. r1 each begin where the previous rank ends: (r'-rank-1) L tokens after e
        const int r1 = static_cast<int>((cu[i1 + 1] - 1) / sh.L);
        for (int rp = rank + 1; rp <= r1; ++rp) {
            t.idx[t.n] = rp;
            t.exps[t.n] = static_cast<float>(rp - rank - 1) * static_cast<float>(sh.L);
            ++t.n;
        }
        if (d_final_state) s_end = d_final_state + static_cast<size_t>(i1) * hdd;
        t.s0_exp = static_cast<float>(cu[i1 + 1] - sh.e);
    } else if (d_final_state) {
        // the last part here ends its sequence; on the last rank the empty sequences at the end come after it
        const int last = sh.e == sh.T ? nseq - 1 : i1;
        s_end = d_final_state + static_cast<size_t>(last) * hdd;
        t.s0_exp = 0.f;
    }
    r = launch_combine_terms(gathered, static_cast<long long>(H), t, s_end, H, D, slopes, h_in,
                             reinterpret_cast<cudaStream_t>(stream));
    if (r == LA_OK) t_last_launches = 1;
    return r;
}

size_t la_prefill_workspace_size(int B, int N, int H, int D, la_dtype dtype) {
    if (B < 1 || N < 0 || H < 1 || (D != 64 && D != 128)) return 0;
    return make_plan(static_cast<int64_t>(B) * N, B, N, H, D, dtype).bytes;
}

la_status la_prefill(const void *q, const void *k, const void *v, void *o, int B, int N, int H, int D, la_dtype dtype,
                     const float *initial_state, float *final_state, const float *slopes, void *workspace,
                     size_t workspace_bytes, la_stream_t stream) {
    if (B < 1 || N < 0) {
        t_last_launches = 0;
        return fail(LA_ERR_INVALID_ARGUMENT, "B=%d must be >= 1 and N=%d >= 0", B, N);
    }
    return prefill_impl(q, k, v, o, nullptr, B, N, static_cast<int64_t>(B) * N, H, D, dtype, initial_state,
                        final_state, slopes, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

size_t la_prefill_varlen_workspace_size(int64_t T, int nseq, int H, int D, la_dtype dtype) {
    if (T < 0 || nseq < 1 || H < 1 || (D != 64 && D != 128)) return 0;
    return make_plan(T, nseq, 0, H, D, dtype).bytes;
}

la_status la_prefill_varlen(const void *q, const void *k, const void *v, void *o, const int32_t *cu_seqlens, int nseq,
                            int64_t T, int H, int D, la_dtype dtype, const float *initial_state, float *final_state,
                            const float *slopes, void *workspace, size_t workspace_bytes, la_stream_t stream) {
    if (!cu_seqlens) {
        t_last_launches = 0;
        return fail(LA_ERR_INVALID_ARGUMENT, "cu_seqlens must be non-null");
    }
    if (!aligned(cu_seqlens, 4)) {
        t_last_launches = 0;
        return fail(LA_ERR_INVALID_ARGUMENT, "cu_seqlens is not 4-byte aligned");
    }
    return prefill_impl(q, k, v, o, cu_seqlens, nseq, 0, T, H, D, dtype, initial_state, final_state, slopes, workspace,
                        workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

size_t la_prefill_backward_workspace_size(int B, int N, int H, int D, la_dtype dtype) {
    if (B < 1 || N < 0 || H < 1 || (D != 64 && D != 128)) return 0;
    return make_bwd_plan(static_cast<int64_t>(B) * N, B, N, H, D, dtype).bytes;
}

la_status la_prefill_backward(const void *q, const void *k, const void *v, const void *dout, void *dq, void *dk,
                              void *dv, int B, int N, int H, int D, la_dtype dtype, const float *initial_state,
                              const float *d_final_state, float *d_initial_state, const float *slopes, void *workspace,
                              size_t workspace_bytes, la_stream_t stream) {
    if (B < 1 || N < 0) {
        t_last_launches = 0;
        return fail(LA_ERR_INVALID_ARGUMENT, "B=%d must be >= 1 and N=%d >= 0", B, N);
    }
    return backward_impl(q, k, v, dout, dq, dk, dv, nullptr, B, N, static_cast<int64_t>(B) * N, H, D, dtype,
                         initial_state, d_final_state, d_initial_state, slopes, workspace, workspace_bytes,
                         reinterpret_cast<cudaStream_t>(stream));
}

size_t la_prefill_varlen_backward_workspace_size(int64_t T, int nseq, int H, int D, la_dtype dtype) {
    if (T < 0 || nseq < 1 || H < 1 || (D != 64 && D != 128)) return 0;
    return make_bwd_plan(T, nseq, 0, H, D, dtype).bytes;
}

la_status la_prefill_varlen_backward(const void *q, const void *k, const void *v, const void *dout, void *dq, void *dk,
                                     void *dv, const int32_t *cu_seqlens, int nseq, int64_t T, int H, int D,
                                     la_dtype dtype, const float *initial_state, const float *d_final_state,
                                     float *d_initial_state, const float *slopes, void *workspace,
                                     size_t workspace_bytes, la_stream_t stream) {
    if (!cu_seqlens || !aligned(cu_seqlens, 4)) {
        t_last_launches = 0;
        return fail(LA_ERR_INVALID_ARGUMENT, "cu_seqlens must be non-null and 4-byte aligned");
    }
    return backward_impl(q, k, v, dout, dq, dk, dv, cu_seqlens, nseq, 0, T, H, D, dtype, initial_state, d_final_state,
                         d_initial_state, slopes, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

la_status la_prefill_norm_gate(const void *q, const void *k, const void *v, const void *gate, const float *norm_weight,
                               float eps, void *o, int B, int N, int H, int D, la_dtype dtype,
                               const float *initial_state, float *final_state, const float *slopes, void *workspace,
                               size_t workspace_bytes, la_stream_t stream) {
    if (B < 1 || N < 0) {
        t_last_launches = 0;
        return fail(LA_ERR_INVALID_ARGUMENT, "B=%d must be >= 1 and N=%d >= 0", B, N);
    }
    const NormGate ng{gate, norm_weight, eps};
    return prefill_norm_gate_impl(q, k, v, ng, o, nullptr, B, N, static_cast<int64_t>(B) * N, H, D, dtype,
                                  initial_state, final_state, slopes, workspace, workspace_bytes,
                                  reinterpret_cast<cudaStream_t>(stream));
}

la_status la_prefill_varlen_norm_gate(const void *q, const void *k, const void *v, const void *gate,
                                      const float *norm_weight, float eps, void *o, const int32_t *cu_seqlens,
                                      int nseq, int64_t T, int H, int D, la_dtype dtype, const float *initial_state,
                                      float *final_state, const float *slopes, void *workspace,
                                      size_t workspace_bytes, la_stream_t stream) {
    if (!cu_seqlens || !aligned(cu_seqlens, 4)) {
        t_last_launches = 0;
        return fail(LA_ERR_INVALID_ARGUMENT, "cu_seqlens must be non-null and 4-byte aligned");
    }
    const NormGate ng{gate, norm_weight, eps};
    return prefill_norm_gate_impl(q, k, v, ng, o, cu_seqlens, nseq, 0, T, H, D, dtype, initial_state, final_state,
                                  slopes, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

la_status la_norm_gate(const void *o, const void *gate, const float *norm_weight, float eps, void *y, int64_t T, int H,
                       int D, la_dtype dtype, la_stream_t stream) {
    t_last_launches = 0;
    if (!valid_dtype(dtype)) return fail(LA_ERR_INVALID_ARGUMENT, "dtype %d is not a la_dtype", dtype);
    if (D != 64 && D != 128) return fail(LA_ERR_UNSUPPORTED, "head dim D=%d: only 64 and 128 are supported", D);
    if (T < 0 || H < 1) return fail(LA_ERR_INVALID_ARGUMENT, "T=%lld >= 0 and H=%d >= 1 required", static_cast<long long>(T), H);
    if (T * H * D >= (int64_t(1) << 31))
        return fail(LA_ERR_UNSUPPORTED, "T*H*D = %lld elements must be < 2^31", static_cast<long long>(T * H * D));
    if (T > 0 && (!o || !y)) return fail(LA_ERR_INVALID_ARGUMENT, "o and y must be non-null");
    if ((o && !aligned(o, 16)) || (y && !aligned(y, 16)))
        return fail(LA_ERR_INVALID_ARGUMENT, "o and y must be 16-byte aligned");
    const size_t n = static_cast<size_t>(T) * H * D, ob = n * out_bytes(dtype);
    if (o != y && ob && overlap(o, ob, y, ob)) return fail(LA_ERR_INVALID_ARGUMENT, "y must be o itself or not overlap it");
    const NormGate ng{gate, norm_weight, eps};
    la_status r = check_norm_gate(&ng, y, ob, n * in_bytes(dtype));
    if (r != LA_OK) return r;
    if ((r = launch_norm_gate(o, ng, y, T, H, D, dtype, reinterpret_cast<cudaStream_t>(stream))) != LA_OK) return r;
    t_last_launches = T > 0 ? 1 : 0;
    return LA_OK;
}

la_status la_decode_steps_norm_gate(const void *q, const void *k, const void *v, const void *gate,
                                    const float *norm_weight, float eps, void *o, float *state, int B, int K, int H,
                                    int D, la_dtype dtype, const float *slopes, la_stream_t stream) {
    const NormGate ng{gate, norm_weight, eps};
    return decode_impl(q, k, v, o, state, B, K, H, D, dtype, slopes, stream, &ng);
}

la_status la_decode_step(const void *q, const void *k, const void *v, void *o, float *state, int B, int H, int D,
                         la_dtype dtype, const float *slopes, la_stream_t stream) {
    return decode_impl(q, k, v, o, state, B, 1, H, D, dtype, slopes, stream);
}

la_status la_decode_steps(const void *q, const void *k, const void *v, void *o, float *state, int B, int K, int H,
                          int D, la_dtype dtype, const float *slopes, la_stream_t stream) {
    return decode_impl(q, k, v, o, state, B, K, H, D, dtype, slopes, stream);
}

const char *la_status_string(la_status s) {
    switch (s) {
        case LA_OK: return "LA_OK";
        case LA_ERR_INVALID_ARGUMENT: return "LA_ERR_INVALID_ARGUMENT";
        case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED";
        case LA_ERR_WORKSPACE: return "LA_ERR_WORKSPACE";
        case LA_ERR_CUDA: return "LA_ERR_CUDA";
        case LA_ERR_DEVICE_TIMEOUT: return "LA_ERR_DEVICE_TIMEOUT";
    }
    return "LA_ERR_UNKNOWN";
}

const char *la_last_error(void) { return t_last_error.c_str(); }

la_status la_trace_enable(int on) {
    t_trace = on != 0;
    return LA_OK;
}

int la_trace_collect(const char **names, float *ms, int max) {
    int n = 0;
    bool ok = true;
    for (const TraceRec &r : t_recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) ok = false;
        if (n < max) {
            if (names) names[n] = r.name;
            if (ms) ms[n] = t;
            ++n;
        }
        t_pool.push_back(r.a);
        t_pool.push_back(r.b);
    }
    t_recs.clear();
    return ok ? n : -1;
}

int la_last_launch_count(void) { return t_last_launches; }

la_status la_validate_cu_seqlens(const int32_t *cu_seqlens, int nseq, int64_t T, la_stream_t stream) {
    if (!cu_seqlens || nseq < 1 || T < 0) return fail(LA_ERR_INVALID_ARGUMENT, "bad arguments");
    std::string host(static_cast<size_t>(nseq + 1) * sizeof(int32_t), '\0');
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&host[0], cu_seqlens, host.size(), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "reading cu_seqlens");
    const int32_t *c = reinterpret_cast<const int32_t *>(host.data());
    if (c[0] != 0) return fail(LA_ERR_INVALID_ARGUMENT, "cu_seqlens[0] = %d, expected 0", c[0]);
    for (int i = 0; i < nseq; ++i)
        if (c[i + 1] < c[i]) return fail(LA_ERR_INVALID_ARGUMENT, "cu_seqlens decreases at %d", i);
    if (c[nseq] != T)
        return fail(LA_ERR_INVALID_ARGUMENT, "cu_seqlens[nseq] = %d, expected T = %lld", c[nseq], static_cast<long long>(T));
    return LA_OK;
}

la_status la_get_device_error(int *code) {
    if (!code) return fail(LA_ERR_INVALID_ARGUMENT, "code must be non-null");
    cudaError_t e = cudaDeviceSynchronize();
    int v = 0;
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&v, la::g_status, sizeof(int));
    const int zero = 0;
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(la::g_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
    *code = v;
    return LA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- la_prefill without caller workspace
// Scratch for la_prefill_noalloc: a fixed array in the library's device image,
// so that callers who cannot allocate still get the segment split. Host code
// must not use the symbol's name as an address (it is a host-side stand-in);
// the device address is looked up once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_static_workspace[LA_STATIC_WORKSPACE_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_static_ws_mu;
void *g_static_ws_ptr[kMaxDevices] = {};

// Device address of g_static_workspace on the current device (looked up on first use).
la_status static_workspace(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(LA_ERR_UNSUPPORTED, "device index %d >= %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lock(g_static_ws_mu);
    if (!g_static_ws_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_workspace);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static workspace)");
        g_static_ws_ptr[dev] = p;
    }
    *out = g_static_ws_ptr[dev];
    return LA_OK;
}
}  // namespace

extern "C" la_status la_prefill_noalloc(const void *q, const void *k, const void *v, void *o, int B, int N, int H,
                                        int D, la_dtype dtype, const float *initial_state, float *final_state,
                                        const float *slopes, la_stream_t stream) {
    t_last_launches = 0;
    if (B < 1 || N < 0) return fail(LA_ERR_INVALID_ARGUMENT, "B=%d must be >= 1 and N=%d >= 0", B, N);
    if (H < 1 || (D != 64 && D != 128)) return la_prefill(q, k, v, o, B, N, H, D, dtype, initial_state, final_state,
                                                          slopes, nullptr, 0, stream);  // reports the argument error
    const size_t need = la_prefill_workspace_size(B, N, H, D, dtype);
    if (need > LA_STATIC_WORKSPACE_BYTES)
        return fail(LA_ERR_WORKSPACE,
                    "this call needs %zu bytes of scratch; la_prefill_noalloc has %u (use la_prefill with a workspace)",
                    need, LA_STATIC_WORKSPACE_BYTES);
    void *ws = nullptr;
    if (need > 0) {
        la_status r = static_workspace(&ws);
        if (r != LA_OK) return r;
    }
    return la_prefill(q, k, v, o, B, N, H, D, dtype, initial_state, final_state, slopes, ws, need, stream);
}

#ifdef LA_TRACE_PHASES
// Profiling builds only: copy the phase timestamps of the traced CTAs of the last launches.
extern "C" int la_debug_phase_dump(long long *out, int n) {
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    const int cap = la::kPhaseSlots * la::kPhaseChunks * la::kPhaseEvents;
    if (n > cap) n = cap;
    return cudaMemcpyFromSymbol(out, la::g_la_phase, sizeof(long long) * n) == cudaSuccess ? n : -1;
}
extern "C" int la_debug_sphase_dump(long long *out, int n) {
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    const int cap = la::kPhaseSlots * la::kPhaseChunks * 8;
    if (n > cap) n = cap;
    return cudaMemcpyFromSymbol(out, la::g_la_sphase, sizeof(long long) * n) == cudaSuccess ? n : -1;
}
#endif
#ifdef LA_TRACE_ANY
extern "C" int la_debug_cta_dump(long long *out, int n) {
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    const int cap = 2 * la::kTraceCtas * 8;
    if (n > cap) n = cap;
    return cudaMemcpyFromSymbol(out, la::g_la_cta, sizeof(long long) * n) == cudaSuccess ? n : -1;
}
#endif
