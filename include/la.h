/*
 * la.h -- C ABI of the B200 (sm_100a) Lightning Attention library.
 *
 * The operator. Lightning Attention is the linear-attention layer of the
 * hybrid Lightning-Attention / MLA stack (Ling & Ring 2.6 Technical Report,
 * blog post news.neo-ai.one/en/article/3021, section "Hybrid Linear Attention":
 * mixed 7:1 with MLA, O(n) along the sequence). The pages give no formula; the
 * operator implemented here is the causal linear attention with per-head decay
 *
 *     o_t = sum_{s<=t} lambda_h^(t-s) (q_t . k_s) v_s,
 *     lambda_h = exp(-2^(-8(h+1)/H)),  h = 0..H-1,
 *
 * in state form S_t = lambda_h S_{t-1} + k_t^T v_t, o_t = q_t S_t, where S is a
 * D x D fp32 matrix per (sequence, head), S[i][j] pairing k_i with v_j. With an
 * initial state S0 the first token sees lambda S0 (the state decays once
 * before the first token), and the final state after N tokens is
 * lambda^N S0 + sum_s lambda^(N-1-s) k_s^T v_s (s 0-based). No 1/sqrt(D)
 * scale, normaliser, feature map or gate is applied inside the operator.
 *
 * Conventions shared by every entry point:
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise. The
 *     caller owns every buffer; the library never allocates, frees or keeps a
 *     pointer after the call returns.
 *   - Every call only validates its arguments on the host and enqueues kernels
 *     on `stream`; it does not synchronise (except la_validate_cu_seqlens and
 *     la_get_device_error, which say so). Calls are thread-safe.
 *   - q, k, v, o and states must be 16-byte aligned and densely packed in the
 *     layouts given below (head dim innermost). o must not alias q, k or v.
 *   - dtype: LA_BF16 (bf16 q/k/v/o), LA_BF16_F16OUT (bf16 q/k/v, fp16 o),
 *     LA_BF16_F32OUT (bf16 q/k/v, fp32 o) or LA_FP32 (fp32 q/k/v/o).
 *     Accumulation and states are always fp32. The output's own rounding is
 *     part of the result: up to 2^-8 relative for bf16 o, 2^-11 for fp16 o
 *     (whose range ends at 65504; values below 2^-14 lose relative precision);
 *     fp32 o is the fp32 accumulator unrounded.
 *   - D (head dim, Dk = Dv = D) must be 64 or 128. bf16 inputs run on the tensor
 *     cores (D = 64 with chunk and output-correction kernels of its own, whose
 *     products run over the 64 real columns; its segment-state pass uses the
 *     128-wide tiles with the missing columns filled with zeros on load);
 *     LA_FP32 runs on the CUDA cores (fp32 FMA), as does a call with no tokens.
 *   - `slopes` is an optional fp32 [H] device array: lambda_h = exp(-slopes[h]),
 *     slopes[h] >= 0. NULL selects the schedule above.
 *   - Arguments are checked before anything is enqueued; on error nothing is
 *     enqueued and la_last_error() describes the problem. A CUDA launch error
 *     is returned as LA_ERR_CUDA.
 *   - Kernels never trap. Every wait inside a kernel is bounded; if one ever
 *     runs out, the kernel records LA_ERR_DEVICE_TIMEOUT in a device status
 *     word (read with la_get_device_error) and returns.
 */
#ifndef LA_H
#define LA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream; NULL is the legacy default stream. */
typedef struct CUstream_st *la_stream_t;

typedef enum {
    LA_OK = 0,
    LA_ERR_INVALID_ARGUMENT = 1,  /* null / misaligned pointer, bad size, o aliasing an input */
    LA_ERR_UNSUPPORTED = 2,       /* valid but not implemented (e.g. D not 64 or 128) */
    LA_ERR_WORKSPACE = 3,         /* workspace NULL or smaller than the queried size */
    LA_ERR_CUDA = 4,              /* a CUDA runtime / driver call or launch failed */
    LA_ERR_DEVICE_TIMEOUT = 5     /* reported by la_get_device_error: a bounded wait ran out */
} la_status;

typedef enum {
    LA_BF16 = 0,         /* q, k, v, o bf16 */
    LA_FP32 = 1,         /* q, k, v, o fp32 */
    LA_BF16_F32OUT = 2,  /* q, k, v bf16; o fp32 */
    LA_BF16_F16OUT = 3   /* q, k, v bf16; o fp16 (11-bit significand; |o| must stay below 65504) */
} la_dtype;

/*
 * Chunked prefill over B sequences of equal length N.
 *   q, k, v, o     : [B, N, H, D] in the types `dtype` names (o written in full).
 *   initial_state  : [B, H, D, D] fp32, or NULL for a zero state.
 *   final_state    : [B, H, D, D] fp32 written with S_N, or NULL. It may be
 *                    the same pointer as initial_state (updated in place).
 *   workspace      : device scratch of at least la_prefill_workspace_size(...)
 *                    bytes (256-byte aligned), or NULL when that size is 0.
 *                    Its contents on entry do not matter; the library owns it
 *                    until the enqueued work has finished.
 * Valid sizes: B >= 1, N >= 0, H >= 1, D in {64, 128}, B*N*H*D < 2^31.
 * Work split: when B*H alone cannot fill the GPU, each sequence is cut into
 * segments processed in parallel. A state-only pass first computes, from a
 * zero start, the state of every fine unit before a sequence's last segment;
 * the CTA of each later segment then sums the decayed states of the units
 * before it as it starts (no separate scan kernel). The split is a fixed
 * function of the arguments (B, N, H, D, dtype), so the workspace size that
 * la_prefill_workspace_size returns is always the one the call needs.
 * Carrying final_state into the next call's initial_state continues the same
 * sequence exactly (the hand-off that the report's context-parallel section,
 * "Long-Context Training: Context Parallel for Lightning Attention", relies on).
 */
size_t la_prefill_workspace_size(int B, int N, int H, int D, la_dtype dtype);
la_status la_prefill(const void *q, const void *k, const void *v, void *o,
                     int B, int N, int H, int D, la_dtype dtype,
                     const float *initial_state, float *final_state, const float *slopes,
                     void *workspace, size_t workspace_bytes, la_stream_t stream);

/*
 * Prefill over nseq sequences of different lengths packed along the token
 * axis (the varlen sequences of the report's context-parallel section).
 *   q, k, v, o     : [T, H, D] in the types `dtype` names; sequence i is tokens
 *                    cu_seqlens[i] .. cu_seqlens[i+1]-1.
 *   cu_seqlens     : DEVICE int32 [nseq + 1]; cu_seqlens[0] = 0, non-decreasing,
 *                    cu_seqlens[nseq] = T. Zero-length sequences are allowed
 *                    (their final state equals their initial state). The host
 *                    cannot read this array without synchronising, so it is
 *                    not checked here: a malformed array is clamped on the
 *                    device (no access outside [0, T)) and recorded as
 *                    LA_ERR_INVALID_ARGUMENT in the device status word; call
 *                    la_validate_cu_seqlens first to check one synchronously.
 *   initial_state, final_state : [nseq, H, D, D] fp32 or NULL (same rules as
 *                    la_prefill; they may alias).
 * Valid sizes: nseq >= 1, T >= 0, H >= 1, D in {64, 128}, T*H*D < 2^31.
 */
size_t la_prefill_varlen_workspace_size(int64_t T, int nseq, int H, int D, la_dtype dtype);
la_status la_prefill_varlen(const void *q, const void *k, const void *v, void *o,
                            const int32_t *cu_seqlens, int nseq, int64_t T, int H, int D,
                            la_dtype dtype, const float *initial_state, float *final_state,
                            const float *slopes, void *workspace, size_t workspace_bytes,
                            la_stream_t stream);

/*
 * Backward pass of la_prefill (training use of the layer; the pages do not
 * treat the backward pass, so this is the derivative of the operator above).
 * Given dout = dL/do and d_final_state = dL/dS_N (NULL for zero), it writes
 *     dq_t = S_t dO_t,   dk_t = G_t v_t,   dv_t = k_t G_t,   dS_0 = lambda G_0,
 * where S_t is the forward state and G_t = q_t^T dO_t + lambda G_{t+1} (with
 * G_{N-1} also holding dS_N) is the gradient of S_t. Each is one run of the
 * chunked recurrence with the roles of q, k, v exchanged: dq forward in time
 * from S0^T, dk and dv backward in time from dS_N^T and dS_N (the dv run's
 * final state is dS_0). The forward's outputs are not needed.
 *   q, k, v, dout  : [B, N, H, D] inputs in the input type of `dtype`.
 *   dq, dk, dv     : [B, N, H, D] written in the output type of `dtype` (bf16,
 *                    fp16 or fp32 as for o); they must not overlap each other
 *                    or any input.
 *   initial_state  : [B, H, D, D] fp32 S0 of the forward call, or NULL (zero).
 *   d_final_state  : [B, H, D, D] fp32 dL/dS_N, or NULL (zero).
 *   d_initial_state: [B, H, D, D] fp32 written with dL/dS0, or NULL. It may be
 *                    the same pointer as d_final_state or initial_state.
 *   workspace      : at least la_prefill_backward_workspace_size(...) bytes
 *                    (never 0), 256-byte aligned.
 * Same sizes, slopes and error rules as la_prefill. Error bound: the three
 * runs have the forward's accuracy, each relative to its own outputs.
 * Streams: the three runs share the GPU; two of them run on internal streams
 * (one pair per host thread and device) that start after the work already on
 * `stream` and are joined back into it through events, so everything enqueued
 * on `stream` afterwards is ordered after the whole backward pass, and the call
 * may be captured into a CUDA graph like any other.
 */
size_t la_prefill_backward_workspace_size(int B, int N, int H, int D, la_dtype dtype);
la_status la_prefill_backward(const void *q, const void *k, const void *v, const void *dout,
                              void *dq, void *dk, void *dv, int B, int N, int H, int D,
                              la_dtype dtype, const float *initial_state, const float *d_final_state,
                              float *d_initial_state, const float *slopes, void *workspace,
                              size_t workspace_bytes, la_stream_t stream);

/*
 * Backward pass of la_prefill_varlen: as la_prefill_backward over packed
 * sequences ([T, H, D] tensors, states [nseq, H, D, D], cu_seqlens as for
 * la_prefill_varlen). A zero-length sequence passes the state gradient
 * through: its dS_0 is its dS_N.
 */
size_t la_prefill_varlen_backward_workspace_size(int64_t T, int nseq, int H, int D, la_dtype dtype);
la_status la_prefill_varlen_backward(const void *q, const void *k, const void *v, const void *dout,
                                     void *dq, void *dk, void *dv, const int32_t *cu_seqlens,
                                     int nseq, int64_t T, int H, int D, la_dtype dtype,
                                     const float *initial_state, const float *d_final_state,
                                     float *d_initial_state, const float *slopes, void *workspace,
                                     size_t workspace_bytes, la_stream_t stream);

/*
 * Output group RMSNorm + sigmoid gate (the report's "linghe" section, blog post
 * news.neo-ai.one/en/article/3021, lists "Group RMSNorm + Sigmoid Gate" among
 * the fused kernels of the attention module's BF16 inference, with no
 * formula). Each (token, head) row of D values is one group:
 *     y = norm_weight[h] * o / sqrt(mean_d(o^2) + eps) * sigmoid(gate),
 * one streaming pass that reads o and the gate and writes y.
 *   o, y           : [T, H, D] in the output type of `dtype`; y may be o itself
 *                    (in place) but must not otherwise overlap it.
 *   gate           : [T, H, D] in the input type of `dtype` (bf16, or fp32 for
 *                    LA_FP32): the gate pre-activation, a projection of the
 *                    layer input made by the caller; must not overlap y.
 *   norm_weight    : [H, D] fp32 (the learned per-channel scale).
 *   eps            : finite, >= 0 (with eps = 0 an all-zero row gives NaN).
 * Valid sizes: T >= 0, H >= 1, D in {64, 128}, T*H*D < 2^31.
 */
la_status la_norm_gate(const void *o, const void *gate, const float *norm_weight, float eps, void *y,
                       int64_t T, int H, int D, la_dtype dtype, la_stream_t stream);

/*
 * la_prefill followed by la_norm_gate in place on o (two launches after the
 * prefill's own): o receives y. gate as in la_norm_gate ([B, N, H, D]);
 * everything else as la_prefill (same workspace size, every dtype and D).
 * (Folding the norm and gate into the prefill kernel's own output store was
 * measured slower on B200: that kernel has no shared memory left for the gate
 * tile, and its one slot that is free before the store frees up too late for
 * the gate's load to arrive.)
 */
la_status la_prefill_norm_gate(const void *q, const void *k, const void *v, const void *gate,
                               const float *norm_weight, float eps, void *o,
                               int B, int N, int H, int D, la_dtype dtype,
                               const float *initial_state, float *final_state, const float *slopes,
                               void *workspace, size_t workspace_bytes, la_stream_t stream);

/* la_prefill_varlen with the fused output norm + gate (gate [T, H, D] bf16). */
la_status la_prefill_varlen_norm_gate(const void *q, const void *k, const void *v, const void *gate,
                                      const float *norm_weight, float eps, void *o,
                                      const int32_t *cu_seqlens, int nseq, int64_t T, int H, int D,
                                      la_dtype dtype, const float *initial_state, float *final_state,
                                      const float *slopes, void *workspace, size_t workspace_bytes,
                                      la_stream_t stream);

/*
 * la_decode_steps with the output norm + gate fused into the decode kernel's
 * store (its outputs are on chip): gate [B, K, H, D] in the input type of
 * `dtype`, norm_weight [H, D] fp32, eps as for la_norm_gate. Every dtype and
 * D in {64, 128}; K = 1 is one step.
 */
la_status la_decode_steps_norm_gate(const void *q, const void *k, const void *v, const void *gate,
                                    const float *norm_weight, float eps, void *o, float *state,
                                    int B, int K, int H, int D, la_dtype dtype, const float *slopes,
                                    la_stream_t stream);

/*
 * One decode step for B sequences, state updated in place: the state form of
 * the operator above, one token at a time (the report's section "Hybrid
 * Linear Attention", blog post news.neo-ai.one/en/article/3021, gives the layer
 * a cost linear in the sequence length for training and decoding: each new
 * token reads and rewrites the fixed-size state instead of the whole history).
 *   S <- lambda_h S + k^T v, then o = q S (the output includes this token).
 *   q, k, v, o : [B, H, D] in the types `dtype` names; state : [B, H, D, D] fp32 (read and
 *   written). Needs no workspace. Valid sizes: B >= 1, H >= 1, D in {64, 128}.
 */
la_status la_decode_step(const void *q, const void *k, const void *v, void *o, float *state,
                         int B, int H, int D, la_dtype dtype, const float *slopes,
                         la_stream_t stream);

/*
 * K consecutive decode steps per sequence in one launch (multi-token or
 * speculative decoding; no counterpart on the report's pages beyond the
 * recurrence itself): for t = 0..K-1, S <- lambda S + k_t^T v_t, o_t = q_t S.
 * q, k, v, o: [B, K, H, D] (token t of sequence b at row b*K + t); state
 * [B, H, D, D] fp32, updated in place and read and written once for all K
 * tokens (the state stays on chip between them). K = 0 does nothing. Same
 * dtypes, alignment and error behaviour as la_decode_step; K = 1 is exactly
 * la_decode_step.
 */
la_status la_decode_steps(const void *q, const void *k, const void *v, void *o, float *state,
                          int B, int K, int H, int D, la_dtype dtype, const float *slopes,
                          la_stream_t stream);

/* Static description of a status code (never NULL). */
const char *la_status_string(la_status s);

/* Description of the last error returned on the calling thread (never NULL; "" if none). */
const char *la_last_error(void);

/*
 * Debug helper, SYNCHRONOUS: copies cu_seqlens to the host on `stream`, waits,
 * and checks cu[0] = 0, cu non-decreasing, cu[nseq] = T.
 */
la_status la_validate_cu_seqlens(const int32_t *cu_seqlens, int nseq, int64_t T, la_stream_t stream);

/*
 * SYNCHRONOUS: waits for the device, then reads and clears the library's
 * device status word. *code receives LA_OK, or the first device-side status
 * recorded since the last call (LA_ERR_DEVICE_TIMEOUT, or
 * LA_ERR_INVALID_ARGUMENT for a malformed cu_seqlens). Returns LA_ERR_CUDA if
 * the device could not be read.
 */
la_status la_get_device_error(int *code);

/* Number of kernels the last successful call on this thread enqueued (for launch accounting). */
int la_last_launch_count(void);

/*
 * Kernel-level tracing, for profiling (no counterpart on the report's pages).
 * la_trace_enable(1) makes every later call on this thread record a CUDA
 * event on `stream` before and after each kernel it enqueues (events are
 * created on first use and reused; no device memory is allocated).
 * la_trace_collect() waits for the recorded events and writes, for at most
 * `max` kernels in launch order since the last collect, a pointer to the
 * kernel's static name and its duration in milliseconds; it returns how many
 * were written (or -1 on a CUDA error) and clears the record.
 * la_trace_enable(0) stops recording.
 */
la_status la_trace_enable(int on);
int la_trace_collect(const char **names, float *ms, int max);

/*
 * la_prefill for callers that cannot allocate device memory at call time (the
 * report's pages have no counterpart; this is a deployment convenience).
 * Some callers have no way to hand the library a scratch buffer: code that runs
 * under a host framework which owns every device allocation and offers no
 * scratch, or code on a latency-critical path where a cudaMalloc (which may
 * synchronise the whole device) is not acceptable. This entry point takes the
 * same arguments as la_prefill minus the workspace and uses instead a scratch
 * array compiled into the library: LA_STATIC_WORKSPACE_BYTES of device memory,
 * which every GPU that loads the library holds until the process exits.
 *   - It allocates nothing: no cudaMalloc / cudaFree, no allocating library call.
 *   - Calls whose la_prefill_workspace_size(...) exceeds LA_STATIC_WORKSPACE_BYTES
 *     are rejected with LA_ERR_WORKSPACE before anything is enqueued; use
 *     la_prefill with your own workspace for those.
 *   - The first call on a device looks up the array's device address (with that
 *     device current); make that first call before any stream capture.
 *   - All calls on a device share the one array and it keeps whatever the last
 *     call left there; every byte a call reads is written earlier in the same
 *     call, so nothing has to be cleared. Calls that can overlap on the GPU
 *     (different streams, or different host threads) race on the array: order
 *     them on one stream or serialise them.
 */
#define LA_STATIC_WORKSPACE_BYTES (32u << 20)
la_status la_prefill_noalloc(const void *q, const void *k, const void *v, void *o,
                             int B, int N, int H, int D, la_dtype dtype,
                             const float *initial_state, float *final_state, const float *slopes,
                             la_stream_t stream);

/*
 * Context parallelism: one batch of sequences sharded along N across the R
 * ranks of a group (Ling & Ring 2.6 Technical Report, section "Long-Context
 * Training: Context Parallel for Lightning Attention": each shard runs its
 * local recursion, then is corrected with the gathered states of the earlier
 * shards). Every rank holds tokens [r*L, (r+1)*L) of each sequence. Per rank:
 *   1. la_shard_state: dS_r = sum over the shard of lambda^(L-1-s) k_s^T v_s,
 *      the state the shard produces from a zero start;
 *   2. an all-gather of dS_r over the group (the caller's collective, e.g.
 *      NCCL through torch.distributed) into gathered[R, B, H, D, D];
 *   3. la_cp_entry_state: the state entering shard r,
 *      S_in = lambda^(r*L) S_0 + sum_{r' < r} lambda^((r-1-r')*L) dS_r';
 *   4. la_prefill on the shard with initial_state = S_in.
 * Outputs are then exactly those of one prefill over the whole sequences, and
 * the last rank's final state is the sequences' final state.
 *
 * la_shard_state: k, v [B, N, H, D] bf16 (dtype one of the bf16-input types;
 * LA_FP32 gives LA_ERR_UNSUPPORTED), D = 64 or 128. delta_state [B, H, D, D] fp32,
 * written (16-byte aligned, caller-owned). The shard is cut into fine units
 * that fill the GPU; their states are combined into delta_state through a
 * caller-owned, 256-byte aligned workspace of
 * la_shard_state_workspace_size(B, N, H, D, dtype) bytes (0 when no split is
 * needed; LA_ERR_WORKSPACE if missing or short). N = 0 writes zeros. slopes as
 * for la_prefill. Asynchronous on `stream`.
 */
size_t la_shard_state_workspace_size(int B, int N, int H, int D, la_dtype dtype);
la_status la_shard_state(const void *k, const void *v, int B, int N, int H, int D, la_dtype dtype,
                         const float *slopes, float *delta_state, void *workspace,
                         size_t workspace_bytes, la_stream_t stream);

/*
 * la_cp_entry_state: gathered [R, B, H, D, D] fp32 holds dS_0 .. dS_{R-1} in
 * rank order (only the first `rank` are read; may be NULL for rank 0), L the
 * tokens per shard, initial_state [B, H, D, D] fp32 or NULL (zero), s_in
 * [B, H, D, D] fp32 written (must not overlap gathered). D = 64 or 128. All
 * pointers are device pointers, 16-byte aligned. LA_ERR_INVALID_ARGUMENT for
 * rank outside [0, R). Asynchronous on `stream`.
 */
la_status la_cp_entry_state(const float *gathered, int R, int rank, int B, int H, int D, int L,
                            const float *initial_state, const float *slopes, float *s_in,
                            la_stream_t stream);

/*
 * Context-parallel backward pass (the training side of the same section).
 * Rank r holds tokens [r*L, (r+1)*L) of every sequence with their output
 * gradient dO, and the loss's gradient dS_N of the sequences' final state (the
 * same on every rank, or NULL). Besides the forward entry state S_in above, the
 * backward pass needs the reversed state entering the shard from its right end:
 *   1. la_shard_state_reverse: the shard's reversed state from a zero start,
 *      dH_r = sum_s lambda^(s+1) q_s^T dO_s (s from the shard's start);
 *   2. all ranks exchange their dH_r into gathered[R, B, H, D, D] (the same
 *      all-gather as dS_r; the two can travel together);
 *   3. la_cp_reverse_entry_state: the state entering shard r from the right,
 *      H_in = lambda^((R-1-r)*L) dS_N + sum_{r' > r} lambda^((r'-r-1)*L) dH_r';
 *   4. la_prefill_backward on the shard with initial_state = S_in and
 *      d_final_state = H_in.
 * The shards' dq, dk, dv are then exactly those of one backward pass over the
 * whole sequences, and rank 0's d_initial_state is the sequences' dS_0.
 *
 * la_shard_state_reverse: q, dout [B, N, H, D] bf16, D = 64 or 128; otherwise as
 * la_shard_state (same workspace size). delta_state is D x D with rows indexed
 * by q's features and columns by dout's.
 * la_cp_reverse_entry_state: gathered holds dH_0 .. dH_{R-1} in rank order
 * (only those after `rank` are read; may be NULL for the last rank);
 * d_final_state [B, H, D, D] fp32 or NULL (zero); h_in written (must not
 * overlap gathered). Otherwise as la_cp_entry_state.
 */
la_status la_shard_state_reverse(const void *q, const void *dout, int B, int N, int H, int D,
                                 la_dtype dtype, const float *slopes, float *delta_state,
                                 void *workspace, size_t workspace_bytes, la_stream_t stream);
la_status la_cp_reverse_entry_state(const float *gathered, int R, int rank, int B, int H, int D,
                                    int L, const float *d_final_state, const float *slopes,
                                    float *h_in, la_stream_t stream);

/*
 * Context parallelism over packed varlen sequences (the same report section:
 * its context parallelism serves "varlen sequences", with the state correction
 * of several sub-sequences in one vectorized form). The packed batch [T, H, D]
 * with cu_seqlens is cut along the token axis into R equal shards: rank r holds
 * tokens [r*L, (r+1)*L), L = T/R, so a sequence may start on one rank and end
 * on any later one. The part of a sequence on a rank is a sub-sequence; a
 * rank's sub-sequences are the sequences meeting its shard, in order (an empty
 * sequence at token p belongs to the rank that holds token p, the last rank for
 * p = T). Only a rank's first sub-sequence can have started on an earlier rank,
 * and only its last can continue on a later one. Per rank:
 *   1. the state its last sub-sequence produces from a zero start
 *      (la_shard_state on that sub-sequence's tokens, B = 1), and, for the
 *      backward pass, the reversed state its first sub-sequence produces from a
 *      zero start (la_shard_state_reverse on that sub-sequence's q and dout);
 *   2. an all-gather of those [H, D, D] states over the group (rank order);
 *   3. la_cp_varlen_entry_state: the state entering the first sub-sequence,
 *      and for the backward pass la_cp_varlen_reverse_entry_state: the reversed
 *      state entering the last sub-sequence from its right end;
 *   4. la_prefill_varlen (or la_prefill_varlen_backward) on the rank's
 *      sub-sequences, the first starting from the entry state, the others from
 *      their sequences' initial states (the last ending with the reversed
 *      entry state as its final-state gradient, the others with their
 *      sequences' final-state gradients).
 * Outputs and gradients are then exactly those of one call over the whole
 * packed batch; a sequence's final state is the final state of its last
 * sub-sequence, and its initial-state gradient that of its first.
 *
 * la_cp_varlen_entry_state:
 *   gathered      : [R, H, D, D] fp32, rank r' at index r': the state of rank r''s
 *                   last sub-sequence from a zero start. Read only for the ranks
 *                   before `rank` that hold part of the sequence entering this
 *                   shard (may be NULL when none do).
 *   cu_seqlens    : HOST int32 [nseq + 1] of the whole packed batch: cu[0] = 0,
 *                   non-decreasing, T = cu[nseq] > 0 divisible by R (checked here;
 *                   LA_ERR_INVALID_ARGUMENT otherwise). 1 <= R <= 64.
 *   initial_state : [nseq, H, D, D] fp32 initial states of all sequences, or NULL.
 *   s_in          : [H, D, D] fp32, written: the state entering this rank's first
 *                   sub-sequence (its sequence's initial state when it starts here).
 * la_cp_varlen_reverse_entry_state: the mirror image. gathered holds each rank's
 *   first-sub-sequence reversed state (read for the ranks after `rank` holding
 *   part of the sequence leaving this shard); d_final_state [nseq, H, D, D] fp32
 *   or NULL; h_in [H, D, D] written: the reversed state entering this rank's last
 *   sub-sequence from its right end (its sequence's final-state gradient when it
 *   ends here).
 * Both: D = 64 or 128, slopes as for la_prefill, device pointers 16-byte aligned
 * except cu_seqlens; the output must not overlap the other arrays.
 * Asynchronous on `stream` (one small kernel).
 */
la_status la_cp_varlen_entry_state(const float *gathered, int R, int rank, const int32_t *cu_seqlens,
                                   int nseq, int H, int D, const float *initial_state,
                                   const float *slopes, float *s_in, la_stream_t stream);
la_status la_cp_varlen_reverse_entry_state(const float *gathered, int R, int rank,
                                           const int32_t *cu_seqlens, int nseq, int H, int D,
                                           const float *d_final_state, const float *slopes,
                                           float *h_in, la_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LA_H */
