/*
 * Lightning Attention oracle: plain, slow, fp64 CPU code.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may call, link or load
 * this file; only the tests, the package's smoke check and the CPU-baseline leg
 * of the benchmark use it. It shares no code with the CUDA library.
 *
 * What it computes (Ling & Ring 2.6 Technical Report, blog post
 * news.neo-ai.one/en/article/3021, section "Hybrid Linear Attention": Lightning
 * Attention is the linear layer of the 7:1 hybrid stack and costs O(n) along
 * the sequence; section "Long-Context Training: Context Parallel for Lightning
 * Attention": it has a recursive dependency along the sequence). The pages give
 * no formula; the operator is the causal linear attention with per-head decay
 *
 *     o_t = sum_{s<=t} lambda_h^(t-s) (q_t . k_s) v_s,
 *     lambda_h = exp(-2^(-8(h+1)/H)),  h = 0..H-1,
 *
 * and, with an initial state S0 (Dk x Dv, S[i][j] pairs k_i with v_j), the
 * recurrent form S_t = lambda S_{t-1} + k_t^T v_t, o_t = q_t S_t, t = 1..N.
 * The initial state therefore decays once before the first token, and the
 * final state is S_N.
 *
 * This file holds the recurrent (state) form, which is O(N Dk Dv) and is the
 * timed CPU baseline, the single decode step, and the backward pass of the
 * recurrent form (its adjoint, token by token). The quadratic masked-decay
 * form and the brute-force triple sum live in oracle/__init__.py (numpy and
 * plain Python), so that two independent codings of the definition check one
 * another.
 *
 * Layouts: q, k are [T, H, Dk]; v, o are [T, H, Dv] (token-major, packed over
 * sequences given by cu_seqlens[nseq+1]); states are [nseq, H, Dk, Dv].
 */
#define _GNU_SOURCE
#include <math.h>
#include <pthread.h>
#include <sched.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* lambda_h = exp(-2^(-8(h+1)/H)): the decay schedule the operator is specified with. */
int la_oracle_decay(int H, double *lam) {
    if (H <= 0 || !lam) return -1;
    for (int h = 0; h < H; ++h) lam[h] = exp(-pow(2.0, -8.0 * (double)(h + 1) / (double)H));
    return 0;
}

/* Number of CPUs this process may run on (the affinity mask), at least 1. */
int la_oracle_default_threads(void) {
    cpu_set_t set;
    CPU_ZERO(&set);
    if (sched_getaffinity(0, sizeof(set), &set) == 0) {
        int n = CPU_COUNT(&set);
        if (n > 0) return n;
    }
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

typedef struct {
    const double *q, *k, *v;
    double *o;
    const int64_t *cu;
    int nseq, H, Dk, Dv;
    const double *lam;
    const double *s0;
    double *sN;
    int64_t next;          /* next (seq, head) pair to take */
    pthread_mutex_t mu;
} rec_job;

/* One (sequence, head): run the recurrence token by token. */
static void rec_one(const rec_job *J, int seq, int h, double *S) {
    const int H = J->H, Dk = J->Dk, Dv = J->Dv;
    const double lam = J->lam[h];
    const size_t ss = (size_t)Dk * Dv;
    if (J->s0) memcpy(S, J->s0 + ((size_t)seq * H + h) * ss, ss * sizeof(double));
    else memset(S, 0, ss * sizeof(double));
    for (int64_t t = J->cu[seq]; t < J->cu[seq + 1]; ++t) {
        const double *qt = J->q + ((size_t)t * H + h) * Dk;
        const double *kt = J->k + ((size_t)t * H + h) * Dk;
        const double *vt = J->v + ((size_t)t * H + h) * Dv;
        double *ot = J->o + ((size_t)t * H + h) * Dv;
        /* S_t = lambda S_{t-1} + k_t^T v_t */
        for (int i = 0; i < Dk; ++i)
            for (int j = 0; j < Dv; ++j) S[(size_t)i * Dv + j] = lam * S[(size_t)i * Dv + j] + kt[i] * vt[j];
        /* o_t = q_t S_t */
        for (int j = 0; j < Dv; ++j) ot[j] = 0.0;
        for (int i = 0; i < Dk; ++i)
            for (int j = 0; j < Dv; ++j) ot[j] += qt[i] * S[(size_t)i * Dv + j];
    }
    if (J->sN) memcpy(J->sN + ((size_t)seq * H + h) * ss, S, ss * sizeof(double));
}

static void *rec_worker(void *arg) {
    rec_job *J = (rec_job *)arg;
    double *S = (double *)malloc((size_t)J->Dk * J->Dv * sizeof(double));
    if (!S) return (void *)1;
    const int64_t total = (int64_t)J->nseq * J->H;
    for (;;) {
        pthread_mutex_lock(&J->mu);
        int64_t u = J->next++;
        pthread_mutex_unlock(&J->mu);
        if (u >= total) break;
        rec_one(J, (int)(u / J->H), (int)(u % J->H), S);
    }
    free(S);
    return NULL;
}

/*
 * Recurrent form over packed sequences. initial_state / final_state may be
 * NULL (zero start / not returned); final_state may alias initial_state.
 * nthreads <= 0 uses every CPU in the affinity mask. Returns 0, or -1 on bad
 * arguments, -2 on allocation / thread failure.
 */
int la_oracle_prefill_recurrent(const double *q, const double *k, const double *v, double *o,
                                const int64_t *cu_seqlens, int nseq, int H, int Dk, int Dv,
                                const double *lam, const double *initial_state, double *final_state,
                                int nthreads) {
    if (!q || !k || !v || !o || !cu_seqlens || !lam || nseq < 1 || H < 1 || Dk < 1 || Dv < 1) return -1;
    if (cu_seqlens[0] != 0) return -1;
    for (int i = 0; i < nseq; ++i)
        if (cu_seqlens[i + 1] < cu_seqlens[i]) return -1;
    /* Aliased initial/final state: each (seq, head) reads its own slot before writing it,
       and no other pair touches that slot, so the alias is safe. */
    rec_job J = {q, k, v, o, cu_seqlens, nseq, H, Dk, Dv, lam, initial_state, final_state, 0,
                 PTHREAD_MUTEX_INITIALIZER};
    if (nthreads <= 0) nthreads = la_oracle_default_threads();
    const int64_t total = (int64_t)nseq * H;
    if (nthreads > total) nthreads = (int)total;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) return -2;
    int started = 0, rc = 0;
    for (; started < nthreads; ++started)
        if (pthread_create(&th[started], NULL, rec_worker, &J) != 0) break;
    if (started == 0) rc = (int)(intptr_t)rec_worker(&J) ? -2 : 0;
    for (int i = 0; i < started; ++i) {
        void *r = NULL;
        pthread_join(th[i], &r);
        if (r) rc = -2;
    }
    free(th);
    return rc;
}

/*
 * One decode step, in place: S <- lambda S + k^T v, then o = q S (the output
 * includes the current token). q, k: [B, H, Dk]; v, o: [B, H, Dv];
 * state: [B, H, Dk, Dv].
 */
int la_oracle_decode_step(const double *q, const double *k, const double *v, double *o, double *state,
                          int B, int H, int Dk, int Dv, const double *lam) {
    if (!q || !k || !v || !o || !state || !lam || B < 1 || H < 1 || Dk < 1 || Dv < 1) return -1;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const size_t bh = (size_t)b * H + h;
            double *S = state + bh * (size_t)Dk * Dv;
            const double *qt = q + bh * Dk, *kt = k + bh * Dk, *vt = v + bh * Dv;
            double *ot = o + bh * Dv;
            for (int i = 0; i < Dk; ++i)
                for (int j = 0; j < Dv; ++j) S[(size_t)i * Dv + j] = lam[h] * S[(size_t)i * Dv + j] + kt[i] * vt[j];
            for (int j = 0; j < Dv; ++j) ot[j] = 0.0;
            for (int i = 0; i < Dk; ++i)
                for (int j = 0; j < Dv; ++j) ot[j] += qt[i] * S[(size_t)i * Dv + j];
        }
    return 0;
}

/*
 * Backward pass (gradients of the operator). With the loss's gradients dO
 * (one per output) and dS_N (of the final state, or zero), the recurrence
 * S_t = lambda S_{t-1} + k_t^T v_t, o_t = q_t S_t has the adjoint
 *
 *     dq_t = S_t dO_t                         (dq_t[i] = sum_j S_t[i][j] dO_t[j]),
 *     G_t  = q_t^T dO_t + lambda G_{t+1},     G_N-1 also gets dS_N,
 *     dk_t = G_t v_t,  dv_t = k_t G_t,        dS_0 = lambda G_0,
 *
 * G_t being the gradient with respect to S_t. The pages do not treat the
 * backward pass; this is the derivative of the recurrent form above, step by
 * step (a forward sweep for dq, a reverse sweep for dk, dv and dS_0).
 */
typedef struct {
    const double *q, *k, *v, *dout;
    double *dq, *dk, *dv;
    const int64_t *cu;
    int nseq, H, Dk, Dv;
    const double *lam;
    const double *s0, *dsN;
    double *ds0;
    int64_t next;
    pthread_mutex_t mu;
} bwd_job;

static void bwd_one(const bwd_job *J, int seq, int h, double *S) {
    const int H = J->H, Dk = J->Dk, Dv = J->Dv;
    const double lam = J->lam[h];
    const size_t ss = (size_t)Dk * Dv;
    /* forward sweep: dq_t = S_t dO_t */
    if (J->s0) memcpy(S, J->s0 + ((size_t)seq * H + h) * ss, ss * sizeof(double));
    else memset(S, 0, ss * sizeof(double));
    for (int64_t t = J->cu[seq]; t < J->cu[seq + 1]; ++t) {
        const double *kt = J->k + ((size_t)t * H + h) * Dk;
        const double *vt = J->v + ((size_t)t * H + h) * Dv;
        const double *gt = J->dout + ((size_t)t * H + h) * Dv;
        double *dqt = J->dq + ((size_t)t * H + h) * Dk;
        for (int i = 0; i < Dk; ++i)
            for (int j = 0; j < Dv; ++j) S[(size_t)i * Dv + j] = lam * S[(size_t)i * Dv + j] + kt[i] * vt[j];
        for (int i = 0; i < Dk; ++i) {
            double acc = 0.0;
            for (int j = 0; j < Dv; ++j) acc += S[(size_t)i * Dv + j] * gt[j];
            dqt[i] = acc;
        }
    }
    /* reverse sweep: G accumulates q_t^T dO_t, then gives dk_t and dv_t, then decays */
    if (J->dsN) memcpy(S, J->dsN + ((size_t)seq * H + h) * ss, ss * sizeof(double));
    else memset(S, 0, ss * sizeof(double));
    for (int64_t t = J->cu[seq + 1] - 1; t >= J->cu[seq]; --t) {
        const double *qt = J->q + ((size_t)t * H + h) * Dk;
        const double *kt = J->k + ((size_t)t * H + h) * Dk;
        const double *vt = J->v + ((size_t)t * H + h) * Dv;
        const double *gt = J->dout + ((size_t)t * H + h) * Dv;
        double *dkt = J->dk + ((size_t)t * H + h) * Dk;
        double *dvt = J->dv + ((size_t)t * H + h) * Dv;
        for (int i = 0; i < Dk; ++i)
            for (int j = 0; j < Dv; ++j) S[(size_t)i * Dv + j] += qt[i] * gt[j];
        for (int i = 0; i < Dk; ++i) {
            double acc = 0.0;
            for (int j = 0; j < Dv; ++j) acc += S[(size_t)i * Dv + j] * vt[j];
            dkt[i] = acc;
        }
        for (int j = 0; j < Dv; ++j) dvt[j] = 0.0;
        for (int i = 0; i < Dk; ++i)
            for (int j = 0; j < Dv; ++j) dvt[j] += kt[i] * S[(size_t)i * Dv + j];
        for (size_t e = 0; e < ss; ++e) S[e] *= lam;
    }
    if (J->ds0) memcpy(J->ds0 + ((size_t)seq * H + h) * ss, S, ss * sizeof(double));
}

static void *bwd_worker(void *arg) {
    bwd_job *J = (bwd_job *)arg;
    double *S = (double *)malloc((size_t)J->Dk * J->Dv * sizeof(double));
    if (!S) return (void *)1;
    const int64_t total = (int64_t)J->nseq * J->H;
    for (;;) {
        pthread_mutex_lock(&J->mu);
        int64_t u = J->next++;
        pthread_mutex_unlock(&J->mu);
        if (u >= total) break;
        bwd_one(J, (int)(u / J->H), (int)(u % J->H), S);
    }
    free(S);
    return NULL;
}

/*
 * Gradients over packed sequences: dq, dk [T, H, Dk]; dv [T, H, Dv] from dout
 * [T, H, Dv]. initial_state (the forward's S0), d_final_state (dS_N) and
 * d_initial_state (dS_0, output) may each be NULL; d_initial_state may alias
 * d_final_state. Returns 0, -1 on bad arguments, -2 on allocation / thread
 * failure.
 */
int la_oracle_prefill_backward_recurrent(const double *q, const double *k, const double *v, const double *dout,
                                         double *dq, double *dk, double *dv, const int64_t *cu_seqlens, int nseq,
                                         int H, int Dk, int Dv, const double *lam, const double *initial_state,
                                         const double *d_final_state, double *d_initial_state, int nthreads) {
    if (!q || !k || !v || !dout || !dq || !dk || !dv || !cu_seqlens || !lam || nseq < 1 || H < 1 || Dk < 1 ||
        Dv < 1)
        return -1;
    if (cu_seqlens[0] != 0) return -1;
    for (int i = 0; i < nseq; ++i)
        if (cu_seqlens[i + 1] < cu_seqlens[i]) return -1;
    bwd_job J = {q, k, v, dout, dq, dk, dv, cu_seqlens, nseq, H, Dk, Dv, lam, initial_state, d_final_state,
                 d_initial_state, 0, PTHREAD_MUTEX_INITIALIZER};
    if (nthreads <= 0) nthreads = la_oracle_default_threads();
    const int64_t total = (int64_t)nseq * H;
    if (nthreads > total) nthreads = (int)total;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) return -2;
    int started = 0, rc = 0;
    for (; started < nthreads; ++started)
        if (pthread_create(&th[started], NULL, bwd_worker, &J) != 0) break;
    if (started == 0) rc = (int)(intptr_t)bwd_worker(&J) ? -2 : 0;
    for (int i = 0; i < started; ++i) {
        void *r = NULL;
        pthread_join(th[i], &r);
        if (r) rc = -2;
    }
    free(th);
    return rc;
}
