/*
 * Lightning-attention oracle: plain, slow, fp64 CPU implementation.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the test suite, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header or constant with the CUDA path.
 *
 * What it computes (MiniMax-01 "Scaling Foundation Models with Lightning
 * Attention", as summarised by the CSDN digest, section 2.1, and the mizuki
 * blog, appendix "key concepts"): causal linear attention in the
 * NormAttention style -- no softmax, no denominator, no feature map -- for each
 * packed sequence s, head h and position i of s:
 *
 *     O[i]  = sum_{j <= i, j in s} (q_i . k_j) v_j              (quadratic form)
 *           = q_i^T KV_i,  KV_i = KV_{i-1} + k_i v_i^T,  KV = 0 at start(s)
 *                                                           (recurrent form)
 *     y[i]  = O[i] / sqrt(mean_d O[i]_d^2 + eps)      (optional output RMSNorm)
 *     state = KV_end(s) = K_s^T V_s
 *
 * and the block-tiled evaluation that the pages call lightning attention
 * (intra-block masked left product plus inter-block right product, CSDN
 * digest section 2.1; mizuki blog appendix): per block b of size beta,
 *     O_b = [(Q_b K_b^T) (.) M] V_b + Q_b KV,   then   KV += K_b^T V_b.
 *
 * Decode (jvyan.cn article, section 2 "compute optimisation": length-1
 * requests get their own kernel): KV <- KV + k v^T, then o = q^T KV.  The
 * readout includes the current token, matching the causal diagonal j <= i.
 *
 * Initial state (optional, state_in != NULL): a sequence may continue from a
 * state X = KV at its start instead of 0, as a chunk of a longer sequence does
 * (LASP+: local prefix sums of the chunk states, all-gathered, after which each
 * chunk runs from the sum of the states before it -- mizuki blog, section 5
 * "pretraining" and appendix "key concepts"; jvyan.cn article, section 3).  Then
 *     O[i]  = q_i^T X + sum_{j <= i, j in s} (q_i . k_j) v_j,
 *     KV_{start(s)-1} = X,   state = X + K_s^T V_s.
 *
 * Layouts: q, k, v, o are [T][H][D] fp64 row-major (T = total tokens).
 * cu[] has S+1 non-decreasing entries from 0 to T; sequence s owns tokens
 * cu[s] .. cu[s+1]-1.  state is [S][H][D][D] with state[s][h][r][c] =
 * sum_t k_t[r] v_t[c].  Work is split over (sequence, head) pairs with pthreads;
 * each pair is computed by one thread in the plain loop order written below.
 *
 * All functions return 0 on success and a negative value on a bad argument.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* LA_ORACLE_MUTANT selects a deliberately wrong variant (0 = the oracle).  It
 * exists only so that the test suite can show that its pins catch plausible
 * mistakes; the shipped build always uses 0. */
#ifndef LA_ORACLE_MUTANT
#define LA_ORACLE_MUTANT 0
#endif
#define MUT(n) (LA_ORACLE_MUTANT == (n))

typedef struct {
    const double *q, *k, *v;
    double *o;      /* may be NULL (state only) */
    double *state;  /* may be NULL */
    const double *state_in; /* decode: input state (may alias state); prefill: initial
                               state per (sequence, head), or NULL for zero */
    int64_t T;
    int H, D, S;
    const int64_t *cu;
    int rmsnorm;
    double eps;
    int beta;
    int form;       /* 0 quadratic, 1 recurrent, 2 blocked, 3 decode */
    int64_t njobs;
    int64_t next;   /* shared job counter */
} job_t;

static inline const double *row(const double *x, int64_t t, int h, int H, int D) {
    return x + ((size_t)t * (size_t)H + (size_t)h) * (size_t)D;
}
static inline double *rowm(double *x, int64_t t, int h, int H, int D) {
    return x + ((size_t)t * (size_t)H + (size_t)h) * (size_t)D;
}

static double dot(const double *a, const double *b, int D) {
    double s = 0.0;
    for (int d = 0; d < D; ++d) s += a[d] * b[d];
    return s;
}

/* y = x / sqrt(mean(x^2) + eps), in place. */
static void rmsnorm_row(double *x, int D, double eps) {
    double ss = 0.0;
    for (int d = 0; d < D; ++d) ss += x[d] * x[d];
    double r = MUT(2) ? sqrt(ss / (double)D) + eps : MUT(8) ? sqrt(ss + eps) : sqrt(ss / (double)D + eps);
    for (int d = 0; d < D; ++d) x[d] = x[d] / r;
}

/* KV = X (an initial state), D x D row-major. */
static void init_state(double *KV, const double *X, int D) {
    for (int r = 0; r < D; ++r)
        for (int c = 0; c < D; ++c)
            KV[(size_t)r * D + c] = MUT(10) ? X[(size_t)c * D + r] : X[(size_t)r * D + c];
}

/* Quadratic masked form: O = [(Q K^T) (.) M] V, one row at a time. */
static void run_quadratic(const job_t *J, int s, int h) {
    const int H = J->H, D = J->D;
    const int64_t a = J->cu[s], b = J->cu[s + 1];
    const double *X = J->state_in ? J->state_in + ((size_t)s * H + h) * (size_t)D * D : NULL;
    for (int64_t i = a; i < b; ++i) {
        double *oi = rowm(J->o, i, h, H, D);
        for (int d = 0; d < D; ++d) oi[d] = 0.0;
        const double *qi = row(J->q, i, h, H, D);
        for (int64_t j = a; MUT(1) ? j < i : j <= i; ++j) {
            double w = dot(qi, row(J->k, j, h, H, D), D);
            const double *vj = row(J->v, j, h, H, D);
            for (int d = 0; d < D; ++d) oi[d] += w * vj[d];
        }
        if (X && !MUT(9))                                /* + q_i^T X */
            for (int c = 0; c < D; ++c)
                for (int r = 0; r < D; ++r) oi[c] += qi[r] * X[(size_t)r * D + c];
        if (J->rmsnorm) rmsnorm_row(oi, D, J->eps);
    }
    if (J->state) {
        double *st = J->state + ((size_t)s * H + h) * (size_t)D * D;
        for (int r = 0; r < D * D; ++r) st[r] = X && !MUT(11) ? X[r] : 0.0;
        for (int64_t j = a; j < b; ++j) {
            const double *kj = row(J->k, j, h, H, D), *vj = row(J->v, j, h, H, D);
            for (int r = 0; r < D; ++r)
                for (int c = 0; c < D; ++c) st[(size_t)r * D + c] += kj[r] * vj[c];
        }
    }
}

/* Token-by-token recurrent form: KV += k v^T, then o = q^T KV. */
static void run_recurrent(const job_t *J, int s, int h) {
    const int H = J->H, D = J->D;
    const int64_t a = J->cu[s], b = J->cu[s + 1];
    double *KV = (double *)calloc((size_t)D * D, sizeof(double));
    if (J->state_in)                                     /* KV_{start-1} = X */
        init_state(KV, J->state_in + ((size_t)s * H + h) * (size_t)D * D, D);
    for (int64_t i = a; i < b; ++i) {
        const double *ki = row(J->k, i, h, H, D), *vi = row(J->v, i, h, H, D);
        if (!MUT(5))
            for (int r = 0; r < D; ++r)
                for (int c = 0; c < D; ++c) KV[(size_t)r * D + c] += ki[r] * vi[c];
        if (J->o) {
            const double *qi = row(J->q, i, h, H, D);
            double *oi = rowm(J->o, i, h, H, D);
            for (int c = 0; c < D; ++c) {
                double acc = 0.0;
                for (int r = 0; r < D; ++r)
                    acc += qi[r] * (MUT(3) ? KV[(size_t)c * D + r] : KV[(size_t)r * D + c]);
                oi[c] = acc;
            }
            if (J->rmsnorm) rmsnorm_row(oi, D, J->eps);
        }
        if (MUT(5))
            for (int r = 0; r < D; ++r)
                for (int c = 0; c < D; ++c) KV[(size_t)r * D + c] += ki[r] * vi[c];
    }
    if (J->state) memcpy(J->state + ((size_t)s * H + h) * (size_t)D * D, KV,
                         (size_t)D * D * sizeof(double));
    free(KV);
}

/* Block-tiled form: intra-block masked left product, inter-block right
 * product with the running state, then the state update with the block. */
static void run_blocked(const job_t *J, int s, int h) {
    const int H = J->H, D = J->D, beta = J->beta;
    const int64_t a = J->cu[s], b = J->cu[s + 1];
    double *KV = (double *)calloc((size_t)D * D, sizeof(double));
    if (J->state_in)                                     /* KV before the first block = X */
        init_state(KV, J->state_in + ((size_t)s * H + h) * (size_t)D * D, D);
    double *intra = (double *)malloc((size_t)D * sizeof(double));
    double *inter = (double *)malloc((size_t)D * sizeof(double));
    for (int64_t p = a; p < b; p += beta) {
        int64_t e = p + beta < b ? p + beta : b;
        for (int64_t i = p; i < e; ++i) {
            const double *qi = row(J->q, i, h, H, D);
            for (int d = 0; d < D; ++d) intra[d] = 0.0;
            for (int64_t j = MUT(7) ? a : p; j <= i; ++j) { /* mask M: j <= i, same block */
                double w = dot(qi, row(J->k, j, h, H, D), D);
                const double *vj = row(J->v, j, h, H, D);
                for (int d = 0; d < D; ++d) intra[d] += w * vj[d];
            }
            for (int c = 0; c < D; ++c) {               /* Q_b . KV (previous blocks) */
                double acc = 0.0;
                for (int r = 0; r < D; ++r) acc += qi[r] * KV[(size_t)r * D + c];
                inter[c] = acc;
            }
            double *oi = rowm(J->o, i, h, H, D);
            for (int d = 0; d < D; ++d) oi[d] = MUT(4) ? intra[d] : intra[d] + inter[d];
            if (J->rmsnorm) rmsnorm_row(oi, D, J->eps);
        }
        for (int64_t j = p; j < e; ++j) {               /* KV += K_b^T V_b */
            const double *kj = row(J->k, j, h, H, D), *vj = row(J->v, j, h, H, D);
            for (int r = 0; r < D; ++r)
                for (int c = 0; c < D; ++c) KV[(size_t)r * D + c] += kj[r] * vj[c];
        }
    }
    if (J->state) memcpy(J->state + ((size_t)s * H + h) * (size_t)D * D, KV,
                         (size_t)D * D * sizeof(double));
    free(KV);
    free(intra);
    free(inter);
}

/* One decode step for sequence (slot) s, head h: q,k,v,o are [S][H][D]. */
static void run_decode(const job_t *J, int s, int h) {
    const int H = J->H, D = J->D;
    const size_t off = ((size_t)s * H + h) * (size_t)D * D;
    const double *KV0 = J->state_in + off;
    double *KV = J->state + off;
    const double *qi = row(J->q, s, h, H, D), *ki = row(J->k, s, h, H, D),
                 *vi = row(J->v, s, h, H, D);
    double *oi = rowm(J->o, s, h, H, D);
    if (MUT(6))
        for (int c = 0; c < D; ++c) {
            double acc = 0.0;
            for (int r = 0; r < D; ++r) acc += qi[r] * KV0[(size_t)r * D + c];
            oi[c] = acc;
        }
    for (int r = 0; r < D; ++r)
        for (int c = 0; c < D; ++c) KV[(size_t)r * D + c] = KV0[(size_t)r * D + c] + ki[r] * vi[c];
    if (!MUT(6))
        for (int c = 0; c < D; ++c) {
            double acc = 0.0;
            for (int r = 0; r < D; ++r) acc += qi[r] * KV[(size_t)r * D + c];
            oi[c] = acc;
        }
    if (J->rmsnorm) rmsnorm_row(oi, D, J->eps);
}

static void *worker(void *arg) {
    job_t *J = (job_t *)arg;
    for (;;) {
        int64_t jid = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (jid >= J->njobs) break;
        int s = (int)(jid / J->H), h = (int)(jid % J->H);
        switch (J->form) {
            case 0: run_quadratic(J, s, h); break;
            case 1: run_recurrent(J, s, h); break;
            case 2: run_blocked(J, s, h); break;
            default: run_decode(J, s, h); break;
        }
    }
    return NULL;
}

static int run_all(job_t *J, int nthreads) {
    J->njobs = (int64_t)J->S * J->H;
    J->next = 0;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if ((int64_t)nthreads > J->njobs) nthreads = (int)(J->njobs > 0 ? J->njobs : 1);
    pthread_t tid[256];
    int started = 0;
    for (int t = 1; t < nthreads; ++t)
        if (pthread_create(&tid[started], NULL, worker, J) == 0) ++started;
    worker(J);
    for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
    return 0;
}

static int check_cu(const int64_t *cu, int S, int64_t T) {
    if (!cu || S < 0) return -1;
    if (cu[0] != 0 || cu[S] != T) return -1;
    for (int s = 0; s < S; ++s)
        if (cu[s + 1] < cu[s]) return -1;
    return 0;
}

int la_oracle_prefill(int form, const double *q, const double *k, const double *v, double *o,
                      double *state, const double *state_in, int64_t T, int H, int D,
                      const int64_t *cu, int S, int beta, int rmsnorm, double eps, int nthreads) {
    if (H < 1 || D < 1 || T < 0 || form < 0 || form > 2) return -1;
    if (check_cu(cu, S, T)) return -2;
    if (form == 2 && beta < 1) return -3;
    if (!q || !k || !v) return -4;
    if (!o && form != 1) return -4;
    job_t J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v; J.o = o; J.state = state; J.state_in = state_in;
    J.T = T; J.H = H; J.D = D; J.S = S; J.cu = cu;
    J.rmsnorm = rmsnorm; J.eps = eps; J.beta = beta; J.form = form;
    return run_all(&J, nthreads);
}

int la_oracle_decode_step(const double *q, const double *k, const double *v,
                          const double *state_in, double *state_out, double *o,
                          int B, int H, int D, int rmsnorm, double eps, int nthreads) {
    if (B < 0 || H < 1 || D < 1 || !q || !k || !v || !state_in || !state_out || !o) return -1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v; J.o = o; J.state = state_out; J.state_in = state_in;
    J.H = H; J.D = D; J.S = B; J.rmsnorm = rmsnorm; J.eps = eps; J.form = 3;
    return run_all(&J, nthreads);
}
