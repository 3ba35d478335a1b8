/*
 * ssd_oracle.c -- plain, slow, fp64 CPU oracle for the selective state-space
 * recurrence.  TEST INFRASTRUCTURE ONLY: nothing in the product path may link,
 * load or call this file.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference arm of bench.py use it.
 *
 * What it computes (and where that is defined):
 *   - The recurrence h_t = Abar_t h_{t-1} + Bbar_t x_t  ("5.3 Tensor Parallelism
 *     support and large-cluster training", section 2.1).
 *   - A_t = a_t * I: one scalar decay per (token, head), shared by all N state
 *     dimensions (same page, section 3.1).
 *   - Discretisation Abar_t = exp(d_t * A_h), Bbar_t = d_t * B_t with
 *     d_t = softplus(dt_t + dt_bias_h); output y_t = C_t^T h_t + D_h x_t.  The
 *     page leaves Abar/Bbar symbolic; this is the plain reading adopted for the
 *     whole library (Euler step on B, exact exponential on A).
 *   - State of size N x P per head (same page, section 3.2), stored row-major
 *     (n, p).
 *   - Packed variable-length input: at the first token of every packed sequence
 *     the carried state is forgotten (the page's "A_t = 0" reset, section 4.3,
 *     read as the discrete multiplier Abar = 0) and replaced by that sequence's
 *     own initial state (zero when none is given).
 *   - The state carried from prefill into decode ("Scaling State-Space Models on
 *     Multiple GPUs with Tensor Parallelism", abstract): oracle_state_update is
 *     one step of the same recurrence applied to a cached state.
 *
 * Everything is a literal token-by-token loop in double precision.  There is
 * no chunking, blocking or reordering: the oracle is the definition.
 *
 * Parity pins (tests/test_oracle.py) tie it to things other than itself: a
 * hand-derived worked example, closed forms (L = 1, A = 0 cumulative sum,
 * constant-input geometric series), the brute-force materialised
 * semiseparable matrix, the independently written block-decomposed form, and
 * invariants (state-cache continuation, packing = separate runs, causality,
 * linearity, group replication).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* softplus(z) = log(1 + e^z), evaluated without overflow. */
double oracle_softplus(double z) {
    if (z > 0.0) return z + log1p(exp(-z));
    return log1p(exp(z));
}

typedef struct {
    int64_t batch, seqlen, nheads, headdim, dstate, ngroups, nseqs;
    const double *x, *dt, *dt_bias, *A, *B, *C, *D, *init_state;
    const int32_t *seq_idx;
    double *y, *final_state;
    /* work distribution */
    int64_t n_items;
    int64_t next_item;
    pthread_mutex_t lock;
} scan_job;

/* One work item = (batch row or packed sequence, head).  The token range is
 * [t0, t1) of batch row `row`; `s` indexes init_state/final_state. */
static void run_item(scan_job *j, int64_t item, double *state) {
    const int64_t H = j->nheads, P = j->headdim, N = j->dstate, G = j->ngroups;
    const int64_t L = j->seqlen;
    const int64_t heads_per_group = H / G;
    const int64_t h = item % H;
    const int64_t s = item / H;
    const int64_t g = h / heads_per_group;
    int64_t row, t0, t1;
    if (j->seq_idx) {
        /* packed: batch == 1, sequence s = the run of tokens with seq_idx == s */
        row = 0;
        t0 = 0;
        while (t0 < L && j->seq_idx[t0] != s) t0++;
        t1 = t0;
        while (t1 < L && j->seq_idx[t1] == s) t1++;
    } else {
        row = s;
        t0 = 0;
        t1 = L;
    }
    const double bias = j->dt_bias ? j->dt_bias[h] : 0.0;
    const double Ah = j->A[h];
    const double Dh = j->D ? j->D[h] : 0.0;

    /* h_{-1}: the sequence's own initial state, or zero. */
    if (j->init_state) {
        memcpy(state, j->init_state + (s * H + h) * N * P, sizeof(double) * N * P);
    } else {
        memset(state, 0, sizeof(double) * N * P);
    }
    for (int64_t t = t0; t < t1; ++t) {
        const int64_t tok = row * L + t;
        const double d = oracle_softplus(j->dt[tok * H + h] + bias);
        const double decay = exp(d * Ah);
        const double *xt = j->x + (tok * H + h) * P;
        const double *Bt = j->B + (tok * G + g) * N;
        const double *Ct = j->C + (tok * G + g) * N;
        double *yt = j->y + (tok * H + h) * P;
        /* h_t = exp(d A) h_{t-1} + d B_t x_t^T */
        for (int64_t n = 0; n < N; ++n) {
            const double dB = d * Bt[n];
            double *hn = state + n * P;
            for (int64_t p = 0; p < P; ++p) hn[p] = decay * hn[p] + dB * xt[p];
        }
        /* y_t = C_t^T h_t + D x_t */
        for (int64_t p = 0; p < P; ++p) yt[p] = Dh * xt[p];
        for (int64_t n = 0; n < N; ++n) {
            const double c = Ct[n];
            const double *hn = state + n * P;
            for (int64_t p = 0; p < P; ++p) yt[p] += c * hn[p];
        }
    }
    if (j->final_state) {
        memcpy(j->final_state + (s * H + h) * N * P, state, sizeof(double) * N * P);
    }
}

static void *worker(void *arg) {
    scan_job *j = (scan_job *)arg;
    double *state = (double *)malloc(sizeof(double) * j->dstate * j->headdim);
    if (!state) return (void *)1;
    for (;;) {
        pthread_mutex_lock(&j->lock);
        int64_t item = j->next_item++;
        pthread_mutex_unlock(&j->lock);
        if (item >= j->n_items) break;
        run_item(j, item, state);
    }
    free(state);
    return NULL;
}

/* Validates the packed-sequence index: starts at 0, steps of 0 or +1, ends at
 * nseqs - 1.  Returns 0 when valid. */
static int check_seq_idx(const int32_t *seq_idx, int64_t L, int64_t nseqs) {
    if (L == 0) return nseqs == 0 ? 0 : -1;
    if (seq_idx[0] != 0) return -1;
    for (int64_t t = 1; t < L; ++t) {
        int32_t step = seq_idx[t] - seq_idx[t - 1];
        if (step != 0 && step != 1) return -1;
    }
    return seq_idx[L - 1] == nseqs - 1 ? 0 : -1;
}

/*
 * Full-sequence scan.  Layouts (row-major, all double unless noted):
 *   x (batch, seqlen, nheads, headdim); dt (batch, seqlen, nheads);
 *   dt_bias (nheads) or NULL; A (nheads); B, C (batch, seqlen, ngroups, dstate);
 *   D (nheads) or NULL; init_state (S, nheads, dstate, headdim) or NULL;
 *   seq_idx int32 (seqlen) with batch == 1, or NULL;
 *   y (batch, seqlen, nheads, headdim); final_state (S, ...) or NULL.
 *   S = nseqs when seq_idx is given, else batch.
 * Returns 0 on success, -1 on invalid arguments, -2 on allocation failure.
 */
int oracle_ssd_scan(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                    int64_t dstate, int64_t ngroups, int64_t nseqs,
                    const double *x, const double *dt, const double *dt_bias,
                    const double *A, const double *B, const double *C, const double *D,
                    const double *init_state, const int32_t *seq_idx,
                    double *y, double *final_state, int nthreads) {
    if (batch < 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 ||
        ngroups <= 0 || nheads % ngroups != 0)
        return -1;
    if (!A || (batch * seqlen > 0 && (!x || !dt || !B || !C || !y))) return -1;
    int64_t S = batch;
    if (seq_idx) {
        if (batch != 1) return -1;
        if (check_seq_idx(seq_idx, seqlen, nseqs) != 0) return -1;
        S = nseqs;
    }
    scan_job j;
    memset(&j, 0, sizeof(j));
    j.batch = batch; j.seqlen = seqlen; j.nheads = nheads; j.headdim = headdim;
    j.dstate = dstate; j.ngroups = ngroups; j.nseqs = nseqs;
    j.x = x; j.dt = dt; j.dt_bias = dt_bias; j.A = A; j.B = B; j.C = C; j.D = D;
    j.init_state = init_state; j.seq_idx = seq_idx; j.y = y; j.final_state = final_state;
    j.n_items = S * nheads;
    j.next_item = 0;
    pthread_mutex_init(&j.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > j.n_items) nthreads = (int)(j.n_items > 0 ? j.n_items : 1);
    int rc = 0;
    pthread_t *tids = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    if (!tids) { pthread_mutex_destroy(&j.lock); return -2; }
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (pthread_create(&tids[i], NULL, worker, &j) != 0) break;
        started++;
    }
    if (started == 0) { worker(&j); }
    for (int i = 0; i < started; ++i) {
        void *ret = NULL;
        pthread_join(tids[i], &ret);
        if (ret) rc = -2;
    }
    free(tids);
    pthread_mutex_destroy(&j.lock);
    return rc;
}

/*
 * One decode step on a cached state, in place (the prefill -> decode state
 * cache).  state (batch, nheads, dstate, headdim); x (batch, nheads, headdim);
 * dt (batch, nheads); B, C (batch, ngroups, dstate); y (batch, nheads, headdim).
 */
int oracle_state_update(int64_t batch, int64_t nheads, int64_t headdim, int64_t dstate,
                        int64_t ngroups, double *state, const double *x, const double *dt,
                        const double *dt_bias, const double *A, const double *B,
                        const double *C, const double *D, double *y) {
    if (batch < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0 ||
        nheads % ngroups != 0)
        return -1;
    const int64_t H = nheads, P = headdim, N = dstate, G = ngroups;
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            const int64_t g = h / (H / G);
            const double d = oracle_softplus(dt[b * H + h] + (dt_bias ? dt_bias[h] : 0.0));
            const double decay = exp(d * A[h]);
            const double *xt = x + (b * H + h) * P;
            const double *Bt = B + (b * G + g) * N;
            const double *Ct = C + (b * G + g) * N;
            double *st = state + (b * H + h) * N * P;
            double *yt = y + (b * H + h) * P;
            for (int64_t n = 0; n < N; ++n)
                for (int64_t p = 0; p < P; ++p)
                    st[n * P + p] = decay * st[n * P + p] + d * Bt[n] * xt[p];
            for (int64_t p = 0; p < P; ++p) {
                double acc = (D ? D[h] : 0.0) * xt[p];
                for (int64_t n = 0; n < N; ++n) acc += Ct[n] * st[n * P + p];
                yt[p] = acc;
            }
        }
    }
    return 0;
}
