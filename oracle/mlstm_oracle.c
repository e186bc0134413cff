/*
 * mLSTM / retention sequential recurrence in fp64 -- TEST INFRASTRUCTURE ONLY.
 *
 * This file is the oracle: a plain, slow, obviously correct CPU statement of
 * what the GPU path computes.  Only tests, the smoke check and the benchmark's
 * CPU-baseline leg may load it.  It shares no code, header or constant with the
 * CUDA library and must never be reached from the product path.
 *
 * What it computes (one token at a time, per (batch, head, block) slice):
 *
 *   mLSTM matrix memory, DeepChrInteract-v2 "mLSTM Model", "Core idea":
 *       C_t = f_t C_{t-1} + i_t (v_t outer k_t)
 *   with the normaliser n_t = f_t n_{t-1} + i_t k_t and the read-out
 *       h_t = o_t * (C_t q_t) / max(|n_t . q_t|, 1),
 *   an exponential input gate i_t = exp(itilde_t), a log-sigmoid forget gate
 *   log f_t = logsigmoid(ftilde_t), and the gates "stabilized in log space"
 *   ("Core idea", same page) by the running maximum
 *       m_t = max(log f_t + m_{t-1}, log i_t).
 *   The state is carried in stabilised units C'_t = C_t e^{-m_t},
 *   n'_t = n_t e^{-m_t}; the floor 1 on |n . q| becomes e^{-m_t} in those units,
 *   so the stabiliser never changes h.
 *
 *   Block-diagonal memory, Edifice.Recurrent.XLSTMv2, "Key Improvements" #1:
 *   each head's q, k, v are split into num_blocks contiguous slices; block j
 *   has its own C_j [dv/nb x dk/nb] and n_j, and shares the head's gates and m.
 *
 *   Retention, Edifice.Attention.RetNet, "Key Innovation" (recurrent form)
 *   and "Multi-Scale Retention": s_n = gamma s_{n-1} + K_n^T V_n, o_n = Q_n s_n
 *   with gamma_h = 1 - 2^(-5-h) for head h (0-based).  Stored here as C = s^T,
 *   i.e. C_t = gamma C_{t-1} + v_t k_t^T and h_t = C_t q_t (no normaliser,
 *   no stabiliser, no gates).
 *
 * Layouts (row-major, last index fastest):
 *   q, k [B,NH,S,DHQK]   v, o, h [B,NH,S,DHV]   igate, fgate [B,NH,S]
 *   C [B,NH,nb,DHV/nb,DHQK/nb] (value row, key column)   n [B,NH,nb,DHQK/nb]   m [B,NH]
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int B, NH, S, DHQK, DHV, nb, retention;
    const double *q, *k, *v, *ig, *fg, *og, *C0, *n0, *m0;
    double *h, *C, *n, *m;
    int n_slices, next_stride, first;
} job_t;

/* log(sigmoid(x)) written in the form that cannot overflow. */
static double log_sigmoid(double x) {
    return (x < 0.0 ? x : 0.0) - log1p(exp(-fabs(x)));
}

static void run_slice(const job_t* J, int slice) {
    const int nb = J->nb, dk = J->DHQK / nb, dv = J->DHV / nb, S = J->S;
    const int blk = slice % nb, bh = slice / nb, head = bh % J->NH;
    double* C = (double*)malloc(sizeof(double) * (size_t)dv * dk);
    double* n = (double*)malloc(sizeof(double) * (size_t)dk);
    double m = 0.0;
    size_t c_off = ((size_t)bh * nb + blk) * (size_t)dv * dk;
    size_t n_off = ((size_t)bh * nb + blk) * (size_t)dk;
    for (size_t i = 0; i < (size_t)dv * dk; ++i) C[i] = J->C0 ? J->C0[c_off + i] : 0.0;
    for (int i = 0; i < dk; ++i) n[i] = J->n0 ? J->n0[n_off + i] : 0.0;
    if (J->m0) m = J->m0[bh];
    const double gamma = 1.0 - ldexp(1.0, -5 - head);

    for (int t = 0; t < S; ++t) {
        const size_t tok = (size_t)bh * S + t;
        const double* qt = J->q + tok * J->DHQK + (size_t)blk * dk;
        const double* kt = J->k + tok * J->DHQK + (size_t)blk * dk;
        const double* vt = J->v + tok * J->DHV + (size_t)blk * dv;
        double* ht = J->h + tok * J->DHV + (size_t)blk * dv;
        double fprime, iprime;
        if (J->retention) {
            fprime = gamma;
            iprime = 1.0;
        } else {
            const double lf = log_sigmoid(J->fg[tok]);
            const double li = J->ig[tok];
            const double m_new = (lf + m > li) ? lf + m : li;
            fprime = exp(lf + m - m_new);
            iprime = exp(li - m_new);
            m = m_new;
        }
        /* C' <- f' C' + i' v k^T ; n' <- f' n' + i' k */
        for (int r = 0; r < dv; ++r)
            for (int c = 0; c < dk; ++c)
                C[(size_t)r * dk + c] = fprime * C[(size_t)r * dk + c] + iprime * vt[r] * kt[c];
        double nq = 0.0;
        if (!J->retention) {
            for (int c = 0; c < dk; ++c) {
                n[c] = fprime * n[c] + iprime * kt[c];
                nq += n[c] * qt[c];
            }
        }
        const double den = J->retention ? 1.0 : fmax(fabs(nq), exp(-m));
        for (int r = 0; r < dv; ++r) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += C[(size_t)r * dk + c] * qt[c];
            double o = (J->og && !J->retention) ? J->og[tok * J->DHV + (size_t)blk * dv + r] : 1.0;
            ht[r] = o * acc / den;
        }
    }
    if (J->C) memcpy(J->C + c_off, C, sizeof(double) * (size_t)dv * dk);
    if (J->n && !J->retention) memcpy(J->n + n_off, n, sizeof(double) * (size_t)dk);
    if (J->m && !J->retention && blk == 0) J->m[bh] = m;
    free(C);
    free(n);
}

static void* worker(void* arg) {
    job_t* J = (job_t*)arg;
    for (int s = J->first; s < J->n_slices; s += J->next_stride) run_slice(J, s);
    return NULL;
}

/*
 * Runs the recurrence over every (b, h, block) slice.  Pointers o, C0, n0, m0
 * may be NULL (o = 1, zero initial state, m0 = 0).  C, n, m may be NULL (not
 * written).  In retention mode ig, fg, o, n0, m0, n, m are ignored.
 * Returns 0 on success, -1 on a bad shape.
 */
int oracle_mlstm_sequential(int B, int NH, int S, int DHQK, int DHV, int nb, int retention,
                            const double* q, const double* k, const double* v,
                            const double* ig, const double* fg, const double* og,
                            const double* C0, const double* n0, const double* m0,
                            double* h, double* C, double* n, double* m, int nthreads) {
    if (B < 0 || NH < 0 || S < 0 || nb <= 0 || DHQK % nb || DHV % nb) return -1;
    if (!retention && S > 0 && (!ig || !fg)) return -1;
    job_t base = {B, NH, S, DHQK, DHV, nb, retention, q, k, v, ig, fg, og, C0, n0, m0,
                  h, C, n, m, B * NH * nb, 1, 0};
    if (nthreads < 1) nthreads = 1;
    if (nthreads > base.n_slices) nthreads = base.n_slices > 0 ? base.n_slices : 1;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
    job_t* jobs = (job_t*)malloc(sizeof(job_t) * nthreads);
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = base;
        jobs[i].first = i;
        jobs[i].next_stride = nthreads;
        pthread_create(&th[i], NULL, worker, &jobs[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    free(jobs);
    return 0;
}
