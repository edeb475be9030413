/*
 * mlstm_oracle.c -- plain fp64 CPU oracle of the mLSTM matrix-memory cell.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path (the CUDA library,
 * its Python binding) may include, link or call this file.  Only the tests,
 * the smoke check and the CPU-baseline leg of the benchmark use it.  It shares
 * no code, header, table or helper with the CUDA kernels.
 *
 * What it computes (one head at a time, token by token, no chunking, no
 * reordering):
 *
 *   log f_t = logsigmoid(f~_t)                 forget gate kept in log space
 *   m_t     = max(log f_t + m_{t-1}, i~_t)     stabilizer state
 *   f'_t    = exp(log f_t + m_{t-1} - m_t)     stabilized forget gate
 *   i'_t    = exp(i~_t - m_t)                  stabilized input gate
 *   C_t     = f'_t C_{t-1} + i'_t k_t v_t^T    matrix memory, stored [DHQK][DHV]
 *   n_t     = f'_t n_{t-1} + i'_t k_t          normalizer state
 *   qh      = q_t / sqrt(DHQK)
 *   h_t[j]  = o_t[j] * (sum_i qh[i] C_t[i][j]) / max(|n_t . qh|, exp(-m_t))
 *
 * Sources: "xLSTM Guide: Extended LSTM Architecture & Matrix Memory",
 * sections "The Stabilizer State: Preventing Numerical Overflow" (running-max
 * stabilizer and the stabilized exponential gates) and "mLSTM: Matrix
 * Key-Value Memory and Covariance Updates", "Recurrent Formulation (Inference
 * Mode)" (the C, n and h updates).  Readings where the pages are loose: the
 * forget gate is the sigmoid gate taken in log space; q (not k) carries the
 * 1/sqrt(DHQK) factor, so C and n hold raw k; the denominator floor is
 * exp(-m_t), which on the unstabilized states is the guide's floor of 1; the
 * memory is stored as k v^T ([DHQK][DHV]) and read out as C^T qh; the output
 * gate arrives already activated (NULL means o = 1).
 *
 * Inputs arrive as float (an exact image of fp32 and bf16 data) and are
 * widened to double; all arithmetic is double precision with the host libm.
 */
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* logsigmoid(x) = -log(1 + exp(-x)), evaluated without overflow. */
static double log_sigmoid(double x)
{
    if (x >= 0.0)
        return -log1p(exp(-x));
    return x - log1p(exp(x));
}

/*
 * Runs the recurrence for T tokens of one head, starting from the state
 * (C, n, *m) and leaving the final state there.  h (T x dv) may be NULL when
 * only the state is wanted.
 */
static void recurrent_head(int T, int dk, int dv,
                           const float *q, const float *k, const float *v,
                           const float *ig, const float *fg, const float *og,
                           double *C, double *n, double *m, double *h)
{
    const double scale = 1.0 / sqrt((double)dk);
    double *qh = (double *)malloc(sizeof(double) * (size_t)dk);
    double *kt = (double *)malloc(sizeof(double) * (size_t)dk);
    double *vt = (double *)malloc(sizeof(double) * (size_t)dv);
    double m_prev = *m;

    for (int t = 0; t < T; ++t) {
        const float *qt = q + (size_t)t * dk;
        const float *ktf = k + (size_t)t * dk;
        const float *vtf = v + (size_t)t * dv;
        const double lf = log_sigmoid((double)fg[t]);
        const double it = (double)ig[t];
        const double m_new = fmax(lf + m_prev, it);
        const double fp = exp(lf + m_prev - m_new);
        const double ip = exp(it - m_new);

        for (int i = 0; i < dk; ++i) {
            kt[i] = (double)ktf[i];
            qh[i] = (double)qt[i] * scale;
        }
        for (int j = 0; j < dv; ++j)
            vt[j] = (double)vtf[j];

        /* C_t = f' C_{t-1} + i' k v^T ;  n_t = f' n_{t-1} + i' k */
        for (int i = 0; i < dk; ++i) {
            double *row = C + (size_t)i * dv;
            const double ik = ip * kt[i];
            for (int j = 0; j < dv; ++j)
                row[j] = fp * row[j] + ik * vt[j];
            n[i] = fp * n[i] + ip * kt[i];
        }

        if (h) {
            double den = 0.0;
            for (int i = 0; i < dk; ++i)
                den += n[i] * qh[i];
            const double denom = fmax(fabs(den), exp(-m_new));
            double *ht = h + (size_t)t * dv;
            for (int j = 0; j < dv; ++j)
                ht[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double *row = C + (size_t)i * dv;
                const double qi = qh[i];
                for (int j = 0; j < dv; ++j)
                    ht[j] += qi * row[j];
            }
            const float *ot = og ? og + (size_t)t * dv : NULL;
            for (int j = 0; j < dv; ++j)
                ht[j] = (ot ? (double)ot[j] : 1.0) * ht[j] / denom;
        }
        m_prev = m_new;
    }
    *m = m_prev;
    free(qh);
    free(kt);
    free(vt);
}

typedef struct {
    int BH, T, dk, dv;
    const float *q, *k, *v, *ig, *fg, *og;
    double *C, *n, *m, *h;
    int next;                 /* next head to take */
    pthread_mutex_t lock;
} job_t;

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int bh = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (bh >= J->BH)
            break;
        const size_t T = (size_t)J->T;
        recurrent_head(J->T, J->dk, J->dv,
                       J->q + (size_t)bh * T * J->dk, J->k + (size_t)bh * T * J->dk,
                       J->v + (size_t)bh * T * J->dv, J->ig + (size_t)bh * T,
                       J->fg + (size_t)bh * T,
                       J->og ? J->og + (size_t)bh * T * J->dv : NULL,
                       J->C + (size_t)bh * J->dk * J->dv, J->n + (size_t)bh * J->dk,
                       J->m + bh,
                       J->h ? J->h + (size_t)bh * T * J->dv : NULL);
    }
    return NULL;
}

/* Number of worker threads a call with nthreads <= 0 uses. */
int oracle_default_threads(void)
{
    long c = sysconf(_SC_NPROCESSORS_ONLN);
    return c > 0 ? (int)c : 1;
}

/*
 * Runs T tokens for every (batch, head) from the state (C, n, m), which is
 * updated in place: C [BH][dk][dv], n [BH][dk], m [BH].  Token inputs are
 * [BH][T][dk|dv] and [BH][T]; og may be NULL.  h [BH][T][dv] may be NULL.
 * Heads are spread over nthreads threads (<= 0: all online cores).
 * Returns 0, or -1 on a bad argument.
 */
int oracle_mlstm_run(int BH, int T, int dk, int dv,
                     const float *q, const float *k, const float *v,
                     const float *ig, const float *fg, const float *og,
                     double *C, double *n, double *m, double *h, int nthreads)
{
    if (BH < 0 || T < 0 || dk <= 0 || dv <= 0 || !C || !n || !m)
        return -1;
    if (T > 0 && (!q || !k || !v || !ig || !fg))
        return -1;
    if (BH == 0 || T == 0)
        return 0;
    if (nthreads <= 0)
        nthreads = oracle_default_threads();
    if (nthreads > BH)
        nthreads = BH;

    job_t J = {BH, T, dk, dv, q, k, v, ig, fg, og, C, n, m, h, 0};
    pthread_mutex_init(&J.lock, NULL);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int i = 0; i < nthreads; ++i)
        pthread_create(&th[i], NULL, worker, &J);
    for (int i = 0; i < nthreads; ++i)
        pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return 0;
}

/*
 * Forward pass from the zero state (C = 0, n = 0, m = 0) over S tokens:
 * fills h [BH][S][dv] and the final state.  Any output may be NULL except
 * that the state buffers are needed as working memory, so NULL state
 * pointers make the oracle allocate its own.
 */
int oracle_mlstm_fwd(int BH, int S, int dk, int dv,
                     const float *q, const float *k, const float *v,
                     const float *ig, const float *fg, const float *og,
                     double *h, double *C_final, double *n_final, double *m_final,
                     int nthreads)
{
    if (BH < 0 || dk <= 0 || dv <= 0)
        return -1;
    const size_t nC = (size_t)BH * dk * dv, nn = (size_t)BH * dk, nm = (size_t)BH;
    double *C = C_final ? C_final : (double *)malloc(sizeof(double) * (nC ? nC : 1));
    double *n = n_final ? n_final : (double *)malloc(sizeof(double) * (nn ? nn : 1));
    double *m = m_final ? m_final : (double *)malloc(sizeof(double) * (nm ? nm : 1));
    memset(C, 0, sizeof(double) * nC);
    memset(n, 0, sizeof(double) * nn);
    for (size_t i = 0; i < nm; ++i)
        m[i] = 0.0;
    const int rc = oracle_mlstm_run(BH, S, dk, dv, q, k, v, ig, fg, og, C, n, m, h, nthreads);
    if (!C_final) free(C);
    if (!n_final) free(n);
    if (!m_final) free(m);
    return rc;
}

/* One decode step: the recurrence body applied once, state updated in place. */
int oracle_mlstm_step(int BH, int dk, int dv, double *C, double *n, double *m,
                      const float *q, const float *k, const float *v,
                      const float *ig, const float *fg, const float *og,
                      double *h, int nthreads)
{
    return oracle_mlstm_run(BH, 1, dk, dv, q, k, v, ig, fg, og, C, n, m, h, nthreads);
}
