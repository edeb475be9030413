/*
 * mlstm_adjoint.c -- fp64 CPU gradients of the mLSTM recurrence by reverse-mode differentiation
 * written out token by token (the adjoint of the recurrence).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path (the CUDA library, its Python binding)
 * may include, link or call this file.  It shares no code, header, table or helper with the CUDA
 * kernels (nor with mlstm_oracle.c).
 *
 * The forward pass is the recurrence of mlstm_oracle.c, from the zero state, per head:
 *   log f_t = logsigmoid(f~_t),  m_t = max(log f_t + m_{t-1}, i~_t),
 *   f'_t = exp(log f_t + m_{t-1} - m_t),  i'_t = exp(i~_t - m_t),
 *   C_t = f'_t C_{t-1} + i'_t k_t v_t^T,  n_t = f'_t n_{t-1} + i'_t k_t,
 *   h_t = o_t * (C_t^T qh_t) / max(|n_t . qh_t|, exp(-m_t)),  qh_t = q_t / sqrt(DHQK)
 * ("xLSTM Guide: Extended LSTM Architecture & Matrix Memory", "The Stabilizer State" and
 * "Recurrent Formulation (Inference Mode)"; the same readings as mlstm_oracle.c).
 *
 * What it computes: the gradients of L = sum_t dh_t . h_t with respect to q, k, v, i~, f~ and o.
 * h does not depend on the stabilizer (any sequence m_t gives the same h), so m is held fixed and
 * each step is differentiated with the chain rule, last token first:
 *   read-out:  num = C_t^T qh,  den = n_t . qh,  N = max(|den|, exp(-m_t)),  h = o num / N
 *     dL/do = dh num / N,  dnum = o dh / N,  dN = -sum(dh o num) / N^2,
 *     dden = dN sign(den) when |den| > exp(-m_t) (the branch the forward pass took), else 0,
 *     dqh = C_t dnum + dden n_t,  dC_t += qh dnum^T,  dn_t += dden qh;
 *   update:    C_t = f' C_{t-1} + i' k v^T,  n_t = f' n_{t-1} + i' k
 *     dk = i' (dC_t v + dn_t),  dv = i' dC_t^T k,
 *     df' = <dC_t, C_{t-1}> + dn_t . n_{t-1},  di' = k . (dC_t v + dn_t),
 *     dL/dlog f_t = f' df',  dL/di~_t = i' di',  dL/df~_t = dL/dlog f_t * sigmoid(-f~_t),
 *     dC_{t-1} = f' dC_t,  dn_{t-1} = f' dn_t;
 *   dL/dq = dqh / sqrt(DHQK).
 * The states C_{t-1}, C_t are recomputed forward from checkpoints kept every K tokens.
 *
 * Inputs arrive as float (an exact image of fp32 and bf16 data) and are widened to double; all
 * arithmetic is double precision with the host libm.
 */
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

static double log_sigmoid(double x)
{
    if (x >= 0.0)
        return -log1p(exp(-x));
    return x - log1p(exp(x));
}

static double sigmoid(double x)
{
    if (x >= 0.0)
        return 1.0 / (1.0 + exp(-x));
    const double e = exp(x);
    return e / (1.0 + e);
}

/* One forward step: (C, n, m) before token t -> after it (in place). */
static void step(int dk, int dv, const float *k, const float *v, double ig, double fg, double *C, double *n,
                 double *m)
{
    const double lf = log_sigmoid(fg);
    const double m_new = fmax(lf + *m, ig);
    const double fp = exp(lf + *m - m_new);
    const double ip = exp(ig - m_new);
    for (int i = 0; i < dk; ++i) {
        double *row = C + (size_t)i * dv;
        const double ik = ip * (double)k[i];
        for (int j = 0; j < dv; ++j)
            row[j] = fp * row[j] + ik * (double)v[j];
        n[i] = fp * n[i] + ip * (double)k[i];
    }
    *m = m_new;
}

typedef struct {
    int T, dk, dv;
    const float *q, *k, *v, *ig, *fg, *og, *dh;
    double *dq, *dkk, *dvv, *dig, *dfg, *dog;
} head_t;

static void adjoint_head(const head_t *H)
{
    const int T = H->T, dk = H->dk, dv = H->dv;
    const size_t nC = (size_t)dk * dv;
    const double scale = 1.0 / sqrt((double)dk);
    int K = (int)ceil(sqrt((double)(T > 0 ? T : 1)));
    if (K < 1)
        K = 1;
    const int nck = (T + K - 1) / K;
    double *ckC = (double *)calloc((size_t)(nck > 0 ? nck : 1) * nC, sizeof(double));
    double *ckn = (double *)calloc((size_t)(nck > 0 ? nck : 1) * dk, sizeof(double));
    double *ckm = (double *)calloc((size_t)(nck > 0 ? nck : 1), sizeof(double));
    double *segC = (double *)malloc(sizeof(double) * (size_t)(K + 1) * nC);
    double *segn = (double *)malloc(sizeof(double) * (size_t)(K + 1) * dk);
    double *segm = (double *)malloc(sizeof(double) * (size_t)(K + 1));
    double *C = (double *)calloc(nC, sizeof(double));
    double *n = (double *)calloc((size_t)dk, sizeof(double));
    double *dC = (double *)calloc(nC, sizeof(double));
    double *dn = (double *)calloc((size_t)dk, sizeof(double));
    double *qh = (double *)malloc(sizeof(double) * (size_t)dk);
    double *num = (double *)malloc(sizeof(double) * (size_t)dv);
    double *dnum = (double *)malloc(sizeof(double) * (size_t)dv);
    double *dCv = (double *)malloc(sizeof(double) * (size_t)dk);
    double m = 0.0;

    /* forward pass: the state before every K-th token */
    for (int t = 0; t < T; ++t) {
        if (t % K == 0) {
            const int c = t / K;
            memcpy(ckC + (size_t)c * nC, C, sizeof(double) * nC);
            memcpy(ckn + (size_t)c * dk, n, sizeof(double) * (size_t)dk);
            ckm[c] = m;
        }
        step(dk, dv, H->k + (size_t)t * dk, H->v + (size_t)t * dv, H->ig[t], H->fg[t], C, n, &m);
    }

    /* backward, one checkpoint segment at a time, last first */
    for (int c = nck - 1; c >= 0; --c) {
        const int t0 = c * K, t1 = (t0 + K < T) ? t0 + K : T;
        memcpy(segC, ckC + (size_t)c * nC, sizeof(double) * nC);
        memcpy(segn, ckn + (size_t)c * dk, sizeof(double) * (size_t)dk);
        segm[0] = ckm[c];
        for (int t = t0; t < t1; ++t) {   /* states after each token of the segment */
            const int j = t - t0;
            memcpy(segC + (size_t)(j + 1) * nC, segC + (size_t)j * nC, sizeof(double) * nC);
            memcpy(segn + (size_t)(j + 1) * dk, segn + (size_t)j * dk, sizeof(double) * (size_t)dk);
            segm[j + 1] = segm[j];
            step(dk, dv, H->k + (size_t)t * dk, H->v + (size_t)t * dv, H->ig[t], H->fg[t],
                 segC + (size_t)(j + 1) * nC, segn + (size_t)(j + 1) * dk, &segm[j + 1]);
        }
        for (int t = t1 - 1; t >= t0; --t) {
            const int j = t - t0;
            const double *Cp = segC + (size_t)j * nC, *Ct = segC + (size_t)(j + 1) * nC;
            const double *np_ = segn + (size_t)j * dk, *nt = segn + (size_t)(j + 1) * dk;
            const double mp = segm[j], mt = segm[j + 1];
            const float *qt = H->q + (size_t)t * dk, *kt = H->k + (size_t)t * dk, *vt = H->v + (size_t)t * dv;
            const float *ot = H->og ? H->og + (size_t)t * dv : NULL;
            const float *dht = H->dh + (size_t)t * dv;
            const double lf = log_sigmoid((double)H->fg[t]);
            const double fp = exp(lf + mp - mt);
            const double ip = exp((double)H->ig[t] - mt);

            /* read-out of token t */
            for (int i = 0; i < dk; ++i)
                qh[i] = (double)qt[i] * scale;
            double den = 0.0;
            for (int i = 0; i < dk; ++i)
                den += nt[i] * qh[i];
            for (int jj = 0; jj < dv; ++jj)
                num[jj] = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double *row = Ct + (size_t)i * dv;
                for (int jj = 0; jj < dv; ++jj)
                    num[jj] += qh[i] * row[jj];
            }
            const double floor_ = exp(-mt);
            const double N = fmax(fabs(den), floor_);
            double dN = 0.0;
            for (int jj = 0; jj < dv; ++jj) {
                const double o = ot ? (double)ot[jj] : 1.0;
                const double d = (double)dht[jj];
                if (H->dog)
                    H->dog[(size_t)t * dv + jj] = d * num[jj] / N;
                dnum[jj] = o * d / N;
                dN -= d * o * num[jj] / (N * N);
            }
            const double dden = fabs(den) > floor_ ? (den > 0.0 ? dN : -dN) : 0.0;
            for (int i = 0; i < dk; ++i) {
                const double *row = Ct + (size_t)i * dv;
                double a = 0.0;
                for (int jj = 0; jj < dv; ++jj)
                    a += row[jj] * dnum[jj];
                H->dq[(size_t)t * dk + i] = (a + dden * nt[i]) * scale;
            }
            for (int i = 0; i < dk; ++i) {
                double *drow = dC + (size_t)i * dv;
                for (int jj = 0; jj < dv; ++jj)
                    drow[jj] += qh[i] * dnum[jj];
                dn[i] += dden * qh[i];
            }

            /* the update of token t */
            double dfp = 0.0, dip = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double *drow = dC + (size_t)i * dv, *prow = Cp + (size_t)i * dv;
                double a = 0.0, b = 0.0;
                for (int jj = 0; jj < dv; ++jj) {
                    a += drow[jj] * (double)vt[jj];
                    b += drow[jj] * prow[jj];
                }
                dCv[i] = a + dn[i];
                dfp += b + dn[i] * np_[i];
                dip += (double)kt[i] * dCv[i];
                H->dkk[(size_t)t * dk + i] = ip * dCv[i];
            }
            for (int jj = 0; jj < dv; ++jj) {
                double a = 0.0;
                for (int i = 0; i < dk; ++i)
                    a += dC[(size_t)i * dv + jj] * (double)kt[i];
                H->dvv[(size_t)t * dv + jj] = ip * a;
            }
            H->dig[t] = ip * dip;
            H->dfg[t] = fp * dfp * sigmoid(-(double)H->fg[t]);
            for (size_t e = 0; e < nC; ++e)
                dC[e] *= fp;
            for (int i = 0; i < dk; ++i)
                dn[i] *= fp;
        }
    }
    free(ckC); free(ckn); free(ckm); free(segC); free(segn); free(segm);
    free(C); free(n); free(dC); free(dn); free(qh); free(num); free(dnum); free(dCv);
}

typedef struct {
    int BH, T, dk, dv;
    const float *q, *k, *v, *ig, *fg, *og, *dh;
    double *dq, *dkk, *dvv, *dig, *dfg, *dog;
    int next;
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
        head_t H = {J->T, J->dk, J->dv,
                    J->q + (size_t)bh * T * J->dk, J->k + (size_t)bh * T * J->dk, J->v + (size_t)bh * T * J->dv,
                    J->ig + (size_t)bh * T, J->fg + (size_t)bh * T, J->og ? J->og + (size_t)bh * T * J->dv : NULL,
                    J->dh + (size_t)bh * T * J->dv,
                    J->dq + (size_t)bh * T * J->dk, J->dkk + (size_t)bh * T * J->dk, J->dvv + (size_t)bh * T * J->dv,
                    J->dig + (size_t)bh * T, J->dfg + (size_t)bh * T, J->dog ? J->dog + (size_t)bh * T * J->dv : NULL};
        adjoint_head(&H);
    }
    return NULL;
}

/*
 * Gradients of sum(dh * h) for BH independent heads of T tokens from the zero state.  Token
 * inputs [BH][T][dk|dv] and [BH][T] (og NULL = no output gate); outputs [BH][T][dk|dv], [BH][T]
 * (dog ignored without og).  Heads are spread over nthreads threads (<= 0: all online cores).
 * Returns 0, or -1 on a bad argument.
 */
int oracle_mlstm_adjoint(int BH, int T, int dk, int dv, const float *q, const float *k, const float *v,
                         const float *ig, const float *fg, const float *og, const float *dh, double *dq,
                         double *dkk, double *dvv, double *dig, double *dfg, double *dog, int nthreads)
{
    if (BH < 0 || T < 0 || dk <= 0 || dv <= 0)
        return -1;
    if (BH == 0 || T == 0)
        return 0;
    if (!q || !k || !v || !ig || !fg || !dh || !dq || !dkk || !dvv || !dig || !dfg || (og && !dog))
        return -1;
    if (nthreads <= 0) {
        long c = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = c > 0 ? (int)c : 1;
    }
    if (nthreads > BH)
        nthreads = BH;
    job_t J = {BH, T, dk, dv, q, k, v, ig, fg, og, dh, dq, dkk, dvv, dig, dfg, og ? dog : NULL, 0};
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
