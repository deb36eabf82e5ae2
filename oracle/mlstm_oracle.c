/*
 * mLSTM forward oracle: a plain, slow, float64 CPU restatement of the mLSTM
 * recurrence with exponential gating.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library.
 *
 * Sources (page title, section, equation):
 *   - "xLSTM: LSTM의 발명자가 현대 LLM 시대에 맞게 재설계한 확장 LSTM"
 *     (obsidian-dorae222.pages.dev), section "mLSTM (matrix LSTM)":
 *       eq. (1) C_t = f_t C_{t-1} + i_t v_t k_t^T
 *       eq. (2) n_t = f_t n_{t-1} + i_t k_t
 *       eq. (3) h_t = o_t * C_t q_t / max(|n_t^T q_t|, 1)
 *     section "sLSTM", stabilizer paragraph:
 *       m_t = max(f~_t + m_{t-1}, i~_t),
 *       f'_t = exp(f~_t + m_{t-1} - m_t),  i'_t = exp(i~_t - m_t)
 *     and the page's forward_recurrent listing, which applies that stabilizer
 *     to the mLSTM, stores v k^T as a (d_v x d_k) matrix and reads C q.
 *
 * Readings taken where the page is silent or inconsistent:
 *   - C is d_v x d_qk, stored row-major [d_v][d_qk]: the outer product v k^T
 *     and the readout C q in eq. (1)/(3) fix that orientation (the prose line
 *     "C in R^{d_k x d_v}" is the odd one out).
 *   - The output gate o_t is not part of this computation; h~ is the pre-gate
 *     readout.
 *   - The state carried between steps is the stabilized triple
 *     (C~, n~, m) with C = e^m C~ and n = e^m n~.  Dividing eq. (1)-(2) by e^{m_t}
 *     gives the stabilized update below, and dividing numerator and
 *     denominator of eq. (3) by e^{m_t} turns max(|n^T q|, 1) into
 *     max(|n~^T q|, e^{-m_t}); h~ is unchanged in exact arithmetic.
 *   - q is multiplied by qk_scale before it is used (qk_scale = 1 is the page
 *     literally; 1/sqrt(d_qk) is the usual attention scaling).
 *   - Absent initial state means C~ = 0, n~ = 0, m = 0.
 *
 * No blocking, fusion or reordering: one token at a time, in the order of the
 * recurrence.  Independent (batch, head) pairs run on separate threads; that
 * does not change any arithmetic.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int64_t T, dqk, dv;
    double qk_scale;
    const double *q, *k, *v, *ig, *fg;        /* this head's inputs          */
    double *C, *n, *m;                        /* this head's state, in/out   */
    double *h;                                /* this head's outputs [T][dv] */
} head_job;

/* One (batch, head): run the stabilized recurrence over t = 0..T-1. */
static void run_head(const head_job *j)
{
    const int64_t dqk = j->dqk, dv = j->dv;
    double *qs = (double *)malloc((size_t)(dqk > 0 ? dqk : 1) * sizeof(double));
    double m = *j->m;
    for (int64_t t = 0; t < j->T; ++t) {
        const double *qt = j->q + t * dqk;
        const double *kt = j->k + t * dqk;
        const double *vt = j->v + t * dv;
        const double it = j->ig[t];
        const double ft = j->fg[t];

        for (int64_t c = 0; c < dqk; ++c) qs[c] = j->qk_scale * qt[c];

        /* stabilizer: m_t = max(f~_t + m_{t-1}, i~_t) */
        const double a = ft + m;
        const double m_new = (a > it) ? a : it;
        /* stabilized gates f'_t, i'_t */
        const double fp = exp(ft + m - m_new);
        const double ip = exp(it - m_new);

        /* eq. (1): C~ <- f' C~ + i' v k^T   (row r = value index) */
        for (int64_t r = 0; r < dv; ++r) {
            double *Cr = j->C + r * dqk;
            for (int64_t c = 0; c < dqk; ++c)
                Cr[c] = fp * Cr[c] + ip * vt[r] * kt[c];
        }
        /* eq. (2): n~ <- f' n~ + i' k */
        for (int64_t c = 0; c < dqk; ++c) j->n[c] = fp * j->n[c] + ip * kt[c];

        /* eq. (3), stabilized: h~ = C~ q / max(|n~^T q|, exp(-m_t)) */
        double nq = 0.0;
        for (int64_t c = 0; c < dqk; ++c) nq += j->n[c] * qs[c];
        const double lower = exp(-m_new);
        const double den = (fabs(nq) > lower) ? fabs(nq) : lower;
        double *ht = j->h + t * dv;
        for (int64_t r = 0; r < dv; ++r) {
            const double *Cr = j->C + r * dqk;
            double num = 0.0;
            for (int64_t c = 0; c < dqk; ++c) num += Cr[c] * qs[c];
            ht[r] = num / den;
        }
        m = m_new;
    }
    *j->m = m;
    free(qs);
}

typedef struct {
    head_job *jobs;
    int64_t njobs;
    int64_t next;
    pthread_mutex_t lock;
} job_queue;

static void *worker(void *arg)
{
    job_queue *qu = (job_queue *)arg;
    for (;;) {
        pthread_mutex_lock(&qu->lock);
        int64_t idx = qu->next++;
        pthread_mutex_unlock(&qu->lock);
        if (idx >= qu->njobs) break;
        run_head(&qu->jobs[idx]);
    }
    return NULL;
}

/*
 * Full forward over a sequence.
 *   q, k : [B][H][T][dqk]   v : [B][H][T][dv]   ig, fg : [B][H][T]
 *   C0   : [B][H][dv][dqk]  n0 : [B][H][dqk]    m0 : [B][H]   (each may be NULL = zero)
 *   h    : [B][H][T][dv]    C, n, m : final stabilized state, same shapes as C0, n0, m0
 * Returns 0, or -1 on bad sizes / allocation failure.
 */
int mlstm_oracle_forward(int64_t B, int64_t H, int64_t T, int64_t dqk, int64_t dv,
                         double qk_scale,
                         const double *q, const double *k, const double *v,
                         const double *ig, const double *fg,
                         const double *C0, const double *n0, const double *m0,
                         double *h, double *C, double *n, double *m,
                         int nthreads)
{
    if (B < 0 || H < 0 || T < 0 || dqk < 0 || dv < 0) return -1;
    const int64_t BH = B * H;
    const int64_t csz = dv * dqk;
    for (int64_t bh = 0; bh < BH; ++bh) {
        if (C0) memcpy(C + bh * csz, C0 + bh * csz, (size_t)csz * sizeof(double));
        else memset(C + bh * csz, 0, (size_t)csz * sizeof(double));
        if (n0) memcpy(n + bh * dqk, n0 + bh * dqk, (size_t)dqk * sizeof(double));
        else memset(n + bh * dqk, 0, (size_t)dqk * sizeof(double));
        m[bh] = m0 ? m0[bh] : 0.0;
    }
    if (BH == 0 || T == 0) return 0;

    head_job *jobs = (head_job *)calloc((size_t)BH, sizeof(head_job));
    if (!jobs) return -1;
    for (int64_t bh = 0; bh < BH; ++bh) {
        head_job *j = &jobs[bh];
        j->T = T; j->dqk = dqk; j->dv = dv; j->qk_scale = qk_scale;
        j->q = q + bh * T * dqk;
        j->k = k + bh * T * dqk;
        j->v = v + bh * T * dv;
        j->ig = ig + bh * T;
        j->fg = fg + bh * T;
        j->C = C + bh * csz;
        j->n = n + bh * dqk;
        j->m = m + bh;
        j->h = h + bh * T * dv;
    }

    if (nthreads <= 1 || BH == 1) {
        for (int64_t bh = 0; bh < BH; ++bh) run_head(&jobs[bh]);
        free(jobs);
        return 0;
    }
    if (nthreads > BH) nthreads = (int)BH;
    job_queue qu;
    qu.jobs = jobs; qu.njobs = BH; qu.next = 0;
    pthread_mutex_init(&qu.lock, NULL);
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    int started = 0;
    for (int i = 0; i < nthreads; ++i)
        if (pthread_create(&th[i], NULL, worker, &qu) == 0) ++started;
    if (started == 0) worker(&qu);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&qu.lock);
    free(th);
    free(jobs);
    return 0;
}

/*
 * One decode step (the page's forward_recurrent, without projections and o_t):
 *   q, k : [B][H][dqk]  v : [B][H][dv]  ig, fg : [B][H]
 *   C, n, m : state in (stabilized); C1, n1, m1 : state out; h : [B][H][dv]
 */
int mlstm_oracle_step(int64_t B, int64_t H, int64_t dqk, int64_t dv, double qk_scale,
                      const double *q, const double *k, const double *v,
                      const double *ig, const double *fg,
                      const double *C, const double *n, const double *m,
                      double *h, double *C1, double *n1, double *m1, int nthreads)
{
    return mlstm_oracle_forward(B, H, 1, dqk, dv, qk_scale, q, k, v, ig, fg,
                                C, n, m, h, C1, n1, m1, nthreads);
}

/*
 * Output stage of the mLSTM (xLSTM page, "mLSTM (matrix LSTM)" eq. 3, and the
 * o_t line of the page's forward_recurrent listing): h_t = o_t * h~_t with
 * o_t the logistic sigmoid of the output-gate pre-activation, element by
 * element.  count elements of h_tilde and o_pre; h may alias neither.
 */
int mlstm_oracle_output_gate(int64_t count, const double *h_tilde, const double *o_pre, double *h)
{
    if (count < 0 || (count > 0 && (!h_tilde || !o_pre || !h)))
        return 1;
    for (int64_t i = 0; i < count; ++i)
        h[i] = h_tilde[i] / (1.0 + exp(-o_pre[i]));
    return 0;
}
