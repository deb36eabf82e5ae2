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

/*
 * Reverse-mode derivative of the forward above (vector-Jacobian product).
 *
 * What is differentiated: the method's readout in its literal form, eq. (3)
 * with the true states of eq. (1)-(2), h_t = C_t q_t / max(|n_t^T q_t|, 1), f_t =
 * exp(f~_t), i_t = exp(i~_t); the stabilized triple (C~, n~, m) is only how those
 * states are stored.  h~ does not depend on the gauge m, so m is a constant of
 * the derivative (it is never differentiated through its max), and every
 * quantity below is the true one rescaled by e^{m_t}, so that no factor exceeds 1:
 *   adjoint of C~_t:  dC~_t = e^{m_t} dL/dC_t, carried back by f'_t;
 *   at token t, with dn~um = dh_t / den~_t, g = dh_t . h~_t, s = n~_t . q_t,
 *   ds = -(g / den~_t) sign(s) where |s| > e^{-m_t} (0 where the clamp holds):
 *     dC~_t += dn~um q_t^T,  dn~_t += ds q_t,
 *     dq_t  = qk_scale (C~_t^T dn~um + ds n~_t),
 *     dv_t  = i'_t dC~_t k_t,   dk_t = i'_t (dC~_t^T v_t + dn~_t),
 *     di~_t = k_t . dk_t        (i~ scales both places k_t enters),
 *     df~_t = f'_t (<dC~_t, C~_{t-1}> + <dn~_t, n~_{t-1}>),
 *   then dC~_{t-1} = f'_t dC~_t, dn~_{t-1} = f'_t dn~_t.
 * The upstream gradient of the final state (dC_T, dn_T, for the stored C~_T, n~_T)
 * is taken as that of a consumer of the true state (the next call of the
 * recurrence is one): dC~_T = dC_T.  The initial state's gradients follow from
 * C_0 = e^{m_0} C~_0: dC~_0, dn~_0 and dm_0 = <dC~_0, C~_0> + <dn~_0, n~_0>.
 *
 * The backward sweep needs the state before every token; it keeps the state at
 * every 64th token and recomputes the 64 states of a stretch with the same
 * token_step as the forward (identical arithmetic, less memory).
 */
enum { BWD_STRETCH = 64 };

typedef struct {
    int64_t T, dqk, dv;
    double qk_scale;
    const double *q, *k, *v, *ig, *fg;        /* this head's inputs                   */
    const double *C0, *n0;                    /* initial state, or NULL (zero)        */
    double m0;
    const double *dh, *dCT, *dnT;             /* upstream: [T][dv], final state or NULL */
    double *dq, *dk, *dv_, *dig, *dfg;        /* gradients of the inputs              */
    double *dC0, *dn0, *dm0;                  /* gradients of the initial state       */
    int status;
} bwd_job;

/* One token of the stabilized recurrence on (C, n) in place, as in run_head;
 * returns m_t and the quantities the derivative needs. */
static double token_step(int64_t dqk, int64_t dv, double qk_scale, double m, const double *qt,
                         const double *kt, const double *vt, double it, double ft, double *C, double *n,
                         double *qs, double *ht, double *fp_o, double *ip_o, double *s_o, double *lower_o,
                         double *den_o)
{
    for (int64_t c = 0; c < dqk; ++c) qs[c] = qk_scale * qt[c];
    const double a = ft + m;
    const double m_new = (a > it) ? a : it;
    const double fp = exp(ft + m - m_new);
    const double ip = exp(it - m_new);
    for (int64_t r = 0; r < dv; ++r)
        for (int64_t c = 0; c < dqk; ++c) C[r * dqk + c] = fp * C[r * dqk + c] + ip * vt[r] * kt[c];
    for (int64_t c = 0; c < dqk; ++c) n[c] = fp * n[c] + ip * kt[c];
    double s = 0.0;
    for (int64_t c = 0; c < dqk; ++c) s += n[c] * qs[c];
    const double lower = exp(-m_new);
    const double den = (fabs(s) > lower) ? fabs(s) : lower;
    for (int64_t r = 0; r < dv; ++r) {
        double num = 0.0;
        for (int64_t c = 0; c < dqk; ++c) num += C[r * dqk + c] * qs[c];
        ht[r] = num / den;
    }
    *fp_o = fp; *ip_o = ip; *s_o = s; *lower_o = lower; *den_o = den;
    return m_new;
}

static void run_head_bwd(bwd_job *j)
{
    const int64_t T = j->T, dqk = j->dqk, dv = j->dv, csz = dv * dqk, K = BWD_STRETCH;
    const int64_t nck = (T + K - 1) / K;
    /* checkpoints: the state before tokens 0, K, 2K, ...; one stretch of states */
    double *ckC = (double *)malloc((size_t)(nck + 1) * (size_t)(csz > 0 ? csz : 1) * sizeof(double));
    double *ckn = (double *)malloc((size_t)(nck + 1) * (size_t)(dqk > 0 ? dqk : 1) * sizeof(double));
    double *ckm = (double *)malloc((size_t)(nck + 1) * sizeof(double));
    double *stC = (double *)malloc((size_t)(K + 1) * (size_t)(csz > 0 ? csz : 1) * sizeof(double));
    double *stn = (double *)malloc((size_t)(K + 1) * (size_t)(dqk > 0 ? dqk : 1) * sizeof(double));
    double *sth = (double *)malloc((size_t)K * (size_t)(dv > 0 ? dv : 1) * sizeof(double));
    double *stf = (double *)malloc((size_t)K * 6 * sizeof(double));   /* fp, ip, s, lower, den, m */
    double *qs = (double *)malloc((size_t)(dqk > 0 ? dqk : 1) * sizeof(double));
    double *dC = (double *)malloc((size_t)(csz > 0 ? csz : 1) * sizeof(double));
    double *dn = (double *)malloc((size_t)(dqk > 0 ? dqk : 1) * sizeof(double));
    double *dnum = (double *)malloc((size_t)(dv > 0 ? dv : 1) * sizeof(double));
    if (!ckC || !ckn || !ckm || !stC || !stn || !sth || !stf || !qs || !dC || !dn || !dnum) {
        j->status = -1;
        goto out;
    }
    /* forward sweep, keeping the checkpoints */
    {
        double *C = stC, *n = stn, m = j->m0, f[5];
        for (int64_t x = 0; x < csz; ++x) C[x] = j->C0 ? j->C0[x] : 0.0;
        for (int64_t c = 0; c < dqk; ++c) n[c] = j->n0 ? j->n0[c] : 0.0;
        for (int64_t t = 0; t < T; ++t) {
            if (t % K == 0) {
                memcpy(ckC + (t / K) * csz, C, (size_t)csz * sizeof(double));
                memcpy(ckn + (t / K) * dqk, n, (size_t)dqk * sizeof(double));
                ckm[t / K] = m;
            }
            m = token_step(dqk, dv, j->qk_scale, m, j->q + t * dqk, j->k + t * dqk, j->v + t * dv, j->ig[t],
                           j->fg[t], C, n, qs, sth, &f[0], &f[1], &f[2], &f[3], &f[4]);
        }
    }
    /* backward sweep */
    for (int64_t x = 0; x < csz; ++x) dC[x] = j->dCT ? j->dCT[x] : 0.0;
    for (int64_t c = 0; c < dqk; ++c) dn[c] = j->dnT ? j->dnT[c] : 0.0;
    for (int64_t b = nck - 1; b >= 0; --b) {
        const int64_t t0 = b * K, len = (T - t0 < K) ? T - t0 : K;
        /* the stretch's states: stC[0] = before token t0, stC[i + 1] = after token t0 + i */
        memcpy(stC, ckC + b * csz, (size_t)csz * sizeof(double));
        memcpy(stn, ckn + b * dqk, (size_t)dqk * sizeof(double));
        double m = ckm[b];
        for (int64_t i = 0; i < len; ++i) {
            const int64_t t = t0 + i;
            memcpy(stC + (i + 1) * csz, stC + i * csz, (size_t)csz * sizeof(double));
            memcpy(stn + (i + 1) * dqk, stn + i * dqk, (size_t)dqk * sizeof(double));
            double *f = stf + 6 * i;
            m = token_step(dqk, dv, j->qk_scale, m, j->q + t * dqk, j->k + t * dqk, j->v + t * dv, j->ig[t],
                           j->fg[t], stC + (i + 1) * csz, stn + (i + 1) * dqk, qs, sth + i * dv, &f[0], &f[1],
                           &f[2], &f[3], &f[4]);
            f[5] = m;
        }
        for (int64_t i = len - 1; i >= 0; --i) {
            const int64_t t = t0 + i;
            const double *f = stf + 6 * i;
            const double fp = f[0], ip = f[1], s = f[2], lower = f[3], den = f[4];
            const double *Ct = stC + (i + 1) * csz, *Cp = stC + i * csz;
            const double *nt = stn + (i + 1) * dqk, *np_ = stn + i * dqk;
            const double *ht = sth + i * dv, *dht = j->dh + t * dv;
            const double *qt = j->q + t * dqk, *kt = j->k + t * dqk, *vt = j->v + t * dv;
            for (int64_t c = 0; c < dqk; ++c) qs[c] = j->qk_scale * qt[c];
            /* readout: h~ = C~ q / den~ */
            double g = 0.0;
            for (int64_t r = 0; r < dv; ++r) {
                dnum[r] = dht[r] / den;
                g += dht[r] * ht[r];
            }
            const double ds = (fabs(s) > lower) ? -(g / den) * (s > 0.0 ? 1.0 : -1.0) : 0.0;
            /* this token's direct terms join the carried adjoint */
            for (int64_t r = 0; r < dv; ++r)
                for (int64_t c = 0; c < dqk; ++c) dC[r * dqk + c] += dnum[r] * qs[c];
            for (int64_t c = 0; c < dqk; ++c) dn[c] += ds * qs[c];
            /* dq */
            for (int64_t c = 0; c < dqk; ++c) {
                double acc = ds * nt[c];
                for (int64_t r = 0; r < dv; ++r) acc += Ct[r * dqk + c] * dnum[r];
                j->dq[t * dqk + c] = j->qk_scale * acc;
            }
            /* dv, dk, di~ */
            for (int64_t r = 0; r < dv; ++r) {
                double acc = 0.0;
                for (int64_t c = 0; c < dqk; ++c) acc += dC[r * dqk + c] * kt[c];
                j->dv_[t * dv + r] = ip * acc;
            }
            double di = 0.0;
            for (int64_t c = 0; c < dqk; ++c) {
                double acc = dn[c];
                for (int64_t r = 0; r < dv; ++r) acc += dC[r * dqk + c] * vt[r];
                j->dk[t * dqk + c] = ip * acc;
                di += kt[c] * j->dk[t * dqk + c];
            }
            j->dig[t] = di;
            /* df~: the carried state's share */
            double df = 0.0;
            for (int64_t x = 0; x < csz; ++x) df += dC[x] * Cp[x];
            for (int64_t c = 0; c < dqk; ++c) df += dn[c] * np_[c];
            j->dfg[t] = fp * df;
            /* adjoint of the state before token t */
            for (int64_t x = 0; x < csz; ++x) dC[x] *= fp;
            for (int64_t c = 0; c < dqk; ++c) dn[c] *= fp;
        }
    }
    {
        double dm = 0.0;
        for (int64_t x = 0; x < csz; ++x) {
            j->dC0[x] = dC[x];
            dm += dC[x] * (j->C0 ? j->C0[x] : 0.0);
        }
        for (int64_t c = 0; c < dqk; ++c) {
            j->dn0[c] = dn[c];
            dm += dn[c] * (j->n0 ? j->n0[c] : 0.0);
        }
        *j->dm0 = dm;
    }
    j->status = 0;
out:
    free(ckC); free(ckn); free(ckm); free(stC); free(stn); free(sth); free(stf); free(qs);
    free(dC); free(dn); free(dnum);
}

typedef struct {
    bwd_job *jobs;
    int64_t njobs, next;
    pthread_mutex_t lock;
} bwd_queue;

static void *bwd_worker(void *arg)
{
    bwd_queue *qu = (bwd_queue *)arg;
    for (;;) {
        pthread_mutex_lock(&qu->lock);
        int64_t idx = qu->next++;
        pthread_mutex_unlock(&qu->lock);
        if (idx >= qu->njobs) break;
        run_head_bwd(&qu->jobs[idx]);
    }
    return NULL;
}

/*
 * Backward over a sequence: shapes as in mlstm_oracle_forward; dh [B][H][T][dv];
 * dCT [B][H][dv][dqk], dnT [B][H][dqk] (each may be NULL = zero); C0, n0, m0 as in
 * the forward (NULL = zero state).  Outputs dq, dk [B][H][T][dqk], dv [B][H][T][dv],
 * dig, dfg [B][H][T], dC0 [B][H][dv][dqk], dn0 [B][H][dqk], dm0 [B][H].
 * Returns 0, or -1 on bad sizes / allocation failure.
 */
int mlstm_oracle_backward(int64_t B, int64_t H, int64_t T, int64_t dqk, int64_t dv, double qk_scale,
                          const double *q, const double *k, const double *v, const double *ig,
                          const double *fg, const double *C0, const double *n0, const double *m0,
                          const double *dh, const double *dCT, const double *dnT,
                          double *dq, double *dk, double *dv_, double *dig, double *dfg,
                          double *dC0, double *dn0, double *dm0, int nthreads)
{
    if (B < 0 || H < 0 || T < 0 || dqk < 0 || dv < 0) return -1;
    const int64_t BH = B * H, csz = dv * dqk;
    if (BH == 0) return 0;
    bwd_job *jobs = (bwd_job *)calloc((size_t)BH, sizeof(bwd_job));
    if (!jobs) return -1;
    for (int64_t bh = 0; bh < BH; ++bh) {
        bwd_job *j = &jobs[bh];
        j->T = T; j->dqk = dqk; j->dv = dv; j->qk_scale = qk_scale;
        j->q = q + bh * T * dqk; j->k = k + bh * T * dqk; j->v = v + bh * T * dv;
        j->ig = ig + bh * T; j->fg = fg + bh * T;
        j->C0 = C0 ? C0 + bh * csz : NULL;
        j->n0 = n0 ? n0 + bh * dqk : NULL;
        j->m0 = m0 ? m0[bh] : 0.0;
        j->dh = dh + bh * T * dv;
        j->dCT = dCT ? dCT + bh * csz : NULL;
        j->dnT = dnT ? dnT + bh * dqk : NULL;
        j->dq = dq + bh * T * dqk; j->dk = dk + bh * T * dqk; j->dv_ = dv_ + bh * T * dv;
        j->dig = dig + bh * T; j->dfg = dfg + bh * T;
        j->dC0 = dC0 + bh * csz; j->dn0 = dn0 + bh * dqk; j->dm0 = dm0 + bh;
    }
    if (nthreads > BH) nthreads = (int)BH;
    if (nthreads <= 1) {
        for (int64_t bh = 0; bh < BH; ++bh) run_head_bwd(&jobs[bh]);
    } else {
        bwd_queue qu;
        qu.jobs = jobs; qu.njobs = BH; qu.next = 0;
        pthread_mutex_init(&qu.lock, NULL);
        pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
        int started = 0;
        for (int i = 0; i < nthreads; ++i)
            if (pthread_create(&th[i], NULL, bwd_worker, &qu) == 0) ++started;
        if (started == 0) bwd_worker(&qu);
        for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
        pthread_mutex_destroy(&qu.lock);
        free(th);
    }
    int rc = 0;
    for (int64_t bh = 0; bh < BH; ++bh)
        if (jobs[bh].status != 0) rc = -1;
    free(jobs);
    return rc;
}
