/*
 * kd_oracle.c -- fp64 CPU oracle for the Kronecker delta rule token mixer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no source,
 * header, table or helper with the CUDA library; it is the plain definition of
 * what that library computes, written token by token in double precision.
 *
 * Sources (web pages on the method; cited by title and section):
 *  [digest]  "KronLSTM이 스칼라 보정으로 긴 문맥 선형 어텐션의 기억 간섭을 줄인다"
 *            (a digest of the KronLSTM paper)
 *              - section "어떻게 동작하나": the Kronecker delta rule corrects one
 *                scalar association v^T S k toward a target along the outer
 *                product v k^T; erase amount beta, write amount c (target c/beta).
 *              - section "어떻게 쓰나": a diagonal forget gate on the key
 *                dimension decays the memory from the right; beta and c are
 *                per-head scalars; the only state is one matrix per head.
 *  [review]  "[논문리뷰] Kronecker Delta Rule for Long Context Linear Attention",
 *            section "Key Terms & Definitions" (Kronecker Delta Rule entry).
 *
 * One token step, per head, state S in R^{dv x dk} (row r = value channel,
 * column j = key channel):
 *      Sbar = S diag(f),  f = exp(logf)          (decay from the right)
 *      b    = v^T Sbar k                          (current association)
 *      u    = c - beta * b                        (erase by beta, write by c)
 *      S    = Sbar + u v k^T
 *      o    = S q                                 (read after the write)
 * Readings of the pages where they are silent: the write gate c enters
 * directly (c/beta is never formed, so beta = 0 is legal); the decay is applied
 * before the erase read; the output reads the state after the write; q is not
 * rescaled; k and v are used as given (no renormalisation).
 *
 * The reverse recurrence is reverse-mode differentiation of the step above
 * (the pages give none); it recomputes states from checkpoints every 64 tokens.
 *
 * Layouts: q,k,v,o,dO: [B,T,H,d]; beta,c: [B,T,H]; logf: [B,T,H,dk];
 * states: [B,H,dv,dk] row-major.  All double.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define KDO_CKPT 64

/* ------------------------------------------------------------------------ */
/* One token step for one head.  S (dv x dk) is updated in place.           */
/* Writes o (dv), and optionally the association b and coefficient u.       */
/* ------------------------------------------------------------------------ */
static void kdo_token_step(double *S, const double *q, const double *k,
                           const double *v, double beta, double c,
                           const double *logf, int dk, int dv, double *o,
                           double *b_out, double *u_out)
{
    /* decay from the right: column j scaled by f_j */
    for (int r = 0; r < dv; ++r)
        for (int j = 0; j < dk; ++j)
            S[(size_t)r * dk + j] *= exp(logf[j]);
    /* b = v^T Sbar k */
    double b = 0.0;
    for (int r = 0; r < dv; ++r) {
        double row = 0.0;
        for (int j = 0; j < dk; ++j)
            row += S[(size_t)r * dk + j] * k[j];
        b += v[r] * row;
    }
    double u = c - beta * b;
    /* S = Sbar + u v k^T */
    for (int r = 0; r < dv; ++r)
        for (int j = 0; j < dk; ++j)
            S[(size_t)r * dk + j] += u * v[r] * k[j];
    /* o = S q */
    for (int r = 0; r < dv; ++r) {
        double acc = 0.0;
        for (int j = 0; j < dk; ++j)
            acc += S[(size_t)r * dk + j] * q[j];
        o[r] = acc;
    }
    if (b_out) *b_out = b;
    if (u_out) *u_out = u;
}

/* Public single-head step (used by the invariant tests). */
int kdo_step(double *S, const double *q, const double *k, const double *v,
             double beta, double c, const double *logf, int dk, int dv,
             double *o, double *b_out, double *u_out)
{
    if (!S || !q || !k || !v || !logf || !o || dk <= 0 || dv <= 0) return 1;
    kdo_token_step(S, q, k, v, beta, c, logf, dk, dv, o, b_out, u_out);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Thread pool over (b,h) units.                                            */
/* ------------------------------------------------------------------------ */
typedef struct {
    const double *q, *k, *v, *beta, *c, *logf, *S0, *dO, *dST;
    double *O, *ST, *bt, *ut;
    double *dq, *dk, *dv, *dbeta, *dc, *dlogf, *dS0;
    int B, H, T, DK, DV;
    int next;               /* next unit, guarded by mu */
    pthread_mutex_t mu;
    int status;
} kdo_job;

static int kdo_take(kdo_job *jb)
{
    pthread_mutex_lock(&jb->mu);
    int u = jb->next < jb->B * jb->H ? jb->next++ : -1;
    pthread_mutex_unlock(&jb->mu);
    return u;
}

static void kdo_fail(kdo_job *jb)
{
    pthread_mutex_lock(&jb->mu);
    jb->status = 2;
    pthread_mutex_unlock(&jb->mu);
}

static int kdo_threads(int want, int units)
{
    if (want <= 0) {
        long n = sysconf(_SC_NPROCESSORS_ONLN);
        want = n > 0 ? (int)n : 1;
    }
    if (want > units) want = units;
    return want < 1 ? 1 : want;
}

static void kdo_run(kdo_job *jb, void *(*fn)(void *), int nthreads)
{
    int n = kdo_threads(nthreads, jb->B * jb->H);
    if (n == 1) { fn(jb); return; }
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n);
    int started = 0;
    for (int i = 0; i < n; ++i)
        if (pthread_create(&th[i], NULL, fn, jb) == 0) ++started;
    if (started == 0) fn(jb);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
}

/* Gather token t of unit (b,h) from a [B,T,H,d] array. */
static inline const double *kdo_tok(const double *x, int b, int t, int h,
                                    int T, int H, int d)
{
    return x + (((size_t)b * T + t) * H + h) * (size_t)d;
}

/* ------------------------------------------------------------------------ */
/* Forward: token recurrence over t = 1..T for every (b,h).                 */
/* ------------------------------------------------------------------------ */
static void *kdo_fwd_worker(void *arg)
{
    kdo_job *jb = (kdo_job *)arg;
    const int T = jb->T, H = jb->H, DK = jb->DK, DV = jb->DV;
    double *S = (double *)malloc(sizeof(double) * (size_t)DK * DV);
    if (!S) { kdo_fail(jb); return NULL; }
    int unit;
    while ((unit = kdo_take(jb)) >= 0) {
        int b = unit / H, h = unit % H;
        size_t soff = (size_t)unit * DV * DK;
        if (jb->S0) memcpy(S, jb->S0 + soff, sizeof(double) * (size_t)DK * DV);
        else memset(S, 0, sizeof(double) * (size_t)DK * DV);
        for (int t = 0; t < T; ++t) {
            size_t g = ((size_t)b * T + t) * H + h;
            double bb, uu;
            kdo_token_step(S, kdo_tok(jb->q, b, t, h, T, H, DK),
                           kdo_tok(jb->k, b, t, h, T, H, DK),
                           kdo_tok(jb->v, b, t, h, T, H, DV), jb->beta[g],
                           jb->c[g], kdo_tok(jb->logf, b, t, h, T, H, DK), DK,
                           DV, jb->O + g * DV, &bb, &uu);
            if (jb->bt) jb->bt[g] = bb;
            if (jb->ut) jb->ut[g] = uu;
        }
        if (jb->ST) memcpy(jb->ST + soff, S, sizeof(double) * (size_t)DK * DV);
    }
    free(S);
    return NULL;
}

/*
 * kdo_fwd: O [B,T,H,dv] and ST [B,H,dv,dk] (nullable).  S0 nullable => 0.
 * bt, ut (nullable, [B,T,H]) receive the per-token association b_t and write
 * coefficient u_t.  nthreads <= 0 => all online cores.  Returns 0 on success.
 */
int kdo_fwd(const double *q, const double *k, const double *v,
            const double *beta, const double *c, const double *logf,
            const double *S0, double *O, double *ST, double *bt, double *ut,
            int B, int H, int T, int dk, int dv, int nthreads)
{
    if (!q || !k || !v || !beta || !c || !logf || !O) return 1;
    if (B <= 0 || H <= 0 || T < 0 || dk <= 0 || dv <= 0) return 1;
    kdo_job jb;
    memset(&jb, 0, sizeof(jb));
    jb.q = q; jb.k = k; jb.v = v; jb.beta = beta; jb.c = c; jb.logf = logf;
    jb.S0 = S0; jb.O = O; jb.ST = ST; jb.bt = bt; jb.ut = ut;
    jb.B = B; jb.H = H; jb.T = T; jb.DK = dk; jb.DV = dv;
    pthread_mutex_init(&jb.mu, NULL);
    kdo_run(&jb, kdo_fwd_worker, nthreads);
    pthread_mutex_destroy(&jb.mu);
    return jb.status;
}

/* ------------------------------------------------------------------------ */
/* Backward: reverse-mode of the token step, newest token first.            */
/*   G = dL/dS_t (starts at dST, or 0)                                      */
/*   G += dO_t q_t^T ; dq_t = S_t^T dO_t                                   */
/*   du = v^T G k ; dv = u G k ; dk = u G^T v                               */
/*   dc = du ; dbeta = -b du ; db = -beta du                                */
/*   Gbar = G + db v k^T ; dv += db Sbar k ; dk += db Sbar^T v              */
/*   dlogf_j = sum_r Gbar[r,j] Sbar[r,j] ; G = Gbar diag(f)                 */
/* States inside each 64-token segment are recomputed from a checkpoint.   */
/* ------------------------------------------------------------------------ */
static void *kdo_bwd_worker(void *arg)
{
    kdo_job *jb = (kdo_job *)arg;
    const int T = jb->T, H = jb->H, DK = jb->DK, DV = jb->DV;
    const size_t SZ = (size_t)DK * DV;
    const int nseg = (T + KDO_CKPT - 1) / KDO_CKPT;
    double *ckpt = (double *)malloc(sizeof(double) * SZ * (size_t)(nseg > 0 ? nseg : 1));
    /* seg[i] = state after token (seg_start + i - 1); seg[0] = checkpoint */
    double *seg = (double *)malloc(sizeof(double) * SZ * (KDO_CKPT + 1));
    double *G = (double *)malloc(sizeof(double) * SZ);
    double *Sbar = (double *)malloc(sizeof(double) * SZ);
    double *o = (double *)malloc(sizeof(double) * (size_t)DV);
    double *bseg = (double *)malloc(sizeof(double) * KDO_CKPT);
    double *useg = (double *)malloc(sizeof(double) * KDO_CKPT);
    if (!ckpt || !seg || !G || !Sbar || !o || !bseg || !useg) {
        kdo_fail(jb);
        free(ckpt); free(seg); free(G); free(Sbar); free(o); free(bseg); free(useg);
        return NULL;
    }
    int unit;
    while ((unit = kdo_take(jb)) >= 0) {
        int b = unit / H, h = unit % H;
        size_t soff = (size_t)unit * SZ;
        /* forward sweep, keeping one checkpoint per segment */
        double *S = seg; /* scratch */
        if (jb->S0) memcpy(S, jb->S0 + soff, sizeof(double) * SZ);
        else memset(S, 0, sizeof(double) * SZ);
        for (int t = 0; t < T; ++t) {
            if (t % KDO_CKPT == 0)
                memcpy(ckpt + (size_t)(t / KDO_CKPT) * SZ, S, sizeof(double) * SZ);
            size_t g = ((size_t)b * T + t) * H + h;
            kdo_token_step(S, kdo_tok(jb->q, b, t, h, T, H, DK),
                           kdo_tok(jb->k, b, t, h, T, H, DK),
                           kdo_tok(jb->v, b, t, h, T, H, DV), jb->beta[g],
                           jb->c[g], kdo_tok(jb->logf, b, t, h, T, H, DK), DK,
                           DV, o, NULL, NULL);
        }
        if (jb->dST) memcpy(G, jb->dST + soff, sizeof(double) * SZ);
        else memset(G, 0, sizeof(double) * SZ);

        for (int sgi = nseg - 1; sgi >= 0; --sgi) {
            int t0 = sgi * KDO_CKPT;
            int t1 = t0 + KDO_CKPT < T ? t0 + KDO_CKPT : T;
            /* recompute the states of this segment */
            memcpy(seg, ckpt + (size_t)sgi * SZ, sizeof(double) * SZ);
            for (int t = t0; t < t1; ++t) {
                double *Sn = seg + (size_t)(t - t0 + 1) * SZ;
                memcpy(Sn, seg + (size_t)(t - t0) * SZ, sizeof(double) * SZ);
                size_t g = ((size_t)b * T + t) * H + h;
                kdo_token_step(Sn, kdo_tok(jb->q, b, t, h, T, H, DK),
                               kdo_tok(jb->k, b, t, h, T, H, DK),
                               kdo_tok(jb->v, b, t, h, T, H, DV), jb->beta[g],
                               jb->c[g], kdo_tok(jb->logf, b, t, h, T, H, DK),
                               DK, DV, o, &bseg[t - t0], &useg[t - t0]);
            }
            for (int t = t1 - 1; t >= t0; --t) {
                size_t g = ((size_t)b * T + t) * H + h;
                const double *qt = kdo_tok(jb->q, b, t, h, T, H, DK);
                const double *kt = kdo_tok(jb->k, b, t, h, T, H, DK);
                const double *vt = kdo_tok(jb->v, b, t, h, T, H, DV);
                const double *lf = kdo_tok(jb->logf, b, t, h, T, H, DK);
                const double *dOt = kdo_tok(jb->dO, b, t, h, T, H, DV);
                const double *Sprev = seg + (size_t)(t - t0) * SZ;
                const double *Scur = seg + (size_t)(t - t0 + 1) * SZ;
                double *dqt = jb->dq + g * DK;
                double *dkt = jb->dk + g * DK;
                double *dvt = jb->dv + g * DV;
                double *dlf = jb->dlogf + g * DK;
                double beta = jb->beta[g];
                double bb = bseg[t - t0], uu = useg[t - t0];
                /* output o_t = S_t q_t */
                for (int r = 0; r < DV; ++r)
                    for (int j = 0; j < DK; ++j)
                        G[(size_t)r * DK + j] += dOt[r] * qt[j];
                for (int j = 0; j < DK; ++j) {
                    double acc = 0.0;
                    for (int r = 0; r < DV; ++r) acc += Scur[(size_t)r * DK + j] * dOt[r];
                    dqt[j] = acc;
                }
                /* S_t = Sbar + u v k^T */
                double du = 0.0;
                for (int r = 0; r < DV; ++r) {
                    double acc = 0.0;
                    for (int j = 0; j < DK; ++j) acc += G[(size_t)r * DK + j] * kt[j];
                    dvt[r] = uu * acc;
                    du += vt[r] * acc;
                }
                for (int j = 0; j < DK; ++j) {
                    double acc = 0.0;
                    for (int r = 0; r < DV; ++r) acc += G[(size_t)r * DK + j] * vt[r];
                    dkt[j] = uu * acc;
                }
                /* u = c - beta b */
                jb->dc[g] = du;
                jb->dbeta[g] = -bb * du;
                double db = -beta * du;
                /* b = v^T Sbar k ; Sbar = S_{t-1} diag(f) */
                for (int r = 0; r < DV; ++r)
                    for (int j = 0; j < DK; ++j)
                        Sbar[(size_t)r * DK + j] = Sprev[(size_t)r * DK + j] * exp(lf[j]);
                for (int r = 0; r < DV; ++r)
                    for (int j = 0; j < DK; ++j)
                        G[(size_t)r * DK + j] += db * vt[r] * kt[j];
                for (int r = 0; r < DV; ++r) {
                    double acc = 0.0;
                    for (int j = 0; j < DK; ++j) acc += Sbar[(size_t)r * DK + j] * kt[j];
                    dvt[r] += db * acc;
                }
                for (int j = 0; j < DK; ++j) {
                    double acc = 0.0, accl = 0.0;
                    for (int r = 0; r < DV; ++r) {
                        acc += Sbar[(size_t)r * DK + j] * vt[r];
                        accl += G[(size_t)r * DK + j] * Sbar[(size_t)r * DK + j];
                    }
                    dkt[j] += db * acc;
                    dlf[j] = accl;
                }
                for (int r = 0; r < DV; ++r)
                    for (int j = 0; j < DK; ++j)
                        G[(size_t)r * DK + j] *= exp(lf[j]);
            }
        }
        if (jb->dS0) memcpy(jb->dS0 + soff, G, sizeof(double) * SZ);
    }
    free(ckpt); free(seg); free(G); free(Sbar); free(o); free(bseg); free(useg);
    return NULL;
}

/*
 * kdo_bwd: gradients of the loss l = <dO, O> + <dST, S_T> with respect to
 * q, k, v, beta, c, logf and S0.  dST and S0 nullable (=> 0); dS0 nullable.
 */
int kdo_bwd(const double *q, const double *k, const double *v,
            const double *beta, const double *c, const double *logf,
            const double *S0, const double *dO, const double *dST, double *dq,
            double *dk, double *dv, double *dbeta, double *dc, double *dlogf,
            double *dS0, int B, int H, int T, int dk_, int dv_, int nthreads)
{
    if (!q || !k || !v || !beta || !c || !logf || !dO) return 1;
    if (!dq || !dk || !dv || !dbeta || !dc || !dlogf) return 1;
    if (B <= 0 || H <= 0 || T < 0 || dk_ <= 0 || dv_ <= 0) return 1;
    kdo_job jb;
    memset(&jb, 0, sizeof(jb));
    jb.q = q; jb.k = k; jb.v = v; jb.beta = beta; jb.c = c; jb.logf = logf;
    jb.S0 = S0; jb.dO = dO; jb.dST = dST;
    jb.dq = dq; jb.dk = dk; jb.dv = dv; jb.dbeta = dbeta; jb.dc = dc;
    jb.dlogf = dlogf; jb.dS0 = dS0;
    jb.B = B; jb.H = H; jb.T = T; jb.DK = dk_; jb.DV = dv_;
    pthread_mutex_init(&jb.mu, NULL);
    kdo_run(&jb, kdo_bwd_worker, nthreads);
    pthread_mutex_destroy(&jb.mu);
    return jb.status;
}

/*
 * kdo_decode: one token per (b,h).  S [B,H,dv,dk] updated in place;
 * q,k [B,H,dk], v [B,H,dv], beta,c [B,H], logf [B,H,dk] -> o [B,H,dv].
 * The same step as the forward recurrence with T = 1.
 */
int kdo_decode(const double *q, const double *k, const double *v,
               const double *beta, const double *c, const double *logf,
               double *S, double *o, int B, int H, int dk, int dv)
{
    if (!q || !k || !v || !beta || !c || !logf || !S || !o) return 1;
    if (B <= 0 || H <= 0 || dk <= 0 || dv <= 0) return 1;
    for (int unit = 0; unit < B * H; ++unit)
        kdo_token_step(S + (size_t)unit * dv * dk, q + (size_t)unit * dk,
                       k + (size_t)unit * dk, v + (size_t)unit * dv,
                       beta[unit], c[unit], logf + (size_t)unit * dk, dk, dv,
                       o + (size_t)unit * dv, NULL, NULL);
    return 0;
}
