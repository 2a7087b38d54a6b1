/*
 * gdr_oracle.c -- fp64 CPU oracle of the gated delta rule.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark load this file's library.  It shares no code, header,
 * table or constant with the CUDA library and never touches a GPU.
 *
 * What it computes: the plain token-by-token recurrence, in the d_v x d_k
 * orientation,
 *
 *     S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = S_t q_t,
 *
 * as the first line of the induction in "Reading notes: Kimi Delta
 * Attention" (mzeromiko), section 4 "Forward pass", writes it:
 * S_t = S_{t-1}Diag(alpha_t) + beta_t (v_t - S_{t-1}Diag(alpha_t) k_t) k_t^T.
 * Each token is done in the order the pseudo-code of "KDA vs Gated DeltaNet"
 * (brenchcc), section 4 "How the source maps to the formulas", gives:
 * decay the state, predict the value from the decayed state, form the
 * delta, write it along the key, read the output with the query.
 *
 *   - per-channel gate (KDA): alpha_t = exp(max(g_t, -5)) per key channel;
 *     the -5 lower bound is the g_min of the KDA gate in "Lightweight LLM
 *     reproduction: Linear Attention" (aitujian), section 3.1 [7a].
 *   - scalar gate (Gated DeltaNet): alpha_t = exp(g_t) for the whole head,
 *     "Token Mixer I", section "Gated Delta Networks" (no bound applied).
 *
 * Oracle-only extension used by the pins: the erase and write strengths may
 * be given apart from beta (the tied-scalar case of Gated DeltaNet-2's erase
 * and write gates, "Token Mixer I", section "Gated DeltaNet-2 / Decoupling
 * erase and write"): delta = w_t v_t - e_t (S~ k_t).  With e = w = beta it is
 * the method itself; e = 0, w = 1 gives (gated) linear attention.
 *
 * Gated Delta Rule-2 (gdr2_oracle_forward): the erase gate b_t in [0,1]^dk
 * and the write gate w_t in [0,1]^dv of "Token Mixer I", section "Gated
 * DeltaNet-2: Decoupling Erase and Write in Linear Attention", eq. (10).  The
 * state is read along e_t = b_t * k_t (elementwise) and the written target is
 * z_t = w_t * v_t; the write direction stays k_t.  In this orientation:
 *
 *     S~ = S_{t-1} Diag(alpha_t),   delta = w_t * v_t - S~ (b_t * k_t),
 *     S_t = S~ + delta k_t^T,       o_t = S_t q_t,
 *
 * the residual z_t - S~^T e_t of the section's fast-weight paragraph, taken
 * in the same order as above (decay, read, delta, write, read out).
 *
 * Layouts (row-major, contiguous, fp64):
 *   q, k   [B,H,T,dk]      v, O [B,H,T,dv]
 *   g      [B,H,T,dk] (per-channel) or [B,H,T] (scalar)
 *   beta, erase, write  [B,H,T]      (erase / write may be NULL -> beta)
 *   GDR-2: b [B,H,T,dk], w [B,H,T,dv] (in place of beta)
 *   S0, S_T [B,H,dv,dk]              (S0 NULL -> zeros, S_T NULL -> not written)
 * Heads are independent; they are spread over nthreads POSIX threads
 * (nthreads <= 0 -> all online cores).  Returns 0, or -1 on a bad argument
 * or allocation failure.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    const double *q, *k, *v, *g, *beta, *erase, *write, *S0;
    const double *eb, *ww;   /* GDR-2 erase gate [B,H,T,dk] and write gate [B,H,T,dv], or NULL */
    double *O, *S_T;
    int B, H, T, dk, dv, per_channel, clamp;
    int head_begin, head_end;
    int status;
} oracle_job;

static void run_head(const oracle_job *J, int head, double *S, double *a, double *delta, double *ek)
{
    const int T = J->T, dk = J->dk, dv = J->dv;
    const size_t hk = (size_t)head * T * dk, hv = (size_t)head * T * dv, hs = (size_t)head * T;
    const size_t hS = (size_t)head * dv * dk;

    if (J->S0) memcpy(S, J->S0 + hS, sizeof(double) * dv * dk);
    else memset(S, 0, sizeof(double) * dv * dk);

    for (int t = 0; t < T; ++t) {
        const double *qt = J->q + hk + (size_t)t * dk;
        const double *kt = J->k + hk + (size_t)t * dk;
        const double *vt = J->v + hv + (size_t)t * dv;
        double *ot = J->O + hv + (size_t)t * dv;

        /* gate: alpha_t */
        if (J->per_channel) {
            const double *gt = J->g + hk + (size_t)t * dk;
            for (int c = 0; c < dk; ++c) {
                double gc = gt[c];
                if (J->clamp && gc < -5.0) gc = -5.0;
                a[c] = exp(gc);
            }
        } else {
            const double as = exp(J->g[hs + t]);
            for (int c = 0; c < dk; ++c) a[c] = as;
        }
        if (J->eb) {
            /* GDR-2: decay, read along e = b * k, delta = w * v - S~ e */
            const double *bt = J->eb + hk + (size_t)t * dk;
            const double *wt = J->ww + hv + (size_t)t * dv;
            for (int c = 0; c < dk; ++c) ek[c] = bt[c] * kt[c];
            for (int i = 0; i < dv; ++i) {
                double *row = S + (size_t)i * dk;
                double p = 0.0;
                for (int c = 0; c < dk; ++c) {
                    row[c] *= a[c];
                    p += row[c] * ek[c];
                }
                delta[i] = wt[i] * vt[i] - p;
            }
        } else {
            const double e = J->erase ? J->erase[hs + t] : J->beta[hs + t];
            const double w = J->write ? J->write[hs + t] : J->beta[hs + t];

            /* decay, then predict from the decayed state: p = S~ k */
            for (int i = 0; i < dv; ++i) {
                double *row = S + (size_t)i * dk;
                double p = 0.0;
                for (int c = 0; c < dk; ++c) {
                    row[c] *= a[c];
                    p += row[c] * kt[c];
                }
                delta[i] = w * vt[i] - e * p;
            }
        }
        /* write the delta along k, then read with q: o = S_t q */
        for (int i = 0; i < dv; ++i) {
            double *row = S + (size_t)i * dk;
            double o = 0.0;
            for (int c = 0; c < dk; ++c) {
                row[c] += delta[i] * kt[c];
                o += row[c] * qt[c];
            }
            ot[i] = o;
        }
    }
    if (J->S_T) memcpy(J->S_T + hS, S, sizeof(double) * dv * dk);
}

static void *worker(void *arg)
{
    oracle_job *J = (oracle_job *)arg;
    double *S = (double *)malloc(sizeof(double) * (size_t)J->dv * J->dk);
    double *a = (double *)malloc(sizeof(double) * (size_t)J->dk);
    double *delta = (double *)malloc(sizeof(double) * (size_t)J->dv);
    double *ek = (double *)malloc(sizeof(double) * (size_t)J->dk);
    if (!S || !a || !delta || !ek) {
        J->status = -1;
    } else {
        for (int h = J->head_begin; h < J->head_end; ++h) run_head(J, h, S, a, delta, ek);
    }
    free(ek);
    free(S);
    free(a);
    free(delta);
    return NULL;
}

static int run_jobs(const double *q, const double *k, const double *v, const double *g,
                    const double *beta, const double *erase, const double *write,
                    const double *eb, const double *ww,
                    const double *S0, double *O, double *S_T,
                    int B, int H, int T, int dk, int dv,
                    int gate_scalar, int clamp, int nthreads)
{
    const int heads = B * H;
    if (heads == 0) return 0;
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > heads) nthreads = heads;

    oracle_job *jobs = (oracle_job *)calloc((size_t)nthreads, sizeof(oracle_job));
    pthread_t *tid = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !tid) {
        free(jobs);
        free(tid);
        return -1;
    }
    int status = 0;
    for (int j = 0; j < nthreads; ++j) {
        oracle_job *J = &jobs[j];
        J->q = q; J->k = k; J->v = v; J->g = g; J->beta = beta;
        J->erase = erase; J->write = write; J->S0 = S0; J->O = O; J->S_T = S_T;
        J->eb = eb; J->ww = ww;
        J->B = B; J->H = H; J->T = T; J->dk = dk; J->dv = dv;
        J->per_channel = !gate_scalar;
        J->clamp = clamp;
        J->head_begin = (int)((long long)heads * j / nthreads);
        J->head_end = (int)((long long)heads * (j + 1) / nthreads);
        J->status = 0;
    }
    int started = 0;
    for (int j = 1; j < nthreads; ++j) {
        if (pthread_create(&tid[j], NULL, worker, &jobs[j]) != 0) {
            /* fall back to running this share on the calling thread */
            worker(&jobs[j]);
            tid[j] = 0;
        } else {
            ++started;
        }
    }
    worker(&jobs[0]);
    for (int j = 1; j < nthreads; ++j)
        if (tid[j]) pthread_join(tid[j], NULL);
    for (int j = 0; j < nthreads; ++j)
        if (jobs[j].status) status = -1;
    (void)started;
    free(jobs);
    free(tid);
    return status;
}

int gdr_oracle_forward(const double *q, const double *k, const double *v, const double *g,
                       const double *beta, const double *erase, const double *write,
                       const double *S0, double *O, double *S_T,
                       int B, int H, int T, int dk, int dv,
                       int gate_scalar, int clamp, int nthreads)
{
    if (!q || !k || !v || !g || !O || B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return -1;
    if (!beta && (!erase || !write)) return -1;
    return run_jobs(q, k, v, g, beta, erase, write, NULL, NULL, S0, O, S_T, B, H, T, dk, dv, gate_scalar, clamp,
                    nthreads);
}

/* Gated Delta Rule-2: b [B,H,T,dk] erase gate, w [B,H,T,dv] write gate (both required). */
int gdr2_oracle_forward(const double *q, const double *k, const double *v, const double *g,
                        const double *b, const double *w, const double *S0, double *O, double *S_T,
                        int B, int H, int T, int dk, int dv, int gate_scalar, int clamp, int nthreads)
{
    if (!q || !k || !v || !g || !b || !w || !O || B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return -1;
    return run_jobs(q, k, v, g, NULL, NULL, NULL, b, w, S0, O, S_T, B, H, T, dk, dv, gate_scalar, clamp, nthreads);
}

/*
 * Backward pass (reverse mode through the same token recurrence), the
 * reference of the library's chunked backward.  Given dO [B,H,T,dv] and
 * dS_T [B,H,dv,dk] (NULL -> zeros) it returns the gradients of
 * L = <dO, O> + <dS_T, S_T> with respect to q, k ([B,H,T,dk]), v ([B,H,T,dv]),
 * g (the layout of g), beta ([B,H,T]) and S0 ([B,H,dv,dk]; dS0 may be NULL).
 * Each token's forward step (decay, predict, delta, write, read out) is
 * undone in reverse order with the chain rule; the per-channel -5 bound
 * passes the gradient where g >= -5 and blocks it below.  States are
 * recomputed forward from checkpoints every 64 tokens (plain recomputation,
 * no algebra).
 */
typedef struct {
    const double *q, *k, *v, *g, *beta, *S0, *dO, *dST;
    double *dq, *dk, *dv, *dg, *dbeta, *dS0;
    int B, H, T, dk_, dv_, per_channel, clamp;
    int head_begin, head_end;
    int status;
} bwd_job;

#define SEG 64

static void decay_of(const bwd_job *J, int head, int t, double *a, double *gate_pass)
{
    const int dk = J->dk_, T = J->T;
    if (J->per_channel) {
        const double *gt = J->g + ((size_t)head * T + t) * dk;
        for (int c = 0; c < dk; ++c) {
            double gc = gt[c];
            gate_pass[c] = 1.0;
            if (J->clamp && gc < -5.0) {
                gc = -5.0;
                gate_pass[c] = 0.0;
            }
            a[c] = exp(gc);
        }
    } else {
        const double as = exp(J->g[(size_t)head * T + t]);
        for (int c = 0; c < dk; ++c) {
            a[c] = as;
            gate_pass[c] = 1.0;
        }
    }
}

/* one forward token step from S (in place): returns p = S~ k and delta in the buffers */
static void fwd_step(const bwd_job *J, int head, int t, double *S, const double *a, double *p, double *delta)
{
    const int dk = J->dk_, dv = J->dv_, T = J->T;
    const double *kt = J->k + ((size_t)head * T + t) * dk;
    const double *vt = J->v + ((size_t)head * T + t) * dv;
    const double b = J->beta[(size_t)head * T + t];
    for (int i = 0; i < dv; ++i) {
        double *row = S + (size_t)i * dk, acc = 0.0;
        for (int c = 0; c < dk; ++c) {
            row[c] *= a[c];
            acc += row[c] * kt[c];
        }
        p[i] = acc;
        delta[i] = b * (vt[i] - acc);
    }
    for (int i = 0; i < dv; ++i) {
        double *row = S + (size_t)i * dk;
        for (int c = 0; c < dk; ++c) row[c] += delta[i] * kt[c];
    }
}

static void bwd_head(const bwd_job *J, int head, double *ckpt, double *seg, double *dS, double *a, double *gp,
                     double *p, double *delta, double *ddelta, double *tmp)
{
    const int T = J->T, dk = J->dk_, dv = J->dv_;
    const size_t SS = (size_t)dv * dk;
    const int nseg = (T + SEG - 1) / SEG;
    /* forward: checkpoints S at the start of every segment */
    double *S = seg;   /* scratch */
    if (J->S0) memcpy(S, J->S0 + (size_t)head * SS, sizeof(double) * SS);
    else memset(S, 0, sizeof(double) * SS);
    for (int s = 0; s < nseg; ++s) {
        memcpy(ckpt + (size_t)s * SS, S, sizeof(double) * SS);
        const int e = (s + 1) * SEG < T ? (s + 1) * SEG : T;
        for (int t = s * SEG; t < e; ++t) {
            decay_of(J, head, t, a, gp);
            fwd_step(J, head, t, S, a, p, delta);
        }
    }
    /* reverse */
    if (J->dST) memcpy(dS, J->dST + (size_t)head * SS, sizeof(double) * SS);
    else memset(dS, 0, sizeof(double) * SS);
    for (int s = nseg - 1; s >= 0; --s) {
        const int t0 = s * SEG, e = (s + 1) * SEG < T ? (s + 1) * SEG : T;
        /* states S_{t-1} for t in [t0, e): seg[t - t0] */
        memcpy(seg, ckpt + (size_t)s * SS, sizeof(double) * SS);
        for (int t = t0; t < e - 1; ++t) {
            memcpy(seg + (size_t)(t - t0 + 1) * SS, seg + (size_t)(t - t0) * SS, sizeof(double) * SS);
            decay_of(J, head, t, a, gp);
            fwd_step(J, head, t, seg + (size_t)(t - t0 + 1) * SS, a, p, delta);
        }
        for (int t = e - 1; t >= t0; --t) {
            const double *Sp = seg + (size_t)(t - t0) * SS;   /* S_{t-1} */
            const size_t tk = ((size_t)head * T + t) * dk, tv = ((size_t)head * T + t) * dv;
            const double *qt = J->q + tk, *kt = J->k + tk, *vt = J->v + tv, *dOt = J->dO + tv;
            const double b = J->beta[(size_t)head * T + t];
            decay_of(J, head, t, a, gp);
            /* recompute S~ (tmp), p, delta and S_t (tmp + delta k^T) */
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int c = 0; c < dk; ++c) {
                    tmp[(size_t)i * dk + c] = Sp[(size_t)i * dk + c] * a[c];
                    acc += tmp[(size_t)i * dk + c] * kt[c];
                }
                p[i] = acc;
                delta[i] = b * (vt[i] - acc);
            }
            /* o_t = S_t q_t: dS_t += dO_t q_t^T; dq_t = S_t^T dO_t */
            double *dqt = J->dq + tk, *dkt = J->dk + tk;
            for (int c = 0; c < dk; ++c) dqt[c] = 0.0, dkt[c] = 0.0;
            for (int i = 0; i < dv; ++i)
                for (int c = 0; c < dk; ++c) {
                    const double st = tmp[(size_t)i * dk + c] + delta[i] * kt[c];
                    dqt[c] += st * dOt[i];
                    dS[(size_t)i * dk + c] += dOt[i] * qt[c];
                }
            /* S_t = S~ + delta k^T: d delta = dS_t k; dk += dS_t^T delta; dS~ = dS_t */
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int c = 0; c < dk; ++c) {
                    acc += dS[(size_t)i * dk + c] * kt[c];
                    dkt[c] += dS[(size_t)i * dk + c] * delta[i];
                }
                ddelta[i] = acc;
            }
            /* delta = beta (v - p) */
            double db = 0.0;
            double *dvt = J->dv + tv;
            for (int i = 0; i < dv; ++i) {
                db += ddelta[i] * (vt[i] - p[i]);
                dvt[i] = b * ddelta[i];
            }
            J->dbeta[(size_t)head * T + t] = db;
            /* p = S~ k: dS~ += dp k^T (dp = -beta d delta); dk += S~^T dp */
            for (int i = 0; i < dv; ++i) {
                const double dp = -b * ddelta[i];
                for (int c = 0; c < dk; ++c) {
                    dS[(size_t)i * dk + c] += dp * kt[c];
                    dkt[c] += tmp[(size_t)i * dk + c] * dp;
                }
            }
            /* S~ = S_{t-1} Diag(a): da = sum_i dS~ * S_{t-1}; dS_{t-1} = dS~ Diag(a) */
            double dgs = 0.0;
            for (int c = 0; c < dk; ++c) {
                double da = 0.0;
                for (int i = 0; i < dv; ++i) da += dS[(size_t)i * dk + c] * Sp[(size_t)i * dk + c];
                const double dgc = da * a[c] * gp[c];
                if (J->per_channel) J->dg[tk + c] = dgc;
                else dgs += dgc;
            }
            if (!J->per_channel) J->dg[(size_t)head * T + t] = dgs;
            for (int i = 0; i < dv; ++i)
                for (int c = 0; c < dk; ++c) dS[(size_t)i * dk + c] *= a[c];
        }
    }
    if (J->dS0) memcpy(J->dS0 + (size_t)head * SS, dS, sizeof(double) * SS);
}

static void *bwd_worker(void *arg)
{
    bwd_job *J = (bwd_job *)arg;
    const int dk = J->dk_, dv = J->dv_;
    const size_t SS = (size_t)dv * dk;
    const int nseg = (J->T + SEG - 1) / SEG;
    const int md = dk > dv ? dk : dv;
    double *ckpt = (double *)malloc(sizeof(double) * SS * (size_t)(nseg > 0 ? nseg : 1));
    double *seg = (double *)malloc(sizeof(double) * SS * SEG);
    double *dS = (double *)malloc(sizeof(double) * SS);
    double *tmp = (double *)malloc(sizeof(double) * SS);
    double *a = (double *)malloc(sizeof(double) * dk), *gp = (double *)malloc(sizeof(double) * dk);
    double *p = (double *)malloc(sizeof(double) * md), *delta = (double *)malloc(sizeof(double) * dv);
    double *ddelta = (double *)malloc(sizeof(double) * dv);
    if (!ckpt || !seg || !dS || !tmp || !a || !gp || !p || !delta || !ddelta) J->status = -1;
    else
        for (int h = J->head_begin; h < J->head_end; ++h) bwd_head(J, h, ckpt, seg, dS, a, gp, p, delta, ddelta, tmp);
    free(ckpt); free(seg); free(dS); free(tmp); free(a); free(gp); free(p); free(delta); free(ddelta);
    return NULL;
}

int gdr_oracle_backward(const double *q, const double *k, const double *v, const double *g, const double *beta,
                        const double *S0, const double *dO, const double *dST,
                        double *dq, double *dk, double *dv, double *dg, double *dbeta, double *dS0,
                        int B, int H, int T, int dk_, int dv_, int gate_scalar, int clamp, int nthreads)
{
    if (!q || !k || !v || !g || !beta || !dO || !dq || !dk || !dv || !dg || !dbeta) return -1;
    if (B < 0 || H < 0 || T < 0 || dk_ <= 0 || dv_ <= 0) return -1;
    const int heads = B * H;
    if (heads == 0) return 0;
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > heads) nthreads = heads;
    bwd_job *jobs = (bwd_job *)calloc((size_t)nthreads, sizeof(bwd_job));
    pthread_t *tid = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !tid) {
        free(jobs);
        free(tid);
        return -1;
    }
    for (int j = 0; j < nthreads; ++j) {
        bwd_job *J = &jobs[j];
        J->q = q; J->k = k; J->v = v; J->g = g; J->beta = beta; J->S0 = S0; J->dO = dO; J->dST = dST;
        J->dq = dq; J->dk = dk; J->dv = dv; J->dg = dg; J->dbeta = dbeta; J->dS0 = dS0;
        J->B = B; J->H = H; J->T = T; J->dk_ = dk_; J->dv_ = dv_;
        J->per_channel = !gate_scalar;
        J->clamp = clamp;
        J->head_begin = (int)((long long)heads * j / nthreads);
        J->head_end = (int)((long long)heads * (j + 1) / nthreads);
    }
    for (int j = 1; j < nthreads; ++j)
        if (pthread_create(&tid[j], NULL, bwd_worker, &jobs[j]) != 0) {
            bwd_worker(&jobs[j]);
            tid[j] = 0;
        }
    bwd_worker(&jobs[0]);
    int status = 0;
    for (int j = 1; j < nthreads; ++j)
        if (tid[j]) pthread_join(tid[j], NULL);
    for (int j = 0; j < nthreads; ++j)
        if (jobs[j].status) status = -1;
    free(jobs);
    free(tid);
    return status;
}

int gdr_oracle_online_cores(void)
{
    return (int)sysconf(_SC_NPROCESSORS_ONLN);
}
