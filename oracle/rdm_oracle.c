/*
 * rdm_oracle.c -- plain fp64 CPU oracle for the DDTS-gated linear-attention
 * recurrence of Rodimus.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check
 * and the CPU-baseline leg of the bench call it; the product path never does.
 * It shares no source, header or helper with the CUDA library.
 *
 * What it computes (per batch b and head h, token by token, in double):
 *
 *   gates   alpha_t     = exp(-g_t * tau_t)                 (element-wise over d_k)
 *           alpha_hat_t = g_t ^ tau_t  (C pow: 0^0 = 1, 0^x = 0 for x > 0)
 *     "Rodimus*: Breaking the Accuracy-Efficiency Trade-Off with Efficient
 *      Attentions", digest.lyk-ai.com summary, section "Method", first Rodimus
 *      bullet (the DDTS selection gate g_t and temperature gate tau_t).
 *   state   S_t = diag(alpha_t) S_{t-1} + (alpha_hat_t * k_t)(beta_hat_t * v_t)^T
 *   readout o_t = S_t^T q_t          (the state after the update of token t)
 *     The update is diagonal along the key dimension n = d_k (paperhub.cn
 *     OpenReview rebuttal, "Efficient Parallelization" bullet, pointing to
 *     Sec. 3.1.3 / App. B3); beta_hat gates the input side only (atlas.scime.ai
 *     summary, ablation table rows on hat-beta and on beta in the transition);
 *     the state is a fixed d_k x d_v matrix carried across tokens (paperhub.cn
 *     rebuttal Q2 and Q5-3, Table 4 "State size n x m").
 *
 * Feedthrough (optional): o_t += d (.) v_t with d one weight per head and value
 *   channel, d[h][j]: the feedthrough d_t of the paper's Eq. (11), which the
 *   paperhub.cn OpenReview rebuttal (answer to Q6) names the SSM feedthrough
 *   as used in Mamba and Mamba2, a learned skip from the SSM input (here v_t)
 *   to the output.  Its shape and input are not printed; this is the reading.
 *
 * Backward: reverse-mode differentiation of exactly that loop, step by step
 * (no chunking, no cumulative-sum identities).  States S_{t-1} needed by the
 * reverse step are recomputed from checkpoints taken every CKPT tokens.
 *
 * Layouts: sequences [B,H,T,D] row-major, states [B,H,d_k,d_v], decode inputs
 * [B,H,D].  All arrays are double.  Work is split over (b,h) pairs across
 * nthreads POSIX threads (nthreads <= 0 means 1).
 *
 * Conventions at the edge of the domain (g >= 0, tau >= 0 assumed):
 *   d alpha_hat / d g   = tau * g^(tau-1)     (0 when tau == 0; +inf at g == 0, tau < 1)
 *   d alpha_hat / d tau = alpha_hat * ln g    (0 when alpha_hat == 0)
 *
 * Return value: 0 on success, -1 on a bad argument or an allocation failure.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

#define CKPT 64

typedef struct {
    int B, H, T, dk, dv;
    const double *q, *k, *v, *g, *tau, *beta, *S0, *dO, *dST;
    double *o, *ST;
    double *dq, *dk_, *dv_, *dg, *dtau, *dbeta, *dS0;
    const double *dfeed;    /* feedthrough weights [H][dv], or NULL */
    double *ddfeed;         /* per-(b,h) feedthrough gradient [B*H][dv], or NULL */
    int next;               /* next (b,h) pair to take */
    int failed;
    pthread_mutex_t lock;
} job_t;

static double gate_alpha(double g, double tau) { return exp(-g * tau); }
static double gate_alpha_hat(double g, double tau) { return pow(g, tau); }

/* One token of the recurrence for one (b,h):  S <- diag(alpha) S + khat vhat^T,
 * then o = S^T q.  x_t vectors are the token's rows. */
static void step_token(int dk, int dv, const double *q, const double *k, const double *v,
                       const double *g, const double *tau, const double *beta,
                       double *S, double *o)
{
    for (int i = 0; i < dk; ++i) {
        double al = gate_alpha(g[i], tau[i]);
        double kh = gate_alpha_hat(g[i], tau[i]) * k[i];
        double *row = S + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) row[j] = al * row[j] + kh * (beta[j] * v[j]);
    }
    if (o) {
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * q[i];
            o[j] = acc;
        }
    }
}

/* Feedthrough of one token: o += d (.) v. */
static void add_feedthrough(int dv, const double *d, const double *v, double *o)
{
    for (int j = 0; j < dv; ++j) o[j] += d[j] * v[j];
}

static int take_pair(job_t *J)
{
    pthread_mutex_lock(&J->lock);
    int p = J->next < J->B * J->H ? J->next++ : -1;
    pthread_mutex_unlock(&J->lock);
    return p;
}

/* ---------------------------------------------------------------- forward */
static void *fwd_worker(void *arg)
{
    job_t *J = (job_t *)arg;
    const int T = J->T, dk = J->dk, dv = J->dv;
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    if (!S) { J->failed = 1; return NULL; }
    for (int p; (p = take_pair(J)) >= 0;) {
        size_t sk = (size_t)p * T * dk, sv = (size_t)p * T * dv, ss = (size_t)p * dk * dv;
        if (J->S0) memcpy(S, J->S0 + ss, sizeof(double) * dk * dv);
        else memset(S, 0, sizeof(double) * dk * dv);
        for (int t = 0; t < T; ++t) {
            size_t ok = sk + (size_t)t * dk, ov = sv + (size_t)t * dv;
            step_token(dk, dv, J->q + ok, J->k + ok, J->v + ov, J->g + ok, J->tau + ok,
                       J->beta + ov, S, J->o ? J->o + ov : NULL);
            if (J->o && J->dfeed) add_feedthrough(dv, J->dfeed + (size_t)(p % J->H) * dv,
                                                  J->v + ov, J->o + ov);
        }
        if (J->ST) memcpy(J->ST + ss, S, sizeof(double) * dk * dv);
    }
    free(S);
    return NULL;
}

static int run_pool(job_t *J, void *(*fn)(void *), int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > J->B * J->H) nthreads = J->B * J->H;
    if (nthreads < 1) return 0;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    if (!th) return -1;
    pthread_mutex_init(&J->lock, NULL);
    J->next = 0;
    J->failed = 0;
    int started = 0;
    for (int i = 0; i < nthreads; ++i)
        if (pthread_create(&th[i], NULL, fn, J) == 0) ++started;
    if (started == 0) fn(J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&J->lock);
    free(th);
    return J->failed ? -1 : 0;
}

static int dims_ok(int B, int H, int T, int dk, int dv)
{
    return B >= 0 && H >= 0 && T >= 0 && dk > 0 && dv > 0;
}

int rdm_oracle_fwd(int B, int H, int T, int dk, int dv,
                   const double *q, const double *k, const double *v,
                   const double *g, const double *tau, const double *beta,
                   const double *S0, const double *dfeed, double *o, double *ST, int nthreads)
{
    if (!dims_ok(B, H, T, dk, dv)) return -1;
    if (T > 0 && (!q || !k || !v || !g || !tau || !beta)) return -1;
    job_t J;
    memset(&J, 0, sizeof(J));
    J.B = B; J.H = H; J.T = T; J.dk = dk; J.dv = dv;
    J.q = q; J.k = k; J.v = v; J.g = g; J.tau = tau; J.beta = beta; J.S0 = S0;
    J.o = o; J.ST = ST; J.dfeed = dfeed;
    return run_pool(&J, fwd_worker, nthreads);
}

/* ----------------------------------------------------------------- decode */
static void *decode_worker(void *arg)
{
    job_t *J = (job_t *)arg;
    const int dk = J->dk, dv = J->dv;
    for (int p; (p = take_pair(J)) >= 0;) {
        size_t ok = (size_t)p * dk, ov = (size_t)p * dv;
        step_token(dk, dv, J->q + ok, J->k + ok, J->v + ov, J->g + ok, J->tau + ok,
                   J->beta + ov, J->ST + (size_t)p * dk * dv, J->o ? J->o + ov : NULL);
        if (J->o && J->dfeed) add_feedthrough(dv, J->dfeed + (size_t)(p % J->H) * dv,
                                              J->v + ov, J->o + ov);
    }
    return NULL;
}

/* One token for every (b,h): S [B,H,dk,dv] updated in place, o [B,H,dv]
 * (o may be NULL).  The same step function as the forward loop. */
int rdm_oracle_decode_step(int B, int H, int dk, int dv,
                           const double *q, const double *k, const double *v,
                           const double *g, const double *tau, const double *beta,
                           const double *dfeed, double *S, double *o, int nthreads)
{
    if (!dims_ok(B, H, 1, dk, dv) || !S || !q || !k || !v || !g || !tau || !beta) return -1;
    job_t J;
    memset(&J, 0, sizeof(J));
    J.B = B; J.H = H; J.T = 1; J.dk = dk; J.dv = dv;
    J.q = q; J.k = k; J.v = v; J.g = g; J.tau = tau; J.beta = beta;
    J.ST = S; J.o = o; J.dfeed = dfeed;
    return run_pool(&J, decode_worker, nthreads);
}

/* --------------------------------------------------------------- backward */
static void *bwd_worker(void *arg)
{
    job_t *J = (job_t *)arg;
    const int T = J->T, dk = J->dk, dv = J->dv;
    const size_t SS = (size_t)dk * dv;
    const int nck = (T + CKPT - 1) / CKPT;
    /* ck[c] = state before token c*CKPT; seg[u] = state after token c*CKPT+u-1 */
    double *ck = (double *)malloc(sizeof(double) * SS * (size_t)(nck > 0 ? nck : 1));
    double *seg = (double *)malloc(sizeof(double) * SS * (CKPT + 1));
    double *dS = (double *)malloc(sizeof(double) * SS);
    double *al = (double *)malloc(sizeof(double) * dk);
    double *ah = (double *)malloc(sizeof(double) * dk);
    double *kh = (double *)malloc(sizeof(double) * dk);
    double *vh = (double *)malloc(sizeof(double) * dv);
    double *dkh = (double *)malloc(sizeof(double) * dk);
    double *dvh = (double *)malloc(sizeof(double) * dv);
    double *dal = (double *)malloc(sizeof(double) * dk);
    if (!ck || !seg || !dS || !al || !ah || !kh || !vh || !dkh || !dvh || !dal) {
        J->failed = 1;
        goto out;
    }
    for (int p; (p = take_pair(J)) >= 0;) {
        size_t sk = (size_t)p * T * dk, sv = (size_t)p * T * dv, ss = (size_t)p * SS;
        /* forward sweep: checkpoints only */
        double *S = seg;
        if (J->S0) memcpy(S, J->S0 + ss, sizeof(double) * SS);
        else memset(S, 0, sizeof(double) * SS);
        for (int t = 0; t < T; ++t) {
            if (t % CKPT == 0) memcpy(ck + (size_t)(t / CKPT) * SS, S, sizeof(double) * SS);
            size_t ok = sk + (size_t)t * dk, ov = sv + (size_t)t * dv;
            step_token(dk, dv, J->q + ok, J->k + ok, J->v + ov, J->g + ok, J->tau + ok,
                       J->beta + ov, S, NULL);
        }
        /* reverse sweep */
        if (J->dST) memcpy(dS, J->dST + ss, sizeof(double) * SS);
        else memset(dS, 0, sizeof(double) * SS);
        for (int c = nck - 1; c >= 0; --c) {
            int t0 = c * CKPT, t1 = t0 + CKPT < T ? t0 + CKPT : T;
            memcpy(seg, ck + (size_t)c * SS, sizeof(double) * SS);
            for (int t = t0; t < t1; ++t) {
                memcpy(seg + (size_t)(t - t0 + 1) * SS, seg + (size_t)(t - t0) * SS,
                       sizeof(double) * SS);
                size_t ok = sk + (size_t)t * dk, ov = sv + (size_t)t * dv;
                step_token(dk, dv, J->q + ok, J->k + ok, J->v + ov, J->g + ok, J->tau + ok,
                           J->beta + ov, seg + (size_t)(t - t0 + 1) * SS, NULL);
            }
            for (int t = t1 - 1; t >= t0; --t) {
                const double *St = seg + (size_t)(t - t0 + 1) * SS;   /* S_t     */
                const double *Sp = seg + (size_t)(t - t0) * SS;       /* S_{t-1} */
                size_t ok = sk + (size_t)t * dk, ov = sv + (size_t)t * dv;
                const double *q = J->q + ok, *k = J->k + ok, *g = J->g + ok, *tau = J->tau + ok;
                const double *v = J->v + ov, *beta = J->beta + ov, *dO = J->dO + ov;
                for (int i = 0; i < dk; ++i) {
                    al[i] = gate_alpha(g[i], tau[i]);
                    ah[i] = gate_alpha_hat(g[i], tau[i]);
                    kh[i] = ah[i] * k[i];
                }
                for (int j = 0; j < dv; ++j) vh[j] = beta[j] * v[j];
                /* readout o_t = S_t^T q_t */
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) dS[(size_t)i * dv + j] += q[i] * dO[j];
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += St[(size_t)i * dv + j] * dO[j];
                    J->dq[ok + i] = acc;
                }
                /* update S_t = diag(al) S_{t-1} + kh vh^T */
                for (int i = 0; i < dk; ++i) {
                    double a1 = 0.0, a2 = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        a1 += dS[(size_t)i * dv + j] * vh[j];
                        a2 += dS[(size_t)i * dv + j] * Sp[(size_t)i * dv + j];
                    }
                    dkh[i] = a1;
                    dal[i] = a2;
                }
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += dS[(size_t)i * dv + j] * kh[i];
                    dvh[j] = acc;
                }
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) dS[(size_t)i * dv + j] *= al[i];
                /* gates */
                for (int i = 0; i < dk; ++i) {
                    double dah = k[i] * dkh[i];
                    double dah_dg = tau[i] == 0.0 ? 0.0 : tau[i] * pow(g[i], tau[i] - 1.0);
                    double dah_dtau = ah[i] == 0.0 ? 0.0 : ah[i] * log(g[i]);
                    J->dk_[ok + i] = ah[i] * dkh[i];
                    J->dg[ok + i] = dal[i] * (-tau[i] * al[i]) + dah * dah_dg;
                    J->dtau[ok + i] = dal[i] * (-g[i] * al[i]) + dah * dah_dtau;
                }
                for (int j = 0; j < dv; ++j) {
                    J->dv_[ov + j] = beta[j] * dvh[j];
                    J->dbeta[ov + j] = v[j] * dvh[j];
                }
                /* feedthrough o_t += d (.) v_t */
                if (J->dfeed) {
                    const double *d = J->dfeed + (size_t)(p % J->H) * dv;
                    for (int j = 0; j < dv; ++j) {
                        J->dv_[ov + j] += d[j] * dO[j];
                        if (J->ddfeed) J->ddfeed[(size_t)p * dv + j] += dO[j] * v[j];
                    }
                }
            }
        }
        if (J->dS0) memcpy(J->dS0 + ss, dS, sizeof(double) * SS);
    }
out:
    free(ck); free(seg); free(dS); free(al); free(ah); free(kh); free(vh);
    free(dkh); free(dvh); free(dal);
    return NULL;
}

int rdm_oracle_bwd(int B, int H, int T, int dk, int dv,
                   const double *q, const double *k, const double *v,
                   const double *g, const double *tau, const double *beta,
                   const double *S0, const double *dO, const double *dST,
                   const double *dfeed,
                   double *dq, double *dk_, double *dv_, double *dg, double *dtau,
                   double *dbeta, double *dS0, double *ddfeed, int nthreads)
{
    if (!dims_ok(B, H, T, dk, dv)) return -1;
    if (T > 0 && (!q || !k || !v || !g || !tau || !beta || !dO || !dq || !dk_ || !dv_ ||
                  !dg || !dtau || !dbeta))
        return -1;
    job_t J;
    memset(&J, 0, sizeof(J));
    J.B = B; J.H = H; J.T = T; J.dk = dk; J.dv = dv;
    J.q = q; J.k = k; J.v = v; J.g = g; J.tau = tau; J.beta = beta; J.S0 = S0;
    J.dO = dO; J.dST = dST;
    J.dq = dq; J.dk_ = dk_; J.dv_ = dv_; J.dg = dg; J.dtau = dtau; J.dbeta = dbeta; J.dS0 = dS0;
    J.dfeed = dfeed; J.ddfeed = ddfeed;
    return run_pool(&J, bwd_worker, nthreads);
}

/* ------------------------------------------------------------- short conv
 * ShortConv of the Rodimus block (digest.lyk-ai.com summary, "Method", third
 * Rodimus bullet: a short convolution for local context next to the GLU).  The
 * pages print neither its width, placement nor activation; the reading taken
 * is a causal depthwise convolution along the tokens, one filter of width W per
 * (head, channel):
 *     z[b,h,t,c] = bias[h,c] + sum_{i=0}^{W-1} w[h,c,i] * x[b,h,t-i,c]
 *     y = z, or y = z * sigmoid(z) (SiLU) when silu != 0
 * with x at t - i < 0 taken from the carried-in state xs[b,h,W-1+(t-i),c] (the
 * previous W-1 tokens, oldest first; zeros when xs is NULL).  The state after
 * the sequence (its last W-1 inputs, including carried-in ones when T < W-1)
 * is written to xs_out when non-NULL.  Layouts: x, y [B,H,T,D]; w [H,D,W];
 * bias [H,D] or NULL; xs, xs_out [B,H,W-1,D]. */
static double conv_input(const double *x, const double *xs, int T, int D, int W, int t, int c)
{
    if (t >= 0) return t < T ? x[(size_t)t * D + c] : 0.0;
    int s = W - 1 + t;            /* position in the carried-in state */
    return (xs && s >= 0) ? xs[(size_t)s * D + c] : 0.0;
}

int rdm_oracle_shortconv_fwd(int B, int H, int T, int D, int W, const double *x,
                             const double *w, const double *bias, const double *xs,
                             int silu, double *y, double *xs_out)
{
    if (B < 0 || H < 0 || T < 0 || D < 1 || W < 1 || !w) return -1;
    for (int p = 0; p < B * H; ++p) {
        const int h = p % H;
        const double *xp = x + (size_t)p * T * D;
        const double *sp = xs ? xs + (size_t)p * (W - 1) * D : NULL;
        for (int t = 0; t < T; ++t)
            for (int c = 0; c < D; ++c) {
                double z = bias ? bias[(size_t)h * D + c] : 0.0;
                for (int i = 0; i < W; ++i)
                    z += w[((size_t)h * D + c) * W + i] * conv_input(xp, sp, T, D, W, t - i, c);
                y[((size_t)p * T + t) * D + c] = silu ? z / (1.0 + exp(-z)) : z;
            }
        if (xs_out)
            for (int s = 0; s < W - 1; ++s)
                for (int c = 0; c < D; ++c)
                    xs_out[((size_t)p * (W - 1) + s) * D + c] =
                        conv_input(xp, sp, T, D, W, T - (W - 1) + s, c);
    }
    return 0;
}

/* Reverse mode of rdm_oracle_shortconv_fwd for the loss with dL/dy = dy (and
 * dL/dxs_out = dxs_out when non-NULL): dx [B,H,T,D], dw [H,D,W], dbias [H,D]
 * (NULL = skip), dxs [B,H,W-1,D] (NULL = skip).  Written by direct
 * differentiation of the loops above: z is recomputed per output. */
int rdm_oracle_shortconv_bwd(int B, int H, int T, int D, int W, const double *x,
                             const double *w, const double *bias, const double *xs, int silu,
                             const double *dy, const double *dxs_out, double *dx, double *dw,
                             double *dbias, double *dxs)
{
    if (B < 0 || H < 0 || T < 0 || D < 1 || W < 1 || !w || !dx || !dw) return -1;
    memset(dx, 0, sizeof(double) * (size_t)B * H * T * D);
    memset(dw, 0, sizeof(double) * (size_t)H * D * W);
    if (dbias) memset(dbias, 0, sizeof(double) * (size_t)H * D);
    if (dxs) memset(dxs, 0, sizeof(double) * (size_t)B * H * (W - 1) * D);
    for (int p = 0; p < B * H; ++p) {
        const int h = p % H;
        const double *xp = x + (size_t)p * T * D;
        const double *sp = xs ? xs + (size_t)p * (W - 1) * D : NULL;
        /* the carried-out state is a copy of inputs: route its gradient back */
        if (dxs_out)
            for (int s = 0; s < W - 1; ++s)
                for (int c = 0; c < D; ++c) {
                    const double gsv = dxs_out[((size_t)p * (W - 1) + s) * D + c];
                    const int t = T - (W - 1) + s;
                    if (t >= 0) dx[((size_t)p * T + t) * D + c] += gsv;
                    else if (dxs && W - 1 + t >= 0) dxs[((size_t)p * (W - 1) + W - 1 + t) * D + c] += gsv;
                }
        for (int t = 0; t < T; ++t)
            for (int c = 0; c < D; ++c) {
                double z = bias ? bias[(size_t)h * D + c] : 0.0;
                for (int i = 0; i < W; ++i)
                    z += w[((size_t)h * D + c) * W + i] * conv_input(xp, sp, T, D, W, t - i, c);
                double gz = dy[((size_t)p * T + t) * D + c];
                if (silu) {
                    const double s = 1.0 / (1.0 + exp(-z));
                    gz *= s * (1.0 + z * (1.0 - s));
                }
                if (dbias) dbias[(size_t)h * D + c] += gz;
                for (int i = 0; i < W; ++i) {
                    const int ti = t - i;
                    dw[((size_t)h * D + c) * W + i] += gz * conv_input(xp, sp, T, D, W, ti, c);
                    const double gx = gz * w[((size_t)h * D + c) * W + i];
                    if (ti >= 0) dx[((size_t)p * T + ti) * D + c] += gx;
                    else if (dxs && W - 1 + ti >= 0) dxs[((size_t)p * (W - 1) + W - 1 + ti) * D + c] += gx;
                }
            }
    }
    return 0;
}

/* ------------------------------------------------------------------ SW-SKA
 * Sliding-window shared-key attention of Rodimus+ (digest.lyk-ai.com summary,
 * "Method", Rodimus+ bullets: attention over a sliding window for local context,
 * with one key shared by all heads to shrink the KV cache; paperhub.cn
 * OpenReview rebuttal, answer to Q1: multi-head query and value projections
 * and a multi-query key projection).  The pages print neither the window nor
 * the score scale; the reading taken is, per batch b, head h and token t,
 *     s_u = scale * q[b,h,t] . k[b,u]        for u = max(0, t-w+1) .. t
 *     o[b,h,t] = sum_u softmax(s)_u v[b,h,u]
 * with one key row per token shared by every head.  Layouts: q [B,H,T,dk],
 * k [B,T,dk], v [B,H,T,dv], o [B,H,T,dv].  The softmax subtracts the largest
 * score first, which leaves the exact value unchanged. */
static void ska_attend(int n, int dk, int dv, double scale, const double *q,
                       const double *const *krow, const double *const *vrow, double *p,
                       double *o)
{
    double mx = -INFINITY, sum = 0.0;
    for (int u = 0; u < n; ++u) {
        double a = 0.0;
        for (int i = 0; i < dk; ++i) a += q[i] * krow[u][i];
        p[u] = scale * a;
        if (p[u] > mx) mx = p[u];
    }
    for (int u = 0; u < n; ++u) {
        p[u] = exp(p[u] - mx);
        sum += p[u];
    }
    for (int j = 0; j < dv; ++j) o[j] = 0.0;
    for (int u = 0; u < n; ++u)
        for (int j = 0; j < dv; ++j) o[j] += (p[u] / sum) * vrow[u][j];
}

int rdm_oracle_ska_fwd(int B, int H, int T, int dk, int dv, int w, double scale,
                       const double *q, const double *k, const double *v, double *o)
{
    if (B < 0 || H < 0 || T < 0 || dk < 1 || dv < 1 || w < 1) return -1;
    double *p = (double *)malloc(sizeof(double) * (size_t)w);
    const double **kr = (const double **)malloc(sizeof(double *) * (size_t)w);
    const double **vr = (const double **)malloc(sizeof(double *) * (size_t)w);
    if (!p || !kr || !vr) { free(p); free(kr); free(vr); return -1; }
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const size_t bh = (size_t)b * H + h;
            for (int t = 0; t < T; ++t) {
                const int u0 = t - w + 1 > 0 ? t - w + 1 : 0;
                for (int u = u0; u <= t; ++u) {
                    kr[u - u0] = k + ((size_t)b * T + u) * dk;
                    vr[u - u0] = v + (bh * T + u) * dv;
                }
                ska_attend(t - u0 + 1, dk, dv, scale, q + (bh * T + t) * dk, kr, vr, p,
                           o + (bh * T + t) * dv);
            }
        }
    free(p); free(kr); free(vr);
    return 0;
}

/* One decode step against a ring KV cache of w slots: token position pos[b]
 * (the number of tokens seen before this one) goes to slot pos[b] mod w, so the
 * cache holds positions max(0, pos-w+1) .. pos after the write.  Layouts:
 * q [B,H,dk], k [B,dk], v [B,H,dv], kc [B,w,dk], vc [B,H,w,dv], o [B,H,dv].
 * The cached positions are visited oldest first. */
int rdm_oracle_ska_decode(int B, int H, int dk, int dv, int w, double scale,
                          const long long *pos, const double *q, const double *k,
                          const double *v, double *kc, double *vc, double *o)
{
    if (B < 0 || H < 0 || dk < 1 || dv < 1 || w < 1) return -1;
    double *p = (double *)malloc(sizeof(double) * (size_t)w);
    const double **kr = (const double **)malloc(sizeof(double *) * (size_t)w);
    const double **vr = (const double **)malloc(sizeof(double *) * (size_t)w);
    if (!p || !kr || !vr) { free(p); free(kr); free(vr); return -1; }
    for (int b = 0; b < B; ++b) {
        if (pos[b] < 0) { free(p); free(kr); free(vr); return -1; }
        const long long t = pos[b], u0 = t - w + 1 > 0 ? t - w + 1 : 0;
        const int slot = (int)(t % w);
        for (int i = 0; i < dk; ++i) kc[((size_t)b * w + slot) * dk + i] = k[(size_t)b * dk + i];
        for (int h = 0; h < H; ++h)
            for (int j = 0; j < dv; ++j)
                vc[(((size_t)b * H + h) * w + slot) * dv + j] = v[((size_t)b * H + h) * dv + j];
        for (int h = 0; h < H; ++h) {
            for (long long u = u0; u <= t; ++u) {
                kr[u - u0] = kc + ((size_t)b * w + (size_t)(u % w)) * dk;
                vr[u - u0] = vc + (((size_t)b * H + h) * w + (size_t)(u % w)) * dv;
            }
            ska_attend((int)(t - u0 + 1), dk, dv, scale, q + ((size_t)b * H + h) * dk, kr, vr,
                       p, o + ((size_t)b * H + h) * dv);
        }
    }
    free(p); free(kr); free(vr);
    return 0;
}
