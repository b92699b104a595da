/*
 * Kalman Delta Network memory recurrence -- the ORACLE.
 *
 * TEST INFRASTRUCTURE ONLY.  Plain fp64, token by token, no blocking, no
 * fusion, no reordering beyond the order the method states.  Only the tests,
 * the package's smoke check and the benchmark's CPU-baseline leg may load
 * this library; the product path never does.  It shares no code with the CUDA
 * path: nothing here is included by, or includes, anything of the package.
 *
 * Notation (per head): key k, query q in R^dk; value v in R^dv; memory
 * S in R^{dk x dv} (read as S^T k); per-channel decay alpha in [0,1]^dk;
 * per-channel process-noise variance sigma; scalar observation-noise
 * variance r; per-channel key-space uncertainty P (the diagonal of the
 * covariance); information scaling mu.
 *
 * Sources (pages as titled):
 *  - "给记忆装一个信任度探测器：Kalman Delta Networks ..." (techwalker), sections
 *    "把记忆问题重新想成一个滤波问题" (predict / update with a gain from the
 *    uncertainty and the observation reliability) and "对角近似" (diagonal
 *    predict, dense posterior projected back to a diagonal by a KL-minimising
 *    mean-field step, exact mean, information scaling mu on the precision
 *    increment, no effect of mu on the current write).
 *  - "Kalman Delta Networks: Uncertainty-aware Associative Memory"
 *    (aifromscratch), "Approximation 1: Diagonal KDN".
 *  - "Gated KalmaNet" blog (csdn), section 2.1: the full-covariance gain form
 *    S - (S k - v) k^T Phi / (1/eta + k^T Phi k).
 *  - "Память с поправкой" (delta rule tutorial): read v^ = S^T k, error
 *    e = v - v^, write S += beta k e^T.
 *  - "معماری KDA" (dothoosh): per-channel decay D_t = diag(alpha_t) applied
 *    before the delta update; readout from the memory.
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository):
 *  - predict of the diagonal uncertainty: P^- = alpha^2 * P + sigma (a variance
 *    under S -> diag(alpha) S scales by alpha^2);
 *  - the mean-field projection keeps the diagonal of the posterior PRECISION:
 *    1/P = 1/P^- + mu * k^2 / r;
 *  - the readout o_t = S_t^T q_t is taken after the write, without scaling;
 *  - isotropic KDN (one uncertainty p per head; explainer "各向同性近似",
 *    aifromscratch "Approximation 2: Isotropic KDN"): the predicted covariance
 *    diag(alpha^2) p + diag(sigma) is brought back to a multiple of the identity
 *    keeping its trace, p^- = mean(alpha^2) p + mean(sigma) (the pages require the
 *    isotropic recursion to stay a Moebius map, which the trace keeps and the
 *    precision average would not); the gain p^- k / (r + p^- |k|^2) is exact for an
 *    isotropic prior; the posterior is projected like the diagonal one, by its
 *    precision, averaged over the d_k directions: 1/p = 1/p^- + mu |k|^2 / (d_k r).
 *
 * Layout: tokens flattened as [ntok, H, d] (dense batch b,t -> b*T + t);
 * sequence s covers tokens [cu[s], cu[s+1]); states S [nseq, H, dk, dv],
 * P [nseq, H, dk], full covariances [nseq, H, dk, dk].  All row-major fp64.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- shared steps */

/* Decayed delta write (delta-rule tutorial steps "read, compare, correct" with the
 * KDA per-channel decay applied first):
 *   W = diag(alpha) S ;  u = v - W^T k ;  S = W + g u^T.
 * g is the write key: beta*k for the delta family, the Kalman gain for KDN. */
static void delta_write(double *S, int dk, int dv, const double *alpha,
                        const double *k, const double *g, const double *v, double *u)
{
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j)
            S[(size_t)i * dv + j] *= alpha[i];
    for (int j = 0; j < dv; ++j) {
        double pred = 0.0;
        for (int i = 0; i < dk; ++i)
            pred += S[(size_t)i * dv + j] * k[i];
        u[j] = v[j] - pred;
    }
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j)
            S[(size_t)i * dv + j] += g[i] * u[j];
}

/* Readout o = S^T q. */
static void readout(const double *S, int dk, int dv, const double *q, double *o)
{
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i)
            acc += S[(size_t)i * dv + j] * q[i];
        o[j] = acc;
    }
}

/* ---------------------------------------------------------------- work split */

typedef struct {
    int mode;                 /* 0 diagonal KDN, 1 full covariance, 2 constant beta, 3 isotropic KDN */
    int nseq, H, dk, dv;
    const int64_t *cu;
    const double *q, *k, *v, *alpha, *sigma, *r, *beta;
    const double *S0, *P0;    /* P0: [nseq,H,dk] (diag), [nseq,H,dk,dk] (full), [nseq,H] (isotropic) */
    double mu;
    double *o, *S_out, *P_out;
    double *Pm_trace, *P_trace, *g_trace, *beff_trace;
    int next;                 /* work counter (atomic) */
    int status;
} job_t;

static void run_item(job_t *J, int item)
{
    const int H = J->H, dk = J->dk, dv = J->dv;
    const int s = item / H, h = item % H;
    const int64_t t0 = J->cu[s], t1 = J->cu[s + 1];
    const size_t sh = (size_t)s * H + h;

    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *u = (double *)malloc(sizeof(double) * (size_t)dv);
    double *g = (double *)malloc(sizeof(double) * (size_t)dk);
    double *Pm = (double *)malloc(sizeof(double) * (size_t)dk);
    double *P = NULL, *Sig = NULL, *Sm = NULL, *Sk = NULL;
    if (!S || !u || !g || !Pm) { J->status = -1; goto done; }

    if (J->S0) memcpy(S, J->S0 + sh * dk * dv, sizeof(double) * (size_t)dk * dv);
    else memset(S, 0, sizeof(double) * (size_t)dk * dv);

    if (J->mode == 1) {
        Sig = (double *)malloc(sizeof(double) * (size_t)dk * dk);
        Sm = (double *)malloc(sizeof(double) * (size_t)dk * dk);
        Sk = (double *)malloc(sizeof(double) * (size_t)dk);
        if (!Sig || !Sm || !Sk) { J->status = -1; goto done; }
        if (J->P0) memcpy(Sig, J->P0 + sh * dk * dk, sizeof(double) * (size_t)dk * dk);
        else for (int i = 0; i < dk; ++i) for (int j = 0; j < dk; ++j) Sig[(size_t)i * dk + j] = (i == j);
    } else if (J->mode == 3) {
        P = (double *)malloc(sizeof(double));
        if (!P) { J->status = -1; goto done; }
        P[0] = J->P0 ? J->P0[sh] : 1.0;
    } else {
        P = (double *)malloc(sizeof(double) * (size_t)dk);
        if (!P) { J->status = -1; goto done; }
        for (int i = 0; i < dk; ++i) P[i] = J->P0 ? J->P0[sh * dk + i] : 1.0;
    }

    for (int64_t t = t0; t < t1; ++t) {
        const size_t th = (size_t)t * H + h;
        const double *q = J->q + th * dk, *k = J->k + th * dk, *v = J->v + th * dv;
        const double *al = J->alpha + th * dk;
        const double r = J->r ? J->r[th] : 0.0;

        if (J->mode == 0) {
            /* predict: the decay keeps the covariance diagonal; variance scales by alpha^2 */
            const double *sg = J->sigma + th * dk;
            for (int i = 0; i < dk; ++i) Pm[i] = al[i] * al[i] * P[i] + sg[i];
            /* gain from the predicted uncertainty and the observation noise */
            double den = r;
            for (int i = 0; i < dk; ++i) den += Pm[i] * k[i] * k[i];
            for (int i = 0; i < dk; ++i) g[i] = Pm[i] * k[i] / den;
        } else if (J->mode == 1) {
            /* full covariance: Sigma^- = D Sigma D + diag(sigma); K = Sigma^- k / (r + k^T Sigma^- k) */
            const double *sg = J->sigma + th * dk;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dk; ++j)
                    Sm[(size_t)i * dk + j] = al[i] * Sig[(size_t)i * dk + j] * al[j] + (i == j ? sg[i] : 0.0);
            double den = r;
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += Sm[(size_t)i * dk + j] * k[j];
                Sk[i] = acc;
                den += k[i] * acc;
            }
            for (int i = 0; i < dk; ++i) g[i] = Sk[i] / den;
            /* posterior covariance Sigma = Sigma^- - (Sigma^- k)(Sigma^- k)^T / den, symmetrised */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dk; ++j)
                    Sig[(size_t)i * dk + j] = Sm[(size_t)i * dk + j] - Sk[i] * Sk[j] / den;
            for (int i = 0; i < dk; ++i)
                for (int j = i + 1; j < dk; ++j) {
                    double m = 0.5 * (Sig[(size_t)i * dk + j] + Sig[(size_t)j * dk + i]);
                    Sig[(size_t)i * dk + j] = Sig[(size_t)j * dk + i] = m;
                }
        } else if (J->mode == 3) {
            /* isotropic predict: the trace of diag(alpha^2) p + diag(sigma), per direction */
            const double *sg = J->sigma + th * dk;
            double a2 = 0.0, sm = 0.0, kk = 0.0;
            for (int i = 0; i < dk; ++i) { a2 += al[i] * al[i]; sm += sg[i]; kk += k[i] * k[i]; }
            Pm[0] = (a2 / dk) * P[0] + sm / dk;
            /* exact gain for an isotropic prior: g = p^- k / (r + p^- |k|^2) */
            const double den = r + Pm[0] * kk;
            for (int i = 0; i < dk; ++i) g[i] = Pm[0] * k[i] / den;
        } else {
            /* delta family: the write key is beta * k */
            const double b = J->beta[th];
            for (int i = 0; i < dk; ++i) g[i] = b * k[i];
        }

        delta_write(S, dk, dv, al, k, g, v, u);
        readout(S, dk, dv, q, J->o + th * dv);

        if (J->g_trace) memcpy(J->g_trace + th * dk, g, sizeof(double) * (size_t)dk);
        if (J->beff_trace) {
            double b = 0.0;
            for (int i = 0; i < dk; ++i) b += k[i] * g[i];
            J->beff_trace[th] = b;
        }
        if (J->mode == 0) {
            if (J->Pm_trace) memcpy(J->Pm_trace + th * dk, Pm, sizeof(double) * (size_t)dk);
            /* mean-field update: diagonal of the posterior precision, increment scaled by mu */
            for (int i = 0; i < dk; ++i) P[i] = Pm[i] / (1.0 + J->mu * Pm[i] * k[i] * k[i] / r);
            if (J->P_trace) memcpy(J->P_trace + th * dk, P, sizeof(double) * (size_t)dk);
        } else if (J->mode == 3) {
            if (J->Pm_trace) J->Pm_trace[th] = Pm[0];
            /* precision of the posterior averaged over the d_k directions, increment scaled by mu */
            double kk = 0.0;
            for (int i = 0; i < dk; ++i) kk += k[i] * k[i];
            P[0] = Pm[0] / (1.0 + J->mu * Pm[0] * kk / (dk * r));
            if (J->P_trace) J->P_trace[th] = P[0];
        }
    }

    if (J->S_out) memcpy(J->S_out + sh * dk * dv, S, sizeof(double) * (size_t)dk * dv);
    if (J->P_out) {
        if (J->mode == 1) memcpy(J->P_out + sh * dk * dk, Sig, sizeof(double) * (size_t)dk * dk);
        else if (J->mode == 0) memcpy(J->P_out + sh * dk, P, sizeof(double) * (size_t)dk);
        else if (J->mode == 3) J->P_out[sh] = P[0];
    }
done:
    free(S); free(u); free(g); free(Pm); free(P); free(Sig); free(Sm); free(Sk);
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    const int n = J->nseq * J->H;
    for (;;) {
        int item = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (item >= n) break;
        run_item(J, item);
    }
    return NULL;
}

static int run_job(job_t *J, int nthreads)
{
    const int n = J->nseq * J->H;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n) nthreads = n > 0 ? n : 1;
    J->next = 0;
    J->status = 0;
    if (nthreads == 1) { worker(J); return J->status; }
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) return -1;
    int started = 0;
    for (int i = 0; i < nthreads; ++i)
        if (pthread_create(&th[i], NULL, worker, J) == 0) ++started;
    if (started == 0) worker(J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    return J->status;
}

static int check_cu(int nseq, const int64_t *cu)
{
    if (nseq < 0 || !cu || cu[0] != 0) return -2;
    for (int s = 0; s < nseq; ++s) if (cu[s + 1] < cu[s]) return -2;
    return 0;
}

/* ---------------------------------------------------------------- entry points */

/* Diagonal KDN, per token:
 *   1. P^- = alpha^2 * P + sigma
 *   2. g   = P^- * k / (r + sum_i P^-_i k_i^2)
 *   3. W = diag(alpha) S ; u = v - W^T k ; S = W + g u^T
 *   4. o   = S^T q
 *   5. P   = P^- / (1 + mu * P^- * k^2 / r)
 * S0 NULL -> zeros, P0 NULL -> ones.  Traces (per token, may be NULL): P^-, P, g, k^T g. */
int kdn_oracle_diag(int nseq, const int64_t *cu, int H, int dk, int dv,
                    const double *q, const double *k, const double *v,
                    const double *alpha, const double *sigma, const double *r,
                    const double *S0, const double *P0, double mu,
                    double *o, double *S_out, double *P_out,
                    double *Pm_trace, double *P_trace, double *g_trace, double *beff_trace,
                    int nthreads)
{
    if (check_cu(nseq, cu) || H <= 0 || dk <= 0 || dv <= 0 || !q || !k || !v || !alpha || !sigma || !r || !o)
        return -2;
    job_t J = {0};
    J.mode = 0; J.nseq = nseq; J.H = H; J.dk = dk; J.dv = dv; J.cu = cu;
    J.q = q; J.k = k; J.v = v; J.alpha = alpha; J.sigma = sigma; J.r = r;
    J.S0 = S0; J.P0 = P0; J.mu = mu; J.o = o; J.S_out = S_out; J.P_out = P_out;
    J.Pm_trace = Pm_trace; J.P_trace = P_trace; J.g_trace = g_trace; J.beff_trace = beff_trace;
    return run_job(&J, nthreads);
}

/* Full-covariance Kalman filter over the same observation model (tiny sizes only):
 *   Sigma^- = D Sigma D + diag(sigma) ; K = Sigma^- k / (r + k^T Sigma^- k)
 *   S = D S + K (v - (D S)^T k)^T ; Sigma = Sigma^- - K k^T Sigma^- ; o = S^T q.
 * Sigma0 [nseq,H,dk,dk] (NULL -> identity); Sigma_out likewise. */
int kdn_oracle_fullkf(int nseq, const int64_t *cu, int H, int dk, int dv,
                      const double *q, const double *k, const double *v,
                      const double *alpha, const double *sigma, const double *r,
                      const double *S0, const double *Sigma0,
                      double *o, double *S_out, double *Sigma_out, double *g_trace, int nthreads)
{
    if (check_cu(nseq, cu) || H <= 0 || dk <= 0 || dv <= 0 || !q || !k || !v || !alpha || !sigma || !r || !o)
        return -2;
    job_t J = {0};
    J.mode = 1; J.nseq = nseq; J.H = H; J.dk = dk; J.dv = dv; J.cu = cu;
    J.q = q; J.k = k; J.v = v; J.alpha = alpha; J.sigma = sigma; J.r = r;
    J.S0 = S0; J.P0 = Sigma0; J.o = o; J.S_out = S_out; J.P_out = Sigma_out; J.g_trace = g_trace;
    return run_job(&J, nthreads);
}

/* Delta family with a given write strength: g = beta_t k_t, then the same decayed
 * write and readout (alpha = 1: DeltaNet; alpha a per-token scalar broadcast:
 * Gated DeltaNet; per-channel alpha: KDA).  beta: [ntok, H]. */
int kdn_oracle_delta(int nseq, const int64_t *cu, int H, int dk, int dv,
                     const double *q, const double *k, const double *v,
                     const double *alpha, const double *beta, const double *S0,
                     double *o, double *S_out, int nthreads)
{
    if (check_cu(nseq, cu) || H <= 0 || dk <= 0 || dv <= 0 || !q || !k || !v || !alpha || !beta || !o)
        return -2;
    job_t J = {0};
    J.mode = 2; J.nseq = nseq; J.H = H; J.dk = dk; J.dv = dv; J.cu = cu;
    J.q = q; J.k = k; J.v = v; J.alpha = alpha; J.beta = beta;
    J.S0 = S0; J.o = o; J.S_out = S_out;
    return run_job(&J, nthreads);
}

/* Isotropic KDN, per token (one uncertainty p per head):
 *   1. p^- = mean_i(alpha_i^2) p + mean_i(sigma_i)
 *   2. g   = p^- k / (r + p^- |k|^2)
 *   3. W = diag(alpha) S ; u = v - W^T k ; S = W + g u^T
 *   4. o   = S^T q
 *   5. p   = p^- / (1 + mu p^- |k|^2 / (d_k r))
 * S0 NULL -> zeros, P0 [nseq,H] NULL -> ones.  Traces per token: p^- and p [ntok,H],
 * g [ntok,H,dk], k^T g [ntok,H]. */
int kdn_oracle_iso(int nseq, const int64_t *cu, int H, int dk, int dv,
                   const double *q, const double *k, const double *v,
                   const double *alpha, const double *sigma, const double *r,
                   const double *S0, const double *P0, double mu,
                   double *o, double *S_out, double *P_out,
                   double *Pm_trace, double *P_trace, double *g_trace, double *beff_trace,
                   int nthreads)
{
    if (check_cu(nseq, cu) || H <= 0 || dk <= 0 || dv <= 0 || !q || !k || !v || !alpha || !sigma || !r || !o)
        return -2;
    job_t J = {0};
    J.mode = 3; J.nseq = nseq; J.H = H; J.dk = dk; J.dv = dv; J.cu = cu;
    J.q = q; J.k = k; J.v = v; J.alpha = alpha; J.sigma = sigma; J.r = r;
    J.S0 = S0; J.P0 = P0; J.mu = mu; J.o = o; J.S_out = S_out; J.P_out = P_out;
    J.Pm_trace = Pm_trace; J.P_trace = P_trace; J.g_trace = g_trace; J.beff_trace = beff_trace;
    return run_job(&J, nthreads);
}
