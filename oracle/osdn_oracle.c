/*
 * OSDN oracle: a plain, slow, token-by-token CPU recurrence in float64.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path (the CUDA library and
 * its Python binding) links, imports or calls this file. Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg use it. It shares no code,
 * header, table or helper with the CUDA kernels.
 *
 * What it computes (page "OSDN: Improving Delta Rule with Provable Online
 * Preconditioning in Linear Attention", gist.science technical summary):
 *
 *   Section 1 (problem statement): per-token regression loss
 *       f_t(S) = 1/2 || S k_t - v_t ||^2,   S in R^{dv x dk}.
 *   Section 2.1 (algebraic equivalence): right-preconditioned step
 *       S_t = S_{t-1} - beta_t grad f_t(S_{t-1}) D_t,  D_t = diag(d_t),
 *   which equals the write-side scaled key form
 *       S_t = S_{t-1} + beta_t (v_t - S_{t-1} k_t) (d_t (.) k_t)^T.
 *   The read/erase key stays k_t; only the write key is scaled.
 *   Output o_t = S_t q_t (read after the write, no 1/sqrt(dk) scale).
 *   Section 2.2 (decoupled hypergradient): closed form
 *       h_t(d) = ((1 - beta_t <d, k_t^2>)^2 - 1) / (2 ||k_t||^2),
 *   gradient  grad_d h_t(d) = -beta_t (1 - beta_t <d, k_t^2>) k_t^2 / ||k_t||^2.
 *   Section 2.3 (APF): d_{t+1} = r_t d_t - eta grad_d h_t(d_t)
 *       = r_t d_t + eta beta_t (1 - beta_t <d_t, k_t^2>) k_t^2 / ||k_t||^2.
 *
 * Readings fixed here (the pages leave them open):
 *   - online gradient DESCENT on h (the page writes "+ eta grad h"; descent is
 *     what "OGD on h" means and what drives beta <d, k^2> toward the gated
 *     Newton condition beta <d*, k^2> = 1 of Theorem 5.2);
 *   - no projection step after the APF update (the recurrence stays affine);
 *   - play-then-update: token t writes with d_t, and d_1 = d0;
 *   - r_t is an input per (token, head); r == NULL means APF off (r == 1);
 *   - ||k_t||^2 == 0 skips the gradient term (h is undefined there).
 *
 * Gated OSDN (an option; the gated delta rule backbone the pages run OSDN on):
 *       S_t = alpha_t S_{t-1} (I - beta_t k_t (d_t (.) k_t)^T) + beta_t v_t (d_t (.) k_t)^T,
 * i.e. the step above applied to the decayed state alpha_t S_{t-1}; d is unchanged.
 *
 * Anchored APF (an option; the "refresh the calibration" reading of the APF
 * section): the retention pulls d toward its initial value d0 instead of 0,
 *       d_{t+1} = r_t d_t + (1 - r_t) d0 - eta grad_d h_t(d_t).
 *
 * Diagnostic (technical summary sections 4-5, the contraction factor of the
 * gated Newton analysis): the residual ratio of token t,
 *       rho_t = f_t(S_t) / f_t(S_{t-1}) = (1 - beta_t <d_t, k_t^2>)^2,
 * from the same <d_t, k_t^2> the d step uses (pinned against the S
 * trajectory in the tests).
 *
 * Backward (training; the pages give no backward, so this is the plain
 * reverse-mode derivative of the recurrence above, token by token): for a
 * scalar loss L with given dL/do_t, dL/dS_T and dL/dd_T, it returns dL/d of
 * every input (q, k, v, beta, r, alpha, d0, S0). Adjoint of one token, with
 * Sh = alpha S_{t-1}, e = Sh k - v, kw = d (.) k, S_t = Sh - beta e kw^T,
 * a = k^2, n = ||k||^2, s = <d, a>, x = eta beta (1 - beta s) / n (0 when n = 0),
 * d_{t+1} = r d + (1 - r) d0 [anchored only] + x a; LS = dL/dS_t, Ld = dL/dd_{t+1}:
 *       LS += dO q^T;        dq = S_t^T dO;       g = LS kw;
 *       dv = beta g;         dbeta = -<e, g> + dx eta (1 - 2 beta s) / n;
 *       dkw = -beta LS^T e;  LSh = LS - beta g k^T;  dk = Sh^T (-beta g) + dkw (.) d + 2 k (.) da;
 *       dalpha = <LSh, S_{t-1}>;  dL/dS_{t-1} = alpha LSh;
 *       dx = <a, Ld>;  dr = <d - d0 [anchored], Ld>;  da = x Ld - dx (eta beta^2 / n) d - dx x / n;
 *       dL/dd_t = r Ld + dkw (.) k - dx (eta beta^2 / n) a;  dd0 += (1 - r) Ld [anchored].
 * Pinned in the tests by central finite differences of fwd() and by the
 * linearity of (o, S_T) in (v, S0) and of o in q.
 */
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int B, T, H, dk, dv;
    double eta;
    const double *q, *k, *v, *beta, *r, *d0, *S0, *alpha;
    double *out, *S_final, *d_final, *rho;
    int anchor;                         /* anchored APF: retention toward d0 */
    int unit_begin, unit_end;
} oracle_job;

/* One token of the recurrence for one (sequence, head). S is dv x dk
 * row-major, d has dk entries; both are updated in place. o receives dv
 * values. e and a are scratch of dv and dk entries. */
static void oracle_token(int dk, int dv, double eta, double *S, double *d,
                         const double *q, const double *k, const double *v,
                         double beta, double r, double *o, double *e, double *a, double *rho,
                         const double *anchor, double alpha)
{
    if (alpha != 1.0)                                  /* gated: decay the state first */
        for (size_t i = 0; i < (size_t)dv * dk; ++i) S[i] *= alpha;
    double n = 0.0, s = 0.0;
    for (int i = 0; i < dk; ++i) {
        a[i] = k[i] * k[i];           /* k_t^2, elementwise */
        n += a[i];                    /* ||k_t||^2 */
        s += d[i] * a[i];             /* <d_t, k_t^2> with the pre-update d */
    }
    if (rho) *rho = (1.0 - beta * s) * (1.0 - beta * s);
    /* residual e = S_{t-1} k_t - v_t (gradient of f_t is e k_t^T) */
    for (int row = 0; row < dv; ++row) {
        double acc = 0.0;
        const double *Srow = S + (size_t)row * dk;
        for (int i = 0; i < dk; ++i) acc += Srow[i] * k[i];
        e[row] = acc - v[row];
    }
    /* S_t = S_{t-1} - beta e (d (.) k)^T */
    for (int row = 0; row < dv; ++row) {
        double *Srow = S + (size_t)row * dk;
        double be = beta * e[row];
        for (int i = 0; i < dk; ++i) Srow[i] -= be * (d[i] * k[i]);
    }
    /* o_t = S_t q_t */
    for (int row = 0; row < dv; ++row) {
        double acc = 0.0;
        const double *Srow = S + (size_t)row * dk;
        for (int i = 0; i < dk; ++i) acc += Srow[i] * q[i];
        o[row] = acc;
    }
    /* d_{t+1} = r d_t (+ (1 - r) d0 when anchored) + eta beta (1 - beta s) k^2 / ||k||^2 */
    double x = 0.0;
    if (n > 0.0) x = eta * beta * (1.0 - beta * s) / n;
    for (int i = 0; i < dk; ++i) d[i] = r * d[i] + (anchor ? (1.0 - r) * anchor[i] : 0.0) + x * a[i];
}

static void *oracle_worker(void *arg)
{
    oracle_job *J = (oracle_job *)arg;
    const int dk = J->dk, dv = J->dv, T = J->T, H = J->H;
    double *S = (double *)malloc(sizeof(double) * (size_t)dv * dk);
    double *d = (double *)malloc(sizeof(double) * (size_t)dk);
    double *e = (double *)malloc(sizeof(double) * (size_t)dv);
    double *a = (double *)malloc(sizeof(double) * (size_t)dk);
    double *d_start = (double *)malloc(sizeof(double) * (size_t)dk);
    for (int u = J->unit_begin; u < J->unit_end; ++u) {
        const int b = u / H, h = u % H;
        if (J->S0) memcpy(S, J->S0 + (size_t)u * dv * dk, sizeof(double) * (size_t)dv * dk);
        else memset(S, 0, sizeof(double) * (size_t)dv * dk);
        if (J->d0) memcpy(d, J->d0 + (size_t)u * dk, sizeof(double) * (size_t)dk);
        else for (int i = 0; i < dk; ++i) d[i] = 1.0;
        memcpy(d_start, d, sizeof(double) * (size_t)dk);
        for (int t = 0; t < T; ++t) {
            const size_t tok = ((size_t)b * T + t) * H + h;  /* [B, T, H] */
            oracle_token(dk, dv, J->eta, S, d,
                         J->q + tok * dk, J->k + tok * dk, J->v + tok * dv,
                         J->beta[tok], J->r ? J->r[tok] : 1.0,
                         J->out + tok * dv, e, a, J->rho ? J->rho + tok : NULL,
                         J->anchor ? d_start : NULL, J->alpha ? J->alpha[tok] : 1.0);
        }
        if (J->S_final) memcpy(J->S_final + (size_t)u * dv * dk, S, sizeof(double) * (size_t)dv * dk);
        if (J->d_final) memcpy(J->d_final + (size_t)u * dk, d, sizeof(double) * (size_t)dk);
    }
    free(S); free(d); free(e); free(a); free(d_start);
    return NULL;
}

/* Forward over a whole sequence batch.
 * q, k: [B, T, H, dk]; v, out: [B, T, H, dv]; beta, r: [B, T, H] (r may be NULL);
 * d0: [B, H, dk] (NULL = ones); S0: [B, H, dv, dk] (NULL = zeros);
 * S_final: [B, H, dv, dk], d_final: [B, H, dk], rho: [B, T, H] (any may be NULL).
 * The (b, h) units are independent; nthreads host threads share them.
 * Returns 0, or -1 on bad sizes. */
int osdn_oracle_fwd_ex(int B, int T, int H, int dk, int dv, double eta, int anchor,
                       const double *q, const double *k, const double *v,
                       const double *beta, const double *r, const double *alpha,
                       const double *d0, const double *S0,
                       double *out, double *S_final, double *d_final, double *rho,
                       int nthreads)
{
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    const int units = B * H;
    if (units == 0) return 0;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > units) nthreads = units;
    oracle_job *jobs = (oracle_job *)calloc((size_t)nthreads, sizeof(oracle_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int w = 0; w < nthreads; ++w) {
        oracle_job J = {B, T, H, dk, dv, eta, q, k, v, beta, r, d0, S0, alpha,
                        out, S_final, d_final, rho, anchor,
                        (int)((long long)units * w / nthreads),
                        (int)((long long)units * (w + 1) / nthreads)};
        jobs[w] = J;
    }
    for (int w = 1; w < nthreads; ++w) pthread_create(&th[w], NULL, oracle_worker, &jobs[w]);
    oracle_worker(&jobs[0]);
    for (int w = 1; w < nthreads; ++w) pthread_join(th[w], NULL);
    free(jobs); free(th);
    return 0;
}

int osdn_oracle_fwd_rho(int B, int T, int H, int dk, int dv, double eta,
                        const double *q, const double *k, const double *v,
                        const double *beta, const double *r,
                        const double *d0, const double *S0,
                        double *out, double *S_final, double *d_final, double *rho,
                        int nthreads)
{
    return osdn_oracle_fwd_ex(B, T, H, dk, dv, eta, 0, q, k, v, beta, r, NULL, d0, S0, out, S_final, d_final, rho,
                              nthreads);
}

int osdn_oracle_fwd(int B, int T, int H, int dk, int dv, double eta,
                    const double *q, const double *k, const double *v,
                    const double *beta, const double *r,
                    const double *d0, const double *S0,
                    double *out, double *S_final, double *d_final,
                    int nthreads)
{
    return osdn_oracle_fwd_ex(B, T, H, dk, dv, eta, 0, q, k, v, beta, r, NULL, d0, S0, out, S_final, d_final, NULL,
                              nthreads);
}

/* One decode token for every (b, h): q, k [B, H, dk]; v, out [B, H, dv];
 * beta, r, alpha [B, H] (r, alpha may be NULL); S [B, H, dv, dk] and d
 * [B, H, dk] updated in place; d_anchor [B, H, dk] (NULL: plain APF, non-NULL:
 * anchored APF toward it). Same arithmetic as one step of osdn_oracle_fwd_ex. */
int osdn_oracle_step_ex(int B, int H, int dk, int dv, double eta,
                        const double *q, const double *k, const double *v,
                        const double *beta, const double *r, const double *alpha, const double *d_anchor,
                        double *S, double *d, double *out)
{
    if (B < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    double *e = (double *)malloc(sizeof(double) * (size_t)dv);
    double *a = (double *)malloc(sizeof(double) * (size_t)dk);
    for (int u = 0; u < B * H; ++u) {
        oracle_token(dk, dv, eta, S + (size_t)u * dv * dk, d + (size_t)u * dk,
                     q + (size_t)u * dk, k + (size_t)u * dk, v + (size_t)u * dv,
                     beta[u], r ? r[u] : 1.0, out + (size_t)u * dv, e, a, NULL,
                     d_anchor ? d_anchor + (size_t)u * dk : NULL, alpha ? alpha[u] : 1.0);
    }
    free(e); free(a);
    return 0;
}

int osdn_oracle_step(int B, int H, int dk, int dv, double eta,
                     const double *q, const double *k, const double *v,
                     const double *beta, const double *r,
                     double *S, double *d, double *out)
{
    return osdn_oracle_step_ex(B, H, dk, dv, eta, q, k, v, beta, r, NULL, NULL, S, d, out);
}

/* ------------------------------------------------------------------------- */
/* Backward: reverse-mode gradients of osdn_oracle_fwd_ex.                    */

typedef struct {
    int B, T, H, dk, dv;
    double eta;
    int anchor;
    const double *q, *k, *v, *beta, *r, *alpha, *d0, *S0, *dout, *dS_final, *dd_final;
    double *dq, *dk_, *dv_, *dbeta, *dr, *dalpha, *dd0, *dS0;
    int unit_begin, unit_end;
} oracle_bwd_job;

/* Adjoint of one token (the formulas in the header). Sp = S_{t-1} before the
 * decay, d = d_t. LS (dv x dk) enters as dL/dS_t from the later tokens and
 * leaves as dL/dS_{t-1}; Ld (dk) enters as dL/dd_{t+1} and leaves as dL/dd_t;
 * dd_anchor accumulates (1 - r) Ld under anchored APF. The per-token gradients
 * are written to gq, gk, gv (overwritten) and *gbeta, *gr, *galpha (when non-NULL). */
static void oracle_token_bwd(int dk, int dv, double eta, const double *Sp, const double *d,
                             const double *q, const double *k, const double *v,
                             double beta, double r, double alpha, const double *dO,
                             const double *anchor, double *LS, double *Ld, double *dd_anchor,
                             double *gq, double *gk, double *gv, double *gbeta, double *gr, double *galpha,
                             double *Sh, double *e, double *a, double *kw, double *g, double *dkw, double *ddl)
{
    const size_t nS = (size_t)dv * dk;
    for (size_t i = 0; i < nS; ++i) Sh[i] = alpha * Sp[i];
    double n = 0.0, s = 0.0;
    for (int i = 0; i < dk; ++i) {
        a[i] = k[i] * k[i];
        n += a[i];
        s += d[i] * a[i];
        kw[i] = d[i] * k[i];
    }
    double edo = 0.0;
    for (int row = 0; row < dv; ++row) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += Sh[(size_t)row * dk + i] * k[i];
        e[row] = acc - v[row];
        edo += e[row] * dO[row];
    }
    /* o_t = S_t q_t with S_t = Sh - beta e kw^T */
    for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        for (int row = 0; row < dv; ++row) acc += Sh[(size_t)row * dk + i] * dO[row];
        gq[i] = acc - beta * kw[i] * edo;
    }
    for (int row = 0; row < dv; ++row)
        for (int i = 0; i < dk; ++i) LS[(size_t)row * dk + i] += dO[row] * q[i];
    /* through the write S_t = Sh - beta e kw^T */
    double gb = 0.0;
    for (int row = 0; row < dv; ++row) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += LS[(size_t)row * dk + i] * kw[i];
        g[row] = acc;
        gv[row] = beta * acc;            /* e = Sh k - v, de = -beta g */
        gb -= e[row] * acc;
    }
    for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        for (int row = 0; row < dv; ++row) acc += LS[(size_t)row * dk + i] * e[row];
        dkw[i] = -beta * acc;
    }
    /* through e = Sh k - v: dL/dSh = LS + (-beta g) k^T, dk += Sh^T (-beta g) */
    for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        for (int row = 0; row < dv; ++row) acc += Sh[(size_t)row * dk + i] * g[row];
        gk[i] = -beta * acc;
    }
    for (int row = 0; row < dv; ++row)
        for (int i = 0; i < dk; ++i) LS[(size_t)row * dk + i] -= beta * g[row] * k[i];
    if (galpha) {
        double acc = 0.0;
        for (size_t i = 0; i < nS; ++i) acc += LS[i] * Sp[i];
        *galpha = acc;
    }
    if (alpha != 1.0)
        for (size_t i = 0; i < nS; ++i) LS[i] *= alpha;
    /* through kw = d (.) k */
    for (int i = 0; i < dk; ++i) {
        gk[i] += dkw[i] * d[i];
        ddl[i] = dkw[i] * k[i];
    }
    /* through d_{t+1} = r d + (1 - r) d0 [anchored] + x a */
    if (gr) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += (d[i] - (anchor ? anchor[i] : 0.0)) * Ld[i];
        *gr = acc;
    }
    if (anchor)
        for (int i = 0; i < dk; ++i) dd_anchor[i] += (1.0 - r) * Ld[i];
    if (n > 0.0) {
        const double x = eta * beta * (1.0 - beta * s) / n;
        double dx = 0.0;
        for (int i = 0; i < dk; ++i) dx += a[i] * Ld[i];
        gb += dx * eta * (1.0 - 2.0 * beta * s) / n;
        const double ds = -dx * eta * beta * beta / n;   /* dL/ds */
        const double dn = -dx * x / n;                   /* dL/dn */
        for (int i = 0; i < dk; ++i) {
            const double da = x * Ld[i] + ds * d[i] + dn;
            gk[i] += 2.0 * k[i] * da;
            ddl[i] += ds * a[i];
        }
    }
    for (int i = 0; i < dk; ++i) Ld[i] = r * Ld[i] + ddl[i];
    *gbeta = gb;
}

static void *oracle_bwd_worker(void *arg)
{
    oracle_bwd_job *J = (oracle_bwd_job *)arg;
    const int dk = J->dk, dv = J->dv, T = J->T, H = J->H;
    const int seg = 64;                                /* checkpoint spacing (tokens) */
    const int nseg = (T + seg - 1) / seg;
    const size_t nS = (size_t)dv * dk;
    double *ckS = (double *)malloc(sizeof(double) * nS * (size_t)(nseg > 0 ? nseg : 1));
    double *ckd = (double *)malloc(sizeof(double) * (size_t)dk * (size_t)(nseg > 0 ? nseg : 1));
    double *Sbuf = (double *)malloc(sizeof(double) * nS * (size_t)seg);
    double *dbuf = (double *)malloc(sizeof(double) * (size_t)dk * (size_t)seg);
    double *S = (double *)malloc(sizeof(double) * nS);
    double *d = (double *)malloc(sizeof(double) * (size_t)dk);
    double *d_start = (double *)malloc(sizeof(double) * (size_t)dk);
    double *LS = (double *)malloc(sizeof(double) * nS);
    double *Ld = (double *)malloc(sizeof(double) * (size_t)dk);
    double *dd_anchor = (double *)calloc((size_t)dk, sizeof(double));
    double *Sh = (double *)malloc(sizeof(double) * nS);
    double *o = (double *)malloc(sizeof(double) * (size_t)dv);
    double *e = (double *)malloc(sizeof(double) * (size_t)dv);
    double *g = (double *)malloc(sizeof(double) * (size_t)dv);
    double *a = (double *)malloc(sizeof(double) * (size_t)dk);
    double *kw = (double *)malloc(sizeof(double) * (size_t)dk);
    double *dkw = (double *)malloc(sizeof(double) * (size_t)dk);
    double *ddl = (double *)malloc(sizeof(double) * (size_t)dk);
    for (int u = J->unit_begin; u < J->unit_end; ++u) {
        const int b = u / H, h = u % H;
        if (J->S0) memcpy(S, J->S0 + (size_t)u * nS, sizeof(double) * nS);
        else memset(S, 0, sizeof(double) * nS);
        if (J->d0) memcpy(d, J->d0 + (size_t)u * dk, sizeof(double) * (size_t)dk);
        else for (int i = 0; i < dk; ++i) d[i] = 1.0;
        memcpy(d_start, d, sizeof(double) * (size_t)dk);
        const double *anc = J->anchor ? d_start : NULL;
        /* forward pass: state checkpoints at the start of every segment */
        for (int t = 0; t < T; ++t) {
            if (t % seg == 0) {
                memcpy(ckS + (size_t)(t / seg) * nS, S, sizeof(double) * nS);
                memcpy(ckd + (size_t)(t / seg) * dk, d, sizeof(double) * (size_t)dk);
            }
            const size_t tok = ((size_t)b * T + t) * H + h;
            oracle_token(dk, dv, J->eta, S, d, J->q + tok * dk, J->k + tok * dk, J->v + tok * dv,
                         J->beta[tok], J->r ? J->r[tok] : 1.0, o, e, a, NULL, anc,
                         J->alpha ? J->alpha[tok] : 1.0);
        }
        /* reverse pass, one segment at a time: replay the segment forward from its
           checkpoint to recover S_{t-1} and d_t, then walk its tokens backward */
        if (J->dS_final) memcpy(LS, J->dS_final + (size_t)u * nS, sizeof(double) * nS);
        else memset(LS, 0, sizeof(double) * nS);
        if (J->dd_final) memcpy(Ld, J->dd_final + (size_t)u * dk, sizeof(double) * (size_t)dk);
        else memset(Ld, 0, sizeof(double) * (size_t)dk);
        memset(dd_anchor, 0, sizeof(double) * (size_t)dk);
        for (int sg = nseg - 1; sg >= 0; --sg) {
            const int t0 = sg * seg, t1 = (t0 + seg < T) ? t0 + seg : T;
            memcpy(S, ckS + (size_t)sg * nS, sizeof(double) * nS);
            memcpy(d, ckd + (size_t)sg * dk, sizeof(double) * (size_t)dk);
            for (int t = t0; t < t1; ++t) {
                memcpy(Sbuf + (size_t)(t - t0) * nS, S, sizeof(double) * nS);
                memcpy(dbuf + (size_t)(t - t0) * dk, d, sizeof(double) * (size_t)dk);
                const size_t tok = ((size_t)b * T + t) * H + h;
                oracle_token(dk, dv, J->eta, S, d, J->q + tok * dk, J->k + tok * dk, J->v + tok * dv,
                             J->beta[tok], J->r ? J->r[tok] : 1.0, o, e, a, NULL, anc,
                             J->alpha ? J->alpha[tok] : 1.0);
            }
            for (int t = t1 - 1; t >= t0; --t) {
                const size_t tok = ((size_t)b * T + t) * H + h;
                oracle_token_bwd(dk, dv, J->eta, Sbuf + (size_t)(t - t0) * nS, dbuf + (size_t)(t - t0) * dk,
                                 J->q + tok * dk, J->k + tok * dk, J->v + tok * dv, J->beta[tok],
                                 J->r ? J->r[tok] : 1.0, J->alpha ? J->alpha[tok] : 1.0,
                                 J->dout + tok * dv, anc, LS, Ld, dd_anchor,
                                 J->dq + tok * dk, J->dk_ + tok * dk, J->dv_ + tok * dv, J->dbeta + tok,
                                 J->dr ? J->dr + tok : NULL, J->dalpha ? J->dalpha + tok : NULL,
                                 Sh, e, a, kw, g, dkw, ddl);
            }
        }
        if (J->dS0) memcpy(J->dS0 + (size_t)u * nS, LS, sizeof(double) * nS);
        if (J->dd0)
            for (int i = 0; i < dk; ++i) J->dd0[(size_t)u * dk + i] = Ld[i] + dd_anchor[i];
    }
    free(ckS); free(ckd); free(Sbuf); free(dbuf); free(S); free(d); free(d_start); free(LS); free(Ld);
    free(dd_anchor); free(Sh); free(o); free(e); free(g); free(a); free(kw); free(dkw); free(ddl);
    return NULL;
}

/* Gradients of L = sum <dout, out> + <dS_final, S_final> + <dd_final, d_final>
 * of osdn_oracle_fwd_ex with the same inputs (dS_final, dd_final NULL = 0).
 * dq, dk: [B, T, H, dk]; dv: [B, T, H, dv]; dbeta, dr, dalpha: [B, T, H];
 * dd0: [B, H, dk]; dS0: [B, H, dv, dk]. dr, dalpha, dd0, dS0 may be NULL (not
 * written); dr is only meaningful with r, dalpha only with alpha.
 * Returns 0, or -1 on bad sizes. */
int osdn_oracle_bwd_ex(int B, int T, int H, int dk, int dv, double eta, int anchor,
                       const double *q, const double *k, const double *v,
                       const double *beta, const double *r, const double *alpha,
                       const double *d0, const double *S0,
                       const double *dout, const double *dS_final, const double *dd_final,
                       double *dq, double *dk_, double *dv_, double *dbeta,
                       double *dr, double *dalpha, double *dd0, double *dS0,
                       int nthreads)
{
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    const int units = B * H;
    if (units == 0) return 0;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > units) nthreads = units;
    oracle_bwd_job *jobs = (oracle_bwd_job *)calloc((size_t)nthreads, sizeof(oracle_bwd_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int w = 0; w < nthreads; ++w) {
        oracle_bwd_job J = {B, T, H, dk, dv, eta, anchor, q, k, v, beta, r, alpha, d0, S0,
                            dout, dS_final, dd_final, dq, dk_, dv_, dbeta, dr, dalpha, dd0, dS0,
                            (int)((long long)units * w / nthreads),
                            (int)((long long)units * (w + 1) / nthreads)};
        jobs[w] = J;
    }
    for (int w = 1; w < nthreads; ++w) pthread_create(&th[w], NULL, oracle_bwd_worker, &jobs[w]);
    oracle_bwd_worker(&jobs[0]);
    for (int w = 1; w < nthreads; ++w) pthread_join(th[w], NULL);
    free(jobs); free(th);
    return 0;
}
