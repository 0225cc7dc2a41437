/*
 * mesa_oracle.c -- plain, slow, fp64 CPU reference of the Mesa layer.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark load this code. It shares nothing with the
 * CUDA library (no headers, helpers, tables or constants) and the CUDA
 * library never calls it.
 *
 * What it computes. Source: "MesaNet: Sequence Modeling by Locally Optimal
 * Test-Time Training" (gist.science/ja/paper/2506.05233; the ko and hi
 * editions carry the same formula), Technical summary > Method > Mesa layer.
 *
 *   Objective (Mesa layer equation):
 *     Phi_t = argmin_Phi 1/2 sum_{t'<=t} zeta_{tt'} |v_t' - Phi k_t'|^2
 *                        + 1/2 Tr(Phi Lambda Phi^T)
 *   with zeta the cumulative forget factors and Lambda symmetric positive
 *   definite. Setting the gradient to zero gives Phi_t = G_t (H_t+Lambda)^-1,
 *   H_t = sum zeta k k^T, G_t = sum zeta v k^T, and the output
 *   Delta_t = Phi_t q_t = G_t x_t with x_t = (H_t + Lambda)^-1 q_t, the
 *   "optimal query response" that the page says is found by conjugate
 *   gradient rather than recursive least squares.
 *
 *   Reading of zeta (the page only says "cumulative forget factors"):
 *     zeta_{tt'} = beta_t' * prod_{s=t'+1..t} gamma_s, i.e. the gated
 *     recurrences H_t = gamma_t H_{t-1} + beta_t k_t k_t^T and
 *     G_t = gamma_t G_{t-1} + beta_t v_t k_t^T, H_0 = G_0 = 0.
 *   Lambda = diag(lambda[h]) per head, constant in t and not decayed (it sits
 *   outside the zeta sum in the objective).
 *
 *   CG rule (the page names CG and a per-token stopping criterion under
 *   "Dynamic compute" but gives no details; readings):
 *     x_0 = 0, r_0 = q, p_0 = q (no warm start: the page lists warm starts as
 *     future work). Before every update k = 0..N-1: if tol > 0 and
 *     |r_k|_2 <= tol |q|_2, stop. Breakdown: if r.r <= 0 or p.Ap <= 0 or
 *     p.Ap is not finite, stop (the token keeps its current x). Otherwise
 *     alpha = r.r / p.Ap, x += alpha p, r -= alpha Ap, rho = r'.r'/r.r,
 *     p = r' + rho p. iters = number of updates applied. tol <= 0: exactly N
 *     updates unless breakdown.
 *
 *   Chunked form (the page: CG over many time steps is equivalent to gated
 *   linear attention; the layer keeps G_t and H_t and solves the systems in
 *   parallel per chunk). For chunk c = [c0, c1) with chunk-start states
 *   H_c, G_c and in-chunk log-cumsum b_t = sum_{s=c0..t} log gamma_s:
 *     H_t p = e^{b_t} H_c p + sum_{j=c0..t} beta_j e^{b_t-b_j} (k_j.p) k_j
 *     G_t x = e^{b_t} G_c x + sum_{j=c0..t} beta_j e^{b_t-b_j} (k_j.x) v_j
 *     H_{c+1} = e^{b_{c1-1}} H_c + sum_j beta_j e^{b_{c1-1}-b_j} k_j k_j^T
 *   (and the same for G). The matrices H_t are never formed.
 *
 * Everything is in fp64. Loops run in the order the definitions are written;
 * the only parallelism is over independent (b, h) sequences.
 */
#include "mesa_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Conjugate gradient with a caller-supplied matrix-vector product.          */
/* ------------------------------------------------------------------------ */

typedef void (*matvec_fn)(const void* ctx, const double* p, double* y);

static double dot(int n, const double* a, const double* b) {
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += a[i] * b[i];
    return s;
}

/* Solves A x = b by CG, A given only through mv, starting from x0 (NULL:
 * x0 = 0). The first residual is r0 = b - A x0 and the first direction
 * p0 = r0; the stopping test compares |r_k| with tol |b| whatever the start.
 * work: 3n doubles. */
static int cg_generic_x0(int n, matvec_fn mv, const void* ctx, const double* b, const double* x0,
                         int cg_steps, double tol, double* x, double* work) {
    double* r = work;
    double* p = work + n;
    double* y = work + 2 * n;
    if (x0) {
        for (int i = 0; i < n; ++i) x[i] = x0[i];
        mv(ctx, x, y);
        for (int i = 0; i < n; ++i) { r[i] = b[i] - y[i]; p[i] = r[i]; }
    } else {
        for (int i = 0; i < n; ++i) { x[i] = 0.0; r[i] = b[i]; p[i] = b[i]; }
    }
    double rr = dot(n, r, r);
    const double bnorm = sqrt(dot(n, b, b));
    int it = 0;
    for (int kstep = 0; kstep < cg_steps; ++kstep) {
        if (tol > 0.0 && sqrt(rr) <= tol * bnorm) break;   /* stopping criterion */
        mv(ctx, p, y);
        const double pAp = dot(n, p, y);
        if (!(rr > 0.0) || !(pAp > 0.0) || !isfinite(pAp)) break;   /* breakdown */
        const double alpha = rr / pAp;
        for (int i = 0; i < n; ++i) { x[i] += alpha * p[i]; r[i] -= alpha * y[i]; }
        const double rr_new = dot(n, r, r);
        ++it;
        const double rho = rr_new / rr;
        for (int i = 0; i < n; ++i) p[i] = r[i] + rho * p[i];
        rr = rr_new;
    }
    return it;
}

static int cg_generic(int n, matvec_fn mv, const void* ctx, const double* b,
                      int cg_steps, double tol, double* x, double* work) {
    return cg_generic_x0(n, mv, ctx, b, NULL, cg_steps, tol, x, work);
}

/* Dense (H + Lambda) p: the matrix is formed explicitly. */
typedef struct { int n; const double* A; } dense_ctx;

static void dense_mv(const void* vctx, const double* p, double* y) {
    const dense_ctx* c = (const dense_ctx*)vctx;
    for (int i = 0; i < c->n; ++i) y[i] = dot(c->n, c->A + (size_t)i * c->n, p);
}

int oracle_cg_dense(int n, const double* A, const double* b, const double* x0, int cg_steps, double tol,
                    double* x, int32_t* iters) {
    if (n <= 0 || !A || !b || !x || cg_steps < 0) return -1;
    double* work = (double*)malloc(sizeof(double) * 3 * (size_t)n);
    if (!work) return -2;
    dense_ctx c = {n, A};
    int it = cg_generic_x0(n, dense_mv, &c, b, x0, cg_steps, tol, x, work);
    if (iters) *iters = it;
    free(work);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Argument checks shared by the entry points.                               */
/* ------------------------------------------------------------------------ */

static int bad_dims(int B, int H, int T, int dk, int dv) {
    return B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0;
}

/* Gated rank-1 updates of the explicit statistics (the recurrence above). */
static void update_state(int dk, int dv, double g, double bta, const double* kt,
                         const double* vt, double* Hm, double* Gm) {
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dk; ++j)
            Hm[(size_t)i * dk + j] = g * Hm[(size_t)i * dk + j] + bta * kt[i] * kt[j];
    for (int i = 0; i < dv; ++i)
        for (int j = 0; j < dk; ++j)
            Gm[(size_t)i * dk + j] = g * Gm[(size_t)i * dk + j] + bta * vt[i] * kt[j];
}

static void init_state(size_t n, const double* src, double* dst) {
    if (src) memcpy(dst, src, n * sizeof(double));
    else memset(dst, 0, n * sizeof(double));
}

/* ------------------------------------------------------------------------ */
/* Per-token recurrence + CG                                                  */
/* ------------------------------------------------------------------------ */

int oracle_forward_cg(const double* q, const double* k, const double* v,
                      const double* gamma, const double* beta, const double* lambda,
                      int B, int H, int T, int dk, int dv, int cg_steps, double tol,
                      const double* H_init, const double* G_init,
                      double* out, int32_t* iters, double* H_final, double* G_final) {
    if (bad_dims(B, H, T, dk, dv) || cg_steps < 0) return -1;
    if (T > 0 && (!q || !k || !v || !gamma || !beta || !out)) return -1;
    if (!lambda) return -1;
    const int BH = B * H;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int bh = 0; bh < BH; ++bh) {
        const int h = bh % H;
        double* Hm = (double*)malloc(sizeof(double) * (size_t)dk * dk);
        double* Gm = (double*)malloc(sizeof(double) * (size_t)dv * dk);
        double* A = (double*)malloc(sizeof(double) * (size_t)dk * dk);
        double* x = (double*)malloc(sizeof(double) * (size_t)dk);
        double* work = (double*)malloc(sizeof(double) * 3 * (size_t)dk);
        if (!Hm || !Gm || !A || !x || !work) {
            err |= 1;
        } else {
            init_state((size_t)dk * dk, H_init ? H_init + (size_t)bh * dk * dk : NULL, Hm);
            init_state((size_t)dv * dk, G_init ? G_init + (size_t)bh * dv * dk : NULL, Gm);
            for (int t = 0; t < T; ++t) {
                const size_t bt = (size_t)bh * T + t;
                const double* qt = q + bt * dk;
                const double* kt = k + bt * dk;
                const double* vt = v + bt * dv;
                update_state(dk, dv, gamma[bt], beta[bt], kt, vt, Hm, Gm);
                /* A = H_t + Lambda */
                for (int i = 0; i < dk; ++i) {
                    for (int j = 0; j < dk; ++j) A[(size_t)i * dk + j] = Hm[(size_t)i * dk + j];
                    A[(size_t)i * dk + i] += lambda[(size_t)h * dk + i];
                }
                dense_ctx c = {dk, A};
                int it = cg_generic(dk, dense_mv, &c, qt, cg_steps, tol, x, work);
                if (iters) iters[bt] = it;
                /* o_t = G_t x_t */
                double* ot = out + bt * dv;
                for (int i = 0; i < dv; ++i) ot[i] = dot(dk, Gm + (size_t)i * dk, x);
            }
            if (H_final) memcpy(H_final + (size_t)bh * dk * dk, Hm, sizeof(double) * (size_t)dk * dk);
            if (G_final) memcpy(G_final + (size_t)bh * dv * dk, Gm, sizeof(double) * (size_t)dv * dk);
        }
        free(Hm); free(Gm); free(A); free(x); free(work);
    }
    return err ? -2 : 0;
}

/* The per-token forward with a warm-started CG (MesaNet page, Significance
 * and claims: warm starts named as the way to cut the solver's cost): token
 * t's CG starts from x0[b,h,t,:] (NULL: from zero, which is exactly
 * oracle_forward_cg), r_0 = q_t - (H_t + Lambda) x0_t, p_0 = r_0, and the
 * stopping test stays |r_k| <= tol |q_t|. x_out [B,H,T,dk] (or NULL)
 * receives every token's solution. */
int oracle_forward_cg_x0(const double* q, const double* k, const double* v,
                         const double* gamma, const double* beta, const double* lambda,
                         int B, int H, int T, int dk, int dv, int cg_steps, double tol,
                         const double* x0, const double* H_init, const double* G_init,
                         double* out, int32_t* iters, double* x_out, double* H_final, double* G_final) {
    if (bad_dims(B, H, T, dk, dv) || cg_steps < 0) return -1;
    if (T > 0 && (!q || !k || !v || !gamma || !beta || !out)) return -1;
    if (!lambda) return -1;
    const int BH = B * H;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int bh = 0; bh < BH; ++bh) {
        const int h = bh % H;
        double* Hm = (double*)malloc(sizeof(double) * (size_t)dk * dk);
        double* Gm = (double*)malloc(sizeof(double) * (size_t)dv * dk);
        double* A = (double*)malloc(sizeof(double) * (size_t)dk * dk);
        double* x = (double*)malloc(sizeof(double) * (size_t)dk);
        double* work = (double*)malloc(sizeof(double) * 3 * (size_t)dk);
        if (!Hm || !Gm || !A || !x || !work) {
            err |= 1;
        } else {
            init_state((size_t)dk * dk, H_init ? H_init + (size_t)bh * dk * dk : NULL, Hm);
            init_state((size_t)dv * dk, G_init ? G_init + (size_t)bh * dv * dk : NULL, Gm);
            for (int t = 0; t < T; ++t) {
                const size_t bt = (size_t)bh * T + t;
                update_state(dk, dv, gamma[bt], beta[bt], k + bt * dk, v + bt * dv, Hm, Gm);
                for (int i = 0; i < dk; ++i) {
                    for (int j = 0; j < dk; ++j) A[(size_t)i * dk + j] = Hm[(size_t)i * dk + j];
                    A[(size_t)i * dk + i] += lambda[(size_t)h * dk + i];
                }
                dense_ctx c = {dk, A};
                const int it = cg_generic_x0(dk, dense_mv, &c, q + bt * dk, x0 ? x0 + bt * dk : NULL, cg_steps, tol,
                                             x, work);
                if (iters) iters[bt] = it;
                if (x_out) memcpy(x_out + bt * dk, x, sizeof(double) * (size_t)dk);
                double* ot = out + bt * dv;
                for (int i = 0; i < dv; ++i) ot[i] = dot(dk, Gm + (size_t)i * dk, x);
            }
            if (H_final) memcpy(H_final + (size_t)bh * dk * dk, Hm, sizeof(double) * (size_t)dk * dk);
            if (G_final) memcpy(G_final + (size_t)bh * dv * dk, Gm, sizeof(double) * (size_t)dv * dk);
        }
        free(Hm); free(Gm); free(A); free(x); free(work);
    }
    return err ? -2 : 0;
}

/* ------------------------------------------------------------------------ */
/* Per-token recurrence + exact Cholesky solve                                */
/* ------------------------------------------------------------------------ */

/* In-place Cholesky A = L L^T (lower triangle holds L). Returns 0 if SPD. */
static int cholesky(int n, double* A) {
    for (int j = 0; j < n; ++j) {
        double s = A[(size_t)j * n + j];
        for (int m = 0; m < j; ++m) s -= A[(size_t)j * n + m] * A[(size_t)j * n + m];
        if (!(s > 0.0)) return -1;
        const double ljj = sqrt(s);
        A[(size_t)j * n + j] = ljj;
        for (int i = j + 1; i < n; ++i) {
            double t = A[(size_t)i * n + j];
            for (int m = 0; m < j; ++m) t -= A[(size_t)i * n + m] * A[(size_t)j * n + m];
            A[(size_t)i * n + j] = t / ljj;
        }
    }
    return 0;
}

/* Solves L L^T x = b given the factor in the lower triangle of A. */
static void chol_solve(int n, const double* A, const double* b, double* x) {
    for (int i = 0; i < n; ++i) {          /* L z = b */
        double s = b[i];
        for (int m = 0; m < i; ++m) s -= A[(size_t)i * n + m] * x[m];
        x[i] = s / A[(size_t)i * n + i];
    }
    for (int i = n - 1; i >= 0; --i) {     /* L^T x = z */
        double s = x[i];
        for (int m = i + 1; m < n; ++m) s -= A[(size_t)m * n + i] * x[m];
        x[i] = s / A[(size_t)i * n + i];
    }
}

int oracle_forward_cholesky(const double* q, const double* k, const double* v,
                            const double* gamma, const double* beta, const double* lambda,
                            int B, int H, int T, int dk, int dv,
                            const double* H_init, const double* G_init,
                            double* out, double* H_final, double* G_final) {
    if (bad_dims(B, H, T, dk, dv)) return -1;
    if (T > 0 && (!q || !k || !v || !gamma || !beta || !out)) return -1;
    if (!lambda) return -1;
    const int BH = B * H;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int bh = 0; bh < BH; ++bh) {
        const int h = bh % H;
        double* Hm = (double*)malloc(sizeof(double) * (size_t)dk * dk);
        double* Gm = (double*)malloc(sizeof(double) * (size_t)dv * dk);
        double* A = (double*)malloc(sizeof(double) * (size_t)dk * dk);
        double* x = (double*)malloc(sizeof(double) * (size_t)dk);
        if (!Hm || !Gm || !A || !x) {
            err |= 1;
        } else {
            init_state((size_t)dk * dk, H_init ? H_init + (size_t)bh * dk * dk : NULL, Hm);
            init_state((size_t)dv * dk, G_init ? G_init + (size_t)bh * dv * dk : NULL, Gm);
            for (int t = 0; t < T && !err; ++t) {
                const size_t bt = (size_t)bh * T + t;
                update_state(dk, dv, gamma[bt], beta[bt], k + bt * dk, v + bt * dv, Hm, Gm);
                for (int i = 0; i < dk; ++i) {
                    for (int j = 0; j < dk; ++j) A[(size_t)i * dk + j] = Hm[(size_t)i * dk + j];
                    A[(size_t)i * dk + i] += lambda[(size_t)h * dk + i];
                }
                if (cholesky(dk, A) != 0) { err |= 2; break; }
                chol_solve(dk, A, q + bt * dk, x);
                double* ot = out + bt * dv;
                for (int i = 0; i < dv; ++i) ot[i] = dot(dk, Gm + (size_t)i * dk, x);
            }
            if (H_final) memcpy(H_final + (size_t)bh * dk * dk, Hm, sizeof(double) * (size_t)dk * dk);
            if (G_final) memcpy(G_final + (size_t)bh * dv * dk, Gm, sizeof(double) * (size_t)dv * dk);
        }
        free(Hm); free(Gm); free(A); free(x);
    }
    return err ? -2 : 0;
}

/* ------------------------------------------------------------------------ */
/* Chunked form                                                               */
/* ------------------------------------------------------------------------ */

typedef struct {
    int dk, t;              /* t: position of the token inside the chunk */
    const double* Hc;       /* chunk-start state, dk x dk */
    const double* kc;       /* keys of the chunk, n x dk */
    const double* bcum;     /* in-chunk inclusive log-cumsum of gamma */
    const double* betac;    /* beta of the chunk */
    const double* lam;      /* diagonal of Lambda */
} chunk_ctx;

/* (H_t + Lambda) p with H_t never formed. */
static void chunk_mv(const void* vctx, const double* p, double* y) {
    const chunk_ctx* c = (const chunk_ctx*)vctx;
    const int dk = c->dk, t = c->t;
    const double decay_t = exp(c->bcum[t]);
    for (int i = 0; i < dk; ++i) y[i] = decay_t * dot(dk, c->Hc + (size_t)i * dk, p);
    for (int j = 0; j <= t; ++j) {
        const double m = c->betac[j] * exp(c->bcum[t] - c->bcum[j]);
        const double s = m * dot(dk, c->kc + (size_t)j * dk, p);
        for (int i = 0; i < dk; ++i) y[i] += s * c->kc[(size_t)j * dk + i];
    }
    for (int i = 0; i < dk; ++i) y[i] += c->lam[i] * p[i];
}

int oracle_forward_chunked(const double* q, const double* k, const double* v,
                           const double* gamma, const double* beta, const double* lambda,
                           int B, int H, int T, int dk, int dv, int chunk,
                           int cg_steps, double tol,
                           const double* H_init, const double* G_init,
                           double* out, int32_t* iters, double* H_final, double* G_final) {
    if (bad_dims(B, H, T, dk, dv) || cg_steps < 0 || chunk <= 0) return -1;
    if (T > 0 && (!q || !k || !v || !gamma || !beta || !out)) return -1;
    if (!lambda) return -1;
    const int BH = B * H;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int bh = 0; bh < BH; ++bh) {
        const int h = bh % H;
        double* Hc = (double*)malloc(sizeof(double) * (size_t)dk * dk);
        double* Gc = (double*)malloc(sizeof(double) * (size_t)dv * dk);
        double* bcum = (double*)malloc(sizeof(double) * (size_t)chunk);
        double* x = (double*)malloc(sizeof(double) * (size_t)dk);
        double* work = (double*)malloc(sizeof(double) * 3 * (size_t)dk);
        if (!Hc || !Gc || !bcum || !x || !work) {
            err |= 1;
        } else {
            init_state((size_t)dk * dk, H_init ? H_init + (size_t)bh * dk * dk : NULL, Hc);
            init_state((size_t)dv * dk, G_init ? G_init + (size_t)bh * dv * dk : NULL, Gc);
            for (int c0 = 0; c0 < T; c0 += chunk) {
                const int n = (T - c0 < chunk) ? (T - c0) : chunk;
                const size_t base = (size_t)bh * T + c0;
                const double* kc = k + base * dk;
                const double* vc = v + base * dv;
                const double* betac = beta + base;
                double acc = 0.0;
                for (int t = 0; t < n; ++t) { acc += log(gamma[base + t]); bcum[t] = acc; }
                for (int t = 0; t < n; ++t) {
                    chunk_ctx c = {dk, t, Hc, kc, bcum, betac, lambda + (size_t)h * dk};
                    int it = cg_generic(dk, chunk_mv, &c, q + (base + t) * dk, cg_steps, tol, x, work);
                    if (iters) iters[base + t] = it;
                    /* o_t = e^{b_t} G_c x + sum_j beta_j e^{b_t-b_j} (k_j.x) v_j */
                    double* ot = out + (base + t) * dv;
                    const double decay_t = exp(bcum[t]);
                    for (int i = 0; i < dv; ++i) ot[i] = decay_t * dot(dk, Gc + (size_t)i * dk, x);
                    for (int j = 0; j <= t; ++j) {
                        const double s = betac[j] * exp(bcum[t] - bcum[j]) * dot(dk, kc + (size_t)j * dk, x);
                        for (int i = 0; i < dv; ++i) ot[i] += s * vc[(size_t)j * dv + i];
                    }
                }
                /* carry the states to the next chunk */
                const double blast = bcum[n - 1];
                const double Gam = exp(blast);
                for (size_t e = 0; e < (size_t)dk * dk; ++e) Hc[e] *= Gam;
                for (size_t e = 0; e < (size_t)dv * dk; ++e) Gc[e] *= Gam;
                for (int j = 0; j < n; ++j) {
                    const double w = betac[j] * exp(blast - bcum[j]);
                    const double* kj = kc + (size_t)j * dk;
                    const double* vj = vc + (size_t)j * dv;
                    for (int a = 0; a < dk; ++a)
                        for (int b2 = 0; b2 < dk; ++b2) Hc[(size_t)a * dk + b2] += w * kj[a] * kj[b2];
                    for (int a = 0; a < dv; ++a)
                        for (int b2 = 0; b2 < dk; ++b2) Gc[(size_t)a * dk + b2] += w * vj[a] * kj[b2];
                }
            }
            if (H_final) memcpy(H_final + (size_t)bh * dk * dk, Hc, sizeof(double) * (size_t)dk * dk);
            if (G_final) memcpy(G_final + (size_t)bh * dv * dk, Gc, sizeof(double) * (size_t)dv * dk);
        }
        free(Hc); free(Gc); free(bcum); free(x); free(work);
    }
    return err ? -2 : 0;
}

/* ------------------------------------------------------------------------ */
/* One decode step: O(1) per token on explicit state                          */
/* ------------------------------------------------------------------------ */

/* ------------------------------------------------------------------------ */
/* Input preprocessing (MesaNet page, Architecture, "Preprocessing"): a causal */
/* depthwise convolution over time, then L2 normalisation per token.          */
/* ------------------------------------------------------------------------ */

int oracle_preprocess(const double* x, const double* conv, int B, int H, int T, int d, int W, double* y) {
    if (bad_dims(B, H, T, d, d) || W < 1 || !x || !conv || !y) return -1;
    const int BH = B * H;
#pragma omp parallel for schedule(static)
    for (int bh = 0; bh < BH; ++bh) {
        const int h = bh % H;
        const double* xs = x + (size_t)bh * T * d;
        double* ys = y + (size_t)bh * T * d;
        for (int t = 0; t < T; ++t) {
            double nn = 0.0;
            for (int i = 0; i < d; ++i) {
                double u = 0.0;
                for (int w = 0; w < W && w <= t; ++w)
                    u += conv[((size_t)h * W + w) * d + i] * xs[(size_t)(t - w) * d + i];
                ys[(size_t)t * d + i] = u;
                nn += u * u;
            }
            const double nrm = sqrt(nn);
            const double inv = 1.0 / (nrm > 1e-6 ? nrm : 1e-6);
            for (int i = 0; i < d; ++i) ys[(size_t)t * d + i] *= inv;
        }
    }
    return 0;
}

int oracle_step(const double* q, const double* k, const double* v,
                const double* gamma, const double* beta, const double* lambda,
                int B, int H, int dk, int dv, double* Hstate, double* Gstate,
                int cg_steps, double tol, double* out, int32_t* iters) {
    return oracle_step_warm(q, k, v, gamma, beta, lambda, B, H, dk, dv, Hstate, Gstate, NULL, cg_steps, tol,
                            out, iters);
}

/* One decode step whose CG starts from x_state (MesaNet page, Significance and
 * claims: warm starts named as the way to cut the solver's cost). x_state
 * [B, H, dk] holds the starting guess on entry and the solution on exit;
 * NULL starts from zero. */
int oracle_step_warm(const double* q, const double* k, const double* v,
                     const double* gamma, const double* beta, const double* lambda,
                     int B, int H, int dk, int dv, double* Hstate, double* Gstate, double* x_state,
                     int cg_steps, double tol, double* out, int32_t* iters) {
    if (bad_dims(B, H, 1, dk, dv) || cg_steps < 0) return -1;
    if (!q || !k || !v || !gamma || !beta || !lambda || !Hstate || !Gstate || !out) return -1;
    const int BH = B * H;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int bh = 0; bh < BH; ++bh) {
        const int h = bh % H;
        double* Hm = Hstate + (size_t)bh * dk * dk;
        double* Gm = Gstate + (size_t)bh * dv * dk;
        double* A = (double*)malloc(sizeof(double) * (size_t)dk * dk);
        double* x = (double*)malloc(sizeof(double) * (size_t)dk);
        double* work = (double*)malloc(sizeof(double) * 3 * (size_t)dk);
        if (!A || !x || !work) {
            err |= 1;
        } else {
            update_state(dk, dv, gamma[bh], beta[bh], k + (size_t)bh * dk, v + (size_t)bh * dv, Hm, Gm);
            for (int i = 0; i < dk; ++i) {
                for (int j = 0; j < dk; ++j) A[(size_t)i * dk + j] = Hm[(size_t)i * dk + j];
                A[(size_t)i * dk + i] += lambda[(size_t)h * dk + i];
            }
            dense_ctx c = {dk, A};
            int it = cg_generic_x0(dk, dense_mv, &c, q + (size_t)bh * dk, x_state ? x_state + (size_t)bh * dk : NULL,
                                   cg_steps, tol, x, work);
            if (iters) iters[bh] = it;
            for (int i = 0; i < dv; ++i) out[(size_t)bh * dv + i] = dot(dk, Gm + (size_t)i * dk, x);
            if (x_state)
                for (int i = 0; i < dk; ++i) x_state[(size_t)bh * dk + i] = x[i];
        }
        free(A); free(x); free(work);
    }
    return err ? -2 : 0;
}

/* ------------------------------------------------------------------------ */
/* Backward pass: gradients of a scalar loss L through o_t = G_t x_t         */
/* ------------------------------------------------------------------------ */
/*
 * The pages claim the layer trains in time linear in T but give no backward
 * method. Reading taken here: implicit differentiation of the solution map
 * x_t = (H_t + Lambda)^-1 q_t, the adjoint system solved by the same CG rule
 * (same step count; the stopping test relative to its own right-hand side).
 * Given do_t = dL/do_t (tokens t = 0..T-1, zero initial states):
 *   dG_t = do_t x_t^T                     (o_t = G_t x_t)
 *   u_t  = CG_N(H_t + Lambda, G_t^T do_t)  (adjoint; exactly A_t^-1 G_t^T do_t)
 *   dq_t = u_t,   dH_t = -u_t x_t^T,   dlambda_i += -u_ti x_ti
 * then back through the recurrences H_t = gamma_t H_{t-1} + beta_t k_t k_t^T
 * and G_t = gamma_t G_{t-1} + beta_t v_t k_t^T with the running totals
 *   Hbar_t = dH_t + gamma_{t+1} Hbar_{t+1},   Gbar_t = dG_t + gamma_{t+1} Gbar_{t+1}:
 *   dbeta_t  = k_t^T Hbar_t k_t + v_t^T Gbar_t k_t
 *   dk_t     = beta_t (Hbar_t + Hbar_t^T) k_t + beta_t Gbar_t^T v_t
 *   dv_t     = beta_t Gbar_t k_t
 *   dgamma_t = <Hbar_t, H_{t-1}> + <Gbar_t, G_{t-1}>      (Frobenius products)
 * When CG has converged this is the exact gradient of the layer. The states
 * H_t and G_t are kept for every t (memory (T+1)(dk^2 + dv dk) doubles per
 * sequence).
 */
int oracle_backward(const double* q, const double* k, const double* v,
                    const double* gamma, const double* beta, const double* lambda,
                    int B, int H, int T, int dk, int dv, int cg_steps, double tol, const double* dout,
                    double* dq, double* dk_out, double* dv_out, double* dgamma, double* dbeta,
                    double* dlambda, int32_t* iters_fwd, int32_t* iters_adj) {
    if (bad_dims(B, H, T, dk, dv) || cg_steps < 0 || !lambda || !dlambda) return -1;
    if (T > 0 && (!q || !k || !v || !gamma || !beta || !dout || !dq || !dk_out || !dv_out || !dgamma || !dbeta))
        return -1;
    const int BH = B * H;
    const size_t SH = (size_t)dk * dk, SG = (size_t)dv * dk;
    double* part = (double*)calloc((size_t)(BH > 0 ? BH : 1) * dk, sizeof(double));   /* dlambda per sequence */
    if (!part) return -2;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int bh = 0; bh < BH; ++bh) {
        const int h = bh % H;
        double* Hs = (double*)calloc((size_t)(T + 1) * SH, sizeof(double));    /* Hs[t] = state after t tokens */
        double* Gs = (double*)calloc((size_t)(T + 1) * SG, sizeof(double));
        double* X = (double*)malloc(sizeof(double) * ((size_t)T * dk + 1));
        double* U = (double*)malloc(sizeof(double) * ((size_t)T * dk + 1));
        double* A = (double*)malloc(sizeof(double) * SH);
        double* g = (double*)malloc(sizeof(double) * (size_t)dk);
        double* work = (double*)malloc(sizeof(double) * 3 * (size_t)dk);
        double* Hbar = (double*)calloc(SH, sizeof(double));
        double* Gbar = (double*)calloc(SG, sizeof(double));
        if (!Hs || !Gs || !X || !U || !A || !g || !work || !Hbar || !Gbar) {
            err |= 1;
        } else {
            /* forward in time: states, x_t and the adjoint u_t */
            for (int t = 0; t < T; ++t) {
                const size_t bt = (size_t)bh * T + t;
                double* Hm = Hs + (size_t)(t + 1) * SH;
                double* Gm = Gs + (size_t)(t + 1) * SG;
                memcpy(Hm, Hs + (size_t)t * SH, sizeof(double) * SH);
                memcpy(Gm, Gs + (size_t)t * SG, sizeof(double) * SG);
                update_state(dk, dv, gamma[bt], beta[bt], k + bt * dk, v + bt * dv, Hm, Gm);
                for (int i = 0; i < dk; ++i) {
                    for (int j = 0; j < dk; ++j) A[(size_t)i * dk + j] = Hm[(size_t)i * dk + j];
                    A[(size_t)i * dk + i] += lambda[(size_t)h * dk + i];
                }
                dense_ctx c = {dk, A};
                double* xt = X + (size_t)t * dk;
                double* ut = U + (size_t)t * dk;
                const int itf = cg_generic(dk, dense_mv, &c, q + bt * dk, cg_steps, tol, xt, work);
                /* right-hand side of the adjoint system: G_t^T do_t */
                const double* dot_ = dout + bt * dv;
                for (int j = 0; j < dk; ++j) {
                    double s = 0.0;
                    for (int i = 0; i < dv; ++i) s += Gm[(size_t)i * dk + j] * dot_[i];
                    g[j] = s;
                }
                const int ita = cg_generic(dk, dense_mv, &c, g, cg_steps, tol, ut, work);
                if (iters_fwd) iters_fwd[bt] = itf;
                if (iters_adj) iters_adj[bt] = ita;
                for (int i = 0; i < dk; ++i) {
                    dq[bt * dk + i] = ut[i];
                    part[(size_t)bh * dk + i] -= ut[i] * xt[i];
                }
            }
            /* backward in time through the recurrences */
            for (int t = T - 1; t >= 0; --t) {
                const size_t bt = (size_t)bh * T + t;
                const double* kt = k + bt * dk;
                const double* vt = v + bt * dv;
                const double* xt = X + (size_t)t * dk;
                const double* ut = U + (size_t)t * dk;
                const double* dot_ = dout + bt * dv;
                const double gnext = (t + 1 < T) ? gamma[bt + 1] : 0.0;
                for (size_t e = 0; e < SH; ++e) Hbar[e] *= gnext;
                for (size_t e = 0; e < SG; ++e) Gbar[e] *= gnext;
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dk; ++j) Hbar[(size_t)i * dk + j] -= ut[i] * xt[j];
                for (int i = 0; i < dv; ++i)
                    for (int j = 0; j < dk; ++j) Gbar[(size_t)i * dk + j] += dot_[i] * xt[j];
                const double bta = beta[bt];
                double db = 0.0;
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dk; ++j) db += kt[i] * Hbar[(size_t)i * dk + j] * kt[j];
                for (int i = 0; i < dv; ++i)
                    for (int j = 0; j < dk; ++j) db += vt[i] * Gbar[(size_t)i * dk + j] * kt[j];
                dbeta[bt] = db;
                for (int i = 0; i < dk; ++i) {
                    double s = 0.0;
                    for (int j = 0; j < dk; ++j) s += (Hbar[(size_t)i * dk + j] + Hbar[(size_t)j * dk + i]) * kt[j];
                    for (int l = 0; l < dv; ++l) s += Gbar[(size_t)l * dk + i] * vt[l];
                    dk_out[bt * dk + i] = bta * s;
                }
                for (int l = 0; l < dv; ++l) {
                    double s = 0.0;
                    for (int j = 0; j < dk; ++j) s += Gbar[(size_t)l * dk + j] * kt[j];
                    dv_out[bt * dv + l] = bta * s;
                }
                const double* Hprev = Hs + (size_t)t * SH;
                const double* Gprev = Gs + (size_t)t * SG;
                double dg = 0.0;
                for (size_t e = 0; e < SH; ++e) dg += Hbar[e] * Hprev[e];
                for (size_t e = 0; e < SG; ++e) dg += Gbar[e] * Gprev[e];
                dgamma[bt] = dg;
            }
        }
        free(Hs); free(Gs); free(X); free(U); free(A); free(g); free(work); free(Hbar); free(Gbar);
    }
    if (!err) {   /* dlambda[h] = sum over the batch, in batch order */
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < dk; ++i) {
                double s = 0.0;
                for (int b = 0; b < B; ++b) s += part[((size_t)b * H + h) * dk + i];
                dlambda[(size_t)h * dk + i] = s;
            }
    }
    free(part);
    return err ? -2 : 0;
}
