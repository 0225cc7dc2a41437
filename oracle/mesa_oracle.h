/*
 * mesa_oracle.h -- plain fp64 CPU reference of the Mesa layer.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load or call this library. The product
 * (the CUDA library under test_sequence_layer_b200/) neither includes this
 * header nor links this code, and this code includes nothing of the product.
 *
 * Method source: "MesaNet: Sequence Modeling by Locally Optimal Test-Time
 * Training" (gist.science, ja/ko/hi editions), Technical summary > Method >
 * Mesa layer. See mesa_oracle.c for the step-by-step citations.
 *
 * Layouts (all row-major, contiguous, fp64):
 *   q, k   [B, H, T, dk]      v, out [B, H, T, dv]
 *   gamma, beta [B, H, T]     lambda [H, dk]   (diagonal of Lambda per head)
 *   H state [B, H, dk, dk]    G state [B, H, dv, dk]
 *   iters  [B, H, T] int32    (number of CG updates applied to each token)
 * Optional pointers may be NULL. Return value: 0 on success, a negative
 * number for an invalid argument (nothing is written in that case).
 */
#ifndef MESA_ORACLE_H
#define MESA_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Per-token recurrence with explicit H_t, G_t and conjugate gradient. */
int oracle_forward_cg(const double* q, const double* k, const double* v,
                      const double* gamma, const double* beta, const double* lambda,
                      int B, int H, int T, int dk, int dv, int cg_steps, double tol,
                      const double* H_init, const double* G_init,
                      double* out, int32_t* iters, double* H_final, double* G_final);

/* oracle_forward_cg with every token's CG started from x0 [B,H,T,dk] (NULL:
 * zero); x_out [B,H,T,dk] or NULL receives the solutions. */
int oracle_forward_cg_x0(const double* q, const double* k, const double* v,
                         const double* gamma, const double* beta, const double* lambda,
                         int B, int H, int T, int dk, int dv, int cg_steps, double tol,
                         const double* x0, const double* H_init, const double* G_init,
                         double* out, int32_t* iters, double* x_out, double* H_final, double* G_final);

/* Per-token recurrence with an exact Cholesky solve of (H_t + Lambda) x = q. */
int oracle_forward_cholesky(const double* q, const double* k, const double* v,
                            const double* gamma, const double* beta, const double* lambda,
                            int B, int H, int T, int dk, int dv,
                            const double* H_init, const double* G_init,
                            double* out, double* H_final, double* G_final);

/* Chunked form: carried chunk-start states plus decay-masked in-chunk sums;
 * the CG rule is the same as oracle_forward_cg. */
int oracle_forward_chunked(const double* q, const double* k, const double* v,
                           const double* gamma, const double* beta, const double* lambda,
                           int B, int H, int T, int dk, int dv, int chunk,
                           int cg_steps, double tol,
                           const double* H_init, const double* G_init,
                           double* out, int32_t* iters, double* H_final, double* G_final);

/* One recurrent decode step on explicit state (updated in place). */
int oracle_step(const double* q, const double* k, const double* v,
                const double* gamma, const double* beta, const double* lambda,
                int B, int H, int dk, int dv, double* Hstate, double* Gstate,
                int cg_steps, double tol, double* out, int32_t* iters);

/* Input preprocessing of queries or keys (MesaNet page, Architecture,
 * "Preprocessing": keys and queries are normalised, with a short-window
 * convolution before the Mesa layer). Read as: a causal depthwise convolution
 * over time, then L2 normalisation of every token:
 *   u_t[i] = sum_{w=0..W-1} conv[h][w][i] * x[b][h][t-w][i]   (x = 0 before t = 0)
 *   y_t    = u_t / max(|u_t|_2, 1e-6)
 * x, y [B, H, T, d]; conv [H, W, d] (w = lag in tokens). */
int oracle_preprocess(const double* x, const double* conv, int B, int H, int T, int d, int W, double* y);

/* One decode step whose CG starts from x_state ([B, H, dk]: the starting
 * guess on entry, the solution on exit; NULL starts from zero, which is
 * oracle_step). The stopping test stays |r_k| <= tol |q|. */
int oracle_step_warm(const double* q, const double* k, const double* v,
                     const double* gamma, const double* beta, const double* lambda,
                     int B, int H, int dk, int dv, double* Hstate, double* Gstate, double* x_state,
                     int cg_steps, double tol, double* out, int32_t* iters);

/* Dense CG on one SPD system A x = b (A n-by-n row-major), same rule as above,
 * from x0 (NULL: zero). Exposed so tests can pin the CG rule on its own. */
int oracle_cg_dense(int n, const double* A, const double* b, const double* x0, int cg_steps, double tol,
                    double* x, int32_t* iters);

/* Backward pass (reading: implicit differentiation of x_t = (H_t+Lambda)^-1 q_t,
 * adjoint u_t = CG_N(H_t + Lambda, G_t^T do_t) under the same CG rule) for
 * zero initial states. dout [B,H,T,dv] is dL/do. Outputs: dq, dk [B,H,T,dk];
 * dv [B,H,T,dv]; dgamma, dbeta [B,H,T]; dlambda [H,dk] (summed over the
 * batch); iters_fwd / iters_adj [B,H,T] (NULL allowed): CG updates of the
 * forward and the adjoint solve. */
int oracle_backward(const double* q, const double* k, const double* v,
                    const double* gamma, const double* beta, const double* lambda,
                    int B, int H, int T, int dk, int dv, int cg_steps, double tol, const double* dout,
                    double* dq, double* dk_out, double* dv_out, double* dgamma, double* dbeta,
                    double* dlambda, int32_t* iters_fwd, int32_t* iters_adj);

#ifdef __cplusplus
}
#endif
#endif
