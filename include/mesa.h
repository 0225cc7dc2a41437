/*
 * mesa.h -- C ABI of the B200 (sm_100a) Mesa layer library (libmesa_b200.so).
 *
 * The Mesa layer of "MesaNet: Sequence Modeling by Locally Optimal Test-Time
 * Training" (gist.science, ja/ko/hi editions; Technical summary > Method >
 * Mesa layer). For every sequence (b, h) and token t it keeps the gated
 * statistics
 *     H_t = gamma_t H_{t-1} + beta_t k_t k_t^T        (dk x dk)
 *     G_t = gamma_t G_{t-1} + beta_t v_t k_t^T        (dv x dk)
 * (the page's cumulative forget factors zeta read as
 *  zeta_{tt'} = beta_t' prod_{s=t'+1..t} gamma_s), solves
 *     (H_t + Lambda) x_t = q_t
 * by conjugate gradient (the page's "optimal query response"), and emits the
 * locally optimal read-out o_t = G_t x_t (the page's Delta_t = Phi_t q_t with
 * Phi_t = G_t (H_t + Lambda)^-1, the minimiser of its Mesa objective).
 *
 * CG rule (identical in every entry point): x_0 = 0, r_0 = p_0 = q_t; before
 * each of at most cg_steps updates the token stops if tol > 0 and
 * |r|_2 <= tol |q_t|_2 (the page's per-token stopping criterion under
 * "Dynamic compute"); it also stops, keeping its x, if r.r <= 0 or
 * p.(H+Lambda)p <= 0 or is not finite. iters = number of updates applied.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller (except
 *     mesa_forward_host, whose tensors are host pointers). The library
 *     allocates no device memory in any call; scratch space is the caller's
 *     workspace.
 *   - Layouts are contiguous row-major: q, k [B,H,T,dk]; v, out [B,H,T,dv];
 *     gamma, beta, iters [B,H,T]; lambda [H,dk] (the diagonal of Lambda for
 *     each head, shared by the batch); H states [B,H,dk,dk]; G states
 *     [B,H,dv,dk].
 *   - Preconditions on values (not checked, the caller's contract):
 *     0 < gamma <= 1, beta >= 0, lambda > 0, all finite. A non-finite input
 *     makes the outputs of its chunk (on the tensor-core path: of its pair
 *     of chunks, which share every MMA) and of every later token of its
 *     sequence non-finite; it never hangs and touches no other sequence.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Device calls are asynchronous on it.
 *   - Argument errors are returned synchronously and nothing is launched.
 *     A failed launch returns MESA_ERR_CUDA. A kernel that gives up a bounded
 *     wait records MESA_ERR_DEVICE_TIMEOUT in a per-device error word that
 *     mesa_get_error() reads and clears.
 */
#ifndef MESA_H
#define MESA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MESA_OK = 0,
    MESA_ERR_INVALID_ARG = 1,    /* null pointer, bad size, misalignment, bad tol */
    MESA_ERR_UNSUPPORTED = 2,    /* valid but not implemented (dk, dv, chunk) */
    MESA_ERR_WORKSPACE = 3,      /* workspace missing or smaller than required */
    MESA_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed */
    MESA_ERR_DEVICE_TIMEOUT = 5  /* a kernel gave up a bounded wait (see mesa_get_error) */
} mesa_status;

typedef enum {
    MESA_F32 = 0,    /* q, k, v are float32 */
    MESA_BF16 = 1    /* q, k, v are bfloat16 (gamma, beta, lambda stay float32) */
} mesa_dtype;

/*
 * Bytes of device workspace mesa_forward needs for these sizes (0 if the
 * sizes are invalid or unsupported). The workspace holds the chunk-start
 * states {H_c, G_c} of every chunk (the layer's carried inter-chunk state).
 */
size_t mesa_forward_workspace_size(int B, int H, int T, int dk, int dv, int chunk,
                                   mesa_dtype dtype);

/*
 * Chunkwise-parallel forward of the Mesa layer over a whole sequence.
 * Source: the MesaNet page, Technical summary > Method > Mesa layer
 * (objective; CG solve of q*_t) and its "Parallelisation" paragraph (CG over
 * many time steps is gated linear attention; the layer keeps G_t and H_t
 * and solves the systems of a chunk in parallel).
 *
 *   q, k, v      input tensors, element type `dtype`, 16-byte aligned.
 *   gamma, beta  float32 [B,H,T], 4-byte aligned.
 *   lambda       float32 [H,dk], > 0.
 *   B, H, T      batch, heads, tokens; B,H >= 1, T >= 0 (T = 0: only the
 *                final-state outputs are written, as copies of the initial
 *                state or zeros).
 *   dk, dv       key and value width. Supported: dk == dv in {16,32,64,128}.
 *   chunk        chunk length C in {16,32,64}; T need not be a multiple of C
 *                (the tail behaves as if padded with beta = 0, gamma = 1).
 *                The tensor-core path serves dtype = MESA_BF16,
 *                dk = dv = 128, chunk = 64; every other supported shape runs
 *                the fp32 CUDA-core path. The tensor-core path divides every
 *                MMA operand (keys, values, decay mask, states, CG
 *                directions) by a power of two at or above its largest entry
 *                before rounding it to fp16, so it accepts the same range of
 *                magnitudes as float32; its rounding is ~2^-11 relative per
 *                operand, which the solve amplifies by up to the condition
 *                number of H_t + Lambda (bf16-mode accuracy holds while
 *                beta |k|^2 stays within a few hundred times lambda).
 *   cg_steps     maximum CG updates per token, 0..1024.
 *   tol          relative residual tolerance; <= 0 runs exactly cg_steps
 *                updates (unless breakdown). NaN is an argument error.
 *   out          float32 [B,H,T,dv], 16-byte aligned (written).
 *   iters_out    int32 [B,H,T] or NULL: CG updates applied per token.
 *   H_in, G_in   float32 initial states or NULL (zero), 16-byte aligned.
 *   H_out, G_out float32 final states (after token T-1) or NULL. May not
 *                alias H_in / G_in.
 *   workspace    device memory of at least mesa_forward_workspace_size()
 *                bytes, 256-byte aligned. Its contents on entry do not
 *                matter; calls sharing a workspace must not overlap.
 */
mesa_status mesa_forward(const void* q, const void* k, const void* v,
                         const float* gamma, const float* beta, const float* lambda,
                         int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype,
                         int cg_steps, float tol,
                         float* out, int32_t* iters_out,
                         const float* H_in, const float* G_in,
                         float* H_out, float* G_out,
                         void* workspace, size_t ws_bytes, void* stream);

/*
 * mesa_forward with a warm-started CG: token t's solve starts from a caller-
 * given guess x0_t instead of zero. Source: the MesaNet page, Significance
 * and claims (warm starts are named as the way to cut the solver's cost; the
 * pages give no rule). Reading taken: x_0 = x0_t, r_0 = q_t - (H_t + Lambda)
 * x0_t, p_0 = r_0, and the stopping test stays |r_k| <= tol |q_t|, so a
 * guess within the tolerance takes no step; iters counts the updates after
 * the start. In the one-pass forward every token of a block is solved at
 * once, so no token's neighbour has a solution to offer; the guesses come
 * from the caller, e.g. the solutions of an earlier forward over a context
 * that has since been edited or extended (x_out below).
 *
 *   x0       float32 [B,H,T,dk], 16-byte aligned, or NULL (start from zero:
 *            then the call equals mesa_forward).
 *   x_out    float32 [B,H,T,dk], 16-byte aligned, or NULL: every token's
 *            solution x_t. May be the same buffer as x0 (updated in place);
 *            otherwise neither may overlap the other or `out`.
 * Every other argument, and the cost of a cold call, as for mesa_forward; a
 * warm start adds one matrix-vector product per token (one more CG-step's
 * worth of work) and the read of x0.
 */
mesa_status mesa_forward_warm(const void* q, const void* k, const void* v,
                              const float* gamma, const float* beta, const float* lambda,
                              int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype,
                              int cg_steps, float tol, const float* x0, float* x_out,
                              float* out, int32_t* iters_out,
                              const float* H_in, const float* G_in,
                              float* H_out, float* G_out,
                              void* workspace, size_t ws_bytes, void* stream);

/*
 * Size of the fixed device scratch array behind mesa_forward_noalloc.
 */
#define MESA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/*
 * mesa_forward without a workspace argument, for callers that cannot
 * allocate device memory at all: plug-in code inside a host framework that
 * owns every device allocation and passes in only its tensors, or latency-
 * bound loops that must never call cudaMalloc (which can synchronise the
 * device). The MesaNet pages have no counterpart to this entry point; it
 * exists for those callers only.
 *
 * Arguments, layouts and results are exactly those of mesa_forward minus
 * `workspace` and `ws_bytes`. The scratch the forward needs (chunk-start
 * states) comes from a library-owned device array of
 * MESA_NOALLOC_SCRATCH_BYTES (32 MiB) that every GPU loading the library
 * holds until the process exits. Nothing is allocated by the call.
 *   - Sizes whose scratch (mesa_forward_workspace_size) exceeds
 *     MESA_NOALLOC_SCRATCH_BYTES are refused with MESA_ERR_WORKSPACE before
 *     any device work.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *     The address is cached per device for the device's primary context
 *     (the CUDA runtime's): calls from another driver context, or after
 *     cudaDeviceReset, are not supported.
 *   - All calls on a device share the array, which keeps the previous call's
 *     contents; every byte is written before it is read, so no clearing is
 *     needed. Calls that overlap on the GPU (different streams, or host
 *     threads without ordering) race on the array: serialise them.
 */
mesa_status mesa_forward_noalloc(const void* q, const void* k, const void* v,
                                 const float* gamma, const float* beta, const float* lambda,
                                 int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype,
                                 int cg_steps, float tol,
                                 float* out, int32_t* iters_out,
                                 const float* H_in, const float* G_in,
                                 float* H_out, float* G_out, void* stream);

/*
 * Input preprocessing of queries and keys, the layer's own input path
 * ("MesaNet" page, Technical summary > Architecture > "Preprocessing": keys
 * and queries are normalised, with a short-window convolution before the
 * Mesa layer; read as the convolution first, then the normalisation, so that
 * the layer receives unit-norm keys and queries). For every (b, h, t) and
 * channel i, separately for q and k with their own weights:
 *     u_t[i] = sum_{w=0..W-1} conv[h][w][i] * x_{t-w}[i]   (x = 0 before t = 0)
 *     y_t    = u_t / max(|u_t|_2, 1e-6)
 * q_raw, k_raw, q_out, k_out: [B,H,T,d] in `dtype` (MESA_BF16 rounds the
 * outputs to bf16, nearest-even; the arithmetic is fp32). conv_q, conv_k:
 * [H,W,d] fp32, w = lag in tokens (w = 0 multiplies the current token).
 * 1 <= W <= 4; d in {16, 32, 64, 128}; B*H <= 65535. The outputs are ready
 * to pass to mesa_forward as q and k. Outputs must not overlap the inputs or
 * each other (MESA_ERR_INVALID_ARG). Pointers are DEVICE pointers, 16-byte
 * aligned (conv 4-byte aligned). Asynchronous on `stream`; T = 0 is a no-op.
 */
mesa_status mesa_preprocess(const void* q_raw, const void* k_raw, const float* conv_q, const float* conv_k,
                            int B, int H, int T, int d, int W, mesa_dtype dtype, void* q_out, void* k_out,
                            void* stream);

/*
 * The forward with the q/k input preprocessing of mesa_preprocess applied on
 * the way in: equals mesa_preprocess(q_raw, k_raw, conv_q, conv_k, W)
 * followed by mesa_forward on its outputs, bit for bit. Source: the MesaNet
 * page, Technical summary > Architecture > "Preprocessing" (read as for
 * mesa_preprocess: causal depthwise convolution, then L2 normalisation, the
 * convolution starting from zero rows at the call's first token).
 *
 * On the tensor-core shape (MESA_BF16, dk = dv = 128, chunk = 64) nothing is
 * preprocessed ahead: the chunk-state scan and the solve convolve and
 * normalise the raw rows as they stage them (each 128-token block with the
 * three rows before it), so the preprocessed q and k never go to memory.
 * Every other shape runs the two steps, with the preprocessed q and k in
 * the workspace.
 *
 *   q_raw, k_raw  raw queries and keys, [B,H,T,dk] in `dtype`, 16-byte aligned.
 *   conv_q, conv_k  float32 [H,W,dk] weights (w = lag), 4-byte aligned.
 *   W             window, 1..4.
 *   workspace     at least mesa_forward_preprocessed_workspace_size() bytes,
 *                 256-byte aligned.
 * Every other argument as for mesa_forward.
 */
size_t mesa_forward_preprocessed_workspace_size(int B, int H, int T, int dk, int dv, int chunk,
                                                mesa_dtype dtype);
mesa_status mesa_forward_preprocessed(const void* q_raw, const void* k_raw, const void* v,
                                      const float* gamma, const float* beta, const float* lambda,
                                      const float* conv_q, const float* conv_k, int W,
                                      int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype,
                                      int cg_steps, float tol,
                                      float* out, int32_t* iters_out,
                                      const float* H_in, const float* G_in,
                                      float* H_out, float* G_out,
                                      void* workspace, size_t ws_bytes, void* stream);

/*
 * Backward pass of the layer (training): gradients of a scalar loss L given
 * dout = dL/do for the inputs of a mesa_forward call with zero initial
 * states. The pages claim training in time linear in T but give no backward
 * method; the reading implemented is implicit differentiation of the
 * solution map x_t = (H_t + Lambda)^-1 q_t, with the adjoint system
 *     u_t = CG(H_t + Lambda, G_t^T dout_t)
 * solved under the same CG rule as the forward (same cg_steps; the tolerance
 * test relative to |G_t^T dout_t|). Then dq_t = u_t, dlambda_i = -sum u_ti x_ti,
 * and back through the gated recurrences of H and G (with
 * Hbar_t = -sum_{t'>=t} (prod gamma) u_t' x_t'^T and
 * Gbar_t = sum_{t'>=t} (prod gamma) dout_t' x_t'^T):
 *     dk_t = beta_t ((Hbar_t + Hbar_t^T) k_t + Gbar_t^T v_t),  dv_t = beta_t Gbar_t k_t,
 *     dbeta_t = k_t^T Hbar_t k_t + v_t^T Gbar_t k_t,
 *     dgamma_t = <Hbar_t, H_{t-1}> + <Gbar_t, G_{t-1}>.
 * When CG has converged this is the exact gradient of the layer.
 *
 *   q, k, v, gamma, beta, lambda, B, H, T, dk, dv, chunk, dtype, cg_steps,
 *                tol: as in mesa_forward (every supported shape and dtype).
 *                On the tensor-core shape (MESA_BF16, dk = dv = 128,
 *                chunk = 64) the forward solve, the right-hand sides
 *                G_t^T dout_t and the adjoint solve run on the tensor cores
 *                (fp16 operands, fp32 accumulation: the bf16-mode accuracy);
 *                the reverse gradient scans and every other shape are fp32 on
 *                the CUDA cores.
 *   dout         float32 [B,H,T,dv].
 *   dq, dk_out   float32 [B,H,T,dk];  dv_out float32 [B,H,T,dv].
 *   dgamma, dbeta float32 [B,H,T].    dlambda float32 [H,dk] (summed over
 *                the batch).
 *   workspace    device memory of at least mesa_backward_workspace_size()
 *                bytes, 256-byte aligned (it holds the chunk states, the
 *                forward solutions and the reverse gradient states).
 * All pointers are DEVICE pointers, 16-byte aligned (gamma, beta, lambda,
 * dgamma, dbeta, dlambda 4-byte aligned); the outputs must not overlap the
 * inputs. Asynchronous on `stream`. T = 0 writes zeros to dlambda only.
 */
size_t mesa_backward_workspace_size(int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype);

mesa_status mesa_backward(const void* q, const void* k, const void* v,
                          const float* gamma, const float* beta, const float* lambda,
                          int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype,
                          int cg_steps, float tol, const float* dout,
                          float* dq, float* dk_out, float* dv_out, float* dgamma, float* dbeta, float* dlambda,
                          void* workspace, size_t ws_bytes, void* stream);

/*
 * Sequence sharding (a long sequence split into consecutive slices, one per
 * GPU). The layer carries the states H_t, G_t from chunk to chunk ("MesaNet"
 * page, Mesa layer, "Parallelisation"); the state after a slice s from an
 * initial state S is D_s S + Delta_s, with Delta_s the state after the slice
 * from zero and D_s = prod_{t in s} gamma_t. So each slice needs only the
 * state entering it:
 *     S_0 = 0,  S_{s+1} = D_s S_s + Delta_s.
 * A sharded forward: mesa_chunk_state on the slice (from zero) -> exchange
 * (Delta_s, D_s) of every slice (an all-gather) -> mesa_state_prefix for the
 * caller's slice r -> mesa_forward on the slice with H_in, G_in = S_r.
 *
 * mesa_chunk_state: the scan of mesa_forward without the solve. For every
 * (b, h): H_out, G_out = the states after the T tokens from H_in, G_in (NULL:
 * zero) and decay_out [B,H] = prod_t gamma_t. Arguments as in mesa_forward;
 * H_out, G_out float32 [B,H,dk,dk] / [B,H,dv,dk], 16-byte aligned, distinct
 * from the inputs; decay_out float32 [B,H]. Workspace: at least
 * mesa_chunk_state_workspace_size() bytes, 256-byte aligned. T = 0 copies
 * (or zeroes) the state and writes decay 1.
 */
size_t mesa_chunk_state_workspace_size(int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype);

mesa_status mesa_chunk_state(const void* k, const void* v, const float* gamma, const float* beta,
                             int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype,
                             const float* H_in, const float* G_in, float* H_out, float* G_out, float* decay_out,
                             void* workspace, size_t ws_bytes, void* stream);

/*
 * The state entering slice r (0 <= r <= n_slices) from the summaries of the
 * slices before it, in sequence order: H_slices float32 [n_slices,B,H,dk,dk]
 * and G_slices [n_slices,B,H,dv,dk] (each from a zero state), decay_slices
 * [n_slices,B,H]. Writes H_in, G_in (float32 [B,H,dk,dk] / [B,H,dv,dk],
 * 16-byte aligned, not overlapping the inputs or each other). r = 0 writes
 * zeros; r = n_slices gives the state after the whole sequence. dk == dv in
 * {16,32,64,128}. Asynchronous on `stream`.
 */
mesa_status mesa_state_prefix(const float* H_slices, const float* G_slices, const float* decay_slices,
                              int n_slices, int r, int B, int H, int dk, int dv,
                              float* H_in, float* G_in, void* stream);

/*
 * Bytes of device workspace mesa_forward_host needs: the mesa_forward
 * workspace plus device staging for every tensor argument.
 */
size_t mesa_forward_host_workspace_size(int B, int H, int T, int dk, int dv, int chunk,
                                        mesa_dtype dtype);

/*
 * The same forward with every tensor in HOST memory (page-locked memory is
 * needed for the copies to overlap; pageable memory works but is slower).
 * The batch is split into slices of sequences (one slice when the inputs are
 * under 16 MiB): with 16 or more batch rows, up to 32 groups of whole rows;
 * with fewer, runs of heads inside one batch row (about 16 slices). Slice by
 * slice, the inputs are copied to
 * the device on a library copy-in stream, the forward runs on one of two
 * library compute streams once they have landed, and the outputs are copied
 * back on a library copy-out stream, so both copy directions overlap the
 * kernels. The library streams start after the work already enqueued on
 * `stream`, `stream` waits for the last copy, and the call synchronises
 * `stream` before returning, so the host outputs are valid on MESA_OK.
 * Calls from several host threads are serialised by a library lock (the
 * library streams are shared per device). No host alignment is required.
 * `workspace` is DEVICE memory of at least mesa_forward_host_workspace_size()
 * bytes, 256-byte aligned.
 */
mesa_status mesa_forward_host(const void* q, const void* k, const void* v,
                              const float* gamma, const float* beta, const float* lambda,
                              int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype,
                              int cg_steps, float tol,
                              float* out, int32_t* iters_out,
                              const float* H_in, const float* G_in,
                              float* H_out, float* G_out,
                              void* workspace, size_t ws_bytes, void* stream);

/*
 * One recurrent decode step on explicit state, O(1) per token (the MesaNet
 * page, "Parallelisation": O(1) inference with the state variables G_t, H_t).
 * For every (b, h): H <- gamma H + beta k k^T, G <- gamma G + beta v k^T,
 * x = CG(H + Lambda, q), out = G x.
 *
 *   q, k         float32 [B,H,dk];  v float32 [B,H,dv]; 16-byte aligned.
 *   gamma, beta  float32 [B,H].     lambda float32 [H,dk].
 *   dk == dv in {16,32,64,128}.
 *   Hstate       float32 [B,H,dk,dk], read and overwritten in place.
 *   Gstate       float32 [B,H,dv,dk], read and overwritten in place.
 *   cg_steps, tol as in mesa_forward.
 *   out          float32 [B,H,dv] (written).  iters_out int32 [B,H] or NULL.
 * No workspace is needed.
 */
mesa_status mesa_step(const float* q, const float* k, const float* v,
                      const float* gamma, const float* beta, const float* lambda,
                      int B, int H, int dk, int dv,
                      float* Hstate, float* Gstate,
                      int cg_steps, float tol,
                      float* out, int32_t* iters_out, void* stream);

/*
 * mesa_step with a warm-started solve: the CG of each head starts from the
 * guess in x_state instead of zero (the pages name warm starts as the way to
 * cut the solver's cost: "MesaNet" page, Significance and claims). x_state
 * [B,H,dk] fp32 DEVICE buffer, in/out: on entry the starting guess x0 (for
 * example the previous step's solution; zeros make this call mesa_step), on
 * exit this step's solution x. The CG rule is mesa_step's with r0 = q -
 * (H + Lambda) x0 and p0 = r0; the stopping test stays |r_k| <= tol |q|, so a
 * good guess stops after fewer updates (iters counts the updates applied).
 * x_state may be NULL (cold start); it must not alias q or out. Other
 * arguments, errors and the state update are those of mesa_step.
 */
mesa_status mesa_step_warm(const float* q, const float* k, const float* v,
                           const float* gamma, const float* beta, const float* lambda,
                           int B, int H, int dk, int dv,
                           float* Hstate, float* Gstate, float* x_state,
                           int cg_steps, float tol,
                           float* out, int32_t* iters_out, void* stream);

/*
 * Synchronises `stream`, then reads and clears the calling device's error
 * word. Returns MESA_OK if no kernel recorded an error since the last call,
 * MESA_ERR_DEVICE_TIMEOUT if one gave up a bounded wait, MESA_ERR_CUDA if the
 * synchronisation itself failed.
 */
mesa_status mesa_get_error(void* stream);

/* Static, human-readable name of a status code (never NULL). */
const char* mesa_status_string(mesa_status s);

/*
 * Kernel timing (a profiling aid, off by default). While enabled, every
 * kernel the library launches is bracketed by CUDA events recorded on the
 * call's stream, and counted. mesa_timing_read() synchronises those events
 * and returns, for up to `max` kernel kinds, the kind's name, its number of
 * launches and its summed device time in milliseconds since the last read;
 * it then clears the records. Returns the number of kinds written, or -1 on
 * a CUDA error. Not thread-safe; enable it only in one host thread.
 */
mesa_status mesa_timing_enable(int on);
int mesa_timing_read(const char** names, int* launches, double* total_ms, int max);

/* Library version: major*10000 + minor*100 + patch. */
int mesa_version(void);

#ifdef MESA_DEBUG
/*
 * Debug builds only (libmesa_b200_debug.so, compiled with -DMESA_DEBUG):
 * fault injection for the failure-detection tests; the pages have no
 * counterpart. The next `launches` launches of the tensor-core solve kernel
 * (bf16, d = 128, chunk 64) leave out the completion signal of their first
 * Z product. Every thread's bounded wait on it (about one second of clock
 * cycles) then runs out; the kernel records a timeout in the error word,
 * lets every issued MMA and copy drain (bounded again), frees its tensor
 * memory and returns, leaving the context usable. The forward's outputs are
 * then undefined and mesa_get_error() returns MESA_ERR_DEVICE_TIMEOUT.
 * Returns MESA_ERR_INVALID_ARG for launches < 0.
 */
mesa_status mesa_debug_skip_commit(int launches);
#endif

#ifdef __cplusplus
}
#endif
#endif /* MESA_H */
