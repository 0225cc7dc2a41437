// mesa_internal.h -- host-side declarations shared by the library's .cu files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "mesa.h"

namespace mesa {

// Validated arguments of one forward call (device pointers).
struct ForwardArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* gamma;
    const float* beta;
    const float* lambda;
    int B, H, T, dk, dv, chunk;
    mesa_dtype dtype;
    int cg_steps;
    float tol;
    float* out;
    int32_t* iters;
    const float* H_in;
    const float* G_in;
    float* H_out;
    float* G_out;
    void* workspace;
    size_t ws_bytes;
    float* x_out = nullptr;     // the CG solutions x_t [B,H,T,dk] (fp32), when not null
    const float* x0 = nullptr;  // per-token CG starting guesses [B,H,T,dk] (fp32), when not null
    // fused input preprocessing (tensor-core path): q and k are raw, and the
    // kernels convolve and normalise them as they stage them (weights [H,W,dk])
    const float* conv_q = nullptr;
    const float* conv_k = nullptr;
    int conv_w = 0;
    bool scan_only = false;     // fp32 CUDA-core path only: the chunk-state scan, no solve
};

struct BackwardArgs {
    ForwardArgs f;              // the forward's inputs (out, iters, states unused)
    const float* dout;          // dL/do [B,H,T,dv]
    float* dq;                  // [B,H,T,dk]
    float* dk;                  // [B,H,T,dk]
    float* dv;                  // [B,H,T,dv]
    float* dgamma;              // [B,H,T]
    float* dbeta;               // [B,H,T]
    float* dlambda;             // [H,dk]
};

// Device address of the calling device's error word (nullptr on failure).
unsigned* error_word_ptr();

// Kernel kinds for the optional timing records (mesa_timing_enable).
enum KernelKind : int {
    kKindSimtScan = 0, kKindSimtCg, kKindStep, kKindTcScan, kKindTcCg, kKindPre,
    kKindBwdAdj, kKindBwdRscan, kKindBwdGrad, kKindBwdReduce, kKindShard, kKindBwdRhs, kKindCount
};

// Brackets one launch with CUDA events on `st` while timing is enabled.
class LaunchTimer {
  public:
    LaunchTimer(int kind, cudaStream_t st);
    ~LaunchTimer();
    LaunchTimer(const LaunchTimer&) = delete;
    LaunchTimer& operator=(const LaunchTimer&) = delete;

  private:
    int slot_;
    cudaStream_t st_;
};

// fp32 CUDA-core path (simt_forward.cu).
size_t simt_workspace_bytes(int B, int H, int T, int dk, int dv, int chunk);
cudaError_t forward_simt(const ForwardArgs& a, cudaStream_t st);
size_t backward_workspace_bytes(int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype);
// Sequence sharding: the state after a slice and its total decay; the state
// entering slice r from the summaries of slices 0..r-1 (sharded.cu).
cudaError_t chunk_state(const ForwardArgs& a, float* decay_out, cudaStream_t st);
cudaError_t state_prefix(const float* H_s, const float* G_s, const float* decay_s, int r, int BH, int dk, int dv,
                         float* H_in, float* G_in, cudaStream_t st);
cudaError_t backward_simt(const BackwardArgs& a, cudaStream_t st);

// Tensor-core path (tc_forward.cu): bf16 inputs, dk = dv = 128, chunk = 64.
bool tc_supported(int dk, int dv, int chunk, mesa_dtype dtype);
size_t tc_workspace_bytes(int B, int H, int T);
size_t tc_images_bytes(int B, int H, int T);     // the state images at the start of the workspace
cudaError_t forward_tc(const ForwardArgs& a, cudaStream_t st);
// Chunk-state scan of the tensor-core forward: state images and scales into
// img / scales (layout in tc_layout.cuh), final states into a.H_out / a.G_out.
cudaError_t tc_scan_launch(const ForwardArgs& a, void* img, float* scales, unsigned* err, cudaStream_t st);
// The backward's reverse chunk scan of the gradient states on the tensor
// cores (d = 128, C = 64): per chunk the fp32 states carried in from the
// tokens after it, [B*H][chunks][Hhat, Ghat][128][128].
cudaError_t tc_rscan_launch(const float* dout, const float* u, const float* xsol, const float* gamma, int B, int H,
                            int T, float* rstates, unsigned* err, cudaStream_t st);
// The backward's adjoint solve on the tensor cores, from the images a
// forward_tc call left at the start of `images_ws`: the right-hand side
// g_t = G_t^T dout_t (into rhs_buf), then u_t = CG(H_t + Lambda, g_t) into dq
// and e_t = g_t . x_t - u_t . (H_t x_t) into zt.
cudaError_t tc_adjoint(const ForwardArgs& f, const void* images_ws, const float* dout, const float* xsol,
                       float* rhs_buf, float* dq, float* zt, cudaStream_t st);
#ifdef MESA_DEBUG
// The next `launches` launches of the tensor-core solve kernel leave out the
// completion signal of their first Z product (fault injection, debug builds).
cudaError_t tc_debug_skip_commit(int launches);
#endif

// Decode step (decode.cu).
struct StepArgs {
    const float* q;
    const float* k;
    const float* v;
    const float* gamma;
    const float* beta;
    const float* lambda;
    int B, H, dk, dv;
    float* Hs;
    float* Gs;
    int cg_steps;
    float tol;
    float* out;
    int32_t* iters;
    float* xs;           // optional warm start [B,H,dk], in/out
};
cudaError_t step_launch(const StepArgs& a, cudaStream_t st);

// Input preprocessing (preprocess.cu).
struct PreArgs {
    const void* xq;
    const void* xk;
    const float* conv_q;
    const float* conv_k;
    int B, H, T, d, W;
    mesa_dtype dtype;
    void* yq;
    void* yk;
};
cudaError_t preprocess_launch(const PreArgs& a, cudaStream_t st);

}  // namespace mesa
