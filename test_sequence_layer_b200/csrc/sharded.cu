// sharded.cu -- the two device steps of a sequence-sharded forward.
//
// Method: "MesaNet: Sequence Modeling by Locally Optimal Test-Time Training"
// (gist.science), Technical summary > Method > Mesa layer, "Parallelisation":
// the layer carries the states H_t, G_t from chunk to chunk, so a sequence
// split into consecutive slices (one per rank) needs only the state entering
// each slice. With the gated recurrence H_t = gamma_t H_{t-1} + beta_t k_t k_t^T,
// the state after slice s from an initial state S is D_s S + Delta_s, where
// Delta_s is the state after the slice from zero and D_s = prod_{t in s} gamma_t.
// So the state entering slice r is the exclusive prefix
//     S_0 = 0,   S_{s+1} = D_s S_s + Delta_s      (s < r),
// the same for G. chunk_state computes (Delta_s, D_s) of the caller's slice
// (the scan of the forward, no solve); after an all-gather of those across
// ranks, state_prefix forms S_r; the slice's forward then starts from it.
#include "mesa_internal.h"

namespace mesa {
namespace {

// D = exp(sum_t log gamma_t) per sequence; one CTA per sequence, fixed-order
// tree sum of per-thread partials (deterministic).
__global__ void __launch_bounds__(256) slice_decay_kernel(const float* __restrict__ gamma, int T,
                                                          float* __restrict__ decay) {
    __shared__ float part[256];
    const size_t off = (size_t)blockIdx.x * T;
    float s = 0.f;
    for (int t = threadIdx.x; t < T; t += 256) s += logf(gamma[off + t]);
    part[threadIdx.x] = s;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) decay[blockIdx.x] = expf(part[0]);
}

// S_r[e] for every element e of the [BH][rows][dk] states: slices in order.
__global__ void state_prefix_kernel(const float* __restrict__ S_s, const float* __restrict__ decay_s, int r,
                                    int BH, int per_seq, float* __restrict__ S_in) {
    const size_t n = (size_t)BH * per_seq;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        const int bh = (int)(e / per_seq);
        float acc = 0.f;
        for (int s = 0; s < r; ++s) acc = fmaf(decay_s[(size_t)s * BH + bh], acc, S_s[(size_t)s * n + e]);
        S_in[e] = acc;
    }
}

int prefix_grid(size_t n) {
    const size_t g = (n + 255) / 256;
    return (int)(g < 148 * 8 ? g : 148 * 8);
}

}  // namespace

cudaError_t chunk_state(const ForwardArgs& a, float* decay_out, cudaStream_t st) {
    cudaError_t e = cudaSuccess;
    if (a.T == 0) {
        // the caller has passed the state through; only the decay (1) is left
    } else if (tc_supported(a.dk, a.dv, a.chunk, a.dtype)) {
        char* ws = static_cast<char*>(a.workspace);
        e = tc_scan_launch(a, ws, reinterpret_cast<float*>(ws + tc_images_bytes(a.B, a.H, a.T)), error_word_ptr(), st);
    } else {
        ForwardArgs s = a;
        s.scan_only = true;
        e = forward_simt(s, st);
    }
    if (e != cudaSuccess) return e;
    LaunchTimer timer(kKindShard, st);
    slice_decay_kernel<<<a.B * a.H, 256, 0, st>>>(a.gamma, a.T, decay_out);
    return cudaGetLastError();
}

cudaError_t state_prefix(const float* H_s, const float* G_s, const float* decay_s, int r, int BH, int dk, int dv,
                         float* H_in, float* G_in, cudaStream_t st) {
    LaunchTimer timer(kKindShard, st);
    const size_t nh = (size_t)BH * dk * dk, ng = (size_t)BH * dv * dk;
    state_prefix_kernel<<<prefix_grid(nh), 256, 0, st>>>(H_s, decay_s, r, BH, dk * dk, H_in);
    state_prefix_kernel<<<prefix_grid(ng), 256, 0, st>>>(G_s, decay_s, r, BH, dv * dk, G_in);
    return cudaGetLastError();
}

}  // namespace mesa
