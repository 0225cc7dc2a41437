// api.cu -- the extern "C" entry points of libmesa_b200.so (declared in mesa.h):
// argument validation, workspace carving, kernel dispatch, the host-buffer
// variant and the per-device error word.
#include <math.h>
#include <string.h>

#include <mutex>
#include <nvtx3/nvToolsExt.h>
#include <vector>

#include "mesa_common.cuh"
#include "mesa_internal.h"

namespace mesa {

__device__ unsigned g_error_word = 0;

namespace {

constexpr int kMaxDevices = 64;
unsigned* g_err_ptr[kMaxDevices] = {nullptr};

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool supported_width(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

// Shape checks shared by every forward entry point (no pointers involved).
mesa_status check_shape(int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype,
                        int cg_steps, float tol) {
    if (B < 1 || H < 1 || T < 0 || dk < 1 || dv < 1 || chunk < 1) return MESA_ERR_INVALID_ARG;
    if (dtype != MESA_F32 && dtype != MESA_BF16) return MESA_ERR_INVALID_ARG;
    if (cg_steps < 0 || cg_steps > 1024 || isnan(tol)) return MESA_ERR_INVALID_ARG;
    if ((long long)B * H > 65535) return MESA_ERR_UNSUPPORTED;           // grid.y limit
    if (!supported_width(dk) || dk != dv) return MESA_ERR_UNSUPPORTED;
    if (chunk != 16 && chunk != 32 && chunk != 64) return MESA_ERR_UNSUPPORTED;
    if ((long long)(T + chunk - 1) / chunk > 0x7fffffffLL) return MESA_ERR_UNSUPPORTED;
    return MESA_OK;
}

size_t workspace_bytes(int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype) {
    if (tc_supported(dk, dv, chunk, dtype)) return tc_workspace_bytes(B, H, T);
    return simt_workspace_bytes(B, H, T, dk, dv, chunk);
}

size_t elem_size(mesa_dtype d) { return d == MESA_BF16 ? 2 : 4; }

mesa_status launch_forward(const ForwardArgs& a, cudaStream_t st) {
    const size_t sbytes = (size_t)a.B * a.H * a.dk * a.dk * sizeof(float);
    const size_t gbytes = (size_t)a.B * a.H * a.dv * a.dk * sizeof(float);
    if (a.T == 0) {
        // Nothing to read out; the final state is the initial state.
        if (a.H_out) {
            cudaError_t e = a.H_in ? cudaMemcpyAsync(a.H_out, a.H_in, sbytes, cudaMemcpyDeviceToDevice, st)
                                   : cudaMemsetAsync(a.H_out, 0, sbytes, st);
            if (e != cudaSuccess) return MESA_ERR_CUDA;
        }
        if (a.G_out) {
            cudaError_t e = a.G_in ? cudaMemcpyAsync(a.G_out, a.G_in, gbytes, cudaMemcpyDeviceToDevice, st)
                                   : cudaMemsetAsync(a.G_out, 0, gbytes, st);
            if (e != cudaSuccess) return MESA_ERR_CUDA;
        }
        return MESA_OK;
    }
    cudaError_t e = tc_supported(a.dk, a.dv, a.chunk, a.dtype) ? forward_tc(a, st) : forward_simt(a, st);
    return e == cudaSuccess ? MESA_OK : MESA_ERR_CUDA;
}

// ---- kernel timing records ----
const char* const kKindNames[kKindCount] = {"simt_scan", "simt_cg", "decode_step", "tc_scan", "tc_cg",
                                             "preprocess", "bwd_adjoint", "bwd_rscan", "bwd_grad", "bwd_reduce",
                                             "shard", "bwd_rhs"};
struct TimingRec {
    int kind;
    cudaEvent_t start, stop;
};
bool g_timing_on = false;
std::vector<TimingRec> g_recs;
std::vector<cudaEvent_t> g_event_pool;
constexpr size_t kMaxRecs = 1 << 16;

cudaEvent_t take_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

}  // namespace

// Every launch is also an NVTX range named after its kernel kind, so that
// Nsight tools show the library's kernels by name on the host timeline.
LaunchTimer::LaunchTimer(int kind, cudaStream_t st) : slot_(-1), st_(st) {
    nvtxRangePushA(kKindNames[kind]);
    if (!g_timing_on || g_recs.size() >= kMaxRecs) return;
    TimingRec r{kind, take_event(), take_event()};
    if (!r.start || !r.stop || cudaEventRecord(r.start, st) != cudaSuccess) {
        if (r.start) g_event_pool.push_back(r.start);
        if (r.stop) g_event_pool.push_back(r.stop);
        return;
    }
    slot_ = (int)g_recs.size();
    g_recs.push_back(r);
}

LaunchTimer::~LaunchTimer() {
    if (slot_ >= 0) cudaEventRecord(g_recs[slot_].stop, st_);
    nvtxRangePop();
}

unsigned* error_word_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    if (!g_err_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
        g_err_ptr[dev] = static_cast<unsigned*>(p);
    }
    return g_err_ptr[dev];
}

}  // namespace mesa

using namespace mesa;

namespace mesa {
namespace {

// Streams and events of the host-buffer pipeline, created once per device and
// kept for the life of the process. The pipeline splits the batch into slices
// of sequences (every (b, h) sequence is independent): a slice is a run of
// nh heads of one batch row b, so it is contiguous in every [B,H,...] tensor
// and runs as a forward with B = 1, H = nh and lambda offset to its first
// head. Slice i's inputs go up on the copy-in stream, its forward runs on
// compute stream i % 2 once they have landed, and its outputs come down on the
// copy-out stream once it is done, so the two copy directions and the kernels
// overlap.
constexpr int kMaxSlices = 32;
constexpr int kTargetSlices = 16;
struct HostPipe {
    bool ready = false;
    cudaStream_t in = nullptr, out = nullptr, comp[2] = {nullptr, nullptr};
    cudaEvent_t start = nullptr, end = nullptr, landed[kMaxSlices] = {}, done[kMaxSlices] = {};
};
HostPipe g_pipe[kMaxDevices];
std::mutex g_pipe_mutex;

HostPipe* host_pipe() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    HostPipe& hp = g_pipe[dev];
    if (hp.ready) return &hp;
    const unsigned sf = cudaStreamNonBlocking, ef = cudaEventDisableTiming;
    bool ok = cudaStreamCreateWithFlags(&hp.in, sf) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.out, sf) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.comp[0], sf) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.comp[1], sf) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.start, ef) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.end, ef) == cudaSuccess;
    for (int i = 0; ok && i < kMaxSlices; ++i)
        ok = cudaEventCreateWithFlags(&hp.landed[i], ef) == cudaSuccess &&
             cudaEventCreateWithFlags(&hp.done[i], ef) == cudaSuccess;
    if (!ok) return nullptr;
    hp.ready = true;
    return &hp;
}

}  // namespace
}  // namespace mesa

extern "C" {

int mesa_version(void) { return 10000; }

const char* mesa_status_string(mesa_status s) {
    switch (s) {
        case MESA_OK: return "MESA_OK";
        case MESA_ERR_INVALID_ARG: return "MESA_ERR_INVALID_ARG";
        case MESA_ERR_UNSUPPORTED: return "MESA_ERR_UNSUPPORTED";
        case MESA_ERR_WORKSPACE: return "MESA_ERR_WORKSPACE";
        case MESA_ERR_CUDA: return "MESA_ERR_CUDA";
        case MESA_ERR_DEVICE_TIMEOUT: return "MESA_ERR_DEVICE_TIMEOUT";
    }
    return "MESA_ERR_UNKNOWN";
}

size_t mesa_forward_workspace_size(int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype) {
    if (check_shape(B, H, T, dk, dv, chunk, dtype, 0, 0.f) != MESA_OK) return 0;
    return workspace_bytes(B, H, T, dk, dv, chunk, dtype);
}

mesa_status mesa_forward(const void* q, const void* k, const void* v,
                         const float* gamma, const float* beta, const float* lambda,
                         int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype,
                         int cg_steps, float tol,
                         float* out, int32_t* iters_out,
                         const float* H_in, const float* G_in,
                         float* H_out, float* G_out,
                         void* workspace, size_t ws_bytes, void* stream) {
    mesa_status s = check_shape(B, H, T, dk, dv, chunk, dtype, cg_steps, tol);
    if (s != MESA_OK) return s;
    if (!lambda || !aligned(lambda, 4)) return MESA_ERR_INVALID_ARG;
    if (T > 0) {
        if (!q || !k || !v || !gamma || !beta || !out) return MESA_ERR_INVALID_ARG;
        if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return MESA_ERR_INVALID_ARG;
        if (!aligned(gamma, 4) || !aligned(beta, 4)) return MESA_ERR_INVALID_ARG;
        if (iters_out && !aligned(iters_out, 4)) return MESA_ERR_INVALID_ARG;
    }
    for (const void* p : {(const void*)H_in, (const void*)G_in, (const void*)H_out, (const void*)G_out})
        if (p && !aligned(p, 16)) return MESA_ERR_INVALID_ARG;
    if ((H_out && H_out == H_in) || (G_out && G_out == G_in)) return MESA_ERR_INVALID_ARG;
    const size_t need = workspace_bytes(B, H, T, dk, dv, chunk, dtype);
    if (T > 0 && need > 0) {
        if (!workspace || ws_bytes < need) return MESA_ERR_WORKSPACE;
        if (!aligned(workspace, 256)) return MESA_ERR_INVALID_ARG;
    }
    ForwardArgs a{q, k, v, gamma, beta, lambda, B, H, T, dk, dv, chunk, dtype, cg_steps, tol,
                  out, iters_out, H_in, G_in, H_out, G_out, workspace, ws_bytes};
    return launch_forward(a, static_cast<cudaStream_t>(stream));
}

mesa_status mesa_forward_warm(const void* q, const void* k, const void* v,
                              const float* gamma, const float* beta, const float* lambda,
                              int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype,
                              int cg_steps, float tol, const float* x0, float* x_out,
                              float* out, int32_t* iters_out,
                              const float* H_in, const float* G_in,
                              float* H_out, float* G_out,
                              void* workspace, size_t ws_bytes, void* stream) {
    if (T > 0) {
        if ((x0 && !aligned(x0, 16)) || (x_out && !aligned(x_out, 16))) return MESA_ERR_INVALID_ARG;
        // x0 and x_out are read and written row by row by the same block of
        // threads, so they may be the same buffer; they must not overlap anything else
        const size_t xb = (size_t)B * H * T * dk * sizeof(float);
        const char* ob = reinterpret_cast<const char*>(out);
        const size_t outb = (size_t)B * H * T * dv * sizeof(float);
        for (const void* xp : {(const void*)x0, (const void*)x_out}) {
            const char* c = static_cast<const char*>(xp);
            if (c && ob && c < ob + outb && ob < c + xb) return MESA_ERR_INVALID_ARG;
        }
        if (x0 && x_out && x0 != x_out) {
            const char* a = reinterpret_cast<const char*>(x0);
            const char* b = reinterpret_cast<const char*>(x_out);
            if (a < b + xb && b < a + xb) return MESA_ERR_INVALID_ARG;
        }
    }
    mesa_status s = check_shape(B, H, T, dk, dv, chunk, dtype, cg_steps, tol);
    if (s != MESA_OK) return s;
    if (!lambda || !aligned(lambda, 4)) return MESA_ERR_INVALID_ARG;
    if (T > 0) {
        if (!q || !k || !v || !gamma || !beta || !out) return MESA_ERR_INVALID_ARG;
        if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return MESA_ERR_INVALID_ARG;
        if (!aligned(gamma, 4) || !aligned(beta, 4)) return MESA_ERR_INVALID_ARG;
        if (iters_out && !aligned(iters_out, 4)) return MESA_ERR_INVALID_ARG;
    }
    for (const void* p : {(const void*)H_in, (const void*)G_in, (const void*)H_out, (const void*)G_out})
        if (p && !aligned(p, 16)) return MESA_ERR_INVALID_ARG;
    if ((H_out && H_out == H_in) || (G_out && G_out == G_in)) return MESA_ERR_INVALID_ARG;
    const size_t need = workspace_bytes(B, H, T, dk, dv, chunk, dtype);
    if (T > 0 && need > 0) {
        if (!workspace || ws_bytes < need) return MESA_ERR_WORKSPACE;
        if (!aligned(workspace, 256)) return MESA_ERR_INVALID_ARG;
    }
    ForwardArgs a{q, k, v, gamma, beta, lambda, B, H, T, dk, dv, chunk, dtype, cg_steps, tol,
                  out, iters_out, H_in, G_in, H_out, G_out, workspace, ws_bytes};
    a.x0 = T > 0 ? x0 : nullptr;
    a.x_out = T > 0 ? x_out : nullptr;
    return launch_forward(a, static_cast<cudaStream_t>(stream));
}

size_t mesa_forward_preprocessed_workspace_size(int B, int H, int T, int dk, int dv, int chunk,
                                                mesa_dtype dtype) {
    if (check_shape(B, H, T, dk, dv, chunk, dtype, 0, 0.f) != MESA_OK) return 0;
    const size_t fw = workspace_bytes(B, H, T, dk, dv, chunk, dtype);
    if (tc_supported(dk, dv, chunk, dtype)) return fw;          // fused: the forward's own workspace
    return round_up((size_t)B * H * T * dk * elem_size(dtype), 256) * 2 + fw;   // + preprocessed q, k
}

mesa_status mesa_forward_preprocessed(const void* q_raw, const void* k_raw, const void* v,
                                      const float* gamma, const float* beta, const float* lambda,
                                      const float* conv_q, const float* conv_k, int W,
                                      int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype,
                                      int cg_steps, float tol,
                                      float* out, int32_t* iters_out,
                                      const float* H_in, const float* G_in,
                                      float* H_out, float* G_out,
                                      void* workspace, size_t ws_bytes, void* stream) {
    mesa_status s = check_shape(B, H, T, dk, dv, chunk, dtype, cg_steps, tol);
    if (s != MESA_OK) return s;
    if (W < 1 || W > 4 || !conv_q || !conv_k || !aligned(conv_q, 4) || !aligned(conv_k, 4)) return MESA_ERR_INVALID_ARG;
    if (!lambda || !aligned(lambda, 4)) return MESA_ERR_INVALID_ARG;
    if (T > 0) {
        if (!q_raw || !k_raw || !v || !gamma || !beta || !out) return MESA_ERR_INVALID_ARG;
        if (!aligned(q_raw, 16) || !aligned(k_raw, 16) || !aligned(v, 16) || !aligned(out, 16))
            return MESA_ERR_INVALID_ARG;
        if (!aligned(gamma, 4) || !aligned(beta, 4)) return MESA_ERR_INVALID_ARG;
        if (iters_out && !aligned(iters_out, 4)) return MESA_ERR_INVALID_ARG;
    }
    for (const void* p : {(const void*)H_in, (const void*)G_in, (const void*)H_out, (const void*)G_out})
        if (p && !aligned(p, 16)) return MESA_ERR_INVALID_ARG;
    if ((H_out && H_out == H_in) || (G_out && G_out == G_in)) return MESA_ERR_INVALID_ARG;
    const size_t need = mesa_forward_preprocessed_workspace_size(B, H, T, dk, dv, chunk, dtype);
    if (T > 0 && need > 0) {
        if (!workspace || ws_bytes < need) return MESA_ERR_WORKSPACE;
        if (!aligned(workspace, 256)) return MESA_ERR_INVALID_ARG;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    ForwardArgs a{q_raw, k_raw, v, gamma, beta, lambda, B, H, T, dk, dv, chunk, dtype, cg_steps, tol,
                  out, iters_out, H_in, G_in, H_out, G_out, workspace, ws_bytes};
    if (T > 0 && tc_supported(dk, dv, chunk, dtype)) {
        // the scan and the solve convolve and normalise the raw rows as they stage them
        a.conv_q = conv_q;
        a.conv_k = conv_k;
        a.conv_w = W;
        return launch_forward(a, st);
    }
    if (T > 0) {      // the other shapes: preprocessing into the workspace, then the forward
        const size_t qb = round_up((size_t)B * H * T * dk * elem_size(dtype), 256);
        char* w = static_cast<char*>(workspace);
        PreArgs pa{q_raw, k_raw, conv_q, conv_k, B, H, T, dk, W, dtype, w, w + qb};
        if (preprocess_launch(pa, st) != cudaSuccess) return MESA_ERR_CUDA;
        a.q = w;
        a.k = w + qb;
        a.workspace = w + 2 * qb;
        a.ws_bytes = ws_bytes - 2 * qb;
    }
    return launch_forward(a, st);
}

size_t mesa_backward_workspace_size(int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype) {
    if (check_shape(B, H, T, dk, dv, chunk, dtype, 0, 0.f) != MESA_OK) return 0;
    return backward_workspace_bytes(B, H, T, dk, dv, chunk, dtype);
}

mesa_status mesa_backward(const void* q, const void* k, const void* v,
                          const float* gamma, const float* beta, const float* lambda,
                          int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype,
                          int cg_steps, float tol, const float* dout,
                          float* dq, float* dk_out, float* dv_out, float* dgamma, float* dbeta, float* dlambda,
                          void* workspace, size_t ws_bytes, void* stream) {
    mesa_status s = check_shape(B, H, T, dk, dv, chunk, dtype, cg_steps, tol);
    if (s != MESA_OK) return s;
    if (!lambda || !dlambda || !aligned(lambda, 4) || !aligned(dlambda, 4)) return MESA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) return cudaMemsetAsync(dlambda, 0, (size_t)H * dk * sizeof(float), st) == cudaSuccess
                           ? MESA_OK : MESA_ERR_CUDA;
    const void* in16[] = {q, k, v, dout};
    const void* out16[] = {dq, dk_out, dv_out};
    for (const void* p : in16)
        if (!p || !aligned(p, 16)) return MESA_ERR_INVALID_ARG;
    for (const void* p : out16)
        if (!p || !aligned(p, 16)) return MESA_ERR_INVALID_ARG;
    for (const void* p : {(const void*)gamma, (const void*)beta, (const void*)dgamma, (const void*)dbeta})
        if (!p || !aligned(p, 4)) return MESA_ERR_INVALID_ARG;
    // no output may overlap an input or another output
    const size_t tok = (size_t)B * H * T, es = elem_size(dtype);
    struct Range { const char* p; size_t n; };
    const Range ranges[] = {
        {(const char*)q, tok * dk * es}, {(const char*)k, tok * dk * es}, {(const char*)v, tok * dv * es},
        {(const char*)gamma, tok * 4}, {(const char*)beta, tok * 4}, {(const char*)lambda, (size_t)H * dk * 4},
        {(const char*)dout, tok * dv * 4}, {(const char*)dq, tok * dk * 4}, {(const char*)dk_out, tok * dk * 4},
        {(const char*)dv_out, tok * dv * 4}, {(const char*)dgamma, tok * 4}, {(const char*)dbeta, tok * 4},
        {(const char*)dlambda, (size_t)H * dk * 4}};
    constexpr int kFirstOut = 7, kRanges = 13;
    for (int o = kFirstOut; o < kRanges; ++o)
        for (int r = 0; r < kRanges; ++r)
            if (r != o && ranges[o].p < ranges[r].p + ranges[r].n && ranges[r].p < ranges[o].p + ranges[o].n)
                return MESA_ERR_INVALID_ARG;
    const size_t need = backward_workspace_bytes(B, H, T, dk, dv, chunk, dtype);
    if (!workspace || ws_bytes < need) return MESA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return MESA_ERR_INVALID_ARG;
    BackwardArgs a{{q, k, v, gamma, beta, lambda, B, H, T, dk, dv, chunk, dtype, cg_steps, tol, nullptr, nullptr,
                    nullptr, nullptr, nullptr, nullptr, workspace, ws_bytes},
                   dout, dq, dk_out, dv_out, dgamma, dbeta, dlambda};
    return backward_simt(a, st) == cudaSuccess ? MESA_OK : MESA_ERR_CUDA;
}

size_t mesa_chunk_state_workspace_size(int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype) {
    if (check_shape(B, H, T, dk, dv, chunk, dtype, 0, 0.f) != MESA_OK) return 0;
    return workspace_bytes(B, H, T, dk, dv, chunk, dtype);
}

mesa_status mesa_chunk_state(const void* k, const void* v, const float* gamma, const float* beta,
                             int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype,
                             const float* H_in, const float* G_in, float* H_out, float* G_out, float* decay_out,
                             void* workspace, size_t ws_bytes, void* stream) {
    mesa_status s = check_shape(B, H, T, dk, dv, chunk, dtype, 0, 0.f);
    if (s != MESA_OK) return s;
    if (!H_out || !G_out || !decay_out) return MESA_ERR_INVALID_ARG;
    if (!aligned(H_out, 16) || !aligned(G_out, 16) || !aligned(decay_out, 4)) return MESA_ERR_INVALID_ARG;
    for (const void* p : {(const void*)H_in, (const void*)G_in})
        if (p && !aligned(p, 16)) return MESA_ERR_INVALID_ARG;
    if (H_out == H_in || G_out == G_in) return MESA_ERR_INVALID_ARG;
    if (T > 0) {
        if (!k || !v || !gamma || !beta) return MESA_ERR_INVALID_ARG;
        if (!aligned(k, 16) || !aligned(v, 16) || !aligned(gamma, 4) || !aligned(beta, 4)) return MESA_ERR_INVALID_ARG;
        const size_t need = workspace_bytes(B, H, T, dk, dv, chunk, dtype);
        if (!workspace || ws_bytes < need) return MESA_ERR_WORKSPACE;
        if (!aligned(workspace, 256)) return MESA_ERR_INVALID_ARG;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    ForwardArgs a{nullptr, k, v, gamma, beta, nullptr, B, H, T, dk, dv, chunk, dtype, 0, 0.f,
                  nullptr, nullptr, H_in, G_in, H_out, G_out, workspace, ws_bytes};
    if (T == 0) {   // the state passes through unchanged; the decay of an empty slice is 1
        if (launch_forward(a, st) != MESA_OK) return MESA_ERR_CUDA;
    }
    return chunk_state(a, decay_out, st) == cudaSuccess ? MESA_OK : MESA_ERR_CUDA;
}

mesa_status mesa_state_prefix(const float* H_slices, const float* G_slices, const float* decay_slices,
                              int n_slices, int r, int B, int H, int dk, int dv,
                              float* H_in, float* G_in, void* stream) {
    if (B < 1 || H < 1 || n_slices < 0 || r < 0 || r > n_slices) return MESA_ERR_INVALID_ARG;
    if (!supported_width(dk) || dk != dv) return MESA_ERR_UNSUPPORTED;
    if (!H_in || !G_in || !aligned(H_in, 16) || !aligned(G_in, 16)) return MESA_ERR_INVALID_ARG;
    if (r > 0 && (!H_slices || !G_slices || !decay_slices)) return MESA_ERR_INVALID_ARG;
    const size_t BH = (size_t)B * H;
    const size_t nh = BH * dk * dk * 4, ng = BH * dv * dk * 4;
    const char* hi = (const char*)H_in;
    const char* gi = (const char*)G_in;
    if (hi < gi + ng && gi < hi + nh) return MESA_ERR_INVALID_ARG;
    if (r > 0) {
        const struct { const char* p; size_t n; } in[] = {{(const char*)H_slices, nh * n_slices},
                                                          {(const char*)G_slices, ng * n_slices},
                                                          {(const char*)decay_slices, BH * 4 * n_slices}};
        for (const auto& x : in)
            if ((hi < x.p + x.n && x.p < hi + nh) || (gi < x.p + x.n && x.p < gi + ng)) return MESA_ERR_INVALID_ARG;
    }
    return state_prefix(H_slices, G_slices, decay_slices, r, (int)BH, dk, dv, H_in, G_in,
                        static_cast<cudaStream_t>(stream)) == cudaSuccess ? MESA_OK : MESA_ERR_CUDA;
}

size_t mesa_forward_host_workspace_size(int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype) {
    if (check_shape(B, H, T, dk, dv, chunk, dtype, 0, 0.f) != MESA_OK) return 0;
    const size_t tok = (size_t)B * H * T;
    const size_t es = elem_size(dtype);
    // forward scratch: one region per compute stream of the pipeline (each sized
    // for a slice), never more than two slices' worth of the whole batch, plus padding
    size_t n = round_up(workspace_bytes(B, H, T, dk, dv, chunk, dtype), 256) + 2 * 256;
    n += round_up(tok * dk * es, 256) * 2 + round_up(tok * dv * es, 256);      // q, k, v
    n += round_up(tok * 4, 256) * 2 + round_up((size_t)H * dk * 4, 256);      // gamma, beta, lambda
    n += round_up(tok * dv * 4, 256) + round_up(tok * 4, 256);                // out, iters
    n += (round_up((size_t)B * H * dk * dk * 4, 256) + round_up((size_t)B * H * dv * dk * 4, 256)) * 2;
    return n;
}


mesa_status mesa_forward_host(const void* q, const void* k, const void* v,
                              const float* gamma, const float* beta, const float* lambda,
                              int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype,
                              int cg_steps, float tol,
                              float* out, int32_t* iters_out,
                              const float* H_in, const float* G_in,
                              float* H_out, float* G_out,
                              void* workspace, size_t ws_bytes, void* stream) {
    mesa_status s = check_shape(B, H, T, dk, dv, chunk, dtype, cg_steps, tol);
    if (s != MESA_OK) return s;
    if (!lambda) return MESA_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !gamma || !beta || !out)) return MESA_ERR_INVALID_ARG;
    if ((H_out && H_out == H_in) || (G_out && G_out == G_in)) return MESA_ERR_INVALID_ARG;
    const size_t need = mesa_forward_host_workspace_size(B, H, T, dk, dv, chunk, dtype);
    if (!workspace || ws_bytes < need) return MESA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return MESA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    const size_t tok = (size_t)B * H * T;
    const size_t es = elem_size(dtype);
    // slices: with at least kTargetSlices batch rows, groups of whole rows (at
    // most kMaxSlices slices); with fewer, runs of nh heads inside one row (nh
    // halves while it divides evenly, to about kTargetSlices slices); one
    // slice for small or empty problems
    const size_t in_bytes = tok * (2 * dk + dv) * es + tok * 8;
    const bool split = T > 0 && in_bytes >= ((size_t)16 << 20);
    int nslices = 1, Bs = B, Hs_ = H, per_row = 1;
    if (split && B >= kTargetSlices) {
        Bs = (B + kMaxSlices - 1) / kMaxSlices;
        nslices = (B + Bs - 1) / Bs;
    } else if (split) {
        while (Hs_ % 2 == 0 && B * (H / Hs_) < kTargetSlices) Hs_ /= 2;
        per_row = H / Hs_;
        nslices = B * per_row;                         // < 2 kTargetSlices = kMaxSlices
        Bs = 1;
    }
    char* w = static_cast<char*>(workspace);
    const size_t fws_slice = round_up(workspace_bytes(Bs, Hs_, T, dk, dv, chunk, dtype), 256);
    const size_t fws_total = round_up(workspace_bytes(B, H, T, dk, dv, chunk, dtype), 256) + 2 * 256;
    const int ncomp = (nslices > 1 && 2 * fws_slice <= fws_total) ? 2 : 1;   // compute streams
    char* fws[2] = {w, ncomp == 2 ? w + fws_slice : w};
    char* cur = w + fws_total;
    auto carve = [&](size_t bytes) { char* p = cur; cur += round_up(bytes, 256); return p; };
    char* dq = carve(tok * dk * es);
    char* dk_ = carve(tok * dk * es);
    char* dv_ = carve(tok * dv * es);
    float* dg = reinterpret_cast<float*>(carve(tok * 4));
    float* db = reinterpret_cast<float*>(carve(tok * 4));
    float* dl = reinterpret_cast<float*>(carve((size_t)H * dk * 4));
    float* dout = reinterpret_cast<float*>(carve(tok * dv * 4));
    int32_t* dit = reinterpret_cast<int32_t*>(carve(tok * 4));
    const size_t hs = (size_t)dk * dk, gs = (size_t)dv * dk;     // floats per sequence
    float* dHi = reinterpret_cast<float*>(carve((size_t)B * H * hs * 4));
    float* dGi = reinterpret_cast<float*>(carve((size_t)B * H * gs * 4));
    float* dHo = reinterpret_cast<float*>(carve((size_t)B * H * hs * 4));
    float* dGo = reinterpret_cast<float*>(carve((size_t)B * H * gs * 4));

    std::lock_guard<std::mutex> lock(g_pipe_mutex);
    HostPipe* hp = host_pipe();
    if (!hp) return MESA_ERR_CUDA;
    auto cp = [](void* dst, const void* src, size_t bytes, cudaMemcpyKind kind, cudaStream_t sm) {
        return bytes == 0 || cudaMemcpyAsync(dst, src, bytes, kind, sm) == cudaSuccess;
    };
    const cudaMemcpyKind H2D = cudaMemcpyHostToDevice, D2H = cudaMemcpyDeviceToHost;
    bool ok = cudaEventRecord(hp->start, st) == cudaSuccess;       // after the caller's earlier work
    for (cudaStream_t sm : {hp->in, hp->comp[0], hp->comp[1], hp->out})
        ok = ok && cudaStreamWaitEvent(sm, hp->start, 0) == cudaSuccess;
    ok = ok && cp(dl, lambda, (size_t)H * dk * 4, H2D, hp->in);
    // slice i: sequences s0 .. s0+ns-1, run as a forward over nb batch rows of
    // nhs heads starting at head h0 (lambda is offset to h0)
    auto slice = [&](int i, size_t& s0, size_t& ns, int& h0, int& nb, int& nhs) {
        if (per_row > 1) {
            const int b = i / per_row;
            h0 = (i % per_row) * Hs_;
            nb = 1;
            nhs = Hs_;
            s0 = (size_t)b * H + h0;
        } else {
            const int b0 = i * Bs;
            nb = (B - b0 < Bs) ? B - b0 : Bs;
            h0 = 0;
            nhs = H;
            s0 = (size_t)b0 * H;
        }
        ns = (size_t)nb * nhs;
    };
    for (int i = 0; ok && i < nslices; ++i) {
        size_t s0, ns;
        int h0, nb, nhs;
        slice(i, s0, ns, h0, nb, nhs);
        const size_t t0 = s0 * T, nt = ns * T;                        // tokens
        const char* hq = static_cast<const char*>(q);
        const char* hk = static_cast<const char*>(k);
        const char* hv = static_cast<const char*>(v);
        if (T > 0) {
            ok = ok && cp(dq + t0 * dk * es, hq + t0 * dk * es, nt * dk * es, H2D, hp->in);
            ok = ok && cp(dk_ + t0 * dk * es, hk + t0 * dk * es, nt * dk * es, H2D, hp->in);
            ok = ok && cp(dv_ + t0 * dv * es, hv + t0 * dv * es, nt * dv * es, H2D, hp->in);
            ok = ok && cp(dg + t0, gamma + t0, nt * 4, H2D, hp->in) && cp(db + t0, beta + t0, nt * 4, H2D, hp->in);
        }
        if (H_in) ok = ok && cp(dHi + s0 * hs, H_in + s0 * hs, ns * hs * 4, H2D, hp->in);
        if (G_in) ok = ok && cp(dGi + s0 * gs, G_in + s0 * gs, ns * gs * 4, H2D, hp->in);
        ok = ok && cudaEventRecord(hp->landed[i], hp->in) == cudaSuccess;
    }
    for (int i = 0; ok && i < nslices; ++i) {
        size_t s0, ns;
        int h0, nb, nhs;
        slice(i, s0, ns, h0, nb, nhs);
        const size_t t0 = s0 * T;
        cudaStream_t cs = hp->comp[i % ncomp];
        ok = cudaStreamWaitEvent(cs, hp->landed[i], 0) == cudaSuccess;
        if (!ok) break;
        ForwardArgs a{dq + t0 * dk * es, dk_ + t0 * dk * es, dv_ + t0 * dv * es, dg + t0, db + t0, dl + (size_t)h0 * dk,
                      nb, nhs, T, dk, dv, chunk, dtype, cg_steps, tol,
                      dout + t0 * dv, iters_out ? dit + t0 : nullptr,
                      H_in ? dHi + s0 * hs : nullptr, G_in ? dGi + s0 * gs : nullptr,
                      H_out ? dHo + s0 * hs : nullptr, G_out ? dGo + s0 * gs : nullptr,
                      fws[i % ncomp], fws_slice};
        s = launch_forward(a, cs);
        if (s != MESA_OK) {
            ok = false;
            break;
        }
        ok = cudaEventRecord(hp->done[i], cs) == cudaSuccess;
    }
    for (int i = 0; ok && i < nslices; ++i) {
        size_t s0, ns;
        int h0, nb, nhs;
        slice(i, s0, ns, h0, nb, nhs);
        const size_t t0 = s0 * T, nt = ns * T;
        ok = cudaStreamWaitEvent(hp->out, hp->done[i], 0) == cudaSuccess;
        if (T > 0) ok = ok && cp(out + t0 * dv, dout + t0 * dv, nt * dv * 4, D2H, hp->out);
        if (T > 0 && iters_out) ok = ok && cp(iters_out + t0, dit + t0, nt * 4, D2H, hp->out);
        if (H_out) ok = ok && cp(H_out + s0 * hs, dHo + s0 * hs, ns * hs * 4, D2H, hp->out);
        if (G_out) ok = ok && cp(G_out + s0 * gs, dGo + s0 * gs, ns * gs * 4, D2H, hp->out);
    }
    // the caller's stream resumes after the last copy; the call returns once it has landed
    ok = ok && cudaEventRecord(hp->end, hp->out) == cudaSuccess && cudaStreamWaitEvent(st, hp->end, 0) == cudaSuccess;
    if (!ok) {
        // a failure after the first copy was queued: the caller's stream still
        // waits for whatever the pipeline streams hold (copies reading the
        // caller's host buffers, kernels on the workspace), so that an error
        // return keeps the ordering guarantee of a successful call
        for (cudaStream_t sm : {hp->in, hp->comp[0], hp->comp[1], hp->out})
            if (cudaEventRecord(hp->end, sm) == cudaSuccess) cudaStreamWaitEvent(st, hp->end, 0);
    }
    const bool synced = cudaStreamSynchronize(st) == cudaSuccess;
    if (s != MESA_OK) return s;
    return ok && synced ? MESA_OK : MESA_ERR_CUDA;
}

mesa_status mesa_step_warm(const float* q, const float* k, const float* v,
                           const float* gamma, const float* beta, const float* lambda,
                           int B, int H, int dk, int dv,
                           float* Hstate, float* Gstate, float* x_state,
                           int cg_steps, float tol,
                           float* out, int32_t* iters_out, void* stream) {
    if (B < 1 || H < 1 || dk < 1 || dv < 1) return MESA_ERR_INVALID_ARG;
    if (cg_steps < 0 || cg_steps > 1024 || isnan(tol)) return MESA_ERR_INVALID_ARG;
    if (!supported_width(dk) || dk != dv) return MESA_ERR_UNSUPPORTED;
    if ((long long)B * H > 0x7fffffffLL) return MESA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !gamma || !beta || !lambda || !Hstate || !Gstate || !out) return MESA_ERR_INVALID_ARG;
    for (const void* p : {(const void*)q, (const void*)k, (const void*)v, (const void*)Hstate,
                          (const void*)Gstate, (const void*)out})
        if (!aligned(p, 16)) return MESA_ERR_INVALID_ARG;
    if (!aligned(gamma, 4) || !aligned(beta, 4) || !aligned(lambda, 4)) return MESA_ERR_INVALID_ARG;
    if (iters_out && !aligned(iters_out, 4)) return MESA_ERR_INVALID_ARG;
    if (x_state && !aligned(x_state, 4)) return MESA_ERR_INVALID_ARG;
    if (Hstate == Gstate) return MESA_ERR_INVALID_ARG;
    if (x_state && ((const void*)x_state == (const void*)q || x_state == out)) return MESA_ERR_INVALID_ARG;
    StepArgs a{q, k, v, gamma, beta, lambda, B, H, dk, dv, Hstate, Gstate, cg_steps, tol, out, iters_out, x_state};
    return step_launch(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MESA_OK : MESA_ERR_CUDA;
}

mesa_status mesa_step(const float* q, const float* k, const float* v,
                      const float* gamma, const float* beta, const float* lambda,
                      int B, int H, int dk, int dv,
                      float* Hstate, float* Gstate,
                      int cg_steps, float tol,
                      float* out, int32_t* iters_out, void* stream) {
    return mesa_step_warm(q, k, v, gamma, beta, lambda, B, H, dk, dv, Hstate, Gstate, nullptr, cg_steps, tol,
                          out, iters_out, stream);
}

mesa_status mesa_preprocess(const void* q_raw, const void* k_raw, const float* conv_q, const float* conv_k,
                            int B, int H, int T, int d, int W, mesa_dtype dtype, void* q_out, void* k_out,
                            void* stream) {
    if (B < 1 || H < 1 || T < 0 || W < 1 || W > 4) return MESA_ERR_INVALID_ARG;
    if (dtype != MESA_F32 && dtype != MESA_BF16) return MESA_ERR_INVALID_ARG;
    if (!supported_width(d)) return MESA_ERR_UNSUPPORTED;
    if ((long long)B * H > 65535) return MESA_ERR_UNSUPPORTED;                 // grid.y limit
    if (T == 0) return MESA_OK;
    if (!q_raw || !k_raw || !conv_q || !conv_k || !q_out || !k_out) return MESA_ERR_INVALID_ARG;
    for (const void* p : {q_raw, k_raw, (const void*)q_out, (const void*)k_out})
        if (!aligned(p, 16)) return MESA_ERR_INVALID_ARG;
    if (!aligned(conv_q, 4) || !aligned(conv_k, 4)) return MESA_ERR_INVALID_ARG;
    // outputs must not overlap the inputs: rows are read by the warp after their own
    const size_t bytes = (size_t)B * H * T * d * elem_size(dtype);
    auto overlap = [bytes](const void* a, const void* b) {
        const char* x = static_cast<const char*>(a);
        const char* y = static_cast<const char*>(b);
        return x < y + bytes && y < x + bytes;
    };
    if (overlap(q_out, q_raw) || overlap(q_out, k_raw) || overlap(k_out, q_raw) || overlap(k_out, k_raw) ||
        overlap(q_out, k_out))
        return MESA_ERR_INVALID_ARG;
    PreArgs a{q_raw, k_raw, conv_q, conv_k, B, H, T, d, W, dtype, q_out, k_out};
    return preprocess_launch(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MESA_OK : MESA_ERR_CUDA;
}

mesa_status mesa_timing_enable(int on) {
    g_timing_on = on != 0;
    return MESA_OK;
}

int mesa_timing_read(const char** names, int* launches, double* total_ms, int max) {
    int counts[kKindCount] = {0};
    double ms[kKindCount] = {0.0};
    int rc = 0;
    for (const TimingRec& r : g_recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess)
            rc = -1;
        counts[r.kind] += 1;
        ms[r.kind] += t;
        g_event_pool.push_back(r.start);
        g_event_pool.push_back(r.stop);
    }
    g_recs.clear();
    if (rc < 0) return -1;
    int n = 0;
    for (int k = 0; k < kKindCount && n < max; ++k) {
        if (counts[k] == 0) continue;
        if (names) names[n] = kKindNames[k];
        if (launches) launches[n] = counts[k];
        if (total_ms) total_ms[n] = ms[k];
        ++n;
    }
    return n;
}

#ifdef MESA_DEBUG
mesa_status mesa_debug_skip_commit(int launches) {
    if (launches < 0) return MESA_ERR_INVALID_ARG;
    return tc_debug_skip_commit(launches) == cudaSuccess ? MESA_OK : MESA_ERR_CUDA;
}
#endif

mesa_status mesa_get_error(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MESA_ERR_CUDA;
    unsigned w = 0;
    if (cudaMemcpyFromSymbol(&w, g_error_word, sizeof(w)) != cudaSuccess) return MESA_ERR_CUDA;
    if (w == 0) return MESA_OK;
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return MESA_ERR_CUDA;
    return MESA_ERR_DEVICE_TIMEOUT;
}

}  // extern "C"
