// noalloc.cu -- mesa_forward_noalloc: the chunkwise forward with its scratch
// taken from a fixed, library-owned device array instead of a caller-supplied
// workspace.
//
// Who needs this: callers that cannot allocate device memory at all, e.g.
// plug-in code running inside a host framework that owns every device
// allocation and hands out only the tensors it passes in, or latency-bound
// loops that must never call cudaMalloc (which can synchronise the device).
// Such callers cannot provide the workspace mesa_forward asks for.
//
// The scratch lives in kScratchBytes of file-scope device memory. Every GPU
// that loads this library holds that memory until the process exits. All
// calls on a device share it and it keeps the last call's contents: the
// forward writes every byte it later reads (chunk-start states and their
// scales), so nothing needs clearing between calls; calls that overlap on the
// GPU (other streams, or host threads, without ordering) race on it.
#include <atomic>

#include "mesa_common.cuh"
#include "mesa_internal.h"

namespace mesa {
namespace {

constexpr size_t kScratchBytes = MESA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDev = 64;
std::atomic<void*> g_scratch_addr[kMaxDev];

// Device address of the scratch array on the current device. Looked up once
// per device, in the device's primary context (the runtime API's context; the
// host-side name of the array is only a stand-in, never a device address).
// Host threads that race on the first call each store the same address, so
// the cached value is written atomically and read without a lock. Returns
// nullptr if the lookup fails.
void* scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
    void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
        g_scratch_addr[dev].store(p, std::memory_order_release);
    }
    return p;
}

}  // namespace
}  // namespace mesa

extern "C" mesa_status mesa_forward_noalloc(const void* q, const void* k, const void* v,
                                            const float* gamma, const float* beta, const float* lambda,
                                            int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype,
                                            int cg_steps, float tol,
                                            float* out, int32_t* iters_out,
                                            const float* H_in, const float* G_in,
                                            float* H_out, float* G_out, void* stream) {
    // Sizes first: a shape whose scratch exceeds the fixed array is refused
    // before anything touches the device.
    const size_t need = mesa_forward_workspace_size(B, H, T, dk, dv, chunk, dtype);
    if (need > mesa::kScratchBytes) return MESA_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (need > 0) {           // zero: invalid or unsupported sizes, or T = 0 (mesa_forward sorts these out)
        scratch = mesa::scratch_address();
        if (!scratch) return MESA_ERR_CUDA;
    }
    return mesa_forward(q, k, v, gamma, beta, lambda, B, H, T, dk, dv, chunk, dtype, cg_steps, tol, out,
                        iters_out, H_in, G_in, H_out, G_out, scratch, scratch ? mesa::kScratchBytes : 0, stream);
}
