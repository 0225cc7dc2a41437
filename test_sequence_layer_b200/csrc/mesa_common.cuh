// mesa_common.cuh -- shared device helpers of the Mesa layer library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mesa.h"

namespace mesa {

// Bits of the per-device error word (read and cleared by mesa_get_error).
enum : unsigned {
    kErrTimeout = 1u,     // a bounded wait ran out of iterations
};

// Kernels that can fail on the device get the address of the calling device's
// error word (api.cu, error_word_ptr()) and OR their failure bits into it.
__device__ __forceinline__ void record_error(unsigned* word, unsigned bits) {
    if (word) atomicOr(word, bits);
}

// Element loads that widen the layer's input types to float.
__device__ __forceinline__ float ld_in(const float* p, size_t i) { return p[i]; }
__device__ __forceinline__ float ld_in(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }

// CG stopping/breakdown rule shared by every kernel (see mesa.h):
// a token keeps iterating while this holds.
__device__ __forceinline__ bool cg_may_continue(float rr, float qnorm, float tol) {
    if (!(rr > 0.f)) return false;
    if (tol > 0.f && sqrtf(rr) <= tol * qnorm) return false;
    return true;
}

__device__ __forceinline__ bool cg_curvature_ok(float pAp) { return pAp > 0.f && isfinite(pAp); }

}  // namespace mesa
