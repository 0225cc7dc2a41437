// tc_layout.cuh -- what the tensor-core scan (tc_scan.cu) and the
// tensor-core solve (tc_forward.cu) share: the head size and chunk length
// they are built for, the fp16 state-image format and the scaling helpers.
//
// State image: the state before a 128-token block of one sequence as fp16
// values divided by a power-of-two scale s >= 1 stored beside it: H with
// rows i and columns l, G transposed (row l, column i holds G[i][l]), both
// 128 x 128. Two 64-column blocks of 16 KB; row i of a
// block is 128 bytes whose 16-byte units (8 columns each) are permuted by
// XOR with (i & 7): the K-major 128-byte-swizzle layout that tcgen05.mma
// reads, so the solve loads an image with one bulk copy. Images of sequence
// bh, block p (np blocks per sequence): H at image_index(bh, np, p, 0), G at
// image_index(bh, np, p, 1); scales use the same index.
#pragma once
#include "mesa_common.cuh"
#include "tc_common.cuh"

namespace mesa {
namespace tc {

constexpr int kD = 128;          // dk = dv
constexpr int kC = 64;           // chunk length
constexpr uint32_t kImgBytes = kD * kD * 2;      // one fp16 state image
constexpr size_t kImgHalves = (size_t)kD * kD;

// The smallest power of two >= m, for a bound m >= 0 on the magnitudes a
// tensor-core operand is divided by before it is rounded to fp16 (so the
// operand's entries lie in [-1, 1], inside fp16's normal range down to 2^-14
// of its largest entry). The exponent is kept in [-120, 126] so that the
// scale and its reciprocal are normal floats; m = 0 (an all-zero operand) or
// a non-finite m gives 1.
__device__ __forceinline__ float pow2_ceil(float m) {
    if (!(m > 0.f) || !(m <= 3.0e38f)) return 1.f;
    const uint32_t b = __float_as_uint(m);
    int e = (int)((b >> 23) & 0xffu) - 127 + ((b & 0x7fffffu) ? 1 : 0);
    e = max(-120, min(126, e));
    return __uint_as_float((uint32_t)(e + 127) << 23);
}

// Power of two 2^floor(e/2) with 2^e <= rr < 2^(e+1): a scale within a factor
// sqrt(2) of |r| whose reciprocal is exact (1 for rr <= 0 or denormal rr).
__device__ __forceinline__ float pow2_sqrt_scale(float rr) {
    const int e = ((__float_as_int(rr) >> 23) & 0xff) - 127;
    if (!(rr > 0.f) || e <= -126 || e >= 127) return 1.f;
    return __int_as_float((((e >> 1) + 127) & 0xff) << 23);
}

__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 raw, float scale) {
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&raw);
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(b[i]);
        ow[i] = pack_half2(f.x * scale, f.y * scale);
    }
    return o;
}

__host__ __device__ __forceinline__ size_t image_index(int bh, int np, int p, int m) {
    return ((size_t)bh * np + p) * 2 + m;
}

}  // namespace tc
}  // namespace mesa
