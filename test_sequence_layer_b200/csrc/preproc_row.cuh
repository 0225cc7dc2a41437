// preproc_row.cuh -- the per-token arithmetic of the q/k input preprocessing
// ("MesaNet" page, Technical summary > Architecture > "Preprocessing": keys
// and queries are normalised, with a short-window convolution before the Mesa
// layer): a causal depthwise convolution over time, then L2 normalisation of
// the token's row,
//     u_t[i] = sum_{w < W} conv[h][w][i] x_{t-w}[i]     (x = 0 before t = 0)
//     y_t    = u_t / max(|u_t|_2, 1e-6).
// Shared by the standalone preprocessing kernel and by the tensor-core scan
// and solve kernels, which apply it to the raw rows they stage: every path
// performs the same operations in the same order, so all produce the same
// bits. A lane holds eight channels of a row as four fp32 pairs; the LPR
// lanes holding one row are consecutive (a row of D channels spans D / 8).
#pragma once
#include "mesa_common.cuh"

namespace mesa {
namespace pre {

constexpr int kMaxW = 4;     // longest convolution window

// Eight channels of token t: u = c[0] x[0] + c[1] x[1] + c[2] x[2] + c[3] x[3]
// in this order, x[w] the token w steps back and c[w] its weights (zero for
// lags at or past the window, which leave u unchanged for finite x).
__device__ __forceinline__ void conv8(const float2 (&c)[kMaxW][4], const float2 (&x)[kMaxW][4], float2 (&u)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) u[j] = __fmul2_rn(c[0][j], x[0][j]);
#pragma unroll
    for (int w = 1; w < kMaxW; ++w)
#pragma unroll
        for (int j = 0; j < 4; ++j) u[j] = __ffma2_rn(c[w][j], x[w][j], u[j]);
}

// u / max(|u|_2, 1e-6) for the row whose D = 8 LPR channels sit in LPR
// consecutive lanes (a partial sum per lane, then a butterfly over the lanes).
template <int LPR>
__device__ __forceinline__ void norm8(float2 (&u)[4]) {
    float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 4; ++j) ss2 = __ffma2_rn(u[j], u[j], ss2);
    float ss = ss2.x + ss2.y;
#pragma unroll
    for (int off = LPR / 2; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off, LPR);
    const float inv = 1.f / fmaxf(sqrtf(ss), 1e-6f);
    const float2 iv = make_float2(inv, inv);
#pragma unroll
    for (int j = 0; j < 4; ++j) u[j] = __fmul2_rn(u[j], iv);
}

__device__ __forceinline__ void bf16x8_to_f2(uint4 r, float2 (&v)[4]) {
    v[0] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
    v[1] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
    v[2] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.z));
    v[3] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.w));
}

__device__ __forceinline__ uint4 f2_to_bf16x8(const float2 (&v)[4]) {
    uint4 r;
    uint32_t* w = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 b = __float22bfloat162_rn(v[i]);
        w[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    return r;
}

// The weights of eight channels c0..c0+7 for every lag (zero past the window W),
// from a [W][D] array (global or shared memory).
template <int D>
__device__ __forceinline__ void load_weights8(const float* conv, int W, int c0, float2 (&c)[kMaxW][4]) {
#pragma unroll
    for (int w = 0; w < kMaxW; ++w)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            c[w][j] = w < W ? make_float2(conv[w * D + c0 + 2 * j], conv[w * D + c0 + 2 * j + 1]) : make_float2(0.f, 0.f);
}

// One bf16 piece of a preprocessed row (bf16 rows in, bf16 out, as the
// standalone kernel writes them): x[w] are the raw pieces of tokens t-w.
template <int LPR>
__device__ __forceinline__ uint4 conv_norm_bf16x8(const float2 (&c)[kMaxW][4], const uint4 (&x)[kMaxW]) {
    float2 xs[kMaxW][4], u[4];
#pragma unroll
    for (int w = 0; w < kMaxW; ++w) bf16x8_to_f2(x[w], xs[w]);
    conv8(c, xs, u);
    norm8<LPR>(u);
    return f2_to_bf16x8(u);
}

}  // namespace pre
}  // namespace mesa

namespace mesa {
namespace pre {

// conv_norm_bf16x8 with the weights read lag by lag from a zero-padded
// [kMaxW][D] shared-memory array (fewer live registers; the same operations
// in the same order, so the same bits).
template <int D, int LPR>
__device__ __forceinline__ uint4 conv_norm_bf16x8_sw(const float* sw, int c0, const uint4 (&x)[kMaxW]) {
    float2 u[4], xs[4];
    bf16x8_to_f2(x[0], xs);
    {
        const float4 a = *reinterpret_cast<const float4*>(sw + c0), b = *reinterpret_cast<const float4*>(sw + c0 + 4);
        u[0] = __fmul2_rn(make_float2(a.x, a.y), xs[0]);
        u[1] = __fmul2_rn(make_float2(a.z, a.w), xs[1]);
        u[2] = __fmul2_rn(make_float2(b.x, b.y), xs[2]);
        u[3] = __fmul2_rn(make_float2(b.z, b.w), xs[3]);
    }
#pragma unroll
    for (int w = 1; w < kMaxW; ++w) {
        bf16x8_to_f2(x[w], xs);
        const float4 a = *reinterpret_cast<const float4*>(sw + w * D + c0);
        const float4 b = *reinterpret_cast<const float4*>(sw + w * D + c0 + 4);
        u[0] = __ffma2_rn(make_float2(a.x, a.y), xs[0], u[0]);
        u[1] = __ffma2_rn(make_float2(a.z, a.w), xs[1], u[1]);
        u[2] = __ffma2_rn(make_float2(b.x, b.y), xs[2], u[2]);
        u[3] = __ffma2_rn(make_float2(b.z, b.w), xs[3], u[3]);
    }
    norm8<LPR>(u);
    return f2_to_bf16x8(u);
}

// The weights of one head, [W][D] in global memory, into a [kMaxW][D]
// shared-memory array padded with zeros past W (every thread of the block).
template <int D>
__device__ __forceinline__ void stage_weights(const float* conv, int W, float* sw) {
    for (int e = threadIdx.x; e < kMaxW * D; e += blockDim.x) sw[e] = (e / D < W) ? conv[e] : 0.f;
}

}  // namespace pre
}  // namespace mesa
