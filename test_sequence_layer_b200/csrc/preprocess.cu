// preprocess.cu -- input preprocessing of queries and keys: a causal
// depthwise convolution over time (window W <= 4), then L2 normalisation of
// every token.
//
// Method: "MesaNet: Sequence Modeling by Locally Optimal Test-Time Training"
// (gist.science), Technical summary > Architecture > "Preprocessing": keys and
// queries are normalised, with a short-window convolution before the Mesa
// layer. Read as the convolution first, so that the layer receives unit-norm
// keys and queries:
//     u_t[i] = sum_{w < W} conv[h][w][i] x_{t-w}[i]   (x = 0 before t = 0)
//     y_t    = u_t / max(|u_t|_2, 1e-6)
//
// The kernel is bound by HBM: every token row of q and k is read once and
// written once. Grid (tiles of kTile tokens, B*H, 2): blockIdx.z picks q or k.
// Each CTA brings its tile and the W-1 rows before it into shared memory with
// one bulk async copy (so the bytes in flight do not cost registers), then
// every row is independent: a row of D channels spans D/8 lanes (8 channels
// each, fp32 pairs in packed FMA), its norm is a shuffle reduction over those
// lanes, and the result is written with 16-byte stores.
#include <cuda_bf16.h>

#include "mesa_common.cuh"
#include "mesa_internal.h"
#include "preproc_row.cuh"
#include "tc_common.cuh"

namespace mesa {
namespace {

constexpr int kPreWarps = 8;
constexpr int kTile = 128;                // tokens per CTA
constexpr int kMaxW = pre::kMaxW;

// Eight channels of one row: fp32 (two 16-byte loads) or bf16 (one).
__device__ __forceinline__ void load8(const float* p, float2 (&v)[4]) {
    const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = make_float2(a.x, a.y); v[1] = make_float2(a.z, a.w);
    v[2] = make_float2(b.x, b.y); v[3] = make_float2(b.z, b.w);
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float2 (&v)[4]) {
    const uint4 r = *reinterpret_cast<const uint4*>(p);
    v[0] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
    v[1] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
    v[2] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.z));
    v[3] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.w));
}
__device__ __forceinline__ void store8(float* p, const float2 (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0].x, v[0].y, v[1].x, v[1].y);
    *reinterpret_cast<float4*>(p + 4) = make_float4(v[2].x, v[2].y, v[3].x, v[3].y);
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float2 (&v)[4]) {
    uint4 r;
    uint32_t* w = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 b = __float22bfloat162_rn(v[i]);
        w[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(p) = r;
}

// Shared-memory row slot: eight channels of a row as fp32 pairs.
__device__ __forceinline__ void lds8(const float* p, float2 (&v)[4]) { load8(p, v); }
__device__ __forceinline__ void lds8(const __nv_bfloat16* p, float2 (&v)[4]) { load8(p, v); }

// CTA: kTile tokens of one sequence, of q (blockIdx.z = 0) or k. Rows
// t0-3 .. t0+kTile-1 arrive by one bulk async copy (rows before the sequence
// start are zero-filled). A row of D channels spans LPR = D/8 lanes, 8
// channels each; lane group g of warp w handles rows w*RPS + g, + kRowStride, ...
template <int D, typename E>
__global__ void __launch_bounds__(32 * kPreWarps)
preprocess_kernel(const E* __restrict__ xq, const E* __restrict__ xk, const float* __restrict__ cq,
                  const float* __restrict__ ck, int H, int T, int W, E* __restrict__ yq, E* __restrict__ yk,
                  unsigned* __restrict__ err) {
    constexpr int LPR = D / 8, RPS = 32 / LPR;
    constexpr int kHalo = kMaxW - 1;
    constexpr uint32_t RB = D * sizeof(E);            // bytes per row
    extern __shared__ __align__(128) uint8_t smem_raw[];
    E* rows = reinterpret_cast<E*>(smem_raw);         // (kHalo + kTile) rows
    __shared__ uint64_t bar;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int grp = lane / LPR, c0 = 8 * (lane % LPR);
    const int bh = blockIdx.y, h = bh % H;
    const bool is_k = blockIdx.z != 0;
    const E* x = (is_k ? xk : xq) + (size_t)bh * T * D;
    E* y = (is_k ? yk : yq) + (size_t)bh * T * D;
    const float* conv = (is_k ? ck : cq) + (size_t)h * W * D;
    const int t0 = blockIdx.x * kTile;
    const int n = min(kTile, T - t0);
    const int lo = max(0, t0 - kHalo);                // first row that exists
    const int skip = lo - (t0 - kHalo);               // halo rows before the sequence start

    if (tid == 0) {
        tc::mbar_init(&bar, 1);
        tc::fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        const uint32_t bytes = (uint32_t)(t0 + n - lo) * RB;
        tc::mbar_arrive_expect_tx(&bar, bytes);
        tc::bulk_g2s(rows + (size_t)skip * D, x + (size_t)lo * D, bytes, &bar);
    }
    for (int e = tid; e < skip * D; e += 32 * kPreWarps) rows[e] = E(0.f);
    float2 c[kMaxW][4];                               // weights by lag, channel pairs
    pre::load_weights8<D>(conv, W, c0, c);
    const bool landed = tc::mbar_wait(&bar, 0);
    __syncthreads();                                  // zero-filled halo rows visible
    if (!landed) {
        if (tid == 0) record_error(err, kErrTimeout);
        return;
    }
    constexpr int kRowStride = kPreWarps * RPS;
#pragma unroll 2
    for (int r = warp * RPS + grp; r < n; r += kRowStride) {
        const E* src = rows + (size_t)(r + kHalo) * D + c0;   // token t0 + r
        float2 u[4], xs[kMaxW][4];
#pragma unroll
        for (int w = 0; w < kMaxW; ++w) lds8(src - (size_t)w * D, xs[w]);
        pre::conv8(c, xs, u);
        pre::norm8<LPR>(u);
        store8(y + (size_t)(t0 + r) * D + c0, u);
    }
}

template <int D, typename E>
cudaError_t launch_pre(const PreArgs& a, cudaStream_t st) {
    const size_t smem = (size_t)(kMaxW - 1 + kTile) * D * sizeof(E);
    auto kern = preprocess_kernel<D, E>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int tiles = (a.T + kTile - 1) / kTile;
    LaunchTimer timer(kKindPre, st);
    kern<<<dim3(tiles, a.B * a.H, 2), 32 * kPreWarps, smem, st>>>(
        static_cast<const E*>(a.xq), static_cast<const E*>(a.xk), a.conv_q, a.conv_k, a.H, a.T, a.W,
        static_cast<E*>(a.yq), static_cast<E*>(a.yk), error_word_ptr());
    return cudaGetLastError();
}

template <typename E>
cudaError_t launch_pre_dtype(const PreArgs& a, cudaStream_t st) {
    switch (a.d) {
        case 16: return launch_pre<16, E>(a, st);
        case 32: return launch_pre<32, E>(a, st);
        case 64: return launch_pre<64, E>(a, st);
        case 128: return launch_pre<128, E>(a, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t preprocess_launch(const PreArgs& a, cudaStream_t st) {
    if (a.T == 0) return cudaSuccess;
    return a.dtype == MESA_BF16 ? launch_pre_dtype<__nv_bfloat16>(a, st) : launch_pre_dtype<float>(a, st);
}

}  // namespace mesa
