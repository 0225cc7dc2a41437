// simt_chunk.cuh -- the fp32 CUDA-core building blocks of one chunk that the
// forward (simt_forward.cu) and the backward (simt_backward.cu) share: the
// in-chunk gate cumsum, the shared-memory layout of a chunk, the chunkwise
// matrix-vector product with H_t and the CG iterations on (H_t + Lambda).
//
// Method: "MesaNet: Sequence Modeling by Locally Optimal Test-Time Training"
// (gist.science), Technical summary > Method > Mesa layer and its
// "Parallelisation" paragraph. For chunk c = [t0, t0+C) with chunk-start
// state H_c and in-chunk log-cumsum b_t = sum_{s=t0..t} log gamma_s:
//     H_t p = e^{b_t} H_c p + sum_{j=t0..t} beta_j e^{b_t-b_j} (k_j.p) k_j.
//
// Thread layout (256 threads): thread (tt, ti) = (tid / 16, tid % 16) holds
// rows tt + 16 a (a < CH/16) and columns ti + 16 b (b < D/16) of every
// [CH x D] operand in registers.
#pragma once
#include "mesa_common.cuh"

namespace mesa {
namespace simt {

constexpr int kThreads = 256;

// Inclusive log-cumsum of gamma over one chunk (padded tokens count as
// gamma = 1), done by warp 0. Writes b[t] for t < CH.
template <int CH>
__device__ __forceinline__ void chunk_log_cumsum(const float* __restrict__ gamma, size_t base, int n,
                                                 float* __restrict__ b) {
    static_assert(CH <= 64, "chunk must be <= 64");
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    const int t0 = 2 * lane, t1 = 2 * lane + 1;
    const float l0 = (t0 < n) ? logf(gamma[base + t0]) : 0.f;
    const float l1 = (t1 < n) ? logf(gamma[base + t1]) : 0.f;
    float pair = l0 + l1;
    // inclusive scan of the pair sums across the warp
    float incl = pair;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    const float excl = incl - pair;
    if (t0 < CH) b[t0] = excl + l0;
    if (t1 < CH) b[t1] = excl + l0 + l1;
}

// Sum over the 16 lanes of a half-warp (all 16 receive the total).
__device__ __forceinline__ float sum16(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    return v;
}

// N consecutive floats (N = 1, 2 or 4; the address aligned to N floats).
template <int N>
__device__ __forceinline__ void load_n(const float* p, float (&v)[N]) {
    if constexpr (N == 4) {
        const float4 f = *reinterpret_cast<const float4*>(p);
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    } else if constexpr (N == 2) {
        const float2 f = *reinterpret_cast<const float2*>(p);
        v[0] = f.x; v[1] = f.y;
    } else {
        v[0] = p[0];
    }
}

template <int N>
__device__ __forceinline__ void store_n(float* p, const float (&v)[N]) {
    if constexpr (N == 4) *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    else if constexpr (N == 2) *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
    else p[0] = v[0];
}

// One chunk's contribution to a TL x TL tile of a chunk state: thread
// (ty, tx) = (tid / 16, tid % 16) owns tile rows ty R .. + R - 1 and columns
// tx R .. + R - 1 (R = TL / 16) and forms
//     acc[r][c] = sum_{t < CH} sA[t][ty R + r] * sB[t][tx R + c]
// in order of t, from two [CH][TL + 4] shared tiles (16-byte aligned rows):
// R + R loads per R x R FMAs.
template <int CH, int TL>
__device__ __forceinline__ void tile_outer(const float* sA, const float* sB, float (&acc)[TL / 16][TL / 16]) {
    constexpr int R = TL / 16, TS = TL + 4;
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int c = 0; c < R; ++c) acc[r][c] = 0.f;
#pragma unroll 4
    for (int t = 0; t < CH; ++t) {
        float av[R], bv[R];
        load_n<R>(sA + t * TS + ty * R, av);
        load_n<R>(sB + t * TS + tx * R, bv);
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int c = 0; c < R; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
    }
}

template <int DK, int DV, int CH>
struct CgSmem {
    static constexpr int DKP = DK + 1, DVP = DV + 1, CHP = CH + 1;
    static constexpr int MAXR = DK > DV ? DK : DV;
    static constexpr int oH = 0;                       // H_c, later G_c   [MAXR][DKP]
    static constexpr int oK = oH + MAXR * DKP;         // keys            [CH][DKP]
    static constexpr int oP = oK + CH * DKP;           // CG direction, later x [CH][DKP]
    static constexpr int oV = oP + CH * DKP;           // values          [CH][DVP]
    static constexpr int oW = oV + CH * DVP;           // masked scores   [CH][CHP]
    static constexpr int oM = oW + CH * CHP;           // decay mask      [CH][CHP]
    static constexpr int oE = oM + CH * CHP;           // e^{b_t}         [CH]
    static constexpr int oB = oE + CH;                 // b_t             [CH]
    static constexpr int oL = oB + CH;                 // lambda          [DK]
    static constexpr int total = oL + DK;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

// Masked scores W = M o (A B^T) of two [CH x D] row blocks (row stride DP)
// into sW (row stride CH + 1): W_tj = M_tj (a_t . b_j).
template <int D, int CH>
__device__ __forceinline__ void masked_scores(const float* sA, const float* sB, const float* sM, float* sW) {
    constexpr int TP = CH / 16, JP = CH / 16, DP = D + 1, CHP = CH + 1;
    const int tt = threadIdx.x >> 4, ti = threadIdx.x & 15;
    float s[TP][JP];
#pragma unroll
    for (int a = 0; a < TP; ++a)
#pragma unroll
        for (int b = 0; b < JP; ++b) s[a][b] = 0.f;
#pragma unroll 4
    for (int kk = 0; kk < D; ++kk) {
        float av[TP], bv[JP];
#pragma unroll
        for (int a = 0; a < TP; ++a) av[a] = sA[(tt + 16 * a) * DP + kk];
#pragma unroll
        for (int b = 0; b < JP; ++b) bv[b] = sB[(ti + 16 * b) * DP + kk];
#pragma unroll
        for (int a = 0; a < TP; ++a)
#pragma unroll
            for (int b = 0; b < JP; ++b) s[a][b] = fmaf(av[a], bv[b], s[a][b]);
    }
#pragma unroll
    for (int a = 0; a < TP; ++a)
#pragma unroll
        for (int b = 0; b < JP; ++b) {
            const int t = tt + 16 * a, j = ti + 16 * b;
            sW[t * CHP + j] = sM[t * CHP + j] * s[a][b];
        }
}

// y = e^{b_t} H_c p_t + sum_j M_tj (k_j . p_t) k_j for the rows p_t of sP
// (no Lambda term). sH holds H_c row-major ([i][k], stride DK + 1). Starts
// with the caller's sP complete (a barrier before the call) and ends with
// every thread past its reads of sW; sP, sH, sK are only read.
template <int DK, int CH>
__device__ __forceinline__ void chunk_matvec(const float* sP, const float* sH, const float* sK, float* sW,
                                             const float* sM, const float* sE, float (&y)[CH / 16][DK / 16]) {
    constexpr int TP = CH / 16, IP = DK / 16, DKP = DK + 1, CHP = CH + 1;
    const int tt = threadIdx.x >> 4, ti = threadIdx.x & 15;
    masked_scores<DK, CH>(sP, sK, sM, sW);
    __syncthreads();
#pragma unroll
    for (int a = 0; a < TP; ++a)
#pragma unroll
        for (int b = 0; b < IP; ++b) y[a][b] = 0.f;
#pragma unroll 4
    for (int kk = 0; kk < DK; ++kk) {
        float pv[TP], hv[IP];
#pragma unroll
        for (int a = 0; a < TP; ++a) pv[a] = sP[(tt + 16 * a) * DKP + kk];
#pragma unroll
        for (int b = 0; b < IP; ++b) hv[b] = sH[(ti + 16 * b) * DKP + kk];
#pragma unroll
        for (int a = 0; a < TP; ++a)
#pragma unroll
            for (int b = 0; b < IP; ++b) y[a][b] = fmaf(pv[a], hv[b], y[a][b]);
    }
#pragma unroll
    for (int a = 0; a < TP; ++a) {
        const float e = sE[tt + 16 * a];
#pragma unroll
        for (int b = 0; b < IP; ++b) y[a][b] *= e;
    }
#pragma unroll 4
    for (int jj = 0; jj < CH; ++jj) {
        float wv[TP], kv[IP];
#pragma unroll
        for (int a = 0; a < TP; ++a) wv[a] = sW[(tt + 16 * a) * CHP + jj];
#pragma unroll
        for (int b = 0; b < IP; ++b) kv[b] = sK[jj * DKP + ti + 16 * b];
#pragma unroll
        for (int a = 0; a < TP; ++a)
#pragma unroll
            for (int b = 0; b < IP; ++b) y[a][b] = fmaf(wv[a], kv[b], y[a][b]);
    }
}

// CG on (H_t + Lambda) x_t = rhs_t for the CH rows of the chunk, from x = 0:
// on entry x = 0, r = p = rhs, rr = |rhs|^2, qn = |rhs|, act = (row is a
// token), it = 0, and sP holds p (a barrier after it was written). The rule
// is the library's (mesa.h): stop when |r| <= tol |rhs| (tol > 0), freeze a
// row on breakdown (r.r <= 0, or p.Ap <= 0 or not finite). On return x holds
// the solution, it the update counts.
template <int DK, int CH>
__device__ __forceinline__ void chunk_cg(float* sP, const float* sH, const float* sK, float* sW, const float* sM,
                                         const float* sE, const float* sL, float (&x)[CH / 16][DK / 16],
                                         float (&r)[CH / 16][DK / 16], float (&p)[CH / 16][DK / 16],
                                         float (&rr)[CH / 16], const float (&qn)[CH / 16], bool (&act)[CH / 16],
                                         int (&it)[CH / 16], int cg_steps, float tol) {
    constexpr int TP = CH / 16, IP = DK / 16, DKP = DK + 1;
    const int tt = threadIdx.x >> 4, ti = threadIdx.x & 15;
    float y[TP][IP];
    for (int step = 0; step < cg_steps; ++step) {
        bool any = false;
#pragma unroll
        for (int a = 0; a < TP; ++a) {
            act[a] = act[a] && cg_may_continue(rr[a], qn[a], tol);
            any |= act[a];
        }
        if (!__syncthreads_or(any)) break;
        chunk_matvec<DK, CH>(sP, sH, sK, sW, sM, sE, y);
#pragma unroll
        for (int a = 0; a < TP; ++a) {
            float s = 0.f;
#pragma unroll
            for (int b = 0; b < IP; ++b) {
                y[a][b] = fmaf(sL[ti + 16 * b], p[a][b], y[a][b]);
                s = fmaf(p[a][b], y[a][b], s);
            }
            const float pAp = sum16(s);
            if (act[a] && !cg_curvature_ok(pAp)) act[a] = false;
            float s2 = 0.f;
            if (act[a]) {
                const float alpha = rr[a] / pAp;
#pragma unroll
                for (int b = 0; b < IP; ++b) {
                    x[a][b] = fmaf(alpha, p[a][b], x[a][b]);
                    r[a][b] = fmaf(-alpha, y[a][b], r[a][b]);
                    s2 = fmaf(r[a][b], r[a][b], s2);
                }
            }
            const float rr_new = sum16(s2);
            if (act[a]) {
                const float rho = rr_new / rr[a];
#pragma unroll
                for (int b = 0; b < IP; ++b) p[a][b] = fmaf(rho, p[a][b], r[a][b]);
                rr[a] = rr_new;
                ++it[a];
            }
        }
        __syncthreads();
#pragma unroll
        for (int a = 0; a < TP; ++a)
#pragma unroll
            for (int b = 0; b < IP; ++b) sP[(tt + 16 * a) * DKP + ti + 16 * b] = p[a][b];
        __syncthreads();
    }
}

}  // namespace simt
}  // namespace mesa
