// simt_forward.cu -- fp32 CUDA-core chunkwise forward of the Mesa layer.
//
// Serves the fp32 mode (and every shape the tensor-core path does not take):
// the statistics, the CG vectors and every product stay in fp32 so the result
// tracks the fp64 definition to ~1e-5 relative.
//
// Method: "MesaNet: Sequence Modeling by Locally Optimal Test-Time Training"
// (gist.science), Technical summary > Method > Mesa layer, and its
// "Parallelisation" paragraph: the CG matvec (H_t + Lambda) p of every token
// of a chunk is evaluated as gated linear attention, i.e. for chunk
// c = [t0, t0+C) with chunk-start state H_c and in-chunk log-cumsum
// b_t = sum_{s=t0..t} log gamma_s:
//     H_t p = e^{b_t} H_c p + sum_{j=t0..t} beta_j e^{b_t-b_j} (k_j.p) k_j
// and the read-out G_t x = e^{b_t} G_c x + sum_{j<=t} beta_j e^{b_t-b_j} (k_j.x) v_j.
// The chunk-start states follow H_{c+1} = e^{b_last} H_c + sum_j beta_j
// e^{b_last-b_j} k_j k_j^T (same for G).
//
// Kernels:
//   simt_scan_kernel  grid (state tiles, B*H): one CTA walks the chunks of one
//                     sequence for one 64x64 (d < 64: d x d) tile of H or G, each
//                     thread a 4x4 block of it (1x1, 2x2 for d = 16, 32), writing
//                     the chunk-start states to the workspace.
//   simt_cg_kernel    grid (chunks, B*H): one CTA runs all CG iterations of one
//                     chunk with H_c, K, V, P and the decay mask in shared
//                     memory, then the read-out.
#include "mesa_internal.h"
#include "simt_chunk.cuh"

namespace mesa {
namespace {

using namespace simt;

template <int DK, int DV, int CH, typename Tin>
__global__ void __launch_bounds__(kThreads)
simt_scan_kernel(const Tin* __restrict__ k, const Tin* __restrict__ v,
                 const float* __restrict__ gamma, const float* __restrict__ beta,
                 int T, int nc, const float* __restrict__ H_in, const float* __restrict__ G_in,
                 float* __restrict__ states, float* __restrict__ H_out, float* __restrict__ G_out) {
    static_assert(DK == DV, "dk == dv");
    constexpr int TL = DK < 64 ? DK : 64;                  // tile edge
    constexpr int R = TL / 16;                             // each thread: R x R elements of the tile
    constexpr int TS = TL + 4;                             // shared row stride (16-byte rows)
    constexpr int TPR = DK / TL;                           // tiles per row of a matrix
    constexpr int H_TILES = TPR * TPR;
    constexpr size_t SE = (size_t)DK * DK + (size_t)DV * DK;

    __shared__ __align__(16) float sA[CH * TS];
    __shared__ __align__(16) float sKc[CH * TS];
    __shared__ float sb[CH];
    __shared__ float sw[CH];

    const int bh = blockIdx.y;
    int tile = blockIdx.x;
    const bool isG = tile >= H_TILES;
    if (isG) tile -= H_TILES;
    const int i0 = (tile / TPR) * TL + (threadIdx.x >> 4) * R;   // this thread's first row ...
    const int j0 = (tile % TPR) * TL + (threadIdx.x & 15) * R;   // ... and column in the matrix
    const int tcol = (tile % TPR) * TL, trow = (tile / TPR) * TL;
    const Tin* A = isG ? v : k;
    const size_t mat_off = isG ? (size_t)DK * DK : 0;
    const float* init = isG ? G_in : H_in;
    float* fin = isG ? G_out : H_out;

    float S[R][R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int c = 0; c < R; ++c)
            S[r][c] = init ? init[(size_t)bh * DK * DK + (size_t)(i0 + r) * DK + j0 + c] : 0.f;
    }

    for (int c = 0; c < nc; ++c) {
        const int t0 = c * CH;
        const int n = min(CH, T - t0);
        const size_t base = (size_t)bh * T + t0;
        float* dst = states + ((size_t)bh * nc + c) * SE + mat_off;
#pragma unroll
        for (int r = 0; r < R; ++r) store_n<R>(dst + (size_t)(i0 + r) * DK + j0, S[r]);
        chunk_log_cumsum<CH>(gamma, base, n, sb);
        __syncthreads();
        const float blast = sb[CH - 1];
        for (int t = threadIdx.x; t < CH; t += kThreads)
            sw[t] = (t < n) ? beta[base + t] * expf(blast - sb[t]) : 0.f;
        __syncthreads();
        for (int idx = threadIdx.x; idx < CH * TL; idx += kThreads) {
            const int t = idx / TL, col = idx % TL;
            const bool ok = t < n;
            sA[t * TS + col] = ok ? sw[t] * ld_in(A, (base + t) * DK + trow + col) : 0.f;
            sKc[t * TS + col] = ok ? ld_in(k, (base + t) * DK + tcol + col) : 0.f;
        }
        __syncthreads();
        const float Gam = expf(blast);
        float acc[R][R];
        tile_outer<CH, TL>(sA, sKc, acc);
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int cc = 0; cc < R; ++cc) S[r][cc] = fmaf(Gam, S[r][cc], acc[r][cc]);
        __syncthreads();
    }
    if (fin) {
#pragma unroll
        for (int r = 0; r < R; ++r) store_n<R>(fin + (size_t)bh * DK * DK + (size_t)(i0 + r) * DK + j0, S[r]);
    }
}

template <int DK, int DV, int CH, typename Tin>
__global__ void __launch_bounds__(kThreads, 1)
simt_cg_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
               const float* __restrict__ gamma, const float* __restrict__ beta,
               const float* __restrict__ lambda, int H, int T, int nc, int cg_steps, float tol,
               const float* __restrict__ states, float* __restrict__ out, int32_t* __restrict__ iters,
               float* __restrict__ x_out, const float* __restrict__ x0) {
    static_assert(DK % 16 == 0 && DV % 16 == 0 && CH % 16 == 0, "multiples of 16");
    using L = CgSmem<DK, DV, CH>;
    constexpr int TP = CH / 16, IP = DK / 16, VP = DV / 16;
    constexpr int DKP = L::DKP, DVP = L::DVP, CHP = L::CHP;
    constexpr size_t SE = (size_t)DK * DK + (size_t)DV * DK;
    extern __shared__ float smem[];
    float* sH = smem + L::oH;
    float* sK = smem + L::oK;
    float* sP = smem + L::oP;
    float* sV = smem + L::oV;
    float* sW = smem + L::oW;
    float* sM = smem + L::oM;
    float* sE = smem + L::oE;
    float* sB = smem + L::oB;
    float* sL = smem + L::oL;

    const int c = blockIdx.x, bh = blockIdx.y, h = bh % H;
    const int t0 = c * CH;
    const int n = min(CH, T - t0);
    const size_t base = (size_t)bh * T + t0;
    const int tid = threadIdx.x, tt = tid >> 4, ti = tid & 15;
    const float* Hc = states + ((size_t)bh * nc + c) * SE;
    const float* Gc = Hc + (size_t)DK * DK;

    // ---- stage the chunk: H_c, K, V, lambda, gates, decay mask ----
    for (int e = tid; e < DK * DK; e += kThreads) sH[(e / DK) * DKP + e % DK] = Hc[e];
    for (int e = tid; e < CH * DK; e += kThreads) {
        const int t = e / DK, d = e % DK;
        sK[t * DKP + d] = (t < n) ? ld_in(k, (base + t) * DK + d) : 0.f;
    }
    for (int e = tid; e < CH * DV; e += kThreads) {
        const int t = e / DV, d = e % DV;
        sV[t * DVP + d] = (t < n) ? ld_in(v, (base + t) * DV + d) : 0.f;
    }
    for (int d = tid; d < DK; d += kThreads) sL[d] = lambda[(size_t)h * DK + d];
    chunk_log_cumsum<CH>(gamma, base, n, sB);
    __syncthreads();
    for (int t = tid; t < CH; t += kThreads) sE[t] = expf(sB[t]);
    for (int e = tid; e < CH * CH; e += kThreads) {
        const int t = e / CH, j = e % CH;
        sM[t * CHP + j] = (j <= t && t < n) ? beta[base + j] * expf(sB[t] - sB[j]) : 0.f;
    }

    // ---- CG init: x = 0, r = p = q ----
    float x[TP][IP], r[TP][IP], p[TP][IP];
    float rr[TP], qn[TP];
    bool act[TP];
    int it[TP];
#pragma unroll
    for (int a = 0; a < TP; ++a) {
        const int t = tt + 16 * a;
        float s = 0.f;
#pragma unroll
        for (int b = 0; b < IP; ++b) {
            const int i = ti + 16 * b;
            const float qv = (t < n) ? ld_in(q, (base + t) * DK + i) : 0.f;
            x[a][b] = 0.f;
            r[a][b] = qv;
            p[a][b] = qv;
            sP[t * DKP + i] = qv;
            s = fmaf(qv, qv, s);
        }
        rr[a] = sum16(s);
        qn[a] = sqrtf(rr[a]);
        act[a] = t < n;
        it[a] = 0;
    }
    __syncthreads();
    if (x0) {
        // warm start: x = x0, r = p = q - (H_t + Lambda) x0 (one more matvec);
        // the stopping test stays relative to |q|
#pragma unroll
        for (int a = 0; a < TP; ++a) {
            const int t = tt + 16 * a;
#pragma unroll
            for (int b = 0; b < IP; ++b) {
                const int i = ti + 16 * b;
                x[a][b] = (t < n) ? x0[(base + t) * DK + i] : 0.f;
                sP[t * DKP + i] = x[a][b];
            }
        }
        __syncthreads();
        float y[TP][IP];
        chunk_matvec<DK, CH>(sP, sH, sK, sW, sM, sE, y);
#pragma unroll
        for (int a = 0; a < TP; ++a) {
            const int t = tt + 16 * a;
            float s = 0.f;
#pragma unroll
            for (int b = 0; b < IP; ++b) {
                r[a][b] = r[a][b] - fmaf(sL[ti + 16 * b], x[a][b], y[a][b]);
                p[a][b] = r[a][b];
                s = fmaf(r[a][b], r[a][b], s);
            }
            rr[a] = sum16(s);
            if (!(t < n)) rr[a] = 0.f;
        }
        __syncthreads();                                 // every thread past its reads of sP
#pragma unroll
        for (int a = 0; a < TP; ++a)
#pragma unroll
            for (int b = 0; b < IP; ++b) sP[(tt + 16 * a) * DKP + ti + 16 * b] = p[a][b];
        __syncthreads();
    }

    chunk_cg<DK, CH>(sP, sH, sK, sW, sM, sE, sL, x, r, p, rr, qn, act, it, cg_steps, tol);

    // ---- the solution, if asked for, then the read-out o = e^{b_t} G_c x + (M (.) X K^T) V ----
    if (x_out) {
#pragma unroll
        for (int a = 0; a < TP; ++a) {
            const int t = tt + 16 * a;
            if (t < n) {
#pragma unroll
                for (int b = 0; b < IP; ++b) x_out[(base + t) * DK + ti + 16 * b] = x[a][b];
            }
        }
    }
    if (!out) {
        if (iters) {
#pragma unroll
            for (int a = 0; a < TP; ++a) {
                const int t = tt + 16 * a;
                if (t < n && ti == 0) iters[base + t] = it[a];
            }
        }
        return;
    }
    __syncthreads();
#pragma unroll
    for (int a = 0; a < TP; ++a)
#pragma unroll
        for (int b = 0; b < IP; ++b) sP[(tt + 16 * a) * DKP + ti + 16 * b] = x[a][b];
    for (int e = tid; e < DV * DK; e += kThreads) sH[(e / DK) * DKP + e % DK] = Gc[e];
    __syncthreads();
    masked_scores<DK, CH>(sP, sK, sM, sW);
    __syncthreads();
    float o[TP][VP];
#pragma unroll
    for (int a = 0; a < TP; ++a)
#pragma unroll
        for (int b = 0; b < VP; ++b) o[a][b] = 0.f;
#pragma unroll 4
    for (int kk = 0; kk < DK; ++kk) {
        float xv[TP], gv[VP];
#pragma unroll
        for (int a = 0; a < TP; ++a) xv[a] = sP[(tt + 16 * a) * DKP + kk];
#pragma unroll
        for (int b = 0; b < VP; ++b) gv[b] = sH[(ti + 16 * b) * DKP + kk];
#pragma unroll
        for (int a = 0; a < TP; ++a)
#pragma unroll
            for (int b = 0; b < VP; ++b) o[a][b] = fmaf(xv[a], gv[b], o[a][b]);
    }
#pragma unroll
    for (int a = 0; a < TP; ++a) {
        const float e = sE[tt + 16 * a];
#pragma unroll
        for (int b = 0; b < VP; ++b) o[a][b] *= e;
    }
#pragma unroll 4
    for (int jj = 0; jj < CH; ++jj) {
        float wv[TP], vv[VP];
#pragma unroll
        for (int a = 0; a < TP; ++a) wv[a] = sW[(tt + 16 * a) * CHP + jj];
#pragma unroll
        for (int b = 0; b < VP; ++b) vv[b] = sV[jj * DVP + ti + 16 * b];
#pragma unroll
        for (int a = 0; a < TP; ++a)
#pragma unroll
            for (int b = 0; b < VP; ++b) o[a][b] = fmaf(wv[a], vv[b], o[a][b]);
    }
#pragma unroll
    for (int a = 0; a < TP; ++a) {
        const int t = tt + 16 * a;
        if (t < n) {
#pragma unroll
            for (int b = 0; b < VP; ++b) out[(base + t) * DV + ti + 16 * b] = o[a][b];
            if (iters && ti == 0) iters[base + t] = it[a];
        }
    }
}

template <int D, int CH, typename Tin>
cudaError_t launch_simt(const ForwardArgs& a, cudaStream_t st) {
    const int nc = (a.T + CH - 1) / CH;
    const int BH = a.B * a.H;
    float* states = reinterpret_cast<float*>(a.workspace);
    constexpr int TL = D < 64 ? D : 64;
    constexpr int tiles = 2 * (D / TL) * (D / TL);
    {
        LaunchTimer timer(kKindSimtScan, st);
        simt_scan_kernel<D, D, CH, Tin><<<dim3(tiles, BH), kThreads, 0, st>>>(
            static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.v), a.gamma, a.beta, a.T, nc,
            a.H_in, a.G_in, states, a.H_out, a.G_out);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || a.scan_only) return e;
    using L = CgSmem<D, D, CH>;
    auto kern = simt_cg_kernel<D, D, CH, Tin>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
    if (e != cudaSuccess) return e;
    {
        LaunchTimer timer(kKindSimtCg, st);
        kern<<<dim3(nc, BH), kThreads, L::bytes, st>>>(
            static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.v),
            a.gamma, a.beta, a.lambda, a.H, a.T, nc, a.cg_steps, a.tol, states, a.out, a.iters, a.x_out, a.x0);
    }
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t dispatch_simt(const ForwardArgs& a, cudaStream_t st) {
#define MESA_SIMT_CASE(D_, C_) \
    if (a.dk == D_ && a.chunk == C_) return launch_simt<D_, C_, Tin>(a, st);
    MESA_SIMT_CASE(16, 16) MESA_SIMT_CASE(16, 32) MESA_SIMT_CASE(16, 64)
    MESA_SIMT_CASE(32, 16) MESA_SIMT_CASE(32, 32) MESA_SIMT_CASE(32, 64)
    MESA_SIMT_CASE(64, 16) MESA_SIMT_CASE(64, 32) MESA_SIMT_CASE(64, 64)
    MESA_SIMT_CASE(128, 16) MESA_SIMT_CASE(128, 32) MESA_SIMT_CASE(128, 64)
#undef MESA_SIMT_CASE
    return cudaErrorInvalidValue;
}

}  // namespace

size_t simt_workspace_bytes(int B, int H, int T, int dk, int dv, int chunk) {
    const size_t nc = (size_t)((T + chunk - 1) / chunk);
    return (size_t)B * H * nc * ((size_t)dk * dk + (size_t)dv * dk) * sizeof(float);
}

cudaError_t forward_simt(const ForwardArgs& a, cudaStream_t st) {
    return a.dtype == MESA_BF16 ? dispatch_simt<__nv_bfloat16>(a, st) : dispatch_simt<float>(a, st);
}

}  // namespace mesa
