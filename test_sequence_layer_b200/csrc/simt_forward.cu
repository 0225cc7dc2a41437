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
//                     sequence for one 32x32 (or 16x16) tile of H or G, writing
//                     the chunk-start states to the workspace.
//   simt_cg_kernel    grid (chunks, B*H): one CTA runs all CG iterations of one
//                     chunk with H_c, K, V, P and the decay mask in shared
//                     memory, then the read-out.
#include "mesa_common.cuh"
#include "mesa_internal.h"

namespace mesa {
namespace {

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

template <int DK, int DV, int CH, typename Tin>
__global__ void __launch_bounds__(kThreads)
simt_scan_kernel(const Tin* __restrict__ k, const Tin* __restrict__ v,
                 const float* __restrict__ gamma, const float* __restrict__ beta,
                 int T, int nc, const float* __restrict__ H_in, const float* __restrict__ G_in,
                 float* __restrict__ states, float* __restrict__ H_out, float* __restrict__ G_out) {
    static_assert(DK == DV, "dk == dv");
    constexpr int TL = DK < 32 ? DK : 32;                  // tile edge
    constexpr int TPR = DK / TL;                           // tiles per row of a matrix
    constexpr int H_TILES = TPR * TPR;
    constexpr int EPT = (TL * TL + kThreads - 1) / kThreads;
    constexpr size_t SE = (size_t)DK * DK + (size_t)DV * DK;

    __shared__ float sA[CH][TL + 1];
    __shared__ float sKc[CH][TL + 1];
    __shared__ float sb[CH];
    __shared__ float sw[CH];

    const int bh = blockIdx.y;
    int tile = blockIdx.x;
    const bool isG = tile >= H_TILES;
    if (isG) tile -= H_TILES;
    const int i0 = (tile / TPR) * TL, j0 = (tile % TPR) * TL;
    const Tin* A = isG ? v : k;
    const size_t mat_off = isG ? (size_t)DK * DK : 0;
    const float* init = isG ? G_in : H_in;
    float* fin = isG ? G_out : H_out;

    float S[EPT];
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
        const int idx = threadIdx.x + kThreads * e;
        S[e] = 0.f;
        if (idx < TL * TL && init) S[e] = init[(size_t)bh * DK * DK + (size_t)(i0 + idx / TL) * DK + j0 + idx % TL];
    }

    for (int c = 0; c < nc; ++c) {
        const int t0 = c * CH;
        const int n = min(CH, T - t0);
        const size_t base = (size_t)bh * T + t0;
        float* dst = states + ((size_t)bh * nc + c) * SE + mat_off;
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
            const int idx = threadIdx.x + kThreads * e;
            if (idx < TL * TL) dst[(size_t)(i0 + idx / TL) * DK + j0 + idx % TL] = S[e];
        }
        chunk_log_cumsum<CH>(gamma, base, n, sb);
        __syncthreads();
        const float blast = sb[CH - 1];
        for (int t = threadIdx.x; t < CH; t += kThreads)
            sw[t] = (t < n) ? beta[base + t] * expf(blast - sb[t]) : 0.f;
        __syncthreads();
        for (int idx = threadIdx.x; idx < CH * TL; idx += kThreads) {
            const int t = idx / TL, col = idx % TL;
            const bool ok = t < n;
            sA[t][col] = ok ? sw[t] * ld_in(A, (base + t) * DK + i0 + col) : 0.f;
            sKc[t][col] = ok ? ld_in(k, (base + t) * DK + j0 + col) : 0.f;
        }
        __syncthreads();
        const float Gam = expf(blast);
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
            const int idx = threadIdx.x + kThreads * e;
            if (idx < TL * TL) {
                const int i = idx / TL, j = idx % TL;
                float acc = 0.f;
#pragma unroll 8
                for (int t = 0; t < CH; ++t) acc = fmaf(sA[t][i], sKc[t][j], acc);
                S[e] = fmaf(Gam, S[e], acc);
            }
        }
        __syncthreads();
    }
    if (fin) {
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
            const int idx = threadIdx.x + kThreads * e;
            if (idx < TL * TL) fin[(size_t)bh * DK * DK + (size_t)(i0 + idx / TL) * DK + j0 + idx % TL] = S[e];
        }
    }
}

// Sum over the 16 lanes of a half-warp (all 16 receive the total).
__device__ __forceinline__ float sum16(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    return v;
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

template <int DK, int DV, int CH, typename Tin>
__global__ void __launch_bounds__(kThreads, 1)
simt_cg_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
               const float* __restrict__ gamma, const float* __restrict__ beta,
               const float* __restrict__ lambda, int H, int T, int nc, int cg_steps, float tol,
               const float* __restrict__ states, float* __restrict__ out, int32_t* __restrict__ iters) {
    static_assert(DK % 16 == 0 && DV % 16 == 0 && CH % 16 == 0, "multiples of 16");
    using L = CgSmem<DK, DV, CH>;
    constexpr int TP = CH / 16, IP = DK / 16, VP = DV / 16, JP = CH / 16;
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
    float x[TP][IP], r[TP][IP], p[TP][IP], y[TP][IP];
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

    for (int step = 0; step < cg_steps; ++step) {
        bool any = false;
#pragma unroll
        for (int a = 0; a < TP; ++a) {
            act[a] = act[a] && cg_may_continue(rr[a], qn[a], tol);
            any |= act[a];
        }
        if (!__syncthreads_or(any)) break;

        // S = P K^T, W = M (.) S
        {
            float s[TP][JP];
#pragma unroll
            for (int a = 0; a < TP; ++a)
#pragma unroll
                for (int b = 0; b < JP; ++b) s[a][b] = 0.f;
#pragma unroll 4
            for (int kk = 0; kk < DK; ++kk) {
                float pv[TP], kv[JP];
#pragma unroll
                for (int a = 0; a < TP; ++a) pv[a] = sP[(tt + 16 * a) * DKP + kk];
#pragma unroll
                for (int b = 0; b < JP; ++b) kv[b] = sK[(ti + 16 * b) * DKP + kk];
#pragma unroll
                for (int a = 0; a < TP; ++a)
#pragma unroll
                    for (int b = 0; b < JP; ++b) s[a][b] = fmaf(pv[a], kv[b], s[a][b]);
            }
#pragma unroll
            for (int a = 0; a < TP; ++a)
#pragma unroll
                for (int b = 0; b < JP; ++b) {
                    const int t = tt + 16 * a, j = ti + 16 * b;
                    sW[t * CHP + j] = sM[t * CHP + j] * s[a][b];
                }
        }
        __syncthreads();

        // y = e^{b_t} H_c p + W K + lambda p
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

        // CG update
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

    // ---- read-out: o = e^{b_t} G_c x + (M (.) X K^T) V ----
    __syncthreads();
#pragma unroll
    for (int a = 0; a < TP; ++a)
#pragma unroll
        for (int b = 0; b < IP; ++b) sP[(tt + 16 * a) * DKP + ti + 16 * b] = x[a][b];
    for (int e = tid; e < DV * DK; e += kThreads) sH[(e / DK) * DKP + e % DK] = Gc[e];
    __syncthreads();
    {
        float s[TP][JP];
#pragma unroll
        for (int a = 0; a < TP; ++a)
#pragma unroll
            for (int b = 0; b < JP; ++b) s[a][b] = 0.f;
#pragma unroll 4
        for (int kk = 0; kk < DK; ++kk) {
            float pv[TP], kv[JP];
#pragma unroll
            for (int a = 0; a < TP; ++a) pv[a] = sP[(tt + 16 * a) * DKP + kk];
#pragma unroll
            for (int b = 0; b < JP; ++b) kv[b] = sK[(ti + 16 * b) * DKP + kk];
#pragma unroll
            for (int a = 0; a < TP; ++a)
#pragma unroll
                for (int b = 0; b < JP; ++b) s[a][b] = fmaf(pv[a], kv[b], s[a][b]);
        }
#pragma unroll
        for (int a = 0; a < TP; ++a)
#pragma unroll
            for (int b = 0; b < JP; ++b) {
                const int t = tt + 16 * a, j = ti + 16 * b;
                sW[t * CHP + j] = sM[t * CHP + j] * s[a][b];
            }
    }
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
    constexpr int TL = D < 32 ? D : 32;
    constexpr int tiles = 2 * (D / TL) * (D / TL);
    {
        LaunchTimer timer(kKindSimtScan, st);
        simt_scan_kernel<D, D, CH, Tin><<<dim3(tiles, BH), kThreads, 0, st>>>(
            static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.v), a.gamma, a.beta, a.T, nc,
            a.H_in, a.G_in, states, a.H_out, a.G_out);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    using L = CgSmem<D, D, CH>;
    auto kern = simt_cg_kernel<D, D, CH, Tin>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
    if (e != cudaSuccess) return e;
    {
        LaunchTimer timer(kKindSimtCg, st);
        kern<<<dim3(nc, BH), kThreads, L::bytes, st>>>(
            static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.v),
            a.gamma, a.beta, a.lambda, a.H, a.T, nc, a.cg_steps, a.tol, states, a.out, a.iters);
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
