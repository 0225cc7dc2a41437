// simt_backward.cu -- chunkwise backward of the Mesa layer on the CUDA cores (fp32).
//
// The pages claim the layer trains in time linear in T but give no backward
// method. Reading taken here: implicit differentiation of the solution map
// x_t = (H_t + Lambda)^-1 q_t, with the adjoint system solved by the same CG
// rule (same step count; the stopping test relative to its own right-hand
// side). For a loss L with do_t = dL/do_t (zero initial states):
//   u_t  = CG_N(H_t + Lambda, G_t^T do_t)          dq_t = u_t
//   dlambda_i = -sum_t u_ti x_ti
//   Gbar_s = sum_{t>=s} (prod_{r=s+1..t} gamma_r) do_t x_t^T
//   Hbar_s = -sum_{t>=s} (prod_{r=s+1..t} gamma_r) u_t x_t^T
//   dv_s = beta_s Gbar_s k_s,   dk_s = beta_s ((Hbar_s + Hbar_s^T) k_s + Gbar_s^T v_s)
//   dbeta_s = k_s^T Hbar_s k_s + v_s^T Gbar_s k_s
//   gamma_s dgamma_s = sum_{t>=s} z_t,   z_t = e_t - beta_t dbeta_t,
//   e_t = (G_t^T do_t) . x_t - u_t . (H_t x_t)
// The last line is the Frobenius form <Hbar_s, H_{s-1}> + <Gbar_s, G_{s-1}>
// rewritten over the pairs (t, s) that the factor gamma_s enters, so no state
// before every token is needed.
//
// Every product is chunkwise, as in the forward: within chunk c = [t0, t0+C)
// with b_t the in-chunk log-cumsum of gamma, the reversed decay is
// N_st = e^{b_t - b_s} for t >= s, and the gradient states carried backwards
// across chunks obey
//   Ghat_{c-1} = e^{b_last} Ghat_c + sum_{t in c} e^{b_t} do_t x_t^T
// (Hhat the same with u_t), so for s in chunk c
//   Gbar_s = sum_{t in c, t>=s} N_st do_t x_t^T + e^{b_last - b_s} Ghat_c.
//
// Kernels (all fp32, 256 threads, thread layout of simt_chunk.cuh):
//   the forward solutions x_t: the fp32 scan + CG of simt_forward.cu, or,
//                     for bf16 inputs at d = 128, C = 64, the tensor-core
//                     scan and solve (x stored in fp32);
//   simt_adj_kernel   grid (chunks, B*H): right-hand side G_t^T do_t, the
//                     adjoint CG, H_t x_t, then dq, e_t and per-chunk dlambda
//                     sums; for bf16 inputs at d = 128, C = 64 the same on the
//                     tensor cores instead (tc_adjoint in tc_forward.cu, from
//                     the forward's state images) and dlambda_part_kernel;
//   simt_rscan_kernel grid (64 x 64 state tiles, B*H): the reverse chunk scan of
//                     Hhat_c and Ghat_c;
//   simt_grad_kernel  grid (chunks, B*H): dk, dv, dbeta and z_t;
//   dgamma_kernel     grid (B*H): the suffix sums of z;
//   dlambda_kernel    the batch and chunk sums of dlambda, in a fixed order.
#include "mesa_internal.h"
#include "simt_chunk.cuh"

namespace mesa {
namespace {

using namespace simt;

template <int DK, int DV, int CH, typename Tin>
__global__ void __launch_bounds__(kThreads, 1)
simt_adj_kernel(const Tin* __restrict__ k, const Tin* __restrict__ v, const float* __restrict__ gamma,
                const float* __restrict__ beta, const float* __restrict__ lambda, const float* __restrict__ dout,
                const float* __restrict__ xsol, int H, int T, int nc, int cg_steps, float tol,
                const float* __restrict__ states, float* __restrict__ dq, float* __restrict__ z,
                float* __restrict__ dlam_part) {
    static_assert(DK == DV && DK % 16 == 0 && CH % 16 == 0, "dk == dv, multiples of 16");
    using L = CgSmem<DK, DV, CH>;
    constexpr int TP = CH / 16, IP = DK / 16;
    constexpr int DKP = L::DKP, DVP = L::DVP, CHP = L::CHP;
    constexpr size_t SE = (size_t)DK * DK + (size_t)DV * DK;
    static_assert(CH * DVP >= 16 * DK, "the value buffer holds the dlambda partials");
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

    // ---- stage: G_c, K, V, the rows of dL/do (in the direction buffer), lambda, gates, mask ----
    for (int e = tid; e < DV * DK; e += kThreads) sH[(e / DK) * DKP + e % DK] = Gc[e];
    for (int e = tid; e < CH * DK; e += kThreads) {
        const int t = e / DK, d = e % DK;
        sK[t * DKP + d] = (t < n) ? ld_in(k, (base + t) * DK + d) : 0.f;
        sP[t * DKP + d] = (t < n) ? dout[(base + t) * DV + d] : 0.f;
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
    __syncthreads();

    // ---- right-hand side g_t = G_t^T do_t = e^{b_t} G_c^T do_t + sum_j M_tj (v_j . do_t) k_j ----
    masked_scores<DK, CH>(sP, sV, sM, sW);
    __syncthreads();
    float g[TP][IP];
#pragma unroll
    for (int a = 0; a < TP; ++a)
#pragma unroll
        for (int b = 0; b < IP; ++b) g[a][b] = 0.f;
#pragma unroll 4
    for (int l = 0; l < DV; ++l) {
        float dv_[TP], gv[IP];
#pragma unroll
        for (int a = 0; a < TP; ++a) dv_[a] = sP[(tt + 16 * a) * DKP + l];
#pragma unroll
        for (int b = 0; b < IP; ++b) gv[b] = sH[l * DKP + ti + 16 * b];
#pragma unroll
        for (int a = 0; a < TP; ++a)
#pragma unroll
            for (int b = 0; b < IP; ++b) g[a][b] = fmaf(dv_[a], gv[b], g[a][b]);
    }
#pragma unroll
    for (int a = 0; a < TP; ++a) {
        const float e = sE[tt + 16 * a];
#pragma unroll
        for (int b = 0; b < IP; ++b) g[a][b] *= e;
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
            for (int b = 0; b < IP; ++b) g[a][b] = fmaf(wv[a], kv[b], g[a][b]);
    }
    // g . x with the forward solution (the first term of e_t)
    float gx[TP];
#pragma unroll
    for (int a = 0; a < TP; ++a) {
        const int t = tt + 16 * a;
        float s = 0.f;
#pragma unroll
        for (int b = 0; b < IP; ++b) s = fmaf(g[a][b], (t < n) ? xsol[(base + t) * DK + ti + 16 * b] : 0.f, s);
        gx[a] = sum16(s);
    }
    __syncthreads();                                   // reads of G_c and of the dL/do rows are done

    // ---- adjoint CG on (H_t + Lambda) u_t = g_t ----
    for (int e = tid; e < DK * DK; e += kThreads) sH[(e / DK) * DKP + e % DK] = Hc[e];
    float x[TP][IP], r[TP][IP];
    float rr[TP], qn[TP];
    bool act[TP];
    int it[TP];
#pragma unroll
    for (int a = 0; a < TP; ++a) {
        const int t = tt + 16 * a;
        float s = 0.f;
#pragma unroll
        for (int b = 0; b < IP; ++b) {
            x[a][b] = 0.f;
            r[a][b] = g[a][b];
            sP[t * DKP + ti + 16 * b] = g[a][b];
            s = fmaf(g[a][b], g[a][b], s);
        }
        rr[a] = sum16(s);
        qn[a] = sqrtf(rr[a]);
        act[a] = t < n;
        it[a] = 0;
    }
    __syncthreads();
    chunk_cg<DK, CH>(sP, sH, sK, sW, sM, sE, sL, x, r, g, rr, qn, act, it, cg_steps, tol);

    // ---- H_t x_t with the forward solution, then e_t = g.x - u.(H x) ----
    __syncthreads();
#pragma unroll
    for (int a = 0; a < TP; ++a) {
        const int t = tt + 16 * a;
#pragma unroll
        for (int b = 0; b < IP; ++b) sP[t * DKP + ti + 16 * b] = (t < n) ? xsol[(base + t) * DK + ti + 16 * b] : 0.f;
    }
    __syncthreads();
    float hx[TP][IP];
    chunk_matvec<DK, CH>(sP, sH, sK, sW, sM, sE, hx);
    float lp[IP];
#pragma unroll
    for (int b = 0; b < IP; ++b) lp[b] = 0.f;
#pragma unroll
    for (int a = 0; a < TP; ++a) {
        const int t = tt + 16 * a;
        float s = 0.f;
#pragma unroll
        for (int b = 0; b < IP; ++b) {
            s = fmaf(x[a][b], hx[a][b], s);
            lp[b] = fmaf(x[a][b], sP[t * DKP + ti + 16 * b], lp[b]);
        }
        const float e = gx[a] - sum16(s);
        if (t < n) {
#pragma unroll
            for (int b = 0; b < IP; ++b) dq[(base + t) * DK + ti + 16 * b] = x[a][b];
            if (ti == 0) z[base + t] = e;
        }
    }
    // dlambda partial of the chunk: -sum_t u_ti x_ti, summed over the 16 row groups in order
    float* red = sV;                                   // values were last read before the first CG barrier
#pragma unroll
    for (int b = 0; b < IP; ++b) red[tt * DK + ti + 16 * b] = lp[b];
    __syncthreads();
    for (int i = tid; i < DK; i += kThreads) {
        float s = 0.f;
        for (int rg = 0; rg < 16; ++rg) s += red[rg * DK + i];
        dlam_part[((size_t)bh * nc + c) * DK + i] = -s;
    }
}

// Reverse chunk scan of the gradient states: CTA (tile, bh) walks the chunks
// of sequence bh from the last to the first for one tile of Hhat (rows from
// u) or Ghat (rows from dL/do), columns from x. Writes, per chunk c, the state
// carried in from the tokens after it.
// Four CTAs per SM (at most 64 registers a thread): with 2 x (d / 64)^2 tiles
// per sequence the grid is 1024 CTAs at d = 128, B x H = 128, which then runs
// in two waves of 592 instead of three of 444.
template <int DK, int DV, int CH>
__global__ void __launch_bounds__(kThreads, 4)
simt_rscan_kernel(const float* __restrict__ dout, const float* __restrict__ u, const float* __restrict__ xsol,
                  const float* __restrict__ gamma, int T, int nc, float* __restrict__ rstates) {
    static_assert(DK == DV, "dk == dv");
    constexpr int TL = DK < 64 ? DK : 64;                  // tile edge
    constexpr int R = TL / 16;                             // each thread: R x R elements of the tile
    constexpr int TS = TL + 4;                             // shared row stride (16-byte rows)
    constexpr int TPR = DK / TL;
    constexpr int H_TILES = TPR * TPR;
    constexpr size_t SE = (size_t)DK * DK + (size_t)DV * DK;

    __shared__ __align__(16) float sA[CH * TS];
    __shared__ __align__(16) float sX[CH * TS];
    __shared__ float sb[CH];
    __shared__ float sw[CH];

    const int bh = blockIdx.y;
    int tile = blockIdx.x;
    const bool isG = tile >= H_TILES;
    if (isG) tile -= H_TILES;
    const int trow = (tile / TPR) * TL, tcol = (tile % TPR) * TL;
    const int i0 = trow + (threadIdx.x >> 4) * R, j0 = tcol + (threadIdx.x & 15) * R;
    const float* A = isG ? dout : u;
    const size_t mat_off = isG ? (size_t)DK * DK : 0;

    float S[R][R];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int c = 0; c < R; ++c) S[r][c] = 0.f;
    // warp 0 holds the gammas of the next chunk (positions 2 lane, 2 lane + 1;
    // 1 past the sequence end), loaded a chunk ahead so their latency hides
    // under the current chunk's copies and products
    const int lane = threadIdx.x & 31;
    const bool gw = threadIdx.x < 32;
    float g0 = 1.f, g1 = 1.f;
    auto load_gates = [&](int cc) {
        const int nn = min(CH, T - cc * CH);
        const size_t gb = (size_t)bh * T + (size_t)cc * CH;
        g0 = 2 * lane < nn ? gamma[gb + 2 * lane] : 1.f;
        g1 = 2 * lane + 1 < nn ? gamma[gb + 2 * lane + 1] : 1.f;
    };
    if (gw && nc > 0) load_gates(nc - 1);
    for (int c = nc - 1; c >= 0; --c) {
        const int t0 = c * CH;
        const int n = min(CH, T - t0);
        const size_t base = (size_t)bh * T + t0;
        float* dst = rstates + ((size_t)bh * nc + c) * SE + mat_off;
#pragma unroll
        for (int r = 0; r < R; ++r) store_n<R>(dst + (size_t)(i0 + r) * DK + j0, S[r]);
        if (gw) {                                      // b = the in-chunk log-cumsum of gamma
            const float l0 = logf(g0), l1 = logf(g1);
            const float pair = l0 + l1;
            float incl = pair;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float o = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += o;
            }
            const float excl = incl - pair;
            if (2 * lane < CH) sb[2 * lane] = excl + l0;
            if (2 * lane + 1 < CH) sb[2 * lane + 1] = excl + l0 + l1;
            if (c > 0) load_gates(c - 1);
        }
        __syncthreads();
        const float blast = sb[CH - 1];
        for (int t = threadIdx.x; t < CH; t += kThreads) sw[t] = (t < n) ? expf(sb[t]) : 0.f;
        __syncthreads();
#pragma unroll 4
        for (int idx = threadIdx.x; idx < CH * TL / 4; idx += kThreads) {   // 16-byte pieces (TL, TS multiples of 4)
            const int t = idx / (TL / 4), col = 4 * (idx % (TL / 4));
            float4 a4 = make_float4(0.f, 0.f, 0.f, 0.f), x4 = a4;
            if (t < n) {
                const float wt = sw[t];
                a4 = *reinterpret_cast<const float4*>(A + (base + t) * DK + trow + col);
                a4 = make_float4(wt * a4.x, wt * a4.y, wt * a4.z, wt * a4.w);
                x4 = *reinterpret_cast<const float4*>(xsol + (base + t) * DK + tcol + col);
            }
            *reinterpret_cast<float4*>(sA + t * TS + col) = a4;
            *reinterpret_cast<float4*>(sX + t * TS + col) = x4;
        }
        __syncthreads();
        const float Gam = expf(blast);
        float acc[R][R];
        tile_outer<CH, TL>(sA, sX, acc);
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int cc = 0; cc < R; ++cc) S[r][cc] = fmaf(Gam, S[r][cc], acc[r][cc]);
        __syncthreads();
    }
}

// Shared tiles of the gradient kernel: rows of D floats, no padding. The
// tiles read down their columns (the state, x and the dL/do / u rows) are
// swizzled: the 16-byte piece j of row rho sits at piece j ^ (rho & SWM), so
// eight threads reading one piece of eight consecutive rows hit distinct
// banks, and a thread reads four consecutive elements of a row at once.
// Four consecutive input elements (16-byte aligned for float, 8-byte for bf16), widened to float.
__device__ __forceinline__ float4 ld_in4(const float* p, size_t i) { return *reinterpret_cast<const float4*>(p + i); }
__device__ __forceinline__ float4 ld_in4(const __nv_bfloat16* p, size_t i) {
    const uint2 u = *reinterpret_cast<const uint2*>(p + i);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

template <int D>
struct GradSwz {
    static constexpr int SWM = (D / 4 < 8 ? D / 4 : 8) - 1;
    // element (row, col)
    static __device__ __forceinline__ int at(int row, int col) {
        return row * D + ((((col >> 2) ^ (row & SWM))) << 2) + (col & 3);
    }
    // the 16-byte piece j of row `row`
    static __device__ __forceinline__ float4* piece(float* tile, int row, int j) {
        return reinterpret_cast<float4*>(tile + row * D + ((j ^ (row & SWM)) << 2));
    }
};

template <int D, int CH>
struct GradSmem {
    static constexpr int DP = D, CHP = CH + 1;
    static constexpr int oR = 0;                       // Ghat_c, later Hhat_c  [D][D] swizzled
    static constexpr int oK = oR + D * DP;             // keys                  [CH][D]
    static constexpr int oV = oK + CH * DP;            // values                [CH][D]
    static constexpr int oX = oV + CH * DP;            // forward solutions x   [CH][D] swizzled
    static constexpr int oD = oX + CH * DP;            // dL/do rows, later u   [CH][D] swizzled
    static constexpr int oW = oD + CH * DP;            // reversed masked scores [CH][CHP]
    static constexpr int oW1 = oW + CH * CHP;          // N_st (k_s . x_t), kept for the second half [CH][CHP]
    static constexpr int oB = oW1 + CH * CHP;          // b_t                   [CH]
    static constexpr int oBeta = oB + CH;              // beta_t                [CH]
    static constexpr int total = oBeta + CH;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

// W_st = e^{b_t - b_s} (a_s . c_t) for s <= t < n, else 0 (rows s, columns t).
template <int D, int CH>
__device__ __forceinline__ void rev_scores(const float* sA, const float* sC, const float* sB, int n, float* sW) {
    constexpr int TP = CH / 16, JP = CH / 16, DP = GradSmem<D, CH>::DP, CHP = CH + 1;
    const int tt = threadIdx.x >> 4, ti = threadIdx.x & 15;
    float s[TP][JP];
#pragma unroll
    for (int a = 0; a < TP; ++a)
#pragma unroll
        for (int b = 0; b < JP; ++b) s[a][b] = 0.f;
#pragma unroll 2
    for (int kk = 0; kk < D; kk += 4) {                // four k at a time, in order
        float4 av[TP], cv[JP];
#pragma unroll
        for (int a = 0; a < TP; ++a) av[a] = *reinterpret_cast<const float4*>(sA + (tt + 16 * a) * DP + kk);
#pragma unroll
        for (int b = 0; b < JP; ++b)                   // sC swizzled; (ti + 16 b) & SWM = ti & SWM
            cv[b] = *reinterpret_cast<const float4*>(sC + (ti + 16 * b) * DP + (((kk >> 2) ^ (ti & GradSwz<D>::SWM)) << 2));
#pragma unroll
        for (int a = 0; a < TP; ++a)
#pragma unroll
            for (int b = 0; b < JP; ++b) {
                s[a][b] = fmaf(av[a].x, cv[b].x, s[a][b]);
                s[a][b] = fmaf(av[a].y, cv[b].y, s[a][b]);
                s[a][b] = fmaf(av[a].z, cv[b].z, s[a][b]);
                s[a][b] = fmaf(av[a].w, cv[b].w, s[a][b]);
            }
    }
#pragma unroll
    for (int a = 0; a < TP; ++a)
#pragma unroll
        for (int b = 0; b < JP; ++b) {
            const int r = tt + 16 * a, t = ti + 16 * b;
            sW[r * CHP + t] = (t >= r && t < n) ? expf(sB[t] - sB[r]) * s[a][b] : 0.f;
        }
}

// acc[s][o] += sum_t W_st R_t[o]   (rows s = tt + 16 a, columns o = ti + 16 b)
template <int D, int CH>
__device__ __forceinline__ void add_wr(const float* sW, const float* sR, float (&acc)[CH / 16][D / 16]) {
    constexpr int TP = CH / 16, IP = D / 16, DP = GradSmem<D, CH>::DP, CHP = CH + 1;
    const int tt = threadIdx.x >> 4, ti = threadIdx.x & 15;
#pragma unroll 4
    for (int t = 0; t < CH; ++t) {
        float wv[TP], rv[IP];
#pragma unroll
        for (int a = 0; a < TP; ++a) wv[a] = sW[(tt + 16 * a) * CHP + t];
        // sR swizzled: column ti + 16 b of row t (the swizzle flips bit 0 of b
        // when bit 2 of t & SWM is set, and the low piece bits by t & 3)
        const int x = t & GradSwz<D>::SWM, flip = (x >> 2) << 4;
        const float* rrow = sR + t * DP + (((ti >> 2) ^ (x & 3)) << 2) + (ti & 3);
#pragma unroll
        for (int b = 0; b < IP; ++b) rv[b] = rrow[16 * b + ((b & 1) ? -flip : flip)];
#pragma unroll
        for (int a = 0; a < TP; ++a)
#pragma unroll
            for (int b = 0; b < IP; ++b) acc[a][b] = fmaf(wv[a], rv[b], acc[a][b]);
    }
}

// acc[s][o] += sum_r A_s[r] M[o][r] (COL = false) or A_s[r] M[r][o] (COL = true)
template <int D, int CH, bool COL>
__device__ __forceinline__ void add_state(const float* sA, const float* sM, float (&acc)[CH / 16][D / 16]) {
    constexpr int TP = CH / 16, IP = D / 16, DP = GradSmem<D, CH>::DP;
    const int tt = threadIdx.x >> 4, ti = threadIdx.x & 15;
#pragma unroll 1
    for (int r = 0; r < D; r += 4) {                   // four r at a time, in order
        float4 av[TP];
#pragma unroll
        for (int a = 0; a < TP; ++a) av[a] = *reinterpret_cast<const float4*>(sA + (tt + 16 * a) * DP + r);
        if constexpr (COL) {                           // rows of M: one float per column, per r
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float mv[IP];
                const int x = (r + j) & GradSwz<D>::SWM, flip = (x >> 2) << 4;
                const float* mrow = sM + (r + j) * DP + (((ti >> 2) ^ (x & 3)) << 2) + (ti & 3);
#pragma unroll
                for (int b = 0; b < IP; ++b) mv[b] = mrow[16 * b + ((b & 1) ? -flip : flip)];
#pragma unroll
                for (int a = 0; a < TP; ++a) {
                    const float aj = j == 0 ? av[a].x : j == 1 ? av[a].y : j == 2 ? av[a].z : av[a].w;
#pragma unroll
                    for (int b = 0; b < IP; ++b) acc[a][b] = fmaf(aj, mv[b], acc[a][b]);
                }
            }
        } else {                                       // columns of M: four r per vector load
#pragma unroll
            for (int b = 0; b < IP; ++b) {
                const float4 m4 =
                    *reinterpret_cast<const float4*>(sM + (ti + 16 * b) * DP + (((r >> 2) ^ (ti & GradSwz<D>::SWM)) << 2));
#pragma unroll
                for (int a = 0; a < TP; ++a) {
                    acc[a][b] = fmaf(av[a].x, m4.x, acc[a][b]);
                    acc[a][b] = fmaf(av[a].y, m4.y, acc[a][b]);
                    acc[a][b] = fmaf(av[a].z, m4.z, acc[a][b]);
                    acc[a][b] = fmaf(av[a].w, m4.w, acc[a][b]);
                }
            }
        }
    }
}

template <int CH, int IP>
__device__ __forceinline__ void zero2(float (&m)[CH / 16][IP]) {
#pragma unroll
    for (int a = 0; a < CH / 16; ++a)
#pragma unroll
        for (int b = 0; b < IP; ++b) m[a][b] = 0.f;
}

// dk, dv, dbeta and z_t = e_t - beta_t dbeta_t for the tokens of one chunk.
template <int DK, int DV, int CH, typename Tin>
__global__ void __launch_bounds__(kThreads, 1)
simt_grad_kernel(const Tin* __restrict__ k, const Tin* __restrict__ v, const float* __restrict__ gamma,
                 const float* __restrict__ beta, const float* __restrict__ dout, const float* __restrict__ u,
                 const float* __restrict__ xsol, int T, int nc, const float* __restrict__ rstates,
                 float* __restrict__ dk_out, float* __restrict__ dv_out, float* __restrict__ dbeta,
                 float* __restrict__ z) {
    static_assert(DK == DV && DK % 16 == 0 && CH % 16 == 0, "dk == dv, multiples of 16");
    using G = GradSmem<DK, CH>;
    constexpr int TP = CH / 16, IP = DK / 16, DP = G::DP;
    constexpr size_t SE = (size_t)DK * DK + (size_t)DV * DK;
    extern __shared__ float smem[];
    float* sR = smem + G::oR;
    float* sK = smem + G::oK;
    float* sV = smem + G::oV;
    float* sX = smem + G::oX;
    float* sD = smem + G::oD;
    float* sW = smem + G::oW;
    float* sW1 = smem + G::oW1;
    float* sB = smem + G::oB;
    float* sBeta = smem + G::oBeta;
    using Z = GradSwz<DK>;                             // layout of sR, sX and sD

    const int c = blockIdx.x, bh = blockIdx.y;
    const int t0 = c * CH;
    const int n = min(CH, T - t0);
    const size_t base = (size_t)bh * T + t0;
    const int tid = threadIdx.x, tt = tid >> 4, ti = tid & 15;
    const float* Hh = rstates + ((size_t)bh * nc + c) * SE;
    const float* Gh = Hh + (size_t)DK * DK;

    // 16-byte pieces: the state, then the rows (zero past n)
    constexpr int PR = DK / 4;                         // pieces per row
#pragma unroll 16
    for (int e = tid; e < DV * PR; e += kThreads)
        *Z::piece(sR, e / PR, e % PR) = *reinterpret_cast<const float4*>(Gh + 4 * (size_t)e);
#pragma unroll 8
    for (int e = tid; e < CH * PR; e += kThreads) {
        const int t = e / PR, j = e % PR;
        const bool ok = t < n;
        const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
        const size_t g = (base + t) * DK + 4 * j;
        *reinterpret_cast<float4*>(sK + t * DP + 4 * j) = ok ? ld_in4(k, g) : zero;
        *reinterpret_cast<float4*>(sV + t * DP + 4 * j) = ok ? ld_in4(v, g) : zero;
        *Z::piece(sX, t, j) = ok ? *reinterpret_cast<const float4*>(xsol + g) : zero;
        *Z::piece(sD, t, j) = ok ? *reinterpret_cast<const float4*>(dout + g) : zero;
    }
    chunk_log_cumsum<CH>(gamma, base, n, sB);
    for (int t = tid; t < CH; t += kThreads) sBeta[t] = (t < n) ? beta[base + t] : 0.f;
    __syncthreads();
    float cs[TP];                                      // e^{b_last - b_s}
#pragma unroll
    for (int a = 0; a < TP; ++a) cs[a] = expf(sB[CH - 1] - sB[tt + 16 * a]);

    float acc[TP][IP], stt[TP][IP], dk_acc[TP][IP], dbt[TP];
    // ---- value statistics: Gbar_s k_s (-> dv) and Gbar_s^T v_s (-> dk) ----
    rev_scores<DK, CH>(sK, sX, sB, n, sW1);            // N_st (k_s . x_t), used again below
    __syncthreads();
    zero2<CH, IP>(acc);
    zero2<CH, IP>(stt);
    add_wr<DK, CH>(sW1, sD, acc);
    add_state<DK, CH, false>(sK, sR, stt);
#pragma unroll
    for (int a = 0; a < TP; ++a) {
        const int s = tt + 16 * a;
        const float bs = sBeta[s];
        float d = 0.f;
#pragma unroll
        for (int b = 0; b < IP; ++b) {
            const float gv = fmaf(cs[a], stt[a][b], acc[a][b]);
            d = fmaf(sV[s * DP + ti + 16 * b], gv, d);
            if (s < n) dv_out[(base + s) * DV + ti + 16 * b] = bs * gv;
        }
        dbt[a] = sum16(d);
    }
    __syncthreads();
    rev_scores<DK, CH>(sV, sD, sB, n, sW);             // N_st (v_s . do_t)
    __syncthreads();
    zero2<CH, IP>(acc);
    zero2<CH, IP>(stt);
    add_wr<DK, CH>(sW, sX, acc);
    add_state<DK, CH, true>(sV, sR, stt);
#pragma unroll
    for (int a = 0; a < TP; ++a)
#pragma unroll
        for (int b = 0; b < IP; ++b) dk_acc[a][b] = fmaf(cs[a], stt[a][b], acc[a][b]);
    __syncthreads();                                   // done with Ghat, the dL/do rows and the scores

    // ---- key statistics: Hbar_s k_s and Hbar_s^T k_s (-> dk, dbeta) ----
#pragma unroll 16
    for (int e = tid; e < DK * PR; e += kThreads)
        *Z::piece(sR, e / PR, e % PR) = *reinterpret_cast<const float4*>(Hh + 4 * (size_t)e);
#pragma unroll 8
    for (int e = tid; e < CH * PR; e += kThreads) {
        const int t = e / PR, j = e % PR;
        *Z::piece(sD, t, j) = (t < n) ? *reinterpret_cast<const float4*>(u + (base + t) * DK + 4 * j)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();                                   // Hhat and the u rows are in place
    zero2<CH, IP>(acc);
    zero2<CH, IP>(stt);
    add_wr<DK, CH>(sW1, sD, acc);                      // the same N_st (k_s . x_t) as the first half
    add_state<DK, CH, false>(sK, sR, stt);
#pragma unroll
    for (int a = 0; a < TP; ++a) {
        const int s = tt + 16 * a;
        float d = 0.f;
#pragma unroll
        for (int b = 0; b < IP; ++b) {
            const float hk = -fmaf(cs[a], stt[a][b], acc[a][b]);
            d = fmaf(sK[s * DP + ti + 16 * b], hk, d);
            dk_acc[a][b] += hk;
        }
        dbt[a] += sum16(d);
    }
    __syncthreads();
    rev_scores<DK, CH>(sK, sD, sB, n, sW);             // N_st (k_s . u_t)
    __syncthreads();
    zero2<CH, IP>(acc);
    zero2<CH, IP>(stt);
    add_wr<DK, CH>(sW, sX, acc);
    add_state<DK, CH, true>(sK, sR, stt);
#pragma unroll
    for (int a = 0; a < TP; ++a) {
        const int s = tt + 16 * a;
        if (s < n) {
            const float bs = sBeta[s];
#pragma unroll
            for (int b = 0; b < IP; ++b)
                dk_out[(base + s) * DK + ti + 16 * b] = bs * (dk_acc[a][b] - fmaf(cs[a], stt[a][b], acc[a][b]));
            if (ti == 0) {
                dbeta[base + s] = dbt[a];
                z[base + s] -= bs * dbt[a];
            }
        }
    }
}

// gamma_t dgamma_t = sum_{t' >= t} z_t': one CTA per sequence, fp64 sums.
__global__ void __launch_bounds__(256) dgamma_kernel(const float* __restrict__ z, const float* __restrict__ gamma,
                                                     int T, float* __restrict__ dgamma) {
    __shared__ double part[256];
    const size_t off = (size_t)blockIdx.x * T;
    const int seg = (T + 255) / 256;
    const int lo = min(T, (int)threadIdx.x * seg), hi = min(T, lo + seg);
    double s = 0.0;
    for (int t = lo; t < hi; ++t) s += z[off + t];
    part[threadIdx.x] = s;
    __syncthreads();
    double acc = 0.0;
    for (int j = 255; j > (int)threadIdx.x; --j) acc += part[j];
    for (int t = hi - 1; t >= lo; --t) {
        acc += z[off + t];
        dgamma[off + t] = (float)(acc / gamma[off + t]);
    }
}

// dlambda[h][i] = sum over batch rows b, then chunks c, of the chunk partials.
// Per-chunk sums -sum_{t in c} u_ti x_ti of the dlambda partials from u (dq)
// and x, one block per (chunk, b*h) and one thread per key channel, in token
// order: the layout simt_adj_kernel writes, for dlambda_kernel.
__global__ void dlambda_part_kernel(const float* __restrict__ u, const float* __restrict__ x, int T, int chunk,
                                    int nc, int dk, float* __restrict__ part) {
    const int c = blockIdx.x, bh = blockIdx.y;
    for (int i = threadIdx.x; i < dk; i += blockDim.x) {
        const int t0 = c * chunk, t1 = min(T, t0 + chunk);
        float s = 0.f;
        for (int t = t0; t < t1; ++t) {
            const size_t e = ((size_t)bh * T + t) * dk + i;
            s = fmaf(-u[e], x[e], s);
        }
        part[((size_t)bh * nc + c) * dk + i] = s;
    }
}

__global__ void dlambda_kernel(const float* __restrict__ part, int B, int H, int nc, int dk,
                               float* __restrict__ dlambda) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= H * dk) return;
    const int h = idx / dk, i = idx % dk;
    float s = 0.f;
    for (int b = 0; b < B; ++b)
        for (int c = 0; c < nc; ++c) s += part[(((size_t)b * H + h) * nc + c) * dk + i];
    dlambda[idx] = s;
}

struct BwdLayout {
    size_t states, x, z, rstates, part, tcws, oscr, total;
};

// With the tensor-core solve (bf16, d = 128, C = 64) the forward solutions
// come from it: its workspace and a scratch read-out follow the rest.
BwdLayout bwd_layout(int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t nc = (size_t)((T + chunk - 1) / chunk);
    const size_t BH = (size_t)B * H;
    const size_t se = nc * ((size_t)dk * dk + (size_t)dv * dk) * sizeof(float);
    BwdLayout l;
    l.states = 0;                      // fp32 chunk-start states: the CUDA-core adjoint only
    l.x = l.states + (tc_supported(dk, dv, chunk, dtype) ? 0 : up(BH * se));
    l.z = l.x + up(BH * T * dk * sizeof(float));
    l.rstates = l.z + up(BH * T * sizeof(float));
    l.part = l.rstates + up(BH * se);
    l.tcws = l.part + up(BH * nc * dk * sizeof(float));
    l.oscr = l.tcws;
    l.total = l.tcws;
    if (tc_supported(dk, dv, chunk, dtype)) {
        l.oscr = l.tcws + up(tc_workspace_bytes(B, H, T));
        l.total = l.oscr + up(BH * T * dv * sizeof(float));
    }
    return l;
}

template <int D, int CH, typename Tin>
cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t st) {
    const ForwardArgs& f = a.f;
    const int nc = (f.T + CH - 1) / CH;
    const int BH = f.B * f.H;
    const BwdLayout l = bwd_layout(f.B, f.H, f.T, D, D, CH, f.dtype);
    char* ws = static_cast<char*>(f.workspace);
    float* states = reinterpret_cast<float*>(ws + l.states);
    float* X = reinterpret_cast<float*>(ws + l.x);
    float* Z = reinterpret_cast<float*>(ws + l.z);
    float* R = reinterpret_cast<float*>(ws + l.rstates);
    float* part = reinterpret_cast<float*>(ws + l.part);

    // forward: the solutions x_t (and whatever chunk states the adjoint reads)
    ForwardArgs fa = f;
    fa.out = nullptr;
    fa.iters = nullptr;
    fa.H_in = fa.G_in = nullptr;
    fa.H_out = fa.G_out = nullptr;
    fa.workspace = states;
    fa.x_out = X;
    cudaError_t e;
    if (tc_supported(f.dk, f.dv, f.chunk, f.dtype)) {
        // bf16 inputs at d = 128, C = 64, all on the tensor cores (the
        // bf16-mode precision): the scan and solve give x and leave their
        // fp16 state images in the workspace; the adjoint reads those
        // images, so no fp32 states are formed. The read-out buffer, which
        // the backward does not need, holds g_t = G_t^T dout_t.
        ForwardArgs ft = fa;
        ft.workspace = ws + l.tcws;
        ft.ws_bytes = l.oscr - l.tcws;
        float* scratch = reinterpret_cast<float*>(ws + l.oscr);
        ft.out = scratch;
        if ((e = forward_tc(ft, st)) != cudaSuccess) return e;
        if ((e = tc_adjoint(f, ws + l.tcws, a.dout, X, scratch, a.dq, Z, st)) != cudaSuccess) return e;
        LaunchTimer timer(kKindBwdReduce, st);
        dlambda_part_kernel<<<dim3(nc, BH), 128, 0, st>>>(a.dq, X, f.T, CH, nc, D, part);
    } else {
        if ((e = forward_simt(fa, st)) != cudaSuccess) return e;
        using L = CgSmem<D, D, CH>;
        auto adj = simt_adj_kernel<D, D, CH, Tin>;
        e = cudaFuncSetAttribute(adj, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
        if (e != cudaSuccess) return e;
        LaunchTimer timer(kKindBwdAdj, st);
        adj<<<dim3(nc, BH), kThreads, L::bytes, st>>>(
            static_cast<const Tin*>(f.k), static_cast<const Tin*>(f.v), f.gamma, f.beta, f.lambda, a.dout, X, f.H,
            f.T, nc, f.cg_steps, f.tol, states, a.dq, Z, part);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (tc_supported(f.dk, f.dv, f.chunk, f.dtype)) {
        // the reverse scan on the tensor cores at the same bf16-mode precision
        if ((e = tc_rscan_launch(a.dout, a.dq, X, f.gamma, f.B, f.H, f.T, R, error_word_ptr(), st)) != cudaSuccess)
            return e;
    } else {
        constexpr int TL = D < 64 ? D : 64;
        constexpr int tiles = 2 * (D / TL) * (D / TL);
        LaunchTimer timer(kKindBwdRscan, st);
        simt_rscan_kernel<D, D, CH><<<dim3(tiles, BH), kThreads, 0, st>>>(a.dout, a.dq, X, f.gamma, f.T, nc, R);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    using G = GradSmem<D, CH>;
    auto grad = simt_grad_kernel<D, D, CH, Tin>;
    e = cudaFuncSetAttribute(grad, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::bytes);
    if (e != cudaSuccess) return e;
    {
        LaunchTimer timer(kKindBwdGrad, st);
        grad<<<dim3(nc, BH), kThreads, G::bytes, st>>>(
            static_cast<const Tin*>(f.k), static_cast<const Tin*>(f.v), f.gamma, f.beta, a.dout, a.dq, X, f.T, nc,
            R, a.dk, a.dv, a.dbeta, Z);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    {
        LaunchTimer timer(kKindBwdReduce, st);
        dgamma_kernel<<<BH, 256, 0, st>>>(Z, f.gamma, f.T, a.dgamma);
        dlambda_kernel<<<(f.H * D + 255) / 256, 256, 0, st>>>(part, f.B, f.H, nc, D, a.dlambda);
    }
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t dispatch_backward(const BackwardArgs& a, cudaStream_t st) {
    const ForwardArgs& f = a.f;
#define MESA_BWD_CASE(D_, C_) \
    if (f.dk == D_ && f.chunk == C_) return launch_backward<D_, C_, Tin>(a, st);
    MESA_BWD_CASE(16, 16) MESA_BWD_CASE(16, 32) MESA_BWD_CASE(16, 64)
    MESA_BWD_CASE(32, 16) MESA_BWD_CASE(32, 32) MESA_BWD_CASE(32, 64)
    MESA_BWD_CASE(64, 16) MESA_BWD_CASE(64, 32) MESA_BWD_CASE(64, 64)
    MESA_BWD_CASE(128, 16) MESA_BWD_CASE(128, 32) MESA_BWD_CASE(128, 64)
#undef MESA_BWD_CASE
    return cudaErrorInvalidValue;
}

}  // namespace

size_t backward_workspace_bytes(int B, int H, int T, int dk, int dv, int chunk, mesa_dtype dtype) {
    return bwd_layout(B, H, T, dk, dv, chunk, dtype).total;
}

cudaError_t backward_simt(const BackwardArgs& a, cudaStream_t st) {
    return a.f.dtype == MESA_BF16 ? dispatch_backward<__nv_bfloat16>(a, st) : dispatch_backward<float>(a, st);
}

}  // namespace mesa
