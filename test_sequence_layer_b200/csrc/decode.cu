// decode.cu -- one recurrent decode step of the Mesa layer on explicit state.
//
// Method: "MesaNet: Sequence Modeling by Locally Optimal Test-Time Training"
// (gist.science), Technical summary > Method > Mesa layer ("Parallelisation":
// the layer keeps the state variables G_t and H_t and runs inference at O(1)
// cost per token). Per (b, h):
//     H <- gamma H + beta k k^T,  G <- gamma G + beta v k^T,
//     x  = CG(H + Lambda, q)      (rule in mesa.h),   out = G x.
//
// The step is bound by HBM: each head reads and writes its fp32 H and G
// (4 * 4 * d^2 bytes = 256 KiB at d = 128). One CTA of 8 warps serves one
// head:
//   * the G matrix is prefetched into shared memory with cp.async at entry,
//     so its read overlaps the H update and the CG iterations;
//   * H is read with coalesced vector loads, updated, written back, and kept
//     in registers (warp w owns rows w, w+8, ...; lane l owns columns
//     l*CPL .. l*CPL+CPL-1), so every CG matvec runs from registers;
//   * each matvec reduces its per-lane partial row sums with a butterfly
//     transpose-reduction (R rows over 32 lanes in R-1+log2(32/R)... shuffles)
//     instead of R full warp reductions; the block sums use a double-buffered
//     scratch, one barrier each;
//   * with x_state the CG starts from the caller's guess (warm start; the
//     pages name warm starts as the way to cut the solver's cost, MesaNet
//     page, Significance and claims): r0 = q - (H + Lambda) x0, and the
//     solution is written back to x_state.
#include "mesa_common.cuh"
#include "mesa_internal.h"

namespace mesa {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;

// Reduces R per-lane partial sums across the warp. On return the lane holds
// the full sum of row row_of_lane<R>(lane).
template <int R>
__device__ __forceinline__ float butterfly_reduce(float (&v)[R], int lane) {
    int off = 16;
#pragma unroll
    for (int cnt = R; cnt > 1; cnt >>= 1, off >>= 1) {
        const int half = cnt >> 1;
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int m = 0; m < half; ++m) {
            const float send = upper ? v[m] : v[m + half];
            const float keep = upper ? v[m + half] : v[m];
            v[m] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    float s = v[0];
    for (; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    return s;
}

template <int R>
__device__ __forceinline__ int row_of_lane(int lane) {
    int row = 0, off = 16;
#pragma unroll
    for (int cnt = R; cnt > 1; cnt >>= 1, off >>= 1)
        if (lane & off) row += cnt >> 1;
    return row;
}

// Block-wide sum; exactly one lane per row contributes (contrib == true).
// red holds two kWarps-slot buffers used alternately (par flips per call):
// the barrier of the call in between orders a buffer's readers before its
// next writers, so each call needs one barrier.
__device__ __forceinline__ float block_sum(float v, bool contrib, float* red, int& par, int warp, int lane) {
    float s = contrib ? v : 0.f;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    float* rb = red + par * kWarps;
    if (lane == 0) rb[warp] = s;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) tot += rb[w];
    par ^= 1;
    return tot;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
step_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
            const float* __restrict__ gamma, const float* __restrict__ beta,
            const float* __restrict__ lambda, int H, float* __restrict__ Hs, float* __restrict__ Gs,
            int cg_steps, float tol, float* __restrict__ out, int32_t* __restrict__ iters,
            float* __restrict__ xs) {
    constexpr int RPW = D / kWarps;                  // rows per warp
    constexpr int CPL = D >= 32 ? D / 32 : 1;        // columns per lane
    constexpr int DUP = 32 / RPW;                    // lanes sharing one row after the reduction
    static_assert(RPW >= 1 && (RPW & (RPW - 1)) == 0, "rows per warp must be a power of two");

    extern __shared__ __align__(16) float smem[];
    float* sG = smem;             // D*D, prefetched G
    float* sk = sG + D * D;       // D
    float* sv = sk + D;           // D
    float* sp = sv + D;           // D (CG direction, later x)
    float* red = sp + D;          // 2 x kWarps

    const int bh = blockIdx.x, h = bh % H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float* Hm = Hs + (size_t)bh * D * D;
    float* Gm = Gs + (size_t)bh * D * D;

    // Prefetch G into shared memory (16-byte async copies, no register staging).
    {
        const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(sG);
        for (int e = tid; e < D * D / 4; e += kThreads) {
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sbase + 16u * e),
                         "l"(Gm + 4 * e)
                         : "memory");
        }
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    }
    for (int e = tid; e < D; e += kThreads) {
        sk[e] = k[(size_t)bh * D + e];
        sv[e] = v[(size_t)bh * D + e];
        sp[e] = q[(size_t)bh * D + e];
    }
    const float g = gamma[bh], bt = beta[bh];
    __syncthreads();

    // H <- gamma H + beta k k^T, written back and kept in registers.
    const int col0 = lane * CPL;
    const bool col_ok = col0 < D;
    float kc[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) kc[c] = col_ok ? sk[col0 + c] : 0.f;
    float Hr[RPW][CPL];
#pragma unroll
    for (int m = 0; m < RPW; ++m) {
        const int i = warp + kWarps * m;
        const float bki = bt * sk[i];
        float* row = Hm + (size_t)i * D + col0;
        if (col_ok) {
            if constexpr (CPL == 4) {
                float4 h4 = *reinterpret_cast<const float4*>(row);
                h4.x = fmaf(g, h4.x, bki * kc[0]);
                h4.y = fmaf(g, h4.y, bki * kc[1]);
                h4.z = fmaf(g, h4.z, bki * kc[2]);
                h4.w = fmaf(g, h4.w, bki * kc[3]);
                *reinterpret_cast<float4*>(row) = h4;
                Hr[m][0] = h4.x; Hr[m][1] = h4.y; Hr[m][2] = h4.z; Hr[m][3] = h4.w;
            } else {
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    const float hv = fmaf(g, row[c], bki * kc[c]);
                    row[c] = hv;
                    Hr[m][c] = hv;
                }
            }
        } else {
#pragma unroll
            for (int c = 0; c < CPL; ++c) Hr[m][c] = 0.f;
        }
    }

    // CG on (H + Lambda) x = q; this lane tracks row `ri` of every vector.
    const int ri = warp + kWarps * row_of_lane<RPW>(lane);
    const bool contrib = (lane & (DUP - 1)) == 0;
    const float lam_i = lambda[(size_t)h * D + ri];
    int par = 0;
    // (H + Lambda) applied to the vector in sp, for row ri (sp must be
    // published by a barrier before the call)
    auto matvec_row = [&](float own) {
        float pc[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) pc[c] = col_ok ? sp[col0 + c] : 0.f;
        float part[RPW];
#pragma unroll
        for (int m = 0; m < RPW; ++m) {
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) acc = fmaf(Hr[m][c], pc[c], acc);
            part[m] = acc;
        }
        return fmaf(lam_i, own, butterfly_reduce<RPW>(part, lane));
    };
    const float q_i = sp[ri];
    float xi = 0.f, r_i = q_i;
    const float qq = block_sum(q_i * q_i, contrib, red, par, warp, lane);   // its barrier ends the reads of q
    const float qn = sqrtf(qq);
    float rr = qq;
    if (xs) {                                           // r0 = q - (H + Lambda) x0
        xi = xs[(size_t)bh * D + ri];
        if (contrib) sp[ri] = xi;
        __syncthreads();
        r_i = q_i - matvec_row(xi);
        rr = block_sum(r_i * r_i, contrib, red, par, warp, lane);          // its barrier ends the reads of x0
        if (contrib) sp[ri] = r_i;                      // p0 = r0
        __syncthreads();
    }
    float pi = r_i;
    int it = 0;
    for (int s = 0; s < cg_steps; ++s) {
        if (!cg_may_continue(rr, qn, tol)) break;   // block-uniform
        const float yi = matvec_row(pi);
        const float pAp = block_sum(pi * yi, contrib, red, par, warp, lane);
        if (!cg_curvature_ok(pAp)) break;
        const float alpha = rr / pAp;
        xi = fmaf(alpha, pi, xi);
        r_i = fmaf(-alpha, yi, r_i);
        const float rr_new = block_sum(r_i * r_i, contrib, red, par, warp, lane);
        pi = fmaf(rr_new / rr, pi, r_i);
        rr = rr_new;
        ++it;
        if (contrib) sp[ri] = pi;       // block_sum's barriers order this after all reads
        __syncthreads();
    }

    // G <- gamma G + beta v k^T (written back), out = G x.
    __syncthreads();
    if (contrib) sp[ri] = xi;
    asm volatile("cp.async.wait_all;\n" ::: "memory");
    __syncthreads();
    float xc[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) xc[c] = col_ok ? sp[col0 + c] : 0.f;
    float part[RPW];
#pragma unroll
    for (int m = 0; m < RPW; ++m) {
        const int i = warp + kWarps * m;
        const float bvi = bt * sv[i];
        float acc = 0.f;
        if (col_ok) {
            float gr[CPL];
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                gr[c] = fmaf(g, sG[i * D + col0 + c], bvi * kc[c]);
                acc = fmaf(gr[c], xc[c], acc);
            }
            float* row = Gm + (size_t)i * D + col0;
            if constexpr (CPL == 4) {
                *reinterpret_cast<float4*>(row) = make_float4(gr[0], gr[1], gr[2], gr[3]);
            } else {
#pragma unroll
                for (int c = 0; c < CPL; ++c) row[c] = gr[c];
            }
        }
        part[m] = acc;
    }
    const float oi = butterfly_reduce<RPW>(part, lane);
    if (contrib) out[(size_t)bh * D + ri] = oi;
    if (iters && tid == 0) iters[bh] = it;
    if (xs && contrib) xs[(size_t)bh * D + ri] = xi;
}

template <int D>
cudaError_t launch_step(const StepArgs& a, cudaStream_t st) {
    const size_t smem = sizeof(float) * ((size_t)D * D + 3 * D + 2 * kWarps);
    auto kern = step_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    {
        LaunchTimer timer(kKindStep, st);
        kern<<<a.B * a.H, kThreads, smem, st>>>(a.q, a.k, a.v, a.gamma, a.beta, a.lambda, a.H, a.Hs, a.Gs,
                                                a.cg_steps, a.tol, a.out, a.iters, a.xs);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t step_launch(const StepArgs& a, cudaStream_t st) {
    switch (a.dk) {
        case 16: return launch_step<16>(a, st);
        case 32: return launch_step<32>(a, st);
        case 64: return launch_step<64>(a, st);
        case 128: return launch_step<128>(a, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace mesa
