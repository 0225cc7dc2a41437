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
// (4 * 4 * d^2 bytes = 256 KiB at d = 128). A CTA of 8 warps serves one head
// at a time, and two CTAs per SM walk the heads (CTA i takes heads i,
// i + grid, ...):
//   * the H of the CTA's next head is copied into shared memory by one bulk
//     async copy while the CTA solves its current head, so the read of H is
//     off the critical path and the SM's two CTAs drift apart in phase,
//     which keeps HBM busy while either of them iterates;
//   * H is updated from that copy, written back, and kept in registers (warp
//     w owns rows w, w+8, ...; lane l owns columns l*CPL .. l*CPL+CPL-1), so
//     every CG matvec runs from registers;
//   * each matvec reduces its per-lane partial row sums with a butterfly
//     transpose-reduction (R rows over 32 lanes in R-1+log2(32/R)... shuffles)
//     instead of R full warp reductions; the block sums use a double-buffered
//     scratch, one barrier each, and the new residual rides on the barrier of
//     the r.r sum, so an iteration has two barriers;
//   * G is read once the CG ends, all of a thread's rows at once, updated,
//     written back and applied to x;
//   * with x_state the CG starts from the caller's guess (warm start; the
//     pages name warm starts as the way to cut the solver's cost, MesaNet
//     page, Significance and claims): r0 = q - (H + Lambda) x0, and the
//     solution is written back to x_state.
// The wait for a copy is bounded: if it runs out, the kernel records a
// timeout in the error word and stops.
#include "mesa_common.cuh"
#include "mesa_internal.h"
#include "tc_common.cuh"

namespace mesa {
namespace {

using namespace tc;

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
// The contributing lanes are those whose lane index is a multiple of DUP, so
// the butterfly stops at offset DUP: lane 0 then holds the warp's sum. The 8
// warp sums are read as two float4 (red is 16-byte aligned) and added as a tree.
template <int DUP>
__device__ __forceinline__ float block_sum(float v, bool contrib, float* red, int& par, int warp, int lane) {
    static_assert(kWarps == 8, "two float4 of warp sums");
    float s = contrib ? v : 0.f;
#pragma unroll
    for (int off = 16; off >= DUP; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    float* rb = red + par * kWarps;
    if (lane == 0) rb[warp] = s;
    __syncthreads();
    const float4 a = *reinterpret_cast<const float4*>(rb), b = *reinterpret_cast<const float4*>(rb + 4);
    par ^= 1;
    return ((a.x + a.y) + (a.z + a.w)) + ((b.x + b.y) + (b.z + b.w));
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
step_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
            const float* __restrict__ gamma, const float* __restrict__ beta,
            const float* __restrict__ lambda, int H, int nheads, float* __restrict__ Hs, float* __restrict__ Gs,
            int cg_steps, float tol, float* __restrict__ out, int32_t* __restrict__ iters,
            float* __restrict__ xs, unsigned* __restrict__ err) {
    constexpr int RPW = D / kWarps;                  // rows per warp
    constexpr int CPL = D >= 32 ? D / 32 : 1;        // columns per lane
    constexpr int DUP = 32 / RPW;                    // lanes sharing one row after the reduction
    constexpr uint32_t kStateBytes = (uint32_t)D * D * 4;
    static_assert(RPW >= 1 && (RPW & (RPW - 1)) == 0, "rows per warp must be a power of two");

    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem_raw);           // the H copy's barrier
    int* gave_up = reinterpret_cast<int*>(smem_raw + 8);              // a bounded wait ran out
    float* sH = reinterpret_cast<float*>(smem_raw + 16);              // D*D: this head's H, by bulk copy
    float* sk = sH + D * D;       // D
    float* sv = sk + D;           // D
    float* sp = sv + D;           // D (q, the warm start's x0 and r0, then x)
    float* sr = sp + D;           // D (the CG residual, published each iteration)
    float* red = sr + D;          // 2 x kWarps

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int col0 = lane * CPL;
    const bool col_ok = col0 < D;
    const bool contrib = (lane & (DUP - 1)) == 0;
    const int ri = warp + kWarps * row_of_lane<RPW>(lane);    // the row this lane tracks in the CG

    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        *gave_up = 0;
    }
    __syncthreads();
    // Each CTA walks heads blockIdx.x, blockIdx.x + gridDim.x, ...; the H of
    // its next head is copied into shared memory while it solves this one.
    int bh = blockIdx.x;
    if (tid == 0 && bh < nheads) {
        mbar_arrive_expect_tx(bar, kStateBytes);
        bulk_g2s(sH, Hs + (size_t)bh * D * D, kStateBytes, bar);
    }
    uint32_t parity = 0;
    for (; bh < nheads; bh += gridDim.x) {
        const int h = bh % H;
        float* Hm = Hs + (size_t)bh * D * D;
        float* Gm = Gs + (size_t)bh * D * D;
        for (int e = tid; e < D; e += kThreads) {        // the previous head's last reads ended at a barrier
            sk[e] = k[(size_t)bh * D + e];
            sv[e] = v[(size_t)bh * D + e];
            sp[e] = q[(size_t)bh * D + e];
        }
        const float g = gamma[bh], bt = beta[bh];
        if (tid == 0 && !mbar_wait(bar, parity)) *gave_up = 1;
        __syncthreads();
        if (*gave_up) break;                             // block-uniform
        parity ^= 1;

        // H <- gamma H + beta k k^T, written back and kept in registers.
        float kc[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) kc[c] = col_ok ? sk[col0 + c] : 0.f;
        float Hr[RPW][CPL];
#pragma unroll
        for (int m = 0; m < RPW; ++m) {
            const int i = warp + kWarps * m;
            const float bki = bt * sk[i];
            const float* srow = sH + i * D + col0;
            float* row = Hm + (size_t)i * D + col0;
            if (col_ok) {
                if constexpr (CPL == 4) {
                    float4 h4 = *reinterpret_cast<const float4*>(srow);
                    h4.x = fmaf(g, h4.x, bki * kc[0]);
                    h4.y = fmaf(g, h4.y, bki * kc[1]);
                    h4.z = fmaf(g, h4.z, bki * kc[2]);
                    h4.w = fmaf(g, h4.w, bki * kc[3]);
                    *reinterpret_cast<float4*>(row) = h4;
                    Hr[m][0] = h4.x; Hr[m][1] = h4.y; Hr[m][2] = h4.z; Hr[m][3] = h4.w;
                } else {
#pragma unroll
                    for (int c = 0; c < CPL; ++c) {
                        const float hv = fmaf(g, srow[c], bki * kc[c]);
                        row[c] = hv;
                        Hr[m][c] = hv;
                    }
                }
            } else {
#pragma unroll
                for (int c = 0; c < CPL; ++c) Hr[m][c] = 0.f;
            }
        }
        __syncthreads();                                 // every read of this head's H is done
        if (tid == 0 && bh + (int)gridDim.x < nheads) {  // the next head's H, during this head's CG
            fence_proxy_async();
            mbar_arrive_expect_tx(bar, kStateBytes);
            bulk_g2s(sH, Hs + (size_t)(bh + gridDim.x) * D * D, kStateBytes, bar);
        }

        // CG on (H + Lambda) x = q; this lane tracks row `ri` of every vector.
        const float lam_i = lambda[(size_t)h * D + ri];
        int par = 0;
        // (H + Lambda) applied to a vector whose columns col0.. this lane
        // holds in vc, for row ri (own = the vector's entry ri)
        auto matvec_row = [&](const float (&vc)[CPL], float own) {
            float part[RPW];
#pragma unroll
            for (int m = 0; m < RPW; ++m) {
                float acc = 0.f;
#pragma unroll
                for (int c = 0; c < CPL; ++c) acc = fmaf(Hr[m][c], vc[c], acc);
                part[m] = acc;
            }
            return fmaf(lam_i, own, butterfly_reduce<RPW>(part, lane));
        };
        // Every lane keeps two views of the direction p: entry ri (pi), and
        // its matvec columns col0.. (pc). Both follow p = r + (rr_new / rr) p
        // with the same operands, so they stay equal bit for bit; the new
        // residual reaches the column view through sr, which the barrier of
        // the r.r sum publishes. One barrier per block sum, two per iteration.
        float pc[CPL];
        const float q_i = sp[ri];
#pragma unroll
        for (int c = 0; c < CPL; ++c) pc[c] = col_ok ? sp[col0 + c] : 0.f;
        float xi = 0.f, r_i = q_i;
        const float qq = block_sum<DUP>(q_i * q_i, contrib, red, par, warp, lane);   // its barrier ends the reads of q
        const float qn = sqrtf(qq);
        float rr = qq;
        if (xs) {                                           // r0 = q - (H + Lambda) x0
            xi = xs[(size_t)bh * D + ri];
            if (contrib) sp[ri] = xi;
            __syncthreads();
            float xc0[CPL];
#pragma unroll
            for (int c = 0; c < CPL; ++c) xc0[c] = col_ok ? sp[col0 + c] : 0.f;
            r_i = q_i - matvec_row(xc0, xi);
            if (contrib) sr[ri] = r_i;
            rr = block_sum<DUP>(r_i * r_i, contrib, red, par, warp, lane);          // publishes r0 in sr
#pragma unroll
            for (int c = 0; c < CPL; ++c) pc[c] = col_ok ? sr[col0 + c] : 0.f;   // p0 = r0
        }
        float pi = r_i;
        int it = 0;
        for (int s = 0; s < cg_steps; ++s) {
            if (!cg_may_continue(rr, qn, tol)) break;   // block-uniform
            const float yi = matvec_row(pc, pi);
            const float pAp = block_sum<DUP>(pi * yi, contrib, red, par, warp, lane);   // also ends the reads of sr
            if (!cg_curvature_ok(pAp)) break;
            // alpha and rho feed recurrences that CG corrects: the fast
            // division (a few ulp) suffices and is off the chain's critical
            // path sooner than the IEEE one
            const float alpha = __fdividef(rr, pAp);
            xi = fmaf(alpha, pi, xi);
            r_i = fmaf(-alpha, yi, r_i);
            if (contrib) sr[ri] = r_i;
            const float rr_new = block_sum<DUP>(r_i * r_i, contrib, red, par, warp, lane);   // publishes sr
            const float rho = __fdividef(rr_new, rr);
            pi = fmaf(rho, pi, r_i);
#pragma unroll
            for (int c = 0; c < CPL; ++c) pc[c] = col_ok ? fmaf(rho, pc[c], sr[col0 + c]) : 0.f;
            rr = rr_new;
            ++it;
        }

        // G <- gamma G + beta v k^T (written back), out = G x. The rows of G are
        // read straight from global memory, all of this thread's at once.
        __syncthreads();
        if (contrib) sp[ri] = xi;
        float gr[RPW][CPL];
#pragma unroll
        for (int m = 0; m < RPW; ++m) {
            const float* row = Gm + (size_t)(warp + kWarps * m) * D + col0;
            if (col_ok) {
                if constexpr (CPL == 4) {
                    const float4 g4 = *reinterpret_cast<const float4*>(row);
                    gr[m][0] = g4.x; gr[m][1] = g4.y; gr[m][2] = g4.z; gr[m][3] = g4.w;
                } else {
#pragma unroll
                    for (int c = 0; c < CPL; ++c) gr[m][c] = row[c];
                }
            }
        }
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
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    gr[m][c] = fmaf(g, gr[m][c], bvi * kc[c]);
                    acc = fmaf(gr[m][c], xc[c], acc);
                }
                float* row = Gm + (size_t)i * D + col0;
                if constexpr (CPL == 4) {
                    *reinterpret_cast<float4*>(row) = make_float4(gr[m][0], gr[m][1], gr[m][2], gr[m][3]);
                } else {
#pragma unroll
                    for (int c = 0; c < CPL; ++c) row[c] = gr[m][c];
                }
            }
            part[m] = acc;
        }
        const float oi = butterfly_reduce<RPW>(part, lane);
        if (contrib) out[(size_t)bh * D + ri] = oi;
        if (iters && tid == 0) iters[bh] = it;
        if (xs && contrib) xs[(size_t)bh * D + ri] = xi;
        __syncthreads();                                 // sk, sv, sp are rewritten for the next head
    }
    if (*gave_up && tid == 0) {
        record_error(err, kErrTimeout);
        mbar_wait(bar, parity);                          // one more bounded chance for the copy to land
    }
}

// Dynamic shared memory of step_kernel<D>: the barrier and flag (16 bytes),
// one D x D state, k, v, the two CG vectors and the reduction scratch.
template <int D>
constexpr size_t step_smem_bytes() {
    return 16 + sizeof(float) * ((size_t)D * D + 4 * D + 2 * kWarps);
}

template <int D>
cudaError_t launch_step(const StepArgs& a, cudaStream_t st) {
    const size_t smem = step_smem_bytes<D>();
    auto kern = step_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int nheads = a.B * a.H;
    const int grid = nheads < 2 * sms ? nheads : 2 * sms;     // two resident CTAs per SM
    {
        LaunchTimer timer(kKindStep, st);
        kern<<<grid, kThreads, smem, st>>>(a.q, a.k, a.v, a.gamma, a.beta, a.lambda, a.H, nheads, a.Hs, a.Gs,
                                           a.cg_steps, a.tol, a.out, a.iters, a.xs, error_word_ptr());
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
