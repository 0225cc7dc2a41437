// tc_forward.cu -- tensor-core (tcgen05) chunkwise forward of the Mesa layer
// for bf16 inputs, dk = dv = 128, chunk C = 64.
//
// Method: "MesaNet: Sequence Modeling by Locally Optimal Test-Time Training"
// (gist.science), Technical summary > Method > Mesa layer and its
// "Parallelisation" paragraph (every CG matvec of a chunk is a gated linear
// attention pass over a carried d x d state plus a decay-masked intra-chunk
// term). With b_t the in-chunk log-cumsum of gamma, M_tj = beta_j e^{b_t-b_j}
// (j <= t), chunk-start state H_c and a CG direction matrix P (one row per
// token of the chunk):
//     Y = diag(e^b) P H_c^T + (M o P K^T) K + P diag(lambda)
//     O = diag(e^b) X G_c^T + (M o X K^T) V
//     H_{c+1} = e^{b_last} H_c + K^T diag(w) K,  w_j = beta_j e^{b_last-b_j}
//
// Numerics. Every tensor-core operand is fp16 (same tensor rate as bf16,
// 8x finer rounding), accumulation is fp32:
//   * bf16 q, k, v convert exactly to fp16 (normalised keys and queries are
//     far inside the fp16 range; v is scaled per chunk by a power of two);
//   * the chunk-start states are stored as fp16 images scaled per chunk by a
//     power of two s >= 1 (so |H/s| <= 1);
//   * the CG direction of each token is scaled by 1/|r| before rounding, so
//     its fp16 image has unit-order entries; every CG vector (x, r, p) and
//     scalar stays fp32;
//   * the scan splits beta_j e^{b_last-b_j} k_j into an fp16 hi/lo pair, so
//     the fp32 running states carry ~22-bit products.
//
// Kernels:
//   tc_scan_kernel  grid (2, B*H): CTA (m, bh) walks the chunks of sequence bh
//                   for m = 0 (H) or 1 (G). Per chunk one M=128,N=128,K=128
//                   MMA forms the weighted outer-product sum in TMEM; the
//                   running fp32 state lives in registers (thread: one row,
//                   64 columns) and each chunk-start state is written as a
//                   swizzled fp16 image ready to be a shared-memory operand.
//   tc_cg_kernel    grid (chunks, B*H), 2 CTAs per SM: one CTA runs every CG
//                   iteration of one chunk and the read-out. Tokens are the
//                   MMA M dimension (M = 64), so each token's CG vectors sit
//                   in the registers of 8 threads and every dot product is a
//                   thread-local sum plus a 4-lane shuffle and one shared-
//                   memory exchange. x lives in TMEM.
#include "mesa_common.cuh"
#include "mesa_internal.h"
#include "tc_common.cuh"

namespace mesa {
namespace {

using namespace tc;

constexpr int kD = 128;          // dk = dv
constexpr int kC = 64;           // chunk length
constexpr int kThreads = 256;
constexpr uint32_t kImgBytes = kD * kD * 2;      // one fp16 state image
constexpr size_t kImgHalves = (size_t)kD * kD;

// Power of two >= max(m, 1).
__device__ __forceinline__ float pow2_ceil_at_least_one(float m) {
    if (!(m > 1.f)) return 1.f;
    int e;
    const float f = frexpf(m, &e);       // m = f * 2^e, f in [0.5, 1)
    return ldexpf(1.f, f == 0.5f ? e - 1 : e);
}

// Inclusive log-cumsum of gamma over a 64-token chunk by warp 0 (padded
// tokens count as gamma = 1).
__device__ __forceinline__ void chunk_gates(const float* __restrict__ gamma, size_t base, int n, float* b) {
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    const int t0 = 2 * lane, t1 = 2 * lane + 1;
    const float l0 = (t0 < n) ? logf(gamma[base + t0]) : 0.f;
    const float l1 = (t1 < n) ? logf(gamma[base + t1]) : 0.f;
    const float pair = l0 + l1;
    float incl = pair;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    const float excl = incl - pair;
    b[t0] = excl + l0;
    b[t1] = excl + l0 + l1;
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

// =====================================================================
// Chunk-state scan
// =====================================================================
struct ScanSmem {
    static constexpr int oAhi = 0;                // MN-major [64 j][128 i] fp16, 16 KB
    static constexpr int oAlo = 16384;
    static constexpr int oB = 32768;              // keys, MN-major [64 j][128 k]
    static constexpr int oGate = 49152;           // b[64], w[64]
    static constexpr int oRed = oGate + 512;      // 8 floats
    static constexpr int oBar = oRed + 64;        // mbarrier
    static constexpr int oSlot = oBar + 16;
    static constexpr int bytes = oSlot + 16;
};

__global__ void __launch_bounds__(kThreads, 2)
tc_scan_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
               const float* __restrict__ gamma, const float* __restrict__ beta, int T, int nc,
               const float* __restrict__ H_in, const float* __restrict__ G_in, __half* __restrict__ img,
               float* __restrict__ scales, float* __restrict__ H_out, float* __restrict__ G_out,
               unsigned* __restrict__ err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* Ahi = smem + ScanSmem::oAhi;
    uint8_t* Alo = smem + ScanSmem::oAlo;
    uint8_t* Bk = smem + ScanSmem::oB;
    float* sb = reinterpret_cast<float*>(smem + ScanSmem::oGate);
    float* sw = sb + kC;
    float* red = reinterpret_cast<float*>(smem + ScanSmem::oRed);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + ScanSmem::oBar);
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + ScanSmem::oSlot);

    const int m = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int q4 = w & 3, hh = w >> 2;
    const int row = 32 * q4 + lane;               // state row owned by this thread
    const int col0 = 64 * hh;                     // its 64 columns (one K block of the image)
    const __nv_bfloat16* A = m ? v : k;
    const float* init = m ? G_in : H_in;
    float* fin = m ? G_out : H_out;

    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    if (w == 0) tmem_alloc(slot, 128);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *slot;

    float S[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) S[i] = 0.f;
    if (init) {
        const float4* src = reinterpret_cast<const float4*>(init + ((size_t)bh * kD + row) * kD + col0);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float4 f = src[i];
            S[4 * i] = f.x; S[4 * i + 1] = f.y; S[4 * i + 2] = f.z; S[4 * i + 3] = f.w;
        }
    }

    constexpr uint32_t kIdesc = idesc_f16(128, 128, true, true);
    bool ok = true;
    for (int c = 0; c <= nc; ++c) {
        // ---- emit the state before chunk c: fp16 image + scale (or the final fp32 state) ----
        float mx = 0.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) mx = fmaxf(mx, fabsf(S[i]));
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) red[w] = mx;
        __syncthreads();
        if (c < nc) {
            float gm = red[0];
#pragma unroll
            for (int i = 1; i < 8; ++i) gm = fmaxf(gm, red[i]);
            const float s = pow2_ceil_at_least_one(gm);
            const float inv = 1.f / s;
            const size_t ci = ((size_t)bh * nc + c) * 2 + m;
            if (tid == 0) scales[ci] = s;
            uint8_t* dst = reinterpret_cast<uint8_t*>(img + ci * kImgHalves) + hh * 16384 + row * 128;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                uint4 o;
                o.x = pack_half2(S[8 * g] * inv, S[8 * g + 1] * inv);
                o.y = pack_half2(S[8 * g + 2] * inv, S[8 * g + 3] * inv);
                o.z = pack_half2(S[8 * g + 4] * inv, S[8 * g + 5] * inv);
                o.w = pack_half2(S[8 * g + 6] * inv, S[8 * g + 7] * inv);
                *reinterpret_cast<uint4*>(dst + ((g ^ (row & 7)) << 4)) = o;
            }
        } else {
            if (fin) {
                float4* d4 = reinterpret_cast<float4*>(fin + ((size_t)bh * kD + row) * kD + col0);
#pragma unroll
                for (int i = 0; i < 16; ++i) d4[i] = make_float4(S[4 * i], S[4 * i + 1], S[4 * i + 2], S[4 * i + 3]);
            }
            break;
        }

        // ---- gates of chunk c ----
        const int t0 = c * kC;
        const int n = min(kC, T - t0);
        const size_t base = (size_t)bh * T + t0;
        chunk_gates(gamma, base, n, sb);
        __syncthreads();
        const float blast = sb[kC - 1];
        if (tid < kC) sw[tid] = (tid < n) ? beta[base + tid] * expf(blast - sb[tid]) : 0.f;
        __syncthreads();

        // ---- operand images: A = w_j a_j (hi/lo), B = k_j, both [j][d] ----
#pragma unroll
        for (int rep = 0; rep < 4; ++rep) {
            const int cid = tid + kThreads * rep;          // 1024 16-byte chunks
            const int j = cid >> 4, cc = cid & 15;
            uint4 ra = make_uint4(0, 0, 0, 0), rk = make_uint4(0, 0, 0, 0);
            if (j < n) {
                ra = *reinterpret_cast<const uint4*>(A + (base + j) * kD + 8 * cc);
                rk = *reinterpret_cast<const uint4*>(k + (base + j) * kD + 8 * cc);
            }
            const float wj = sw[j];
            const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&ra);
            uint4 hi, lo;
            uint32_t* hw = reinterpret_cast<uint32_t*>(&hi);
            uint32_t* lw = reinterpret_cast<uint32_t*>(&lo);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(a2[i]);
                const float x0 = wj * f.x, x1 = wj * f.y;
                const __half2 h2 = __floats2half2_rn(x0, x1);
                const float2 hb = __half22float2(h2);
                hw[i] = *reinterpret_cast<const uint32_t*>(&h2);
                lw[i] = pack_half2(x0 - hb.x, x1 - hb.y);
            }
            const uint32_t off = (uint32_t)((cc >> 3) * 8192 + j * 128 + (((cc & 7) ^ (j & 7)) << 4));
            *reinterpret_cast<uint4*>(Ahi + off) = hi;
            *reinterpret_cast<uint4*>(Alo + off) = lo;
            *reinterpret_cast<uint4*>(Bk + off) = bf16x8_to_f16x8(rk, 1.f);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- Delta = A^T B over the chunk (K = 64 tokens, hi then lo) ----
        if (tid == 0) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint8_t* Asrc = (ks < 4) ? Ahi : Alo;
                const int kk = ks & 3;
                mma_f16(tbase, sdesc(smem_addr(Asrc) + kk * 2048, 8192, 1024),
                        sdesc(smem_addr(Bk) + kk * 2048, 8192, 1024), kIdesc, ks > 0 ? 1u : 0u);
            }
            mma_commit(bar);
        }
        ok = mbar_wait(bar, c & 1) && ok;
        const int all_ok = __syncthreads_and(ok ? 1 : 0);
        tc_fence_after();
        if (!all_ok) break;

        // ---- S <- e^{b_last} S + Delta ----
        const float Gam = expf(blast);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float dv[32];
            tmem_ld32_x32(tbase + ((uint32_t)(32 * q4) << 16) + col0 + 32 * half, dv);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) S[32 * half + i] = fmaf(Gam, S[32 * half + i], dv[i]);
        }
        tc_fence_before();
        __syncthreads();       // TMEM and the operand images are free for the next chunk
        tc_fence_after();
    }

    if (!__syncthreads_and(ok)) {
        if (tid == 0) record_error(err, kErrTimeout);
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tbase, 128);
}

// =====================================================================
// Fused CG iterations + read-out, one chunk per CTA
// =====================================================================
struct CgSmem {
    static constexpr int oH = 0;                  // H_c image, later G_c   32 KB
    static constexpr int oK = 32768;              // key image, later value image   16 KB
    static constexpr int oP = 49152;              // P-hat image, later X-hat  16 KB
    static constexpr int oPt = 65536;             // P-tilde image, later X-tilde  16 KB
    static constexpr int oW = 81920;              // masked scores image  8 KB
    static constexpr int kMStride = 72;           // padded row stride of the decay mask
    static constexpr int oM = 90112;              // decay mask fp32 [64][72]
    static constexpr int oLam = oM + kC * kMStride * 4;   // lambda [128]
    static constexpr int oEb = oLam + 512;        // e^{b_t} [64]
    static constexpr int oB = oEb + 256;          // b_t [64]
    static constexpr int oRed = oB + 256;         // [2 buffers][2 halves][64 tokens]
    static constexpr int oMisc = oRed + 1024;     // 16 floats
    static constexpr int oBar = oMisc + 64;        // 2 mbarriers
    static constexpr int oSlot = oBar + 16;
    static constexpr int bytes = oSlot + 16;
};

// Sum over the 8 threads that hold one token (4 lanes x 2 column halves).
__device__ __forceinline__ void token_sum2(float& a0, float& a1, float* redbuf, int hh, int tok0, int tok1,
                                           int lane) {
    a0 += __shfl_xor_sync(0xffffffffu, a0, 1);
    a0 += __shfl_xor_sync(0xffffffffu, a0, 2);
    a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
    a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
    if ((lane & 3) == 0) {
        redbuf[hh * 64 + tok0] = a0;
        redbuf[hh * 64 + tok1] = a1;
    }
    __syncthreads();
    a0 = redbuf[tok0] + redbuf[64 + tok0];
    a1 = redbuf[tok1] + redbuf[64 + tok1];
}

// Writes this thread's two tokens x 16 columns of a [64 t][128 k] fp16 image.
__device__ __forceinline__ void store_rows(uint8_t* imgbase, int hh, int tok0, int tok1, int lane,
                                           const float (&v0)[16], const float (&v1)[16], float s0, float s1) {
    uint8_t* blk = imgbase + hh * 8192;
    const int cw = 4 * (lane & 3);
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        *reinterpret_cast<uint32_t*>(blk + tok0 * 128 + ((g ^ (tok0 & 7)) << 4) + cw) =
            pack_half2(v0[2 * g] * s0, v0[2 * g + 1] * s0);
        *reinterpret_cast<uint32_t*>(blk + tok1 * 128 + ((g ^ (tok1 & 7)) << 4) + cw) =
            pack_half2(v1[2 * g] * s1, v1[2 * g + 1] * s1);
    }
}

__global__ void __launch_bounds__(kThreads, 2)
tc_cg_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
             const __nv_bfloat16* __restrict__ v, const float* __restrict__ gamma,
             const float* __restrict__ beta, const float* __restrict__ lambda, int H, int T, int nc,
             int cg_steps, float tol, const __half* __restrict__ img, const float* __restrict__ scales,
             float* __restrict__ out, int32_t* __restrict__ iters, unsigned* __restrict__ err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* Hs = smem + CgSmem::oH;
    uint8_t* Ks = smem + CgSmem::oK;
    uint8_t* Ps = smem + CgSmem::oP;
    uint8_t* Pt = smem + CgSmem::oPt;
    uint8_t* Ws = smem + CgSmem::oW;
    float* Mk = reinterpret_cast<float*>(smem + CgSmem::oM);
    float* slam = reinterpret_cast<float*>(smem + CgSmem::oLam);
    float* seb = reinterpret_cast<float*>(smem + CgSmem::oEb);
    float* sbc = reinterpret_cast<float*>(smem + CgSmem::oB);
    float* red = reinterpret_cast<float*>(smem + CgSmem::oRed);
    float* misc = reinterpret_cast<float*>(smem + CgSmem::oMisc);
    uint64_t* bar_ld = reinterpret_cast<uint64_t*>(smem + CgSmem::oBar);
    uint64_t* bar_mma = bar_ld + 1;
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + CgSmem::oSlot);

    const int c = blockIdx.x, bh = blockIdx.y, head = bh % H;
    const int t0 = c * kC;
    const int n = min(kC, T - t0);
    const size_t base = (size_t)bh * T + t0;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int q4 = w & 3, hh = w >> 2;
    const int tok0 = 16 * q4 + (lane >> 2), tok1 = tok0 + 8;
    const int cb = 64 * hh + 2 * (lane & 3);      // column of (group g, e): cb + 8g + e
    const size_t ci = (size_t)bh * nc + c;
    const __half* Himg = img + (ci * 2 + 0) * kImgHalves;
    const __half* Gimg = img + (ci * 2 + 1) * kImgHalves;

    // ---- set-up: barriers, TMEM, async load of the H_c image ----
    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        misc[15] = 0.f;                          // abort flag: set by a thread whose wait gave up
    }
    if (w == 0) tmem_alloc(slot, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *slot;
    const uint32_t tq = tbase + ((uint32_t)(32 * q4) << 16);    // this warp's lane quadrant
    if (tid == 0) {
        mbar_arrive_expect_tx(bar_ld, kImgBytes);
        bulk_g2s(Hs, Himg, kImgBytes, bar_ld);
    }

    // gates and decay mask
    chunk_gates(gamma, base, n, sbc);
    for (int d = tid; d < kD; d += kThreads) slam[d] = lambda[(size_t)head * kD + d];
    // key image (bf16 -> fp16 is exact for normalised keys)
#pragma unroll
    for (int rep = 0; rep < 4; ++rep) {
        const int cid = tid + kThreads * rep;
        const int j = cid >> 4, cc = cid & 15;
        uint4 rk = make_uint4(0, 0, 0, 0);
        if (j < n) rk = *reinterpret_cast<const uint4*>(k + (base + j) * kD + 8 * cc);
        *reinterpret_cast<uint4*>(Ks + (cc >> 3) * 8192 + j * 128 + (((cc & 7) ^ (j & 7)) << 4)) =
            bf16x8_to_f16x8(rk, 1.f);
    }
    __syncthreads();
    if (tid < kC) seb[tid] = expf(sbc[tid]);
    for (int e = tid; e < kC * kC; e += kThreads) {
        const int tt = e >> 6, j = e & 63;
        Mk[tt * CgSmem::kMStride + j] = (j <= tt && tt < n) ? beta[base + j] * expf(sbc[tt] - sbc[j]) : 0.f;
    }

    // CG state: x = 0 (TMEM), r = p = q; this thread holds 2 tokens x 16 columns
    float r0[16], r1[16], p0[16], p1[16];
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        const int col = cb + 8 * g;
        float2 a = make_float2(0.f, 0.f), b = make_float2(0.f, 0.f);
        if (tok0 < n) a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(q + (base + tok0) * kD + col));
        if (tok1 < n) b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(q + (base + tok1) * kD + col));
        r0[2 * g] = a.x; r0[2 * g + 1] = a.y;
        r1[2 * g] = b.x; r1[2 * g + 1] = b.y;
        p0[2 * g] = a.x; p0[2 * g + 1] = a.y;
        p1[2 * g] = b.x; p1[2 * g + 1] = b.y;
    }
    {
        float z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0.f;
        tmem_st16_x8(tq + 128 + 64 * hh, z);
        tmem_wait_st();
    }
    float rr0 = 0.f, rr1 = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        rr0 = fmaf(r0[i], r0[i], rr0);
        rr1 = fmaf(r1[i], r1[i], rr1);
    }
    int rb = 0;   // alternating reduction buffer
    token_sum2(rr0, rr1, red + 128 * rb, hh, tok0, tok1, lane);
    rb ^= 1;
    const float qn0 = sqrtf(rr0), qn1 = sqrtf(rr1);
    bool act0 = tok0 < n, act1 = tok1 < n;
    int it0 = 0, it1 = 0;
    const float eb0 = seb[tok0], eb1 = seb[tok1];
    float s0 = rr0 > 0.f ? sqrtf(rr0) : 1.f, s1 = rr1 > 0.f ? sqrtf(rr1) : 1.f;
    store_rows(Ps, hh, tok0, tok1, lane, p0, p1, 1.f / s0, 1.f / s1);
    store_rows(Pt, hh, tok0, tok1, lane, p0, p1, eb0 / s0, eb1 / s1);

    bool ok = mbar_wait(bar_ld, 0);
    const float sH = scales[ci * 2 + 0], sG = scales[ci * 2 + 1];
    const float inv_sH = 1.f / sH;
    uint32_t mma_phase = 0;
    constexpr uint32_t kIdS = idesc_f16(64, 64, false, false);
    constexpr uint32_t kIdU = idesc_f16(64, 128, false, false);
    constexpr uint32_t kIdZ = idesc_f16(64, 128, false, true);
    float wsc = inv_sH;     // scale folded into the masked scores (1/sH in CG, sV/sG in the read-out)

    for (int step = 0; step < cg_steps; ++step) {
        act0 = act0 && cg_may_continue(rr0, qn0, tol);
        act1 = act1 && cg_may_continue(rr1, qn1, tol);
        if (!ok) misc[15] = 1.f;
        fence_proxy_async();
        tc_fence_before();
        const int any = __syncthreads_or((act0 || act1) ? 1 : 0);
        tc_fence_after();
        if (!any || misc[15] != 0.f) break;      // uniform: every thread reads the same flag

        // S = P-hat K^T  (M=64 tokens, N=64 keys, K=128)
        if (tid == 0 && ok) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t ko = (ks >> 2) * 8192 + (ks & 3) * 32;
                mma_f16(tbase, sdesc(smem_addr(Ps) + ko, 16, 1024), sdesc(smem_addr(Ks) + ko, 16, 1024), kIdS,
                        ks > 0 ? 1u : 0u);
            }
            mma_commit(bar_mma);
        }
        ok = mbar_wait(bar_mma, mma_phase & 1) && ok;
        ++mma_phase;
        tc_fence_after();
        {
            float sv[16];
            tmem_ld16_x4(tq + 32 * hh, sv);
            tmem_wait_ld();
            const int cw = 4 * (lane & 3);
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const int j = 32 * hh + 8 * g + 2 * (lane & 3);
                const float2 m0 = *reinterpret_cast<const float2*>(Mk + tok0 * CgSmem::kMStride + j);
                const float2 m1 = *reinterpret_cast<const float2*>(Mk + tok1 * CgSmem::kMStride + j);
                const int chunk = (4 * hh + g);
                *reinterpret_cast<uint32_t*>(Ws + tok0 * 128 + ((chunk ^ (tok0 & 7)) << 4) + cw) =
                    pack_half2(m0.x * sv[4 * g] * wsc, m0.y * sv[4 * g + 1] * wsc);
                *reinterpret_cast<uint32_t*>(Ws + tok1 * 128 + ((chunk ^ (tok1 & 7)) << 4) + cw) =
                    pack_half2(m1.x * sv[4 * g + 2] * wsc, m1.y * sv[4 * g + 3] * wsc);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // Y = P-tilde H^T + W K   (M=64, N=128)
        if (tid == 0 && ok) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t ka = (ks >> 2) * 8192 + (ks & 3) * 32;
                const uint32_t kb = (ks >> 2) * 16384 + (ks & 3) * 32;
                mma_f16(tbase, sdesc(smem_addr(Pt) + ka, 16, 1024), sdesc(smem_addr(Hs) + kb, 16, 1024), kIdU,
                        ks > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_f16(tbase, sdesc(smem_addr(Ws) + ks * 32, 16, 1024),
                        sdesc(smem_addr(Ks) + ks * 2048, 8192, 1024), kIdZ, 1u);
            mma_commit(bar_mma);
        }
        ok = mbar_wait(bar_mma, mma_phase & 1) && ok;
        ++mma_phase;
        tc_fence_after();

        float yv[32];
        tmem_ld16_x8(tq + 64 * hh, yv);
        tmem_wait_ld();
        const float ys0 = s0 * sH, ys1 = s1 * sH;
        float pa0 = 0.f, pa1 = 0.f;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            const float2 lm = *reinterpret_cast<const float2*>(slam + cb + 8 * g);
            yv[4 * g + 0] = fmaf(yv[4 * g + 0], ys0, lm.x * p0[2 * g]);
            yv[4 * g + 1] = fmaf(yv[4 * g + 1], ys0, lm.y * p0[2 * g + 1]);
            yv[4 * g + 2] = fmaf(yv[4 * g + 2], ys1, lm.x * p1[2 * g]);
            yv[4 * g + 3] = fmaf(yv[4 * g + 3], ys1, lm.y * p1[2 * g + 1]);
            pa0 = fmaf(p0[2 * g], yv[4 * g], fmaf(p0[2 * g + 1], yv[4 * g + 1], pa0));
            pa1 = fmaf(p1[2 * g], yv[4 * g + 2], fmaf(p1[2 * g + 1], yv[4 * g + 3], pa1));
        }
        token_sum2(pa0, pa1, red + 128 * rb, hh, tok0, tok1, lane);
        rb ^= 1;
        if (act0 && !cg_curvature_ok(pa0)) act0 = false;
        if (act1 && !cg_curvature_ok(pa1)) act1 = false;
        const float al0 = act0 ? rr0 / pa0 : 0.f, al1 = act1 ? rr1 / pa1 : 0.f;
        float rn0 = 0.f, rn1 = 0.f;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                if (act0) r0[2 * g + e] = fmaf(-al0, yv[4 * g + e], r0[2 * g + e]);
                if (act1) r1[2 * g + e] = fmaf(-al1, yv[4 * g + 2 + e], r1[2 * g + e]);
                rn0 = fmaf(r0[2 * g + e], r0[2 * g + e], rn0);
                rn1 = fmaf(r1[2 * g + e], r1[2 * g + e], rn1);
            }
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {   // x += alpha p (x in TMEM, same layout as Y)
            float xv[16];
            const uint32_t xa = tq + 128 + 64 * hh + 32 * half;
            tmem_ld16_x4(xa, xv);
            tmem_wait_ld();
#pragma unroll
            for (int g = 0; g < 4; ++g) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int pi = 2 * (4 * half + g) + e;
                    if (act0) xv[4 * g + e] = fmaf(al0, p0[pi], xv[4 * g + e]);
                    if (act1) xv[4 * g + 2 + e] = fmaf(al1, p1[pi], xv[4 * g + 2 + e]);
                }
            }
            tmem_st16_x4(xa, xv);
            tmem_wait_st();
        }
        token_sum2(rn0, rn1, red + 128 * rb, hh, tok0, tok1, lane);
        rb ^= 1;
        if (act0) {
            const float rho = rn0 / rr0;
#pragma unroll
            for (int i = 0; i < 16; ++i) p0[i] = fmaf(rho, p0[i], r0[i]);
            rr0 = rn0;
            ++it0;
            s0 = rr0 > 0.f ? sqrtf(rr0) : 1.f;
        }
        if (act1) {
            const float rho = rn1 / rr1;
#pragma unroll
            for (int i = 0; i < 16; ++i) p1[i] = fmaf(rho, p1[i], r1[i]);
            rr1 = rn1;
            ++it1;
            s1 = rr1 > 0.f ? sqrtf(rr1) : 1.f;
        }
        store_rows(Ps, hh, tok0, tok1, lane, p0, p1, 1.f / s0, 1.f / s1);
        store_rows(Pt, hh, tok0, tok1, lane, p0, p1, eb0 / s0, eb1 / s1);
    }

    // ---- read-out: o = e^{b_t} G_c x + (M o X K^T) V ----
    float xr0[16], xr1[16];
    {
        float xv[32];
        tmem_ld16_x8(tq + 128 + 64 * hh, xv);
        tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            xr0[2 * g] = xv[4 * g]; xr0[2 * g + 1] = xv[4 * g + 1];
            xr1[2 * g] = xv[4 * g + 2]; xr1[2 * g + 1] = xv[4 * g + 3];
        }
    }
    float xx0 = 0.f, xx1 = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        xx0 = fmaf(xr0[i], xr0[i], xx0);
        xx1 = fmaf(xr1[i], xr1[i], xx1);
    }
    // the values of the chunk, scaled by a power of two so fp16 holds them
    uint4 vraw[4];
    float vmax = 0.f;
#pragma unroll
    for (int rep = 0; rep < 4; ++rep) {
        const int cid = tid + kThreads * rep;
        const int j = cid >> 4, cc = cid & 15;
        vraw[rep] = make_uint4(0, 0, 0, 0);
        if (j < n) vraw[rep] = *reinterpret_cast<const uint4*>(v + (base + j) * kD + 8 * cc);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&vraw[rep]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(b2[i]);
            vmax = fmaxf(vmax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, off));
    if (lane == 0) misc[w] = vmax;
    token_sum2(xx0, xx1, red + 128 * rb, hh, tok0, tok1, lane);   // its barrier also publishes misc[]
    rb ^= 1;
    float vm = misc[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) vm = fmaxf(vm, misc[i]);
    const float sV = pow2_ceil_at_least_one(vm);
    const float xs0 = xx0 > 0.f ? sqrtf(xx0) : 1.f, xs1 = xx1 > 0.f ? sqrtf(xx1) : 1.f;
    store_rows(Ps, hh, tok0, tok1, lane, xr0, xr1, 1.f / xs0, 1.f / xs1);
    store_rows(Pt, hh, tok0, tok1, lane, xr0, xr1, eb0 / xs0, eb1 / xs1);
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        // every MMA that read the H image has completed: reuse its buffer for G_c
        mbar_arrive_expect_tx(bar_ld, kImgBytes);
        bulk_g2s(Hs, Gimg, kImgBytes, bar_ld);
        // S' = X-hat K^T
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t ko = (ks >> 2) * 8192 + (ks & 3) * 32;
            mma_f16(tbase, sdesc(smem_addr(Ps) + ko, 16, 1024), sdesc(smem_addr(Ks) + ko, 16, 1024), kIdS,
                    ks > 0 ? 1u : 0u);
        }
        mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, mma_phase & 1) && ok;
    ++mma_phase;
    tc_fence_after();
    wsc = sV / sG;
    {
        float sv[16];
        tmem_ld16_x4(tq + 32 * hh, sv);
        tmem_wait_ld();
        const int cw = 4 * (lane & 3);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int j = 32 * hh + 8 * g + 2 * (lane & 3);
            const float2 m0 = *reinterpret_cast<const float2*>(Mk + tok0 * CgSmem::kMStride + j);
            const float2 m1 = *reinterpret_cast<const float2*>(Mk + tok1 * CgSmem::kMStride + j);
            const int chunk = (4 * hh + g);
            *reinterpret_cast<uint32_t*>(Ws + tok0 * 128 + ((chunk ^ (tok0 & 7)) << 4) + cw) =
                pack_half2(m0.x * sv[4 * g] * wsc, m0.y * sv[4 * g + 1] * wsc);
            *reinterpret_cast<uint32_t*>(Ws + tok1 * 128 + ((chunk ^ (tok1 & 7)) << 4) + cw) =
                pack_half2(m1.x * sv[4 * g + 2] * wsc, m1.y * sv[4 * g + 3] * wsc);
        }
    }
    // the key image is dead (S' done): overwrite it with the value image
    const float inv_sV = 1.f / sV;
#pragma unroll
    for (int rep = 0; rep < 4; ++rep) {
        const int cid = tid + kThreads * rep;
        const int j = cid >> 4, cc = cid & 15;
        *reinterpret_cast<uint4*>(Ks + (cc >> 3) * 8192 + j * 128 + (((cc & 7) ^ (j & 7)) << 4)) =
            bf16x8_to_f16x8(vraw[rep], inv_sV);
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    ok = mbar_wait(bar_ld, 1) && ok;
    if (tid == 0 && ok) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t ka = (ks >> 2) * 8192 + (ks & 3) * 32;
            const uint32_t kb = (ks >> 2) * 16384 + (ks & 3) * 32;
            mma_f16(tbase, sdesc(smem_addr(Pt) + ka, 16, 1024), sdesc(smem_addr(Hs) + kb, 16, 1024), kIdU,
                    ks > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_f16(tbase, sdesc(smem_addr(Ws) + ks * 32, 16, 1024), sdesc(smem_addr(Ks) + ks * 2048, 8192, 1024),
                    kIdZ, 1u);
        mma_commit(bar_mma);
    }
    if (__syncthreads_and(ok ? 1 : 0)) {
        ok = mbar_wait(bar_mma, mma_phase & 1) && ok;
        ++mma_phase;
        tc_fence_after();
        float ov[32];
        tmem_ld16_x8(tq + 64 * hh, ov);
        tmem_wait_ld();
        const float os0 = xs0 * sG, os1 = xs1 * sG;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            const int col = cb + 8 * g;
            if (tok0 < n)
                *reinterpret_cast<float2*>(out + (base + tok0) * kD + col) =
                    make_float2(ov[4 * g] * os0, ov[4 * g + 1] * os0);
            if (tok1 < n)
                *reinterpret_cast<float2*>(out + (base + tok1) * kD + col) =
                    make_float2(ov[4 * g + 2] * os1, ov[4 * g + 3] * os1);
        }
        if (iters && hh == 0 && (lane & 3) == 0) {
            if (tok0 < n) iters[base + tok0] = it0;
            if (tok1 < n) iters[base + tok1] = it1;
        }
    }
    if (!__syncthreads_and(ok ? 1 : 0)) {
        if (tid == 0) record_error(err, kErrTimeout);
        // give in-flight work one more bounded chance to drain before TMEM is released
        mbar_wait(bar_mma, (mma_phase & 1));
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tbase, 256);
}

}  // namespace

bool tc_supported(int dk, int dv, int chunk, mesa_dtype dtype) {
    return dtype == MESA_BF16 && dk == kD && dv == kD && chunk == kC;
}

static size_t images_bytes(int B, int H, int T) {
    const size_t nc = (size_t)((T + kC - 1) / kC);
    return (size_t)B * H * nc * 2 * kImgBytes;
}

size_t tc_workspace_bytes(int B, int H, int T) {
    const size_t nc = (size_t)((T + kC - 1) / kC);
    return images_bytes(B, H, T) + ((size_t)B * H * nc * 2 * sizeof(float) + 255) / 256 * 256;
}

cudaError_t forward_tc(const ForwardArgs& a, cudaStream_t st) {
    const int nc = (a.T + kC - 1) / kC;
    const int BH = a.B * a.H;
    __half* img = reinterpret_cast<__half*>(a.workspace);
    float* scales = reinterpret_cast<float*>(static_cast<char*>(a.workspace) + images_bytes(a.B, a.H, a.T));
    unsigned* err = error_word_ptr();
    const int scan_smem = ScanSmem::bytes + 1024;
    const int cg_smem = CgSmem::bytes + 1024;
    cudaError_t e = cudaFuncSetAttribute(tc_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, scan_smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_cg_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, cg_smem);
    if (e != cudaSuccess) return e;
    {
        LaunchTimer timer(kKindTcScan, st);
        tc_scan_kernel<<<dim3(2, BH), kThreads, scan_smem, st>>>(
            static_cast<const __nv_bfloat16*>(a.k), static_cast<const __nv_bfloat16*>(a.v), a.gamma, a.beta, a.T,
            nc, a.H_in, a.G_in, img, scales, a.H_out, a.G_out, err);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    {
        LaunchTimer timer(kKindTcCg, st);
        tc_cg_kernel<<<dim3(nc, BH), kThreads, cg_smem, st>>>(
            static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
            static_cast<const __nv_bfloat16*>(a.v), a.gamma, a.beta, a.lambda, a.H, a.T, nc, a.cg_steps, a.tol,
            img, scales, a.out, a.iters, err);
    }
    return cudaGetLastError();
}

}  // namespace mesa
