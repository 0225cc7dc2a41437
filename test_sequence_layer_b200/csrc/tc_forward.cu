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

// Power of two 2^floor(e/2) with 2^e <= rr < 2^(e+1): a scale within a factor
// sqrt(2) of |r| whose reciprocal is exact (1 for rr <= 0 or denormal rr).
__device__ __forceinline__ float pow2_sqrt_scale(float rr) {
    const int e = ((__float_as_int(rr) >> 23) & 0xff) - 127;
    if (!(rr > 0.f) || e <= -126 || e >= 127) return 1.f;
    return __int_as_float((((e >> 1) + 127) & 0xff) << 23);
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
// The fp16 image of a chunk-start state is scaled by s = 2^ceil(log2 max(Bnd,1))
// where Bnd bounds every entry: Bnd_0 = max|S_in| and
// Bnd_{c+1} = e^{b_last} Bnd_c + sum_j w_j |a_j|_inf |k_j|_inf (a = k for H,
// a = v for G), since |(a_j k_j^T)_il| <= |a_j|_inf |k_j|_inf. Every CTA of a
// sequence evaluates the same scalar recurrence, so the column blocks of one
// state agree on its scale without communicating.
constexpr int kScanNB = 2;                       // 64-column blocks per state matrix

struct ScanSmem {
    static constexpr int oRawA = 0;               // 2 x [64][128] bf16 rows of a (16 KB each)
    static constexpr int oRawK = 32768;           // 2 x [64][128] bf16 rows of k
    static constexpr int oAhi = 65536;            // MN-major [64 j][128 i] fp16, 16 KB
    static constexpr int oAlo = 81920;
    static constexpr int oB = 98304;              // MN-major [64 j][64 l] fp16, 8 KB
    static constexpr int oGate = 106496;          // b[64], w[64], amax[64], kmax[64]
    static constexpr int oRed = oGate + 1024;     // 16 floats
    static constexpr int oBar = oRed + 64;        // raw[2], mma
    static constexpr int oSlot = oBar + 32;
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
    const int m = blockIdx.x / kScanNB, nb = blockIdx.x % kScanNB, bh = blockIdx.y;
    uint8_t* rawK = smem + ScanSmem::oRawK;
    uint8_t* rawA = m ? smem + ScanSmem::oRawA : rawK;     // for H the left factor is k itself
    uint8_t* Ahi = smem + ScanSmem::oAhi;
    uint8_t* Alo = smem + ScanSmem::oAlo;
    uint8_t* Bk = smem + ScanSmem::oB;
    float* sb = reinterpret_cast<float*>(smem + ScanSmem::oGate);
    float* sw = sb + kC;
    float* amax = sw + kC;
    float* kmax = amax + kC;
    float* red = reinterpret_cast<float*>(smem + ScanSmem::oRed);
    uint64_t* bar_raw = reinterpret_cast<uint64_t*>(smem + ScanSmem::oBar);
    uint64_t* bar_mma = bar_raw + 2;
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + ScanSmem::oSlot);

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int q4 = w & 3, hh = w >> 2;
    const int row = 32 * q4 + lane;               // state row owned by this thread
    const int lcol = 32 * hh;                     // its 32 columns within the block
    const int col0 = 64 * nb + lcol;              // ... within the matrix
    const __nv_bfloat16* A = m ? v : k;
    const float* init = m ? G_in : H_in;
    float* fin = m ? G_out : H_out;
    const size_t seq = (size_t)bh * T;

    auto prefetch = [&](int cc) {                 // raw rows of chunk cc -> buffer cc & 1 (thread 0)
        const int nn = min(kC, T - cc * kC);
        const uint32_t bytes = (uint32_t)nn * kD * 2;
        const int buf = cc & 1;
        mbar_arrive_expect_tx(bar_raw + buf, m ? 2 * bytes : bytes);
        bulk_g2s(rawK + buf * 16384, k + (seq + (size_t)cc * kC) * kD, bytes, bar_raw + buf);
        if (m) bulk_g2s(rawA + buf * 16384, A + (seq + (size_t)cc * kC) * kD, bytes, bar_raw + buf);
    };

    if (tid == 0) {
        mbar_init(bar_raw, 1);
        mbar_init(bar_raw + 1, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        red[15] = 0.f;                            // abort flag
    }
    if (w == 0) tmem_alloc(slot, 64);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *slot;
    if (tid == 0 && nc > 0) {
        prefetch(0);
        if (nc > 1) prefetch(1);
    }

    float S[32];
    float bound = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) S[i] = 0.f;
    if (init) {
        const float4* src = reinterpret_cast<const float4*>(init + ((size_t)bh * kD + row) * kD + col0);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 f = src[i];
            S[4 * i] = f.x; S[4 * i + 1] = f.y; S[4 * i + 2] = f.z; S[4 * i + 3] = f.w;
        }
        // bound on the whole matrix, identical in every CTA of the sequence
        float mx = 0.f;
        const float4* all = reinterpret_cast<const float4*>(init + (size_t)bh * kD * kD);
        for (int i = tid; i < kD * kD / 4; i += kThreads) {
            const float4 f = all[i];
            mx = fmaxf(mx, fmaxf(fmaxf(fabsf(f.x), fabsf(f.y)), fmaxf(fabsf(f.z), fabsf(f.w))));
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) red[w] = mx;
        __syncthreads();
        bound = red[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) bound = fmaxf(bound, red[i]);
        __syncthreads();
    }

    constexpr uint32_t kIdesc = idesc_f16(128, 64, true, true);
    const uint64_t dAhi = sdesc(smem_addr(Ahi), 8192, 1024), dAlo = sdesc(smem_addr(Alo), 8192, 1024);
    const uint64_t dB = sdesc(smem_addr(Bk), 8192, 1024);
    uint32_t mma_phase = 0;
    bool ok = true;
    for (int c = 0; c <= nc; ++c) {
        // ---- emit the state before chunk c (fp16 image block + scale), or the final state ----
        if (c < nc) {
            const float s = pow2_ceil_at_least_one(bound);
            const float inv = 1.f / s;
            const size_t ci = ((size_t)bh * nc + c) * 2 + m;
            if (tid == 0 && nb == 0) scales[ci] = s;
            uint8_t* dst = reinterpret_cast<uint8_t*>(img + ci * kImgHalves) + nb * 16384 + row * 128;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                uint4 o;
                o.x = pack_half2(S[8 * g] * inv, S[8 * g + 1] * inv);
                o.y = pack_half2(S[8 * g + 2] * inv, S[8 * g + 3] * inv);
                o.z = pack_half2(S[8 * g + 4] * inv, S[8 * g + 5] * inv);
                o.w = pack_half2(S[8 * g + 6] * inv, S[8 * g + 7] * inv);
                *reinterpret_cast<uint4*>(dst + ((((lcol >> 3) + g) ^ (row & 7)) << 4)) = o;
            }
        } else {
            if (fin) {
                float4* d4 = reinterpret_cast<float4*>(fin + ((size_t)bh * kD + row) * kD + col0);
#pragma unroll
                for (int i = 0; i < 8; ++i) d4[i] = make_float4(S[4 * i], S[4 * i + 1], S[4 * i + 2], S[4 * i + 3]);
            }
            break;
        }

        // ---- chunk c: wait for its rows, gates ----
        const int t0 = c * kC;
        const int n = min(kC, T - t0);
        const size_t base = seq + t0;
        const int buf = c & 1;
        if (tid == 0 && !mbar_wait(bar_raw + buf, (c >> 1) & 1)) red[15] = 1.f;
        chunk_gates(gamma, base, n, sb);
        __syncthreads();
        if (red[15] != 0.f) {
            ok = false;
            break;
        }
        const float blast = sb[kC - 1];
        if (tid < kC) sw[tid] = (tid < n) ? beta[base + tid] * expf(blast - sb[tid]) : 0.f;
        __syncthreads();

        // ---- operand images: A = w_j a_j (hi/lo) [j][i], B = k_j block [j][l]; row maxima ----
        const uint8_t* ra = rawA + buf * 16384;
        const uint8_t* rk = rawK + buf * 16384;
#pragma unroll
        for (int rep = 0; rep < 4; ++rep) {
            const int cid = tid + kThreads * rep;          // 1024 16-byte chunks of a
            const int j = cid >> 4, cc = cid & 15;
            uint4 raw = make_uint4(0, 0, 0, 0);
            if (j < n) raw = *reinterpret_cast<const uint4*>(ra + j * 256 + cc * 16);
            const float wj = sw[j];
            const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
            uint4 hi, lo;
            uint32_t* hw = reinterpret_cast<uint32_t*>(&hi);
            uint32_t* lw = reinterpret_cast<uint32_t*>(&lo);
            float mx = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(a2[i]);
                mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
                const float x0 = wj * f.x, x1 = wj * f.y;
                const __half2 h2 = __floats2half2_rn(x0, x1);
                const float2 hb = __half22float2(h2);
                hw[i] = *reinterpret_cast<const uint32_t*>(&h2);
                lw[i] = pack_half2(x0 - hb.x, x1 - hb.y);
            }
            const uint32_t off = (uint32_t)((cc >> 3) * 8192 + j * 128 + (((cc & 7) ^ (j & 7)) << 4));
            *reinterpret_cast<uint4*>(Ahi + off) = hi;
            *reinterpret_cast<uint4*>(Alo + off) = lo;
            // row max over the 16 threads (same half-warp) that hold row j
#pragma unroll
            for (int o2 = 8; o2 >= 1; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
            if (cc == 0) amax[j] = mx;
            if (m) {   // key row maxima for the value-state bound
                uint4 kr = make_uint4(0, 0, 0, 0);
                if (j < n) kr = *reinterpret_cast<const uint4*>(rk + j * 256 + cc * 16);
                const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kr);
                float km = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __bfloat1622float2(k2[i]);
                    km = fmaxf(km, fmaxf(fabsf(f.x), fabsf(f.y)));
                }
#pragma unroll
                for (int o2 = 8; o2 >= 1; o2 >>= 1) km = fmaxf(km, __shfl_xor_sync(0xffffffffu, km, o2));
                if (cc == 0) kmax[j] = km;
            }
        }
#pragma unroll
        for (int rep = 0; rep < 2; ++rep) {
            const int cid = tid + kThreads * rep;          // 512 16-byte chunks of the k block
            const int j = cid >> 3, cc = cid & 7;
            uint4 raw = make_uint4(0, 0, 0, 0);
            if (j < n) raw = *reinterpret_cast<const uint4*>(rk + j * 256 + (8 * nb + cc) * 16);
            *reinterpret_cast<uint4*>(Bk + j * 128 + ((cc ^ (j & 7)) << 4)) = bf16x8_to_f16x8(raw, 1.f);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            if (c + 2 < nc) prefetch(c + 2);       // raw buffer `buf` is consumed
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t ko = ((ks & 3) * 2048) >> 4;
                mma_f16(tbase, (ks < 4 ? dAhi : dAlo) + ko, dB + ko, kIdesc, ks > 0 ? 1u : 0u);
            }
            mma_commit(bar_mma);
        }
        // bound update: every warp reduces the same 64 terms in the same order,
        // so every thread of every CTA of this sequence gets the same value
        {
            const float* km = m ? kmax : amax;
            float add = sw[lane] * (amax[lane] * km[lane]) + sw[lane + 32] * (amax[lane + 32] * km[lane + 32]);
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) add += __shfl_xor_sync(0xffffffffu, add, off);
            bound = fmaf(expf(blast), bound, add);
        }
        if (tid == 0 && !mbar_wait(bar_mma, mma_phase & 1)) red[15] = 1.f;
        ++mma_phase;
        __syncthreads();
        tc_fence_after();
        if (red[15] != 0.f) {
            ok = false;
            break;
        }

        // ---- S <- e^{b_last} S + Delta ----
        const float Gam = expf(blast);
        float dv[32];
        tmem_ld32_x32(tbase + ((uint32_t)(32 * q4) << 16) + lcol, dv);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) S[i] = fmaf(Gam, S[i], dv[i]);
        tc_fence_before();
        __syncthreads();       // TMEM and the operand images are free for the next chunk
        tc_fence_after();
    }

    if (!ok) {
        if (tid == 0) {
            record_error(err, kErrTimeout);
            mbar_wait(bar_mma, mma_phase & 1);    // one more bounded chance for in-flight work to drain
        }
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tbase, 64);
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
    static constexpr int oM = 90112;              // decay mask / sH, fp32 [64][72]
    static constexpr int oLam = oM + kC * kMStride * 4;   // lambda [128]
    static constexpr int oEb = oLam + 512;        // e^{b_t} [64]
    static constexpr int oB = oEb + 256;          // b_t [64]
    static constexpr int oRed = oB + 256;         // [2 halves][64 tokens][4] partial sums
    static constexpr int oMisc = oRed + 2048;     // 16 floats / flags
    static constexpr int oBar = oMisc + 64;       // 3 mbarriers
    static constexpr int oSlot = oBar + 32;
    static constexpr int bytes = oSlot + 16;
};

// Sums NV (<= 4) per-token partials over the 8 threads that hold one token
// (4 lanes x 2 column halves). One barrier. v0/v1: the two tokens of this thread.
template <int NV>
__device__ __forceinline__ void token_sums(float (&v0)[NV], float (&v1)[NV], float4* red, int hh, int tok0, int tok1,
                                           int lane) {
    static_assert(NV >= 1 && NV <= 4, "at most 4 partials");
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        v0[i] += __shfl_xor_sync(0xffffffffu, v0[i], 1);
        v0[i] += __shfl_xor_sync(0xffffffffu, v0[i], 2);
        v1[i] += __shfl_xor_sync(0xffffffffu, v1[i], 1);
        v1[i] += __shfl_xor_sync(0xffffffffu, v1[i], 2);
    }
    if ((lane & 3) == 0) {
        float a[4] = {0.f, 0.f, 0.f, 0.f}, b[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            a[i] = v0[i];
            b[i] = v1[i];
        }
        red[hh * 64 + tok0] = make_float4(a[0], a[1], a[2], a[3]);
        red[hh * 64 + tok1] = make_float4(b[0], b[1], b[2], b[3]);
    }
    __syncthreads();
    const float4 a0 = red[tok0], b0 = red[64 + tok0], a1 = red[tok1], b1 = red[64 + tok1];
    const float s0[4] = {a0.x + b0.x, a0.y + b0.y, a0.z + b0.z, a0.w + b0.w};
    const float s1[4] = {a1.x + b1.x, a1.y + b1.y, a1.z + b1.z, a1.w + b1.w};
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        v0[i] = s0[i];
        v1[i] = s1[i];
    }
}

// Writes this thread's two tokens x 16 columns (as float2 pairs) of a
// [64 t][128 k] fp16 image, each token scaled by its own factor.
__device__ __forceinline__ void store_rows(uint8_t* img0, uint8_t* img1, uint32_t phase,
                                           const float2 (&v0)[8], const float2 (&v1)[8], float s0, float s1) {
    const float2 f0 = make_float2(s0, s0), f1 = make_float2(s1, s1);
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        const float2 a = __fmul2_rn(v0[g], f0), b = __fmul2_rn(v1[g], f1);
        const uint32_t o = ((uint32_t)g ^ phase) << 4;
        *reinterpret_cast<uint32_t*>(img0 + o) = pack_half2(a.x, a.y);
        *reinterpret_cast<uint32_t*>(img1 + o) = pack_half2(b.x, b.y);
    }
}

// One thread issues, waits (bounded) and records failure; the barrier then
// releases the CTA. Returns the CTA-uniform success flag.
__device__ __forceinline__ bool wait_mma_cta(uint64_t* bar, uint32_t parity, int tid, float* abort_flag) {
    if (tid == 0) {
        if (!mbar_wait(bar, parity)) *abort_flag = 1.f;
    }
    __syncthreads();
    tc_fence_after();
    return *abort_flag == 0.f;
}

// Every thread waits on the MMA barrier itself (no CTA barrier); a thread
// whose bounded wait gave up raises the abort flag, which the next CTA
// barrier makes visible to all.
__device__ __forceinline__ void wait_mma_each(uint64_t* bar, uint32_t parity, float* abort_flag) {
    if (!mbar_wait(bar, parity)) *abort_flag = 1.f;
    tc_fence_after();
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
    float4* red = reinterpret_cast<float4*>(smem + CgSmem::oRed);
    float* misc = reinterpret_cast<float*>(smem + CgSmem::oMisc);
    float* abort_flag = misc + 15;
    uint64_t* bar_ld = reinterpret_cast<uint64_t*>(smem + CgSmem::oBar);
    uint64_t* bar_s = bar_ld + 1;        // scores S ready
    uint64_t* bar_y = bar_ld + 2;        // Y = U + Z ready
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

    // this thread's 32-bit slot of group g in a [64][128] fp16 image is
    // row0/row1 + ((g ^ phase) << 4) + cw (both tokens share the swizzle
    // phase: tok1 = tok0 + 8)
    const uint32_t phase = (uint32_t)(tok0 & 7), cw = 4u * (uint32_t)(lane & 3);
    const uint32_t row0 = (uint32_t)(hh * 8192 + tok0 * 128) + cw, row1 = row0 + 8 * 128;

    // ---- set-up: barriers, TMEM, async load of the H_c image ----
    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_y, 1);
        fence_mbar_init();
        *abort_flag = 0.f;
    }
    if (w == 0) tmem_alloc(slot, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *slot;
    // TMEM: columns [0,128) lanes 16g..16g+15 (M=64 rows) hold Y = U + Z; the
    // idle lanes 16g+16..16g+31 of the same columns hold x (same token order);
    // columns [128,192) hold the scores S.
    const uint32_t tq = tbase + ((uint32_t)(32 * q4) << 16);    // this warp's lane quadrant
    const uint32_t tx = tq + (16u << 16);                        // ... and its x lanes
    constexpr uint32_t kColS = 128;
    if (tid == 0) {
        mbar_arrive_expect_tx(bar_ld, kImgBytes);
        bulk_g2s(Hs, Himg, kImgBytes, bar_ld);
    }
    const float sH = scales[ci * 2 + 0], sG = scales[ci * 2 + 1];
    const float inv_sH = 1.f / sH;

    // gates, lambda and the key image (bf16 -> fp16 is exact for normalised keys)
    chunk_gates(gamma, base, n, sbc);
    for (int d = tid; d < kD; d += kThreads) slam[d] = lambda[(size_t)head * kD + d];
#pragma unroll
    for (int rep = 0; rep < 4; ++rep) {
        const int cid = tid + kThreads * rep;
        const int j = cid >> 4, cc = cid & 15;
        uint4 rk = make_uint4(0, 0, 0, 0);
        if (j < n) rk = *reinterpret_cast<const uint4*>(k + (base + j) * kD + 8 * cc);
        *reinterpret_cast<uint4*>(Ks + (cc >> 3) * 8192 + j * 128 + (((cc & 7) ^ (j & 7)) << 4)) =
            bf16x8_to_f16x8(rk, 1.f);
    }
    // CG state: x = 0 (TMEM), r = p = q; this thread holds 2 tokens x 8 column pairs
    float2 r0[8], r1[8], p0[8], p1[8];
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        const int col = cb + 8 * g;
        float2 a = make_float2(0.f, 0.f), b = make_float2(0.f, 0.f);
        if (tok0 < n) a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(q + (base + tok0) * kD + col));
        if (tok1 < n) b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(q + (base + tok1) * kD + col));
        r0[g] = a; p0[g] = a;
        r1[g] = b; p1[g] = b;
    }
    __syncthreads();                                   // gates visible
    if (tid < kC) seb[tid] = expf(sbc[tid]);
    for (int e = tid; e < kC * kC; e += kThreads) {
        const int tt = e >> 6, j = e & 63;
        Mk[tt * CgSmem::kMStride + j] =
            (j <= tt && tt < n) ? beta[base + j] * expf(sbc[tt] - sbc[j]) * inv_sH : 0.f;
    }
    {
        float z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0.f;
        tmem_st16_x8(tx + 64 * hh, z);
        tmem_wait_st();
    }
    float rr0, rr1;
    {
        float a0[1] = {0.f}, a1[1] = {0.f};
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            a0[0] = fmaf(r0[g].x, r0[g].x, fmaf(r0[g].y, r0[g].y, a0[0]));
            a1[0] = fmaf(r1[g].x, r1[g].x, fmaf(r1[g].y, r1[g].y, a1[0]));
        }
        token_sums<1>(a0, a1, red, hh, tok0, tok1, lane);   // barrier also publishes seb
        rr0 = a0[0];
        rr1 = a1[0];
    }
    const float qn0 = sqrtf(rr0), qn1 = sqrtf(rr1);
    bool act0 = tok0 < n, act1 = tok1 < n;
    int it0 = 0, it1 = 0;
    const float eb0 = seb[tok0], eb1 = seb[tok1];
    float s0 = pow2_sqrt_scale(rr0), s1 = pow2_sqrt_scale(rr1);
    float is0 = 1.f / s0, is1 = 1.f / s1;                   // exact: powers of two
    store_rows(Ps + row0, Ps + row1, phase, p0, p1, is0, is1);
    store_rows(Pt + row0, Pt + row1, phase, p0, p1, eb0 * is0, eb1 * is1);

    // MMA issue (one thread). Descriptor address fields are the low 14 bits,
    // so byte offsets (>> 4) add directly.
    constexpr uint32_t kIdS = idesc_f16(64, 64, false, false);
    constexpr uint32_t kIdU = idesc_f16(64, 128, false, false);
    constexpr uint32_t kIdZ = idesc_f16(64, 128, false, true);
    auto issue_S = [&](const uint8_t* A) {   // S = A K^T: M=64 tokens, N=64 keys, K=128
        const uint64_t dA = sdesc(smem_addr(A), 16, 1024), dK = sdesc(smem_addr(Ks), 16, 1024);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t ko = ((ks >> 2) * 8192 + (ks & 3) * 32) >> 4;
            mma_f16(tbase + kColS, dA + ko, dK + ko, kIdS, ks > 0 ? 1u : 0u);
        }
    };
    auto issue_U = [&](const uint8_t* A, const uint8_t* B) {   // Y = A B^T: M=64, N=128, K=128
        const uint64_t dA = sdesc(smem_addr(A), 16, 1024), dB = sdesc(smem_addr(B), 16, 1024);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t ka = ((ks >> 2) * 8192 + (ks & 3) * 32) >> 4;
            const uint32_t kb = ((ks >> 2) * 16384 + (ks & 3) * 32) >> 4;
            mma_f16(tbase, dA + ka, dB + kb, kIdU, ks > 0 ? 1u : 0u);
        }
    };
    auto issue_Z = [&]() {                   // Y += W Kmn: M=64, N=128, K=64
        const uint64_t dW = sdesc(smem_addr(Ws), 16, 1024), dKmn = sdesc(smem_addr(Ks), 8192, 1024);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) mma_f16(tbase, dW + ((ks * 32) >> 4), dKmn + ((ks * 2048) >> 4), kIdZ, 1u);
    };
    // S (in TMEM) -> masked, scaled scores -> fp16 image
    auto masked_scores = [&](float extra) {
        float sv[16];
        tmem_ld16_x4(tq + kColS + 32 * hh, sv);
        tmem_wait_ld();
        const float2 ex = make_float2(extra, extra);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int j = 32 * hh + 8 * g + 2 * (lane & 3);
            const float2 m0 = __fmul2_rn(*reinterpret_cast<const float2*>(Mk + tok0 * CgSmem::kMStride + j), ex);
            const float2 m1 = __fmul2_rn(*reinterpret_cast<const float2*>(Mk + tok1 * CgSmem::kMStride + j), ex);
            const float2 w0 = __fmul2_rn(m0, make_float2(sv[4 * g], sv[4 * g + 1]));
            const float2 w1 = __fmul2_rn(m1, make_float2(sv[4 * g + 2], sv[4 * g + 3]));
            const uint32_t o = ((((uint32_t)(4 * hh + g)) ^ phase) << 4) + cw;
            *reinterpret_cast<uint32_t*>(Ws + tok0 * 128 + o) = pack_half2(w0.x, w0.y);
            *reinterpret_cast<uint32_t*>(Ws + tok1 * 128 + o) = pack_half2(w1.x, w1.y);
        }
    };

    bool ok = mbar_wait(bar_ld, 0);
    if (!ok) *abort_flag = 1.f;
    uint32_t mma_phase = 0;

    for (int step = 0; step < cg_steps; ++step) {
        act0 = act0 && cg_may_continue(rr0, qn0, tol);
        act1 = act1 && cg_may_continue(rr1, qn1, tol);
        fence_proxy_async();
        tc_fence_before();
        const int any = __syncthreads_or((act0 || act1) ? 1 : 0);
        tc_fence_after();
        if (!any || *abort_flag != 0.f) break;

        // S first, then U straight behind it: U runs while the scores are masked
        if (tid == 0) {
            issue_S(Ps);
            mma_commit(bar_s);
            issue_U(Pt, Hs);
        }
        wait_mma_each(bar_s, mma_phase & 1, abort_flag);
        masked_scores(1.f);
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (*abort_flag != 0.f) break;
        if (tid == 0) {
            issue_Z();
            mma_commit(bar_y);
        }
        wait_mma_each(bar_y, mma_phase & 1, abort_flag);
        ++mma_phase;

        // y = (s sH) Y + lambda p, written back over Y; partials p.y, r.y, y.y, r.r
        float d0[4], d1[4];
        {
            const float2 ys0 = make_float2(s0 * sH, s0 * sH), ys1 = make_float2(s1 * sH, s1 * sH);
            float2 a = make_float2(0.f, 0.f), b = a, cc = a, e = a, f = a, h = a, ra = a, rb2 = a;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float yv[16];
                const uint32_t ya = tq + 64 * hh + 32 * half;
                tmem_ld16_x4(ya, yv);
                tmem_wait_ld();
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int gg = 4 * half + g;
                    const float2 lm = *reinterpret_cast<const float2*>(slam + cb + 8 * gg);
                    const float2 y0 = __ffma2_rn(make_float2(yv[4 * g], yv[4 * g + 1]), ys0, __fmul2_rn(lm, p0[gg]));
                    const float2 y1 = __ffma2_rn(make_float2(yv[4 * g + 2], yv[4 * g + 3]), ys1, __fmul2_rn(lm, p1[gg]));
                    a = __ffma2_rn(p0[gg], y0, a);
                    b = __ffma2_rn(r0[gg], y0, b);
                    cc = __ffma2_rn(y0, y0, cc);
                    e = __ffma2_rn(p1[gg], y1, e);
                    f = __ffma2_rn(r1[gg], y1, f);
                    h = __ffma2_rn(y1, y1, h);
                    ra = __ffma2_rn(r0[gg], r0[gg], ra);
                    rb2 = __ffma2_rn(r1[gg], r1[gg], rb2);
                    yv[4 * g] = y0.x; yv[4 * g + 1] = y0.y; yv[4 * g + 2] = y1.x; yv[4 * g + 3] = y1.y;
                }
                tmem_st16_x4(ya, yv);
            }
            d0[0] = a.x + a.y; d0[1] = b.x + b.y; d0[2] = cc.x + cc.y; d0[3] = ra.x + ra.y;
            d1[0] = e.x + e.y; d1[1] = f.x + f.y; d1[2] = h.x + h.y; d1[3] = rb2.x + rb2.y;
        }
        tmem_wait_st();
        token_sums<4>(d0, d1, red, hh, tok0, tok1, lane);
        if (act0 && !cg_curvature_ok(d0[0])) act0 = false;
        if (act1 && !cg_curvature_ok(d1[0])) act1 = false;
        // rr is refreshed from the true |r|^2 every iteration (no drift); the next
        // |r - alpha y|^2 = rr - 2 alpha r.y + alpha^2 y.y is only needed one step
        // ahead, for rho and the next stopping test.
        if (act0) rr0 = d0[3];
        if (act1) rr1 = d1[3];
        const float al0 = act0 ? rr0 / d0[0] : 0.f, al1 = act1 ? rr1 / d1[0] : 0.f;
        const float rn0 = fmaxf(fmaf(al0, fmaf(al0, d0[2], -2.f * d0[1]), rr0), 0.f);
        const float rn1 = fmaxf(fmaf(al1, fmaf(al1, d1[2], -2.f * d1[1]), rr1), 0.f);
        const float rho0 = act0 ? rn0 / rr0 : 0.f, rho1 = act1 ? rn1 / rr1 : 0.f;
        const float2 pa0 = make_float2(al0, al0), pa1 = make_float2(al1, al1);
        const float2 na0 = make_float2(-al0, -al0), na1 = make_float2(-al1, -al1);
        const float2 rh0 = make_float2(rho0, rho0), rh1 = make_float2(rho1, rho1);
#pragma unroll
        for (int half = 0; half < 2; ++half) {   // x += alpha p (TMEM), r -= alpha y, p = r + rho p
            float xv[16], yv[16];
            const uint32_t xa = tx + 64 * hh + 32 * half;
            tmem_ld16_x4(xa, xv);
            tmem_ld16_x4(tq + 64 * hh + 32 * half, yv);
            tmem_wait_ld();
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const int gg = 4 * half + g;
                const float2 x0 = __ffma2_rn(pa0, p0[gg], make_float2(xv[4 * g], xv[4 * g + 1]));
                const float2 x1 = __ffma2_rn(pa1, p1[gg], make_float2(xv[4 * g + 2], xv[4 * g + 3]));
                xv[4 * g] = x0.x; xv[4 * g + 1] = x0.y; xv[4 * g + 2] = x1.x; xv[4 * g + 3] = x1.y;
                if (act0) {
                    r0[gg] = __ffma2_rn(na0, make_float2(yv[4 * g], yv[4 * g + 1]), r0[gg]);
                    p0[gg] = __ffma2_rn(rh0, p0[gg], r0[gg]);
                }
                if (act1) {
                    r1[gg] = __ffma2_rn(na1, make_float2(yv[4 * g + 2], yv[4 * g + 3]), r1[gg]);
                    p1[gg] = __ffma2_rn(rh1, p1[gg], r1[gg]);
                }
            }
            tmem_st16_x4(xa, xv);
        }
        if (act0) {
            rr0 = rn0;
            ++it0;
            s0 = pow2_sqrt_scale(rr0);
            is0 = 1.f / s0;
        }
        if (act1) {
            rr1 = rn1;
            ++it1;
            s1 = pow2_sqrt_scale(rr1);
            is1 = 1.f / s1;
        }
        tmem_wait_st();
        store_rows(Ps + row0, Ps + row1, phase, p0, p1, is0, is1);
        store_rows(Pt + row0, Pt + row1, phase, p0, p1, eb0 * is0, eb1 * is1);
    }

    // ---- read-out: o = e^{b_t} G_c x + (M o X K^T) V ----
    float2 xr0[8], xr1[8];
    {
        float xv[32];
        tmem_ld16_x8(tx + 64 * hh, xv);
        tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            xr0[g] = make_float2(xv[4 * g], xv[4 * g + 1]);
            xr1[g] = make_float2(xv[4 * g + 2], xv[4 * g + 3]);
        }
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
    float xs0, xs1;
    {
        float a0[1] = {0.f}, a1[1] = {0.f};
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            a0[0] = fmaf(xr0[g].x, xr0[g].x, fmaf(xr0[g].y, xr0[g].y, a0[0]));
            a1[0] = fmaf(xr1[g].x, xr1[g].x, fmaf(xr1[g].y, xr1[g].y, a1[0]));
        }
        token_sums<1>(a0, a1, red, hh, tok0, tok1, lane);   // its barrier also publishes misc[]
        xs0 = a0[0] > 0.f ? sqrtf(a0[0]) : 1.f;
        xs1 = a1[0] > 0.f ? sqrtf(a1[0]) : 1.f;
    }
    float vm = misc[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) vm = fmaxf(vm, misc[i]);
    const float sV = pow2_ceil_at_least_one(vm);
    store_rows(Ps + row0, Ps + row1, phase, xr0, xr1, 1.f / xs0, 1.f / xs1);
    store_rows(Pt + row0, Pt + row1, phase, xr0, xr1, eb0 / xs0, eb1 / xs1);
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    ok = *abort_flag == 0.f;
    if (ok) {
        if (tid == 0) {
            // every MMA that read the H image has completed: reuse its buffer for G_c
            mbar_arrive_expect_tx(bar_ld, kImgBytes);
            bulk_g2s(Hs, Gimg, kImgBytes, bar_ld);
            issue_S(Ps);                       // S' = X-hat K^T
            mma_commit(bar_s);
        }
        ok = wait_mma_cta(bar_s, mma_phase & 1, tid, abort_flag);
    }
    if (ok) {
        masked_scores(sH * sV / sG);           // mask holds 1/sH
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
        if (tid == 0) {
            if (!mbar_wait(bar_ld, 1)) {
                *abort_flag = 1.f;
            } else {
                issue_U(Pt, Hs);               // O = X-tilde G^T + W' V
                issue_Z();
                mma_commit(bar_y);
            }
        }
        ok = wait_mma_cta(bar_y, mma_phase & 1, tid, abort_flag);
        ++mma_phase;
    }
    if (ok) {
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
    } else {
        if (tid == 0) {
            record_error(err, kErrTimeout);
            // one more bounded chance for every MMA issued so far to drain
            mma_commit(bar_ld);
            mbar_wait(bar_ld, 0);
            mbar_wait(bar_ld, 1);
        }
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
        tc_scan_kernel<<<dim3(2 * kScanNB, BH), kThreads, scan_smem, st>>>(
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
