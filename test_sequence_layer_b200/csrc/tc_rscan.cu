// tc_rscan.cu -- the backward's reverse chunk scan of the gradient states on
// the tensor cores, for the tensor-core shape (d = 128, C = 64).
//
// Method: "MesaNet: Sequence Modeling by Locally Optimal Test-Time Training"
// (gist.science), Technical summary > Method > Mesa layer ("Parallelisation":
// training in time linear in T). The gradient states carried backwards across
// chunks (implicit differentiation, see simt_backward.cu) obey
//     Hhat_{c-1} = e^{b_last} Hhat_c + sum_{t in c} e^{b_t} u_t x_t^T,
//     Ghat_{c-1} = e^{b_last} Ghat_c + sum_{t in c} e^{b_t} do_t x_t^T,
// with b_t the in-chunk log-cumsum of gamma; per chunk c the state carried in
// from the tokens after it is written in fp32 (the gradient kernel's input).
//
// Numerics: per chunk, e^{b_t} a_t / sA (a = u or dL/do) is split into fp16
// hi/lo pairs and multiplied by x_t / sX in fp16 on the tensor cores with fp32
// accumulation into the fp32 running state; sA and sX are the powers of two
// at or above the chunk's largest |e^{b_t} a_t| and |x_t| entries. x enters
// with 11 bits, so the products carry ~2^-12 relative error: the bf16-mode
// precision the tensor-core backward runs at.
#include "mesa_internal.h"
#include "tc_layout.cuh"

namespace mesa {
namespace {

using namespace tc;

constexpr int kRThreads = 512;

struct RscanSmem {
    static constexpr int oRawA = 0;               // 2 x [64][128] fp32 rows of a (32 KB each)
    static constexpr int oRawX = 65536;           // 2 x [64][128] fp32 rows of x
    static constexpr int oImg = 131072;           // {A hi, A lo, X}: MN-major SW128, 16 KB each
    static constexpr int oGate = oImg + 49152;    // b[64], w[64]
    static constexpr int oRed = oGate + 512;      // 32 floats; [31] is the abort flag
    static constexpr int oCmax = oRed + 128;      // {max w|a|, max |x|} (int bits of non-negative floats)
    static constexpr int oBar = oCmax + 16;       // raw[2], mma
    static constexpr int oSlot = oBar + 32;
    static constexpr int bytes = oSlot + 16;
};
static_assert(RscanSmem::oImg % 1024 == 0, "SW128 images need 1 KB alignment");

__device__ __forceinline__ float absmax4(float4 v) {
    return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
}

// 8 x 8 transpose of 16-byte units among the lanes of each lane octet: on
// entry lane 8o + a holds units 0..7 of its own row, on return U[s] is unit a
// of row 8o + s. Three butterfly rounds: lanes a and a ^ m swap the units whose
// index differs from the lane's in bit m.
__device__ __forceinline__ void octet_transpose(uint4 (&U)[8], int lane) {
#pragma unroll
    for (int m = 4; m >= 1; m >>= 1) {
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (k & m) continue;                  // each pair (k, k | m) once
            const uint4 send = up ? U[k] : U[k | m];
            uint4 recv;
            recv.x = __shfl_xor_sync(0xffffffffu, send.x, m);
            recv.y = __shfl_xor_sync(0xffffffffu, send.y, m);
            recv.z = __shfl_xor_sync(0xffffffffu, send.z, m);
            recv.w = __shfl_xor_sync(0xffffffffu, send.w, m);
            if (up) U[k] = recv;
            else U[k | m] = recv;
        }
    }
}

// CTA (bh, m) walks the chunks of sequence bh from the last to the first for
// Hhat (m = 0, rows from u) or Ghat (m = 1, rows from dL/do). Warp w serves
// TMEM lane quadrant w % 4 (state rows 32 (w % 4) .. + 31, one per thread)
// and the 32 columns 32 (w / 4) .. + 31; tensor memory holds the chunk's
// product (columns 0 .. 127) and the running state (128 .. 255). Per chunk:
// the gates (warp 1), the operand scales from the chunk's maxima, the fp16
// images, one M = N = 128, K = 64 product (hi and lo), during which the state
// carried into the chunk is written out, and the state update. The rows of
// the chunk after next are on their way by bulk copy meanwhile.
__global__ void __launch_bounds__(kRThreads, 1)
tc_rscan_kernel(const float* __restrict__ dout, const float* __restrict__ u, const float* __restrict__ xsol,
                const float* __restrict__ gamma, int T, int nc, float* __restrict__ rstates,
                unsigned* __restrict__ err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int bh = blockIdx.x, m = blockIdx.y;
    const float* A = m ? dout : u;
    float* rawA = reinterpret_cast<float*>(smem + RscanSmem::oRawA);
    float* rawX = reinterpret_cast<float*>(smem + RscanSmem::oRawX);
    uint8_t* img = smem + RscanSmem::oImg;
    float* sb = reinterpret_cast<float*>(smem + RscanSmem::oGate);
    float* sw = sb + kC;
    float* red = reinterpret_cast<float*>(smem + RscanSmem::oRed);
    int* cmax = reinterpret_cast<int*>(smem + RscanSmem::oCmax);
    uint64_t* bar_raw = reinterpret_cast<uint64_t*>(smem + RscanSmem::oBar);
    uint64_t* bar_mma = bar_raw + 2;
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + RscanSmem::oSlot);

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int q4 = w & 3;
    const int row = 32 * q4 + lane;
    const int col0 = 32 * (w >> 2);
    const size_t seq = (size_t)bh * T;
    constexpr size_t SE = 2 * (size_t)kD * kD;

    // rows of the cc-th chunk walked (chunk nc - 1 - cc) into buffer cc & 1 (thread 0)
    int prefetched = 0;
    auto prefetch = [&](int cc) {
        const int c = nc - 1 - cc;
        const int nn = min(kC, T - c * kC);
        const uint32_t bytes = (uint32_t)nn * kD * 4;
        const int buf = cc & 1;
        mbar_arrive_expect_tx(bar_raw + buf, 2 * bytes);
        bulk_g2s(rawA + buf * kC * kD, A + (seq + (size_t)c * kC) * kD, bytes, bar_raw + buf);
        bulk_g2s(rawX + buf * kC * kD, xsol + (seq + (size_t)c * kC) * kD, bytes, bar_raw + buf);
        prefetched = cc + 1;
    };
    // warp 1: gamma of chunk c into registers (positions 2 lane, 2 lane + 1; 1 past the end)
    float g0 = 1.f, g1 = 1.f;
    auto load_gates = [&](int c) {
        const int nn = min(kC, T - c * kC);
        const size_t base = seq + (size_t)c * kC;
        g0 = 2 * lane < nn ? gamma[base + 2 * lane] : 1.f;
        g1 = 2 * lane + 1 < nn ? gamma[base + 2 * lane + 1] : 1.f;
    };

    if (tid == 0) {
        mbar_init(bar_raw, 1);
        mbar_init(bar_raw + 1, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        red[31] = 0.f;
    }
    if (w == 0) tmem_alloc(slot, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *slot;
    const uint32_t tl = tbase + ((uint32_t)(32 * q4) << 16) + col0;
    {
        float z[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) z[e] = 0.f;
        tmem_st32_x16(tl + 128, z);
        tmem_st32_x16(tl + 144, z);
        tmem_wait_st();
    }
    if (tid == 0 && nc > 0) {
        prefetch(0);
        if (nc > 1) prefetch(1);
    }
    if (w == 1 && nc > 0) load_gates(nc - 1);

    constexpr uint32_t kIdesc = idesc_f16(128, 128, true, true);
    int mma_issued = 0, mma_seen = 0;             // thread 0
    bool ok = true;
    for (int cc = 0; cc < nc; ++cc) {
        const int c = nc - 1 - cc;
        const int n = min(kC, T - c * kC);
        const int buf = cc & 1;
        const float* ra = rawA + buf * kC * kD;
        const float* rx = rawX + buf * kC * kD;
        if (w == 1) {                             // b (inclusive log-cumsum) and w_t = e^{b_t} (0 past n)
            const float l0 = logf(g0), l1 = logf(g1);
            const float pair = l0 + l1;
            float incl = pair;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float o = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += o;
            }
            const float b0 = incl - pair + l0, b1 = incl;
            sb[2 * lane] = b0;
            sb[2 * lane + 1] = b1;
            sw[2 * lane] = 2 * lane < n ? expf(b0) : 0.f;
            sw[2 * lane + 1] = 2 * lane + 1 < n ? expf(b1) : 0.f;
            if (cc + 1 < nc) load_gates(c - 1);
        }
        if (tid < 2) cmax[tid] = 0;
        if (!mbar_wait(bar_raw + buf, (cc >> 1) & 1)) red[31] = 1.f;
        __syncthreads();                          // gates, cleared maxima, rows landed
        if (red[31] != 0.f) {
            ok = false;
            break;
        }
        // the chunk's maxima of w_t |a_t| and |x_t| (rows past n hold stale data: skipped)
        {
            float ma = 0.f, mx = 0.f;
#pragma unroll
            for (int rep = 0; rep < 4; ++rep) {
                const int e = tid + kRThreads * rep;       // 2048 float4 pieces of each chunk's rows
                const int t = e >> 5, q = e & 31;
                if (t < n) {
                    ma = fmaxf(ma, sw[t] * absmax4(*reinterpret_cast<const float4*>(ra + t * kD + 4 * q)));
                    mx = fmaxf(mx, absmax4(*reinterpret_cast<const float4*>(rx + t * kD + 4 * q)));
                }
            }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
                ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, off));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            }
            if (lane == 0) {
                atomicMax(cmax, __float_as_int(ma));
                atomicMax(cmax + 1, __float_as_int(mx));
            }
        }
        __syncthreads();
        const float sA = pow2_ceil(__int_as_float(cmax[0])), sX = pow2_ceil(__int_as_float(cmax[1]));
        {
            const float iA = 1.f / sA, iX = 1.f / sX;             // powers of two: exact
#pragma unroll
            for (int rep = 0; rep < 2; ++rep) {
                const int e = tid + kRThreads * rep;       // 1024 units of 8 columns of each image
                const int t = e >> 4, cc16 = e & 15;
                float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0, x0 = a0, x1 = a0;
                if (t < n) {
                    a0 = *reinterpret_cast<const float4*>(ra + t * kD + 8 * cc16);
                    a1 = *reinterpret_cast<const float4*>(ra + t * kD + 8 * cc16 + 4);
                    x0 = *reinterpret_cast<const float4*>(rx + t * kD + 8 * cc16);
                    x1 = *reinterpret_cast<const float4*>(rx + t * kD + 8 * cc16 + 4);
                }
                const float f = sw[t] * iA;
                const float av[8] = {a0.x * f, a0.y * f, a0.z * f, a0.w * f, a1.x * f, a1.y * f, a1.z * f, a1.w * f};
                uint4 hi, lo, xo;
                uint32_t* hw = reinterpret_cast<uint32_t*>(&hi);
                uint32_t* lw = reinterpret_cast<uint32_t*>(&lo);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const __half2 h2 = __floats2half2_rn(av[2 * i], av[2 * i + 1]);
                    const float2 hb = __half22float2(h2);
                    hw[i] = *reinterpret_cast<const uint32_t*>(&h2);
                    lw[i] = pack_half2(av[2 * i] - hb.x, av[2 * i + 1] - hb.y);
                }
                xo.x = pack_half2(x0.x * iX, x0.y * iX);
                xo.y = pack_half2(x0.z * iX, x0.w * iX);
                xo.z = pack_half2(x1.x * iX, x1.y * iX);
                xo.w = pack_half2(x1.z * iX, x1.w * iX);
                const uint32_t off = (uint32_t)((cc16 >> 3) * 8192 + t * 128 + (((cc16 & 7) ^ (t & 7)) << 4));
                *reinterpret_cast<uint4*>(img + off) = hi;
                *reinterpret_cast<uint4*>(img + 16384 + off) = lo;
                *reinterpret_cast<uint4*>(img + 32768 + off) = xo;
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();                          // images written; the chunk's raw rows are read
        tc_fence_after();
        if (tid == 0) {
            const uint64_t dAhi = sdesc(smem_addr(img), 8192, 1024), dAlo = sdesc(smem_addr(img + 16384), 8192, 1024);
            const uint64_t dX = sdesc(smem_addr(img + 32768), 8192, 1024);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t ko = ((ks & 3) * 2048) >> 4;
                mma_f16(tbase, (ks < 4 ? dAhi : dAlo) + ko, dX + ko, kIdesc, ks > 0 ? 1u : 0u);
            }
            mma_commit(bar_mma);
            ++mma_issued;
            if (cc + 2 < nc) prefetch(cc + 2);    // buffer cc & 1 is read
        }
        // under the product: the state carried into chunk c, to rstates (rows of
        // 128 bytes per thread, written a full line per four lanes after a transpose)
        {
            float s0[16], s1[16];
            tmem_ld32_x16(tl + 128, s0);
            tmem_ld32_x16(tl + 144, s1);
            tmem_wait_ld();
            uint4 U[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                U[k] = make_uint4(__float_as_uint(s0[4 * k]), __float_as_uint(s0[4 * k + 1]),
                                  __float_as_uint(s0[4 * k + 2]), __float_as_uint(s0[4 * k + 3]));
                U[4 + k] = make_uint4(__float_as_uint(s1[4 * k]), __float_as_uint(s1[4 * k + 1]),
                                      __float_as_uint(s1[4 * k + 2]), __float_as_uint(s1[4 * k + 3]));
            }
            octet_transpose(U, lane);
            float* dst = rstates + ((size_t)bh * nc + c) * SE + (size_t)m * kD * kD + col0 + 4 * (lane & 7);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const int r = 32 * q4 + (lane & ~7) + s;
                *reinterpret_cast<uint4*>(dst + (size_t)r * kD) = U[s];
            }
        }
        if (tid == 0) {
            if (mbar_wait(bar_mma, cc & 1)) mma_seen = mma_issued;
            else red[31] = 1.f;
        }
        __syncthreads();                          // the product is done
        tc_fence_after();
        if (red[31] != 0.f) {
            ok = false;
            break;
        }
        {
            const float Gam = expf(sb[kC - 1]), ds = sA * sX;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float dv[16], S[16];
                tmem_ld32_x16(tl + 16 * h, dv);
                tmem_ld32_x16(tl + 128 + 16 * h, S);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) S[e] = fmaf(Gam, S[e], ds * dv[e]);
                tmem_st32_x16(tl + 128 + 16 * h, S);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();                          // product and state read: the next product may start
        tc_fence_after();
    }
    if (tid == 0 && !ok) {
        record_error(err, kErrTimeout);
        // one more bounded chance for the product and the row copies in flight to drain
        if (mma_issued > mma_seen) mbar_wait(bar_mma, (mma_issued - 1) & 1);
        for (int cc = 0; cc < prefetched; ++cc) mbar_wait(bar_raw + (cc & 1), (cc >> 1) & 1);
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tbase, 256);
}

}  // namespace

cudaError_t tc_rscan_launch(const float* dout, const float* u, const float* xsol, const float* gamma, int B, int H,
                            int T, float* rstates, unsigned* err, cudaStream_t st) {
    const int nc = (T + kC - 1) / kC;
    const int smem = RscanSmem::bytes + 1024;
    const cudaError_t e = cudaFuncSetAttribute(tc_rscan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    LaunchTimer timer(kKindBwdRscan, st);
    tc_rscan_kernel<<<dim3(B * H, 2), kRThreads, smem, st>>>(dout, u, xsol, gamma, T, nc, rstates, err);
    return cudaGetLastError();
}

}  // namespace mesa
