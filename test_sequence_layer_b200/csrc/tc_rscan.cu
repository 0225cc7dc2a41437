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

// Shared memory of a CTA carrying kNM states. kNM = 1: the rows of a and x in
// two buffers each (the chunk after next is requested once a chunk's rows are
// read); kNM = 2: the rows of u, dL/do and x in one buffer each (the next
// chunk is requested then). Then the fp16 images {A hi, A lo} per state and X,
// MN-major SW128, 16 KB each; both layouts end at the same offset.
template <int kNM>
struct RscanSmem {
    static constexpr int kBufs = kNM == 1 ? 2 : 1;           // row buffers
    static constexpr int oRawA = 0;                          // [kBufs][kNM][64][128] fp32 rows of a
    static constexpr int oRawX = kBufs * kNM * 32768;        // [kBufs][64][128] fp32 rows of x
    static constexpr int oImg = oRawX + kBufs * 32768;       // A hi/lo of state slot i at 32 KB i, X after them
    static constexpr int oX = kNM * 32768;
    static constexpr int oGate = oImg + oX + 16384;          // b[64], w[64]
    static constexpr int oRed = oGate + 512;                 // 32 floats; [31] is the abort flag
    static constexpr int oCmax = oRed + 128;                 // {max |x|, max w|a| per slot} (int bits)
    static constexpr int oBar = oCmax + 16;                  // raw[2], mma
    static constexpr int oSlot = oBar + 32;
    static constexpr int bytes = oSlot + 16;
    static_assert(oImg % 1024 == 0, "SW128 images need 1 KB alignment");
};

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

// CTA bh walks the chunks of sequence bh from the last to the first for both
// states (kNM = 2) or for state blockIdx.y (kNM = 1): Hhat (rows from u) or
// Ghat (rows from dL/do); both share x. Warp w serves
// TMEM lane quadrant w % 4 (state rows 32 (w % 4) .. + 31, one per thread)
// and the 32 columns 32 (w / 4) .. + 31; tensor memory holds the chunk's
// product of state slot i (columns 128 i ..) and its running state
// (128 (kNM + i) ..). Per chunk: the gates (warp 1), the operand scales from
// the chunk's maxima, the fp16 images, one M = N = 128, K = 64 product (hi and
// lo) per state, during which the states carried into the chunk are written
// out, and the state updates. The rows of a later chunk are on their way by
// bulk copy meanwhile.
template <int kNM>
__global__ void __launch_bounds__(kRThreads, 1)
tc_rscan_kernel(const float* __restrict__ dout, const float* __restrict__ u, const float* __restrict__ xsol,
                const float* __restrict__ gamma, int T, int nc, float* __restrict__ rstates,
                unsigned* __restrict__ err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    using L = RscanSmem<kNM>;
    constexpr int NB = L::kBufs;
    const int bh = blockIdx.x;
    const int m0 = kNM == 2 ? 0 : (int)blockIdx.y;   // state of slot 0 (0: Hhat, 1: Ghat)
    float* rawA = reinterpret_cast<float*>(smem + L::oRawA);
    float* rawX = reinterpret_cast<float*>(smem + L::oRawX);
    uint8_t* img = smem + L::oImg;
    float* sb = reinterpret_cast<float*>(smem + L::oGate);
    float* sw = sb + kC;
    float* red = reinterpret_cast<float*>(smem + L::oRed);
    int* cmax = reinterpret_cast<int*>(smem + L::oCmax);
    uint64_t* bar_raw = reinterpret_cast<uint64_t*>(smem + L::oBar);
    uint64_t* bar_mma = bar_raw + 2;
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L::oSlot);

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int q4 = w & 3;
    const int row = 32 * q4 + lane;
    const int col0 = 32 * (w >> 2);
    const size_t seq = (size_t)bh * T;
    constexpr size_t SE = 2 * (size_t)kD * kD;

    // rows of the cc-th chunk walked (chunk nc - 1 - cc) into buffer cc % NB (thread 0)
    int prefetched = 0;
    auto prefetch = [&](int cc) {
        const int c = nc - 1 - cc;
        const int nn = min(kC, T - c * kC);
        const uint32_t bytes = (uint32_t)nn * kD * 4;
        const int buf = cc % NB;
        mbar_arrive_expect_tx(bar_raw + buf, (kNM + 1) * bytes);
#pragma unroll
        for (int i = 0; i < kNM; ++i) {
            const float* A = m0 + i ? dout : u;
            bulk_g2s(rawA + (buf * kNM + i) * kC * kD, A + (seq + (size_t)c * kC) * kD, bytes, bar_raw + buf);
        }
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
    if (w == 0) tmem_alloc(slot, 256 * kNM);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *slot;
    const uint32_t tl = tbase + ((uint32_t)(32 * q4) << 16) + col0;
    {
        float z[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) z[e] = 0.f;
#pragma unroll
        for (int i = 0; i < kNM; ++i) {
            tmem_st32_x16(tl + 128 * (kNM + i), z);
            tmem_st32_x16(tl + 128 * (kNM + i) + 16, z);
        }
        tmem_wait_st();
    }
    if (tid == 0 && nc > 0) {
        prefetch(0);
        if (NB == 2 && nc > 1) prefetch(1);
    }
    if (w == 1 && nc > 0) load_gates(nc - 1);

    constexpr uint32_t kIdesc = idesc_f16(128, 128, true, true);
    int mma_issued = 0, mma_seen = 0;             // thread 0
    bool ok = true;
    for (int cc = 0; cc < nc; ++cc) {
        const int c = nc - 1 - cc;
        const int n = min(kC, T - c * kC);
        const int buf = cc % NB;
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
        if (tid < kNM + 1) cmax[tid] = 0;
        if (!mbar_wait(bar_raw + buf, (cc / NB) & 1)) red[31] = 1.f;
        __syncthreads();                          // gates, cleared maxima, rows landed
        if (red[31] != 0.f) {
            ok = false;
            break;
        }
        // the chunk's maxima of |x_t| and w_t |a_t| (rows past n hold stale data: skipped)
        {
            float mx = 0.f, ma[kNM];
#pragma unroll
            for (int i = 0; i < kNM; ++i) ma[i] = 0.f;
#pragma unroll
            for (int rep = 0; rep < 4; ++rep) {
                const int e = tid + kRThreads * rep;       // 2048 float4 pieces of each chunk's rows
                const int t = e >> 5, q = e & 31;
                if (t < n) {
                    mx = fmaxf(mx, absmax4(*reinterpret_cast<const float4*>(rx + t * kD + 4 * q)));
#pragma unroll
                    for (int i = 0; i < kNM; ++i)
                        ma[i] = fmaxf(ma[i], sw[t] * absmax4(*reinterpret_cast<const float4*>(
                                                             rawA + (buf * kNM + i) * kC * kD + t * kD + 4 * q)));
                }
            }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
#pragma unroll
                for (int i = 0; i < kNM; ++i) ma[i] = fmaxf(ma[i], __shfl_xor_sync(0xffffffffu, ma[i], off));
            }
            if (lane == 0) {
                atomicMax(cmax, __float_as_int(mx));
#pragma unroll
                for (int i = 0; i < kNM; ++i) atomicMax(cmax + 1 + i, __float_as_int(ma[i]));
            }
        }
        __syncthreads();
        const float sX = pow2_ceil(__int_as_float(cmax[0]));
        float sA[kNM];
#pragma unroll
        for (int i = 0; i < kNM; ++i) sA[i] = pow2_ceil(__int_as_float(cmax[1 + i]));
        {
            const float iX = 1.f / sX;                              // powers of two: exact
            float iA[kNM];
#pragma unroll
            for (int i = 0; i < kNM; ++i) iA[i] = 1.f / sA[i];
#pragma unroll
            for (int rep = 0; rep < 2; ++rep) {
                const int e = tid + kRThreads * rep;       // 1024 units of 8 columns of each image
                const int t = e >> 4, cc16 = e & 15;
                const uint32_t off = (uint32_t)((cc16 >> 3) * 8192 + t * 128 + (((cc16 & 7) ^ (t & 7)) << 4));
                float4 x0 = make_float4(0.f, 0.f, 0.f, 0.f), x1 = x0;
                if (t < n) {
                    x0 = *reinterpret_cast<const float4*>(rx + t * kD + 8 * cc16);
                    x1 = *reinterpret_cast<const float4*>(rx + t * kD + 8 * cc16 + 4);
                }
                uint4 xo;
                xo.x = pack_half2(x0.x * iX, x0.y * iX);
                xo.y = pack_half2(x0.z * iX, x0.w * iX);
                xo.z = pack_half2(x1.x * iX, x1.y * iX);
                xo.w = pack_half2(x1.z * iX, x1.w * iX);
                *reinterpret_cast<uint4*>(img + L::oX + off) = xo;
#pragma unroll
                for (int i = 0; i < kNM; ++i) {
                    const float* ra = rawA + (buf * kNM + i) * kC * kD;
                    float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
                    if (t < n) {
                        a0 = *reinterpret_cast<const float4*>(ra + t * kD + 8 * cc16);
                        a1 = *reinterpret_cast<const float4*>(ra + t * kD + 8 * cc16 + 4);
                    }
                    const float f = sw[t] * iA[i];
                    const float av[8] = {a0.x * f, a0.y * f, a0.z * f, a0.w * f,
                                         a1.x * f, a1.y * f, a1.z * f, a1.w * f};
                    uint4 hi, lo;
                    uint32_t* hw = reinterpret_cast<uint32_t*>(&hi);
                    uint32_t* lw = reinterpret_cast<uint32_t*>(&lo);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const __half2 h2 = __floats2half2_rn(av[2 * k], av[2 * k + 1]);
                        const float2 hb = __half22float2(h2);
                        hw[k] = *reinterpret_cast<const uint32_t*>(&h2);
                        lw[k] = pack_half2(av[2 * k] - hb.x, av[2 * k + 1] - hb.y);
                    }
                    *reinterpret_cast<uint4*>(img + 32768 * i + off) = hi;
                    *reinterpret_cast<uint4*>(img + 32768 * i + 16384 + off) = lo;
                }
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();                          // images written; the chunk's raw rows are read
        tc_fence_after();
        if (tid == 0) {
            const uint64_t dX = sdesc(smem_addr(img + L::oX), 8192, 1024);
#pragma unroll
            for (int i = 0; i < kNM; ++i) {
                const uint64_t dAhi = sdesc(smem_addr(img + 32768 * i), 8192, 1024);
                const uint64_t dAlo = sdesc(smem_addr(img + 32768 * i + 16384), 8192, 1024);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t ko = ((ks & 3) * 2048) >> 4;
                    mma_f16(tbase + 128 * i, (ks < 4 ? dAhi : dAlo) + ko, dX + ko, kIdesc, ks > 0 ? 1u : 0u);
                }
            }
            mma_commit(bar_mma);
            ++mma_issued;
            if (cc + NB < nc) prefetch(cc + NB);  // buffer cc % NB is read
        }
        // under the product: the state carried into chunk c, to rstates (rows of
        // 128 bytes per thread, written a full line per four lanes after a transpose)
#pragma unroll
        for (int i = 0; i < kNM; ++i) {
            float s0[16], s1[16];
            tmem_ld32_x16(tl + 128 * (kNM + i), s0);
            tmem_ld32_x16(tl + 128 * (kNM + i) + 16, s1);
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
            float* dst = rstates + ((size_t)bh * nc + c) * SE + (size_t)(m0 + i) * kD * kD + col0 + 4 * (lane & 7);
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
            const float Gam = expf(sb[kC - 1]);
#pragma unroll
            for (int i = 0; i < kNM; ++i) {
                const float ds = sA[i] * sX;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float dv[16], S[16];
                    tmem_ld32_x16(tl + 128 * i + 16 * h, dv);
                    tmem_ld32_x16(tl + 128 * (kNM + i) + 16 * h, S);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) S[e] = fmaf(Gam, S[e], ds * dv[e]);
                    tmem_st32_x16(tl + 128 * (kNM + i) + 16 * h, S);
                }
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
        for (int cc = max(0, prefetched - NB); cc < prefetched; ++cc)     // each buffer's latest copy
            mbar_wait(bar_raw + cc % NB, (cc / NB) & 1);
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tbase, 256 * kNM);
}

}  // namespace

// One CTA per state and sequence while all 2 B H of them fit on the SMs at
// once; one CTA per sequence carrying both states (x read once) otherwise.
cudaError_t tc_rscan_launch(const float* dout, const float* u, const float* xsol, const float* gamma, int B, int H,
                            int T, float* rstates, unsigned* err, cudaStream_t st) {
    const int nc = (T + kC - 1) / kC;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long seqs = (long long)B * H;
    const bool split = 2 * seqs <= sms;
    const int smem = (split ? RscanSmem<1>::bytes : RscanSmem<2>::bytes) + 1024;
    auto kern = split ? tc_rscan_kernel<1> : tc_rscan_kernel<2>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    LaunchTimer timer(kKindBwdRscan, st);
    kern<<<dim3((unsigned)seqs, split ? 2 : 1), kRThreads, smem, st>>>(dout, u, xsol, gamma, T, nc, rstates, err);
    return cudaGetLastError();
}

}  // namespace mesa
