// tc_scan.cu -- tensor-core chunk-state scan of the Mesa layer for bf16
// inputs, dk = dv = 128, chunk C = 64.
//
// Method: "MesaNet: Sequence Modeling by Locally Optimal Test-Time Training"
// (gist.science), Technical summary > Method > Mesa layer and its
// "Parallelisation" paragraph: the states carried from chunk to chunk obey
//     H_{c+1} = e^{b_last} H_c + K^T diag(w) K,   G_{c+1} = e^{b_last} G_c + V^T diag(w) K,
// with b_t the in-chunk log-cumsum of gamma and w_j = beta_j e^{b_last-b_j}.
// One CTA walks the chunks of one sequence and carries both states (or, for
// small batches, one CTA per state and sequence): they live in tensor memory
// as fp32 beside the chunk products, and the state before every 128-token
// block of the solve is written as a scaled fp16 image (format in
// tc_layout.cuh), plus the final states.
//
// Numerics: per chunk, the fp16 keys k_j / sK multiply w_j k_j / sAH and
// w_j v_j / sAG, split into fp16 hi/lo pairs, on the tensor cores with fp32
// accumulation, so each chunk's sum carries ~22-bit products into the fp32
// running states. sAH, sAG and sK are the powers of two at or above
// the chunk's largest |w_j k_j|, |w_j v_j| and |k_j| entries, so every operand
// lies in [-1, 1] whatever the size of beta, k or v; a state takes sA sK
// times its sum.
//
// Pipeline per chunk c: the products of chunk c run while the CTA writes
// chunk c+1's operand images (a second set) and reads chunk c+2's rows and
// forms their maxima; then both states take their products, the threads that
// hold them write the states before every even chunk as images, warp 1 forms
// chunk c+3's gates, and chunk c+3's rows are on their way.
#include "mesa_internal.h"
#include "preproc_row.cuh"
#include "tc_layout.cuh"

namespace mesa {
namespace {

using namespace tc;

// =====================================================================
// Chunk-state scan
// =====================================================================
// The fp16 image of a chunk-start state is scaled by s = 2^ceil(log2 Bnd)
// where Bnd bounds every entry: Bnd_0 = max|S_in| and
// Bnd_{c+1} = e^{b_last} Bnd_c + sum_j w_j |a_j|_inf |k_j|_inf (a = k for H,
// a = v for G), since |(a_j k_j^T)_il| <= |a_j|_inf |k_j|_inf. Every warp of
// the CTA evaluates the same scalar recurrences in the same order, so all
// threads agree on the scales without communicating.
constexpr int kScanThreads = 512;

struct ScanSmem {
    static constexpr int oRawK = 0;               // [64][128] bf16 rows of k (16 KB)
    static constexpr int oRawV = 16384;           // [64][128] bf16 rows of v (16 KB)
    static constexpr int oImg = 32768;            // 2 operand sets, MN-major SW128, 16 KB per image:
    static constexpr int kSet = 81920;            //   {W hi of slot 0, 1; W lo of slot 0, 1; K}
    static constexpr int oLo = 32768;             // offsets in a set (W hi of slot i at 16384 i)
    static constexpr int oK = 65536;
    static constexpr int oGate = oImg + 2 * kSet; // b[4][64], w[4][64], kmax[4][64], vmax[4][64]
    static constexpr int oRed = oGate + 4096;     // 64 floats: warp partials of H [0, 16) and G [16, 32); [32] abort
    static constexpr int oCmax = oRed + 256;      // [2 buffers][4] {max w|k|, max w|v|, max |k|, -} (int bits)
    static constexpr int oBar = oCmax + 32;       // raw, mma
    static constexpr int oSlot = oBar + 16;
    static constexpr int oConv = oSlot + 16;      // key convolution weights [4 lags][128] (fused preprocessing)
    static constexpr int oHalo = oConv + 2048;    // 2 x the 3 raw key rows before a chunk (fused preprocessing)
    static constexpr int bytes = oHalo + 2 * 768;
};
static_assert(ScanSmem::oImg % 1024 == 0 && ScanSmem::kSet % 1024 == 0, "SW128 images need 1 KB alignment");
static_assert(ScanSmem::oCmax % 16 == 0 && ScanSmem::oBar % 8 == 0, "vector and barrier alignment");

// Tensor memory of a CTA carrying kNM states (kNM = 2: H and G; kNM = 1: the
// one blockIdx.y names): the chunk product of state slot i in columns
// 128 i .. 128 i + 127, the running state of slot i in 128 (kNM + i) .. .
__host__ __device__ constexpr uint32_t col_acc(int i) { return 128u * (uint32_t)i; }
template <int kNM>
__device__ constexpr uint32_t col_state(int i) { return 128u * (uint32_t)(kNM + i); }
constexpr int kAbort = 32;

// The bf16 piece x times f, split into fp16 hi and lo parts (x f = hi + lo to
// ~22 bits).
__device__ __forceinline__ void split_hilo(uint4 raw, float f, uint4& hi, uint4& lo) {
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
    uint32_t* hw = reinterpret_cast<uint32_t*>(&hi);
    uint32_t* lw = reinterpret_cast<uint32_t*>(&lo);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(a2[i]);
        const float x0 = f * x.x, x1 = f * x.y;
        const __half2 h2 = __floats2half2_rn(x0, x1);
        const float2 hb = __half22float2(h2);
        hw[i] = *reinterpret_cast<const uint32_t*>(&h2);
        lw[i] = pack_half2(x0 - hb.x, x1 - hb.y);
    }
}

// 4 x 4 transpose of 16-byte units among the lanes of each lane quad: on
// entry lane 4q + a holds units 0..3 of its own row, on return U[s] is unit a
// of row 4q + s (the row of lane 4q + s). Two butterfly rounds: lanes a and
// a ^ m swap the units whose index differs from the lane's in bit m.
__device__ __forceinline__ void quad_transpose(uint4 (&U)[4], int lane) {
#pragma unroll
    for (int m = 2; m >= 1; m >>= 1) {
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
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

__device__ __forceinline__ float absmax8(uint4 raw) {
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
    float mx = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(a2[i]);
        mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    return mx;
}

// CTA bh walks the chunks of sequence bh, for both states (kNM = 2) or for
// state blockIdx.y (kNM = 1: H for 0, G for 1; twice the CTAs, each chunk
// about 0.7 of the time, which pays while 2 B H CTAs fit on the SMs at once).
// Warp w serves TMEM lane quadrant w % 4 (state rows 32 (w % 4) .. + 31, one
// per thread) and the 32 columns 32 (w / 4) .. + 31 of each state. Per
// chunk, with w_j = beta_j e^{b_last - b_j},
//     H <- e^{b_last} H + sAH sK sum_j (w_j k_j / sAH) (k_j / sK)^T
//     G <- e^{b_last} G + sAG sK sum_j (w_j v_j / sAG) (k_j / sK)^T
// Both sums are one product over the chunk's tokens with the keys as the
// left factor: D[l][n] = sum_j (k_j[l] / sK) W_j[n], with W_j = [w_j k_j / sAH |
// w_j v_j / sAG] (N = 256; N = 128 with one state), issued for the hi and the
// lo fp16 parts of W. Row l of D holds H[l][.] and G[.][l]: tensor memory
// carries G transposed, and so do its images (row l, column i hold G[i][l]);
// G_in and G_out keep the [i][l] layout of the interface and are read and
// written down their columns.
template <int kNM>
__global__ void __launch_bounds__(kScanThreads, 1)
tc_scan_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
               const float* __restrict__ gamma, const float* __restrict__ beta, int T, int nc,
               const float* __restrict__ H_in, const float* __restrict__ G_in, __half* __restrict__ img,
               float* __restrict__ scales, float* __restrict__ H_out, float* __restrict__ G_out,
               unsigned* __restrict__ err, const float* __restrict__ conv_k, int conv_w, int H) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int bh = blockIdx.x;
    const int m0 = kNM == 2 ? 0 : (int)blockIdx.y;     // state of slot 0 (0: H, 1: G)
    const bool with_h = kNM == 2 || m0 == 0, with_g = kNM == 2 || m0 == 1;   // with_g: v rows are needed
    uint8_t* rawK = smem + ScanSmem::oRawK;
    uint8_t* rawV = smem + ScanSmem::oRawV;
    float* sb = reinterpret_cast<float*>(smem + ScanSmem::oGate);      // [4][64]
    float* sw = sb + 4 * kC;                                            // [4][64]
    float* kmx = sw + 4 * kC;                                           // [4][64] row maxima |k_j|_inf
    float* vmx = kmx + 4 * kC;                                          // [4][64] row maxima |v_j|_inf
    float* red = reinterpret_cast<float*>(smem + ScanSmem::oRed);
    // Chunk maxima, kept as the bit patterns of non-negative floats (which
    // order like the floats), so each warp folds its maximum in with one
    // shared-memory atomicMax; buffer cc & 1, cleared after its chunk's images
    // are written.
    int* cmax = reinterpret_cast<int*>(smem + ScanSmem::oCmax);
    uint64_t* bar_raw = reinterpret_cast<uint64_t*>(smem + ScanSmem::oBar);
    uint64_t* bar_mma = bar_raw + 1;
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + ScanSmem::oSlot);
    float* sconv = reinterpret_cast<float*>(smem + ScanSmem::oConv);
    uint8_t* halo = smem + ScanSmem::oHalo;           // [2][3 rows][256 B]

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int q4 = w & 3;
    const int row = 32 * q4 + lane;               // state row owned by this thread
    const int col0 = 32 * (w >> 2);               // its 32 columns
    const size_t seq = (size_t)bh * T;
    const int np = (nc + 1) >> 1;

    // Rows of chunk cc (k, and v for G) into the row buffers (thread 0). One copy is
    // in flight at a time: the next is issued once every thread has read the
    // rows of the previous one, so the barrier's phase parity is cc & 1.
    int prefetched = 0;
    auto prefetch = [&](int cc) {
        const int nn = min(kC, T - cc * kC);
        const uint32_t bytes = (uint32_t)nn * kD * 2;
        mbar_arrive_expect_tx(bar_raw, with_g ? 2 * bytes : bytes);
        bulk_g2s(rawK, k + (seq + (size_t)cc * kC) * kD, bytes, bar_raw);
        if (with_g) bulk_g2s(rawV, v + (seq + (size_t)cc * kC) * kD, bytes, bar_raw);
        prefetched = cc + 1;
    };
    auto wait_rows = [&](int cc) {                // every thread: chunk cc's rows have landed
        if (!mbar_wait(bar_raw, cc & 1)) red[kAbort] = 1.f;
    };
    // Warp 1: gamma and beta of chunk cc into registers (lane: positions 2 lane, 2 lane + 1;
    // padding positions read as gamma = 1, beta = 0).
    float pg0 = 1.f, pg1 = 1.f, pb0 = 0.f, pb1 = 0.f;
    auto load_gates = [&](int cc) {
        const int nn = min(kC, T - cc * kC);
        const size_t base = seq + (size_t)cc * kC;
        const int t0 = 2 * lane, t1 = 2 * lane + 1;
        pg0 = t0 < nn ? gamma[base + t0] : 1.f;
        pg1 = t1 < nn ? gamma[base + t1] : 1.f;
        pb0 = t0 < nn ? beta[base + t0] : 0.f;
        pb1 = t1 < nn ? beta[base + t1] : 0.f;
    };
    // Warp 1: from the loaded gates of chunk cc, b (the in-chunk inclusive
    // log-cumsum of gamma) and w_j = beta_j e^{b_last - b_j} into buffer cc & 3.
    auto chunk_gates = [&](int cc) {
        float* b = sb + (cc & 3) * kC;
        float* wv = sw + (cc & 3) * kC;
        const float l0 = logf(pg0), l1 = logf(pg1);
        const float pair = l0 + l1;
        float incl = pair;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o;
        }
        const float b0 = incl - pair + l0, b1 = incl;
        const float bl = __shfl_sync(0xffffffffu, incl, 31);     // b at the chunk's last position
        b[2 * lane] = b0;
        b[2 * lane + 1] = b1;
        wv[2 * lane] = pb0 * expf(bl - b0);
        wv[2 * lane + 1] = pb1 * expf(bl - b1);
    };
    // Operand images of chunk cc, in two phases a pipeline stage apart.
    // build_load (stage cc-2): this thread's two 16-byte pieces of the k and
    // v rows into registers, the row maxima of |k| and |v| into buffer cc & 3
    // (for the state bounds) and this warp's maxima of w_j |k_j|, w_j |v_j|
    // and |k_j| into cmax buffer cc & 1 (for the chunk's operand scales).
    // build_store (stage cc-1): the scales from cmax, then w_j k_j / sAH and
    // w_j v_j / sAG (hi/lo) [j][i] and K = k_j / sK [j][l] into set cc & 1,
    // all MN-major SW128 in 64-column blocks; returns (sAH sK, sAG sK), the
    // factors the chunk's products carry.
    // Fused input preprocessing of the keys (conv_k given): the raw piece of
    // row j of chunk cc becomes its convolved, normalised bf16 piece. The rows
    // before it come from the chunk's raw rows or, for its first three rows,
    // from the halo buffer cc & 1, which holds the previous chunk's last three
    // raw rows (zero before the sequence start); the chunk's own last three
    // raw rows go to halo buffer (cc + 1) & 1. Padding rows (j >= n) give zero.
    auto preprocess_key = [&](int cc, int n, int j, int cc16, uint4 raw) -> uint4 {
        uint4 x[pre::kMaxW];
        x[0] = raw;
#pragma unroll
        for (int w = 1; w < pre::kMaxW; ++w)
            x[w] = j >= w ? *reinterpret_cast<const uint4*>(rawK + (j - w) * 256 + cc16 * 16)
                          : *reinterpret_cast<const uint4*>(halo + (cc & 1) * 768 + (3 + j - w) * 256 + cc16 * 16);
        if (j >= kC - 3) *reinterpret_cast<uint4*>(halo + ((cc + 1) & 1) * 768 + (j - (kC - 3)) * 256 + cc16 * 16) = raw;
        const uint4 y = pre::conv_norm_bf16x8_sw<kD, 16>(sconv, cc16 * 8, x);
        return j < n ? y : make_uint4(0, 0, 0, 0);
    };
    uint4 rk[2], rv[2];
    auto build_load = [&](int cc) {
        const int n = min(kC, T - cc * kC);
        const float* swc = sw + (cc & 3) * kC;
        float* km = kmx + (cc & 3) * kC;
        float* vm = vmx + (cc & 3) * kC;
        float wk = 0.f, wv = 0.f, kk = 0.f;
#pragma unroll
        for (int rep = 0; rep < 2; ++rep) {
            const int cid = tid + kScanThreads * rep;      // 1024 16-byte pieces of each chunk's rows
            const int j = cid >> 4, cc16 = cid & 15;
            rk[rep] = make_uint4(0, 0, 0, 0);
            rv[rep] = make_uint4(0, 0, 0, 0);
            if (j < n) {
                rk[rep] = *reinterpret_cast<const uint4*>(rawK + j * 256 + cc16 * 16);
                if (with_g) rv[rep] = *reinterpret_cast<const uint4*>(rawV + j * 256 + cc16 * 16);
            }
            if (conv_k) rk[rep] = preprocess_key(cc, n, j, cc16, rk[rep]);
            float mk = absmax8(rk[rep]), mv = absmax8(rv[rep]);
            // row maxima over the 16 threads (same half-warp) that hold row j
#pragma unroll
            for (int o2 = 8; o2 >= 1; o2 >>= 1) {
                mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, o2));
                mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, o2));
            }
            if (cc16 == 0) {
                km[j] = mk;
                vm[j] = mv;
            }
            wk = fmaxf(wk, swc[j] * mk);
            wv = fmaxf(wv, swc[j] * mv);
            kk = fmaxf(kk, mk);
        }
        wk = fmaxf(wk, __shfl_xor_sync(0xffffffffu, wk, 16));   // the warp's other row
        wv = fmaxf(wv, __shfl_xor_sync(0xffffffffu, wv, 16));
        kk = fmaxf(kk, __shfl_xor_sync(0xffffffffu, kk, 16));
        if (lane == 0) {
            atomicMax(cmax + 4 * (cc & 1), __float_as_int(wk));
            atomicMax(cmax + 4 * (cc & 1) + 1, __float_as_int(wv));
            atomicMax(cmax + 4 * (cc & 1) + 2, __float_as_int(kk));
        }
    };
    auto build_store = [&](int cc) -> float2 {
        const float* swc = sw + (cc & 3) * kC;
        uint8_t* set = smem + ScanSmem::oImg + (cc & 1) * ScanSmem::kSet;
        const int4 c4 = *reinterpret_cast<const int4*>(cmax + 4 * (cc & 1));
        const float sAH = pow2_ceil(__int_as_float(c4.x)), sAG = pow2_ceil(__int_as_float(c4.y));
        const float sK = pow2_ceil(__int_as_float(c4.z));
        const float iAH = 1.f / sAH, iAG = 1.f / sAG, iK = 1.f / sK;   // powers of two: exact
#pragma unroll
        for (int rep = 0; rep < 2; ++rep) {
            const int cid = tid + kScanThreads * rep;
            const int j = cid >> 4, cc16 = cid & 15;
            const uint32_t off = (uint32_t)((cc16 >> 3) * 8192 + j * 128 + (((cc16 & 7) ^ (j & 7)) << 4));
            uint4 hi, lo;
            if (with_h) {                          // slot 0
                split_hilo(rk[rep], swc[j] * iAH, hi, lo);
                *reinterpret_cast<uint4*>(set + off) = hi;
                *reinterpret_cast<uint4*>(set + ScanSmem::oLo + off) = lo;
            }
            if (with_g) {                          // slot kNM - 1
                split_hilo(rv[rep], swc[j] * iAG, hi, lo);
                *reinterpret_cast<uint4*>(set + 16384 * (kNM - 1) + off) = hi;
                *reinterpret_cast<uint4*>(set + ScanSmem::oLo + 16384 * (kNM - 1) + off) = lo;
            }
            *reinterpret_cast<uint4*>(set + ScanSmem::oK + off) = bf16x8_to_f16x8(rk[rep], iK);
        }
        return make_float2(sAH * sK, sAG * sK);
    };
    // The state row's 32 columns as fp16 / s: 16 columns (col0 + 16 h ..)
    // into units 2h, 2h + 1; then the row's four units into the image at
    // index ci (the solve's layout: two 64-column blocks, 16-byte units
    // XOR-permuted by row & 7). After a transpose within each lane quad, the
    // four lanes of a quad write the 64 contiguous bytes of one row per store.
    auto pack_units16 = [&](uint4 (&U)[4], int h, const float (&St)[16], float inv) {
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            uint4 o;
            o.x = pack_half2(St[8 * g] * inv, St[8 * g + 1] * inv);
            o.y = pack_half2(St[8 * g + 2] * inv, St[8 * g + 3] * inv);
            o.z = pack_half2(St[8 * g + 4] * inv, St[8 * g + 5] * inv);
            o.w = pack_half2(St[8 * g + 6] * inv, St[8 * g + 7] * inv);
            U[2 * h + g] = o;
        }
    };
    auto write_units = [&](size_t ci, uint4 (&U)[4]) {
        quad_transpose(U, lane);
        const int a = lane & 3;
        uint8_t* blk = reinterpret_cast<uint8_t*>(img + ci * kImgHalves) + (col0 >> 6) * 16384;
        const int u = ((col0 & 63) >> 3) + a;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int r = 32 * q4 + (lane & ~3) + s;
            *reinterpret_cast<uint4*>(blk + r * 128 + ((u ^ (r & 7)) << 4)) = U[s];
        }
    };

    // 16 entries of a state as this thread holds them (TMEM lane `row`,
    // columns col0 + 16 h ..): H[row][col] for H (mm = 0), G[col][row] for G,
    // which tensor memory carries transposed; the G accesses are coalesced
    // across the warp's consecutive rows.
    auto load16 = [&](const float* src, int mm, int h, float (&S)[16]) {
        const float* base = src + (size_t)bh * kD * kD;
        if (mm == 0) {
            const float4* s4 = reinterpret_cast<const float4*>(base + (size_t)row * kD + col0 + 16 * h);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 f = s4[i];
                S[4 * i] = f.x; S[4 * i + 1] = f.y; S[4 * i + 2] = f.z; S[4 * i + 3] = f.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) S[i] = base[(size_t)(col0 + 16 * h + i) * kD + row];
        }
    };
    auto store16 = [&](float* dst, int mm, int h, const float (&S)[16]) {
        float* base = dst + (size_t)bh * kD * kD;
        if (mm == 0) {
            float4* d4 = reinterpret_cast<float4*>(base + (size_t)row * kD + col0 + 16 * h);
#pragma unroll
            for (int i = 0; i < 4; ++i) d4[i] = make_float4(S[4 * i], S[4 * i + 1], S[4 * i + 2], S[4 * i + 3]);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) base[(size_t)(col0 + 16 * h + i) * kD + row] = S[i];
        }
    };

    if (tid == 0) {
        mbar_init(bar_raw, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        red[kAbort] = 0.f;
    }
    if (tid < 8) cmax[tid] = 0;
    if (conv_k) {                                  // fused preprocessing: weights, zero rows before t = 0
        pre::stage_weights<kD>(conv_k + (size_t)(bh % H) * conv_w * kD, conv_w, sconv);
        for (int e = tid; e < 768 / 16; e += kScanThreads) reinterpret_cast<uint4*>(halo)[e] = make_uint4(0, 0, 0, 0);
    }
    if (w == 0) tmem_alloc(slot, 256 * kNM);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *slot;
    const uint32_t tl = tbase + ((uint32_t)(32 * q4) << 16) + col0;    // this thread's lane and first column
    if (tid == 0 && nc > 0) prefetch(0);

    // The initial states (zero without H_in / G_in) into tensor memory, and
    // max |S_in| over each matrix for the entry bounds.
#pragma unroll
    for (int i = 0; i < kNM; ++i) {
        const int mm = m0 + i;
        const float* init = mm ? G_in : H_in;
        float* fin = mm ? G_out : H_out;
        float mx = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float S[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) S[e] = 0.f;
            if (init) load16(init, mm, h, S);
#pragma unroll
            for (int e = 0; e < 16; ++e) mx = fmaxf(mx, fabsf(S[e]));
            if (nc == 0 && fin) store16(fin, mm, h, S);    // no tokens: the final state is the initial one
            tmem_st32_x16(tl + col_state<kNM>(i) + 16 * h, S);
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) red[16 * i + w] = mx;
    }
    tmem_wait_st();
    if (w == 1) {                                  // gates of chunks 0..2, gamma and beta of chunk 3
        for (int cc = 0; cc < 3 && cc < nc; ++cc) {
            load_gates(cc);
            chunk_gates(cc);
        }
        if (nc > 3) load_gates(3);
    }
    tc_fence_before();
    __syncthreads();                              // gates and the bounds' partials visible
    tc_fence_after();
    float bnd[kNM];                               // entry bounds of the slots' states
#pragma unroll
    for (int i = 0; i < kNM; ++i) {
        bnd[i] = red[16 * i];
#pragma unroll
        for (int e = 1; e < 16; ++e) bnd[i] = fmaxf(bnd[i], red[16 * i + e]);
    }
    bool ok = red[kAbort] == 0.f;

    constexpr uint32_t kIdesc = idesc_f16(128, 128 * kNM, true, true);
    auto issue_mma = [&](int cc) {                // thread 0: the chunk's 8 K steps (W hi, then W lo) into TMEM
        const uint8_t* set = smem + ScanSmem::oImg + (cc & 1) * ScanSmem::kSet;
        const uint64_t dA = sdesc(smem_addr(set + ScanSmem::oK), 8192, 1024);
        const uint64_t dBhi = sdesc(smem_addr(set), 8192, 1024), dBlo = sdesc(smem_addr(set + ScanSmem::oLo), 8192, 1024);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t ko = ((ks & 3) * 2048) >> 4;
            mma_f16(tbase + col_acc(0), dA + ko, (ks < 4 ? dBhi : dBlo) + ko, kIdesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar_mma);
    };
    int mma_issued = 0, mma_seen = 0;             // thread 0
    float2 ds_cur = make_float2(1.f, 1.f), ds_next = ds_cur;   // sA sK of the chunk in the MMA, of the next chunk
    if (ok && nc > 0) {
        // the states before chunk 0 (block 0's images), chunk 0's operands, chunk 1's rows
#pragma unroll
        for (int i = 0; i < kNM; ++i) {
            const size_t ci = image_index(bh, np, 0, m0 + i);
            const float inv = 1.f / pow2_ceil(bnd[i]);
            uint4 U[4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float S[16];
                tmem_ld32_x16(tl + col_state<kNM>(i) + 16 * h, S);
                tmem_wait_ld();
                pack_units16(U, h, S, inv);
            }
            write_units(ci, U);
        }
        if (tid == 0)
            for (int i = 0; i < kNM; ++i) scales[image_index(bh, np, 0, m0 + i)] = pow2_ceil(bnd[i]);
        wait_rows(0);
        build_load(0);
        __syncthreads();                          // chunk 0's maxima; its rows are read
        if (tid == 0 && nc > 1) prefetch(1);
        ds_cur = build_store(0);
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid < 4) cmax[tid] = 0;               // buffer 0 is free for chunk 2
        if (tid == 0 && red[kAbort] == 0.f) {
            issue_mma(0);
            ++mma_issued;
        }
        if (nc > 1) {
            wait_rows(1);
            build_load(1);
        }
        __syncthreads();                          // chunk 1's maxima; its rows are read
        if (tid == 0 && nc > 2) prefetch(2);
        ok = red[kAbort] == 0.f;
    }
    int c = 0;
    for (; ok && c < nc; ++c) {
        // ---- under the products of chunk c: chunk c+1's images, chunk c+2's
        //      rows and maxima, the bounds after chunk c ----
        if (c + 1 < nc) ds_next = build_store(c + 1);
        if (c + 2 < nc) {
            wait_rows(c + 2);
            build_load(c + 2);
        }
        const float blast = sb[(c & 3) * kC + kC - 1];
        {
            // every warp reduces the same 64 terms in the same order, so every
            // thread gets the same values
            const float* swc = sw + (c & 3) * kC;
            const float* km = kmx + (c & 3) * kC;
            const float* vm = vmx + (c & 3) * kC;
            float addH = swc[lane] * (km[lane] * km[lane]) + swc[lane + 32] * (km[lane + 32] * km[lane + 32]);
            float addG = swc[lane] * (vm[lane] * km[lane]) + swc[lane + 32] * (vm[lane + 32] * km[lane + 32]);
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
                addH += __shfl_xor_sync(0xffffffffu, addH, off);
                addG += __shfl_xor_sync(0xffffffffu, addG, off);
            }
            const float eb = expf(blast);
#pragma unroll
            for (int i = 0; i < kNM; ++i) bnd[i] = fmaf(eb, bnd[i], m0 + i ? addG : addH);
        }
        const bool emit = c + 1 < nc && ((c + 1) & 1) == 0;
        if (tid == 0) {
            if (mbar_wait(bar_mma, c & 1)) mma_seen = mma_issued;
            else red[kAbort] = 1.f;
        }
        __syncthreads();                          // products of c done; images of c+1, maxima of c+2 written
        tc_fence_after();
        if (red[kAbort] != 0.f) {
            ok = false;
            break;
        }
        if (tid == 0 && c + 3 < nc) prefetch(c + 3);        // chunk c+2's rows are read
        if (tid < 4) cmax[4 * ((c + 1) & 1) + tid] = 0;      // chunk c+1's images are written: free for c+3
        // warp 1: chunk c+3's gates (its buffer last served chunk c-1's bound),
        // next to the other warps' tensor-memory traffic
        if (w == 1 && c + 3 < nc) {
            chunk_gates(c + 3);
            if (c + 4 < nc) load_gates(c + 4);
        }
        // ---- S <- e^{b_last} S + sA sK Delta, for H and G; the images of the
        //      states before chunk c+1 when it starts a block; the final states ----
        const float Gam = expf(blast);
        const bool last = c + 1 == nc;
#pragma unroll
        for (int i = 0; i < kNM; ++i) {
            const int mm = m0 + i;
            const float ds = mm ? ds_cur.y : ds_cur.x;
            const float inv = 1.f / pow2_ceil(bnd[i]);
            const size_t ci = image_index(bh, np, (c + 1) >> 1, mm);
            float* fin = mm ? G_out : H_out;
            uint4 U[4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float dv[16], S[16];
                tmem_ld32_x16(tl + col_acc(i) + 16 * h, dv);
                tmem_ld32_x16(tl + col_state<kNM>(i) + 16 * h, S);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) S[e] = fmaf(Gam, S[e], ds * dv[e]);
                if (last) {
                    if (fin) store16(fin, mm, h, S);
                } else {
                    tmem_st32_x16(tl + col_state<kNM>(i) + 16 * h, S);
                    if (emit) pack_units16(U, h, S, inv);
                }
            }
            if (!last && emit) write_units(ci, U);
        }
        if (last) break;
        tmem_wait_st();
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();                          // products read; chunk c+1's images written
        tc_fence_after();
        if (tid == 0) {
            if (emit)
                for (int i = 0; i < kNM; ++i) scales[image_index(bh, np, (c + 1) >> 1, m0 + i)] = pow2_ceil(bnd[i]);
            issue_mma(c + 1);
            ++mma_issued;
        }
        ds_cur = ds_next;
    }
    if (tid == 0 && !ok) {
        record_error(err, kErrTimeout);
        // one more bounded chance for the products and the row copy in flight to drain
        if (mma_issued > mma_seen) mbar_wait(bar_mma, (mma_issued - 1) & 1);
        if (prefetched > 0) mbar_wait(bar_raw, (prefetched - 1) & 1);
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tbase, 256 * kNM);
}

}  // namespace

// One CTA per state and sequence while all 2 B H of them fit on the SMs at
// once (a chain of chunks is then as short as it gets); one CTA per sequence
// carrying both states otherwise (half the CTAs, each chunk ~1.45 times as long).
cudaError_t tc_scan_launch(const ForwardArgs& a, void* img, float* scales, unsigned* err, cudaStream_t st) {
    const int nc = (a.T + kC - 1) / kC;
    const int smem = ScanSmem::bytes + 1024;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long seqs = (long long)a.B * a.H;
    const bool split = 2 * seqs <= sms;
    auto kern = split ? tc_scan_kernel<1> : tc_scan_kernel<2>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    LaunchTimer timer(kKindTcScan, st);
    kern<<<dim3((unsigned)seqs, split ? 2 : 1), kScanThreads, smem, st>>>(
        static_cast<const __nv_bfloat16*>(a.k), static_cast<const __nv_bfloat16*>(a.v), a.gamma, a.beta, a.T, nc,
        a.H_in, a.G_in, static_cast<__half*>(img), scales, a.H_out, a.G_out, err, a.conv_k, a.conv_w, a.H);
    return cudaGetLastError();
}

}  // namespace mesa
