// tc_scan.cu -- tensor-core chunk-state scan of the Mesa layer for bf16
// inputs, dk = dv = 128, chunk C = 64.
//
// Method: "MesaNet: Sequence Modeling by Locally Optimal Test-Time Training"
// (gist.science), Technical summary > Method > Mesa layer and its
// "Parallelisation" paragraph: the states carried from chunk to chunk obey
//     H_{c+1} = e^{b_last} H_c + K^T diag(w) K,   G_{c+1} = e^{b_last} G_c + V^T diag(w) K,
// with b_t the in-chunk log-cumsum of gamma and w_j = beta_j e^{b_last-b_j}.
// The kernel walks the chunks of each sequence, keeps the running state in
// fp32 registers and writes the state before every 128-token block of the
// solve as a scaled fp16 image (format in tc_layout.cuh), plus the final state.
//
// Numerics: per chunk, w_j a_j / sA is split into an fp16 hi/lo pair and
// multiplied by the fp16 keys k_j / sK on the tensor cores with fp32
// accumulation, so each chunk's sum carries ~22-bit products into the fp32
// running state. sA and sK are the powers of two at or above the chunk's
// largest |w_j a_j| and |k_j| entries, so every operand lies in [-1, 1]
// whatever the size of beta, k or v; the state takes sA sK times the sum.
//
// Pipeline per chunk c: MMA(c) runs while the CTA writes chunk c+1's operand
// images (a second set), reads chunk c+2's rows and forms their maxima, and
// warp 1 forms chunk c+3's gates; then the state takes Delta_c, and the state
// before every even chunk is staged in shared memory and stored with one bulk
// copy.
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
// the CTA evaluates the same scalar recurrence in the same order, so all
// threads agree on the scale without communicating.
constexpr int kScanThreads = 512;

struct ScanSmem {
    static constexpr int oRawA = 0;               // 2 x [64][128] bf16 rows of a (16 KB each)
    static constexpr int oRawK = 32768;           // 2 x [64][128] bf16 rows of k
    static constexpr int oImg = 65536;            // 2 operand sets {A hi, A lo, B}, MN-major SW128, 16 KB each
    static constexpr int kSet = 49152;
    static constexpr int oStage = oImg + 2 * kSet;    // staged state image for the bulk store (32 KB)
    static constexpr int oGate = oStage + 32768;  // b[4][64], w[4][64], amax[4][64], kmax[4][64]
    static constexpr int oRed = oGate + 4096;     // 32 floats; [31] is the abort flag
    static constexpr int oCmax = oRed + 128;      // [2 buffers] {max w|a|, max |k|} of a chunk (as int bits)
    static constexpr int oBar = oCmax + 256;      // raw[2], mma
    static constexpr int oSlot = oBar + 32;
    static constexpr int oConv = oSlot + 16;      // key convolution weights [4 lags][128] (fused preprocessing)
    static constexpr int oHalo = oConv + 2048;    // 2 x the 3 raw key rows before a chunk (fused preprocessing)
    static constexpr int bytes = oHalo + 2 * 768;
};

// CTA (m, bh) walks the chunks of sequence bh for m = 0 (H, a = k) or m = 1
// (G, a = v) and holds the whole 128 x 128 running state in registers: warp w
// serves TMEM lane quadrant w % 4 (state rows 32 (w % 4) .. + 31, one per
// thread) and the 32 columns 32 (w / 4) .. + 31. Per chunk, with
// w_j = beta_j e^{b_last - b_j},
//     S <- e^{b_last} S + sA sK sum_j (w_j a_j / sA) (k_j / sK)^T
// where the sum is one M = 128, N = 128, K = 64 MMA over the chunk's tokens,
// issued for the hi and the lo fp16 parts of w_j a_j / sA. The chunks are
// pipelined so that everything but the state update runs under the MMA of
// chunk c: the operand images of chunk c+1 are written (a second set, with
// scales from chunk c+1's maxima, formed one chunk earlier), the rows of
// chunk c+2 are read into registers and their maxima formed, warp 1 forms
// chunk c+3's gates from gamma and beta it loaded a chunk earlier, and the
// rows of chunk c+4 are on their way. The state before every even chunk is
// staged in shared memory in the solve's image layout and written with one
// bulk copy.
__global__ void __launch_bounds__(kScanThreads, 1)
tc_scan_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
               const float* __restrict__ gamma, const float* __restrict__ beta, int T, int nc,
               const float* __restrict__ H_in, const float* __restrict__ G_in, __half* __restrict__ img,
               float* __restrict__ scales, float* __restrict__ H_out, float* __restrict__ G_out,
               unsigned* __restrict__ err, const float* __restrict__ conv_k, int conv_w, int H) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int m = blockIdx.x, bh = blockIdx.y;
    uint8_t* rawK = smem + ScanSmem::oRawK;
    uint8_t* rawA = m ? smem + ScanSmem::oRawA : rawK;     // for H the left factor is k itself
    uint8_t* stage = smem + ScanSmem::oStage;
    float* sb = reinterpret_cast<float*>(smem + ScanSmem::oGate);      // [4][64]
    float* sw = sb + 4 * kC;                                            // [4][64]
    float* amax = sw + 4 * kC;                                          // [4][64]
    float* kmax = amax + 4 * kC;                                        // [4][64]
    float* red = reinterpret_cast<float*>(smem + ScanSmem::oRed);
    // Chunk maxima, kept as the bit patterns of non-negative floats (which
    // order like the floats), so each warp folds its maximum in with one
    // shared-memory atomicMax; buffer cc & 1, cleared after its chunk's images
    // are written.
    int* cmax = reinterpret_cast<int*>(smem + ScanSmem::oCmax);
    uint64_t* bar_raw = reinterpret_cast<uint64_t*>(smem + ScanSmem::oBar);
    uint64_t* bar_mma = bar_raw + 2;
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + ScanSmem::oSlot);
    float* sconv = reinterpret_cast<float*>(smem + ScanSmem::oConv);
    uint8_t* halo = smem + ScanSmem::oHalo;           // [2][3 rows][256 B]

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int q4 = w & 3;
    const int row = 32 * q4 + lane;               // state row owned by this thread
    const int col0 = 32 * (w >> 2);               // its 32 columns
    const __nv_bfloat16* A = m ? v : k;
    const float* init = m ? G_in : H_in;
    float* fin = m ? G_out : H_out;
    const size_t seq = (size_t)bh * T;
    const int np = (nc + 1) >> 1;

    int prefetched = 0;                           // chunks whose row copies were issued (thread 0)
    auto prefetch = [&](int cc) {                 // rows of chunk cc -> buffer cc & 1 (thread 0)
        const int nn = min(kC, T - cc * kC);
        const uint32_t bytes = (uint32_t)nn * kD * 2;
        const int buf = cc & 1;
        mbar_arrive_expect_tx(bar_raw + buf, m ? 2 * bytes : bytes);
        bulk_g2s(rawK + buf * 16384, k + (seq + (size_t)cc * kC) * kD, bytes, bar_raw + buf);
        if (m) bulk_g2s(rawA + buf * 16384, A + (seq + (size_t)cc * kC) * kD, bytes, bar_raw + buf);
        prefetched = cc + 1;
    };
    auto wait_rows = [&](int cc) {                // every thread: chunk cc's rows have landed
        if (!mbar_wait(bar_raw + (cc & 1), (cc >> 1) & 1)) red[31] = 1.f;
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
    // build_load (stage cc-2): this thread's two 16-byte pieces of the rows of
    // a (and of k for G) into registers, the row maxima of |a| and |k| into
    // buffer cc & 3 (for the state bound) and this warp's maxima of w_j |a_j|
    // and |k_j| into cmax buffer cc & 1 (for the chunk's operand scales).
    // build_store (stage cc-1): sA, sK from cmax, then A = w_j a_j / sA (hi/lo)
    // [j][i] and B = k_j / sK [j][l] into set cc & 1, both MN-major SW128 in two
    // 64-column blocks; returns sA sK, the factor the chunk's product carries.
    // Fused input preprocessing of the keys (conv_k given): the raw piece of
    // row j of chunk cc becomes its convolved, normalised bf16 piece. The rows
    // before it come from the chunk's raw rows or, for its first three rows,
    // from the halo buffer cc & 1, which holds the previous chunk's last three
    // raw rows (zero before the sequence start); the chunk's own last three
    // raw rows go to halo buffer (cc + 1) & 1. Padding rows (j >= n) give zero.
    auto preprocess_key = [&](int cc, int n, int j, int cc16, const uint8_t* rows, uint4 raw) -> uint4 {
        uint4 x[pre::kMaxW];
        x[0] = raw;
#pragma unroll
        for (int w = 1; w < pre::kMaxW; ++w)
            x[w] = j >= w ? *reinterpret_cast<const uint4*>(rows + (j - w) * 256 + cc16 * 16)
                          : *reinterpret_cast<const uint4*>(halo + (cc & 1) * 768 + (3 + j - w) * 256 + cc16 * 16);
        if (j >= kC - 3) *reinterpret_cast<uint4*>(halo + ((cc + 1) & 1) * 768 + (j - (kC - 3)) * 256 + cc16 * 16) = raw;
        const uint4 y = pre::conv_norm_bf16x8_sw<kD, 16>(sconv, cc16 * 8, x);
        return j < n ? y : make_uint4(0, 0, 0, 0);
    };
    uint4 ra[2], rk[2];
    auto build_load = [&](int cc) {
        const int n = min(kC, T - cc * kC);
        const float* swc = sw + (cc & 3) * kC;
        const uint8_t* rpa = rawA + (cc & 1) * 16384;
        const uint8_t* rpk = rawK + (cc & 1) * 16384;
        float* am = amax + (cc & 3) * kC;
        float* km = kmax + (cc & 3) * kC;
        float wa = 0.f, wk = 0.f;
#pragma unroll
        for (int rep = 0; rep < 2; ++rep) {
            const int cid = tid + kScanThreads * rep;      // 1024 16-byte chunks of the rows
            const int j = cid >> 4, cc16 = cid & 15;
            ra[rep] = make_uint4(0, 0, 0, 0);
            if (j < n) ra[rep] = *reinterpret_cast<const uint4*>(rpa + j * 256 + cc16 * 16);
            if (conv_k && !m) ra[rep] = preprocess_key(cc, n, j, cc16, rpa, ra[rep]);
            const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&ra[rep]);
            float mx = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(a2[i]);
                mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
            // row max over the 16 threads (same half-warp) that hold row j
#pragma unroll
            for (int o2 = 8; o2 >= 1; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
            if (cc16 == 0) am[j] = mx;
            float kmx = mx;
            if (m) {   // key rows: the B operand and the key row maxima for the value-state bound
                rk[rep] = make_uint4(0, 0, 0, 0);
                if (j < n) rk[rep] = *reinterpret_cast<const uint4*>(rpk + j * 256 + cc16 * 16);
                if (conv_k) rk[rep] = preprocess_key(cc, n, j, cc16, rpk, rk[rep]);
                const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&rk[rep]);
                kmx = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __bfloat1622float2(k2[i]);
                    kmx = fmaxf(kmx, fmaxf(fabsf(f.x), fabsf(f.y)));
                }
#pragma unroll
                for (int o2 = 8; o2 >= 1; o2 >>= 1) kmx = fmaxf(kmx, __shfl_xor_sync(0xffffffffu, kmx, o2));
                if (cc16 == 0) km[j] = kmx;
            }
            wa = fmaxf(wa, swc[j] * mx);
            wk = fmaxf(wk, kmx);
        }
        wa = fmaxf(wa, __shfl_xor_sync(0xffffffffu, wa, 16));   // the warp's other row
        wk = fmaxf(wk, __shfl_xor_sync(0xffffffffu, wk, 16));
        if (lane == 0) {
            atomicMax(cmax + 2 * (cc & 1), __float_as_int(wa));
            atomicMax(cmax + 2 * (cc & 1) + 1, __float_as_int(wk));
        }
    };
    auto build_store = [&](int cc) -> float {
        const float* swc = sw + (cc & 3) * kC;
        uint8_t* Ahi = smem + ScanSmem::oImg + (cc & 1) * ScanSmem::kSet;
        uint8_t* Alo = Ahi + 16384;
        uint8_t* Bk = Ahi + 32768;
        const int2 c2 = *reinterpret_cast<const int2*>(cmax + 2 * (cc & 1));
        const float sA = pow2_ceil(__int_as_float(c2.x)), sK = pow2_ceil(__int_as_float(c2.y));
        const float inv_sA = 1.f / sA, inv_sK = 1.f / sK;       // powers of two: exact
#pragma unroll
        for (int rep = 0; rep < 2; ++rep) {
            const int cid = tid + kScanThreads * rep;
            const int j = cid >> 4, cc16 = cid & 15;
            const float wj = swc[j] * inv_sA;
            const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&ra[rep]);
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
            const uint32_t off = (uint32_t)((cc16 >> 3) * 8192 + j * 128 + (((cc16 & 7) ^ (j & 7)) << 4));
            *reinterpret_cast<uint4*>(Ahi + off) = hi;
            *reinterpret_cast<uint4*>(Alo + off) = lo;
            *reinterpret_cast<uint4*>(Bk + off) = bf16x8_to_f16x8(m ? rk[rep] : ra[rep], inv_sK);
        }
        return sA * sK;
    };
    // The state / s as fp16 into the staging image (the solve's layout);
    // returns the power-of-two scale s from the entry bound.
    auto stage_state = [&](const float (&St)[32], float bnd) {
        const float s = pow2_ceil(bnd);
        const float inv = 1.f / s;
        uint8_t* dst = stage + (col0 >> 6) * 16384 + row * 128;
        const int g0 = (col0 & 63) >> 3;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            uint4 o;
            o.x = pack_half2(St[8 * g] * inv, St[8 * g + 1] * inv);
            o.y = pack_half2(St[8 * g + 2] * inv, St[8 * g + 3] * inv);
            o.z = pack_half2(St[8 * g + 4] * inv, St[8 * g + 5] * inv);
            o.w = pack_half2(St[8 * g + 6] * inv, St[8 * g + 7] * inv);
            *reinterpret_cast<uint4*>(dst + (((g0 + g) ^ (row & 7)) << 4)) = o;
        }
        return s;
    };

    if (tid == 0) {
        mbar_init(bar_raw, 1);
        mbar_init(bar_raw + 1, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        red[31] = 0.f;
    }
    if (tid < 4) cmax[tid] = 0;
    if (conv_k) {                                  // fused preprocessing: weights, zero rows before t = 0
        pre::stage_weights<kD>(conv_k + (size_t)(bh % H) * conv_w * kD, conv_w, sconv);
        for (int e = tid; e < 768 / 16; e += kScanThreads) reinterpret_cast<uint4*>(halo)[e] = make_uint4(0, 0, 0, 0);
    }
    if (w == 0) tmem_alloc(slot, 128);
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
        // max |S_in| over the matrix: each thread's own 32 entries, then the CTA
        float mx = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) mx = fmaxf(mx, fabsf(S[i]));
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) red[w] = mx;
        __syncthreads();
        bound = red[0];
#pragma unroll
        for (int i = 1; i < kScanThreads / 32; ++i) bound = fmaxf(bound, red[i]);
    }
    if (w == 1) {                                  // gates of chunks 0..2, gamma and beta of chunk 3
        for (int cc = 0; cc < 3 && cc < nc; ++cc) {
            load_gates(cc);
            chunk_gates(cc);
        }
        if (nc > 3) load_gates(3);
    }
    __syncthreads();                              // gates visible (and the bound's partials read)
    bool ok = red[31] == 0.f;

    constexpr uint32_t kIdesc = idesc_f16(128, 128, true, true);
    auto issue_mma = [&](int cc) {                // thread 0: the chunk's 8 K steps (hi, then lo) into TMEM
        const uint8_t* Ahi = smem + ScanSmem::oImg + (cc & 1) * ScanSmem::kSet;
        const uint64_t dAhi = sdesc(smem_addr(Ahi), 8192, 1024), dAlo = sdesc(smem_addr(Ahi + 16384), 8192, 1024);
        const uint64_t dB = sdesc(smem_addr(Ahi + 32768), 8192, 1024);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t ko = ((ks & 3) * 2048) >> 4;
            mma_f16(tbase, (ks < 4 ? dAhi : dAlo) + ko, dB + ko, kIdesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar_mma);
    };
    int mma_issued = 0, mma_seen = 0;             // thread 0
    float ds_cur = 1.f, ds_next = 1.f;            // sA sK of the chunk in the MMA, of the next chunk
    if (ok && nc > 0) {
        // the state before chunk 0 (block 0's image), chunk 0's operands, chunk 1's rows
        wait_rows(0);
        build_load(0);
        __syncthreads();                          // chunk 0's maxima
        ds_cur = build_store(0);
        const float s0 = stage_state(S, bound);
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid < 2) cmax[tid] = 0;               // buffer 0 is free for chunk 2
        if (tid == 0) {
            const size_t ci = image_index(bh, np, 0, m);
            bulk_s2g(img + ci * kImgHalves, stage, kImgBytes);
            bulk_commit();
            scales[ci] = s0;
            if (red[31] == 0.f) {
                issue_mma(0);
                ++mma_issued;
            }
            if (nc > 2) prefetch(2);              // raw buffer 0 is consumed
        }
        if (nc > 1) {
            wait_rows(1);
            build_load(1);
        }
        __syncthreads();                          // chunk 1's maxima; raw buffer 1 consumed
        if (tid == 0 && nc > 3) prefetch(3);
        ok = red[31] == 0.f;
    }
    int c = 0;
    for (; ok && c < nc; ++c) {
        // ---- under MMA(c): chunk c+1's images, chunk c+2's rows and maxima,
        //      chunk c+3's gates, the bound after chunk c ----
        if (c + 1 < nc) ds_next = build_store(c + 1);
        if (c + 2 < nc) {
            wait_rows(c + 2);
            build_load(c + 2);
        }
        if (w == 1 && c + 3 < nc) {
            chunk_gates(c + 3);
            if (c + 4 < nc) load_gates(c + 4);
        }
        const float blast = sb[(c & 3) * kC + kC - 1];
        {
            // every warp reduces the same 64 terms in the same order, so every
            // thread gets the same value
            const float* swc = sw + (c & 3) * kC;
            const float* am = amax + (c & 3) * kC;
            const float* km = (m ? kmax : amax) + (c & 3) * kC;
            float add = swc[lane] * (am[lane] * km[lane]) + swc[lane + 32] * (am[lane + 32] * km[lane + 32]);
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) add += __shfl_xor_sync(0xffffffffu, add, off);
            bound = fmaf(expf(blast), bound, add);
        }
        const bool emit = c + 1 < nc && ((c + 1) & 1) == 0;
        if (tid == 0) {
            if (mbar_wait(bar_mma, c & 1)) mma_seen = mma_issued;
            else red[31] = 1.f;
            if (emit) bulk_wait_read_all();       // the staging buffer is free again
        }
        __syncthreads();                          // MMA(c) done; images of c+1, maxima of c+2, gates of c+3 written
        tc_fence_after();
        if (red[31] != 0.f) {
            ok = false;
            break;
        }
        // ---- S <- e^{b_last} S + sA sK Delta ----
        if (tid < 2) cmax[2 * ((c + 1) & 1) + tid] = 0;     // chunk c+1's images are written: free for c+3
        const float Gam = expf(blast);
        {
            float dv[32];
            tmem_ld32_x32(tbase + ((uint32_t)(32 * q4) << 16) + col0, dv);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) S[i] = fmaf(Gam, S[i], ds_cur * dv[i]);
        }
        if (c + 1 == nc) {                        // the final state
            if (fin) {
                float4* d4 = reinterpret_cast<float4*>(fin + ((size_t)bh * kD + row) * kD + col0);
#pragma unroll
                for (int i = 0; i < 8; ++i) d4[i] = make_float4(S[4 * i], S[4 * i + 1], S[4 * i + 2], S[4 * i + 3]);
            }
            break;
        }
        float s_img = 0.f;
        if (emit) s_img = stage_state(S, bound);  // the state before chunk c+1 starts block (c+1)/2
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();                          // TMEM read; staging image and chunk c+1's images written
        tc_fence_after();
        if (tid == 0) {
            if (emit) {
                const size_t ci = image_index(bh, np, (c + 1) >> 1, m);
                bulk_s2g(img + ci * kImgHalves, stage, kImgBytes);
                bulk_commit();
                scales[ci] = s_img;
            }
            issue_mma(c + 1);
            ++mma_issued;
            if (c + 4 < nc) prefetch(c + 4);      // raw buffer c & 1 is consumed (chunk c+2's rows)
        }
        ds_cur = ds_next;
    }
    if (nc == 0 && fin) {                         // no tokens: the final state is the initial one
        float4* d4 = reinterpret_cast<float4*>(fin + ((size_t)bh * kD + row) * kD + col0);
#pragma unroll
        for (int i = 0; i < 8; ++i) d4[i] = make_float4(S[4 * i], S[4 * i + 1], S[4 * i + 2], S[4 * i + 3]);
    }
    if (tid == 0) {
        if (!ok) {
            record_error(err, kErrTimeout);
            // one more bounded chance for the MMA and the row copies in flight to drain
            if (mma_issued > mma_seen) mbar_wait(bar_mma, (mma_issued - 1) & 1);
            for (int cc = 0; cc < prefetched; ++cc) mbar_wait(bar_raw + (cc & 1), (cc >> 1) & 1);
        }
        bulk_wait_all();                          // the image stores have landed before the CTA leaves
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tbase, 128);
}

}  // namespace

cudaError_t tc_scan_launch(const ForwardArgs& a, void* img, float* scales, unsigned* err, cudaStream_t st) {
    const int nc = (a.T + kC - 1) / kC;
    const int smem = ScanSmem::bytes + 1024;
    const cudaError_t e = cudaFuncSetAttribute(tc_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    LaunchTimer timer(kKindTcScan, st);
    tc_scan_kernel<<<dim3(2, a.B * a.H), kScanThreads, smem, st>>>(
        static_cast<const __nv_bfloat16*>(a.k), static_cast<const __nv_bfloat16*>(a.v), a.gamma, a.beta, a.T, nc,
        a.H_in, a.G_in, static_cast<__half*>(img), scales, a.H_out, a.G_out, err, a.conv_k, a.conv_w, a.H);
    return cudaGetLastError();
}

}  // namespace mesa
