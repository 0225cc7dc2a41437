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
// 8x finer rounding), accumulation is fp32. Each fp16 image is divided by a
// power of two chosen from a bound on its entries, so that it lies in
// [-1, 1] (or, for the score images, within a small fixed multiple of 1)
// whatever the magnitudes of beta, Lambda, k or v; every scale is undone
// exactly in the fp32 epilogue:
//   * keys: K / sK, sK >= max |k| over the block; values: V / sV likewise;
//   * the decay mask: M sK^2 / sW with sW >= max_j beta_j sK^2 >= max M sK^2;
//   * the chunk-start states: fp16 images H / sH, G / sG with sH, sG >= a
//     bound on the state's entries (tc_scan.cu);
//   * the CG direction of each token is scaled by ~1/|r| before rounding, and
//     the solution by 1/|x| for the read-out; every CG vector (x, r, p) and
//     scalar stays fp32;
//   * the scan splits beta_j e^{b_last-b_j} k_j into an fp16 hi/lo pair, so
//     the fp32 running states carry ~22-bit products (tc_scan.cu).
//
// Kernels (the scan that produces the chunk-start state images is in
// tc_scan.cu):
//   tc_cg_kernel    grid (ceil(T/128), B*H), one CTA per SM: one CTA runs every
//                   CG iteration of a 128-token block and the read-out. Tokens
//                   are the MMA M dimension (M = 128, lane = token); x and r
//                   live in TMEM, p in registers (thread: one token, 32
//                   columns); every dot product is a thread-local sum plus one
//                   shared-memory exchange across the four column quarters.
#include "mesa_internal.h"
#include "preproc_row.cuh"
#include "tc_layout.cuh"

namespace mesa {
namespace {

#ifdef MESA_DEBUG
// Debug builds only: when set, the solve kernel leaves out the completion
// signal of its first Z product, so every thread's bounded wait on it runs
// out, the kernel records a timeout in the error word and returns.
__device__ int g_debug_skip_commit = 0;
int g_debug_skip_launches = 0;
#endif

using namespace tc;

// Every thread waits on the MMA barrier itself (no CTA barrier); a thread
// whose bounded wait gave up raises the abort flag, which the next CTA
// barrier makes visible to all.
__device__ __forceinline__ void wait_mma_each(uint64_t* bar, uint32_t parity, float* abort_flag) {
    if (!mbar_wait(bar, parity)) *abort_flag = 1.f;
    tc_fence_after();
}

// =====================================================================
// Fused CG iterations + read-out, 128 tokens per CTA
// =====================================================================
// CTA blk takes tokens t0 .. t0+127 of one sequence (t0 = 128 blk, i.e. the
// even chunk c = 2 blk and the chunk after it) and the state H_c before them.
// With b_t the log-cumsum of gamma from t0 over all 128 tokens and
// M_tj = beta_j e^{b_t-b_j} (t0 <= j <= t),
//     H_t = e^{b_t} H_c + sum_j M_tj k_j k_j^T
// for every token of the block. This is the chunkwise form of two 64-token
// chunks with the second chunk's state H_{c+1} expanded into its definition,
// so one chunk-start state serves 128 tokens and every product has M = N = 128:
//   S = P K^T,  W = M o S (lower triangular),  U = P H_c^T,  Z = W K,
//   y_t = s_t (sH e^{b_t} U_t + sW Z_t) + lambda p_t
// with P the direction images p_t / s_t, K = k / sK and M the mask image
// M_tj sK^2 / sW.
// Thread layout: 16 warps; warp w holds the 32 tokens of TMEM lane quadrant
// w % 4 (lane = token) and the 32 columns 32 * (w / 4) .. + 31 of each.
// TMEM columns: U [0,128), S / Z / y [128,256), x [256,384), r [384,512);
// p stays in registers.
constexpr int kBlk = 2 * kC;                      // tokens per CTA
constexpr int kBlkThreads = 512;

struct BlkSmem {
    static constexpr int oH = 0;                  // state image [128 i][128 k] (32 KB); later G
    static constexpr int oK = 32768;              // key image [128 j][128 k] (32 KB); later values
    static constexpr int oP = 65536;              // P-hat image [128 t][128 k] (32 KB); later X-hat
    static constexpr int oW = 98304;              // masked scores [128 t][128 j] (32 KB)
    static constexpr int oG = 131072;             // value-state image [128 l][128 i] (G transposed, 32 KB), fetched at start
    static constexpr int kMS = 136;               // mask row stride in halves (conflict-free 16-byte rows)
    static constexpr int oM = 163840;             // decay mask M sK^2 / sW, fp16 [128 t][128 j], stride kMS
    static constexpr int oLam = oM + kBlk * kMS * 2;   // lambda [128]
    static constexpr int oEb = oLam + 512;        // e^{b_t} [128]
    static constexpr int oB = oEb + 512;          // b_t [128]
    static constexpr int oBeta = oB + 512;        // beta_j [128]
    static constexpr int oRed = oBeta + 512;      // [4 column quarters][128 tokens] float4
    static constexpr int oMisc = oRed + 8192;     // 32 floats
    static constexpr int oBar = oMisc + 128;      // mbarriers: ld (H), s, u, z, g (G), in (rows), v (values)
    static constexpr int oSlot = oBar + 64;
    static constexpr int oConvK = oSlot + 16;     // fused preprocessing: key and query weights [4][128],
    static constexpr int oConvQ = oConvK + 2048;
    static constexpr int oHaloK = oConvQ + 2048;  // and the 3 raw key and query rows before the block
    static constexpr int oHaloQ = oHaloK + 768;
    static constexpr int oGx = oHaloQ + 768;      // adjoint: g_t . x_t per token [128]
    static constexpr int oEcol = oGx + 512;       // decay mask column factors [128]
    static constexpr int bytes = oEcol + 512;
};

// Decay mask M_tj sK^2 / sW = msc beta_j e^{b_t - b_j} for j <= t < n, zero
// elsewhere, fp16 in Mk (row stride kMS). Part 1 takes the 16-column group
// that holds each row's diagonal, from one exponential per entry, and leaves
// the column factors ecol[j] = beta_j e^{b_r - b_j} (r = the last column of
// j's group) for part 2, which fills every other group. Part 1 needs b (sbc)
// and beta in shared memory; part 2 needs ecol, so a CTA barrier separates
// the two. One item per (row, column pair) or (row, group); rows run fastest
// across a warp, so the shared loads broadcast and the stores hit distinct banks.
static_assert(kBlkThreads == 512 && kBlk == 128, "decay mask items assume 512 threads over 128 rows");

__device__ __forceinline__ void decay_mask_diag(__half* Mk, const float* sbc, const float* sbeta, float* ecol, int n,
                                                float msc, int tid) {
#pragma unroll
    for (int rep = 0; rep < 2; ++rep) {
        const int e = tid + kBlkThreads * rep;         // row tt, pair e / 128 of its diagonal group
        const int tt = e & (kBlk - 1), j = (tt & ~15) + 2 * (e >> 7);
        float m0 = 0.f, m1 = 0.f;
        if (tt < n) {
            const float bt = sbc[tt];
            if (j <= tt) m0 = sbeta[j] * __expf(bt - sbc[j]) * msc;
            if (j + 1 <= tt) m1 = sbeta[j + 1] * __expf(bt - sbc[j + 1]) * msc;
        }
        *reinterpret_cast<__half2*>(Mk + tt * BlkSmem::kMS + j) = __floats2half2_rn(m0, m1);
    }
    if (tid < kBlk) ecol[tid] = sbeta[tid] * __expf(sbc[tid | 15] - sbc[tid]);
}

// Part 2: left of the diagonal group, e^{b_t - b_j} = e^{b_t - b_r} e^{b_r - b_j}
// with j <= r < t. For 0 < gamma <= 1 both exponents are <= 0: neither factor
// overflows, and neither underflows unless their product does.
__device__ __forceinline__ void decay_mask_rest(__half* Mk, const float* sbc, const float* ecol, int n, float msc,
                                                int tid) {
#pragma unroll
    for (int rep = 0; rep < 2; ++rep) {
        const int e = tid + kBlkThreads * rep;         // row tt, 16-column group g
        const int tt = e & (kBlk - 1), g = e >> 7;
        if (g == (tt >> 4)) continue;                  // part 1's group
        uint4 h0 = make_uint4(0, 0, 0, 0), h1 = h0;
        if (tt < n && g < (tt >> 4)) {
            const float f = msc * __expf(sbc[tt] - sbc[16 * g + 15]);
            const float4* ec = reinterpret_cast<const float4*>(ecol + 16 * g);
            const float4 c0 = ec[0], c1 = ec[1], c2 = ec[2], c3 = ec[3];
            h0 = make_uint4(pack_half2(f * c0.x, f * c0.y), pack_half2(f * c0.z, f * c0.w),
                            pack_half2(f * c1.x, f * c1.y), pack_half2(f * c1.z, f * c1.w));
            h1 = make_uint4(pack_half2(f * c2.x, f * c2.y), pack_half2(f * c2.z, f * c2.w),
                            pack_half2(f * c3.x, f * c3.y), pack_half2(f * c3.z, f * c3.w));
        }
        uint4* dst = reinterpret_cast<uint4*>(Mk + tt * BlkSmem::kMS + 16 * g);
        dst[0] = h0;
        dst[1] = h1;
    }
}

// Output rows go out through a staging tile in shared memory: each thread
// holds one token's 32 columns, so direct stores would touch 32 rows per warp
// instruction. The tile's rows are padded by 16 bytes, so a warp's 32
// consecutive rows fall in distinct banks; a warp then writes whole 512-byte rows.
constexpr int kOutPitch = kD * 4 + 16;
static_assert(kBlk * kOutPitch <= BlkSmem::oG, "output staging must fit the four 32 KB images before G");

__device__ __forceinline__ void stage_out16(uint8_t* stage, int tok, int col, const float (&uv)[16],
                                            const float (&zv)[16], float cu, float cz) {
    float4* dst = reinterpret_cast<float4*>(stage + tok * kOutPitch + col * 4);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        dst[i] = make_float4(fmaf(uv[4 * i], cu, zv[4 * i] * cz), fmaf(uv[4 * i + 1], cu, zv[4 * i + 1] * cz),
                             fmaf(uv[4 * i + 2], cu, zv[4 * i + 2] * cz), fmaf(uv[4 * i + 3], cu, zv[4 * i + 3] * cz));
}

__device__ __forceinline__ void stage_copy16(uint8_t* stage, int tok, int col, const float (&v)[16]) {
    float4* dst = reinterpret_cast<float4*>(stage + tok * kOutPitch + col * 4);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

// This thread's 32 columns of TMEM columns [c0, c0 + 128) (fp32) into the
// staging tile, then, after a CTA barrier, rows 0..n-1 of the tile to dst.
// Every thread of the CTA calls it; the tile's previous readers must be done.
__device__ __forceinline__ void tmem_rows_out(uint8_t* stage, uint32_t tl, uint32_t c0, int tok, int col0,
                                              float* dst, int n, int w, int lane);

// Rows 0..n-1 of the staging tile to dst (row-major, kD floats a row); warp w
// takes rows w, w + 16, ...
__device__ __forceinline__ void write_staged_rows(const uint8_t* stage, float* dst, int n, int w, int lane) {
    for (int r = w; r < n; r += kBlkThreads / 32)
        reinterpret_cast<float4*>(dst + (size_t)r * kD)[lane] =
            *reinterpret_cast<const float4*>(stage + r * kOutPitch + 16 * lane);
}

__device__ __forceinline__ void tmem_rows_out(uint8_t* stage, uint32_t tl, uint32_t c0, int tok, int col0,
                                              float* dst, int n, int w, int lane) {
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
        float v[16];
        tmem_ld32_x16(tl + c0 + col0 + 16 * h2, v);
        tmem_wait_ld();
        stage_copy16(stage, tok, col0 + 16 * h2, v);
    }
    __syncthreads();
    write_staged_rows(stage, dst, n, w, lane);
}

// b[t], t < 128: cumulative sum of log gamma over positions 0..t of the first
// n positions, held constant past n. One warp, four positions per lane.
__device__ __forceinline__ void warp_gate_cumsum128(const float* g, int n, float* b) {
    const int lane = threadIdx.x & 31;
    float l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) l[i] = (4 * lane + i < n) ? logf(g[4 * lane + i]) : 0.f;
    const float quad = (l[0] + l[1]) + (l[2] + l[3]);
    float incl = quad;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    float acc = incl - quad;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc += l[i];
        b[4 * lane + i] = acc;
    }
}

// Sums 4 per-token partials over the 4 column quarters (one barrier).
__device__ __forceinline__ float4 quarter_sum(float4 v, float4* red, int cq, int tok) {
    red[cq * 128 + tok] = v;
    __syncthreads();
    const float4 a = red[tok], b = red[128 + tok], c = red[256 + tok], d = red[384 + tok];
    return make_float4((a.x + b.x) + (c.x + d.x), (a.y + b.y) + (c.y + d.y), (a.z + b.z) + (c.z + d.z),
                       (a.w + b.w) + (c.w + d.w));
}

// 32 consecutive columns (col0..col0+31) of one token row of a [128][128]
// fp16 K-major image (two 64-column blocks of 16 KB), each value times s.
__device__ __forceinline__ void store_row32(uint8_t* img, int tok, int col0, const float2 (&v)[16], float s) {
    uint8_t* row = img + (col0 >> 6) * 16384 + tok * 128;
    const int c8 = (col0 & 63) >> 3;
    const float2 f = make_float2(s, s);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const float2 a = __fmul2_rn(v[4 * g], f), b = __fmul2_rn(v[4 * g + 1], f);
        const float2 c = __fmul2_rn(v[4 * g + 2], f), d = __fmul2_rn(v[4 * g + 3], f);
        uint4 o;
        o.x = pack_half2(a.x, a.y);
        o.y = pack_half2(b.x, b.y);
        o.z = pack_half2(c.x, c.y);
        o.w = pack_half2(d.x, d.y);
        *reinterpret_cast<uint4*>(row + (((c8 + g) ^ (tok & 7)) << 4)) = o;
    }
}

// Eight K = 16 steps of one fp16 product into TMEM address d. A is a K-major
// SW128 image (64-element K blocks a_kb bytes apart); B is K-major (b_k16 = 32)
// or MN-major (b_lbo = MN block stride, b_k16 = 2048), its K blocks b_kb apart.
__device__ __forceinline__ void issue_k128(uint32_t d, uint32_t a, uint32_t b, uint32_t b_lbo, uint32_t a_kb,
                                        uint32_t b_kb, uint32_t b_k16, uint32_t idesc) {
    const uint64_t da = sdesc(a, 16, 1024), db = sdesc(b, b_lbo, 1024);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        const uint32_t oa = ((ks >> 2) * a_kb + (ks & 3) * 32) >> 4;
        const uint32_t ob = ((ks >> 2) * b_kb + (ks & 3) * b_k16) >> 4;
        mma_f16(d, da + oa, db + ob, idesc, ks > 0 ? 1u : 0u);
    }
}

// kAdj = false: the forward (right-hand side q, read-out o = G x).
// kAdj = true: the adjoint solve of the backward, (H_t + Lambda) u_t = g_t with
// g_t = G_t^T dout_t read from `rhs` (fp32, tc_rhs_kernel) under the same CG
// rule; writes dq_t = u_t and e_t = g_t . x_t - u_t . (H_t x_t), with x_t the
// forward's solutions (`xsol`) and H_t x_t one more product of the same kind.
// kAdj: the backward's adjoint solve (no read-out); kXout: the forward also
// stores its solutions x in x_out (a separate instantiation keeps that path's
// registers out of the plain forward).
template <bool kAdj, bool kXout>
__global__ void __launch_bounds__(kBlkThreads, 1)
tc_cg_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
             const __nv_bfloat16* __restrict__ v, const float* __restrict__ gamma,
             const float* __restrict__ beta, const float* __restrict__ lambda, int H, int T, int np,
             int cg_steps, float tol, const __half* __restrict__ img, const float* __restrict__ scales,
             float* __restrict__ out, int32_t* __restrict__ iters, unsigned* __restrict__ err,
             float* __restrict__ x_out, const float* __restrict__ x0, const float* __restrict__ conv_q,
             const float* __restrict__ conv_k, int conv_w, const float* __restrict__ rhs,
             const float* __restrict__ xsol, float* __restrict__ dq, float* __restrict__ zt) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* Hs = smem + BlkSmem::oH;
    uint8_t* Ks = smem + BlkSmem::oK;
    uint8_t* Ps = smem + BlkSmem::oP;
    uint8_t* Ws = smem + BlkSmem::oW;
    uint8_t* Gs = smem + BlkSmem::oG;
    __half* Mk = reinterpret_cast<__half*>(smem + BlkSmem::oM);
    float* slam = reinterpret_cast<float*>(smem + BlkSmem::oLam);
    float* seb = reinterpret_cast<float*>(smem + BlkSmem::oEb);
    float* sbc = reinterpret_cast<float*>(smem + BlkSmem::oB);
    float* sbeta = reinterpret_cast<float*>(smem + BlkSmem::oBeta);
    float* ecol = reinterpret_cast<float*>(smem + BlkSmem::oEcol);
    float4* red = reinterpret_cast<float4*>(smem + BlkSmem::oRed);
    float* misc = reinterpret_cast<float*>(smem + BlkSmem::oMisc);
    float* abort_flag = misc + 31;
    uint64_t* bar_ld = reinterpret_cast<uint64_t*>(smem + BlkSmem::oBar);
    uint64_t* bar_s = bar_ld + 1;
    uint64_t* bar_u = bar_ld + 2;
    uint64_t* bar_z = bar_ld + 3;
    uint64_t* bar_g = bar_ld + 4;
    uint64_t* bar_in = bar_ld + 5;
    uint64_t* bar_v = bar_ld + 6;
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + BlkSmem::oSlot);
    float* sconvK = reinterpret_cast<float*>(smem + BlkSmem::oConvK);
    float* sconvQ = reinterpret_cast<float*>(smem + BlkSmem::oConvQ);
    uint8_t* haloK = smem + BlkSmem::oHaloK;
    uint8_t* haloQ = smem + BlkSmem::oHaloQ;

    const int blk = blockIdx.x, bh = blockIdx.y, head = bh % H;
    const int t0 = blk * kBlk;
    const int n = min(kBlk, T - t0);
    const size_t base = (size_t)bh * T + t0;       // token tok of the CTA is base + tok
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int q4 = w & 3, cq = w >> 2;
    const int tok = 32 * q4 + lane;                  // 0..127 = TMEM lane
    const bool valid = tok < n;
    // The MMA-issuing thread: tcgen05.mma stalls its thread while the tensor
    // pipe is full, so the issuer is the first thread of warp 8 (tokens 0..31,
    // columns 64..95), whose block of masked scores lies above the diagonal and
    // is never computed: it issues S and U while the other warps mask scores.
    constexpr int kIssuer = 256;
    const int col0 = 32 * cq;                         // this thread's 32 columns
    const size_t iH = image_index(bh, np, blk, 0), iG = image_index(bh, np, blk, 1);   // state images of the block

    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_u, 1);
        mbar_init(bar_z, 1);
        mbar_init(bar_g, 1);
        mbar_init(bar_in, 1);
        mbar_init(bar_v, 1);
        fence_mbar_init();
        *abort_flag = 0.f;
    }
    if (w == 0) tmem_alloc(slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *slot;
    const uint32_t tl = tbase + ((uint32_t)(32 * q4) << 16);     // this warp's lane quadrant
    constexpr uint32_t kColU = 0, kColS = 128, kColX = 256, kColR = 384;

    // Bulk copies: first what the set-up reads (the raw key rows staged in the
    // P-hat buffer, the raw query rows staged in the score buffer and, for a
    // full aligned block, gamma and beta staged in the reduction buffer); the
    // two state images follow once those have landed, so that they do not
    // share the memory bandwidth with them (H is first read by the first MMA,
    // G by the read-out).
    const uint32_t row_bytes = (uint32_t)n * kD * 2;
    const bool gates_bulk = n == kBlk && ((reinterpret_cast<uintptr_t>(gamma + base) |
                                            reinterpret_cast<uintptr_t>(beta + base)) & 15) == 0;
    float* gstage = reinterpret_cast<float*>(red);
    // Fused input preprocessing (conv_k given): q and k arrive raw, with the
    // three rows before the block, and are convolved and normalised here.
    const bool fuse = conv_k != nullptr;
    const bool halo_rows = fuse && t0 >= pre::kMaxW - 1;
    // The adjoint has no query rows and no read-out: its right-hand sides g_t
    // and the forward solutions x_t (fp32 rows) are staged instead, g in the
    // score and G buffers (64 KB, both free until the first masked scores)
    // and x in the H and key buffers (the H image follows once x is read).
    // A warm-started forward (the instantiation that stores its solutions)
    // stages its x0 rows (fp32) in the H and key buffers the same way.
    const uint32_t frow_bytes = (uint32_t)n * kD * 4;
    const bool x0_staged = kXout && !kAdj && x0 != nullptr;
    if (tid == 0) {
        mbar_arrive_expect_tx(bar_in, (kAdj ? row_bytes + 2u * frow_bytes : 2u * row_bytes + (x0_staged ? frow_bytes : 0u)) +
                                          (gates_bulk ? 2u * kBlk * 4u : 0u) + (halo_rows ? 2u * 768u : 0u));
        bulk_g2s(Ps, k + base * kD, row_bytes, bar_in);
        if (!kAdj) {
            bulk_g2s(Ws, q + base * kD, row_bytes, bar_in);
            if (x0_staged) bulk_g2s(Hs, x0 + base * kD, frow_bytes, bar_in);
        } else {
            bulk_g2s(Ws, rhs + base * kD, frow_bytes, bar_in);
            bulk_g2s(Hs, xsol + base * kD, frow_bytes, bar_in);
        }
        if (gates_bulk) {
            bulk_g2s(gstage, gamma + base, kBlk * 4, bar_in);
            bulk_g2s(gstage + kBlk, beta + base, kBlk * 4, bar_in);
        }
        if (halo_rows) {
            bulk_g2s(haloK, k + (base - 3) * kD, 768, bar_in);
            bulk_g2s(haloQ, q + (base - 3) * kD, 768, bar_in);
        }
    }
    if (fuse) {
        pre::stage_weights<kD>(conv_k + (size_t)head * conv_w * kD, conv_w, sconvK);
        pre::stage_weights<kD>(conv_q + (size_t)head * conv_w * kD, conv_w, sconvQ);
        if (!halo_rows)                                // rows before the sequence start are zero
            for (int e = tid; e < 2 * 768 / 16; e += kBlkThreads) reinterpret_cast<uint4*>(haloK)[e] = make_uint4(0, 0, 0, 0);
    }
    const float sH = scales[iH];
    if (tid >= kBlk && tid < kBlk + kD) slam[tid - kBlk] = lambda[(size_t)head * kD + tid - kBlk];
    if (tid == 0) {
        if (!mbar_wait(bar_in, 0)) *abort_flag = 1.f;
        if (!kAdj && !x0_staged) {                     // (else the H image follows the staged fp32 rows)
            mbar_arrive_expect_tx(bar_ld, kImgBytes);
            bulk_g2s(Hs, img + iH * kImgHalves, kImgBytes, bar_ld);
        }
        if (!kAdj) {                                   // the adjoint has no read-out
            mbar_arrive_expect_tx(bar_g, kImgBytes);
            bulk_g2s(Gs, img + iG * kImgHalves, kImgBytes, bar_g);
        }
    }
    __syncthreads();

    // gates and beta; the raw key rows (held in registers until the key image
    // is written) and the block's maxima of |k| and beta, per warp into misc
    if (w == 0) warp_gate_cumsum128(gates_bulk ? gstage : gamma + base, n, sbc);
    float bmax = 0.f, kmax = 0.f;
    if (tid < kBlk) {
        bmax = (tid < n) ? (gates_bulk ? gstage[kBlk + tid] : beta[base + tid]) : 0.f;
        sbeta[tid] = bmax;
    }
    // a raw piece (row j, channels 8 cc..) of staged rows -> its preprocessed piece
    auto preprocess_piece = [&](const uint8_t* rows, const uint8_t* halo, const float* sw, int j, int cc,
                                uint4 raw) -> uint4 {
        uint4 x[pre::kMaxW];
        x[0] = raw;
#pragma unroll
        for (int wl = 1; wl < pre::kMaxW; ++wl)
            x[wl] = j >= wl ? *reinterpret_cast<const uint4*>(rows + (j - wl) * 256 + cc * 16)
                            : *reinterpret_cast<const uint4*>(halo + (3 + j - wl) * 256 + cc * 16);
        const uint4 y = pre::conv_norm_bf16x8_sw<kD, 16>(sw, cc * 8, x);
        return j < n ? y : make_uint4(0, 0, 0, 0);
    };
    uint4 kraw[4];
#pragma unroll
    for (int rep = 0; rep < 4; ++rep) {
        const int cid = tid + kBlkThreads * rep;       // 2048 16-byte chunks
        const int j = cid >> 4, cc = cid & 15;
        kraw[rep] = make_uint4(0, 0, 0, 0);
        if (j < n) kraw[rep] = *reinterpret_cast<const uint4*>(Ps + j * 256 + cc * 16);
        if (fuse) kraw[rep] = preprocess_piece(Ps, haloK, sconvK, j, cc, kraw[rep]);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&kraw[rep]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(b2[i]);
            kmax = fmaxf(kmax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        kmax = fmaxf(kmax, __shfl_xor_sync(0xffffffffu, kmax, off));
        bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, off));
    }
    if (lane == 0) {
        misc[w] = kmax;
        if (w < 4) misc[16 + w] = bmax;
    }
    if (fuse) {                                        // queries preprocessed in place in their staging buffer
        uint4 qp[4];
#pragma unroll
        for (int rep = 0; rep < 4; ++rep) {
            const int cid = tid + kBlkThreads * rep;
            const int j = cid >> 4, cc = cid & 15;
            uint4 raw = make_uint4(0, 0, 0, 0);
            if (j < n) raw = *reinterpret_cast<const uint4*>(Ws + j * 256 + cc * 16);
            qp[rep] = preprocess_piece(Ws, haloQ, sconvQ, j, cc, raw);
        }
        __syncthreads();                               // every raw query row read
#pragma unroll
        for (int rep = 0; rep < 4; ++rep) {
            const int cid = tid + kBlkThreads * rep;
            *reinterpret_cast<uint4*>(Ws + (cid >> 4) * 256 + (cid & 15) * 16) = qp[rep];
        }
        __syncthreads();
    }
    // CG state: x = 0 and r = q in TMEM, p = q in registers; this thread: token tok, columns col0..col0+31
    // (the adjoint: r = p = g_t from rhs, and the partial g_t . x_t for e_t)
    float2 p[16];
    float gx = 0.f;
    if constexpr (kAdj) {
        // this token's g_t and x_t columns from the staged rows (one row per lane)
        const float4* gr = reinterpret_cast<const float4*>(Ws) + tok * (kD / 4) + col0 / 4;
        const float4* xr = reinterpret_cast<const float4*>(Hs) + tok * (kD / 4) + col0 / 4;
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            float4 f = make_float4(0.f, 0.f, 0.f, 0.f), xf = f;
            if (valid) {
                f = gr[g];
                xf = xr[g];
            }
            acc = __ffma2_rn(make_float2(f.x, f.y), make_float2(xf.x, xf.y), acc);
            acc = __ffma2_rn(make_float2(f.z, f.w), make_float2(xf.z, xf.w), acc);
            p[2 * g] = make_float2(f.x, f.y);
            p[2 * g + 1] = make_float2(f.z, f.w);
        }
        gx = acc.x + acc.y;
    } else {
        // The staged rows are 256 bytes apart, one per lane: lane l reads its
        // four 16-byte pieces starting from piece l mod 4, so that a
        // quarter-warp's eight reads fall in four bank groups, not one; the
        // pieces are then rotated back into order.
        const int rot = lane & 3;
        uint4 raw[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            raw[g] = make_uint4(0, 0, 0, 0);
            if (valid) raw[g] = *reinterpret_cast<const uint4*>(Ws + tok * 256 + col0 * 2 + 16 * ((g + rot) & 3));
        }
        uint4 t[4];                                    // piece c = raw[(c - rot) mod 4]
#pragma unroll
        for (int c = 0; c < 4; ++c) t[c] = (rot & 1) ? raw[(c + 3) & 3] : raw[c];
#pragma unroll
        for (int c = 0; c < 4; ++c) raw[c] = (rot & 2) ? t[(c + 2) & 3] : t[c];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&raw[g]);
#pragma unroll
            for (int i = 0; i < 4; ++i) p[4 * g + i] = __bfloat1622float2(b2[i]);
        }
    }
    // r = q; x = x0 (a warm start) or 0. With x0, p = x0 for the extra first
    // step that forms r = q - (H_t + Lambda) x0 (below).
    float qq = 0.f;
    {
        float2 a = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 16; ++i) a = __ffma2_rn(p[i], p[i], a);
        qq = a.x + a.y;
    }
#pragma unroll
    for (int h2 = 0; h2 < 4; ++h2) {
        float z[8], rv[8];
        float4 xa = make_float4(0.f, 0.f, 0.f, 0.f), xb = xa;
        if (x0 && valid) {                             // this token's x0 columns: staged rows, else global memory
            const float4* src = x0_staged ? reinterpret_cast<const float4*>(Hs) + tok * (kD / 4) + (col0 + 8 * h2) / 4
                                          : reinterpret_cast<const float4*>(x0 + (base + tok) * kD + col0 + 8 * h2);
            xa = src[0];
            xb = src[1];
        }
        z[0] = xa.x; z[1] = xa.y; z[2] = xa.z; z[3] = xa.w;
        z[4] = xb.x; z[5] = xb.y; z[6] = xb.z; z[7] = xb.w;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            rv[2 * i] = p[4 * h2 + i].x;
            rv[2 * i + 1] = p[4 * h2 + i].y;
            if (x0) p[4 * h2 + i] = make_float2(z[2 * i], z[2 * i + 1]);
        }
        tmem_st32_x8(tl + kColX + col0 + 8 * h2, z);
        tmem_st32_x8(tl + kColR + col0 + 8 * h2, rv);
    }
    __syncthreads();                                   // gates, beta, maxima visible; staged rows consumed
    if ((kAdj || x0_staged) && tid == 0) {             // the H image, now that the staged fp32 rows are read
        fence_proxy_async();
        mbar_arrive_expect_tx(bar_ld, kImgBytes);
        bulk_g2s(Hs, img + iH * kImgHalves, kImgBytes, bar_ld);
    }
    // key scale sK >= max |k| and mask scale sW >= max_j beta_j sK^2 (powers of two)
    float sK, sW;
    {
        float km = misc[0], bm = misc[16];
#pragma unroll
        for (int i = 1; i < 16; ++i) km = fmaxf(km, misc[i]);
#pragma unroll
        for (int i = 17; i < 20; ++i) bm = fmaxf(bm, misc[i]);
        sK = pow2_ceil(km);
        sW = pow2_ceil(bm * sK * sK);
        const float inv_sK = 1.f / sK;
#pragma unroll
        for (int rep = 0; rep < 4; ++rep) {            // key image K / sK
            const int cid = tid + kBlkThreads * rep;
            const int j = cid >> 4, cc = cid & 15;
            *reinterpret_cast<uint4*>(Ks + (cc >> 3) * 16384 + j * 128 + (((cc & 7) ^ (j & 7)) << 4)) =
                bf16x8_to_f16x8(kraw[rep], inv_sK);
        }
    }
    if (tid < kBlk) seb[tid] = expf(sbc[tid]);
#pragma unroll
    for (int rep = 0; rep < 4; ++rep) reinterpret_cast<uint4*>(Ws)[tid + kBlkThreads * rep] = make_uint4(0, 0, 0, 0);
    // M_tj sK^2 / sW (at most 1), part 1. The exponents are <= 0; the fast
    // exponential's few-ulp error is far below the fp16 rounding that follows.
    const float msc = sK * sK / sW;                    // powers of two: exact
    decay_mask_diag(Mk, sbc, sbeta, ecol, n, msc, tid);
    float rr, pp;
    {
        float2 a = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 16; ++i) a = __ffma2_rn(p[i], p[i], a);
        const float4 d = quarter_sum(make_float4(qq, a.x + a.y, gx, 0.f), red, cq, tok);   // barrier publishes seb, Mk
        rr = d.x;                                      // |q|^2 = |r|^2
        pp = d.y;                                      // |p|^2 (|x0|^2 for a warm start)
        if (kAdj && cq == 0) reinterpret_cast<float*>(smem + BlkSmem::oGx)[tok] = d.z;   // adjoint: g_t . x_t
    }
    decay_mask_rest(Mk, sbc, ecol, n, msc, tid);       // published by the first step's barrier
    tmem_wait_st();
    const float qn = sqrtf(rr);
    bool act = valid;
    int it = 0;
    const float eb = seb[tok];
    float s = pow2_sqrt_scale(pp), is = 1.f / s;
    store_row32(Ps, tok, col0, p, is);

    constexpr uint32_t kIdKK = idesc_f16(128, 128, false, false);     // A and B K-major
    constexpr uint32_t kIdKM = idesc_f16(128, 128, false, true);      // B MN-major
    auto issue_S = [&]() {      // S = P K^T -> columns [128, 256)
        issue_k128(tbase + kColS, smem_addr(Ps), smem_addr(Ks), 16, 16384, 16384, 32, kIdKK);
    };
    auto issue_U = [&]() {      // U = P H^T -> columns [0, 128)
        issue_k128(tbase + kColU, smem_addr(Ps), smem_addr(Hs), 16, 16384, 16384, 32, kIdKK);
    };
    auto issue_Z = [&]() {      // Z = W K -> columns [128, 256)
        issue_k128(tbase + kColS, smem_addr(Ws), smem_addr(Ks), 16384, 16384, 8192, 2048, kIdKM);
    };
    // S (TMEM) -> decay-masked scores -> score image. The quarter of
    // tokens 0..63 against keys 64..127 lies above the diagonal: it stays zero.
    auto masked_scores = [&]() {
        if (q4 < 2 && cq >= 2) return;                 // warp-uniform
        const __half* mrow = Mk + tok * BlkSmem::kMS + col0;
        float2 wv[16];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            float sv[16];
            tmem_ld32_x16(tl + kColS + col0 + 16 * h2, sv);
            tmem_wait_ld();
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                const uint4 m8 = *reinterpret_cast<const uint4*>(mrow + 16 * h2 + 8 * g);
                const __half2* m2 = reinterpret_cast<const __half2*>(&m8);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int c = 4 * g + i;
                    wv[8 * h2 + c] = __fmul2_rn(__half22float2(m2[i]), make_float2(sv[2 * c], sv[2 * c + 1]));
                }
            }
        }
        store_row32(Ws, tok, col0, wv, 1.f);
    };

    if (tid == 0 && !mbar_wait(bar_ld, 0)) *abort_flag = 1.f;
    uint32_t ph = 0;
    auto fetch_values = [&]() {                        // raw value rows into the dead H buffer
        mbar_arrive_expect_tx(bar_v, row_bytes);
        bulk_g2s(Hs, v + base * kD, row_bytes, bar_v);
    };
    auto fetch_xsol = [&]() {                          // adjoint: the x_t rows (fp32) into the score and G buffers
        mbar_arrive_expect_tx(bar_v, frow_bytes);
        bulk_g2s(Ws, xsol + base * kD, frow_bytes, bar_v);
    };
    const int first_step = x0 ? -1 : 0;
    int step = first_step;
    // step -1 (warm start only): the matvec of x0; its update leaves x = x0 and
    // turns r = q into r_0 = q - (H_t + Lambda) x0, with p_0 = r_0
    for (; step < cg_steps; ++step) {
        if (step >= 0) act = act && cg_may_continue(rr, qn, tol);
        fence_proxy_async();
        tc_fence_before();
        const int any = __syncthreads_or(act ? 1 : 0);
        tc_fence_after();
        if (!any || *abort_flag != 0.f) break;
        if (tid == kIssuer) {
            issue_S();
            mma_commit(bar_s);
            issue_U();
            mma_commit(bar_u);
        }
        wait_mma_each(bar_s, ph & 1, abort_flag);
        masked_scores();
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (*abort_flag != 0.f) break;
        if (tid == kIssuer) {
            issue_Z();
#ifdef MESA_DEBUG
            if (!(step == 0 && g_debug_skip_commit))   // fault injection: nothing signals Z of step 0
#endif
            mma_commit(bar_z);
        }
        wait_mma_each(bar_u, ph & 1, abort_flag);
        wait_mma_each(bar_z, ph & 1, abort_flag);
        ++ph;
        // with a fixed step count the last U product is known: H is dead from
        // here, and the read-out's value rows can be on their way during this
        // step's CUDA-core work
        if (!kAdj && tid == 0 && tol <= 0.f && step == cg_steps - 1) fetch_values();
        // the adjoint's tail re-reads x_t: with a fixed step count its rows can
        // be on their way into the score and G buffers (dead from here)
        if (kAdj && tid == 0 && tol <= 0.f && step == cg_steps - 1) fetch_xsol();

        // y = s (sH e^b U + sW Z) + lambda p (written over Z); partials p.y, r.y, y.y, r.r
        const float c_u = s * sH * eb, c_z = s * sW;
        float4 d;
        {
            float2 a = make_float2(0.f, 0.f), b = a, cc = a, e = a;
#pragma unroll
            for (int h2 = 0; h2 < 4; ++h2) {
                float uv[8], zv[8], rv[8];
                tmem_ld32_x8(tl + kColU + col0 + 8 * h2, uv);
                tmem_ld32_x8(tl + kColS + col0 + 8 * h2, zv);
                tmem_ld32_x8(tl + kColR + col0 + 8 * h2, rv);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int pi = 4 * h2 + i;
                    const float2 lm = *reinterpret_cast<const float2*>(slam + col0 + 2 * pi);
                    const float2 rp = make_float2(rv[2 * i], rv[2 * i + 1]);
                    float2 y = __ffma2_rn(make_float2(uv[2 * i], uv[2 * i + 1]), make_float2(c_u, c_u),
                                          __fmul2_rn(lm, p[pi]));
                    y = __ffma2_rn(make_float2(zv[2 * i], zv[2 * i + 1]), make_float2(c_z, c_z), y);
                    a = __ffma2_rn(p[pi], y, a);
                    b = __ffma2_rn(rp, y, b);
                    cc = __ffma2_rn(y, y, cc);
                    e = __ffma2_rn(rp, rp, e);
                    zv[2 * i] = y.x;
                    zv[2 * i + 1] = y.y;
                }
                tmem_st32_x8(tl + kColS + col0 + 8 * h2, zv);
            }
            d = make_float4(a.x + a.y, b.x + b.y, cc.x + cc.y, e.x + e.y);
        }
        tmem_wait_st();
        d = quarter_sum(d, red, cq, tok);
        const bool warm = step < 0;
        if (act && !warm && !cg_curvature_ok(d.x)) act = false;
        if (act) rr = d.w;                             // true |r|^2 of the current residual
        // alpha and rho feed recurrences that CG corrects: the fast division suffices
        const float al = act ? (warm ? 1.f : __fdividef(rr, d.x)) : 0.f;
        const float rn = fmaxf(fmaf(al, fmaf(al, d.z, -2.f * d.y), rr), 0.f);
        const float rho = (act && !warm) ? __fdividef(rn, rr) : 0.f;
        const float ax = warm ? 0.f : al;              // the warm step keeps x = x0
        const float2 pa = make_float2(ax, ax), na = make_float2(-al, -al), rh = make_float2(rho, rho);
        // the next direction's image is written round by round (its scale is known here)
        const float s_new = act ? pow2_sqrt_scale(rn) : s;
        const float is_new = 1.f / s_new;
        uint8_t* prow = Ps + (col0 >> 6) * 16384 + tok * 128;
#pragma unroll
        for (int h2 = 0; h2 < 4; ++h2) {               // x += alpha p; r -= alpha y; p = r + rho p
            float xv[8], yv[8], rv[8];
            tmem_ld32_x8(tl + kColX + col0 + 8 * h2, xv);
            tmem_ld32_x8(tl + kColS + col0 + 8 * h2, yv);
            tmem_ld32_x8(tl + kColR + col0 + 8 * h2, rv);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int pi = 4 * h2 + i;
                const float2 x = __ffma2_rn(pa, p[pi], make_float2(xv[2 * i], xv[2 * i + 1]));
                xv[2 * i] = x.x;
                xv[2 * i + 1] = x.y;
                if (act) {
                    const float2 r = __ffma2_rn(na, make_float2(yv[2 * i], yv[2 * i + 1]),
                                                make_float2(rv[2 * i], rv[2 * i + 1]));
                    p[pi] = __ffma2_rn(rh, p[pi], r);
                    rv[2 * i] = r.x;
                    rv[2 * i + 1] = r.y;
                }
            }
            tmem_st32_x8(tl + kColX + col0 + 8 * h2, xv);
            tmem_st32_x8(tl + kColR + col0 + 8 * h2, rv);
            {
                const float2 f = make_float2(is_new, is_new);
                const float2 a0 = __fmul2_rn(p[4 * h2], f), a1 = __fmul2_rn(p[4 * h2 + 1], f);
                const float2 a2 = __fmul2_rn(p[4 * h2 + 2], f), a3 = __fmul2_rn(p[4 * h2 + 3], f);
                *reinterpret_cast<uint4*>(prow + (((((col0 & 63) >> 3) + h2) ^ (tok & 7)) << 4)) =
                    make_uint4(pack_half2(a0.x, a0.y), pack_half2(a1.x, a1.y), pack_half2(a2.x, a2.y),
                               pack_half2(a3.x, a3.y));
            }
        }
        if (act) {
            rr = rn;
            if (!warm) ++it;
        }
        s = s_new;
        is = is_new;
        tmem_wait_st();
    }

    if constexpr (kAdj) {
        // ---- adjoint tail: dq = u, then H_t x_t by one more product with
        // X-hat = x / s_x, and e_t = g_t . x_t - u_t . (H_t x_t) ----
        // the x_t rows: sent during the last fixed step, else now (the
        // masked scores are dead once the loop has ended)
        const bool x_sent = tol <= 0.f && step == cg_steps && cg_steps > first_step;
        if (tid == 0 && !x_sent) fetch_xsol();
        if (tid == 0 && !mbar_wait(bar_v, 0)) *abort_flag = 1.f;
        __syncthreads();                               // x rows landed; last reduction's readers are done with red[]
        float ux_part = 0.f;
        {
            float2 xr[16];
            const float4* xrow = reinterpret_cast<const float4*>(Ws) + tok * (kD / 4) + col0 / 4;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
                if (valid) f = xrow[g];
                xr[2 * g] = make_float2(f.x, f.y);
                xr[2 * g + 1] = make_float2(f.z, f.w);
            }
            float2 a = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 16; ++i) a = __ffma2_rn(xr[i], xr[i], a);
            ux_part = a.x + a.y;
            const float xx = quarter_sum(make_float4(ux_part, 0.f, 0.f, 0.f), red, cq, tok).x;   // every x row read
            s = pow2_sqrt_scale(xx);
            store_row32(Ps, tok, col0, xr, 1.f / s);
            // the staged rows overwrote the score image's quarter above the
            // diagonal (tokens 0..63, keys 64..127), which the masked scores
            // never rewrite: zero it again (8 KB, one 16-byte piece a thread)
            reinterpret_cast<uint4*>(Ws + 16384)[tid] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        bool ok = *abort_flag == 0.f;
        if (ok) {
            if (tid == kIssuer) {
                issue_S();
                mma_commit(bar_s);
                issue_U();
                mma_commit(bar_u);
            }
            wait_mma_each(bar_s, ph & 1, abort_flag);
            masked_scores();
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            ok = *abort_flag == 0.f;
        }
        if (ok) {
            if (tid == kIssuer) {
                issue_Z();
                mma_commit(bar_z);
            }
            wait_mma_each(bar_u, ph & 1, abort_flag);
            wait_mma_each(bar_z, ph & 1, abort_flag);
            ++ph;
            // H_t x_t = s_x (sH e^b U + sW Z) (no Lambda term); the partial u . (H_t x_t)
            const float c_u = s * sH * eb, c_z = s * sW;
            float2 a = make_float2(0.f, 0.f);
#pragma unroll
            for (int h2 = 0; h2 < 4; ++h2) {
                float uv[8], zv[8], xv[8];
                tmem_ld32_x8(tl + kColU + col0 + 8 * h2, uv);
                tmem_ld32_x8(tl + kColS + col0 + 8 * h2, zv);
                tmem_ld32_x8(tl + kColX + col0 + 8 * h2, xv);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float2 hx = __fmul2_rn(make_float2(uv[2 * i], uv[2 * i + 1]), make_float2(c_u, c_u));
                    hx = __ffma2_rn(make_float2(zv[2 * i], zv[2 * i + 1]), make_float2(c_z, c_z), hx);
                    a = __ffma2_rn(make_float2(xv[2 * i], xv[2 * i + 1]), hx, a);
                }
            }
            const float uhx = quarter_sum(make_float4(a.x + a.y, 0.f, 0.f, 0.f), red, cq, tok).x;
            if (cq == 0 && valid) zt[base + tok] = reinterpret_cast<const float*>(smem + BlkSmem::oGx)[tok] - uhx;
            if (iters && cq == 0 && valid) iters[base + tok] = it;
            // dq = u, still in the x columns of TMEM, through the staging tile (every image is dead)
            tmem_rows_out(smem, tl, kColX, tok, col0, dq + base * kD, n, w, lane);
            ok = *abort_flag == 0.f;
        }
        if (!ok && tid == kIssuer) {
            record_error(err, kErrTimeout);
            // one more bounded chance for every MMA issued so far to drain
            mma_commit(bar_ld);
            mbar_wait(bar_ld, 0);
            mbar_wait(bar_ld, 1);
        }
    } else {
        // ---- read-out: o = e^{b_t} G_c x + (M o X K^T) V, on the same MMA pattern,
        // with X-hat = x / |x|, V / sV (sV >= max |v|) and the same key and mask images ----
        // unless the last fixed step already sent them (the loop ran to its end)
        const bool v_sent = tol <= 0.f && step == cg_steps && cg_steps > first_step;
        if (tid == 0 && !v_sent) fetch_values();          // while x is normalised
        __syncthreads();                                   // last reduction's readers are done with red[]
        float xs;
        {
            float2 xr[16];
    #pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                float xv[16];
                tmem_ld32_x16(tl + kColX + col0 + 16 * h2, xv);
                tmem_wait_ld();
    #pragma unroll
                for (int i = 0; i < 8; ++i) xr[8 * h2 + i] = make_float2(xv[2 * i], xv[2 * i + 1]);
            }
            float2 a = make_float2(0.f, 0.f);
    #pragma unroll
            for (int i = 0; i < 16; ++i) a = __ffma2_rn(xr[i], xr[i], a);
            const float xx = quarter_sum(make_float4(a.x + a.y, 0.f, 0.f, 0.f), red, cq, tok).x;
            xs = xx > 0.f ? sqrtf(xx) : 1.f;
            store_row32(Ps, tok, col0, xr, 1.f / xs);
        }
        // values of the block (kept in registers until the key image is free) and max |v|
        if (!mbar_wait(bar_v, 0)) *abort_flag = 1.f;
        uint4 vraw[4];
        float vmax = 0.f;
    #pragma unroll
        for (int rep = 0; rep < 4; ++rep) {
            const int cid = tid + kBlkThreads * rep;
            const int j = cid >> 4, cc = cid & 15;
            vraw[rep] = make_uint4(0, 0, 0, 0);
            if (j < n) vraw[rep] = *reinterpret_cast<const uint4*>(Hs + j * 256 + cc * 16);
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
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();                                   // publishes X-hat and misc
        tc_fence_after();
        float vm = misc[0];
    #pragma unroll
        for (int i = 1; i < 16; ++i) vm = fmaxf(vm, misc[i]);
        const float sV = pow2_ceil(vm);
        const float sG = scales[iG];
        bool ok = *abort_flag == 0.f;
        if (ok) {
            if (tid == kIssuer) {
                issue_S();                         // S' = X-hat K^T
                mma_commit(bar_s);
            }
            wait_mma_each(bar_s, ph & 1, abort_flag);
            masked_scores();                       // W' = (M sK^2 / sW) o (X-hat (K / sK)^T)
            const float inv_sV = 1.f / sV;
    #pragma unroll
            for (int rep = 0; rep < 4; ++rep) {    // the key image is dead: values take its place
                const int cid = tid + kBlkThreads * rep;
                const int j = cid >> 4, cc = cid & 15;
                *reinterpret_cast<uint4*>(Ks + (cc >> 3) * 16384 + j * 128 + (((cc & 7) ^ (j & 7)) << 4)) =
                    bf16x8_to_f16x8(vraw[rep], inv_sV);
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            ok = *abort_flag == 0.f;
        }
        if (ok) {
            if (tid == kIssuer) {
                if (!mbar_wait(bar_g, 0)) {
                    *abort_flag = 1.f;
                    mma_commit(bar_u);
                    mma_commit(bar_z);
                } else {
                    // U' = X-hat G^T: the image holds G transposed (row l, column i), the
                    // right operand MN-major like the key image
                    issue_k128(tbase + kColU, smem_addr(Ps), smem_addr(Gs), 16384, 16384, 8192, 2048, kIdKM);
                    mma_commit(bar_u);
                    issue_Z();                     // Z' = W' V
                    mma_commit(bar_z);
                }
            }
            wait_mma_each(bar_u, ph & 1, abort_flag);
            wait_mma_each(bar_z, ph & 1, abort_flag);
            ++ph;
            __syncthreads();
            ok = *abort_flag == 0.f;
        }
        if (ok) {
            // G x = xs sG U';  sum_j M_tj (x.k_j) v_j = xs sV sW / sK Z'
            const float cu = xs * sG * eb, cz = xs * sV * sW / sK;
    #pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {           // every image is dead: the staging tile takes their place
                float uv[16], zv[16];
                tmem_ld32_x16(tl + kColU + col0 + 16 * h2, uv);
                tmem_ld32_x16(tl + kColS + col0 + 16 * h2, zv);
                tmem_wait_ld();
                stage_out16(smem, tok, col0 + 16 * h2, uv, zv, cu, cz);
            }
            if (iters && cq == 0 && valid) iters[base + tok] = it;
            __syncthreads();
            write_staged_rows(smem, out + base * kD, n, w, lane);
            if (kXout && x_out) {                          // the solutions themselves (fp32), x still in TMEM
                __syncthreads();                           // the tile's rows are read
                tmem_rows_out(smem, tl, kColX, tok, col0, x_out + base * kD, n, w, lane);
            }
        } else if (tid == kIssuer) {
            record_error(err, kErrTimeout);
            // one more bounded chance for every MMA issued so far to drain
            mma_commit(bar_ld);
            mbar_wait(bar_ld, 0);
            mbar_wait(bar_ld, 1);
            mbar_wait(bar_g, 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tbase, 512);
}

// =====================================================================
// Right-hand side of the adjoint solve, 128 tokens per CTA
// =====================================================================
// g_t = G_t^T dout_t for every token of the block, in the chunk form of the
// read-out with the roles of the two factors swapped:
//     g_t = e^{b_t} G_c^T dout_t + sum_{j <= t} M_tj (dout_t . v_j) k_j.
// Images: D = dout_t / s_t (per-token power of two), V / sV, K / sK, the mask
// M sK^2 / sW as in the solve, and the G image read K-major (it holds G
// transposed: its rows are the key index l). Products: S = D V^T,
// W = mask o S, U = D G, Z = W K, so
//     g_t = s_t (sG e^{b_t} U_t + sW sV / sK Z_t).
__global__ void __launch_bounds__(kBlkThreads, 1)
tc_rhs_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
              const float* __restrict__ gamma, const float* __restrict__ beta, const float* __restrict__ dout,
              int T, int np, const __half* __restrict__ img, const float* __restrict__ scales,
              float* __restrict__ rhs, unsigned* __restrict__ err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* Vr = smem + BlkSmem::oH;             // raw value rows
    uint8_t* Ks = smem + BlkSmem::oK;             // key image
    uint8_t* Ds = smem + BlkSmem::oP;             // raw key rows, then the dout image
    uint8_t* Ws = smem + BlkSmem::oW;             // value image, then the masked scores
    uint8_t* Gs = smem + BlkSmem::oG;             // value-state image
    __half* Mk = reinterpret_cast<__half*>(smem + BlkSmem::oM);
    float* seb = reinterpret_cast<float*>(smem + BlkSmem::oEb);
    float* sbc = reinterpret_cast<float*>(smem + BlkSmem::oB);
    float* sbeta = reinterpret_cast<float*>(smem + BlkSmem::oBeta);
    float* ecol = reinterpret_cast<float*>(smem + BlkSmem::oEcol);
    float4* red = reinterpret_cast<float4*>(smem + BlkSmem::oRed);
    float* misc = reinterpret_cast<float*>(smem + BlkSmem::oMisc);
    float* abort_flag = misc + 31;
    uint64_t* bar_in = reinterpret_cast<uint64_t*>(smem + BlkSmem::oBar);
    uint64_t* bar_g = bar_in + 1;
    uint64_t* bar_s = bar_in + 2;
    uint64_t* bar_u = bar_in + 3;
    uint64_t* bar_z = bar_in + 4;
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + BlkSmem::oSlot);

    const int blk = blockIdx.x, bh = blockIdx.y;
    const int t0 = blk * kBlk;
    const int n = min(kBlk, T - t0);
    const size_t base = (size_t)bh * T + t0;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int q4 = w & 3, cq = w >> 2;
    const int tok = 32 * q4 + lane;
    const bool valid = tok < n;
    constexpr int kIssuer = 256;
    const int col0 = 32 * cq;
    const size_t iG = image_index(bh, np, blk, 1);

    if (tid == 0) {
        mbar_init(bar_in, 1);
        mbar_init(bar_g, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_u, 1);
        mbar_init(bar_z, 1);
        fence_mbar_init();
        *abort_flag = 0.f;
        misc[20] = 0.f;                                // max |v| (as int bits, atomicMax)
    }
    if (w == 0) tmem_alloc(slot, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *slot;
    const uint32_t tl = tbase + ((uint32_t)(32 * q4) << 16);
    constexpr uint32_t kColU = 0, kColS = 128;

    const uint32_t row_bytes = (uint32_t)n * kD * 2;
    float* gstage = reinterpret_cast<float*>(red);
    const bool gates_bulk = n == kBlk && ((reinterpret_cast<uintptr_t>(gamma + base) |
                                            reinterpret_cast<uintptr_t>(beta + base)) & 15) == 0;
    // the dout rows (fp32) are staged too: tokens 0..63 in the key-image
    // buffer and 64..127 in the score buffer, both free until the images are
    // written after the maxima
    const int n_lo = n < 64 ? n : 64, n_hi = n - n_lo;
    if (tid == 0) {
        mbar_arrive_expect_tx(bar_in, 2 * row_bytes + (uint32_t)n * kD * 4 + (gates_bulk ? 2u * kBlk * 4u : 0u));
        bulk_g2s(Ds, k + base * kD, row_bytes, bar_in);
        bulk_g2s(Vr, v + base * kD, row_bytes, bar_in);
        bulk_g2s(Ks, dout + base * kD, (uint32_t)n_lo * kD * 4, bar_in);
        if (n_hi > 0) bulk_g2s(Ws, dout + (base + 64) * kD, (uint32_t)n_hi * kD * 4, bar_in);
        if (gates_bulk) {
            bulk_g2s(gstage, gamma + base, kBlk * 4, bar_in);
            bulk_g2s(gstage + kBlk, beta + base, kBlk * 4, bar_in);
        }
        mbar_arrive_expect_tx(bar_g, kImgBytes);
        bulk_g2s(Gs, img + iG * kImgHalves, kImgBytes, bar_g);
    }
    if (tid == 0 && !mbar_wait(bar_in, 0)) *abort_flag = 1.f;
    __syncthreads();
    // this thread's token row of dout (32 columns, fp32), from the staged rows
    float2 dd[16];
    {
        const float4* drow = reinterpret_cast<const float4*>(tok < 64 ? Ks : Ws) + (tok & 63) * (kD / 4) + col0 / 4;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
            if (valid) f = drow[g];
            dd[2 * g] = make_float2(f.x, f.y);
            dd[2 * g + 1] = make_float2(f.z, f.w);
        }
    }

    // gates, beta, the raw key and value rows and their maxima
    if (w == 0) warp_gate_cumsum128(gates_bulk ? gstage : gamma + base, n, sbc);
    float bmax = 0.f, kmax = 0.f, vmax = 0.f;
    if (tid < kBlk) {
        bmax = (tid < n) ? (gates_bulk ? gstage[kBlk + tid] : beta[base + tid]) : 0.f;
        sbeta[tid] = bmax;
    }
    uint4 kraw[4], vraw[4];
#pragma unroll
    for (int rep = 0; rep < 4; ++rep) {
        const int cid = tid + kBlkThreads * rep;
        const int j = cid >> 4, cc = cid & 15;
        kraw[rep] = vraw[rep] = make_uint4(0, 0, 0, 0);
        if (j < n) {
            kraw[rep] = *reinterpret_cast<const uint4*>(Ds + j * 256 + cc * 16);
            vraw[rep] = *reinterpret_cast<const uint4*>(Vr + j * 256 + cc * 16);
        }
        const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kraw[rep]);
        const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&vraw[rep]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 fk = __bfloat1622float2(k2[i]), fv = __bfloat1622float2(v2[i]);
            kmax = fmaxf(kmax, fmaxf(fabsf(fk.x), fabsf(fk.y)));
            vmax = fmaxf(vmax, fmaxf(fabsf(fv.x), fabsf(fv.y)));
        }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        kmax = fmaxf(kmax, __shfl_xor_sync(0xffffffffu, kmax, off));
        bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, off));
        vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, off));
    }
    if (lane == 0) {
        misc[w] = kmax;
        if (w < 4) misc[16 + w] = bmax;
        atomicMax(reinterpret_cast<int*>(misc + 20), __float_as_int(vmax));
    }
    __syncthreads();                                   // maxima visible; raw key rows read
    float sK, sW, sV;
    {
        float km = misc[0], bm = misc[16];
#pragma unroll
        for (int i = 1; i < 16; ++i) km = fmaxf(km, misc[i]);
#pragma unroll
        for (int i = 17; i < 20; ++i) bm = fmaxf(bm, misc[i]);
        sK = pow2_ceil(km);
        sW = pow2_ceil(bm * sK * sK);
        sV = pow2_ceil(misc[20]);
        const float inv_sK = 1.f / sK, inv_sV = 1.f / sV;
#pragma unroll
        for (int rep = 0; rep < 4; ++rep) {            // key image K / sK and value image V / sV (K-major)
            const int cid = tid + kBlkThreads * rep;
            const int j = cid >> 4, cc = cid & 15;
            const uint32_t off = (cc >> 3) * 16384 + j * 128 + (((cc & 7) ^ (j & 7)) << 4);
            *reinterpret_cast<uint4*>(Ks + off) = bf16x8_to_f16x8(kraw[rep], inv_sK);
            *reinterpret_cast<uint4*>(Ws + off) = bf16x8_to_f16x8(vraw[rep], inv_sV);
        }
    }
    if (tid < kBlk) seb[tid] = expf(sbc[tid]);
    const float msc = sK * sK / sW;
    decay_mask_diag(Mk, sbc, sbeta, ecol, n, msc, tid);
    // the dout image D = dout_t / s_t (the raw key rows in this buffer are consumed)
    float sd;
    {
        float2 a = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 16; ++i) a = __ffma2_rn(dd[i], dd[i], a);
        const float dn = quarter_sum(make_float4(a.x + a.y, 0.f, 0.f, 0.f), red, cq, tok).x;   // publishes seb, Mk
        sd = pow2_sqrt_scale(dn);
        store_row32(Ds, tok, col0, dd, 1.f / sd);
    }
    decay_mask_rest(Mk, sbc, ecol, n, msc, tid);
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    constexpr uint32_t kIdKK = idesc_f16(128, 128, false, false);
    constexpr uint32_t kIdKM = idesc_f16(128, 128, false, true);
    bool ok = *abort_flag == 0.f;
    if (ok) {
        if (tid == kIssuer) {
            issue_k128(tbase + kColS, smem_addr(Ds), smem_addr(Ws), 16, 16384, 16384, 32, kIdKK);   // S = D V^T
            mma_commit(bar_s);
            if (!mbar_wait(bar_g, 0)) {
                *abort_flag = 1.f;
            } else {
                // U = D G: the image's rows are G's columns l, so it is read K-major
                issue_k128(tbase + kColU, smem_addr(Ds), smem_addr(Gs), 16, 16384, 16384, 32, kIdKK);
            }
            mma_commit(bar_u);
        }
        wait_mma_each(bar_s, 0, abort_flag);
        // masked scores over the value image (S is complete, so V is dead); the
        // quarter of tokens 0..63 against keys 64..127 is written as zeros
        {
            const bool zero_blk = q4 < 2 && cq >= 2;
            const __half* mrow = Mk + tok * BlkSmem::kMS + col0;
            float2 wv[16];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                float sv[16];
                if (!zero_blk) {
                    tmem_ld32_x16(tl + kColS + col0 + 16 * h2, sv);
                    tmem_wait_ld();
                }
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    const uint4 m8 = *reinterpret_cast<const uint4*>(mrow + 16 * h2 + 8 * g);
                    const __half2* m2 = reinterpret_cast<const __half2*>(&m8);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int c = 4 * g + i;
                        wv[8 * h2 + c] = zero_blk ? make_float2(0.f, 0.f)
                                                  : __fmul2_rn(__half22float2(m2[i]), make_float2(sv[2 * c], sv[2 * c + 1]));
                    }
                }
            }
            store_row32(Ws, tok, col0, wv, 1.f);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        ok = *abort_flag == 0.f;
    }
    if (ok) {
        if (tid == kIssuer) {
            issue_k128(tbase + kColS, smem_addr(Ws), smem_addr(Ks), 16384, 16384, 8192, 2048, kIdKM);   // Z = W K
            mma_commit(bar_z);
        }
        wait_mma_each(bar_u, 0, abort_flag);
        wait_mma_each(bar_z, 0, abort_flag);
        __syncthreads();
        ok = *abort_flag == 0.f;
    }
    if (ok) {
        const float sG = scales[iG];
        const float cu = sd * sG * seb[tok], cz = sd * sW * sV / sK;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            float uv[16], zv[16];
            tmem_ld32_x16(tl + kColU + col0 + 16 * h2, uv);
            tmem_ld32_x16(tl + kColS + col0 + 16 * h2, zv);
            tmem_wait_ld();
            stage_out16(smem, tok, col0 + 16 * h2, uv, zv, cu, cz);
        }
        __syncthreads();
        write_staged_rows(smem, rhs + base * kD, n, w, lane);
    } else if (tid == kIssuer) {
        record_error(err, kErrTimeout);
        mma_commit(bar_in);                            // one more bounded chance for the MMAs to drain
        mbar_wait(bar_in, 1);
        mbar_wait(bar_g, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tbase, 256);
}

}  // namespace

bool tc_supported(int dk, int dv, int chunk, mesa_dtype dtype) {
    return dtype == MESA_BF16 && dk == kD && dv == kD && chunk == kC;
}

// One H and one G image (and their scales) per 128-token block.
size_t tc_images_bytes(int B, int H, int T) {
    const size_t np = (size_t)((T + kBlk - 1) / kBlk);
    return (size_t)B * H * np * 2 * kImgBytes;
}

size_t tc_workspace_bytes(int B, int H, int T) {
    const size_t np = (size_t)((T + kBlk - 1) / kBlk);
    return tc_images_bytes(B, H, T) + ((size_t)B * H * np * 2 * sizeof(float) + 255) / 256 * 256;
}

cudaError_t forward_tc(const ForwardArgs& a, cudaStream_t st) {
    const int nc = (a.T + kC - 1) / kC;
    const int BH = a.B * a.H;
    __half* img = reinterpret_cast<__half*>(a.workspace);
    float* scales = reinterpret_cast<float*>(static_cast<char*>(a.workspace) + tc_images_bytes(a.B, a.H, a.T));
    unsigned* err = error_word_ptr();
    const int cg_smem = BlkSmem::bytes + 1024;
    cudaError_t e = tc_scan_launch(a, img, scales, err, st);
    if (e != cudaSuccess) return e;
    auto kern = a.x_out ? tc_cg_kernel<false, true> : tc_cg_kernel<false, false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, cg_smem);
    if (e != cudaSuccess) return e;
#ifdef MESA_DEBUG
    static const int kOne = 1, kZero = 0;
    const bool inject = g_debug_skip_launches > 0;
    if (inject) {
        --g_debug_skip_launches;
        e = cudaMemcpyToSymbolAsync(g_debug_skip_commit, &kOne, sizeof(int), 0, cudaMemcpyHostToDevice, st);
        if (e != cudaSuccess) return e;
    }
#endif
    {
        LaunchTimer timer(kKindTcCg, st);
        kern<<<dim3((nc + 1) / 2, BH), kBlkThreads, cg_smem, st>>>(
            static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
            static_cast<const __nv_bfloat16*>(a.v), a.gamma, a.beta, a.lambda, a.H, a.T, (nc + 1) / 2, a.cg_steps, a.tol,
            img, scales, a.out, a.iters, err, a.x_out, a.x0, a.conv_q, a.conv_k, a.conv_w, nullptr, nullptr,
            nullptr, nullptr);
    }
#ifdef MESA_DEBUG
    if (inject) {
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        return cudaMemcpyToSymbolAsync(g_debug_skip_commit, &kZero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
    }
#endif
    return cudaGetLastError();
}

// The adjoint solve of the backward on the tensor-core path, from the state
// images and scales a forward_tc call over the same inputs left in
// `images_ws`: g = G_t^T dout into rhs_buf, then u and e_t.
cudaError_t tc_adjoint(const ForwardArgs& f, const void* images_ws, const float* dout, const float* xsol,
                       float* rhs_buf, float* dq, float* zt, cudaStream_t st) {
    const int nc = (f.T + kC - 1) / kC, np = (nc + 1) / 2;
    const int BH = f.B * f.H;
    const __half* img = reinterpret_cast<const __half*>(images_ws);
    const float* scales =
        reinterpret_cast<const float*>(static_cast<const char*>(images_ws) + tc_images_bytes(f.B, f.H, f.T));
    unsigned* err = error_word_ptr();
    const int smem = BlkSmem::bytes + 1024;
    cudaError_t e = cudaFuncSetAttribute(tc_rhs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_cg_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    {
        LaunchTimer timer(kKindBwdRhs, st);
        tc_rhs_kernel<<<dim3(np, BH), kBlkThreads, smem, st>>>(
            static_cast<const __nv_bfloat16*>(f.k), static_cast<const __nv_bfloat16*>(f.v), f.gamma, f.beta, dout,
            f.T, np, img, scales, rhs_buf, err);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    {
        LaunchTimer timer(kKindBwdAdj, st);
        tc_cg_kernel<true, false><<<dim3(np, BH), kBlkThreads, smem, st>>>(
            nullptr, static_cast<const __nv_bfloat16*>(f.k), static_cast<const __nv_bfloat16*>(f.v), f.gamma,
            f.beta, f.lambda, f.H, f.T, np, f.cg_steps, f.tol, img, scales, nullptr, nullptr, err, nullptr, nullptr,
            nullptr, nullptr, 0, rhs_buf, xsol, dq, zt);
    }
    return cudaGetLastError();
}

#ifdef MESA_DEBUG
cudaError_t tc_debug_skip_commit(int launches) {
    g_debug_skip_launches = launches;
    return cudaSuccess;
}
#endif

}  // namespace mesa
