// mlp_tc.cu -- TTT-MLP prefill: fp32 masters in tensor memory, 5th-generation tensor-core
// updates (tcgen05), warp-level MMAs for the small per-mini-batch products.
//
// The hidden state is the two-layer MLP f(x) = gelu(x W1 + b1) W2 + b2, d = 64 -> 256 -> 64
// (ttt-lm-pytorch README: "TTT-MLP ... a two-layer MLP"; "代码连连看——TTT": "TTTMLP is two
// TTTLinear stacked").  Each mini-batch takes the layer-wise dual update of TTT-Linear:
//   Z1 = XK W1 + b1, X2 = gelu(Z1), Z2 = X2 W2 + b2, g2 = ln_fused_l2_bwd(Z2, XV - XK),
//   g1 = (g2 W2^T) * gelu'(Z1),
//   Zbar1 = XQ W1 + b1 - M1 g1, Xbar2 = gelu(Zbar1), Zbar2 = Xbar2 W2 + b2 - M2 g2,
//   M1 = eta * tril(XQ XK^T + 1), M2 = eta * tril(Xbar2 X2^T + 1), out = XQ + LN(Zbar2),
//   full mini-batch: W1 -= (eta[K-1,:] XK)^T g1, W2 -= (eta[K-1,:] X2)^T g2, biases alike.
//
// Design (one CTA of 8 warps per (batch, head) chain, the whole sequence on chip):
//  * The fp32 masters W1^T (256 x 64) and W2 (256 x 64) live in tensor memory (hidden unit =
//    lane, two 128-lane tiles each, 256 columns) and take their rank-16 updates as accumulating
//    tcgen05 MMAs: W1^T += g1^T (-t lr XK), W2 += X2^T (-t lr g2).  They are issued as soon as
//    their operands exist and run while the warps compute the output path.  Afterwards the
//    masters are read back (tcgen05.ld) into bf16 shadows in 128-byte-swizzled shared memory.
//  * The per-mini-batch products involve 16 tokens, so they run as mma.sync m16n8k16 on all 8
//    warps at once (a tcgen05 MMA needs M >= 64 and a commit/wait round trip per dependent
//    step): warp w owns hidden units 32w..32w+31 of Z1, XQ W1, X2, g2 W2^T, g1, Zbar1, Xbar2,
//    and outputs 8w..8w+7 of Z2 and Zbar2.  The W shadows are the B operands (ldmatrix, plain
//    or transposed), the token tiles the A operands.
//  * The accumulator layout of a warp's [16 tokens x 32 hidden] tiles is reused as operand
//    layout without shared memory: as A of Xbar2 X2^T (k = hidden) directly, and as B of the
//    same product (k = hidden, n = token) directly; g1 reaches the B operand of M1 g1 by
//    movmatrix transposes.  X2, Xbar2 and g1 go to shared memory only where other warps or the
//    tensor cores read them.
//  * The two LayerNorms (loss gradient on Z2, output on Zbar2) run on token rows, 16 lanes per
//    row, after the warps' output slices meet in shared memory.
//  * XQ, XK, XV tiles arrive by TMA (K rows of 128 bytes from a 4-D tensor map, head-major or
//    token-major, 128-byte swizzle, no multicast) into a ring.
//    One thread issues the tcgen05 MMAs and commits to one mbarrier; all waits are bounded.
//  * Operand precision: every tensor-core operand is fp16 (11-bit significand), with fp32
//    accumulation.  The state path (both layers' products and updates) feeds back into itself
//    for every mini-batch, and with bf16 operands (8-bit) a few chains of the B=8, H=32, L=2048
//    workload end above 1e-2 relative error on b2.  The XQ and XK tiles are converted to fp16 in
//    place (the next mini-batch's at the end of each one; exact for bf16 values of magnitude up
//    to 65504, larger ones saturate), XV stays bf16; the W1 update scales g1 (not XK) by -t lr
//    so that no operand falls into fp16's subnormal range.  (In place, because two CTAs of this
//    kernel share an SM only while each needs under half of the SM's shared memory.)
#include "tc5.cuh"
#include "ttt_common.cuh"
#include "ttt_internal.h"

#include <cuda_fp16.h>

namespace ttt {
namespace {

constexpr int kThreads = 256;
constexpr int kHid = TTT_HIDDEN;
constexpr int kStages = 2;
constexpr int kTile = TTT_KMAX * 128;  // [16 rows x 128 bytes] bf16 tile
constexpr uint32_t kTmemCols = 256;
constexpr long long kDrainPolls = 1ll << 24;
constexpr uint32_t cW1 = 0;    // + 64 mt: W1^T tile mt (rows = hidden 128mt.., cols = input dim)
constexpr uint32_t cW2 = 128;  // + 64 mt: W2 tile mt (rows = hidden, cols = output dim)

struct __align__(1024) MlpSmem {
    uint8_t stage[kStages][3 * kTile];  // XK | XQ | XV, bf16 as loaded; XK, XQ then fp16 in place
    uint8_t W1s[2][128 * 128];          // fp16 W1^T shadow [tile][128 hidden rows x 128 B (64 inputs)]
    uint8_t W2s[kHid * 128];            // fp16 W2 shadow [256 hidden rows x 128 B (64 outputs)]
    uint8_t X2s[4 * kTile];             // fp16 X2     [4 hidden blocks][16 token rows x 128 B]
    uint8_t XB2s[4 * kTile];            // fp16 Xbar2
    uint8_t G1s[4 * kTile];             // fp16 -t_{K-1} lr g1
    uint8_t G2s[kTile];                 // fp16 g2 [16 token rows x 128 B (64 outputs)]
    uint8_t G2Ls[kTile];                // fp16 -t_{K-1} lr g2
    union {                             // (disjoint lifetimes inside a mini-batch)
        float Zt[TTT_KMAX][TTT_D];      // Z2, then Zbar2, as token rows (b2 included)
        __half A2p[8][TTT_KMAX][TTT_KMAX];  // Xbar2 X2^T over each warp's hidden slice
    };
    float A2[TTT_KMAX][TTT_KMAX];       // their sum
    float b2[TTT_D];
    float lr[kStages][TTT_KMAX];
    float te[TTT_KMAX];
    uint64_t full[kStages];
    uint64_t mma_bar;
    uint64_t drain_bar;
    uint32_t tmem_base;
    int fail;
    long long out_off;                  // element offset of this chain's token 0 in out
};

// byte offset of bf16 element (row r, col c < 64) in a [rows x 128 B] tile, 128-byte swizzle
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return static_cast<uint32_t>(r * 128 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1));
}

__device__ __forceinline__ float tanh_fast(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// tanh form of GELU and its derivative
__device__ __forceinline__ void gelu2(float x, float& y, float& dy) {
    const float k = 0.7978845608028654f, c = 0.044715f;
    const float th = tanh_fast(k * fmaf(c * x, x * x, x));
    y = 0.5f * x * (1.0f + th);
    dy = 0.5f * (1.0f + th) + 0.5f * x * (1.0f - th * th) * k * fmaf(3.0f * c, x * x, 1.0f);
}
__device__ __forceinline__ float gelu(float x) {
    const float k = 0.7978845608028654f, c = 0.044715f;
    return 0.5f * x * (1.0f + tanh_fast(k * fmaf(c * x, x * x, x)));
}

// The same for two elements at once with paired fp32 arithmetic (one FFMA2 per two FFMAs).
__device__ __forceinline__ void gelu2_pair(float2 x, float2& y, float2& dy) {
    const float2 k = make_float2(0.7978845608028654f, 0.7978845608028654f), c = make_float2(0.044715f, 0.044715f);
    const float2 h = make_float2(0.5f, 0.5f), one = make_float2(1.0f, 1.0f);
    const float2 x2 = __fmul2_rn(x, x);
    const float2 u = __fmul2_rn(k, __ffma2_rn(__fmul2_rn(c, x), x2, x));
    const float2 th = make_float2(tanh_fast(u.x), tanh_fast(u.y));
    const float2 hx = __fmul2_rn(h, x), op = __fadd2_rn(one, th);
    y = __fmul2_rn(hx, op);
    const float2 sech2 = __ffma2_rn(__fmul2_rn(th, th), make_float2(-1.0f, -1.0f), one);
    const float2 poly = __fmul2_rn(k, __ffma2_rn(make_float2(3.0f * 0.044715f, 3.0f * 0.044715f), x2, one));
    dy = __ffma2_rn(__fmul2_rn(hx, sech2), poly, __fmul2_rn(h, op));
}
__device__ __forceinline__ float2 gelu_pair(float2 x) {
    const float2 k = make_float2(0.7978845608028654f, 0.7978845608028654f), c = make_float2(0.044715f, 0.044715f);
    const float2 u = __fmul2_rn(k, __ffma2_rn(__fmul2_rn(c, x), __fmul2_rn(x, x), x));
    const float2 th = make_float2(tanh_fast(u.x), tanh_fast(u.y));
    return __fmul2_rn(__fmul2_rn(make_float2(0.5f, 0.5f), x), __fadd2_rn(make_float2(1.0f, 1.0f), th));
}

// Mean and 1/sqrt(var + eps) of a 64-value row held 4 per lane by 16 lanes (Chan merges).
__device__ __forceinline__ void row_stats16(const float (&v)[4], float eps, float& mu, float& rstd) {
    float m = 0.25f * ((v[0] + v[1]) + (v[2] + v[3]));
    float M2 = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) M2 = fmaf(v[i] - m, v[i] - m, M2);
#pragma unroll
    for (int off = 1; off < 16; off <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, off);
        const float M2o = __shfl_xor_sync(0xffffffffu, M2, off);
        const float dm = mo - m;
        M2 = M2 + M2o + dm * dm * (2.0f * off);
        m = 0.5f * (m + mo);
    }
    mu = m;
    rstd = rsqrtf(M2 * (1.0f / TTT_D) + eps);
}

__device__ __forceinline__ float sum16(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    return v;
}

// 4 consecutive bf16 of row r starting at column c (c % 4 == 0) -> floats
__device__ __forceinline__ void ld4_bf16(const uint8_t* tile, int r, int c, float* out) {
    const uint2 v = *reinterpret_cast<const uint2*>(tile + swz(r, c));
    const float2 a = unpack_bf16x2(v.x), b = unpack_bf16x2(v.y);
    out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
}
__device__ __forceinline__ void st4_f16(uint8_t* tile, int r, int c, float a, float b, float d, float e) {
    *reinterpret_cast<uint2*>(tile + swz(r, c)) = make_uint2(pack_f16x2(a, b), pack_f16x2(d, e));
}

// A stage's XK and XQ tiles from bf16 to fp16 in place: thread tid converts one 16-byte chunk,
// of XK for tid < 128 and of XQ otherwise.
__device__ __forceinline__ void convert_stage(uint8_t* stage, int tid) {
    uint4* p = reinterpret_cast<uint4*>(stage + 16u * static_cast<uint32_t>(tid & 127) +
                                        static_cast<uint32_t>(tid >> 7) * kTile);
    const uint4 v = *p;
    *p = make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z), bf16x2_to_f16x2(v.w));
}

// 4 consecutive fp16 of row r starting at column c (c % 4 == 0) -> floats
__device__ __forceinline__ void ld4_f16(const uint8_t* tile, int r, int c, float* out) {
    const uint2 v = *reinterpret_cast<const uint2*>(tile + swz(r, c));
    const float2 a = unpack_f16x2(v.x), b = unpack_f16x2(v.y);
    out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
}

// [16 tokens x 32 hidden] slice of this warp: four m16n8 accumulator tiles (hidden 8nt + 2t + e,
// rows g and g+8), written as bf16 pairs into a [4 blocks][16 x 128 B] token-row operand tile.
__device__ __forceinline__ void store_slice(uint8_t* tiles, int w, int g, int t, const uint32_t (&p)[4][2]) {
    uint8_t* blk = tiles + (w >> 1) * kTile;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        const int c = 32 * (w & 1) + 8 * nt + 2 * t;
        *reinterpret_cast<uint32_t*>(blk + swz(g, c)) = p[nt][0];
        *reinterpret_cast<uint32_t*>(blk + swz(g + 8, c)) = p[nt][1];
    }
}

// D[16 x 8] += A[16 x 256] B[256 x 8] with A a [4 blocks][16 x 128 B] token-row tile (X2 or Xbar2)
// and B the W2 shadow's 8 output columns 8w.. (k = hidden rows, read transposed).  Two
// accumulators (even and odd k-steps) halve the dependent chain.
__device__ __forceinline__ void tokens_times_w2(float (&acc)[2][4], uint32_t a_tiles, uint32_t w2, int w, int lane,
                                                int lrow, int lchunk) {
#pragma unroll
    for (int p = 0; p < 8; ++p) {  // pairs of k-steps: hidden rows 32p .. 32p + 31
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(w2 + swz128(32 * p + lane, w), b0, b1, b2, b3);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int ks = 2 * p + hh;  // hidden 16 ks .. 16 ks + 15
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(a_tiles + (ks >> 2) * kTile + swz128(lrow, 2 * (ks & 3) + lchunk), a0, a1, a2, a3);
            mma_f16_16816(acc[hh], a0, a1, a2, a3, hh ? b2 : b0, hh ? b3 : b1);
        }
    }
}

__global__ void __launch_bounds__(kThreads, 2)
mlp_tc_kernel(const MlpArgs a, const __grid_constant__ LinearMaps maps) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    MlpSmem& s = *reinterpret_cast<MlpSmem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));

    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int q = w & 3, mt = w >> 2;            // tensor-memory lane quarter and 128-lane tile
    const int u = 128 * mt + 32 * q + lane;      // the hidden unit whose master rows this thread moves
    const int g = lane >> 2, t = lane & 3;
    const int chain = blockIdx.x;
    const int h = chain % a.H, bi = chain / a.H;
    const int K = a.K;
    const int n_full = static_cast<int>(a.n_full);
    const int n_mb = n_full + (a.rem > 0 ? 1 : 0);
    const float eps = a.eps;
    const long long wait_limit = a.wait_limit;
    const float* lr_g = a.lr + static_cast<long long>(chain) * a.L;
    const uint32_t tile_tx = static_cast<uint32_t>(K) * TTT_D * 2;

    // ---- set-up --------------------------------------------------------------------------------
    if (w == 0) tc5::alloc(&s.tmem_base, kTmemCols);
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) mbar_init(&s.full[i], 1);
        mbar_init(&s.mma_bar, 1);
        mbar_init(&s.drain_bar, 1);
        fence_mbarrier_init();
        tma_prefetch_desc(&maps.xq);
        tma_prefetch_desc(&maps.xk);
        tma_prefetch_desc(&maps.xv);
        s.fail = 0;
        s.out_off = bi * a.act_b + h * a.act_h;
    }
    for (int i = tid; i < kStages * 3 * kTile / 16; i += kThreads)
        reinterpret_cast<uint4*>(&s.stage[0][0])[i] = make_uint4(0, 0, 0, 0);  // rows >= K stay zero
    if (tid < TTT_KMAX) s.te[tid] = a.token_eta ? (tid < K ? a.token_eta[tid] : 0.f) : 1.0f / (tid + 1);
    const long long w0off = a.w0_chain_stride ? static_cast<long long>(chain) * a.w0_chain_stride
                                              : static_cast<long long>(h) * TTT_D * kHid;
    const long long b1off = a.w0_chain_stride ? static_cast<long long>(chain) * kHid : static_cast<long long>(h) * kHid;
    const long long b2off = a.w0_chain_stride ? static_cast<long long>(chain) * TTT_D : static_cast<long long>(h) * TTT_D;
    if (tid < TTT_D) s.b2[tid] = a.b2_0[b2off + tid];
    // b1 at this thread's accumulator columns: hidden 32w + 8nt + 2t + e
    float b1r[4][2];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) b1r[nt][e] = a.b1_0[b1off + 32 * w + 8 * nt + 2 * t + e];
    fence_proxy_async_smem();
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();
    const uint32_t tm = s.tmem_base;
    const uint32_t my_lane = static_cast<uint32_t>(32 * q);  // base lane of this warp's quarter

    // masters into tensor memory, bf16 shadows into shared memory
    {
        const float* W1 = a.W1_0 + w0off;  // [64 in][256 hid]
        const float* W2 = a.W2_0 + w0off;  // [256 hid][64 out]
        const int r = u & 127;             // row of this thread in its 128-row tile
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float v1[16], v2[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                v1[i] = W1[(16 * c + i) * kHid + u];
                v2[i] = W2[u * TTT_D + 16 * c + i];
            }
            tc5::st16(tc5::taddr(tm, my_lane, cW1 + 64 * mt + 16 * c), v1);
            tc5::st16(tc5::taddr(tm, my_lane, cW2 + 64 * mt + 16 * c), v2);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int cc = 16 * c + 8 * half;  // 8 columns = one 16-byte chunk
                uint4 p1, p2;
                p1.x = pack_f16x2(v1[8 * half + 0], v1[8 * half + 1]); p1.y = pack_f16x2(v1[8 * half + 2], v1[8 * half + 3]);
                p1.z = pack_f16x2(v1[8 * half + 4], v1[8 * half + 5]); p1.w = pack_f16x2(v1[8 * half + 6], v1[8 * half + 7]);
                p2.x = pack_f16x2(v2[8 * half + 0], v2[8 * half + 1]); p2.y = pack_f16x2(v2[8 * half + 2], v2[8 * half + 3]);
                p2.z = pack_f16x2(v2[8 * half + 4], v2[8 * half + 5]); p2.w = pack_f16x2(v2[8 * half + 6], v2[8 * half + 7]);
                *reinterpret_cast<uint4*>(&s.W1s[mt][0] + swz(r, cc)) = p1;
                *reinterpret_cast<uint4*>(&s.W2s[0] + swz(u, cc)) = p2;
            }
        }
        tc5::wait_st();
    }
    fence_proxy_async_smem();
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();

    // producer (warp 0): mini-batch mm into stage st.  lr comes by one bulk copy when its slice
    // is 16-byte aligned and a multiple of 16 bytes (one arrival on the stage's barrier), else by
    // plain loads of the warp before the arrival (per-lane asynchronous arrivals would serialise
    // in the barrier unit while every other warp waits for this one)
    const bool lr_bulk = (K % 4 == 0) && (a.L % 4 == 0) && ((reinterpret_cast<uintptr_t>(a.lr) & 15) == 0);
    auto issue = [&](int mm, int st) {
        const int Kmm = mm < n_full ? K : static_cast<int>(a.rem);
        const int row0 = mm * K;
        const bool bulk = lr_bulk && (Kmm % 4 == 0);
        if (!bulk) {
            if (lane < TTT_KMAX) s.lr[st][lane] = lane < Kmm ? lr_g[row0 + lane] : 0.f;
            __syncwarp();
        }
        if (lane == 0) {
            if (bulk)
                for (int j = Kmm; j < TTT_KMAX; ++j) s.lr[st][j] = 0.f;
            const uint32_t lr_tx = bulk ? static_cast<uint32_t>(Kmm) * 4 : 0u;
            mbar_arrive_expect_tx(&s.full[st], 3 * tile_tx + lr_tx);  // (release: orders the stores above)
            // coordinates (0, token, h, b) head-major, (0, h, token, b) token-major
            const int c1 = a.tok_major ? h : row0, c2 = a.tok_major ? row0 : h;
            tma_load_4d(&s.stage[st][0], &maps.xk, 0, c1, c2, bi, &s.full[st]);
            tma_load_4d(&s.stage[st][kTile], &maps.xq, 0, c1, c2, bi, &s.full[st]);
            tma_load_4d(&s.stage[st][2 * kTile], &maps.xv, 0, c1, c2, bi, &s.full[st]);
            if (bulk) bulk_load(&s.lr[st][0], lr_g + row0, lr_tx, &s.full[st]);
        }
    };
    if (w == 0)
        for (int mm = 0; mm < kStages - 1 && mm < n_mb; ++mm) issue(mm, mm);

    // row-phase geometry (all 8 warps): token row rr, features f4..f4+3 (16 lanes per row)
    const int rr = tid >> 4, f4 = 4 * (tid & 15);
    float lw[4], lb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        lw[i] = a.ln_w[h * TTT_D + f4 + i];
        lb[i] = a.ln_b[h * TTT_D + f4 + i];
    }
    const float tl = s.te[K - 1];
    const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;  // ldmatrix row supplied by this lane
    const int lchunk = lane >> 4;
    // -t_i on the lower triangle j <= i, zero above, at this lane's (i, j) positions of a 16x16
    // accumulator: M[i][j] = c (A[i][j] + 1), c = tmask lr_j
    float tmask[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int i = g + 8 * (e >> 1), j = 8 * nt + 2 * t + (e & 1);
            tmask[nt][e] = (j <= i) ? -s.te[i] : 0.f;
        }
    const uint32_t idUp = tc5::idesc_f16(128, 64, 1, 1);
    const uint64_t dX2m = tc5::sdesc(smem_u32(&s.X2s[0]), kTile, 1024);     // X2^T, MN-major A
    const uint64_t dG1m = tc5::sdesc(smem_u32(&s.G1s[0]), kTile, 1024);     // (-t lr g1)^T, MN-major A
    const uint64_t dXK16m = tc5::sdesc(smem_u32(&s.stage[0][0]), kTile, 1024);  // XK (fp16) of stage 0, MN-major B
    const uint64_t dG2Lm = tc5::sdesc(smem_u32(&s.G2Ls[0]), kTile, 1024);   // -t lr g2, MN-major B
    const uint32_t w1_s = smem_u32(&s.W1s[(32 * w) >> 7][0]);  // this warp's 32 hidden rows live in one tile
    const int w1_row0 = (32 * w) & 127;
    const uint32_t w2_s = smem_u32(&s.W2s[0]);
    const uint32_t x2_s = smem_u32(&s.X2s[0]), xb2_s = smem_u32(&s.XB2s[0]), g2_s = smem_u32(&s.G2s[0]);

    // M = c (A + 1) of a 16x16 accumulator pair, as the A operand of a 16x16x16 MMA
    auto m_operand = [&](const float (&at)[2][4], const float* lr_s, uint32_t (&ma)[4]) {
        const float2 l01 = *reinterpret_cast<const float2*>(&lr_s[2 * t]);
        const float2 l89 = *reinterpret_cast<const float2*>(&lr_s[2 * t + 8]);
        const float c00 = tmask[0][0] * l01.x, c01 = tmask[0][1] * l01.y, c02 = tmask[0][2] * l01.x, c03 = tmask[0][3] * l01.y;
        const float c10 = tmask[1][0] * l89.x, c11 = tmask[1][1] * l89.y, c12 = tmask[1][2] * l89.x, c13 = tmask[1][3] * l89.y;
        ma[0] = pack_f16x2(fmaf(c00, at[0][0], c00), fmaf(c01, at[0][1], c01));
        ma[1] = pack_f16x2(fmaf(c02, at[0][2], c02), fmaf(c03, at[0][3], c03));
        ma[2] = pack_f16x2(fmaf(c10, at[1][0], c10), fmaf(c11, at[1][1], c11));
        ma[3] = pack_f16x2(fmaf(c12, at[1][2], c12), fmaf(c13, at[1][3], c13));
    };

    // the fp16 copy of stage 0 before the loop; that of mini-batch m + 1 at the end of m
    if (n_mb > 0) {
        if (!mbar_wait_bounded(&s.full[0], 0, wait_limit, a.status)) s.fail = 1;
        convert_stage(&s.stage[0][0], tid);
    }
    __syncthreads();

    uint32_t mpar = 0;  // phase parity of mma_bar
    int st = 0;
    uint32_t par = 0;
    int m_stop = n_mb;  // first mini-batch whose loads may still be in flight (failure path)
    for (int m = 0; m < n_mb; ++m, st = (st + 1 == kStages ? 0 : st + 1), par ^= (st == 0)) {
        const bool full_mb = m < n_full;
        const int Km = full_mb ? K : static_cast<int>(a.rem);
        if (w == 0 && m + kStages - 1 < n_mb) issue(m + kStages - 1, (m + kStages - 1) % kStages);
        if (!mbar_wait_bounded(&s.full[st], par, wait_limit, a.status)) s.fail = 1;
        const uint8_t* xk_t = &s.stage[st][0];  // fp16 (converted)
        const uint8_t* xq_t = &s.stage[st][kTile];
        const uint8_t* xv_t = &s.stage[st][2 * kTile];  // bf16
        const float* lr_s = s.lr[st];
        const uint32_t xk_s = smem_u32(xk_t), xq_s = smem_u32(xq_t);

        // (1) Z1 = XK W1 + b1, XQ W1 + b1 on this warp's 32 hidden units; XQ XK^T
        float z1[4][4], zb1[4][4], at1[2][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            z1[nt][0] = z1[nt][2] = zb1[nt][0] = zb1[nt][2] = b1r[nt][0];
            z1[nt][1] = z1[nt][3] = zb1[nt][1] = zb1[nt][3] = b1r[nt][1];
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) at1[0][e] = at1[1][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t k0, k1, k2, k3, q0, q1, q2, q3;
            ldmatrix_x4(xk_s + swz128(lrow, 2 * kk + lchunk), k0, k1, k2, k3);
            ldmatrix_x4(xq_s + swz128(lrow, 2 * kk + lchunk), q0, q1, q2, q3);
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {  // hidden 32w + 16hb .. + 15: n-tiles 2hb, 2hb + 1
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(w1_s + swz128(w1_row0 + 16 * hb + lrow, 2 * kk + lchunk), b0, b1, b2, b3);
                mma_f16_16816(z1[2 * hb], k0, k1, k2, k3, b0, b2);
                mma_f16_16816(z1[2 * hb + 1], k0, k1, k2, k3, b1, b3);
                mma_f16_16816(zb1[2 * hb], q0, q1, q2, q3, b0, b2);
                mma_f16_16816(zb1[2 * hb + 1], q0, q1, q2, q3, b1, b3);
            }
            mma_f16_16816(at1[0], q0, q1, q2, q3, k0, k2);  // tokens 0-7 of XK as B
            mma_f16_16816(at1[1], q0, q1, q2, q3, k1, k3);  // tokens 8-15
        }

        // (2) X2 = gelu(Z1), keep gelu'(Z1); X2 to shared memory (A of Z2, A of W2's update)
        float dg[4][4];
        uint32_t x2p[4][2];  // X2 as bf16 pairs: [n-tile][row g, row g + 8]
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            float2 y0, y1, d0, d1;
            gelu2_pair(make_float2(z1[nt][0], z1[nt][1]), y0, d0);
            gelu2_pair(make_float2(z1[nt][2], z1[nt][3]), y1, d1);
            dg[nt][0] = d0.x; dg[nt][1] = d0.y; dg[nt][2] = d1.x; dg[nt][3] = d1.y;
            x2p[nt][0] = pack_f16x2(y0.x, y0.y);
            x2p[nt][1] = pack_f16x2(y1.x, y1.y);
        }
        store_slice(&s.X2s[0], w, g, t, x2p);
        __syncthreads();

        // (3) Z2 = X2 W2 + b2 on this warp's outputs 8w..8w+7 -> token rows in Zt
        {
            float z2[2][4];
            const float2 bb = *reinterpret_cast<const float2*>(&s.b2[8 * w + 2 * t]);
            z2[0][0] = z2[0][2] = bb.x;
            z2[0][1] = z2[0][3] = bb.y;
#pragma unroll
            for (int e = 0; e < 4; ++e) z2[1][e] = 0.f;
            tokens_times_w2(z2, x2_s, w2_s, w, lane, lrow, lchunk);
            *reinterpret_cast<float2*>(&s.Zt[g][8 * w + 2 * t]) = make_float2(z2[0][0] + z2[1][0], z2[0][1] + z2[1][1]);
            *reinterpret_cast<float2*>(&s.Zt[g + 8][8 * w + 2 * t]) = make_float2(z2[0][2] + z2[1][2], z2[0][3] + z2[1][3]);
        }
        __syncthreads();

        // (4) g2 = ln_fused_l2_bwd(Z2, XV - XK) on token rows; -t lr g2 and -t lr XK for the updates
        {
            float z[4], xk[4], xv[4];
            const float4 zz = *reinterpret_cast<const float4*>(&s.Zt[rr][f4]);
            z[0] = zz.x; z[1] = zz.y; z[2] = zz.z; z[3] = zz.w;
            ld4_f16(xk_t, rr, f4, xk);
            ld4_bf16(xv_t, rr, f4, xv);
            float mu, rs;
            row_stats16(z, eps, mu, rs);
            float xh[4], qv[4], sq = 0.f, sqx = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xh[i] = (z[i] - mu) * rs;
                qv[i] = lw[i] * (fmaf(lw[i], xh[i], lb[i]) - (xv[i] - xk[i]));
                sq += qv[i];
                sqx = fmaf(qv[i], xh[i], sqx);
            }
            sq = sum16(sq);
            sqx = sum16(sqx);
            const float sc = (rr < Km) ? rs * (1.0f / TTT_D) : 0.f;
            float g2[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) g2[i] = fmaf(-xh[i], sqx, fmaf(static_cast<float>(TTT_D), qv[i], -sq)) * sc;
            st4_f16(&s.G2s[0], rr, f4, g2[0], g2[1], g2[2], g2[3]);
            const float ls = -tl * lr_s[rr];
            st4_f16(&s.G2Ls[0], rr, f4, ls * g2[0], ls * g2[1], ls * g2[2], ls * g2[3]);
        }
        __syncthreads();

        // (5) g2 W2^T on this warp's hidden units; (6) g1 = (g2 W2^T) * gelu'(Z1)
        float g1[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) g1[nt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(g2_s + swz128(lrow, 2 * kk + lchunk), a0, a1, a2, a3);
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
                uint32_t b0, b1, b2, b3;  // W2 rows = hidden (n), outputs = k
                ldmatrix_x4(w2_s + swz128(32 * w + 16 * hb + lrow, 2 * kk + lchunk), b0, b1, b2, b3);
                mma_f16_16816(g1[2 * hb], a0, a1, a2, a3, b0, b2);
                mma_f16_16816(g1[2 * hb + 1], a0, a1, a2, a3, b1, b3);
            }
        }
        uint32_t g1p[4][2], g1s[4][2];  // g1, and -t_{K-1} lr g1 for W1's update, as fp16 pairs
        {
            const float lg = lr_s[g], lg8 = lr_s[g + 8];
            const float sg = -tl * lg, sg8 = -tl * lg8;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) g1[nt][e] *= dg[nt][e];
                g1p[nt][0] = pack_f16x2(g1[nt][0], g1[nt][1]);
                g1p[nt][1] = pack_f16x2(g1[nt][2], g1[nt][3]);
                g1s[nt][0] = pack_f16x2(sg * g1[nt][0], sg * g1[nt][1]);
                g1s[nt][1] = pack_f16x2(sg8 * g1[nt][2], sg8 * g1[nt][3]);
                // b1 -= t_{K-1} sum_j lr_j g1_j (sum over the 16 token rows: lanes g = 0..7)
                if (full_mb) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        float v = fmaf(lg, g1[nt][e], lg8 * g1[nt][2 + e]);
                        v += __shfl_xor_sync(0xffffffffu, v, 4);
                        v += __shfl_xor_sync(0xffffffffu, v, 8);
                        v += __shfl_xor_sync(0xffffffffu, v, 16);
                        b1r[nt][e] -= tl * v;
                    }
                }
            }
        }
        store_slice(&s.G1s[0], w, g, t, g1s);
        // the state update on a full mini-batch, on the tensor cores while the output path runs:
        // W1^T += g1^T (-t lr XK), W2 += X2^T (-t lr g2)
        fence_proxy_async_smem();
        tc5::fence_before();
        __syncthreads();
        tc5::fence_after();
        if (tid == 0 && full_mb) {
#pragma unroll
            for (int t2 = 0; t2 < 2; ++t2) {
                tc5::mma_ss(tm + cW1 + 64 * t2, tc5::sdesc_add(dG1m, t2 * 2 * kTile),
                            tc5::sdesc_add(dXK16m, st * 3 * kTile), idUp, 1);
                tc5::mma_ss(tm + cW2 + 64 * t2, tc5::sdesc_add(dX2m, t2 * 2 * kTile), dG2Lm, idUp, 1);
            }
            tc5::commit(&s.mma_bar);
        }

        // (7) Zbar1 = XQ W1 + b1 - M1 g1 (M1 = eta * tril(XQ XK^T + 1), g1 as B by transposes)
        {
            uint32_t ma[4];
            m_operand(at1, lr_s, ma);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
                mma_f16_16816(zb1[nt], ma[0], ma[1], ma[2], ma[3], movmatrix_trans(g1p[nt][0]),
                               movmatrix_trans(g1p[nt][1]));
        }

        // (8) Xbar2 = gelu(Zbar1); Xbar2 X2^T over this warp's hidden units, summed over warps
        {
            uint32_t xb2p[4][2];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const float2 y0 = gelu_pair(make_float2(zb1[nt][0], zb1[nt][1]));
                const float2 y1 = gelu_pair(make_float2(zb1[nt][2], zb1[nt][3]));
                xb2p[nt][0] = pack_f16x2(y0.x, y0.y);
                xb2p[nt][1] = pack_f16x2(y1.x, y1.y);
            }
            store_slice(&s.XB2s[0], w, g, t, xb2p);
            float a2[2][4] = {};
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {  // hidden n-tiles 2kk, 2kk + 1 form one k-step
                // A = Xbar2 (rows = tokens), B = X2 (k = hidden, n = tokens), both from accumulators
                mma_f16_16816(a2[0], xb2p[2 * kk][0], xb2p[2 * kk][1], xb2p[2 * kk + 1][0], xb2p[2 * kk + 1][1],
                               x2p[2 * kk][0], x2p[2 * kk + 1][0]);
                mma_f16_16816(a2[1], xb2p[2 * kk][0], xb2p[2 * kk][1], xb2p[2 * kk + 1][0], xb2p[2 * kk + 1][1],
                               x2p[2 * kk][1], x2p[2 * kk + 1][1]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                *reinterpret_cast<__half2*>(&s.A2p[w][g][8 * nt + 2 * t]) = __floats2half2_rn(a2[nt][0], a2[nt][1]);
                *reinterpret_cast<__half2*>(&s.A2p[w][g + 8][8 * nt + 2 * t]) = __floats2half2_rn(a2[nt][2], a2[nt][3]);
            }
        }
        __syncthreads();
        {  // one element of the 16x16 sum per thread
            const __half* p = &s.A2p[0][0][0] + tid;
            constexpr int kS = TTT_KMAX * TTT_KMAX;
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = __half2float(p[i * kS]);
            (&s.A2[0][0])[tid] = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
        }
        __syncthreads();

        // (9) Zbar2 = Xbar2 W2 + b2 - M2 g2 on this warp's outputs -> token rows in Zt
        float b2d[2];
        {
            float at2[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                at2[nt][0] = s.A2[g][8 * nt + 2 * t];
                at2[nt][1] = s.A2[g][8 * nt + 2 * t + 1];
                at2[nt][2] = s.A2[g + 8][8 * nt + 2 * t];
                at2[nt][3] = s.A2[g + 8][8 * nt + 2 * t + 1];
            }
            uint32_t ma[4];
            m_operand(at2, lr_s, ma);
            float zb2[2][4];
            const float2 bb = *reinterpret_cast<const float2*>(&s.b2[8 * w + 2 * t]);
            zb2[0][0] = zb2[0][2] = bb.x;
            zb2[0][1] = zb2[0][3] = bb.y;
#pragma unroll
            for (int e = 0; e < 4; ++e) zb2[1][e] = 0.f;
            tokens_times_w2(zb2, xb2_s, w2_s, w, lane, lrow, lchunk);
            {
                uint32_t b0, b1, d0, d1;  // g2 (k = tokens, n = outputs 8w..), transposed from token rows
                ldmatrix_x4_trans(g2_s + swz128(lrow, w), b0, b1, d0, d1);
                mma_f16_16816(zb2[1], ma[0], ma[1], ma[2], ma[3], b0, b1);
                // sum_j lr_j g2_j for b2's update: an A operand whose row 0 is lr
                const uint32_t r0 = g == 0 ? pack_f16x2(lr_s[2 * t], lr_s[2 * t + 1]) : 0u;
                const uint32_t r2 = g == 0 ? pack_f16x2(lr_s[2 * t + 8], lr_s[2 * t + 9]) : 0u;
                float bd[4] = {0.f, 0.f, 0.f, 0.f};
                mma_f16_16816(bd, r0, 0u, r2, 0u, b0, b1);
                b2d[0] = bd[0];  // row 0, outputs 8w + 2t, 8w + 2t + 1 (lanes g == 0)
                b2d[1] = bd[1];
            }
            *reinterpret_cast<float2*>(&s.Zt[g][8 * w + 2 * t]) = make_float2(zb2[0][0] + zb2[1][0], zb2[0][1] + zb2[1][1]);
            *reinterpret_cast<float2*>(&s.Zt[g + 8][8 * w + 2 * t]) = make_float2(zb2[0][2] + zb2[1][2], zb2[0][3] + zb2[1][3]);
        }
        __syncthreads();

        // (10) out = XQ + LN(Zbar2) on token rows
        {
            float z[4], xq[4];
            const float4 zz = *reinterpret_cast<const float4*>(&s.Zt[rr][f4]);
            z[0] = zz.x; z[1] = zz.y; z[2] = zz.z; z[3] = zz.w;
            ld4_f16(xq_t, rr, f4, xq);
            float mu, rs;
            row_stats16(z, eps, mu, rs);
            if (rr < Km) {
                float o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) o[i] = xq[i] + fmaf(lw[i], (z[i] - mu) * rs, lb[i]);
                __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) + s.out_off +
                                     (static_cast<long long>(m) * K + rr) * a.act_t;
                *reinterpret_cast<uint2*>(out + f4) = make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
            }
        }

        // (11) new state: b2, and the bf16 shadows of the updated masters
        if (full_mb) {
            if (!mbar_wait_bounded(&s.mma_bar, mpar, wait_limit, a.status)) s.fail = 1;
            mpar ^= 1;
            tc5::fence_after();
            __syncthreads();  // every warp is done reading the shadows
            if (g == 0) {
                s.b2[8 * w + 2 * t] -= tl * b2d[0];
                s.b2[8 * w + 2 * t + 1] -= tl * b2d[1];
            }
            const int r = u & 127;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float v1[16], v2[16];
                tc5::ld16(tc5::taddr(tm, my_lane, cW1 + 64 * mt + 16 * c), v1);
                tc5::ld16(tc5::taddr(tm, my_lane, cW2 + 64 * mt + 16 * c), v2);
                tc5::wait_ld();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int cc = 16 * c + 8 * half;
                    uint4 p1, p2;
                    p1.x = pack_f16x2(v1[8 * half + 0], v1[8 * half + 1]); p1.y = pack_f16x2(v1[8 * half + 2], v1[8 * half + 3]);
                    p1.z = pack_f16x2(v1[8 * half + 4], v1[8 * half + 5]); p1.w = pack_f16x2(v1[8 * half + 6], v1[8 * half + 7]);
                    p2.x = pack_f16x2(v2[8 * half + 0], v2[8 * half + 1]); p2.y = pack_f16x2(v2[8 * half + 2], v2[8 * half + 3]);
                    p2.z = pack_f16x2(v2[8 * half + 4], v2[8 * half + 5]); p2.w = pack_f16x2(v2[8 * half + 6], v2[8 * half + 7]);
                    *reinterpret_cast<uint4*>(&s.W1s[mt][0] + swz(r, cc)) = p1;
                    *reinterpret_cast<uint4*>(&s.W2s[0] + swz(u, cc)) = p2;
                }
            }
        }
        if (m + 1 < n_mb) {  // fp16 copy of the next mini-batch's XK and XQ (loaded since the top of m)
            const int st1 = st ^ 1;
            if (!mbar_wait_bounded(&s.full[st1], par ^ (st1 == 0 ? 1u : 0u), wait_limit, a.status)) s.fail = 1;
            convert_stage(&s.stage[st1][0], tid);
        }
        tc5::fence_before();
        __syncthreads();
        tc5::fence_after();
        if (s.fail) {
            m_stop = m;
            break;
        }
    }

    // ---- final state (the masters) ----------------------------------------------------------------
    if (!s.fail) {
        float* W1l = a.W1_last + static_cast<long long>(chain) * TTT_D * kHid;
        float* W2l = a.W2_last + static_cast<long long>(chain) * TTT_D * kHid;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float v1[16], v2[16];
            tc5::ld16(tc5::taddr(tm, my_lane, cW1 + 64 * mt + 16 * c), v1);
            tc5::ld16(tc5::taddr(tm, my_lane, cW2 + 64 * mt + 16 * c), v2);
            tc5::wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                W1l[(16 * c + i) * kHid + u] = v1[i];
                W2l[u * TTT_D + 16 * c + i] = v2[i];
            }
        }
        if (g == 0)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                a.b1_last[static_cast<long long>(chain) * kHid + 32 * w + 8 * nt + 2 * t] = b1r[nt][0];
                a.b1_last[static_cast<long long>(chain) * kHid + 32 * w + 8 * nt + 2 * t + 1] = b1r[nt][1];
            }
        if (tid < TTT_D) a.b2_last[static_cast<long long>(chain) * TTT_D + tid] = s.b2[tid];
    } else if (tid == 0) {
        // A wait gave up: let the MMAs and the loads still in flight land (bounded) before the
        // tensor memory is freed and the CTA exits.  Mini-batches m_stop .. issued-1 were loaded
        // but not consumed; the drain commit arrives once every MMA issued so far has finished.
        tc5::commit(&s.drain_bar);
        mbar_wait_bounded(&s.drain_bar, 0, kDrainPolls, nullptr);
        const int issued = min(n_mb, m_stop + kStages);
        for (int mm = m_stop; mm < issued; ++mm)
            mbar_wait_bounded(&s.full[mm % kStages], static_cast<uint32_t>((mm / kStages) & 1), kDrainPolls, nullptr);
    }
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();
    if (w == 0) tc5::dealloc(tm, kTmemCols);
}

}  // namespace

cudaError_t launch_mlp_tc(const MlpArgs& a, const LinearMaps& maps, cudaStream_t st) {
    const size_t smem = sizeof(MlpSmem) + 1024;  // + alignment slack
    cudaError_t e = cudaFuncSetAttribute(mlp_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    // two CTAs (chains) per SM: ask for the largest shared-memory carve-out
    e = cudaFuncSetAttribute(mlp_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    mlp_tc_kernel<<<static_cast<unsigned>(a.B * a.H), kThreads, smem, st>>>(a, maps);
    return cudaGetLastError();
}

}  // namespace ttt
